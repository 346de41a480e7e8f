// Backward of the PyTorch3D mesh rasterizer to screen-space vertex positions ("Accelerating
// 3D Deep Learning with PyTorch3D"; tutorial summary 3:52: gradients flow from 2-D pixels
// back to the 3-D model).  For each valid (pixel, slot) the face's edge-function weights,
// inside flag, nearest edge and its segment parameter are recomputed and differentiated
// with the candidate set, the inside flag and the nearest edge held fixed:
//
//   C_k = cross(V1 - p, V2 - p) for (V1, V2) = (b, c), (c, a), (a, b);  w_k = C_k / A
//   d cross(U - p, V - p)/dU = (V.y - p.y, -(V.x - p.x)),  /dV = (-(U.y - p.y), U.x - p.x)
//   dA/da = (b.y - c.y, c.x - b.x), dA/db = (c.y - a.y, a.x - c.x), dA/dc = (a.y - b.y, b.x - a.x)
//   dw_k = (dC_k - w_k dA) / A
//   perspective: u_k = w_k / z_k, S = sum u, bary_m = u_m / S, z = 1 / S
//   plain:       bary_k = w_k,     z = sum w_k z_k
//   squared distance to the nearest edge u -> v at q = u + t (v - u):
//       dd2/du = -2 (p - q)(1 - t),  dd2/dv = -2 (p - q) t;   dist = -d2 inside, +d2 outside.
//
// Contributions are scattered with float32 atomics (red.global.add): the general kernel
// adds into grad_verts (zeroed first); the fused silhouette kernel adds (x, y) pairs into
// a float2 accumulator that a final pass copies to grad_verts.
#include <cfloat>
#include <cmath>

#include "mr_common.cuh"
#include "mr_silhouette.cuh"

namespace mr {
namespace {

__device__ __forceinline__ bool load_face(const int64_t* __restrict__ faces, int64_t V, int64_t f, int64_t (&vid)[3]) {
    vid[0] = faces[3 * f];
    vid[1] = faces[3 * f + 1];
    vid[2] = faces[3 * f + 2];
    return vid[0] >= 0 && vid[0] < V && vid[1] >= 0 && vid[1] < V && vid[2] >= 0 && vid[2] < V;
}

// General backward: one thread per slot, float64 arithmetic; each of the face's vertices
// receives one float4 (x, y, z, 0) atomic into a padded accumulator.
template <bool PERSP>
__global__ void k_raster_bwd(const float* __restrict__ verts, int64_t V, const int64_t* __restrict__ faces,
                             int64_t F, const int64_t* __restrict__ p2f, int64_t nslots, int H, int W, int K,
                             const float* __restrict__ gz, const float* __restrict__ gb,
                             const float* __restrict__ gd, float4* __restrict__ acc, int* __restrict__ err) {
    for (int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; s < nslots; s += (int64_t)gridDim.x * blockDim.x) {
        const int64_t f = p2f[s];
        if (f == -1) continue;
        if (f < -1 || f >= F) {
            atomicOr(err, kErrSlotIndex);
            continue;
        }
        int64_t vid[3];
        if (!load_face(faces, V, f, vid)) {
            atomicOr(err, kErrFaceIndex);
            continue;
        }
        const int64_t pix = s / K;
        const int64_t rem = pix % ((int64_t)H * W);
        const int i = (int)(rem / W), j = (int)(rem % W);
        const double px = -1.0 + (2.0 * j + 1.0) / W;
        const double py = 1.0 - (2.0 * i + 1.0) / H;
        double x[3], y[3], z[3];
#pragma unroll
        for (int q = 0; q < 3; ++q) {
            x[q] = verts[3 * vid[q]];
            y[q] = verts[3 * vid[q] + 1];
            z[q] = verts[3 * vid[q] + 2];
        }
        const double A = (x[1] - x[0]) * (y[2] - y[0]) - (y[1] - y[0]) * (x[2] - x[0]);
        if (fabs(A) <= kDegenerateArea) continue;
        double rx[3], ry[3];   // vertex - pixel
#pragma unroll
        for (int q = 0; q < 3; ++q) { rx[q] = x[q] - px; ry[q] = y[q] - py; }
        double w[3];
        w[0] = (rx[1] * ry[2] - ry[1] * rx[2]) / A;
        w[1] = (rx[2] * ry[0] - ry[2] * rx[0]) / A;
        w[2] = (rx[0] * ry[1] - ry[0] * rx[1]) / A;
        const bool inside = w[0] >= 0.0 && w[1] >= 0.0 && w[2] >= 0.0;
        double g[3][3] = {{0, 0, 0}, {0, 0, 0}, {0, 0, 0}};   // [vertex][x, y, z]
        if (gd) {
            int eu = 0;
            double best = DBL_MAX, bt = 0.0;
#pragma unroll
            for (int k = 0; k < 3; ++k) {
                const int k1 = k == 2 ? 0 : k + 1;
                const double ex = x[k1] - x[k], ey = y[k1] - y[k];
                const double len2 = ex * ex + ey * ey;
                double t = len2 > 0.0 ? ((px - x[k]) * ex + (py - y[k]) * ey) / len2 : 0.0;
                t = fmin(fmax(t, 0.0), 1.0);
                const double dx = px - (x[k] + t * ex), dy = py - (y[k] + t * ey);
                const double d2 = dx * dx + dy * dy;
                if (d2 < best) { best = d2; eu = k; bt = t; }
            }
            const int ev = eu == 2 ? 0 : eu + 1;
            const double gdist = (double)gd[s] * (inside ? -1.0 : 1.0);
            const double qx = x[eu] + bt * (x[ev] - x[eu]), qy = y[eu] + bt * (y[ev] - y[eu]);
            const double dx = px - qx, dy = py - qy;
            g[eu][0] += gdist * (-2.0 * dx * (1.0 - bt));
            g[eu][1] += gdist * (-2.0 * dy * (1.0 - bt));
            g[ev][0] += gdist * (-2.0 * dx * bt);
            g[ev][1] += gdist * (-2.0 * dy * bt);
        }
        if (gb || gz) {
            double gbar[3] = {0, 0, 0};
            if (gb) { gbar[0] = gb[3 * s]; gbar[1] = gb[3 * s + 1]; gbar[2] = gb[3 * s + 2]; }
            const double gzz = gz ? (double)gz[s] : 0.0;
            double gw[3];
            if (PERSP) {
                double u[3], S = 0.0;
#pragma unroll
                for (int k = 0; k < 3; ++k) { u[k] = w[k] / z[k]; S += u[k]; }
                double bar[3] = {u[0] / S, u[1] / S, u[2] / S};
                const double zz = 1.0 / S;
                const double dot = gbar[0] * bar[0] + gbar[1] * bar[1] + gbar[2] * bar[2];
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    const double gu = (gbar[k] - dot) / S - gzz * zz * zz;
                    gw[k] = gu / z[k];
                    g[k][2] += -gu * u[k] / z[k];
                }
            } else {
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    gw[k] = gbar[k] + gzz * z[k];
                    g[k][2] += gzz * w[k];
                }
            }
            const double G = gw[0] * w[0] + gw[1] * w[1] + gw[2] * w[2];
            const double dA[3][2] = {{y[1] - y[2], x[2] - x[1]}, {y[2] - y[0], x[0] - x[2]}, {y[0] - y[1], x[1] - x[0]}};
            // sum_k gw_k dC_k / d(vertex)
            double dc[3][2];
            dc[0][0] = gw[1] * (-ry[2]) + gw[2] * (ry[1]);
            dc[0][1] = gw[1] * (rx[2]) + gw[2] * (-rx[1]);
            dc[1][0] = gw[0] * (ry[2]) + gw[2] * (-ry[0]);
            dc[1][1] = gw[0] * (-rx[2]) + gw[2] * (rx[0]);
            dc[2][0] = gw[0] * (-ry[1]) + gw[1] * (ry[0]);
            dc[2][1] = gw[0] * (rx[1]) + gw[1] * (-rx[0]);
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                g[q][0] += (dc[q][0] - G * dA[q][0]) / A;
                g[q][1] += (dc[q][1] - G * dA[q][1]) / A;
            }
        }
#pragma unroll
        for (int q = 0; q < 3; ++q)
            if (g[q][0] != 0.0 || g[q][1] != 0.0 || g[q][2] != 0.0)
                atomicAdd(acc + vid[q], make_float4((float)g[q][0], (float)g[q][1], (float)g[q][2], 0.f));
    }
}

// grad_verts (V x 3) from the padded (x, y, z, 0) accumulator.
__global__ void k_xyzw_to_xyz(const float4* __restrict__ acc, int64_t V, float* __restrict__ gv) {
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < V; v += (int64_t)gridDim.x * blockDim.x) {
        const float4 a = acc[v];
        gv[3 * v] = a.x;
        gv[3 * v + 1] = a.y;
        gv[3 * v + 2] = a.z;
    }
}

// Fused silhouette backward + distance backward: one thread per pixel (32 consecutive
// pixels per warp), float32.  Per slot the nearest edge u -> v is recomputed and its two
// end points receive -2 (p - q)(1 - t) and -2 (p - q) t times dL/ddist.
template <int KC>
__global__ void __launch_bounds__(256)
k_sil_raster_bwd(const float* __restrict__ verts, int64_t V, const int64_t* __restrict__ faces, int64_t F,
                 const int64_t* __restrict__ p2f, const float* __restrict__ dists,
                 const float* __restrict__ grad_alpha, int64_t npix, int H, int W, int K, float sigma,
                 float2* __restrict__ acc, int* __restrict__ err) {
    const int lane = threadIdx.x & 31;
    const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t base = wid * 32; base < npix; base += nw * 32) {
        const int64_t q = base + lane;
        const bool live = q < npix;
        float d[KC], g[KC];
        bool v[KC];
        int64_t fk[KC];
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            const bool in = live && k < K;
            fk[k] = in ? p2f[q * K + k] : -1;
            if (fk[k] < -1) atomicOr(err, kErrSlotIndex);
            v[k] = fk[k] >= 0;
            d[k] = in ? dists[q * K + k] : 0.f;
        }
        const float ga = live ? grad_alpha[q] : 0.f;
        silhouette_grad<KC>(d, v, K, sigma, ga, g);
        const int64_t rem = (live ? q : 0) % ((int64_t)H * W);
        const int i = (int)(rem / W), j = (int)(rem % W);
        const double pxd = -1.0 + (2.0 * j + 1.0) / W, pyd = 1.0 - (2.0 * i + 1.0) / H;
        const float pxh = (float)pxd, pyh = (float)pyd;
        const float pxl = (float)(pxd - (double)pxh), pyl = (float)(pyd - (double)pyh);
        // per slot: the nearest edge's two end points and their (x, y) contributions
        constexpr int NT = KC <= 8 ? 2 * KC : 2;
        int tid[NT];
        float2 tv[NT];
        bool alive[NT];
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            bool act = k < K && v[k] && g[k] != 0.f;
            if constexpr (KC <= 8) {
                tid[2 * k] = tid[2 * k + 1] = -1;
                tv[2 * k] = tv[2 * k + 1] = make_float2(0.f, 0.f);
            }
            if (act) {
                int64_t vid[3];
                if (fk[k] >= F) {
                    atomicOr(err, kErrSlotIndex);
                    act = false;
                } else if (!load_face(faces, V, fk[k], vid)) {
                    atomicOr(err, kErrFaceIndex);
                    act = false;
                } else {
                    float x[3], y[3];
#pragma unroll
                    for (int e = 0; e < 3; ++e) {
                        x[e] = verts[3 * vid[e]];
                        y[e] = verts[3 * vid[e] + 1];
                    }
                    int eu = 0;
                    float best = FLT_MAX, bt = 0.f, brx = 0.f, bry = 0.f;
#pragma unroll
                    for (int e = 0; e < 3; ++e) {
                        const int e1 = e == 2 ? 0 : e + 1;
                        const float ex = x[e1] - x[e], ey = y[e1] - y[e];
                        const float ax = (pxh - x[e]) + pxl, ay = (pyh - y[e]) + pyl;
                        const float len2 = fmaf(ex, ex, ey * ey);
                        const float t = len2 > 0.f ? __saturatef(__fdividef(fmaf(ax, ex, ay * ey), len2)) : 0.f;
                        const float rx = fmaf(-t, ex, ax), ry = fmaf(-t, ey, ay);
                        const float d2 = fmaf(rx, rx, ry * ry);
                        if (d2 < best) { best = d2; eu = e; bt = t; brx = rx; bry = ry; }
                    }
                    const int ev = eu == 2 ? 0 : eu + 1;
                    const float gdist = d[k] < 0.f ? -g[k] : g[k];
                    const float su = -2.f * gdist * (1.f - bt), sv = -2.f * gdist * bt;
                    if constexpr (KC <= 8) {
                        tv[2 * k] = make_float2(su * brx, su * bry);
                        tv[2 * k + 1] = make_float2(sv * brx, sv * bry);
                        tid[2 * k] = (int)vid[eu];
                        tid[2 * k + 1] = (int)vid[ev];
                    } else {
                        atomicAdd(acc + vid[eu], make_float2(su * brx, su * bry));
                        atomicAdd(acc + vid[ev], make_float2(sv * brx, sv * bry));
                        act = false;
                    }
                }
            }
            if constexpr (KC <= 8) alive[2 * k] = alive[2 * k + 1] = act;
        }
        // The K faces of a pixel are neighbours and often share the nearest edge's end
        // points: sum equal vertex ids of this pixel first (the two ends of one slot
        // always differ), then one float2 atomic per distinct vertex (up to K = 8; larger K
        // would spend more registers on the comparisons than the atomics cost).
#pragma unroll
        for (int t = 2; t < (KC <= 8 ? NT : 0); ++t)
#pragma unroll
            for (int u = 0; u < (t & ~1); ++u)
                if (alive[u] && alive[t] && tid[u] == tid[t]) {
                    tv[u].x += tv[t].x;
                    tv[u].y += tv[t].y;
                    alive[t] = false;
                }
#pragma unroll
        for (int t = 0; t < (KC <= 8 ? NT : 0); ++t)
            if (alive[t]) atomicAdd(acc + tid[t], tv[t]);
    }
}

// grad_verts (V x 3) from the (x, y) accumulator; the silhouette has no z gradient.
__global__ void k_xy_to_xyz(const float2* __restrict__ acc, int64_t V, float* __restrict__ gv) {
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < V; v += (int64_t)gridDim.x * blockDim.x) {
        const float2 a = acc[v];
        gv[3 * v] = a.x;
        gv[3 * v + 1] = a.y;
        gv[3 * v + 2] = 0.f;
    }
}

int validate_bwd(const float* verts, int64_t V, const int64_t* faces, int64_t F, const int64_t* p2f, int32_t N,
                 int32_t H, int32_t W, int32_t K, float* grad_verts) {
    if (N < 0 || H < 1 || W < 1 || K < 1 || K > MR_KMAX || V < 0 || F < 0 || V > INT32_MAX) {
        set_error("invalid shape N=%d H=%d W=%d K=%d V=%lld F=%lld", N, H, W, K, (long long)V, (long long)F);
        return MR_ERR_ARG;
    }
    if (V > 0 && (!verts || !grad_verts)) {
        set_error("null vertex pointer");
        return MR_ERR_ARG;
    }
    if (N > 0 && (!p2f || (F > 0 && !faces))) {
        set_error("null input pointer");
        return MR_ERR_ARG;
    }
    return MR_OK;
}

inline int grid_for(int64_t n) { return (int)std::min<int64_t>((n + 255) / 256, 148 * 32); }

}  // namespace
}  // namespace mr

extern "C" {

int mr_rasterize_bwd(const float* verts, int64_t V, const int64_t* faces, int64_t F, const int64_t* pix_to_face,
                     int32_t N, int32_t H, int32_t W, int32_t K, int32_t perspective_correct, const float* grad_zbuf,
                     const float* grad_bary, const float* grad_dists, float* grad_verts, void* stream) {
    int rc = mr::validate_bwd(verts, V, faces, F, pix_to_face, N, H, W, K, grad_verts);
    if (rc != MR_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t nslots = (int64_t)N * H * W * K;
    if (V == 0) return MR_OK;
    if (nslots == 0 || (!grad_zbuf && !grad_bary && !grad_dists)) {
        MR_CUDA(cudaMemsetAsync(grad_verts, 0, sizeof(float) * 3 * (size_t)V, s));
        return MR_OK;
    }
    int* err = mr::device_error_word();
    if (!err) {
        mr::set_error("cannot locate the device error word");
        return MR_ERR_CUDA;
    }
    float4* acc = nullptr;
    rc = mr::scratch_alloc(reinterpret_cast<void**>(&acc), sizeof(float4) * (size_t)V, s);
    if (rc != MR_OK) return rc;
    cudaError_t e = cudaMemsetAsync(acc, 0, sizeof(float4) * (size_t)V, s);
    if (e == cudaSuccess) {
        const int g = mr::grid_for(nslots);
        mr::ProfScope ps(MR_STAGE_RASTER_BWD, s);
        if (perspective_correct)
            mr::k_raster_bwd<true><<<g, 256, 0, s>>>(verts, V, faces, F, pix_to_face, nslots, H, W, K, grad_zbuf,
                                                     grad_bary, grad_dists, acc, err);
        else
            mr::k_raster_bwd<false><<<g, 256, 0, s>>>(verts, V, faces, F, pix_to_face, nslots, H, W, K, grad_zbuf,
                                                      grad_bary, grad_dists, acc, err);
        mr::k_xyzw_to_xyz<<<mr::grid_for(V), 256, 0, s>>>(acc, V, grad_verts);
        e = cudaGetLastError();
    }
    mr::scratch_free(acc, s);
    if (e != cudaSuccess) return mr::cuda_fail(e, "rasterizer backward launch");
    return MR_OK;
}

int mr_silhouette_rasterize_bwd(const float* verts, int64_t V, const int64_t* faces, int64_t F,
                                const int64_t* pix_to_face, const float* dists, int32_t N, int32_t H, int32_t W,
                                int32_t K, float sigma, const float* grad_alpha, float* grad_verts, void* stream) {
    int rc = mr::validate_bwd(verts, V, faces, F, pix_to_face, N, H, W, K, grad_verts);
    if (rc != MR_OK) return rc;
    if (!(sigma > 0.f) || !std::isfinite(sigma)) {
        mr::set_error("sigma must be finite and > 0");
        return MR_ERR_ARG;
    }
    if (N > 0 && (!dists || !grad_alpha)) {
        mr::set_error("null dists or grad_alpha");
        return MR_ERR_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t npix = (int64_t)N * H * W;
    if (npix == 0 || V == 0) {
        if (V > 0) MR_CUDA(cudaMemsetAsync(grad_verts, 0, sizeof(float) * 3 * (size_t)V, s));
        return MR_OK;
    }
    int* err = mr::device_error_word();
    if (!err) {
        mr::set_error("cannot locate the device error word");
        return MR_ERR_CUDA;
    }
    float2* acc = nullptr;
    rc = mr::scratch_alloc(reinterpret_cast<void**>(&acc), sizeof(float2) * (size_t)V, s);
    if (rc != MR_OK) return rc;
    cudaError_t e = cudaMemsetAsync(acc, 0, sizeof(float2) * (size_t)V, s);
    if (e == cudaSuccess) {
        const int g = mr::grid_for(npix);
        mr::ProfScope ps(MR_STAGE_SILHOUETTE_RASTER_BWD, s);
#define MR_SRB(KC)                                                                                            \
    mr::k_sil_raster_bwd<KC><<<g, 256, 0, s>>>(verts, V, faces, F, pix_to_face, dists, grad_alpha, npix, H, W, K, \
                                               sigma, acc, err)
        if (K <= 1) MR_SRB(1);
        else if (K <= 2) MR_SRB(2);
        else if (K <= 4) MR_SRB(4);
        else if (K <= 8) MR_SRB(8);
        else if (K <= 16) MR_SRB(16);
        else MR_SRB(32);
#undef MR_SRB
        mr::k_xy_to_xyz<<<mr::grid_for(V), 256, 0, s>>>(acc, V, grad_verts);
        e = cudaGetLastError();
    }
    mr::scratch_free(acc, s);
    if (e != cudaSuccess) return mr::cuda_fail(e, "silhouette-rasterizer backward launch");
    return MR_OK;
}

}  // extern "C"
