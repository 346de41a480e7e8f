// Stage two of the PyTorch3D renderer beyond the silhouette ("Accelerating 3D Deep Learning
// with PyTorch3D", method: pluggable Gouraud / Phong shaders over the K faces kept per
// pixel): per-vertex attribute interpolation over the fragments and the soft RGB blend of
// SoftRas (the renderer the paper compares against), with their backward passes.
//
//   interpolation   out[s, d] = sum_m bary[s, m] attr[v_m, d]  (0 for an empty slot)
//   blend           p_k = 1 / (1 + exp(d_k / sigma)),
//                   w_k = p_k exp((z_near_k - z_k) / (gamma (zfar - znear))), where z_near_k is
//                   the pixel's nearest fragment depth (the normalised-nearness shift),
//                   w_b = exp((eps - s_max) / gamma), s = (zfar - z) / (zfar - znear),
//                   rgb = (sum w_k c_k + w_b bg) / (sum w_k + w_b),  alpha = 1 - prod (1 - p_k).
// The depth weight is formed from the depth difference, not from two rounded nearness
// values, so float32 keeps it accurate when gamma is small (1e-4 makes a 1e-7 nearness
// error a 1e-3 weight error).
#include <cfloat>
#include <cmath>

#include "mr_common.cuh"
#include "mr_silhouette.cuh"

namespace mr {
namespace {

constexpr float kBlendEps = 1e-10f;

__device__ __forceinline__ bool face_ids(const int64_t* __restrict__ faces, int64_t V, int64_t f, int64_t (&v)[3]) {
    v[0] = faces[3 * f];
    v[1] = faces[3 * f + 1];
    v[2] = faces[3 * f + 2];
    return v[0] >= 0 && v[0] < V && v[1] >= 0 && v[1] < V && v[2] >= 0 && v[2] < V;
}

__global__ void k_interpolate_fwd(const int64_t* __restrict__ p2f, const float* __restrict__ bary, int64_t nslots,
                                  const int64_t* __restrict__ faces, int64_t F, const float* __restrict__ attr,
                                  int64_t V, int D, float* __restrict__ out, int* __restrict__ err) {
    for (int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; s < nslots; s += (int64_t)gridDim.x * blockDim.x) {
        const int64_t f = p2f[s];
        int64_t v[3];
        bool ok = f >= 0;
        if (f < -1 || f >= F) {
            atomicOr(err, kErrSlotIndex);
            ok = false;
        } else if (ok && !face_ids(faces, V, f, v)) {
            atomicOr(err, kErrFaceIndex);
            ok = false;
        }
        float b0 = 0.f, b1 = 0.f, b2 = 0.f;
        if (ok) {
            b0 = bary[3 * s];
            b1 = bary[3 * s + 1];
            b2 = bary[3 * s + 2];
        }
        for (int d = 0; d < D; ++d)
            out[s * D + d] = ok ? fmaf(b0, attr[v[0] * D + d], fmaf(b1, attr[v[1] * D + d], b2 * attr[v[2] * D + d]))
                                : 0.f;
    }
}

// Gradient of the interpolation.  For D <= 4 the attribute gradient is summed into a
// padded V x 4 accumulator with one float4 atomic per (slot, vertex) (three per slot
// instead of 3 D scalar ones), then copied out; wider attributes use scalar atomics.
template <bool VEC4>
__global__ void k_interpolate_bwd(const int64_t* __restrict__ p2f, const float* __restrict__ bary, int64_t nslots,
                                  const int64_t* __restrict__ faces, int64_t F, const float* __restrict__ attr,
                                  int64_t V, int D, const float* __restrict__ grad_out, float* __restrict__ grad_attr,
                                  float4* __restrict__ acc4, float* __restrict__ grad_bary, int* __restrict__ err) {
    for (int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; s < nslots; s += (int64_t)gridDim.x * blockDim.x) {
        const int64_t f = p2f[s];
        int64_t v[3];
        bool ok = f >= 0;
        if (f < -1 || f >= F) {
            atomicOr(err, kErrSlotIndex);
            ok = false;
        } else if (ok && !face_ids(faces, V, f, v)) {
            atomicOr(err, kErrFaceIndex);
            ok = false;
        }
        float gb[3] = {0.f, 0.f, 0.f};
        if (ok) {
            const float b[3] = {bary[3 * s], bary[3 * s + 1], bary[3 * s + 2]};
            if (VEC4) {
                float g[4] = {0.f, 0.f, 0.f, 0.f};
                for (int d = 0; d < D; ++d) g[d] = grad_out[s * D + d];
#pragma unroll
                for (int m = 0; m < 3; ++m) {
                    for (int d = 0; d < D; ++d) gb[m] = fmaf(attr[v[m] * D + d], g[d], gb[m]);
                    atomicAdd(acc4 + v[m], make_float4(b[m] * g[0], b[m] * g[1], b[m] * g[2], b[m] * g[3]));
                }
            } else {
                for (int d = 0; d < D; ++d) {
                    const float g = grad_out[s * D + d];
                    if (g == 0.f) continue;
#pragma unroll
                    for (int m = 0; m < 3; ++m) {
                        gb[m] = fmaf(attr[v[m] * D + d], g, gb[m]);
                        if (b[m] != 0.f) atomicAdd(grad_attr + v[m] * D + d, b[m] * g);
                    }
                }
            }
        }
        if (grad_bary) {
            grad_bary[3 * s] = gb[0];
            grad_bary[3 * s + 1] = gb[1];
            grad_bary[3 * s + 2] = gb[2];
        }
    }
}

__global__ void k_acc4_to_rows(const float4* __restrict__ acc4, int64_t V, int D, float* __restrict__ out) {
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < V; v += (int64_t)gridDim.x * blockDim.x) {
        const float4 a = acc4[v];
        const float x[4] = {a.x, a.y, a.z, a.w};
        for (int d = 0; d < D; ++d) out[v * D + d] = x[d];
    }
}

struct BlendParams {
    float bg[MR_BLEND_DMAX];
    float sigma, gamma, znear, zfar;
};

// Per-pixel blend state from the K slots' face ids, distances and depths: coverage
// weights p, depth weights w, the background weight wb and the normaliser den.
template <int KC>
__device__ __forceinline__ void blend_state(const int64_t (&f)[KC], const float (&dist)[KC], const float (&zv)[KC],
                                            int K, const BlendParams& P, bool (&valid)[KC], float (&d)[KC],
                                            float (&p)[KC], float (&w)[KC], float& wb, float& den) {
    float zmin = FLT_MAX;
    float z[KC];
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        valid[k] = k < K && f[k] >= 0;
        d[k] = valid[k] ? dist[k] : 0.f;
        z[k] = valid[k] ? zv[k] : 0.f;
        if (valid[k]) zmin = fminf(zmin, z[k]);
    }
    const float range = P.zfar - P.znear;
    const float s_max = (P.zfar - zmin) / range;        // nearness of the nearest fragment
    const bool shifted = s_max > kBlendEps;              // else the shift is eps itself
    den = 0.f;
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        const float x = d[k] / P.sigma;
        p[k] = valid[k] ? 1.f / (1.f + expf(x)) : 0.f;
        float e;
        if (shifted) e = (zmin - z[k]) / (P.gamma * range);
        else e = ((P.zfar - z[k]) / range - kBlendEps) / P.gamma;
        w[k] = valid[k] ? p[k] * expf(e) : 0.f;
        den += w[k];
    }
    wb = expf((kBlendEps - (shifted ? s_max : kBlendEps)) / P.gamma);
    den += wb;
}

// The same from memory (pixel q, K slots, element-wise loads).
template <int KC>
__device__ __forceinline__ void blend_weights(const int64_t* __restrict__ p2f, const float* __restrict__ dists,
                                              const float* __restrict__ zbuf, int64_t q, int K, const BlendParams& P,
                                              bool (&valid)[KC], float (&d)[KC], float (&p)[KC], float (&w)[KC],
                                              float& wb, float& den) {
    int64_t f[KC];
    float dd[KC], zz[KC];
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        f[k] = k < K ? p2f[q * K + k] : -1;
        dd[k] = f[k] >= 0 ? dists[q * K + k] : 0.f;
        zz[k] = f[k] >= 0 ? zbuf[q * K + k] : 0.f;
    }
    blend_state<KC>(f, dd, zz, K, P, valid, d, p, w, wb, den);
}

// RGB blend with K == KC (a multiple of 4) and 16-byte aligned arrays: every per-pixel run
// (ids, distances, depths, 3 KC colours, rgba, gradients) moves in 16-byte accesses.
template <int KC>
__global__ void k_blend_fwd_rgb(const int64_t* __restrict__ p2f, const float* __restrict__ colors,
                                const float* __restrict__ dists, const float* __restrict__ zbuf, int64_t npix,
                                BlendParams P, float* __restrict__ out) {
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < npix; q += (int64_t)gridDim.x * blockDim.x) {
        int64_t f[KC];
        float dd[KC], zz[KC], col[3 * KC];
        ld_vec<KC>(p2f + q * KC, f);
        ld_vec<KC>(dists + q * KC, dd);
        ld_vec<KC>(zbuf + q * KC, zz);
        ld_vec<3 * KC>(colors + q * 3 * KC, col);
        bool valid[KC];
        float d[KC], p[KC], w[KC], wb, den;
        blend_state<KC>(f, dd, zz, KC, P, valid, d, p, w, wb, den);
        float o[4];
#pragma unroll
        for (int c = 0; c < 3; ++c) {
            float acc = wb * P.bg[c];
#pragma unroll
            for (int k = 0; k < KC; ++k)
                if (valid[k]) acc = fmaf(w[k], col[3 * k + c], acc);
            o[c] = acc / den;
        }
        o[3] = silhouette_alpha<KC>(d, valid, KC, P.sigma);
        st_vec<4>(out + q * 4, o);
    }
}

template <int KC>
__global__ void k_blend_bwd_rgb(const int64_t* __restrict__ p2f, const float* __restrict__ colors,
                                const float* __restrict__ dists, const float* __restrict__ zbuf, int64_t npix,
                                BlendParams P, const float* __restrict__ grad_rgba, float* __restrict__ grad_colors,
                                float* __restrict__ grad_dists, float* __restrict__ grad_zbuf) {
    const float inv_gz = 1.f / (P.gamma * (P.zfar - P.znear));
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < npix; q += (int64_t)gridDim.x * blockDim.x) {
        int64_t f[KC];
        float dd[KC], zz[KC], col[3 * KC], g4[4];
        ld_vec<KC>(p2f + q * KC, f);
        ld_vec<KC>(dists + q * KC, dd);
        ld_vec<KC>(zbuf + q * KC, zz);
        ld_vec<3 * KC>(colors + q * 3 * KC, col);
        ld_vec<4>(grad_rgba + q * 4, g4);
        bool valid[KC];
        float d[KC], p[KC], w[KC], wb, den;
        blend_state<KC>(f, dd, zz, KC, P, valid, d, p, w, wb, den);
        const float inv_den = 1.f / den;
        float rgb[3];
#pragma unroll
        for (int c = 0; c < 3; ++c) {
            float acc = wb * P.bg[c];
#pragma unroll
            for (int k = 0; k < KC; ++k)
                if (valid[k]) acc = fmaf(w[k], col[3 * k + c], acc);
            rgb[c] = acc * inv_den;
        }
        float ga[KC], gc[3 * KC], gdv[KC], gzv[KC];
        silhouette_grad<KC>(d, valid, KC, P.sigma, g4[3], ga);
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            float gw = 0.f;
#pragma unroll
            for (int c = 0; c < 3; ++c) {
                gc[3 * k + c] = valid[k] ? w[k] * inv_den * g4[c] : 0.f;
                gw = fmaf(col[3 * k + c] - rgb[c], g4[c], gw);
            }
            gw *= inv_den;
            gdv[k] = valid[k] ? gw * w[k] * (-(1.f - p[k]) / P.sigma) + ga[k] : 0.f;
            gzv[k] = valid[k] ? -gw * w[k] * inv_gz : 0.f;
        }
        if (grad_colors) st_vec<3 * KC>(grad_colors + q * 3 * KC, gc);
        if (grad_dists) st_vec<KC>(grad_dists + q * KC, gdv);
        if (grad_zbuf) st_vec<KC>(grad_zbuf + q * KC, gzv);
    }
}

template <int KC>
__global__ void k_blend_fwd(const int64_t* __restrict__ p2f, const float* __restrict__ colors,
                            const float* __restrict__ dists, const float* __restrict__ zbuf, int64_t npix, int K,
                            int D, BlendParams P, float* __restrict__ out) {
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < npix; q += (int64_t)gridDim.x * blockDim.x) {
        bool valid[KC];
        float d[KC], p[KC], w[KC], wb, den;
        blend_weights<KC>(p2f, dists, zbuf, q, K, P, valid, d, p, w, wb, den);
        for (int c = 0; c < D; ++c) {
            float acc = wb * P.bg[c];
#pragma unroll
            for (int k = 0; k < KC; ++k)
                if (valid[k]) acc = fmaf(w[k], colors[(q * K + k) * D + c], acc);
            out[q * (D + 1) + c] = acc / den;
        }
        out[q * (D + 1) + D] = silhouette_alpha<KC>(d, valid, K, P.sigma);
    }
}

template <int KC>
__global__ void k_blend_bwd(const int64_t* __restrict__ p2f, const float* __restrict__ colors,
                            const float* __restrict__ dists, const float* __restrict__ zbuf, int64_t npix, int K,
                            int D, BlendParams P, const float* __restrict__ grad_rgba,
                            float* __restrict__ grad_colors, float* __restrict__ grad_dists,
                            float* __restrict__ grad_zbuf) {
    const float inv_gz = 1.f / (P.gamma * (P.zfar - P.znear));
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < npix; q += (int64_t)gridDim.x * blockDim.x) {
        bool valid[KC];
        float d[KC], p[KC], w[KC], wb, den;
        blend_weights<KC>(p2f, dists, zbuf, q, K, P, valid, d, p, w, wb, den);
        const float inv_den = 1.f / den;
        float rgb[MR_BLEND_DMAX], g[MR_BLEND_DMAX];
        for (int c = 0; c < D; ++c) {
            float acc = wb * P.bg[c];
#pragma unroll
            for (int k = 0; k < KC; ++k)
                if (valid[k]) acc = fmaf(w[k], colors[(q * K + k) * D + c], acc);
            rgb[c] = acc * inv_den;
            g[c] = grad_rgba[q * (D + 1) + c];
        }
        float ga[KC];
        silhouette_grad<KC>(d, valid, K, P.sigma, grad_rgba[q * (D + 1) + D], ga);
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            if (k >= K) break;
            const int64_t s = q * K + k;
            float gw = 0.f;
            for (int c = 0; c < D; ++c) {
                if (grad_colors) grad_colors[s * D + c] = valid[k] ? w[k] * inv_den * g[c] : 0.f;
                if (valid[k]) gw = fmaf(colors[s * D + c] - rgb[c], g[c], gw);
            }
            gw *= inv_den;
            if (grad_dists) grad_dists[s] = valid[k] ? gw * w[k] * (-(1.f - p[k]) / P.sigma) + ga[k] : 0.f;
            if (grad_zbuf) grad_zbuf[s] = valid[k] ? -gw * w[k] * inv_gz : 0.f;
        }
    }
}


// 16-byte alignment of an optional array (a null pointer does not stop the vector path).
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_blend(int64_t npix, int K, int D, float sigma, float gamma, float znear, float zfar) {
    if (npix < 0 || K < 1 || K > MR_KMAX || D < 1 || D > MR_BLEND_DMAX) {
        set_error("invalid shape npix=%lld K=%d D=%d (D <= %d)", (long long)npix, K, D, MR_BLEND_DMAX);
        return MR_ERR_ARG;
    }
    if (!(sigma > 0.f) || !(gamma > 0.f) || !(zfar > znear) || !std::isfinite(sigma) || !std::isfinite(gamma) ||
        !std::isfinite(znear) || !std::isfinite(zfar)) {
        set_error("blend needs finite sigma > 0, gamma > 0 and zfar > znear");
        return MR_ERR_ARG;
    }
    return MR_OK;
}

}  // namespace
}  // namespace mr

extern "C" {

int mr_interpolate_fwd(const int64_t* pix_to_face, const float* bary, int64_t npix, int32_t K, const int64_t* faces,
                       int64_t F, const float* attr, int64_t V, int32_t D, float* out, void* stream) {
    if (npix < 0 || K < 1 || K > MR_KMAX || D < 1 || V < 0 || F < 0) {
        mr::set_error("invalid shape npix=%lld K=%d D=%d", (long long)npix, K, D);
        return MR_ERR_ARG;
    }
    const int64_t nslots = npix * K;
    if (nslots == 0) return MR_OK;
    if (!pix_to_face || !bary || !out || (F > 0 && (!faces || !attr))) {
        mr::set_error("null pointer");
        return MR_ERR_ARG;
    }
    int* err = mr::device_error_word();
    if (!err) {
        mr::set_error("cannot locate the device error word");
        return MR_ERR_CUDA;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    {
        mr::ProfScope ps(MR_STAGE_INTERPOLATE_FWD, s);
        mr::k_interpolate_fwd<<<mr::grid_for(nslots), 256, 0, s>>>(pix_to_face, bary, nslots, faces, F, attr, V, D, out,
                                                                  err);
    }
    MR_CUDA(cudaGetLastError());
    return MR_OK;
}

int mr_interpolate_bwd(const int64_t* pix_to_face, const float* bary, int64_t npix, int32_t K, const int64_t* faces,
                       int64_t F, const float* attr, int64_t V, int32_t D, const float* grad_out, float* grad_attr,
                       float* grad_bary, void* stream) {
    if (npix < 0 || K < 1 || K > MR_KMAX || D < 1 || V < 0 || F < 0) {
        mr::set_error("invalid shape npix=%lld K=%d D=%d", (long long)npix, K, D);
        return MR_ERR_ARG;
    }
    if ((V > 0 && !grad_attr) || (npix > 0 && (!pix_to_face || !bary || !grad_out))) {
        mr::set_error("null pointer");
        return MR_ERR_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t nslots = npix * K;
    if (nslots == 0 || V == 0) {
        if (V > 0) MR_CUDA(cudaMemsetAsync(grad_attr, 0, sizeof(float) * (size_t)(V * D), s));
        return MR_OK;
    }
    int* err = mr::device_error_word();
    if (!err) {
        mr::set_error("cannot locate the device error word");
        return MR_ERR_CUDA;
    }
    if (D > 4) {
        MR_CUDA(cudaMemsetAsync(grad_attr, 0, sizeof(float) * (size_t)(V * D), s));
        mr::ProfScope ps(MR_STAGE_INTERPOLATE_BWD, s);
        mr::k_interpolate_bwd<false><<<mr::grid_for(nslots), 256, 0, s>>>(pix_to_face, bary, nslots, faces, F, attr, V,
                                                                         D, grad_out, grad_attr, nullptr, grad_bary,
                                                                         err);
        MR_CUDA(cudaGetLastError());
        return MR_OK;
    }
    float4* acc = nullptr;
    int rc = mr::scratch_alloc(reinterpret_cast<void**>(&acc), sizeof(float4) * (size_t)V, s);
    if (rc != MR_OK) return rc;
    cudaError_t e = cudaMemsetAsync(acc, 0, sizeof(float4) * (size_t)V, s);
    if (e == cudaSuccess) {
        mr::ProfScope ps(MR_STAGE_INTERPOLATE_BWD, s);
        mr::k_interpolate_bwd<true><<<mr::grid_for(nslots), 256, 0, s>>>(pix_to_face, bary, nslots, faces, F, attr, V,
                                                                        D, grad_out, nullptr, acc, grad_bary, err);
        mr::k_acc4_to_rows<<<mr::grid_for(V), 256, 0, s>>>(acc, V, D, grad_attr);
        e = cudaGetLastError();
    }
    mr::scratch_free(acc, s);
    if (e != cudaSuccess) return mr::cuda_fail(e, "interpolation backward");
    return MR_OK;
}

int mr_blend_fwd(const int64_t* pix_to_face, const float* colors, const float* dists, const float* zbuf, int64_t npix,
                 int32_t K, int32_t D, const float* background, float sigma, float gamma, float znear, float zfar,
                 float* rgba, void* stream) {
    int rc = mr::check_blend(npix, K, D, sigma, gamma, znear, zfar);
    if (rc != MR_OK || npix == 0) return rc;
    if (!pix_to_face || !colors || !dists || !zbuf || !background || !rgba) {
        mr::set_error("null pointer");
        return MR_ERR_ARG;
    }
    mr::BlendParams P;
    for (int c = 0; c < MR_BLEND_DMAX; ++c) P.bg[c] = c < D ? background[c] : 0.f;
    P.sigma = sigma; P.gamma = gamma; P.znear = znear; P.zfar = zfar;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int g = mr::grid_for(npix);
    mr::ProfScope ps(MR_STAGE_BLEND_FWD, s);
    if (D == 3 && (K == 4 || K == 8) && mr::aligned16(pix_to_face) && mr::aligned16(colors) && mr::aligned16(dists) &&
        mr::aligned16(zbuf) && mr::aligned16(rgba)) {
        if (K == 4) mr::k_blend_fwd_rgb<4><<<g, 256, 0, s>>>(pix_to_face, colors, dists, zbuf, npix, P, rgba);
        else mr::k_blend_fwd_rgb<8><<<g, 256, 0, s>>>(pix_to_face, colors, dists, zbuf, npix, P, rgba);
        MR_CUDA(cudaGetLastError());
        return MR_OK;
    }
#define MR_BF(KC) mr::k_blend_fwd<KC><<<g, 256, 0, s>>>(pix_to_face, colors, dists, zbuf, npix, K, D, P, rgba)
    if (K <= 1) MR_BF(1);
    else if (K <= 2) MR_BF(2);
    else if (K <= 4) MR_BF(4);
    else if (K <= 8) MR_BF(8);
    else if (K <= 16) MR_BF(16);
    else MR_BF(32);
#undef MR_BF
    MR_CUDA(cudaGetLastError());
    return MR_OK;
}

int mr_blend_bwd(const int64_t* pix_to_face, const float* colors, const float* dists, const float* zbuf, int64_t npix,
                 int32_t K, int32_t D, const float* background, float sigma, float gamma, float znear, float zfar,
                 const float* grad_rgba, float* grad_colors, float* grad_dists, float* grad_zbuf, void* stream) {
    int rc = mr::check_blend(npix, K, D, sigma, gamma, znear, zfar);
    if (rc != MR_OK || npix == 0) return rc;
    if (!pix_to_face || !colors || !dists || !zbuf || !background || !grad_rgba) {
        mr::set_error("null pointer");
        return MR_ERR_ARG;
    }
    mr::BlendParams P;
    for (int c = 0; c < MR_BLEND_DMAX; ++c) P.bg[c] = c < D ? background[c] : 0.f;
    P.sigma = sigma; P.gamma = gamma; P.znear = znear; P.zfar = zfar;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int g = mr::grid_for(npix);
    mr::ProfScope ps(MR_STAGE_BLEND_BWD, s);
    if (D == 3 && (K == 4 || K == 8) && mr::aligned16(pix_to_face) && mr::aligned16(colors) && mr::aligned16(dists) &&
        mr::aligned16(zbuf) && mr::aligned16(grad_rgba) && mr::aligned16(grad_colors) && mr::aligned16(grad_dists) &&
        mr::aligned16(grad_zbuf)) {
        if (K == 4)
            mr::k_blend_bwd_rgb<4><<<g, 256, 0, s>>>(pix_to_face, colors, dists, zbuf, npix, P, grad_rgba, grad_colors,
                                                     grad_dists, grad_zbuf);
        else
            mr::k_blend_bwd_rgb<8><<<g, 256, 0, s>>>(pix_to_face, colors, dists, zbuf, npix, P, grad_rgba, grad_colors,
                                                     grad_dists, grad_zbuf);
        MR_CUDA(cudaGetLastError());
        return MR_OK;
    }
#define MR_BB(KC)                                                                                          \
    mr::k_blend_bwd<KC><<<g, 256, 0, s>>>(pix_to_face, colors, dists, zbuf, npix, K, D, P, grad_rgba, grad_colors, \
                                          grad_dists, grad_zbuf)
    if (K <= 1) MR_BB(1);
    else if (K <= 2) MR_BB(2);
    else if (K <= 4) MR_BB(4);
    else if (K <= 8) MR_BB(8);
    else if (K <= 16) MR_BB(16);
    else MR_BB(32);
#undef MR_BB
    MR_CUDA(cudaGetLastError());
    return MR_OK;
}

}  // extern "C"
