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
// Contributions are scattered with float32 vector atomics (red.global.add): the general
// kernel adds (x, y, z, 0) rows into a float4 accumulator, the fused silhouette kernel
// (x, y) pairs into a float2 one; a final pass copies either to grad_verts.
#include <algorithm>
#include <cfloat>
#include <cmath>
#include <cstdint>

#include "mr_common.cuh"
#include "mr_silhouette.cuh"

namespace mr {
namespace {

// acc[id] += v for every lane with on set, after summing over runs of equal ids in
// consecutive lanes: consecutive lanes are neighbouring pixels of a row, which usually share
// a face and so its vertices, and atomics to one address serialise in L2 (on the 64-image
// batch the real vertex ids took 0.65 ms where the same number of atomics to spread
// addresses took 0.40).  A segmented suffix sum (shuffles, stopped once no lane still has
// a partner) leaves each run's total in its first lane, which issues the one atomic.  Must
// be called by all 32 lanes of the warp.
__device__ __forceinline__ void warp_run_add(float2* __restrict__ acc, int id, float2 v, bool on, int lane) {
    if (!__ballot_sync(0xffffffffu, on)) return;
    const int key = on ? id : -1;
    const int up = __shfl_up_sync(0xffffffffu, key, 1);
    const bool head = lane == 0 || up != key;
    const unsigned heads = __ballot_sync(0xffffffffu, head);
    if (heads != 0xffffffffu) {
        const unsigned later = lane == 31 ? 0u : (heads & (0xffffffffu << (lane + 1)));
        const int next = later ? __ffs(later) - 1 : 32;   // this run's end (exclusive)
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const bool take = lane + off < next;
            if (!__any_sync(0xffffffffu, take)) break;
            const float ox = __shfl_down_sync(0xffffffffu, v.x, off);
            const float oy = __shfl_down_sync(0xffffffffu, v.y, off);
            if (take) {
                v.x += ox;
                v.y += oy;
            }
        }
    }
    if (on && head) atomicAdd(acc + id, v);
}

__device__ __forceinline__ bool load_face(const int64_t* __restrict__ faces, int64_t V, int64_t f, int64_t (&vid)[3]) {
    vid[0] = faces[3 * f];
    vid[1] = faces[3 * f + 1];
    vid[2] = faces[3 * f + 2];
    return vid[0] >= 0 && vid[0] < V && vid[1] >= 0 && vid[1] < V && vid[2] >= 0 && vid[2] < V;
}

// Chain rule of one slot's barycentric and depth outputs into its three vertices'
// (x, y, z), in arithmetic type T.  r = vertex - pixel centre, w = the edge-function
// weights C_k / A, invA = 1 / A; g[vertex][x, y, z] is added to.
template <typename T, bool PERSP>
__device__ __forceinline__ void bary_z_grad(const T (&rx)[3], const T (&ry)[3], const T (&w)[3], T invA,
                                            const float (&x)[3], const float (&y)[3], const float (&z)[3],
                                            const float (&gbar)[3], float gzz, float (&g)[3][3]) {
    T gw[3];
    if constexpr (PERSP) {
        T u[3], S = 0;
#pragma unroll
        for (int e = 0; e < 3; ++e) { u[e] = w[e] / (T)z[e]; S += u[e]; }
        const T iS = (T)1 / S;
        const T dot = ((T)gbar[0] * u[0] + (T)gbar[1] * u[1] + (T)gbar[2] * u[2]) * iS;
#pragma unroll
        for (int e = 0; e < 3; ++e) {
            const T gu = ((T)gbar[e] - dot) * iS - (T)gzz * iS * iS;
            gw[e] = gu / (T)z[e];
            g[e][2] -= (float)(gu * u[e] / (T)z[e]);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 3; ++e) {
            gw[e] = (T)gzz * (T)z[e] + (T)gbar[e];
            g[e][2] += (float)((T)gzz * w[e]);
        }
    }
    const T G = gw[0] * w[0] + gw[1] * w[1] + gw[2] * w[2];
    // d A / d vertex and sum_k gw_k d C_k / d vertex (C_k = cross of two rows of r)
    const T dA[3][2] = {{(T)y[1] - (T)y[2], (T)x[2] - (T)x[1]}, {(T)y[2] - (T)y[0], (T)x[0] - (T)x[2]},
                        {(T)y[0] - (T)y[1], (T)x[1] - (T)x[0]}};
    const T dc[3][2] = {{gw[2] * ry[1] - gw[1] * ry[2], gw[1] * rx[2] - gw[2] * rx[1]},
                        {gw[0] * ry[2] - gw[2] * ry[0], gw[2] * rx[0] - gw[0] * rx[2]},
                        {gw[1] * ry[0] - gw[0] * ry[1], gw[0] * rx[1] - gw[1] * rx[0]}};
#pragma unroll
    for (int e = 0; e < 3; ++e) {
        g[e][0] += (float)((dc[e][0] - G * dA[e][0]) * invA);
        g[e][1] += (float)((dc[e][1] - G * dA[e][1]) * invA);
    }
}

// One slot's contributions g[vertex][x, y, z] to its face's three vertices (x, y, z:
// their screen-space coordinates), added to g; false for a degenerate face.  The distance part runs in float32 in face-local
// coordinates (vertex minus pixel centre, the centre given as a double and as a float
// pair; near-tied edges re-decided in float64), the barycentric and depth part in float64
// (its terms scale with 1/A and cancel for slivers seen edge-on).
template <bool PERSP>
__device__ __forceinline__ bool slot_grad(const float (&x)[3], const float (&y)[3], const float (&z)[3], double pxd,
                                          double pyd, float pxh, float pyh, float pxl, float pyl, int64_t s,
                                          const float* __restrict__ gz, const float* __restrict__ gb,
                                          const float* __restrict__ gd, float (&g)[3][3]) {
    float rx[3], ry[3];
#pragma unroll
    for (int e = 0; e < 3; ++e) {
        rx[e] = (x[e] - pxh) - pxl;   // vertex - pixel centre
        ry[e] = (y[e] - pyh) - pyl;
    }
    const double Ad = ((double)x[1] - x[0]) * ((double)y[2] - y[0]) - ((double)y[1] - y[0]) * ((double)x[2] - x[0]);
    if (fabs(Ad) <= kDegenerateArea) return false;
    // edge-function weights in float64: the barycentric chain below divides by A and
    // cancels large terms for slivers seen edge-on, which float32 cannot carry
    double rxd[3], ryd[3], wd[3];
#pragma unroll
    for (int e = 0; e < 3; ++e) { rxd[e] = x[e] - pxd; ryd[e] = y[e] - pyd; }
    const double iAd = 1.0 / Ad;
    wd[0] = (rxd[1] * ryd[2] - ryd[1] * rxd[2]) * iAd;
    wd[1] = (rxd[2] * ryd[0] - ryd[2] * rxd[0]) * iAd;
    wd[2] = (rxd[0] * ryd[1] - ryd[0] * rxd[1]) * iAd;
    if (gd) {
        const float gds = gd[s];
        if (gds != 0.f) {
            const bool inside = wd[0] >= 0.0 && wd[1] >= 0.0 && wd[2] >= 0.0;
            int eu = 0, vbest = -1, vsecond = -2;   // nearest point's vertex (-1: inside an edge)
            float best = FLT_MAX, second = FLT_MAX, bt = 0.f, bdx = 0.f, bdy = 0.f;
#pragma unroll
            for (int e = 0; e < 3; ++e) {
                const int e1 = e == 2 ? 0 : e + 1;
                const float ex = x[e1] - x[e], ey = y[e1] - y[e];
                const float ax = -rx[e], ay = -ry[e];        // pixel - edge start
                const float len2 = fmaf(ex, ex, ey * ey);
                const float t = len2 > 0.f ? __saturatef(fmaf(ax, ex, ay * ey) / len2) : 0.f;
                const float dx = fmaf(-t, ex, ax), dy = fmaf(-t, ey, ay);   // pixel - nearest point
                const float d2 = fmaf(dx, dx, dy * dy);
                const int vtx = t == 0.f ? e : (t == 1.f ? e1 : -1 - e);
                if (d2 < best) {
                    second = best;
                    vsecond = vbest;
                    best = d2; eu = e; bt = t; bdx = dx; bdy = dy;
                    vbest = vtx;
                } else if (d2 < second) {
                    second = d2;
                    vsecond = vtx;
                }
            }
            // Two edges almost equally near (the pixel sits on an angle bisector
            // inside the face): float32 may pick the other edge than the exact
            // distances do, and the two picks feed different vertices.  Decide
            // such near-ties again in float64 (rare).  Two edges whose nearest
            // point is the same shared vertex are no tie: both feed that vertex.
            if (second - best <= 1e-5f * best && !(vbest >= 0 && vbest == vsecond)) {
                double bd = DBL_MAX;
#pragma unroll
                for (int e = 0; e < 3; ++e) {
                    const int e1 = e == 2 ? 0 : e + 1;
                    const double ex = (double)x[e1] - x[e], ey = (double)y[e1] - y[e];
                    const double ax = pxd - x[e], ay = pyd - y[e];
                    const double len2 = ex * ex + ey * ey;
                    double t = len2 > 0.0 ? (ax * ex + ay * ey) / len2 : 0.0;
                    t = fmin(fmax(t, 0.0), 1.0);
                    const double dx = ax - t * ex, dy = ay - t * ey;
                    const double d2 = dx * dx + dy * dy;
                    if (d2 < bd) { bd = d2; eu = e; bt = (float)t; bdx = (float)dx; bdy = (float)dy; }
                }
            }
            const int ev = eu == 2 ? 0 : eu + 1;
            const float gdist = inside ? -gds : gds;
            const float su = -2.f * gdist * (1.f - bt), sv = -2.f * gdist * bt;
            g[eu][0] += su * bdx;
            g[eu][1] += su * bdy;
            g[ev][0] += sv * bdx;
            g[ev][1] += sv * bdy;
        }
    }
    if (gb || gz) {
        float gbar[3] = {0.f, 0.f, 0.f};
        if (gb) { gbar[0] = gb[3 * s]; gbar[1] = gb[3 * s + 1]; gbar[2] = gb[3 * s + 2]; }
        const float gzz = gz ? gz[s] : 0.f;
        bary_z_grad<double, PERSP>(rxd, ryd, wd, iAd, x, y, z, gbar, gzz, g);
    }
    return true;
}

// General backward: one thread per pixel, its K slots in turn; each valid slot's
// contributions (slot_grad) go out as one float4 atomic per vertex into a padded
// (x, y, z, 0) accumulator.  Measured alternatives that lost on this scatter: summing
// equal vertex ids within a pixel, or along a run of lanes, before the atomics; issuing
// the K slots' gathers phase by phase (more registers, fewer resident warps); packing the
// valid slots of a warp's pixels into a shared-memory queue so that no lane idles; a
// per-call table of face records (three 16-byte loads per slot instead of the face ids
// and nine scalar vertex loads: 1.74 -> 1.71 ms, not worth its 48 bytes per face).
template <int KC, bool PERSP>
__global__ void __launch_bounds__(256, 4)   // 64 registers: 4 CTAs per SM (measured 1.75 -> 1.63 ms)
k_raster_bwd(const float* __restrict__ verts, int64_t V, const int64_t* __restrict__ faces, int64_t F,
             const int64_t* __restrict__ p2f, int64_t npix, int H, int W, int K, const float* __restrict__ gz,
             const float* __restrict__ gb, const float* __restrict__ gd, float4* __restrict__ acc,
             int* __restrict__ err) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const double inv_w = 1.0 / W, inv_h = 1.0 / H;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < npix; q += stride) {
        int i, j;
        pixel_rc(q, H, W, i, j);
        const double pxd = pixel_x(j, W, inv_w), pyd = pixel_y(i, H, inv_h);
        const float pxh = (float)pxd, pyh = (float)pyd;
        const float pxl = (float)(pxd - (double)pxh), pyl = (float)(pyd - (double)pyh);
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            if (k >= K) break;
            const int64_t s = q * K + k;
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
            float x[3], y[3], z[3];
#pragma unroll
            for (int e = 0; e < 3; ++e) {
                x[e] = verts[3 * vid[e]];
                y[e] = verts[3 * vid[e] + 1];
                z[e] = verts[3 * vid[e] + 2];
            }
            float g[3][3] = {{0.f, 0.f, 0.f}, {0.f, 0.f, 0.f}, {0.f, 0.f, 0.f}};   // [vertex][x, y, z]
            if (!slot_grad<PERSP>(x, y, z, pxd, pyd, pxh, pyh, pxl, pyl, s, gz, gb, gd, g)) continue;
#pragma unroll
            for (int e = 0; e < 3; ++e)
                if (g[e][0] != 0.f || g[e][1] != 0.f || g[e][2] != 0.f)
                    atomicAdd(acc + vid[e], make_float4(g[e][0], g[e][1], g[e][2], 0.f));
        }
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
// end points receive -2 (p - q)(1 - t) and -2 (p - q) t times dL/ddist.  EXACT: H and W are
// powers of two, so 1/W and 1/H are exact, the pixel centres exact float32 values and their
// float-float low parts 0.  VEC: K == KC and 16-byte aligned rows, so a pixel's K ids and
// distances come in 16-byte loads (on the 64-image batch, K = 4: 0.557 -> 0.542 ms, the
// sums equal up to the order of the atomics).
template <int KC, bool EXACT, bool VEC>
__global__ void __launch_bounds__(256, 6)   // 40 registers: 6 CTAs per SM (4 / 5 / 8: 0.619 / 0.567 / 0.597 ms)
k_sil_raster_bwd(const float* __restrict__ verts, int64_t V, const int64_t* __restrict__ faces, int64_t F,
                 const int64_t* __restrict__ p2f, const float* __restrict__ dists,
                 const float* __restrict__ grad_alpha, int64_t npix, int H, int W, int K, float sigma,
                 float2* __restrict__ acc, int* __restrict__ err) {
    const int lane = threadIdx.x & 31;
    const bool small = npix <= 0x7fffffff;                  // pixel ids fit 32-bit division
    const unsigned hw = (unsigned)H * (unsigned)W;
    const double inv_w = 1.0 / W, inv_h = 1.0 / H;
    const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t base = wid * 32; base < npix; base += nw * 32) {
        const int64_t q = base + lane;
        const bool live = q < npix;
        float d[KC], g[KC];
        bool v[KC];
        int64_t fk[KC];
        int ebits = 0;   // error flags of this pixel, set in the device word once at the end
        bool work = false;
        if constexpr (VEC) {
            static_assert(KC % 4 == 0, "16-byte loads of the ids in pairs, of the distances in fours");
            if (live) {
#pragma unroll
                for (int k = 0; k < KC; k += 2) {
                    const longlong2 pr = *reinterpret_cast<const longlong2*>(p2f + q * KC + k);
                    fk[k] = pr.x;
                    fk[k + 1] = pr.y;
                }
            } else {
#pragma unroll
                for (int k = 0; k < KC; ++k) fk[k] = -1;
            }
        } else {
#pragma unroll
            for (int k = 0; k < KC; ++k) fk[k] = live && k < K ? p2f[q * K + k] : -1;
        }
#pragma unroll
        for (int k = 0; k < KC; ++k) work |= fk[k] != -1;
        // a warp of pixels with every slot empty (background) has nothing to add: skip its
        // distance and dL/dalpha reads and the arithmetic
        if (!__any_sync(0xffffffffu, work)) continue;
        if constexpr (VEC) {
#pragma unroll
            for (int k = 0; k < KC; k += 4) {
                const float4 dv = live ? *reinterpret_cast<const float4*>(dists + q * KC + k)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
                d[k] = dv.x;
                d[k + 1] = dv.y;
                d[k + 2] = dv.z;
                d[k + 3] = dv.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < KC; ++k) d[k] = live && k < K ? dists[q * K + k] : 0.f;
        }
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            if (fk[k] < -1) ebits |= kErrSlotIndex;
            v[k] = fk[k] >= 0;
        }
        const float ga = live ? grad_alpha[q] : 0.f;
        silhouette_grad<KC>(d, v, K, sigma, ga, g);
        int i, j;
        if (small) {
            const unsigned rem = (unsigned)(live ? q : 0) % hw;
            i = (int)(rem / (unsigned)W);
            j = (int)(rem - (unsigned)i * (unsigned)W);
        } else {
            const int64_t rem = (live ? q : 0) % ((int64_t)H * W);
            i = (int)(rem / W);
            j = (int)(rem % W);
        }
        const double pxd = EXACT ? (double)(2 * j + 1 - W) * inv_w : -1.0 + (2.0 * j + 1.0) / W;
        const double pyd = EXACT ? (double)(H - 2 * i - 1) * inv_h : 1.0 - (2.0 * i + 1.0) / H;
        const float pxh = (float)pxd, pyh = (float)pyd;
        const float pxl = EXACT ? 0.f : (float)(pxd - (double)pxh), pyl = EXACT ? 0.f : (float)(pyd - (double)pyh);
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
                    ebits |= kErrSlotIndex;
                    act = false;
                } else if (!load_face(faces, V, fk[k], vid)) {
                    ebits |= kErrFaceIndex;
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
                        const float ax = EXACT ? pxh - x[e] : (pxh - x[e]) + pxl;
                        const float ay = EXACT ? pyh - y[e] : (pyh - y[e]) + pyl;
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
        // always differ), then over runs of equal ids in neighbouring lanes, then one
        // float2 atomic per run (up to K = 8; larger K would spend more registers on the
        // comparisons than the atomics cost).
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
        for (int t = 0; t < (KC <= 8 ? NT : 0); ++t) warp_run_add(acc, tid[t], tv[t], alive[t], lane);
        if (ebits) atomicOr(err, ebits);
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
        const int64_t npix = (int64_t)N * H * W;
        const int g = mr::grid_for(npix);
        mr::ProfScope ps(MR_STAGE_RASTER_BWD, s);
#define MR_RB(KC, PC)                                                                                           \
    mr::k_raster_bwd<KC, PC><<<g, 256, 0, s>>>(verts, V, faces, F, pix_to_face, npix, H, W, K, grad_zbuf, grad_bary, \
                                               grad_dists, acc, err)
#define MR_RB_K(PC)               \
    if (K <= 1) MR_RB(1, PC);     \
    else if (K <= 2) MR_RB(2, PC); \
    else if (K <= 4) MR_RB(4, PC); \
    else if (K <= 8) MR_RB(8, PC); \
    else if (K <= 16) MR_RB(16, PC); \
    else MR_RB(32, PC)
        if (perspective_correct) {
            MR_RB_K(true);
        } else {
            MR_RB_K(false);
        }
#undef MR_RB_K
#undef MR_RB
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
        // 148 x 64 blocks of 256 (0.561 -> 0.558 ms against 148 x 32)
        const int g = (int)std::min<int64_t>((npix + 255) / 256, 148 * 64);
        mr::ProfScope ps(MR_STAGE_SILHOUETTE_RASTER_BWD, s);
        const bool exact = (H & (H - 1)) == 0 && (W & (W - 1)) == 0;
        // 16-byte loads of each pixel's ids and distances (K = 4, the rows aligned; K = 8
        // spills more in that form and was not measured faster)
        const bool vec = K == 4 &&
                         ((reinterpret_cast<uintptr_t>(pix_to_face) | reinterpret_cast<uintptr_t>(dists)) & 15) == 0;
#define MR_SRB3(KC, X, VC)                                                                                  \
    mr::k_sil_raster_bwd<KC, X, VC><<<g, 256, 0, s>>>(verts, V, faces, F, pix_to_face, dists, grad_alpha, npix, \
                                                      H, W, K, sigma, acc, err)
#define MR_SRB(KC)                     \
    if (exact) MR_SRB3(KC, true, false); \
    else MR_SRB3(KC, false, false)
#define MR_SRBV(KC)                                    \
    if (vec && exact) MR_SRB3(KC, true, true);         \
    else if (vec) MR_SRB3(KC, false, true);            \
    else MR_SRB(KC)
        if (K <= 1) { MR_SRB(1); }
        else if (K <= 2) { MR_SRB(2); }
        else if (K <= 4) { MR_SRBV(4); }
        else if (K <= 8) { MR_SRB(8); }
        else if (K <= 16) { MR_SRB(16); }
        else { MR_SRB(32); }
#undef MR_SRBV
#undef MR_SRB
#undef MR_SRB3
        mr::k_xy_to_xyz<<<mr::grid_for(V), 256, 0, s>>>(acc, V, grad_verts);
        e = cudaGetLastError();
    }
    mr::scratch_free(acc, s);
    if (e != cudaSuccess) return mr::cuda_fail(e, "silhouette-rasterizer backward launch");
    return MR_OK;
}

}  // extern "C"
