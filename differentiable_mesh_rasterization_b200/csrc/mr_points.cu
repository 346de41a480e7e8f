// The point-cloud renderer ("Accelerating 3D Deep Learning with PyTorch3D": the same
// two-stage renderer draws point clouds as well as meshes, over heterogeneous batches).
//
// Stage one, for every pixel of image n: the K points of cloud n nearest in depth among
// those with z >= 0 whose squared 2-D distance to the pixel centre is at most r^2, ordered
// by (z, point id); idx (global point id), zbuf = z, dists = squared distance; -1 pads.
// Stage two composites per-point features over those K slots with weights
// a_k = 1 - dists_k / r^2: front-to-back alpha compositing (out = sum a_k T_k f_k,
// T_k = prod_{j<k} (1 - a_j)) or the norm-weighted sum (sum a_k f_k / max(sum a_k, 1e-4)).
//
// Pipeline: points are binned into 16 x 16-pixel screen bins of their image (count ->
// exclusive scan -> one stream sync for the total -> fill, like the mesh path); one CTA per
// bin then stages the bin's points in shared memory in chunks of 256 and every thread
// (one pixel) keeps its K nearest in registers; 16-byte stores write the slots.
#include <algorithm>
#include <cfloat>
#include <cmath>
#include <vector>

#include "mr_common.cuh"
#include "mr_scan.cuh"

namespace mr {
namespace {

constexpr int kPtBin = 16;          // bin side in pixels (one 256-thread CTA per bin)
constexpr float kNormFloor = 1e-4f;

// Image of point p: the cloud whose range [first, first + num) holds it (binary search
// over the cloud starts, which are ascending), or -1.
__device__ __forceinline__ int cloud_of(int64_t p, const int64_t* __restrict__ first, const int64_t* __restrict__ num,
                                       int N) {
    int lo = 0, hi = N - 1, n = -1;
    while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        if (first[mid] <= p) {
            n = mid;
            lo = mid + 1;
        } else {
            hi = mid - 1;
        }
    }
    return n >= 0 && p < first[n] + num[n] ? n : -1;
}

// Inclusive pixel ranges whose centres lie within r of (x, y), widened by 1e-5 NDC so that
// every pixel the float32 test can accept is inside; false if empty.
__device__ __forceinline__ bool point_box(float x, float y, float r, int H, int W, int& j0, int& j1, int& i0,
                                          int& i1) {
    const double rr = (double)r + 1e-5;
    const double a = ((double)x - rr + 1.0) * W * 0.5 - 0.5, b = ((double)x + rr + 1.0) * W * 0.5 - 0.5;
    const double c = (1.0 - (double)y - rr) * H * 0.5 - 0.5, d = (1.0 - (double)y + rr) * H * 0.5 - 0.5;
    if (!(b >= 0.0) || !(a <= W - 1.0) || !(d >= 0.0) || !(c <= H - 1.0)) return false;   // also NaN
    j0 = (int)fmax(ceil(a), 0.0);
    j1 = (int)fmin(floor(b), W - 1.0);
    i0 = (int)fmax(ceil(c), 0.0);
    i1 = (int)fmin(floor(d), H - 1.0);
    return j0 <= j1 && i0 <= i1;
}

template <bool FILL>
__global__ void k_point_bins(const float* __restrict__ pts, int64_t P, const int64_t* __restrict__ first,
                             const int64_t* __restrict__ num, int N, int H, int W, float r, int nbx, int nby,
                             int* __restrict__ counts, const int* __restrict__ offsets, int* __restrict__ list) {
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < P; p += (int64_t)gridDim.x * blockDim.x) {
        const int n = cloud_of(p, first, num, N);
        if (n < 0) continue;
        const float x = pts[3 * p], y = pts[3 * p + 1], z = pts[3 * p + 2];
        if (!(z >= 0.f)) continue;
        int j0, j1, i0, i1;
        if (!point_box(x, y, r, H, W, j0, j1, i0, i1)) continue;
        for (int by = i0 / kPtBin; by <= i1 / kPtBin; ++by)
            for (int bx = j0 / kPtBin; bx <= j1 / kPtBin; ++bx) {
                const int b = (n * nby + by) * nbx + bx;
                const int at = atomicAdd(counts + b, 1);
                if (FILL) list[offsets[b] + at] = (int)p;
            }
    }
}

// A slot key: the depth's bits above the point id.  Depths here are >= 0 (negative ones
// never reach the fine pass and -0 is made +0), and non-negative floats order like their
// bits, so one 64-bit compare orders (z, id).  kEmpty sorts after every point.
constexpr unsigned long long kEmpty = (0x7F7FFFFFull << 32) | 0xFFFFFFFFull;

__device__ __forceinline__ unsigned long long point_key(float z, int id) {
    return ((unsigned long long)__float_as_uint(z + 0.f) << 32) | (unsigned)id;
}

// Sorted insertion of (key, d2) into a register list of KC entries (the caller has checked
// key < the list's last key).
template <int KC>
__device__ __forceinline__ void insert_point(unsigned long long (&kk)[KC], float (&kd)[KC], unsigned long long key,
                                             float d2) {
#pragma unroll
    for (int k = KC - 1; k > 0; --k) {
        const bool shift = key < kk[k - 1];
        const bool here = !shift && key < kk[k];
        kk[k] = shift ? kk[k - 1] : (here ? key : kk[k]);
        kd[k] = shift ? kd[k - 1] : (here ? d2 : kd[k]);
    }
    if (key < kk[0]) {
        kk[0] = key;
        kd[0] = d2;
    }
}

// One pixel's K slots from its register list (16-byte stores when K is a multiple of 4 and
// the outputs are 16-byte aligned).
template <int KC>
__device__ __forceinline__ void write_point_slots(const unsigned long long (&kk)[KC], const float (&kd)[KC], int K,
                                                  int64_t o, bool vec, int64_t* __restrict__ idx,
                                                  float* __restrict__ zbuf, float* __restrict__ dists) {
    long long v[KC];
    float z[KC], d[KC];
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        const bool ok = kk[k] != kEmpty;
        v[k] = ok ? (long long)(unsigned)(kk[k] & 0xffffffffu) : -1;
        z[k] = ok ? __uint_as_float((unsigned)(kk[k] >> 32)) : -1.f;
        d[k] = ok ? kd[k] : -1.f;
    }
    if constexpr (KC >= 4) {
        if (vec && (K & 3) == 0) {
#pragma unroll
            for (int k = 0; k < KC; k += 4) {
                if (k >= K) break;
                reinterpret_cast<longlong2*>(idx + o + k)[0] = make_longlong2(v[k], v[k + 1]);
                reinterpret_cast<longlong2*>(idx + o + k)[1] = make_longlong2(v[k + 2], v[k + 3]);
                *reinterpret_cast<float4*>(zbuf + o + k) = make_float4(z[k], z[k + 1], z[k + 2], z[k + 3]);
                *reinterpret_cast<float4*>(dists + o + k) = make_float4(d[k], d[k + 1], d[k + 2], d[k + 3]);
            }
            return;
        }
    }
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        if (k >= K) break;
        idx[o + k] = v[k];
        zbuf[o + k] = z[k];
        dists[o + k] = d[k];
    }
}

// Fine pass: one CTA of 256 threads per 16 x 16 bin, one thread per pixel; the bin's
// points are staged in shared memory 256 at a time and every thread keeps its K nearest in
// registers.  While staging, each point's pixel box (the one that binned it) is tested
// against the eight 4 x 8 warp tiles of the bin; every warp then compacts the staged
// points whose box meets its tile (ballot) and tests only those.  Measured and rejected:
// a bounded grid walking the bins (load imbalance, 1.45 vs 1.13 ms on the benchmark
// batch) and sorting each chunk by depth in shared memory so that a full list can stop
// early (1.53 ms: the warp waits for its slowest lane).
template <int KC>
__global__ void __launch_bounds__(256, KC <= 8 ? 5 : 1) k_point_fine(const float* __restrict__ pts, const int* __restrict__ offsets,
                                                    const int* __restrict__ list, int H, int W, float r, float r2,
                                                    int K, int nbx, int nby, int64_t* __restrict__ idx,
                                                    float* __restrict__ zbuf, float* __restrict__ dists, bool vec,
                                                    double inv_w, double inv_h) {
    __shared__ float4 sp[256];
    __shared__ unsigned char smask[256];          // bit w: the point's box meets warp w's tile
    __shared__ unsigned char wl[8][256];          // per warp: its staged points, compacted
    const int b = blockIdx.x;
    const int n = b / (nbx * nby), by = (b / nbx) % nby, bx = b % nbx;
    // each warp takes a 4 x 8 block of the bin (a point's disc meets fewer warps than with
    // 2 x 16 rows, so fewer warps run the insertion for it)
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = by * kPtBin + (w >> 1) * 4 + (lane >> 3), j = bx * kPtBin + (w & 1) * 8 + (lane & 7);
    unsigned long long kk[KC];
    float kd[KC];
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        kk[k] = kEmpty;
        kd[k] = -1.f;
    }
    const int beg = offsets[b], end = offsets[b + 1];
    if (beg == end) {                             // an empty bin (the whole CTA): padding only
        if (i < H && j < W)
            write_point_slots<KC>(kk, kd, K, (((int64_t)n * H + i) * W + j) * K, vec, idx, zbuf, dists);
        return;
    }
    // pixel centre as a float pair (hi + lo): the offset to a point is then exact to ~1e-15
    const double pxd = pixel_x(j, W, inv_w), pyd = pixel_y(i, H, inv_h);
    const float pxh = (float)pxd, pyh = (float)pyd;
    const float pxl = (float)(pxd - (double)pxh), pyl = (float)(pyd - (double)pyh);
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int c0 = beg; c0 < end; c0 += 256) {
        __syncthreads();
        unsigned mask = 0;
        if (c0 + (int)threadIdx.x < end) {
            const int p = list[c0 + threadIdx.x];
            const float x = pts[3 * (int64_t)p], y = pts[3 * (int64_t)p + 1];
            sp[threadIdx.x] = make_float4(x, y, pts[3 * (int64_t)p + 2], __int_as_float(p));
            // pixel ranges whose centres lie within r + 2e-5 of the point, in float32: the
            // margin (2e-5 NDC) is far above the rounding of these few operations, so the
            // ranges hold every pixel the test below can accept
            const float R = r + 2e-5f, hw = 0.5f * W, hh = 0.5f * H;
            const int j0 = (int)ceilf((x - R + 1.f) * hw - 0.5f), j1 = (int)floorf((x + R + 1.f) * hw - 0.5f);
            const int i0 = (int)ceilf((1.f - y - R) * hh - 0.5f), i1 = (int)floorf((1.f - y + R) * hh - 0.5f);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const int ti = by * kPtBin + (v >> 1) * 4, tj = bx * kPtBin + (v & 1) * 8;
                if (j0 <= tj + 7 && j1 >= tj && i0 <= ti + 3 && i1 >= ti) mask |= 1u << v;
            }
        }
        smask[threadIdx.x] = (unsigned char)mask;
        __syncthreads();
        int nw = 0;                               // this warp's points of the chunk
#pragma unroll
        for (int s0 = 0; s0 < 256; s0 += 32) {
            const bool mine = (smask[s0 + lane] >> w) & 1u;
            const unsigned bal = __ballot_sync(0xffffffffu, mine);
            if (mine) wl[w][nw + __popc(bal & lt_mask)] = (unsigned char)(s0 + lane);
            nw += __popc(bal);
        }
        __syncwarp();
        for (int u = 0; u < nw; ++u) {
            const float4 q = sp[wl[w][u]];
            const float dx = (pxh - q.x) + pxl, dy = (pyh - q.y) + pyl;
            const float d2 = fmaf(dx, dx, dy * dy);
            const unsigned long long key = point_key(q.z, __float_as_int(q.w));
            if (d2 <= r2 && key < kk[KC - 1]) insert_point<KC>(kk, kd, key, d2);
        }
    }
    if (i < H && j < W)
        write_point_slots<KC>(kk, kd, K, (((int64_t)n * H + i) * W + j) * K, vec, idx, zbuf, dists);
}

// Backward of the point rasterizer: thread per slot, one float4 (x, y, z, 0) atomic per
// valid slot into a padded accumulator.
__global__ void k_point_raster_bwd(const float* __restrict__ pts, int64_t P, const int64_t* __restrict__ idx,
                                   int64_t nslots, int H, int W, int K, const float* __restrict__ gz,
                                   const float* __restrict__ gd, float4* __restrict__ acc, int* __restrict__ err) {
    for (int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; s < nslots; s += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = idx[s];
        if (m == -1) continue;
        if (m < -1 || m >= P) {
            atomicOr(err, kErrSlotIndex);
            continue;
        }
        float4 c = make_float4(0.f, 0.f, gz ? gz[s] : 0.f, 0.f);
        if (gd) {
            const int64_t rem = (s / K) % ((int64_t)H * W);
            const int i = (int)(rem / W), j = (int)(rem % W);
            const double pxd = -1.0 + (2.0 * j + 1.0) / W, pyd = 1.0 - (2.0 * i + 1.0) / H;
            const float g = gd[s];
            c.x = -2.f * g * (float)(pxd - (double)pts[3 * m]);
            c.y = -2.f * g * (float)(pyd - (double)pts[3 * m + 1]);
        }
        if (c.x != 0.f || c.y != 0.f || c.z != 0.f) atomicAdd(acc + m, c);
    }
}

__global__ void k_xyzw_rows(const float4* __restrict__ acc, int64_t P, float* __restrict__ out) {
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < P; p += (int64_t)gridDim.x * blockDim.x) {
        const float4 a = acc[p];
        out[3 * p] = a.x;
        out[3 * p + 1] = a.y;
        out[3 * p + 2] = a.z;
    }
}

// r^2 as a float pair and 1/r^2: a = 1 - d / r^2 is formed as ((r2h - d) + r2l) / r^2, so
// that a keeps its relative accuracy where it is small (a point near the radius; the
// norm-weighted sum divides by sum a down to the 1e-4 floor).
struct Radius2 {
    float h, l, inv;
};

__device__ __forceinline__ float point_weight(float d, const Radius2& R) { return ((R.h - d) + R.l) * R.inv; }

inline Radius2 radius2(float radius) {
    const double r2 = (double)radius * radius;
    Radius2 R;
    R.h = (float)r2;
    R.l = (float)(r2 - (double)R.h);
    R.inv = (float)(1.0 / r2);
    return R;
}

// Compositing, thread per pixel.  MODE 0: alpha, 1: norm-weighted.
// A pixel's K slot ids and distances: 16-byte loads when VEC (K == KC, a multiple of 4,
// aligned arrays), else element-wise.
template <int KC, bool VEC>
__device__ __forceinline__ void load_slots(const int64_t* __restrict__ idx, const float* __restrict__ dists, int64_t q,
                                           int K, int64_t (&m)[KC], float (&d)[KC]) {
    if constexpr (VEC) {
        ld_vec<KC>(idx + q * KC, m);
        ld_vec<KC>(dists + q * KC, d);
    } else {
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            m[k] = k < K ? idx[q * K + k] : -1;
            d[k] = m[k] >= 0 ? dists[q * K + k] : 0.f;
        }
    }
}

template <int KC, int MODE, bool VEC>
__global__ void k_composite_fwd(const int64_t* __restrict__ idx, const float* __restrict__ dists, int64_t npix, int K,
                                const float* __restrict__ feat, int64_t P, int C, Radius2 R,
                                float* __restrict__ out, int* __restrict__ err) {
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < npix; q += (int64_t)gridDim.x * blockDim.x) {
        int64_t m[KC];
        float w[KC], dv[KC];
        float T = 1.f, wsum = 0.f;
        load_slots<KC, VEC>(idx, dists, q, K, m, dv);
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            if (m[k] < -1 || m[k] >= P) {
                atomicOr(err, kErrSlotIndex);
                m[k] = -1;
            }
            const float a = m[k] >= 0 ? point_weight(dv[k], R) : 0.f;
            w[k] = MODE == 0 ? a * T : a;
            T *= 1.f - a;
            wsum += a;
        }
        const float scale = MODE == 0 ? 1.f : 1.f / fmaxf(wsum, kNormFloor);
        for (int c = 0; c < C; ++c) {
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < KC; ++k)
                if (m[k] >= 0) acc = fmaf(w[k], feat[m[k] * C + c], acc);
            out[q * C + c] = acc * scale;
        }
    }
}

// Backward of the compositing.  Alpha: with R_k = the composite behind slot k relative to
// the transmittance after it (R_last = 0, R_{k-1} = a_k (f_k . g) + (1 - a_k) R_k),
// dL/da_k = T_k ((f_k . g) - R_k) -- no division by 1 - a_k.  Norm-weighted:
// dL/da_k = (f_k - out) . g / den (den = sum a > floor) or f_k . g / den.  Feature
// gradients w_k g go to a padded accumulator (float4 per point for C <= 4, else scalars).
template <int KC, int MODE, bool VEC4, bool VEC>
__global__ void k_composite_bwd(const int64_t* __restrict__ idx, const float* __restrict__ dists, int64_t npix, int K,
                                const float* __restrict__ feat, int64_t P, int C, Radius2 R,
                                const float* __restrict__ grad_out, float* __restrict__ gfeat,
                                float4* __restrict__ gfeat4, float* __restrict__ grad_dists, int* __restrict__ err) {
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < npix; q += (int64_t)gridDim.x * blockDim.x) {
        int64_t m[KC];
        float a[KC], T[KC], fg[KC], dv[KC], gdv[KC];
        float t = 1.f, wsum = 0.f;
        load_slots<KC, VEC>(idx, dists, q, K, m, dv);
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            if (m[k] < -1 || m[k] >= P) {
                atomicOr(err, kErrSlotIndex);
                m[k] = -1;
            }
            a[k] = m[k] >= 0 ? point_weight(dv[k], R) : 0.f;
            T[k] = t;
            t *= 1.f - a[k];
            wsum += a[k];
            fg[k] = 0.f;
        }
        const float den = fmaxf(wsum, kNormFloor);
        const float inv_den = 1.f / den;
        float og = 0.f;              // out . g (norm-weighted)
        for (int c = 0; c < C; ++c) {
            const float g = grad_out[q * C + c];
            float o = 0.f;
#pragma unroll
            for (int k = 0; k < KC; ++k)
                if (m[k] >= 0) {
                    const float f = feat[m[k] * C + c];
                    fg[k] = fmaf(f, g, fg[k]);
                    o = fmaf(a[k], f, o);
                }
            og = fmaf(o * inv_den, g, og);
        }
        float rest = 0.f;            // R_k of the comment above
#pragma unroll
        for (int k = KC - 1; k >= 0; --k) {
            float ga = 0.f;
            if (m[k] >= 0) {
                if (MODE == 0) ga = T[k] * (fg[k] - rest);
                else ga = (wsum > kNormFloor ? fg[k] - og : fg[k]) * inv_den;
                if (MODE == 0) rest = fmaf(a[k], fg[k], (1.f - a[k]) * rest);
                const float wk = MODE == 0 ? a[k] * T[k] : a[k] * inv_den;
                if (VEC4) {
                    float g4[4] = {0.f, 0.f, 0.f, 0.f};
                    for (int c = 0; c < C; ++c) g4[c] = wk * grad_out[q * C + c];
                    atomicAdd(gfeat4 + m[k], make_float4(g4[0], g4[1], g4[2], g4[3]));
                } else {
                    for (int c = 0; c < C; ++c) atomicAdd(gfeat + m[k] * C + c, wk * grad_out[q * C + c]);
                }
            }
            gdv[k] = -ga * R.inv;
            if (!VEC && grad_dists && k < K) grad_dists[q * K + k] = gdv[k];
        }
        if (VEC && grad_dists) st_vec<KC>(grad_dists + q * KC, gdv);
    }
}

__global__ void k_acc4_cols(const float4* __restrict__ acc, int64_t P, int C, float* __restrict__ out) {
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < P; p += (int64_t)gridDim.x * blockDim.x) {
        const float4 a = acc[p];
        const float x[4] = {a.x, a.y, a.z, a.w};
        for (int c = 0; c < C; ++c) out[p * C + c] = x[c];
    }
}

int check_clouds(const int64_t* first, const int64_t* num, int N, int64_t P, const char* what) {
    for (int n = 0; n < N; ++n) {
        if (first[n] < 0 || num[n] < 0 || first[n] + num[n] > P || (n > 0 && first[n] < first[n - 1] + num[n - 1])) {
            set_error("%s: cloud %d range [%lld, %lld) outside [0, %lld) or not ascending", what, n,
                      (long long)first[n], (long long)(first[n] + num[n]), (long long)P);
            return MR_ERR_ARG;
        }
    }
    return MR_OK;
}

}  // namespace
}  // namespace mr

extern "C" {

int mr_rasterize_points_fwd(const float* points, int64_t P, const int64_t* cloud_first_idx,
                            const int64_t* num_points_per_cloud, int32_t N, int32_t H, int32_t W, float radius,
                            int32_t K, int64_t* idx, float* zbuf, float* dists, void* stream) {
    using namespace mr;
    if (N < 0 || H < 1 || W < 1 || H > MR_MAX_SIDE || W > MR_MAX_SIDE || K < 1 || K > MR_KMAX || P < 0 ||
        P > INT32_MAX || !(radius >= 0.f) || !std::isfinite(radius)) {
        set_error("invalid arguments N=%d H=%d W=%d K=%d P=%lld radius=%g", N, H, W, K, (long long)P, (double)radius);
        return MR_ERR_ARG;
    }
    if (N == 0) return MR_OK;
    if (!cloud_first_idx || !num_points_per_cloud || !idx || !zbuf || !dists || (P > 0 && !points)) {
        set_error("null pointer");
        return MR_ERR_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    std::vector<int64_t> staged;
    int rc = host_indices(s, N, staged, {&cloud_first_idx, &num_points_per_cloud});
    if (rc != MR_OK) return rc;
    rc = check_clouds(cloud_first_idx, num_points_per_cloud, N, P, "mr_rasterize_points_fwd");
    if (rc != MR_OK) return rc;
    const int nbx = (W + kPtBin - 1) / kPtBin, nby = (H + kPtBin - 1) / kPtBin;
    const int64_t nbins64 = (int64_t)N * nbx * nby;
    if (nbins64 >= INT32_MAX / 2) {
        set_error("too many bins");
        return MR_ERR_ARG;
    }
    const int nbins = (int)nbins64;
    const int ntiles = (nbins + kScanTile - 1) / kScanTile;
    // scratch: cloud ranges, counts, offsets (+1), tile sums, total
    const size_t sz_cl = sizeof(int64_t) * 2 * (size_t)N, sz_cnt = sizeof(int) * (size_t)nbins,
                 sz_off = sizeof(int) * ((size_t)nbins + 1), sz_tile = sizeof(long long) * ((size_t)ntiles + 1);
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t bytes = up(sz_cl) + up(sz_cnt) + up(sz_off) + up(sz_tile);
    char* base = nullptr;
    rc = scratch_alloc(reinterpret_cast<void**>(&base), bytes, s);
    if (rc != MR_OK) return rc;
    int64_t* cl = reinterpret_cast<int64_t*>(base);
    int* counts = reinterpret_cast<int*>(base + up(sz_cl));
    int* offsets = reinterpret_cast<int*>(base + up(sz_cl) + up(sz_cnt));
    long long* tile = reinterpret_cast<long long*>(base + up(sz_cl) + up(sz_cnt) + up(sz_off));
    long long* total_d = tile + ntiles;
    // the per-cloud arrays through pinned staging when it can be had (a copy from pageable
    // memory may first wait for the stream); the synchronisation below completes the copy
    std::vector<int64_t> host;
    int64_t* hs = static_cast<int64_t*>(host_staging(sizeof(int64_t) * 2 * (size_t)N));
    if (!hs) {
        host.resize(2 * (size_t)N);
        hs = host.data();
    }
    std::copy(cloud_first_idx, cloud_first_idx + N, hs);
    std::copy(num_points_per_cloud, num_points_per_cloud + N, hs + N);
    int* list = nullptr;
    long long total = 0;
    cudaError_t e = cudaMemcpyAsync(cl, hs, sz_cl, cudaMemcpyHostToDevice, s);
    const float r2 = radius * radius;
    const int gp = grid_for(std::max<int64_t>(P, 1));
    if (e == cudaSuccess) e = cudaMemsetAsync(counts, 0, sz_cnt, s);
    if (e == cudaSuccess) {
        ProfScope ps(MR_STAGE_POINTS_BIN, s);
        if (P > 0)
            k_point_bins<false><<<gp, 256, 0, s>>>(points, P, cl, cl + N, N, H, W, radius, nbx, nby, counts, nullptr,
                                                   nullptr);
        k_scan_tiles<<<ntiles, 1024, 0, s>>>(counts, nbins, offsets, tile);
        k_scan_tops<<<1, 1024, 0, s>>>(tile, ntiles, total_d);
        k_scan_add<<<std::min((nbins + 256) / 256, 148 * 8), 256, 0, s>>>(offsets, nbins, tile, total_d);
        e = cudaGetLastError();
    }
    // the one sync: the list's size, read back without a copy engine when a mapped host
    // word is at hand
    const Mailbox mb = host_mailbox();
    if (e == cudaSuccess)
        e = mb.dev ? post_counts(total_d, nullptr, nullptr, mb.dev, s)
                   : cudaMemcpyAsync(&total, total_d, sizeof(long long), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess && mb.dev) total = mb.host[0];
    if (e == cudaSuccess && total > INT32_MAX) {
        scratch_free(base, s);
        set_error("%lld point-bin entries exceed the int32 list (radius too large for this batch)", total);
        return MR_ERR_ARG;
    }
    if (e == cudaSuccess && total > 0) {
        rc = scratch_alloc(reinterpret_cast<void**>(&list), sizeof(int) * (size_t)total, s);
        if (rc != MR_OK) {
            scratch_free(base, s);
            return rc;
        }
        e = cudaMemsetAsync(counts, 0, sz_cnt, s);
        if (e == cudaSuccess) {
            ProfScope ps(MR_STAGE_POINTS_BIN, s);
            k_point_bins<true><<<gp, 256, 0, s>>>(points, P, cl, cl + N, N, H, W, radius, nbx, nby, counts, offsets,
                                                  list);
            e = cudaGetLastError();
        }
    }
    if (e == cudaSuccess) {
        const bool vec = (reinterpret_cast<uintptr_t>(idx) & 15) == 0 && (reinterpret_cast<uintptr_t>(zbuf) & 15) == 0 &&
                         (reinterpret_cast<uintptr_t>(dists) & 15) == 0;
        ProfScope ps(MR_STAGE_POINTS_FINE, s);
#define MR_PF(KC) \
    k_point_fine<KC><<<nbins, 256, 0, s>>>(points, offsets, list, H, W, radius, r2, K, nbx, nby, idx, zbuf, dists, vec, \
                                           1.0 / W, 1.0 / H)
        if (K <= 1) MR_PF(1);
        else if (K <= 2) MR_PF(2);
        else if (K <= 4) MR_PF(4);
        else if (K <= 8) MR_PF(8);
        else if (K <= 16) MR_PF(16);
        else MR_PF(32);
#undef MR_PF
        e = cudaGetLastError();
    }
    if (list) scratch_free(list, s);
    scratch_free(base, s);
    if (e != cudaSuccess) return cuda_fail(e, "point rasterization");
    return MR_OK;
}

int mr_rasterize_points_bwd(const float* points, int64_t P, const int64_t* idx, int32_t N, int32_t H, int32_t W,
                            int32_t K, const float* grad_zbuf, const float* grad_dists, float* grad_points,
                            void* stream) {
    using namespace mr;
    if (N < 0 || H < 1 || W < 1 || K < 1 || K > MR_KMAX || P < 0) {
        set_error("invalid shape");
        return MR_ERR_ARG;
    }
    if (P > 0 && (!points || !grad_points)) {
        set_error("null point pointer");
        return MR_ERR_ARG;
    }
    if (P == 0) return MR_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t nslots = (int64_t)N * H * W * K;
    if (nslots == 0 || (!grad_zbuf && !grad_dists)) {
        MR_CUDA(cudaMemsetAsync(grad_points, 0, sizeof(float) * 3 * (size_t)P, s));
        return MR_OK;
    }
    if (!idx) {
        set_error("null idx");
        return MR_ERR_ARG;
    }
    int* err = device_error_word();
    if (!err) {
        set_error("cannot locate the device error word");
        return MR_ERR_CUDA;
    }
    float4* acc = nullptr;
    int rc = scratch_alloc(reinterpret_cast<void**>(&acc), sizeof(float4) * (size_t)P, s);
    if (rc != MR_OK) return rc;
    cudaError_t e = cudaMemsetAsync(acc, 0, sizeof(float4) * (size_t)P, s);
    if (e == cudaSuccess) {
        ProfScope ps(MR_STAGE_POINTS_BWD, s);
        k_point_raster_bwd<<<grid_for(nslots), 256, 0, s>>>(points, P, idx, nslots, H, W, K, grad_zbuf, grad_dists,
                                                           acc, err);
        k_xyzw_rows<<<grid_for(P), 256, 0, s>>>(acc, P, grad_points);
        e = cudaGetLastError();
    }
    scratch_free(acc, s);
    if (e != cudaSuccess) return cuda_fail(e, "point rasterizer backward");
    return MR_OK;
}

int mr_composite_points_fwd(const int64_t* idx, const float* dists, int64_t npix, int32_t K, const float* features,
                            int64_t P, int32_t C, float radius, int32_t mode, float* out, void* stream) {
    using namespace mr;
    if (npix < 0 || K < 1 || K > MR_KMAX || C < 1 || P < 0 || (mode != 0 && mode != 1) || !(radius > 0.f) ||
        !std::isfinite(radius)) {
        set_error("invalid arguments npix=%lld K=%d C=%d mode=%d radius=%g", (long long)npix, K, C, mode,
                  (double)radius);
        return MR_ERR_ARG;
    }
    if (npix == 0) return MR_OK;
    if (!idx || !dists || !out || (P > 0 && !features)) {
        set_error("null pointer");
        return MR_ERR_ARG;
    }
    int* err = device_error_word();
    if (!err) {
        set_error("cannot locate the device error word");
        return MR_ERR_CUDA;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const Radius2 R = radius2(radius);
    const int g = grid_for(npix);
    ProfScope ps(MR_STAGE_COMPOSITE_FWD, s);
    const bool vec = (K == 4 || K == 8) && ((reinterpret_cast<uintptr_t>(idx) | reinterpret_cast<uintptr_t>(dists)) & 15) == 0;
#define MR_CF2(KC, V)                                                                                              \
    (mode == 0 ? k_composite_fwd<KC, 0, V><<<g, 256, 0, s>>>(idx, dists, npix, K, features, P, C, R, out, err) \
               : k_composite_fwd<KC, 1, V><<<g, 256, 0, s>>>(idx, dists, npix, K, features, P, C, R, out, err))
#define MR_CF(KC) MR_CF2(KC, false)
    if (vec && K == 4) MR_CF2(4, true);
    else if (vec) MR_CF2(8, true);
    else if (K <= 1) MR_CF(1);
    else if (K <= 2) MR_CF(2);
    else if (K <= 4) MR_CF(4);
    else if (K <= 8) MR_CF(8);
    else if (K <= 16) MR_CF(16);
    else MR_CF(32);
#undef MR_CF
#undef MR_CF2
    MR_CUDA(cudaGetLastError());
    return MR_OK;
}

int mr_composite_points_bwd(const int64_t* idx, const float* dists, int64_t npix, int32_t K, const float* features,
                            int64_t P, int32_t C, float radius, int32_t mode, const float* grad_out,
                            float* grad_features, float* grad_dists, void* stream) {
    using namespace mr;
    if (npix < 0 || K < 1 || K > MR_KMAX || C < 1 || P < 0 || (mode != 0 && mode != 1) || !(radius > 0.f) ||
        !std::isfinite(radius)) {
        set_error("invalid arguments");
        return MR_ERR_ARG;
    }
    if ((P > 0 && (!features || !grad_features)) || (npix > 0 && (!idx || !dists || !grad_out))) {
        set_error("null pointer");
        return MR_ERR_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (npix == 0 || P == 0) {
        if (P > 0) MR_CUDA(cudaMemsetAsync(grad_features, 0, sizeof(float) * (size_t)(P * C), s));
        if (npix > 0 && grad_dists) MR_CUDA(cudaMemsetAsync(grad_dists, 0, sizeof(float) * (size_t)(npix * K), s));
        return MR_OK;
    }
    int* err = device_error_word();
    if (!err) {
        set_error("cannot locate the device error word");
        return MR_ERR_CUDA;
    }
    const bool vec4 = C <= 4;
    float4* acc = nullptr;
    if (vec4) {
        int rc = scratch_alloc(reinterpret_cast<void**>(&acc), sizeof(float4) * (size_t)P, s);
        if (rc != MR_OK) return rc;
    }
    cudaError_t e = vec4 ? cudaMemsetAsync(acc, 0, sizeof(float4) * (size_t)P, s)
                         : cudaMemsetAsync(grad_features, 0, sizeof(float) * (size_t)(P * C), s);
    const Radius2 R = radius2(radius);
    const int g = grid_for(npix);
    if (e == cudaSuccess) {
        ProfScope ps(MR_STAGE_COMPOSITE_BWD, s);
        const bool vec = (K == 4 || K == 8) && ((reinterpret_cast<uintptr_t>(idx) | reinterpret_cast<uintptr_t>(dists) |
                                                  reinterpret_cast<uintptr_t>(grad_dists)) & 15) == 0;
#define MR_CB3(KC, MODE, V)                                                                                       \
    (vec4 ? k_composite_bwd<KC, MODE, true, V><<<g, 256, 0, s>>>(idx, dists, npix, K, features, P, C, R,        \
                                                                 grad_out, nullptr, acc, grad_dists, err)         \
          : k_composite_bwd<KC, MODE, false, V><<<g, 256, 0, s>>>(idx, dists, npix, K, features, P, C, R,       \
                                                                  grad_out, grad_features, nullptr, grad_dists, err))
#define MR_CB2(KC, V) (mode == 0 ? MR_CB3(KC, 0, V) : MR_CB3(KC, 1, V))
#define MR_CB(KC) MR_CB2(KC, false)
        if (vec && K == 4) MR_CB2(4, true);
        else if (vec) MR_CB2(8, true);
        else if (K <= 1) MR_CB(1);
        else if (K <= 2) MR_CB(2);
        else if (K <= 4) MR_CB(4);
        else if (K <= 8) MR_CB(8);
        else if (K <= 16) MR_CB(16);
        else MR_CB(32);
#undef MR_CB
#undef MR_CB2
#undef MR_CB3
        if (vec4) k_acc4_cols<<<grid_for(P), 256, 0, s>>>(acc, P, C, grad_features);
        e = cudaGetLastError();
    }
    if (acc) scratch_free(acc, s);
    if (e != cudaSuccess) return cuda_fail(e, "compositing backward");
    return MR_OK;
}

}  // extern "C"
