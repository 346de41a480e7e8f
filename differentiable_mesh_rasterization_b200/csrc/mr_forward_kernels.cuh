// Kernels and launch helpers of the stage-one forward pipeline (internal header).
//
// Shared by the allocating entry points (mr_forward.cu) and the scratch-free variant
// (mr_noalloc.cu); everything sits in an unnamed namespace, so each translation unit
// compiles its own copy.  The pipeline is described in mr_forward.cu.
#pragma once

#include <algorithm>
#include <cfloat>
#include <climits>
#include <cmath>
#include <vector>

#include "mr_common.cuh"
#include "mr_scan.cuh"
#include "mr_silhouette.cuh"

namespace mr {
namespace {


// ------------------------------------------------------------------ face setup
// Per-face plane constants of the fine pass, computed in float64 from the exact float32
// vertices and rounded once.  The origin is the face's first vertex a, so a pixel enters
// as (dx, dy) = p - a.  The winding is made counter-clockwise (b and c swapped if needed)
// so every edge function is positive inside.  Per edge u -> v with unit direction e and
// length L:
//     c(d) = -e.y * d.x + e.x * d.y + ng   signed distance to the edge line (inside > 0)
//     s(d) =  e.x * d.x + e.y * d.y + tg   position along the edge from its midpoint
//     squared distance to the segment = c^2 + max(|s| - L/2, 0)^2.
// The depth key is the plane through (x, y, z) -- or (x, y, -1/z) with perspective
// correction, where 1/z is screen-affine -- written as k_hi + (gx dx + gy dy + k_lo);
// the float-float constant keeps the key within half an ulp plus the plane terms.
// Layout (6 float4): (ax, ay, gx, gy) (k_hi, k_lo, L0/2, L1/2) (e0.x, e0.y, ng0, tg0)
//                    (e1.x, e1.y, ng1, tg1) (e2.x, e2.y, ng2, tg2) (L2/2, face id, 0, 0)
constexpr int kConstF4 = 6;

__device__ __forceinline__ void setup_face(const float* __restrict__ verts, int64_t V,
                                           const int64_t* __restrict__ faces, int64_t f, int H, int W,
                                           double reach, int persp, FaceGeom* __restrict__ geom,
                                           FaceBox* __restrict__ box, float4* __restrict__ fconst,
                                           int* __restrict__ err, float& qlo, float& qhi) {
    int64_t i0 = faces[3 * f], i1 = faces[3 * f + 1], i2 = faces[3 * f + 2];
    FaceBox bx = {1, 0, 1, 0, 0.f, 0};
    float4* out = fconst + kConstF4 * f;
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i0 < 0 || i0 >= V || i1 < 0 || i1 >= V || i2 < 0 || i2 >= V) {
        atomicOr(err, kErrFaceIndex);
        geom[f] = FaceGeom{zero, zero, zero};
        box[f] = bx;
        return;
    }
    float4 a = make_float4(verts[3 * i0], verts[3 * i0 + 1], verts[3 * i0 + 2], 0.f);
    float4 b = make_float4(verts[3 * i1], verts[3 * i1 + 1], verts[3 * i1 + 2], 0.f);
    float4 c = make_float4(verts[3 * i2], verts[3 * i2 + 1], verts[3 * i2 + 2], 0.f);
    double ax = a.x, ay = a.y, bxx = b.x, byy = b.y, cx = c.x, cy = c.y;
    double area2 = (bxx - ax) * (cy - ay) - (byy - ay) * (cx - ax);
    if (!(fabs(area2) > kDegenerateArea)) {
        geom[f] = FaceGeom{a, b, c};
        box[f] = bx;
        return;
    }
    // 1 / (2 area) as a float-float pair for the epilogue's float64 barycentrics
    const double inv_area2 = 1.0 / area2;
    a.w = (float)inv_area2;
    b.w = (float)(inv_area2 - (double)a.w);
    geom[f] = FaceGeom{a, b, c};
    double xmin = fmin(ax, fmin(bxx, cx)) - reach, xmax = fmax(ax, fmax(bxx, cx)) + reach;
    double ymin = fmin(ay, fmin(byy, cy)) - reach, ymax = fmax(ay, fmax(byy, cy)) + reach;
    // pixel j has centre x = -1 + (2j+1)/W; row i has y = 1 - (2i+1)/H.  The 1e-4
    // pixel pad keeps the box a superset under rounding.
    double jl = ceil((xmin + 1.0) * 0.5 * W - 0.5 - 1e-4);
    double jh = floor((xmax + 1.0) * 0.5 * W - 0.5 + 1e-4);
    double il = ceil((1.0 - ymax) * 0.5 * H - 0.5 - 1e-4);
    double ih = floor((1.0 - ymin) * 0.5 * H - 0.5 + 1e-4);
    jl = fmax(jl, 0.0); il = fmax(il, 0.0);
    jh = fmin(jh, (double)(W - 1)); ih = fmin(ih, (double)(H - 1));
    const bool on_screen = jl <= jh && il <= ih;

    double x[3] = {0.0, bxx - ax, cx - ax};
    double y[3] = {0.0, byy - ay, cy - ay};
    double q[3];
    if (persp) {
        q[0] = -1.0 / (double)a.z; q[1] = -1.0 / (double)b.z; q[2] = -1.0 / (double)c.z;
    } else {
        q[0] = a.z; q[1] = b.z; q[2] = c.z;
    }
    const double nx = y[1] * (q[2] - q[0]) - (q[1] - q[0]) * y[2];
    const double ny = (q[1] - q[0]) * x[2] - x[1] * (q[2] - q[0]);
    const double gx = -nx * inv_area2, gy = -ny * inv_area2;
    const float khi = (float)q[0];
    const float klo = (float)(q[0] - (double)khi);
    if (on_screen) {
        // lowest key over the box's pixel centres (a plane: one corner), lowered by a
        // margin well above the float32 evaluation error of the key
        const double xl = -1.0 + (2.0 * jl + 1.0) / W - ax, xh = -1.0 + (2.0 * jh + 1.0) / W - ax;
        const double yl = 1.0 - (2.0 * ih + 1.0) / H - ay, yh = 1.0 - (2.0 * il + 1.0) / H - ay;
        const double tx = fmin(gx * xl, gx * xh), ty = fmin(gy * yl, gy * yh);
        const double span = fabs(q[0]) + fmax(fabs(gx * xl), fabs(gx * xh)) + fmax(fabs(gy * yl), fabs(gy * yh));
        bx = FaceBox{(short)jl, (short)jh, (short)il, (short)ih, __double2float_rd(q[0] + tx + ty - 1e-6 * span), 0};
        qlo = (float)fmin(q[0], fmin(q[1], q[2]));
        qhi = (float)fmax(q[0], fmax(q[1], q[2]));
    }
    box[f] = bx;
    if (area2 < 0.0) {
        double t = x[1]; x[1] = x[2]; x[2] = t;
        t = y[1]; y[1] = y[2]; y[2] = t;
    }
    float e[3][5];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const int k1 = k == 2 ? 0 : k + 1;
        const double ex = x[k1] - x[k], ey = y[k1] - y[k];
        const double L = sqrt(ex * ex + ey * ey);
        const double inv_L = 1.0 / L;
        const double ux = ex * inv_L, uy = ey * inv_L;
        e[k][0] = (float)ux;
        e[k][1] = (float)uy;
        e[k][2] = (float)(uy * x[k] - ux * y[k]);
        e[k][3] = (float)(-(ux * x[k] + uy * y[k]) - 0.5 * L);
        e[k][4] = (float)(0.5 * L);
    }
    out[0] = make_float4(a.x, a.y, (float)gx, (float)gy);
    out[1] = make_float4(khi, klo, e[0][4], e[1][4]);
    out[2] = make_float4(e[0][0], e[0][1], e[0][2], e[0][3]);
    out[3] = make_float4(e[1][0], e[1][1], e[1][2], e[1][3]);
    out[4] = make_float4(e[2][0], e[2][1], e[2][2], e[2][3]);
    out[5] = make_float4(e[2][4], __int_as_float((int)f), 0.f, 0.f);
}

// Ordered unsigned image of a float (monotone), for atomic min / max of depth keys.
__device__ __forceinline__ unsigned float_order(float f) {
    const unsigned u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float order_float(unsigned u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// (image, face) pairs are enumerated image by image: pair q belongs to image n with
// pair_prefix[n] <= q < pair_prefix[n+1] and is face first[n] + q - pair_prefix[n].
__device__ __forceinline__ int pair_image(const int64_t* prefix, int N, int64_t q) {
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= q) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Face setup over the (image, face) pairs (a face shared by several images is set up
// once per image, with identical results), and each image's range of vertex depth keys
// (ordered-unsigned minima in krange[0, N), maxima in krange[N, 2N); one atomic pair per
// warp when the warp sits in one image).
// 64 registers, 4 CTAs per SM: the kernel waits on its dependent face -> vertex gathers, so
// residency pays (0.144 -> 0.135 ms on the 64-image batch; 5 or 6 CTAs spill: 0.140 / 0.147)
__global__ void __launch_bounds__(256, 4)
k_face_setup(const float* __restrict__ verts, int64_t V, const int64_t* __restrict__ faces,
                             const int64_t* __restrict__ prefix, const int64_t* __restrict__ first, int N,
                             int64_t pairs, int H, int W, double reach, int persp, FaceGeom* __restrict__ geom,
                             FaceBox* __restrict__ box, float4* __restrict__ fconst, unsigned* __restrict__ krange,
                             int* __restrict__ err) {
    for (int64_t q0 = (int64_t)blockIdx.x * blockDim.x; q0 < pairs; q0 += (int64_t)gridDim.x * blockDim.x) {
        const int64_t q = q0 + threadIdx.x;
        const bool live = q < pairs;
        int n = 0;
        float qlo = FLT_MAX, qhi = -FLT_MAX;
        if (live) {
            n = pair_image(prefix, N, q);
            setup_face(verts, V, faces, first[n] + (q - prefix[n]), H, W, reach, persp, geom, box, fconst, err, qlo,
                       qhi);
        }
        const int n0 = __shfl_sync(0xffffffffu, n, 0);
        if (__all_sync(0xffffffffu, !live || n == n0)) {
            for (int o = 16; o > 0; o >>= 1) {
                qlo = fminf(qlo, __shfl_xor_sync(0xffffffffu, qlo, o));
                qhi = fmaxf(qhi, __shfl_xor_sync(0xffffffffu, qhi, o));
            }
            if ((threadIdx.x & 31) == 0 && qlo <= qhi) {
                atomicMin(&krange[n0], float_order(qlo));
                atomicMax(&krange[N + n0], float_order(qhi));
            }
        } else if (live && qlo <= qhi) {
            atomicMin(&krange[n], float_order(qlo));
            atomicMax(&krange[N + n], float_order(qhi));
        }
    }
}

// ------------------------------------------------------------------ binning
// Each bin's face list is split into kDepthBuckets sub-lists by the face's key lower
// bound, relative to its image's range of vertex keys, nearest bucket first.  The fine
// pass then meets near faces first, so its depth culls reject more of the rest.
constexpr int kDepthBuckets = 8;

__device__ __forceinline__ int depth_bucket(float kmin, float lo, float hi) {
    if (!(hi > lo)) return 0;
    const float t = (kmin - lo) / (hi - lo) * (float)kDepthBuckets;
    return t <= 0.f ? 0 : (t >= (float)(kDepthBuckets - 1) ? kDepthBuckets - 1 : (int)t);
}

template <bool FILL>
__global__ void k_bin_pairs(const FaceBox* __restrict__ box, const int64_t* __restrict__ prefix,
                            const int64_t* __restrict__ first, int N, int64_t pairs, int nbx, int nby,
                            const unsigned* __restrict__ krange, int* __restrict__ counts,
                            const int* __restrict__ offsets, int* __restrict__ list) {
    const unsigned lane = threadIdx.x & 31;
    for (int64_t q0 = (int64_t)blockIdx.x * blockDim.x; q0 < pairs; q0 += (int64_t)gridDim.x * blockDim.x) {
        int64_t q = q0 + threadIdx.x;
        bool live = q < pairs;
        int n = 0, bucket = 0;
        int64_t f = 0;
        FaceBox b = {1, 0, 1, 0, 0.f, 0};
        if (live) {
            n = pair_image(prefix, N, q);
            f = first[n] + (q - prefix[n]);
            b = box[f];
            bucket = depth_bucket(b.kmin, order_float(krange[n]), order_float(krange[N + n]));
        }
        int bx0 = 0, bx1 = -1, by0 = 0, by1 = -1;
        if (live && b.x0 <= b.x1) {
            bx0 = b.x0 / kBin; bx1 = b.x1 / kBin; by0 = b.y0 / kBin; by1 = b.y1 / kBin;
        }
        // Walk the touched bins in lock-step across the warp; neighbouring faces share
        // (bin, bucket) slots, so a run of equal slots in neighbouring lanes takes one atomic
        // per step, issued by the run's first lane (match.any, which groups equal slots
        // anywhere in the warp, cost more than it saved: count 0.079 -> 0.076 ms, fill
        // 0.095 -> 0.093 ms on the 64-image batch).
        int nx = bx1 - bx0 + 1, ny = by1 - by0 + 1;
        int mine = (nx > 0 && ny > 0) ? nx * ny : 0;
        int most = mine;
        for (int o = 16; o > 0; o >>= 1) most = max(most, __shfl_xor_sync(0xffffffffu, most, o));
        for (int s = 0; s < most; ++s) {
            bool act = s < mine;
            int slot = -1;
            if (act) slot = ((n * nby + by0 + s / nx) * nbx + bx0 + s % nx) * kDepthBuckets + bucket;
            const int up = __shfl_up_sync(0xffffffffu, slot, 1);
            const bool head = lane == 0 || up != slot;
            const unsigned heads = __ballot_sync(0xffffffffu, head);
            const int run0 = 31 - __clz(heads & (0xffffffffu >> (31 - lane)));   // this run's first lane
            const unsigned later = lane == 31 ? 0u : (heads & (0xffffffffu << (lane + 1)));
            const int run1 = later ? __ffs(later) - 1 : 32;                       // and its end
            int base = 0;
            if (act && head) base = atomicAdd(&counts[slot], run1 - (int)lane);
            base = __shfl_sync(0xffffffffu, base, run0);
            if (!act) continue;
            if (FILL) list[offsets[slot] + base + ((int)lane - run0)] = (int)f;
        }
    }
}

// ------------------------------------------------------------------ launch order of the bins
// The fine pass's time is set by its longest bin lists when they start late (a crowded
// bin's warps walk its whole list); the bins are therefore launched longest first: a
// histogram of the list lengths in 33 classes (0, then 2^(c-1) <= length < 2^c), then each
// bin written to its class's next place, classes from the longest down.  Order inside a
// class is free; the outputs do not depend on the order.
constexpr int kLenClasses = 33;

__device__ __forceinline__ int len_class(int len) { return len > 0 ? 32 - __clz(len) : 0; }

__global__ void k_bin_hist(const int* __restrict__ offsets, int nbins, int* __restrict__ hist) {
    __shared__ int h[kLenClasses];
    for (int c = threadIdx.x; c < kLenClasses; c += blockDim.x) h[c] = 0;
    __syncthreads();
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < nbins; b += gridDim.x * blockDim.x)
        atomicAdd(&h[len_class(offsets[(b + 1) * kDepthBuckets] - offsets[b * kDepthBuckets])], 1);
    __syncthreads();
    for (int c = threadIdx.x; c < kLenClasses; c += blockDim.x)
        if (h[c]) atomicAdd(&hist[c], h[c]);
}

// Rounds of blockDim bins: ranks inside the round from shared-memory atomics, then one
// global atomic per class and round reserves the round's places in that class.
__global__ void k_bin_order(const int* __restrict__ offsets, int nbins, const int* __restrict__ hist,
                            int* __restrict__ cursor, int* __restrict__ order) {
    __shared__ int start[kLenClasses], cnt[kLenClasses], base[kLenClasses];
    if (threadIdx.x == 0) {
        int at = 0;
        for (int c = kLenClasses - 1; c >= 0; --c) {
            start[c] = at;
            at += hist[c];
        }
    }
    for (int b0 = blockIdx.x * blockDim.x; b0 < nbins; b0 += gridDim.x * blockDim.x) {
        for (int c = threadIdx.x; c < kLenClasses; c += blockDim.x) cnt[c] = 0;
        __syncthreads();
        const int b = b0 + threadIdx.x;
        int c = 0, r = 0;
        if (b < nbins) {
            c = len_class(offsets[(b + 1) * kDepthBuckets] - offsets[b * kDepthBuckets]);
            r = atomicAdd(&cnt[c], 1);
        }
        __syncthreads();
        for (int k = threadIdx.x; k < kLenClasses; k += blockDim.x)
            base[k] = cnt[k] ? start[k] + atomicAdd(&cursor[k], cnt[k]) : 0;
        __syncthreads();
        if (b < nbins) order[base[c] + r] = b;
        __syncthreads();
    }
}

// ------------------------------------------------------------------ fine pass
// The K nearest candidates of a lane in registers, sorted by (key, face id).  Keys are held
// as unsigned images that order like the float keys: without perspective correction the
// keys are depths >= 0, whose bit patterns already do; with it they are negative, and
// float_order maps them.  (key, face id) then compares as one unsigned 64-bit value: all K
// compares first (independent of each other), then each slot takes its left neighbour, the
// new entry or itself.  On the 64-image batch the fine pass took 1.483 instead of 1.548 ms
// with this form over a serial chain of float compares with an id tie-break, results the
// same bit for bit.
template <int KC>
__device__ __forceinline__ void topk_insert(unsigned (&kb)[KC], int (&ff)[KC], unsigned key, int fid) {
    const unsigned long long x = ((unsigned long long)key << 32) | (unsigned)fid;
    bool c[KC];
#pragma unroll
    for (int k = 0; k < KC; ++k) c[k] = x < (((unsigned long long)kb[k] << 32) | (unsigned)ff[k]);
#pragma unroll
    for (int k = KC - 1; k > 0; --k) {
        kb[k] = c[k - 1] ? kb[k - 1] : (c[k] ? key : kb[k]);
        ff[k] = c[k - 1] ? ff[k - 1] : (c[k] ? fid : ff[k]);
    }
    kb[0] = c[0] ? key : kb[0];
    ff[0] = c[0] ? fid : ff[0];
}

// Two CTAs of four warps per 16x16 bin; each of the bin's eight warps owns an 8x4 pixel
// tile and runs on its own (no block barriers).  A warp reads the bin's face list 32 ids at a time, tests
// each face's pixel box against its tile, compacts the hits with a ballot and copies
// their constants into its shared-memory slots.  For each staged face the warp first
// evaluates the depth key alone; if no lane could admit the face into its top-K (face
// behind the camera or not nearer than the lane's K-th key) the face is skipped, else
// every lane runs the full candidacy test.  EXACT: the pixel centres are exact float32
// values (H and W powers of two), so the float-float low parts vanish.
template <int KC, bool PERSP, bool EXACT>
__global__ void __launch_bounds__(kFineThreads, (KC <= 4 ? 6 : 4) * kFineCtasPerBin)
k_fine(const float4* __restrict__ fconst, const FaceBox* __restrict__ box, const int* __restrict__ offsets,
       const int* __restrict__ list, const int* __restrict__ order, int nbx, int nby, int H, int W, int K, float blur,
       bool vec, int64_t* __restrict__ p2f) {
    __shared__ __align__(16) float4 s_c[kFineWarps][32][kConstF4];

    const int bin = order[blockIdx.x / kFineCtasPerBin];
    const int bxi = bin % nbx;
    const int byi = (bin / nbx) % nby;
    const int n = bin / (nbx * nby);
    const int lwarp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int warp = (blockIdx.x % kFineCtasPerBin) * kFineWarps + lwarp;   // the warp tile within the bin
    const int tj0 = bxi * kBin + (warp & 1) * kWarpTileW;
    const int ti0 = byi * kBin + (warp >> 1) * kWarpTileH;
    if (tj0 >= W || ti0 >= H) return;                        // tile entirely off the image
    const int j = tj0 + (lane & 7), i = ti0 + (lane >> 3);
    const bool in_img = i < H && j < W;
    const double pxd = -1.0 + (2.0 * j + 1.0) / W;
    const double pyd = 1.0 - (2.0 * i + 1.0) / H;
    const float pxh = (float)pxd, pyh = (float)pyd;
    const float pxl = (float)(pxd - (double)pxh), pyl = (float)(pyd - (double)pyh);
    const unsigned lt_mask = (1u << lane) - 1u;

    unsigned kb[KC];   // the keys' order images (see topk_insert); off-image lanes are never written
    int ff[KC];
    const unsigned far_key = PERSP ? float_order(FLT_MAX) : __float_as_uint(FLT_MAX);
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        kb[k] = in_img ? far_key : 0u;
        ff[k] = INT_MAX;
    }

    const int beg = offsets[bin * kDepthBuckets], cnt = offsets[(bin + 1) * kDepthBuckets] - beg;
    float4(*slots)[kConstF4] = s_c[lwarp];
    // the next batch's face id and box are loaded while the current batch is tested
    int nfid = 0;
    FaceBox nbox = {1, 0, 1, 0, 0.f, 0};
    if (lane < cnt) {
        nfid = list[beg + lane];
        nbox = box[nfid];
    }
    for (int base = 0; base < cnt; base += 32) {
        const int fid = nfid;
        const FaceBox b = nbox;
        // tile depth cull: the farthest K-th key over the warp's pixels; a face whose lowest
        // key over its box lies beyond it cannot enter any lane's top K
        // one warp reduction over the order images (off-image lanes give 0, the lowest)
        const unsigned zfar_b = __reduce_max_sync(0xffffffffu, in_img ? kb[KC - 1] : 0u);
        const float zfar = PERSP ? order_float(zfar_b) : __uint_as_float(zfar_b);
        const bool hit = base + lane < cnt && b.x0 <= tj0 + kWarpTileW - 1 && b.x1 >= tj0 &&
                         b.y0 <= ti0 + kWarpTileH - 1 && b.y1 >= ti0 && b.kmin <= zfar;
        if (base + 32 + lane < cnt) {
            nfid = list[beg + base + 32 + lane];
            nbox = box[nfid];
        }
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (hit) {
            const int slot = __popc(m & lt_mask);
            const float4* src = fconst + (int64_t)kConstF4 * fid;
#pragma unroll
            for (int u = 0; u < kConstF4; ++u) cp_async16(&slots[slot][u], src + u);
        }
        cp_wait_all();
        __syncwarp();
        const int nh = __popc(m);
        for (int qi = 0; qi < nh; ++qi) {
            const float4 q0 = slots[qi][0], q1 = slots[qi][1];
            float dx = pxh - q0.x, dy = pyh - q0.y;
            if (!EXACT) { dx += pxl; dy += pyl; }
            const float key = q1.x + fmaf(q0.z, dx, fmaf(q0.w, dy, q1.y));
            // admissible: in front of the camera and not behind the lane's K-th key.  Without
            // perspective the keys are depths >= 0, whose float order is their bit order,
            // so one unsigned compare does both (negative keys wrap to huge values).
            const unsigned kbits = PERSP ? float_order(key) : __float_as_uint(key);
            const bool maybe = PERSP ? (key < 0.f && kbits <= kb[KC - 1]) : kbits <= kb[KC - 1];
            if (!__any_sync(0xffffffffu, maybe)) continue;
            const float4 e0 = slots[qi][2], e1 = slots[qi][3], e2 = slots[qi][4], q5 = slots[qi][5];
            const float c0 = fmaf(-e0.y, dx, fmaf(e0.x, dy, e0.z));
            const float s0 = fmaf(e0.x, dx, fmaf(e0.y, dy, e0.w));
            const float c1 = fmaf(-e1.y, dx, fmaf(e1.x, dy, e1.z));
            const float s1 = fmaf(e1.x, dx, fmaf(e1.y, dy, e1.w));
            const float c2 = fmaf(-e2.y, dx, fmaf(e2.x, dy, e2.z));
            const float s2 = fmaf(e2.x, dx, fmaf(e2.y, dy, e2.w));
            const float o0 = fmaxf(fabsf(s0) - q1.z, 0.f);
            const float o1 = fmaxf(fabsf(s1) - q1.w, 0.f);
            const float o2 = fmaxf(fabsf(s2) - q5.x, 0.f);
            const float d0 = fmaf(o0, o0, c0 * c0);
            const float d1 = fmaf(o1, o1, c1 * c1);
            const float d2 = fmaf(o2, o2, c2 * c2);
            const bool inside = fminf(c0, fminf(c1, c2)) >= 0.f;
            const float dmin = fminf(d0, fminf(d1, d2));
            if (maybe && (inside || dmin <= blur)) topk_insert<KC>(kb, ff, kbits, __float_as_int(q5.y));
        }
        __syncwarp();
    }
    if (!in_img) return;
    // the winners go straight into pix_to_face (global face ids, -1 past the candidates);
    // the epilogue reads them back from there
    const int64_t pix = ((int64_t)n * H + i) * W + j;
    if ((KC % 2) == 0 && K == KC && vec) {
#pragma unroll
        for (int k2 = 0; k2 < KC; k2 += 2)
            *reinterpret_cast<longlong2*>(p2f + pix * KC + k2) =
                make_longlong2(ff[k2] == INT_MAX ? -1 : ff[k2], ff[k2 + 1] == INT_MAX ? -1 : ff[k2 + 1]);
    } else {
#pragma unroll
        for (int k = 0; k < KC; ++k)
            if (k < K) p2f[pix * K + k] = ff[k] == INT_MAX ? -1 : ff[k];
    }
}

// Per-slot outputs from the original vertices, the definition written out.  The
// barycentrics and z are evaluated in float64 -- edge functions from exact float64
// differences, times the float64 1/(2 area) kept as a float-float pair in a.w, b.w --
// because extrapolated blur-ring faces reach |w| in the hundreds, where float32 cannot
// hold them to 1e-5.  The squared distance only needs float32: the nearest-edge
// distance in face-local differences is good to ~1e-10 in NDC^2.
template <bool PERSP, bool EXACT = false>
__device__ __forceinline__ void slot_outputs(const FaceGeom& g, double pxd, double pyd, float pxh, float pxl,
                                             float pyh, float pyl, float* z_out, float* b_out, float* d_out) {
    const double inv_area2 = (double)g.a.w + (double)g.b.w;
    const double rx0 = (double)g.a.x - pxd, ry0 = (double)g.a.y - pyd;
    const double rx1 = (double)g.b.x - pxd, ry1 = (double)g.b.y - pyd;
    const double rx2 = (double)g.c.x - pxd, ry2 = (double)g.c.y - pyd;
    const double w0 = (rx1 * ry2 - ry1 * rx2) * inv_area2;
    const double w1 = (rx2 * ry0 - ry2 * rx0) * inv_area2;
    const double w2 = (rx0 * ry1 - ry0 * rx1) * inv_area2;
    const bool inside = w0 >= 0.0 && w1 >= 0.0 && w2 >= 0.0;
    const double z0 = g.a.z, z1 = g.b.z, z2 = g.c.z;
    double b0 = w0, b1 = w1, b2 = w2, z;
    if (PERSP) {
        // u_k = w_k / z_k renormalised; multiplied through by z0 z1 z2 to keep one division
        const double u0 = w0 * z1 * z2, u1 = w1 * z0 * z2, u2 = w2 * z0 * z1;
        const double inv = 1.0 / (u0 + u1 + u2);
        b0 = u0 * inv; b1 = u1 * inv; b2 = u2 * inv;
        z = z0 * z1 * z2 * inv;
    } else {
        z = w0 * z0 + w1 * z1 + w2 * z2;
    }
    // squared distance to the nearest edge, float32, pixel - vertex differences; the segment
    // parameter t takes the fast division (len2 is a normal float32 of an edge the setup kept:
    // its error of a few ulp moves d2 far below the 1e-5 of the outputs)
    // EXACT: the pixel centre is an exact float32 (H, W powers of two), its low part is 0
    const float qx[3] = {EXACT ? pxh - g.a.x : (pxh - g.a.x) + pxl, EXACT ? pxh - g.b.x : (pxh - g.b.x) + pxl,
                         EXACT ? pxh - g.c.x : (pxh - g.c.x) + pxl};
    const float qy[3] = {EXACT ? pyh - g.a.y : (pyh - g.a.y) + pyl, EXACT ? pyh - g.b.y : (pyh - g.b.y) + pyl,
                         EXACT ? pyh - g.c.y : (pyh - g.c.y) + pyl};
    const float vx[3] = {g.a.x, g.b.x, g.c.x}, vy[3] = {g.a.y, g.b.y, g.c.y};
    float d2 = FLT_MAX;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const int k1 = k == 2 ? 0 : k + 1;
        const float ex = vx[k1] - vx[k], ey = vy[k1] - vy[k];
        const float len2 = fmaf(ex, ex, ey * ey);
        const float t = len2 > 0.f ? __saturatef(__fdividef(fmaf(qx[k], ex, qy[k] * ey), len2)) : 0.f;
        const float rx = fmaf(-t, ex, qx[k]), ry = fmaf(-t, ey, qy[k]);
        d2 = fminf(d2, fmaf(rx, rx, ry * ry));
    }
    *z_out = (float)z;
    b_out[0] = (float)b0;
    b_out[1] = (float)b1;
    b_out[2] = (float)b2;
    *d_out = inside ? -d2 : d2;
}

// One thread per pixel: the K winners' outputs (and the fused silhouette), written
// contiguously per pixel; VEC (K == KC, a multiple of 4, 16-byte aligned outputs) with
// 16-byte loads and stores.  Pixels are taken in 16 x 16 tiles (one tile per 256
// consecutive work items), so the threads of a block gather the faces of one screen
// region and the geometry reads hit L1.
template <int KC, bool PERSP, bool SIL, bool VEC, bool EXACT>
__global__ void __launch_bounds__(256, 4)
k_epilogue(const FaceGeom* __restrict__ geom, const int* __restrict__ offsets, int64_t* __restrict__ p2f, int N,
           int H, int W, int K, float sigma, float* __restrict__ zbuf, float* __restrict__ bary,
           float* __restrict__ dists, float* __restrict__ alpha) {
    static_assert(kBin == 16, "the tile arithmetic below takes 16 x 16 tiles");
    const int tw = (W + kBin - 1) / kBin, th = (H + kBin - 1) / kBin;
    const int64_t items = (int64_t)N * th * tw * (kBin * kBin);
    const bool small = (int64_t)N * th * tw <= 0x7fffffff;   // tile ids fit 32-bit division
    const bool ragged = (H % kBin) != 0 || (W % kBin) != 0;   // some tiles stick out of the image
    const double inv_w = 1.0 / W, inv_h = 1.0 / H;
    for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items;
         it += (int64_t)gridDim.x * blockDim.x) {
        const int64_t tile = it >> 8;                           // kBin * kBin = 256 items per tile
        const int r = (int)(it & 255);
        int tx, ty;
        int64_t n;
        if (small) {
            const unsigned t = (unsigned)tile, t2 = t / (unsigned)tw;
            tx = (int)(t - t2 * (unsigned)tw);
            ty = (int)(t2 % (unsigned)th);
            n = t2 / (unsigned)th;
        } else {
            tx = (int)(tile % tw);
            const int64_t t2 = tile / tw;
            ty = (int)(t2 % th);
            n = t2 / th;
        }
        const int i = ty * kBin + (r >> 4), j = tx * kBin + (r & 15);
        if (ragged && (i >= H || j >= W)) continue;
        const int64_t pix = (n * H + i) * W + j;
        // a tile is a bin: the fine pass did not run for an empty one, whose pixels get the
        // padding here (-1 in every slot, alpha 0)
        if (offsets[(tile + 1) * kDepthBuckets] == offsets[tile * kDepthBuckets]) {
            if (VEC) {
                const float4 m1 = make_float4(-1.f, -1.f, -1.f, -1.f);
#pragma unroll
                for (int k4 = 0; k4 < KC; k4 += 4) {
                    const int64_t s = pix * KC + k4;
                    reinterpret_cast<longlong2*>(p2f + s)[0] = make_longlong2(-1, -1);
                    reinterpret_cast<longlong2*>(p2f + s)[1] = make_longlong2(-1, -1);
                    *reinterpret_cast<float4*>(zbuf + s) = m1;
                    *reinterpret_cast<float4*>(dists + s) = m1;
                    float4* bp = reinterpret_cast<float4*>(bary + 3 * s);
                    bp[0] = m1;
                    bp[1] = m1;
                    bp[2] = m1;
                }
            } else {
                for (int k = 0; k < K; ++k) {
                    const int64_t s = pix * K + k;
                    p2f[s] = -1;
                    zbuf[s] = -1.f;
                    dists[s] = -1.f;
                    bary[3 * s] = bary[3 * s + 1] = bary[3 * s + 2] = -1.f;
                }
            }
            if (SIL) alpha[pix] = 0.f;
            continue;
        }
        // EXACT (H, W powers of two): 1/W and 1/H are exact, so the centre is one exact
        // product instead of a division (the same float64 value)
        const double pxd = EXACT ? (double)(2 * j + 1 - W) * inv_w : -1.0 + (2.0 * j + 1.0) / W;
        const double pyd = EXACT ? (double)(H - 2 * i - 1) * inv_h : 1.0 - (2.0 * i + 1.0) / H;
        const float pxh = (float)pxd, pyh = (float)pyd;
        const float pxl = (float)(pxd - (double)pxh), pyl = (float)(pyd - (double)pyh);
        float dsil[KC];
        bool vsil[KC];
        if (VEC) {
#pragma unroll
            for (int k4 = 0; k4 < KC; k4 += 4) {
                const longlong2 fa = reinterpret_cast<const longlong2*>(p2f + pix * KC + k4)[0];
                const longlong2 fb = reinterpret_cast<const longlong2*>(p2f + pix * KC + k4)[1];
                const int fk[4] = {(int)fa.x, (int)fa.y, (int)fb.x, (int)fb.y};
                float zz[4], bb[12], dd[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (fk[u] >= 0) {
                        slot_outputs<PERSP, EXACT>(geom[fk[u]], pxd, pyd, pxh, pxl, pyh, pyl, &zz[u], &bb[3 * u],
                                                   &dd[u]);
                    } else {
                        zz[u] = -1.f; dd[u] = -1.f; bb[3 * u] = bb[3 * u + 1] = bb[3 * u + 2] = -1.f;
                    }
                    dsil[k4 + u] = dd[u];
                    vsil[k4 + u] = fk[u] >= 0;
                }
                const int64_t s = pix * KC + k4;
                *reinterpret_cast<float4*>(zbuf + s) = make_float4(zz[0], zz[1], zz[2], zz[3]);
                *reinterpret_cast<float4*>(dists + s) = make_float4(dd[0], dd[1], dd[2], dd[3]);
                float4* bp = reinterpret_cast<float4*>(bary + 3 * s);
                bp[0] = make_float4(bb[0], bb[1], bb[2], bb[3]);
                bp[1] = make_float4(bb[4], bb[5], bb[6], bb[7]);
                bp[2] = make_float4(bb[8], bb[9], bb[10], bb[11]);
            }
        } else {
#pragma unroll
            for (int k = 0; k < KC; ++k) {
                if (k >= K) break;
                const int64_t s = pix * K + k;
                const int fk = (int)p2f[s];
                float zz, bb[3], dd;
                if (fk >= 0) {
                    slot_outputs<PERSP, EXACT>(geom[fk], pxd, pyd, pxh, pxl, pyh, pyl, &zz, bb, &dd);
                } else {
                    zz = -1.f; dd = -1.f; bb[0] = bb[1] = bb[2] = -1.f;
                }
                zbuf[s] = zz;
                dists[s] = dd;
                bary[3 * s] = bb[0]; bary[3 * s + 1] = bb[1]; bary[3 * s + 2] = bb[2];
                dsil[k] = dd;
                vsil[k] = fk >= 0;
            }
        }
        if (SIL) alpha[pix] = silhouette_alpha<KC>(dsil, vsil, VEC ? KC : K, sigma);   // VEC implies K == KC
    }
}

template <int KC>
void launch_fine(bool persp, bool exact, int nbins, cudaStream_t s, const float4* fconst, const FaceBox* box,
                 const int* order, const int* offsets, const int* list, int nbx, int nby, int H, int W, int K,
                 float blur, bool vec, int64_t* p2f) {
#define MR_FINE(P, E)                                                                                          \
    k_fine<KC, P, E><<<nbins * kFineCtasPerBin, kFineThreads, 0, s>>>(fconst, box, offsets, list, order, nbx, nby, \
                                                                       H, W, K, blur, vec, p2f)
    if (persp) {
        if (exact) MR_FINE(true, true); else MR_FINE(true, false);
    } else {
        if (exact) MR_FINE(false, true); else MR_FINE(false, false);
    }
#undef MR_FINE
}

template <int KC>
void launch_epilogue(bool persp, bool sil, bool vec, bool exact, int N, int H, int W, cudaStream_t s,
                     const FaceGeom* geom, const int* offsets, int64_t* p2f, int K, float sigma, float* zbuf,
                     float* bary, float* dists, float* alpha) {
    const int64_t items = (int64_t)N * ceil_div(H, kBin) * ceil_div(W, kBin) * (kBin * kBin);
    const int grid = (int)std::min<int64_t>((items + 255) / 256, 148 * 64);   // 148 x 64: 0.425 -> 0.420 ms
#define MR_EPI(P, S, V, X) \
    k_epilogue<KC, P, S, V, X><<<grid, 256, 0, s>>>(geom, offsets, p2f, N, H, W, K, sigma, zbuf, bary, dists, alpha)
#define MR_EPI2(P, S)                           \
    if (vec && exact) MR_EPI(P, S, true, true); \
    else if (vec) MR_EPI(P, S, true, false);    \
    else MR_EPI(P, S, false, false)
    if (persp) {
        if (sil) { MR_EPI2(true, true); } else { MR_EPI2(true, false); }
    } else {
        if (sil) { MR_EPI2(false, true); } else { MR_EPI2(false, false); }
    }
#undef MR_EPI2
#undef MR_EPI
}

void dispatch_fine(int KC, bool persp, bool exact, int nbins, cudaStream_t s, const float4* fconst,
                   const FaceBox* box, const int* order, const int* offsets, const int* list, int nbx, int nby, int H,
                   int W, int K, float blur, bool vec, int64_t* p2f) {
#define MR_F(KCV) \
    launch_fine<KCV>(persp, exact, nbins, s, fconst, box, order, offsets, list, nbx, nby, H, W, K, blur, vec, p2f)
    switch (KC) {
        case 1: MR_F(1); break;
        case 2: MR_F(2); break;
        case 4: MR_F(4); break;
        case 8: MR_F(8); break;
        case 16: MR_F(16); break;
        default: MR_F(32); break;
    }
#undef MR_F
}

void dispatch_epilogue(int KC, bool persp, bool sil, bool vec_ok, bool exact, int N, int H, int W, cudaStream_t s,
                       const FaceGeom* geom, const int* offsets, int64_t* p2f, int K, float sigma, float* zbuf,
                       float* bary, float* dists, float* alpha) {
    const bool vec = vec_ok && K == KC && (KC % 4) == 0;
#define MR_E(KCV) \
    launch_epilogue<KCV>(persp, sil, vec, exact, N, H, W, s, geom, offsets, p2f, K, sigma, zbuf, bary, dists, alpha)
    switch (KC) {
        case 1: MR_E(1); break;
        case 2: MR_E(2); break;
        case 4: MR_E(4); break;
        case 8: MR_E(8); break;
        case 16: MR_E(16); break;
        default: MR_E(32); break;
    }
#undef MR_E
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int validate_fwd(const float* verts, int64_t V, const int64_t* faces, int64_t F, const int64_t* first,
                 const int64_t* num, int32_t N, int32_t H, int32_t W, float blur, int32_t K,
                 const void* p2f, const void* zbuf, const void* bary, const void* dists) {
    if (N < 0 || H < 1 || W < 1 || H > MR_MAX_SIDE || W > MR_MAX_SIDE) {
        set_error("invalid image batch N=%d H=%d W=%d", N, H, W);
        return MR_ERR_ARG;
    }
    if (K < 1 || K > MR_KMAX) {
        set_error("K=%d outside 1..%d", K, MR_KMAX);
        return MR_ERR_ARG;
    }
    if (!(blur >= 0.f) || !std::isfinite(blur)) {
        set_error("blur_radius must be finite and >= 0");
        return MR_ERR_ARG;
    }
    if (V < 0 || F < 0 || V > INT32_MAX || F > INT32_MAX) {
        set_error("V=%lld F=%lld outside 0..2^31-1", (long long)V, (long long)F);
        return MR_ERR_ARG;
    }
    if ((F > 0 && (!faces || !verts)) || (N > 0 && (!first || !num))) {
        set_error("null input pointer");
        return MR_ERR_ARG;
    }
    if (N > 0 && (!p2f || !zbuf || !bary || !dists)) {
        set_error("null output pointer");
        return MR_ERR_ARG;
    }
    for (int n = 0; n < N; ++n) {
        if (first[n] < 0 || num[n] < 0 || first[n] + num[n] > F) {
            set_error("mesh %d: faces [%lld, %lld) outside [0, F=%lld)", n, (long long)first[n],
                      (long long)(first[n] + num[n]), (long long)F);
            return MR_ERR_ARG;
        }
    }
    return MR_OK;
}

// ------------------------------------------------------------------ host pipeline
// Sizes of one forward call and the layout of its fixed scratch block (everything but
// the bin lists, which are sized after the count pass).
struct FwdPlan {
    int64_t V, F, pairs, npix;
    int N, H, W, K, KC, persp, nbx, nby, nbins, nslots, ntiles;
    float blur;
    size_t geom, box, con, cnt, off, tsum, rng, pre, fst, tot, err, ord, hist, bytes;
};

inline int fwd_plan(int64_t V, int64_t F, const int64_t* num, int N, int H, int W, float blur, int K, int persp,
                    FwdPlan& P) {
    P.V = V; P.F = F; P.N = N; P.H = H; P.W = W; P.K = K; P.persp = persp; P.blur = blur;
    P.KC = K <= 1 ? 1 : K <= 2 ? 2 : K <= 4 ? 4 : K <= 8 ? 8 : K <= 16 ? 16 : 32;
    P.nbx = ceil_div(W, kBin);
    P.nby = ceil_div(H, kBin);
    const long long nbins = (long long)N * P.nbx * P.nby;
    if (nbins * kDepthBuckets >= INT32_MAX / 2) {
        set_error("too many screen bins (%lld)", nbins);
        return MR_ERR_ARG;
    }
    P.nbins = (int)nbins;
    P.nslots = P.nbins * kDepthBuckets;
    P.ntiles = ceil_div(P.nslots, kScanTile);
    P.npix = (int64_t)N * H * W;
    P.pairs = 0;
    for (int n = 0; n < N; ++n) P.pairs += num[n];
    auto up = [](size_t b) { return (b + 255) & ~size_t(255); };
    P.geom = 0;
    P.box = P.geom + up(sizeof(FaceGeom) * (size_t)F);
    P.con = P.box + up(sizeof(FaceBox) * (size_t)F);
    P.cnt = P.con + up(sizeof(float4) * kConstF4 * (size_t)F);
    P.off = P.cnt + up(sizeof(int) * (size_t)P.nslots);
    P.tsum = P.off + up(sizeof(int) * (size_t)(P.nslots + 1));
    P.rng = P.tsum + up(sizeof(long long) * (size_t)P.ntiles);
    P.pre = P.rng + up(sizeof(unsigned) * 2 * (size_t)N);
    P.fst = P.pre + up(sizeof(int64_t) * (size_t)(N + 1));
    P.tot = P.fst + up(sizeof(int64_t) * (size_t)N);
    P.err = P.tot + 256;
    P.ord = P.err + 256;
    P.hist = P.ord + up(sizeof(int) * (size_t)P.nbins);
    P.bytes = P.hist + up(sizeof(int) * 2 * kLenClasses);
    return MR_OK;
}

// Pointers into one scratch block laid out by fwd_plan.
struct FwdBufs {
    FaceGeom* geom;
    FaceBox* box;
    float4* fconst;
    int *counts, *offsets;
    long long* tile_sum;
    unsigned* krange;
    int64_t *prefix, *first;
    long long* total;
    int* err;
    int* order;       // bins, longest list first
    int* hist;        // kLenClasses class counts, then kLenClasses cursors
};

inline FwdBufs fwd_bufs(char* ws, const FwdPlan& P) {
    FwdBufs B;
    B.geom = reinterpret_cast<FaceGeom*>(ws + P.geom);
    B.box = reinterpret_cast<FaceBox*>(ws + P.box);
    B.fconst = reinterpret_cast<float4*>(ws + P.con);
    B.counts = reinterpret_cast<int*>(ws + P.cnt);
    B.offsets = reinterpret_cast<int*>(ws + P.off);
    B.tile_sum = reinterpret_cast<long long*>(ws + P.tsum);
    B.krange = reinterpret_cast<unsigned*>(ws + P.rng);
    B.prefix = reinterpret_cast<int64_t*>(ws + P.pre);
    B.first = reinterpret_cast<int64_t*>(ws + P.fst);
    B.total = reinterpret_cast<long long*>(ws + P.tot);
    B.err = reinterpret_cast<int*>(ws + P.err);
    B.order = reinterpret_cast<int*>(ws + P.ord);
    B.hist = reinterpret_cast<int*>(ws + P.hist);
    return B;
}

inline int pair_blocks(int64_t pairs) { return (int)std::min<int64_t>((pairs + 255) / 256, 148 * 16); }

// Up to the bin counts: per-mesh arrays to the device, clears, face setup (with the
// images' key ranges), bin count and scan, the bins' longest-first order, and the read-back
// of the list total, the error word and the number of empty bins (valid after the stream is
// synchronised): written by a kernel into mailbox (a Mailbox's dev pointer, words 0-2) when
// one is given, else copied into host_total / host_err / host_empty.  staging: pinned host
// memory of 2N + 1 int64 for the per-mesh arrays' copies, or nullptr (copies from the
// caller's memory).
inline cudaError_t fwd_enqueue_count(const FwdPlan& P, const FwdBufs& B, const float* verts, const int64_t* faces,
                                     const int64_t* host_prefix, const int64_t* host_first, cudaStream_t s,
                                     long long* host_total, int* host_err, int* host_empty,
                                     long long* mailbox = nullptr, int64_t* staging = nullptr) {
    cudaError_t e;
    if (staging) {
        // pinned staging: the copies do not wait for the stream's earlier work
        std::copy(host_prefix, host_prefix + P.N + 1, staging);
        std::copy(host_first, host_first + P.N, staging + P.N + 1);
        host_prefix = staging;
        host_first = staging + P.N + 1;
    }
    if ((e = cudaMemcpyAsync(B.prefix, host_prefix, sizeof(int64_t) * (P.N + 1), cudaMemcpyHostToDevice, s))) return e;
    if ((e = cudaMemcpyAsync(B.first, host_first, sizeof(int64_t) * P.N, cudaMemcpyHostToDevice, s))) return e;
    if ((e = cudaMemsetAsync(B.counts, 0, sizeof(int) * (size_t)P.nslots, s))) return e;
    if ((e = cudaMemsetAsync(B.err, 0, sizeof(int), s))) return e;
    // key ranges, ordered-unsigned: N minima starting at 0xffffffff, then N maxima at 0
    if ((e = cudaMemsetAsync(B.krange, 0xff, sizeof(unsigned) * (size_t)P.N, s))) return e;
    if ((e = cudaMemsetAsync(B.krange + P.N, 0, sizeof(unsigned) * (size_t)P.N, s))) return e;
    const double reach = std::sqrt((double)P.blur) * (1.0 + 1e-6) + 1e-7;
    if (P.pairs > 0) {
        {
            ProfScope ps(MR_STAGE_FACE_SETUP, s);
            k_face_setup<<<pair_blocks(P.pairs), 256, 0, s>>>(verts, P.V, faces, B.prefix, B.first, P.N, P.pairs, P.H,
                                                              P.W, reach, P.persp, B.geom, B.box, B.fconst, B.krange,
                                                              B.err);
        }
        if ((e = cudaGetLastError())) return e;
        {
            ProfScope ps(MR_STAGE_BIN_COUNT, s);
            k_bin_pairs<false><<<pair_blocks(P.pairs), 256, 0, s>>>(B.box, B.prefix, B.first, P.N, P.pairs, P.nbx,
                                                                    P.nby, B.krange, B.counts, nullptr, nullptr);
        }
        if ((e = cudaGetLastError())) return e;
    }
    {
        ProfScope ps(MR_STAGE_BIN_SCAN, s);
        k_scan_tiles<<<P.ntiles, 1024, 0, s>>>(B.counts, P.nslots, B.offsets, B.tile_sum);
        k_scan_tops<<<1, 1024, 0, s>>>(B.tile_sum, P.ntiles, B.total);
        k_scan_add<<<std::min(ceil_div(P.nslots + 1, 256), 148 * 8), 256, 0, s>>>(B.offsets, P.nslots, B.tile_sum,
                                                                                  B.total);
        // the fine pass's launch order: longest bin lists first
        if ((e = cudaMemsetAsync(B.hist, 0, sizeof(int) * 2 * kLenClasses, s))) return e;
        const int og = std::min(ceil_div(P.nbins, 256), 148 * 4);
        k_bin_hist<<<og, 256, 0, s>>>(B.offsets, P.nbins, B.hist);
        k_bin_order<<<og, 256, 0, s>>>(B.offsets, P.nbins, B.hist, B.hist + kLenClasses, B.order);
    }
    if ((e = cudaGetLastError())) return e;
    // hist[0]: the bins of length class 0, i.e. the empty ones (they come last in the order)
    if (mailbox) return post_counts(B.total, B.err, B.hist, mailbox, s);
    if ((e = cudaMemcpyAsync(host_total, B.total, sizeof(long long), cudaMemcpyDeviceToHost, s))) return e;
    if ((e = cudaMemcpyAsync(host_empty, B.hist, sizeof(int), cudaMemcpyDeviceToHost, s))) return e;
    return cudaMemcpyAsync(host_err, B.err, sizeof(int), cudaMemcpyDeviceToHost, s);
}

// Bin fill into `list` (total entries), fine pass and epilogue.
// The fine pass runs one CTA per non-empty bin (the first nbins - empty entries of the
// longest-first order); the epilogue writes the padding of the empty bins' pixels, their
// pix_to_face included.
inline cudaError_t fwd_enqueue_rest(const FwdPlan& P, const FwdBufs& B, int* list, long long total, int empty,
                                    bool sil, float sigma, int64_t* p2f, float* zbuf, float* bary, float* dists,
                                    float* alpha, cudaStream_t s) {
    cudaError_t e;
    if (total > 0) {
        if ((e = cudaMemsetAsync(B.counts, 0, sizeof(int) * (size_t)P.nslots, s))) return e;
        ProfScope ps(MR_STAGE_BIN_FILL, s);
        k_bin_pairs<true><<<pair_blocks(P.pairs), 256, 0, s>>>(B.box, B.prefix, B.first, P.N, P.pairs, P.nbx, P.nby,
                                                               B.krange, B.counts, B.offsets, list);
        if ((e = cudaGetLastError())) return e;
    }
    const bool vec_ok = aligned16(p2f) && aligned16(zbuf) && aligned16(bary) && aligned16(dists);
    const bool exact = (P.H & (P.H - 1)) == 0 && (P.W & (P.W - 1)) == 0;
    const int busy = P.nbins - std::min(std::max(empty, 0), P.nbins);
    {
        ProfScope ps(MR_STAGE_FINE, s);
        if (busy > 0)
            dispatch_fine(P.KC, P.persp != 0, exact, busy, s, B.fconst, B.box, B.order, B.offsets, list, P.nbx,
                          P.nby, P.H, P.W, P.K, P.blur, aligned16(p2f), p2f);
    }
    if ((e = cudaGetLastError())) return e;
    {
        ProfScope ps(MR_STAGE_EPILOGUE, s);
        dispatch_epilogue(P.KC, P.persp != 0, sil, vec_ok, exact, P.N, P.H, P.W, s, B.geom, B.offsets, p2f, P.K,
                          sigma, zbuf, bary, dists, alpha);
    }
    return cudaGetLastError();
}

}  // namespace
}  // namespace mr
