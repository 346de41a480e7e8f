// Shared definitions of the sm_100a mesh rasterizer library (internal header).
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include <cstdio>
#include <initializer_list>
#include <string>
#include <vector>

#include "meshrast.h"

namespace mr {

// Screen tile of the coarse pass and of one fine-pass CTA: 16 x 16 pixels, split into
// eight 8 x 4 warp tiles (two across, four down).
constexpr int kBin = 16;
constexpr int kWarpTileW = 8;
constexpr int kWarpTileH = 4;
constexpr int kWarpsPerBin = (kBin / kWarpTileW) * (kBin / kWarpTileH);   // 8
// The fine pass runs a bin as two CTAs of four warps: a CTA retires when its slowest warp
// does, and half-bin CTAs hold fewer finished warps' slots (1.379 -> 1.357 ms against one
// CTA of eight warps per bin; two or one warp per CTA: 1.365 / 1.418 ms).
constexpr int kFineWarps = 4;
constexpr int kFineCtasPerBin = kWarpsPerBin / kFineWarps;                 // 2
constexpr int kFineThreads = kFineWarps * 32;                              // 128
constexpr double kDegenerateArea = 1e-12;

// Two float32 lanes in one 64-bit register pair, and the packed (sm_100) arithmetic on
// them; each lane is rounded exactly as the scalar instruction would round it.
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 pack2(float lo, float hi) {
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unpack2(f32x2 v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
    f32x2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Asynchronous 16-byte global -> shared copies (no register round trip); a thread sees
// its own copies after cp_wait_all, the other lanes' after a following __syncwarp.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_wait_all() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

// Device error bits.
constexpr int kErrFaceIndex = 1;    // a face vertex id outside [0, V)
constexpr int kErrSlotIndex = 2;    // a pix_to_face entry outside [-1, F)

// Face geometry as written by the setup pass: the three vertices in their original
// order (x, y, z, unused).  Exact copies of the caller's float32 values.
struct __align__(16) FaceGeom {
    float4 a, b, c;
};

// Inclusive pixel box of a face grown by sqrt(blur_radius), clipped to the image, and a
// lower bound of the face's depth key over the pixel centres of that box.  x0 > x1 marks
// a face that touches no pixel (off-screen or degenerate).
struct __align__(16) FaceBox {
    short x0, x1, y0, y1;
    float kmin;
    int unused;
};

void set_error(const char* fmt, ...);
int cuda_fail(cudaError_t e, const char* what);

#define MR_CUDA(call)                                        \
    do {                                                     \
        cudaError_t e_ = (call);                             \
        if (e_ != cudaSuccess) return ::mr::cuda_fail(e_, #call); \
    } while (0)

// Per-mesh (per-cloud) index arrays may be given in host or in device memory.  Each
// pointer in `arrays` that is device memory is replaced by a host copy of its n entries
// held in `buf` (one device-to-host copy per array on stream s, then one synchronisation
// of s); host-readable pointers are left as they are.
int host_indices(cudaStream_t s, int64_t n, std::vector<int64_t>& buf,
                 std::initializer_list<const int64_t**> arrays);

// A mapped (zero-copy) pinned host buffer of 64 bytes (three 64-bit words in use), one per
// calling thread and device: the values a call reads back in the middle (a list total, the
// device error word, a count) are written there by a kernel, so reading them needs no copy engine -- a copy
// would queue behind the caller's own large transfers on that engine.  dev is nullptr when
// no such buffer can be had; the caller then copies instead.
struct Mailbox {
    volatile long long* host;
    long long* dev;
};
Mailbox host_mailbox();
// Pinned host memory of at least `bytes`, one growing buffer per calling thread and
// device, or nullptr when it cannot be had.  Host-to-device copies of small per-call arrays
// go through it: a copy from pageable memory may first synchronise the stream (to stage
// the data), which leaves the GPU idle until the call has launched its first kernel.  The
// buffer may be rewritten by the thread's next call, so a caller only uses it for copies
// that its own stream synchronisation has completed before it returns.
void* host_staging(size_t bytes);

// Enqueues on s: out[0] = *total, out[1] = err ? *err : 0, out[2] = extra ? *extra : 0 (out: a
// Mailbox's dev pointer).
cudaError_t post_counts(const long long* total, const int* err, const int* extra, long long* out, cudaStream_t s);

// Scratch allocation on the caller's stream (stream-ordered pool).
int scratch_alloc(void** p, size_t bytes, cudaStream_t s);
void scratch_free(void* p, cudaStream_t s);

// Grid of 256-thread blocks for a grid-stride loop over n items: at most 32 blocks per
// SM of the 148.
inline int grid_for(int64_t n) { return (int)(n < 148 * 32 * 256 ? (n + 255) / 256 : 148 * 32); }

// Row i and column j of flat pixel index q (images of H x W, row-major): 32-bit division
// when q fits (64-bit division costs several times more).
__device__ __forceinline__ void pixel_rc(int64_t q, int H, int W, int& i, int& j) {
    if (q <= 0x7fffffff) {
        const unsigned r = (unsigned)q % ((unsigned)H * (unsigned)W);
        i = (int)(r / (unsigned)W);
        j = (int)(r - (unsigned)i * (unsigned)W);
    } else {
        const int64_t r = q % ((int64_t)H * W);
        i = (int)(r / W);
        j = (int)(r % W);
    }
}

// Centre of pixel column j in NDC, -1 + (2j + 1) / W, in float64; inv_w = 1.0 / W.  For W a
// power of two 1/W is exact and so is the product: the same value without a division.
__device__ __forceinline__ double pixel_x(int j, int W, double inv_w) {
    return (W & (W - 1)) == 0 ? (double)(2 * j + 1 - W) * inv_w : -1.0 + (2.0 * j + 1.0) / W;
}
// Centre of pixel row i, 1 - (2i + 1) / H.
__device__ __forceinline__ double pixel_y(int i, int H, double inv_h) {
    return (H & (H - 1)) == 0 ? (double)(H - 2 * i - 1) * inv_h : 1.0 - (2.0 * i + 1.0) / H;
}

// 16-byte loads and stores of N consecutive values (N a multiple of 4 floats or 2 int64;
// the address 16-byte aligned).
template <int N>
__device__ __forceinline__ void ld_vec(const float* __restrict__ a, float (&v)[N]) {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
        const float4 t = reinterpret_cast<const float4*>(a)[i];
        v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
}
template <int N>
__device__ __forceinline__ void st_vec(float* __restrict__ a, const float (&v)[N]) {
#pragma unroll
    for (int i = 0; i < N / 4; ++i)
        reinterpret_cast<float4*>(a)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}
template <int N>
__device__ __forceinline__ void ld_vec(const int64_t* __restrict__ a, int64_t (&v)[N]) {
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
        const longlong2 t = reinterpret_cast<const longlong2*>(a)[i];
        v[2 * i] = t.x; v[2 * i + 1] = t.y;
    }
}

// Device-wide sticky error word (asynchronous kernels).
int* device_error_word();

// Stage timing: while profiling is enabled, a ProfScope records a CUDA event pair
// around the launches in its scope on stream s.
bool profiling_enabled();
void profile_record(int stage, cudaEvent_t start, cudaEvent_t stop);
cudaEvent_t profile_event();
// Each scope is also an NVTX range named after its stage (host-side enqueue of the stage's
// launches; free unless a tracing tool is attached).
const char* stage_name(int stage);
struct ProfScope {
    int stage;
    cudaStream_t s;
    cudaEvent_t a = nullptr, b = nullptr;
    ProfScope(int st, cudaStream_t str) : stage(st), s(str) {
        nvtxRangePushA(stage_name(st));
        if (profiling_enabled()) {
            a = profile_event();
            b = profile_event();
            if (a && b) cudaEventRecord(a, s);
        }
    }
    ~ProfScope() {
        if (a && b) {
            cudaEventRecord(b, s);
            profile_record(stage, a, b);
        }
        nvtxRangePop();
    }
};

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace mr
