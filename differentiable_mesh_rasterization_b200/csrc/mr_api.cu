// Host-side plumbing of the C ABI: error reporting, stream-ordered scratch, the device
// error word and the status query.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "mr_common.cuh"

namespace {
thread_local char g_last_error[512] = "";
__device__ int g_device_error = 0;
std::mutex g_pool_mutex;
bool g_pool_ready[64] = {};

struct ProfEntry {
    int stage;
    cudaEvent_t a, b;
};
std::mutex g_prof_mutex;
bool g_prof_on = false;
std::vector<ProfEntry> g_prof_pending;
std::vector<cudaEvent_t> g_prof_free;

// One-shot failure of the scratch allocator, armed by mr_inject_fault (tests only).
std::atomic<int> g_inject_kind{0};
std::atomic<int> g_inject_skip{0};
}  // namespace

namespace mr {

void set_error(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
}

int cuda_fail(cudaError_t e, const char* what) {
    set_error("%s failed: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
    return MR_ERR_CUDA;
}

// Freed scratch stays in the device's default pool instead of returning to the driver
// at every synchronisation; the attribute is per process and per device.
static int ensure_pool(int dev) {
    if (dev < 0 || dev >= 64) return MR_OK;
    std::lock_guard<std::mutex> g(g_pool_mutex);
    if (g_pool_ready[dev]) return MR_OK;
    cudaMemPool_t pool;
    MR_CUDA(cudaDeviceGetDefaultMemPool(&pool, dev));
    uint64_t keep = UINT64_MAX;
    MR_CUDA(cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep));
    g_pool_ready[dev] = true;
    return MR_OK;
}

int scratch_alloc(void** p, size_t bytes, cudaStream_t s) {
    *p = nullptr;
    if (bytes == 0) return MR_OK;
    const int kind = g_inject_kind.load();
    if (kind != MR_INJECT_OFF && g_inject_skip.fetch_sub(1) <= 0) {
        g_inject_kind.store(MR_INJECT_OFF);        // one shot: disarmed before returning
        if (kind == MR_INJECT_OOM) {
            set_error("scratch allocation of %zu bytes failed (injected)", bytes);
            return MR_ERR_OOM;
        }
        set_error("cudaMallocAsync failed: cudaErrorLaunchFailure (injected)");
        return MR_ERR_CUDA;
    }
    int dev = 0;
    MR_CUDA(cudaGetDevice(&dev));
    int rc = ensure_pool(dev);
    if (rc != MR_OK) return rc;
    cudaError_t e = cudaMallocAsync(p, bytes, s);
    if (e == cudaErrorMemoryAllocation) {
        cudaGetLastError();
        set_error("scratch allocation of %zu bytes failed", bytes);
        return MR_ERR_OOM;
    }
    if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync");
    return MR_OK;
}

void scratch_free(void* p, cudaStream_t s) {
    if (p) cudaFreeAsync(p, s);
}

namespace {
__global__ void k_post_counts(const long long* __restrict__ total, const int* __restrict__ err,
                              const int* __restrict__ extra, long long* __restrict__ out) {
    out[0] = *total;
    out[1] = err ? (long long)*err : 0;
    out[2] = extra ? (long long)*extra : 0;
    __threadfence_system();
}

struct MailboxSlots {
    Mailbox m[64] = {};
    bool tried[64] = {};
};
thread_local MailboxSlots g_mail;
}  // namespace

Mailbox host_mailbox() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return Mailbox{nullptr, nullptr};
    }
    if (!g_mail.tried[dev]) {
        g_mail.tried[dev] = true;
        void* h = nullptr;
        void* d = nullptr;
        // 64 bytes per thread and device, kept for the life of the thread
        if (cudaHostAlloc(&h, 64, cudaHostAllocMapped | cudaHostAllocPortable) == cudaSuccess &&
            cudaHostGetDevicePointer(&d, h, 0) == cudaSuccess) {
            g_mail.m[dev] = Mailbox{static_cast<volatile long long*>(h), static_cast<long long*>(d)};
        } else {
            cudaGetLastError();
            if (h) cudaFreeHost(h);
        }
    }
    return g_mail.m[dev];
}

namespace {
struct StagingSlots {
    void* p[64] = {};
    size_t cap[64] = {};
};
thread_local StagingSlots g_stage;
}  // namespace

void* host_staging(size_t bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return nullptr;
    }
    if (g_stage.cap[dev] < bytes) {
        if (g_stage.p[dev]) cudaFreeHost(g_stage.p[dev]);
        g_stage.p[dev] = nullptr;
        g_stage.cap[dev] = 0;
        const size_t want = std::max<size_t>(bytes, 4096);
        void* h = nullptr;
        if (cudaHostAlloc(&h, want, cudaHostAllocPortable) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_stage.p[dev] = h;
        g_stage.cap[dev] = want;
    }
    return g_stage.p[dev];
}

cudaError_t post_counts(const long long* total, const int* err, const int* extra, long long* out, cudaStream_t s) {
    k_post_counts<<<1, 1, 0, s>>>(total, err, extra, out);
    return cudaGetLastError();
}

int host_indices(cudaStream_t s, int64_t n, std::vector<int64_t>& buf,
                 std::initializer_list<const int64_t**> arrays) {
    if (n <= 0) return MR_OK;
    std::vector<const int64_t**> on_device;
    for (const int64_t** a : arrays) {
        if (!*a) continue;
        cudaPointerAttributes at;
        if (cudaPointerGetAttributes(&at, *a) != cudaSuccess) {
            cudaGetLastError();          // a pointer CUDA does not know: plain host memory
            continue;
        }
        if (at.type == cudaMemoryTypeDevice) on_device.push_back(a);
    }
    if (on_device.empty()) return MR_OK;
    buf.resize((size_t)n * on_device.size());
    for (size_t i = 0; i < on_device.size(); ++i)
        MR_CUDA(cudaMemcpyAsync(buf.data() + i * n, *on_device[i], sizeof(int64_t) * (size_t)n,
                                cudaMemcpyDeviceToHost, s));
    MR_CUDA(cudaStreamSynchronize(s));
    for (size_t i = 0; i < on_device.size(); ++i) *on_device[i] = buf.data() + i * n;
    return MR_OK;
}

bool profiling_enabled() { return g_prof_on; }

const char* stage_name(int stage) {
    static const char* const names[MR_NUM_STAGES] = {
        "mr:face_setup", "mr:bin_count", "mr:bin_scan", "mr:bin_fill", "mr:fine", "mr:silhouette_fwd",
        "mr:silhouette_bwd", "mr:raster_bwd", "mr:silhouette_raster_bwd", "mr:epilogue", "mr:interpolate_fwd",
        "mr:interpolate_bwd", "mr:blend_fwd", "mr:blend_bwd", "mr:phong_fwd", "mr:phong_bwd", "mr:phong_shade_fwd",
        "mr:phong_shade_bwd", "mr:points_bin", "mr:points_fine", "mr:points_bwd", "mr:composite_fwd",
        "mr:composite_bwd", "mr:knn", "mr:knn_bwd"};
    return stage >= 0 && stage < MR_NUM_STAGES ? names[stage] : "mr:stage";
}

cudaEvent_t profile_event() {
    std::lock_guard<std::mutex> g(g_prof_mutex);
    if (!g_prof_free.empty()) {
        cudaEvent_t e = g_prof_free.back();
        g_prof_free.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return e;
}

void profile_record(int stage, cudaEvent_t a, cudaEvent_t b) {
    std::lock_guard<std::mutex> g(g_prof_mutex);
    g_prof_pending.push_back(ProfEntry{stage, a, b});
}

int* device_error_word() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return static_cast<int*>(p);
}

}  // namespace mr

namespace mr {
// Independent FFMA chains (8 per thread, each 4 deep per iteration) for the issue-rate
// probe; the result is stored only if it is exactly zero, which never happens for a
// multiplier above 1, so nothing is optimised away and nothing is written.
__global__ void __launch_bounds__(256) k_fma_probe(int iters, float m, float* __restrict__ sink) {
    float x[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) x[c] = (float)(threadIdx.x + c) * 1e-3f;
    for (int it = 0; it < iters; ++it)
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 8; ++c) x[c] = fmaf(x[c], m, 1e-7f);
    float t = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) t += x[c];
    if (t == 0.f) sink[blockIdx.x * blockDim.x + threadIdx.x] = t;
}
}  // namespace mr

extern "C" {

const char* mr_last_error(void) { return g_last_error; }

int mr_profile_enable(int32_t on) {
    std::lock_guard<std::mutex> g(g_prof_mutex);
    g_prof_on = on != 0;
    return MR_OK;
}

int mr_profile_read(double* stage_ms, int64_t* launches, int32_t nstages) {
    std::vector<ProfEntry> pending;
    {
        std::lock_guard<std::mutex> g(g_prof_mutex);
        pending.swap(g_prof_pending);
    }
    for (int i = 0; i < nstages; ++i) {
        if (stage_ms) stage_ms[i] = 0.0;
        if (launches) launches[i] = 0;
    }
    int rc = MR_OK;
    for (const ProfEntry& e : pending) {
        float ms = 0.f;
        cudaError_t err = cudaEventSynchronize(e.b);
        if (err == cudaSuccess) err = cudaEventElapsedTime(&ms, e.a, e.b);
        if (err != cudaSuccess && rc == MR_OK) rc = mr::cuda_fail(err, "cudaEventElapsedTime");
        if (e.stage >= 0 && e.stage < nstages) {
            if (stage_ms) stage_ms[e.stage] += ms;
            if (launches) launches[e.stage] += 1;
        }
    }
    std::lock_guard<std::mutex> g(g_prof_mutex);
    for (const ProfEntry& e : pending) {
        g_prof_free.push_back(e.a);
        g_prof_free.push_back(e.b);
    }
    return rc;
}

int mr_version(void) { return 10000; }

int mr_inject_fault(int32_t kind, int32_t skip) {
    if (kind < MR_INJECT_OFF || kind > MR_INJECT_CUDA || skip < 0) {
        mr::set_error("mr_inject_fault: kind=%d skip=%d", kind, skip);
        return MR_ERR_ARG;
    }
    g_inject_kind.store(MR_INJECT_OFF);
    g_inject_skip.store(skip);
    g_inject_kind.store(kind);
    return MR_OK;
}

int mr_scratch_peak(int64_t* bytes, int32_t reset) {
    if (!bytes) {
        mr::set_error("null output");
        return MR_ERR_ARG;
    }
    int dev = 0;
    MR_CUDA(cudaGetDevice(&dev));
    cudaMemPool_t pool;
    MR_CUDA(cudaDeviceGetDefaultMemPool(&pool, dev));
    uint64_t high = 0;
    MR_CUDA(cudaMemPoolGetAttribute(pool, cudaMemPoolAttrUsedMemHigh, &high));
    *bytes = (int64_t)high;
    if (reset) {
        uint64_t zero = 0;
        MR_CUDA(cudaMemPoolSetAttribute(pool, cudaMemPoolAttrUsedMemHigh, &zero));
    }
    return MR_OK;
}

int mr_scratch_in_use(int64_t* bytes) {
    if (!bytes) {
        mr::set_error("null output");
        return MR_ERR_ARG;
    }
    int dev = 0;
    MR_CUDA(cudaGetDevice(&dev));
    cudaMemPool_t pool;
    MR_CUDA(cudaDeviceGetDefaultMemPool(&pool, dev));
    uint64_t used = 0;
    MR_CUDA(cudaMemPoolGetAttribute(pool, cudaMemPoolAttrUsedMemCurrent, &used));
    *bytes = (int64_t)used;
    return MR_OK;
}

int mr_measure_fp32_peak(double* inst_per_s, void* stream) {
    if (!inst_per_s) {
        mr::set_error("null output");
        return MR_ERR_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int dev = 0, sms = 0;
    MR_CUDA(cudaGetDevice(&dev));
    MR_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    // five timed launches of ~11 ms each after a warm-up; the fastest one counts, so launch
    // and tail effects and a clock still ramping up do not lower the peak
    const int blocks = sms * 8, iters = 40960, runs = 5;
    float* sink = nullptr;
    int rc = mr::scratch_alloc(reinterpret_cast<void**>(&sink), sizeof(float) * (size_t)blocks * 256, s);
    if (rc != MR_OK) return rc;
    cudaEvent_t a = nullptr, b = nullptr;
    cudaError_t e = cudaEventCreate(&a);
    if (e == cudaSuccess) e = cudaEventCreate(&b);
    float ms = 0.f;
    if (e == cudaSuccess) {
        mr::k_fma_probe<<<blocks, 256, 0, s>>>(iters, 1.0001f, sink);   // warm-up
        for (int r = 0; r < runs && e == cudaSuccess; ++r) {
            cudaEventRecord(a, s);
            mr::k_fma_probe<<<blocks, 256, 0, s>>>(iters, 1.0001f, sink);
            cudaEventRecord(b, s);
            e = cudaGetLastError();
            float t = 0.f;
            if (e == cudaSuccess) e = cudaEventSynchronize(b);
            if (e == cudaSuccess) e = cudaEventElapsedTime(&t, a, b);
            if (e == cudaSuccess && t > 0.f && (ms == 0.f || t < ms)) ms = t;
        }
    }
    if (a) cudaEventDestroy(a);
    if (b) cudaEventDestroy(b);
    mr::scratch_free(sink, s);
    if (e != cudaSuccess) return mr::cuda_fail(e, "fp32 probe");
    if (!(ms > 0.f)) {
        mr::set_error("fp32 probe: no elapsed time");
        return MR_ERR_CUDA;
    }
    // 8 chains x 4 FFMA per iteration and thread
    *inst_per_s = (double)blocks * 256.0 * iters * 32.0 / (ms * 1e-3);
    return MR_OK;
}

int mr_device_status(void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int* w = mr::device_error_word();
    if (!w) {
        mr::set_error("cannot locate the device error word");
        return MR_ERR_CUDA;
    }
    int host = 0;
    MR_CUDA(cudaMemcpyAsync(&host, w, sizeof(int), cudaMemcpyDeviceToHost, s));
    MR_CUDA(cudaStreamSynchronize(s));
    if (host != 0) {
        MR_CUDA(cudaMemsetAsync(w, 0, sizeof(int), s));
        MR_CUDA(cudaStreamSynchronize(s));
        mr::set_error("a kernel skipped %s",
                      (host & mr::kErrFaceIndex) ? "a face with a vertex id outside [0, V)"
                                                 : "a pix_to_face entry outside [-1, F)");
        return MR_ERR_DEVICE;
    }
    g_last_error[0] = '\0';
    return MR_OK;
}

}  // extern "C"
