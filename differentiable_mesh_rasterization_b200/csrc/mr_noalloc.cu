// mr_rasterize_fwd_noalloc: stage one of the rasterizer for callers that must not
// allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the moment they render: a
// host that has handed all device memory to its own pool and forbids the driver from
// carving out more, a latency-critical loop where an allocation could block or fail
// under memory pressure, or a plugin that runs inside someone else's memory budget.
// For them this entry point runs the same kernels as mr_rasterize_fwd, but every byte
// of scratch (face records, per-bin counts, their launch order and the bin lists) comes from
// one file-scope device array of fixed size.  The caller still provides the inputs and
// the outputs.
//
// The array is MR_NOALLOC_SCRATCH_BYTES (64 MiB) on every device that loads this part
// of the library and stays there until the process exits.  Its address is looked up
// once per device, by the first call made on that device with the device current; make
// that first call before any stream capture.  Like mr_rasterize_fwd, every call
// synchronises its stream once, after the bin count, to learn the size of the bin lists
// (and once before, when the per-mesh arrays are device memory).  All calls share the
// array and it keeps the previous call's contents (the parts that must start at zero are
// cleared on every call), so two calls whose work overlaps on the GPU -- on different
// streams, or from different threads -- race on it; order them on one stream.
#include <mutex>

#include "mr_forward_kernels.cuh"

static __device__ __align__(256) unsigned char g_noalloc_scratch[MR_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mutex;
char* g_noalloc_ptr[64] = {};

// Device address of the scratch array on the current device (looked up once per device).
int noalloc_scratch(char** out) {
    int dev = 0;
    MR_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) {
        mr::set_error("device ordinal %d outside 0..63", dev);
        return MR_ERR_ARG;
    }
    std::lock_guard<std::mutex> g(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return mr::cuda_fail(e, "cudaGetSymbolAddress(scratch)");
        g_noalloc_ptr[dev] = static_cast<char*>(p);
    }
    *out = g_noalloc_ptr[dev];
    return MR_OK;
}

}  // namespace

namespace mr {
namespace {

int rasterize_noalloc(const float* verts, int64_t V, const int64_t* faces, int64_t F, const int64_t* first,
                      const int64_t* num, int32_t N, int32_t H, int32_t W, float blur, int32_t K, int32_t persp,
                      int64_t* p2f, float* zbuf, float* bary, float* dists, cudaStream_t s) {
    std::vector<int64_t> staged;
    if (N > 0) {
        int rs = host_indices(s, N, staged, {&first, &num});
        if (rs != MR_OK) return rs;
    }
    int rc = validate_fwd(verts, V, faces, F, first, num, N, H, W, blur, K, p2f, zbuf, bary, dists);
    if (rc != MR_OK) return rc;
    if (N == 0) return MR_OK;
    FwdPlan P;
    rc = fwd_plan(V, F, num, N, H, W, blur, K, persp, P);
    if (rc != MR_OK) return rc;
    if (P.bytes > (size_t)MR_NOALLOC_SCRATCH_BYTES) {
        set_error("mr_rasterize_fwd_noalloc: this batch needs %zu bytes of scratch before its bin lists, more "
                  "than the fixed %d bytes; use mr_rasterize_fwd", P.bytes, MR_NOALLOC_SCRATCH_BYTES);
        return MR_ERR_ARG;
    }
    char* ws = nullptr;
    rc = noalloc_scratch(&ws);
    if (rc != MR_OK) return rc;
    std::vector<int64_t> prefix(N + 1, 0);
    for (int n = 0; n < N; ++n) prefix[n + 1] = prefix[n] + num[n];
    const FwdBufs B = fwd_bufs(ws, P);
    int* list = reinterpret_cast<int*>(ws + P.bytes);     // the bin lists follow the fixed block
    long long total = 0;
    int herr = 0, empty = 0;
    MR_CUDA(fwd_enqueue_count(P, B, verts, faces, prefix.data(), first, s, &total, &herr, &empty));
    MR_CUDA(cudaStreamSynchronize(s));
    if (total < 0 || P.bytes + sizeof(int) * (size_t)total > (size_t)MR_NOALLOC_SCRATCH_BYTES) {
        set_error("mr_rasterize_fwd_noalloc: the bin lists need %lld entries, more than the %zu left of the "
                  "fixed %d-byte scratch; use mr_rasterize_fwd", total,
                  ((size_t)MR_NOALLOC_SCRATCH_BYTES - P.bytes) / sizeof(int), MR_NOALLOC_SCRATCH_BYTES);
        return MR_ERR_ARG;
    }
    MR_CUDA(fwd_enqueue_rest(P, B, list, total, empty, false, 0.f, p2f, zbuf, bary, dists, nullptr, s));
    if (herr != 0) {
        set_error("a face references a vertex id outside [0, V=%lld); it was ignored", (long long)V);
        return MR_ERR_DEVICE;
    }
    return MR_OK;
}

}  // namespace
}  // namespace mr

extern "C" int mr_rasterize_fwd_noalloc(const float* verts, int64_t V, const int64_t* faces, int64_t F,
                                        const int64_t* mesh_to_face_first_idx, const int64_t* num_faces_per_mesh,
                                        int32_t N, int32_t H, int32_t W, float blur_radius, int32_t K,
                                        int32_t perspective_correct, int64_t* pix_to_face, float* zbuf, float* bary,
                                        float* dists, void* stream) {
    return mr::rasterize_noalloc(verts, V, faces, F, mesh_to_face_first_idx, num_faces_per_mesh, N, H, W,
                                 blur_radius, K, perspective_correct, pix_to_face, zbuf, bary, dists,
                                 static_cast<cudaStream_t>(stream));
}
