// Stage one of the PyTorch3D two-stage mesh rasterizer ("Accelerating 3D Deep Learning
// with PyTorch3D", method: per-pixel K nearest faces) on sm_100a, plus the fused
// stage-two silhouette.
//
// Pipeline (one CUDA stream):
//   face setup   one thread per (image, face) pair: gather the three vertices, float64
//                signed area (degenerate test), pixel box grown by sqrt(blur_radius), a
//                lower bound of the depth key over the box, the face's plane constants
//                for the fine pass (float64, rounded once), and the image's key range.
//   bin count    one thread per pair: count the 16x16 screen bins the box touches, per
//                depth bucket of the face within its image (one atomic per run of equal
//                slots in neighbouring lanes).
//   bin scan     exclusive scan of the per-(bin, bucket) counts -> list offsets, total;
//                the bins' longest-first order and the number of empty bins.
//   (host)       one stream synchronisation to size the face lists (the total, the error
//                word and the empty-bin count come back through mapped host memory).
//   bin fill     second pass of the pair loop: scatter face ids into the bin lists, so
//                each bin's list runs from its nearest depth bucket to its farthest.
//   fine         two CTAs of four warps per non-empty bin, eight independent warps in all
//                (8x4 pixel tiles): ballot-compacted per-warp face lists staged in shared
//                memory, a warp-wide depth pre-test, the full candidacy test, and a
//                register-resident sorted top-K per pixel; writes the K winning face ids
//                straight into pix_to_face.
//   epilogue     one thread per pixel: barycentrics, z and signed squared distance of
//                the K winners recomputed in float64 from the original vertices, the
//                fused soft silhouette, 16-byte stores; the pixels of empty bins get their
//                padding (pix_to_face included) without reads.
#include "mr_forward_kernels.cuh"

namespace mr {
namespace {

int rasterize_impl(const float* verts, int64_t V, const int64_t* faces, int64_t F, const int64_t* first,
                   const int64_t* num, int32_t N, int32_t H, int32_t W, float blur, int32_t K, int32_t persp,
                   float sigma, bool sil, int64_t* p2f, float* zbuf, float* bary, float* dists, float* alpha,
                   cudaStream_t s) {
    std::vector<int64_t> staged;
    if (N > 0) {
        int rs = host_indices(s, N, staged, {&first, &num});
        if (rs != MR_OK) return rs;
    }
    int rc = validate_fwd(verts, V, faces, F, first, num, N, H, W, blur, K, p2f, zbuf, bary, dists);
    if (rc != MR_OK) return rc;
    if (sil && (!(sigma > 0.f) || !std::isfinite(sigma) || (N > 0 && !alpha))) {
        set_error("silhouette needs a finite sigma > 0 and an alpha buffer");
        return MR_ERR_ARG;
    }
    if (N == 0) return MR_OK;
    FwdPlan P;
    rc = fwd_plan(V, F, num, N, H, W, blur, K, persp, P);
    if (rc != MR_OK) return rc;
    std::vector<int64_t> prefix(N + 1, 0);
    for (int n = 0; n < N; ++n) prefix[n + 1] = prefix[n] + num[n];

    char* ws = nullptr;
    int* list = nullptr;
    rc = scratch_alloc(reinterpret_cast<void**>(&ws), P.bytes, s);
    if (rc != MR_OK) return rc;
    const FwdBufs B = fwd_bufs(ws, P);
    auto finish = [&](int code) {
        scratch_free(list, s);
        scratch_free(ws, s);
        return code;
    };
    long long total = 0;
    int herr = 0, empty = 0;
    const Mailbox mb = host_mailbox();
    int64_t* staging = static_cast<int64_t*>(host_staging(sizeof(int64_t) * (2 * (size_t)N + 1)));
    cudaError_t e = fwd_enqueue_count(P, B, verts, faces, prefix.data(), first, s, &total, &herr, &empty, mb.dev,
                                      staging);
    if (e != cudaSuccess) return finish(cuda_fail(e, "forward: face setup and binning"));
    if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return finish(cuda_fail(e, "cudaStreamSynchronize"));
    if (mb.dev) {
        total = mb.host[0];
        herr = (int)mb.host[1];
        empty = (int)mb.host[2];
    }
    if (total >= INT32_MAX) {
        set_error("bin lists too long (%lld entries)", total);
        return finish(MR_ERR_ARG);
    }
    if (total > 0) {
        rc = scratch_alloc(reinterpret_cast<void**>(&list), sizeof(int) * (size_t)total, s);
        if (rc != MR_OK) return finish(rc);
    }
    e = fwd_enqueue_rest(P, B, list, total, empty, sil, sigma, p2f, zbuf, bary, dists, alpha, s);
    if (e != cudaSuccess) return finish(cuda_fail(e, "forward: fine pass"));
    if (herr != 0) {
        set_error("a face references a vertex id outside [0, V=%lld); it was ignored", (long long)V);
        return finish(MR_ERR_DEVICE);
    }
    return finish(MR_OK);
}

}  // namespace
}  // namespace mr

extern "C" {

int mr_rasterize_fwd(const float* verts, int64_t V, const int64_t* faces, int64_t F,
                     const int64_t* mesh_to_face_first_idx, const int64_t* num_faces_per_mesh, int32_t N,
                     int32_t H, int32_t W, float blur_radius, int32_t K, int32_t perspective_correct,
                     int64_t* pix_to_face, float* zbuf, float* bary, float* dists, void* stream) {
    return mr::rasterize_impl(verts, V, faces, F, mesh_to_face_first_idx, num_faces_per_mesh, N, H, W, blur_radius,
                              K, perspective_correct, 0.f, false, pix_to_face, zbuf, bary, dists, nullptr,
                              static_cast<cudaStream_t>(stream));
}

int mr_rasterize_silhouette_fwd(const float* verts, int64_t V, const int64_t* faces, int64_t F,
                                const int64_t* mesh_to_face_first_idx, const int64_t* num_faces_per_mesh,
                                int32_t N, int32_t H, int32_t W, float blur_radius, int32_t K,
                                int32_t perspective_correct, float sigma, int64_t* pix_to_face, float* zbuf,
                                float* bary, float* dists, float* alpha, void* stream) {
    return mr::rasterize_impl(verts, V, faces, F, mesh_to_face_first_idx, num_faces_per_mesh, N, H, W, blur_radius,
                              K, perspective_correct, sigma, true, pix_to_face, zbuf, bary, dists, alpha,
                              static_cast<cudaStream_t>(stream));
}

}  // extern "C"
