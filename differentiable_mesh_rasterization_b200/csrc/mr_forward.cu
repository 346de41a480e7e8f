// Stage one of the PyTorch3D two-stage mesh rasterizer ("Accelerating 3D Deep Learning
// with PyTorch3D", method: per-pixel K nearest faces) on sm_100a, plus the fused
// stage-two silhouette.
//
// Pipeline (one CUDA stream):
//   face setup   one thread per face: gather the three vertices, float64 signed area
//                (degenerate test), pixel box grown by sqrt(blur_radius), and the face's
//                plane constants for the fine pass (float64, rounded once to float32).
//   bin count    one thread per (image, face) pair: count the 16x16 screen bins the box
//                touches (warp-aggregated atomics).
//   bin scan     exclusive scan of the per-bin counts -> list offsets and the total.
//   (host)       one stream synchronisation to size the face lists.
//   bin fill     second pass of the pair loop: scatter face ids into the bin lists.
//   fine         one CTA per bin, eight independent warps (8x4 pixel tiles): ballot-
//                compacted per-warp face lists staged in shared memory, a warp-wide
//                depth pre-test, the full candidacy test, and a register-resident
//                insertion-sorted top-K per pixel; writes the K winning face ids.
//   epilogue     one thread per pixel: barycentrics, z and signed squared distance of
//                the K winners recomputed in float64 from the original vertices, the
//                fused soft silhouette, 16-byte stores.
#include "mr_forward_kernels.cuh"

namespace mr {
namespace {

int rasterize_impl(const float* verts, int64_t V, const int64_t* faces, int64_t F, const int64_t* first,
                   const int64_t* num, int32_t N, int32_t H, int32_t W, float blur, int32_t K, int32_t persp,
                   float sigma, bool sil, int64_t* p2f, float* zbuf, float* bary, float* dists, float* alpha,
                   cudaStream_t s) {
    int rc = validate_fwd(verts, V, faces, F, first, num, N, H, W, blur, K, p2f, zbuf, bary, dists);
    if (rc != MR_OK) return rc;
    if (sil && (!(sigma > 0.f) || !std::isfinite(sigma) || (N > 0 && !alpha))) {
        set_error("silhouette needs a finite sigma > 0 and an alpha buffer");
        return MR_ERR_ARG;
    }
    if (N == 0) return MR_OK;
    const int nbx = ceil_div(W, kBin), nby = ceil_div(H, kBin);
    const long long nbins_ll = (long long)N * nbx * nby;
    if (nbins_ll >= INT32_MAX / 2) {
        set_error("too many screen bins (%lld)", nbins_ll);
        return MR_ERR_ARG;
    }
    const int nbins = (int)nbins_ll;
    std::vector<int64_t> prefix(N + 1, 0);
    for (int n = 0; n < N; ++n) prefix[n + 1] = prefix[n] + num[n];
    const int64_t pairs = prefix[N];

    const int KC = K <= 1 ? 1 : K <= 2 ? 2 : K <= 4 ? 4 : K <= 8 ? 8 : K <= 16 ? 16 : 32;
    const int64_t npix = (int64_t)N * H * W;
    // one scratch block: geometry | boxes | constants | top-K ids | counts | offsets |
    // prefix | first | total | error
    auto up = [](size_t b) { return (b + 255) & ~size_t(255); };
    const size_t o_geom = 0;
    const size_t o_box = o_geom + up(sizeof(FaceGeom) * (size_t)F);
    const size_t o_con = o_box + up(sizeof(FaceBox) * (size_t)F);
    const size_t o_top = o_con + up(sizeof(float4) * kConstF4 * (size_t)F);
    const size_t o_cnt = o_top + up(sizeof(int) * (size_t)npix * (size_t)K);
    const size_t o_off = o_cnt + up(sizeof(int) * (size_t)nbins);
    const size_t o_pre = o_off + up(sizeof(int) * (size_t)(nbins + 1));
    const size_t o_fst = o_pre + up(sizeof(int64_t) * (size_t)(N + 1));
    const size_t o_tot = o_fst + up(sizeof(int64_t) * (size_t)N);
    const size_t o_err = o_tot + 256;
    const size_t bytes = o_err + 256;
    char* ws = nullptr;
    rc = scratch_alloc(reinterpret_cast<void**>(&ws), bytes, s);
    if (rc != MR_OK) return rc;
    FaceGeom* geom = reinterpret_cast<FaceGeom*>(ws + o_geom);
    FaceBox* box = reinterpret_cast<FaceBox*>(ws + o_box);
    float4* fconst = reinterpret_cast<float4*>(ws + o_con);
    int* topk = reinterpret_cast<int*>(ws + o_top);
    int* counts = reinterpret_cast<int*>(ws + o_cnt);
    int* offsets = reinterpret_cast<int*>(ws + o_off);
    int64_t* d_prefix = reinterpret_cast<int64_t*>(ws + o_pre);
    int64_t* d_first = reinterpret_cast<int64_t*>(ws + o_fst);
    long long* d_total = reinterpret_cast<long long*>(ws + o_tot);
    int* d_err = reinterpret_cast<int*>(ws + o_err);
    int* list = nullptr;

    auto fail = [&](int code) {
        scratch_free(list, s);
        scratch_free(ws, s);
        return code;
    };
#define MR_TRY(call)                                    \
    do {                                                \
        cudaError_t e_ = (call);                        \
        if (e_ != cudaSuccess) return fail(cuda_fail(e_, #call)); \
    } while (0)

    MR_TRY(cudaMemcpyAsync(d_prefix, prefix.data(), sizeof(int64_t) * (N + 1), cudaMemcpyHostToDevice, s));
    MR_TRY(cudaMemcpyAsync(d_first, first, sizeof(int64_t) * N, cudaMemcpyHostToDevice, s));
    MR_TRY(cudaMemsetAsync(counts, 0, sizeof(int) * (size_t)nbins, s));
    MR_TRY(cudaMemsetAsync(d_err, 0, sizeof(int), s));
    const double reach = std::sqrt((double)blur) * (1.0 + 1e-6) + 1e-7;
    if (F > 0) {
        ProfScope ps(MR_STAGE_FACE_SETUP, s);
        k_face_setup<<<(unsigned)((F + 255) / 256), 256, 0, s>>>(verts, V, faces, F, H, W, reach, persp, geom, box,
                                                                  fconst, d_err);
        MR_TRY(cudaGetLastError());
    }
    const int pair_blocks = (int)std::min<int64_t>((pairs + 255) / 256, 148 * 16);
    if (pairs > 0) {
        ProfScope ps(MR_STAGE_BIN_COUNT, s);
        k_bin_pairs<false><<<pair_blocks, 256, 0, s>>>(box, d_prefix, d_first, N, pairs, nbx, nby, counts,
                                                       nullptr, nullptr);
        MR_TRY(cudaGetLastError());
    }
    {
        ProfScope ps(MR_STAGE_BIN_SCAN, s);
        k_scan<<<1, 1024, 0, s>>>(counts, nbins, offsets, d_total);
    }
    MR_TRY(cudaGetLastError());
    long long host[2] = {0, 0};
    MR_TRY(cudaMemcpyAsync(&host[0], d_total, sizeof(long long), cudaMemcpyDeviceToHost, s));
    int herr = 0;
    MR_TRY(cudaMemcpyAsync(&herr, d_err, sizeof(int), cudaMemcpyDeviceToHost, s));
    MR_TRY(cudaStreamSynchronize(s));
    const long long total = host[0];
    if (total >= INT32_MAX) {
        set_error("bin lists too long (%lld entries)", total);
        return fail(MR_ERR_ARG);
    }
    if (total > 0) {
        rc = scratch_alloc(reinterpret_cast<void**>(&list), sizeof(int) * (size_t)total, s);
        if (rc != MR_OK) return fail(rc);
        MR_TRY(cudaMemsetAsync(counts, 0, sizeof(int) * (size_t)nbins, s));
        ProfScope ps(MR_STAGE_BIN_FILL, s);
        k_bin_pairs<true><<<pair_blocks, 256, 0, s>>>(box, d_prefix, d_first, N, pairs, nbx, nby, counts, offsets,
                                                      list);
        MR_TRY(cudaGetLastError());
    }
    const bool vec_ok = aligned16(p2f) && aligned16(zbuf) && aligned16(bary) && aligned16(dists);
    const bool exact = (H & (H - 1)) == 0 && (W & (W - 1)) == 0;
    {
        ProfScope ps(MR_STAGE_FINE, s);
        dispatch_fine(KC, persp != 0, exact, nbins, s, fconst, box, offsets, list, nbx, nby, H, W, K, blur, topk);
    }
    MR_TRY(cudaGetLastError());
    {
        ProfScope ps(MR_STAGE_EPILOGUE, s);
        dispatch_epilogue(KC, persp != 0, sil, npix, s, geom, topk, H, W, K, sigma, vec_ok, p2f, zbuf, bary, dists,
                          alpha);
    }
    MR_TRY(cudaGetLastError());
#undef MR_TRY
    scratch_free(list, s);
    scratch_free(ws, s);
    if (herr != 0) {
        set_error("a face references a vertex id outside [0, V=%lld); it was ignored", (long long)V);
        return MR_ERR_DEVICE;
    }
    return MR_OK;
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
