// Stage two of the PyTorch3D rasterizer as stand-alone kernels: the soft silhouette over
// the K faces kept per pixel and its gradient with respect to their distances.  One
// thread per pixel (grid-stride); the K slots of a pixel are contiguous.
#include <cmath>

#include "mr_common.cuh"
#include "mr_silhouette.cuh"

namespace mr {
namespace {

template <int KC>
__device__ __forceinline__ void load_slots(const int64_t* __restrict__ p2f, const float* __restrict__ dists,
                                           int64_t base, int K, float (&d)[KC], bool (&v)[KC]) {
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        if (k < K) {
            v[k] = __ldg(p2f + base + k) >= 0;
            d[k] = __ldg(dists + base + k);
        } else {
            v[k] = false;
            d[k] = 0.f;
        }
    }
}

template <int KC>
__global__ void k_silhouette_fwd(const int64_t* __restrict__ p2f, const float* __restrict__ dists, int64_t npix,
                                 int K, float sigma, float* __restrict__ alpha) {
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < npix; q += (int64_t)gridDim.x * blockDim.x) {
        float d[KC];
        bool v[KC];
        load_slots<KC>(p2f, dists, q * K, K, d, v);
        alpha[q] = silhouette_alpha<KC>(d, v, K, sigma);
    }
}

template <int KC>
__global__ void k_silhouette_bwd(const float* __restrict__ grad_alpha, const int64_t* __restrict__ p2f,
                                 const float* __restrict__ dists, int64_t npix, int K, float sigma,
                                 float* __restrict__ grad_dists) {
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < npix; q += (int64_t)gridDim.x * blockDim.x) {
        float d[KC], g[KC];
        bool v[KC];
        load_slots<KC>(p2f, dists, q * K, K, d, v);
        silhouette_grad<KC>(d, v, K, sigma, grad_alpha[q], g);
#pragma unroll
        for (int k = 0; k < KC; ++k)
            if (k < K) grad_dists[q * K + k] = g[k];
    }
}

int validate(int32_t N, int32_t H, int32_t W, int32_t K, float sigma, const void* a, const void* b, const void* c,
             const void* d) {
    if (N < 0 || H < 1 || W < 1 || K < 1 || K > MR_KMAX) {
        set_error("invalid shape N=%d H=%d W=%d K=%d", N, H, W, K);
        return MR_ERR_ARG;
    }
    if (!(sigma > 0.f) || !std::isfinite(sigma)) {
        set_error("sigma must be finite and > 0");
        return MR_ERR_ARG;
    }
    if (N > 0 && (!a || !b || !c || !d)) {
        set_error("null pointer");
        return MR_ERR_ARG;
    }
    return MR_OK;
}


}  // namespace
}  // namespace mr

extern "C" {

int mr_silhouette_blend_fwd(const int64_t* pix_to_face, const float* dists, int32_t N, int32_t H, int32_t W,
                            int32_t K, float sigma, float* alpha, void* stream) {
    int rc = mr::validate(N, H, W, K, sigma, pix_to_face, dists, alpha, alpha);
    if (rc != MR_OK || N == 0) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t npix = (int64_t)N * H * W;
    const int g = mr::grid_for(npix);
    mr::ProfScope ps(MR_STAGE_SILHOUETTE_FWD, s);
    if (K <= 1) mr::k_silhouette_fwd<1><<<g, 256, 0, s>>>(pix_to_face, dists, npix, K, sigma, alpha);
    else if (K <= 2) mr::k_silhouette_fwd<2><<<g, 256, 0, s>>>(pix_to_face, dists, npix, K, sigma, alpha);
    else if (K <= 4) mr::k_silhouette_fwd<4><<<g, 256, 0, s>>>(pix_to_face, dists, npix, K, sigma, alpha);
    else if (K <= 8) mr::k_silhouette_fwd<8><<<g, 256, 0, s>>>(pix_to_face, dists, npix, K, sigma, alpha);
    else if (K <= 16) mr::k_silhouette_fwd<16><<<g, 256, 0, s>>>(pix_to_face, dists, npix, K, sigma, alpha);
    else mr::k_silhouette_fwd<32><<<g, 256, 0, s>>>(pix_to_face, dists, npix, K, sigma, alpha);
    MR_CUDA(cudaGetLastError());
    return MR_OK;
}

int mr_silhouette_blend_bwd(const float* grad_alpha, const int64_t* pix_to_face, const float* dists, int32_t N,
                            int32_t H, int32_t W, int32_t K, float sigma, float* grad_dists, void* stream) {
    int rc = mr::validate(N, H, W, K, sigma, grad_alpha, pix_to_face, dists, grad_dists);
    if (rc != MR_OK || N == 0) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t npix = (int64_t)N * H * W;
    const int g = mr::grid_for(npix);
    mr::ProfScope ps(MR_STAGE_SILHOUETTE_BWD, s);
#define MR_SB(KC) mr::k_silhouette_bwd<KC><<<g, 256, 0, s>>>(grad_alpha, pix_to_face, dists, npix, K, sigma, grad_dists)
    if (K <= 1) MR_SB(1);
    else if (K <= 2) MR_SB(2);
    else if (K <= 4) MR_SB(4);
    else if (K <= 8) MR_SB(8);
    else if (K <= 16) MR_SB(16);
    else MR_SB(32);
#undef MR_SB
    MR_CUDA(cudaGetLastError());
    return MR_OK;
}

}  // extern "C"
