// Soft-silhouette arithmetic shared by the fused forward epilogue, the stand-alone
// silhouette kernels and the fused backward (internal header).
//
// PyTorch3D paper, method: the second stage fuses the influence of the K faces kept per
// pixel.  Per valid slot p_k = 1 / (1 + exp(d_k / sigma)); alpha = 1 - prod_k (1 - p_k).
#pragma once

#include <cuda_runtime.h>

namespace mr {

// alpha = 1 - prod_k (1 - p_k) = 1 - 1 / P with P = prod_k (1 + e_k), e_k = exp(-d_k / sigma),
// because 1 - p_k = 1 / (1 + e_k).  P - 1 is carried as its own running value,
// (P - 1)' = (P - 1) + e + (P - 1) e, so alpha = (P - 1) / P keeps full relative accuracy
// for alpha near 0 (far blur ring), and one exponential per slot is the only
// transcendental.  The exponent is capped at 2^115 and P - 1 at 1e30 (alpha is then 1 in
// float32 either way), so an interior slot (e huge) next to a far one (e = 0) cannot form
// inf * 0.
template <int KC>
__device__ __forceinline__ float silhouette_alpha(const float (&d)[KC], const bool (&valid)[KC], int K,
                                                  float sigma) {
    const float c = 1.4426950408889634f / sigma;   // log2(e) / sigma: e_k = 2^(-d_k c)
    float pm1 = 0.f;
#pragma unroll
    for (int k = 0; k < KC; ++k)
        if (k < K && valid[k]) {
            const float e = exp2f(fminf(-d[k] * c, 115.f));
            pm1 = fminf(fmaf(pm1, e, pm1 + e), 1e30f);
        }
    const float r = 1.f / (1.f + pm1);
    return pm1 <= 1.f ? pm1 * r : 1.f - r;
}

// dL/dd_k = -dL/dalpha * prod_{j != k} (1 - p_j) * p_k (1 - p_k) / sigma; 0 for empty slots.
// The product over j != k is formed directly (no division by 1 - p_k).
template <int KC>
__device__ __forceinline__ void silhouette_grad(const float (&d)[KC], const bool (&valid)[KC], int K, float sigma,
                                                float grad_alpha, float (&g)[KC]) {
    float q[KC], p[KC];
    const float inv_sigma = 1.f / sigma;
    const float c = 1.4426950408889634f * inv_sigma;   // log2(e) / sigma
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        // one exponential per slot: with e = exp(-|x|) and r = 1 / (1 + e) the two
        // sigmoids are r and e * r, assigned by the sign of x (no overflow either way);
        // 1 + e lies in (1, 2], where the fast reciprocal is good to about an ulp
        const float e = exp2f(-fabsf(d[k]) * c);
        const float r = __fdividef(1.f, 1.f + e);
        q[k] = d[k] >= 0.f ? r : e * r;    // 1 - p_k
        p[k] = d[k] >= 0.f ? e * r : r;
    }
    const float ga = -grad_alpha * inv_sigma;
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        float others = 1.f;
#pragma unroll
        for (int j = 0; j < KC; ++j)
            if (j != k && j < K && valid[j]) others *= q[j];
        g[k] = (k < K && valid[k]) ? ga * others * p[k] * q[k] : 0.f;
    }
}

}  // namespace mr
