// Batched K nearest neighbours over heterogeneous clouds ("Accelerating 3D Deep Learning
// with PyTorch3D": a custom KNN kernel for batches of point clouds of different sizes).
//
// For query i of cloud n of the first set, the squared Euclidean distance to every point j
// of cloud n of the second set; the K smallest, ordered by (distance, j).
//
// Exact search, tiled: a CTA owns 256 queries of one cloud (one per thread, the query in
// registers) and streams the reference cloud through shared memory in chunks of 1024
// points, with the bounding box of every group of 32 references; a warp skips a group
// whose box lies beyond the K-th distance of all its 32 queries (exact: the box bounds
// every distance in it), otherwise each thread tests the 32 references, four distances at
// a time, against its current K-th distance and keeps its K best in registers.  The
// distance is formed from coordinate differences (not |q|^2 + |r|^2 - 2 q.r, which cancels
// for near neighbours).  Tiles are issued largest reference cloud first.
#include <algorithm>
#include <cfloat>
#include <climits>
#include <cmath>
#include <utility>
#include <vector>

#include "mr_common.cuh"

namespace mr {
namespace {

constexpr int kKnnQueries = 256;     // queries per CTA
constexpr int kKnnChunk = 1024;      // reference points per shared-memory chunk

struct KnnTile {
    int64_t q0, qn;      // queries [q0, q0 + qn)
    int64_t r0, rn;      // references [r0, r0 + rn)
};

template <int KC>
__device__ __forceinline__ void insert_nn(float (&kd)[KC], int (&ki)[KC], float d, int id) {
#pragma unroll
    for (int k = KC - 1; k > 0; --k) {
        const bool shift = d < kd[k - 1] || (d == kd[k - 1] && id < ki[k - 1]);
        const bool here = !shift && (d < kd[k] || (d == kd[k] && id < ki[k]));
        if (shift) {
            kd[k] = kd[k - 1];
            ki[k] = ki[k - 1];
        } else if (here) {
            kd[k] = d;
            ki[k] = id;
        }
    }
    if (d < kd[0] || (d == kd[0] && id < ki[0])) {
        kd[0] = d;
        ki[0] = id;
    }
}

template <int KC, int D>
__global__ void __launch_bounds__(kKnnQueries) k_knn(const float* __restrict__ p1, const float* __restrict__ p2,
                                                     const KnnTile* __restrict__ tiles, int K,
                                                     int64_t* __restrict__ idx, float* __restrict__ dists) {
    constexpr int kGroups = kKnnChunk / 32;
    __shared__ float4 sr[kKnnChunk];
    __shared__ float4 blo[kGroups], bhi[kGroups];     // box of each group of 32 references
    const KnnTile T = tiles[blockIdx.x];
    const int lane = threadIdx.x & 31;
    const int64_t qi = T.q0 + threadIdx.x;
    const bool live = threadIdx.x < T.qn;
    float q[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < D; ++e) q[e] = live ? p1[qi * D + e] : 0.f;
    float kd[KC];
    int ki[KC];
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        kd[k] = FLT_MAX;
        ki[k] = INT_MAX;
    }
    for (int64_t c0 = 0; c0 < T.rn; c0 += kKnnChunk) {
        __syncthreads();
        const int cnt = (int)min((int64_t)kKnnChunk, T.rn - c0);
        // each warp loads groups of 32 references and their bounding box
        for (int t = threadIdx.x; t < kKnnChunk; t += kKnnQueries) {
            const bool in = t < cnt;
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            if (in) {
                const int64_t r = T.r0 + c0 + t;
#pragma unroll
                for (int e = 0; e < D; ++e) v[e] = p2[r * D + e];
            }
            sr[t] = make_float4(v[0], v[1], v[2], v[3]);
            float lo[4], hi[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                lo[e] = in ? v[e] : FLT_MAX;
                hi[e] = in ? v[e] : -FLT_MAX;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int e = 0; e < D; ++e) {
                    lo[e] = fminf(lo[e], __shfl_xor_sync(0xffffffffu, lo[e], o));
                    hi[e] = fmaxf(hi[e], __shfl_xor_sync(0xffffffffu, hi[e], o));
                }
            if (lane == 0) {
                blo[t >> 5] = make_float4(lo[0], lo[1], lo[2], lo[3]);
                bhi[t >> 5] = make_float4(hi[0], hi[1], hi[2], hi[3]);
            }
        }
        __syncthreads();
        const int id0 = (int)(T.r0 + c0);
        const int ngroups = (cnt + 31) >> 5;
        for (int gi = 0; gi < ngroups; ++gi) {
            // skip the group when its box is farther than this lane's K-th distance, for
            // every lane of the warp (the bound is shrunk by 2^-20 against rounding)
            const float4 lo4 = blo[gi], hi4 = bhi[gi];
            const float lo[4] = {lo4.x, lo4.y, lo4.z, lo4.w}, hi[4] = {hi4.x, hi4.y, hi4.z, hi4.w};
            float lb = 0.f;
#pragma unroll
            for (int e = 0; e < D; ++e) {
                const float gap = fmaxf(fmaxf(lo[e] - q[e], q[e] - hi[e]), 0.f);
                lb = fmaf(gap, gap, lb);
            }
            const bool far = !live || lb * (1.f - 0x1p-20f) > kd[KC - 1];
            if (__all_sync(0xffffffffu, far)) continue;
            const int t0 = gi * 32, t1 = min(t0 + 32, cnt);
            for (int t = t0; t < t1; t += 4) {
                float d4[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 r = sr[min(t + u, kKnnChunk - 1)];
                    const float rv[4] = {r.x, r.y, r.z, r.w};
                    float d = 0.f;
#pragma unroll
                    for (int e = 0; e < D; ++e) {
                        const float w = q[e] - rv[e];
                        d = fmaf(w, w, d);
                    }
                    d4[u] = t + u < t1 ? d : FLT_MAX;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)   // ids ascend: a tie keeps the earlier id
                    if (d4[u] < kd[KC - 1]) insert_nn<KC>(kd, ki, d4[u], id0 + t + u);
            }
        }
    }
    if (!live) return;
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        if (k >= K) break;
        const bool ok = ki[k] != INT_MAX;
        idx[qi * K + k] = ok ? ki[k] : -1;
        dists[qi * K + k] = ok ? kd[k] : -1.f;
    }
}

__global__ void k_fill_rows(int64_t* __restrict__ idx, float* __restrict__ dists, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        idx[i] = -1;
        dists[i] = -1.f;
    }
}

// Backward: thread per query; its own gradient is summed in registers, the references'
// go out as one float4 atomic per (query, neighbour) into a padded accumulator.
template <int D>
__global__ void k_knn_bwd(const float* __restrict__ p1, int64_t P1, const float* __restrict__ p2, int64_t P2, int K,
                          const int64_t* __restrict__ idx, const float* __restrict__ g, float* __restrict__ g1,
                          float4* __restrict__ acc, int* __restrict__ err) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < P1; i += (int64_t)gridDim.x * blockDim.x) {
        float q[D], gq[D];
#pragma unroll
        for (int e = 0; e < D; ++e) {
            q[e] = p1[i * D + e];
            gq[e] = 0.f;
        }
        for (int k = 0; k < K; ++k) {
            const int64_t j = idx[i * K + k];
            if (j == -1) continue;
            if (j < -1 || j >= P2) {
                atomicOr(err, kErrSlotIndex);
                continue;
            }
            const float gk = 2.f * g[i * K + k];
            float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int e = 0; e < D; ++e) {
                const float t = gk * (q[e] - p2[j * D + e]);
                gq[e] += t;
                c[e] = -t;
            }
            atomicAdd(acc + j, make_float4(c[0], c[1], c[2], c[3]));
        }
#pragma unroll
        for (int e = 0; e < D; ++e) g1[i * D + e] = gq[e];
    }
}

template <int D>
__global__ void k_acc_to_d(const float4* __restrict__ acc, int64_t P, float* __restrict__ out) {
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < P; p += (int64_t)gridDim.x * blockDim.x) {
        const float4 a = acc[p];
        const float v[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int e = 0; e < D; ++e) out[p * D + e] = v[e];
    }
}

template <int D>
cudaError_t launch_knn(int K, int ntiles, const float* p1, const float* p2, const KnnTile* tiles, int64_t* idx,
                       float* dists, cudaStream_t s) {
#define MR_KNN(KC) k_knn<KC, D><<<ntiles, kKnnQueries, 0, s>>>(p1, p2, tiles, K, idx, dists)
    if (K <= 1) MR_KNN(1);
    else if (K <= 2) MR_KNN(2);
    else if (K <= 4) MR_KNN(4);
    else if (K <= 8) MR_KNN(8);
    else if (K <= 16) MR_KNN(16);
    else MR_KNN(32);
#undef MR_KNN
    return cudaGetLastError();
}

int check_sets(const int64_t* first, const int64_t* num, int N, int64_t P, const char* what) {
    for (int n = 0; n < N; ++n)
        if (first[n] < 0 || num[n] < 0 || first[n] + num[n] > P) {
            set_error("%s: cloud %d range [%lld, %lld) outside [0, %lld)", what, n, (long long)first[n],
                      (long long)(first[n] + num[n]), (long long)P);
            return MR_ERR_ARG;
        }
    return MR_OK;
}

}  // namespace
}  // namespace mr

extern "C" {

int mr_knn_fwd(const float* p1, int64_t P1, const int64_t* first1, const int64_t* num1, const float* p2, int64_t P2,
               const int64_t* first2, const int64_t* num2, int32_t N, int32_t D, int32_t K, int64_t* idx,
               float* dists, void* stream) {
    using namespace mr;
    if (N < 0 || D < 1 || D > MR_KNN_DMAX || K < 1 || K > MR_KMAX || P1 < 0 || P2 < 0 || P2 > INT32_MAX) {
        set_error("invalid arguments N=%d D=%d K=%d P1=%lld P2=%lld", N, D, K, (long long)P1, (long long)P2);
        return MR_ERR_ARG;
    }
    if (P1 == 0) return MR_OK;
    if (!p1 || !idx || !dists || (N > 0 && (!first1 || !num1 || !first2 || !num2)) || (P2 > 0 && !p2)) {
        set_error("null pointer");
        return MR_ERR_ARG;
    }
    int rc = check_sets(first1, num1, N, P1, "mr_knn_fwd queries");
    if (rc == MR_OK) rc = check_sets(first2, num2, N, P2, "mr_knn_fwd references");
    if (rc != MR_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // query clouds must be disjoint; rows outside every cloud are filled with -1
    std::vector<std::pair<int64_t, int64_t>> ranges;
    std::vector<KnnTile> tiles;
    for (int n = 0; n < N; ++n) {
        if (num1[n] > 0) ranges.push_back({first1[n], num1[n]});
        for (int64_t q = first1[n]; q < first1[n] + num1[n]; q += kKnnQueries)
            tiles.push_back({q, std::min<int64_t>(kKnnQueries, first1[n] + num1[n] - q), first2[n], num2[n]});
    }
    std::sort(ranges.begin(), ranges.end());
    int64_t covered = 0, end = 0;
    for (const auto& r : ranges) {
        if (r.first < end) {
            set_error("mr_knn_fwd: query clouds overlap at point %lld", (long long)r.first);
            return MR_ERR_ARG;
        }
        end = r.first + r.second;
        covered += r.second;
    }
    if (covered < P1) {
        k_fill_rows<<<grid_for(P1 * K), 256, 0, s>>>(idx, dists, P1 * K);
        MR_CUDA(cudaGetLastError());
    }
    if (tiles.empty()) return MR_OK;
    std::stable_sort(tiles.begin(), tiles.end(), [](const KnnTile& a, const KnnTile& b) { return a.rn > b.rn; });
    KnnTile* dt = nullptr;
    rc = scratch_alloc(reinterpret_cast<void**>(&dt), sizeof(KnnTile) * tiles.size(), s);
    if (rc != MR_OK) return rc;
    cudaError_t e = cudaMemcpyAsync(dt, tiles.data(), sizeof(KnnTile) * tiles.size(), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) {
        ProfScope ps(MR_STAGE_KNN, s);
        const int nt = (int)tiles.size();
        switch (D) {
            case 1: e = launch_knn<1>(K, nt, p1, p2, dt, idx, dists, s); break;
            case 2: e = launch_knn<2>(K, nt, p1, p2, dt, idx, dists, s); break;
            case 3: e = launch_knn<3>(K, nt, p1, p2, dt, idx, dists, s); break;
            default: e = launch_knn<4>(K, nt, p1, p2, dt, idx, dists, s); break;
        }
    }
    // (a copy from pageable host memory returns once the data is staged: the vector may go)
    scratch_free(dt, s);
    if (e != cudaSuccess) return cuda_fail(e, "knn");
    return MR_OK;
}

int mr_knn_bwd(const float* p1, int64_t P1, const float* p2, int64_t P2, int32_t D, int32_t K, const int64_t* idx,
               const float* grad_dists, float* grad_p1, float* grad_p2, void* stream) {
    using namespace mr;
    if (D < 1 || D > MR_KNN_DMAX || K < 1 || K > MR_KMAX || P1 < 0 || P2 < 0) {
        set_error("invalid arguments");
        return MR_ERR_ARG;
    }
    if ((P1 > 0 && (!p1 || !grad_p1 || !idx || !grad_dists)) || (P2 > 0 && (!p2 || !grad_p2))) {
        set_error("null pointer");
        return MR_ERR_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (P2 == 0) {
        if (P1 > 0) MR_CUDA(cudaMemsetAsync(grad_p1, 0, sizeof(float) * (size_t)(P1 * D), s));
        return MR_OK;
    }
    int* err = device_error_word();
    if (!err) {
        set_error("cannot locate the device error word");
        return MR_ERR_CUDA;
    }
    float4* acc = nullptr;
    int rc = scratch_alloc(reinterpret_cast<void**>(&acc), sizeof(float4) * (size_t)P2, s);
    if (rc != MR_OK) return rc;
    cudaError_t e = cudaMemsetAsync(acc, 0, sizeof(float4) * (size_t)P2, s);
    if (e == cudaSuccess) {
        ProfScope ps(MR_STAGE_KNN_BWD, s);
        const int g1 = grid_for(std::max<int64_t>(P1, 1)), g2 = grid_for(P2);
#define MR_KB(DD)                                                                                            \
    do {                                                                                                     \
        if (P1 > 0) k_knn_bwd<DD><<<g1, 256, 0, s>>>(p1, P1, p2, P2, K, idx, grad_dists, grad_p1, acc, err); \
        k_acc_to_d<DD><<<g2, 256, 0, s>>>(acc, P2, grad_p2);                                                 \
    } while (0)
        switch (D) {
            case 1: MR_KB(1); break;
            case 2: MR_KB(2); break;
            case 3: MR_KB(3); break;
            default: MR_KB(4); break;
        }
#undef MR_KB
        e = cudaGetLastError();
    }
    scratch_free(acc, s);
    if (e != cudaSuccess) return cuda_fail(e, "knn backward");
    return MR_OK;
}

}  // extern "C"
