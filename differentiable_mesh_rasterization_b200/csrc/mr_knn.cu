// Batched K nearest neighbours over heterogeneous clouds ("Accelerating 3D Deep Learning
// with PyTorch3D": a custom KNN kernel for batches of point clouds of different sizes).
//
// For query i of cloud n of the first set, the squared Euclidean distance to every point j
// of cloud n of the second set; the K smallest, ordered by (distance, j).
//
// Exact search over spatially ordered tiles.  Both sets are first ordered, cloud by cloud,
// by a 16^3 grid over the reference cloud's bounding box, cells in Morton order (count ->
// exclusive scan -> fill, like the rasterizer's binning; order inside a cell is free).
// The bounding boxes of every group of 32 consecutive ordered references and of every 32
// groups are then built once.  Each warp owns 32 consecutive ordered queries of one cloud
// (one per lane, in registers) and walks the cloud's super-boxes outward from the one
// holding its first query's cell, so the K-th distances shrink early; a super-box or a
// group box beyond the K-th distance of all 32 lanes is skipped (exact: a box bounds every
// distance in it), a surviving group is staged in the warp's shared memory and each lane
// tests it four distances at a time, keeping its K best as 64-bit keys (distance bits
// above the original id) in registers.  Warps never wait for one another.  The distance is
// formed from coordinate differences (not |q|^2 + |r|^2 - 2 q.r, which cancels for near
// neighbours).  Tiles go out largest reference cloud first.
#include <algorithm>
#include <cfloat>
#include <climits>
#include <cmath>
#include <utility>
#include <vector>

#include "mr_common.cuh"
#include "mr_scan.cuh"

namespace mr {
namespace {

constexpr int kKnnQueries = 256;     // queries per CTA

constexpr int kGrid = 16;            // cells per axis of a cloud's grid
constexpr int kCells = kGrid * kGrid * kGrid;

struct KnnTile {
    int64_t s0;          // first ordered query
    int qn;              // queries in the tile
    int n;               // cloud
};

struct CloudBox {
    float lo[3], hi[3];
};

// Morton code of a point's cell in its cloud's grid (the first three coordinates).
template <int D>
__device__ __forceinline__ int cell_code(const float* __restrict__ x, const CloudBox& B) {
    int c[3] = {0, 0, 0};
#pragma unroll
    for (int e = 0; e < (D < 3 ? D : 3); ++e) {
        const float ext = B.hi[e] - B.lo[e];
        const float t = ext > 0.f ? (x[e] - B.lo[e]) / ext * (float)kGrid : 0.f;
        c[e] = (int)fminf(fmaxf(t, 0.f), (float)(kGrid - 1));   // clamped before the cast; NaN -> 0
    }
    int code = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b)
        code |= (((c[0] >> b) & 1) << (3 * b)) | (((c[1] >> b) & 1) << (3 * b + 1)) | (((c[2] >> b) & 1) << (3 * b + 2));
    return code;
}

// Cloud n of a set as a prefix-sum position: item t of the set's clouds is point
// first[n] + (t - pre[n]) with n the last cloud whose pre <= t.
__device__ __forceinline__ int cloud_at(int64_t t, const int64_t* __restrict__ pre, int N) {
    int lo = 0, hi = N - 1, n = 0;
    while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid] <= t) {
            n = mid;
            lo = mid + 1;
        } else {
            hi = mid - 1;
        }
    }
    return n;
}

// Bounding box of each reference cloud (one CTA per cloud).
template <int D>
__global__ void k_cloud_box(const float* __restrict__ p2, const int64_t* __restrict__ first2,
                            const int64_t* __restrict__ num2, CloudBox* __restrict__ box) {
    __shared__ float red[2][3][8];
    const int n = blockIdx.x;
    float lo[3] = {FLT_MAX, FLT_MAX, FLT_MAX}, hi[3] = {-FLT_MAX, -FLT_MAX, -FLT_MAX};
    for (int64_t j = first2[n] + threadIdx.x; j < first2[n] + num2[n]; j += blockDim.x)
#pragma unroll
        for (int e = 0; e < (D < 3 ? D : 3); ++e) {
            lo[e] = fminf(lo[e], p2[j * D + e]);
            hi[e] = fmaxf(hi[e], p2[j * D + e]);
        }
#pragma unroll
    for (int e = 0; e < 3; ++e)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lo[e] = fminf(lo[e], __shfl_xor_sync(0xffffffffu, lo[e], o));
            hi[e] = fmaxf(hi[e], __shfl_xor_sync(0xffffffffu, hi[e], o));
        }
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0)
#pragma unroll
        for (int e = 0; e < 3; ++e) {
            red[0][e][w] = lo[e];
            red[1][e][w] = hi[e];
        }
    __syncthreads();
    if (threadIdx.x == 0) {
        CloudBox B;
#pragma unroll
        for (int e = 0; e < 3; ++e) {
            B.lo[e] = red[0][e][0];
            B.hi[e] = red[1][e][0];
            for (int k = 1; k < (int)(blockDim.x >> 5); ++k) {
                B.lo[e] = fminf(B.lo[e], red[0][e][k]);
                B.hi[e] = fmaxf(B.hi[e], red[1][e][k]);
            }
        }
        box[n] = B;
    }
}

// Counting sort of a set's cloud points by (cloud, cell): FILL = false counts per bin,
// FILL = true writes the ordered coordinates (float4), original ids and cell codes.
template <int D, bool FILL>
__global__ void k_order_points(const float* __restrict__ p, const int64_t* __restrict__ first,
                               const int64_t* __restrict__ pre, int N, int64_t total,
                               const CloudBox* __restrict__ box, int* __restrict__ counts,
                               const int* __restrict__ offsets, float4* __restrict__ sp, int* __restrict__ sid,
                               short* __restrict__ scode) {
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
        const int n = cloud_at(t, pre, N);
        const int64_t j = first[n] + (t - pre[n]);
        float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < D; ++e) x[e] = p[j * D + e];
        const int code = cell_code<D>(x, box[n]);
        const int b = n * kCells + code;
        const int at = atomicAdd(counts + b, 1);
        if (FILL) {
            const int pos = offsets[b] + at;
            sp[pos] = make_float4(x[0], x[1], x[2], x[3]);
            sid[pos] = (int)j;
            scode[pos] = (short)code;
        }
    }
}

// A neighbour key: the squared distance's bits above the original reference id.  Distances
// are >= 0 and non-negative floats order like their bits, so one 64-bit compare orders
// (distance, id); kNone sorts after every reference and reads back as FLT_MAX.
constexpr unsigned long long kNone = (0x7F7FFFFFull << 32) | 0xFFFFFFFFull;

__device__ __forceinline__ unsigned long long nn_key(float d, int id) {
    return ((unsigned long long)__float_as_uint(d + 0.f) << 32) | (unsigned)id;
}
__device__ __forceinline__ float key_dist(unsigned long long k) { return __uint_as_float((unsigned)(k >> 32)); }

// Sorted insertion into a register list of KC keys (the caller has checked key < the last).
template <int KC>
__device__ __forceinline__ void insert_nn(unsigned long long (&kk)[KC], unsigned long long key) {
#pragma unroll
    for (int k = KC - 1; k > 0; --k) {
        const bool shift = key < kk[k - 1];
        kk[k] = shift ? kk[k - 1] : (key < kk[k] ? key : kk[k]);
    }
    kk[0] = key < kk[0] ? key : kk[0];
}

// Boxes of the ordered references: level 0 = groups of 32 consecutive points of one
// cloud, level 1 = 32 consecutive groups of one cloud.  One warp per box; item t of a
// level belongs to cloud cloud_at(t, pre_level) and starts at its cloud's first item.
__global__ void k_group_boxes(const float4* __restrict__ sr, const int64_t* __restrict__ pre2,
                              const int64_t* __restrict__ num2, const int64_t* __restrict__ gpre, int N,
                              int64_t ngroups, float4* __restrict__ glo, float4* __restrict__ ghi) {
    const int lane = threadIdx.x & 31;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t g = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; g < ngroups; g += nw) {
        const int n = cloud_at(g, gpre, N);
        const int64_t i = (g - gpre[n]) * 32 + lane;             // point within the cloud
        const bool in = i < num2[n];
        const float4 v = in ? sr[pre2[n] + i] : make_float4(0.f, 0.f, 0.f, 0.f);
        float lo[4] = {v.x, v.y, v.z, v.w}, hi[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (!in) {
                lo[e] = FLT_MAX;
                hi[e] = -FLT_MAX;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                lo[e] = fminf(lo[e], __shfl_xor_sync(0xffffffffu, lo[e], o));
                hi[e] = fmaxf(hi[e], __shfl_xor_sync(0xffffffffu, hi[e], o));
            }
        }
        if (lane == 0) {
            glo[g] = make_float4(lo[0], lo[1], lo[2], lo[3]);
            ghi[g] = make_float4(hi[0], hi[1], hi[2], hi[3]);
        }
    }
}

__global__ void k_super_boxes(const float4* __restrict__ glo, const float4* __restrict__ ghi,
                              const int64_t* __restrict__ gpre, const int64_t* __restrict__ spre, int N,
                              int64_t nsupers, int64_t ngroups_total, float4* __restrict__ slo,
                              float4* __restrict__ shi) {
    const int lane = threadIdx.x & 31;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t u = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; u < nsupers; u += nw) {
        const int n = cloud_at(u, spre, N);
        const int64_t gend = n + 1 < N ? gpre[n + 1] : ngroups_total;
        const int64_t g = gpre[n] + (u - spre[n]) * 32 + lane;
        const bool in = g < gend;
        const float4 a = in ? glo[g] : make_float4(FLT_MAX, FLT_MAX, FLT_MAX, FLT_MAX);
        const float4 b = in ? ghi[g] : make_float4(-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX);
        float lo[4] = {a.x, a.y, a.z, a.w}, hi[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                lo[e] = fminf(lo[e], __shfl_xor_sync(0xffffffffu, lo[e], o));
                hi[e] = fmaxf(hi[e], __shfl_xor_sync(0xffffffffu, hi[e], o));
            }
        if (lane == 0) {
            slo[u] = make_float4(lo[0], lo[1], lo[2], lo[3]);
            shi[u] = make_float4(hi[0], hi[1], hi[2], hi[3]);
        }
    }
}

// Lower bound of the squared distance from q to a box, shrunk by 2^-20 against rounding.
template <int D>
__device__ __forceinline__ float box_bound(const float (&q)[4], float4 lo4, float4 hi4) {
    const float lo[4] = {lo4.x, lo4.y, lo4.z, lo4.w}, hi[4] = {hi4.x, hi4.y, hi4.z, hi4.w};
    float lb = 0.f;
#pragma unroll
    for (int e = 0; e < D; ++e) {
        const float gap = fmaxf(fmaxf(lo[e] - q[e], q[e] - hi[e]), 0.f);
        lb = fmaf(gap, gap, lb);
    }
    return lb * (1.f - 0x1p-20f);
}

// The search: every warp owns 32 consecutive ordered queries of one cloud (one per lane)
// and walks the cloud's super-boxes outward from the one holding its first query's cell
// (home, home + 1, home - 1, ...).  A super-box or group box beyond every lane's K-th
// distance is skipped by the whole warp; a group that survives is staged in the warp's
// shared memory (32 points, one array per coordinate, and ids) and every lane tests it
// four distances at a time, two by two with packed two-lane float32 instructions (each
// lane rounds as the scalar instruction would, so the distances are the scalar ones).
// COUNT adds, per warp, the (live query, reference) pairs whose distance it evaluates to
// *work (one atomic per warp at the end): the search's real work, for measurement.
template <int KC, int D, bool COUNT>
__global__ void __launch_bounds__(kKnnQueries) k_knn(const float4* __restrict__ sq, const int* __restrict__ sqid,
                                                     const short* __restrict__ sqcode, const float4* __restrict__ sr,
                                                     const int* __restrict__ srid, const int* __restrict__ roff,
                                                     const int64_t* __restrict__ pre2, const int64_t* __restrict__ num2,
                                                     const int64_t* __restrict__ gpre, const int64_t* __restrict__ spre,
                                                     const float4* __restrict__ glo, const float4* __restrict__ ghi,
                                                     const float4* __restrict__ slo, const float4* __restrict__ shi,
                                                     const KnnTile* __restrict__ tiles, int K,
                                                     int64_t* __restrict__ idx, float* __restrict__ dists,
                                                     unsigned long long* __restrict__ work) {
    __shared__ __align__(16) float wc[kKnnQueries / 32][4][32];
    __shared__ __align__(16) int wid[kKnnQueries / 32][32];
    const KnnTile T = tiles[blockIdx.x];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp * 32 >= T.qn) return;                              // whole warp past the tile: no partner waits
    const bool live = threadIdx.x < T.qn;
    const int n = T.n;
    const int64_t r0 = pre2[n], rn = num2[n];
    float q[4] = {0.f, 0.f, 0.f, 0.f};
    int qid = -1;
    if (live) {
        const float4 v = sq[T.s0 + threadIdx.x];
        q[0] = v.x; q[1] = v.y; q[2] = v.z; q[3] = v.w;
        qid = sqid[T.s0 + threadIdx.x];
    }
    f32x2 qq[D];
#pragma unroll
    for (int e = 0; e < D; ++e) qq[e] = pack2(q[e], q[e]);
    unsigned long long kk[KC];
#pragma unroll
    for (int k = 0; k < KC; ++k) kk[k] = kNone;
    const int64_t g0 = gpre[n], s0 = spre[n];
    const int64_t ngr = (rn + 31) >> 5, nsup = (ngr + 31) >> 5;
    int64_t home = 0;
    if (rn > 0) {
        const int64_t h = (int64_t)roff[n * kCells + sqcode[T.s0 + warp * 32]] - r0;
        home = min(max(h, (int64_t)0), rn - 1) >> 10;           // super-box of the first query's cell
    }
    int64_t up = home + 1, down = home - 1, cur = home;
    unsigned long long evaluated = 0;
    const unsigned live_lanes = COUNT ? (unsigned)__popc(__ballot_sync(0xffffffffu, live)) : 0u;
    for (int64_t it = 0; it < nsup; ++it) {
        if (__all_sync(0xffffffffu, !live || box_bound<D>(q, slo[s0 + cur], shi[s0 + cur]) > key_dist(kk[KC - 1]))) {
            // skipped
        } else {
            const int64_t gb = cur * 32, ge = min(gb + 32, ngr);
            for (int64_t g = gb; g < ge; ++g) {
                if (__all_sync(0xffffffffu, !live || box_bound<D>(q, glo[g0 + g], ghi[g0 + g]) > key_dist(kk[KC - 1])))
                    continue;
                const int64_t pb = g * 32;
                const int cnt = (int)min((int64_t)32, rn - pb);
                if (COUNT) evaluated += (unsigned long long)cnt * live_lanes;
                __syncwarp();
                if (lane < cnt) {
                    const float4 r = sr[r0 + pb + lane];
                    const float rv[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
                    for (int e = 0; e < D; ++e) wc[warp][e][lane] = rv[e];
                    wid[warp][lane] = srid[r0 + pb + lane];
                }
                __syncwarp();
                // slots at or past cnt hold stale values; their distances are computed
                // (t < cnt <= 32 keeps every read inside the arrays) and never inserted
                for (int t = 0; t < cnt; t += 4) {
                    f32x2 dlo = 0, dhi = 0;
#pragma unroll
                    for (int e = 0; e < D; ++e) {
                        const ulonglong2 r = *reinterpret_cast<const ulonglong2*>(&wc[warp][e][t]);
                        const f32x2 wlo = sub2(qq[e], r.x), whi = sub2(qq[e], r.y);
                        dlo = e == 0 ? mul2(wlo, wlo) : fma2(wlo, wlo, dlo);
                        dhi = e == 0 ? mul2(whi, whi) : fma2(whi, whi, dhi);
                    }
                    float d4[4];
                    unpack2(dlo, d4[0], d4[1]);
                    unpack2(dhi, d4[2], d4[3]);
                    const int4 id4 = *reinterpret_cast<const int4*>(&wid[warp][t]);
                    const int ids[4] = {id4.x, id4.y, id4.z, id4.w};
                    // a float compare with the K-th distance screens first (distances >= 0 order
                    // like their bits; the 64-bit key then settles an equal distance by id)
                    const float dlast = key_dist(kk[KC - 1]);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (t + u < cnt && d4[u] <= dlast) {
                            const unsigned long long key = nn_key(d4[u], ids[u]);
                            if (key < kk[KC - 1]) insert_nn<KC>(kk, key);
                        }
                }
            }
        }
        // next super-box: alternate above and below home while both remain
        const bool go_up = (it & 1) == 0 ? up < nsup : down < 0;
        if (go_up && up < nsup) cur = up++;
        else if (down >= 0) cur = down--;
        else cur = up++;
    }
    if (COUNT && lane == 0) atomicAdd(work, evaluated);
    if (!live) return;
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        if (k >= K) break;
        const bool ok = kk[k] != kNone;
        idx[(int64_t)qid * K + k] = ok ? (int64_t)(unsigned)(kk[k] & 0xffffffffu) : -1;
        dists[(int64_t)qid * K + k] = ok ? key_dist(kk[k]) : -1.f;
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

// The ordering passes and the search for one dimension D.
template <int D>
cudaError_t run_knn(int N, int K, const float* p1, const float* p2, const int64_t* d_first1, const int64_t* d_first2,
                    const int64_t* d_pre1, const int64_t* d_pre2, const int64_t* d_num2, const int64_t* d_gpre,
                    const int64_t* d_spre, int64_t S1, int64_t S2, int64_t G, int64_t NS, CloudBox* box, int* counts1,
                    int* counts2, int* off1, int* off2, long long* tile1, long long* tile2, float4* sq, int* sqid,
                    short* sqcode, float4* sr, int* srid, short* srcode, float4* glo, float4* ghi, float4* slo,
                    float4* shi, const KnnTile* tiles, int ntiles, int64_t* idx, float* dists,
                    unsigned long long* work, cudaStream_t s) {
    const int nb = N * kCells, nt = (nb + kScanTile - 1) / kScanTile;
    cudaError_t e;
    k_cloud_box<D><<<N, 256, 0, s>>>(p2, d_first2, d_num2, box);
    if ((e = cudaMemsetAsync(counts1, 0, sizeof(int) * (size_t)nb, s))) return e;
    if ((e = cudaMemsetAsync(counts2, 0, sizeof(int) * (size_t)nb, s))) return e;
    if (S1 > 0)
        k_order_points<D, false><<<grid_for(S1), 256, 0, s>>>(p1, d_first1, d_pre1, N, S1, box, counts1, nullptr,
                                                              nullptr, nullptr, nullptr);
    if (S2 > 0)
        k_order_points<D, false><<<grid_for(S2), 256, 0, s>>>(p2, d_first2, d_pre2, N, S2, box, counts2, nullptr,
                                                              nullptr, nullptr, nullptr);
    k_scan_tiles<<<nt, 1024, 0, s>>>(counts1, nb, off1, tile1);
    k_scan_tops<<<1, 1024, 0, s>>>(tile1, nt, tile1 + nt);
    k_scan_add<<<std::min((nb + 256) / 256, 148 * 8), 256, 0, s>>>(off1, nb, tile1, tile1 + nt);
    k_scan_tiles<<<nt, 1024, 0, s>>>(counts2, nb, off2, tile2);
    k_scan_tops<<<1, 1024, 0, s>>>(tile2, nt, tile2 + nt);
    k_scan_add<<<std::min((nb + 256) / 256, 148 * 8), 256, 0, s>>>(off2, nb, tile2, tile2 + nt);
    if ((e = cudaMemsetAsync(counts1, 0, sizeof(int) * (size_t)nb, s))) return e;
    if ((e = cudaMemsetAsync(counts2, 0, sizeof(int) * (size_t)nb, s))) return e;
    if (S1 > 0)
        k_order_points<D, true><<<grid_for(S1), 256, 0, s>>>(p1, d_first1, d_pre1, N, S1, box, counts1, off1, sq,
                                                             sqid, sqcode);
    if (S2 > 0)
        k_order_points<D, true><<<grid_for(S2), 256, 0, s>>>(p2, d_first2, d_pre2, N, S2, box, counts2, off2, sr,
                                                             srid, srcode);
    if (G > 0) {
        k_group_boxes<<<(int)std::min<int64_t>((G + 7) / 8, 148 * 32), 256, 0, s>>>(sr, d_pre2, d_num2, d_gpre, N, G,
                                                                                    glo, ghi);
        k_super_boxes<<<(int)std::min<int64_t>((NS + 7) / 8, 148 * 32), 256, 0, s>>>(glo, ghi, d_gpre, d_spre, N, NS,
                                                                                     G, slo, shi);
    }
    if ((e = cudaGetLastError())) return e;
#define MR_KNN(KC)                                                                                            \
    if (work)                                                                                                 \
        k_knn<KC, D, true><<<ntiles, kKnnQueries, 0, s>>>(sq, sqid, sqcode, sr, srid, off2, d_pre2, d_num2,   \
                                                          d_gpre, d_spre, glo, ghi, slo, shi, tiles, K, idx, \
                                                          dists, work);                                       \
    else                                                                                                      \
        k_knn<KC, D, false><<<ntiles, kKnnQueries, 0, s>>>(sq, sqid, sqcode, sr, srid, off2, d_pre2, d_num2,  \
                                                           d_gpre, d_spre, glo, ghi, slo, shi, tiles, K, idx, \
                                                           dists, nullptr)
    if (K <= 1) { MR_KNN(1); }
    else if (K <= 2) { MR_KNN(2); }
    else if (K <= 4) { MR_KNN(4); }
    else if (K <= 8) { MR_KNN(8); }
    else if (K <= 16) { MR_KNN(16); }
    else { MR_KNN(32); }
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

// The whole search; with `evaluated` (host) also the number of (query, reference) pairs
// whose distance the search evaluated (one more stream synchronisation).
int knn_impl(const float* p1, int64_t P1, const int64_t* first1, const int64_t* num1, const float* p2, int64_t P2,
             const int64_t* first2, const int64_t* num2, int32_t N, int32_t D, int32_t K, int64_t* idx, float* dists,
             int64_t* evaluated, void* stream) {
    if (evaluated) *evaluated = 0;
    if (N < 0 || D < 1 || D > MR_KNN_DMAX || K < 1 || K > MR_KMAX || P1 < 0 || P2 < 0 || P1 > INT32_MAX ||
        P2 > INT32_MAX) {
        set_error("invalid arguments N=%d D=%d K=%d P1=%lld P2=%lld", N, D, K, (long long)P1, (long long)P2);
        return MR_ERR_ARG;
    }
    if (P1 == 0) return MR_OK;
    if (!p1 || !idx || !dists || (N > 0 && (!first1 || !num1 || !first2 || !num2)) || (P2 > 0 && !p2)) {
        set_error("null pointer");
        return MR_ERR_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    std::vector<int64_t> staged;
    int rc = host_indices(s, N, staged, {&first1, &num1, &first2, &num2});
    if (rc != MR_OK) return rc;
    rc = check_sets(first1, num1, N, P1, "mr_knn_fwd queries");
    if (rc == MR_OK) rc = check_sets(first2, num2, N, P2, "mr_knn_fwd references");
    if (rc != MR_OK) return rc;
    // query clouds must be disjoint; rows outside every cloud are filled with -1
    std::vector<std::pair<int64_t, int64_t>> ranges;
    for (int n = 0; n < N; ++n)
        if (num1[n] > 0) ranges.push_back({first1[n], num1[n]});
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
    if (covered == 0) return MR_OK;
    if ((int64_t)N * kCells >= INT32_MAX / 2) {
        set_error("too many clouds");
        return MR_ERR_ARG;
    }
    // host-side plan: prefix sums of the cloud sizes (ordered positions) and the tiles
    std::vector<int64_t> host(7 * (size_t)N);
    int64_t* h_first1 = host.data();
    int64_t* h_first2 = h_first1 + N;
    int64_t* h_pre1 = h_first2 + N;
    int64_t* h_pre2 = h_pre1 + N;
    int64_t* h_num2 = h_pre2 + N;
    int64_t* h_gpre = h_num2 + N;     // first group box of each cloud (groups of 32 references)
    int64_t* h_spre = h_gpre + N;     // first super box (32 groups)
    int64_t S1 = 0, S2 = 0, G = 0, NS = 0;
    std::vector<KnnTile> tiles;
    for (int n = 0; n < N; ++n) {
        h_first1[n] = first1[n];
        h_first2[n] = first2[n];
        h_pre1[n] = S1;
        h_pre2[n] = S2;
        h_num2[n] = num2[n];
        h_gpre[n] = G;
        h_spre[n] = NS;
        for (int64_t q = 0; q < num1[n]; q += kKnnQueries)
            tiles.push_back({S1 + q, (int)std::min<int64_t>(kKnnQueries, num1[n] - q), n});
        S1 += num1[n];
        S2 += num2[n];
        const int64_t ng = (num2[n] + 31) / 32;
        G += ng;
        NS += (ng + 31) / 32;
    }
    if (S2 > INT32_MAX) {
        set_error("more than 2^31 reference points in the clouds");
        return MR_ERR_ARG;
    }
    std::stable_sort(tiles.begin(), tiles.end(),
                     [&](const KnnTile& a, const KnnTile& b) { return num2[a.n] > num2[b.n]; });
    // one scratch block: int64 plan, boxes, counts/offsets/tile sums of both sets, the
    // ordered sets, the tiles
    const int nb = N * kCells, nt = (nb + kScanTile - 1) / kScanTile;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    size_t sz[13] = {sizeof(int64_t) * host.size(), sizeof(CloudBox) * (size_t)N, sizeof(int) * (size_t)nb,
                     sizeof(int) * (size_t)nb, sizeof(int) * ((size_t)nb + 1), sizeof(int) * ((size_t)nb + 1),
                     sizeof(long long) * ((size_t)nt + 1), sizeof(long long) * ((size_t)nt + 1),
                     (sizeof(float4) + sizeof(int) + sizeof(short)) * (size_t)S1,
                     (sizeof(float4) + sizeof(int) + sizeof(short)) * (size_t)S2, sizeof(KnnTile) * tiles.size(),
                     sizeof(float4) * 2 * (size_t)(G + NS), sizeof(unsigned long long)};
    size_t total = 0, at[13];
    for (int i = 0; i < 13; ++i) {
        at[i] = total;
        total += up(sz[i]);
    }
    char* base = nullptr;
    rc = scratch_alloc(reinterpret_cast<void**>(&base), total, s);
    if (rc != MR_OK) return rc;
    int64_t* plan = reinterpret_cast<int64_t*>(base + at[0]);
    CloudBox* box = reinterpret_cast<CloudBox*>(base + at[1]);
    int* counts1 = reinterpret_cast<int*>(base + at[2]);
    int* counts2 = reinterpret_cast<int*>(base + at[3]);
    int* off1 = reinterpret_cast<int*>(base + at[4]);
    int* off2 = reinterpret_cast<int*>(base + at[5]);
    long long* tile1 = reinterpret_cast<long long*>(base + at[6]);
    long long* tile2 = reinterpret_cast<long long*>(base + at[7]);
    float4* sq = reinterpret_cast<float4*>(base + at[8]);
    int* sqid = reinterpret_cast<int*>(sq + S1);
    short* sqcode = reinterpret_cast<short*>(sqid + S1);
    float4* sr = reinterpret_cast<float4*>(base + at[9]);
    int* srid = reinterpret_cast<int*>(sr + S2);
    short* srcode = reinterpret_cast<short*>(srid + S2);
    KnnTile* dt = reinterpret_cast<KnnTile*>(base + at[10]);
    float4* glo = reinterpret_cast<float4*>(base + at[11]);
    float4* ghi = glo + G;
    float4* slo = ghi + G;
    float4* shi = slo + NS;
    unsigned long long* work = evaluated ? reinterpret_cast<unsigned long long*>(base + at[12]) : nullptr;
    cudaError_t e = cudaMemcpyAsync(plan, host.data(), sz[0], cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dt, tiles.data(), sz[10], cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && work) e = cudaMemsetAsync(work, 0, sizeof(unsigned long long), s);
    if (e == cudaSuccess) {
        ProfScope ps(MR_STAGE_KNN, s);
        const int ntl = (int)tiles.size();
        const int64_t *f1 = plan, *f2 = plan + N, *pr1 = plan + 2 * N, *pr2 = plan + 3 * N, *n2 = plan + 4 * N;
        const int64_t *gp = plan + 5 * N, *sp = plan + 6 * N;
#define MR_RUN(DD)                                                                                                   \
    run_knn<DD>(N, K, p1, p2, f1, f2, pr1, pr2, n2, gp, sp, S1, S2, G, NS, box, counts1, counts2, off1, off2, tile1, \
                tile2, sq, sqid, sqcode, sr, srid, srcode, glo, ghi, slo, shi, dt, ntl, idx, dists, work, s)
        switch (D) {
            case 1: e = MR_RUN(1); break;
            case 2: e = MR_RUN(2); break;
            case 3: e = MR_RUN(3); break;
            default: e = MR_RUN(4); break;
        }
#undef MR_RUN
    }
    unsigned long long count = 0;
    if (e == cudaSuccess && work) {
        e = cudaMemcpyAsync(&count, work, sizeof(count), cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    }
    // (copies from pageable host memory return once the data is staged: the vectors may go)
    scratch_free(base, s);
    if (e != cudaSuccess) return cuda_fail(e, "knn");
    if (evaluated) *evaluated = (int64_t)count;
    return MR_OK;
}

}  // namespace
}  // namespace mr

extern "C" {

int mr_knn_fwd(const float* p1, int64_t P1, const int64_t* first1, const int64_t* num1, const float* p2, int64_t P2,
               const int64_t* first2, const int64_t* num2, int32_t N, int32_t D, int32_t K, int64_t* idx,
               float* dists, void* stream) {
    return mr::knn_impl(p1, P1, first1, num1, p2, P2, first2, num2, N, D, K, idx, dists, nullptr, stream);
}

int mr_knn_count_pairs(const float* p1, int64_t P1, const int64_t* first1, const int64_t* num1, const float* p2,
                       int64_t P2, const int64_t* first2, const int64_t* num2, int32_t N, int32_t D, int32_t K,
                       int64_t* idx, float* dists, int64_t* evaluated_pairs, void* stream) {
    if (!evaluated_pairs) {
        mr::set_error("null evaluated_pairs");
        return MR_ERR_ARG;
    }
    return mr::knn_impl(p1, P1, first1, num1, p2, P2, first2, num2, N, D, K, idx, dists, evaluated_pairs, stream);
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
