// Phong lighting for the stage-two shaders ("Accelerating 3D Deep Learning with PyTorch3D",
// method: pluggable Gouraud and Phong shaders with lights and materials).  The pages give
// no formula; this is the textbook Phong reflection model with one point light:
//
//   n = N/|N|, l = (L - P)/|L - P|, v = (C - P)/|C - P|, cos = n.l, rv = 2 cos (n.v) - l.v
//   colour = (ambient + diffuse max(cos, 0)) c + specular [cos > 0, rv > 0] rv^shininess
//
// and its gradient with the two switches held.  Two forms:
//   * per point (k_phong_fwd / k_phong_bwd): the lighting of Gouraud shading, evaluated at
//     the mesh vertices before the colours are interpolated;
//   * per fragment, fused with the interpolation (k_phong_shade_fwd / _bwd): P, N and c are
//     interpolated from the face's vertices with the slot's barycentrics and lit in
//     registers, so the interpolated attributes (36 bytes per slot) never reach memory.
// float32 except the interpolation sums (float64, see interpolate3); the normalisations
// use 1/sqrt, the specular power powf.
#include <cmath>

#include "mr_common.cuh"

namespace mr {
namespace {

struct PhongParams {
    float L[3], C[3], amb[3], dif[3], spe[3], shine;
};

struct f3 {
    float x, y, z;
};
__device__ __forceinline__ f3 mk(float x, float y, float z) { return {x, y, z}; }
__device__ __forceinline__ f3 operator+(f3 a, f3 b) { return {a.x + b.x, a.y + b.y, a.z + b.z}; }
__device__ __forceinline__ f3 operator-(f3 a, f3 b) { return {a.x - b.x, a.y - b.y, a.z - b.z}; }
__device__ __forceinline__ f3 operator*(float s, f3 a) { return {s * a.x, s * a.y, s * a.z}; }
__device__ __forceinline__ float dot(f3 a, f3 b) { return fmaf(a.x, b.x, fmaf(a.y, b.y, a.z * b.z)); }
__device__ __forceinline__ f3 ld3(const float* __restrict__ p, int64_t i) { return {p[3 * i], p[3 * i + 1], p[3 * i + 2]}; }
__device__ __forceinline__ void st3(float* __restrict__ p, int64_t i, f3 a) {
    p[3 * i] = a.x;
    p[3 * i + 1] = a.y;
    p[3 * i + 2] = a.z;
}

struct PhongState {
    f3 n, l, v;
    float inv_n, inv_l, inv_v;   // 1/|N|, 1/|L - P|, 1/|C - P|
    float cos, nv, lv, rv, td, ts;
    bool lit, shiny;
};

__device__ __forceinline__ void phong_eval(f3 P, f3 N, const PhongParams& Q, PhongState& S) {
    const f3 dl = mk(Q.L[0], Q.L[1], Q.L[2]) - P;
    const f3 dv = mk(Q.C[0], Q.C[1], Q.C[2]) - P;
    S.inv_n = rsqrtf(dot(N, N));
    S.inv_l = rsqrtf(dot(dl, dl));
    S.inv_v = rsqrtf(dot(dv, dv));
    S.n = S.inv_n * N;
    S.l = S.inv_l * dl;
    S.v = S.inv_v * dv;
    S.cos = dot(S.n, S.l);
    S.nv = dot(S.n, S.v);
    S.lv = dot(S.l, S.v);
    S.rv = 2.f * S.cos * S.nv - S.lv;
    S.lit = S.cos > 0.f;
    S.shiny = S.lit && S.rv > 0.f;
    S.td = S.lit ? S.cos : 0.f;
    S.ts = S.shiny ? powf(S.rv, Q.shine) : 0.f;
}

__device__ __forceinline__ f3 phong_colour(const PhongState& S, f3 c, const PhongParams& Q) {
    return mk(fmaf(fmaf(Q.dif[0], S.td, Q.amb[0]), c.x, Q.spe[0] * S.ts),
              fmaf(fmaf(Q.dif[1], S.td, Q.amb[1]), c.y, Q.spe[1] * S.ts),
              fmaf(fmaf(Q.dif[2], S.td, Q.amb[2]), c.z, Q.spe[2] * S.ts));
}

// (g - (g.u) u) / |x| for u = x / |x|: the gradient of the normalisation.
__device__ __forceinline__ f3 unit_bwd(f3 u, float inv_len, f3 g) { return inv_len * (g - dot(g, u) * u); }

// Gradient of one lit point: gP, gN, gc from the colour gradient g.
__device__ __forceinline__ void phong_point_bwd(f3 P, f3 N, f3 c, f3 g, const PhongParams& Q, f3& gP, f3& gN,
                                                f3& gc) {
    PhongState S;
    phong_eval(P, N, Q, S);
    gc = mk(g.x * fmaf(Q.dif[0], S.td, Q.amb[0]), g.y * fmaf(Q.dif[1], S.td, Q.amb[1]),
            g.z * fmaf(Q.dif[2], S.td, Q.amb[2]));
    const float g_td = fmaf(g.x, Q.dif[0] * c.x, fmaf(g.y, Q.dif[1] * c.y, g.z * Q.dif[2] * c.z));
    const float g_ts = fmaf(g.x, Q.spe[0], fmaf(g.y, Q.spe[1], g.z * Q.spe[2]));
    // d rv^s / d rv = s rv^(s - 1) = s ts / rv (rv > 0 where the term is on): the power
    // already formed for the colour, divided once, instead of a second powf
    const float g_rv = S.shiny ? g_ts * Q.shine * __fdividef(S.ts, S.rv) : 0.f;
    const float g_cos = (S.lit ? g_td : 0.f) + 2.f * g_rv * S.nv;
    const float g_nv = 2.f * g_rv * S.cos;
    const float g_lv = -g_rv;
    const f3 gn = g_cos * S.l + g_nv * S.v;
    const f3 gl = g_cos * S.n + g_lv * S.v;
    const f3 gv = g_nv * S.n + g_lv * S.l;
    gN = unit_bwd(S.n, S.inv_n, gn);
    gP = mk(0.f, 0.f, 0.f) - unit_bwd(S.l, S.inv_l, gl) - unit_bwd(S.v, S.inv_v, gv);
}

__global__ void k_phong_fwd(const float* __restrict__ P, const float* __restrict__ N, const float* __restrict__ c,
                            int64_t M, PhongParams Q, float* __restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < M; i += (int64_t)gridDim.x * blockDim.x) {
        PhongState S;
        phong_eval(ld3(P, i), ld3(N, i), Q, S);
        st3(out, i, phong_colour(S, ld3(c, i), Q));
    }
}

__global__ void k_phong_bwd(const float* __restrict__ P, const float* __restrict__ N, const float* __restrict__ c,
                            int64_t M, PhongParams Q, const float* __restrict__ g, float* __restrict__ gP,
                            float* __restrict__ gN, float* __restrict__ gc) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < M; i += (int64_t)gridDim.x * blockDim.x) {
        f3 a, b, d;
        phong_point_bwd(ld3(P, i), ld3(N, i), ld3(c, i), ld3(g, i), Q, a, b, d);
        if (gP) st3(gP, i, a);
        if (gN) st3(gN, i, b);
        if (gc) st3(gc, i, d);
    }
}

// Face vertex ids of slot s, or false (and the error bit) for an invalid entry.
__device__ __forceinline__ bool slot_face(const int64_t* __restrict__ p2f, const int64_t* __restrict__ faces,
                                          int64_t F, int64_t V, int64_t s, int64_t (&v)[3], int* err) {
    const int64_t f = p2f[s];
    if (f == -1) return false;
    if (f < -1 || f >= F) {
        atomicOr(err, kErrSlotIndex);
        return false;
    }
    v[0] = faces[3 * f];
    v[1] = faces[3 * f + 1];
    v[2] = faces[3 * f + 2];
    if (v[0] < 0 || v[0] >= V || v[1] < 0 || v[1] >= V || v[2] < 0 || v[2] >= V) {
        atomicOr(err, kErrFaceIndex);
        return false;
    }
    return true;
}

// sum_m b_m a_m, summed in float64 and rounded once: blur-ring slots of faces seen
// edge-on carry barycentrics of magnitude up to tens, and a float32 sum would lose about
// log2(sum |b_m|) bits to cancellation before the lighting magnifies the error.
__device__ __forceinline__ void interpolate3(const float (&b)[3], f3 a0, f3 a1, f3 a2, f3& out) {
    out.x = (float)((double)b[0] * a0.x + (double)b[1] * a1.x + (double)b[2] * a2.x);
    out.y = (float)((double)b[0] * a0.y + (double)b[1] * a1.y + (double)b[2] * a2.y);
    out.z = (float)((double)b[0] * a0.z + (double)b[1] * a1.z + (double)b[2] * a2.z);
}

__global__ void k_phong_shade_fwd(const int64_t* __restrict__ p2f, const float* __restrict__ bary, int64_t nslots,
                                  const int64_t* __restrict__ faces, int64_t F, const float* __restrict__ vP,
                                  const float* __restrict__ vN, const float* __restrict__ vc, int64_t V, PhongParams Q,
                                  float* __restrict__ out, int* __restrict__ err) {
    for (int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; s < nslots; s += (int64_t)gridDim.x * blockDim.x) {
        int64_t v[3];
        if (!slot_face(p2f, faces, F, V, s, v, err)) {
            st3(out, s, mk(0.f, 0.f, 0.f));
            continue;
        }
        const float b[3] = {bary[3 * s], bary[3 * s + 1], bary[3 * s + 2]};
        f3 P, N, c;
        interpolate3(b, ld3(vP, v[0]), ld3(vP, v[1]), ld3(vP, v[2]), P);
        interpolate3(b, ld3(vN, v[0]), ld3(vN, v[1]), ld3(vN, v[2]), N);
        interpolate3(b, ld3(vc, v[0]), ld3(vc, v[1]), ld3(vc, v[2]), c);
        PhongState S;
        phong_eval(P, N, Q, S);
        st3(out, s, phong_colour(S, c, Q));
    }
}

// Per slot: the lit point's gradient, spread to the three vertices with weights bary_m as
// three float4 atomics each into a V x 3 float4 accumulator (rows: P, N, c; w unused), and
// grad_bary_m = vP_m.gP + vN_m.gN + vc_m.gc.
__global__ void k_phong_shade_bwd(const int64_t* __restrict__ p2f, const float* __restrict__ bary, int64_t nslots,
                                  const int64_t* __restrict__ faces, int64_t F, const float* __restrict__ vP,
                                  const float* __restrict__ vN, const float* __restrict__ vc, int64_t V, PhongParams Q,
                                  const float* __restrict__ g, float4* __restrict__ acc, float* __restrict__ grad_bary,
                                  int* __restrict__ err) {
    for (int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; s < nslots; s += (int64_t)gridDim.x * blockDim.x) {
        int64_t v[3];
        if (!slot_face(p2f, faces, F, V, s, v, err)) {
            if (grad_bary) st3(grad_bary, s, mk(0.f, 0.f, 0.f));
            continue;
        }
        const float b[3] = {bary[3 * s], bary[3 * s + 1], bary[3 * s + 2]};
        f3 Pm[3], Nm[3], cm[3];
#pragma unroll
        for (int m = 0; m < 3; ++m) {
            Pm[m] = ld3(vP, v[m]);
            Nm[m] = ld3(vN, v[m]);
            cm[m] = ld3(vc, v[m]);
        }
        f3 P, N, c;
        interpolate3(b, Pm[0], Pm[1], Pm[2], P);
        interpolate3(b, Nm[0], Nm[1], Nm[2], N);
        interpolate3(b, cm[0], cm[1], cm[2], c);
        f3 gP, gN, gc;
        phong_point_bwd(P, N, c, ld3(g, s), Q, gP, gN, gc);
        float gb[3];
#pragma unroll
        for (int m = 0; m < 3; ++m) {
            gb[m] = dot(Pm[m], gP) + dot(Nm[m], gN) + dot(cm[m], gc);
            float4* a = acc + 3 * v[m];
            atomicAdd(a, make_float4(b[m] * gP.x, b[m] * gP.y, b[m] * gP.z, 0.f));
            atomicAdd(a + 1, make_float4(b[m] * gN.x, b[m] * gN.y, b[m] * gN.z, 0.f));
            atomicAdd(a + 2, make_float4(b[m] * gc.x, b[m] * gc.y, b[m] * gc.z, 0.f));
        }
        if (grad_bary) st3(grad_bary, s, mk(gb[0], gb[1], gb[2]));
    }
}

__global__ void k_acc_to_attributes(const float4* __restrict__ acc, int64_t V, float* __restrict__ gP,
                                    float* __restrict__ gN, float* __restrict__ gc) {
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < V; v += (int64_t)gridDim.x * blockDim.x) {
        const float4 p = acc[3 * v], n = acc[3 * v + 1], c = acc[3 * v + 2];
        st3(gP, v, mk(p.x, p.y, p.z));
        st3(gN, v, mk(n.x, n.y, n.z));
        st3(gc, v, mk(c.x, c.y, c.z));
    }
}

int read_params(const float* params, PhongParams& Q) {
    if (!params) {
        set_error("null params");
        return MR_ERR_ARG;
    }
    for (int i = 0; i < MR_PHONG_NPARAMS; ++i)
        if (!std::isfinite(params[i])) {
            set_error("params[%d] is not finite", i);
            return MR_ERR_ARG;
        }
    if (params[15] < 1.f) {
        set_error("shininess %g < 1", (double)params[15]);
        return MR_ERR_ARG;
    }
    for (int e = 0; e < 3; ++e) {
        Q.L[e] = params[e];
        Q.C[e] = params[3 + e];
        Q.amb[e] = params[6 + e];
        Q.dif[e] = params[9 + e];
        Q.spe[e] = params[12 + e];
    }
    Q.shine = params[15];
    return MR_OK;
}

int check_shade(int64_t npix, int32_t K, int64_t F, int64_t V) {
    if (npix < 0 || K < 1 || K > MR_KMAX || F < 0 || V < 0) {
        set_error("invalid shape npix=%lld K=%d F=%lld V=%lld", (long long)npix, K, (long long)F, (long long)V);
        return MR_ERR_ARG;
    }
    return MR_OK;
}

}  // namespace
}  // namespace mr

extern "C" {

int mr_phong_fwd(const float* points, const float* normals, const float* albedo, int64_t M, const float* params,
                 float* colors, void* stream) {
    mr::PhongParams Q;
    int rc = mr::read_params(params, Q);
    if (rc != MR_OK) return rc;
    if (M < 0) {
        mr::set_error("negative point count");
        return MR_ERR_ARG;
    }
    if (M == 0) return MR_OK;
    if (!points || !normals || !albedo || !colors) {
        mr::set_error("null pointer");
        return MR_ERR_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    {
        mr::ProfScope ps(MR_STAGE_PHONG_FWD, s);
        mr::k_phong_fwd<<<mr::grid_for(M), 256, 0, s>>>(points, normals, albedo, M, Q, colors);
    }
    MR_CUDA(cudaGetLastError());
    return MR_OK;
}

int mr_phong_bwd(const float* points, const float* normals, const float* albedo, int64_t M, const float* params,
                 const float* grad_colors, float* grad_points, float* grad_normals, float* grad_albedo,
                 void* stream) {
    mr::PhongParams Q;
    int rc = mr::read_params(params, Q);
    if (rc != MR_OK) return rc;
    if (M < 0) {
        mr::set_error("negative point count");
        return MR_ERR_ARG;
    }
    if (M == 0 || (!grad_points && !grad_normals && !grad_albedo)) return MR_OK;
    if (!points || !normals || !albedo || !grad_colors) {
        mr::set_error("null pointer");
        return MR_ERR_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    {
        mr::ProfScope ps(MR_STAGE_PHONG_BWD, s);
        mr::k_phong_bwd<<<mr::grid_for(M), 256, 0, s>>>(points, normals, albedo, M, Q, grad_colors, grad_points,
                                                        grad_normals, grad_albedo);
    }
    MR_CUDA(cudaGetLastError());
    return MR_OK;
}

int mr_phong_shade_fwd(const int64_t* pix_to_face, const float* bary, int64_t npix, int32_t K, const int64_t* faces,
                       int64_t F, const float* points, const float* normals, const float* albedo, int64_t V,
                       const float* params, float* colors, void* stream) {
    mr::PhongParams Q;
    int rc = mr::read_params(params, Q);
    if (rc == MR_OK) rc = mr::check_shade(npix, K, F, V);
    if (rc != MR_OK) return rc;
    const int64_t nslots = npix * K;
    if (nslots == 0) return MR_OK;
    if (!pix_to_face || !bary || !colors || (F > 0 && !faces) || (V > 0 && (!points || !normals || !albedo))) {
        mr::set_error("null pointer");
        return MR_ERR_ARG;
    }
    int* err = mr::device_error_word();
    if (!err) {
        mr::set_error("cannot locate the device error word");
        return MR_ERR_CUDA;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    {
        mr::ProfScope ps(MR_STAGE_PHONG_SHADE_FWD, s);
        mr::k_phong_shade_fwd<<<mr::grid_for(nslots), 256, 0, s>>>(pix_to_face, bary, nslots, faces, F, points,
                                                                  normals, albedo, V, Q, colors, err);
    }
    MR_CUDA(cudaGetLastError());
    return MR_OK;
}

int mr_phong_shade_bwd(const int64_t* pix_to_face, const float* bary, int64_t npix, int32_t K, const int64_t* faces,
                       int64_t F, const float* points, const float* normals, const float* albedo, int64_t V,
                       const float* params, const float* grad_colors, float* grad_points, float* grad_normals,
                       float* grad_albedo, float* grad_bary, void* stream) {
    mr::PhongParams Q;
    int rc = mr::read_params(params, Q);
    if (rc == MR_OK) rc = mr::check_shade(npix, K, F, V);
    if (rc != MR_OK) return rc;
    if (V > 0 && (!grad_points || !grad_normals || !grad_albedo)) {
        mr::set_error("null gradient output");
        return MR_ERR_ARG;
    }
    const int64_t nslots = npix * K;
    if (nslots > 0 && (!pix_to_face || !bary || !grad_colors || (F > 0 && !faces) ||
                       (V > 0 && (!points || !normals || !albedo)))) {
        mr::set_error("null pointer");
        return MR_ERR_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (V == 0 && nslots == 0) return MR_OK;
    int* err = mr::device_error_word();
    if (!err) {
        mr::set_error("cannot locate the device error word");
        return MR_ERR_CUDA;
    }
    float4* acc = nullptr;
    const size_t acc_bytes = sizeof(float4) * 3 * (size_t)V;
    if (V > 0) {
        rc = mr::scratch_alloc(reinterpret_cast<void**>(&acc), acc_bytes, s);
        if (rc != MR_OK) return rc;
    }
    cudaError_t e = V > 0 ? cudaMemsetAsync(acc, 0, acc_bytes, s) : cudaSuccess;
    if (e == cudaSuccess) {
        mr::ProfScope ps(MR_STAGE_PHONG_SHADE_BWD, s);
        if (nslots > 0)
            mr::k_phong_shade_bwd<<<mr::grid_for(nslots), 256, 0, s>>>(pix_to_face, bary, nslots, faces, F, points,
                                                                      normals, albedo, V, Q, grad_colors, acc,
                                                                      grad_bary, err);
        if (V > 0)
            mr::k_acc_to_attributes<<<mr::grid_for(V), 256, 0, s>>>(acc, V, grad_points, grad_normals, grad_albedo);
        e = cudaGetLastError();
    }
    if (acc) mr::scratch_free(acc, s);
    if (e != cudaSuccess) return mr::cuda_fail(e, "Phong shading backward");
    return MR_OK;
}

}  // extern "C"
