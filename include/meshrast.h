/*
 * meshrast.h -- C ABI of the B200 (sm_100a) mesh rasterizer hot path.
 *
 * The operation is the two-stage differentiable mesh rasterizer of PyTorch3D
 * ("Accelerating 3D Deep Learning with PyTorch3D"): stage one keeps, for every pixel,
 * the K nearest faces (method summary: the rasterizer is split in two stages, the first
 * choosing K faces per pixel); stage two blends their influence into a soft silhouette;
 * the backward pass carries pixel gradients back to the vertex positions (tutorial
 * summary, 3:52: gradients flow from the image back to the mesh).  The batch is
 * heterogeneous and packed (tutorial summary, 1:00).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Screen space: verts are (x_ndc, y_ndc, z_view) per vertex, float32, row-major
 *    V x 3.  Pixel (i, j) of an H x W image has centre x = -1 + (2j+1)/W,
 *    y = 1 - (2i+1)/H: +x right, +y up, row 0 at the top.
 *  - faces: int64, F x 3, global (packed) vertex ids.  Mesh n owns faces
 *    [mesh_to_face_first_idx[n], mesh_to_face_first_idx[n] + num_faces_per_mesh[n]).
 *  - Per-pixel outputs are N x H x W x K, slot k innermost; bary adds a trailing 3.
 *  - pix_to_face holds the global face id, -1 for an empty slot.  Empty slots hold -1
 *    in zbuf, in all three bary components and in dists.
 *  - dists is the signed squared 2-D distance to the face: negative inside.
 *  - blur_radius is a threshold on that squared distance (NDC^2 units): a face is a
 *    candidate for a pixel iff the pixel centre is inside the closed triangle or
 *    within squared distance blur_radius of it.  Candidates are ordered by (z, face id);
 *    degenerate faces (|2 * area| <= 1e-12) and candidates with z < 0 are dropped.
 *  - Pointers are DEVICE pointers unless marked otherwise.  Per-mesh (per-cloud) index
 *    arrays are HOST OR DEVICE: the library asks CUDA which one a pointer is and reads a
 *    device array with one device-to-host copy on `stream`, followed by a
 *    synchronisation of `stream` (so such an array must be ready in stream order).  The
 *    caller owns every input and
 *    output; the library allocates its own scratch (stream-ordered, from the device's
 *    default memory pool, released before the call returns) and never frees caller
 *    memory.  stream is a cudaStream_t (NULL = legacy default stream).
 *  - Every function returns MR_OK (0) or a negative MR_ERR_* code and never aborts.
 *    Arguments are validated on the host before any launch; on MR_ERR_ARG nothing
 *    was launched.  mr_last_error() gives a thread-local message for the last failure.
 *  - Device-side checks (a face vertex id outside [0, V), a pix_to_face entry outside
 *    [-1, F)) never trap: the offending face or slot is skipped and a device error
 *    word is set.  mr_rasterize_fwd reads it before returning; the asynchronous entry
 *    points leave it for mr_device_status().
 */
#ifndef MESHRAST_H
#define MESHRAST_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MR_OK 0
#define MR_ERR_ARG (-1)     /* invalid argument; nothing launched */
#define MR_ERR_OOM (-2)     /* scratch allocation failed */
#define MR_ERR_CUDA (-3)    /* a CUDA runtime call failed (message in mr_last_error) */
#define MR_ERR_DEVICE (-4)  /* a kernel met an out-of-range index and skipped it */

#define MR_KMAX 32          /* largest K (faces kept per pixel) */
#define MR_MAX_SIDE 32767   /* largest H or W */

/*
 * Stage one (PyTorch3D paper, method: per-pixel K nearest faces; tutorial 32:56:
 * perspective_correct).  For each image n and pixel, the K candidate faces of mesh n
 * nearest in z, with their z, barycentrics and signed squared distance.
 *
 *   verts                    V x 3 float32 (device)
 *   faces                    F x 3 int64 (device), every id in [0, V)
 *   mesh_to_face_first_idx   N int64 (host or device)
 *   num_faces_per_mesh       N int64 (host or device); first + num <= F for every mesh
 *   H, W                     1 .. MR_MAX_SIDE
 *   blur_radius              >= 0, finite (squared NDC units)
 *   K                        1 .. MR_KMAX
 *   perspective_correct      0: barycentrics are the screen-space edge-function
 *                            weights w_k; 1: u_k = w_k / z_k renormalised to sum 1.
 *                            Barycentrics are never clipped (they sum to 1).
 *   pix_to_face              N x H x W x K int64 (device, written)
 *   zbuf, dists              N x H x W x K float32 (device, written)
 *   bary                     N x H x W x K x 3 float32 (device, written)
 *
 * Synchronises `stream` once to size the per-bin face lists (and once more, before any
 * launch, when the per-mesh arrays are device memory).  The list size and the device
 * error word come back through 64 bytes of mapped pinned host memory, allocated on a
 * thread's first call for the current device and kept for the life of the thread; that
 * read-back uses no copy engine, so it does not wait behind the caller's own transfers
 * (where the mapped memory cannot be had, it falls back to a device-to-host copy on
 * `stream`).  The per-mesh arrays go to the device through a pinned host buffer of the
 * same lifetime (2N + 1 int64, grown when a call needs more), so that their copy does not
 * first wait for the stream's earlier work.  Returns MR_ERR_DEVICE if a face referenced a vertex outside [0, V) (that
 * face is then ignored).
 */
int mr_rasterize_fwd(const float* verts, int64_t V, const int64_t* faces, int64_t F,
                     const int64_t* mesh_to_face_first_idx, const int64_t* num_faces_per_mesh,
                     int32_t N, int32_t H, int32_t W, float blur_radius, int32_t K,
                     int32_t perspective_correct, int64_t* pix_to_face, float* zbuf,
                     float* bary, float* dists, void* stream);

/*
 * mr_rasterize_fwd for callers that cannot allocate device memory (no counterpart in the
 * paper: a property of this library's interface).  Some callers may not call cudaMalloc
 * or any allocator while they render -- a host that hands all device memory to its own
 * pool, a latency-critical loop where an allocation could stall or fail under memory
 * pressure, a plugin running inside another program's memory budget.  This entry point
 * computes exactly what mr_rasterize_fwd computes with the same kernels, but takes all
 * of its scratch from one fixed device array of MR_NOALLOC_SCRATCH_BYTES that the
 * library holds on each device using it until the process exits; it calls no cudaMalloc,
 * cudaFree or other allocating routine.  The caller still provides inputs and outputs.
 *  - Batches whose scratch exceeds the array (face records, per-bin counts and lists)
 *    are rejected with MR_ERR_ARG and a message naming the size.
 *  - The first call on a device looks up the array's device address, with that device
 *    current; make that first call before any stream capture.  Every call synchronises
 *    `stream` once, after the bin count, as mr_rasterize_fwd does.
 *  - All calls share the array and it keeps the last call's contents (what must start
 *    at zero is cleared on every call).  Calls whose work overlaps on the GPU race on
 *    it: issue them in order on one stream.
 * Same arguments, outputs, synchronisation and errors as mr_rasterize_fwd.
 */
#define MR_NOALLOC_SCRATCH_BYTES (64 * 1024 * 1024)
int mr_rasterize_fwd_noalloc(const float* verts, int64_t V, const int64_t* faces, int64_t F,
                             const int64_t* mesh_to_face_first_idx,
                             const int64_t* num_faces_per_mesh, int32_t N, int32_t H, int32_t W,
                             float blur_radius, int32_t K, int32_t perspective_correct,
                             int64_t* pix_to_face, float* zbuf, float* bary, float* dists,
                             void* stream);

/*
 * Stage one fused with the stage-two silhouette: the outputs of mr_rasterize_fwd plus
 * alpha (N x H x W float32), bitwise equal to mr_silhouette_blend_fwd applied to the
 * dists written here.  sigma > 0.
 */
int mr_rasterize_silhouette_fwd(const float* verts, int64_t V, const int64_t* faces, int64_t F,
                                const int64_t* mesh_to_face_first_idx,
                                const int64_t* num_faces_per_mesh, int32_t N, int32_t H,
                                int32_t W, float blur_radius, int32_t K,
                                int32_t perspective_correct, float sigma, int64_t* pix_to_face,
                                float* zbuf, float* bary, float* dists, float* alpha,
                                void* stream);

/*
 * Stage two, soft silhouette (PyTorch3D paper, method: the second stage fuses the
 * influence of the K faces; tutorial 22:00: silhouette supervision).  Per pixel,
 * p_k = 1 / (1 + exp(dists_k / sigma)) over slots with pix_to_face >= 0 and
 * alpha = 1 - prod_k (1 - p_k); 0 for a pixel with no face.
 *   pix_to_face N x H x W x K int64, dists N x H x W x K float32, alpha N x H x W float32.
 * Asynchronous.
 */
int mr_silhouette_blend_fwd(const int64_t* pix_to_face, const float* dists, int32_t N,
                            int32_t H, int32_t W, int32_t K, float sigma, float* alpha,
                            void* stream);

/*
 * Gradient of the soft silhouette:
 *   grad_dists_k = -grad_alpha * prod_{j != k} (1 - p_j) * p_k (1 - p_k) / sigma,
 * 0 for empty slots.  grad_alpha N x H x W, grad_dists N x H x W x K (written).
 * Asynchronous.
 */
int mr_silhouette_blend_bwd(const float* grad_alpha, const int64_t* pix_to_face,
                            const float* dists, int32_t N, int32_t H, int32_t W, int32_t K,
                            float sigma, float* grad_dists, void* stream);

/*
 * Backward of stage one to the screen-space vertex positions (tutorial 3:52).  For each
 * valid slot the pixel's barycentrics, z and signed squared distance to face
 * pix_to_face are recomputed and differentiated with the candidate set, the inside
 * flag and the nearest edge held fixed.  grad_zbuf, grad_bary and grad_dists (shaped
 * like zbuf, bary and dists) may each be NULL.  grad_verts (V x 3 float32) is
 * overwritten.  Contributions are summed with float32 atomics, so the low bits of
 * grad_verts depend on scheduling.  Asynchronous; a pix_to_face entry outside [-1, F)
 * or a face vertex outside [0, V) is skipped and flagged for mr_device_status().
 */
int mr_rasterize_bwd(const float* verts, int64_t V, const int64_t* faces, int64_t F,
                     const int64_t* pix_to_face, int32_t N, int32_t H, int32_t W, int32_t K,
                     int32_t perspective_correct, const float* grad_zbuf, const float* grad_bary,
                     const float* grad_dists, float* grad_verts, void* stream);

/*
 * mr_silhouette_blend_bwd followed by mr_rasterize_bwd with only grad_dists, fused so
 * grad_dists never reaches memory.  The inside flag is read from the sign of dists
 * (dists < 0: inside).  grad_verts (V x 3) is overwritten.  Asynchronous.
 */
int mr_silhouette_rasterize_bwd(const float* verts, int64_t V, const int64_t* faces, int64_t F,
                                const int64_t* pix_to_face, const float* dists, int32_t N,
                                int32_t H, int32_t W, int32_t K, float sigma,
                                const float* grad_alpha, float* grad_verts, void* stream);

/*
 * Stage-two shading (PyTorch3D paper, method: pluggable Gouraud and Phong shaders over
 * the K faces kept per pixel; SoftRas, the renderer the paper compares against, is the
 * source of the soft aggregation).  pix_to_face / bary / dists / zbuf are the stage-one
 * outputs (npix = N*H*W pixels of K slots).  All asynchronous.
 *
 * mr_interpolate_fwd: out (npix x K x D float32) = sum_m bary_m attr[v_m] over the face's
 *   vertices v_m, 0 for empty slots (Gouraud: attr = per-vertex colours or normals).
 *   attr: V x D float32 (device).
 * mr_interpolate_bwd: grad_attr (V x D, overwritten; float32 atomics) and grad_bary
 *   (npix x K x 3, may be NULL) from grad_out (npix x K x D).
 * mr_blend_fwd: soft RGB blend of per-slot colours (npix x K x D, D <= MR_BLEND_DMAX) into
 *   rgba (npix x (D + 1) float32: D colour channels, then alpha):
 *     p_k = 1 / (1 + exp(dists_k / sigma)),  s_k = (zfar - zbuf_k) / (zfar - znear),
 *     m = max(max_k s_k, 1e-10),  w_k = p_k exp((s_k - m) / gamma),  w_b = exp((1e-10 - m) / gamma),
 *     rgb = (sum_k w_k colour_k + w_b background) / (sum_k w_k + w_b),  alpha = 1 - prod_k (1 - p_k).
 *   background: D floats (HOST).  sigma, gamma > 0, zfar > znear.
 * mr_blend_bwd: grad_colors (npix x K x D), grad_dists and grad_zbuf (npix x K) from
 *   grad_rgba (npix x (D + 1)); each output may be NULL; empty slots get 0.
 */
#define MR_BLEND_DMAX 8
int mr_interpolate_fwd(const int64_t* pix_to_face, const float* bary, int64_t npix, int32_t K,
                       const int64_t* faces, int64_t F, const float* attr, int64_t V, int32_t D,
                       float* out, void* stream);
int mr_interpolate_bwd(const int64_t* pix_to_face, const float* bary, int64_t npix, int32_t K,
                       const int64_t* faces, int64_t F, const float* attr, int64_t V, int32_t D,
                       const float* grad_out, float* grad_attr, float* grad_bary, void* stream);
int mr_blend_fwd(const int64_t* pix_to_face, const float* colors, const float* dists,
                 const float* zbuf, int64_t npix, int32_t K, int32_t D, const float* background,
                 float sigma, float gamma, float znear, float zfar, float* rgba, void* stream);
int mr_blend_bwd(const int64_t* pix_to_face, const float* colors, const float* dists,
                 const float* zbuf, int64_t npix, int32_t K, int32_t D, const float* background,
                 float sigma, float gamma, float znear, float zfar, const float* grad_rgba,
                 float* grad_colors, float* grad_dists, float* grad_zbuf, void* stream);

/*
 * Phong lighting (PyTorch3D paper, "Accelerating 3D Deep Learning with PyTorch3D", method:
 * Gouraud and Phong shaders with several lights and materials; the pages print no formula,
 * so this is the textbook Phong reflection model with one point light).  params: 16 floats
 * (HOST) = light position L[3], camera position C[3], ambient[3], diffuse[3], specular[3]
 * (each the product of the light's and the material's colour), shininess (>= 1).  At a point
 * P with normal N (any length > 0) and albedo c:
 *   n = N/|N|, l = (L-P)/|L-P|, v = (C-P)/|C-P|, cos = n.l, rv = (2 cos n - l).v,
 *   colour = (ambient + diffuse max(cos, 0)) c + specular [cos > 0 and rv > 0] rv^shininess.
 * Gouraud shading lights the vertices (mr_phong_fwd with M = V) and interpolates the colours
 * with mr_interpolate_fwd; Phong shading lights every fragment (mr_phong_shade_fwd).
 *
 * mr_phong_fwd: colors (M x 3) at M points; points, normals, albedo: M x 3 float32 (device).
 * mr_phong_bwd: grad_points, grad_normals, grad_albedo (M x 3 each, may be NULL) from
 *   grad_colors (M x 3); the two switches are held fixed.
 * mr_phong_shade_fwd: per slot of npix pixels x K, interpolates P, N and c from the face's
 *   vertices (points, normals, albedo: V x 3) with bary, then lights them: colors
 *   (npix x K x 3), 0 for empty slots.  One pass; the interpolated attributes never reach
 *   memory.
 * mr_phong_shade_bwd: grad_points, grad_normals, grad_albedo (V x 3 each, overwritten;
 *   float32 atomics) and grad_bary (npix x K x 3, may be NULL) from grad_colors.
 * Errors: MR_ERR_ARG for negative sizes, K outside [1, MR_KMAX], a NULL required pointer,
 * non-finite params or shininess < 1; out-of-range face or vertex ids are flagged in the
 * device error word (mr_device_status) and the slot is skipped.
 */
#define MR_PHONG_NPARAMS 16
int mr_phong_fwd(const float* points, const float* normals, const float* albedo, int64_t M,
                 const float* params, float* colors, void* stream);
int mr_phong_bwd(const float* points, const float* normals, const float* albedo, int64_t M,
                 const float* params, const float* grad_colors, float* grad_points,
                 float* grad_normals, float* grad_albedo, void* stream);
int mr_phong_shade_fwd(const int64_t* pix_to_face, const float* bary, int64_t npix, int32_t K,
                       const int64_t* faces, int64_t F, const float* points, const float* normals,
                       const float* albedo, int64_t V, const float* params, float* colors,
                       void* stream);
int mr_phong_shade_bwd(const int64_t* pix_to_face, const float* bary, int64_t npix, int32_t K,
                       const int64_t* faces, int64_t F, const float* points, const float* normals,
                       const float* albedo, int64_t V, const float* params, const float* grad_colors,
                       float* grad_points, float* grad_normals, float* grad_albedo, float* grad_bary,
                       void* stream);

/*
 * Point clouds ("Accelerating 3D Deep Learning with PyTorch3D": the renderer draws point
 * clouds with the same two stages, over heterogeneous batches; the pages print no formula,
 * so these are the plain definitions that match the mesh path).  points: P x 3 float32
 * (device), screen space (x_ndc, y_ndc, z) like the mesh vertices; cloud n is points
 * [cloud_first_idx[n], + num_points_per_cloud[n]) (arrays of N in host or device memory, ascending, disjoint)
 * and is drawn into image n.  Pixel centres as for meshes.
 *
 * mr_rasterize_points_fwd: per pixel the K points of its cloud nearest in depth among those
 *   with z >= 0 and squared 2-D distance to the pixel centre <= radius^2, ordered by
 *   (z, point id): idx (global point id, int64), zbuf (= z), dists (squared distance), all
 *   N x H x W x K, -1 in empty slots.  Bins points into 16 x 16-pixel tiles; performs one
 *   stream synchronisation (the bin list's size, read back through the same mapped host
 *   word as mr_rasterize_fwd's).  MR_ERR_ARG also when the bin list would
 *   exceed 2^31 entries (a radius far larger than the image).
 * mr_rasterize_points_bwd: grad_points (P x 3, overwritten) from grad_zbuf and grad_dists
 *   (each nullable): d dists / d (x, y) = -2 (pixel centre - (x, y)), d zbuf / d z = 1.
 * mr_composite_points_fwd: features (P x C float32) composited over each pixel's K slots
 *   with a_k = 1 - dists_k / radius^2 into out (npix x C): mode 0 front-to-back alpha,
 *   out = sum_k a_k T_k f_k with T_k = prod_{j<k} (1 - a_j); mode 1 norm-weighted,
 *   out = sum_k a_k f_k / max(sum_k a_k, 1e-4).  radius > 0.
 * mr_composite_points_bwd: grad_features (P x C, overwritten; float32 atomics) and
 *   grad_dists (npix x K, nullable; 0 in empty slots) from grad_out (npix x C).
 * Out-of-range point ids in idx are flagged in the device error word and skipped.
 */
int mr_rasterize_points_fwd(const float* points, int64_t P, const int64_t* cloud_first_idx,
                            const int64_t* num_points_per_cloud, int32_t N, int32_t H, int32_t W,
                            float radius, int32_t K, int64_t* idx, float* zbuf, float* dists,
                            void* stream);
int mr_rasterize_points_bwd(const float* points, int64_t P, const int64_t* idx, int32_t N, int32_t H,
                            int32_t W, int32_t K, const float* grad_zbuf, const float* grad_dists,
                            float* grad_points, void* stream);
int mr_composite_points_fwd(const int64_t* idx, const float* dists, int64_t npix, int32_t K,
                            const float* features, int64_t P, int32_t C, float radius, int32_t mode,
                            float* out, void* stream);
int mr_composite_points_bwd(const int64_t* idx, const float* dists, int64_t npix, int32_t K,
                            const float* features, int64_t P, int32_t C, float radius, int32_t mode,
                            const float* grad_out, float* grad_features, float* grad_dists,
                            void* stream);

/*
 * Batched K nearest neighbours (PyTorch3D paper: a custom KNN kernel for heterogeneous
 * batches of point clouds).  p1: P1 x D queries, p2: P2 x D references (float32, device);
 * cloud n of p1 (first1[n], num1[n]) searches cloud n of p2 (first2[n], num2[n]); all four
 * in host or device memory.  mr_knn_fwd: idx (P1 x K int64: global ids into p2) and dists (P1 x K float32:
 * squared Euclidean distances), the K nearest ordered by (distance, id); when cloud n of
 * p2 has fewer than K points the rest hold -1 in both; queries in no cloud get -1 rows.
 * 1 <= D <= MR_KNN_DMAX, 1 <= K <= MR_KMAX, P1, P2 < 2^31; MR_ERR_ARG for overlapping query
 * clouds or a range outside its set.  Exact (every reference of the cloud is either tested
 * or bounded away by the box of its group); allocates scratch of about 24 bytes per point
 * of each set, stream-ordered.
 * mr_knn_bwd: grad_p1 (P1 x D) and grad_p2 (P2 x D), both overwritten (float32 atomics into
 * grad_p2), from grad_dists (P1 x K): d dist / d q = 2 (q - r), d dist / d r = -2 (q - r).
 */
#define MR_KNN_DMAX 4
int mr_knn_fwd(const float* p1, int64_t P1, const int64_t* first1, const int64_t* num1, const float* p2,
               int64_t P2, const int64_t* first2, const int64_t* num2, int32_t N, int32_t D, int32_t K,
               int64_t* idx, float* dists, void* stream);
int mr_knn_bwd(const float* p1, int64_t P1, const float* p2, int64_t P2, int32_t D, int32_t K,
               const int64_t* idx, const float* grad_dists, float* grad_p1, float* grad_p2, void* stream);

/*
 * Work count of the KNN search (measurement support; no counterpart on the pages): runs
 * mr_knn_fwd's search (same arguments, same outputs) in a counting build of its kernel and
 * writes to *evaluated_pairs (HOST) the number of (query, reference) pairs whose distance
 * the search evaluated -- the pairs of every group staged for a warp times its live
 * queries; the groups bounded away by their boxes are not counted.  This is the work the
 * KNN roofline divides by; the search is exact, so the count is at most sum_n num1 * num2
 * and usually far below it.  Synchronises `stream`.
 */
int mr_knn_count_pairs(const float* p1, int64_t P1, const int64_t* first1, const int64_t* num1,
                       const float* p2, int64_t P2, const int64_t* first2, const int64_t* num2,
                       int32_t N, int32_t D, int32_t K, int64_t* idx, float* dists,
                       int64_t* evaluated_pairs, void* stream);

/* Synchronises `stream`, then returns MR_ERR_DEVICE (and clears the word) if any
 * asynchronous kernel of this library flagged an out-of-range index on the current
 * device since the last call, else MR_OK (or MR_ERR_CUDA). */
int mr_device_status(void* stream);

/* Thread-local, NUL-terminated message for the last non-zero return ("" if none). */
const char* mr_last_error(void);

/* Library version as 10000 * major + 100 * minor + patch. */
int mr_version(void);

/*
 * Host-side fault injection, for testing callers' and the library's error paths (no
 * counterpart on the pages).  kind = MR_INJECT_OOM or MR_INJECT_CUDA arms a one-shot
 * failure of the library's scratch allocator: the first `skip` allocations after this call
 * succeed, the next one returns MR_ERR_OOM or MR_ERR_CUDA (the message says "injected")
 * without allocating, and the hook disarms itself.  The entry point that meets it frees any
 * scratch it already holds and returns that code; nothing fails on the GPU.  MR_INJECT_OFF
 * disarms.  Process-wide (all threads and devices).  MR_ERR_ARG for another kind or skip < 0.
 */
#define MR_INJECT_OFF 0
#define MR_INJECT_OOM 1
#define MR_INJECT_CUDA 2
int mr_inject_fault(int32_t kind, int32_t skip);

/*
 * Bytes currently allocated from the current device's default memory pool (its
 * used-memory counter), where the library's scratch comes from; *bytes is HOST.  The
 * scratch of a call is released in stream order, so read this after synchronising the
 * call's stream.  For tests of the library's cleanup.
 */
int mr_scratch_in_use(int64_t* bytes);

/*
 * High-water mark of the bytes allocated from the current device's default memory pool
 * since it was last reset (the peak of the library's scratch, and of anything else the
 * process takes from that pool); *bytes is HOST.  reset != 0 clears the mark after reading
 * it (CUDA resets it to zero; it then follows the allocations made from then on).  For
 * memory measurements (the pages compare renderers'
 * memory; no other counterpart there).
 */
int mr_scratch_peak(int64_t* bytes, int32_t reset);

/*
 * FP32 issue-rate probe (measurement support; no counterpart on the pages): times five
 * launches (after a warm-up) of a kernel of independent FFMA chains filling every SM
 * (8 chains per thread, 148 x 8 CTAs of 256 threads on B200, ~11 ms each) with CUDA events
 * on `stream` and writes the FP32 instructions per second of the fastest launch to
 * *inst_per_s (HOST).  Synchronises `stream`; takes about 70 ms.  The roofline
 * of the fine pass divides by this measured figure rather than by unit counts x clock.
 */
int mr_measure_fp32_peak(double* inst_per_s, void* stream);

/*
 * Stage timing (the library's own tracing; no counterpart on the pages).  While enabled,
 * every launch of the stages below is bracketed by two CUDA events recorded on the
 * caller's stream; recording adds no synchronisation.  Independently of this switch, the
 * host-side enqueue of each stage is an NVTX range named "mr:<stage>" (free unless a
 * tracing tool is attached).  mr_profile_read() waits for the
 * recorded events, writes the summed milliseconds and launch counts per stage into
 * stage_ms[0..nstages) and launches[0..nstages) (either may be NULL), and forgets them.
 * Process-wide; intended for one device and one thread at a time.
 */
#define MR_STAGE_FACE_SETUP 0
#define MR_STAGE_BIN_COUNT 1
#define MR_STAGE_BIN_SCAN 2
#define MR_STAGE_BIN_FILL 3
#define MR_STAGE_FINE 4
#define MR_STAGE_SILHOUETTE_FWD 5
#define MR_STAGE_SILHOUETTE_BWD 6
#define MR_STAGE_RASTER_BWD 7
#define MR_STAGE_SILHOUETTE_RASTER_BWD 8
#define MR_STAGE_EPILOGUE 9
#define MR_STAGE_INTERPOLATE_FWD 10
#define MR_STAGE_INTERPOLATE_BWD 11
#define MR_STAGE_BLEND_FWD 12
#define MR_STAGE_BLEND_BWD 13
#define MR_STAGE_PHONG_FWD 14
#define MR_STAGE_PHONG_BWD 15
#define MR_STAGE_PHONG_SHADE_FWD 16
#define MR_STAGE_PHONG_SHADE_BWD 17
#define MR_STAGE_POINTS_BIN 18
#define MR_STAGE_POINTS_FINE 19
#define MR_STAGE_POINTS_BWD 20
#define MR_STAGE_COMPOSITE_FWD 21
#define MR_STAGE_COMPOSITE_BWD 22
#define MR_STAGE_KNN 23
#define MR_STAGE_KNN_BWD 24
#define MR_NUM_STAGES 25
int mr_profile_enable(int32_t on);
int mr_profile_read(double* stage_ms, int64_t* launches, int32_t nstages);

#ifdef __cplusplus
}
#endif

#endif /* MESHRAST_H */
