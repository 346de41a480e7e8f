/*
 * oracle.c -- plain, slow float64 CPU oracle of the mesh rasterizer hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header, table or helper
 * with the CUDA library; the two meet only through seeded inputs.
 *
 * What it computes (PyTorch3D paper, "Accelerating 3D Deep Learning with PyTorch3D",
 * method summary: two-stage rasterization that keeps, for every pixel, the K nearest
 * faces, then a second stage that blends their influence; tutorial summary, 32:56:
 * the perspective_correct switch).  The pages give the concept only; the formulas are
 * the textbook ones, written out below step by step:
 *
 *   1. pixel centre p = (-1 + (2j+1)/W, 1 - (2i+1)/H); +x right, +y up, row 0 at top.
 *   2. a, b, c = the face's three screen-space vertices (x, y, z).
 *      A = cross(b - a, c - a); a face with |A| <= 1e-12 is skipped (degenerate).
 *   3. w0 = cross(b - p, c - p) / A, w1 = cross(c - p, a - p) / A,
 *      w2 = cross(a - p, b - p) / A (each evaluated directly; no back-face culling).
 *   4. inside = w0 >= 0 and w1 >= 0 and w2 >= 0 (closed triangle).
 *   5. d2 = min over edges (a,b), (b,c), (c,a) of the squared distance from p to the
 *      segment; the first minimal edge in that order wins a tie.
 *   6. the face is a candidate iff inside or d2 <= blur_radius (squared NDC units).
 *   7. barycentrics: perspective-correct -> u_k = w_k / z_k, bary_k = u_k / sum(u);
 *      otherwise bary_k = w_k.  Never clipped, so they sum to 1.
 *   8. z = sum bary_k z_k; a candidate with z < 0 is skipped (behind the camera).
 *   9. dist = -d2 inside, +d2 outside.
 *  10. candidates sorted by (z, face id); the first K kept; empty slots hold -1 in
 *      pix_to_face, zbuf, bary and dists.
 *  11. silhouette: p_k = 1 / (1 + exp(dist_k / sigma)) over valid slots,
 *      alpha = 1 - prod_k (1 - p_k).
 *  12. its gradient: dL/ddist_k = -dL/dalpha * prod_{j != k} (1 - p_j) * p_k (1 - p_k) / sigma.
 *  13. rasterizer backward: the chain rule through steps 3, 5, 7, 8 and 9 with the
 *      candidate set, the inside flag and the nearest edge held fixed.
 *  14-21. stage-two shading (attribute interpolation, soft RGB blend, Phong lighting)
 *      and their gradients; see the two sections at the end of this file.
 *
 * Besides the outputs, the forward marks pixels whose integer result is decided by a
 * float64-vs-float32 rounding: (E1) two of the K+1 nearest candidates lie within 1e-6
 * in depth; (E2) a face whose candidacy is within a margin of its threshold
 * (|d2 - blur| < 1e-5 blur, or min w within 1e-6 of 0 when blur is 0) would rank among
 * the first K.  The margins are tens of times the float32 error of evaluating d2 and w
 * in bin-local coordinates.  These flags only steer the comparison; they change nothing.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define DEGENERATE_AREA 1e-12
#define TIE_DEPTH 1e-6
#define MARGIN_W 1e-6       /* E2 margin on min w when blur_radius is 0 */
#define MARGIN_BLUR 1e-5    /* E2 margin on |d2 - blur| relative to blur */

typedef struct { double x, y, z; } vtx;

/* Everything step 2..9 yields for one (pixel, face) pair. */
typedef struct {
    int degenerate;    /* step 2 */
    int inside;        /* step 4 */
    int edge;          /* argmin edge of step 5: 0 = (a,b), 1 = (b,c), 2 = (c,a) */
    double t;          /* segment parameter of the nearest point on that edge */
    double d2;         /* step 5 */
    double w[3];       /* step 3 */
    double bary[3];    /* step 7 */
    double z;          /* step 8 */
    double dist;       /* step 9 */
} pf_eval;

static double cross2(double ux, double uy, double vx, double vy) { return ux * vy - uy * vx; }

static void face_vertices(const float *verts, const int64_t *faces, int64_t f, vtx v[3]) {
    for (int k = 0; k < 3; ++k) {
        int64_t vi = faces[3 * f + k];
        v[k].x = (double)verts[3 * vi + 0];
        v[k].y = (double)verts[3 * vi + 1];
        v[k].z = (double)verts[3 * vi + 2];
    }
}

/* Squared distance from (px,py) to segment u->v, with the clamped parameter t. */
static double segment_dist2(double px, double py, vtx u, vtx v, double *t_out) {
    double ex = v.x - u.x, ey = v.y - u.y;
    double len2 = ex * ex + ey * ey;
    double t = 0.0;
    if (len2 > 0.0) t = ((px - u.x) * ex + (py - u.y) * ey) / len2;
    if (t < 0.0) t = 0.0;
    if (t > 1.0) t = 1.0;
    double qx = u.x + t * ex, qy = u.y + t * ey;
    *t_out = t;
    return (px - qx) * (px - qx) + (py - qy) * (py - qy);
}

/* Steps 2..9 for pixel centre (px, py) and face vertices v[0..2] = a, b, c. */
static void evaluate(double px, double py, const vtx v[3], int persp, pf_eval *r) {
    const vtx a = v[0], b = v[1], c = v[2];
    memset(r, 0, sizeof(*r));
    double A = cross2(b.x - a.x, b.y - a.y, c.x - a.x, c.y - a.y);
    if (fabs(A) <= DEGENERATE_AREA) { r->degenerate = 1; return; }
    r->w[0] = cross2(b.x - px, b.y - py, c.x - px, c.y - py) / A;
    r->w[1] = cross2(c.x - px, c.y - py, a.x - px, a.y - py) / A;
    r->w[2] = cross2(a.x - px, a.y - py, b.x - px, b.y - py) / A;
    r->inside = r->w[0] >= 0.0 && r->w[1] >= 0.0 && r->w[2] >= 0.0;
    double t;
    r->d2 = segment_dist2(px, py, a, b, &t); r->edge = 0; r->t = t;
    double d = segment_dist2(px, py, b, c, &t);
    if (d < r->d2) { r->d2 = d; r->edge = 1; r->t = t; }
    d = segment_dist2(px, py, c, a, &t);
    if (d < r->d2) { r->d2 = d; r->edge = 2; r->t = t; }
    if (persp) {
        double u0 = r->w[0] / a.z, u1 = r->w[1] / b.z, u2 = r->w[2] / c.z;
        double s = u0 + u1 + u2;
        r->bary[0] = u0 / s; r->bary[1] = u1 / s; r->bary[2] = u2 / s;
    } else {
        r->bary[0] = r->w[0]; r->bary[1] = r->w[1]; r->bary[2] = r->w[2];
    }
    r->z = r->bary[0] * a.z + r->bary[1] * b.z + r->bary[2] * c.z;
    r->dist = r->inside ? -r->d2 : r->d2;
}

static int is_candidate(const pf_eval *r, double blur) {
    if (r->degenerate) return 0;
    if (!(r->inside || r->d2 <= blur)) return 0;   /* step 6 */
    if (r->z < 0.0) return 0;                      /* step 8 */
    return 1;
}

/* (z, face id) lexicographic order of step 10. */
static int before(double z1, int64_t f1, double z2, int64_t f2) {
    return z1 < z2 || (z1 == z2 && f1 < f2);
}

/* ------------------------------------------------------------------ forward */
typedef struct {
    const float *verts; const int64_t *faces; const int64_t *first; const int64_t *num;
    int32_t N, H, W, K, persp; double blur;
    const int64_t *pixels; int64_t npix;
    int64_t *p2f; double *zbuf, *bary, *dists; uint8_t *exempt;
    int64_t next; pthread_mutex_t lock;
} fwd_job;

typedef struct { double z; int64_t f; } zf;

static void rasterize_pixel(fwd_job *J, int64_t pix_id, int64_t out_slot, zf *list) {
    const int32_t H = J->H, W = J->W, K = J->K;
    int64_t n = pix_id / ((int64_t)H * W);
    int64_t rem = pix_id % ((int64_t)H * W);
    int i = (int)(rem / W), j = (int)(rem % W);
    double px = -1.0 + (2.0 * j + 1.0) / W;     /* step 1 */
    double py = 1.0 - (2.0 * i + 1.0) / H;
    /* a face farther than sqrt(blur) from p along x or y can be neither inside nor
     * within the blur radius: the reject below is exact (margin 1e-9 for sqrt rounding). */
    double reach = sqrt(J->blur) + 1e-9;
    int kept = 0, cap = K + 1;                   /* K+1 nearest, for the E1 check */
    int64_t f0 = J->first[n], f1 = J->first[n] + J->num[n];
    for (int64_t f = f0; f < f1; ++f) {
        vtx v[3];
        face_vertices(J->verts, J->faces, f, v);
        double xmin = fmin(v[0].x, fmin(v[1].x, v[2].x)), xmax = fmax(v[0].x, fmax(v[1].x, v[2].x));
        double ymin = fmin(v[0].y, fmin(v[1].y, v[2].y)), ymax = fmax(v[0].y, fmax(v[1].y, v[2].y));
        if (px < xmin - reach || px > xmax + reach || py < ymin - reach || py > ymax + reach) continue;
        pf_eval r;
        evaluate(px, py, v, J->persp, &r);
        if (!is_candidate(&r, J->blur)) continue;
        /* insert (z, f) into the sorted list of at most K+1 entries */
        int pos = kept;
        while (pos > 0 && before(r.z, f, list[pos - 1].z, list[pos - 1].f)) --pos;
        if (pos >= cap) continue;
        int last = kept < cap ? kept : cap - 1;
        for (int q = last; q > pos; --q) list[q] = list[q - 1];
        list[pos].z = r.z; list[pos].f = f;
        if (kept < cap) ++kept;
    }
    /* outputs: the first K entries */
    for (int k = 0; k < K; ++k) {
        int64_t s = out_slot * K + k;
        if (k < kept) {
            vtx v[3];
            pf_eval r;
            face_vertices(J->verts, J->faces, list[k].f, v);
            evaluate(px, py, v, J->persp, &r);
            J->p2f[s] = list[k].f;
            J->zbuf[s] = r.z;
            J->bary[3 * s + 0] = r.bary[0]; J->bary[3 * s + 1] = r.bary[1]; J->bary[3 * s + 2] = r.bary[2];
            J->dists[s] = r.dist;
        } else {
            J->p2f[s] = -1;
            J->zbuf[s] = -1.0;
            J->bary[3 * s + 0] = J->bary[3 * s + 1] = J->bary[3 * s + 2] = -1.0;
            J->dists[s] = -1.0;
        }
    }
    if (!J->exempt) return;
    uint8_t ex = 0;
    /* E1: a depth near-tie among the K+1 nearest (the list is sorted) */
    for (int k = 0; k + 1 < kept; ++k)
        if (list[k + 1].z - list[k].z < TIE_DEPTH) ex |= 1;
    /* E2: a face whose candidacy sits on its threshold and that would rank in the first K */
    for (int64_t f = f0; f < f1; ++f) {
        vtx v[3];
        face_vertices(J->verts, J->faces, f, v);
        double xmin = fmin(v[0].x, fmin(v[1].x, v[2].x)), xmax = fmax(v[0].x, fmax(v[1].x, v[2].x));
        double ymin = fmin(v[0].y, fmin(v[1].y, v[2].y)), ymax = fmax(v[0].y, fmax(v[1].y, v[2].y));
        double reach2 = reach + 1e-3;
        if (px < xmin - reach2 || px > xmax + reach2 || py < ymin - reach2 || py > ymax + reach2) continue;
        pf_eval r;
        evaluate(px, py, v, J->persp, &r);
        if (r.degenerate) continue;
        int marginal;
        if (J->blur > 0.0) {
            marginal = !r.inside && fabs(r.d2 - J->blur) < MARGIN_BLUR * J->blur;
        } else {
            double wmin = fmin(r.w[0], fmin(r.w[1], r.w[2]));
            marginal = wmin > -MARGIN_W && wmin < MARGIN_W;
        }
        if (!marginal || r.z < 0.0) continue;
        int ahead = 0;
        for (int k = 0; k < kept; ++k)
            if (list[k].f != f && before(list[k].z, list[k].f, r.z, f)) ++ahead;
        if (ahead < K) ex |= 2;
    }
    J->exempt[out_slot] = ex;
}

static void *fwd_worker(void *arg) {
    fwd_job *J = (fwd_job *)arg;
    int64_t total = J->pixels ? J->npix : (int64_t)J->N * J->H * J->W;
    zf *list = (zf *)malloc(sizeof(zf) * (size_t)(J->K + 2));
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t start = J->next;
        J->next += 64;
        pthread_mutex_unlock(&J->lock);
        if (start >= total) break;
        int64_t end = start + 64 < total ? start + 64 : total;
        for (int64_t s = start; s < end; ++s)
            rasterize_pixel(J, J->pixels ? J->pixels[s] : s, s, list);
    }
    free(list);
    return NULL;
}

static void run_threads(void *(*fn)(void *), void *job, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, fn, job);
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
}

/* Forward over all N*H*W pixels (pixels == NULL) or over the listed pixel ids
 * (id = (n*H + i)*W + j); outputs are then P x K, in list order.  Returns 0, or -1 on
 * invalid arguments. */
int oracle_rasterize_fwd(const float *verts, int64_t V, const int64_t *faces, int64_t F,
                         const int64_t *first, const int64_t *num, int32_t N, int32_t H, int32_t W,
                         double blur, int32_t K, int32_t persp, const int64_t *pixels, int64_t npix,
                         int64_t *p2f, double *zbuf, double *bary, double *dists, uint8_t *exempt,
                         int32_t nthreads) {
    if (N < 0 || H <= 0 || W <= 0 || K <= 0 || !(blur >= 0.0)) return -1;
    for (int32_t n = 0; n < N; ++n)
        if (first[n] < 0 || num[n] < 0 || first[n] + num[n] > F) return -1;
    for (int64_t q = 0; q < 3 * F; ++q)
        if (faces[q] < 0 || faces[q] >= V) return -1;
    fwd_job J;
    memset(&J, 0, sizeof(J));
    J.verts = verts; J.faces = faces; J.first = first; J.num = num;
    J.N = N; J.H = H; J.W = W; J.K = K; J.persp = persp; J.blur = blur;
    J.pixels = pixels; J.npix = npix;
    J.p2f = p2f; J.zbuf = zbuf; J.bary = bary; J.dists = dists; J.exempt = exempt;
    pthread_mutex_init(&J.lock, NULL);
    run_threads(fwd_worker, &J, nthreads);
    pthread_mutex_destroy(&J.lock);
    return 0;
}

/* ------------------------------------------------------------------ silhouette */
/* Step 11 over npix pixels of K slots each. */
void oracle_silhouette_fwd(const int64_t *p2f, const double *dists, int64_t npix, int32_t K,
                           double sigma, double *alpha) {
    for (int64_t q = 0; q < npix; ++q) {
        double keep = 1.0;   /* prod (1 - p_k) */
        for (int k = 0; k < K; ++k) {
            int64_t s = q * K + k;
            if (p2f[s] < 0) continue;
            double p = 1.0 / (1.0 + exp(dists[s] / sigma));
            keep *= 1.0 - p;
        }
        alpha[q] = 1.0 - keep;
    }
}

/* Step 12: the product over j != k is formed directly (no division). */
void oracle_silhouette_bwd(const double *grad_alpha, const int64_t *p2f, const double *dists,
                           int64_t npix, int32_t K, double sigma, double *grad_dists) {
    for (int64_t q = 0; q < npix; ++q) {
        for (int k = 0; k < K; ++k) {
            int64_t s = q * K + k;
            if (p2f[s] < 0) { grad_dists[s] = 0.0; continue; }
            double others = 1.0;
            for (int j = 0; j < K; ++j) {
                int64_t sj = q * K + j;
                if (j == k || p2f[sj] < 0) continue;
                others *= 1.0 - 1.0 / (1.0 + exp(dists[sj] / sigma));
            }
            double p = 1.0 / (1.0 + exp(dists[s] / sigma));
            grad_dists[s] = -grad_alpha[q] * others * p * (1.0 - p) / sigma;
        }
    }
}

/* ------------------------------------------------------------------ backward */
/*
 * Derivatives used below (v = a, b, c is vertex 0, 1, 2; only x, y enter steps 3 and 5):
 *   C_k = cross(V1 - p, V2 - p) for (V1, V2) = (b, c), (c, a), (a, b);  w_k = C_k / A.
 *   d cross(U - p, V - p) / dU = (V.y - p.y, -(V.x - p.x)),  / dV = (-(U.y - p.y), U.x - p.x).
 *   d A / db = (c.y - a.y, -(c.x - a.x)),  d A / dc = (-(b.y - a.y), b.x - a.x),
 *   d A / da = -(dA/db + dA/dc).
 *   d w_k = (d C_k - w_k d A) / A.
 *   Perspective: u_k = w_k / z_k, s = sum u, bary_k = u_k / s, z = 1 / s, so
 *     d bary_m / d u_k = (delta_mk - bary_m) / s,  d z / d u_k = -z^2,
 *     d u_k / d w_k = 1 / z_k,  d u_k / d z_k = -u_k / z_k.
 *   Plain: bary_k = w_k, z = sum w_k z_k, so d z / d w_k = z_k and d z / d z_k = w_k.
 *   Distance to the nearest edge u->v with nearest point q = u + t (v - u):
 *     d d2 / du = -2 (p - q)(1 - t),  d d2 / dv = -2 (p - q) t;  dist = +-d2.
 */
typedef struct {
    const float *verts; const int64_t *faces; const int64_t *p2f;
    int32_t N, H, W, K, persp;
    const double *gz, *gb, *gd;
    double **partial; int64_t V;
    int64_t next; pthread_mutex_t lock; int nthreads; int tid_next;
} bwd_job;

static void accumulate_slot(bwd_job *J, int64_t slot, double *g) {
    int64_t f = J->p2f[slot];
    if (f < 0) return;
    int64_t pix = slot / J->K;
    int64_t rem = pix % ((int64_t)J->H * J->W);
    int i = (int)(rem / J->W), j = (int)(rem % J->W);
    double px = -1.0 + (2.0 * j + 1.0) / J->W;
    double py = 1.0 - (2.0 * i + 1.0) / J->H;
    vtx v[3];
    face_vertices(J->verts, J->faces, f, v);
    pf_eval r;
    evaluate(px, py, v, J->persp, &r);
    if (r.degenerate) return;
    int64_t vid[3] = {J->faces[3 * f], J->faces[3 * f + 1], J->faces[3 * f + 2]};

    /* dists -> the two end points of the nearest edge (x, y) */
    if (J->gd) {
        double gdist = J->gd[slot] * (r.inside ? -1.0 : 1.0);
        int u = r.edge, w = (r.edge + 1) % 3;
        double qx = v[u].x + r.t * (v[w].x - v[u].x), qy = v[u].y + r.t * (v[w].y - v[u].y);
        double rx = px - qx, ry = py - qy;
        g[3 * vid[u] + 0] += gdist * (-2.0 * rx * (1.0 - r.t));
        g[3 * vid[u] + 1] += gdist * (-2.0 * ry * (1.0 - r.t));
        g[3 * vid[w] + 0] += gdist * (-2.0 * rx * r.t);
        g[3 * vid[w] + 1] += gdist * (-2.0 * ry * r.t);
    }
    if (!J->gb && !J->gz) return;

    double gbary[3] = {0, 0, 0}, gzb = 0.0;
    if (J->gb) for (int m = 0; m < 3; ++m) gbary[m] = J->gb[3 * slot + m];
    if (J->gz) gzb = J->gz[slot];
    double gw[3], gzc[3];    /* dL/dw_k and dL/dz_k (vertex depth) */
    if (J->persp) {
        double u[3], s = 0.0;
        for (int k = 0; k < 3; ++k) { u[k] = r.w[k] / v[k].z; s += u[k]; }
        for (int k = 0; k < 3; ++k) {
            double gu = 0.0;
            for (int m = 0; m < 3; ++m) gu += gbary[m] * (((m == k) ? 1.0 : 0.0) - r.bary[m]) / s;
            gu += gzb * (-r.z * r.z);
            gw[k] = gu / v[k].z;
            gzc[k] = gu * (-u[k] / v[k].z);
        }
    } else {
        for (int k = 0; k < 3; ++k) { gw[k] = gbary[k] + gzb * v[k].z; gzc[k] = gzb * r.w[k]; }
    }
    /* d w_k / d (vertex x, y) */
    const vtx a = v[0], b = v[1], c = v[2];
    double A = cross2(b.x - a.x, b.y - a.y, c.x - a.x, c.y - a.y);
    double dA[3][2] = {{b.y - c.y, c.x - b.x}, {c.y - a.y, -(c.x - a.x)}, {-(b.y - a.y), b.x - a.x}};
    double dC[3][3][2];  /* dC[k][vertex][xy] */
    memset(dC, 0, sizeof(dC));
    int pairs[3][2] = {{1, 2}, {2, 0}, {0, 1}};
    for (int k = 0; k < 3; ++k) {
        int U = pairs[k][0], W2 = pairs[k][1];
        dC[k][U][0] = v[W2].y - py;   dC[k][U][1] = -(v[W2].x - px);
        dC[k][W2][0] = -(v[U].y - py); dC[k][W2][1] = v[U].x - px;
    }
    for (int k = 0; k < 3; ++k)
        for (int q = 0; q < 3; ++q)
            for (int e = 0; e < 2; ++e)
                g[3 * vid[q] + e] += gw[k] * (dC[k][q][e] - r.w[k] * dA[q][e]) / A;
    for (int k = 0; k < 3; ++k) g[3 * vid[k] + 2] += gzc[k];
}

static void *bwd_worker(void *arg) {
    bwd_job *J = (bwd_job *)arg;
    pthread_mutex_lock(&J->lock);
    int tid = J->tid_next++;
    pthread_mutex_unlock(&J->lock);
    double *g = J->partial[tid];
    int64_t total = (int64_t)J->N * J->H * J->W * J->K;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t start = J->next;
        J->next += 4096;
        pthread_mutex_unlock(&J->lock);
        if (start >= total) break;
        int64_t end = start + 4096 < total ? start + 4096 : total;
        for (int64_t s = start; s < end; ++s) accumulate_slot(J, s, g);
    }
    return NULL;
}

/* Step 13 over all N*H*W*K slots.  grad_* may be NULL (no gradient from that output).
 * grad_verts (V x 3) is overwritten.  Returns 0, or -1 on invalid arguments. */
int oracle_rasterize_bwd(const float *verts, int64_t V, const int64_t *faces, int64_t F,
                         const int64_t *p2f, int32_t N, int32_t H, int32_t W, int32_t K, int32_t persp,
                         const double *grad_zbuf, const double *grad_bary, const double *grad_dists,
                         double *grad_verts, int32_t nthreads) {
    if (N < 0 || H <= 0 || W <= 0 || K <= 0) return -1;
    int64_t slots = (int64_t)N * H * W * K;
    for (int64_t s = 0; s < slots; ++s) if (p2f[s] >= F) return -1;
    for (int64_t q = 0; q < 3 * F; ++q) if (faces[q] < 0 || faces[q] >= V) return -1;
    if (nthreads < 1) nthreads = 1;
    bwd_job J;
    memset(&J, 0, sizeof(J));
    J.verts = verts; J.faces = faces; J.p2f = p2f;
    J.N = N; J.H = H; J.W = W; J.K = K; J.persp = persp;
    J.gz = grad_zbuf; J.gb = grad_bary; J.gd = grad_dists; J.V = V;
    J.nthreads = nthreads;
    J.partial = (double **)malloc(sizeof(double *) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) J.partial[t] = (double *)calloc((size_t)(3 * V), sizeof(double));
    pthread_mutex_init(&J.lock, NULL);
    run_threads(bwd_worker, &J, nthreads);
    pthread_mutex_destroy(&J.lock);
    for (int64_t q = 0; q < 3 * V; ++q) {
        double s = 0.0;
        for (int t = 0; t < nthreads; ++t) s += J.partial[t][q];
        grad_verts[q] = s;
    }
    for (int t = 0; t < nthreads; ++t) free(J.partial[t]);
    free(J.partial);
    return 0;
}

/* Per-(pixel, face) probe for tests: steps 2..9 for one pixel centre and one face. */
void oracle_probe(double px, double py, const double *abc /* 9: a, b, c as x,y,z */, int32_t persp,
                  double *out /* 13 values, listed below */) {
    vtx v[3];
    for (int k = 0; k < 3; ++k) { v[k].x = abc[3 * k]; v[k].y = abc[3 * k + 1]; v[k].z = abc[3 * k + 2]; }
    pf_eval r;
    evaluate(px, py, v, persp, &r);
    /* out: [degenerate, inside, edge, t, d2, w0, w1, w2, b0, b1, b2, z, dist] */
    out[0] = r.degenerate; out[1] = r.inside; out[2] = r.edge; out[3] = r.t; out[4] = r.d2;
    out[5] = r.w[0]; out[6] = r.w[1]; out[7] = r.w[2];
    out[8] = r.bary[0]; out[9] = r.bary[1]; out[10] = r.bary[2]; out[11] = r.z; out[12] = r.dist;
}

/* ------------------------------------------------------------------ stage two: shading */
/*
 * Gouraud shading and the soft RGB blend (PyTorch3D paper, method: pluggable Gouraud and
 * Phong shaders over the K faces kept per pixel; the soft aggregation is SoftRas's, the
 * renderer the paper compares against).  Written out:
 *
 *  14. interpolation: for a valid slot with face f = (v0, v1, v2) and barycentrics b,
 *      out[d] = sum_m b_m attr[v_m][d]; empty slots give 0.
 *  15. its gradient: d attr[v_m][d] += b_m g[d]; d b_m = sum_d attr[v_m][d] g[d].
 *  16. soft RGB blend over the valid slots of a pixel, with colours c_k (D channels),
 *      signed distances d_k and depths z_k:
 *        p_k = 1 / (1 + exp(d_k / sigma))                      coverage weight
 *        s_k = (zfar - z_k) / (zfar - znear)                   normalised nearness
 *        m   = max(max_k s_k, eps)        (eps = 1e-10; shift for stability only)
 *        w_k = p_k exp((s_k - m) / gamma),  w_b = exp((eps - m) / gamma)
 *        rgb = (sum_k w_k c_k + w_b bg) / (sum_k w_k + w_b)
 *        alpha = 1 - prod_k (1 - p_k)
 *  17. its gradient, with m held fixed (rgb does not depend on it):
 *        d c_k = w_k / D g,  d w_k = (c_k - rgb) . g / D,
 *        d d_k = d w_k * w_k * (-(1 - p_k) / sigma) + (alpha part as in step 12),
 *        d z_k = d w_k * w_k * (-1 / (gamma (zfar - znear))).
 */
#define BLEND_EPS 1e-10

/* Step 14 over npix pixels of K slots: attr V x D, bary (npix x K x 3), out npix x K x D. */
void oracle_interpolate_fwd(const int64_t *p2f, const double *bary, int64_t npix, int32_t K,
                            const int64_t *faces, const double *attr, int32_t D, double *out) {
    for (int64_t s = 0; s < npix * K; ++s) {
        int64_t f = p2f[s];
        for (int d = 0; d < D; ++d) {
            double v = 0.0;
            if (f >= 0)
                for (int m = 0; m < 3; ++m) v += bary[3 * s + m] * attr[faces[3 * f + m] * D + d];
            out[s * D + d] = v;
        }
    }
}

/* Step 15: grad_attr (V x D) is overwritten; grad_bary (npix x K x 3) may be NULL. */
void oracle_interpolate_bwd(const int64_t *p2f, const double *bary, int64_t npix, int32_t K,
                            const int64_t *faces, const double *attr, int64_t V, int32_t D,
                            const double *grad_out, double *grad_attr, double *grad_bary) {
    memset(grad_attr, 0, sizeof(double) * (size_t)(V * D));
    for (int64_t s = 0; s < npix * K; ++s) {
        int64_t f = p2f[s];
        for (int m = 0; m < 3; ++m) {
            double gb = 0.0;
            if (f >= 0) {
                int64_t v = faces[3 * f + m];
                for (int d = 0; d < D; ++d) {
                    grad_attr[v * D + d] += bary[3 * s + m] * grad_out[s * D + d];
                    gb += attr[v * D + d] * grad_out[s * D + d];
                }
            }
            if (grad_bary) grad_bary[3 * s + m] = gb;
        }
    }
}

/* Step 16: colors npix x K x D, out rgba npix x (D + 1) (colour channels, then alpha). */
void oracle_blend_fwd(const int64_t *p2f, const double *colors, const double *dists, const double *zbuf,
                      int64_t npix, int32_t K, int32_t D, const double *background, double sigma,
                      double gamma, double znear, double zfar, double *out) {
    for (int64_t q = 0; q < npix; ++q) {
        double m = BLEND_EPS, keep = 1.0;
        for (int k = 0; k < K; ++k) {
            int64_t s = q * K + k;
            if (p2f[s] < 0) continue;
            double sk = (zfar - zbuf[s]) / (zfar - znear);
            if (sk > m) m = sk;
        }
        double den = exp((BLEND_EPS - m) / gamma);
        for (int d = 0; d < D; ++d) out[q * (D + 1) + d] = den * background[d];
        for (int k = 0; k < K; ++k) {
            int64_t s = q * K + k;
            if (p2f[s] < 0) continue;
            double p = 1.0 / (1.0 + exp(dists[s] / sigma));
            double sk = (zfar - zbuf[s]) / (zfar - znear);
            double w = p * exp((sk - m) / gamma);
            den += w;
            for (int d = 0; d < D; ++d) out[q * (D + 1) + d] += w * colors[s * D + d];
            keep *= 1.0 - p;
        }
        for (int d = 0; d < D; ++d) out[q * (D + 1) + d] /= den;
        out[q * (D + 1) + D] = 1.0 - keep;
    }
}

/* Step 17: grad_rgba npix x (D + 1); writes grad_colors (npix x K x D), grad_dists and
 * grad_zbuf (npix x K); any output may be NULL. */
void oracle_blend_bwd(const int64_t *p2f, const double *colors, const double *dists, const double *zbuf,
                      int64_t npix, int32_t K, int32_t D, const double *background, double sigma,
                      double gamma, double znear, double zfar, const double *grad_rgba,
                      double *grad_colors, double *grad_dists, double *grad_zbuf) {
    double *rgb = (double *)malloc(sizeof(double) * (size_t)(D + 1));
    for (int64_t q = 0; q < npix; ++q) {
        oracle_blend_fwd(p2f + q * K, colors + q * K * D, dists + q * K, zbuf + q * K, 1, K, D, background,
                         sigma, gamma, znear, zfar, rgb);
        double m = BLEND_EPS;
        for (int k = 0; k < K; ++k) {
            int64_t s = q * K + k;
            if (p2f[s] < 0) continue;
            double sk = (zfar - zbuf[s]) / (zfar - znear);
            if (sk > m) m = sk;
        }
        double den = exp((BLEND_EPS - m) / gamma);
        for (int k = 0; k < K; ++k) {
            int64_t s = q * K + k;
            if (p2f[s] < 0) continue;
            double p = 1.0 / (1.0 + exp(dists[s] / sigma));
            den += p * exp(((zfar - zbuf[s]) / (zfar - znear) - m) / gamma);
        }
        const double *g = grad_rgba + q * (D + 1);
        for (int k = 0; k < K; ++k) {
            int64_t s = q * K + k;
            if (p2f[s] < 0) {
                if (grad_colors) for (int d = 0; d < D; ++d) grad_colors[s * D + d] = 0.0;
                if (grad_dists) grad_dists[s] = 0.0;
                if (grad_zbuf) grad_zbuf[s] = 0.0;
                continue;
            }
            double p = 1.0 / (1.0 + exp(dists[s] / sigma));
            double w = p * exp(((zfar - zbuf[s]) / (zfar - znear) - m) / gamma);
            double gw = 0.0;
            for (int d = 0; d < D; ++d) {
                if (grad_colors) grad_colors[s * D + d] = w / den * g[d];
                gw += (colors[s * D + d] - rgb[d]) * g[d] / den;
            }
            /* alpha = 1 - prod (1 - p_j): d alpha / d p_k = prod_{j != k} (1 - p_j) */
            double others = 1.0;
            for (int j = 0; j < K; ++j) {
                int64_t sj = q * K + j;
                if (j == k || p2f[sj] < 0) continue;
                others *= 1.0 - 1.0 / (1.0 + exp(dists[sj] / sigma));
            }
            double dp_dd = -p * (1.0 - p) / sigma;
            if (grad_dists) grad_dists[s] = gw * w * (-(1.0 - p) / sigma) + g[D] * others * dp_dd;
            if (grad_zbuf) grad_zbuf[s] = gw * w * (-1.0 / (gamma * (zfar - znear)));
        }
    }
    free(rgb);
}

/* ------------------------------------------------------------------ stage two: Phong lighting */
/*
 * The Phong reflection model (the PyTorch3D paper names Gouraud and Phong shading and
 * several lights and materials but prints no formula; this is the textbook model of
 * Phong 1975 with one point light, written out).  At a surface point P with normal N,
 * albedo c, light position L and camera position C (one params row of 16 numbers:
 * L[3], C[3], ambient[3], diffuse[3], specular[3], shininess; each colour is the
 * product of the light's and the material's colour):
 *
 *  18. n = N / |N|, l = (L - P) / |L - P|, v = (C - P) / |C - P|, cos = n . l,
 *      r = 2 cos n - l (l mirrored about n), rv = r . v,
 *      diffuse term  t_d = max(cos, 0),
 *      specular term t_s = rv^shininess when cos > 0 and rv > 0, else 0,
 *      colour = (ambient + diffuse t_d) * c + specular t_s   (per channel).
 *      Gouraud shading evaluates this at the vertices and interpolates the colours
 *      (step 14); Phong shading interpolates P, N and c per fragment (step 14) and
 *      evaluates it there (step 20).
 *  19. its gradient: the chain rule through step 18 with the two switches (cos > 0,
 *      rv > 0) held; the normalisation x / |x| has Jacobian (I - x^ x^T) / |x|.
 *  20. Phong shading of the K slots of each pixel: step 14 for P, N and c, then step 18;
 *      empty slots give 0.  Its gradient (step 21) is step 19 followed by step 15 for
 *      each of the three attributes; grad_bary sums the three.
 *
 * The specular term jumps where cos crosses 0 while rv > 0, so a point with
 * |cos| < 1e-6 is flagged (its colour is decided by rounding).
 */
#define PHONG_MARGIN 1e-6

typedef struct {
    double n[3], l[3], v[3];
    double ln, lv, lc;           /* |N|, |L - P|, |C - P| */
    double cos, rv, td, ts, nv, lvd;
    int lit, shiny;
} phong_state;

static double dot3(const double *a, const double *b) { return a[0] * b[0] + a[1] * b[1] + a[2] * b[2]; }

static void phong_eval(const double *P, const double *N, const double *prm, phong_state *S) {
    double dl[3], dv[3];
    for (int e = 0; e < 3; ++e) {
        dl[e] = prm[e] - P[e];
        dv[e] = prm[3 + e] - P[e];
    }
    S->ln = sqrt(dot3(N, N));
    S->lv = sqrt(dot3(dl, dl));
    S->lc = sqrt(dot3(dv, dv));
    for (int e = 0; e < 3; ++e) {
        S->n[e] = N[e] / S->ln;
        S->l[e] = dl[e] / S->lv;
        S->v[e] = dv[e] / S->lc;
    }
    S->cos = dot3(S->n, S->l);
    S->nv = dot3(S->n, S->v);
    S->lvd = dot3(S->l, S->v);
    S->rv = 2.0 * S->cos * S->nv - S->lvd;
    S->lit = S->cos > 0.0;
    S->shiny = S->lit && S->rv > 0.0;
    S->td = S->lit ? S->cos : 0.0;
    S->ts = S->shiny ? pow(S->rv, prm[15]) : 0.0;
}

/* Step 18 over M points (each row of P, N, c holds 3 numbers); flags may be NULL. */
void oracle_phong_fwd(const double *P, const double *N, const double *c, int64_t M, const double *prm,
                      double *out, uint8_t *flags) {
    for (int64_t i = 0; i < M; ++i) {
        phong_state S;
        phong_eval(P + 3 * i, N + 3 * i, prm, &S);
        for (int e = 0; e < 3; ++e) out[3 * i + e] = (prm[6 + e] + prm[9 + e] * S.td) * c[3 * i + e] + prm[12 + e] * S.ts;
        if (flags) flags[i] = fabs(S.cos) < PHONG_MARGIN;
    }
}

/* d x^ given d(x^) for x^ = x / |x|: (g - (g . x^) x^) / |x|. */
static void unit_bwd(const double *xh, double len, const double *g, double *gx) {
    double t = dot3(g, xh);
    for (int e = 0; e < 3; ++e) gx[e] = (g[e] - t * xh[e]) / len;
}

/* Step 19 for one point: gP, gN, gc (3 each) from the colour gradient g. */
static void phong_point_bwd(const double *P, const double *N, const double *c, const double *prm, const double *g,
                            double *gP, double *gN, double *gc) {
    phong_state S;
    phong_eval(P, N, prm, &S);
    double g_td = 0.0, g_ts = 0.0;
    for (int e = 0; e < 3; ++e) {
        gc[e] = g[e] * (prm[6 + e] + prm[9 + e] * S.td);
        g_td += g[e] * prm[9 + e] * c[e];
        g_ts += g[e] * prm[12 + e];
    }
    double g_cos = S.lit ? g_td : 0.0;
    double g_rv = S.shiny ? g_ts * prm[15] * pow(S.rv, prm[15] - 1.0) : 0.0;
    /* rv = 2 cos nv - lv */
    g_cos += g_rv * 2.0 * S.nv;
    double g_nv = g_rv * 2.0 * S.cos, g_lv = -g_rv;
    double gn[3], gl[3], gv[3];
    for (int e = 0; e < 3; ++e) {
        gn[e] = g_cos * S.l[e] + g_nv * S.v[e];
        gl[e] = g_cos * S.n[e] + g_lv * S.v[e];
        gv[e] = g_nv * S.n[e] + g_lv * S.l[e];
    }
    double gdl[3], gdv[3];
    unit_bwd(S.n, S.ln, gn, gN);
    unit_bwd(S.l, S.lv, gl, gdl);
    unit_bwd(S.v, S.lc, gv, gdv);
    for (int e = 0; e < 3; ++e) gP[e] = -gdl[e] - gdv[e];
}

/* Step 19 over M points; each output (M x 3) may be NULL. */
void oracle_phong_bwd(const double *P, const double *N, const double *c, int64_t M, const double *prm,
                      const double *grad, double *gP, double *gN, double *gc) {
    for (int64_t i = 0; i < M; ++i) {
        double a[3], b[3], d[3];
        phong_point_bwd(P + 3 * i, N + 3 * i, c + 3 * i, prm, grad + 3 * i, a, b, d);
        for (int e = 0; e < 3; ++e) {
            if (gP) gP[3 * i + e] = a[e];
            if (gN) gN[3 * i + e] = b[e];
            if (gc) gc[3 * i + e] = d[e];
        }
    }
}

/* One slot's interpolated P, N, c (step 14 with D = 3, three times). */
static void slot_attributes(const int64_t *faces, int64_t f, const double *bary, const double *vP, const double *vN,
                            const double *vc, double *P, double *N, double *c) {
    for (int e = 0; e < 3; ++e) P[e] = N[e] = c[e] = 0.0;
    for (int m = 0; m < 3; ++m) {
        int64_t v = faces[3 * f + m];
        for (int e = 0; e < 3; ++e) {
            P[e] += bary[m] * vP[3 * v + e];
            N[e] += bary[m] * vN[3 * v + e];
            c[e] += bary[m] * vc[3 * v + e];
        }
    }
}

/* Step 20: colors (npix x K x 3); flags (npix x K) may be NULL. */
void oracle_phong_shade_fwd(const int64_t *p2f, const double *bary, int64_t npix, int32_t K, const int64_t *faces,
                            const double *vP, const double *vN, const double *vc, const double *prm, double *out,
                            uint8_t *flags) {
    for (int64_t s = 0; s < npix * K; ++s) {
        int64_t f = p2f[s];
        if (flags) flags[s] = 0;
        if (f < 0) {
            out[3 * s] = out[3 * s + 1] = out[3 * s + 2] = 0.0;
            continue;
        }
        double P[3], N[3], c[3];
        slot_attributes(faces, f, bary + 3 * s, vP, vN, vc, P, N, c);
        oracle_phong_fwd(P, N, c, 1, prm, out + 3 * s, flags ? flags + s : NULL);
    }
}

/* Step 21: gradients into the vertex attributes (V x 3 each, overwritten) and grad_bary
 * (npix x K x 3, may be NULL). */
void oracle_phong_shade_bwd(const int64_t *p2f, const double *bary, int64_t npix, int32_t K, const int64_t *faces,
                            const double *vP, const double *vN, const double *vc, int64_t V, const double *prm,
                            const double *grad, double *gvP, double *gvN, double *gvc, double *grad_bary) {
    memset(gvP, 0, sizeof(double) * 3 * (size_t)V);
    memset(gvN, 0, sizeof(double) * 3 * (size_t)V);
    memset(gvc, 0, sizeof(double) * 3 * (size_t)V);
    for (int64_t s = 0; s < npix * K; ++s) {
        int64_t f = p2f[s];
        if (f < 0) {
            if (grad_bary) grad_bary[3 * s] = grad_bary[3 * s + 1] = grad_bary[3 * s + 2] = 0.0;
            continue;
        }
        double P[3], N[3], c[3], gP[3], gN[3], gc[3];
        slot_attributes(faces, f, bary + 3 * s, vP, vN, vc, P, N, c);
        phong_point_bwd(P, N, c, prm, grad + 3 * s, gP, gN, gc);
        for (int m = 0; m < 3; ++m) {
            int64_t v = faces[3 * f + m];
            double b = bary[3 * s + m], gb = 0.0;
            for (int e = 0; e < 3; ++e) {
                gvP[3 * v + e] += b * gP[e];
                gvN[3 * v + e] += b * gN[e];
                gvc[3 * v + e] += b * gc[e];
                gb += vP[3 * v + e] * gP[e] + vN[3 * v + e] * gN[e] + vc[3 * v + e] * gc[e];
            }
            if (grad_bary) grad_bary[3 * s + m] = gb;
        }
    }
}

/* ------------------------------------------------------------------ point clouds */
/*
 * The point-cloud renderer and the batched K-nearest-neighbour search (PyTorch3D paper:
 * the renderer handles point clouds as well as meshes, with the same two stages, and a
 * custom heterogeneous-batch KNN kernel; the pages print no formula, so the definitions
 * below are the plain ones that match the mesh path).  Points are in screen space
 * (x_ndc, y_ndc, z) like the mesh vertices; cloud n is points [first_n, first_n + num_n)
 * and is drawn into image n.
 *
 *  22. point rasterization: pixel centre p as in step 1; point m of cloud n is a
 *      candidate iff z_m >= 0 and d2 = (p_x - x_m)^2 + (p_y - y_m)^2 <= r^2 (r = the
 *      radius in NDC units); candidates sorted by (z, point id), the first K kept:
 *      idx (global point id), zbuf = z_m, dists = d2; empty slots hold -1 in all three.
 *  23. its gradient: d dists / d (x_m, y_m) = -2 (p - (x_m, y_m)); d zbuf / d z_m = 1.
 *  24. alpha compositing over a pixel's valid slots in order, with per-point features
 *      f_m (C channels) and a_k = 1 - dists_k / r^2:
 *        out = sum_k a_k T_k f_{idx_k},  T_k = prod_{j < k} (1 - a_j).
 *  25. norm-weighted compositing: out = sum_k a_k f_{idx_k} / max(sum_k a_k, 1e-4).
 *  26. their gradients into the features and the dists (the products over j != k are
 *      formed directly; no division by 1 - a_k).
 *  27. batched KNN: for query point i of cloud n of the first set (D coordinates each),
 *      the squared Euclidean distance to every point j of cloud n of the second set; the
 *      K smallest, ordered by (distance, j); idx = the global (packed) id of j, dists the
 *      distance; when cloud n of the second set has fewer than K points the rest hold
 *      -1 in both.
 *  28. its gradient: d dist / d q = 2 (q - r_j), d dist / d r_j = -2 (q - r_j).
 *
 * Flags: step 22 marks pixels where a point within a margin of the radius
 * (|d2 - r^2| < 1e-5 r^2) would rank among the first K; step 27 marks queries whose
 * K-th and (K+1)-th distances lie within 1e-6 (relative) of each other, or whose first
 * K contain such a near tie (the order of near-equal distances is decided by rounding).
 */
#define POINT_MARGIN 1e-5
#define KNN_TIE 1e-6
#define NORM_FLOOR 1e-4

typedef struct {
    double key;
    int64_t id;
    double aux;
} kv;

static int kv_before(const kv *a, const kv *b) { return a->key < b->key || (a->key == b->key && a->id < b->id); }

/* insertion into a sorted list of at most cap entries; returns the new length */
static int kv_insert(kv *list, int n, int cap, kv e) {
    int pos = n;
    while (pos > 0 && kv_before(&e, &list[pos - 1])) --pos;
    if (pos >= cap) return n;
    int last = n < cap ? n : cap - 1;
    for (int t = last; t > pos; --t) list[t] = list[t - 1];
    list[pos] = e;
    return n < cap ? n + 1 : n;
}

/* Step 22 at one pixel (image n, row i, column j) into K slots at idx/zbuf/dists + o;
 * returns the flag.  list: K scratch entries. */
static int point_pixel(const float *pts, int64_t P, const int64_t *first, const int64_t *num, int32_t n, int32_t H,
                       int32_t W, int32_t i, int32_t j, double r2, int32_t K, kv *list, int64_t *idx, double *zbuf,
                       double *dists) {
    double px = -1.0 + (2.0 * j + 1.0) / W, py = 1.0 - (2.0 * i + 1.0) / H;
    int cnt = 0;
    int near_margin = 0;
    kv marg;
    marg.key = 0.0;
    marg.id = 0;
    marg.aux = 0.0;
    for (int64_t m = first[n]; m < first[n] + num[n]; ++m) {
        if (m < 0 || m >= P) continue;
        double x = pts[3 * m], y = pts[3 * m + 1], z = pts[3 * m + 2];
        if (z < 0.0) continue;
        double d2 = (px - x) * (px - x) + (py - y) * (py - y);
        if (fabs(d2 - r2) < POINT_MARGIN * r2) {
            /* decided by rounding: remember the nearest such point */
            kv e = {z, m, d2};
            if (!near_margin || kv_before(&e, &marg)) marg = e;
            near_margin = 1;
        }
        if (d2 > r2) continue;
        kv e = {z, m, d2};
        cnt = kv_insert(list, cnt, K, e);
    }
    for (int k = 0; k < K; ++k) {
        idx[k] = k < cnt ? list[k].id : -1;
        zbuf[k] = k < cnt ? list[k].key : -1.0;
        dists[k] = k < cnt ? list[k].aux : -1.0;
    }
    if (!near_margin) return 0;
    return cnt < K || kv_before(&marg, &list[K - 1]) || marg.id == list[K - 1].id;
}

/* Step 22 for the N images; idx, zbuf, dists are N x H x W x K; flags N x H x W (may be NULL). */
int oracle_rasterize_points(const float *pts, int64_t P, const int64_t *first, const int64_t *num, int32_t N,
                            int32_t H, int32_t W, double radius, int32_t K, int64_t *idx, double *zbuf,
                            double *dists, uint8_t *flags) {
    if (N < 0 || H < 1 || W < 1 || K < 1 || radius < 0) return -1;
    kv *list = (kv *)malloc(sizeof(kv) * (size_t)(K + 1));
    for (int32_t n = 0; n < N; ++n)
        for (int32_t i = 0; i < H; ++i)
            for (int32_t j = 0; j < W; ++j) {
                int64_t q = ((int64_t)n * H + i) * W + j;
                int f = point_pixel(pts, P, first, num, n, H, W, i, j, radius * radius, K, list, idx + q * K,
                                    zbuf + q * K, dists + q * K);
                if (flags) flags[q] = (uint8_t)f;
            }
    free(list);
    return 0;
}

/* Step 22 at npix listed pixels (ids n * H * W + i * W + j); outputs npix x K, flags npix. */
int oracle_rasterize_points_pixels(const float *pts, int64_t P, const int64_t *first, const int64_t *num, int32_t N,
                                   int32_t H, int32_t W, double radius, int32_t K, const int64_t *pixels,
                                   int64_t npix, int64_t *idx, double *zbuf, double *dists, uint8_t *flags) {
    if (N < 0 || H < 1 || W < 1 || K < 1 || radius < 0) return -1;
    kv *list = (kv *)malloc(sizeof(kv) * (size_t)(K + 1));
    for (int64_t t = 0; t < npix; ++t) {
        int64_t q = pixels[t];
        int32_t n = (int32_t)(q / ((int64_t)H * W)), i = (int32_t)((q / W) % H), j = (int32_t)(q % W);
        if (q < 0 || n >= N) {
            free(list);
            return -1;
        }
        flags[t] = (uint8_t)point_pixel(pts, P, first, num, n, H, W, i, j, radius * radius, K, list, idx + t * K,
                                        zbuf + t * K, dists + t * K);
    }
    free(list);
    return 0;
}

/* Step 23: grad_points (P x 3) overwritten; grad_zbuf / grad_dists may be NULL. */
void oracle_rasterize_points_bwd(const float *pts, int64_t P, const int64_t *idx, int32_t N, int32_t H, int32_t W,
                                 int32_t K, const double *grad_zbuf, const double *grad_dists, double *grad) {
    memset(grad, 0, sizeof(double) * 3 * (size_t)P);
    for (int32_t n = 0; n < N; ++n)
        for (int32_t i = 0; i < H; ++i)
            for (int32_t j = 0; j < W; ++j) {
                double px = -1.0 + (2.0 * j + 1.0) / W, py = 1.0 - (2.0 * i + 1.0) / H;
                int64_t o = (((int64_t)n * H + i) * W + j) * K;
                for (int k = 0; k < K; ++k) {
                    int64_t m = idx[o + k];
                    if (m < 0) continue;
                    if (grad_dists) {
                        grad[3 * m] += grad_dists[o + k] * -2.0 * (px - pts[3 * m]);
                        grad[3 * m + 1] += grad_dists[o + k] * -2.0 * (py - pts[3 * m + 1]);
                    }
                    if (grad_zbuf) grad[3 * m + 2] += grad_zbuf[o + k];
                }
            }
}

/* Steps 24-25: mode 0 alpha, 1 norm-weighted; features P x C; out npix x C. */
void oracle_composite_points(const int64_t *idx, const double *dists, int64_t npix, int32_t K, const double *feat,
                             int32_t C, double radius, int32_t mode, double *out) {
    double r2 = radius * radius;
    for (int64_t q = 0; q < npix; ++q) {
        double T = 1.0, wsum = 0.0;
        for (int c = 0; c < C; ++c) out[q * C + c] = 0.0;
        for (int k = 0; k < K; ++k) {
            int64_t m = idx[q * K + k];
            if (m < 0) continue;
            double a = 1.0 - dists[q * K + k] / r2;
            double w = mode == 0 ? a * T : a;
            for (int c = 0; c < C; ++c) out[q * C + c] += w * feat[m * C + c];
            T *= 1.0 - a;
            wsum += a;
        }
        if (mode == 1) {
            double den = wsum > NORM_FLOOR ? wsum : NORM_FLOOR;
            for (int c = 0; c < C; ++c) out[q * C + c] /= den;
        }
    }
}

/* Step 26: grad_feat (P x C) overwritten, grad_dists (npix x K) written (0 for empty slots). */
void oracle_composite_points_bwd(const int64_t *idx, const double *dists, int64_t npix, int32_t K,
                                 const double *feat, int64_t P, int32_t C, double radius, int32_t mode,
                                 const double *grad_out, double *grad_feat, double *grad_dists) {
    double r2 = radius * radius;
    double *fo = (double *)malloc(sizeof(double) * (size_t)C);   /* the normalised output */
    memset(grad_feat, 0, sizeof(double) * (size_t)(P * C));
    for (int64_t q = 0; q < npix; ++q) {
        const double *g = grad_out + q * C;
        double wsum = 0.0;
        for (int k = 0; k < K; ++k)
            if (idx[q * K + k] >= 0) wsum += 1.0 - dists[q * K + k] / r2;
        double den = wsum > NORM_FLOOR ? wsum : NORM_FLOOR;
        for (int c = 0; c < C; ++c) fo[c] = 0.0;
        if (mode == 1)
            for (int k = 0; k < K; ++k) {
                int64_t m = idx[q * K + k];
                if (m < 0) continue;
                double a = 1.0 - dists[q * K + k] / r2;
                for (int c = 0; c < C; ++c) fo[c] += a * feat[m * C + c] / den;
            }
        for (int k = 0; k < K; ++k) {
            int64_t m = idx[q * K + k];
            if (m < 0) {
                grad_dists[q * K + k] = 0.0;
                continue;
            }
            double a = 1.0 - dists[q * K + k] / r2;
            double ga = 0.0;
            if (mode == 0) {
                /* out = sum_l a_l prod_{j<l} (1 - a_j) f_l */
                double Tk = 1.0;
                for (int j = 0; j < k; ++j)
                    if (idx[q * K + j] >= 0) Tk *= 1.0 - (1.0 - dists[q * K + j] / r2);
                for (int c = 0; c < C; ++c) {
                    grad_feat[m * C + c] += a * Tk * g[c];
                    ga += Tk * feat[m * C + c] * g[c];
                }
                for (int l = k + 1; l < K; ++l) {
                    int64_t ml = idx[q * K + l];
                    if (ml < 0) continue;
                    double al = 1.0 - dists[q * K + l] / r2;
                    double Tl_wo_k = 1.0;   /* prod_{j < l, j != k} (1 - a_j) */
                    for (int j = 0; j < l; ++j)
                        if (j != k && idx[q * K + j] >= 0) Tl_wo_k *= 1.0 - (1.0 - dists[q * K + j] / r2);
                    for (int c = 0; c < C; ++c) ga -= al * Tl_wo_k * feat[ml * C + c] * g[c];
                }
            } else {
                for (int c = 0; c < C; ++c) grad_feat[m * C + c] += a / den * g[c];
                if (wsum > NORM_FLOOR)
                    for (int c = 0; c < C; ++c) ga += (feat[m * C + c] - fo[c]) / den * g[c];
                else
                    for (int c = 0; c < C; ++c) ga += feat[m * C + c] / den * g[c];
            }
            grad_dists[q * K + k] = ga * (-1.0 / r2);
        }
    }
    free(fo);
}

/* Step 27: queries (P1 x D, clouds first1/num1), references (P2 x D, first2/num2);
 * idx, dists P1 x K; flags P1 (may be NULL). */
int oracle_knn(const float *p1, const int64_t *first1, const int64_t *num1, const float *p2, const int64_t *first2,
               const int64_t *num2, int32_t N, int32_t D, int32_t K, int64_t *idx, double *dists, uint8_t *flags) {
    if (N < 0 || D < 1 || K < 1) return -1;
    kv *list = (kv *)malloc(sizeof(kv) * (size_t)(K + 1));
    for (int32_t n = 0; n < N; ++n)
        for (int64_t i = first1[n]; i < first1[n] + num1[n]; ++i) {
            int cnt = 0;
            for (int64_t j = first2[n]; j < first2[n] + num2[n]; ++j) {
                double d = 0.0;
                for (int e = 0; e < D; ++e) {
                    double t = (double)p1[i * D + e] - (double)p2[j * D + e];
                    d += t * t;
                }
                kv x = {d, j, 0.0};
                cnt = kv_insert(list, cnt, K + 1, x);   /* K + 1 kept to see the boundary */
            }
            for (int k = 0; k < K; ++k) {
                idx[i * K + k] = k < cnt ? list[k].id : -1;
                dists[i * K + k] = k < cnt ? list[k].key : -1.0;
            }
            if (flags) {
                int f = 0;
                for (int k = 0; k + 1 < cnt && k < K; ++k)
                    if (list[k + 1].key - list[k].key <= KNN_TIE * list[k + 1].key) f = 1;
                flags[i] = (uint8_t)f;
            }
        }
    free(list);
    return 0;
}

/* Step 28: grad_p1 (P1 x D) and grad_p2 (P2 x D) overwritten. */
void oracle_knn_bwd(const float *p1, int64_t P1, const float *p2, int64_t P2, int32_t D, int32_t K,
                    const int64_t *idx, const double *grad_dists, double *grad_p1, double *grad_p2) {
    memset(grad_p1, 0, sizeof(double) * (size_t)(P1 * D));
    memset(grad_p2, 0, sizeof(double) * (size_t)(P2 * D));
    for (int64_t i = 0; i < P1; ++i)
        for (int k = 0; k < K; ++k) {
            int64_t j = idx[i * K + k];
            if (j < 0) continue;
            for (int e = 0; e < D; ++e) {
                double t = 2.0 * ((double)p1[i * D + e] - (double)p2[j * D + e]) * grad_dists[i * K + k];
                grad_p1[i * D + e] += t;
                grad_p2[j * D + e] -= t;
            }
        }
}
