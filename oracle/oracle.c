/*
 * CPU oracle for the ball-tree build, the 45-degree rotation and ball attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
 * bench's CPU-baseline leg load this file.  It shares no code with the CUDA
 * library (no headers, helpers or tables) and is deliberately plain and slow:
 * every tree node is sorted afresh with qsort, attention is a triple loop in
 * double precision.  Build: gcc -O2 -ffp-contract=off -fPIC -shared.
 *
 * What it follows (page titles as the sources give them):
 *  - "Erwin: A Tree-based Hierarchical Transformer for Large-scale Physical
 *    Systems" (bluesky thread, posts 6/N and 9/N; PMLR abstract): a ball tree
 *    recursively divides the points into nested groups of about equal size, each
 *    covered by a ball; at every level a ball's points are contiguous.  The
 *    pages do not print a split rule; this oracle takes the plainest one:
 *    median of the axis of largest extent, ties by original index, leaves in
 *    index order.
 *  - same thread, post 7/N: ball tree attention is scaled dot-product
 *    attention computed independently inside every ball of one tree level.
 *  - thread post on cross-partition exchange (the tree is rotated where Swin
 *    would shift its windows): the rotated layer rebuilds the tree on rotated
 *    coordinates (45 degrees about +z here).
 *  - same thread, posts 8/N and 9/N: coarsening and refinement of the tree
 *    keep the ball size of attention fixed; because the points of a node are
 *    contiguous at every level, pooling to the parent level is a mean over
 *    consecutive slots and refinement copies a parent back to its children.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_SHAPE 2
#define ORC_ERR_NONFINITE 3

/* IEEE order-preserving map float -> uint32 (after -0 is folded into +0). */
static uint32_t ord_key(float f)
{
    uint32_t u;
    if (f == 0.0f) f = 0.0f;
    memcpy(&u, &f, 4);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

static int cmp_u64(const void *a, const void *b)
{
    uint64_t x = *(const uint64_t *)a, y = *(const uint64_t *)b;
    return (x > y) - (x < y);
}

static int cmp_u32(const void *a, const void *b)
{
    uint32_t x = *(const uint32_t *)a, y = *(const uint32_t *)b;
    return (x > y) - (x < y);
}

/*
 * One node of the tree.  ids[0..s) are local point ids of one cloud; ids >= n
 * are dummy points that pad the cloud to m * 2^L slots.
 *   s == m : a leaf, its points in ascending id order.
 *   else   : extents over the real points (float max - min), the widest axis
 *            (lowest axis on equal extents), sort by (coordinate key, id) with
 *            dummies keyed above every real point, lower half left.
 */
static void build_node(const float *c, int64_t n, int32_t m, uint32_t *ids, int64_t s, uint64_t *tmp)
{
    if (s == m) {
        qsort(ids, (size_t)s, sizeof(uint32_t), cmp_u32);
        return;
    }
    float lo[3] = {0, 0, 0}, hi[3] = {0, 0, 0}, ext[3] = {0, 0, 0};
    int any = 0;
    for (int64_t i = 0; i < s; ++i) {
        uint32_t id = ids[i];
        if ((int64_t)id >= n) continue;
        for (int a = 0; a < 3; ++a) {
            float v = c[3 * (int64_t)id + a];
            if (v == 0.0f) v = 0.0f;
            if (!any || v < lo[a]) lo[a] = v;
            if (!any || v > hi[a]) hi[a] = v;
        }
        any = 1;
    }
    if (any)
        for (int a = 0; a < 3; ++a) ext[a] = hi[a] - lo[a];
    int axis = 0;
    if (ext[1] > ext[axis]) axis = 1;
    if (ext[2] > ext[axis]) axis = 2;
    for (int64_t i = 0; i < s; ++i) {
        uint32_t id = ids[i];
        uint64_t key = ((int64_t)id < n) ? ord_key(c[3 * (int64_t)id + axis]) : 0xFFFFFFFFu;
        tmp[i] = (key << 32) | id;
    }
    qsort(tmp, (size_t)s, sizeof(uint64_t), cmp_u64);
    for (int64_t i = 0; i < s; ++i) ids[i] = (uint32_t)tmp[i];
    build_node(c, n, m, ids, s / 2, tmp);
    build_node(c, n, m, ids + s / 2, s / 2, tmp);
}

static int64_t padded(int64_t n, int32_t m)
{
    int64_t leaves = (n + m - 1) / m, p = 1;
    if (leaves < 1) leaves = 1;
    while (p < leaves) p <<= 1;
    return p * m;
}

/*
 * Build the tree of every cloud of a batch.
 *   coords   float [offsets[B], 3], clouds concatenated in row order
 *   offsets  int64 [B+1]
 *   perm_out int32 [sum of padded sizes]: slot -> global row (offsets[b] + local id), -1 for dummies
 *   pad_out  int64 [B+1]: slot offset of every cloud
 */
int orc_build(const float *coords, const int64_t *offsets, int32_t B, int32_t m, int32_t *perm_out,
              int64_t *pad_out)
{
    if (!coords || !offsets || !perm_out || !pad_out || B < 1) return ORC_ERR_ARG;
    if (m < 1) return ORC_ERR_SHAPE;
    for (int64_t i = 0; i < 3 * offsets[B]; ++i)
        if (!isfinite(coords[i])) return ORC_ERR_NONFINITE;
    pad_out[0] = 0;
    for (int32_t b = 0; b < B; ++b) {
        int64_t n = offsets[b + 1] - offsets[b];
        if (n < 1) return ORC_ERR_SHAPE;
        pad_out[b + 1] = pad_out[b] + padded(n, m);
    }
    for (int32_t b = 0; b < B; ++b) {
        int64_t n = offsets[b + 1] - offsets[b], s = pad_out[b + 1] - pad_out[b];
        uint32_t *ids = (uint32_t *)malloc((size_t)s * sizeof(uint32_t));
        uint64_t *tmp = (uint64_t *)malloc((size_t)s * sizeof(uint64_t));
        if (!ids || !tmp) { free(ids); free(tmp); return ORC_ERR_ARG; }
        for (int64_t i = 0; i < s; ++i) ids[i] = (uint32_t)i;
        build_node(coords + 3 * offsets[b], n, m, ids, s, tmp);
        for (int64_t i = 0; i < s; ++i)
            perm_out[pad_out[b] + i] = ((int64_t)ids[i] < n) ? (int32_t)(offsets[b] + ids[i]) : -1;
        free(ids);
        free(tmp);
    }
    return ORC_OK;
}

/*
 * Rotation by 45 degrees counter-clockwise about +z through the origin, in
 * float with every product and sum rounded on its own (no fused multiply-add):
 *   x' = c*x - s*y,  y' = s*x + c*y,  z' = z,  c = s = float(sqrt(1/2)).
 */
void orc_rotate_z(const float *in, int64_t n, float *out)
{
    const uint32_t bits = 0x3F3504F3u; /* nearest float to sqrt(1/2) */
    float c, s;
    memcpy(&c, &bits, 4);
    s = c;
    for (int64_t i = 0; i < n; ++i) {
        float x = in[3 * i], y = in[3 * i + 1], z = in[3 * i + 2];
        volatile float cx = c * x, sy = s * y, sx = s * x, cy = c * y;
        out[3 * i] = cx - sy;
        out[3 * i + 1] = sx + cy;
        out[3 * i + 2] = z;
    }
}

/* element (row, head, k) of a [rows, H, d] tensor, widened to double
   (dtype 0 float, 1 bf16 bits, 2 double) */
static double widen(const void *p, int dtype, int64_t idx)
{
    if (dtype == 0) return (double)((const float *)p)[idx];
    if (dtype == 2) return ((const double *)p)[idx];
    uint32_t u = (uint32_t)((const uint16_t *)p)[idx] << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/*
 * Attention of one query row over a list of key rows, in double:
 *   O = sum_j softmax_j(q . k_j / sqrt(d)) v_j ; no key -> O = 0.
 */
static void attend(const void *Q, const void *K, const void *V, int dtype, int32_t H, int32_t d, int32_t h,
                   int64_t qrow, const int64_t *krows, int64_t nk, double *logit, double *o)
{
    double scale = 1.0 / sqrt((double)d), mx = -INFINITY, den = 0.0;
    for (int k = 0; k < d; ++k) o[k] = 0.0;
    if (nk == 0) return;
    for (int64_t j = 0; j < nk; ++j) {
        double acc = 0.0;
        for (int k = 0; k < d; ++k)
            acc += widen(Q, dtype, (qrow * H + h) * d + k) * widen(K, dtype, (krows[j] * H + h) * d + k);
        logit[j] = acc * scale;
        if (logit[j] > mx) mx = logit[j];
    }
    for (int64_t j = 0; j < nk; ++j) {
        double w = exp(logit[j] - mx);
        den += w;
        for (int k = 0; k < d; ++k) o[k] += w * widen(V, dtype, (krows[j] * H + h) * d + k);
    }
    for (int k = 0; k < d; ++k) o[k] /= den;
}

/*
 * Ball attention.  Slots are grouped in balls of m consecutive slots; slot s
 * holds row perm[s] of Q/K/V (perm == NULL: row s), or a dummy (perm[s] < 0)
 * that is neither a query nor a key.  Output O [rows, H, d] (double) in the
 * original row order; only rows of the listed balls are written
 * (balls == NULL: every ball).  dtype 0 = float32, 1 = bfloat16 bits.
 */
int orc_ball_attention(const void *Q, const void *K, const void *V, int dtype, const int32_t *perm, int64_t npad,
                       int32_t m, int32_t H, int32_t d, const int64_t *balls, int64_t n_balls, double *O)
{
    if (!Q || !K || !V || !O || m < 1 || H < 1 || d < 1 || npad % m) return ORC_ERR_ARG;
    int64_t nb = balls ? n_balls : npad / m;
    int64_t *krows = (int64_t *)malloc((size_t)m * sizeof(int64_t));
    double *logit = (double *)malloc((size_t)m * sizeof(double));
    if (!krows || !logit) { free(krows); free(logit); return ORC_ERR_ARG; }
    for (int64_t t = 0; t < nb; ++t) {
        int64_t b = balls ? balls[t] : t;
        int64_t nk = 0;
        for (int64_t j = 0; j < m; ++j) {
            int64_t r = perm ? perm[b * m + j] : b * m + j;
            if (r >= 0) krows[nk++] = r;
        }
        for (int32_t h = 0; h < H; ++h)
            for (int64_t i = 0; i < nk; ++i)
                attend(Q, K, V, dtype, H, d, h, krows[i], krows, nk, logit, O + (krows[i] * H + h) * d);
    }
    free(krows);
    free(logit);
    return ORC_OK;
}

/*
 * Full attention over all n rows (every row a key) for the listed query rows
 * (rows == NULL: all).  Output O [n, H, d] double.
 */
int orc_full_attention(const void *Q, const void *K, const void *V, int dtype, int64_t n, int32_t H, int32_t d,
                       const int64_t *rows, int64_t n_rows, double *O)
{
    if (!Q || !K || !V || !O || n < 1 || H < 1 || d < 1) return ORC_ERR_ARG;
    int64_t *krows = (int64_t *)malloc((size_t)n * sizeof(int64_t));
    double *logit = (double *)malloc((size_t)n * sizeof(double));
    if (!krows || !logit) { free(krows); free(logit); return ORC_ERR_ARG; }
    for (int64_t j = 0; j < n; ++j) krows[j] = j;
    int64_t nq = rows ? n_rows : n;
    for (int64_t t = 0; t < nq; ++t) {
        int64_t r = rows ? rows[t] : t;
        for (int32_t h = 0; h < H; ++h) attend(Q, K, V, dtype, H, d, h, r, krows, n, logit, O + (r * H + h) * d);
    }
    free(krows);
    free(logit);
    return ORC_OK;
}

/* inverse permutation and composition (slot maps between two trees of one cloud set) */
void orc_invert(const int32_t *perm, int64_t npad, int32_t *inv, int64_t n_rows)
{
    for (int64_t r = 0; r < n_rows; ++r) inv[r] = -1;
    for (int64_t s = 0; s < npad; ++s)
        if (perm[s] >= 0) inv[perm[s]] = (int32_t)s;
}

void orc_compose(const int32_t *invA, const int32_t *permB, int64_t npad, int32_t *map)
{
    for (int64_t s = 0; s < npad; ++s) map[s] = permB[s] >= 0 ? invA[permB[s]] : -1;
}

/*
 * Ball Sparse Attention (page: Pith review of "BSA: Ball Sparse Attention for
 * Large-scale Geometries" - reading notes and referee report).  Three
 * branches per query, mixed by learned sigmoid gates:
 *   ball        - attention inside the query's own ball (as above);
 *   compression - attention over one coarse token per ball: the mean of the
 *                 ball's K and V rows (mean pooling, one token per ball);
 *   selection   - the queries of one group (= one ball of m slots) share one
 *                 set of blocks: the group's pooled query (mean of its q rows)
 *                 is scored against every coarse key, q_bar . k_bar / sqrt(d),
 *                 the group's own ball is masked, and the top-k balls (ties to
 *                 the lower ball index) are attended at full resolution.
 *   gates       - g[i, h, br] = sigmoid(b[3h+br] + sum_c X[i,c] W[c, 3h+br]),
 *                 br = 0 ball, 1 compression, 2 selection.
 *   O = g0 O_ball + g1 O_cmp + g2 O_slc   (per head).
 * Everything in double from the widened inputs.  A ball with no real point
 * gives no coarse token and cannot be selected.
 *
 * coarsen_q: the optional query-coarsening step (BSA with group compression):
 * the compression and selection branches take the group's pooled query q_bar
 * (the mean of its real q rows) in place of each query, so every query of a
 * group gets the same O_cmp and O_slc; the ball branch and the gates stay per
 * query.
 *
 * sel_in (optional, [nb, H, topk]): use this selection instead of computing it
 * (the tests use it where two blocks tie within rounding).  groups (optional):
 * compute output rows only for these groups.  All outputs except O may be
 * NULL.  Rows are [rows, H, d] in original order; scores [nb, H, nb].
 */
static void attend_vec(const double *q, const double *keys, const double *vals, const unsigned char *valid,
                       int64_t n, int32_t d, double *logit, double *o)
{
    double scale = 1.0 / sqrt((double)d), mx = -INFINITY, den = 0.0;
    int any = 0;
    for (int k = 0; k < d; ++k) o[k] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        if (valid && !valid[j]) continue;
        double acc = 0.0;
        for (int k = 0; k < d; ++k) acc += q[k] * keys[j * d + k];
        logit[j] = acc * scale;
        if (logit[j] > mx) mx = logit[j];
        any = 1;
    }
    if (!any) return;
    for (int64_t j = 0; j < n; ++j) {
        if (valid && !valid[j]) continue;
        double w = exp(logit[j] - mx);
        den += w;
        for (int k = 0; k < d; ++k) o[k] += w * vals[j * d + k];
    }
    for (int k = 0; k < d; ++k) o[k] /= den;
}

int orc_bsa(const void *Q, const void *K, const void *V, int dtype, const int32_t *perm, int64_t npad, int64_t rows,
            int32_t m, int32_t H, int32_t d, const float *X, int32_t C, const float *Wg, const float *bg, int32_t topk,
            int32_t mask_own, int32_t coarsen_q, const int32_t *sel_in, const int64_t *groups, int64_t n_groups, double *O,
            double *O_ball, double *O_cmp, double *O_slc, double *gates, int32_t *sel_out, double *scores_out)
{
    if (!Q || !K || !V || !O || !X || !Wg || m < 1 || H < 1 || d < 1 || C < 1 || topk < 0 || npad % m) return ORC_ERR_ARG;
    int64_t nb = npad / m;
    double *qbar = (double *)calloc((size_t)(nb * H * d), sizeof(double));
    double *kbar = (double *)calloc((size_t)(nb * H * d), sizeof(double));
    double *vbar = (double *)calloc((size_t)(nb * H * d), sizeof(double));
    unsigned char *tok = (unsigned char *)calloc((size_t)nb, 1);
    double *logit = (double *)malloc((size_t)((nb > m * (int64_t)(topk + 1) ? nb : m * (int64_t)(topk + 1)) * sizeof(double)));
    double *keys = (double *)malloc((size_t)(m * (int64_t)(topk + 1) * d) * sizeof(double));
    double *vals = (double *)malloc((size_t)(m * (int64_t)(topk + 1) * d) * sizeof(double));
    double *kc = (double *)malloc((size_t)(nb * d) * sizeof(double));
    double *vc = (double *)malloc((size_t)(nb * d) * sizeof(double));
    double *sc = (double *)malloc((size_t)nb * sizeof(double));
    int32_t *sel = (int32_t *)malloc((size_t)(nb * H * (topk > 0 ? topk : 1)) * sizeof(int32_t));
    int64_t *krows = (int64_t *)malloc((size_t)m * sizeof(int64_t));
    double *ob = (double *)malloc((size_t)d * sizeof(double)), *oc = (double *)malloc((size_t)d * sizeof(double));
    double *os = (double *)malloc((size_t)d * sizeof(double)), *qv = (double *)malloc((size_t)d * sizeof(double));
    if (!qbar || !kbar || !vbar || !tok || !logit || !keys || !vals || !kc || !vc || !sc || !sel || !krows || !ob || !oc ||
        !os || !qv)
        return ORC_ERR_ARG;
    /* coarse tokens and pooled queries: means over the real rows of each ball */
    for (int64_t b = 0; b < nb; ++b) {
        int64_t cnt = 0;
        for (int64_t j = 0; j < m; ++j) {
            int64_t r = perm ? perm[b * m + j] : b * m + j;
            if (r < 0) continue;
            ++cnt;
            for (int32_t h = 0; h < H; ++h)
                for (int k = 0; k < d; ++k) {
                    int64_t idx = (r * H + h) * d + k, o = (b * H + h) * d + k;
                    qbar[o] += widen(Q, dtype, idx);
                    kbar[o] += widen(K, dtype, idx);
                    vbar[o] += widen(V, dtype, idx);
                }
        }
        tok[b] = cnt > 0;
        if (cnt)
            for (int64_t o = b * H * d; o < (b + 1) * H * d; ++o) {
                qbar[o] /= (double)cnt;
                kbar[o] /= (double)cnt;
                vbar[o] /= (double)cnt;
            }
    }
    /* group scores and top-k per (group, head) */
    for (int64_t g = 0; g < nb; ++g)
        for (int32_t h = 0; h < H; ++h) {
            for (int64_t b = 0; b < nb; ++b) {
                double acc = 0.0;
                for (int k = 0; k < d; ++k) acc += qbar[(g * H + h) * d + k] * kbar[(b * H + h) * d + k];
                sc[b] = (tok[b] && tok[g] && !(mask_own && b == g)) ? acc / sqrt((double)d) : -INFINITY;
                if (scores_out) scores_out[(g * H + h) * nb + b] = sc[b];
            }
            int32_t *s = sel + (g * H + h) * topk;
            for (int t = 0; t < topk; ++t) {
                int64_t best = -1;
                for (int64_t b = 0; b < nb; ++b) {
                    if (sc[b] == -INFINITY) continue;
                    int taken = 0;
                    for (int u = 0; u < t; ++u) taken |= s[u] == b;
                    if (taken) continue;
                    if (best < 0 || sc[b] > sc[best]) best = b;  /* strict: the lower index wins ties */
                }
                s[t] = (int32_t)best;
            }
            if (sel_in)
                for (int t = 0; t < topk; ++t) s[t] = sel_in[(g * H + h) * topk + t];
            if (sel_out)
                for (int t = 0; t < topk; ++t) sel_out[(g * H + h) * topk + t] = s[t];
        }
    /* branches, gates and the gated sum for every real query row (of the listed groups) */
    for (int64_t gi = 0; gi < (groups ? n_groups : nb); ++gi) {
        int64_t g = groups ? groups[gi] : gi;
        int64_t nk = 0;
        for (int64_t j = 0; j < m; ++j) {
            int64_t r = perm ? perm[g * m + j] : g * m + j;
            if (r >= 0) krows[nk++] = r;
        }
        for (int32_t h = 0; h < H; ++h) {
            for (int64_t b = 0; b < nb; ++b)
                for (int k = 0; k < d; ++k) {
                    kc[b * d + k] = kbar[(b * H + h) * d + k];
                    vc[b * d + k] = vbar[(b * H + h) * d + k];
                }
            int64_t ns = 0;
            const int32_t *s = sel + (g * H + h) * topk;
            for (int t = 0; t < topk; ++t) {
                if (s[t] < 0) continue;
                for (int64_t j = 0; j < m; ++j) {
                    int64_t r = perm ? perm[(int64_t)s[t] * m + j] : (int64_t)s[t] * m + j;
                    if (r < 0) continue;
                    for (int k = 0; k < d; ++k) {
                        keys[ns * d + k] = widen(K, dtype, (r * H + h) * d + k);
                        vals[ns * d + k] = widen(V, dtype, (r * H + h) * d + k);
                    }
                    ++ns;
                }
            }
            for (int64_t i = 0; i < nk; ++i) {
                int64_t r = krows[i];
                for (int k = 0; k < d; ++k) qv[k] = coarsen_q ? qbar[(g * H + h) * d + k] : widen(Q, dtype, (r * H + h) * d + k);
                attend(Q, K, V, dtype, H, d, h, r, krows, nk, logit, ob);
                attend_vec(qv, kc, vc, tok, nb, d, logit, oc);
                attend_vec(qv, keys, vals, NULL, ns, d, logit, os);
                double gv[3];
                for (int br = 0; br < 3; ++br) {
                    double z = bg ? (double)bg[3 * h + br] : 0.0;
                    for (int c = 0; c < C; ++c) z += (double)X[r * C + c] * (double)Wg[(int64_t)c * 3 * H + 3 * h + br];
                    gv[br] = 1.0 / (1.0 + exp(-z));
                    if (gates) gates[(r * H + h) * 3 + br] = gv[br];
                }
                for (int k = 0; k < d; ++k) {
                    int64_t o = (r * H + h) * d + k;
                    O[o] = gv[0] * ob[k] + gv[1] * oc[k] + gv[2] * os[k];
                    if (O_ball) O_ball[o] = ob[k];
                    if (O_cmp) O_cmp[o] = oc[k];
                    if (O_slc) O_slc[o] = os[k];
                }
            }
        }
    }
    (void)rows;
    free(qbar); free(kbar); free(vbar); free(tok); free(logit); free(keys); free(vals); free(kc); free(vc); free(sc);
    free(sel); free(krows); free(ob); free(oc); free(os); free(qv);
    return ORC_OK;
}

/*
 * Coarsening to a higher tree level ("Erwin" thread, posts 8/N and 9/N): the
 * nodes `s` levels up (s = stride, a power of two) hold `stride` consecutive
 * slots each.  Xc[j, c] = mean of X[perm[slot], c] over the real slots of node
 * j (slots j*stride .. j*stride+stride-1 with perm >= 0); a node without a real
 * slot is 0 and gets cperm[j] = -1, otherwise cperm[j] = j.  X is [rows, C] in
 * original row order (dtype as widen()), Xc [npad/stride, C] in coarse slot
 * order, cperm may be NULL.  cperm is a valid perm for the coarse level (rows =
 * npad/stride), so levels chain.
 */
int orc_pool_mean(const void *X, int dtype, const int32_t *perm, int64_t npad, int64_t rows, int32_t C,
                  int32_t stride, double *Xc, int32_t *cperm)
{
    if (!X || !Xc || C < 1 || stride < 1 || npad < 1 || npad % stride) return ORC_ERR_ARG;
    for (int64_t j = 0; j < npad / stride; ++j) {
        int64_t cnt = 0;
        for (int32_t c = 0; c < C; ++c) Xc[j * C + c] = 0.0;
        for (int32_t t = 0; t < stride; ++t) {
            int64_t slot = j * stride + t, r = perm ? perm[slot] : slot;
            if (r < 0) continue;
            if (r >= rows) return ORC_ERR_ARG;
            ++cnt;
            for (int32_t c = 0; c < C; ++c) Xc[j * C + c] += widen(X, dtype, r * C + c);
        }
        if (cnt)
            for (int32_t c = 0; c < C; ++c) Xc[j * C + c] /= (double)cnt;
        if (cperm) cperm[j] = cnt ? (int32_t)j : -1;
    }
    return ORC_OK;
}

/*
 * Refinement back to the finer level (same posts): every real slot takes the
 * value of its node `stride` slots wide: X[perm[slot], c] = Xc[slot / stride, c].
 * Rows that no slot names are left as they are.
 */
int orc_unpool(const double *Xc, const int32_t *perm, int64_t npad, int64_t rows, int32_t C, int32_t stride,
               double *X)
{
    if (!X || !Xc || C < 1 || stride < 1 || npad < 1 || npad % stride) return ORC_ERR_ARG;
    for (int64_t slot = 0; slot < npad; ++slot) {
        int64_t r = perm ? perm[slot] : slot;
        if (r < 0) continue;
        if (r >= rows) return ORC_ERR_ARG;
        for (int32_t c = 0; c < C; ++c) X[r * C + c] = Xc[(slot / stride) * C + c];
    }
    return ORC_OK;
}

/*
 * Projection of features to queries, keys and values (the linear maps that
 * precede ball attention in every Erwin / BSA attention block; the Erwin
 * thread's posts 7/N-9/N apply attention to projected features of the
 * points).  Y = X W in double: X [rows, C] (dtype as widen()), W [C, 3*H*d]
 * (dtype as widen()), columns [0, Hd) give Q, [Hd, 2Hd) K, [2Hd, 3Hd) V, head h
 * at h*d .. h*d+d-1 of each block.  Q, K, V out: double [rows, H, d].
 */
int orc_project(const void *X, int xdtype, const void *W, int wdtype, int64_t rows, int32_t C, int32_t H, int32_t d,
                double *Q, double *K, double *V)
{
    if (!X || !W || !Q || !K || !V || rows < 0 || C < 1 || H < 1 || d < 1) return ORC_ERR_ARG;
    const int64_t hd = (int64_t)H * d;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < 3 * hd; ++j) {
            double acc = 0.0;
            for (int32_t c = 0; c < C; ++c) acc += widen(X, xdtype, r * C + c) * widen(W, wdtype, (int64_t)c * 3 * hd + j);
            double *dst = j < hd ? Q : (j < 2 * hd ? K : V);
            dst[r * hd + (j % hd)] = acc;
        }
    return ORC_OK;
}
