/*
 * bts.h - C ABI of libbts.so: ball-tree build, rotated rebuild, row movement
 * and ball attention on one NVIDIA B200 (sm_100a).
 *
 * Sources (page title, then place on the page):
 *  [E6]  "Erwin: A Tree-based Hierarchical Transformer for Large-scale Physical
 *        Systems", author's thread, post 6/N: a ball tree recursively
 *        divides the points into nested groups of about equal size, each
 *        enclosed by a ball.
 *  [E7]  same thread, post 7/N: pick a tree level and compute attention
 *        within every ball of it in parallel (Ball Tree Attention).
 *  [E9]  same thread, post 9/N: at every level the points of one ball are
 *        kept contiguous in memory, so ball operations are views.
 *  [E15] same thread, post 15/N: the tree construction is a native,
 *        parallel component.
 *  [ROT] thread post on cross-ball exchange: the tree is rotated, where
 *        Swin would shift its windows.
 *  [ABS] PMLR abstract of the same paper: linear-time attention in
 *        fixed-size neighbourhoods of a ball tree partition.
 *
 * The split rule is the one these sources imply and leave open: every node
 * of s slots is cut into two halves of s/2 at the median of the axis of
 * largest extent (float max - min over its real points, lowest axis on equal
 * extents), points ordered by (coordinate, original index) with -0 equal to
 * +0; leaves list their points in ascending original index.
 *
 * Conventions for every call:
 *  - Pointers are DEVICE pointers owned by the caller unless marked "host".
 *    The library allocates nothing; scratch comes from a caller workspace.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Argument errors are returned before anything is
 *    enqueued.  Errors found on the device (non-finite coordinates, a perm
 *    entry outside the tensors, an inter-block wait that ran out) are
 *    recorded, first error wins, in a status word of the stream the call was
 *    enqueued on, and read back (and cleared) by bt_last_device_status(stream).
 *    Builds also keep theirs in the workspace (bt_build_device_status).  Work
 *    captured into a CUDA graph records into the word of the stream it was
 *    captured on, wherever the graph is later launched.  No call traps, aborts
 *    or prints.
 *  - Arrays are row-major and contiguous.  Coordinates are float [rows, 3].
 *    Q/K/V/O are [rows, H, d] (H heads of d values per row).
 *  - Calls may come from several host threads: the per-device set-up on a
 *    device's first call is done once, under a lock inside the library.
 *    Workspaces (and bt_build_noalloc's static scratch) are not shared safely
 *    between builds in flight at the same time; that is the caller's to avoid.
 */
#ifndef BTS_H
#define BTS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BT_OK = 0,
    BT_ERR_ARG = 1,         /* NULL pointer, size out of range, misaligned pointer */
    BT_ERR_SHAPE = 2,       /* N is not m * 2^L (bt_build), m / d / H not supported */
    BT_ERR_NONFINITE = 3,   /* a coordinate is NaN or infinite (found on the device) */
    BT_ERR_WORKSPACE = 4,   /* workspace NULL or smaller than *_workspace_size() */
    BT_ERR_CUDA = 5,        /* a CUDA runtime call failed */
    BT_ERR_TIMEOUT = 6,     /* an inter-block wait gave up (found on the device) */
    BT_ERR_UNSUPPORTED = 7, /* a valid request the library does not handle */
    BT_ERR_INTERNAL = 8     /* a consistency check inside a kernel failed (found on the device);
                               the output of that call is not valid */
} bt_status;

typedef enum { BT_F32 = 0, BT_BF16 = 1 } bt_dtype;

/* Largest batch (number of clouds) one segmented build accepts. */
#define BT_MAX_CLOUDS 64

/* Library version as 10000*major + 100*minor + patch. */
int32_t bt_version(void);

/*
 * Workspace bytes for a (segmented) build of B clouds with ball size m.
 *   offsets  host int64 [B+1]: cloud b is rows offsets[b] .. offsets[b+1]-1.
 * Returns 0 for invalid arguments.  The same workspace may be reused by any
 * later build whose workspace size is not larger; one workspace must not be
 * used by two builds in flight at the same time.
 */
size_t bt_build_workspace_size(const int64_t *offsets, int32_t B, int32_t m);

/*
 * Ball tree of one cloud [E6][E9][E15].
 *   coords  float [N, 3]
 *   N       number of points; must equal m * 2^L for some L >= 0
 *           (otherwise BT_ERR_SHAPE; padding is bt_build_segmented's job)
 *   m       leaf (ball) size, 1 <= m <= 1024
 *   perm    int32 [N] out: perm[slot] = row of the point stored in that slot.
 *           Ball b is slots b*m .. b*m+m-1; a node of level l is a run of
 *           N/2^l consecutive slots.
 *   ws      workspace of at least bt_build_workspace_size({0,N}, 1, m) bytes,
 *           256-byte aligned
 */
bt_status bt_build(const float *coords, int64_t N, int32_t m, int32_t *perm, void *ws, size_t ws_bytes,
                   void *stream);

/*
 * Ball trees of a batch of clouds of any sizes [E6][E9].  Cloud b (n_b points)
 * is padded with dummy points to Npad_b = m * 2^ceil(log2(ceil(n_b/m))) slots;
 * a dummy is keyed above every real point on every axis, never counts in an
 * extent, and so ends in the rightmost slots of its cloud.
 *   coords      float [offsets[B], 3], clouds concatenated
 *   offsets     host int64 [B+1], strictly increasing, offsets[0] = 0
 *   B           1 <= B <= BT_MAX_CLOUDS
 *   perm        int32 [sum Npad_b] out: cloud b owns slots pad[b]..pad[b+1]-1;
 *               perm[slot] = global row (offsets[b] + index in cloud), or -1
 *               for a dummy slot
 *   pad_offsets host int64 [B+1] out (may be NULL): the slot offsets pad[b]
 */
bt_status bt_build_segmented(const float *coords, const int64_t *offsets, int32_t B, int32_t m, int32_t *perm,
                             int64_t *pad_offsets, void *ws, size_t ws_bytes, void *stream);

/* Flags of bt_build_segmented_ex. */
#define BT_BUILD_NARROW 1u

/*
 * bt_build_segmented with flags; the result is the same for every flag.
 *   BT_BUILD_NARROW  where every cloud fits the one-launch build (power-of-two
 *                    slot counts of at most 32,768), give each cloud half the
 *                    SMs of the default: slower alone, for a build that runs
 *                    beside other kernels (a second tree on another stream).
 *                    Without it the library still picks the narrow build when
 *                    a batch has more clouds than the device holds at once.
 * Unknown flag bits: BT_ERR_ARG.  Other arguments and errors as for
 * bt_build_segmented.  The pages build one tree at a time and say nothing of
 * how the work is spread over a GPU; the flag changes only that.
 */
bt_status bt_build_segmented_ex(const float *coords, const int64_t *offsets, int32_t B, int32_t m, int32_t *perm,
                                int64_t *pad_offsets, void *ws, size_t ws_bytes, uint32_t flags, void *stream);

/*
 * bt_build without a caller workspace, for callers that cannot allocate
 * device memory when they build a tree: code inside a region being captured
 * into a CUDA graph, plug-ins whose host framework owns every device
 * allocation, real-time hosts with a memory budget fixed at start-up.  The
 * pages have no counterpart; this is a deployment variant of bt_build.
 *   coords, N, m, perm  as for bt_build; N <= 65,536 (else BT_ERR_UNSUPPORTED,
 *                       returned before anything is enqueued)
 *   status_out          device int32 (may be NULL): receives, in stream order,
 *                       the device-side status (BT_OK, BT_ERR_NONFINITE, ...)
 * Scratch is one 8 MiB array inside the library, held on every GPU that
 * loads it until the process exits, and shared by all calls on that device:
 * calls whose work overlaps on the GPU race and must be serialised.  The
 * first call on each device looks up the array's device address; make that
 * first call before any stream capture.  Allocates nothing.
 */
bt_status bt_build_noalloc(const float *coords, int64_t N, int32_t m, int32_t *perm, int32_t *status_out,
                           void *stream);

/*
 * First device-side error recorded by the library's work enqueued on `stream`
 * since the previous call for that stream (every call of this header that
 * launches kernels): synchronises `stream`, then takes and clears the
 * stream's status word in one atomic step.  Returns BT_OK, BT_ERR_NONFINITE,
 * BT_ERR_TIMEOUT or BT_ERR_INTERNAL (or BT_ERR_CUDA).  Streams keep separate
 * words, so a caller neither sees nor clears another stream's errors (the
 * library holds 1,023 such words per device; streams beyond them share one).
 * Not for use while `stream` is being captured.
 */
bt_status bt_last_device_status(void *stream);

/*
 * Device-side status of the last build that used `ws`: synchronises `stream`,
 * returns BT_OK, BT_ERR_NONFINITE, BT_ERR_TIMEOUT or BT_ERR_INTERNAL (or
 * BT_ERR_CUDA).
 */
bt_status bt_build_device_status(const void *ws, void *stream);

/*
 * Rotation by 45 degrees counter-clockwise about +z through the origin [ROT],
 * in float with each product and sum rounded separately (no FMA):
 *   x' = c*x - s*y,  y' = s*x + c*y,  z' = z,  c = s = float(sqrt(1/2)).
 *   in, out  float [N, 3]; may be the same buffer.
 */
bt_status bt_rotate_z(const float *in, int64_t N, float *out, void *stream);

/*
 * Inverse of a tree permutation [E9]: inv[perm[s]] = s for every real slot.
 *   perm    int32 [npad] (dummies -1); its real slots must hold every row
 *           0..n_rows-1 exactly once (as bt_build* produces)
 *   inv     int32 [n_rows] out
 */
bt_status bt_invert_perm(const int32_t *perm, int64_t npad, int64_t n_rows, int32_t *inv, void *stream);

/*
 * Slot map between two trees of the same points [ROT][E9]:
 *   map[s] = invA[permB[s]] (or -1 where permB[s] < 0), so that rows held in
 *   tree-A slot order move to tree-B slot order by Y[s] = X[map[s]].
 *   invA int32 [rows], permB int32 [npad], map int32 [npad] out
 */
bt_status bt_compose(const int32_t *invA, const int32_t *permB, int64_t npad, int32_t *map, void *stream);

/*
 * Row gather into tree order [E9]: Y[s] = X[idx[s]] for idx[s] >= 0, a zero
 * row where idx[s] < 0.  Rows are row_bytes bytes (1 <= row_bytes <= 65536).
 *   X  [rows, row_bytes] (idx values must be < rows), Y [npad, row_bytes] out
 */
bt_status bt_gather(const void *X, const int32_t *idx, int64_t npad, int32_t row_bytes, void *Y, void *stream);

/*
 * Row scatter back to the original order [E9]: X[idx[s]] = Y[s] for
 * idx[s] >= 0; slots with idx[s] < 0 are dropped.  Real idx values must be
 * distinct.
 */
bt_status bt_scatter(const void *Y, const int32_t *idx, int64_t npad, int32_t row_bytes, void *X, void *stream);

/*
 * Ball Tree Attention [E7][ABS]: for every ball b (slots b*m .. b*m+m-1) and
 * head h, every real query row i of the ball gets
 *     O[i,h,:] = sum_j softmax_j(Q[i,h,:] . K[j,h,:] / sqrt(d)) V[j,h,:]
 * over the real rows j of the same ball.  No bias, no positional term.
 *   Q, K, V  [rows, H, d] of dtype dt (BT_F32: float, BT_BF16: bfloat16)
 *   perm     int32 [npad] slot -> row (dummy slots -1: neither query nor
 *            key, nothing written), or NULL: row s sits in slot s (rows >=
 *            npad, no dummies).  Gathering by perm and scattering O back is
 *            fused into the attention kernel.  An entry >= rows is never
 *            dereferenced: the slot is treated as a dummy and BT_ERR_INTERNAL
 *            is recorded for bt_last_device_status().
 *   npad     number of slots, a multiple of m
 *   rows     number of rows of Q, K, V and O
 *   m        1 <= m <= 256;  H >= 1;  d in {32, 64}
 *   O        [rows, H, d] out, dtype dt, original row order; rows no slot
 *            names are left untouched
 * Accumulation and softmax are in float.  BT_BF16 with m dividing 128 runs on
 * the tcgen05 tensor cores; other shapes run on the CUDA cores.
 * Concurrency: the bf16 kernel for d = 32 and even H hands out its work from a
 * pair of device counters, which launches that run at the same time must not
 * share.  Eager calls take pair k mod 256 (k-th eager call on the device), so
 * at most 256 of them may be in flight together.  A call made while `stream`
 * is being captured gets a pair of its own for the life of the process (4,096
 * such pairs per device; later captured calls use a fixed schedule with no
 * counters); two executable graphs instantiated from ONE captured graph share
 * that pair and must not run at the same time (one executable graph replayed
 * repeatedly is fine: CUDA orders its launches).
 */
bt_status bt_ball_attention(const void *Q, const void *K, const void *V, const int32_t *perm, int64_t npad,
                            int64_t rows, int32_t m, int32_t H, int32_t d, bt_dtype dt, void *O, void *stream);

/*
 * Q/K/V projection of the point features [E7][E9]: the attention layer's
 * queries, keys and values are linear maps of each point's features, and a
 * ball's points sit in consecutive slots, so writing the projections in slot
 * order makes every ball one contiguous tile for bt_ball_attention_tree.
 *   out[o(r), h, k] = sum_c X[r, c] * Wt[t*H*d + h*d + k, c]   (t = 0 Q, 1 K,
 *   2 V) for every row r, with o(r) = inv[r] (slot order) when perm is given
 *   and o(r) = r (original order) when perm is NULL.
 *   X        dt [rows, C] device, original row order
 *   Wt       dt [3*H*d, C] device: row j holds the weights of output column j
 *            (the layout of a linear layer's weight)
 *   perm     int32 [npad] device (slot -> row, -1 dummy) or NULL.  Given
 *            perm, Q, K, V are [npad, H, d] in slot order and the rows of the
 *            dummy slots are set to zero; inv (int32 [rows] device, inv[r] =
 *            the slot of row r, as bt_invert_perm writes it) is required.  An
 *            inv entry outside [0, npad) is skipped and recorded as
 *            BT_ERR_INTERNAL.  NULL: Q, K, V are [rows, H, d] (inv, npad unused).
 *   Q, K, V  dt device out
 * The feature rows are read in their own order as whole tiles; each output
 * row is stored at its slot.  BT_BF16 with C a multiple of 64 (at most 512),
 * 3*H*d >= 256, rows >= 128 and 16-byte aligned pointers runs on the tcgen05
 * tensor cores (fp32 accumulation, outputs rounded to bf16); every other shape
 * on the CUDA cores in float.
 */
bt_status bt_qkv_project(const void *X, int64_t rows, int32_t C, const void *Wt, int32_t H, int32_t d, bt_dtype dt,
                         const int32_t *perm, const int32_t *inv, int64_t npad, void *Q, void *K, void *V,
                         void *stream);

/*
 * Ball attention of Q/K/V that are already in slot order (as bt_qkv_project
 * writes them with tree_order): the same result as bt_ball_attention on the
 * original-order tensors, with every ball loaded as one tile.
 *   Qt, Kt, Vt  bf16 [npad, H, d] device, slot order
 *   perm        int32 [npad] device: the output row of each slot, -1 for a
 *               dummy slot (neither query nor key, nothing written)
 *   O           bf16 [rows, H, d] device out, original row order
 * Shapes: bf16, d = 32, even H, m in {16, 32, 64, 128}, npad >= 128
 * (BT_ERR_UNSUPPORTED otherwise); the concurrency note of bt_ball_attention
 * applies.
 */
bt_status bt_ball_attention_tree(const void *Qt, const void *Kt, const void *Vt, const int32_t *perm, int64_t npad,
                                 int64_t rows, int32_t m, int32_t H, int32_t d, bt_dtype dt, void *O, void *stream);

/*
 * One attention layer from the features [E7][E9]: bt_qkv_project into a
 * workspace, then ball attention.  For the shapes bt_ball_attention_tree takes
 * (and a non-NULL perm) the projections are written in slot order and the
 * attention loads whole tiles; otherwise they are written in the original
 * order and bt_ball_attention gathers them.  Arguments as for the two calls;
 * m and d as for bt_ball_attention.
 *   ws  workspace of bt_projected_workspace_size(npad, rows, H, d, dt) bytes,
 *       256-byte aligned (the projected Q, K and V, and the inverse of perm)
 * With perm, every row must be named by a slot (as in a tree built over the
 * rows); the slot-order path relies on it.
 */
size_t bt_projected_workspace_size(int64_t npad, int64_t rows, int32_t H, int32_t d, bt_dtype dt);

bt_status bt_projected_ball_attention(const void *X, const int32_t *perm, int64_t npad, int64_t rows, int32_t C,
                                      const void *Wt, int32_t m, int32_t H, int32_t d, bt_dtype dt, void *O, void *ws,
                                      size_t ws_bytes, void *stream);

/*
 * Ball Sparse Attention ("BSA: Ball Sparse Attention for Large-scale
 * Geometries", as reviewed on Pith: reading notes and referee report).  Three
 * branches per query row i and head h, mixed by sigmoid gates:
 *   ball        O_ball  attention inside the query's own ball (as above);
 *   compression O_cmp   attention over one coarse token per ball: the mean of
 *                       the ball's real K rows and V rows;
 *   selection   O_slc   the queries of one ball form a group; the group's
 *                       pooled query (mean of its Q rows) is scored against
 *                       every coarse key, s_b = q_bar . k_bar_b / sqrt(d), the
 *                       own ball masked if p.mask_own_ball, and the p.topk best
 *                       balls (ties to the lower ball) are attended at full
 *                       resolution;
 *   O[i,h] = g0 O_ball + g1 O_cmp + g2 O_slc,
 *   g_br = sigmoid(bg[3h+br] + sum_c X[i,c] Wg[c, 3h+br]), br 0 ball,
 *   1 compression, 2 selection.
 *   Q, K, V, perm, npad, rows  as for bt_ball_attention (bf16 only)
 *   m        128 (the ball, the query group and one selected block)
 *   d        32 or 64;  H <= 64;  npad / m <= 2048 balls;  0 <= topk <= 32
 *   X        float [rows, C] gate features (original row order)
 *   Wg       float [C, 3H] gate weights;  bg  float [3H] or NULL (zero);
 *            W is staged in shared memory: C * (3H rounded up to 24) * 4
 *            bytes + 33,792 must not exceed 200 KiB (BT_ERR_UNSUPPORTED)
 *   O        bf16 [rows, H, d] out
 *   sel_out  int32 [npad/m, H, topk] out (may be NULL): the selected balls per
 *            (group, head), -1 where fewer than topk balls can be selected
 *   ws       workspace of bsa_workspace_size() bytes, 256-byte aligned
 * Coarse tokens and scores are float; attention accumulates in float with
 * P rounded to bf16 for the tensor cores.  A ball with no real point gives
 * no coarse token and is never selected.
 * p.coarsen_queries: the optional query-coarsening step of the same paper
 * ("BSA with group compression"): the compression and selection branches
 * attend with the group's pooled query instead of each query, so all rows of
 * a group share O_cmp and O_slc (computed once per group and head on the CUDA
 * cores, softmax in float from the bf16 coarse tokens and K/V rows); the ball
 * branch and the gates stay per row.
 */
typedef struct {
    int32_t topk;          /* blocks selected per (group, head) */
    int32_t mask_own_ball; /* nonzero: a group never selects its own ball */
    int32_t coarsen_queries; /* nonzero: query coarsening, see above */
} bsa_params;

size_t bsa_workspace_size(int64_t npad, int64_t rows, int32_t m, int32_t H, int32_t d, int32_t topk);

bt_status bsa_forward(const void *Q, const void *K, const void *V, const int32_t *perm, int64_t npad,
                      int64_t rows, int32_t m, int32_t H, int32_t d, bt_dtype dt, const float *X, int32_t C,
                      const float *Wg, const float *bg, bsa_params p, void *O, int32_t *sel_out, void *ws,
                      size_t ws_bytes, void *stream);

/*
 * Coarser tree levels (author's thread on Erwin, posts 8/N and 9/N: the tree
 * is coarsened and refined while the attention ball keeps its size; the points
 * of every node are contiguous at every level, so pooling is a mean over
 * consecutive slots).  A node `stride` slots wide is a tree node when the
 * tree was built with a leaf size that divides stride (leaf size 1 makes
 * every power-of-two stride a tree level).
 *
 * bt_pool_mean: Xc[j, :] = mean of X[perm[s], :] over the real slots s of
 * node j (s = j*stride .. j*stride+stride-1, perm[s] >= 0), accumulated in
 * float and rounded to dt; a node without a real slot gets zeros and
 * cperm[j] = -1, every other node cperm[j] = j.  cperm is a perm of the
 * coarse level (rows = npad/stride), so levels chain.
 *   X      dt [rows, C] device, original row order (perm NULL: slot order,
 *          rows >= npad)
 *   perm   int32 [npad] device (slot -> row, -1 dummy) or NULL
 *   stride power of two dividing npad;  C >= 1 elements per row
 *   Xc     dt [npad/stride, C] device out, coarse slot order
 *   cperm  int32 [npad/stride] device out, or NULL
 * A perm entry >= rows is skipped and recorded as BT_ERR_INTERNAL in the
 * stream's status word (bt_last_device_status).
 */
bt_status bt_pool_mean(const void *X, const int32_t *perm, int64_t npad, int64_t rows, int32_t C, int32_t stride,
                       bt_dtype dt, void *Xc, int32_t *cperm, void *stream);

/*
 * bt_unpool: refinement by copy, X[perm[s], :] = Xc[s / stride, :] for every
 * real slot s.  Rows no slot names are not written.  Arguments as for
 * bt_pool_mean, with Xc the input and X the output.
 */
bt_status bt_unpool(const void *Xc, const int32_t *perm, int64_t npad, int64_t rows, int32_t C, int32_t stride,
                    bt_dtype dt, void *X, void *stream);

/*
 * Ball attention log2(stride) levels up the tree: Q, K and V are mean-pooled
 * to nodes of `stride` slots (one launch), ball attention runs over balls of
 * m coarse tokens (m*stride slots) with the coarse slot map as perm, and each
 * node's output is copied back to its real rows of O ([rows, H, d], original
 * order).  Mean pooling commutes with a linear Q/K/V projection, so this is
 * the attention of the coarse level's pooled features.  (npad/stride) % m == 0.
 * ws: bt_coarse_workspace_size() bytes, 256-byte aligned (coarse Q, K, V, O
 * and the coarse slot map).
 */
size_t bt_coarse_workspace_size(int64_t npad, int32_t H, int32_t d, int32_t stride, bt_dtype dt);

bt_status bt_coarse_ball_attention(const void *Q, const void *K, const void *V, const int32_t *perm, int64_t npad,
                                   int64_t rows, int32_t m, int32_t H, int32_t d, bt_dtype dt, int32_t stride, void *O,
                                   void *ws, size_t ws_bytes, void *stream);

/* Same as bt_last_device_status (the name of an earlier version of this library). */
bt_status bt_attention_device_status(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* BTS_H */
