// Ball Sparse Attention (page: Pith review of "BSA: Ball Sparse Attention for
// Large-scale Geometries": reading notes and referee report; figure 1 caption).
// Three branches per query, mixed by per-head sigmoid gates:
//   ball        - attention inside the query's own ball (the ball attention
//                 kernels, into the workspace);
//   compression - attention over one coarse token per ball, the mean of the
//                 ball's K and V rows;
//   selection   - the queries of one group (one ball of 128 slots) share one
//                 set of blocks: the group's pooled query is scored against
//                 every coarse key, its own ball is masked, and the top-k balls
//                 (ties to the lower ball) are attended at full resolution.
//   O = g_ball O_ball + g_cmp O_cmp + g_slc O_slc,
//   g = sigmoid(b + X W) with column 3h + branch of W for head h.
//
// Kernels (all on the caller's stream):
//   k_bsa_means    one CTA per ball: pooled query, coarse key (f32 and bf16)
//                  and coarse value (bf16), number of real points.
//   k_bsa_gates    two rows per thread, W and an X tile in shared memory.
//   k_bsa_topk     one CTA per (head, 8 groups), one warp per group: scores
//                  from the pooled query and the f32 coarse keys, own ball and
//                  empty balls masked, top-k.
//   k_bsa_attn_tc  persistent tcgen05 kernel over (group, head) items: the
//                  compression and selection branches as flash-style online
//                  softmax over chunks of 128 keys (S and P in TMEM, P V on the
//                  tensor core, row sums in registers), then the gated sum with
//                  the ball branch, scattered through perm.
//   k_bsa_coarse   the query-coarsening variant of the two branches: one CTA
//                  per (group, head) with the pooled query, then the gated sum.
// This file is included by bts_attn.cu (one translation unit with the ball
// attention kernel and the attention status word).
#pragma once

namespace bts {

constexpr int kBsaMaxTopk = 32;
constexpr int64_t kBsaMaxBalls = 2048;

// eight bf16 values (one 16-byte load) widened to float
__device__ __forceinline__ void bf16x8_to_f32(const uint4 w, float (&f)[8])
{
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u[e]));
        f[2 * e] = t.x;
        f[2 * e + 1] = t.y;
    }
}

// ---------------------------------------------------------------------------
// Ball means: one CTA of 8 warps per ball.  Warp w sums rows w, w+8, ... of
// the ball; each lane owns 8 consecutive channels (16-byte loads of Q, K and
// V), so one warp covers 256 channels per row.  The 8 partial sums meet in
// shared memory.
constexpr int kMeanWarps = 8;

__global__ void __launch_bounds__(kMeanWarps * 32) k_bsa_means(const __nv_bfloat16 *__restrict__ Q,
                                                              const __nv_bfloat16 *__restrict__ K,
                                                              const __nv_bfloat16 *__restrict__ V,
                                                              const int32_t *__restrict__ perm, int64_t rows,
                                                              int HD, float *__restrict__ qbar,
                                                              float *__restrict__ kbar,
                                                              __nv_bfloat16 *__restrict__ kc,
                                                              __nv_bfloat16 *__restrict__ vc,
                                                              int32_t *__restrict__ cnt, uint32_t *status)
{
    constexpr int M = 128;
    __shared__ int32_t srow[M];
    __shared__ int s_cnt;
    __shared__ float sred[kMeanWarps][3][256];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t b = blockIdx.x;
    if (tid == 0) s_cnt = 0;
    __syncthreads();
    if (tid < M) {
        int32_t r = perm ? perm[b * M + tid] : int32_t(b * M + tid);
        if (r >= rows) {
            record_error(status, BT_ERR_INTERNAL);
            r = -1;
        }
        srow[tid] = r;
        const uint32_t vb = __ballot_sync(0xffffffffu, r >= 0);
        if (lane == 0) atomicAdd(&s_cnt, __popc(vb));
    }
    __syncthreads();
    const int n = s_cnt;
    const float inv = n > 0 ? 1.0f / float(n) : 0.0f;
    for (int c0 = 0; c0 < HD; c0 += 256) {
        const int ch = c0 + 8 * lane;  // this lane's 8 channels
        float aq[8], ak[8], av[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) aq[k] = ak[k] = av[k] = 0.0f;
        if (ch < HD) {
#pragma unroll 4
            for (int j = warp; j < M; j += kMeanWarps) {
                const int32_t r = srow[j];
                if (r < 0) continue;
                const size_t off = size_t(r) * HD + ch;
                float f[8];
                bf16x8_to_f32(*reinterpret_cast<const uint4 *>(Q + off), f);
#pragma unroll
                for (int k = 0; k < 8; ++k) aq[k] += f[k];
                bf16x8_to_f32(*reinterpret_cast<const uint4 *>(K + off), f);
#pragma unroll
                for (int k = 0; k < 8; ++k) ak[k] += f[k];
                bf16x8_to_f32(*reinterpret_cast<const uint4 *>(V + off), f);
#pragma unroll
                for (int k = 0; k < 8; ++k) av[k] += f[k];
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            sred[warp][0][8 * lane + k] = aq[k];
            sred[warp][1][8 * lane + k] = ak[k];
            sred[warp][2][8 * lane + k] = av[k];
        }
        __syncthreads();
        {
            const int c = c0 + tid;  // one channel per thread (256 threads)
            if (c < HD) {
                float sq = 0.f, sk = 0.f, sv = 0.f;
#pragma unroll
                for (int w = 0; w < kMeanWarps; ++w) {
                    sq += sred[w][0][tid];
                    sk += sred[w][1][tid];
                    sv += sred[w][2][tid];
                }
                const size_t o = size_t(b) * HD + c;
                qbar[o] = sq * inv;
                kbar[o] = sk * inv;
                kc[o] = __float2bfloat16_rn(sk * inv);
                vc[o] = __float2bfloat16_rn(sv * inv);
            }
        }
        __syncthreads();  // sred is reused by the next channel block
    }
    if (tid == 0) cnt[b] = n;
}

// ---------------------------------------------------------------------------
// Gates: sigmoid(bg + X W) per row and output.  One CTA per kGateRows rows; thread t takes row t % kGateRows
// and half t / kGateRows of every group of kGateOut outputs (kGateOut / 2 accumulators in registers).  W is
// staged once per CTA with its rows padded to a multiple of kGateOut (zeros).  X streams through shared
// memory kGateCols columns at a time, double-buffered (the next slice is loaded into registers as coalesced
// float4 while the current one is used); its rows are padded by one word, so the 32 rows a warp reads at
// one column sit in 32 banks, and the W reads of a warp are broadcasts.  Many small CTAs keep enough X in
// flight per SM to stream it at memory speed.
constexpr int kGateThreads = 256, kGateRows = 128, kGateCols = 32, kGateOut = 24, kGateHalf = kGateOut / 2;

static int gate_out_padded(int H) { return (3 * H + kGateOut - 1) / kGateOut * kGateOut; }

static size_t gate_smem_bytes(int C, int H)
{
    return (size_t(C) * gate_out_padded(H) + size_t(2) * kGateRows * (kGateCols + 1)) * 4;
}

__global__ void __launch_bounds__(kGateThreads) k_bsa_gates(const float *__restrict__ X, int64_t rows, int C,
                                                            const float *__restrict__ W,
                                                            const float *__restrict__ bg, int H, int NOP,
                                                            float *__restrict__ gates)
{
    extern __shared__ __align__(16) float gsm[];
    constexpr int XP = kGateCols + 1;
    constexpr int U = kGateRows * kGateCols / 4 / kGateThreads;  // float4 of a slice per thread
    const int NO = 3 * H;
    float *sW = gsm, *sX = gsm + size_t(C) * NOP;  // sX: [2][kGateRows][XP]
    const int tid = threadIdx.x;
    {
        // W rows padded to NOP columns with zeros; loads batched 8 per thread ahead of their stores
        const int total = C * NO, pad = NOP - NO;
        for (int i0 = 0; i0 < total; i0 += 8 * kGateThreads) {
            float t[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + u * kGateThreads + tid;
                t[u] = i < total ? W[i] : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + u * kGateThreads + tid;
                if (i < total) {
                    const int c = i / NO, j = i - c * NO;
                    sW[c * NOP + j] = t[u];
                }
            }
        }
        for (int i = tid; i < C * pad; i += kGateThreads) {
            const int c = i / pad, j = NO + (i - c * pad);
            sW[c * NOP + j] = 0.0f;
        }
    }
    const int64_t r0 = int64_t(blockIdx.x) * kGateRows;
    const int rr = tid % kGateRows, half = tid / kGateRows;
    const int64_t row = r0 + rr;
    const bool vec4 = (C % 4) == 0 && (reinterpret_cast<uintptr_t>(X) % 16) == 0;
    const int nslice = (C + kGateCols - 1) / kGateCols;
    // one slice of X into registers: row i / (kGateCols/4) of the tile, columns c0 + 4*(i % (kGateCols/4)) .. +3
    auto load_slice = [&](int c0, float4 (&t)[U]) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = tid + u * kGateThreads, lr = i / (kGateCols / 4), c4 = i % (kGateCols / 4);
            const int c = c0 + 4 * c4;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r0 + lr < rows) {
                const float *src = X + (r0 + lr) * C + c;
                if (vec4 && c + 4 <= C) {
                    v = *reinterpret_cast<const float4 *>(src);
                } else {
                    if (c < C) v.x = src[0];
                    if (c + 1 < C) v.y = src[1];
                    if (c + 2 < C) v.z = src[2];
                    if (c + 3 < C) v.w = src[3];
                }
            }
            t[u] = v;
        }
    };
    auto store_slice = [&](int buf, const float4 (&t)[U]) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = tid + u * kGateThreads, lr = i / (kGateCols / 4), c4 = i % (kGateCols / 4);
            float *d = sX + (size_t(buf) * kGateRows + lr) * XP + 4 * c4;
            d[0] = t[u].x;
            d[1] = t[u].y;
            d[2] = t[u].z;
            d[3] = t[u].w;
        }
    };
    for (int j0 = 0; j0 < NO; j0 += kGateOut) {
        const int jh = j0 + half * kGateHalf;  // this thread's first output
        float acc[kGateHalf];
#pragma unroll
        for (int j = 0; j < kGateHalf; ++j) acc[j] = (bg && jh + j < NO) ? bg[jh + j] : 0.0f;
        float4 t[U];
        load_slice(0, t);
        __syncthreads();  // W is staged; neither buffer is read any more
        store_slice(0, t);
        __syncthreads();
        for (int k = 0; k < nslice; ++k) {
            const int c0 = k * kGateCols;
            if (k + 1 < nslice) load_slice(c0 + kGateCols, t);  // in flight while slice k is used
            const float *xr = sX + (size_t(k & 1) * kGateRows + rr) * XP;
            const float *wr = sW + size_t(c0) * NOP + jh;
            const int ncol = C - c0 < kGateCols ? C - c0 : kGateCols;
#pragma unroll 8
            for (int cc = 0; cc < ncol; ++cc) {
                const float x = xr[cc];
                const float4 *w4 = reinterpret_cast<const float4 *>(wr + size_t(cc) * NOP);
#pragma unroll
                for (int q = 0; q < kGateHalf / 4; ++q) {
                    const float4 w = w4[q];
                    acc[4 * q] = fmaf(x, w.x, acc[4 * q]);
                    acc[4 * q + 1] = fmaf(x, w.y, acc[4 * q + 1]);
                    acc[4 * q + 2] = fmaf(x, w.z, acc[4 * q + 2]);
                    acc[4 * q + 3] = fmaf(x, w.w, acc[4 * q + 3]);
                }
            }
            if (k + 1 < nslice) store_slice((k + 1) & 1, t);  // the other buffer: nobody reads it now
            __syncthreads();
        }
        if (row < rows) {
#pragma unroll
            for (int j = 0; j < kGateHalf; ++j)
                if (jh + j < NO) gates[row * NO + jh + j] = 1.0f / (1.0f + expf(-acc[j]));
        }
    }
}

// ---------------------------------------------------------------------------
// Group scores and top-k: one CTA of 8 warps per (head, 8 consecutive
// groups), one warp per group.  The head's coarse keys are staged through
// shared memory kTopkKeys at a time (rows padded by one word: the lanes read
// different keys at the same element without bank conflicts) and shared by
// the 8 groups; each warp keeps its group's nb scores in shared memory and
// takes the top k by repeated warp argmax.
constexpr int kTopkWarps = 8, kTopkKeys = 256;

static size_t topk_smem_bytes(int D, int nb)
{
    return (size_t(kTopkKeys) * (D + 1) + size_t(kTopkWarps) * nb) * 4;
}

template <int D>
__global__ void __launch_bounds__(kTopkWarps * 32) k_bsa_topk(const float *__restrict__ qbar,
                                                             const float *__restrict__ kbar,
                                                             const int32_t *__restrict__ cnt, int nb, int H, int topk,
                                                             int mask_own, float scale, int32_t *__restrict__ sel)
{
    extern __shared__ __align__(16) float bsa_tsm[];
    constexpr int KP = D + 1;
    float *sK = bsa_tsm, *ssc = bsa_tsm + kTopkKeys * KP;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ngb = (nb + kTopkWarps - 1) / kTopkWarps;
    const int h = int(blockIdx.x) / ngb, g = (int(blockIdx.x) - h * ngb) * kTopkWarps + warp;
    const bool active = g < nb;
    float *sc = ssc + warp * nb;
    float q[D];
#pragma unroll
    for (int k = 0; k < D; ++k) q[k] = active ? qbar[(size_t(g) * H + h) * D + k] : 0.0f;
    const bool gvalid = active && cnt[g] > 0;
    for (int b0 = 0; b0 < nb; b0 += kTopkKeys) {
        const int nk = nb - b0 < kTopkKeys ? nb - b0 : kTopkKeys;
        __syncthreads();  // the previous key tile is consumed
        for (int i = threadIdx.x; i < nk * (D / 4); i += kTopkWarps * 32) {
            const int kk = i / (D / 4), u = i - kk * (D / 4);
            const float4 v = *reinterpret_cast<const float4 *>(kbar + (size_t(b0 + kk) * H + h) * D + 4 * u);
            float *dst = sK + kk * KP + 4 * u;
            dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
        }
        __syncthreads();
        if (active) {
            for (int kk = lane; kk < nk; kk += 32) {
                float acc = 0.0f;
#pragma unroll
                for (int k = 0; k < D; ++k) acc = fmaf(q[k], sK[kk * KP + k], acc);
                const int b = b0 + kk;
                const bool ok = gvalid && cnt[b] > 0 && !(mask_own && b == g);
                sc[b] = ok ? acc * scale : -INFINITY;
            }
        }
    }
    if (!active) return;  // no block-wide synchronisation below
    __syncwarp();
    const int64_t item = int64_t(g) * H + h;
    for (int t = 0; t < topk; ++t) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int b = lane; b < nb; b += 32) {
            const float v = sc[b];
            if (v > bv) {  // candidates are visited in increasing b: strict > keeps the lower index
                bv = v;
                bi = b;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) {
                bv = ov;
                bi = oi;
            }
        }
        const bool found = bv != -INFINITY;
        if (lane == 0) sel[item * topk + t] = found ? bi : -1;
        if (found && lane == (bi & 31)) sc[bi] = -INFINITY;
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// TMEM accesses of 16 / 8 consecutive 32-bit columns, one lane per thread (the load waits for its data).
__device__ __forceinline__ void bsa_tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void bsa_tmem_st8(uint32_t taddr, const uint32_t (&r)[8])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

template <int D>
struct BsaPipe {
    static constexpr uint32_t QK_BYTES = 128 * D * 2;
    static constexpr uint32_t Q_OFF = 0;
    static constexpr uint32_t STAGE_OFF = QK_BYTES;      // 2 stages of (K chunk, V chunk)
    static constexpr uint32_t STAGE = 2 * QK_BYTES;
    static constexpr uint32_t BYTES = STAGE_OFF + 2 * STAGE;
    static constexpr uint32_t COLS = D == 32 ? 128 : 256;
    static constexpr int PER_SM = D == 32 ? 4 : 2;
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, BsaPipe<D>::PER_SM)
    k_bsa_attn_tc(const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ K,
                  const __nv_bfloat16 *__restrict__ V, const int32_t *__restrict__ perm, int64_t rows, int H,
                  int nb, const __nv_bfloat16 *__restrict__ kc, const __nv_bfloat16 *__restrict__ vc,
                  const int32_t *__restrict__ cnt, const int32_t *__restrict__ sel, int topk,
                  const float *__restrict__ gates, const __nv_bfloat16 *__restrict__ Oball, float sl2,
                  __nv_bfloat16 *__restrict__ O, uint32_t *status)
{
    using L = BsaPipe<D>;
    constexpr int KCH = D / 8;
    constexpr int UPT = 128 * KCH / kTcThreads;
    constexpr uint32_t QK_SBO = KCH * 128, V_SBO = 16 * 128;
    constexpr uint32_t IDESC_S = idesc_bf16(128, false);
    constexpr uint32_t IDESC_O = idesc_bf16(D, true);
    extern __shared__ __align__(1024) uint8_t bsm[];
    __shared__ uint32_t sKeyMask[4];
    __shared__ int32_t sSel[kBsaMaxTopk];  // the item's selected balls
    __shared__ __align__(8) uint64_t sBarS, sBarO;
    __shared__ uint32_t sTmem;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t base = smem_u32(bsm);
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sTmem)),
                     "r"(L::COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sBarS)) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sBarO)) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sTmem, tS = tmem, tO = tmem + 64;
    const uint32_t barS = smem_u32(&sBarS), barO = smem_u32(&sBarO);
    const uint32_t lanebase = uint32_t(warp * 32) << 16;
    const int ncc = (nb + 127) / 128;  // compression chunks
    const int64_t items = int64_t(nb) * H;
    uint32_t nS = 0, nO = 0;  // completed waits per barrier (phase parity)
    bool ok = true;

    auto valid_row = [&](int32_t r) -> int32_t {
        if (r >= rows) {
            record_error(status, BT_ERR_INTERNAL);
            return -1;
        }
        return r;
    };
    // The source rows of a key chunk are fetched one chunk ahead (raw values: the ball's point count for a
    // compression key, the perm entry for a selected one) and decoded when the chunk is issued, so the loads
    // of perm and of the counts never stall the chunk in flight.
    auto chunk_live = [&](int c) -> bool { return c < ncc || sSel[c - ncc] >= 0; };
    auto fetch_raw = [&](int c, int r) -> int32_t {
        if (c >= ncc + topk || !chunk_live(c)) return -1;
        if (c < ncc) {
            const int t = c * 128 + r;
            return t < nb ? cnt[t] : 0;
        }
        const int64_t slot = int64_t(sSel[c - ncc]) * 128 + r;
        return perm ? perm[slot] : int32_t(slot);
    };
    auto decode = [&](int c, int r, int32_t raw) -> int32_t {
        if (c < ncc) return raw > 0 ? c * 128 + r : -1;
        return raw >= 0 ? valid_row(raw) : -1;
    };
    int32_t nraw[UPT], nkey;  // the next chunk's raw values: the rows this thread loads, and key row tid
    auto fetch_chunk = [&](int c) {
#pragma unroll
        for (int i = 0; i < UPT; ++i) nraw[i] = fetch_raw(c, (tid + i * kTcThreads) / KCH);
        nkey = fetch_raw(c, tid);
    };
    auto issue_chunk = [&](int h, int c) {
        if (c < ncc + topk && chunk_live(c)) {
            const bool cmp = c < ncc;
            const __nv_bfloat16 *kb = cmp ? kc : K, *vb = cmp ? vc : V;
            uint8_t *sk = bsm + L::STAGE_OFF + (c & 1) * L::STAGE, *sv = sk + L::QK_BYTES;
#pragma unroll
            for (int i = 0; i < UPT; ++i) {
                const int u = tid + i * kTcThreads;
                const int r = u / KCH, cc = u - r * KCH;
                const int32_t rr = decode(c, r, nraw[i]);
                const size_t goff = rr >= 0 ? (size_t(rr) * H + h) * D + cc * 8 : 0;
                cp_async16(sk + (r >> 3) * QK_SBO + cc * 128 + (r & 7) * 16, kb + goff, rr >= 0);
                cp_async16(sv + cc * V_SBO + r * 16, vb + goff, rr >= 0);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
        const int g = int(item / H), h = int(item - int64_t(g) * H);
        if (tid < topk) sSel[tid] = sel[(size_t(g) * H + h) * topk + tid];
        __syncthreads();  // the previous item's chunks are done with sSel
        // Q rows of the group (as the ball attention gathers them)
        {
            uint8_t *sq = bsm + L::Q_OFF;
#pragma unroll
            for (int i = 0; i < UPT; ++i) {
                const int u = tid + i * kTcThreads;
                const int r = u / KCH, cc = u - r * KCH;
                const int32_t rr = perm ? valid_row(perm[int64_t(g) * 128 + r]) : int32_t(int64_t(g) * 128 + r);
                const size_t goff = rr >= 0 ? (size_t(rr) * H + h) * D + cc * 8 : 0;
                cp_async16(sq + (r >> 3) * QK_SBO + cc * 128 + (r & 7) * 16, Q + goff, rr >= 0);
            }
        }
        fetch_chunk(0);
        issue_chunk(h, 0);  // committed together with Q
        int32_t ckey = nkey;  // key row tid of the chunk in flight
        fetch_chunk(1);
        float o_acc[D], o_cmp[D];
        float m_run = -INFINITY, l_run = 0.0f;
        const int nchunks = ncc + topk;
        for (int c = 0; c < nchunks; ++c) {
            issue_chunk(h, c + 1);
            const bool live = chunk_live(c);
            const int32_t kr = live ? decode(c, tid, ckey) : -1;
            ckey = nkey;
            fetch_chunk(c + 2);
            const uint32_t kb = __ballot_sync(0xffffffffu, kr >= 0);
            if (lane == 0) sKeyMask[warp] = kb;
            asm volatile("cp.async.wait_group 1;" ::: "memory");
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            if (c == 0 || c == ncc) {  // a new branch starts: reset the running softmax
                m_run = -INFINITY;
                l_run = 0.0f;
#pragma unroll
                for (int k = 0; k < D; ++k) o_acc[k] = 0.0f;
            }
            if (live) {
                const uint32_t sq = base + L::Q_OFF, sk = base + L::STAGE_OFF + (c & 1) * L::STAGE;
                const uint32_t sv = sk + L::QK_BYTES;
                if (tid == 0 && ok) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_bf16(tS, smem_desc(sq + kk * 256, 128, QK_SBO), smem_desc(sk + kk * 256, 128, QK_SBO),
                                 IDESC_S, kk > 0);
                    mma_commit(barS);
                }
                ok = ok && mbar_wait(barS, nS & 1, status);
                ++nS;
                tc_fence_after();
                uint32_t cmask[4];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) cmask[q4] = sKeyMask[q4];
                float mx = -INFINITY;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    if (cmask[q4] != 0u) {
                        uint32_t v[32];
                        tmem_ld32(tS + lanebase + q4 * 32, v);
                        if (cmask[q4] == 0xffffffffu) {  // every key of the group valid: three-input max
#pragma unroll
                            for (int j = 0; j < 32; j += 2)
                                mx = fmax3(mx, __uint_as_float(v[j]), __uint_as_float(v[j + 1]));
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if ((cmask[q4] >> j) & 1u) mx = fmaxf(mx, __uint_as_float(v[j]));
                        }
                    }
                }
                const float m_new = fmaxf(m_run, mx == -INFINITY ? -INFINITY : mx * sl2);
                const float mref = m_new == -INFINITY ? 0.0f : m_new;
                const float alpha = m_run == -INFINITY ? 0.0f : ex2(m_run - mref);
                float cs0 = 0.0f, cs1 = 0.0f;  // this chunk's row sum of the weights (even and odd keys)
#pragma unroll
                // sixteen keys at a time (the weights of 16 keys are 8 packed columns): few registers live
                for (int q8 = 0; q8 < 8; ++q8) {
                    uint32_t pk[8];
                    const uint32_t cm = (cmask[q8 >> 1] >> (16 * (q8 & 1))) & 0xFFFFu;
                    if (cm == 0xFFFFu) {  // every key valid: no per-key selects
                        uint32_t v[16];
                        bsa_tmem_ld16(tS + lanebase + q8 * 16, v);
#pragma unroll
                        for (int j = 0; j < 16; j += 2) {
                            float p0, p1;
                            ffma2_bcast(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), sl2, -mref, p0, p1);
                            p0 = ex2(p0);
                            p1 = ex2(p1);
                            const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                            pk[j >> 1] = *reinterpret_cast<const uint32_t *>(&pb);
                            fadd2_acc(cs0, cs1, p0, p1);
                        }
                    } else if (cm != 0u) {
                        uint32_t v[16];
                        bsa_tmem_ld16(tS + lanebase + q8 * 16, v);
#pragma unroll
                        for (int j = 0; j < 16; j += 2) {
                            float p0, p1;
                            ffma2_bcast(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), sl2, -mref, p0, p1);
                            p0 = ((cm >> j) & 1u) ? ex2(p0) : 0.0f;
                            p1 = ((cm >> (j + 1)) & 1u) ? ex2(p1) : 0.0f;
                            const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                            pk[j >> 1] = *reinterpret_cast<const uint32_t *>(&pb);
                            fadd2_acc(cs0, cs1, p0, p1);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j) pk[j] = 0u;
                    }
                    bsa_tmem_st8(tS + lanebase + q8 * 8, pk);
                }
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncthreads();
                tc_fence_after();
                if (tid == 0 && ok) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tO, tS + kk * 8, smem_desc(sv + kk * 256, 128, V_SBO), IDESC_O, kk > 0);
                    mma_commit(barO);
                }
                ok = ok && mbar_wait(barO, nO & 1, status);
                ++nO;
                tc_fence_after();
                if (ok) {
                    l_run = l_run * alpha + (cs0 + cs1);
#pragma unroll
                    for (int c32 = 0; c32 < D; c32 += 32) {
                        uint32_t o[32];
                        tmem_ld32(tO + lanebase + c32, o);
#pragma unroll
                        for (int k = 0; k < 32; ++k) o_acc[c32 + k] = o_acc[c32 + k] * alpha + __uint_as_float(o[k]);
                    }
                }
                m_run = m_new;
            }
            if (c == ncc - 1) {  // the compression branch is complete
                const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
#pragma unroll
                for (int k = 0; k < D; ++k) o_cmp[k] = o_acc[k] * inv;
            }
            tc_fence_before();
            __syncthreads();  // S/P, O and this stage are free before the next chunk
            tc_fence_after();
        }
        if (topk == 0) {
            m_run = -INFINITY;
            l_run = 0.0f;
        }
        // gated sum with the ball branch, scattered to the query's row
        const int32_t qrow = perm ? valid_row(perm[int64_t(g) * 128 + tid]) : int32_t(int64_t(g) * 128 + tid);
        if (qrow >= 0 && ok) {
            const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
            const float *gp = gates + (size_t(qrow) * H + h) * 3;
            const float g0 = gp[0], g1 = gp[1], g2 = gp[2];
            const __nv_bfloat16 *ob = Oball + (size_t(qrow) * H + h) * D;
            uint4 *dst = reinterpret_cast<uint4 *>(O + (size_t(qrow) * H + h) * D);
#pragma unroll
            for (int t = 0; t < D / 8; ++t) {
                const uint4 bw = *reinterpret_cast<const uint4 *>(ob + 8 * t);
                const uint32_t bwv[4] = {bw.x, bw.y, bw.z, bw.w};
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 bf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&bwv[e]));
                    const int k = 8 * t + 2 * e;
                    const float y0 = g0 * bf.x + g1 * o_cmp[k] + g2 * (o_acc[k] * inv);
                    const float y1 = g0 * bf.y + g1 * o_cmp[k + 1] + g2 * (o_acc[k + 1] * inv);
                    const __nv_bfloat162 pb = __floats2bfloat162_rn(y0, y1);
                    w[e] = *reinterpret_cast<const uint32_t *>(&pb);
                }
                dst[t] = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(L::COLS) : "memory");
    }
}

// ---------------------------------------------------------------------------
// Query coarsening ("BSA with group compression"): the compression and
// selection branches take the group's pooled query, so each (group, head)
// item is one query vector against the coarse tokens and then against the
// selected balls - matrix-vector work, on the CUDA cores.  One warp per item.
// Lanes form groups of D/8; a lane group takes one key per half-step, each lane
// 8 of its elements (16 bytes of the bf16 row), and keeps its own online
// softmax (log2 domain); the lane groups merge at the end of each branch.  The
// gated sum over the group's query rows follows in the same warp.
template <int G>
__device__ __forceinline__ float lane_group_sum(float s)
{
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// Two keys into one lane group's running softmax (m, l, acc); s0/s1 are the
// scaled logits (log2 domain), -inf for a missing key (its value row is zero).
__device__ __forceinline__ void softmax_push2(float s0, float s1, const float (&v0)[8], const float (&v1)[8], float &m,
                                              float &l, float (&acc)[8])
{
    const float mn = fmaxf(m, fmaxf(s0, s1));
    if (mn == -INFINITY) return;
    const float alpha = ex2(m - mn), p0 = ex2(s0 - mn), p1 = ex2(s1 - mn);
    l = fmaf(l, alpha, p0 + p1);
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = fmaf(acc[k], alpha, fmaf(p0, v0[k], p1 * v1[k]));
    m = mn;
}

// Merge the lane groups' softmax states (lanes with the same element slice):
// afterwards every lane holds the warp's max M, its sum L and its un-normalised
// accumulator for the lane's element slice, all relative to M.
template <int G>
__device__ __forceinline__ void softmax_warp_merge(float &m, float &l, float (&acc)[8])
{
    float M = m;
#pragma unroll
    for (int o = G; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float f = M == -INFINITY ? 0.0f : ex2(m - M);
    l *= f;
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] *= f;
#pragma unroll
    for (int o = G; o < 32; o <<= 1) {
        l += __shfl_xor_sync(0xffffffffu, l, o);
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], o);
    }
    m = M;
}

// One CTA of kCoarseWarps warps per (group, head) item.  The warps split the
// coarse tokens (by half-steps) and the selected balls (one ball at a time),
// merge their softmax states through shared memory, and split the group's
// query rows for the gated sum.
constexpr int kCoarseWarps = 4;

template <int D>
__global__ void __launch_bounds__(kCoarseWarps * 32) k_bsa_coarse(const __nv_bfloat16 *__restrict__ K,
                                                                  const __nv_bfloat16 *__restrict__ V,
                                                                  const int32_t *__restrict__ perm, int64_t rows,
                                                                  int H, int nb, const float *__restrict__ qbar,
                                                                  const __nv_bfloat16 *__restrict__ kc,
                                                                  const __nv_bfloat16 *__restrict__ vc,
                                                                  const int32_t *__restrict__ cnt,
                                                                  const int32_t *__restrict__ sel, int topk,
                                                                  const float *__restrict__ gates,
                                                                  const __nv_bfloat16 *__restrict__ Oball, float sl2,
                                                                  __nv_bfloat16 *__restrict__ O, uint32_t *status)
{
    constexpr int G = D / 8, KPS = 32 / G;  // lanes per key, keys per half-step
    constexpr int NW = kCoarseWarps;
    __shared__ float sM[2][NW], sL[2][NW];
    __shared__ __align__(16) float sAcc[2][NW][D];
    __shared__ __align__(16) float sOut[2][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t item = blockIdx.x;
    const int g = int(item / H), h = int(item - int64_t(g) * H);
    const int sub = lane % G, kslot = lane / G;  // elements [8 sub, 8 sub + 8) of key kslot of each half-step
    const size_t hoff = size_t(h) * D + sub * 8, rstride = size_t(H) * D;
    float q[8];
    {
        const float4 *qp = reinterpret_cast<const float4 *>(qbar + size_t(g) * rstride + hoff);
        const float4 a = qp[0], b = qp[1];
        q[0] = a.x; q[1] = a.y; q[2] = a.z; q[3] = a.w;
        q[4] = b.x; q[5] = b.y; q[6] = b.z; q[7] = b.w;
    }
    auto logit = [&](const uint4 kw, bool valid) -> float {
        float kf[8];
        bf16x8_to_f32(kw, kf);
        float s = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) s = fmaf(q[k], kf[k], s);
        s = lane_group_sum<G>(s);  // every lane of the warp takes part
        return valid ? s * sl2 : -INFINITY;
    };
    auto publish = [&](int br, float m, float l, float (&acc)[8]) {
        softmax_warp_merge<G>(m, l, acc);
        if (kslot == 0) {
#pragma unroll
            for (int k = 0; k < 8; ++k) sAcc[br][warp][sub * 8 + k] = acc[k];
        }
        if (lane == 0) {
            sM[br][warp] = m;
            sL[br][warp] = l;
        }
    };
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);

    // Loads are batched: BI half-step pairs (2*BI keys per lane) are fetched before any is used, and the
    // row indices of a batch before its K/V rows, so a batch costs two round trips to memory.
    constexpr int BI = 2;
    // compression branch: the coarse tokens of balls with a real point; warp w takes half-step pairs w, w+NW, ...
    {
        float m = -INFINITY, l = 0.0f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int base = 2 * warp * KPS; base < nb; base += BI * 2 * NW * KPS) {
            uint4 kk[2 * BI], vv[2 * BI];
            bool ok[2 * BI];
#pragma unroll
            for (int u = 0; u < 2 * BI; ++u) {
                const int b = base + (u >> 1) * 2 * NW * KPS + (u & 1) * KPS + kslot;
                const bool in = b < nb;
                ok[u] = in && cnt[b] > 0;  // the coarse rows exist for every ball: loaded regardless
                kk[u] = in ? *reinterpret_cast<const uint4 *>(kc + size_t(b) * rstride + hoff) : zero;
                vv[u] = in ? *reinterpret_cast<const uint4 *>(vc + size_t(b) * rstride + hoff) : zero;
            }
#pragma unroll
            for (int u = 0; u < BI; ++u) {
                const float s0 = logit(kk[2 * u], ok[2 * u]), s1 = logit(kk[2 * u + 1], ok[2 * u + 1]);
                float v0[8], v1[8];
                bf16x8_to_f32(vv[2 * u], v0);
                bf16x8_to_f32(vv[2 * u + 1], v1);
                softmax_push2(s0, s1, v0, v1, m, l, acc);
            }
        }
        publish(0, m, l, acc);
    }
    // selection branch: the real rows of the selected balls; warp w takes balls w, w+NW, ...
    {
        constexpr int RPL = 128 / KPS;  // rows of a ball per lane
        float m = -INFINITY, l = 0.0f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int t = warp; t < topk; t += NW) {
            const int s = sel[(size_t(g) * H + h) * topk + t];
            if (s < 0) continue;  // uniform across the warp
            if (s >= nb) {
                record_error(status, BT_ERR_INTERNAL);
                continue;
            }
            for (int i0 = 0; i0 < RPL; i0 += 2 * BI) {
                int32_t rw[2 * BI];
#pragma unroll
                for (int u = 0; u < 2 * BI; ++u) {
                    const int64_t j = int64_t(s) * 128 + kslot + KPS * (i0 + u);
                    int32_t row = perm ? perm[j] : int32_t(j);
                    if (row >= rows) {
                        record_error(status, BT_ERR_INTERNAL);
                        row = -1;
                    }
                    rw[u] = row;
                }
                uint4 kk[2 * BI], vv[2 * BI];
#pragma unroll
                for (int u = 0; u < 2 * BI; ++u) {
                    kk[u] = rw[u] >= 0 ? *reinterpret_cast<const uint4 *>(K + size_t(rw[u]) * rstride + hoff) : zero;
                    vv[u] = rw[u] >= 0 ? *reinterpret_cast<const uint4 *>(V + size_t(rw[u]) * rstride + hoff) : zero;
                }
#pragma unroll
                for (int u = 0; u < BI; ++u) {
                    const float s0 = logit(kk[2 * u], rw[2 * u] >= 0), s1 = logit(kk[2 * u + 1], rw[2 * u + 1] >= 0);
                    float v0[8], v1[8];
                    bf16x8_to_f32(vv[2 * u], v0);
                    bf16x8_to_f32(vv[2 * u + 1], v1);
                    softmax_push2(s0, s1, v0, v1, m, l, acc);
                }
            }
        }
        publish(1, m, l, acc);
    }
    __syncthreads();
    // merge the warps: one thread per (branch, element)
    if (threadIdx.x < 2 * D) {
        const int br = threadIdx.x / D, k = threadIdx.x - br * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, sM[br][w]);
        float L = 0.0f, A = 0.0f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float f = ex2(sM[br][w] - M);  // a warp without keys has M_w = -inf: weight 0
                L = fmaf(sL[br][w], f, L);
                A = fmaf(sAcc[br][w][k], f, A);
            }
        }
        sOut[br][k] = L > 0.0f ? A / L : 0.0f;
    }
    __syncthreads();
    float ocmp[8], oslc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        ocmp[k] = sOut[0][sub * 8 + k];
        oslc[k] = sOut[1][sub * 8 + k];
    }
    // gated sum with the ball branch for every real query row of the group; warp w takes rows w*KPS + kslot, ...
    constexpr int ITE = 128 / (NW * KPS);
    int32_t qr[ITE];
#pragma unroll
    for (int it = 0; it < ITE; ++it) {
        const int r = it * NW * KPS + warp * KPS + kslot;
        int32_t qrow = perm ? perm[int64_t(g) * 128 + r] : int32_t(int64_t(g) * 128 + r);
        if (qrow >= rows) {
            record_error(status, BT_ERR_INTERNAL);
            qrow = -1;
        }
        qr[it] = qrow;
    }
#pragma unroll
    for (int it = 0; it < ITE; ++it) {
        const int32_t qrow = qr[it];
        if (qrow < 0) continue;
        const float *gp = gates + (size_t(qrow) * H + h) * 3;
        const float g0 = gp[0], g1 = gp[1], g2 = gp[2];
        float ob[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4 *>(Oball + size_t(qrow) * rstride + hoff), ob);
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int k = 2 * e;
            const float y0 = g0 * ob[k] + g1 * ocmp[k] + g2 * oslc[k];
            const float y1 = g0 * ob[k + 1] + g1 * ocmp[k + 1] + g2 * oslc[k + 1];
            const __nv_bfloat162 pb = __floats2bfloat162_rn(y0, y1);
            w[e] = *reinterpret_cast<const uint32_t *>(&pb);
        }
        *reinterpret_cast<uint4 *>(O + size_t(qrow) * rstride + hoff) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// ---------------------------------------------------------------------------
struct BsaLayout {
    size_t qbar, kbar, kc, vc, cnt, sel, gates, oball, total;
};

static size_t al256(size_t v) { return (v + 255) & ~size_t(255); }

static BsaLayout bsa_layout(int64_t nb, int64_t rows, int H, int d, int topk)
{
    BsaLayout L{};
    const size_t hd = size_t(H) * d;
    L.qbar = 0;
    L.kbar = al256(L.qbar + nb * hd * 4);
    L.kc = al256(L.kbar + nb * hd * 4);
    L.vc = al256(L.kc + nb * hd * 2);
    L.cnt = al256(L.vc + nb * hd * 2);
    L.sel = al256(L.cnt + nb * 4);
    L.gates = al256(L.sel + nb * H * (topk > 0 ? topk : 1) * 4);
    L.oball = al256(L.gates + rows * H * 3 * 4);
    L.total = al256(L.oball + rows * hd * 2);
    return L;
}

static bt_status bsa_check(int64_t npad, int64_t rows, int32_t m, int32_t H, int32_t d, int32_t topk, int32_t C)
{
    if (npad < 1 || rows < 1 || H < 1 || C < 1) return BT_ERR_ARG;
    if (m != 128 || npad % m || (d != 32 && d != 64)) return BT_ERR_SHAPE;
    if (topk < 0 || topk > kBsaMaxTopk || npad / m > kBsaMaxBalls || H > 64 || C > 2048) return BT_ERR_UNSUPPORTED;
    if (gate_smem_bytes(C, H) > 200 * 1024) return BT_ERR_UNSUPPORTED;
    return BT_OK;
}

}  // namespace bts

extern "C" size_t bsa_workspace_size(int64_t npad, int64_t rows, int32_t m, int32_t H, int32_t d, int32_t topk)
{
    if (bts::bsa_check(npad, rows, m, H, d, topk, 1) != BT_OK) return 0;
    return bts::bsa_layout(npad / m, rows, H, d, topk).total;
}

template <int D>
static bt_status bsa_launch(const void *Q, const void *K, const void *V, const int32_t *perm, int64_t npad,
                            int64_t rows, int H, const float *X, int C, const float *Wg, const float *bg,
                            bsa_params p, void *O, int32_t *sel_out, uint8_t *w, cudaStream_t st)
{
    using namespace bts;
    const int nb = int(npad / 128);
    const BsaLayout Lw = bsa_layout(nb, rows, H, D, p.topk);
    float *qbar = reinterpret_cast<float *>(w + Lw.qbar), *kbar = reinterpret_cast<float *>(w + Lw.kbar);
    __nv_bfloat16 *kc = reinterpret_cast<__nv_bfloat16 *>(w + Lw.kc), *vc = reinterpret_cast<__nv_bfloat16 *>(w + Lw.vc);
    int32_t *cnt = reinterpret_cast<int32_t *>(w + Lw.cnt);
    int32_t *sel = sel_out ? sel_out : reinterpret_cast<int32_t *>(w + Lw.sel);
    float *gates = reinterpret_cast<float *>(w + Lw.gates);
    __nv_bfloat16 *oball = reinterpret_cast<__nv_bfloat16 *>(w + Lw.oball);
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(Q), *k = static_cast<const __nv_bfloat16 *>(K),
                        *v = static_cast<const __nv_bfloat16 *>(V);

    static std::atomic<bool> set[64] = {};
    static int sms[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BT_ERR_CUDA;
    auto init = [&]() -> bt_status {
        if (cudaFuncSetAttribute(k_bsa_attn_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(BsaPipe<D>::BYTES)) ||
            cudaFuncSetAttribute(k_bsa_gates, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) ||
            cudaFuncSetAttribute(k_bsa_topk<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(topk_smem_bytes(D, int(kBsaMaxBalls)))))
            return BT_ERR_CUDA;
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return BT_ERR_CUDA;
        if (dev >= 0 && dev < 64) sms[dev] = n;
        return BT_OK;
    };
    const bt_status s0 = (dev >= 0 && dev < 64) ? setup_once(set[dev], init) : init();
    if (s0 != BT_OK) return s0;
    const int nsm = dev < 64 && sms[dev] > 0 ? sms[dev] : 148;
    uint32_t *status = stream_status(st);
    if (!status) return BT_ERR_CUDA;
    k_bsa_means<<<nb, kMeanWarps * 32, 0, st>>>(q, k, v, perm, rows, H * D, qbar, kbar, kc, vc, cnt, status);
    k_bsa_gates<<<unsigned((rows + kGateRows - 1) / kGateRows), kGateThreads, gate_smem_bytes(C, H), st>>>(
        X, rows, C, Wg, bg, H, gate_out_padded(H), gates);
    if (p.topk > 0)
        k_bsa_topk<D><<<unsigned(int64_t(H) * ((nb + kTopkWarps - 1) / kTopkWarps)), kTopkWarps * 32,
                        topk_smem_bytes(D, nb), st>>>(
            qbar, kbar, cnt, nb, H, p.topk, p.mask_own_ball, 1.0f / sqrtf(float(D)), sel);
    bt_status s = (D == 32 && H % 2 == 0 && rows < 0x7FFFFFFF) ? launch_pair(Q, K, V, perm, npad, rows, 7, H, oball, st)
                                                               : launch_tc<D>(Q, K, V, perm, npad, rows, 7, H, oball, st);
    if (s != BT_OK) return s;
    const int64_t items = int64_t(nb) * H;
    if (p.coarsen_queries) {
        k_bsa_coarse<D><<<unsigned(items), kCoarseWarps * 32, 0, st>>>(
            k, v, perm, rows, H, nb, qbar, kc, vc, cnt, sel, p.topk, gates, oball,
            1.4426950408889634f / sqrtf(float(D)), static_cast<__nv_bfloat16 *>(O), status);
        return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
    }
    const int64_t grid = items < int64_t(nsm) * BsaPipe<D>::PER_SM ? items : int64_t(nsm) * BsaPipe<D>::PER_SM;
    k_bsa_attn_tc<D><<<unsigned(grid), kTcThreads, BsaPipe<D>::BYTES, st>>>(
        q, k, v, perm, rows, H, nb, kc, vc, cnt, sel, p.topk, gates, oball, 1.4426950408889634f / sqrtf(float(D)),
        static_cast<__nv_bfloat16 *>(O), status);
    return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
}

extern "C" bt_status bsa_forward(const void *Q, const void *K, const void *V, const int32_t *perm, int64_t npad,
                                 int64_t rows, int32_t m, int32_t H, int32_t d, bt_dtype dt, const float *X,
                                 int32_t C, const float *Wg, const float *bg, bsa_params p, void *O,
                                 int32_t *sel_out, void *ws, size_t ws_bytes, void *stream)
{
    using namespace bts;
    if (!Q || !K || !V || !O || !X || !Wg) return BT_ERR_ARG;
    if (dt != BT_BF16) return BT_ERR_UNSUPPORTED;
    const bt_status s = bsa_check(npad, rows, m, H, d, p.topk, C);
    if (s != BT_OK) return s;
    if (!perm && rows < npad) return BT_ERR_ARG;
    const uintptr_t al = reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) |
                         reinterpret_cast<uintptr_t>(V) | reinterpret_cast<uintptr_t>(O);
    if (al % 16 || (reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(Wg)) % 4) return BT_ERR_ARG;
    if (!ws || reinterpret_cast<uintptr_t>(ws) % 256) return BT_ERR_WORKSPACE;
    if (ws_bytes < bsa_layout(npad / m, rows, H, d, p.topk).total) return BT_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *w = static_cast<uint8_t *>(ws);
    return d == 32 ? bsa_launch<32>(Q, K, V, perm, npad, rows, H, X, C, Wg, bg, p, O, sel_out, w, st)
                   : bsa_launch<64>(Q, K, V, perm, npad, rows, H, X, C, Wg, bg, p, O, sel_out, w, st);
}
