// Ball Sparse Attention (page: Pith review of "BSA: Ball Sparse Attention for
// Large-scale Geometries": reading notes and referee report; figure 1 caption).
// Three branches per query, mixed by per-head sigmoid gates:
//   ball        - attention inside the query's own ball (k_ball_attn_tc2);
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
//   k_bsa_gates    32 rows per CTA, W and the X tile in shared memory.
//   k_bsa_topk     one warp per (group, head): scores from the pooled query and
//                  the f32 coarse keys, own ball and empty balls masked, top-k.
//   k_bsa_attn_tc  persistent tcgen05 kernel over (group, head) items: the
//                  compression and selection branches as flash-style online
//                  softmax over chunks of 128 keys (S and P in TMEM, P V and
//                  the row sums on the tensor core), then the gated sum with
//                  the ball branch, scattered through perm.
//   k_bsa_coarse   the query-coarsening variant of the two branches: one warp
//                  per (group, head) with the pooled query, then the gated sum.
// This file is included by bts_attn.cu (one translation unit with the ball
// attention kernel and the attention status word).
#pragma once

namespace bts {

constexpr int kBsaMaxTopk = 32;
constexpr int64_t kBsaMaxBalls = 2048;

// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) k_bsa_means(const __nv_bfloat16 *__restrict__ Q,
                                                   const __nv_bfloat16 *__restrict__ K,
                                                   const __nv_bfloat16 *__restrict__ V,
                                                   const int32_t *__restrict__ perm, int64_t rows, int H,
                                                   float *__restrict__ qbar, float *__restrict__ kbar,
                                                   __nv_bfloat16 *__restrict__ kc, __nv_bfloat16 *__restrict__ vc,
                                                   int32_t *__restrict__ cnt)
{
    constexpr int M = 128;
    __shared__ int32_t srow[M];
    __shared__ int s_cnt;
    const int tid = threadIdx.x;
    const int64_t b = blockIdx.x;
    if (tid == 0) s_cnt = 0;
    __syncthreads();
    {
        int32_t r = perm ? perm[b * M + tid] : int32_t(b * M + tid);
        if (r >= rows) {
            record_error(&g_attn_status, BT_ERR_INTERNAL);
            r = -1;
        }
        srow[tid] = r;
        const uint32_t vb = __ballot_sync(0xffffffffu, r >= 0);
        if ((tid & 31) == 0) atomicAdd(&s_cnt, __popc(vb));
    }
    __syncthreads();
    const int n = s_cnt;
    const int HD = H * D;
    const float inv = n > 0 ? 1.0f / float(n) : 0.0f;
    for (int t = 2 * tid; t < HD; t += 2 * M) {
        float q0 = 0.f, q1 = 0.f, k0 = 0.f, k1 = 0.f, v0 = 0.f, v1 = 0.f;
#pragma unroll 4
        for (int j = 0; j < M; ++j) {
            const int32_t r = srow[j];
            if (r < 0) continue;
            const size_t off = size_t(r) * HD + t;
            const float2 qf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(Q + off));
            const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(K + off));
            const float2 vf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(V + off));
            q0 += qf.x; q1 += qf.y; k0 += kf.x; k1 += kf.y; v0 += vf.x; v1 += vf.y;
        }
        const size_t o = size_t(b) * HD + t;
        qbar[o] = q0 * inv; qbar[o + 1] = q1 * inv;
        kbar[o] = k0 * inv; kbar[o + 1] = k1 * inv;
        *reinterpret_cast<__nv_bfloat162 *>(kc + o) = __floats2bfloat162_rn(k0 * inv, k1 * inv);
        *reinterpret_cast<__nv_bfloat162 *>(vc + o) = __floats2bfloat162_rn(v0 * inv, v1 * inv);
    }
    if (tid == 0) cnt[b] = n;
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_bsa_gates(const float *__restrict__ X, int64_t rows, int C,
                                                   const float *__restrict__ W, const float *__restrict__ bg, int H,
                                                   float *__restrict__ gates)
{
    extern __shared__ __align__(16) float gsm[];
    const int NO = 3 * H, CP = C + 1;  // X rows padded by one word against bank conflicts
    float *sW = gsm, *sX = gsm + C * NO;
    const int tid = threadIdx.x;
    for (int i = tid; i < C * NO; i += 256) sW[i] = W[i];
    const int64_t r0 = int64_t(blockIdx.x) * 32;
    for (int i = tid; i < 32 * C; i += 256) {
        const int rr = i / C, c = i - rr * C;
        sX[rr * CP + c] = (r0 + rr < rows) ? X[(r0 + rr) * C + c] : 0.0f;
    }
    __syncthreads();
    const int rr = tid >> 3;
    if (r0 + rr >= rows) return;
    for (int j = tid & 7; j < NO; j += 8) {
        float acc = bg ? bg[j] : 0.0f;
        for (int c = 0; c < C; ++c) acc = fmaf(sX[rr * CP + c], sW[c * NO + j], acc);
        gates[(r0 + rr) * NO + j] = 1.0f / (1.0f + expf(-acc));
    }
}

// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) k_bsa_topk(const float *__restrict__ qbar, const float *__restrict__ kbar,
                                                  const int32_t *__restrict__ cnt, int nb, int H, int topk,
                                                  int mask_own, float scale, int32_t *__restrict__ sel)
{
    extern __shared__ float ssc[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t item = int64_t(blockIdx.x) * 4 + warp;
    if (item >= int64_t(nb) * H) return;  // no block-wide synchronisation below
    const int g = int(item / H), h = int(item - int64_t(g) * H);
    float *sc = ssc + warp * nb;
    float q[D];
#pragma unroll
    for (int k = 0; k < D; ++k) q[k] = qbar[(size_t(g) * H + h) * D + k];
    const bool gvalid = cnt[g] > 0;
    for (int b = lane; b < nb; b += 32) {
        const float4 *kp = reinterpret_cast<const float4 *>(kbar + (size_t(b) * H + h) * D);
        float acc = 0.0f;
#pragma unroll
        for (int k4 = 0; k4 < D / 4; ++k4) {
            const float4 kv = kp[k4];
            acc = fmaf(q[4 * k4], kv.x, acc);
            acc = fmaf(q[4 * k4 + 1], kv.y, acc);
            acc = fmaf(q[4 * k4 + 2], kv.z, acc);
            acc = fmaf(q[4 * k4 + 3], kv.w, acc);
        }
        const bool ok = gvalid && cnt[b] > 0 && !(mask_own && b == g);
        sc[b] = ok ? acc * scale : -INFINITY;
    }
    __syncwarp();
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
template <int D>
struct BsaPipe {
    static constexpr uint32_t QK_BYTES = 128 * D * 2;
    static constexpr uint32_t Q_OFF = 0;
    static constexpr uint32_t STAGE_OFF = QK_BYTES;      // 2 stages of (K chunk, V chunk)
    static constexpr uint32_t STAGE = 2 * QK_BYTES;
    static constexpr uint32_t ONES_OFF = STAGE_OFF + 2 * STAGE;
    static constexpr uint32_t BYTES = ONES_OFF + 16 * 128 * 2;
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
                  __nv_bfloat16 *__restrict__ O)
{
    using L = BsaPipe<D>;
    constexpr int KCH = D / 8;
    constexpr int UPT = 128 * KCH / kTcThreads;
    constexpr uint32_t QK_SBO = KCH * 128, V_SBO = 16 * 128, ONES_SBO = 16 * 128;
    constexpr uint32_t IDESC_S = idesc_bf16(128, false);
    constexpr uint32_t IDESC_O = idesc_bf16(D, true);
    constexpr uint32_t IDESC_SUM = idesc_bf16(16, false);
    extern __shared__ __align__(1024) uint8_t bsm[];
    __shared__ uint32_t sKeyMask[4];
    __shared__ __align__(8) uint64_t sBarS, sBarO;
    __shared__ uint32_t sTmem;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t base = smem_u32(bsm);
    for (int i = tid; i < 16 * 128 * 2 / 16; i += kTcThreads) {
        const int c = i >> 4, rr = i & 15;
        const uint32_t off = (rr >> 3) * ONES_SBO + c * 128 + (rr & 7) * 16;
        const uint32_t one = (rr == 0) ? 0x3F803F80u : 0u;
        *reinterpret_cast<uint4 *>(bsm + L::ONES_OFF + off) = make_uint4(one, one, one, one);
    }
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
    const uint32_t tmem = sTmem, tS = tmem, tO = tmem + 64, tSum = tmem + 64 + D;
    const uint32_t barS = smem_u32(&sBarS), barO = smem_u32(&sBarO);
    const uint32_t lanebase = uint32_t(warp * 32) << 16;
    const int ncc = (nb + 127) / 128;  // compression chunks
    const int64_t items = int64_t(nb) * H;
    uint32_t nS = 0, nO = 0;  // completed waits per barrier (phase parity)
    bool ok = true;

    auto valid_row = [&](int32_t r) -> int32_t {
        if (r >= rows) {
            record_error(&g_attn_status, BT_ERR_INTERNAL);
            return -1;
        }
        return r;
    };
    // row r (0..127) of key chunk c of item (g, h): its source row, or -1
    auto chunk_row = [&](int g, int h, int c, int r) -> int32_t {
        if (c < ncc) {
            const int t = c * 128 + r;
            return (t < nb && cnt[t] > 0) ? t : -1;
        }
        const int s = sel[(size_t(g) * H + h) * topk + (c - ncc)];
        if (s < 0) return -1;
        return perm ? valid_row(perm[int64_t(s) * 128 + r]) : int32_t(int64_t(s) * 128 + r);
    };
    auto chunk_live = [&](int g, int h, int c) -> bool {
        return c < ncc || sel[(size_t(g) * H + h) * topk + (c - ncc)] >= 0;
    };
    auto issue_chunk = [&](int g, int h, int c) {
        if (c < ncc + topk && chunk_live(g, h, c)) {
            const bool cmp = c < ncc;
            const __nv_bfloat16 *kb = cmp ? kc : K, *vb = cmp ? vc : V;
            uint8_t *sk = bsm + L::STAGE_OFF + (c & 1) * L::STAGE, *sv = sk + L::QK_BYTES;
#pragma unroll
            for (int i = 0; i < UPT; ++i) {
                const int u = tid + i * kTcThreads;
                const int r = u / KCH, cc = u - r * KCH;
                const int32_t rr = chunk_row(g, h, c, r);
                const size_t goff = rr >= 0 ? (size_t(rr) * H + h) * D + cc * 8 : 0;
                cp_async16(sk + (r >> 3) * QK_SBO + cc * 128 + (r & 7) * 16, kb + goff, rr >= 0);
                cp_async16(sv + cc * V_SBO + r * 16, vb + goff, rr >= 0);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
        const int g = int(item / H), h = int(item - int64_t(g) * H);
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
        issue_chunk(g, h, 0);  // committed together with Q
        float o_acc[D], o_cmp[D];
        float m_run = -INFINITY, l_run = 0.0f;
        const int nchunks = ncc + topk;
        for (int c = 0; c < nchunks; ++c) {
            issue_chunk(g, h, c + 1);
            const bool live = chunk_live(g, h, c);
            const int32_t kr = live ? chunk_row(g, h, c, tid) : -1;
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
                ok = ok && mbar_wait(barS, nS & 1);
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
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if ((cmask[q4] >> j) & 1u) mx = fmaxf(mx, __uint_as_float(v[j]));
                    }
                }
                const float m_new = fmaxf(m_run, mx == -INFINITY ? -INFINITY : mx * sl2);
                const float mref = m_new == -INFINITY ? 0.0f : m_new;
                const float alpha = m_run == -INFINITY ? 0.0f : ex2(m_run - mref);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t pk[16];
                    if (cmask[q4] != 0u) {
                        uint32_t v[32];
                        tmem_ld32(tS + lanebase + q4 * 32, v);
                        const uint32_t cm = cmask[q4];
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            float p0 = ex2(fmaf(__uint_as_float(v[j]), sl2, -mref));
                            float p1 = ex2(fmaf(__uint_as_float(v[j + 1]), sl2, -mref));
                            p0 = ((cm >> j) & 1u) ? p0 : 0.0f;
                            p1 = ((cm >> (j + 1)) & 1u) ? p1 : 0.0f;
                            const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                            pk[j >> 1] = *reinterpret_cast<const uint32_t *>(&pb);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) pk[j] = 0u;
                    }
                    tmem_st16(tS + lanebase + q4 * 16, pk);
                }
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncthreads();
                tc_fence_after();
                if (tid == 0 && ok) {
                    const uint32_t so1 = base + L::ONES_OFF;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        mma_bf16_ts(tO, tS + kk * 8, smem_desc(sv + kk * 256, 128, V_SBO), IDESC_O, kk > 0);
                        mma_bf16_ts(tSum, tS + kk * 8, smem_desc(so1 + kk * 256, 128, ONES_SBO), IDESC_SUM, kk > 0);
                    }
                    mma_commit(barO);
                }
                ok = ok && mbar_wait(barO, nO & 1);
                ++nO;
                tc_fence_after();
                if (ok) {
                    uint32_t sb;
                    tmem_ld1(tSum + lanebase, sb);
                    l_run = l_run * alpha + __uint_as_float(sb);
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

// Merge the lane groups' softmax states (lanes with the same element slice)
// and normalise: out = sum p v / sum p, zero when no key was valid.
template <int G>
__device__ __forceinline__ void softmax_merge(float m, float l, const float (&acc)[8], float (&out)[8])
{
    float M = m;
#pragma unroll
    for (int o = G; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float f = M == -INFINITY ? 0.0f : ex2(m - M);
    float L = l * f;
#pragma unroll
    for (int k = 0; k < 8; ++k) out[k] = acc[k] * f;
#pragma unroll
    for (int o = G; o < 32; o <<= 1) {
        L += __shfl_xor_sync(0xffffffffu, L, o);
#pragma unroll
        for (int k = 0; k < 8; ++k) out[k] += __shfl_xor_sync(0xffffffffu, out[k], o);
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) out[k] *= inv;
}

template <int D>
__global__ void __launch_bounds__(128) k_bsa_coarse(const __nv_bfloat16 *__restrict__ K,
                                                    const __nv_bfloat16 *__restrict__ V,
                                                    const int32_t *__restrict__ perm, int64_t rows, int H, int nb,
                                                    const float *__restrict__ qbar,
                                                    const __nv_bfloat16 *__restrict__ kc,
                                                    const __nv_bfloat16 *__restrict__ vc,
                                                    const int32_t *__restrict__ cnt, const int32_t *__restrict__ sel,
                                                    int topk, const float *__restrict__ gates,
                                                    const __nv_bfloat16 *__restrict__ Oball, float sl2,
                                                    __nv_bfloat16 *__restrict__ O)
{
    constexpr int G = D / 8, KPS = 32 / G;  // lanes per key, keys per half-step
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t item = int64_t(blockIdx.x) * 4 + warp;
    if (item >= int64_t(nb) * H) return;  // no block-wide synchronisation below
    const int g = int(item / H), h = int(item - int64_t(g) * H);
    const int sub = lane % G, kslot = lane / G;
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
        s = lane_group_sum<G>(s);  // every lane takes part: no early exit before this
        return valid ? s * sl2 : -INFINITY;
    };
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);

    // compression branch: every coarse token of a ball with a real point
    float ocmp[8], oslc[8];
    {
        float m = -INFINITY, l = 0.0f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int b0 = kslot; b0 - kslot < nb; b0 += 2 * KPS) {
            const int b1 = b0 + KPS;
            const bool ok0 = b0 < nb && cnt[b0] > 0, ok1 = b1 < nb && cnt[b1] > 0;
            const uint4 k0 = ok0 ? *reinterpret_cast<const uint4 *>(kc + size_t(b0) * rstride + hoff) : zero;
            const uint4 k1 = ok1 ? *reinterpret_cast<const uint4 *>(kc + size_t(b1) * rstride + hoff) : zero;
            const uint4 w0 = ok0 ? *reinterpret_cast<const uint4 *>(vc + size_t(b0) * rstride + hoff) : zero;
            const uint4 w1 = ok1 ? *reinterpret_cast<const uint4 *>(vc + size_t(b1) * rstride + hoff) : zero;
            const float s0 = logit(k0, ok0), s1 = logit(k1, ok1);
            float v0[8], v1[8];
            bf16x8_to_f32(w0, v0);
            bf16x8_to_f32(w1, v1);
            softmax_push2(s0, s1, v0, v1, m, l, acc);
        }
        softmax_merge<G>(m, l, acc, ocmp);
    }
    // selection branch: the real rows of the selected balls, at full resolution
    {
        float m = -INFINITY, l = 0.0f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int t = 0; t < topk; ++t) {
            const int s = sel[(size_t(g) * H + h) * topk + t];
            if (s < 0) continue;  // uniform across the warp
            if (s >= nb) {
                record_error(&g_attn_status, BT_ERR_INTERNAL);
                continue;
            }
#pragma unroll 2
            for (int r0 = kslot; r0 < 128; r0 += 2 * KPS) {
                const int64_t j0 = int64_t(s) * 128 + r0, j1 = j0 + KPS;
                int32_t row0 = perm ? perm[j0] : int32_t(j0), row1 = perm ? perm[j1] : int32_t(j1);
                if (row0 >= rows || row1 >= rows) {
                    record_error(&g_attn_status, BT_ERR_INTERNAL);
                    row0 = row0 >= rows ? -1 : row0;
                    row1 = row1 >= rows ? -1 : row1;
                }
                const bool ok0 = row0 >= 0, ok1 = row1 >= 0;
                const uint4 k0 = ok0 ? *reinterpret_cast<const uint4 *>(K + size_t(row0) * rstride + hoff) : zero;
                const uint4 k1 = ok1 ? *reinterpret_cast<const uint4 *>(K + size_t(row1) * rstride + hoff) : zero;
                const uint4 w0 = ok0 ? *reinterpret_cast<const uint4 *>(V + size_t(row0) * rstride + hoff) : zero;
                const uint4 w1 = ok1 ? *reinterpret_cast<const uint4 *>(V + size_t(row1) * rstride + hoff) : zero;
                const float s0 = logit(k0, ok0), s1 = logit(k1, ok1);
                float v0[8], v1[8];
                bf16x8_to_f32(w0, v0);
                bf16x8_to_f32(w1, v1);
                softmax_push2(s0, s1, v0, v1, m, l, acc);
            }
        }
        softmax_merge<G>(m, l, acc, oslc);
    }
    // gated sum with the ball branch for every real query row of the group
    for (int r = kslot; r < 128; r += KPS) {
        int32_t qrow = perm ? perm[int64_t(g) * 128 + r] : int32_t(int64_t(g) * 128 + r);
        if (qrow >= rows) {
            record_error(&g_attn_status, BT_ERR_INTERNAL);
            qrow = -1;
        }
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
    if (size_t(C) * 3 * H * 4 + size_t(32) * (C + 1) * 4 > 200 * 1024) return BT_ERR_UNSUPPORTED;
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

    static bool set[64] = {false};
    static int sms[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BT_ERR_CUDA;
    if (dev >= 64 || !set[dev]) {
        if (cudaFuncSetAttribute(k_bsa_attn_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(BsaPipe<D>::BYTES)) ||
            cudaFuncSetAttribute(k_bsa_gates, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) ||
            cudaFuncSetAttribute(k_bsa_topk<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(4 * kBsaMaxBalls * 4)))
            return BT_ERR_CUDA;
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return BT_ERR_CUDA;
        if (dev < 64) {
            sms[dev] = n;
            set[dev] = true;
        }
    }
    const int nsm = dev < 64 && sms[dev] > 0 ? sms[dev] : 148;
    k_bsa_means<D><<<nb, 128, 0, st>>>(q, k, v, perm, rows, H, qbar, kbar, kc, vc, cnt);
    const size_t gsmem = (size_t(C) * 3 * H + size_t(32) * (C + 1)) * 4;
    k_bsa_gates<<<unsigned((rows + 31) / 32), 256, gsmem, st>>>(X, rows, C, Wg, bg, H, gates);
    if (p.topk > 0)
        k_bsa_topk<D><<<unsigned((int64_t(nb) * H + 3) / 4), 128, size_t(4) * nb * 4, st>>>(
            qbar, kbar, cnt, nb, H, p.topk, p.mask_own_ball, 1.0f / sqrtf(float(D)), sel);
    bt_status s = launch_tc<D>(Q, K, V, perm, npad, rows, 7, H, oball, st);
    if (s != BT_OK) return s;
    const int64_t items = int64_t(nb) * H;
    if (p.coarsen_queries) {
        k_bsa_coarse<D><<<unsigned((items + 3) / 4), 128, 0, st>>>(
            k, v, perm, rows, H, nb, qbar, kc, vc, cnt, sel, p.topk, gates, oball,
            1.4426950408889634f / sqrtf(float(D)), static_cast<__nv_bfloat16 *>(O));
        return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
    }
    const int64_t grid = items < int64_t(nsm) * BsaPipe<D>::PER_SM ? items : int64_t(nsm) * BsaPipe<D>::PER_SM;
    k_bsa_attn_tc<D><<<unsigned(grid), kTcThreads, BsaPipe<D>::BYTES, st>>>(
        q, k, v, perm, rows, H, nb, kc, vc, cnt, sel, p.topk, gates, oball, 1.4426950408889634f / sqrtf(float(D)),
        static_cast<__nv_bfloat16 *>(O));
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
