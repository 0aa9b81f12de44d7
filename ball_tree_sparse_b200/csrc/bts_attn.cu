// Ball Tree Attention ("Erwin: A Tree-based Hierarchical Transformer for
// Large-scale Physical Systems", author's thread post 7/N; PMLR abstract):
// scaled dot-product attention restricted to every ball of m consecutive
// tree slots, all balls and heads in parallel.
//
// Three kernels:
//  - k_ball_attn_pair bf16, m dividing 128, d = 32, even H: one work item is a
//                     128-slot tile and a pair of heads, one warpgroup per head.
//                     Q/K/V rows are gathered through perm by TMA (tile::gather4,
//                     128-byte pieces holding both heads of a row, 128-byte
//                     swizzle), two stages deep, issued by all eight warps.
//  - k_ball_attn_tc2  bf16, m dividing 128, any d in {32, 64} and H: persistent
//                     CTAs over work items (128-slot tile, head), rows gathered
//                     with cp.async into the canonical no-swizzle layouts.
//    Both tensor-core kernels run S = QK^T on tcgen05 (M=128, N=128) into
//    TMEM, read S back with tcgen05.ld (one row per thread), write P (bf16,
//    unnormalised) back over S in TMEM with tcgen05.st, run O = PV with P as
//    the TMEM A operand and the row sums as P times a ones column, and scale by
//    1/rowsum in the epilogue, which scatters O through perm.  Balls smaller
//    than 128 share a tile; keys of other balls and dummy keys get weight 0.
//  - k_ball_attn_simt fp32 (and any other shape): one CTA per (ball, head) on
//                     the CUDA cores, exact two-pass softmax.
// The BSA kernels (bts_bsa.cuh) and the coarse-level pooling kernels
// (bts_coarse.cuh) are included into this translation unit.
#include <cuda_bf16.h>

#include <atomic>

#include "bts_internal.cuh"
#include "bts_tc.cuh"

namespace bts {


// ---------------------------------------------------------------------------
// CUDA-core kernel
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

template <typename T, int D>
__global__ void k_ball_attn_simt(const T *__restrict__ Q, const T *__restrict__ K, const T *__restrict__ V,
                                 const int32_t *__restrict__ perm, int64_t rows, int m, int H, float scale,
                                 T *__restrict__ O, uint32_t *status)
{
    extern __shared__ __align__(16) float fsm[];
    float *sK = fsm, *sV = fsm + m * D;
    int32_t *sRow = reinterpret_cast<int32_t *>(sV + m * D);
    const int64_t b = blockIdx.x;
    const int h = blockIdx.y;
    for (int j = threadIdx.x; j < m; j += blockDim.x) {
        int32_t r = perm ? perm[b * m + j] : int32_t(b * m + j);
        if (r >= rows) {  // not a row of Q/K/V: never read or write it
            record_error(status, BT_ERR_INTERNAL);
            r = -1;
        }
        sRow[j] = r;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < m * D; e += blockDim.x) {
        const int j = e / D, k = e - j * D;
        const int32_t r = sRow[j];
        float kv = 0.0f, vv = 0.0f;
        if (r >= 0) {
            const size_t off = (size_t(r) * H + h) * D + k;
            kv = to_f(K[off]);
            vv = to_f(V[off]);
        }
        sK[e] = kv;
        sV[e] = vv;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < m; i += blockDim.x) {
        const int32_t r = sRow[i];
        if (r < 0) continue;
        float q[D];
#pragma unroll
        for (int k = 0; k < D; ++k) q[k] = to_f(Q[(size_t(r) * H + h) * D + k]);
        float mx = -INFINITY;
        for (int j = 0; j < m; ++j) {
            if (sRow[j] < 0) continue;
            float s = 0.0f;
#pragma unroll
            for (int k = 0; k < D; ++k) s = fmaf(q[k], sK[j * D + k], s);
            mx = fmaxf(mx, s * scale);
        }
        float den = 0.0f, acc[D];
#pragma unroll
        for (int k = 0; k < D; ++k) acc[k] = 0.0f;
        for (int j = 0; j < m; ++j) {
            if (sRow[j] < 0) continue;
            float s = 0.0f;
#pragma unroll
            for (int k = 0; k < D; ++k) s = fmaf(q[k], sK[j * D + k], s);
            const float w = expf(s * scale - mx);
            den += w;
#pragma unroll
            for (int k = 0; k < D; ++k) acc[k] = fmaf(w, sV[j * D + k], acc[k]);
        }
        const float inv = 1.0f / den;
#pragma unroll
        for (int k = 0; k < D; ++k) O[(size_t(r) * H + h) * D + k] = from_f<T>(acc[k] * inv);
    }
}

// ---------------------------------------------------------------------------
// tcgen05 / TMEM kernel
// ---------------------------------------------------------------------------
constexpr int kTcThreads = 128;

// ---------------------------------------------------------------------------
// Persistent, pipelined tcgen05 kernel.  Each CTA walks work items
// (128-slot tile, head) with heads fastest.  While item i computes, the Q/K/V
// rows of the CTA's next item are in flight (cp.async, gathered through perm)
// and the perm entries of the item after that are loading into registers.
//   S = Q K^T          -> TMEM cols [0,128)            (tcgen05, M=128 N=128 K=d)
//   softmax per row     (tcgen05.ld), P = exp2(...) as bf16 written back over
//                       S: TMEM cols [0,64), two keys per column (tcgen05.st)
//   O = P V            -> TMEM cols [64,64+d)          (A = P from TMEM)
//   rowsum(P) = P e0   -> TMEM col 64+d                (B = a ones column)
//   O / rowsum -> bf16 -> the query's row.
// ---------------------------------------------------------------------------
template <int D>
struct TcPipe {
    static constexpr int NS = 2;                                // stages of Q/K/V
    static constexpr uint32_t QK_BYTES = 128 * D * 2;           // one of Q or K
    static constexpr uint32_t STAGE = 3 * QK_BYTES;             // Q, K, V of one item
    static constexpr uint32_t ONES_OFF = NS * STAGE;
    static constexpr uint32_t BYTES = ONES_OFF + 16 * 128 * 2;  // + ones operand (N=16, K=128)
    static constexpr uint32_t COLS = D == 32 ? 128 : 256;       // S/P 128, O d, rowsum 16
    static constexpr int PER_SM = D == 32 ? 4 : 2;              // CTAs per SM that TMEM and smem allow
};




template <int D>
__global__ void __launch_bounds__(kTcThreads, TcPipe<D>::PER_SM)
    k_ball_attn_tc2(const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ K,
                    const __nv_bfloat16 *__restrict__ V, const int32_t *__restrict__ perm, int64_t npad,
                    int64_t rows, int lm, int H, float sl2, int64_t items, __nv_bfloat16 *__restrict__ O, uint32_t *status)
{
    using L = TcPipe<D>;
    constexpr int KCH = D / 8;                 // 16-byte chunks per row of one head
    constexpr int UPT = 128 * KCH / kTcThreads;  // 16-byte chunks per thread and tensor
    constexpr uint32_t QK_SBO = KCH * 128;
    constexpr uint32_t V_SBO = 16 * 128, ONES_SBO = 16 * 128;
    constexpr uint32_t IDESC_S = idesc_bf16(128, false);
    constexpr uint32_t IDESC_O = idesc_bf16(D, true);
    constexpr uint32_t IDESC_SUM = idesc_bf16(16, false);
    extern __shared__ __align__(1024) uint8_t tsm[];
    __shared__ uint32_t sKeyMask[4];
    __shared__ __align__(8) uint64_t sBarS, sBarO;
    __shared__ uint32_t sTmem;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m = 1 << lm;
    const uint32_t base = smem_u32(tsm);

    // the ones operand (K-major, N=16 x K=128): row 0 all 1.0, rows 1..15 zero
    for (int i = tid; i < 16 * 128 * 2 / 16; i += kTcThreads) {
        const int c = i >> 4, rr = i & 15;
        const uint32_t off = (rr >> 3) * ONES_SBO + c * 128 + (rr & 7) * 16;
        const uint32_t one = (rr == 0) ? 0x3F803F80u : 0u;
        *reinterpret_cast<uint4 *>(tsm + L::ONES_OFF + off) = make_uint4(one, one, one, one);
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

    auto row_of = [&](int64_t item, int r) -> int32_t {
        if (item >= items) return -1;
        const int64_t slot = (item / H) * 128 + r;
        if (slot >= npad) return -1;
        if (!perm) return int32_t(slot);
        const int32_t row = __ldg(perm + slot);
        if (row >= rows) {  // not a row of Q/K/V: never read or write it
            record_error(status, BT_ERR_INTERNAL);
            return -1;
        }
        return row;
    };
    // rows whose chunks this thread copies: chunk u = tid + i*128 belongs to row u / KCH
    auto load_rows = [&](int64_t item, int32_t (&rr)[UPT]) {
#pragma unroll
        for (int i = 0; i < UPT; ++i) rr[i] = row_of(item, (tid + i * kTcThreads) / KCH);
    };
    // gather Q, K (K-major core matrices) and V (MN-major core matrices) of one item into a stage
    auto issue = [&](int64_t item, int stage, const int32_t (&rw)[UPT]) {
        if (item < items) {
            const int h = int(item % H);
            uint8_t *sq = tsm + stage * L::STAGE, *sk = sq + L::QK_BYTES, *sv = sk + L::QK_BYTES;
#pragma unroll
            for (int i = 0; i < UPT; ++i) {
                const int u = tid + i * kTcThreads;
                const int r = u / KCH, c = u - r * KCH;
                const int32_t rr = rw[i];
                const size_t goff = rr >= 0 ? (size_t(rr) * H + h) * D + c * 8 : 0;
                const uint32_t so = (r >> 3) * QK_SBO + c * 128 + (r & 7) * 16;
                cp_async16(sq + so, Q + goff, rr >= 0);
                cp_async16(sk + so, K + goff, rr >= 0);
                cp_async16(sv + c * V_SBO + r * 16, V + goff, rr >= 0);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    const int64_t first = blockIdx.x, stride = gridDim.x;
    int32_t nrows[UPT];
    load_rows(first, nrows);
    issue(first, 0, nrows);
    load_rows(first + stride, nrows);  // rows of the next item, used at the top of the loop
    int32_t qcur = row_of(first, tid), qnext = row_of(first + stride, tid);
    bool ok = true;
    int it = 0;
    for (int64_t item = first; item < items; item += stride, ++it) {
        const int stage = it & 1;
        issue(item + stride, stage ^ 1, nrows);
        load_rows(item + 2 * stride, nrows);  // consumed one iteration later
        const int32_t qafter = row_of(item + 2 * stride, tid);
        const uint32_t kb = __ballot_sync(0xffffffffu, qcur >= 0);
        if (lane == 0) sKeyMask[warp] = kb;
        asm volatile("cp.async.wait_group 1;" ::: "memory");
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        const uint32_t sq = base + stage * L::STAGE, sk = sq + L::QK_BYTES, sv = sk + L::QK_BYTES;
        if (tid == 0 && ok) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_bf16(tS, smem_desc(sq + kk * 256, 128, QK_SBO), smem_desc(sk + kk * 256, 128, QK_SBO), IDESC_S,
                         kk > 0);
            mma_commit(barS);
        }
        ok = ok && mbar_wait(barS, it & 1, status);
        tc_fence_after();

        // softmax of row tid; keys outside its ball or dummy get weight 0
        const int ball0 = (tid >> lm) << lm;
        uint32_t cmask[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t bm;  // keys of chunk c that lie in this row's ball
            if (m >= 32)
                bm = (c * 32 >= ball0 && c * 32 < ball0 + m) ? 0xffffffffu : 0u;
            else
                bm = (c * 32 <= ball0 && ball0 < c * 32 + 32) ? (((1u << m) - 1u) << (ball0 - c * 32)) : 0u;
            cmask[c] = bm & sKeyMask[c];
        }
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (__any_sync(0xffffffffu, cmask[c] != 0u)) {
                uint32_t v[32];
                tmem_ld32(tS + lanebase + c * 32, v);
                if (cmask[c] == 0xffffffffu) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) mx = fmaxf(mx, __uint_as_float(v[j]));
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if ((cmask[c] >> j) & 1u) mx = fmaxf(mx, __uint_as_float(v[j]));
                }
            }
        }
        const float mxs = mx == -INFINITY ? 0.0f : mx * sl2;
        // chunk c of S (cols 32c..32c+31) becomes P cols 16c..16c+15: every S column a P store
        // overwrites has been read into registers by this thread before (its own TMEM lane)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t pk[16];
            if (__any_sync(0xffffffffu, cmask[c] != 0u)) {
                uint32_t v[32];
                tmem_ld32(tS + lanebase + c * 32, v);
                const uint32_t cm = cmask[c];
                if (__all_sync(0xffffffffu, cm == 0xffffffffu)) {  // every key valid: no per-key selects
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        const float p0 = ex2(fmaf(__uint_as_float(v[j]), sl2, -mxs));
                        const float p1 = ex2(fmaf(__uint_as_float(v[j + 1]), sl2, -mxs));
                        const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                        pk[j >> 1] = *reinterpret_cast<const uint32_t *>(&pb);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        float p0 = ex2(fmaf(__uint_as_float(v[j]), sl2, -mxs));
                        float p1 = ex2(fmaf(__uint_as_float(v[j + 1]), sl2, -mxs));
                        p0 = ((cm >> j) & 1u) ? p0 : 0.0f;
                        p1 = ((cm >> (j + 1)) & 1u) ? p1 : 0.0f;
                        const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                        pk[j >> 1] = *reinterpret_cast<const uint32_t *>(&pb);
                    }
                }
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) pk[j] = 0u;
            }
            tmem_st16(tS + lanebase + c * 16, pk);
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
        ok = ok && mbar_wait(barO, it & 1, status);
        tc_fence_after();
        if (ok) {
            uint32_t sum_bits;
            tmem_ld1(tSum + lanebase, sum_bits);
            const float sum = __uint_as_float(sum_bits);
            const float inv = sum > 0.0f ? 1.0f / sum : 0.0f;
            const int h = int(item % H);
#pragma unroll
            for (int c32 = 0; c32 < D; c32 += 32) {
                uint32_t o[32];
                tmem_ld32(tO + lanebase + c32, o);
                if (qcur >= 0) {
                    uint4 *dst = reinterpret_cast<uint4 *>(O + (size_t(qcur) * H + h) * D + c32);
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 pb = __floats2bfloat162_rn(
                                __uint_as_float(o[8 * t + 2 * e]) * inv, __uint_as_float(o[8 * t + 2 * e + 1]) * inv);
                            w[e] = *reinterpret_cast<const uint32_t *>(&pb);
                        }
                        dst[t] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
        }
        qcur = qnext;
        qnext = qafter;
        tc_fence_before();
        __syncthreads();  // every read of S/P, O and of this stage is done before they are reused
        tc_fence_after();
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
// Two heads per work item (d = 32, even H).  The rows of Q, K and V are gathered by TMA
// (tile::gather4 through perm) as 128-byte pieces: the two heads of a row side by side, 128-byte
// swizzled, so each gather moves enough bytes per request to keep HBM busy.  Warpgroup j of the CTA
// owns head j of the pair: its S in TMEM columns [128j, 128j+128), P written back over the first 64 of
// them, O at +64 and the row sums at +96.  The two heads share one K-major swizzle row, so head j's
// operands start 64 bytes into it; V is read MN-major from the same rows.
// ---------------------------------------------------------------------------
struct PairPipe {
    static constexpr int NS = 2;
    static constexpr uint32_t RB = 128;                 // bytes of one row of a head pair
    static constexpr uint32_t TILE = 128 * RB;          // Q, K or V of one item (16 KB)
    static constexpr uint32_t STAGE = 3 * TILE;
    static constexpr uint32_t BYTES = NS * STAGE + 1024;
    static constexpr uint32_t COLS = 256;
    static constexpr int CONSUMERS = 256;               // two warpgroups, one per head of the pair
    static constexpr int PRODUCERS = 64;                // two warps that gather the next item's rows
    static constexpr int THREADS = CONSUMERS + PRODUCERS;
    static constexpr int PER_SM = 2;
};

// Named barrier of one head's warpgroup (ids 1 and 2; 3 is the producers').
__device__ __forceinline__ void head_sync(int hj)
{
    if (hj == 0)
        asm volatile("bar.sync 1, 128;" ::: "memory");
    else
        asm volatile("bar.sync 2, 128;" ::: "memory");
}

// Warps 0-7 compute: warpgroup j (warps 4j..4j+3) owns head j of the pair and runs on its own (its first
// thread issues that head's MMAs, its own mbarriers and named barrier), so one head's MMA waits overlap
// the other head's softmax.  Warps 8-9 only load perm and issue the TMA gathers of the next item into the
// free stage, so the gathers' issue cost is off the compute path.  Stage s is full when its transaction
// count completes (sFull[s]) and free again when both heads' MMAs that read it have completed (sEmpty[s],
// two arrivals, each armed by tcgen05.commit after that head's P V product).
template <bool TREE>
__global__ void __launch_bounds__(PairPipe::THREADS, PairPipe::PER_SM)
    k_ball_attn_pair(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const int32_t *__restrict__ perm, int64_t npad,
                     int64_t rows, int lm, int H, float sl2, int64_t items, __nv_bfloat16 *__restrict__ O,
                     uint32_t *ctr, uint32_t *status)
{
    using L = PairPipe;
    constexpr int NS = L::NS;
    constexpr int D = 32;
    constexpr uint32_t SBO8 = 8 * L::RB, SW128 = 2;
    constexpr uint32_t IDESC_S = idesc_bf16(128, false);
    constexpr uint32_t IDESC_O = idesc_bf16(D, true);
    extern __shared__ __align__(1024) uint8_t psm[];
    __shared__ uint32_t sKeyMask[NS][2][4];  // per stage: valid keys of each head's tile, by 32-key group
    __shared__ __align__(8) uint64_t sBarS[2], sBarO[2], sFull[NS], sEmpty[NS];
    __shared__ uint32_t sTmem;
    __shared__ int32_t sRows[NS][128];  // rows of the stage's item (-1: dummy slot), for the consumers
    __shared__ int64_t sItem[NS];       // the stage's item, -1 when the CTA has no more work
    __shared__ int64_t sClaim;          // next item, claimed by the first producer thread
    __shared__ int sAbort[2];           // a head's warpgroup stops after a wait that ran out
    __shared__ int sLive[2];            // per producer warp: some row of the claimed item is a real point

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m = 1 << lm;
    const int HP = H >> 1;
    const uint32_t base = (smem_u32(psm) + 1023u) & ~1023u;  // swizzled tiles need 1024-byte alignment
    uint8_t *gbase = psm + (base - smem_u32(psm));

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sTmem)),
                     "r"(L::COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid < 2) sAbort[tid] = 0;
    if (tid == 0) {
        for (int j = 0; j < 2; ++j) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sBarS[j])) : "memory");
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sBarO[j])) : "memory");
        }
        for (int s0 = 0; s0 < NS; ++s0) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sFull[s0])) : "memory");
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 2;" ::"r"(smem_u32(&sEmpty[s0])) : "memory");
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sTmem;
    const int32_t oob = rows < 0x7FFFFFFF ? int32_t(rows) : -1;  // a row outside the tensor reads zeros

    auto raw_row = [&](int64_t item, int rr) -> int32_t {  // items < 2^31: 32-bit index arithmetic
        if (item >= items) return -1;
        const int64_t slot = int64_t(uint32_t(item) / uint32_t(HP)) * 128 + rr;
        if (slot >= npad) return -1;
        return perm ? __ldg(perm + slot) : int32_t(slot);
    };
    auto check = [&](int32_t row) -> int32_t {
        if (row >= rows) {  // not a row of Q/K/V: never read or write it
            record_error(status, BT_ERR_INTERNAL);
            return -1;
        }
        return row;
    };

    if (warp >= 8) {
        // ---------------- producers: lanes 0-15 of warp 8 + w take rows 4g..4g+3, g = 16 w + lane ----------------
        // Work is claimed dynamically: the first item of a CTA is its block index, every later one comes from
        // the launch's counter, so CTAs that start late (the GPU busy with other work) simply take fewer items.
        // The next item is claimed, and its perm rows requested, right after the current item's gathers.
        const int pw = warp - 8, g = 16 * pw + lane;
        bool pok = true;
        // the item after `cur`: the launch's next unclaimed item, or without counters a fixed stride of the grid
        auto claim = [&](int64_t cur) -> int64_t {
            return ctr ? int64_t(gridDim.x) + int64_t(atomicAdd(ctr, 1u)) : cur + int64_t(gridDim.x);
        };
        int64_t item = blockIdx.x;
        int32_t crow[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) crow[i] = lane < 16 ? raw_row(item, 4 * g + i) : -1;
        // An item whose 128 slots are all dummies (the padding at the end of a cloud) has no output: it is
        // replaced by the next claimed item before it takes a stage.  A perm entry outside Q/K/V counts as a
        // real row here, so the item still goes through the checks below.
        auto skip_dead = [&]() {
            while (item < items) {
                const bool live = lane < 16 && (crow[0] >= 0 || crow[1] >= 0 || crow[2] >= 0 || crow[3] >= 0);
                const uint32_t bw = __ballot_sync(0xffffffffu, live);
                if (lane == 0) sLive[pw] = bw != 0u;
                asm volatile("bar.sync 3, %0;" ::"n"(L::PRODUCERS) : "memory");
                const bool dead = !sLive[0] && !sLive[1];
                if (dead && tid == 8 * 32) sClaim = pok ? claim(item) : items;
                asm volatile("bar.sync 3, %0;" ::"n"(L::PRODUCERS) : "memory");  // sLive read; sClaim written
                if (!dead) return;
                item = sClaim;
#pragma unroll
                for (int i = 0; i < 4; ++i) crow[i] = lane < 16 ? raw_row(item, 4 * g + i) : -1;
            }
        };
        skip_dead();
        for (int it = 0;; ++it) {
            const int stage = it & (NS - 1);
            const uint32_t bar = smem_u32(&sFull[stage]);
            if (it >= NS) pok = mbar_wait(smem_u32(&sEmpty[stage]), ((it / NS) + 1) & 1, status) && pok;
            if (item >= items) {  // no more work: tell the consumers through the free stage
                if (tid == 8 * 32) {
                    sItem[stage] = -1;
                    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
                }
                break;
            }
            int32_t rr[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int32_t x = check(crow[i]);
                rr[i] = x >= 0 ? x : oob;
                if (lane < 16) sRows[stage][4 * g + i] = x;
            }
            if (tid == 8 * 32) sItem[stage] = item;
            asm volatile("bar.sync 3, %0;" ::"n"(L::PRODUCERS) : "memory");  // rows and item stored
            if (tid == 8 * 32) mbar_expect_tx(bar, L::STAGE);                  // publishes rows and item
            asm volatile("bar.sync 3, %0;" ::"n"(L::PRODUCERS) : "memory");  // armed before any gather lands
            if (lane < 16) {
                const int32_t col = int32_t(uint32_t(item) % uint32_t(HP)) * 2 * D;
                if constexpr (TREE) {
                    // Q/K/V already in slot order: the item's rows are one 128 x 64 tile of each tensor
                    if (g == 0) {
                        const int32_t y = int32_t(uint32_t(item) / uint32_t(HP)) * 128;
                        const uint32_t dq = base + stage * L::STAGE;
                        tma_load_2d(dq, &tmQ, col, y, bar);
                        tma_load_2d(dq + L::TILE, &tmK, col, y, bar);
                        tma_load_2d(dq + 2 * L::TILE, &tmV, col, y, bar);
                    }
                } else {
                    const uint32_t dq = base + stage * L::STAGE + g * 4 * L::RB;
                    tma_gather4(dq, &tmQ, col, rr[0], rr[1], rr[2], rr[3], bar);
                    tma_gather4(dq + L::TILE, &tmK, col, rr[0], rr[1], rr[2], rr[3], bar);
                    tma_gather4(dq + 2 * L::TILE, &tmV, col, rr[0], rr[1], rr[2], rr[3], bar);
                }
            }
            // claim the next item after the gathers are on their way (a producer whose wait ran out hands out
            // no further work); its perm rows load while the next stage frees up
            if (tid == 8 * 32) sClaim = pok ? claim(item) : items;
            asm volatile("bar.sync 3, %0;" ::"n"(L::PRODUCERS) : "memory");
            item = sClaim;
#pragma unroll
            for (int i = 0; i < 4; ++i) crow[i] = lane < 16 ? raw_row(item, 4 * g + i) : -1;
            skip_dead();
        }
        if (tid == 8 * 32 && ctr) {
            // this CTA claims no more work: the last CTA to get here sets the launch's counters back to zero for
            // the next launch that uses them (every CTA's claims come before its count: release and acquire)
            uint32_t prev;
            asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(prev) : "l"(ctr + 1) : "memory");
            if (prev == gridDim.x - 1) {
                ctr[0] = 0u;
                ctr[1] = 0u;
            }
        }
    } else {
        // ---------------- consumers ----------------
        // Per item: S = Q K^T, softmax (row sums in registers, on the FMA pipe), P V, O read into registers; then this
        // head's TMEM is free, so the next item's S is issued before this item's scale-and-store epilogue.
        const int hj = warp >> 2;  // head of the pair this warpgroup owns
        const int r = tid & 127;   // query row (TMEM lane) this thread owns
        const bool issuer = r == 0;
        const uint32_t tS = tmem + 128 * hj, tO = tS + 64;  // this warpgroup's columns
        const uint32_t barS = smem_u32(&sBarS[hj]), barO = smem_u32(&sBarO[hj]);
        const uint32_t lanebase = uint32_t((warp & 3) * 32) << 16;
        bool ok = true;
        // Waits for stage `st` of round `it`, publishes this warp's key mask, and reads the stage's item and
        // this thread's query row after the warpgroup barrier (so every thread takes the same decision).
        auto head = [&](int itn, int st, int32_t &q, int64_t &itm) -> bool {
            ok = ok && mbar_wait(smem_u32(&sFull[st]), (itn / NS) & 1, status);
            if (!ok) sAbort[hj] = 1;
            q = sRows[st][r];  // -1: dummy slot
            const uint32_t kb = __ballot_sync(0xffffffffu, q >= 0);
            if (lane == 0) sKeyMask[st][hj][warp & 3] = kb;
            tc_fence_before();
            head_sync(hj);
            tc_fence_after();
            itm = sItem[st];
            const bool go = itm >= 0 && !sAbort[hj];
            if (go && issuer && ok) {
                const uint32_t sq = base + st * L::STAGE, sk = sq + L::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_bf16(tS, smem_desc_sw(sq + 64 * hj + 32 * kk, 16, SBO8, SW128),
                             smem_desc_sw(sk + 64 * hj + 32 * kk, 16, SBO8, SW128), IDESC_S, kk > 0);
                mma_commit(barS);
            }
            return go;
        };
        int32_t qcur = -1;
        int64_t item = -1;
        bool go = head(0, 0, qcur, item);
        for (int it = 0; go; ++it) {
            const int stage = it & (NS - 1);
            const uint32_t sv = base + stage * L::STAGE + 2 * L::TILE;
            ok = ok && mbar_wait(barS, it & 1, status);
            tc_fence_after();

            // softmax of row r of head hj; keys outside its ball or dummy get weight 0
            const int ball0 = (r >> lm) << lm;
            uint32_t cmask[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t bm;
                if (m >= 32)
                    bm = (c * 32 >= ball0 && c * 32 < ball0 + m) ? 0xffffffffu : 0u;
                else
                    bm = (c * 32 <= ball0 && ball0 < c * 32 + 32) ? (((1u << m) - 1u) << (ball0 - c * 32)) : 0u;
                cmask[c] = bm & sKeyMask[stage][hj][c];
            }
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (__any_sync(0xffffffffu, cmask[c] != 0u)) {
                    uint32_t v[32];
                    tmem_ld32(tS + lanebase + c * 32, v);
                    if (cmask[c] == 0xffffffffu) {
#pragma unroll
                        for (int j = 0; j < 32; j += 2) mx = fmax3(mx, __uint_as_float(v[j]), __uint_as_float(v[j + 1]));
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if ((cmask[c] >> j) & 1u) mx = fmaxf(mx, __uint_as_float(v[j]));
                    }
                }
            }
            const float mxs = mx == -INFINITY ? 0.0f : mx * sl2;
            // row sum of the weights (before their rounding to bf16 for the P V product), even and odd keys
            float rs0 = 0.0f, rs1 = 0.0f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pk[16];
                if (__any_sync(0xffffffffu, cmask[c] != 0u)) {
                    uint32_t v[32];
                    tmem_ld32(tS + lanebase + c * 32, v);
                    const uint32_t cm = cmask[c];
                    if (__all_sync(0xffffffffu, cm == 0xffffffffu)) {  // every key valid: no per-key selects
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            float p0, p1;
                            ffma2_bcast(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), sl2, -mxs, p0, p1);
                            p0 = ex2(p0);
                            p1 = ex2(p1);
                            const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                            pk[j >> 1] = *reinterpret_cast<const uint32_t *>(&pb);
                            fadd2_acc(rs0, rs1, p0, p1);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            float p0, p1;
                            ffma2_bcast(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), sl2, -mxs, p0, p1);
                            p0 = ((cm >> j) & 1u) ? ex2(p0) : 0.0f;
                            p1 = ((cm >> (j + 1)) & 1u) ? ex2(p1) : 0.0f;
                            const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                            pk[j >> 1] = *reinterpret_cast<const uint32_t *>(&pb);
                            fadd2_acc(rs0, rs1, p0, p1);
                        }
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) pk[j] = 0u;
                }
                tmem_st16(tS + lanebase + c * 16, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            head_sync(hj);
            tc_fence_after();
            if (issuer) {
                if (ok) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tO, tS + kk * 8, smem_desc_sw(sv + 64 * hj + kk * 16 * L::RB, 16, SBO8, SW128),
                                    IDESC_O, kk > 0);
                }
                mma_commit(barO);
                mma_commit(smem_u32(&sEmpty[stage]));  // this head is done with the stage
            }
            ok = ok && mbar_wait(barO, it & 1, status);
            tc_fence_after();
            uint32_t o[32];
            tmem_ld32_nowait(tO + lanebase, o);
            tmem_wait_ld();
            tc_fence_before();
            head_sync(hj);  // this head's S/P and O columns are free again
            tc_fence_after();

            // next item's S on the tensor core while this item's rows are scaled and stored
            int32_t qn = -1;
            int64_t itemn = -1;
            go = head(it + 1, (it + 1) & (NS - 1), qn, itemn);
            if (ok && qcur >= 0) {
                const float rsum = rs0 + rs1;
                const float inv = rsum > 0.0f ? 1.0f / rsum : 0.0f;
                const int h = int(uint32_t(item) % uint32_t(HP)) * 2 + hj;
                uint4 *dst = reinterpret_cast<uint4 *>(O + (size_t(qcur) * H + h) * D);
#pragma unroll
                for (int t = 0; t < D / 8; ++t) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 pb = __floats2bfloat162_rn(__uint_as_float(o[8 * t + 2 * e]) * inv,
                                                                        __uint_as_float(o[8 * t + 2 * e + 1]) * inv);
                        w[e] = *reinterpret_cast<const uint32_t *>(&pb);
                    }
                    dst[t] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            qcur = qn;
            item = itemn;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(L::COLS) : "memory");
    }
}

// Tensor maps that view a [rows, H, d] bf16 tensor as rows of H*d elements with a `box`-element window
// per row (the gather unit of the attention kernels), 128-byte swizzled to match the tcgen05 operands.
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

static bool row_map(CUtensorMap *map, const void *base, int64_t rows, int hd, int box)
{
    const EncodeTiledFn fn = encode_tiled();
    if (!fn || rows < 1 || (reinterpret_cast<uintptr_t>(base) & 15)) return false;
    const cuuint64_t dims[2] = {cuuint64_t(hd), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(hd) * 2};
    const cuuint32_t bx[2] = {cuuint32_t(box), 1};
    const cuuint32_t es[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, bx, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A [rows, cols] bf16 matrix viewed in box_rows x box_cols tiles, 128-byte swizzled (whole-tile loads).
static bool tile_map(CUtensorMap *map, const void *base, int64_t rows, int cols, int box_cols, int box_rows)
{
    const EncodeTiledFn fn = encode_tiled();
    if (!fn || rows < 1 || (reinterpret_cast<uintptr_t>(base) & 15)) return false;
    const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(cols) * 2};
    const cuuint32_t bx[2] = {cuuint32_t(box_cols), cuuint32_t(box_rows)};
    const cuuint32_t es[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, bx, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Work counters of the head-pair kernel ([0] items claimed so far, [1] CTAs done claiming; the last CTA of a launch
// sets both back to zero).  Launches that run at the same time need distinct pairs:
//  - eager launches take pair k mod kEagerPairs (the k-th eager launch on the device), so up to kEagerPairs of
//    them may be in flight together;
//  - a launch captured into a CUDA graph keeps its pair for as long as the graph exists, so every captured
//    launch gets a pair of its own from the next kCapturedPairs, never reused; once those are used up,
//    captured launches run without counters, on a fixed schedule (item i of CTA c is c + i * grid).
constexpr int kEagerPairs = 256;
constexpr int kCapturedPairs = 4096;
static __device__ uint32_t g_pair_ctr[kEagerPairs + kCapturedPairs][2];

// tree: Q, K and V are [npad, H, 32] in slot order (whole-tile loads); otherwise [rows, H, 32] in the original
// order, gathered through perm.  perm names the output row of every slot (or -1) either way.
static bt_status launch_pair(const void *Q, const void *K, const void *V, const int32_t *perm, int64_t npad,
                             int64_t rows, int lm, int H, void *O, cudaStream_t st, bool tree = false)
{
    static std::atomic<bool> set[64] = {};
    static int sms[64] = {0};
    static uint32_t *ctrs[64] = {nullptr};
    static std::atomic<uint32_t> next_pair[64] = {};
    static std::atomic<uint32_t> next_captured[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BT_ERR_CUDA;
    if (dev < 0 || dev >= 64) return BT_ERR_UNSUPPORTED;
    const bt_status s0 = setup_once(set[dev], [&]() -> bt_status {
        if (cudaFuncSetAttribute(k_ball_attn_pair<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(PairPipe::BYTES)) ||
            cudaFuncSetAttribute(k_ball_attn_pair<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(PairPipe::BYTES)))
            return BT_ERR_CUDA;
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return BT_ERR_CUDA;
        // host code sees only a stand-in for the counter array: ask the runtime for its device address
        void *addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_pair_ctr) != cudaSuccess || !addr) return BT_ERR_CUDA;
        ctrs[dev] = static_cast<uint32_t *>(addr);
        sms[dev] = n;
        return BT_OK;
    });
    if (s0 != BT_OK) return s0;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return BT_ERR_CUDA;
    uint32_t *ctr = nullptr;
    if (cs == cudaStreamCaptureStatusNone) {
        ctr = ctrs[dev] + 2 * (next_pair[dev].fetch_add(1u) % kEagerPairs);
    } else {
        const uint32_t k = next_captured[dev].fetch_add(1u);
        if (k < uint32_t(kCapturedPairs)) ctr = ctrs[dev] + 2 * (kEagerPairs + k);
    }
    uint32_t *status = stream_status(st);
    if (!status) return BT_ERR_CUDA;
    CUtensorMap mq, mk, mv;
    if (tree) {
        if (!tile_map(&mq, Q, npad, H * 32, 64, 128) || !tile_map(&mk, K, npad, H * 32, 64, 128) ||
            !tile_map(&mv, V, npad, H * 32, 64, 128))
            return BT_ERR_CUDA;
    } else if (!row_map(&mq, Q, rows, H * 32, 64) || !row_map(&mk, K, rows, H * 32, 64) ||
               !row_map(&mv, V, rows, H * 32, 64)) {
        return BT_ERR_CUDA;
    }
    const int nsm = dev < 64 && sms[dev] > 0 ? sms[dev] : 148;
    const int64_t items = (npad + 127) / 128 * (H / 2);
    if (items > 0x7FFFFFFF) return BT_ERR_UNSUPPORTED;
    const int64_t grid = items < int64_t(nsm) * PairPipe::PER_SM ? items : int64_t(nsm) * PairPipe::PER_SM;
    const float sl2 = 1.4426950408889634f / sqrtf(32.0f);
    auto kern = tree ? k_ball_attn_pair<true> : k_ball_attn_pair<false>;
    kern<<<unsigned(grid), PairPipe::THREADS, PairPipe::BYTES, st>>>(
        mq, mk, mv, perm, npad, rows, lm, H, sl2, items, static_cast<__nv_bfloat16 *>(O), ctr, status);
    return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
}

template <typename T, int D>
static bt_status launch_simt(const void *Q, const void *K, const void *V, const int32_t *perm, int64_t npad,
                             int64_t rows, int m, int H, void *O, cudaStream_t st)
{
    const size_t smem = size_t(2) * m * D * 4 + size_t(m) * 4;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(k_ball_attn_simt<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)))
        return BT_ERR_CUDA;
    const int threads = ((m + 31) / 32) * 32;
    dim3 grid(unsigned(npad / m), unsigned(H));
    uint32_t *status = stream_status(st);
    if (!status) return BT_ERR_CUDA;
    k_ball_attn_simt<T, D><<<grid, threads, smem, st>>>(static_cast<const T *>(Q), static_cast<const T *>(K),
                                                        static_cast<const T *>(V), perm, rows, m, H,
                                                        1.0f / sqrtf(float(D)), static_cast<T *>(O), status);
    return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
}

template <int D>
static bt_status launch_tc(const void *Q, const void *K, const void *V, const int32_t *perm, int64_t npad,
                           int64_t rows, int lm, int H, void *O, cudaStream_t st)
{
    constexpr size_t smem = TcPipe<D>::BYTES;
    static std::atomic<bool> set[64] = {};
    static int sms[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BT_ERR_CUDA;
    auto init = [&]() -> bt_status {
        if (cudaFuncSetAttribute(k_ball_attn_tc2<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)))
            return BT_ERR_CUDA;
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return BT_ERR_CUDA;
        if (dev >= 0 && dev < 64) sms[dev] = n;
        return BT_OK;
    };
    const bt_status s0 = (dev >= 0 && dev < 64) ? setup_once(set[dev], init) : init();
    if (s0 != BT_OK) return s0;
    const int nsm = dev < 64 && sms[dev] > 0 ? sms[dev] : 148;
    const int64_t items = (npad + 127) / 128 * H;
    const int per_sm = TcPipe<D>::PER_SM;
    const int64_t grid = items < int64_t(nsm) * per_sm ? items : int64_t(nsm) * per_sm;
    const float sl2 = 1.4426950408889634f / sqrtf(float(D));
    uint32_t *status = stream_status(st);
    if (!status) return BT_ERR_CUDA;
    k_ball_attn_tc2<D><<<unsigned(grid), kTcThreads, smem, st>>>(
        static_cast<const __nv_bfloat16 *>(Q), static_cast<const __nv_bfloat16 *>(K),
        static_cast<const __nv_bfloat16 *>(V), perm, npad, rows, lm, H, sl2, items, static_cast<__nv_bfloat16 *>(O), status);
    return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
}

}  // namespace bts

#include "bts_bsa.cuh"
#include "bts_project.cuh"

using namespace bts;

extern "C" bt_status bt_ball_attention(const void *Q, const void *K, const void *V, const int32_t *perm, int64_t npad,
                                       int64_t rows, int32_t m, int32_t H, int32_t d, bt_dtype dt, void *O, void *stream)
{
    if (!Q || !K || !V || !O || npad < 0 || rows < 0 || H < 1) return BT_ERR_ARG;
    if (m < 1 || m > 256 || (d != 32 && d != 64)) return BT_ERR_SHAPE;
    if (npad % m) return BT_ERR_SHAPE;
    if (dt != BT_F32 && dt != BT_BF16) return BT_ERR_ARG;
    if (!perm && rows < npad) return BT_ERR_ARG;
    if (npad == 0) return BT_OK;
    if (npad / m > 0x7FFFFFFF || int64_t(H) > 65535 || rows > 0x7FFFFFFF) return BT_ERR_UNSUPPORTED;
    const uintptr_t al = reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) |
                         reinterpret_cast<uintptr_t>(V) | reinterpret_cast<uintptr_t>(O);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dt == BT_BF16 && (m == 16 || m == 32 || m == 64 || m == 128)) {
        if (al % 16) return BT_ERR_ARG;
        const int lm = m == 16 ? 4 : m == 32 ? 5 : m == 64 ? 6 : 7;
        if (d == 32 && H % 2 == 0 && rows < 0x7FFFFFFF) return launch_pair(Q, K, V, perm, npad, rows, lm, H, O, st);
        return d == 32 ? launch_tc<32>(Q, K, V, perm, npad, rows, lm, H, O, st)
                       : launch_tc<64>(Q, K, V, perm, npad, rows, lm, H, O, st);
    }
    if (dt == BT_BF16)
        return d == 32 ? launch_simt<__nv_bfloat16, 32>(Q, K, V, perm, npad, rows, m, H, O, st)
                       : launch_simt<__nv_bfloat16, 64>(Q, K, V, perm, npad, rows, m, H, O, st);
    return d == 32 ? launch_simt<float, 32>(Q, K, V, perm, npad, rows, m, H, O, st)
                   : launch_simt<float, 64>(Q, K, V, perm, npad, rows, m, H, O, st);
}

#include "bts_coarse.cuh"

// ---------------------------------------------------------------------------
// Projection into tree order and attention on tree-ordered Q/K/V
// ---------------------------------------------------------------------------
namespace bts {
static bool pair_shape(int32_t m, int32_t H, int32_t d, bt_dtype dt, int64_t rows)
{
    return dt == BT_BF16 && d == 32 && H % 2 == 0 && (m == 16 || m == 32 || m == 64 || m == 128) &&
           rows < 0x7FFFFFFF;
}
static int log2m(int32_t m) { return m == 16 ? 4 : m == 32 ? 5 : m == 64 ? 6 : 7; }
}  // namespace bts

extern "C" bt_status bt_qkv_project(const void *X, int64_t rows, int32_t C, const void *Wt, int32_t H, int32_t d,
                                    bt_dtype dt, const int32_t *perm, const int32_t *inv, int64_t npad, void *Q,
                                    void *K, void *V, void *stream)
{
    if (!X || !Wt || !Q || !K || !V || rows < 0 || C < 1 || H < 1 || d < 1) return BT_ERR_ARG;
    if (dt != BT_F32 && dt != BT_BF16) return BT_ERR_ARG;
    if (perm && (!inv || npad < 0)) return BT_ERR_ARG;
    if (rows > 0x7FFFFFFF || npad > 0x7FFFFFFF || int64_t(H) * d * 3 > 65535) return BT_ERR_UNSUPPORTED;
    if (!perm) npad = rows;
    if (npad == 0 && rows == 0) return BT_OK;
    return launch_project(X, rows, C, Wt, H, d, dt, perm, inv, npad, Q, K, V, static_cast<cudaStream_t>(stream));
}

extern "C" bt_status bt_ball_attention_tree(const void *Qt, const void *Kt, const void *Vt, const int32_t *perm,
                                            int64_t npad, int64_t rows, int32_t m, int32_t H, int32_t d, bt_dtype dt,
                                            void *O, void *stream)
{
    if (!Qt || !Kt || !Vt || !O || !perm || npad < 0 || rows < 0 || H < 1) return BT_ERR_ARG;
    if (m < 1 || npad % m) return BT_ERR_SHAPE;
    if (npad == 0) return BT_OK;
    // whole 128-slot tiles: the slot-ordered tensors must hold at least one
    if (!pair_shape(m, H, d, dt, rows) || npad < 128 || npad > 0x7FFFFFFF) return BT_ERR_UNSUPPORTED;
    const uintptr_t al = reinterpret_cast<uintptr_t>(Qt) | reinterpret_cast<uintptr_t>(Kt) |
                         reinterpret_cast<uintptr_t>(Vt) | reinterpret_cast<uintptr_t>(O);
    if (al % 16) return BT_ERR_ARG;
    return launch_pair(Qt, Kt, Vt, perm, npad, rows, log2m(m), H, O, static_cast<cudaStream_t>(stream), true);
}

extern "C" size_t bt_projected_workspace_size(int64_t npad, int64_t rows, int32_t H, int32_t d, bt_dtype dt)
{
    if (npad < 0 || rows < 0 || H < 1 || d < 1 || (dt != BT_F32 && dt != BT_BF16)) return 0;
    const int64_t n = npad > rows ? npad : rows;
    const size_t one = (size_t(n) * H * d * (dt == BT_F32 ? 4 : 2) + 255) & ~size_t(255);
    return 3 * one + ((size_t(rows) * 4 + 255) & ~size_t(255));  // Q, K, V and the inverse slot map
}

extern "C" bt_status bt_projected_ball_attention(const void *X, const int32_t *perm, int64_t npad, int64_t rows,
                                                 int32_t C, const void *Wt, int32_t m, int32_t H, int32_t d,
                                                 bt_dtype dt, void *O, void *ws, size_t ws_bytes, void *stream)
{
    if (!X || !Wt || !O || npad < 0 || rows < 0 || C < 1 || H < 1) return BT_ERR_ARG;
    if (m < 1 || m > 256 || (d != 32 && d != 64)) return BT_ERR_SHAPE;
    if (npad % m) return BT_ERR_SHAPE;
    if (!perm && rows < npad) return BT_ERR_ARG;
    if (npad == 0) return BT_OK;
    const size_t need = bt_projected_workspace_size(npad, rows, H, d, dt);
    if (!ws || need == 0 || ws_bytes < need) return BT_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return BT_ERR_ARG;
    const int64_t n = npad > rows ? npad : rows;
    const size_t one = (size_t(n) * H * d * (dt == BT_F32 ? 4 : 2) + 255) & ~size_t(255);
    uint8_t *w = static_cast<uint8_t *>(ws);
    void *Q = w, *K = w + one, *V = w + 2 * one;
    int32_t *inv = reinterpret_cast<int32_t *>(w + 3 * one);
    if (perm && pair_shape(m, H, d, dt, rows) && npad >= 128) {
        // Q, K, V written in slot order (each feature row to its slot); the attention then loads every ball as one
        // tile.  Every row must be named by a slot, as in a tree built over these rows.
        bt_status s = bt_invert_perm(perm, npad, rows, inv, stream);
        if (s != BT_OK) return s;
        s = bt_qkv_project(X, rows, C, Wt, H, d, dt, perm, inv, npad, Q, K, V, stream);
        if (s != BT_OK) return s;
        return bt_ball_attention_tree(Q, K, V, perm, npad, rows, m, H, d, dt, O, stream);
    }
    // other shapes: Q, K, V in the original row order, then the gathering attention
    bt_status s = bt_qkv_project(X, rows, C, Wt, H, d, dt, nullptr, nullptr, 0, Q, K, V, stream);
    if (s != BT_OK) return s;
    return bt_ball_attention(Q, K, V, perm, npad, rows, m, H, d, dt, O, stream);
}
