// Q/K/V projection of the point features, written in tree (slot) order.
//
// Erwin's attention layer projects every point's features to queries, keys and values ("Erwin: A
// Tree-based Hierarchical Transformer for Large-scale Physical Systems", author's thread post 7/N: attention
// inside every ball), and the points of a ball sit in consecutive slots (post 9/N), so a projection that
// writes Q, K and V in slot order leaves every ball a contiguous tile: the attention that follows loads
// whole tiles instead of gathering rows.
//
//   Q|K|V[inv[row], :] = X[row, :] Wt^T   (inv[row]: the row's slot; Wt [3 H d, C]: row j holds the weights of
//                                          output column j; columns [0, Hd) are Q, [Hd, 2Hd) K, [2Hd, 3Hd) V)
//
// The feature rows are read in their own order, as whole 128-row tiles (one TMA request per 64 columns), and
// each output row is stored at its slot: scattered 16-byte stores cost the same as ordered ones, while
// gathering the inputs row by row would cost one TMA request per four rows.
// k_qkv_project (bf16, C a multiple of 64 up to 512): weight-stationary, one CTA per SM.  The SMs are shared
// out over the chunks of 256 output columns (128 when C > 256); a CTA loads its chunk of Wt into shared
// memory once and walks its share of the 128-row tiles of X:
//   warp 8     producer: the Wt chunk, then the tiles' 128 x 64 K blocks of X through a 4-stage ring (TMA
//              tile loads, 128-byte swizzle; rows past the end read zeros);
//   warp 9     one thread issues the tcgen05 products D (TMEM, fp32, two accumulator buffers) += X block
//              (K-major) * Wt block (K-major), K = 64 per block;
//   warps 0-7  epilogue: two warps per 32 rows (TMEM lanes), each reading half of the row's columns of a
//              finished tile from TMEM, rounding to bf16 and storing 16-byte pieces to the row's slot of Q, K
//              or V, while the next tile accumulates in the other buffer.
// k_qkv_project_simt (float, or any shape the tensor-core kernel does not take): one thread per (row,
// output column), features staged in shared memory.
// k_zero_slots: zero rows of Q, K and V for the dummy slots (perm < 0), which no feature row fills.
// This file is included into bts_attn.cu (it uses the tensor-map helpers there).
#pragma once

namespace bts {

struct ProjPipe {
    static constexpr int BM = 128;                    // rows per tile
    static constexpr int BK = 64;                     // K elements per block: one 128-byte swizzle span
    static constexpr uint32_t XBLK = BM * BK * 2;     // 16 KB: one K block of an X tile
    static constexpr int XS = 4;                      // X ring stages (one K block each)
    static constexpr int THREADS = 320;                // 8 epilogue warps, producer, tensor-core issuer
    static constexpr int CMAX = 512;
    // output columns per CTA (its Wt chunk stays in shared memory): 256, or 128 when C > 256
    static int bn(int C) { return C <= 256 ? 256 : 128; }
    static uint32_t bytes(int C) { return uint32_t(C / BK) * uint32_t(bn(C)) * 128u + XS * XBLK + 1024; }
};

// Weight-stationary: CTA b owns output chunk b % nch (bn columns of Wt, loaded once into shared memory) and
// walks the 128-row tiles b / nch, b / nch + groups, ...  inv != NULL: feature row r goes to row inv[r] of
// Q/K/V (slot order; a slot outside [0, npad) is skipped and recorded as BT_ERR_INTERNAL); inv == NULL: to
// row r (original order).
template <int BN>
__global__ void __launch_bounds__(ProjPipe::THREADS, 1)
    k_qkv_project(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                  const int32_t *__restrict__ inv, int64_t npad, int64_t rows, int C, int nout, int hd,
                  int64_t tiles, __nv_bfloat16 *__restrict__ Qo, __nv_bfloat16 *__restrict__ Ko,
                  __nv_bfloat16 *__restrict__ Vo, uint32_t *status)
{
    using L = ProjPipe;
    constexpr uint32_t SBO8 = 8 * 128, SW128 = 2;
    constexpr uint32_t IDESC = idesc_bf16(BN, false);
    constexpr uint32_t WBLK = BN * 128;  // one K block of the Wt chunk
    extern __shared__ __align__(1024) uint8_t xsm[];
    __shared__ __align__(8) uint64_t sWFull, sXFull[L::XS], sXEmpty[L::XS], sAccFull[2], sAccEmpty[2];
    __shared__ uint32_t sTmem;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int KB = C / L::BK;
    const int nch = (nout + BN - 1) / BN;
    const int chunk = int(blockIdx.x) % nch;
    const int64_t groups = int64_t(gridDim.x) / nch;
    const int64_t first = int64_t(blockIdx.x) / nch;
    const uint32_t base = (smem_u32(xsm) + 1023u) & ~1023u;   // Wt chunk: KB blocks of [BN][128 B]
    const uint32_t xbase = base + uint32_t(KB) * WBLK;        // X ring

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sTmem)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sWFull)) : "memory");
        for (int i = 0; i < L::XS; ++i) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sXFull[i])) : "memory");
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sXEmpty[i])) : "memory");
        }
        for (int i = 0; i < 2; ++i) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sAccFull[i])) : "memory");
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 8;" ::"r"(smem_u32(&sAccEmpty[i])) : "memory");
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sTmem;

    if (warp == 8) {
        // ---------------- producer (one thread): the Wt chunk once, then the X tiles' K blocks ----------------
        if (lane == 0) {
            bool ok = true;
            mbar_expect_tx(smem_u32(&sWFull), uint32_t(KB) * WBLK);
            for (int k = 0; k < KB; ++k)
                tma_load_2d(base + k * WBLK, &tmW, k * L::BK, chunk * BN, smem_u32(&sWFull));
            int xi = 0;
            for (int64_t tile = first; tile < tiles && ok; tile += groups)
                for (int k = 0; k < KB && ok; ++k, ++xi) {
                    const int s = xi % L::XS;
                    if (xi >= L::XS) ok = mbar_wait(smem_u32(&sXEmpty[s]), ((xi / L::XS) - 1) & 1, status);
                    if (ok) {
                        mbar_expect_tx(smem_u32(&sXFull[s]), L::XBLK);
                        tma_load_2d(xbase + s * L::XBLK, &tmX, k * L::BK, int32_t(tile * L::BM), smem_u32(&sXFull[s]));
                    }
                }
        }
        __syncwarp();
    } else if (warp == 9) {
        // ---------------- tensor-core issue (one thread) ----------------
        if (lane == 0) {
            bool ok = mbar_wait(smem_u32(&sWFull), 0, status);
            tc_fence_after();
            int xi = 0, ai = 0;
            for (int64_t tile = first; tile < tiles && ok; tile += groups, ++ai) {
                const int ab = ai & 1;
                if (ai >= 2) ok = mbar_wait(smem_u32(&sAccEmpty[ab]), ((ai >> 1) - 1) & 1, status);
                tc_fence_after();
                const uint32_t tacc = tmem + uint32_t(ab) * BN;
                for (int k = 0; k < KB && ok; ++k, ++xi) {
                    const int s = xi % L::XS;
                    ok = mbar_wait(smem_u32(&sXFull[s]), (xi / L::XS) & 1, status);
                    tc_fence_after();
                    if (ok) {
                        const uint32_t xa = xbase + s * L::XBLK, wb = base + k * WBLK;
#pragma unroll
                        for (int kk = 0; kk < L::BK / 16; ++kk)
                            mma_bf16(tacc, smem_desc_sw(xa + 32 * kk, 16, SBO8, SW128),
                                     smem_desc_sw(wb + 32 * kk, 16, SBO8, SW128), IDESC, (k | kk) != 0);
                    }
                    mma_commit(smem_u32(&sXEmpty[s]));  // the X stage is free once these products finish
                }
                mma_commit(smem_u32(&sAccFull[ab]));
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: warp w owns TMEM lanes 32 (w % 4) .. +31 (rows of the tile) and the
        // column half w / 4 of the accumulator; two 32-column loads in flight per wait ----------------
        const int r = (warp & 3) * 32 + lane;
        const int half = warp >> 2;
        const uint32_t lanebase = uint32_t((warp & 3) * 32) << 16;
        bool ok = true;
        int ai = 0;
        for (int64_t tile = first; tile < tiles && ok; tile += groups, ++ai) {
            const int64_t row = tile * L::BM + r;
            int32_t orow = -1;
            if (row < rows) {
                orow = inv ? __ldg(inv + row) : int32_t(row);
                if (inv && (orow < 0 || orow >= npad)) {  // not a slot: never write it
                    if (half == 0) record_error(status, BT_ERR_INTERNAL);
                    orow = -1;
                }
            }
            const int ab = ai & 1;
            ok = mbar_wait(smem_u32(&sAccFull[ab]), (ai >> 1) & 1, status);
            tc_fence_after();
            const uint32_t tacc = tmem + uint32_t(ab) * BN + uint32_t(half * (BN / 2)) + lanebase;
#pragma unroll 1
            for (int c = 0; c < BN / 2 / 32; c += 2) {
                const int col0 = chunk * BN + half * (BN / 2) + c * 32;
                if (col0 >= nout) break;  // the same for every thread of the warp
                uint32_t v[2][32];
                tmem_ld32_nowait(tacc + c * 32, v[0]);
                tmem_ld32_nowait(tacc + (c + 1) * 32, v[1]);
                tmem_wait_ld();
                if (ok && orow >= 0) {
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        const int j0 = col0 + 8 * g;
                        if (j0 >= nout) break;  // 3*H*d is a multiple of 8, so a group never straddles it
                        const int t = j0 / hd, within = j0 - t * hd;
                        __nv_bfloat16 *dst = (t == 0 ? Qo : t == 1 ? Ko : Vo) + size_t(orow) * hd + within;
                        const uint32_t *vv = v[g >> 2] + 8 * (g & 3);
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 pb =
                                __floats2bfloat162_rn(__uint_as_float(vv[2 * e]), __uint_as_float(vv[2 * e + 1]));
                            w[e] = *reinterpret_cast<const uint32_t *>(&pb);
                        }
                        *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&sAccEmpty[ab])) : "memory");
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
    }
}

// CUDA-core projection (float or bf16 inputs, any C): block = 32 feature rows x 128 output columns, the 32
// rows staged in shared memory; accumulation in float.  Output rows as for k_qkv_project.
template <typename T>
__global__ void __launch_bounds__(128) k_qkv_project_simt(const T *__restrict__ X, const T *__restrict__ Wt,
                                                          const int32_t *__restrict__ inv, int64_t npad, int64_t rows,
                                                          int C, int nout, int hd, T *__restrict__ Qo,
                                                          T *__restrict__ Ko, T *__restrict__ Vo, uint32_t *status)
{
    extern __shared__ float xs[];  // [32][C]
    __shared__ int32_t sOut[32];
    const int64_t r0 = int64_t(blockIdx.x) * 32;
    if (threadIdx.x < 32) {
        const int64_t row = r0 + threadIdx.x;
        int32_t o = -1;
        if (row < rows) {
            o = inv ? inv[row] : int32_t(row);
            if (inv && (o < 0 || o >= npad)) {
                if (blockIdx.y == 0) record_error(status, BT_ERR_INTERNAL);
                o = -1;
            }
        }
        sOut[threadIdx.x] = o;
    }
    for (int i = threadIdx.x; i < 32 * C; i += blockDim.x) {
        const int rr = i / C, c = i - rr * C;
        xs[i] = r0 + rr < rows ? to_f(X[size_t(r0 + rr) * C + c]) : 0.0f;
    }
    __syncthreads();
    const int j = blockIdx.y * 128 + threadIdx.x;
    if (j >= nout) return;
    const int t = j / hd, within = j - t * hd;
    T *dst = t == 0 ? Qo : t == 1 ? Ko : Vo;
    const T *w = Wt + size_t(j) * C;
    for (int rr = 0; rr < 32; ++rr) {
        if (sOut[rr] < 0) continue;
        float acc = 0.0f;
        for (int c = 0; c < C; ++c) acc = fmaf(xs[rr * C + c], to_f(w[c]), acc);
        dst[size_t(sOut[rr]) * hd + within] = from_f<T>(acc);
    }
}

// Zero rows of Q, K and V for every dummy slot (perm < 0): one thread per slot, which writes the slot's three
// rows (row_units units of U each) only if the slot is a dummy.
template <typename U>
__global__ void __launch_bounds__(256) k_zero_slots(const int32_t *__restrict__ perm, int64_t npad, int row_units,
                                                    U *__restrict__ Q, U *__restrict__ K, U *__restrict__ V)
{
    for (int64_t s = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; s < npad; s += int64_t(gridDim.x) * blockDim.x) {
        if (perm[s] >= 0) continue;
        const size_t o = size_t(s) * row_units;
        for (int u = 0; u < row_units; ++u) {
            Q[o + u] = U{};
            K[o + u] = U{};
            V[o + u] = U{};
        }
    }
}

static bt_status launch_project(const void *X, int64_t rows, int32_t C, const void *Wt, int32_t H, int32_t d,
                                bt_dtype dt, const int32_t *perm, const int32_t *inv, int64_t npad, void *Q, void *K,
                                void *V, cudaStream_t st)
{
    uint32_t *status = stream_status(st);
    if (!status) return BT_ERR_CUDA;
    const int hd = H * d, nout = 3 * hd;
    const size_t esz = dt == BT_F32 ? 4 : 2;
    if (perm) {  // dummy slots: zero rows (no feature row is projected into them)
        const int64_t g = npad < 148 * 8 * 256 ? (npad + 255) / 256 : 148 * 8;
        const size_t row_bytes = size_t(hd) * esz;
        const uintptr_t qa = reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) |
                             reinterpret_cast<uintptr_t>(V);
        if (row_bytes % 16 == 0 && qa % 16 == 0)
            k_zero_slots<uint4><<<unsigned(g > 0 ? g : 1), 256, 0, st>>>(
                perm, npad, int(row_bytes / 16), static_cast<uint4 *>(Q), static_cast<uint4 *>(K),
                static_cast<uint4 *>(V));
        else
            k_zero_slots<uint16_t><<<unsigned(g > 0 ? g : 1), 256, 0, st>>>(
                perm, npad, int(row_bytes / 2), static_cast<uint16_t *>(Q), static_cast<uint16_t *>(K),
                static_cast<uint16_t *>(V));
    }
    if (rows == 0) return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
    const uintptr_t al = reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(Wt) |
                         reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) |
                         reinterpret_cast<uintptr_t>(V);
    if (dt == BT_BF16 && C % ProjPipe::BK == 0 && C <= ProjPipe::CMAX && hd % 8 == 0 && nout >= ProjPipe::bn(C) &&
        al % 16 == 0 && rows >= ProjPipe::BM && rows < 0x7FFFFFFF) {
        static std::atomic<bool> set[64] = {};
        static int sms[64] = {0};
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return BT_ERR_CUDA;
        if (dev < 0 || dev >= 64) return BT_ERR_UNSUPPORTED;
        const bt_status s0 = setup_once(set[dev], [&]() -> bt_status {
            if (cudaFuncSetAttribute(k_qkv_project<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     int(ProjPipe::bytes(256))) ||
                cudaFuncSetAttribute(k_qkv_project<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     int(ProjPipe::bytes(512))))
                return BT_ERR_CUDA;
            int n = 0;
            if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return BT_ERR_CUDA;
            sms[dev] = n;
            return BT_OK;
        });
        if (s0 != BT_OK) return s0;
        const int BN = ProjPipe::bn(C);
        CUtensorMap mx, mw;
        if (!tile_map(&mx, X, rows, C, ProjPipe::BK, ProjPipe::BM) || !tile_map(&mw, Wt, nout, C, ProjPipe::BK, BN))
            return BT_ERR_CUDA;
        const int64_t tiles = (rows + ProjPipe::BM - 1) / ProjPipe::BM;
        const int nch = (nout + BN - 1) / BN;
        // CTAs per output chunk: the SMs shared out, no more than there are tiles
        int64_t groups = sms[dev] / nch;
        if (groups < 1) groups = 1;
        if (groups > tiles) groups = tiles;
        const unsigned grid = unsigned(groups * nch);
        if (BN == 256)
            k_qkv_project<256><<<grid, ProjPipe::THREADS, ProjPipe::bytes(C), st>>>(
                mx, mw, perm ? inv : nullptr, npad, rows, C, nout, hd, tiles, static_cast<__nv_bfloat16 *>(Q),
                static_cast<__nv_bfloat16 *>(K), static_cast<__nv_bfloat16 *>(V), status);
        else
            k_qkv_project<128><<<grid, ProjPipe::THREADS, ProjPipe::bytes(C), st>>>(
                mx, mw, perm ? inv : nullptr, npad, rows, C, nout, hd, tiles, static_cast<__nv_bfloat16 *>(Q),
                static_cast<__nv_bfloat16 *>(K), static_cast<__nv_bfloat16 *>(V), status);
        return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
    }
    const size_t smem = size_t(32) * C * sizeof(float);
    if (smem > 200 * 1024) return BT_ERR_UNSUPPORTED;
    dim3 grid(unsigned((rows + 31) / 32), unsigned((nout + 127) / 128));
    const int32_t *iv = perm ? inv : nullptr;
    if (dt == BT_F32) {
        if (smem > 48 * 1024 && cudaFuncSetAttribute(k_qkv_project_simt<float>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)))
            return BT_ERR_CUDA;
        k_qkv_project_simt<float><<<grid, 128, smem, st>>>(
            static_cast<const float *>(X), static_cast<const float *>(Wt), iv, npad, rows, C, nout, hd,
            static_cast<float *>(Q), static_cast<float *>(K), static_cast<float *>(V), status);
    } else {
        if (smem > 48 * 1024 && cudaFuncSetAttribute(k_qkv_project_simt<__nv_bfloat16>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)))
            return BT_ERR_CUDA;
        k_qkv_project_simt<__nv_bfloat16><<<grid, 128, smem, st>>>(
            static_cast<const __nv_bfloat16 *>(X), static_cast<const __nv_bfloat16 *>(Wt), iv, npad, rows, C, nout,
            hd, static_cast<__nv_bfloat16 *>(Q), static_cast<__nv_bfloat16 *>(K), static_cast<__nv_bfloat16 *>(V),
            status);
    }
    return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
}

}  // namespace bts
