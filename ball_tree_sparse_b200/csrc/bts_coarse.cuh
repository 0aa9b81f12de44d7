// Coarser tree levels (author's thread on Erwin, posts 8/N and 9/N): the tree
// is coarsened and refined while the attention ball keeps its size, and since
// the points of every node are contiguous at every level, pooling to a parent
// level is a mean over consecutive slots and refinement copies a parent back
// to its children.
//   k_pool_mean  one thread per (coarse token, 16-byte unit of the row): the
//                mean over the real slots of the node, in float, plus the
//                coarse slot map (j, or -1 for a node without a real point);
//                blockIdx.y picks one of up to three tensors (Q, K, V).
//   k_unpool     one thread per (slot, 16-byte unit): the node's row copied
//                to the slot's original row.
// Both are HBM streams.  The coarse level's ball attention is the ordinary
// ball attention over the coarse tokens with the coarse slot map as its perm.
// This file is included at the end of bts_attn.cu (one translation unit with
// the attention status word).
#pragma once

#include <type_traits>

namespace bts {

template <typename T>
struct PoolTensors {
    const T *src[3];
    T *dst[3];
};

template <typename T, int EPU>
__device__ __forceinline__ void load_f32(const T *p, float (&f)[EPU])
{
    if constexpr (EPU == 1) {
        if constexpr (std::is_same<T, float>::value) f[0] = p[0];
        else f[0] = __bfloat162float(p[0]);
    } else if constexpr (std::is_same<T, float>::value) {
        const float4 v = *reinterpret_cast<const float4 *>(p);
        f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    } else {
        bf16x8_to_f32(*reinterpret_cast<const uint4 *>(p), f);
    }
}

template <typename T, int EPU>
__device__ __forceinline__ void store_f32(T *p, const float (&f)[EPU])
{
    if constexpr (EPU == 1) {
        if constexpr (std::is_same<T, float>::value) p[0] = f[0];
        else p[0] = __float2bfloat16_rn(f[0]);
    } else if constexpr (std::is_same<T, float>::value) {
        *reinterpret_cast<float4 *>(p) = make_float4(f[0], f[1], f[2], f[3]);
    } else {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
            w[e] = *reinterpret_cast<const uint32_t *>(&b);
        }
        *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

template <typename T, int EPU>
__global__ void __launch_bounds__(256) k_pool_mean(PoolTensors<T> a, const int32_t *__restrict__ perm,
                                                   int64_t ncoarse, int64_t rows, int units, int stride,
                                                   int32_t *__restrict__ cperm, uint32_t *status)
{
    const int y = blockIdx.y;  // selected without a dynamic index into the parameter array
    const T *__restrict__ src = y == 0 ? a.src[0] : y == 1 ? a.src[1] : a.src[2];
    T *__restrict__ dst = y == 0 ? a.dst[0] : y == 1 ? a.dst[1] : a.dst[2];
    const int64_t total = ncoarse * units;
    for (int64_t t = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; t < total; t += int64_t(gridDim.x) * blockDim.x) {
        const int64_t j = t / units;
        const int u = int(t - j * units);
        float acc[EPU];
#pragma unroll
        for (int k = 0; k < EPU; ++k) acc[k] = 0.0f;
        int cnt = 0;
        for (int i = 0; i < stride; ++i) {
            const int64_t slot = j * stride + i;
            int64_t r = perm ? int64_t(perm[slot]) : slot;
            if (r >= rows) {
                record_error(status, BT_ERR_INTERNAL);
                r = -1;
            }
            if (r < 0) continue;
            ++cnt;
            float f[EPU];
            load_f32<T, EPU>(src + (size_t(r) * units + u) * EPU, f);
#pragma unroll
            for (int k = 0; k < EPU; ++k) acc[k] += f[k];
        }
        const float inv = cnt ? 1.0f / float(cnt) : 0.0f;
#pragma unroll
        for (int k = 0; k < EPU; ++k) acc[k] *= inv;
        store_f32<T, EPU>(dst + (size_t(j) * units + u) * EPU, acc);
        if (cperm && u == 0 && blockIdx.y == 0) cperm[j] = cnt ? int32_t(j) : -1;
    }
}

template <typename U>
__global__ void __launch_bounds__(256) k_unpool(const U *__restrict__ src, const int32_t *__restrict__ perm,
                                                int64_t npad, int64_t rows, int units, int stride,
                                                U *__restrict__ dst, uint32_t *status)
{
    const int64_t total = npad * units;
    for (int64_t t = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; t < total; t += int64_t(gridDim.x) * blockDim.x) {
        const int64_t slot = t / units;
        const int u = int(t - slot * units);
        const int64_t r = perm ? int64_t(perm[slot]) : slot;
        if (r >= rows) {
            record_error(status, BT_ERR_INTERNAL);
            continue;
        }
        if (r < 0) continue;
        dst[size_t(r) * units + u] = src[size_t(slot / stride) * units + u];
    }
}

static unsigned stream_grid(int64_t work)
{
    const int64_t g = (work + 255) / 256, cap = int64_t(148) * 16;
    return unsigned(g < 1 ? 1 : (g > cap ? cap : g));
}

static bt_status pool_check(const int32_t *perm, int64_t npad, int64_t rows, int32_t C, int32_t stride, bt_dtype dt)
{
    if (npad < 0 || rows < 0 || C < 1 || stride < 1) return BT_ERR_ARG;
    if (dt != BT_F32 && dt != BT_BF16) return BT_ERR_ARG;
    if ((stride & (stride - 1)) || npad % stride) return BT_ERR_SHAPE;
    if (!perm && rows < npad) return BT_ERR_ARG;
    if (npad > 0x7FFFFFFF || rows > 0x7FFFFFFF) return BT_ERR_UNSUPPORTED;
    return BT_OK;
}

template <typename T>
static bt_status launch_pool(PoolTensors<T> a, int nt, const int32_t *perm, int64_t npad, int64_t rows, int32_t C,
                             int32_t stride, int32_t *cperm, cudaStream_t st)
{
    const int64_t nc = npad / stride;
    if (nc == 0) return BT_OK;
    constexpr int VEC = 16 / sizeof(T);
    uint32_t *status = stream_status(st);
    if (!status) return BT_ERR_CUDA;
    uintptr_t al = 0;
    for (int i = 0; i < nt; ++i) al |= reinterpret_cast<uintptr_t>(a.src[i]) | reinterpret_cast<uintptr_t>(a.dst[i]);
    if (C % VEC == 0 && al % 16 == 0) {
        const int units = C / VEC;
        k_pool_mean<T, VEC><<<dim3(stream_grid(nc * units), nt), 256, 0, st>>>(a, perm, nc, rows, units, stride, cperm, status);
    } else {
        k_pool_mean<T, 1><<<dim3(stream_grid(nc * C), nt), 256, 0, st>>>(a, perm, nc, rows, C, stride, cperm, status);
    }
    return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
}

static size_t al256c(size_t v) { return (v + 255) & ~size_t(255); }

}  // namespace bts

extern "C" bt_status bt_pool_mean(const void *X, const int32_t *perm, int64_t npad, int64_t rows, int32_t C,
                                  int32_t stride, bt_dtype dt, void *Xc, int32_t *cperm, void *stream)
{
    using namespace bts;
    if (!X || !Xc) return BT_ERR_ARG;
    const bt_status s = pool_check(perm, npad, rows, C, stride, dt);
    if (s != BT_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dt == BT_F32) {
        PoolTensors<float> a{{static_cast<const float *>(X)}, {static_cast<float *>(Xc)}};
        return launch_pool<float>(a, 1, perm, npad, rows, C, stride, cperm, st);
    }
    PoolTensors<__nv_bfloat16> a{{static_cast<const __nv_bfloat16 *>(X)}, {static_cast<__nv_bfloat16 *>(Xc)}};
    return launch_pool<__nv_bfloat16>(a, 1, perm, npad, rows, C, stride, cperm, st);
}

extern "C" bt_status bt_unpool(const void *Xc, const int32_t *perm, int64_t npad, int64_t rows, int32_t C,
                               int32_t stride, bt_dtype dt, void *X, void *stream)
{
    using namespace bts;
    if (!X || !Xc) return BT_ERR_ARG;
    const bt_status s = pool_check(perm, npad, rows, C, stride, dt);
    if (s != BT_OK) return s;
    if (npad == 0) return BT_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t row_bytes = int64_t(C) * (dt == BT_F32 ? 4 : 2);
    const uintptr_t al = reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(Xc);
    uint32_t *status = stream_status(st);
    if (!status) return BT_ERR_CUDA;
    if (row_bytes % 16 == 0 && al % 16 == 0) {
        const int units = int(row_bytes / 16);
        k_unpool<uint4><<<stream_grid(npad * units), 256, 0, st>>>(static_cast<const uint4 *>(Xc), perm, npad, rows,
                                                                    units, stride, static_cast<uint4 *>(X), status);
    } else if (row_bytes % 4 == 0 && al % 4 == 0) {
        const int units = int(row_bytes / 4);
        k_unpool<uint32_t><<<stream_grid(npad * units), 256, 0, st>>>(static_cast<const uint32_t *>(Xc), perm, npad,
                                                                       rows, units, stride, static_cast<uint32_t *>(X), status);
    } else {
        const int units = int(row_bytes / 2);
        k_unpool<uint16_t><<<stream_grid(npad * units), 256, 0, st>>>(static_cast<const uint16_t *>(Xc), perm, npad,
                                                                       rows, units, stride, static_cast<uint16_t *>(X), status);
    }
    return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
}

extern "C" size_t bt_coarse_workspace_size(int64_t npad, int32_t H, int32_t d, int32_t stride, bt_dtype dt)
{
    using namespace bts;
    if (npad < 1 || H < 1 || d < 1 || stride < 1 || npad % stride || (dt != BT_F32 && dt != BT_BF16)) return 0;
    const size_t nc = size_t(npad / stride), tb = nc * size_t(H) * d * (dt == BT_F32 ? 4 : 2);
    return 4 * al256c(tb) + al256c(nc * 4);
}

extern "C" bt_status bt_coarse_ball_attention(const void *Q, const void *K, const void *V, const int32_t *perm,
                                              int64_t npad, int64_t rows, int32_t m, int32_t H, int32_t d,
                                              bt_dtype dt, int32_t stride, void *O, void *ws, size_t ws_bytes,
                                              void *stream)
{
    using namespace bts;
    if (!Q || !K || !V || !O || H < 1 || d < 1) return BT_ERR_ARG;
    bt_status s = pool_check(perm, npad, rows, H * d, stride, dt);
    if (s != BT_OK) return s;
    if (npad == 0) return BT_OK;
    if (m < 1 || (npad / stride) % m) return BT_ERR_SHAPE;
    const size_t need = bt_coarse_workspace_size(npad, H, d, stride, dt);
    if (!ws || reinterpret_cast<uintptr_t>(ws) % 256) return BT_ERR_WORKSPACE;
    if (ws_bytes < need) return BT_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t nc = npad / stride;
    const size_t tb = al256c(size_t(nc) * H * d * (dt == BT_F32 ? 4 : 2));
    uint8_t *w = static_cast<uint8_t *>(ws);
    void *qc = w, *kc = w + tb, *vc = w + 2 * tb, *oc = w + 3 * tb;
    int32_t *cperm = reinterpret_cast<int32_t *>(w + 4 * tb);
    if (dt == BT_F32) {
        PoolTensors<float> a{{static_cast<const float *>(Q), static_cast<const float *>(K), static_cast<const float *>(V)},
                             {static_cast<float *>(qc), static_cast<float *>(kc), static_cast<float *>(vc)}};
        s = launch_pool<float>(a, 3, perm, npad, rows, H * d, stride, cperm, st);
    } else {
        using B = __nv_bfloat16;
        PoolTensors<B> a{{static_cast<const B *>(Q), static_cast<const B *>(K), static_cast<const B *>(V)},
                         {static_cast<B *>(qc), static_cast<B *>(kc), static_cast<B *>(vc)}};
        s = launch_pool<B>(a, 3, perm, npad, rows, H * d, stride, cperm, st);
    }
    if (s != BT_OK) return s;
    s = bt_ball_attention(qc, kc, vc, cperm, nc, nc, m, H, d, dt, oc, stream);
    if (s != BT_OK) return s;
    return bt_unpool(oc, perm, npad, rows, H * d, stride, dt, O, stream);
}
