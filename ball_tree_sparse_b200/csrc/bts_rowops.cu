// Element- and row-wise kernels around the tree: the 45-degree rotation for the
// rotated-tree layers (author's thread: cross-partition exchange comes from
// rotating the tree, the counterpart of Swin's window shift), inverse / composed slot maps, and row gather / scatter into
// and out of tree order (thread post 9/N: a ball's points are contiguous).
// All of them are HBM-bound streams; each thread moves 16-byte vectors where
// the layout allows.
#include "bts_internal.cuh"

namespace bts {

constexpr int kRowThreads = 256;

static unsigned grid_for(int64_t work, int per_block)
{
    int64_t g = (work + per_block - 1) / per_block;
    const int64_t cap = 148 * 32;
    return unsigned(g < 1 ? 1 : (g > cap ? cap : g));
}

// x' = c*x - s*y, y' = s*x + c*y with every product and sum rounded on its own
__global__ void k_rotate_z(const float *__restrict__ in, int64_t n, float *__restrict__ out)
{
    const float c = __uint_as_float(0x3F3504F3u), s = c;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
        const float x = in[3 * i], y = in[3 * i + 1], z = in[3 * i + 2];
        const float xr = __fsub_rn(__fmul_rn(c, x), __fmul_rn(s, y));
        const float yr = __fadd_rn(__fmul_rn(s, x), __fmul_rn(c, y));
        out[3 * i] = xr;
        out[3 * i + 1] = yr;
        out[3 * i + 2] = z;
    }
}

__global__ void k_invert(const int32_t *__restrict__ perm, int64_t npad, int32_t *__restrict__ inv)
{
    for (int64_t s = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; s < npad; s += int64_t(gridDim.x) * blockDim.x) {
        const int32_t r = perm[s];
        if (r >= 0) inv[r] = int32_t(s);
    }
}

__global__ void k_compose(const int32_t *__restrict__ invA, const int32_t *__restrict__ permB, int64_t npad,
                          int32_t *__restrict__ map)
{
    for (int64_t s = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; s < npad; s += int64_t(gridDim.x) * blockDim.x) {
        const int32_t r = permB[s];
        map[s] = r >= 0 ? invA[r] : -1;
    }
}

// One 16-byte (VEC) or 4-byte or 1-byte unit per thread step; `units` per row.
template <typename U, bool GATHER>
__global__ void k_rows(const uint8_t *__restrict__ src, const int32_t *__restrict__ idx, int64_t npad, int units,
                       uint8_t *__restrict__ dst)
{
    const int64_t total = npad * units;
    for (int64_t t = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; t < total; t += int64_t(gridDim.x) * blockDim.x) {
        const int64_t s = t / units;
        const int u = int(t - s * units);
        const int32_t r = idx[s];
        if (GATHER) {
            U val{};
            if (r >= 0) val = reinterpret_cast<const U *>(src)[int64_t(r) * units + u];
            reinterpret_cast<U *>(dst)[s * units + u] = val;
        } else if (r >= 0) {
            reinterpret_cast<U *>(dst)[int64_t(r) * units + u] = reinterpret_cast<const U *>(src)[s * units + u];
        }
    }
}

template <bool GATHER>
static bt_status launch_rows(const void *src, const int32_t *idx, int64_t npad, int32_t row_bytes, void *dst,
                             cudaStream_t st)
{
    if (!src || !idx || !dst || npad < 0 || row_bytes < 1 || row_bytes > 65536) return BT_ERR_ARG;
    if (npad == 0) return BT_OK;
    const uintptr_t al = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst);
    const uint8_t *s = static_cast<const uint8_t *>(src);
    uint8_t *d = static_cast<uint8_t *>(dst);
    if ((row_bytes % 16) == 0 && (al % 16) == 0) {
        const int units = row_bytes / 16;
        k_rows<uint4, GATHER><<<grid_for(npad * units, kRowThreads), kRowThreads, 0, st>>>(s, idx, npad, units, d);
    } else if ((row_bytes % 4) == 0 && (al % 4) == 0) {
        const int units = row_bytes / 4;
        k_rows<uint32_t, GATHER><<<grid_for(npad * units, kRowThreads), kRowThreads, 0, st>>>(s, idx, npad, units,
                                                                                             d);
    } else {
        k_rows<uint8_t, GATHER><<<grid_for(npad * row_bytes, kRowThreads), kRowThreads, 0, st>>>(s, idx, npad,
                                                                                                 row_bytes, d);
    }
    return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
}

}  // namespace bts

using namespace bts;

extern "C" int32_t bt_version(void) { return 100; }

extern "C" bt_status bt_rotate_z(const float *in, int64_t N, float *out, void *stream)
{
    if (!in || !out || N < 0) return BT_ERR_ARG;
    if (N == 0) return BT_OK;
    k_rotate_z<<<grid_for(N, kRowThreads), kRowThreads, 0, static_cast<cudaStream_t>(stream)>>>(in, N, out);
    return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
}

extern "C" bt_status bt_invert_perm(const int32_t *perm, int64_t npad, int64_t n_rows, int32_t *inv, void *stream)
{
    if (!perm || !inv || npad < 0 || n_rows < 0 || n_rows > npad) return BT_ERR_ARG;
    if (npad == 0) return BT_OK;
    k_invert<<<grid_for(npad, kRowThreads), kRowThreads, 0, static_cast<cudaStream_t>(stream)>>>(perm, npad, inv);
    return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
}

extern "C" bt_status bt_compose(const int32_t *invA, const int32_t *permB, int64_t npad, int32_t *map, void *stream)
{
    if (!invA || !permB || !map || npad < 0) return BT_ERR_ARG;
    if (npad == 0) return BT_OK;
    k_compose<<<grid_for(npad, kRowThreads), kRowThreads, 0, static_cast<cudaStream_t>(stream)>>>(invA, permB, npad,
                                                                                                 map);
    return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
}

extern "C" bt_status bt_gather(const void *X, const int32_t *idx, int64_t npad, int32_t row_bytes, void *Y,
                               void *stream)
{
    return launch_rows<true>(X, idx, npad, row_bytes, Y, static_cast<cudaStream_t>(stream));
}

extern "C" bt_status bt_scatter(const void *Y, const int32_t *idx, int64_t npad, int32_t row_bytes, void *X,
                                void *stream)
{
    return launch_rows<false>(Y, idx, npad, row_bytes, X, static_cast<cudaStream_t>(stream));
}
