// Internal helpers shared by the libbts kernels (device code for sm_100a).
#pragma once

#include <atomic>
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "bts.h"

namespace bts {

// First-time set-up of per-device host state (function attributes, SM counts, symbol addresses): `init`
// runs under one lock until it succeeds, and `ready` turns true (release) after it, so concurrent first calls
// from several host threads neither race nor repeat it.  Returns init's status, BT_OK once set up.
template <typename F>
inline bt_status setup_once(std::atomic<bool> &ready, F &&init)
{
    if (ready.load(std::memory_order_acquire)) return BT_OK;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    if (ready.load(std::memory_order_relaxed)) return BT_OK;
    const bt_status s = init();
    if (s == BT_OK) ready.store(true, std::memory_order_release);
    return s;
}

// ---------------------------------------------------------------------------
// Device status word: the first error recorded wins; 0 = no error.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void record_error(uint32_t *status, uint32_t code)
{
    if (ld_relaxed(status) == 0u) atomicCAS(status, 0u, code);  // read first: no atomic storm once set
}

// Device address of the status word of stream `st` on the current device (assigned on the stream's first use;
// nullptr if the CUDA runtime refused the look-up).  Kernels record into it with record_error().
uint32_t *stream_status(cudaStream_t st);

// Copies a build workspace's status word into the stream's word (first error wins); called by one thread of
// every CTA of a build's last kernel, after that CTA's own work, so every error of the build reaches it.
__device__ __forceinline__ void fold_status(uint32_t *ws_status, uint32_t *stream_word)
{
    if (!stream_word) return;
    __threadfence();
    const uint32_t v = ld_relaxed(ws_status);
    if (v) record_error(stream_word, v);
}

__device__ __forceinline__ void st_relaxed(uint32_t *p, uint32_t v)
{
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------------------
// Order-preserving float key.  -0 is folded into +0 first, so the two compare
// equal (the index then decides, as for any other tie).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t float_key(float f)
{
    uint32_t u = __float_as_uint(f == 0.0f ? 0.0f : f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_float(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

constexpr uint32_t kDummyKey = 0xFFFFFFFFu;  // above every finite coordinate's key

// ---------------------------------------------------------------------------
// Decoupled look-back over the tiles of one segment.  A tile publishes its
// aggregate (flag 1) and, once it knows its exclusive prefix, its inclusive
// prefix (flag 2), both packed with the 30-bit value in one 32-bit word.
// Tiles get their ids from an atomic counter in launch order, so every
// predecessor is already resident; the spin is bounded all the same, and on
// exhaustion records BT_ERR_TIMEOUT and carries on with a zero prefix.
// ---------------------------------------------------------------------------
constexpr uint32_t kLbAggregate = 1u << 30;
constexpr uint32_t kLbInclusive = 2u << 30;
constexpr uint32_t kLbValue = (1u << 30) - 1u;
constexpr int kSpinLimit = 1 << 20;

template <int LB>
__device__ __forceinline__ uint32_t lookback(uint32_t *self, int stride, int k_in_segment, uint32_t aggregate,
                                             uint32_t *status)
{
    if (k_in_segment == 0) {
        st_relaxed(self, kLbInclusive | aggregate);
        return 0;
    }
    st_relaxed(self, kLbAggregate | aggregate);
    uint32_t excl = 0;
    // predecessors are read LB at a time with independent loads, nearest first, so a tile that
    // has to sum many aggregates pays one round trip per LB predecessors, not one per predecessor
    for (int q0 = k_in_segment - 1; q0 >= 0; q0 -= LB) {
        uint32_t w[LB];
#pragma unroll
        for (int i = 0; i < LB; ++i) w[i] = (q0 - i >= 0) ? ld_relaxed(self - (k_in_segment - q0 + i) * stride) : 0u;
        bool done = false;
#pragma unroll
        for (int i = 0; i < LB; ++i) {
            if (done || q0 - i < 0) break;
            uint32_t x = w[i];
            int spins = 0;
            while ((x >> 30) == 0u) {
                if (++spins > kSpinLimit) {
                    record_error(status, BT_ERR_TIMEOUT);
                    x = kLbInclusive;
                    break;
                }
                __nanosleep(32);
                x = ld_relaxed(self - (k_in_segment - q0 + i) * stride);
            }
            excl += x & kLbValue;
            done = (x >> 30) == 2u;
        }
        if (done) break;
    }
    st_relaxed(self, kLbInclusive | (excl + aggregate));
    return excl;
}

// ---------------------------------------------------------------------------
// Block-wide exclusive scan (any T with +), NT threads.  `scratch` holds
// NT/32 + 1 values.  Every thread of the block must call it.
// ---------------------------------------------------------------------------
template <int NT, typename T>
__device__ __forceinline__ T block_exclusive_scan(T v, T *scratch, T *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    T x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        T y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        T w = (lane < NT / 32) ? scratch[lane] : T(0);
        T s = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            T y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < NT / 32) scratch[lane] = s - w;
        if (lane == NT / 32 - 1) scratch[NT / 32] = s;
    }
    __syncthreads();
    T r = scratch[warp] + x - v;
    if (total) *total = scratch[NT / 32];
    __syncthreads();
    return r;
}

}  // namespace bts
