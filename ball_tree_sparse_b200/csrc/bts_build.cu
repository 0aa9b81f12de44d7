// Ball-tree build on the GPU: median split along the widest axis, emitted as a
// permutation (the tree of "Erwin: A Tree-based Hierarchical Transformer for
// Large-scale Physical Systems", author's thread posts 6/N, 9/N and 15/N).
//
// Design (sm_100a, one cloud or a batch of clouds).  Every shape sorts each
// cloud once per axis (order-preserving float keys, ties by id) and then splits
// the three sorted lists stably at every level: a node's widest axis comes from
// the two ends of its lists, its median is the element at position s/2 of that
// axis' list, and every list stays sorted inside both children, so no level
// needs a selection.  Three shapes of this algorithm, chosen per call:
//   a. k_cluster_build - clouds of at most 32,768 slots (power-of-two slot
//                     counts): the whole build in one launch, one thread-block
//                     cluster per cloud, the lists in distributed shared
//                     memory as 8-byte records ((key, id) while sorting, the
//                     point's three ranks and id afterwards).
//   b. record path  - larger power-of-two clouds (at most 2^21 slots): k_init
//                     (keys, digit histograms), four radix passes
//                     (k_sort_pass, tiles chained by a bounded decoupled
//                     look-back), k_records (every list element becomes the
//                     point's three ranks), one k_level_r launch per level
//                     whose nodes exceed the shared-memory tail, and k_tail_r
//                     (the remaining levels in shared memory, leaves sorted by
//                     id).
//   c. index lists  - any other shape: the same presort, then k_level and
//                     k_tail on the lists X, Y, Z and the index list I, with
//                     the keys gathered through the lists.
#include <algorithm>
#include <cstring>

#include <cooperative_groups.h>

#include "bts_internal.cuh"

namespace bts {

constexpr int kSortTile = 2048;      // keys per radix tile
constexpr int kSortThreads = 256;
constexpr int kLevelThreads = 512;
constexpr int kLevelTileMin = 512;       // smallest wide-level tile, slots per list (or m when m is larger)
constexpr int kLevelTileMax = 4096;      // largest: eight slots of each list per thread
constexpr int kLevelTilesWanted = 148;   // large builds: about one wide-level tile per SM (two fit one)
constexpr int kTailMax = 4096;         // largest node finished in shared memory
constexpr int kTailMin = 512;          // smallest tail node (for m <= 512)
constexpr int kTailCtasWanted = 2 * 148;  // aim for two tail CTAs per SM
constexpr int kCounterLevel0 = 8;

struct Plan {
    int32_t B, m, T, TP, nlev, sort_tiles;
    int32_t rec;  // 1: record path (every cloud a power-of-two slot count of at most 2^21)
    uint32_t *sstatus;  // status word of the call's stream: the build's last kernel folds the workspace word in
    int64_t npad;
    int64_t pad[BT_MAX_CLOUDS + 1];
    int64_t n[BT_MAX_CLOUDS];
    int64_t row0[BT_MAX_CLOUDS];
    int32_t sort_tile0[BT_MAX_CLOUDS + 1];
    int32_t glev[BT_MAX_CLOUDS];
    int32_t tail0[BT_MAX_CLOUDS + 1];
};

// A wide level's per-tile counts words sit one cache line (16 words) apart: every later tile of the node polls
// each of them, and packed into a few lines they were a hot spot.
constexpr size_t kAggStride = 16;

struct Layout {
    size_t counters, hist, sst, lst, ctrl_end, keys, sk, sv, lists, total;
};

static int ilog2(int64_t v)
{
    int r = 0;
    while ((int64_t(1) << (r + 1)) <= v) ++r;
    return r;
}

static int64_t padded_size(int64_t n, int32_t m)
{
    int64_t leaves = max64(1, (n + m - 1) / m), p = 1;
    while (p < leaves) p <<= 1;
    return p * m;
}

static size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Fills the plan; returns BT_OK or an argument/shape error.
static bt_status make_plan(const int64_t *offsets, int32_t B, int32_t m, Plan &P)
{
    if (!offsets || B < 1) return BT_ERR_ARG;
    if (B > BT_MAX_CLOUDS) return BT_ERR_UNSUPPORTED;
    if (m < 1 || m > 1024) return BT_ERR_SHAPE;
    if (offsets[0] != 0) return BT_ERR_ARG;
    std::memset(&P, 0, sizeof(P));
    P.B = B;
    P.m = m;
    // wide-level tile TP = m * 2^k slots: at least kLevelTileMin, about npad / kLevelTilesWanted on large
    // builds (fewer, larger tiles: fewer predecessors to sum), at most kLevelTileMax
    {
        int64_t all = 0;
        for (int b = 0; b < B; ++b) all += padded_size(offsets[b + 1] - offsets[b], m);
        const int64_t want = std::max<int64_t>(kLevelTileMin, all / kLevelTilesWanted);
        int64_t tp = m;
        while (tp < want && 2 * tp <= kLevelTileMax) tp *= 2;
        P.TP = int32_t(tp);
    }
    int64_t npad_all = 0;
    for (int b = 0; b < B; ++b) {
        const int64_t n = offsets[b + 1] - offsets[b];
        if (n < 1) return BT_ERR_ARG;
        npad_all += padded_size(n, m);
    }
    // tail node size T = m * 2^t: small enough that the tail runs on about kTailCtasWanted CTAs
    // when the batch is large, but never below max(4m, 512) slots (each wide level is a launch,
    // so tiny batches keep their levels in shared memory) and never above kTailMax
    {
        const int tmax = ilog2(kTailMax / m);
        const int tmin = std::min(tmax, std::max(2, m <= kTailMin ? ilog2(kTailMin / m) : 0));
        int t = npad_all >= int64_t(kTailCtasWanted) * m ? ilog2(npad_all / (int64_t(kTailCtasWanted) * m)) : 0;
        t = std::max(std::min(t, tmax), tmin);
        P.T = m << t;
    }
    const int t = ilog2(P.T / m);
    // every wide node has at least 2T slots: a wide-level tile must not be larger
    P.TP = std::min(P.TP, 2 * P.T);
    int64_t pad = 0;
    int32_t st = 0, tt = 0, nlev = 0;
    for (int b = 0; b < B; ++b) {
        int64_t n = offsets[b + 1] - offsets[b];
        if (n < 1) return BT_ERR_ARG;
        int64_t np = padded_size(n, m);
        P.pad[b] = pad;
        P.n[b] = n;
        P.row0[b] = offsets[b];
        P.sort_tile0[b] = st;
        P.tail0[b] = tt;
        int L = ilog2(np / m);
        P.glev[b] = std::max(0, L - t);
        nlev = std::max(nlev, P.glev[b]);
        st += int32_t((np + kSortTile - 1) / kSortTile);
        tt += int32_t(1) << P.glev[b];
        pad += np;
    }
    P.pad[B] = pad;
    P.sort_tile0[B] = st;
    P.tail0[B] = tt;
    P.sort_tiles = st;
    P.nlev = nlev;
    P.npad = pad;
    if (pad > (int64_t(1) << 30) || offsets[B] > (int64_t(1) << 30)) return BT_ERR_UNSUPPORTED;
    // invariants the kernels rely on: every wide node splits into whole tiles, tails fit shared memory
    for (int b = 0; b < B; ++b)
        for (int lev = 0; lev < P.glev[b]; ++lev) {
            const int64_t sn = (P.pad[b + 1] - P.pad[b]) >> lev;
            if (sn <= P.T || sn % P.TP || sn / P.TP < 1) return BT_ERR_INTERNAL;
        }
    if (P.TP > kLevelTileMax || P.T > kTailMax || P.T < m || (P.T & 1)) return BT_ERR_INTERNAL;
    P.rec = 1;
    for (int b = 0; b < B; ++b) {
        const int64_t np = P.pad[b + 1] - P.pad[b];
        if ((np & (np - 1)) || np > (int64_t(1) << 21)) P.rec = 0;
    }
    return BT_OK;
}

static Layout make_layout(const Plan &P)
{
    Layout L{};
    const size_t np = size_t(P.npad);
    L.counters = 64;  // word 0 is the device status
    L.hist = 512;
    L.sst = L.hist + size_t(3) * P.B * 4 * 256 * 4;
    L.lst = L.sst + size_t(4) * 3 * P.sort_tiles * 256 * 4;
    L.ctrl_end = align256(L.lst + size_t(std::max(P.nlev, 1)) * (np / P.TP) * 8 * kAggStride);
    L.keys = L.ctrl_end;
    L.sk = align256(L.keys + 3 * np * 4);
    L.sv = align256(L.sk + 2 * 3 * np * 4);
    L.lists = align256(L.sv + 2 * 3 * np * 4);
    L.total = align256(L.lists + 2 * 4 * np * 4);
    return L;
}

// Lanes of the warp whose 8-bit digit equals this lane's (bit i set for lane i), among the lanes with
// `valid` set: eight ballots, one per digit bit (the warp-level multisplit of radix-sort literature).
__device__ __forceinline__ uint32_t digit_peers(uint32_t d, bool valid)
{
    uint32_t mask = __ballot_sync(0xffffffffu, valid);
#pragma unroll
    for (int bit = 0; bit < 8; ++bit) {
        const bool on = (d >> bit) & 1u;
        const uint32_t b = __ballot_sync(0xffffffffu, on);
        mask &= on ? b : ~b;
    }
    return mask;
}

// Distributed shared memory of the cluster, by explicit shared::cluster addresses.
__device__ __forceinline__ uint32_t cluster_addr(const void *local_smem, uint32_t rank)
{
    const uint32_t a = uint32_t(__cvta_generic_to_shared(local_smem));
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long ld_cluster_u64(uint32_t addr)
{
    unsigned long long v;
    asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, const uint4 &v)
{
    asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// ---------------------------------------------------------------------------
// 1. keys, index list, digit histograms
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kSortThreads) k_init(Plan P, const float *__restrict__ coords,
                                                       uint32_t *__restrict__ keys, uint32_t *__restrict__ ilist,
                                                       uint32_t *__restrict__ hist, uint32_t *status)
{
    __shared__ uint32_t sh[3 * 4 * 256];
    const int tid = threadIdx.x, lane = tid & 31;
    for (int i = tid; i < 3 * 4 * 256; i += kSortThreads) sh[i] = 0;
    __syncthreads();
    const int r = blockIdx.x;
    int b = 0;
    while (b + 1 < P.B && P.sort_tile0[b + 1] <= r) ++b;
    const int k = r - P.sort_tile0[b];
    const int64_t base = P.pad[b] + int64_t(k) * kSortTile;
    const int cnt = int(min64(kSortTile, P.pad[b + 1] - base));
    for (int e0 = 0; e0 < kSortTile; e0 += kSortThreads) {
        const int e = e0 + tid;
        const bool ok = e < cnt;
        const int64_t pid = base + e;
        const int64_t local = pid - P.pad[b];
        const bool real = ok && local < P.n[b];
        uint32_t key[3];
#pragma unroll
        for (int a = 0; a < 3; ++a) {
            key[a] = kDummyKey;
            if (real) {
                float c = coords[(P.row0[b] + local) * 3 + a];
                if (!isfinite(c)) record_error(status, BT_ERR_NONFINITE);
                key[a] = float_key(c);
            }
            if (ok) keys[int64_t(a) * P.npad + pid] = key[a];
        }
        if (ok) ilist[pid] = uint32_t(pid);
        const bool full = __all_sync(0xffffffffu, ok);
#pragma unroll
        for (int a = 0; a < 3; ++a) {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const uint32_t d = (key[a] >> (8 * p)) & 255u;
                // high bytes are usually equal across a warp: one atomic instead of 32 colliding ones
                const uint32_t d0 = __shfl_sync(0xffffffffu, d, 0);
                if (full && __all_sync(0xffffffffu, d == d0)) {
                    if (lane == 0) atomicAdd(&sh[(a * 4 + p) * 256 + d], 32u);
                } else if (ok) {
                    atomicAdd(&sh[(a * 4 + p) * 256 + d], 1u);
                }
            }
        }
    }
    __syncthreads();
    for (int i = tid; i < 3 * 4 * 256; i += kSortThreads) {
        const uint32_t v = sh[i];
        if (v) {
            const int a = i >> 10, rest = i & 1023;
            atomicAdd(&hist[(size_t(a) * P.B + b) * 1024 + rest], v);
        }
    }
}

// ---------------------------------------------------------------------------
// 2. one stable LSD radix pass over 8 bits, all (axis, cloud) segments at once
// ---------------------------------------------------------------------------
template <int PASS>
__global__ void __launch_bounds__(kSortThreads, 4) k_sort_pass(Plan P, const uint32_t *__restrict__ kin,
                                                            const uint32_t *__restrict__ vin,
                                                            uint32_t *__restrict__ kout, uint32_t *__restrict__ vout,
                                                            const uint32_t *__restrict__ hist, uint32_t *sst,
                                                            uint32_t *counters, uint32_t *status,
                                                            uint32_t *__restrict__ rank_out)
{
    constexpr int NT = kSortThreads, NW = NT / 32, PER_WARP = kSortTile / NW, ROUNDS = PER_WARP / 32;
    constexpr int SHIFT = 8 * PASS;
    extern __shared__ __align__(16) uint32_t dyn[];
    // sorted keys and values of the tile; the values in input order (kept out of registers: four CTAs fit an SM)
    uint32_t *skey = dyn, *sval = dyn + kSortTile, *vin_s = dyn + 2 * kSortTile;
    __shared__ uint32_t whist[NW][256];
    __shared__ uint32_t tstart[256], gpos[256];
    __shared__ uint32_t scratch[NT / 32 + 1];
    __shared__ uint32_t s_tile;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) s_tile = atomicAdd(&counters[PASS], 1u);
    for (int i = tid; i < NW * 256; i += NT) (&whist[0][0])[i] = 0;
    __syncthreads();
    const int id = int(s_tile);
    // tiles of the three axes interleaved in dispatch order: a third as many tiles of one segment in flight, so
    // the look-back walks back over fewer unfinished predecessors (they still precede in dispatch order)
    const int a = id % 3, r = id / 3;
    int b = 0;
    while (b + 1 < P.B && P.sort_tile0[b + 1] <= r) ++b;
    const int k = r - P.sort_tile0[b];
    const int64_t seg_size = P.pad[b + 1] - P.pad[b];
    const int64_t seg_base = int64_t(a) * P.npad + P.pad[b];
    const int64_t tile_base = seg_base + int64_t(k) * kSortTile;
    const int cnt = int(min64(kSortTile, seg_size - int64_t(k) * kSortTile));

    uint32_t key[ROUNDS], rnk[ROUNDS];
    const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
    for (int q = 0; q < ROUNDS; ++q) {
        const int e = warp * PER_WARP + q * 32 + lane;
        const bool ok = e < cnt;
        key[q] = ok ? kin[tile_base + e] : 0u;
        if (ok) vin_s[e] = PASS == 0 ? uint32_t(P.pad[b] + int64_t(k) * kSortTile + e) : vin[tile_base + e];
    }
    // stable rank of every element among equal digits of its warp, warp counts (the digit is recomputed from
    // the key wherever it is needed; slot e < cnt holds an element)
#pragma unroll
    for (int q = 0; q < ROUNDS; ++q) {
        const bool ok = warp * PER_WARP + q * 32 + lane < cnt;
        const uint32_t dg = (key[q] >> SHIFT) & 255u;
        const uint32_t peers = digit_peers(dg, ok);
        const uint32_t base = ok ? whist[warp][dg] : 0u;
        __syncwarp();
        if (ok && (peers & lt) == 0u) whist[warp][dg] = base + __popc(peers);
        __syncwarp();
        rnk[q] = base + __popc(peers & lt);
    }
    __syncthreads();
    uint32_t dcount = 0;
    if (tid < 256) {
        uint32_t run = 0;
        for (int w = 0; w < NW; ++w) {
            const uint32_t c = whist[w][tid];
            whist[w][tid] = run;
            run += c;
        }
        dcount = run;
    }
    const uint32_t ts = block_exclusive_scan<NT, uint32_t>(tid < 256 ? dcount : 0u, scratch, nullptr);
    const int g = a * P.B + b;
    const uint32_t hc = tid < 256 ? hist[(size_t(g) * 4 + PASS) * 256 + tid] : 0u;
    const uint32_t gb = block_exclusive_scan<NT, uint32_t>(hc, scratch, nullptr);
    if (tid < 256) {
        const uint32_t excl =
            lookback<16>(&sst[(size_t(PASS) * 3 * P.sort_tiles + size_t(a) * P.sort_tiles + r) * 256 + tid], 256,
                         k, dcount, status);
        tstart[tid] = ts;
        gpos[tid] = gb + excl - ts;  // modulo 2^32; + local index gives the position in the segment
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < ROUNDS; ++q) {
        const int e = warp * PER_WARP + q * 32 + lane;
        if (e < cnt) {
            const uint32_t dg = (key[q] >> SHIFT) & 255u;
            const uint32_t j = tstart[dg] + whist[warp][dg] + rnk[q];
            skey[j] = key[q];
            sval[j] = vin_s[e];
        }
    }
    __syncthreads();
    for (int j = tid; j < cnt; j += NT) {
        const uint32_t kk = skey[j];
        const uint32_t d = (kk >> SHIFT) & 255u;
        const int64_t rel = int64_t(uint32_t(gpos[d] + uint32_t(j)));
        if (rel >= seg_size) {  // counts disagree with the histogram: never write outside the segment
            record_error(status, BT_ERR_INTERNAL);
            continue;
        }
        if (kout) kout[seg_base + rel] = kk;  // the last pass writes sorted keys only when asked
        vout[seg_base + rel] = sval[j];
        if (PASS == 3 && rank_out) {  // the id's rank on axis a; ids come from earlier passes: check them
            if (sval[j] < uint32_t(P.pad[b]) || sval[j] >= uint32_t(P.pad[b + 1]))
                record_error(status, BT_ERR_INTERNAL);
            else
                rank_out[int64_t(a) * P.npad + sval[j]] = uint32_t(rel);
        }
    }
}

// ---------------------------------------------------------------------------
// 3. one wide level: split every node larger than T at the median of its widest axis
// ---------------------------------------------------------------------------
// (key, id) < (pivot key, pivot id): the composite order that makes every key distinct
__device__ __forceinline__ bool before(uint32_t key, uint32_t id, uint32_t pkey, uint32_t pid)
{
    return key < pkey || (key == pkey && id < pid);
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v)
{
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Sum of two 64-bit values over the block (every thread calls; the result is returned to all).
template <int NT>
__device__ __forceinline__ void block_sum2(unsigned long long &a, unsigned long long &b, unsigned long long *red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
    }
    if (lane == 0) {
        red[2 * warp] = a;
        red[2 * warp + 1] = b;
    }
    __syncthreads();
    a = 0;
    b = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        a += red[2 * w];
        b += red[2 * w + 1];
    }
    __syncthreads();
}

// A wide-level tile publishes one word: bit 63 set, and the left counts of its four lists in 15-bit fields
// (a tile holds at most kLevelTileMax = 4096 slots of each list).
constexpr unsigned long long kAggPublished = 1ull << 63;
static_assert(kLevelTileMax < (1 << 15), "left counts of a tile must fit 15 bits");

// One launch per wide level.  Tile j of a node (EPT*NT >= TP slots of each of the four lists) loads its
// slots, finds its node's widest axis and median from the two ends of the sorted lists, classifies every
// slot against the median (the node's own axis list splits by position; the other three lists compare
// keys gathered by id), and publishes its four left counts at once.  Its offsets inside the node are the
// sums of the counts of tiles 0..j-1 of the same node, read in one round by many threads: no tile waits on
// a chain of inclusive prefixes.  Tiles take ids from an atomic counter, so every tile a tile waits on
// has started before it and publishes before it waits on anything.
template <int EPT>
__global__ void __launch_bounds__(kLevelThreads, EPT <= 2 ? 2 : 1) k_level(Plan P, int lev, const uint32_t *__restrict__ keys,
                                                            const uint32_t *__restrict__ lin,
                                                            uint32_t *__restrict__ lout, unsigned long long *agg,
                                                            uint32_t *counters, uint32_t *status)
{
    constexpr int NT = kLevelThreads;
    extern __shared__ __align__(16) uint32_t sl[];  // [4][TP]
    __shared__ unsigned long long scratch[2 * (NT / 32) + 1];
    __shared__ uint32_t s_tile, s_excl[4], s_pkey, s_pid, s_cand[3], s_ckey[3];
    __shared__ int s_axis;
    __shared__ float s_ext[3];
    const int tid = threadIdx.x;
    if (tid == 0) s_tile = atomicAdd(&counters[kCounterLevel0 + lev], 1u);
    __syncthreads();
    const int id = int(s_tile);
    const int64_t np = P.npad;
    const int TP = P.TP;
    int b = 0;
    int64_t r = id;
    for (;;) {
        const int64_t sb = P.pad[b + 1] - P.pad[b];
        const int64_t nt = ((sb >> lev) > P.T) ? sb / TP : 0;
        if (r < nt || b + 1 >= P.B) break;
        r -= nt;
        ++b;
    }
    const int64_t s = (P.pad[b + 1] - P.pad[b]) >> lev, half = s >> 1;
    const int64_t tps = s / TP;
    if (tps < 1 || TP > EPT * NT) {  // cannot happen for a valid plan; never divide by zero or index out of the lists
        if (tid == 0) record_error(status, BT_ERR_INTERNAL);
        return;
    }
    const int64_t kseg = r / tps;
    const int j = int(r - kseg * tps);
    const int64_t seg = P.pad[b] + kseg * s;
    const int64_t nreal = max64(0, min64(s, P.n[b] - kseg * s));
    const int64_t tile0 = seg + int64_t(j) * TP;
    const uint32_t id_lo = uint32_t(P.pad[b]), id_hi = uint32_t(P.pad[b + 1]);  // ids of this cloud
    if (tid < 3) {
        // extent and candidate pivot of axis tid, all loads independent of the axis choice
        uint32_t pp = lin[tid * np + seg + half];
        float e = 0.0f;
        if (nreal > 0) {
            uint32_t p0 = lin[tid * np + seg], p1 = lin[tid * np + seg + nreal - 1];
            if (p0 < id_lo || p0 >= id_hi || p1 < id_lo || p1 >= id_hi) {  // never index with a foreign id
                record_error(status, BT_ERR_INTERNAL);
                p0 = p1 = id_lo;
            }
            e = __fsub_rn(key_float(keys[tid * np + p1]), key_float(keys[tid * np + p0]));
        }
        if (pp < id_lo || pp >= id_hi) {
            record_error(status, BT_ERR_INTERNAL);
            pp = id_lo;
        }
        s_ext[tid] = e;
        s_cand[tid] = pp;
        s_ckey[tid] = keys[tid * np + pp];
    }
    {
        // the tile's slots of all four lists: every load issued before the first store
        uint32_t t[4][EPT];
#pragma unroll
        for (int l = 0; l < 4; ++l)
#pragma unroll
            for (int q = 0; q < EPT; ++q) {
                const int i = tid + q * NT;
                t[l][q] = i < TP ? lin[l * np + tile0 + i] : 0u;
            }
#pragma unroll
        for (int l = 0; l < 4; ++l)
#pragma unroll
            for (int q = 0; q < EPT; ++q) {
                const int i = tid + q * NT;
                if (i < TP) sl[l * TP + i] = t[l][q];
            }
    }
    __syncthreads();
    if (tid == 0) {
        int ax = 0;
        if (s_ext[1] > s_ext[ax]) ax = 1;
        if (s_ext[2] > s_ext[ax]) ax = 2;
        s_axis = ax;
        s_pid = s_cand[ax];
        s_pkey = s_ckey[ax];
    }
    __syncthreads();
    const int ax = s_axis;
    const uint32_t pkey = s_pkey, ppid = s_pid;
    const uint32_t *kax = keys + ax * np;
    const int ept = (TP + NT - 1) / NT;
    const int i0 = tid * ept;
    uint32_t v[4][EPT], kk[4][EPT];
    uint32_t bad = 0;
#pragma unroll
    for (int l = 0; l < 4; ++l)
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int i = i0 + q;
            v[l][q] = (q < ept && i < TP) ? sl[l * TP + i] : 0u;
        }
    // key gathers of the three lists that are not the split axis' own: all issued before the first compare
#pragma unroll
    for (int l = 0; l < 4; ++l)
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            kk[l][q] = 0u;
            if (l != ax && q < ept && i0 + q < TP) {
                const uint32_t pid = v[l][q];
                if (pid < id_lo || pid >= id_hi)
                    bad |= 1u << (l * EPT + q);
                else
                    kk[l][q] = kax[pid];
            }
        }
    if (bad) record_error(status, BT_ERR_INTERNAL);
    uint32_t lbits[4] = {0, 0, 0, 0};
    unsigned long long packed = 0;
#pragma unroll
    for (int l = 0; l < 4; ++l)
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int i = i0 + q;
            if (q < ept && i < TP) {
                bool left;
                if (l == ax)
                    left = int64_t(j) * TP + i < half;
                else
                    left = !((bad >> (l * EPT + q)) & 1u) && before(kk[l][q], v[l][q], pkey, ppid);
                if (left) {
                    lbits[l] |= 1u << q;
                    packed += 1ull << (16 * l);
                }
            }
        }
    unsigned long long tot = 0;
    const unsigned long long ex = block_exclusive_scan<NT, unsigned long long>(packed, scratch, &tot);
    unsigned long long *node_agg = agg + (size_t(lev) * (np / TP) + (id - j)) * kAggStride;
    if (tid == 0) {
        unsigned long long w = kAggPublished;
#pragma unroll
        for (int l = 0; l < 4; ++l) w |= ((tot >> (16 * l)) & 0xFFFFull) << (15 * l);
        st_relaxed_u64(node_agg + size_t(j) * kAggStride, w);
    }
    {
        // left counts of the tiles before this one in the node: two 32-bit sums per 64-bit word
        unsigned long long a01 = 0, a23 = 0;
        for (int t = tid; t < j; t += NT) {
            unsigned long long w = ld_relaxed_u64(node_agg + size_t(t) * kAggStride);
            int spins = 0;
            while (!(w & kAggPublished)) {
                if (++spins > kSpinLimit) {
                    record_error(status, BT_ERR_TIMEOUT);
                    w = kAggPublished;
                    break;
                }
                __nanosleep(32);
                w = ld_relaxed_u64(node_agg + size_t(t) * kAggStride);
            }
            a01 += (w & 0x7FFFull) | (((w >> 15) & 0x7FFFull) << 32);
            a23 += ((w >> 30) & 0x7FFFull) | (((w >> 45) & 0x7FFFull) << 32);
        }
        block_sum2<NT>(a01, a23, scratch);
        if (tid == 0) {
            s_excl[0] = uint32_t(a01);
            s_excl[1] = uint32_t(a01 >> 32);
            s_excl[2] = uint32_t(a23);
            s_excl[3] = uint32_t(a23 >> 32);
        }
    }
#pragma unroll
    for (int l = 0; l < 4; ++l) {
        const int nl = int((tot >> (16 * l)) & 0xFFFFu);
        int run = int((ex >> (16 * l)) & 0xFFFFu);
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int i = i0 + q;
            if (q < ept && i < TP) {
                const bool left = (lbits[l] >> q) & 1u;
                const int pos = left ? run : nl + (i - run);
                run += left;
                sl[l * TP + pos] = v[l][q];
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int l = 0; l < 4; ++l) {
        const int nl = int((tot >> (16 * l)) & 0xFFFFu);
        const int64_t exl = s_excl[l];
        for (int i = tid; i < TP; i += NT) {
            const int64_t dst = i < nl ? exl + i : half + (int64_t(j) * TP - exl) + (i - nl);
            if ((i < nl && dst >= half) || dst < 0 || dst >= s) {  // left count != s/2: a broken invariant
                record_error(status, BT_ERR_INTERNAL);
                continue;
            }
            lout[l * np + seg + dst] = sl[l * TP + i];
        }
    }
}

// ---------------------------------------------------------------------------
// 4. the remaining levels of one node of at most T slots, in shared memory.
//    Points are renamed to local indices 0..sT-1 in ascending id order (the
//    node's index list), so the index list itself is the identity and every
//    list fits in 16 bits.  An id's local index is its rank in the node's
//    ascending id list, found by binary search in shared memory.
// ---------------------------------------------------------------------------
// A local index read from a tail list; out of range only after an invariant broke (then recorded)
__device__ __forceinline__ uint32_t local_ok(uint32_t v, int sT, uint32_t *status)
{
    if (v < uint32_t(sT)) return v;
    record_error(status, BT_ERR_INTERNAL);
    return 0;
}

template <int NT>
__global__ void __launch_bounds__(NT) k_tail(Plan P, const uint32_t *__restrict__ keys,
                                             const uint32_t *__restrict__ lists, int32_t *__restrict__ perm,
                                             uint32_t *status)
{
    constexpr int EPT = 4;  // slots per thread: T <= 1024 runs with 256 threads, T <= 4096 with 1024
    static_assert(kTailMax <= 1024 * EPT && 1024 <= 256 * EPT, "tail slots per thread");
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ unsigned long long scratch[NT / 32 + 1];
    const int T = P.T;
    uint32_t *ps = reinterpret_cast<uint32_t *>(dsm);            // [T] point ids, ascending
    uint32_t *k3 = ps + T;                                       // [3][T] keys by local index
    unsigned long long *segpre = reinterpret_cast<unsigned long long *>(k3 + 3 * T);  // [T/2]
    uint32_t *pkey = reinterpret_cast<uint32_t *>(segpre + T / 2);  // [T/2] pivot keys
    uint16_t *ppv = reinterpret_cast<uint16_t *>(pkey + T / 2);     // [T/2] pivot local index
    uint16_t *lst = ppv + T / 2;                                 // [2][4][T]
    uint8_t *axs = reinterpret_cast<uint8_t *>(lst + 8 * T);     // [T/2]

    const int tid = threadIdx.x;
    const int id = blockIdx.x;
    int b = 0;
    while (b + 1 < P.B && P.tail0[b + 1] <= id) ++b;
    const int k = id - P.tail0[b];
    const int64_t np = P.npad;
    const int sT = int(min64(P.pad[b + 1] - P.pad[b], T));
    const int64_t seg = P.pad[b] + int64_t(k) * sT;
    const int nreal = int(max64(0, min64(sT, P.n[b] - int64_t(k) * sT)));
    const uint32_t *lin = lists + size_t(P.glev[b] & 1) * 4 * np;
    const int m = P.m;

    const uint32_t id_lo = uint32_t(P.pad[b]), id_hi = uint32_t(P.pad[b + 1]);  // ids of this cloud
    {
        // all list loads of this thread's slots first, then the keys of its ids: two round trips
        uint32_t pI[EPT], pA[3][EPT], kk[3][EPT];
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int e = tid + q * NT;
            const bool ok = e < sT;
            pI[q] = ok ? lin[3 * np + seg + e] : id_lo;
#pragma unroll
            for (int a = 0; a < 3; ++a) pA[a][q] = ok ? lin[a * np + seg + e] : id_lo;
        }
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            if (pI[q] < id_lo || pI[q] >= id_hi) {  // never index with a foreign id
                record_error(status, BT_ERR_INTERNAL);
                pI[q] = id_lo;
            }
#pragma unroll
            for (int a = 0; a < 3; ++a) kk[a][q] = tid + q * NT < sT ? keys[a * np + pI[q]] : 0u;
        }
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int e = tid + q * NT;
            if (e < sT) {
                ps[e] = pI[q];
#pragma unroll
                for (int a = 0; a < 3; ++a) k3[a * T + e] = kk[a][q];
                lst[3 * T + e] = uint16_t(e);
            }
        }
        __syncthreads();  // ps[] holds the node's ids in ascending order
        // local index of an id = its rank in ps[]: a fixed-length binary search in shared memory
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int e = tid + q * NT;
            if (e >= sT) continue;
#pragma unroll
            for (int a = 0; a < 3; ++a) {
                const uint32_t pid = pA[a][q];
                int lo = 0;
#pragma unroll
                for (int step = kTailMax / 2; step > 0; step >>= 1)
                    if (lo + step < sT && ps[lo + step] <= pid) lo += step;
                if (ps[lo] != pid) {  // lists disagree on the node's points
                    record_error(status, BT_ERR_INTERNAL);
                    lo = 0;
                }
                lst[a * T + e] = uint16_t(lo);
            }
        }
    }
    __syncthreads();

    int cur = 0;
    const int ept = (sT + NT - 1) / NT;
    const int i0 = tid * ept;
    for (int sz = sT; sz > m; sz >>= 1) {
        const int half = sz >> 1, nsub = sT / sz;
        uint16_t *L = lst + cur * 4 * T, *Ln = lst + (cur ^ 1) * 4 * T;
        for (int q = tid; q < nsub; q += NT) {
            const int start = q * sz;
            const int nr = max(0, min(sz, nreal - start));
            float ext[3] = {0.0f, 0.0f, 0.0f};
            if (nr > 0) {
#pragma unroll
                for (int a = 0; a < 3; ++a)
                    ext[a] = __fsub_rn(key_float(k3[a * T + local_ok(L[a * T + start + nr - 1], sT, status)]),
                                       key_float(k3[a * T + local_ok(L[a * T + start], sT, status)]));
            }
            int ax = 0;
            if (ext[1] > ext[ax]) ax = 1;
            if (ext[2] > ext[ax]) ax = 2;
            const uint32_t pv = local_ok(L[ax * T + start + half], sT, status);
            axs[q] = uint8_t(ax);
            ppv[q] = uint16_t(pv);
            pkey[q] = k3[ax * T + pv];
        }
        __syncthreads();
        uint32_t lbits[4] = {0, 0, 0, 0};
        unsigned long long packed = 0;
        int sub = i0 / sz, sub_start = sub * sz;
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int e = i0 + q;
            if (q < ept && e < sT) {
                if (e - sub_start >= sz) {
                    ++sub;
                    sub_start += sz;
                }
                const int ax = axs[sub];
                const uint32_t pk = pkey[sub], pv = ppv[sub];
                const uint32_t *ka = k3 + ax * T;
#pragma unroll
                for (int l = 0; l < 4; ++l) {
                    const uint32_t v = local_ok(L[l * T + e], sT, status);
                    const bool left = (l == ax) ? (e - sub_start) < half : before(ka[v], v, pk, pv);
                    if (left) {
                        lbits[l] |= 1u << q;
                        packed += 1ull << (16 * l);
                    }
                }
            }
        }
        const unsigned long long ex = block_exclusive_scan<NT, unsigned long long>(packed, scratch, nullptr);
        {
            unsigned long long run = ex;
            int sub2 = i0 / sz, st2 = sub2 * sz;
#pragma unroll
            for (int q = 0; q < EPT; ++q) {
                const int e = i0 + q;
                if (q < ept && e < sT) {
                    if (e - st2 >= sz) {
                        ++sub2;
                        st2 += sz;
                    }
                    if (e == st2) segpre[sub2] = run;
#pragma unroll
                    for (int l = 0; l < 4; ++l)
                        if ((lbits[l] >> q) & 1u) run += 1ull << (16 * l);
                }
            }
        }
        __syncthreads();
        {
            unsigned long long run = ex;
            int sub3 = i0 / sz, start = sub3 * sz;
            unsigned long long sp = ept > 0 && i0 < sT ? segpre[sub3] : 0ull;
#pragma unroll
            for (int q = 0; q < EPT; ++q) {
                const int e = i0 + q;
                if (q < ept && e < sT) {
                    if (e - start >= sz) {
                        ++sub3;
                        start += sz;
                        sp = segpre[sub3];
                    }
#pragma unroll
                    for (int l = 0; l < 4; ++l) {
                        const int pre = int(((run >> (16 * l)) & 0xFFFFu) - ((sp >> (16 * l)) & 0xFFFFu));
                        const bool left = (lbits[l] >> q) & 1u;
                        const int dst = left ? start + pre : start + half + (e - start - pre);
                        if ((left && pre >= half) || dst < start || dst >= start + sz) {
                            record_error(status, BT_ERR_INTERNAL);  // never write outside the node
                        } else {
                            Ln[l * T + dst] = L[l * T + e];
                        }
                        if (left) run += 1ull << (16 * l);
                    }
                }
            }
        }
        __syncthreads();
        cur ^= 1;
    }
    const uint16_t *L = lst + cur * 4 * T;
    for (int e = tid; e < sT; e += NT) {
        const uint32_t pid = ps[local_ok(L[3 * T + e], sT, status)];
        const int64_t li = int64_t(pid) - P.pad[b];
        perm[seg + e] = li < P.n[b] ? int32_t(P.row0[b] + li) : -1;
    }
    __syncthreads();
    if (threadIdx.x == 0) fold_status(status, P.sstatus);
}

// ---------------------------------------------------------------------------
// 4b. record path for large clouds (every cloud a power-of-two slot count of
//     at most 2^21): after the presort, every list element becomes an 8-byte
//     record of the point's ranks on x, y and z (its positions in the three
//     sorted orders, 21 bits each).  Ranks are distinct, so comparing ranks is
//     comparing (coordinate, id): the wide levels and the tail classify by
//     rank, move only records, and gather nothing.  The index list is not
//     carried: the tail sorts every leaf's ids at the end.
// ---------------------------------------------------------------------------
constexpr int kRankBits = 21;
constexpr uint64_t kRankMask = (uint64_t(1) << kRankBits) - 1;

__device__ __forceinline__ uint32_t rrank(uint64_t r, int a) { return uint32_t((r >> (kRankBits * a)) & kRankMask); }

// R0[a][p] = ranks of the point at position p of axis a's sorted list.
__global__ void __launch_bounds__(256) k_records(Plan P, const uint32_t *__restrict__ ids,
                                                 const uint32_t *__restrict__ rnk, unsigned long long *__restrict__ rec,
                                                 uint32_t *status)
{
    const int64_t np = P.npad;
    const int64_t t = int64_t(blockIdx.x) * 256 + threadIdx.x;
    if (t >= 3 * np) return;
    const int a = int(t / np);
    const int64_t p = t - a * np;
    int b = 0;
    while (b + 1 < P.B && P.pad[b + 1] <= p) ++b;
    const uint32_t id = ids[t];
    if (id < uint32_t(P.pad[b]) || id >= uint32_t(P.pad[b + 1])) {  // never index with a foreign id
        record_error(status, BT_ERR_INTERNAL);
        rec[t] = 0;
        return;
    }
    uint64_t r = 0;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const uint32_t v = k == a ? uint32_t(p - P.pad[b]) : rnk[k * np + id];
        r |= uint64_t(v & uint32_t(kRankMask)) << (kRankBits * k);
    }
    rec[t] = r;
}

// One wide level on records (the same tiling and offsets as k_level, three lists of 8-byte records).
template <int EPT>
__global__ void __launch_bounds__(kLevelThreads, 2) k_level_r(
    Plan P, int lev, const uint32_t *__restrict__ skeys, const unsigned long long *__restrict__ rin,
    unsigned long long *__restrict__ rout, unsigned long long *agg, uint32_t *counters, uint32_t *status)
{
    constexpr int NT = kLevelThreads;
    extern __shared__ __align__(16) unsigned long long sr[];  // [3][TP]
    __shared__ unsigned long long scratch[2 * (NT / 32) + 1];
    __shared__ uint16_t s_wcnt[3][EPT][NT / 32];  // left slots per (list, round, warp), then their prefixes
    __shared__ uint32_t s_tile, s_excl[3], s_cand[3], s_ltot[3];
    __shared__ int s_axis;
    __shared__ float s_ext[3];
    const int tid = threadIdx.x;
    if (tid == 0) s_tile = atomicAdd(&counters[kCounterLevel0 + lev], 1u);
    __syncthreads();
    const int id = int(s_tile);
    const int64_t np = P.npad;
    const int TP = P.TP;
    int b = 0;
    int64_t r = id;
    for (;;) {
        const int64_t sb = P.pad[b + 1] - P.pad[b];
        const int64_t nt = ((sb >> lev) > P.T) ? sb / TP : 0;
        if (r < nt || b + 1 >= P.B) break;
        r -= nt;
        ++b;
    }
    const int64_t s = (P.pad[b + 1] - P.pad[b]) >> lev, half = s >> 1;
    const int64_t tps = s / TP;
    if (tps < 1 || TP > EPT * NT) {
        if (tid == 0) record_error(status, BT_ERR_INTERNAL);
        return;
    }
    const int64_t kseg = r / tps;
    const int j = int(r - kseg * tps);
    const int64_t seg = P.pad[b] + kseg * s;
    const int64_t nreal = max64(0, min64(s, P.n[b] - kseg * s));
    const int64_t tile0 = seg + int64_t(j) * TP;
    if (tid < 3) {
        // extent of axis tid from the keys at the node's lowest and highest real rank; candidate median rank
        const unsigned long long *la = rin + tid * np;
        const uint32_t pr = rrank(la[seg + half], tid);
        float e = 0.0f;
        if (nreal > 0) {
            uint32_t r0 = rrank(la[seg], tid), r1 = rrank(la[seg + nreal - 1], tid);
            const uint32_t nb = uint32_t(P.pad[b + 1] - P.pad[b]);
            if (r0 >= nb || r1 >= nb) {  // a rank outside the cloud: never index with it
                record_error(status, BT_ERR_INTERNAL);
                r0 = r1 = 0;
            }
            const uint32_t *ka = skeys + tid * np + P.pad[b];
            e = __fsub_rn(key_float(ka[r1]), key_float(ka[r0]));
        }
        s_ext[tid] = e;
        s_cand[tid] = pr;
    }
    // the tile's records stay in shared memory (not registers), so two CTAs fit an SM
#pragma unroll
    for (int l = 0; l < 3; ++l) {
        unsigned long long t[EPT];
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int i = tid + q * NT;
            t[q] = i < TP ? rin[l * np + tile0 + i] : 0ull;
        }
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int i = tid + q * NT;
            if (i < TP) sr[l * TP + i] = t[q];
        }
    }
    __syncthreads();
    if (tid == 0) {
        int ax = 0;
        if (s_ext[1] > s_ext[ax]) ax = 1;
        if (s_ext[2] > s_ext[ax]) ax = 2;
        s_axis = ax;
    }
    __syncthreads();
    const int ax = s_axis;
    const uint32_t prank = s_cand[ax];
    // classification in coalesced order (slot i = q * NT + tid, conflict-free shared-memory reads): a ballot
    // per (list, round) gives each slot's rank among the left slots of its warp's 32, and a scan of the
    // per-(round, warp) counts in slot order gives the tile's offsets
    const int lane = tid & 31, warp = tid >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t bal[3][EPT];
#pragma unroll
    for (int l = 0; l < 3; ++l)
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int i = q * NT + tid;
            bool left = false;
            if (i < TP) left = (l == ax) ? (int64_t(j) * TP + i < half) : (rrank(sr[l * TP + i], ax) < prank);
            bal[l][q] = __ballot_sync(0xffffffffu, left);
            if (lane == 0) s_wcnt[l][q][warp] = uint16_t(__popc(bal[l][q]));
        }
    __syncthreads();
    if (warp < 3) {
        // exclusive scan of list `warp`'s EPT * (NT / 32) counts, slot order (round-major), one lane per 4
        constexpr int NC = EPT * (NT / 32), PER = (NC + 31) / 32;
        uint16_t *c = &s_wcnt[warp][0][0];
        uint32_t loc[PER], run = 0;
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int k = lane * PER + u;
            loc[u] = k < NC ? c[k] : 0u;
            run += loc[u];
        }
        uint32_t inc = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        uint32_t ex = inc - run;
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int k = lane * PER + u;
            if (k < NC) c[k] = uint16_t(ex);
            ex += loc[u];
        }
        if (lane == 31) s_ltot[warp] = inc;
    }
    __syncthreads();
    const unsigned long long tot =
        uint64_t(s_ltot[0]) | (uint64_t(s_ltot[1]) << 16) | (uint64_t(s_ltot[2]) << 32);
    unsigned long long *node_agg = agg + (size_t(lev) * (np / TP) + (id - j)) * kAggStride;
    if (tid == 0) {
        unsigned long long w = kAggPublished;
#pragma unroll
        for (int l = 0; l < 3; ++l) w |= ((tot >> (16 * l)) & 0xFFFFull) << (15 * l);
        st_relaxed_u64(node_agg + size_t(j) * kAggStride, w);
    }
    {
        unsigned long long a01 = 0, a2 = 0;
        for (int t = tid; t < j; t += NT) {
            unsigned long long w = ld_relaxed_u64(node_agg + size_t(t) * kAggStride);
            int spins = 0;
            while (!(w & kAggPublished)) {
                if (++spins > kSpinLimit) {
                    record_error(status, BT_ERR_TIMEOUT);
                    w = kAggPublished;
                    break;
                }
                __nanosleep(32);
                w = ld_relaxed_u64(node_agg + size_t(t) * kAggStride);
            }
            a01 += (w & 0x7FFFull) | (((w >> 15) & 0x7FFFull) << 32);
            a2 += (w >> 30) & 0x7FFFull;
        }
        block_sum2<NT>(a01, a2, scratch);
        if (tid == 0) {
            s_excl[0] = uint32_t(a01);
            s_excl[1] = uint32_t(a01 >> 32);
            s_excl[2] = uint32_t(a2);
        }
    }
    __syncthreads();
    // every record straight to its place in the node: a warp's left slots land in one run of consecutive
    // positions and its right slots in another
#pragma unroll
    for (int l = 0; l < 3; ++l) {
        const int64_t exl = s_excl[l];
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int i = q * NT + tid;
            if (i < TP) {
                const bool left = (bal[l][q] >> lane) & 1u;
                const int lb = int(s_wcnt[l][q][warp]) + __popc(bal[l][q] & lt);  // left slots before i
                const int64_t dst = left ? exl + lb : half + (int64_t(j) * TP - exl) + (i - lb);
                if ((left && dst >= half) || dst < 0 || dst >= s) {
                    record_error(status, BT_ERR_INTERNAL);
                    continue;
                }
                rout[l * np + seg + dst] = sr[l * TP + i];
            }
        }
    }
}

constexpr int kTailRThreads = 512;

static size_t tail_r_smem_bytes(int T)
{
    // records [2][3][T] + per node of the levels: pivot rank (4 B), axis (1 B), scan prefix (8 B) for T/2 nodes
    return size_t(48) * T + size_t(T / 2) * 13 + 16;
}

// The remaining levels of one node of T slots (T a power of two) on records in shared memory; then each leaf's
// ids (from the x ranks) are sorted ascending and written to perm.
template <int EPT>  // slots per thread: 4 for nodes of up to 2048 slots (two CTAs per SM), 8 for 4096
__global__ void __launch_bounds__(kTailRThreads, EPT <= 4 ? 2 : 1) k_tail_r(Plan P, const uint32_t *__restrict__ skeys,
                                                         const unsigned long long *__restrict__ r0buf,
                                                         const unsigned long long *__restrict__ r1buf,
                                                         const uint32_t *__restrict__ xids, int32_t *__restrict__ perm,
                                                         uint32_t *status)
{
    constexpr int NT = kTailRThreads;
    extern __shared__ __align__(16) uint8_t dsm[];
    const int T = P.T;
    unsigned long long *R = reinterpret_cast<unsigned long long *>(dsm);  // [2][3][T]
    unsigned long long *segpre = R + 6 * T;                              // [T/2]
    uint32_t *pvr = reinterpret_cast<uint32_t *>(segpre + T / 2);         // [T/2] pivot rank
    uint8_t *axs = reinterpret_cast<uint8_t *>(pvr + T / 2);              // [T/2]
    __shared__ uint16_t wcnt[3 * EPT * (kTailRThreads / 32)];             // left slots per (list, round, warp)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    const int id = blockIdx.x;
    int b = 0;
    while (b + 1 < P.B && P.tail0[b + 1] <= id) ++b;
    const int k = id - P.tail0[b];
    const int64_t np = P.npad;
    const int sT = int(min64(P.pad[b + 1] - P.pad[b], T));
    const int64_t seg = P.pad[b] + int64_t(k) * sT;
    const int nreal = int(max64(0, min64(sT, P.n[b] - int64_t(k) * sT)));
    const unsigned long long *rin = (P.glev[b] & 1) ? r1buf : r0buf;
    const int m = P.m;
    const int lsT = 31 - __clz(sT);
    const int64_t sTc = P.pad[b + 1] - P.pad[b];  // slots of the cloud: every rank is below it
    for (int i = tid; i < 3 * sT; i += NT) {
        const int l = i >> lsT, e = i & (sT - 1);
        R[l * T + e] = rin[l * np + seg + e];
    }
    __syncthreads();
    int cur = 0;
    const uint32_t *kb = skeys + P.pad[b];
    for (int sz = sT, lsz = lsT; sz > m; sz >>= 1, --lsz) {
        const int half = sz >> 1, nsub = sT >> lsz;
        unsigned long long *L = R + cur * 3 * T, *Ln = R + (cur ^ 1) * 3 * T;
        for (int q = tid; q < nsub; q += NT) {
            const int start = q << lsz;
            const int nr = max(0, min(sz, nreal - start));
            float ext[3] = {0.0f, 0.0f, 0.0f};
            if (nr > 0) {
#pragma unroll
                for (int a = 0; a < 3; ++a) {
                    uint32_t r1 = rrank(L[a * T + start + nr - 1], a), r0 = rrank(L[a * T + start], a);
                    if (r0 >= uint32_t(sTc) || r1 >= uint32_t(sTc)) {  // a rank outside the cloud
                        record_error(status, BT_ERR_INTERNAL);
                        r0 = r1 = 0;
                    }
                    ext[a] = __fsub_rn(key_float(kb[a * np + r1]), key_float(kb[a * np + r0]));
                }
            }
            int ax = 0;
            if (ext[1] > ext[ax]) ax = 1;
            if (ext[2] > ext[ax]) ax = 2;
            axs[q] = uint8_t(ax);
            pvr[q] = rrank(L[ax * T + start + half], ax);
        }
        __syncthreads();
        // coalesced classification (slot e = q * NT + tid): ballots, then a scan of the per-(round, warp)
        // left counts in slot order; a node's offsets are that prefix minus the prefix at the node's start
        unsigned long long v[3][EPT];
        uint32_t bal[3][EPT];
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int e = q * NT + tid;
            const bool ok = e < sT;
            const int sub = ok ? (e >> lsz) : 0;
            const int ax = axs[sub];
            const uint32_t pr = pvr[sub];
#pragma unroll
            for (int l = 0; l < 3; ++l) {
                v[l][q] = ok ? L[l * T + e] : 0ull;
                const bool left = ok && ((l == ax) ? (e & (sz - 1)) < half : rrank(v[l][q], ax) < pr);
                bal[l][q] = __ballot_sync(0xffffffffu, left);
                if (lane == 0) wcnt[(l * EPT + q) * (NT / 32) + warp] = uint16_t(__popc(bal[l][q]));
            }
        }
        __syncthreads();
        if (warp < 3) {
            constexpr int NC = EPT * (NT / 32), PER = (NC + 31) / 32;
            uint16_t *c = wcnt + warp * NC;
            uint32_t loc[PER], run = 0;
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int k = lane * PER + u;
                loc[u] = k < NC ? c[k] : 0u;
                run += loc[u];
            }
            uint32_t inc = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += y;
            }
            uint32_t ex = inc - run;
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int k = lane * PER + u;
                if (k < NC) c[k] = uint16_t(ex);
                ex += loc[u];
            }
        }
        __syncthreads();
        uint32_t lb[3][EPT];  // left slots before each of this thread's slots, over the whole tile
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int e = q * NT + tid;
#pragma unroll
            for (int l = 0; l < 3; ++l)
                lb[l][q] = uint32_t(wcnt[(l * EPT + q) * (NT / 32) + warp]) + __popc(bal[l][q] & lt);
            if (e < sT && (e & (sz - 1)) == 0)
                segpre[e >> lsz] = uint64_t(lb[0][q]) | (uint64_t(lb[1][q]) << 16) | (uint64_t(lb[2][q]) << 32);
        }
        __syncthreads();
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int e = q * NT + tid;
            if (e < sT) {
                const int sub = e >> lsz, start = sub << lsz;
                const unsigned long long sp = segpre[sub];
#pragma unroll
                for (int l = 0; l < 3; ++l) {
                    const int pre = int(lb[l][q] - uint32_t((sp >> (16 * l)) & 0xFFFFu));
                    const bool left = (bal[l][q] >> lane) & 1u;
                    const int dst = left ? start + pre : start + half + (e - start - pre);
                    if ((left && pre >= half) || dst < start || dst >= start + sz)
                        record_error(status, BT_ERR_INTERNAL);  // never store outside the node
                    else
                        Ln[l * T + dst] = v[l][q];
                }
            }
        }
        __syncthreads();
        cur ^= 1;
    }
    // ids of every slot (from the x rank), then every leaf of m slots sorted ascending by id (bitonic, in place)
    uint32_t *ids = reinterpret_cast<uint32_t *>(R + (cur ^ 1) * 3 * T);  // the free record buffer
    {
        const unsigned long long *L = R + cur * 3 * T;
        const uint32_t *xb = xids + P.pad[b];
        for (int e = tid; e < sT; e += NT) {
            const uint32_t rx = rrank(L[e], 0);
            if (rx >= uint32_t(sTc)) {  // a rank outside the cloud: never index with it
                record_error(status, BT_ERR_INTERNAL);
                ids[e] = uint32_t(P.pad[b]);
            } else {
                ids[e] = xb[rx];
            }
        }
    }
    __syncthreads();
    const int lm = 31 - __clz(m);  // m is a power of two on this path
    for (int kk = 2; kk <= m; kk <<= 1) {
        for (int jj = kk >> 1; jj > 0; jj >>= 1) {
            for (int i = tid; i < sT / 2; i += NT) {
                // pair (lo, lo + jj): lo has bit jj clear
                const int lo = ((i & ~(jj - 1)) << 1) | (i & (jj - 1));
                const int hi = lo + jj;
                const bool up = kk == m ? true : ((lo & kk) == 0);
                const uint32_t x = ids[lo], y = ids[hi];
                if ((x > y) == up) {
                    ids[lo] = y;
                    ids[hi] = x;
                }
            }
            __syncthreads();
        }
    }
    (void)lm;
    for (int e = tid; e < sT; e += NT) {
        const uint32_t pid = ids[e];
        const int64_t li = int64_t(pid) - P.pad[b];
        if (li < 0 || li >= P.pad[b + 1] - P.pad[b]) {
            record_error(status, BT_ERR_INTERNAL);
            perm[seg + e] = -1;
            continue;
        }
        perm[seg + e] = li < P.n[b] ? int32_t(P.row0[b] + li) : -1;
    }
    __syncthreads();
    if (threadIdx.x == 0) fold_status(status, P.sstatus);
}

// ---------------------------------------------------------------------------
// 5. whole build of clouds of at most kClusterMaxCtas * kClusterMaxChunk slots
//    in one launch: one thread-block cluster per cloud, the cloud's lists in
//    the distributed shared memory of its CTAs as 8-byte records.
//
// CTA r of a cluster holds slots r*C .. r*C+C-1 of each list (C = npad / NC).
//   sort    - three lists (X, Y, Z) of (key, id) records, four stable 8-bit
//             LSD passes over the cluster: every CTA ranks its slots locally
//             (ballot digit matching, per-warp digit counts), pushes its digit
//             counts to every CTA and stores every record into the CTA that
//             holds its global position.  The last pass stores, in place of
//             the record, its key into the axis' sorted-key table and its
//             position - the point's rank on that axis - into the rank table
//             of the CTA that owns the point's id.
//   records - every CTA packs the three ranks and the id of each of its
//             points into one 64-bit rank record and stores it at its rank in
//             each of the three lists.  A rank orders points by (key, id) on
//             its axis, so every later comparison is one of ranks.
//   levels  - while a node spans several CTAs: each CTA classifies its slots
//             against the median rank on the node's widest axis (extents from
//             the sorted-key tables at the first and last rank of each list),
//             publishes its three left counts, sums those of the node's CTAs
//             before it and stores every record at its position in the other
//             list buffer of the owning CTA.  Below that, nodes lie inside one
//             CTA and the levels run in its own shared memory.
//   output  - perm from list X's ids (ascending inside every leaf).
// Every CTA of a cluster takes the same sequence of cluster barriers.
// ---------------------------------------------------------------------------
constexpr int kClusterThreads = 512;
constexpr int kClusterMaxChunk = 2048;   // slots per CTA (narrow clusters, and clouds of 32,768 slots)
constexpr int kClusterWideChunk = 1024;  // slots per CTA of the default (wide) clusters
constexpr int kClusterMaxCtas = 16;     // non-portable cluster size (B200 allows 16)
constexpr int kClusterRankWarps = 4;    // warps that rank one axis' slots in a sort pass
static_assert(int64_t(kClusterMaxCtas) * kClusterMaxChunk <= 65536, "ranks and ids fit 16-bit fields");

// Field a of a rank record: the rank on axis a (0..2) or the cloud-local id (3).
__device__ __forceinline__ uint32_t rfield(unsigned long long r, int a) { return uint32_t(r >> (16 * a)) & 0xFFFFu; }

__device__ __forceinline__ void st_cluster_u64(uint32_t addr, unsigned long long v)
{
    asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(addr), "l"(v) : "memory");
}

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v)
{
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void st_cluster_u16(uint32_t addr, uint16_t v)
{
    asm volatile("st.shared::cluster.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

// Split cluster barrier: arrive, other work, then wait.  Every thread of every CTA of the cluster takes
// both, in this order, between any two cluster.sync() calls.
__device__ __forceinline__ void cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory"); }
__device__ __forceinline__ void cluster_arrive_release() { asm volatile("barrier.cluster.arrive.release;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait_acquire() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }

// Scratch shared by the phases in turn: per-warp digit counts [3][RW][256] u16 (sort), the rank table
// [3][CS] u16 (last pass, records), per-node prefix, pivot rank and axis [CS/2] (u64 + u16 + u8, levels),
// leaf ids [CS] u32 (output).
__host__ __device__ __forceinline__ size_t cluster_scratch_bytes(int CS)
{
    const size_t counts = size_t(3) * kClusterRankWarps * 256 * 2, tables = size_t(6) * CS;
    return counts > tables ? counts : tables;
}

// records [2][3][CS] u64 + sorted keys [3][CS] u32 + scratch + received digit counts [NC][3][256] u16 +
// digit starts and offsets [2][3][256] u32
static size_t cluster_smem_bytes(int NC, int CS)
{
    return size_t(6) * CS * 8 + size_t(3) * CS * 4 + cluster_scratch_bytes(CS) + size_t(NC) * 3 * 256 * 2 +
           size_t(6) * 256 * 4;
}

// Sorts the ids (field 3) of every leaf of 32*E slots in X[0..C) ascending, one warp per leaf: lane l holds the
// leaf's slots l*E .. l*E+E-1 in registers; a bitonic network whose compare-exchanges are in-register for
// partners in the same lane and shuffles across lanes otherwise.  emit(i, id) receives slot i's sorted id.
template <int E, typename F>
__device__ __forceinline__ void warp_sort_leaves(const unsigned long long *X, int C, int warp, int lane, int nwarps,
                                                 F &&emit)
{
    constexpr int N = 32 * E;
    for (int leaf = warp; leaf * N < C; leaf += nwarps) {
        uint32_t v[E];
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = rfield(X[leaf * N + lane * E + e], 3);
#pragma unroll
        for (int k = 2; k <= N; k <<= 1) {
#pragma unroll
            for (int j = k >> 1; j > 0; j >>= 1) {
                if (j < E) {
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        if ((e & j) == 0) {
                            const bool up = ((lane * E + e) & k) == 0;
                            const uint32_t a = v[e], c = v[e | j];
                            if ((a > c) == up) {
                                v[e] = c;
                                v[e | j] = a;
                            }
                        }
                    }
                } else {
                    const int lj = j / E;
                    const bool lower = (lane & lj) == 0;
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        const uint32_t o = __shfl_xor_sync(0xffffffffu, v[e], lj);
                        const bool up = ((lane * E + e) & k) == 0;
                        v[e] = (lower == up) ? min(v[e], o) : max(v[e], o);
                    }
                }
            }
        }
#pragma unroll
        for (int e = 0; e < E; ++e) emit(leaf * N + lane * E + e, v[e]);
    }
}

// NC CTAs per cluster; every cloud has a power-of-two slot count npad, and CTA r holds slots r*C..r*C+C-1
// with C = npad / NC = 2^lc.  CS (>= every cloud's C, <= CMAX) is the list stride in shared memory.
template <int NC, int CMAX>
__global__ void __launch_bounds__(kClusterThreads, 1)
    k_cluster_build(Plan P, int CS, const float *__restrict__ coords, int32_t *__restrict__ perm, uint32_t *status)
{
    namespace cg = cooperative_groups;
    constexpr int NT = kClusterThreads, EPT = CMAX / NT > 0 ? CMAX / NT : 1;
    constexpr int RW = kClusterRankWarps;
    constexpr int RQ = CMAX / RW / 32;  // rounds per ranking warp (at most)
    static_assert(RQ >= 1 && 3 * RW <= NT / 32, "ranking warps");
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ __align__(16) uint8_t dsm[];
    unsigned long long *const recs = reinterpret_cast<unsigned long long *>(dsm);  // [2][3][CS]
    uint32_t *const kt = reinterpret_cast<uint32_t *>(recs + 6 * CS);              // [3][CS] sorted keys
    uint8_t *const scr = reinterpret_cast<uint8_t *>(kt + 3 * CS);
    uint16_t *const wh = reinterpret_cast<uint16_t *>(scr);   // [3][RW][256]
    uint16_t *const rtab = reinterpret_cast<uint16_t *>(scr); // [3][CS] rank of each of this CTA's ids
    uint16_t *const rcv = reinterpret_cast<uint16_t *>(scr + cluster_scratch_bytes(CS));  // [NC][3][256]
    uint32_t *const tst = reinterpret_cast<uint32_t *>(rcv + NC * 3 * 256);  // [3][256] starts here
    uint32_t *const off = tst + 3 * 256;                                       // [3][256] global position - local
    __shared__ unsigned long long scratch[NT / 32 + 1];
    __shared__ unsigned long long s_cnt, s_excl;
    __shared__ uint32_t s_pr[3], s_piv;
    __shared__ float s_ext[3];
    __shared__ int s_ax;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rank = int(cluster.block_rank());
    const int b = int(blockIdx.x) / NC;
    const int npad = int(P.pad[b + 1] - P.pad[b]);
    const int lnp = 31 - __clz(npad);
    const int lc = lnp - (31 - __clz(NC));
    const int C = 1 << lc, cmask = C - 1;
    const int n = int(P.n[b]);
    const int m = P.m;
    const int pos0 = rank << lc;  // cloud-local position of this CTA's first slot, and id of its first point
    auto L = [&](int buf, int l) { return recs + (buf * 3 + l) * CS; };
    // the key at rank r of axis a (every rank below npad by the bounds checks of its callers)
    auto key_at = [&](int a, uint32_t r) { return ld_cluster_u32(cluster_addr(kt + a * CS + (r & cmask), r >> lc)); };

    // No CTA touches another's shared memory before every CTA of the cluster has started (this arrive, and
    // its wait before the first remote store), or after that CTA may have exited (the arrive after the last
    // remote load, and its wait at the end).
    cluster_arrive_relaxed();

    // --- (key, id) records of this CTA's points; every list starts in id order
    for (int i = tid; i < C; i += NT) {
        const int id = pos0 + i;
        uint32_t k[3] = {kDummyKey, kDummyKey, kDummyKey};
        if (id < n) {
            const float *c = coords + (P.row0[b] + id) * 3;
            const float x = c[0], y = c[1], z = c[2];
            if (!isfinite(x) || !isfinite(y) || !isfinite(z)) record_error(status, BT_ERR_NONFINITE);
            k[0] = float_key(x);
            k[1] = float_key(y);
            k[2] = float_key(z);
        }
#pragma unroll
        for (int l = 0; l < 3; ++l) L(0, l)[i] = k[l] | (uint64_t(id) << 32);
    }

    // --- presort: list a ends sorted by (key of axis a, id) -----------------
    // Warps RW*a..RW*a+RW-1 rank axis a: warp RW*a+w takes the w-th block of the CTA's slots, 32 per round.
    const int QW = C >= RW * 32 ? C / RW : 32;  // slots of one ranking warp's contiguous block
    const int ra = warp / RW, rw = warp % RW;   // axis and block of a ranking warp (ra < 3)
    const uint32_t lt = (1u << lane) - 1u;
    for (int pass = 0; pass < 4; ++pass) {
        const int sh = 8 * pass;
        for (int i = tid; i < 3 * RW * 256 / 8; i += NT) reinterpret_cast<uint4 *>(wh)[i] = make_uint4(0, 0, 0, 0);
        __syncthreads();
        unsigned long long rec[RQ];
        uint32_t dig[RQ], rnk[RQ];
        if (ra < 3) {
            const unsigned long long *cur = L(0, ra);
            uint16_t *w = wh + (ra * RW + rw) * 256;
#pragma unroll
            for (int q = 0; q < RQ; ++q) {
                const int e = rw * QW + q * 32 + lane;
                const bool ok = q * 32 < QW && e < C;
                rec[q] = ok ? cur[e] : 0ull;
                dig[q] = ok ? ((uint32_t(rec[q]) >> sh) & 255u) : 256u;
            }
#pragma unroll
            for (int q = 0; q < RQ; ++q) {
                const bool ok = dig[q] < 256u;
                const uint32_t peers = digit_peers(dig[q], ok);
                const uint32_t base = ok ? w[dig[q]] : 0u;
                __syncwarp();
                if (ok && (peers & lt) == 0u) w[dig[q]] = uint16_t(base + __popc(peers));
                __syncwarp();
                rnk[q] = base + __popc(peers & lt);
            }
        }
        __syncthreads();
        unsigned long long pk = 0;
        if (tid < 256) {
#pragma unroll
            for (int a = 0; a < 3; ++a) {
                uint32_t run = 0;
#pragma unroll
                for (int w = 0; w < RW; ++w) {
                    const uint32_t c = wh[(a * RW + w) * 256 + tid];
                    wh[(a * RW + w) * 256 + tid] = uint16_t(run);
                    run += c;
                }
                rcv[(rank * 3 + a) * 256 + tid] = uint16_t(run);  // this CTA's row of the exchanged counts
                pk |= uint64_t(run) << (16 * a);
            }
        }
        const unsigned long long ts = block_exclusive_scan<NT, unsigned long long>(pk, scratch, nullptr);
        if (tid < 256) {
#pragma unroll
            for (int a = 0; a < 3; ++a) tst[a * 256 + tid] = uint32_t((ts >> (16 * a)) & 0xFFFFu);
        }
        __syncthreads();
        if (pass == 0) cluster_wait_acquire();  // every CTA of the cluster has started
        // push this CTA's digit counts to every other CTA of the cluster (posted stores)
        for (int i = tid; i < (NC - 1) * 96; i += NT) {
            const int c = (rank + 1 + i / 96) % NC, part = i % 96;
            const uint4 v = reinterpret_cast<const uint4 *>(rcv + rank * 3 * 256)[part];
            st_cluster_v4(cluster_addr(reinterpret_cast<const uint4 *>(rcv + rank * 3 * 256) + part, c), v);
        }
        if (ra < 3) {
            unsigned long long *stg = L(1, ra);
            const uint16_t *w = wh + (ra * RW + rw) * 256;
#pragma unroll
            for (int q = 0; q < RQ; ++q)
                if (dig[q] < 256u) stg[tst[ra * 256 + dig[q]] + w[dig[q]] + rnk[q]] = rec[q];
        }
        cluster.sync();  // every CTA's digit counts have arrived and its locally ordered runs are ready
        {
            unsigned long long tot = 0;
            uint32_t pre[3] = {0, 0, 0};
            if (tid < 256) {
                uint32_t t3[3] = {0, 0, 0};
#pragma unroll
                for (int c = 0; c < NC; ++c)
#pragma unroll
                    for (int a = 0; a < 3; ++a) {
                        const uint32_t v = rcv[(c * 3 + a) * 256 + tid];
                        t3[a] += v;
                        if (c < rank) pre[a] += v;
                    }
                tot = t3[0] | (uint64_t(t3[1]) << 16) | (uint64_t(t3[2]) << 32);
            }
            const unsigned long long base = block_exclusive_scan<NT, unsigned long long>(tot, scratch, nullptr);
            if (tid < 256) {
#pragma unroll
                for (int a = 0; a < 3; ++a)
                    off[a * 256 + tid] = uint32_t((base >> (16 * a)) & 0xFFFFu) + pre[a] - tst[a * 256 + tid];
            }
        }
        __syncthreads();
#pragma unroll
        for (int a = 0; a < 3; ++a) {
            const unsigned long long *stg = L(1, a);
            for (int j = tid; j < C; j += NT) {
                const unsigned long long r = stg[j];
                const uint32_t key = uint32_t(r), id = uint32_t(r >> 32);
                const uint32_t g = off[a * 256 + ((key >> sh) & 255u)] + uint32_t(j);
                if (g >= uint32_t(npad) || id >= uint32_t(npad)) {  // never store outside the cluster's lists
                    record_error(status, BT_ERR_INTERNAL);
                    continue;
                }
                if (pass < 3) {
                    st_cluster_u64(cluster_addr(L(0, a) + (g & cmask), g >> lc), r);
                } else {  // g is the point's rank on axis a
                    st_cluster_u32(cluster_addr(kt + a * CS + (g & cmask), g >> lc), key);
                    st_cluster_u16(cluster_addr(rtab + a * CS + (id & cmask), id >> lc), uint16_t(g));
                }
            }
        }
        cluster.sync();  // every record (last pass: every key and rank) is in place
    }

    // --- rank records, stored at their rank in each list (buffer 1) ---------
    for (int i = tid; i < C; i += NT) {
        const uint32_t r3[3] = {rtab[i], rtab[CS + i], rtab[2 * CS + i]};
        if (r3[0] >= uint32_t(npad) || r3[1] >= uint32_t(npad) || r3[2] >= uint32_t(npad)) {
            record_error(status, BT_ERR_INTERNAL);
            continue;
        }
        const unsigned long long rec = r3[0] | (uint64_t(r3[1]) << 16) | (uint64_t(r3[2]) << 32) |
                                       (uint64_t(pos0 + i) << 48);
#pragma unroll
        for (int a = 0; a < 3; ++a) st_cluster_u64(cluster_addr(L(1, a) + (r3[a] & cmask), r3[a] >> lc), rec);
    }
    cluster.sync();  // every list holds its rank records

    // --- levels whose nodes span several CTAs ------------------------------
    int cb = 1;
    int ls = lnp;  // log2 of the node size
    while ((1 << ls) > m && ls > lc) {
        const int s = 1 << ls, half = s >> 1;
        const int lper = ls - lc;  // log2 of the CTAs per node
        const int k = rank >> lper, j = rank & ((1 << lper) - 1);
        const int nstart = k << ls;
        const int nreal = max(0, min(s, n - nstart));
        if (tid < 3) {
            const int a = tid;
            const unsigned long long *La = L(cb, a);
            const int pm = nstart + half;
            const unsigned long long med = ld_cluster_u64(cluster_addr(La + (pm & cmask), pm >> lc));
            float e = 0.0f;
            if (nreal > 0) {
                const int p1 = nstart + nreal - 1;
                const uint32_t r0 = rfield(ld_cluster_u64(cluster_addr(La + (nstart & cmask), nstart >> lc)), a);
                const uint32_t r1 = rfield(ld_cluster_u64(cluster_addr(La + (p1 & cmask), p1 >> lc)), a);
                if (r0 >= uint32_t(npad) || r1 >= uint32_t(npad))
                    record_error(status, BT_ERR_INTERNAL);
                else
                    e = __fsub_rn(key_float(key_at(a, r1)), key_float(key_at(a, r0)));
            }
            s_ext[a] = e;
            s_pr[a] = rfield(med, a);
        }
        __syncthreads();
        if (tid == 0) {
            int ax = 0;
            if (s_ext[1] > s_ext[ax]) ax = 1;
            if (s_ext[2] > s_ext[ax]) ax = 2;
            s_ax = ax;
            s_piv = s_pr[ax];
        }
        __syncthreads();
        const int ax = s_ax;
        const uint32_t piv = s_piv;
        const int ept = C >= NT ? C / NT : 1;
        const int i0 = tid * ept;
        unsigned long long v[3][EPT];
        uint32_t lbits[3] = {0, 0, 0};
        unsigned long long packed = 0;
#pragma unroll
        for (int l = 0; l < 3; ++l)
#pragma unroll
            for (int q = 0; q < EPT; ++q) {
                const int i = i0 + q;
                v[l][q] = 0ull;
                if (q < ept && i < C) {
                    v[l][q] = L(cb, l)[i];
                    const bool left = (l == ax) ? ((j << lc) + i < half) : (rfield(v[l][q], ax) < piv);
                    if (left) {
                        lbits[l] |= 1u << q;
                        packed += 1ull << (16 * l);
                    }
                }
            }
        unsigned long long tot = 0;
        const unsigned long long ex = block_exclusive_scan<NT, unsigned long long>(packed, scratch, &tot);
        if (tid == 0) s_cnt = tot;
        cluster.sync();  // every CTA's left counts are published
        if (warp == 0) {
            unsigned long long sum = 0;
            for (int t = lane; t < j; t += 32) sum += ld_cluster_u64(cluster_addr(&s_cnt, (k << lper) + t));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if (lane == 0) s_excl = sum;
        }
        __syncthreads();
        const unsigned long long exn = s_excl;
#pragma unroll
        for (int l = 0; l < 3; ++l) {
            const int excl = int((exn >> (16 * l)) & 0xFFFFu);
            int run = int((ex >> (16 * l)) & 0xFFFFu);
            unsigned long long *Ln = L(cb ^ 1, l);
#pragma unroll
            for (int q = 0; q < EPT; ++q) {
                const int i = i0 + q;
                if (q < ept && i < C) {
                    const bool left = (lbits[l] >> q) & 1u;
                    const int dst = left ? excl + run : half + ((j << lc) - excl) + (i - run);
                    run += left;
                    if ((left && dst >= half) || dst < 0 || dst >= s) {  // never store outside the node
                        record_error(status, BT_ERR_INTERNAL);
                        continue;
                    }
                    const int pos = nstart + dst;
                    if ((pos >> lc) == rank)  // stays in this CTA (the split axis' own list always does)
                        Ln[pos & cmask] = v[l][q];
                    else
                        st_cluster_u64(cluster_addr(Ln + (pos & cmask), pos >> lc), v[l][q]);
                }
            }
        }
        cluster.sync();  // the next level reads the other buffer
        cb ^= 1;
        --ls;
    }

    // --- levels inside this CTA --------------------------------------------
    {
        unsigned long long *segpre = reinterpret_cast<unsigned long long *>(scr);  // [C/2] left counts before a node
        uint16_t *spr = reinterpret_cast<uint16_t *>(segpre + CS / 2);            // [C/2] pivot rank per node
        uint8_t *sax = reinterpret_cast<uint8_t *>(spr + CS / 2);                 // [C/2] split axis per node
        const int ept = C >= NT ? C / NT : 1;
        const int i0 = tid * ept;
        for (; (1 << ls) > m; --ls) {
            const int sz = 1 << ls, half = sz >> 1, nsub = C >> ls;
            for (int q = tid; q < nsub; q += NT) {
                const int start = q << ls;
                const int nr = max(0, min(sz, n - (pos0 + start)));
                float e[3] = {0.0f, 0.0f, 0.0f};
                if (nr > 0) {
#pragma unroll
                    for (int a = 0; a < 3; ++a) {
                        const uint32_t r0 = rfield(L(cb, a)[start], a), r1 = rfield(L(cb, a)[start + nr - 1], a);
                        if (r0 >= uint32_t(npad) || r1 >= uint32_t(npad))
                            record_error(status, BT_ERR_INTERNAL);
                        else
                            e[a] = __fsub_rn(key_float(key_at(a, r1)), key_float(key_at(a, r0)));
                    }
                }
                int ax = 0;
                if (e[1] > e[ax]) ax = 1;
                if (e[2] > e[ax]) ax = 2;
                sax[q] = uint8_t(ax);
                spr[q] = uint16_t(rfield(L(cb, ax)[start + half], ax));
            }
            __syncthreads();
            unsigned long long v[3][EPT];
            uint32_t lbits[3] = {0, 0, 0};
            unsigned long long packed = 0;
#pragma unroll
            for (int q = 0; q < EPT; ++q) {
                const int i = i0 + q;
                if (q < ept && i < C) {
                    const int sub = i >> ls, off_in = i & (sz - 1);
                    const int ax = sax[sub];
                    const uint32_t pr = spr[sub];
#pragma unroll
                    for (int l = 0; l < 3; ++l) {
                        v[l][q] = L(cb, l)[i];
                        const bool left = (l == ax) ? off_in < half : rfield(v[l][q], ax) < pr;
                        if (left) {
                            lbits[l] |= 1u << q;
                            packed += 1ull << (16 * l);
                        }
                    }
                }
            }
            const unsigned long long ex = block_exclusive_scan<NT, unsigned long long>(packed, scratch, nullptr);
            {
                unsigned long long run = ex;
#pragma unroll
                for (int q = 0; q < EPT; ++q) {
                    const int i = i0 + q;
                    if (q < ept && i < C) {
                        if ((i & (sz - 1)) == 0) segpre[i >> ls] = run;
#pragma unroll
                        for (int l = 0; l < 3; ++l)
                            if ((lbits[l] >> q) & 1u) run += 1ull << (16 * l);
                    }
                }
            }
            __syncthreads();
            {
                unsigned long long run = ex;
#pragma unroll
                for (int q = 0; q < EPT; ++q) {
                    const int i = i0 + q;
                    if (q < ept && i < C) {
                        const int sub = i >> ls, start = sub << ls;
                        const unsigned long long sp = segpre[sub];
#pragma unroll
                        for (int l = 0; l < 3; ++l) {
                            const int pre = int(((run >> (16 * l)) & 0xFFFFu) - ((sp >> (16 * l)) & 0xFFFFu));
                            const bool left = (lbits[l] >> q) & 1u;
                            const int dst = left ? start + pre : start + half + (i - start - pre);
                            if ((left && pre >= half) || dst < start || dst >= start + sz)
                                record_error(status, BT_ERR_INTERNAL);  // never store outside the node
                            else
                                L(cb ^ 1, l)[dst] = v[l][q];
                            if (left) run += 1ull << (16 * l);
                        }
                    }
                }
            }
            __syncthreads();
            cb ^= 1;
        }
    }

    // the in-CTA levels read other CTAs' sorted-key tables: no CTA leaves before all of them are done
    cluster_arrive_release();

    // --- perm: every leaf's ids (from list X), sorted ascending ----
    // Leaves of 32..256 slots: one warp per leaf sorts the ids in registers (bitonic network, no block barrier);
    // other leaf sizes: one bitonic network over the CTA's slots in shared memory.
    {
        const unsigned long long *X = L(cb, 0);
        auto emit = [&](int i, uint32_t id) { perm[P.pad[b] + pos0 + i] = int(id) < n ? int32_t(P.row0[b] + id) : -1; };
        if (m == 128)
            warp_sort_leaves<4>(X, C, warp, lane, NT / 32, emit);
        else if (m == 64)
            warp_sort_leaves<2>(X, C, warp, lane, NT / 32, emit);
        else if (m == 32)
            warp_sort_leaves<1>(X, C, warp, lane, NT / 32, emit);
        else if (m == 256)
            warp_sort_leaves<8>(X, C, warp, lane, NT / 32, emit);
        else {
            uint32_t *ids = reinterpret_cast<uint32_t *>(scr);  // [C]
            for (int i = tid; i < C; i += NT) ids[i] = rfield(X[i], 3);
            __syncthreads();
            for (int kk = 2; kk <= m; kk <<= 1) {
                for (int jj = kk >> 1; jj > 0; jj >>= 1) {
                    for (int i = tid; i < C / 2; i += NT) {
                        const int lo = ((i & ~(jj - 1)) << 1) | (i & (jj - 1)), hi = lo + jj;
                        const bool up = kk == m || (lo & kk) == 0;  // every leaf of m slots ends ascending
                        const uint32_t x = ids[lo], y = ids[hi];
                        if ((x > y) == up) {
                            ids[lo] = y;
                            ids[hi] = x;
                        }
                    }
                    __syncthreads();
                }
            }
            for (int i = tid; i < C; i += NT) emit(i, ids[i]);
        }
    }
    cluster_wait_acquire();
    __syncthreads();
    if (threadIdx.x == 0) fold_status(status, P.sstatus);
}

static size_t tail_smem_bytes(int T)
{
    // ps + k3 (16 B) + segpre (4 B) + pivot key (2 B) + pivot index (1 B) + lists (16 B) + axis (0.5 B) per slot
    return size_t(T) * 16 + size_t(T / 2) * (8 + 4 + 2 + 1) + size_t(8) * T * 2 + 16;
}

// Cluster size, chunk bound and list stride for the one-launch path, or false when a cloud does not fit it:
// every cloud's slot count must be a power of two (m a power of two) of at most kClusterMaxCtas *
// kClusterMaxChunk.  Wide clusters hold 1,024 slots per CTA (the fastest build of one batch on an idle
// device); narrow ones 2,048, so a cloud takes half the SMs.
static bool cluster_shape(const Plan &P, bool narrow, int &NC, int &CMAX, int &CS)
{
    int64_t mx = 0;
    for (int b = 0; b < P.B; ++b) {
        const int64_t np = P.pad[b + 1] - P.pad[b];
        if (np & (np - 1)) return false;
        mx = std::max<int64_t>(mx, np);
    }
    if (mx > int64_t(kClusterMaxCtas) * kClusterMaxChunk) return false;
    const int chunk = narrow ? kClusterMaxChunk : kClusterWideChunk;
    CMAX = mx > int64_t(kClusterMaxCtas) * chunk ? kClusterMaxChunk : chunk;
    NC = 4;  // at least four CTAs: a small cloud spread over four runs faster than in one CTA alone
    while (NC < kClusterMaxCtas && mx > int64_t(NC) * CMAX) NC *= 2;
    for (int b = 0; b < P.B; ++b)
        if ((P.pad[b + 1] - P.pad[b]) < int64_t(NC) * P.m) return false;  // every leaf inside one CTA
    CS = int(std::max<int64_t>(mx / NC, 16));  // a stride of at least 16 keeps every array 16-byte aligned
    return true;
}

template <int NC, int CMAX>
static cudaError_t cluster_launch(const Plan &P, int CS, const float *coords, int32_t *perm, uint32_t *status,
                                  cudaStream_t st, int *max_clusters)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(P.B * NC));
    cfg.blockDim = dim3(kClusterThreads);
    cfg.dynamicSmemBytes = cluster_smem_bytes(NC, CS);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = unsigned(NC);
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (max_clusters) {  // set-up query: attributes, then how many such clusters fit the device
        cudaError_t e = cudaFuncSetAttribute(k_cluster_build<NC, CMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(cluster_smem_bytes(NC, CMAX)));
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k_cluster_build<NC, CMAX>,
                                                       cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        cfg.gridDim = dim3(unsigned(NC));
        cfg.dynamicSmemBytes = cluster_smem_bytes(NC, CMAX);
        if (e == cudaSuccess) e = cudaOccupancyMaxActiveClusters(max_clusters, k_cluster_build<NC, CMAX>, &cfg);
        return e;
    }
    return cudaLaunchKernelEx(&cfg, k_cluster_build<NC, CMAX>, P, CS, coords, perm, status);
}

static cudaError_t cluster_dispatch(int NC, int CMAX, const Plan &P, int CS, const float *coords, int32_t *perm,
                                    uint32_t *status, cudaStream_t st, int *max_clusters)
{
    if (CMAX == 1024) {
        switch (NC) {
        case 4: return cluster_launch<4, 1024>(P, CS, coords, perm, status, st, max_clusters);
        case 8: return cluster_launch<8, 1024>(P, CS, coords, perm, status, st, max_clusters);
        case 16: return cluster_launch<16, 1024>(P, CS, coords, perm, status, st, max_clusters);
        default: return cudaErrorInvalidValue;
        }
    }
    if (CMAX == 2048) {
        switch (NC) {
        case 4: return cluster_launch<4, 2048>(P, CS, coords, perm, status, st, max_clusters);
        case 8: return cluster_launch<8, 2048>(P, CS, coords, perm, status, st, max_clusters);
        case 16: return cluster_launch<16, 2048>(P, CS, coords, perm, status, st, max_clusters);
        default: return cudaErrorInvalidValue;
        }
    }
    return cudaErrorInvalidValue;
}

// How many clusters of NC CTAs with the largest chunk's shared memory the device holds at once (0: none;
// cached per device).
static int cluster_capacity(int dev, int NC, int CMAX)
{
    // -1 none, else the count; 0 unknown; index log2(NC), CMAX / 2048.  Concurrent first queries from several
    // host threads compute the same value; each entry is one atomic word.
    static std::atomic<int> cache[64][5][2] = {};
    int li = 0;
    while ((1 << li) < NC) ++li;
    const int ci = CMAX == kClusterMaxChunk ? 1 : 0;
    if (dev < 0 || dev >= 64 || li > 4) return 0;
    const int known = cache[dev][li][ci].load(std::memory_order_relaxed);
    if (known) return std::max(known, 0);
    int nclusters = 0;
    const bool ok = cluster_dispatch(NC, CMAX, Plan{}, CMAX, nullptr, nullptr, nullptr, nullptr, &nclusters) ==
                        cudaSuccess &&
                    nclusters > 0;
    (void)cudaGetLastError();  // a refused query is not an error of this call
    cache[dev][li][ci].store(ok ? nclusters : -1, std::memory_order_relaxed);
    return ok ? nclusters : 0;
}

static bt_status launch_build(const float *coords, const Plan &P0, int32_t *perm, void *ws, size_t ws_bytes,
                              uint32_t flags, cudaStream_t st)
{
    Plan P = P0;
    P.sstatus = stream_status(st);
    if (!P.sstatus) return BT_ERR_CUDA;
    const Layout L = make_layout(P);
    if (!ws) return BT_ERR_WORKSPACE;
    if (ws_bytes < L.total) return BT_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return BT_ERR_ARG;
    uint8_t *w = static_cast<uint8_t *>(ws);
    uint32_t *status = reinterpret_cast<uint32_t *>(w);
    uint32_t *counters = reinterpret_cast<uint32_t *>(w + L.counters);
    uint32_t *hist = reinterpret_cast<uint32_t *>(w + L.hist);
    uint32_t *sst = reinterpret_cast<uint32_t *>(w + L.sst);
    unsigned long long *lagg = reinterpret_cast<unsigned long long *>(w + L.lst);
    uint32_t *keys = reinterpret_cast<uint32_t *>(w + L.keys);
    uint32_t *sk = reinterpret_cast<uint32_t *>(w + L.sk);
    uint32_t *sv = reinterpret_cast<uint32_t *>(w + L.sv);
    uint32_t *lists = reinterpret_cast<uint32_t *>(w + L.lists);
    const size_t np = size_t(P.npad);

    static std::atomic<bool> attrs_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BT_ERR_CUDA;
    const size_t sort_smem = size_t(3) * kSortTile * 4;  // sorted keys, sorted values, values in input order
    const size_t tail_smem = tail_smem_bytes(P.T);
    auto init = [&]() -> bt_status {
        if (cudaFuncSetAttribute(k_sort_pass<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sort_smem)) ||
            cudaFuncSetAttribute(k_sort_pass<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sort_smem)) ||
            cudaFuncSetAttribute(k_sort_pass<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sort_smem)) ||
            cudaFuncSetAttribute(k_sort_pass<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sort_smem)) ||
            cudaFuncSetAttribute(k_level<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(4 * kLevelTileMax * sizeof(uint32_t))) ||
            cudaFuncSetAttribute(k_level_r<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(3 * 4 * kLevelThreads * sizeof(uint64_t))) ||
            cudaFuncSetAttribute(k_level_r<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(3 * kLevelTileMax * sizeof(uint64_t))) ||
            cudaFuncSetAttribute(k_tail_r<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(tail_r_smem_bytes(4 * kTailRThreads))) ||
            cudaFuncSetAttribute(k_tail_r<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(tail_r_smem_bytes(8 * kTailRThreads))) ||
            cudaFuncSetAttribute(k_tail<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(tail_smem_bytes(1024))) ||
            cudaFuncSetAttribute(k_tail<1024>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(tail_smem_bytes(kTailMax))))
            return BT_ERR_CUDA;
        return BT_OK;
    };
    const bt_status s0 = (dev >= 0 && dev < 64) ? setup_once(attrs_set[dev], init) : init();
    if (s0 != BT_OK) return s0;
    int NC = 0, CMAX = 0, CS = 0, cap = 0;
    const bool narrow = (flags & BT_BUILD_NARROW) != 0;
    if (cluster_shape(P, narrow, NC, CMAX, CS) && (cap = cluster_capacity(dev, NC, CMAX)) > 0) {
        int nNC = 0, nCMAX = 0, nCS = 0, ncap = 0;
        if (!narrow && P.B > cap && cluster_shape(P, true, nNC, nCMAX, nCS) &&
            (ncap = cluster_capacity(dev, nNC, nCMAX)) > 0 && (P.B + ncap - 1) / ncap < (P.B + cap - 1) / cap) {
            // more clouds than wide clusters fit at once: narrow ones finish the batch in fewer waves
            NC = nNC;
            CMAX = nCMAX;
            CS = nCS;
        }
        // every cloud fits one cluster: the whole build is one launch; only the status word needs clearing
        if (cudaMemsetAsync(ws, 0, 64, st) != cudaSuccess) return BT_ERR_CUDA;
        if (cluster_dispatch(NC, CMAX, P, CS, coords, perm, status, st, nullptr) != cudaSuccess) return BT_ERR_CUDA;
        return BT_OK;
    }
    if (cudaMemsetAsync(ws, 0, L.ctrl_end, st) != cudaSuccess) return BT_ERR_CUDA;
    k_init<<<P.sort_tiles, kSortThreads, 0, st>>>(P, coords, keys, lists + 3 * np, hist, status);
    if (P.rec) {
        // presort; the last pass also leaves the sorted keys (list buffer 1) and every id's rank on each axis
        // (over the keys, no longer needed); then records, wide levels and tail on records
        const int sort_grid = 3 * P.sort_tiles;
        uint32_t *skeys = lists + 4 * np;
        unsigned long long *R0 = reinterpret_cast<unsigned long long *>(sk);
        unsigned long long *R1 = reinterpret_cast<unsigned long long *>(sv);
        k_sort_pass<0><<<sort_grid, kSortThreads, sort_smem, st>>>(P, keys, nullptr, sk, sv, hist, sst, counters,
                                                                   status, nullptr);
        k_sort_pass<1><<<sort_grid, kSortThreads, sort_smem, st>>>(P, sk, sv, sk + 3 * np, sv + 3 * np, hist, sst,
                                                                   counters, status, nullptr);
        k_sort_pass<2><<<sort_grid, kSortThreads, sort_smem, st>>>(P, sk + 3 * np, sv + 3 * np, sk, sv, hist, sst,
                                                                   counters, status, nullptr);
        k_sort_pass<3><<<sort_grid, kSortThreads, sort_smem, st>>>(P, sk, sv, skeys, lists, hist, sst, counters,
                                                                   status, keys);
        k_records<<<unsigned((3 * np + 255) / 256), 256, 0, st>>>(P, lists, keys, R0, status);
        for (int lev = 0; lev < P.nlev; ++lev) {
            int64_t tiles = 0;
            for (int b = 0; b < P.B; ++b) {
                const int64_t sb = P.pad[b + 1] - P.pad[b];
                if ((sb >> lev) > P.T) tiles += sb / P.TP;
            }
            const unsigned long long *rin = (lev & 1) ? R1 : R0;
            unsigned long long *rout = (lev & 1) ? R0 : R1;
            const size_t lsm = size_t(3) * P.TP * sizeof(uint64_t);
            const unsigned g = unsigned(tiles);
            if (P.TP <= kLevelThreads)
                k_level_r<1><<<g, kLevelThreads, lsm, st>>>(P, lev, skeys, rin, rout, lagg, counters, status);
            else if (P.TP <= 2 * kLevelThreads)
                k_level_r<2><<<g, kLevelThreads, lsm, st>>>(P, lev, skeys, rin, rout, lagg, counters, status);
            else if (P.TP <= 4 * kLevelThreads)
                k_level_r<4><<<g, kLevelThreads, lsm, st>>>(P, lev, skeys, rin, rout, lagg, counters, status);
            else
                k_level_r<8><<<g, kLevelThreads, lsm, st>>>(P, lev, skeys, rin, rout, lagg, counters, status);
        }
        if (P.T <= 4 * kTailRThreads)
            k_tail_r<4><<<P.tail0[P.B], kTailRThreads, tail_r_smem_bytes(P.T), st>>>(P, skeys, R0, R1, lists, perm,
                                                                                     status);
        else
            k_tail_r<8><<<P.tail0[P.B], kTailRThreads, tail_r_smem_bytes(P.T), st>>>(P, skeys, R0, R1, lists, perm,
                                                                                     status);
        return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
    }
    const int sort_grid = 3 * P.sort_tiles;
    k_sort_pass<0><<<sort_grid, kSortThreads, sort_smem, st>>>(P, keys, nullptr, sk, sv, hist, sst, counters, status,
                                                               nullptr);
    k_sort_pass<1><<<sort_grid, kSortThreads, sort_smem, st>>>(P, sk, sv, sk + 3 * np, sv + 3 * np, hist, sst,
                                                               counters, status, nullptr);
    k_sort_pass<2><<<sort_grid, kSortThreads, sort_smem, st>>>(P, sk + 3 * np, sv + 3 * np, sk, sv, hist, sst,
                                                               counters, status, nullptr);
    k_sort_pass<3><<<sort_grid, kSortThreads, sort_smem, st>>>(P, sk, sv, nullptr, lists, hist, sst, counters,
                                                               status, nullptr);
    for (int lev = 0; lev < P.nlev; ++lev) {
        int64_t tiles = 0;
        for (int b = 0; b < P.B; ++b) {
            const int64_t sb = P.pad[b + 1] - P.pad[b];
            if ((sb >> lev) > P.T) tiles += sb / P.TP;
        }
        const uint32_t *lin = lists + size_t(lev & 1) * 4 * np;
        uint32_t *lout = lists + size_t((lev + 1) & 1) * 4 * np;
        const size_t lsm = size_t(4) * P.TP * sizeof(uint32_t);
        const unsigned g = unsigned(tiles);
        if (P.TP <= kLevelThreads)
            k_level<1><<<g, kLevelThreads, lsm, st>>>(P, lev, keys, lin, lout, lagg, counters, status);
        else if (P.TP <= 2 * kLevelThreads)
            k_level<2><<<g, kLevelThreads, lsm, st>>>(P, lev, keys, lin, lout, lagg, counters, status);
        else if (P.TP <= 4 * kLevelThreads)
            k_level<4><<<g, kLevelThreads, lsm, st>>>(P, lev, keys, lin, lout, lagg, counters, status);
        else
            k_level<8><<<g, kLevelThreads, lsm, st>>>(P, lev, keys, lin, lout, lagg, counters, status);
    }
    if (P.T <= 1024)
        k_tail<256><<<P.tail0[P.B], 256, tail_smem, st>>>(P, keys, lists, perm, status);
    else
        k_tail<1024><<<P.tail0[P.B], 1024, tail_smem, st>>>(P, keys, lists, perm, status);
    return cudaPeekAtLastError() == cudaSuccess ? BT_OK : BT_ERR_CUDA;
}

}  // namespace bts

using namespace bts;

extern "C" size_t bt_build_workspace_size(const int64_t *offsets, int32_t B, int32_t m)
{
    Plan P;
    if (make_plan(offsets, B, m, P) != BT_OK) return 0;
    return make_layout(P).total;
}

extern "C" bt_status bt_build_segmented_ex(const float *coords, const int64_t *offsets, int32_t B, int32_t m,
                                           int32_t *perm, int64_t *pad_offsets, void *ws, size_t ws_bytes,
                                           uint32_t flags, void *stream)
{
    if (!coords || !perm) return BT_ERR_ARG;
    if (flags & ~uint32_t(BT_BUILD_NARROW)) return BT_ERR_ARG;
    Plan P;
    const bt_status s = make_plan(offsets, B, m, P);
    if (s != BT_OK) return s;
    for (int b = 1; b <= B; ++b)
        if (offsets[b] <= offsets[b - 1]) return BT_ERR_ARG;
    if (pad_offsets)
        for (int b = 0; b <= B; ++b) pad_offsets[b] = P.pad[b];
    return launch_build(coords, P, perm, ws, ws_bytes, flags, static_cast<cudaStream_t>(stream));
}

extern "C" bt_status bt_build_segmented(const float *coords, const int64_t *offsets, int32_t B, int32_t m,
                                        int32_t *perm, int64_t *pad_offsets, void *ws, size_t ws_bytes,
                                        void *stream)
{
    return bt_build_segmented_ex(coords, offsets, B, m, perm, pad_offsets, ws, ws_bytes, 0u, stream);
}

extern "C" bt_status bt_build(const float *coords, int64_t N, int32_t m, int32_t *perm, void *ws, size_t ws_bytes,
                              void *stream)
{
    if (!coords || !perm || N < 1) return BT_ERR_ARG;
    if (m < 1 || m > 1024 || N % m) return BT_ERR_SHAPE;
    const int64_t leaves = N / m;
    if (leaves & (leaves - 1)) return BT_ERR_SHAPE;
    const int64_t offsets[2] = {0, N};
    return bt_build_segmented(coords, offsets, 1, m, perm, nullptr, ws, ws_bytes, stream);
}

extern "C" bt_status bt_build_device_status(const void *ws, void *stream)
{
    if (!ws) return BT_ERR_ARG;
    uint32_t h = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return BT_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return BT_ERR_CUDA;
    return static_cast<bt_status>(h);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of bt_build.
//
// Some callers cannot allocate device memory at the point where they build a
// tree: code inside a region being captured into a CUDA graph (where a
// cudaMalloc would break or end the capture), plug-ins hosted by a framework
// that owns every device allocation through its own pool, and real-time hosts
// that fix their memory budget at start-up.  For them this entry point takes
// its scratch from one file-scope device array of kStaticWsBytes (8 MiB) that
// every GPU which loads this library holds until the process exits, instead
// of a caller workspace.  It serves clouds of at most kStaticMaxPoints points.
//
// The array is shared by every call on a device and keeps the last call's
// contents; each call clears the part that must start at zero.  Two calls
// whose work overlaps on the GPU (different streams, or host threads racing)
// race on the array and produce garbage: serialise them.
// ---------------------------------------------------------------------------
namespace bts {
constexpr size_t kStaticWsBytes = size_t(8) << 20;
constexpr int64_t kStaticMaxPoints = 65536;
static __device__ __align__(256) uint8_t g_static_ws[kStaticWsBytes];
static std::atomic<void *> g_static_ws_addr[64] = {};  // device address of g_static_ws, per device ordinal
}  // namespace bts

extern "C" bt_status bt_build_noalloc(const float *coords, int64_t N, int32_t m, int32_t *perm, int32_t *status_out,
                                      void *stream)
{
    if (!coords || !perm || N < 1) return BT_ERR_ARG;
    if (m < 1 || m > 1024 || N % m) return BT_ERR_SHAPE;
    const int64_t leaves = N / m;
    if (leaves & (leaves - 1)) return BT_ERR_SHAPE;
    if (N > kStaticMaxPoints) return BT_ERR_UNSUPPORTED;  // beyond the static scratch
    const int64_t offsets[2] = {0, N};
    Plan P;
    bt_status s = make_plan(offsets, 1, m, P);
    if (s != BT_OK) return s;
    if (make_layout(P).total > kStaticWsBytes) return BT_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BT_ERR_CUDA;
    void *ws = g_static_ws_addr[dev].load(std::memory_order_acquire);
    if (!ws) {
        // host code only sees a stand-in for the array: ask the runtime for its device address (the same
        // address for every thread that asks)
        if (cudaGetSymbolAddress(&ws, g_static_ws) != cudaSuccess || !ws) return BT_ERR_CUDA;
        g_static_ws_addr[dev].store(ws, std::memory_order_release);
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = launch_build(coords, P, perm, ws, kStaticWsBytes, 0u, st);
    if (s == BT_OK && status_out &&
        cudaMemcpyAsync(status_out, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) !=
            cudaSuccess)
        return BT_ERR_CUDA;
    return s;
}
