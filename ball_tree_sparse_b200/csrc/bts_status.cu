// Per-stream device status words.
//
// Every kernel of the library that can detect an error on the device (a non-finite coordinate, a perm entry
// outside the tensors, a wait that ran out) records it, first error wins, in the status word of the stream
// the call was enqueued on.  bt_last_device_status(stream) reads and clears that word.  Keeping one word per
// stream means that concurrent callers on different streams neither see nor wipe each other's errors.
//
// The words live in a file-scope device array (one copy per GPU that loads the library): slot 0 is shared
// by streams that arrive after the table is full, every other slot belongs to one stream handle for the
// life of the process.  Host code sees only a stand-in for the array, so its device address is looked up
// once per device with cudaGetSymbolAddress.
#include <mutex>
#include <unordered_map>

#include "bts_internal.cuh"

namespace bts {

constexpr int kStatusSlots = 1024;
static __device__ uint32_t g_stream_status[kStatusSlots];
static __device__ uint32_t g_status_taken[kStatusSlots];

namespace {
struct StatusTable {
    std::mutex mu;
    std::unordered_map<uintptr_t, int> slot;
    uint32_t *words = nullptr;
    uint32_t *taken = nullptr;
    int next = 1;
};
StatusTable g_tables[64];

// Slot of `st` on the current device (assigned on first use when `assign`); -1 when none.
int status_slot(cudaStream_t st, bool assign, StatusTable *&tab)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    tab = &g_tables[dev];
    std::lock_guard<std::mutex> lock(tab->mu);
    if (!tab->words) {
        if (!assign) return -1;
        void *a = nullptr, *b = nullptr;
        if (cudaGetSymbolAddress(&a, g_stream_status) != cudaSuccess || !a) return -1;
        if (cudaGetSymbolAddress(&b, g_status_taken) != cudaSuccess || !b) return -1;
        tab->words = static_cast<uint32_t *>(a);
        tab->taken = static_cast<uint32_t *>(b);
    }
    const uintptr_t key = reinterpret_cast<uintptr_t>(st);
    auto it = tab->slot.find(key);
    if (it != tab->slot.end()) return it->second;
    if (!assign) return -1;
    const int s = tab->next < kStatusSlots ? tab->next++ : 0;
    tab->slot.emplace(key, s);
    return s;
}
}  // namespace

uint32_t *stream_status(cudaStream_t st)
{
    StatusTable *tab = nullptr;
    const int s = status_slot(st, true, tab);
    return s < 0 ? nullptr : tab->words + s;
}

__global__ void k_take_status(uint32_t *word, uint32_t *taken) { *taken = atomicExch(word, 0u); }

}  // namespace bts

using namespace bts;

extern "C" bt_status bt_last_device_status(void *stream)
{
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    StatusTable *tab = nullptr;
    const int s = status_slot(st, false, tab);
    if (s < 0) {  // nothing was ever enqueued with a status word on this stream
        return cudaStreamSynchronize(st) == cudaSuccess ? BT_OK : BT_ERR_CUDA;
    }
    uint32_t h = 0;
    k_take_status<<<1, 1, 0, st>>>(tab->words + s, tab->taken + s);
    if (cudaPeekAtLastError() != cudaSuccess) return BT_ERR_CUDA;
    if (cudaMemcpyAsync(&h, tab->taken + s, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return BT_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return BT_ERR_CUDA;
    return static_cast<bt_status>(h);
}

extern "C" bt_status bt_attention_device_status(void *stream) { return bt_last_device_status(stream); }
