// Host-only check of bts::setup_once (per-device first-call set-up): 16 threads race their first calls, the
// first set-up attempt fails, and the next one succeeds.  Expect exactly two set-up runs, every call after the
// success to return BT_OK, and the ready flag set.  Exit status 0 on success.
#include <chrono>
#include <cstdio>
#include <thread>
#include <vector>

#include "bts_internal.cuh"

int main()
{
    static std::atomic<bool> ready = {};
    std::atomic<int> runs{0}, fails_left{1}, ok{0};
    std::vector<std::thread> th;
    for (int t = 0; t < 16; ++t)
        th.emplace_back([&]() {
            for (int rep = 0; rep < 3; ++rep) {
                const bt_status s = bts::setup_once(ready, [&]() -> bt_status {
                    runs.fetch_add(1);
                    std::this_thread::sleep_for(std::chrono::milliseconds(20));
                    return fails_left.fetch_sub(1) > 0 ? BT_ERR_CUDA : BT_OK;
                });
                if (s == BT_OK) ok.fetch_add(1);
            }
        });
    for (auto &x : th) x.join();
    std::printf("set-up runs %d, calls returning OK %d of 48, ready %d\n", runs.load(), ok.load(), int(ready.load()));
    return (runs.load() == 2 && ok.load() == 47 && ready.load()) ? 0 : 1;
}
