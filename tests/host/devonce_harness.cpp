// Host test of kvq::once_per_device (kvq_devonce.h): prints "ok" when the
// per-device bookkeeping behaves as documented.
#include <cstdio>
#include <thread>
#include <vector>

#include "kvq_devonce.h"

static int fail(const char* what) {
    std::printf("FAIL %s\n", what);
    return 1;
}

int main() {
    std::atomic<uint64_t> done{0};
    int calls[70] = {0};
    auto run = [&](int dev, int status) {
        return kvq::once_per_device(done, dev, 0, [&] { ++calls[dev]; return status; });
    };
    // first call per device runs the set-up, later calls do not
    if (run(0, 0) != 0 || run(0, 0) != 0 || calls[0] != 1) return fail("device 0 once");
    // a second device is set up on its own, independently of the first
    if (run(1, 0) != 0 || calls[1] != 1 || run(1, 0) != 0 || calls[1] != 1) return fail("device 1");
    // a failed set-up is reported and retried
    if (run(2, 7) != 7 || calls[2] != 1) return fail("failure reported");
    if (run(2, 0) != 0 || calls[2] != 2 || run(2, 0) != 0 || calls[2] != 2) return fail("retry");
    // ordinals beyond the word's bits set up on every call
    run(65, 0); run(65, 0);
    if (calls[65] != 2) return fail("large ordinal");
    // concurrent threads: every device ends set up, at least once each
    std::atomic<uint64_t> done2{0};
    std::atomic<int> per_dev[8];
    for (auto& c : per_dev) c = 0;
    std::vector<std::thread> th;
    for (int t = 0; t < 16; ++t)
        th.emplace_back([&, t] {
            for (int i = 0; i < 1000; ++i) {
                const int dev = (t + i) % 8;
                kvq::once_per_device(done2, dev, 0, [&] { ++per_dev[dev]; return 0; });
            }
        });
    for (auto& x : th) x.join();
    for (int d = 0; d < 8; ++d)
        if (per_dev[d] < 1 || per_dev[d] > 16) return fail("threads");
    if (done2.load() != 0xffu) return fail("threads mask");
    std::printf("ok\n");
    return 0;
}
