// kvq_devonce.h -- host-side "once per device" bookkeeping for set-up whose
// effect belongs to one device's context (kernel attributes).  Plain C++ with
// no CUDA dependency, so that it is unit-tested on the host.
#pragma once

#include <atomic>
#include <cstdint>

namespace kvq {

// Runs set_up() for device ordinal `dev` unless an earlier call for the same
// ordinal succeeded (returned `ok`).  One bit per ordinal in `done`, updated
// atomically, so concurrent host threads are safe; two threads may both run
// set_up() the first time, which must therefore be idempotent.  A failed
// set_up() is retried on the next call; ordinals outside [0, 64) run it on
// every call.
template <class Status, class F>
Status once_per_device(std::atomic<uint64_t>& done, int dev, Status ok, F&& set_up) {
    const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t{1} << dev) : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return ok;
    const Status st = set_up();
    if (st == ok && bit) done.fetch_or(bit, std::memory_order_release);
    return st;
}

}  // namespace kvq
