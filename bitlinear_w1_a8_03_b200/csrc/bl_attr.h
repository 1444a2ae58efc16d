// Per-device bookkeeping of one-time kernel attribute settings.
//
// cudaFuncSetAttribute (e.g. the opt-in to more than 48 KiB of dynamic shared
// memory) applies to the device that is current when it is called, so a
// process that launches a kernel on several GPUs must set the attribute once
// on each of them.  AttrOnce remembers, per (kernel, device), that the setting
// succeeded; a failed setting is not remembered and is tried again on the next
// launch.  No CUDA types appear here, so the bookkeeping builds and is tested
// on a machine without a GPU.
#pragma once

#include <stdint.h>

#include <mutex>

namespace bl {

class AttrOnce {
public:
    static constexpr int kDevices = 64;
    static constexpr int kKeys = 64;

    // Runs set() (returning 0 on success, anything else is an error code) the
    // first time `key` is seen on `device`, and records a success.  Returns 0
    // when the setting is in place, set()'s error otherwise, and -1 for a
    // device or key outside the table.
    template <typename Setter>
    int ensure(const void* key, int device, Setter set) {
        if (device < 0 || device >= kDevices) return -1;
        std::lock_guard<std::mutex> lock(mu_);
        int slot = -1;
        for (int i = 0; i < used_; ++i)
            if (keys_[i] == key) slot = i;
        if (slot < 0) {
            if (used_ == kKeys) return -1;
            slot = used_++;
            keys_[slot] = key;
            done_[slot] = 0;
        }
        const uint64_t bit = (uint64_t)1 << device;
        if (done_[slot] & bit) return 0;
        const int rc = set();
        if (rc == 0) done_[slot] |= bit;
        return rc;
    }

    // True when `key` has been set successfully on `device`.
    bool is_set(const void* key, int device) {
        if (device < 0 || device >= kDevices) return false;
        std::lock_guard<std::mutex> lock(mu_);
        for (int i = 0; i < used_; ++i)
            if (keys_[i] == key) return (done_[i] >> device) & 1u;
        return false;
    }

private:
    std::mutex mu_;
    const void* keys_[kKeys] = {};
    uint64_t done_[kKeys] = {};
    int used_ = 0;
};

}  // namespace bl
