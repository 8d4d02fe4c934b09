// context_cache.h -- a small table of device addresses keyed by CUDA context.
//
// The device address of a file-scope __device__ array belongs to the module
// instance loaded into one context.  Keying by device number alone goes
// stale when the context is destroyed and created again (cudaDeviceReset,
// or the primary context released and retained anew): the module loads
// again, possibly at another address.  Each context has a process-unique id
// (cuCtxGetId), so the key here is (device, context id), and an entry whose
// context has gone simply never matches again.
//
// Plain C++ with no CUDA types, so the host tests can compile and check it.
// Not thread-safe on its own: the caller holds a lock.
#pragma once

#include <stdint.h>

namespace bimamba {

struct ContextKey {
    int device;
    unsigned long long ctx_id;
    bool operator==(const ContextKey& o) const { return device == o.device && ctx_id == o.ctx_id; }
};

template <int N>
class ContextAddressCache {
  public:
    // The cached address for `key`, or nullptr.
    void* find(const ContextKey& key) const {
        for (int i = 0; i < N; ++i)
            if (used_[i] && keys_[i] == key) return addrs_[i];
        return nullptr;
    }
    // Remember `addr` for `key`: replaces the key's entry if it has one, else
    // takes a free slot, else the oldest entry (round robin).
    void put(const ContextKey& key, void* addr) {
        for (int i = 0; i < N; ++i)
            if (used_[i] && keys_[i] == key) {
                addrs_[i] = addr;
                return;
            }
        int slot = -1;
        for (int i = 0; i < N && slot < 0; ++i)
            if (!used_[i]) slot = i;
        if (slot < 0) {
            slot = next_;
            next_ = (next_ + 1) % N;
        }
        keys_[slot] = key;
        addrs_[slot] = addr;
        used_[slot] = true;
    }

  private:
    ContextKey keys_[N] = {};
    void* addrs_[N] = {};
    bool used_[N] = {};
    int next_ = 0;
};

}  // namespace bimamba
