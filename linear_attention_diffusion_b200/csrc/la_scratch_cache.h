// Host-side cache of a device symbol's address, one slot per device, keyed on
// the CUDA context that was current when the address was looked up.
//
// A `static __device__` array lives in a module that the runtime loads into a
// context. If that context is torn down and a new one is created on the same
// device (cudaDeviceReset, or a primary context released and retained again),
// the module is loaded again and the array may sit at another address. An
// address cached per device ordinal alone would then point at memory the new
// context does not own. The key here is the context's unique id (cuCtxGetId:
// ids are never reused within a process), so a new context always misses the
// cache and the address is looked up again.
//
// Pure C++: no CUDA header, so the keying rule is checked on the host.
#pragma once

#include <mutex>

namespace la {

struct SymbolSlot {
  bool valid = false;
  unsigned long long ctx_id = 0;
  void* addr = nullptr;
};

template <int kMaxDevices>
class SymbolAddressCache {
 public:
  // Address for (dev, ctx_id): the cached one when this slot was filled under
  // the same context id, otherwise resolve(&addr) is called (it returns 0 on
  // success) and its result stored under ctx_id. Returns resolve's non-zero
  // code on failure (the slot is then left empty), -1 for a bad device.
  template <class Resolve>
  int get(int dev, unsigned long long ctx_id, Resolve&& resolve, void** out) {
    if (dev < 0 || dev >= kMaxDevices) return -1;
    std::lock_guard<std::mutex> lock(mu_);
    SymbolSlot& s = slots_[dev];
    if (!(s.valid && s.ctx_id == ctx_id)) {
      s.valid = false;
      void* addr = nullptr;
      const int rc = resolve(&addr);
      if (rc != 0) return rc;
      s.addr = addr;
      s.ctx_id = ctx_id;
      s.valid = true;
    }
    *out = s.addr;
    return 0;
  }

 private:
  std::mutex mu_;
  SymbolSlot slots_[kMaxDevices];
};

}  // namespace la
