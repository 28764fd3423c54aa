// Host-side cache of the device addresses of this library's __device__
// variables (the error word, the static scratch array).
//
// In host code such a variable's name is only a stand-in; its device address
// comes from cudaGetSymbolAddress and belongs to one CUDA context.  A
// cudaDeviceReset ends the device's primary context, and a caller may make
// another context current, so an address cached per device ordinal could
// point into memory the current context does not own.  The cache is therefore
// keyed on the unique id of the context current on the calling thread (the
// driver's cuCtxGetId, unique for the life of the process) and looks the
// address up again whenever that id is new.
#pragma once

#include <cuda_runtime.h>

#include <mutex>

namespace mlstm {

// Unique id of the CUDA context current on the calling thread; false if no
// context is current or the id cannot be read.
bool current_context_id(unsigned long long* id);

struct DeviceAddressCache {
  static constexpr int kSlots = 16;
  std::mutex mu;
  unsigned long long ctx_id[kSlots] = {};
  void* ptr[kSlots] = {};
  int used = 0, next = 0;
};

// Device address of a __device__ variable in the current context.  `lookup`
// is called as lookup(&ptr) and returns a cudaError_t (cudaGetSymbolAddress on
// the variable, made in the file that defines it).  Returns nullptr, with the
// runtime's last error cleared, if the lookup fails.
template <typename Lookup>
void* cached_device_address(DeviceAddressCache& c, Lookup&& lookup) {
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  std::lock_guard<std::mutex> lk(c.mu);
  if (have_id)
    for (int i = 0; i < c.used; ++i)
      if (c.ctx_id[i] == id) return c.ptr[i];
  void* p = nullptr;
  if (lookup(&p) != cudaSuccess || !p) {
    (void)cudaGetLastError();
    return nullptr;
  }
  // The lookup makes the device's primary context current if none was.
  if (!have_id) have_id = current_context_id(&id);
  if (have_id) {
    const int slot = c.used < DeviceAddressCache::kSlots ? c.used++ : c.next++ % c.kSlots;
    c.ctx_id[slot] = id;
    c.ptr[slot] = p;
  }
  return p;
}

}  // namespace mlstm
