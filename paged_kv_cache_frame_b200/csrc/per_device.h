// A per-device "done once" flag for settings that CUDA applies to the current
// device only (cudaFuncSetAttribute, for one). Plain host C++: the setter is
// passed in, so the flag logic runs without a GPU in the host tests.
#pragma once
#include <atomic>
#include <cstdint>

namespace pkv {

constexpr int kMaxDevices = 256;

// Runs set() on device `dev` unless it already succeeded there, and records a
// success in done[dev] (an array of kMaxDevices flags owned by the caller,
// one array per setting). Returns set()'s result, or `invalid` for a device
// index out of range. Two threads racing on a first call may both run set(),
// which is harmless for idempotent settings.
template <typename Err, typename SetFn>
Err once_per_device(int dev, std::atomic<uint8_t>* done, Err ok, Err invalid, SetFn set) {
  if (dev < 0 || dev >= kMaxDevices) return invalid;
  if (done[dev].load(std::memory_order_acquire)) return ok;
  const Err e = set();
  if (e == ok) done[dev].store(1, std::memory_order_release);
  return e;
}

}  // namespace pkv
