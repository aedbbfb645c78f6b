// Host test of the per-device "done once" flag used for the attention
// kernels' dynamic shared-memory attribute (which CUDA applies to the current
// device only). Prints one line per check; exits non-zero on a failure.
#include <cstdio>

#include "per_device.h"

namespace {
int failures = 0;
void check(bool ok, const char* what) {
  std::printf("%s %s\n", ok ? "ok" : "FAIL", what);
  if (!ok) ++failures;
}
}  // namespace

int main() {
  std::atomic<uint8_t> done[pkv::kMaxDevices];
  for (auto& d : done) d.store(0);
  int calls[pkv::kMaxDevices] = {};
  int fail_next = -1;   // device whose next set() fails
  auto on = [&](int dev) {
    return pkv::once_per_device(dev, done, 0, -2, [&]() {
      if (dev >= 0 && dev < pkv::kMaxDevices) ++calls[dev];
      if (dev == fail_next) { fail_next = -1; return 7; }
      return 0;
    });
  };
  check(on(0) == 0 && calls[0] == 1, "first call on device 0 sets it");
  check(on(0) == 0 && calls[0] == 1, "second call on device 0 does not set it again");
  check(on(1) == 0 && calls[1] == 1, "device 1 is set on its own first call, not by device 0's");
  check(on(1) == 0 && calls[1] == 1 && calls[0] == 1, "device 1 once; device 0 untouched");
  fail_next = 2;
  check(on(2) == 7 && calls[2] == 1, "a failing setter's error is returned");
  check(on(2) == 0 && calls[2] == 2, "a failed device is set again on its next call");
  check(on(-1) == -2, "a negative device index is rejected");
  check(on(pkv::kMaxDevices) == -2, "a device index past the table is rejected");
  int others = 0;
  for (int d = 3; d < pkv::kMaxDevices; ++d) others += calls[d] + done[d].load();
  check(others == 0, "no other device was marked");
  return failures == 0 ? 0 : 1;
}
