// Exercises the per-device caches of the host code (csrc/device_cache.h)
// without a GPU: set-up runs once per (device, key) under concurrent callers,
// failures are retried, devices are kept apart, values are cached per device.
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

#include "device_cache.h"

#define CHECK(c)                                              \
  do {                                                        \
    if (!(c)) {                                               \
      std::fprintf(stderr, "FAILED line %d: %s\n", __LINE__, #c); \
      return 1;                                               \
    }                                                         \
  } while (0)

int main() {
  llama::OncePerDevice once;
  static int kern_a, kern_b;   // stand-ins for two kernels' addresses
  std::atomic<int> calls[2][2];
  for (auto& r : calls)
    for (auto& c : r) c = 0;
  std::vector<std::thread> th;
  for (int t = 0; t < 16; ++t)
    th.emplace_back([&, t] {
      for (int i = 0; i < 200; ++i) {
        const int dev = (t + i) & 1;
        const void* key = (i % 3) ? (const void*)&kern_a : (const void*)&kern_b;
        const int k = key == (const void*)&kern_a ? 0 : 1;
        once.run(dev, key, [&] { calls[dev][k]++; return 0; });
      }
    });
  for (auto& x : th) x.join();
  for (int d = 0; d < 2; ++d)
    for (int k = 0; k < 2; ++k) CHECK(calls[d][k] == 1);   // once per device and kernel
  CHECK(once.done(0, &kern_a) && once.done(1, &kern_b));
  CHECK(!once.done(2, &kern_a));                           // a third device is not set up yet

  // a failing set-up is not remembered
  int tries = 0;
  CHECK(once.run(5, &kern_a, [&] { ++tries; return -4; }) == -4);
  CHECK(!once.done(5, &kern_a));
  CHECK(once.run(5, &kern_a, [&] { ++tries; return 0; }) == 0);
  CHECK(once.run(5, &kern_a, [&] { ++tries; return 0; }) == 0);
  CHECK(tries == 2);

  llama::PerDeviceValue<int> sms;
  std::atomic<int> q{0};
  CHECK(sms.get(0, [&] { q++; return 148; }, 1) == 148);
  CHECK(sms.get(0, [&] { q++; return 132; }, 1) == 148);  // cached for device 0
  CHECK(sms.get(1, [&] { q++; return 132; }, 1) == 132);  // device 1 has its own value
  CHECK(sms.get(2, [&] { q++; return 0; }, 148) == 148);  // a failed query gives the fallback ...
  CHECK(sms.get(2, [&] { q++; return 100; }, 148) == 100); // ... and is retried
  CHECK(q == 4);
  std::printf("device cache ok\n");
  return 0;
}
