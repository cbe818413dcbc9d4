// Host-only check of PerDeviceOnce (block_diffusion_decoding_denoising_b200/csrc/dlm_per_device.h):
// once per device, retried after a failure, once under concurrent first calls, and a bad
// index rejected without running the set-up.  Prints "ok" and exits 0 on success.
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

#include "dlm_per_device.h"

#define CHECK(c)                                              \
  do {                                                        \
    if (!(c)) {                                               \
      std::printf("FAILED line %d: %s\n", __LINE__, #c);     \
      return 1;                                               \
    }                                                         \
  } while (0)

int main() {
  using dlm::PerDeviceOnce;
  {
    PerDeviceOnce once;
    int calls[4] = {0, 0, 0, 0};
    for (int rep = 0; rep < 3; ++rep)
      for (int dev = 0; dev < 4; ++dev) CHECK(once.run(dev, [&] { ++calls[dev]; return 0; }) == 0);
    for (int dev = 0; dev < 4; ++dev) CHECK(calls[dev] == 1 && once.done(dev));
    CHECK(!once.done(4));
  }
  {
    PerDeviceOnce once;
    int calls = 0;
    CHECK(once.run(1, [&] { ++calls; return 7; }) == 7);  // failure: returned, not marked
    CHECK(!once.done(1));
    CHECK(once.run(1, [&] { ++calls; return 0; }) == 0);  // retried
    CHECK(once.run(1, [&] { ++calls; return 0; }) == 0);
    CHECK(calls == 2 && once.done(1) && !once.done(0));
  }
  {
    PerDeviceOnce once;
    int calls = 0;
    CHECK(once.run(-1, [&] { ++calls; return 0; }) == PerDeviceOnce::kBadDevice);
    CHECK(once.run(dlm::kMaxDevices, [&] { ++calls; return 0; }) == PerDeviceOnce::kBadDevice);
    CHECK(once.run(dlm::kMaxDevices - 1, [&] { ++calls; return 0; }) == 0);
    CHECK(calls == 1 && once.done(dlm::kMaxDevices - 1));
  }
  {
    PerDeviceOnce once;
    std::atomic<int> calls[8];
    for (auto& c : calls) c = 0;
    std::atomic<bool> go{false};
    std::vector<std::thread> th;
    for (int t = 0; t < 16; ++t)
      th.emplace_back([&, t] {
        while (!go.load()) {
        }
        for (int dev = 0; dev < 8; ++dev) once.run((dev + t) % 8, [&, dev, t] {
          calls[(dev + t) % 8]++;
          std::this_thread::yield();
          return 0;
        });
      });
    go = true;
    for (auto& x : th) x.join();
    for (int dev = 0; dev < 8; ++dev) CHECK(calls[dev].load() == 1);
  }
  std::printf("ok\n");
  return 0;
}
