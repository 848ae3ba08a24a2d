// CPU check of the per-device set-up flags the launchers use
// (sink_aware_sliding_head_b200/csrc/device_once.h): each device runs its
// set-up once, a failed set-up is retried, devices are independent, devices
// outside the table are never cached, and concurrent first calls run the
// set-up once.
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

#include "device_once.h"

#define CHECK(c)                                             \
  do {                                                       \
    if (!(c)) {                                              \
      std::printf("FAIL line %d: %s\n", __LINE__, #c);       \
      return 1;                                              \
    }                                                        \
  } while (0)

int main() {
  using flint::PerDeviceOnce;
  {
    PerDeviceOnce once;
    int calls[flint::kMaxDevices] = {};
    for (int rep = 0; rep < 3; ++rep)
      for (int dev = 0; dev < flint::kMaxDevices; ++dev)
        CHECK(once.run(dev, [&] { ++calls[dev]; return 0; }) == 0);
    for (int dev = 0; dev < flint::kMaxDevices; ++dev) {
      CHECK(calls[dev] == 1);
      CHECK(once.done(dev));
    }
  }
  {  // device 1 set up first must not mark device 0 (the old per-process flag did)
    PerDeviceOnce once;
    int c0 = 0, c1 = 0;
    CHECK(once.run(1, [&] { ++c1; return 0; }) == 0);
    CHECK(!once.done(0) && once.done(1));
    CHECK(once.run(0, [&] { ++c0; return 0; }) == 0);
    CHECK(c0 == 1 && c1 == 1);
  }
  {  // a failing set-up reports its error and is retried
    PerDeviceOnce once;
    int calls = 0;
    CHECK(once.run(3, [&] { ++calls; return 7; }) == 7);
    CHECK(!once.done(3));
    CHECK(once.run(3, [&] { ++calls; return 0; }) == 0);
    CHECK(once.run(3, [&] { ++calls; return 0; }) == 0);
    CHECK(calls == 2 && once.done(3));
  }
  {  // out-of-range devices run every time and are never marked
    PerDeviceOnce once;
    int calls = 0;
    for (int dev : {-1, flint::kMaxDevices, flint::kMaxDevices + 5})
      for (int rep = 0; rep < 2; ++rep) CHECK(once.run(dev, [&] { ++calls; return 0; }) == 0);
    CHECK(calls == 6);
    CHECK(!once.done(-1) && !once.done(flint::kMaxDevices));
  }
  {  // many threads, first use of several devices at once
    PerDeviceOnce once;
    std::atomic<int> calls[4];
    for (auto& c : calls) c = 0;
    std::vector<std::thread> th;
    for (int t = 0; t < 16; ++t)
      th.emplace_back([&, t] {
        for (int rep = 0; rep < 1000; ++rep) {
          const int dev = (t + rep) % 4;
          once.run(dev, [&] { calls[dev].fetch_add(1); return 0; });
        }
      });
    for (auto& x : th) x.join();
    for (auto& c : calls) CHECK(c.load() == 1);
  }
  std::printf("device once ok\n");
  return 0;
}
