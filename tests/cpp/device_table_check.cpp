// Host-only check of ivc::DeviceTable (ivc_device_once.h): values are kept
// per (key, device ordinal), apply() runs only when a value must grow and is
// recorded only on success, and out-of-range ordinals are refused.
#include <cstdio>

#include "ivc_device_once.h"

#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      std::printf("FAILED line %d: %s\n", __LINE__, #cond);      \
      return 1;                                                  \
    }                                                            \
  } while (0)

int main() {
  ivc::DeviceTable t;
  static const char k1 = 0, k2 = 0;
  int calls = 0;
  auto ok = [&] { ++calls; return 0; };
  auto fail = [&] { ++calls; return 7; };

  // first use on device 0 applies; the same or a smaller size does not
  CHECK(t.raise(&k1, 0, 1000, ok) == 0 && calls == 1);
  CHECK(t.raise(&k1, 0, 1000, ok) == 0 && calls == 1);
  CHECK(t.raise(&k1, 0, 500, ok) == 0 && calls == 1);
  // another device has its own entry: a process that drives two GPUs
  // applies the attribute on each
  CHECK(t.get(&k1, 1) == 0);
  CHECK(t.raise(&k1, 1, 1000, ok) == 0 && calls == 2);
  CHECK(t.get(&k1, 1) == 1000 && t.get(&k1, 0) == 1000);
  // a larger size on device 0 applies again
  CHECK(t.raise(&k1, 0, 2000, ok) == 0 && calls == 3 && t.get(&k1, 0) == 2000);
  // another key (kernel) is independent
  CHECK(t.get(&k2, 0) == 0);
  // a failed apply is not recorded, so the next call tries again
  CHECK(t.raise(&k2, 3, 64, fail) == 7 && calls == 4 && t.get(&k2, 3) == 0);
  CHECK(t.raise(&k2, 3, 64, ok) == 0 && calls == 5 && t.get(&k2, 3) == 64);
  // ordinals outside the table are refused without calling apply
  CHECK(t.raise(&k1, -1, 8, ok) == -1 && t.raise(&k1, ivc::kMaxDevices, 8, ok) == -1);
  CHECK(calls == 5);
  std::printf("device table ok\n");
  return 0;
}
