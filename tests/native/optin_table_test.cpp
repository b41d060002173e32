// Host test of the per-device dynamic shared-memory opt-in record
// (block_sparse_attention_candidate_b200/csrc/optin.h) with a fake setter in
// place of cudaFuncSetAttribute.  Prints "ok" and exits 0 when every check holds.
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

#include "optin.h"

#define CHECK(c)                                                   \
  do {                                                             \
    if (!(c)) {                                                    \
      std::printf("FAILED line %d: %s\n", __LINE__, #c);           \
      return 1;                                                    \
    }                                                              \
  } while (0)

int main() {
  dynrad::OptInTable t;
  int calls[dynrad::OptInTable::kMaxDevices] = {};
  auto setter_for = [&](int dev) { return [&calls, dev](int) { ++calls[dev]; return true; }; };

  // first use on a device sets the attribute; later uses of the same size do not
  CHECK(t.ensure(0, 200000, setter_for(0)));
  CHECK(t.ensure(0, 200000, setter_for(0)));
  CHECK(calls[0] == 1 && t.granted(0) == 200000);
  // a second device needs its own call (the attribute belongs to that context)
  CHECK(t.ensure(1, 200000, setter_for(1)));
  CHECK(calls[1] == 1 && t.granted(1) == 200000);
  // a smaller size is covered; a larger one is set again
  CHECK(t.ensure(1, 1000, setter_for(1)) && calls[1] == 1);
  CHECK(t.ensure(1, 230000, setter_for(1)) && calls[1] == 2 && t.granted(1) == 230000);
  // a failing setter is not recorded, so the next call tries again
  bool fail = true;
  auto flaky = [&](int) { ++calls[2]; return !fail; };
  CHECK(!t.ensure(2, 5000, flaky) && t.granted(2) == 0);
  fail = false;
  CHECK(t.ensure(2, 5000, flaky) && calls[2] == 2 && t.granted(2) == 5000);
  // ordinals outside the table are refused without calling the setter
  int outside = 0;
  auto count = [&](int) { ++outside; return true; };
  CHECK(!t.ensure(-1, 10, count) && !t.ensure(dynrad::OptInTable::kMaxDevices, 10, count) && outside == 0);
  // many threads on one fresh device: exactly one setter call
  std::atomic<int> concurrent_calls{0};
  std::vector<std::thread> th;
  for (int i = 0; i < 16; ++i)
    th.emplace_back([&] { t.ensure(5, 4096, [&](int) { ++concurrent_calls; return true; }); });
  for (auto& x : th) x.join();
  CHECK(concurrent_calls.load() == 1 && t.granted(5) == 4096);
  std::printf("ok\n");
  return 0;
}
