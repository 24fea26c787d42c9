"""Per-device kernel-attribute bookkeeping (csrc/device_once.hpp), on the CPU.

The tensor-core kernels raise their dynamic shared-memory limit once per
device (the attribute belongs to each device's context).  The bookkeeping is
host-only C++, so this test compiles a small driver with g++ against the
library's header and checks: one set-up per device on success, a failed
set-up retried, untracked device ids set up every time, and many threads on
many devices each seeing every device done with at most one set-up per
thread.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "paged_kv_cache_483_b200", "csrc")

DRIVER = r"""
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <thread>
#include <vector>
#include "device_once.hpp"

#define CHECK(c) do { if (!(c)) { std::printf("FAIL line %d: %s\n", __LINE__, #c); return 1; } } while (0)

int main() {
  {
    pa::PerDeviceOnce once;
    int calls = 0;
    auto ok = [&] { ++calls; return 0; };
    CHECK(!once.done(0) && !once.done(3));
    CHECK(once.run(0, ok) == 0 && calls == 1);
    CHECK(once.run(0, ok) == 0 && calls == 1);       // done on device 0
    CHECK(once.done(0) && !once.done(3));
    CHECK(once.run(3, ok) == 0 && calls == 2);       // device 3 is separate
    CHECK(once.run(63, ok) == 0 && calls == 3 && once.done(63));
    CHECK(once.run(64, ok) == 0 && once.run(64, ok) == 0 && calls == 5);  // untracked
    CHECK(once.run(-1, ok) == 0 && calls == 6 && !once.done(-1) && !once.done(64));
  }
  {
    pa::PerDeviceOnce once;
    int calls = 0;
    CHECK(once.run(2, [&] { ++calls; return 7; }) == 7);   // failure: not recorded
    CHECK(!once.done(2));
    CHECK(once.run(2, [&] { ++calls; return 0; }) == 0 && once.done(2));
    CHECK(once.run(2, [&] { ++calls; return 9; }) == 0 && calls == 2);
  }
  {
    pa::PerDeviceOnce once;
    const int kThreads = 16, kDevices = 8;
    std::atomic<int> per_dev[kDevices];
    for (auto& c : per_dev) c = 0;
    std::vector<std::thread> ts;
    for (int t = 0; t < kThreads; ++t)
      ts.emplace_back([&, t] {
        for (int r = 0; r < 1000; ++r) {
          const int dev = (t + r) % kDevices;
          if (once.run(dev, [&] { per_dev[dev]++; return 0; }) != 0) std::abort();
        }
      });
    for (auto& th : ts) th.join();
    for (int d = 0; d < kDevices; ++d) {
      CHECK(once.done(d));
      CHECK(per_dev[d] >= 1 && per_dev[d] <= kThreads);
    }
  }
  std::printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_per_device_once_bookkeeping(tmp_path):
    src = tmp_path / "device_once_test.cpp"
    exe = tmp_path / "device_once_test"
    src.write_text(DRIVER)
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", f"-I{HDR}", str(src), "-o",
                    str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
