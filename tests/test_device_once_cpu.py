"""The per-device one-time set-up helper (csrc/device_once.h), checked on the CPU.

Kernel attribute opt-ins apply to the device that is current when they are set,
so the library keys every one-time set-up by device. This compiles a small C++
program against the header (no CUDA needed) and checks: the set-up runs once per
device index, not once per process; a failed set-up is retried on the next call;
the cached value is per device; out-of-range indices are refused; and concurrent
callers run each device's set-up exactly once.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gated_delta_rule_58_b200", "csrc")

PROGRAM = r"""
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <thread>
#include <vector>
#include "device_once.h"

using gdn::PerDeviceOnce;
using gdn::run_once_per_device;

#define CHECK(c) do { if (!(c)) { std::printf("FAIL line %d: %s\n", __LINE__, #c); return 1; } } while (0)

int main() {
  {  // once per device, values cached per device
    PerDeviceOnce once;
    int calls = 0, v = -1;
    auto setup = [&](int dev, int* out) { ++calls; *out = 100 + dev; return true; };
    CHECK(run_once_per_device(once, 0, setup, &v) && v == 100 && calls == 1);
    CHECK(run_once_per_device(once, 0, setup, &v) && v == 100 && calls == 1);
    CHECK(run_once_per_device(once, 1, setup, &v) && v == 101 && calls == 2);  // a second device sets up again
    CHECK(run_once_per_device(once, 0, setup, &v) && v == 100 && calls == 2);
    CHECK(!run_once_per_device(once, -1, setup, &v) && calls == 2);
    CHECK(!run_once_per_device(once, gdn::kMaxDevicesOnce, setup, &v) && calls == 2);
  }
  {  // a failure is not remembered: the next call retries
    PerDeviceOnce once;
    int calls = 0;
    auto flaky = [&](int, int* out) { ++calls; *out = 7; return calls >= 2; };
    CHECK(!run_once_per_device(once, 3, flaky));
    CHECK(run_once_per_device(once, 3, flaky) && calls == 2);
    CHECK(run_once_per_device(once, 3, flaky) && calls == 2);
  }
  {  // concurrent callers: each device's set-up runs exactly once
    PerDeviceOnce once;
    std::atomic<int> calls[4];
    for (auto& c : calls) c = 0;
    std::vector<std::thread> th;
    for (int t = 0; t < 16; ++t)
      th.emplace_back([&, t] {
        for (int i = 0; i < 1000; ++i) {
          const int dev = (t + i) & 3;
          int v = 0;
          run_once_per_device(once, dev, [&](int d, int* out) { calls[d]++; *out = d; return true; }, &v);
          if (v != dev) std::abort();
        }
      });
    for (auto& x : th) x.join();
    for (int d = 0; d < 4; ++d) CHECK(calls[d] == 1);
  }
  std::printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_run_once_per_device_is_keyed_by_device(tmp_path):
    src = tmp_path / "once.cpp"
    exe = tmp_path / "once"
    src.write_text(PROGRAM)
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-pthread", "-I", CSRC, str(src), "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
