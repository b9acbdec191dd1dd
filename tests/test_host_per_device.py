"""Host logic of the per-device caches (csrc/per_device.h), compiled with g++ and run on the CPU.

Kernel attributes and occupancy figures belong to one device, so the library keeps them per device
index.  The cache must compute a device's value once even when several host threads ask at the same
time, keep devices apart, reject indices outside its table and never keep a failed computation.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "nvfp4_w4a4_gemm_fs_b200", "csrc")

PROGRAM = r"""
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>
#include "per_device.h"

int main() {
  fs::PerDevice<int> cache;
  std::atomic<int> calls[fs::kMaxDevices];
  for (auto& c : calls) c = 0;
  std::atomic<int> bad{0};
  std::vector<std::thread> threads;
  for (int t = 0; t < 16; ++t)
    threads.emplace_back([&, t] {
      for (int i = 0; i < fs::kMaxDevices; ++i) {
        const int d = (i + 7 * t) % fs::kMaxDevices;     // threads visit devices in different orders
        int v = -1;
        const bool ok = cache.get(d, &v, [&](int* out) { calls[d]++; *out = 1000 + d; return true; });
        if (!ok || v != 1000 + d) bad++;
      }
    });
  for (auto& th : threads) th.join();
  for (int d = 0; d < fs::kMaxDevices; ++d)
    if (calls[d] != 1) { std::printf("device %d computed %d times\n", d, calls[d].load()); return 1; }
  if (bad) { std::printf("%d wrong values\n", bad.load()); return 1; }
  int v = 0;
  if (cache.get(-1, &v, [](int* o) { *o = 1; return true; })) return 2;
  if (cache.get(fs::kMaxDevices, &v, [](int* o) { *o = 1; return true; })) return 3;
  fs::PerDevice<int> flaky;
  int tries = 0;
  if (flaky.get(3, &v, [&](int*) { ++tries; return false; })) return 4;
  if (!flaky.get(3, &v, [&](int* o) { ++tries; *o = 7; return true; }) || v != 7) return 5;
  if (!flaky.get(3, &v, [&](int* o) { ++tries; *o = 9; return true; }) || v != 7 || tries != 2) return 6;
  std::printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_per_device_cache(tmp_path):
    src = tmp_path / "per_device_test.cpp"
    exe = tmp_path / "per_device_test"
    src.write_text(PROGRAM)
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-I", CSRC, str(src), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
