"""Per-device launcher state (csrc/per_device.h), driven on the CPU with fake devices.

The launchers set kernel attributes and read occupancy once per GPU.  This test
compiles the same header with the host compiler and checks, with a counting fake
in place of the CUDA calls: one set-up per device (not per process), a retry after
a failed set-up, values kept apart per device, devices outside the table never
cached, and one set-up per device when many threads race on the first call.
"""
import os
import shutil
import subprocess

import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "weight_sequence_mixing_b200",
                    "csrc")

PROGRAM = r"""
#include <cstdio>
#include <thread>
#include <vector>
#include "per_device.h"

static int calls[256];

int main() {
  using namespace ttt;
  int bad = 0;
  // set-up once per device: device 0, then device 1, then both again
  {
    OncePerDevice once;
    auto setup = [](int dev) { return [dev] { ++calls[dev]; return 0; }; };
    for (int rep = 0; rep < 3; ++rep)
      for (int dev : {0, 1}) bad |= once.run(dev, setup(dev)) != 0;
    bad |= (calls[0] != 1 || calls[1] != 1) << 1;
  }
  // a failed set-up is retried on the next call, and cached once it succeeds
  {
    OncePerDevice once;
    int attempts = 0;
    auto flaky = [&] { return ++attempts < 3 ? 7 : 0; };
    bad |= (once.run(2, flaky) != 7) << 2;
    bad |= (once.run(2, flaky) != 7) << 3;
    bad |= (once.run(2, flaky) != 0) << 4;
    bad |= (once.run(2, flaky) != 0 || attempts != 3) << 5;
  }
  // values per device: each device keeps its own answer
  {
    IntPerDevice v;
    int asked = 0;
    for (int rep = 0; rep < 2; ++rep)
      for (int dev = 0; dev < 4; ++dev) bad |= (v.get(dev, [&] { ++asked; return 100 + dev; }) != 100 + dev) << 6;
    bad |= (asked != 4) << 7;
  }
  // devices outside the table are never cached
  {
    IntPerDevice v;
    int asked = 0;
    for (int rep = 0; rep < 3; ++rep) v.get(-1, [&] { ++asked; return 1; });
    for (int rep = 0; rep < 3; ++rep) v.get(kPerDeviceSlots, [&] { ++asked; return 1; });
    bad |= (asked != 6) << 8;
  }
  // many threads racing on the first call of two devices: one set-up each
  {
    OncePerDevice once;
    std::atomic<int> per_dev[2] = {};
    std::vector<std::thread> ts;
    for (int t = 0; t < 16; ++t)
      ts.emplace_back([&, t] {
        for (int rep = 0; rep < 1000; ++rep) once.run(t & 1, [&] { per_dev[t & 1].fetch_add(1); return 0; });
      });
    for (auto& th : ts) th.join();
    bad |= (per_dev[0].load() != 1 || per_dev[1].load() != 1) << 9;
  }
  std::printf("%d\n", bad);
  return bad != 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs the host C++ compiler")
def test_per_device_state_with_fake_devices(tmp_path):
    src = tmp_path / "per_device_test.cpp"
    src.write_text(PROGRAM)
    exe = tmp_path / "per_device_test"
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-I", CSRC, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, f"failed checks (bit mask): {out.stdout.strip()} {out.stderr}"
