"""Host logic of the per-device kernel-attribute record (csrc/attr_cache.h),
compiled with g++ and run on the CPU: the shared-memory limit of a kernel is
raised on every device it launches on (cudaFuncSetAttribute acts on the
current device only), only when a launch needs more than recorded, never
lowered by a smaller concurrent request, and a failed raise is not recorded."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "precision_quantized_gemm_b200", "csrc")

DRIVER = r"""
#include "attr_cache.h"
#include <cstdio>
#include <thread>
#include <vector>
#include <atomic>
int main() {
  qg::GrowOnlyAttr a;
  int calls[4] = {0, 0, 0, 0};
  int dev_value[4] = {0, 0, 0, 0};
  auto setter = [&](int dev) { return [&, dev](int v) { ++calls[dev]; dev_value[dev] = v; return 0; }; };
  // device 0: first launch raises, same or smaller sizes do not, larger does
  if (a.ensure(0, 100000, setter(0)) || calls[0] != 1 || dev_value[0] != 100000) return 1;
  if (a.ensure(0, 100000, setter(0)) || a.ensure(0, 50000, setter(0)) || calls[0] != 1) return 2;
  if (a.ensure(0, 150000, setter(0)) || calls[0] != 2 || dev_value[0] != 150000) return 3;
  // device 1 is configured on its own first launch, even at a size device 0 has
  if (a.ensure(1, 100000, setter(1)) || calls[1] != 1 || dev_value[1] != 100000) return 4;
  // a failing raise is reported and not recorded; the next launch retries
  if (a.ensure(2, 90000, [&](int) { ++calls[2]; return 7; }) != 7 || a.recorded(2) != 0) return 5;
  if (a.ensure(2, 90000, setter(2)) || calls[2] != 2 || a.recorded(2) != 90000) return 6;
  // concurrent launches of mixed sizes on device 3: the largest wins, the
  // value set last is the recorded one, and it is never lowered
  std::atomic<int> last{0}, n{0};
  std::vector<std::thread> th;
  for (int t = 0; t < 16; ++t)
    th.emplace_back([&, t] {
      for (int i = 0; i < 2000; ++i) {
        const int v = 1000 * (1 + (t * 7 + i) % 200);
        a.ensure(3, v, [&](int x) { ++n; last.store(x); return 0; });
      }
    });
  for (auto& x : th) x.join();
  if (a.recorded(3) != 200000 || last.load() != 200000 || n.load() > 200) return 8;
  std::printf("ok %d\n", n.load());
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_grow_only_attr_per_device(tmp_path):
    src = tmp_path / "drv.cpp"
    src.write_text(DRIVER)
    exe = tmp_path / "drv"
    r = subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-I", CSRC, str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.startswith("ok"), (r.returncode, r.stdout, r.stderr)
