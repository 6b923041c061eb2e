"""Host-side check of the address cache behind la_state_reduce_static.

The entry point keeps its scratch in a `static __device__` array whose device
address it looks up once per CUDA context. The cache key must be the context,
not only the device ordinal: after cudaDeviceReset (or a primary context
released and created again) the library's module is loaded again and the
array may sit elsewhere, so an address kept per ordinal would be stale.

This test compiles a small C++ driver against the cache header (pure C++, no
CUDA) and checks the keying rule with a fake resolver: a hit under the same
context id, a fresh lookup under a new id on the same device, independent
slots per device, a failed lookup that leaves the slot empty, and a refused
device ordinal. No GPU is involved.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "linear_attention_diffusion_b200", "csrc")

DRIVER = r"""
#include <cstdio>
#include "la_scratch_cache.h"

static int calls = 0;
static char arena[64];

int main() {
  la::SymbolAddressCache<4> cache;
  void* out = nullptr;
  // resolver that hands out a different address on every call
  auto resolve = [](void** a) { *a = arena + (calls++ % 64); return 0; };
  auto fail = [](void** a) { *a = nullptr; ++calls; return 7; };

  // first call in context 101 on device 0: one lookup
  if (cache.get(0, 101, resolve, &out) != 0 || calls != 1 || out != arena + 0) return 1;
  void* first = out;
  // same context again: cached, no lookup
  if (cache.get(0, 101, resolve, &out) != 0 || calls != 1 || out != first) return 2;
  // the context was destroyed and created again (new id, same device): fresh lookup
  if (cache.get(0, 202, resolve, &out) != 0 || calls != 2 || out == first) return 3;
  void* second = out;
  if (cache.get(0, 202, resolve, &out) != 0 || calls != 2 || out != second) return 4;
  // going back to an older id is a miss too (ids are never reused; the slot
  // holds one context)
  if (cache.get(0, 101, resolve, &out) != 0 || calls != 3) return 5;
  // another device has its own slot
  if (cache.get(1, 101, resolve, &out) != 0 || calls != 4) return 6;
  if (cache.get(0, 101, resolve, &out) != 0 || calls != 4) return 7;
  // a failed lookup returns its code and leaves the slot empty
  out = arena;
  if (cache.get(2, 5, fail, &out) != 7 || calls != 5) return 8;
  if (cache.get(2, 5, resolve, &out) != 0 || calls != 6) return 9;
  // a device ordinal outside the table is refused without a lookup
  if (cache.get(4, 5, resolve, &out) != -1 || cache.get(-1, 5, resolve, &out) != -1) return 10;
  if (calls != 6) return 11;
  std::puts("ok");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="no host C++ compiler")
def test_scratch_address_cache_is_keyed_on_the_context(tmp_path):
    src = tmp_path / "cache_check.cpp"
    src.write_text(DRIVER)
    exe = tmp_path / "cache_check"
    r = subprocess.run(["g++", "-std=c++17", "-O1", "-Wall", "-Werror", "-I", CSRC, str(src),
                        "-o", str(exe), "-pthread"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=30)
    assert r.returncode == 0 and r.stdout.strip() == "ok", f"check {r.returncode} failed"
