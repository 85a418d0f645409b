"""Host logic of the decode split plan (kvq_plan.h), compiled with g++ and checked over a grid of
shapes: every plan covers the sequence with whole 64-token units and no empty split, respects the
largest chunk, and never asks for more splits than max_splits() -- the bound the workspace is
sized from -- for any length up to the capacity. Also the plan of the 8B-shaped decode step.
"""
import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "bit_kv_cache_seeded_b200", "csrc")

DRIVER = r"""
#include <cstdio>
#include "kvq_plan.h"
using namespace kvq;

// resident CTAs per SM as a function of the chunk: constant, or falling with the chunk's logits
// (shared memory) the way the tensor-core kernel's do
static int slots_const1(int) { return 1; }
static int slots_const4(int) { return 4; }
static int slots_smem(int units) {
  const int per = 14336 + 16 * (units * 64 + 8) + 4096 + 1152;
  const int n = 233472 / per;
  return n < 1 ? 1 : (n > 4 ? 4 : n);
}
// shaped like the 1-bit instance's: registers allow 7 CTAs per SM, shared memory (the chunk's
// logits) fewer for long chunks
static int slots_onebit(int units) {
  const int per = 5120 + 16 * (units * 64 + 8) + 2048 + 1152;
  const int n = 233472 / per;
  return n < 1 ? 1 : (n > 7 ? 7 : n);
}

template <class F>
int check(const F& slots, const char* name) {
  const int pairs_[] = {1, 2, 3, 8, 16, 64, 128, 512, 2048, 8192};
  const int sms_[] = {1, 2, 148, 1024};
  const int max_units_[] = {1, 35, 1 << 30};
  const int waves_[] = {2, 16};
  const int caps_[] = {1, 63, 64, 65, 200, 2240, 2241, 8192 + 64, 32768, 131072};
  long cases = 0;
  for (int pairs : pairs_) for (int sms : sms_) for (int mu : max_units_) for (int wb : waves_) for (int cap : caps_) {
    const int tiles = (cap + 63) / 64 * 2;
    const int bound = max_splits(pairs, sms, tiles, mu, wb);
    const int step = cap > 5000 ? 97 : 1;
    for (int len = 0;; len = len + step < cap ? len + step : cap) {  // 0, step, 2 step, ..., cap
      int splits = 0, chunk = 0;
      plan_splits(pairs, sms, slots, mu, wb, len, &splits, &chunk);
      const int units = len > 0 ? (len + 63) / 64 : 1, cu = chunk / 64;
      if (chunk <= 0 || chunk % 64 != 0 || cu > mu || splits < 1) { printf("%s shape p%d s%d mu%d len%d\n", name, pairs, sms, mu, len); return 1; }
      if ((long)splits * cu < units || (long)(splits - 1) * cu >= units) { printf("%s cover p%d s%d mu%d len%d: %d x %d\n", name, pairs, sms, mu, len, splits, cu); return 1; }
      if (splits > bound) { printf("%s workspace p%d s%d mu%d wb%d cap%d len%d: %d > %d\n", name, pairs, sms, mu, wb, cap, len, splits, bound); return 1; }
      ++cases;
      if (len == cap) break;
    }
  }
  return cases > 0 ? 0 : 1;
}

int main() {
  if (check(slots_const1, "1") || check(slots_const4, "4") || check(slots_smem, "smem") || check(slots_onebit, "onebit"))
    return 1;
  // the 8B-shaped decode step: 16 x 8 rows, 8192 + 1 tokens, four CTAs per SM, 35-unit chunks
  int splits = 0, chunk = 0;
  plan_splits(128, 148, slots_const4, 35, 16, 8193, &splits, &chunk);
  printf("llama8b %d %d\n", splits, chunk);
  // the 1-bit layer's shape: 256 x 8 rows, 16384 + 1 tokens; shorter chunks let 7 CTAs share an SM
  plan_splits(2048, 148, slots_onebit, 35, 16, 16385, &splits, &chunk);
  printf("onebit %d %d\n", splits, chunk);
  return 0;
}
"""


def test_split_plan_invariants(tmp_path):
    src = tmp_path / "plan_check.cpp"
    src.write_text(DRIVER)
    exe = tmp_path / "plan_check"
    try:
        subprocess.run(["g++", "-O2", "-std=c++17", "-I", CSRC, str(src), "-o", str(exe)], check=True,
                       capture_output=True, text=True)
    except FileNotFoundError:
        pytest.skip("g++ not available")
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    # 129 units over 4 splits of 33: 512 CTAs, one wave of four per SM
    assert out.stdout.split()[-6:-3] == ["llama8b", "4", "2112"], out.stdout
    # 257 units over 11 splits of 24 (1536 tokens), 7 CTAs per SM, rather than 8 splits of the
    # largest chunk (5 per SM)
    assert out.stdout.split()[-3:] == ["onebit", "11", "1536"], out.stdout
