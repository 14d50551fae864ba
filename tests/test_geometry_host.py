"""The expert kernels' panel geometry on the CPU.

A host program that includes the kernel headers (compiled by nvcc, run on the
host: only __host__ __device__ helpers and constants are used) checks the
invariants the token classes rely on:
  * every class's stage is 64 KB of weights, and every class keeps the same
    accumulators per consumer thread (16 warps);
  * stages are whole 16-row k-steps and whole 64-column x 16-row TMA boxes,
    panels whole m-tiles per warp and whole 128-column tcgen05 slots;
  * a DOWN stage's activation rows lie inside one UP panel of its class, so
    one published panel is all it waits for;
  * the weight, activation and tcgen05 token buffers hold the largest class,
    and the stage ring fits the 227 KB a block can use;
  * for any hidden / intermediate size (multiples of 8), panels x width and
    stages x rows cover the matrix with less than one panel / stage to spare,
    and the panel counters (max_up_panels) cover every class.
"""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "moe_decode_block_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include "moe_device.cuh"
#include "expert_mma.cuh"
#include "expert_tc.cuh"
using namespace moe;
static int bad = 0;
#define CHECK(c) do { if (!(c)) { std::printf("FAIL %s (line %d)\n", #c, __LINE__); ++bad; } } while (0)
int main() {
  for (int c = 0; c < kNumClasses; ++c) {
    const int lw = class_lw(c), R = class_rows(c), nt = class_nt(c);
    CHECK(lw * R * 2 == 65536);
    for (int kc = c; kc < kNumClasses; ++kc) CHECK(class_mt(c, consumer_warps_for(kc)) * nt <= acc_frags(kc));
    const int cw = consumer_warps_for(c);
    CHECK(acc_frags(c) == (c == 0 ? class_mt(0, cw) * nt : cmax(acc_frags(c - 1), class_mt(c, cw) * nt)));
    CHECK(acc_frags(c) * 4 <= 64);  // accumulator floats a consumer thread holds
    CHECK(cw == 8 && expert_threads(c) == 288);
    CHECK(consumer_warps_for(c, true) == 16 && expert_threads(c, true) == 544);
    for (int kc = c; kc < kNumClasses; ++kc) CHECK(class_frags(c, consumer_warps_for(kc, true), true) <= acc_frags(kc, true));
    CHECK(lw % (consumer_warps_for(c) * 16) == 0);
    CHECK(R % 16 == 0 && R % kBoxRows == 0);
    CHECK((lw / 2) % (kChunkCols * kBoxChunks) == 0);
    CHECK((lw / 2) % R == 0);
    CHECK(lw % 128 == 0);
    CHECK(stage_w_bytes(c) <= kStageWBytes);
    CHECK(kUnitTok * (R * 2 + 16) <= kStageXBytes);
    CHECK(kUnitTok * R * 2 <= kTcBBytes);
    CHECK(class_for_tokens(8 * nt) == c);
    if (c + 1 < kNumClasses) CHECK(class_for_tokens(8 * nt + 1) == c + 1);
  }
  CHECK(class_for_tokens(kUnitTok) == kNumClasses - 1);
  CHECK(kStageBytesMma % 1024 == 0 && kStageBytesMma >= kStageWBytes + kStageXBytes);
  CHECK(mma_smem_bytes(kMaxStagesMma) <= 232448);
  CHECK(tc_smem_bytes(2) <= 232448);
  for (int H = 8; H <= 16384; H += 8 * 13) {
    for (int I = 8; I <= 16384; I += 8 * 11) {
      for (int c = 0; c < kNumClasses; ++c) {
        const int lw = class_lw(c), R = class_rows(c);
        const int pu = unit_panels(c, true, H, I), su = unit_panel_stages(c, true, H, I);
        const int pd = unit_panels(c, false, H, I), sd = unit_panel_stages(c, false, H, I);
        CHECK(pu * (lw / 2) >= I && (pu - 1) * (lw / 2) < I);
        CHECK(su * R >= H && (su - 1) * R < H);
        CHECK(pd * lw >= H && (pd - 1) * lw < H);
        CHECK(sd * R >= I && (sd - 1) * R < I);
        CHECK(unit_stages(c, true, H, I) == pu * su && unit_stages(c, false, H, I) == pd * sd);
        CHECK(pu <= max_up_panels(I));
        if (bad > 20) return 1;
      }
    }
  }
  if (!bad) std::printf("ok\n");
  return bad ? 1 : 0;
}
"""


def _nvcc():
    for p in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if p and os.path.exists(p):
            return p
    return None


@pytest.mark.skipif(_nvcc() is None, reason="needs nvcc")
def test_token_class_geometry():
    with tempfile.TemporaryDirectory() as d:
        cu = os.path.join(d, "geometry_check.cu")
        exe = os.path.join(d, "geometry_check")
        with open(cu, "w") as f:
            f.write(PROGRAM)
        subprocess.check_call([_nvcc(), "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                               f"-I{CSRC}", "-o", exe, cu])
        out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout[-3000:]
