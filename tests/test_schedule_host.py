"""The expert kernel's ticket schedule on the CPU.

The schedule functions (struct Sched, make_round, make_sched, sched_range) are
taken as they stand from the kernel header, their device qualifiers dropped,
and compiled with the host C++ compiler, so the checks run the arithmetic the
kernel runs.  Properties, for many stage counts T and grid sizes G:
  * the tickets cut [0, T) into consecutive, non-empty chunks, each stage once;
  * make_sched's chunks hold at most kMaxChunk stages, and its tail of
    one-stage tickets stays bounded (about 2G, whatever T is);
  * make_round hands out whole-grid rounds: a chunk size of max(T / G, 1).
  * with staggered starts, the first G big chunks are c_big - (tk mod stag)
    stages, never under half a big chunk, and the tiling properties hold.
A lost stage would drop part of a weight matrix from the sums; a repeated one
would count it twice.
"""
import os
import re
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "moe_decode_block_b200", "csrc", "expert_mma.cuh")

CHECKER = r"""
#include <cstdio>
#include <algorithm>
constexpr int kMaxChunk = %(max_chunk)d;
%(sched)s
static int fail(const char* what, int T, int G) {
  std::printf("FAIL %%s T=%%d G=%%d\n", what, T, G);
  return 1;
}
// tickets tile [0, T) in order
static void walk(const Sched& s, int T, int G, int max_chunk, int* bad) {
  int next = 0;
  for (int tk = 0; tk < s.n_tickets; ++tk) {
    int b, e;
    sched_range(s, tk, b, e);
    if (b != next || e <= b || e - b > max_chunk) { *bad = fail("tiling", T, G); return; }
    next = e;
  }
  if (next != T) *bad = fail("coverage", T, G);
}
// make_sched's bands: big chunks, then about three quarter chunks per CTA,
// then a one-stage tail of min(T, 2G) stages plus the quarter band's
// remainder (smaller than one quarter chunk)
static void check_bands(const Sched& s, int T, int G, int* bad) {
  const int tail = s.n_tickets - s.n_big - s.n_mid;
  const int taken = sched_stagger_sum(std::min(s.n_big, G), s.stag);
  if (tail != T - s.T2) *bad = fail("tail tickets", T, G);
  if (tail > std::min(T, 2 * G) + s.c_mid - 1) *bad = fail("tail length", T, G);
  if (s.n_mid > 3 * G + s.c_big / s.c_mid + 1 + taken / s.c_mid) *bad = fail("quarter band", T, G);
  if (s.c_mid != std::max(s.c_big / 4, 1)) *bad = fail("quarter size", T, G);
  if (s.stag > 1 && s.stag > s.c_big / 2) *bad = fail("stagger bound", T, G);
}
// staggered starts: the first G big chunks have c_big - (tk mod stag) stages
static void check_stagger(const Sched& s, int T, int G, int* bad) {
  for (int tk = 0; tk < std::min(s.n_big, G); ++tk) {
    int b, e;
    sched_range(s, tk, b, e);
    const int want = s.c_big - (s.stag > 1 ? tk %% s.stag : 0);
    if (e - b != want || e - b < (s.c_big + 1) / 2) { *bad = fail("staggered chunk", T, G); return; }
  }
}
int main() {
  const int grids[] = {1, 2, 3, 7, 64, 74, 148, 296};
  int bad = 0;
  for (int G : grids) {
    for (int T = 0; T <= 6000 && !bad; ++T) {
      const Sched a = make_round(T, G);
      walk(a, T, G, 1 << 30, &bad);
      if (T > 0 && a.c_big != std::max(T / G, 1)) bad = fail("round chunk", T, G);
      const Sched b = make_sched(T, G, 4);
      walk(b, T, G, kMaxChunk, &bad);
      check_bands(b, T, G, &bad);
      for (int stag : {4, 8, 13}) {
        const Sched c = make_sched(T, G, 4, stag);
        walk(c, T, G, kMaxChunk, &bad);
        check_bands(c, T, G, &bad);
        check_stagger(c, T, G, &bad);
      }
    }
    const int big[] = {20000, 131071, 390000, 524287};
    for (int T : big) {
      walk(make_round(T, G), T, G, 1 << 30, &bad);
      const Sched b = make_sched(T, G, 4);
      walk(b, T, G, kMaxChunk, &bad);
      check_bands(b, T, G, &bad);
      for (int stag : {4, 8, 13}) {
        const Sched c = make_sched(T, G, 4, stag);
        walk(c, T, G, kMaxChunk, &bad);
        check_bands(c, T, G, &bad);
        check_stagger(c, T, G, &bad);
      }
    }
  }
  if (!bad) std::printf("ok\n");
  return bad;
}
"""


def _schedule_source():
    src = open(HEADER).read()
    beg = src.index("struct Sched {")
    end = src.index("__device__", src.index("void sched_range("))
    body = src[beg:end].replace("__device__ __forceinline__", "inline")
    assert "__" not in re.sub(r"//.*", "", body), "the schedule code is expected to be plain C++"
    max_chunk = int(re.search(r"constexpr int kMaxChunk = (\d+);", src).group(1))
    return body, max_chunk


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs a host C++ compiler")
def test_ticket_schedule_tiles_every_stage_once():
    body, max_chunk = _schedule_source()
    with tempfile.TemporaryDirectory() as d:
        cpp = os.path.join(d, "sched_check.cpp")
        exe = os.path.join(d, "sched_check")
        with open(cpp, "w") as f:
            f.write(CHECKER % {"max_chunk": max_chunk, "sched": body})
        subprocess.check_call(["g++", "-std=c++17", "-O2", "-o", exe, cpp])
        out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout[-2000:]
