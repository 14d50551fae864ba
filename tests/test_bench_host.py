"""Host-side helpers of bench.py (no GPU): the code-only source hash that
decides whether a committed ncu traffic figure still describes the kernels."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_only_drops_comments_and_keeps_literals():
    src = ('int a = 1;  // trailing\n'
           '/* block\n   comment */ const char* s = "x // y /* z */";\n'
           "char q = '\\''; char r = '/';  // the CTA's\n"
           '\n   \n'
           'int b;\n')
    assert bench.code_only(src) == ('int a = 1;\n'
                                    ' const char* s = "x // y /* z */";\n'
                                    "char q = '\\''; char r = '/';\n"
                                    'int b;')


def test_code_only_is_blind_to_comment_edits_but_not_to_code_edits():
    a = "__global__ void k(int* p) {\n  // store one\n  *p = 1;\n}\n"
    b = "__global__ void k(int* p) {\n  // store the value one (reworded)\n  *p = 1;  /* note */\n}\n"
    c = "__global__ void k(int* p) {\n  // store one\n  *p = 2;\n}\n"
    assert bench.code_only(a) == bench.code_only(b)
    assert bench.code_only(a) != bench.code_only(c)


def test_traffic_is_reported_only_for_the_code_it_was_captured_on(monkeypatch):
    import json
    with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
        ent = json.load(f)["expert_mlp/full_b1"]
    monkeypatch.setattr(bench, "kernel_sources_sha", lambda: ent["sources_sha256"])
    assert bench.ncu_traffic("expert_mlp", "full_b1") == float(ent["dram_bytes_per_launch"])
    assert bench.ncu_traffic("expert_mlp", "no_such_workload") is None
    monkeypatch.setattr(bench, "kernel_sources_sha", lambda: "0" * 64)
    assert bench.ncu_traffic("expert_mlp", "full_b1") is None
