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


def test_stored_input_counters_are_the_margin_rejections_of_the_script():
    # the benchmark reads its rows' redraw counters from bench_inputs.json;
    # recompute a few with the committed script's own function (the oracle's
    # router on the host-drawn router weights) and compare
    import importlib.util
    import json

    from moe_decode_block_b200 import synth
    path = os.path.join(ROOT, "tests", "golden", "make_bench_inputs.py")
    spec = importlib.util.spec_from_file_location("make_bench_inputs", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    with open(bench.INPUTS_JSON) as f:
        stored = json.load(f)["workloads"]
    for name, x_seed in (("tiny_b1", 0), ("full_b8", 0), ("zipf_b32", 0), ("full_b64", 3000)):
        wl = synth.WORKLOADS[name]
        router_w, bias = synth.make_router(wl.shape, seed=0, routing=wl.routing)
        att = mod.attempts_for(wl.shape, wl.batch, router_w, bias, x_seed)
        assert att.tolist() == stored[name][str(x_seed)], name
        assert bench.x_attempts(name, x_seed) == stored[name][str(x_seed)]
    assert bench.x_attempts("no_such_workload", 0) is None


def test_parity_check_accepts_the_oracle_and_rejects_a_wrong_forward():
    import numpy as np
    import torch

    import oracle
    from moe_decode_block_b200 import synth
    s = synth.TINY
    wts = synth.make_weights(s, seed=0, device="cpu")
    x = synth.make_x(3, s.hidden, seed=0, attempts=[0, 0, 0])
    xb = synth.bf16_bits(x)
    o_out, o_ids, o_w, _ = oracle.moe_forward(xb, synth.bf16_bits(wts.router_w),
                                              [synth.bf16_bits(t) for t in wts.w13],
                                              [synth.bf16_bits(t) for t in wts.w2], synth.bf16_bits(wts.shared_w13),
                                              synth.bf16_bits(wts.shared_w2), s.top_k)
    out = torch.tensor(o_out, dtype=torch.float32).to(torch.bfloat16)
    ids = torch.tensor(o_ids)
    w = torch.tensor(o_w, dtype=torch.float32)
    good = bench.check_against_oracle(wts, x, out, ids, w, s.top_k)
    assert good["ok"] and good["ids_exact"] and good["max_out_err"] <= good["tol"]
    # the same check given the oracle's result directly
    assert bench.check_against_oracle(wts, x, out, ids, w, s.top_k, ref=(o_out, o_ids, o_w))["ok"]
    bad_out = out.clone()
    bad_out[1, 7] += 1.0
    assert not bench.check_against_oracle(wts, x, bad_out, ids, w, s.top_k)["ok"]
    bad_ids = ids.clone()
    bad_ids[0] = bad_ids[0].flip(0)
    assert not bench.check_against_oracle(wts, x, out, bad_ids, w, s.top_k)["ok"]
    nan_out = out.clone()
    nan_out[2, 0] = float("nan")
    assert not bench.check_against_oracle(wts, x, nan_out, ids, w, s.top_k)["ok"]
    assert np.isfinite(good["max_w_err"])
