"""Pins of the fp64 oracle against facts that do not come from the oracle
itself: a hand-derived closed-form example, invariants of the definition,
brute force over every expert subset, and special cases that reduce to
library routines (scipy softmax, torch silu, float64 matmul).

Both oracle implementations (C and numpy) are pinned.  CPU only.
"""
import ctypes
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle import moe_oracle_np as npo
from moe_decode_block_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers ---

def to_bits(a):
    """float array -> bf16 bit patterns (values must be bf16-exact here)."""
    t = torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.tensor(np.asarray(a, dtype=np.float32))), "not bf16-exact"
    return t.view(torch.int16).numpy().view(np.uint16)


def rand_block(B=4, H=32, E=16, k=2, I=8, Is=8, seed=0, std=0.02, xstd=1.0, bias=False):
    g = torch.Generator().manual_seed(seed)

    def rb(*shape, s=std):
        return (torch.randn(*shape, generator=g) * s).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)

    d = dict(
        x=rb(B, H, s=xstd), router_w=rb(H, E, s=0.3),
        w13=[rb(H, 2 * I, s=0.3) for _ in range(E)], w2=[rb(I, H, s=0.3) for _ in range(E)],
        sw13=rb(H, 2 * Is, s=0.3), sw2=rb(Is, H, s=0.3), k=k,
        bias=(torch.randn(E, generator=g).numpy().astype(np.float32) if bias else None),
    )
    return d


def run(impl, d, **over):
    d = {**d, **over}
    if impl == "c":
        return oracle.moe_forward(d["x"], d["router_w"], d["w13"], d["w2"], d["sw13"], d["sw2"], d["k"], d["bias"])
    return npo.moe_forward(d["x"], d["router_w"], d["w13"], d["w2"], d["sw13"], d["sw2"], d["k"], d["bias"])


def run_block(impl, d, ids, w):
    if impl == "c":
        return oracle.block(d["x"], ids, w, d["w13"], d["w2"], d["sw13"], d["sw2"])
    return npo.block(d["x"], ids, w, d["w13"], d["w2"], d["sw13"], d["sw2"])


def f64(bits):
    return npo.bf16_bits_to_f64(bits)


def torch_mlp(xf, W13, W2):
    """Dense SwiGLU MLP from library routines (torch float64 matmul + silu)."""
    x = torch.tensor(xf, dtype=torch.float64)
    w13 = torch.tensor(f64(W13))
    w2 = torch.tensor(f64(W2))
    inter = w13.shape[1] // 2
    gu = x @ w13
    return (torch.nn.functional.silu(gu[..., :inter]) * gu[..., inter:] @ w2).numpy()


IMPLS = ["c", "np"]


# ------------------------------------------------------------------ pins ----

@pytest.mark.parametrize("impl", IMPLS)
def test_worked_example_closed_form(impl):
    with open(os.path.join(GOLDEN, "worked_example.json")) as f:
        g = json.load(f)
    d = dict(x=to_bits(g["x"]), router_w=to_bits(g["router_w"]),
             w13=[to_bits(w) for w in g["w13"]], w2=[to_bits(w) for w in g["w2"]],
             sw13=to_bits(g["shared_w13"]), sw2=to_bits(g["shared_w2"]), k=2, bias=None)
    out, ids, w, logits = run(impl, d)
    ex = g["expected"]
    np.testing.assert_array_equal(ids, np.array(ex["topk_ids"]))
    np.testing.assert_allclose(logits, ex["logits"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(w, ex["topk_w"], rtol=1e-14, atol=0)
    np.testing.assert_allclose(out, ex["out"], rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("impl", IMPLS)
def test_renormalised_weights_sum_to_one(impl):
    d = rand_block(B=16, E=16, k=4, seed=1, bias=True)
    _, _, w, _ = run(impl, d)
    assert np.all(w > 0)
    assert np.max(np.abs(w.sum(axis=1) - 1.0)) <= 1e-12


@pytest.mark.parametrize("impl", IMPLS)
def test_weights_equal_softmax_over_selected_logits(impl):
    # renormalising the full softmax over S equals a softmax over S alone
    d = rand_block(B=8, E=16, k=3, seed=2)
    _, ids, w, logits = run(impl, d)
    for b in range(8):
        ref = scipy.special.softmax(logits[b, ids[b]])
        np.testing.assert_allclose(w[b], ref, rtol=1e-13)
        # and the ratio of two weights is exp of the logit gap (sign of the exponent)
        assert math.isclose(w[b, 0] / w[b, 1], math.exp(logits[b, ids[b, 0]] - logits[b, ids[b, 1]]), rel_tol=1e-12)


def test_c_logits_match_library_matmul():
    d = rand_block(B=5, H=64, E=16, seed=3, bias=True)
    logits, _, _ = oracle.router(d["x"], d["router_w"], 2, d["bias"])
    ref = f64(d["x"]) @ f64(d["router_w"]) + d["bias"].astype(np.float64)[None]
    np.testing.assert_allclose(logits, ref, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("impl", IMPLS)
def test_one_hot_token_reads_one_router_row(impl):
    d = rand_block(B=1, H=32, E=16, seed=4, bias=True)
    for h in (0, 7, 31):
        x = np.zeros((1, 32), np.float32); x[0, h] = 1.0
        logits = (oracle.router(to_bits(x), d["router_w"], 2, d["bias"])[0] if impl == "c"
                  else npo.router(to_bits(x), d["router_w"], 2, d["bias"])[0])
        np.testing.assert_array_equal(logits[0], f64(d["router_w"])[h] + d["bias"].astype(np.float64))


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("k", [1, 2, 3])
def test_selection_brute_force_over_all_subsets(impl, k):
    # tiny shape: 16 experts; the chosen set maximises the sum of logits over
    # all C(16,k) subsets and comes out ordered by logit descending
    d = rand_block(B=6, H=32, E=16, k=k, seed=5 + k)
    _, ids, _, logits = run(impl, d, k=k)
    for b in range(6):
        best = max(itertools.combinations(range(16), k), key=lambda s: sum(logits[b, list(s)]))
        assert sorted(best) == sorted(ids[b].tolist())
        assert all(logits[b, ids[b, j]] > logits[b, ids[b, j + 1]] for j in range(k - 1))


@pytest.mark.parametrize("impl", IMPLS)
def test_ties_go_to_smaller_expert_id(impl):
    d = rand_block(B=3, H=16, E=8, k=3, seed=9)
    R = f64(d["router_w"]).astype(np.float32)
    x = np.zeros((3, 16), np.float32); x[:, 0] = 1.0
    # only row 0 of R matters; experts 2 and 5 get bitwise-equal logits 4.0
    R[0, :] = [0.5, 0.25, 4.0, -1.0, 0.0, 4.0, 1.0, 3.0]
    _, ids, w, _ = run(impl, d, router_w=to_bits(R), x=to_bits(x), bias=None)
    for b in range(3):
        assert ids[b].tolist() == [2, 5, 7]
        assert w[b, 0] == w[b, 1]


@pytest.mark.parametrize("impl", IMPLS)
def test_forced_routing_matches_and_other_subsets_differ(impl):
    d = rand_block(B=2, H=32, E=16, k=2, seed=11)
    out, ids, w, logits = run(impl, d)
    np.testing.assert_array_equal(run_block(impl, d, ids, w), out)
    # any other subset (with its own renormalised weights) changes the output
    for b in range(2):
        for s in itertools.islice(itertools.combinations(range(16), 2), 0, 120, 7):
            if sorted(s) == sorted(ids[b].tolist()):
                continue
            sid = np.array([s], np.int32)
            sw = scipy.special.softmax(logits[b, list(s)])[None]
            alt = run_block(impl, {**d, "x": d["x"][b:b + 1]}, sid, sw)
            assert np.max(np.abs(alt - out[b:b + 1])) > 1e-6


@pytest.mark.parametrize("impl", IMPLS)
def test_identical_experts_reduce_to_one_dense_mlp(impl):
    # routing-independent: sum_j w_j = 1, so the routed part is MLP(x) exactly
    d = rand_block(B=5, H=32, E=16, k=4, I=8, seed=12, bias=True)
    d["w13"] = [d["w13"][3]] * 16
    d["w2"] = [d["w2"][3]] * 16
    out, _, _, _ = run(impl, d)
    X = f64(d["x"])
    ref = X + torch_mlp(X, d["w13"][0], d["w2"][0]) + torch_mlp(X, d["sw13"], d["sw2"])
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("impl", IMPLS)
def test_block_equals_library_composition(impl):
    # distinct experts: out = x + sum_j softmax(logits[S])_j * MLP_{S_j}(x) + MLP_s(x)
    d = rand_block(B=3, H=32, E=16, k=3, I=8, seed=13)
    out, ids, _, _ = run(impl, d)
    X = f64(d["x"])
    logits = X @ f64(d["router_w"])
    for b in range(3):
        S = np.argsort(-logits[b], kind="stable")[:3]
        np.testing.assert_array_equal(ids[b], S)
        wts = scipy.special.softmax(logits[b, S])
        ref = X[b] + sum(wts[j] * torch_mlp(X[b], d["w13"][S[j]], d["w2"][S[j]]) for j in range(3))
        ref = ref + torch_mlp(X[b], d["sw13"], d["sw2"])
        np.testing.assert_allclose(out[b], ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("impl", IMPLS)
def test_silu_and_gate_up_order_one_hot(impl):
    # x = e_0, gate column c = g_c, up column = 1, W2 = identity:
    # y_c = silu(g_c) = g_c * expit(g_c)  (scipy), which pins the activation,
    # the sign of its exponent and that the gate is the first half of w13
    H = I = 8
    gvals = np.array([1.0, -1.0, 2.0, -2.0, 0.5, 0.0, 4.0, -0.25], np.float32)
    W13 = np.zeros((H, 2 * I), np.float32)
    W13[0, :I] = gvals
    W13[0, I:] = 1.0
    W2 = np.eye(I, H, dtype=np.float32)
    x = np.zeros((1, H), np.float32); x[0, 0] = 1.0
    zeros = np.zeros((H, 2 * I), np.float32)
    d = dict(x=to_bits(x), router_w=to_bits(np.zeros((H, 2), np.float32)),
             w13=[to_bits(W13), to_bits(W13)], w2=[to_bits(W2), to_bits(W2)],
             sw13=to_bits(zeros), sw2=to_bits(np.zeros((I, H), np.float32)), k=1, bias=None)
    out, ids, w, _ = run(impl, d)
    assert ids[0, 0] == 0 and w[0, 0] == 1.0
    expected = x[0].astype(np.float64) + gvals * scipy.special.expit(gvals.astype(np.float64))
    np.testing.assert_allclose(out[0], expected, rtol=1e-15, atol=1e-16)
    np.testing.assert_allclose(expected[0] - 1.0, 0.7310585786300049, rtol=1e-15)  # silu(1) = e/(1+e)


@pytest.mark.parametrize("impl", IMPLS)
def test_batch_rows_are_permutation_equivariant(impl):
    d = rand_block(B=7, seed=14, bias=True)
    out, ids, w, _ = run(impl, d)
    perm = np.random.default_rng(0).permutation(7)
    out_p, ids_p, w_p, _ = run(impl, d, x=d["x"][perm])
    np.testing.assert_array_equal(out_p, out[perm])
    np.testing.assert_array_equal(ids_p, ids[perm])
    np.testing.assert_array_equal(w_p, w[perm])


@pytest.mark.parametrize("impl", IMPLS)
def test_expert_relabelling(impl):
    d = rand_block(B=4, E=16, k=3, seed=15, bias=True)
    out, ids, w, _ = run(impl, d)
    perm = np.random.default_rng(1).permutation(16)  # new id n holds old expert perm[n]
    inv = np.argsort(perm)
    d2 = dict(d, router_w=np.ascontiguousarray(d["router_w"][:, perm]),
              w13=[d["w13"][perm[n]] for n in range(16)], w2=[d["w2"][perm[n]] for n in range(16)],
              bias=d["bias"][perm])
    out2, ids2, w2, _ = run(impl, d2)
    np.testing.assert_array_equal(ids2, inv[ids])
    # the full-softmax denominator is summed in the new expert order: rounding only
    np.testing.assert_allclose(w2, w, rtol=1e-14, atol=0)
    np.testing.assert_allclose(out2, out, rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("impl", IMPLS)
def test_zero_down_projections_leave_the_residual(impl):
    d = rand_block(B=3, seed=16)
    z = np.zeros_like(d["w2"][0])
    out, _, _, _ = run(impl, d, w2=[z] * 16, sw2=np.zeros_like(d["sw2"]))
    np.testing.assert_array_equal(out, f64(d["x"]))


@pytest.mark.parametrize("impl", IMPLS)
def test_shared_expert_alone(impl):
    d = rand_block(B=3, seed=17)
    z = np.zeros_like(d["w2"][0])
    out, _, _, _ = run(impl, d, w2=[z] * 16)
    X = f64(d["x"])
    np.testing.assert_allclose(out, X + torch_mlp(X, d["sw13"], d["sw2"]), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("impl", IMPLS)
def test_top1_weight_is_exactly_one(impl):
    d = rand_block(B=5, k=1, seed=18)
    _, _, w, _ = run(impl, d, k=1)
    assert np.all(w == 1.0)


@pytest.mark.parametrize("impl", IMPLS)
def test_large_bias_forces_an_expert_first(impl):
    d = rand_block(B=4, E=16, k=2, seed=19)
    bias = np.zeros(16, np.float32); bias[13] = 1.0e3
    _, ids, w, logits = run(impl, d, bias=bias)
    assert np.all(ids[:, 0] == 13)
    assert np.all(w[:, 0] > 1 - 1e-12)
    np.testing.assert_allclose(logits[:, 13] - 1e3, f64(d["x"]) @ f64(d["router_w"])[:, 13], atol=1e-10)


@pytest.mark.parametrize("impl", IMPLS)
def test_routed_part_is_linear_in_w2(impl):
    d = rand_block(B=3, seed=20)
    out1, _, _, _ = run(impl, d)
    w2x2 = [to_bits(2.0 * f64(w)) for w in d["w2"]]  # doubling is bf16-exact
    out2, _, _, _ = run(impl, d, w2=w2x2)
    X = f64(d["x"])
    s = torch_mlp(X, d["sw13"], d["sw2"])
    np.testing.assert_allclose(out2 - X - s, 2.0 * (out1 - X - s), rtol=1e-12, atol=1e-12)


def test_c_and_numpy_oracles_agree():
    for seed in range(3):
        d = rand_block(B=6, H=64, E=16, k=2, I=16, Is=24, seed=100 + seed, bias=bool(seed % 2))
        oc, ic, wc, lc = run("c", d)
        on, in_, wn, ln = run("np", d)
        np.testing.assert_array_equal(ic, in_)
        np.testing.assert_allclose(lc, ln, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(wc, wn, rtol=1e-13)
        np.testing.assert_allclose(oc, on, rtol=1e-12, atol=1e-12)


def test_c_oracle_does_not_depend_on_thread_count():
    d = rand_block(B=3, H=256, E=16, k=2, I=128, Is=128, seed=21)
    gomp = ctypes.CDLL("libgomp.so.1")
    n0 = oracle.num_threads()
    try:
        gomp.omp_set_num_threads(1)
        o1 = run("c", d)[0]
        gomp.omp_set_num_threads(max(2, n0))
        o2 = run("c", d)[0]
    finally:
        gomp.omp_set_num_threads(n0)
    np.testing.assert_array_equal(o1, o2)


def test_tiny_config_inputs_through_both_oracles():
    # the tiny workload itself (seed 0), checked C vs numpy and on its invariants
    wl = synth.WORKLOADS["tiny_b1"]
    s = wl.shape
    wts = synth.make_weights(s, seed=0)
    x = synth.bf16_bits(synth.make_x(1, s.hidden, seed=0))
    args = (x, synth.bf16_bits(wts.router_w), [synth.bf16_bits(w) for w in wts.w13],
            [synth.bf16_bits(w) for w in wts.w2], synth.bf16_bits(wts.shared_w13), synth.bf16_bits(wts.shared_w2), 2)
    oc, ic, wc, lc = oracle.moe_forward(*args)
    on, in_, wn, _ = npo.moe_forward(*args)
    np.testing.assert_array_equal(ic, in_)
    np.testing.assert_allclose(oc, on, rtol=1e-12, atol=1e-12)
    assert abs(wc.sum() - 1) < 1e-12
    assert oracle.topk_margin(lc, 2)[0] > 0


# ------------------------------------------- expert-at-a-time driver ---

@pytest.mark.parametrize("B,k,shared", [(1, 2, True), (7, 3, True), (16, 8, False), (33, 16, True)])
def test_streamed_block_is_bitwise_the_block(B, k, shared):
    # block_streamed evaluates each selected expert for the tokens that chose
    # it and sums in block's order, so it must equal block() bit for bit; it
    # fetches every selected expert exactly once, in ascending id order, and
    # nothing else
    d = rand_block(B=B, H=48, E=24, k=k, I=16, Is=24, seed=40 + B)
    _, ids, w = oracle.router(d["x"], d["router_w"], k, None)
    sw13, sw2 = (d["sw13"], d["sw2"]) if shared else (None, None)
    ref = oracle.block(d["x"], ids, w, d["w13"], d["w2"], sw13, sw2)
    fetched = []

    def fetch(e):
        fetched.append(e)
        return d["w13"][e], d["w2"][e]

    got = oracle.block_streamed(d["x"], ids, w, fetch, sw13, sw2)
    assert np.array_equal(got, ref)
    assert fetched == sorted(set(ids.ravel().tolist()))


def test_expert_outputs_is_one_swiglu_mlp_per_row():
    # one expert's outputs for a row list equal the block of a top-1 routing
    # to that expert with the residual taken away (weight 1, no shared)
    d = rand_block(B=5, H=32, E=8, k=1, I=8, Is=8, seed=9)
    rows = np.array([4, 0, 2, 2], dtype=np.int32)
    y = oracle.expert_outputs(d["x"], d["w13"][3], d["w2"][3], rows)
    ids = np.full((5, 1), 3, np.int32)
    full = oracle.block(d["x"], ids, np.ones((5, 1)), d["w13"], d["w2"])
    resid = d["x"].astype(np.uint32) << 16
    xr = resid.view(np.float32).astype(np.float64)
    np.testing.assert_allclose(y, (full - xr)[rows], rtol=0, atol=1e-12)


# ------------------------------------------------------- FP8 expert weights ---

def _fp8_expert(I, H, seed, scale_lo=0.5, scale_hi=2.0):
    g = torch.Generator().manual_seed(seed)
    q13 = torch.randint(0, 256, (2 * I, H), generator=g, dtype=torch.uint8)
    q2 = torch.randint(0, 256, (H, I), generator=g, dtype=torch.uint8)
    q13[(q13 & 0x7F) == 0x7F] = 0x38  # no NaN codes (replace with 1.0)
    q2[(q2 & 0x7F) == 0x7F] = 0x38
    s13 = (scale_lo + (scale_hi - scale_lo) * torch.rand(-(-2 * I // 128), -(-H // 128), generator=g)) * 2 ** -9
    s2 = (scale_lo + (scale_hi - scale_lo) * torch.rand(-(-H // 128), -(-I // 128), generator=g)) * 2 ** -9
    return q13.numpy(), s13.numpy().astype(np.float32), q2.numpy(), s2.numpy().astype(np.float32)


def _torch_decode(q):
    return torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).double().numpy()


def test_e4m3_decoding_matches_torch_for_every_code():
    ref = _torch_decode(np.arange(256, dtype=np.uint8))
    for code in range(256):
        v = oracle.e4m3_value(code)
        if np.isnan(ref[code]):
            assert np.isnan(v), code
        else:
            assert v == ref[code], (code, v, ref[code])
    assert oracle.e4m3_value(0x7E) == 448.0 and oracle.e4m3_value(0x01) == 2.0 ** -9


def _dequant(q, s):
    d = _torch_decode(q)
    o, i = q.shape
    full = np.repeat(np.repeat(s.astype(np.float64), 128, axis=0), 128, axis=1)[:o, :i]
    return d * full


def test_fp8_expert_with_unit_scales_is_the_bf16_expert_bitwise():
    # e4m3 values are exact in bf16: with unit scales the fp8 expert must be
    # the bf16 oracle's expert on the decoded (transposed) weights, bit for bit
    H, I = 256, 192
    q13, s13, q2, s2 = _fp8_expert(I, H, seed=1)
    s13[:] = 1.0
    s2[:] = 1.0
    x = rand_block(B=3, H=H, seed=2)["x"]
    y8 = oracle.expert_outputs_fp8(x, q13, s13, q2, s2, [0, 2, 1])
    w13 = to_bits(_torch_decode(q13).T.astype(np.float32))
    w2 = to_bits(_torch_decode(q2).T.astype(np.float32))
    y16 = oracle.expert_outputs(x, w13, w2, [0, 2, 1])
    assert np.array_equal(y8, y16)


def test_fp8_block_scale_applies_to_its_block_only():
    # doubling one scale equals doubling exactly that 128 x 128 block of the
    # dequantized weights (a power-of-two scaling is exact, and the doubled
    # values are still exact in bf16): compare with the bf16 oracle on the
    # decoded weights with that block doubled
    H, I = 384, 256
    q13, s13, q2, s2 = _fp8_expert(I, H, seed=3)
    s13[:] = 1.0
    s2[:] = 1.0
    x = rand_block(B=2, H=H, seed=4)["x"]
    s13b = s13.copy()
    s13b[1, 2] = 2.0  # outputs 128..255, inputs 256..383
    y = oracle.expert_outputs_fp8(x, q13, s13b, q2, s2, [0, 1])
    d13 = _torch_decode(q13)
    d13[128:256, 256:384] *= 2.0
    y16 = oracle.expert_outputs(x, to_bits(d13.T.astype(np.float32)), to_bits(_torch_decode(q2).T.astype(np.float32)),
                                [0, 1])
    assert np.array_equal(y, y16)


def test_fp8_expert_matches_a_library_composition():
    # torch's e4m3 decoding, numpy fp64 matmuls and scipy's logistic function
    H, I = 256, 160
    q13, s13, q2, s2 = _fp8_expert(I, H, seed=5)
    x = rand_block(B=4, H=H, seed=6)["x"]
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    W13 = _dequant(q13, s13)  # [2I, H]
    W2 = _dequant(q2, s2)     # [H, I]
    gu = xf @ W13.T
    a = gu[:, :I] * scipy.special.expit(gu[:, :I]) * gu[:, I:]
    ref = a @ W2.T
    y = oracle.expert_outputs_fp8(x, q13, s13, q2, s2, np.arange(4))
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12)


def test_fp8_streamed_block_combines_like_the_block():
    # routing, residual and shared expert around fp8 experts: the fp8 block
    # with unit scales equals the bf16 oracle's block on the decoded weights
    H, I, E, k = 128, 128, 6, 2
    experts = [_fp8_expert(I, H, seed=20 + e) for e in range(E)]
    for q13, s13, q2, s2 in experts:
        s13[:] = 1.0
        s2[:] = 1.0
    shared = _fp8_expert(I, H, seed=40)
    shared[1][:] = 1.0
    shared[3][:] = 1.0
    d = rand_block(B=5, H=H, E=E, k=k, seed=7)
    _, ids, w = oracle.router(d["x"], d["router_w"], k, None)
    out8 = oracle.block_streamed_fp8(d["x"], ids, w, lambda e: experts[e], shared)
    tb = lambda q: to_bits(_torch_decode(q).T.astype(np.float32))
    out16 = oracle.block(d["x"], ids, w, [tb(e[0]) for e in experts], [tb(e[2]) for e in experts],
                         tb(shared[0]), tb(shared[2]))
    assert np.array_equal(out8, out16)
