"""CUDA path vs the fp64 oracle on a B200, through the C ABI.

Bar: expert ids exact, renormalised weights within 1e-5, outputs within
2e-2 * rms(oracle out).  Both execution plans are covered: the default one
(router kernel + one expert kernel with the shared expert, routed experts and
combine) and the two-stream one (shared expert on the aux stream, separate
combine kernel).  Inputs are seeded and synthetic (weights ~ N(0,0.02),
x ~ N(0,1), bf16) with a top-k logit margin >= 1e-3.  Every configuration,
full size included, is compared element by element on every token (the
oracle streams one selected expert at a time from the device).
"""
import numpy as np
import pytest
import torch

from moe_decode_block_b200 import MOE_OK, MoEDecode, synth
import oracle
from gpu_helpers import Run, expected_stages, margin_x, oracle_check

pytestmark = pytest.mark.gpu


PLANS = ["default", "two_stream"]


@pytest.fixture(scope="module", params=PLANS + ["tcgen05"])
def tiny(request):
    wts = synth.make_weights(synth.TINY, seed=0, device="cuda")
    return Run(synth.TINY, wts, max_batch=64, two_stream=request.param == "two_stream",
               tcgen05=request.param == "tcgen05")


@pytest.fixture(scope="module")
def full():
    wts = synth.make_weights(synth.FULL, seed=0, device="cuda")
    run = Run(synth.FULL, wts, max_batch=64)
    yield run
    run.blk.close()
    del run.wts, wts
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ tiny ----

@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 7, 8, 13, 32, 64])
def test_tiny_every_element(tiny, B):
    x = margin_x(B, synth.TINY.hidden, tiny.wts, synth.TINY.top_k, seed=B)
    before = tiny.blk.stats()
    out, ids, w = tiny.forward(x)
    oracle_check(tiny.wts, synth.TINY.top_k, x, out, ids, w)
    st = tiny.blk.stats()
    assert st["last_kernels"] == tiny.kernels_per_forward()
    assert st["last_token_tiles"] == (min(B, 32) + 7) // 8
    # the device counted the stages of the token classes this routing needs
    up, down = expected_stages(synth.TINY, ids.cpu().numpy(), B)
    assert [a - b for a, b in zip(st["stages_up"], before["stages_up"])] == up
    assert [a - b for a, b in zip(st["stages_down"], before["stages_down"])] == down
    assert tiny.blk.status() == MOE_OK


def test_tiny_config_seed0(tiny):
    x = margin_x(1, synth.TINY.hidden, tiny.wts, synth.TINY.top_k, seed=0)
    out, ids, w = tiny.forward(x)
    oracle_check(tiny.wts, synth.TINY.top_k, x, out, ids, w)


@pytest.mark.parametrize("plan", PLANS)
def test_tiny_top1_and_no_shared(plan):
    s = synth.BlockShape(hidden=256, n_experts=16, top_k=1, inter=128, shared_inter=0, n_shared=0)
    wts = synth.make_weights(s, seed=3, device="cuda")
    run = Run(s, wts, max_batch=8, two_stream=plan == "two_stream")
    x = margin_x(8, s.hidden, wts, 1, seed=3)
    out, ids, w = run.forward(x)
    assert torch.all(w == 1.0)
    oracle_check(wts, 1, x, out, ids, w)
    assert run.blk.stats()["last_kernels"] == run.kernels_per_forward()


@pytest.mark.parametrize("plan", PLANS)
def test_tiny_odd_shapes_several_panels_and_ragged_steps(plan):
    # inter 2056 -> two UP panels (gate/up pairs) with a ragged last panel;
    # hidden 4104 -> two DOWN panels and a ragged last 512-column combine
    # block; K not a multiple of 64 -> row-copy path, ragged steps; batch 40
    # -> two shared-expert units and a split routed unit
    s = synth.BlockShape(hidden=4104, n_experts=24, top_k=3, inter=2056, shared_inter=136, n_shared=1)
    wts = synth.make_weights(s, seed=4, device="cuda")
    run = Run(s, wts, max_batch=40, two_stream=plan == "two_stream")
    for B in (1, 6, 16, 40):
        x = margin_x(B, s.hidden, wts, s.top_k, seed=40 + B)
        out, ids, w = run.forward(x)
        oracle_check(wts, s.top_k, x, out, ids, w)


@pytest.mark.parametrize("H,E,k,B", [
    (256, 8, 8, 64),     # k == E: every token selects every expert (64 tokens -> two units each)
    (256, 64, 12, 8),    # k > 8: the router's k-round argmax path (64-expert instance)
    (512, 64, 32, 64),   # the largest top-k: 2048 assignments, experts above 32 tokens split
    (256, 384, 16, 8),   # k > 8 on the 384-expert router instance
    (256, 1024, 8, 64),  # the largest expert count (the 256-thread router instance), top-8 path
    (256, 1024, 12, 8),  # ... and its k-round path
])
def test_wide_top_k_and_every_expert_selected(H, E, k, B):
    s = synth.BlockShape(hidden=H, n_experts=E, top_k=k, inter=128, shared_inter=128, n_shared=1)
    wts = synth.make_weights(s, seed=5, device="cuda")
    run = Run(s, wts, max_batch=B)
    try:
        x = margin_x(B, s.hidden, wts, k, seed=50 + k)
        out, ids, w = run.forward(x)
        oracle_check(wts, k, x, out, ids, w)
        assert run.blk.status() == MOE_OK
    finally:
        run.blk.close()


def test_zero_down_weights_give_the_input_bitwise(tiny):
    wts = tiny.wts
    z2 = torch.zeros_like(wts.w2)
    blk = tiny.blk
    x = margin_x(5, synth.TINY.hidden, wts, synth.TINY.top_k, seed=77)
    out = torch.empty_like(x)
    ids = torch.empty(5, 2, dtype=torch.int32, device="cuda")
    w = torch.empty(5, 2, dtype=torch.float32, device="cuda")
    blk.forward(x, wts.router_w, wts.w13, z2, wts.shared_w13, torch.zeros_like(wts.shared_w2), out, ids, w)
    torch.cuda.synchronize()
    assert torch.equal(out, x)


def test_batch_zero_is_a_no_op(tiny):
    x = torch.empty(0, synth.TINY.hidden, dtype=torch.bfloat16, device="cuda")
    sentinel = torch.full((1, synth.TINY.hidden), 7.0, dtype=torch.bfloat16, device="cuda")
    ids = torch.full((1, 2), -1, dtype=torch.int32, device="cuda")
    w = torch.zeros(1, 2, device="cuda")
    before = tiny.blk.stats()["forwards"]
    tiny.blk.forward(x, tiny.wts.router_w, tiny.wts.w13, tiny.wts.w2, tiny.wts.shared_w13, tiny.wts.shared_w2,
                     sentinel, ids, w, batch=0)
    torch.cuda.synchronize()
    assert torch.all(sentinel == 7.0) and torch.all(ids == -1)
    assert tiny.blk.stats()["forwards"] == before


def test_separate_expert_tensors_and_a_single_stream(tiny):
    wts = tiny.wts
    w13 = [wts.w13[e].clone() for e in range(synth.TINY.n_experts)]
    w2 = [wts.w2[e].clone() for e in range(synth.TINY.n_experts)]
    x = margin_x(6, synth.TINY.hidden, wts, 2, seed=5)
    main = torch.cuda.current_stream()
    out, ids, w = tiny.forward(x, stream_aux=main, w13=w13, w2=w2)
    oracle_check(wts, 2, x, out, ids, w)


def test_repeated_calls_are_consistent(tiny):
    # the workspace returns to zero after every call
    x = margin_x(9, synth.TINY.hidden, tiny.wts, 2, seed=6)
    o1, i1, w1 = tiny.forward(x)
    for _ in range(5):
        o2, i2, w2 = tiny.forward(x)
        assert torch.equal(i1, i2)
        assert torch.max(torch.abs(w1 - w2)) <= 1e-6
        assert torch.max(torch.abs(o1.float() - o2.float())) <= 2 * 2 ** -7 * o1.float().abs().max()
    oracle_check(tiny.wts, 2, x, o2, i2, w2)


@pytest.mark.parametrize("kind,B", [("pinned", 4), ("pageable", 4), ("mixed", 4), ("pinned", 13)])
def test_host_buffer_entry_point(tiny, kind, B):
    # pinned (mapped) outputs are stored by the kernels directly; pageable or
    # mixed ones go through device staging and copies
    wts = tiny.wts
    x = margin_x(B, synth.TINY.hidden, wts, 2, seed=8 + B).cpu()
    out = torch.empty_like(x)
    ids = torch.empty(B, 2, dtype=torch.int32)
    w = torch.empty(B, 2, dtype=torch.float32)
    if kind == "pinned":
        x, out, ids, w = x.pin_memory(), out.pin_memory(), ids.pin_memory(), w.pin_memory()
    elif kind == "mixed":
        out = out.pin_memory()
    for _ in range(2):
        out.fill_(float("nan"))
        ids.fill_(-1)
        w.fill_(float("nan"))
        tiny.blk.forward_host(x, wts.router_w, wts.w13, wts.w2, wts.shared_w13, wts.shared_w2, out, ids, w)
        oracle_check(wts, 2, x, out, ids, w)
    assert tiny.blk.status() == MOE_OK


def test_host_buffer_entry_point_replays_follow_new_inputs(tiny):
    # with pinned, mapped buffers the host-buffer entry point captures the
    # copy of x and the forward once and replays them: new contents of the
    # same buffers must give new results, and another batch a new capture
    wts = tiny.wts
    B = 6
    x = torch.empty(B, synth.TINY.hidden, dtype=torch.bfloat16).pin_memory()
    out = torch.empty_like(x).pin_memory()
    ids = torch.empty(B, 2, dtype=torch.int32).pin_memory()
    w = torch.empty(B, 2, dtype=torch.float32).pin_memory()
    before = tiny.blk.stats()["forwards"]
    for seed, b in ((30, B), (31, B), (32, B), (33, 4), (34, B)):
        x[:b].copy_(margin_x(b, synth.TINY.hidden, wts, 2, seed=seed).cpu())
        out.fill_(float("nan"))
        ids.fill_(-1)
        tiny.blk.forward_host(x[:b], wts.router_w, wts.w13, wts.w2, wts.shared_w13, wts.shared_w2, out[:b], ids[:b],
                              w[:b], batch=b)
        oracle_check(wts, 2, x[:b], out[:b], ids[:b], w[:b])
    assert tiny.blk.stats()["forwards"] == before + 5
    assert tiny.blk.status() == MOE_OK


def _graph_alternating(run, xa, xb, replays=20):
    """Capture [x <- xa; forward; x <- xb; forward] in one graph and replay it:
    an activation read hoisted above a grid-dependency wait would show up as
    one output computed from the other input.  Every replay is compared with
    eager forwards of the same inputs, and the last replay's two outputs with
    the fp64 oracle."""
    s = run.s
    B = xa.shape[0]
    xbuf = torch.empty_like(xa)
    outs = [torch.empty_like(xa) for _ in range(2)]
    ids = [torch.empty(B, s.top_k, dtype=torch.int32, device="cuda") for _ in range(2)]
    ws = [torch.empty(B, s.top_k, dtype=torch.float32, device="cuda") for _ in range(2)]
    ref = [run.forward(xa), run.forward(xb)]
    stream = torch.cuda.Stream()
    aux = torch.cuda.Stream()
    wts = run.wts
    args = (wts.router_w, wts.w13, wts.w2, wts.shared_w13, wts.shared_w2)
    with torch.cuda.stream(stream):
        # warm-up outside capture
        xbuf.copy_(xa)
        run.blk.forward(xbuf, *args, outs[0], ids[0], ws[0], stream_main=stream, stream_aux=aux)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        cur = torch.cuda.current_stream()
        xbuf.copy_(xa)
        run.blk.forward(xbuf, *args, outs[0], ids[0], ws[0], stream_main=cur, stream_aux=aux)
        xbuf.copy_(xb)
        run.blk.forward(xbuf, *args, outs[1], ids[1], ws[1], stream_main=cur, stream_aux=aux)
    for _ in range(replays):
        for o in outs:
            o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for i in range(2):
            assert torch.equal(ids[i], ref[i][1])
            err = torch.max(torch.abs(outs[i].float() - ref[i][0].float()))
            assert err <= 2 * 2 ** -7 * ref[i][0].float().abs().max()
    for i, xi in enumerate((xa, xb)):
        oracle_check(run.wts, s.top_k, xi, outs[i], ids[i], ws[i])
    del g


def test_graph_replay_alternating_inputs_tiny(tiny):
    xa = margin_x(3, synth.TINY.hidden, tiny.wts, 2, seed=9)
    xb = margin_x(3, synth.TINY.hidden, tiny.wts, 2, seed=10)
    _graph_alternating(tiny, xa, xb)


# ------------------------------------------------------------- full size ----

@pytest.mark.parametrize("B", [1, 8])
def test_full_size_every_token(full, B):
    x = margin_x(B, synth.FULL.hidden, full.wts, synth.FULL.top_k, seed=0)
    before = full.blk.stats()
    out, ids, w = full.forward(x)
    oracle_check(full.wts, synth.FULL.top_k, x, out, ids, w)
    st = full.blk.stats()
    up, down = expected_stages(synth.FULL, ids.cpu().numpy(), B)
    assert [a - b for a, b in zip(st["stages_up"], before["stages_up"])] == up
    assert [a - b for a, b in zip(st["stages_down"], before["stages_down"])] == down


def test_full_size_batch64_every_token(full):
    x = margin_x(64, synth.FULL.hidden, full.wts, synth.FULL.top_k, seed=0)
    out, ids, w = full.forward(x)
    distinct = len(set(ids.cpu().numpy().ravel().tolist()))
    assert distinct > 200  # most experts touched
    oracle_check(full.wts, synth.FULL.top_k, x, out, ids, w)


@pytest.mark.parametrize("B", [1, 2, 4, 8, 16, 32, 64])
def test_zipf_sweep(full, B):
    # same seeded weights as the uniform block; routing="zipf" only adds the
    # Zipf(1.2) log-prior bias to the router logits
    wts = full.wts
    zipf = synth.BlockWeights(wts.router_w, wts.w13, wts.w2, wts.shared_w13, wts.shared_w2,
                              synth.zipf_log_prior(synth.FULL.n_experts, seed=0, device="cuda"))
    run = Run(synth.FULL, zipf, max_batch=64)
    try:
        x = margin_x(B, synth.FULL.hidden, zipf, synth.FULL.top_k, seed=B)
        out, ids, w = run.forward(x)
        oracle_check(zipf, synth.FULL.top_k, x, out, ids, w)
        assert run.blk.status() == MOE_OK
    finally:
        run.blk.close()


def test_all_tokens_routed_to_the_same_experts(full):
    # a +30 bias on eight experts sends every token to them: each of those
    # experts receives all 64 tokens (the maximum-reuse extreme).  Natural
    # logits are ~N(0, 1.7^2), so +30 always wins, while fp32 logits near 30
    # still resolve 4e-6 (a +1000 bias would blur the weights to ~6e-5).
    wts = full.wts
    bias = torch.zeros(synth.FULL.n_experts, dtype=torch.float32, device="cuda")
    hot = torch.tensor([3, 77, 128, 200, 255, 301, 350, 383], device="cuda")
    bias[hot] = 30.0
    biased = synth.BlockWeights(wts.router_w, wts.w13, wts.w2, wts.shared_w13, wts.shared_w2, bias)
    run = Run(synth.FULL, biased, max_batch=64)
    try:
        x = margin_x(64, synth.FULL.hidden, biased, synth.FULL.top_k, seed=123)
        out, ids, w = run.forward(x)
        assert set(ids.cpu().numpy().ravel().tolist()) == set(hot.tolist())
        oracle_check(biased, synth.FULL.top_k, x, out, ids, w)
    finally:
        run.blk.close()


def test_graph_replay_alternating_inputs_full_b8(full):
    xa = margin_x(8, synth.FULL.hidden, full.wts, 8, seed=11)
    xb = margin_x(8, synth.FULL.hidden, full.wts, 8, seed=12)
    _graph_alternating(full, xa, xb, replays=5)


@pytest.mark.parametrize("B", [1, 8, 40])
def test_full_size_tcgen05_expert_kernel(full, B):
    # the expert kernel on tcgen05 with TMEM accumulators (MOE_FLAG_TCGEN05)
    run = Run(synth.FULL, full.wts, max_batch=64, tcgen05=True)
    try:
        x = margin_x(B, synth.FULL.hidden, full.wts, synth.FULL.top_k, seed=300 + B)
        out, ids, w = run.forward(x)
        oracle_check(full.wts, synth.FULL.top_k, x, out, ids, w)
        assert run.blk.status() == MOE_OK
    finally:
        run.blk.close()


@pytest.mark.parametrize("B", [1, 8, 40])
def test_full_size_two_stream_plan(full, B):
    run = Run(synth.FULL, full.wts, max_batch=64, two_stream=True)
    try:
        x = margin_x(B, synth.FULL.hidden, full.wts, synth.FULL.top_k, seed=200 + B)
        out, ids, w = run.forward(x)
        oracle_check(full.wts, synth.FULL.top_k, x, out, ids, w)
        assert run.blk.stats()["last_kernels"] == 4
        assert run.blk.status() == MOE_OK
    finally:
        run.blk.close()


@pytest.mark.parametrize("plan", PLANS)
def test_exact_logit_ties_go_to_the_smaller_id(plan):
    # router columns 2p and 2p+1 identical: their logits are equal in fp64 and
    # bitwise equal on the GPU (one thread sums both columns in the same order
    # and one vector reduction adds them), so every selected pair must come
    # out smaller id first; x is drawn so that distinct pairs keep a margin
    s = synth.TINY
    wts = synth.make_weights(s, seed=21, device="cuda")
    rw = wts.router_w.clone()
    rw[:, 1::2] = rw[:, 0::2]
    tied = synth.BlockWeights(rw, wts.w13, wts.w2, wts.shared_w13, wts.shared_w2, None)
    run = Run(s, tied, max_batch=8, two_stream=plan == "two_stream")
    B = 6
    rows = []
    attempt = 0
    while len(rows) < B:
        x1 = synth.make_x(1, s.hidden, seed=500 + attempt)
        attempt += 1
        logits, _, _ = oracle.router(synth.bf16_bits(x1), synth.bf16_bits(rw), s.top_k, None)
        pair = np.sort(logits[0, 0::2])[::-1]
        if pair[0] - pair[1] >= 1e-3:
            rows.append(x1)
    x = torch.cat(rows).to("cuda")
    out, ids, w = run.forward(x)
    ids_h = ids.cpu().numpy()
    assert np.all(ids_h[:, 0] % 2 == 0) and np.all(ids_h[:, 1] == ids_h[:, 0] + 1)
    oracle_check(tied, s.top_k, x, out, ids, w)
