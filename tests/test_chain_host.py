"""Host-side checks of the block chain's arguments (no GPU)."""
import pytest

from moe_decode_block_b200.chain import check_chain_args


def _w():
    return (object(), object(), object(), object(), object())


def test_matching_lengths_pass():
    outs = [object(), object(), object()]
    check_chain_args(3, [_w(), _w(), _w()], outs, [1, 2, 3], [1, 2, 3])


@pytest.mark.parametrize("bad", ["weights", "outs", "topk_ids", "topk_w"])
def test_a_short_sequence_is_rejected(bad):
    seqs = dict(weights=[_w(), _w()], outs=[object(), object()], topk_ids=[1, 2], topk_w=[1, 2])
    seqs[bad] = seqs[bad][:1]
    with pytest.raises(ValueError, match=bad):
        check_chain_args(2, **seqs)


def test_weights_need_five_tensors_and_outputs_distinct_buffers():
    with pytest.raises(ValueError, match="weights"):
        check_chain_args(1, [_w()[:4]], [object()], [1], [1])
    o = object()
    with pytest.raises(ValueError, match="distinct"):
        check_chain_args(2, [_w(), _w()], [o, o], [1, 2], [1, 2])
    with pytest.raises(ValueError, match="at least one"):
        check_chain_args(0, [], [], [], [])
