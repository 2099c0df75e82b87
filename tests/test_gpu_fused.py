"""GPU: fp8_paged_decode_append_attention -- the append and the attention in
one launch. The pools must hold exactly the codes the oracle's append writes
(bit-exact, nothing else changed), and the output must match the oracle's
attention over positions + 1 keys of the updated cache."""

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from tests._common import assert_attention_close, np_

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F(cuda_device):
    import fp8_paged_decode_split_b200 as F
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)
    return F


@pytest.fixture(autouse=True, params=[1, 3], ids=["uniform", "proportional"])
def schedule(F, request):
    """The fused call runs the split kernel: uniform and proportional splits."""
    F.fp8pd_set_option(F.OPT_SCHEDULE, request.param)
    yield request.param
    F.fp8pd_set_option(F.OPT_SCHEDULE, 0)


@pytest.fixture(params=[(1, 1), (0, 0), (0, 1), (2, 1)], ids=["cvt", "bits", "kbits-vcvt", "mma8"])
def kdecode(F, request):
    F.fp8pd_set_option(F.OPT_K_DECODE, request.param[0])
    F.fp8pd_set_option(F.OPT_V_DECODE, request.param[1])
    yield request.param
    F.fp8pd_set_option(F.OPT_K_DECODE, 1)
    F.fp8pd_set_option(F.OPT_V_DECODE, 1)


def _fused_vs_oracle(F, case, li=0, positions=None, where=""):
    """Runs the fused call on layer li; checks the pools and the output
    against the oracle's append followed by its attention."""
    layer = case.layers[li]
    pos = case.positions if positions is None else positions
    kp0, vp0 = np_(layer.k_pages).copy(), np_(layer.v_pages).copy()
    out = F.fp8_paged_decode_append_attention(
        layer.q, layer.k_new, layer.v_new, layer.k_pages, layer.v_pages, layer.k_scale,
        layer.v_scale, layer.block_table, pos, window=layer.window, sinks=layer.sinks,
        sm_scale=layer.sm_scale)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0, where
    O.kv_append(np_(layer.k_new), np_(layer.v_new), kp0, vp0, np_(layer.k_scale),
                np_(layer.v_scale), np_(layer.block_table), np_(pos))
    assert np.array_equal(np_(layer.k_pages), kp0), f"{where}: K pool differs from the oracle"
    assert np.array_equal(np_(layer.v_pages), vp0), f"{where}: V pool differs from the oracle"
    want = O.paged_decode_attention(np_(layer.q), kp0, vp0, np_(layer.k_scale),
                                    np_(layer.v_scale), np_(layer.block_table),
                                    np_(pos).astype(np.int64) + 1, window=layer.window,
                                    sinks=np_(layer.sinks), sm_scale=layer.sm_scale)
    assert_attention_close(np_(out), want, where)
    return out


@pytest.mark.parametrize("nsplit", [0, 1, 3])
def test_llama_like_reduced(F, cuda_device, kdecode, nsplit):
    """GQA 32/8, D=128, per-(page, head) scales, several split counts."""
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, nsplit)
    try:
        case = W.make_case("llama", cuda_device, B=6, seq_len=(40, 700))
        _fused_vs_oracle(F, case, where=f"llama splits={nsplit}")
    finally:
        F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)


def test_positions_at_page_edges_and_empty_cache(F, cuda_device):
    """The new token as the first key of an empty cache, at the first and the
    last slot of a page, and mid-page; positions may also rewrite an earlier
    slot (the call appends at `positions` whatever the cache held there)."""
    case = W.make_case("llama", cuda_device, B=8, seq_len=(300, 400))
    pos = torch.tensor([0, 15, 16, 17, 31, 32, 200, 299], dtype=torch.int32, device=cuda_device)
    _fused_vs_oracle(F, case, positions=pos, where="page edges")


@pytest.mark.parametrize("name", ["gptoss_w128", "gptoss_full"])
def test_gptoss_like_sinks_and_window(F, cuda_device, kdecode, name):
    """D=64, G=8, sink logits; the 128-key window includes the new token."""
    case = W.make_case(name, cuda_device, B=3, seq_len=1000, append=True)
    _fused_vs_oracle(F, case, where=name)


def test_mixed_pool_head_dims_256_and_512(F, cuda_device):
    """Two layers sharing one pool of 65,536-byte pages: the sliding D=256
    layer and the full D=512 layer, per-(page, head) scales, N(0,2) values
    with outliers. Each layer appends into its own pages."""
    case = W.make_case("mixed", cuda_device, B=3, seq_len=(100, 3000), append=True)
    _fused_vs_oracle(F, case, li=0, where="mixed D=256")
    _fused_vs_oracle(F, case, li=1, where="mixed D=512")


def test_more_than_eight_query_heads_per_kv_head(F, cuda_device):
    """G = 16: two head groups attend the same tile; the first stores the new
    token, both use the codes they computed."""
    spec = W.Spec("g16", B=3, ps=16, layers=(W.LayerSpec(32, 2, 128, 0, None),),
                  seq_len=(50, 900), scale_mode="page", append=True, seed=11)
    _fused_vs_oracle(F, W.make_case(spec, cuda_device), where="G=16")


def test_long_sequence_many_splits(F, cuda_device):
    """20,000 keys in one sequence: many splits and the two-level merge."""
    case = W.make_case("long_b1", cuda_device, seq_len=20000)
    _fused_vs_oracle(F, case, where="long")


def test_same_bytes_as_append_then_attention(F, cuda_device):
    """For a fixed plan the fused call gives the same pools and the same
    output, bit for bit, as fp8_kv_append followed by the attention call."""
    a = W.make_case("llama", cuda_device, B=5, seq_len=(40, 900))
    b = W.make_case("llama", cuda_device, B=5, seq_len=(40, 900))
    la, lb = a.layers[0], b.layers[0]
    got = F.fp8_paged_decode_append_attention(
        la.q, la.k_new, la.v_new, la.k_pages, la.v_pages, la.k_scale, la.v_scale,
        la.block_table, a.positions, sm_scale=la.sm_scale)
    F.fp8_kv_append(lb.k_new, lb.v_new, lb.k_pages, lb.v_pages, lb.k_scale, lb.v_scale,
                    lb.block_table, b.positions)
    want = F.fp8_paged_decode_attention(lb.q, lb.k_pages, lb.v_pages, lb.k_scale, lb.v_scale,
                                        lb.block_table, b.attend_lens, sm_scale=lb.sm_scale)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    assert torch.equal(la.k_pages, lb.k_pages) and torch.equal(la.v_pages, lb.v_pages)
    assert torch.equal(got, want)


def test_out_of_range_position_is_flagged_and_not_written(F, cuda_device):
    case = W.make_case("llama", cuda_device, B=4, seq_len=(100, 200))
    layer = case.layers[0]
    lim = layer.block_table.shape[1] * case.spec.ps
    pos = case.positions.clone()
    pos[1] = lim            # one past the table
    pos[2] = -3
    kp0, vp0 = layer.k_pages.clone(), layer.v_pages.clone()
    out = F.fp8_paged_decode_append_attention(
        layer.q, layer.k_new, layer.v_new, layer.k_pages, layer.v_pages, layer.k_scale,
        layer.v_scale, layer.block_table, pos, sm_scale=layer.sm_scale)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() & F.FLAG_POS_OOB
    assert torch.all(out[1] == 0) and torch.all(out[2] == 0)
    # sequences 1 and 2 wrote nothing; 0 and 3 wrote only their new slots
    k_np, k0_np = np_(layer.k_pages), np_(kp0)
    O.kv_append(np_(layer.k_new)[[0, 3]], np_(layer.v_new)[[0, 3]], k0_np, np_(vp0),
                np_(layer.k_scale), np_(layer.v_scale), np_(layer.block_table)[[0, 3]],
                np_(pos)[[0, 3]])
    assert np.array_equal(k_np, k0_np)
