"""GPU: context-parallel split-KV on one GPU, the ranks run in turn.

Each "rank" attends its key slice of every sequence with
fp8_paged_decode_attention_partial, the slices' partials are stacked in rank
order (what the all-gather returns) and fp8pd_combine_partials merges them;
the result is the decode attention over all keys, checked against the
oracle. The slices either read one shared pool or each rank's own pool (its
pages only, the rest of its block table unused), as separate GPUs would.
Kernels that wait on one another never run here: the ranks' launches are
independent.
"""

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from fp8_paged_decode_split_b200.context_parallel import attention as cp_attention, key_slices
from tests._common import ATOL_REL, assert_attention_close, np_, oracle_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F(cuda_device):
    import fp8_paged_decode_split_b200 as F
    return F


@pytest.fixture(autouse=True, params=[1, 3], ids=["uniform", "proportional"])
def schedule(F, request):
    F.fp8pd_set_option(F.OPT_SCHEDULE, request.param)
    yield
    F.fp8pd_set_option(F.OPT_SCHEDULE, 0)


def _ranks_partials(F, layer, lens, slices, pools=None):
    outs_o, outs_ml = [], []
    for r in range(slices.shape[0]):
        kp, vp, ks, vs, tbl = pools[r] if pools else (layer.k_pages, layer.v_pages, layer.k_scale,
                                                       layer.v_scale, layer.block_table)
        kr = torch.as_tensor(slices[r], device=layer.q.device)
        o, ml = F.fp8_paged_decode_attention_partial(layer.q, kp, vp, ks, vs, tbl, lens, kr,
                                                     window=layer.window, sm_scale=layer.sm_scale)
        outs_o.append(o)
        outs_ml.append(ml)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    return torch.stack(outs_o), torch.stack(outs_ml)


@pytest.mark.parametrize("name,overrides,world", [
    ("long_b1", dict(seq_len=20000), 2),
    ("long_b1", dict(seq_len=20000), 8),
    ("llama", dict(B=6, seq_len=(40, 3000)), 3),
    ("gptoss_full", dict(B=3, seq_len=3000), 4),       # sinks, added once by the combine
    ("gptoss_w128", dict(B=3, seq_len=3000), 4),       # window: most slices empty
    ("mixed", dict(B=3, seq_len=(500, 4000)), 2),
])
def test_slices_combined_equal_the_full_attention(F, cuda_device, name, overrides, world):
    case = W.make_case(name, cuda_device, **overrides)
    lens = case.attend_lens
    slices = key_slices(lens.cpu().numpy(), case.spec.ps, world)
    for li, layer in enumerate(case.layers):
        all_o, all_ml = _ranks_partials(F, layer, lens, slices)
        out = F.fp8pd_combine_partials(all_o, all_ml, sinks=layer.sinks)
        torch.cuda.synchronize()
        assert_attention_close(np_(out), oracle_attention(layer, lens), f"{name}[{li}] x{world}")


def test_partials_match_the_oracle_partials(F, cuda_device):
    """The partial of each slice itself: normalized numerator o / l within
    the attention tolerance, l and m (log2 units) within f32 rounding of the
    oracle's; empty slices give (-inf, 0)."""
    case = W.make_case("llama", cuda_device, B=5, seq_len=(40, 2000))
    layer = case.layers[0]
    lens = case.attend_lens
    slices = key_slices(lens.cpu().numpy(), case.spec.ps, 4)
    slices[1, 0] = (0, 0)                                   # one empty slice
    all_o, all_ml = _ranks_partials(F, layer, lens, slices)
    for r in range(4):
        o, ml = O.paged_decode_partial(np_(layer.q), np_(layer.k_pages), np_(layer.v_pages),
                                       np_(layer.k_scale), np_(layer.v_scale),
                                       np_(layer.block_table), np_(lens), slices[r],
                                       sm_scale=layer.sm_scale)
        g_o, g_ml = np_(all_o[r]), np_(all_ml[r])
        empty = ml[:, :, 0] == -np.inf
        assert np.array_equal(g_ml[empty][:, 0], ml[empty][:, 0])
        assert np.all(g_ml[empty][:, 1] == 0)
        ne = ~empty
        assert np.allclose(g_ml[ne][:, 0], ml[ne][:, 0], rtol=1e-5, atol=1e-4)
        # numerators and sums are relative to each side's own maximum
        shift = np.exp2(g_ml[:, :, 0] - np.where(empty, 0, ml[:, :, 0]))
        l_g = np.where(ne, g_ml[:, :, 1] * shift, 0)
        assert np.allclose(l_g[ne], ml[:, :, 1][ne], rtol=1e-3)
        norm_g = g_o[ne] / g_ml[ne][:, 1:2]
        norm_w = o[ne] / ml[ne][:, 1:2]
        err = np.abs(norm_g - norm_w) / np.maximum(1.0, np.abs(norm_w))
        assert err.max() <= ATOL_REL


def _rank_pool(layer, lens, kr, ps):
    """Rank r's own pool: only the pages its slice touches, renumbered, and a
    block table that marks every other logical page unused (-1)."""
    tbl = layer.block_table.cpu().numpy()
    own = np.full_like(tbl, -1)
    ids = []
    for b in range(tbl.shape[0]):
        s, e = int(kr[b][0]), int(kr[b][1])
        if e <= s:
            continue
        for lp in range(s // ps, (e - 1) // ps + 1):
            own[b, lp] = len(ids)
            ids.append(int(tbl[b, lp]))
    idx = torch.as_tensor(ids if ids else [0], device=layer.q.device)
    per_page = lambda sc: sc[idx] if sc.dim() >= 2 else sc  # noqa: E731
    return (layer.k_pages[idx].contiguous(), layer.v_pages[idx].contiguous(),
            per_page(layer.k_scale), per_page(layer.v_scale),
            torch.as_tensor(own, device=layer.q.device))


@pytest.mark.parametrize("world", [2, 4])
def test_each_rank_holds_only_its_pages(F, cuda_device, world):
    case = W.make_case("llama", cuda_device, B=4, seq_len=(500, 3000))
    layer = case.layers[0]
    lens = case.attend_lens
    slices = key_slices(lens.cpu().numpy(), case.spec.ps, world)
    pools = [_rank_pool(layer, lens, slices[r], case.spec.ps) for r in range(world)]
    all_o, all_ml = _ranks_partials(F, layer, lens, slices, pools)
    out = F.fp8pd_combine_partials(all_o, all_ml, sinks=None)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    assert_attention_close(np_(out), oracle_attention(layer, lens), f"own pools x{world}")


def test_single_rank_helper_equals_plain_attention(F, cuda_device):
    """context_parallel.attention without a process group: one slice (all
    keys), its partial and the combine: the plain decode attention."""
    case = W.make_case("gptoss_full", cuda_device, B=2, seq_len=2000)
    layer = case.layers[0]
    lens = case.attend_lens
    kr = torch.as_tensor(key_slices(lens.cpu().numpy(), case.spec.ps, 1)[0], device=cuda_device)
    out = cp_attention(layer.q, layer.k_pages, layer.v_pages, layer.k_scale, layer.v_scale,
                       layer.block_table, lens, kr, window=layer.window, sinks=layer.sinks,
                       sm_scale=layer.sm_scale)
    torch.cuda.synchronize()
    assert_attention_close(np_(out), oracle_attention(layer, lens), "single rank")


def test_combine_refuses_bad_arguments(F, cuda_device):
    o = torch.zeros(2, 1, 4, 64, device=cuda_device)
    ml = torch.zeros(2, 1, 4, 2, device=cuda_device)
    with pytest.raises(F.Fp8pdError) as e:
        F.fp8pd_combine_partials(o, ml[:, :, :3])
    assert e.value.status == -3
    with pytest.raises(F.Fp8pdError) as e:
        F.fp8pd_combine_partials(o[:, :, :, :62], ml)
    assert e.value.status in (-4, -5)
