"""GPU: the split kernel's head-dim split at D = 512 against the float64 oracle.

At head dim 512 with page or head scales, f32 compute and the hardware-cvt
decodes (and no fused append), each tile stream of a block is run by two or
four warps (a build setting): each copies and contracts its part of the head
dim, and the parts of the scores are summed in shared memory once per tile.
Every test checks that this path ran (fp8pd_last_run_info()["dim_split"] > 1)
or, for the modes it does not take, that the whole-width kernel did (== 1).
Tolerance as everywhere: max |got - ref| <= 1e-3 * max(1, |ref|) per output
element.
"""

import math

import numpy as np
import pytest
import torch

import workloads as W
from tests._common import assert_attention_close, gpu_attention, np_, oracle_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F(cuda_device):
    import fp8_paged_decode_split_b200 as F
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)
    return F


@pytest.fixture(autouse=True, params=[1, 3], ids=["split", "proportional"])
def schedule(F, request):
    F.fp8pd_set_option(F.OPT_SCHEDULE, request.param)
    yield request.param
    F.fp8pd_set_option(F.OPT_SCHEDULE, 0)


@pytest.fixture
def splits(F):
    def set_(n):
        F.fp8pd_set_option(F.OPT_NUM_SPLITS, n)
    yield set_
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)


def _spec(name, B=3, Hq=16, Hkv=2, window=0, seq_len=(17, 900), scale_mode="page", sinks=True,
          seed=5, ps=32):
    return W.Spec(name, B=B, ps=ps, layers=(W.LayerSpec(Hq, Hkv, 512, window, 1 / 128),),
                  seq_len=seq_len, scale_mode=scale_mode, sinks=sinks, dist="normal2_outliers",
                  seed=seed)


def _check(F, layer, lens, where, split=True):
    got = gpu_attention(F, layer, lens)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0, where
    run = F.fp8pd_last_run_info()
    assert run["kernel"] == 1, (where, run)
    assert (run["dim_split"] in (2, 4)) if split else run["dim_split"] == 1, (where, run)
    return assert_attention_close(np_(got), oracle_attention(layer, lens), where)


def test_mixed_pool_full_layer_reduced(F, cuda_device):
    """The mixed pool's D = 512 layer (B = 3, 300 to 1,500 keys), which reads
    the pool shared with the D = 256 layer."""
    case = W.make_case("mixed", cuda_device, B=3, seq_len=(300, 1500))
    _check(F, case.layers[1], case.attend_lens, "mixed full layer")


@pytest.mark.parametrize("scale_mode", ["page", "head"])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 1), (16, 2), (24, 2), (12, 4)])
def test_group_sizes_and_scale_forms(F, cuda_device, Hq, Hkv, scale_mode):
    spec = _spec("gs", B=2, Hq=Hq, Hkv=Hkv, seq_len=(17, 400), scale_mode=scale_mode,
                 seed=Hq + Hkv)
    case = W.make_case(spec, cuda_device)
    _check(F, case.layers[0], case.attend_lens, f"Hq={Hq} Hkv={Hkv} {scale_mode}")


@pytest.mark.parametrize("ps", [16, 32, 64, 256])
def test_page_sizes(F, cuda_device, ps):
    case = W.make_case(_spec("ps", ps=ps, seq_len=(1, 700), seed=ps), cuda_device)
    _check(F, case.layers[0], case.attend_lens, f"ps={ps}")


@pytest.mark.parametrize("window", [1, 2, 15, 16, 17, 100, 600, 10 ** 6])
def test_windows(F, cuda_device, window):
    case = W.make_case(_spec("win", window=window, seq_len=(30, 700), seed=window % 89),
                       cuda_device)
    _check(F, case.layers[0], case.attend_lens, f"window={window}")


@pytest.mark.parametrize("nsplit", [1, 2, 5, 19])
def test_split_counts(F, cuda_device, splits, nsplit):
    splits(nsplit)
    case = W.make_case(_spec("sp", B=2, seq_len=(2000, 5000), seed=nsplit), cuda_device)
    _check(F, case.layers[0], case.attend_lens, f"splits={nsplit}")


def test_ragged_batch_with_empty_and_single_key_sequences(F, cuda_device):
    case = W.make_case(_spec("ragged", B=24, seq_len=(0, 2500), seed=77), cuda_device)
    lens = case.attend_lens.clone()
    lens[::5] = 0
    lens[3] = min(1, int(lens[3]))
    _check(F, case.layers[0], lens, "ragged")
    got = np_(gpu_attention(F, case.layers[0], lens))
    assert np.array_equal(got[0], np.zeros_like(got[0]))  # an empty sequence gives 0


def test_nan_codes_outside_the_attended_keys_are_ignored(F, cuda_device):
    case = W.make_case(_spec("nan", B=4, seq_len=(5, 300), ps=16, seed=9), cuda_device)
    layer = case.layers[0]
    ps = layer.k_pages.shape[1]
    lens = case.attend_lens.cpu().numpy()
    tbl = layer.block_table.cpu().numpy()
    for b, L in enumerate(lens):
        s = L % ps
        if s:
            layer.k_pages[tbl[b, (L - 1) // ps], s:] = 0x7F
            layer.v_pages[tbl[b, (L - 1) // ps], s:] = 0xFF
    _check(F, layer, case.attend_lens, "nan codes")


@pytest.mark.parametrize("qscale", [1e-6, 30.0, 3000.0])
def test_query_magnitudes(F, cuda_device, qscale):
    case = W.make_case(_spec("q", B=3, seq_len=(5, 300), sinks=False, seed=4), cuda_device)
    layer = case.layers[0]
    q = (layer.q.float() * qscale).to(torch.bfloat16)
    lc = W.LayerCase(**{**layer.__dict__, "q": q, "sm_scale": (1 / 128) / max(1.0, qscale / 30)})
    _check(F, lc, case.attend_lens, f"qscale={qscale}")


def test_partial_slices_combine_to_the_full_attention(F, cuda_device):
    from fp8_paged_decode_split_b200 import context_parallel as CP
    case = W.make_case(_spec("cp", B=2, seq_len=(1500, 4000), seed=21), cuda_device)
    layer = case.layers[0]
    lens = case.attend_lens
    slices = CP.key_slices(lens.cpu().numpy(), layer.k_pages.shape[1], 3)
    outs_o, outs_ml = [], []
    for r in range(3):
        kr = torch.from_numpy(slices[r]).to(cuda_device)
        o, ml = F.fp8_paged_decode_attention_partial(
            layer.q, layer.k_pages, layer.v_pages, layer.k_scale, layer.v_scale,
            layer.block_table, lens, kr, window=layer.window, sm_scale=layer.sm_scale)
        assert F.fp8pd_last_run_info()["dim_split"] in (2, 4)
        outs_o.append(o)
        outs_ml.append(ml)
    out = F.fp8pd_combine_partials(torch.stack(outs_o), torch.stack(outs_ml), sinks=layer.sinks)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    assert_attention_close(np_(out), oracle_attention(layer, lens), "slices")


def test_cuda_graph_capture_and_replay(F, cuda_device, splits):
    splits(3)
    case = W.make_case(_spec("graph", B=2, seq_len=(1000, 3000), seed=13), cuda_device)
    layer = case.layers[0]
    plan = F.fp8pd_plan(layer.q, layer.k_pages, layer.block_table, layer.window)
    gpu_attention(F, layer, case.attend_lens)
    ds = F.fp8pd_last_run_info()["dim_split"]
    # warps per block: tile streams (at least 4) x the warps of each stream
    wpb, rem = divmod(plan["warps"], plan["grid_blocks"])
    assert ds in (2, 4) and rem == 0 and wpb % ds == 0 and wpb >= 4 * ds
    F.fp8pd_reserve_workspace(plan["workspace_bytes"])
    out = torch.empty(layer.q.shape, dtype=torch.float32, device=cuda_device)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        gpu_attention(F, layer, case.attend_lens, out=out)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        gpu_attention(F, layer, case.attend_lens, out=out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    assert_attention_close(np_(out), oracle_attention(layer, case.attend_lens), "graph replay")


def test_no_alloc_entry_point(F, cuda_device):
    case = W.make_case(_spec("na", B=3, seq_len=(200, 2000), seed=31), cuda_device)
    layer = case.layers[0]
    out = torch.empty(layer.q.shape, dtype=torch.float32, device=cuda_device)
    F.fp8_paged_decode_attention_noalloc(
        layer.q, layer.k_pages, layer.v_pages, layer.k_scale, layer.v_scale, layer.block_table,
        case.attend_lens, window=layer.window, sinks=layer.sinks, sm_scale=layer.sm_scale, out=out)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    assert F.fp8pd_last_run_info()["dim_split"] in (2, 4)
    assert_attention_close(np_(out), oracle_attention(layer, case.attend_lens), "no-alloc")


def test_modes_it_does_not_take_run_whole_width(F, cuda_device):
    """Per-token scales, K as E4M3 MMAs, the bit-assembly decode and the fp8
    compute path run the whole-width kernel at D = 512."""
    case = W.make_case(_spec("tok", B=2, seq_len=(10, 300), scale_mode="token", seed=3),
                       cuda_device)
    _check(F, case.layers[0], case.attend_lens, "per-token scales", split=False)
    case = W.make_case(_spec("pg", B=2, seq_len=(10, 300), seed=4), cuda_device)
    for opt, val in ((F.OPT_K_DECODE, 2), (F.OPT_K_DECODE, 0), (F.OPT_V_DECODE, 0)):
        F.fp8pd_set_option(opt, val)
        try:
            _check(F, case.layers[0], case.attend_lens, f"option {opt}={val}", split=False)
        finally:
            F.fp8pd_set_option(opt, 1)
    F.fp8pd_set_option(F.OPT_COMPUTE, 1)
    try:
        gpu_attention(F, case.layers[0], case.attend_lens)
        torch.cuda.synchronize()
        assert F.fp8pd_check_errors() == 0
        assert F.fp8pd_last_run_info()["dim_split"] == 1
    finally:
        F.fp8pd_set_option(F.OPT_COMPUTE, 0)


def test_fused_append_runs_whole_width(F, cuda_device):
    """The fused append-attention call at D = 512 stores the same bytes as
    fp8_kv_append and attends over position + 1 keys, on the whole-width
    kernel."""
    spec = W.Spec("app", B=3, ps=32, layers=(W.LayerSpec(16, 2, 512, 0, 1 / 128),),
                  seq_len=(20, 900), scale_mode="page", sinks=True, append=True, seed=8)
    case = W.make_case(spec, cuda_device)
    layer = case.layers[0]
    kp, vp = layer.k_pages.clone(), layer.v_pages.clone()
    F.fp8_kv_append(layer.k_new, layer.v_new, kp, vp, layer.k_scale, layer.v_scale,
                    layer.block_table, case.positions)
    out = F.fp8_paged_decode_append_attention(
        layer.q, layer.k_new, layer.v_new, layer.k_pages, layer.v_pages, layer.k_scale,
        layer.v_scale, layer.block_table, case.positions, window=layer.window,
        sinks=layer.sinks, sm_scale=layer.sm_scale)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    assert F.fp8pd_last_run_info()["dim_split"] == 1
    assert torch.equal(layer.k_pages, kp) and torch.equal(layer.v_pages, vp)
    assert_attention_close(np_(out), oracle_attention(layer, case.positions + 1), "fused")
