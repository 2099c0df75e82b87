"""GPU: the tensor-memory kernel (tcgen05 MMAs, TMEM accumulators,
FP8PD_OPT_KERNEL = 2) against the float64 oracle.

Every test asks for the tensor-memory kernel and checks that it ran
(fp8pd_last_run_info()["kernel"] == 2) wherever it applies: head dim 64 or
128, page or head scales, f32 compute. The tolerance is the same as the split
kernel's: max |got - ref| <= 1e-3 * max(1, |ref|) per output element; the
append is bit-exact.
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
    F.fp8pd_set_option(F.OPT_KERNEL, 2)
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)
    yield F
    F.fp8pd_set_option(F.OPT_KERNEL, 0)


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


def _check(F, layer, lens, where, kernel=2):
    got = gpu_attention(F, layer, lens)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0, where
    assert F.fp8pd_last_run_info()["kernel"] == kernel, where
    return assert_attention_close(np_(got), oracle_attention(layer, lens), where)


def test_tiny_config_full_size(F, cuda_device):
    case = W.make_case("tiny", cuda_device)
    _check(F, case.layers[0], case.attend_lens, "tiny")


@pytest.mark.parametrize("nsplit", [0, 1, 3])
def test_llama_like_reduced(F, cuda_device, splits, nsplit):
    splits(nsplit)
    case = W.make_case("llama", cuda_device, B=6, seq_len=(40, 700))
    _check(F, case.layers[0], case.attend_lens, f"llama splits={nsplit}")


@pytest.mark.parametrize("name", ["gptoss_w128", "gptoss_full"])
def test_gptoss_like_reduced_sinks(F, cuda_device, name):
    case = W.make_case(name, cuda_device, B=3, seq_len=1000)
    _check(F, case.layers[0], case.attend_lens, name)


@pytest.mark.parametrize("nsplit", [0, 7, 40])
def test_long_context_reduced_split(F, cuda_device, splits, nsplit):
    splits(nsplit)
    case = W.make_case("long_b1", cuda_device, seq_len=20000)
    _check(F, case.layers[0], case.attend_lens, f"long splits={nsplit}")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 2), (12, 4), (16, 1), (24, 2)])
def test_head_dims_and_group_sizes(F, cuda_device, D, Hq, Hkv):
    spec = W.Spec("shape", B=2, ps=16, layers=(W.LayerSpec(Hq, Hkv, D, 0, 0.7 / math.sqrt(D)),),
                  seq_len=(17, 161), scale_mode="page", sinks=True, seed=D + Hq)
    case = W.make_case(spec, cuda_device)
    _check(F, case.layers[0], case.attend_lens, f"D={D} Hq={Hq} Hkv={Hkv}")


@pytest.mark.parametrize("ps", [16, 32, 64, 128, 256])
def test_page_sizes(F, cuda_device, ps):
    spec = W.Spec("ps", B=3, ps=ps, layers=(W.LayerSpec(16, 4, 128, 0, None),),
                  seq_len=(1, 600), scale_mode="head", seed=ps)
    case = W.make_case(spec, cuda_device)
    _check(F, case.layers[0], case.attend_lens, f"ps={ps}")


@pytest.mark.parametrize("window", [1, 2, 15, 16, 17, 100, 127, 128, 129, 599, 10 ** 6])
def test_windows(F, cuda_device, window):
    spec = W.Spec("win", B=3, ps=16, layers=(W.LayerSpec(8, 2, 64, window, 0.125),),
                  seq_len=(30, 600), scale_mode="page", sinks=True, seed=window % 97)
    case = W.make_case(spec, cuda_device)
    _check(F, case.layers[0], case.attend_lens, f"window={window}")


def test_ragged_batch_with_empty_and_long_sequences(F, cuda_device):
    spec = W.Spec("ragged", B=40, ps=16, layers=(W.LayerSpec(32, 8, 128, 0, None),),
                  seq_len=(0, 3000), scale_mode="page", sinks=True, seed=77)
    case = W.make_case(spec, cuda_device)
    lens = case.attend_lens.clone()
    lens[::7] = 0
    lens[3] = min(1, int(lens[3]))
    _check(F, case.layers[0], lens, "ragged")
    got = np_(gpu_attention(F, case.layers[0], lens))
    assert np.array_equal(got[0], np.zeros_like(got[0]))  # an empty sequence gives 0


def test_nan_codes_outside_the_attended_keys_are_ignored(F, cuda_device):
    """Slots past the last key hold E4M3 NaN codes: never attended, the output
    stays finite and equal to the oracle's."""
    spec = W.Spec("edge", B=4, ps=16, layers=(W.LayerSpec(8, 2, 128, 0, 0.09),),
                  seq_len=(5, 300), scale_mode="page", sinks=True, seed=9)
    case = W.make_case(spec, cuda_device)
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


@pytest.mark.parametrize("qscale", [1e-6, 1e-3, 30.0, 3000.0])
def test_query_magnitudes(F, cuda_device, qscale):
    spec = W.Spec("edge", B=4, ps=16, layers=(W.LayerSpec(8, 2, 128, 0, 0.09),),
                  seq_len=(5, 300), scale_mode="page", seed=9)
    case = W.make_case(spec, cuda_device)
    layer = case.layers[0]
    q = (layer.q.float() * qscale).to(torch.bfloat16)
    lc = W.LayerCase(**{**layer.__dict__, "q": q, "sm_scale": 0.09 / max(1.0, qscale / 30)})
    _check(F, lc, case.attend_lens, f"qscale={qscale}")


@pytest.mark.parametrize("nsplit", [1, 2, 5, 19])
def test_split_count_does_not_change_the_result(F, cuda_device, splits, nsplit):
    splits(nsplit)
    case = W.make_case("long_b1", cuda_device, seq_len=5000)
    _check(F, case.layers[0], case.attend_lens, f"splits={nsplit}")


def test_fused_append_matches_append_then_attention(F, cuda_device):
    """The fused call stores the same E4M3 bytes as fp8_kv_append (bit-exact)
    and attends over position + 1 keys within the tolerance."""
    case = W.make_case("llama", cuda_device, B=5, seq_len=(20, 900))
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
    assert F.fp8pd_last_run_info()["kernel"] == 2
    assert torch.equal(layer.k_pages, kp) and torch.equal(layer.v_pages, vp)
    assert_attention_close(np_(out), oracle_attention(layer, case.positions + 1), "fused")


def test_partial_slices_combine_to_the_full_attention(F, cuda_device):
    """Context-parallel slices through the partial entry point, merged by the
    combine kernel, equal the oracle's full attention."""
    from fp8_paged_decode_split_b200 import context_parallel as CP
    case = W.make_case("long_b1", cuda_device, seq_len=6000)
    layer = case.layers[0]
    lens = case.attend_lens
    slices = CP.key_slices(lens.cpu().numpy(), layer.k_pages.shape[1], 3)
    outs_o, outs_ml = [], []
    for r in range(3):
        kr = torch.from_numpy(slices[r]).to(cuda_device)
        o, ml = F.fp8_paged_decode_attention_partial(
            layer.q, layer.k_pages, layer.v_pages, layer.k_scale, layer.v_scale,
            layer.block_table, lens, kr, window=layer.window, sm_scale=layer.sm_scale)
        assert F.fp8pd_last_run_info()["kernel"] == 2
        outs_o.append(o)
        outs_ml.append(ml)
    out = F.fp8pd_combine_partials(torch.stack(outs_o), torch.stack(outs_ml), sinks=layer.sinks)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    assert_attention_close(np_(out), oracle_attention(layer, lens), "slices")


def test_cuda_graph_capture_and_replay(F, cuda_device, splits):
    splits(4)
    case = W.make_case("long_b1", cuda_device, seq_len=5000)
    layer = case.layers[0]
    plan = F.fp8pd_plan(layer.q, layer.k_pages, layer.block_table, layer.window)
    F.fp8pd_reserve_workspace(plan["workspace_bytes"])
    out = torch.empty(layer.q.shape, dtype=torch.float32, device=cuda_device)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        gpu_attention(F, layer, case.attend_lens, out=out)   # warm up on the side stream
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        gpu_attention(F, layer, case.attend_lens, out=out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    assert_attention_close(np_(out), oracle_attention(layer, case.attend_lens), "graph replay")


def test_modes_it_does_not_take_run_the_split_kernel(F, cuda_device):
    """Per-token scales and head dims 256 / 512 run the split kernel even with
    the tensor-memory kernel asked for."""
    spec = W.Spec("tok", B=3, ps=16, layers=(W.LayerSpec(8, 2, 128, 0, None),),
                  seq_len=(10, 300), scale_mode="token", seed=3)
    case = W.make_case(spec, cuda_device)
    _check(F, case.layers[0], case.attend_lens, "per-token scales", kernel=1)
    spec = W.Spec("d256", B=2, ps=16, layers=(W.LayerSpec(8, 2, 256, 0, None),),
                  seq_len=(10, 300), scale_mode="page", seed=4)
    case = W.make_case(spec, cuda_device)
    _check(F, case.layers[0], case.attend_lens, "D=256", kernel=1)
