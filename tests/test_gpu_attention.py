"""GPU: fp8_paged_decode_attention against the float64 oracle.

Tolerance: max |got - ref| <= 1e-3 * max(1, |ref|) per output element. The
reduced workloads keep the shapes of the serving configurations but shorter
sequences, so the oracle computes every output; they still span several
16-token tiles, several pages and ragged last pages.
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
    """Every test runs with each schedule: uniform splits and proportional
    splits (no forced split count)."""
    F.fp8pd_set_option(F.OPT_SCHEDULE, request.param)
    yield request.param
    F.fp8pd_set_option(F.OPT_SCHEDULE, 0)


@pytest.fixture(params=[(1, 1), (0, 0), (2, 1)], ids=["cvt", "bits", "mma8"])
def kdecode(F, request):
    """Run a test with each E4M3 -> f16 decode of K and V (hardware cvt, bit
    assembly), and with K's E4M3 bytes in E4M3 MMAs (V by the cvt)."""
    F.fp8pd_set_option(F.OPT_K_DECODE, request.param[0])
    F.fp8pd_set_option(F.OPT_V_DECODE, request.param[1])
    yield request.param
    F.fp8pd_set_option(F.OPT_K_DECODE, 1)
    F.fp8pd_set_option(F.OPT_V_DECODE, 1)


@pytest.fixture(params=[(1, 0), (0, 1)], ids=["kcvt-vbits", "kbits-vcvt"])
def mixed_decode(F, request):
    F.fp8pd_set_option(F.OPT_K_DECODE, request.param[0])
    F.fp8pd_set_option(F.OPT_V_DECODE, request.param[1])
    yield request.param
    F.fp8pd_set_option(F.OPT_K_DECODE, 1)
    F.fp8pd_set_option(F.OPT_V_DECODE, 1)


@pytest.fixture
def splits(F):
    """Force a split count for one test; restore the planner afterwards."""
    def set_(n):
        F.fp8pd_set_option(F.OPT_NUM_SPLITS, n)
    yield set_
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)


def _check_layer(F, case, li=0, lens=None, where=""):
    layer = case.layers[li]
    lens = case.attend_lens if lens is None else lens
    got = gpu_attention(F, layer, lens)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0, where
    want = oracle_attention(layer, lens)
    return assert_attention_close(np_(got), want, where)


# --------------------------------------------------------------- workloads

def test_tiny_config_full_size(F, cuda_device, kdecode):
    case = W.make_case("tiny", cuda_device)
    _check_layer(F, case, where="tiny")


@pytest.mark.parametrize("nsplit", [0, 1, 3])
def test_llama_like_reduced_with_append(F, cuda_device, splits, nsplit):
    """GQA 32/8, D=128, per-(page, head) scales: append the new token, then
    attend over seq_len + 1 keys; the append is bit-exact, the output within
    tolerance."""
    import oracle as O
    splits(nsplit)
    case = W.make_case("llama", cuda_device, B=6, seq_len=(40, 700))
    layer = case.layers[0]
    kp0, vp0 = np_(layer.k_pages).copy(), np_(layer.v_pages).copy()
    F.fp8_kv_append(layer.k_new, layer.v_new, layer.k_pages, layer.v_pages, layer.k_scale,
                    layer.v_scale, layer.block_table, case.positions)
    O.kv_append(np_(layer.k_new), np_(layer.v_new), kp0, vp0, np_(layer.k_scale),
                np_(layer.v_scale), np_(layer.block_table), np_(case.positions))
    assert np.array_equal(np_(layer.k_pages), kp0) and np.array_equal(np_(layer.v_pages), vp0)
    _check_layer(F, case, where=f"llama splits={nsplit}")


@pytest.mark.parametrize("name", ["gptoss_w128", "gptoss_full"])
def test_gptoss_like_reduced_sinks(F, cuda_device, name, kdecode):
    case = W.make_case(name, cuda_device, B=3, seq_len=1000)
    _check_layer(F, case, where=name)


def test_mixed_pool_two_geometries(F, cuda_device, kdecode):
    """A sliding layer (D=256, window) and a full layer (D=512) read one pool
    with a 65,536-byte page stride; N(0,2) values with 1% x20 outliers."""
    case = W.make_case("mixed", cuda_device, B=3, seq_len=(300, 1500))
    object.__setattr__(case.layers[0], "window", 200)
    _check_layer(F, case, 0, where="mixed sliding")
    _check_layer(F, case, 1, where="mixed full")


@pytest.mark.parametrize("nsplit", [0, 7, 40])
def test_long_context_reduced_split(F, cuda_device, splits, nsplit):
    splits(nsplit)
    case = W.make_case("long_b1", cuda_device, seq_len=20000)
    _check_layer(F, case, where=f"long splits={nsplit}")
    if nsplit == 40:
        assert F.fp8pd_last_run_info()["combine"] == 1


def test_mixed_decodes(F, cuda_device, mixed_decode):
    case = W.make_case("llama", cuda_device, B=3, seq_len=(40, 400))
    _check_layer(F, case, where=f"decode {mixed_decode}")


@pytest.mark.parametrize("window", [0, 37])
def test_nan_codes_outside_the_attended_keys_are_ignored(F, cuda_device, kdecode, window):
    """Slots past the last key, and keys before the window, hold E4M3 NaN
    codes: they are never attended, so the output stays finite and equal to
    the oracle's (which never reads them)."""
    case = _small(cuda_device, sinks=True)
    layer = case.layers[0]
    lc = W.LayerCase(**{**layer.__dict__, "window": window})
    ps = layer.k_pages.shape[1]
    lens = case.attend_lens.cpu().numpy()
    tbl = layer.block_table.cpu().numpy()
    for b, L in enumerate(lens):
        last = tbl[b, (L - 1) // ps]
        s = L % ps
        if s:
            layer.k_pages[last, s:] = 0x7F
            layer.v_pages[last, s:] = 0xFF
        if window:
            lo = max(0, L - window)
            first = tbl[b, lo // ps]
            if lo % ps:
                layer.k_pages[first, : lo % ps] = 0xFF
                layer.v_pages[first, : lo % ps] = 0x7F
    _check_layer(F, W.Case(**{**case.__dict__, "layers": [lc]}), where=f"nan codes w={window}")


# --------------------------------------------------------------- shapes

@pytest.mark.parametrize("D", [64, 128, 256, 512])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 2), (12, 4), (16, 1), (24, 2)])
def test_head_dims_and_group_sizes(F, cuda_device, D, Hq, Hkv, kdecode):
    spec = W.Spec("shape", B=2, ps=16, layers=(W.LayerSpec(Hq, Hkv, D, 0, 0.7 / math.sqrt(D)),),
                  seq_len=(17, 161), scale_mode="page", sinks=True, seed=D + Hq)
    _check_layer(F, W.make_case(spec, cuda_device), where=f"D={D} Hq={Hq} Hkv={Hkv}")


@pytest.mark.parametrize("ps", [16, 32, 48, 64, 128, 256])
def test_page_sizes(F, cuda_device, ps):
    spec = W.Spec("ps", B=3, ps=ps, layers=(W.LayerSpec(16, 4, 128, 0, None),),
                  seq_len=(1, 600), scale_mode="head", seed=ps)
    _check_layer(F, W.make_case(spec, cuda_device), where=f"ps={ps}")


@pytest.mark.parametrize("window", [1, 2, 15, 16, 17, 100, 599, 600, 10 ** 6])
def test_windows(F, cuda_device, window):
    spec = W.Spec("win", B=3, ps=16, layers=(W.LayerSpec(8, 2, 64, window, 0.125),),
                  seq_len=(30, 600), scale_mode="page", sinks=True, seed=window % 97)
    _check_layer(F, W.make_case(spec, cuda_device), where=f"window={window}")


def test_the_requested_kernel_runs(F, cuda_device, schedule):
    case = W.make_case("llama", cuda_device, B=6, seq_len=(40, 700))
    _check_layer(F, case, where="llama")
    assert F.fp8pd_last_run_info()["schedule"] == schedule


def test_ragged_batch_with_empty_and_long_sequences(F, cuda_device, kdecode):
    """40 sequences from 0 to 3,000 keys, every seventh empty and one of a
    single key: proportional splits give the long ones many blocks and the
    empty ones none."""
    spec = W.Spec("ragged", B=40, ps=16, layers=(W.LayerSpec(32, 8, 128, 0, None),),
                  seq_len=(0, 3000), scale_mode="page", sinks=True, seed=77)
    case = W.make_case(spec, cuda_device)
    lens = case.attend_lens.clone()
    lens[::7] = 0
    lens[3] = min(1, int(lens[3]))
    _check_layer(F, case, lens=lens, where="ragged")


# --------------------------------------------------------------- edge cases

def _small(cuda_device, **kw):
    spec = W.Spec("edge", B=4, ps=16, layers=(W.LayerSpec(8, 2, 128, 0, 0.09),),
                  seq_len=(5, 300), scale_mode="page", sinks=kw.pop("sinks", False), seed=9)
    return W.make_case(W.spec_with(spec, **kw), cuda_device)


def test_empty_and_single_key_sequences(F, cuda_device):
    case = _small(cuda_device, sinks=True)
    lens = case.attend_lens.clone()
    lens[:3] = torch.tensor([0, 1, 2], dtype=torch.int32)
    _check_layer(F, case, lens=lens, where="empty/single")
    layer = case.layers[0]
    got = np_(gpu_attention(F, layer, lens))
    assert np.array_equal(got[0], np.zeros_like(got[0]))


def test_sink_minus_inf_equals_no_sink(F, cuda_device):
    case = _small(cuda_device, sinks=True)
    layer = case.layers[0]
    with_inf = gpu_attention(F, W.LayerCase(**{**layer.__dict__, "sinks": torch.full_like(layer.sinks, -math.inf)}),
                             case.attend_lens)
    without = gpu_attention(F, W.LayerCase(**{**layer.__dict__, "sinks": None}), case.attend_lens)
    assert torch.equal(with_inf, without)


def test_zero_query_gives_mean_of_values(F, cuda_device):
    case = _small(cuda_device)
    layer = case.layers[0]
    z = W.LayerCase(**{**layer.__dict__, "q": torch.zeros_like(layer.q)})
    got = np_(gpu_attention(F, z, case.attend_lens))
    want = oracle_attention(z, case.attend_lens)
    assert_attention_close(got, want, "q=0")


@pytest.mark.parametrize("qscale", [1e-6, 1e-3, 30.0, 3000.0])
def test_query_magnitudes(F, cuda_device, qscale, kdecode):
    case = _small(cuda_device)
    layer = case.layers[0]
    q = (layer.q.float() * qscale).to(torch.bfloat16)
    lc = W.LayerCase(**{**layer.__dict__, "q": q, "sm_scale": 0.09 / max(1.0, qscale / 30)})
    got = np_(gpu_attention(F, lc, case.attend_lens))
    assert_attention_close(got, oracle_attention(lc, case.attend_lens), f"qscale={qscale}")


def test_extreme_scales_and_subnormal_codes(F, cuda_device, kdecode):
    """Scales far from 1 and caches made of E4M3 subnormal codes only."""
    case = _small(cuda_device)
    layer = case.layers[0]
    g = torch.Generator(device=cuda_device).manual_seed(4)
    sub = torch.randint(0, 8, layer.k_pages.shape, generator=g, device=cuda_device, dtype=torch.uint8)
    sign = torch.randint(0, 2, layer.k_pages.shape, generator=g, device=cuda_device, dtype=torch.uint8) << 7
    layer.k_pages.copy_(sub | sign)
    layer.v_pages.copy_(torch.flip(sub | sign, dims=[0]))
    for ks, vs in ((1e4, 1e-4), (1e-3, 3e3)):
        lc = W.LayerCase(**{**layer.__dict__, "k_scale": layer.k_scale * ks, "v_scale": layer.v_scale * vs})
        got = np_(gpu_attention(F, lc, case.attend_lens))
        assert_attention_close(got, oracle_attention(lc, case.attend_lens), f"scales {ks},{vs}")


def test_strided_query_and_output(F, cuda_device):
    case = _small(cuda_device)
    layer = case.layers[0]
    qbig = torch.zeros(4, 8, 2, 128, dtype=torch.bfloat16, device=cuda_device)
    qbig[:, :, 1] = layer.q
    qv = qbig[:, :, 1]
    out_big = torch.full((4, 10, 132), 7.0, device=cuda_device)
    out = out_big[:, 1:9, :128]
    lc = W.LayerCase(**{**layer.__dict__, "q": qv})
    gpu_attention(F, lc, case.attend_lens, out=out)
    want = oracle_attention(layer, case.attend_lens)
    assert_attention_close(np_(out), want, "strided q/out")
    assert torch.all(out_big[:, 0] == 7.0) and torch.all(out_big[:, 9] == 7.0)
    assert torch.all(out_big[:, :, 128:] == 7.0)


# --------------------------------------------------------------- invariances

def test_page_placement_is_bit_exact_for_a_fixed_plan(F, cuda_device, splits):
    """The same logical cache on permuted vs identity page ids gives identical
    bits (a fixed split plan)."""
    splits(3)
    case = _small(cuda_device)
    layer = case.layers[0]
    lens = case.attend_lens
    a = gpu_attention(F, layer, lens).clone()
    # relocate every used page to a fresh pool in logical order
    tbl = layer.block_table
    B, mp = tbl.shape
    ids = tbl.clamp(min=0).reshape(-1)
    kp2 = layer.k_pages[ids].contiguous()
    vp2 = layer.v_pages[ids].contiguous()
    ks2 = layer.k_scale[ids].contiguous()
    vs2 = layer.v_scale[ids].contiguous()
    tbl2 = torch.arange(B * mp, dtype=torch.int32, device=cuda_device).reshape(B, mp)
    lc = W.LayerCase(**{**layer.__dict__, "k_pages": kp2, "v_pages": vp2, "k_scale": ks2,
                        "v_scale": vs2, "block_table": tbl2})
    b = gpu_attention(F, lc, lens)
    assert torch.equal(a, b)


def test_gqa_equals_repeated_kv_heads(F, cuda_device):
    case = _small(cuda_device)
    layer = case.layers[0]
    G = 4
    kp = layer.k_pages.repeat_interleave(G, dim=2).contiguous()
    vp = layer.v_pages.repeat_interleave(G, dim=2).contiguous()
    lc = W.LayerCase(**{**layer.__dict__, "k_pages": kp, "v_pages": vp,
                        "k_scale": layer.k_scale.repeat_interleave(G, dim=1),
                        "v_scale": layer.v_scale.repeat_interleave(G, dim=1)})
    a = np_(gpu_attention(F, layer, case.attend_lens))
    b = np_(gpu_attention(F, lc, case.attend_lens))
    assert_attention_close(a, b, "gqa vs repeated")


@pytest.mark.parametrize("nsplit", [1, 2, 5, 19])
def test_split_count_does_not_change_the_result(F, cuda_device, splits, nsplit):
    case = _small(cuda_device, sinks=True)
    splits(nsplit)
    _check_layer(F, case, where=f"splits={nsplit}")


# --------------------------------------------------------------- device errors

def test_bad_lengths_and_page_ids_are_flagged(F, cuda_device):
    case = _small(cuda_device)
    layer = case.layers[0]
    mp = layer.block_table.shape[1]
    lens = case.attend_lens.clone()
    lens[1] = mp * 16 + 1          # beyond the block table
    lens[2] = -3
    assert F.fp8pd_check_errors() == 0
    got = np_(gpu_attention(F, layer, lens))
    flags = F.fp8pd_check_errors()
    assert flags & F.FLAG_SEQLEN_OOB
    assert np.all(got[1] == 0) and np.all(got[2] == 0)
    want = oracle_attention(layer, case.attend_lens)
    assert_attention_close(got[[0, 3]], want[[0, 3]], "unaffected rows")
    tbl = layer.block_table.clone()
    tbl[3, 0] = layer.k_pages.shape[0] + 5
    lc = W.LayerCase(**{**layer.__dict__, "block_table": tbl})
    gpu_attention(F, lc, case.attend_lens)
    assert F.fp8pd_check_errors() & F.FLAG_PAGE_OOB
    assert F.fp8pd_check_errors() == 0


def test_workspace_reuse_across_call_shapes(F, cuda_device):
    """Split calls of different shapes share the device's workspace: a call
    with few ticket counters and a later one with more must both be right
    (the later call's counters must not sit where the earlier call wrote its
    split partials)."""
    small = W.Spec("few-units", B=3, ps=16, layers=(W.LayerSpec(16, 4, 128, 0, None),),
                   seq_len=(300, 600), scale_mode="head", seed=16)
    for spec in (small, W.spec_with("llama", B=6, seq_len=(40, 700)), small,
                 W.spec_with("long_b1", seq_len=20000), W.spec_with("llama", B=6, seq_len=(40, 700))):
        case = W.make_case(spec, cuda_device)
        assert F.fp8pd_plan(case.layers[0].q, case.layers[0].k_pages, case.layers[0].block_table,
                            case.layers[0].window)["combine"] == 1
        _check_layer(F, case, where=spec.name)


# --------------------------------------------------------------- graphs

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
    want = oracle_attention(layer, case.attend_lens)
    assert_attention_close(np_(out), want, "graph replay")
