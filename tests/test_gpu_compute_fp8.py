"""GPU: the opt-in fp8 compute path (FP8PD_OPT_COMPUTE = 1) against the oracle.

The solution page's "Two compute paths" table gives the fp8 path (one E4M3
rounding on q and on p, E4M3 dot products) a tolerance of 1.5e-1; its
"Limitations" say why it is wider. Each case is checked against the oracle's
own fp8 variant and against the f32 oracle, both within
1.5e-1 * max(1, |ref|) per element. Where nothing rounds (q = 0: every weight
is exactly 1, and E4M3 values are exact in every operand) the path is held to
the f32 tolerance 1e-3, which pins the byte layout of its V and P operands.
"""

import dataclasses

import numpy as np
import pytest
import torch

import workloads as W
from tests._common import ATOL_REL, assert_attention_close, gpu_attention, np_, oracle_attention

pytestmark = pytest.mark.gpu

FP8_TOL = 1.5e-1


@pytest.fixture(scope="module")
def F(cuda_device):
    import fp8_paged_decode_split_b200 as F
    return F


@pytest.fixture(autouse=True, params=[1, 3], ids=["uniform", "proportional"])
def fp8_mode(F, request):
    F.fp8pd_set_option(F.OPT_COMPUTE, 1)
    F.fp8pd_set_option(F.OPT_SCHEDULE, request.param)
    yield
    F.fp8pd_set_option(F.OPT_COMPUTE, 0)
    F.fp8pd_set_option(F.OPT_SCHEDULE, 0)


def _close(got, want, tol, where):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - want) / np.maximum(1.0, np.abs(want))
    assert np.all(np.isfinite(got)), where
    assert err.max() <= tol, f"{where}: max scaled error {err.max():.3e} > {tol}"
    return float(err.max())


def _check(F, layer, lens, where):
    got = np_(gpu_attention(F, layer, lens))
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0, where
    assert F.fp8pd_last_run_info()["compute"] == 1
    e8 = _close(got, oracle_attention(layer, lens, compute="fp8"), FP8_TOL, where + " vs fp8 oracle")
    e32 = _close(got, oracle_attention(layer, lens), FP8_TOL, where + " vs f32 oracle")
    return e8, e32


@pytest.mark.parametrize("name,overrides", [
    ("tiny", {}),
    ("llama", dict(B=5, seq_len=(40, 700))),
    ("gptoss_w128", dict(B=3, seq_len=1000)),
    ("gptoss_full", dict(B=2, seq_len=1500)),
    ("mixed", dict(B=3, seq_len=(300, 2500))),
    ("long_b1", dict(seq_len=6000)),
])
def test_fp8_compute_on_the_serving_shapes(F, cuda_device, name, overrides):
    case = W.make_case(name, cuda_device, **overrides)
    for li, layer in enumerate(case.layers):
        _check(F, layer, case.attend_lens, f"{name}[{li}]")


@pytest.mark.parametrize("D", [64, 128, 256, 512])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 2), (16, 1)])
def test_fp8_compute_head_dims_and_groups(F, cuda_device, D, Hq, Hkv):
    spec = W.Spec("f8shape", B=2, ps=16, layers=(W.LayerSpec(Hq, Hkv, D, 0, D ** -0.5),),
                  seq_len=(17, 300), scale_mode="page", sinks=True, seed=D + Hq)
    case = W.make_case(spec, cuda_device)
    _check(F, case.layers[0], case.attend_lens, f"D={D} Hq={Hq} Hkv={Hkv}")


@pytest.mark.parametrize("D", [64, 128, 512])
def test_fp8_compute_zero_query_is_exact(F, cuda_device, D):
    """q = 0 with one V scale per KV head: every score is 0, every weight
    exactly 1, so the rounded operand (weight * v_scale / max v_scale * 2^8 =
    2^8) is exact, and V enters the MMA as its own bytes: the only rounding
    left is the f32 accumulation, so the f32 tolerance holds. A wrong token or
    entry in the V and P operands would fail it. (With per-page V scales the
    rounded operand carries the page's scale ratio, so it is not exact.)"""
    spec = W.Spec("f8zero", B=3, ps=16, layers=(W.LayerSpec(16, 2, D, 0, D ** -0.5),),
                  seq_len=(1, 400), scale_mode="head", seed=D)
    case = W.make_case(spec, cuda_device)
    layer = dataclasses.replace(case.layers[0], q=torch.zeros_like(case.layers[0].q))
    got = np_(gpu_attention(F, layer, case.attend_lens))
    torch.cuda.synchronize()
    assert_attention_close(got, oracle_attention(layer, case.attend_lens), f"q=0 D={D}")
    assert ATOL_REL == 1e-3


@pytest.mark.parametrize("window", [0, 37])
def test_fp8_compute_ignores_nan_codes_outside_the_keys(F, cuda_device, window):
    """Masked slots hold E4M3 NaN codes; the fp8 path zeroes their V bytes
    before the MMA (a NaN times a zero weight is still NaN)."""
    spec = W.Spec("f8nan", B=4, ps=16, layers=(W.LayerSpec(8, 2, 128, window, 0.09),),
                  seq_len=(5, 300), scale_mode="page", sinks=True, seed=9)
    case = W.make_case(spec, cuda_device)
    layer = case.layers[0]
    ps = layer.k_pages.shape[1]
    lens = case.attend_lens.cpu().numpy()
    tbl = layer.block_table.cpu().numpy()
    for b, L in enumerate(lens):
        last = tbl[b, (L - 1) // ps]
        if L % ps:
            layer.k_pages[last, L % ps:] = 0x7F
            layer.v_pages[last, L % ps:] = 0xFF
        if window:
            lo = max(0, L - window)
            first = tbl[b, lo // ps]
            if lo % ps:
                layer.k_pages[first, : lo % ps] = 0xFF
                layer.v_pages[first, : lo % ps] = 0x7F
    _check(F, layer, case.attend_lens, f"nan codes w={window}")


def test_fp8_compute_fused_append(F, cuda_device):
    """The fused append + attention on the fp8 path: codes bit-exact against
    the oracle's append, the output within the fp8 tolerance."""
    import oracle as O
    case = W.make_case("llama", cuda_device, B=4, seq_len=(40, 500))
    layer = case.layers[0]
    kp, vp = np_(layer.k_pages).copy(), np_(layer.v_pages).copy()
    O.kv_append(np_(layer.k_new), np_(layer.v_new), kp, vp, np_(layer.k_scale), np_(layer.v_scale),
                np_(layer.block_table), np_(case.positions))
    out = F.fp8_paged_decode_append_attention(
        layer.q, layer.k_new, layer.v_new, layer.k_pages, layer.v_pages, layer.k_scale,
        layer.v_scale, layer.block_table, case.positions, window=0, sinks=None,
        sm_scale=layer.sm_scale)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    assert np.array_equal(np_(layer.k_pages), kp) and np.array_equal(np_(layer.v_pages), vp)
    want = O.paged_decode_attention(np_(layer.q), kp, vp, np_(layer.k_scale), np_(layer.v_scale),
                                    np_(layer.block_table), np_(case.attend_lens),
                                    sm_scale=layer.sm_scale, compute="fp8")
    _close(np_(out), want, FP8_TOL, "fused fp8")


def test_fp8_compute_refuses_per_token_scales(F, cuda_device):
    case = W.make_case("llama", cuda_device, B=2, seq_len=(40, 100), scale_mode="token")
    layer = case.layers[0]
    out = torch.full(layer.q.shape, 3.0, device=cuda_device)
    with pytest.raises(F.Fp8pdError) as e:
        gpu_attention(F, layer, case.attend_lens, out=out)
    assert e.value.status == -5
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)
