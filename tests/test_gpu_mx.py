"""GPU: the MXFP8 cache (E4M3 codes, one E8M0 scale per 32 head-dim entries
of each stored token and KV head) against the float64 oracle.

Attention with MX K and V (or either one beside a float scale form) within
1e-3 * max(1, |ref|); the appends, unfused and fused, write codes and scale
bytes bit-exact against the oracle's MX quantizer. V blocks whose scales
span many binades inside one tile check the kernel's exact power-of-two
rescaling of decoded V (exact while a block is at most 14 binades below the
tile's largest).
"""

import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from tests._common import assert_attention_close, gpu_attention, np_, oracle_attention

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


def _check(F, layer, lens, where):
    got = np_(gpu_attention(F, layer, lens))
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0, where
    return assert_attention_close(got, oracle_attention(layer, lens), where)


@pytest.mark.parametrize("D", [64, 128, 256, 512])
@pytest.mark.parametrize("ps", [16, 64])
def test_mx_attention_head_dims_and_pages(F, cuda_device, D, ps):
    spec = W.Spec("mx", B=3, ps=ps, layers=(W.LayerSpec(16, 2, D, 0, D ** -0.5),),
                  seq_len=(5, 700), scale_mode="mx", sinks=True, seed=D + ps)
    case = W.make_case(spec, cuda_device)
    _check(F, case.layers[0], case.attend_lens, f"mx D={D} ps={ps}")


@pytest.mark.parametrize("name,overrides", [
    ("llama", dict(B=5, seq_len=(40, 1500))),
    ("gptoss_w128", dict(B=3, seq_len=900)),
    ("mixed", dict(B=3, seq_len=(300, 2500))),
    ("long_b1", dict(seq_len=9000)),
])
def test_mx_serving_shapes(F, cuda_device, name, overrides):
    case = W.make_case(name, cuda_device, scale_mode="mx", **overrides)
    for li, layer in enumerate(case.layers):
        _check(F, layer, case.attend_lens, f"mx {name}[{li}]")


def test_mx_beside_float_scales(F, cuda_device):
    """MX K with per-page V scales, and per-token K scales with MX V."""
    mx = W.make_case("llama", cuda_device, B=3, seq_len=(40, 600), scale_mode="mx")
    pg = W.make_case("llama", cuda_device, B=3, seq_len=(40, 600), scale_mode="page")
    tk = W.make_case("llama", cuda_device, B=3, seq_len=(40, 600), scale_mode="token")
    a, b, c = mx.layers[0], pg.layers[0], tk.layers[0]
    mixed1 = dataclasses.replace(a, v_pages=b.v_pages, v_scale=b.v_scale)
    _check(F, mixed1, mx.attend_lens, "K mx, V per page")
    mixed2 = dataclasses.replace(a, k_pages=c.k_pages, k_scale=c.k_scale)
    _check(F, mixed2, mx.attend_lens, "K per token, V mx")


@pytest.mark.parametrize("spread", [6, 14])
def test_mx_v_blocks_far_apart_in_one_tile(F, cuda_device, spread):
    """V scale codes drawn over `spread` binades per token and block: the
    kernel rescales decoded V by 2^(code - tile max), exact in f16 down to
    14 binades."""
    spec = W.Spec("mxs", B=2, ps=16, layers=(W.LayerSpec(8, 2, 128, 0, 128 ** -0.5),),
                  seq_len=(100, 400), scale_mode="mx", seed=spread)
    case = W.make_case(spec, cuda_device)
    layer = case.layers[0]
    g = torch.Generator(device=cuda_device).manual_seed(spread)
    shift = torch.randint(0, spread + 1, layer.v_scale.shape, generator=g, device=cuda_device,
                          dtype=torch.int32)
    layer.v_scale.copy_((layer.v_scale.to(torch.int32) - shift).clamp(1, 254).to(torch.uint8))
    _check(F, layer, case.attend_lens, f"mx V spread {spread}")


def test_mx_append_bit_exact(F, cuda_device):
    case = W.make_case("llama", cuda_device, B=6, seq_len=(40, 700), scale_mode="mx")
    layer = case.layers[0]
    want = [np_(t).copy() for t in (layer.k_pages, layer.v_pages, layer.k_scale, layer.v_scale)]
    O.kv_append(np_(layer.k_new), np_(layer.v_new), *want, np_(layer.block_table),
                np_(case.positions))
    F.fp8_kv_append(layer.k_new, layer.v_new, layer.k_pages, layer.v_pages, layer.k_scale,
                    layer.v_scale, layer.block_table, case.positions)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    for got, w in zip((layer.k_pages, layer.v_pages, layer.k_scale, layer.v_scale), want):
        assert np.array_equal(np_(got), w)


def test_mx_fused_append_attention(F, cuda_device):
    case = W.make_case("llama", cuda_device, B=5, seq_len=(40, 900), scale_mode="mx")
    layer = case.layers[0]
    want = [np_(t).copy() for t in (layer.k_pages, layer.v_pages, layer.k_scale, layer.v_scale)]
    O.kv_append(np_(layer.k_new), np_(layer.v_new), *want, np_(layer.block_table),
                np_(case.positions))
    out = F.fp8_paged_decode_append_attention(
        layer.q, layer.k_new, layer.v_new, layer.k_pages, layer.v_pages, layer.k_scale,
        layer.v_scale, layer.block_table, case.positions, window=0, sinks=None,
        sm_scale=layer.sm_scale)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    for got, w in zip((layer.k_pages, layer.v_pages, layer.k_scale, layer.v_scale), want):
        assert np.array_equal(np_(got), w)
    ref = O.paged_decode_attention(np_(layer.q), want[0], want[1], want[2], want[3],
                                   np_(layer.block_table), np_(case.attend_lens),
                                   sm_scale=layer.sm_scale)
    assert_attention_close(np_(out), ref, "mx fused")


def test_mx_refused_on_the_fp8_compute_path(F, cuda_device):
    case = W.make_case("llama", cuda_device, B=2, seq_len=(40, 100), scale_mode="mx")
    F.fp8pd_set_option(F.OPT_COMPUTE, 1)
    try:
        with pytest.raises(F.Fp8pdError) as e:
            gpu_attention(F, case.layers[0], case.attend_lens)
        assert e.value.status == -5
    finally:
        F.fp8pd_set_option(F.OPT_COMPUTE, 0)
