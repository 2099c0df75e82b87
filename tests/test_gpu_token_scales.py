"""GPU: per-token-per-head K/V scales -- one float32 per stored token and KV
head, shaped [num_pages, ps, Hkv] -- through the attention, the append and
the fused call, against the oracle. The append writes the new token's own
scale (max|x| / 448) beside its codes: both must be bit-exact."""

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from tests._common import (assert_attention_close, footer_pool, footer_views, gpu_attention, np_,
                           oracle_attention)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F(cuda_device):
    import fp8_paged_decode_split_b200 as F
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)
    return F


@pytest.fixture(autouse=True, params=[1, 3], ids=["uniform", "proportional"])
def schedule(F, request):
    """Per-token scales under uniform and proportional splits."""
    F.fp8pd_set_option(F.OPT_SCHEDULE, request.param)
    yield request.param
    F.fp8pd_set_option(F.OPT_SCHEDULE, 0)


def _attention(F, case, li=0, where=""):
    layer = case.layers[li]
    out = gpu_attention(F, layer, case.cache_lens)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0, where
    assert_attention_close(np_(out), oracle_attention(layer, case.cache_lens), where)
    return out


def _fused(F, case, li=0, positions=None, where=""):
    """Fused call on layer li: pools and scales bit-exact against the
    oracle's append, output within tolerance of its attention."""
    layer = case.layers[li]
    pos = case.positions if positions is None else positions
    kp0, vp0 = np_(layer.k_pages).copy(), np_(layer.v_pages).copy()
    ks0, vs0 = np_(layer.k_scale).copy(), np_(layer.v_scale).copy()
    out = F.fp8_paged_decode_append_attention(
        layer.q, layer.k_new, layer.v_new, layer.k_pages, layer.v_pages, layer.k_scale,
        layer.v_scale, layer.block_table, pos, window=layer.window, sinks=layer.sinks,
        sm_scale=layer.sm_scale)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0, where
    O.kv_append(np_(layer.k_new), np_(layer.v_new), kp0, vp0, ks0, vs0, np_(layer.block_table),
                np_(pos))
    assert np.array_equal(np_(layer.k_scale), ks0), f"{where}: K scales differ from the oracle"
    assert np.array_equal(np_(layer.v_scale), vs0), f"{where}: V scales differ from the oracle"
    assert np.array_equal(np_(layer.k_pages), kp0), f"{where}: K pool differs from the oracle"
    assert np.array_equal(np_(layer.v_pages), vp0), f"{where}: V pool differs from the oracle"
    want = O.paged_decode_attention(np_(layer.q), kp0, vp0, ks0, vs0, np_(layer.block_table),
                                    np_(pos).astype(np.int64) + 1, window=layer.window,
                                    sinks=np_(layer.sinks), sm_scale=layer.sm_scale)
    assert_attention_close(np_(out), want, where)
    return out


# ---------------------------------------------------------------- attention

def test_llama_like(F, cuda_device):
    """GQA 32/8, D = 128, ps = 16, ragged lengths."""
    case = W.make_case("llama", cuda_device, B=6, seq_len=(1, 700), scale_mode="token")
    _attention(F, case, where="llama token scales")


@pytest.mark.parametrize("name", ["gptoss_w128", "gptoss_full"])
def test_gptoss_like_sinks_and_window(F, cuda_device, name):
    """D = 64 (one tile per softmax step with per-token scales), sinks."""
    case = W.make_case(name, cuda_device, B=3, seq_len=(20, 1000), scale_mode="token")
    _attention(F, case, where=name)


def test_mixed_pool_head_dims_256_and_512(F, cuda_device):
    """Shared pool of 65,536-byte pages, ps = 32, N(0,2) values with outliers:
    per-token scales follow every outlier row."""
    case = W.make_case("mixed", cuda_device, B=3, seq_len=(100, 3000), scale_mode="token")
    _attention(F, case, li=0, where="mixed D=256")
    _attention(F, case, li=1, where="mixed D=512")


def test_page_size_64_many_splits(F, cuda_device):
    case = W.make_case("long_b1", cuda_device, seq_len=9000, scale_mode="token", append=False)
    _attention(F, case, where="ps=64")


@pytest.mark.parametrize("kd,vd", [(0, 0), (0, 1), (1, 0)], ids=["bits", "kbits-vcvt", "kcvt-vbits"])
def test_decode_variants(F, cuda_device, kd, vd):
    F.fp8pd_set_option(F.OPT_K_DECODE, kd)
    F.fp8pd_set_option(F.OPT_V_DECODE, vd)
    try:
        for name, D in (("gptoss_full", 64), ("llama", 128)):
            case = W.make_case(name, cuda_device, B=3, seq_len=(30, 600), scale_mode="token")
            _attention(F, case, where=f"D={D} decode {kd}{vd}")
    finally:
        F.fp8pd_set_option(F.OPT_K_DECODE, 1)
        F.fp8pd_set_option(F.OPT_V_DECODE, 1)


def test_constant_over_slots_equals_per_page(F, cuda_device):
    """A per-token view that repeats each page's scale (slot stride 0) gives
    the per-page result."""
    case = W.make_case("llama", cuda_device, B=5, seq_len=(30, 900), scale_mode="page")
    layer = case.layers[0]
    P, ps, Hkv = layer.k_pages.shape[0], layer.k_pages.shape[1], layer.k_pages.shape[2]
    ks3 = layer.k_scale.unsqueeze(1).expand(P, ps, Hkv)
    vs3 = layer.v_scale.unsqueeze(1).expand(P, ps, Hkv)
    a = gpu_attention(F, layer, case.cache_lens)
    b = F.fp8_paged_decode_attention(layer.q, layer.k_pages, layer.v_pages, ks3, vs3,
                                     layer.block_table, case.cache_lens, sm_scale=layer.sm_scale)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    assert torch.allclose(a, b, rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("k_tok", [True, False], ids=["k-token-v-page", "k-page-v-token"])
def test_mixed_scale_forms(F, cuda_device, k_tok):
    """K and V scales in different forms: one per token, the other per page
    (the per-token array's slot 0, a valid if coarser dequantization)."""
    case = W.make_case("llama", cuda_device, B=4, seq_len=(30, 700), scale_mode="token")
    layer = case.layers[0]
    if k_tok:
        layer.v_scale = layer.v_scale[:, 0, :].contiguous()
    else:
        layer.k_scale = layer.k_scale[:, 0, :].contiguous()
    _attention(F, case, where=f"k_tok={k_tok}")


def test_strided_scale_view(F, cuda_device):
    """Scales stored [num_pages, Hkv, ps] and passed as a permuted view."""
    case = W.make_case("llama", cuda_device, B=4, seq_len=(30, 700), scale_mode="token")
    layer = case.layers[0]
    layer.k_scale = layer.k_scale.permute(0, 2, 1).contiguous().permute(0, 2, 1)
    layer.v_scale = layer.v_scale.permute(0, 2, 1).contiguous().permute(0, 2, 1)
    assert layer.k_scale.stride(1) == 1
    _attention(F, case, where="strided scales")


# ---------------------------------------------------------------- append

@pytest.mark.parametrize("D", [64, 128, 96])
def test_append_writes_codes_and_scale(F, cuda_device, D):
    """fp8_kv_append with per-token scales: codes and the written scale
    bit-exact against the oracle; nothing else changes. D = 96 is not an
    attention head dim but the append takes any D."""
    g = torch.Generator(device=cuda_device).manual_seed(40 + D)
    P, ps, Hkv, B = 12, 16, 3, 5
    kp = torch.randint(0, 256, (P, ps, Hkv, D), dtype=torch.uint8, device=cuda_device, generator=g)
    vp = torch.randint(0, 256, (P, ps, Hkv, D), dtype=torch.uint8, device=cuda_device, generator=g)
    ks = torch.rand(P, ps, Hkv, device=cuda_device, generator=g) + 0.5
    vs = torch.rand(P, ps, Hkv, device=cuda_device, generator=g) + 0.5
    kn = (torch.randn(B, Hkv, D, device=cuda_device, generator=g) * 5).to(torch.bfloat16)
    vn = (torch.randn(B, Hkv, D, device=cuda_device, generator=g) * 1e-3).to(torch.bfloat16)
    kn[0, 1] = 0.0          # an all-zero row takes scale 1
    vn[2, 0, 3] = float("nan")  # a NaN entry is skipped by the maximum
    table = torch.tensor(np.random.default_rng(D).permutation(P)[:B * 2].reshape(B, 2),
                         dtype=torch.int32, device=cuda_device)
    pos = torch.tensor([0, 5, 16, 31, 17], dtype=torch.int32, device=cuda_device)
    want = [np_(t).copy() for t in (kp, vp, ks, vs)]
    F.fp8_kv_append(kn, vn, kp, vp, ks, vs, table, pos)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    O.kv_append(np_(kn), np_(vn), *want, np_(table), np_(pos))
    for got, w, name in zip((kp, vp, ks, vs), want, ("K pool", "V pool", "K scale", "V scale")):
        assert np.array_equal(np_(got), w), name
    assert np_(ks)[table[0, 0].item(), 0, 1] == 1.0


# ---------------------------------------------------------------- fused

def test_fused_llama_like(F, cuda_device):
    case = W.make_case("llama", cuda_device, B=6, seq_len=(40, 700), scale_mode="token")
    _fused(F, case, where="fused llama")


def test_fused_positions_at_page_edges(F, cuda_device):
    case = W.make_case("llama", cuda_device, B=8, seq_len=(300, 400), scale_mode="token")
    pos = torch.tensor([0, 15, 16, 17, 31, 32, 200, 299], dtype=torch.int32, device=cuda_device)
    _fused(F, case, positions=pos, where="fused page edges")


@pytest.mark.parametrize("name", ["gptoss_w128", "gptoss_full"])
def test_fused_gptoss_like(F, cuda_device, name):
    case = W.make_case(name, cuda_device, B=3, seq_len=1000, append=True, scale_mode="token")
    _fused(F, case, where=f"fused {name}")


def test_fused_mixed_and_g16(F, cuda_device):
    case = W.make_case("mixed", cuda_device, B=3, seq_len=(100, 3000), append=True,
                       scale_mode="token")
    _fused(F, case, li=0, where="fused mixed D=256")
    _fused(F, case, li=1, where="fused mixed D=512")
    spec = W.Spec("g16", B=3, ps=16, layers=(W.LayerSpec(32, 2, 128, 0, None),),
                  seq_len=(50, 900), scale_mode="token", append=True, seed=11)
    _fused(F, W.make_case(spec, cuda_device), where="fused G=16")


def test_fused_same_bytes_as_append_then_attention(F, cuda_device):
    a = W.make_case("llama", cuda_device, B=5, seq_len=(40, 900), scale_mode="token")
    b = W.make_case("llama", cuda_device, B=5, seq_len=(40, 900), scale_mode="token")
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
    assert torch.equal(la.k_scale, lb.k_scale) and torch.equal(la.v_scale, lb.v_scale)
    assert torch.equal(la.k_pages, lb.k_pages) and torch.equal(la.v_pages, lb.v_pages)
    assert torch.equal(got, want)


# ---------------------------------------------------------------- sub-row K groups

@pytest.mark.parametrize("name,G", [("gptoss_full", 2), ("gptoss_w128", 4), ("llama", 2),
                                    ("llama", 8), ("mixed", 16)])
def test_key_groups_attention(F, cuda_device, name, G):
    """K scales [num_pages, ps, Hkv, G]: each group of D / G head-dim entries
    has its own scale per token (D / G >= 16)."""
    case = W.make_case(name, cuda_device, B=3, seq_len=(20, 1500), scale_mode="token",
                       k_groups=G)
    for li in range(len(case.layers)):
        _attention(F, case, li=li, where=f"{name} k_groups={G} layer {li}")


def test_key_groups_decode_variants(F, cuda_device):
    F.fp8pd_set_option(F.OPT_K_DECODE, 0)
    F.fp8pd_set_option(F.OPT_V_DECODE, 0)
    try:
        case = W.make_case("llama", cuda_device, B=3, seq_len=(30, 600), scale_mode="token",
                           k_groups=4)
        _attention(F, case, where="k_groups=4 bit assembly")
    finally:
        F.fp8pd_set_option(F.OPT_K_DECODE, 1)
        F.fp8pd_set_option(F.OPT_V_DECODE, 1)


def test_one_key_group_equals_per_token(F, cuda_device):
    case = W.make_case("llama", cuda_device, B=4, seq_len=(30, 700), scale_mode="token")
    layer = case.layers[0]
    a = gpu_attention(F, layer, case.cache_lens)
    b = F.fp8_paged_decode_attention(layer.q, layer.k_pages, layer.v_pages,
                                     layer.k_scale.unsqueeze(-1), layer.v_scale.unsqueeze(-1),
                                     layer.block_table, case.cache_lens, sm_scale=layer.sm_scale)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    assert torch.equal(a, b)


@pytest.mark.parametrize("D,G", [(64, 4), (128, 8), (80, 16), (96, 2)])
def test_append_key_groups(F, cuda_device, D, G):
    """fp8_kv_append with sub-row K groups: codes and group scales bit-exact
    against the oracle. D = 80, G = 16 puts group starts at odd entries."""
    g = torch.Generator(device=cuda_device).manual_seed(60 + D)
    P, ps, Hkv, B = 10, 16, 2, 4
    kp = torch.randint(0, 256, (P, ps, Hkv, D), dtype=torch.uint8, device=cuda_device, generator=g)
    vp = kp.clone()
    ks = torch.rand(P, ps, Hkv, G, device=cuda_device, generator=g) + 0.5
    vs = torch.rand(P, ps, Hkv, device=cuda_device, generator=g) + 0.5
    mag = torch.logspace(-3, 2, G, device=cuda_device).repeat_interleave(D // G)
    kn = (torch.randn(B, Hkv, D, device=cuda_device, generator=g) * mag).to(torch.bfloat16)
    vn = torch.randn(B, Hkv, D, device=cuda_device, generator=g).to(torch.bfloat16)
    kn[1, 0, :D // G] = 0.0                      # one all-zero group
    table = torch.tensor(np.random.default_rng(D).permutation(P)[:B * 2].reshape(B, 2),
                         dtype=torch.int32, device=cuda_device)
    pos = torch.tensor([0, 7, 16, 31], dtype=torch.int32, device=cuda_device)
    want = [np_(t).copy() for t in (kp, vp, ks, vs)]
    F.fp8_kv_append(kn, vn, kp, vp, ks, vs, table, pos)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    O.kv_append(np_(kn), np_(vn), *want, np_(table), np_(pos))
    for got, w, name in zip((kp, vp, ks, vs), want, ("K pool", "V pool", "K scale", "V scale")):
        assert np.array_equal(np_(got), w), name


@pytest.mark.parametrize("name,G", [("llama", 4), ("gptoss_w128", 4), ("mixed", 16)])
def test_fused_key_groups(F, cuda_device, name, G):
    case = W.make_case(name, cuda_device, B=3, seq_len=(40, 1200), append=True,
                       scale_mode="token", k_groups=G)
    for li in range(len(case.layers)):
        _fused(F, case, li=li, where=f"fused {name} k_groups={G} layer {li}")


def test_fused_key_groups_same_bytes_as_two_calls(F, cuda_device):
    kw = dict(B=5, seq_len=(40, 900), scale_mode="token", k_groups=8)
    a = W.make_case("llama", cuda_device, **kw)
    b = W.make_case("llama", cuda_device, **kw)
    la, lb = a.layers[0], b.layers[0]
    # page-edge positions, none past the slot each sequence's table reserves
    pos = torch.minimum(torch.tensor([0, 15, 16, 400, 17], dtype=torch.int32, device=cuda_device),
                        a.positions)
    got = F.fp8_paged_decode_append_attention(
        la.q, la.k_new, la.v_new, la.k_pages, la.v_pages, la.k_scale, la.v_scale,
        la.block_table, pos, sm_scale=la.sm_scale)
    F.fp8_kv_append(lb.k_new, lb.v_new, lb.k_pages, lb.v_pages, lb.k_scale, lb.v_scale,
                    lb.block_table, pos)
    want = F.fp8_paged_decode_attention(lb.q, lb.k_pages, lb.v_pages, lb.k_scale, lb.v_scale,
                                        lb.block_table, pos + 1, sm_scale=lb.sm_scale)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    assert torch.equal(la.k_scale, lb.k_scale) and torch.equal(la.v_scale, lb.v_scale)
    assert torch.equal(la.k_pages, lb.k_pages) and torch.equal(la.v_pages, lb.v_pages)
    assert torch.equal(got, want)


def test_page1_worked_example_per_token(F, cuda_device):
    """The solution page's worked example as it is written there: 16-token
    blocks quantized per token and KV head into a permuted block table
    (2, 0, 1), GQA 2:1, 40 live tokens, one decode query, D ** -0.5."""
    BT, HKV, HQ, D, T = 16, 2, 4, 64, 40
    table = np.array([[2, 0, 1]], np.int32)
    g = torch.Generator().manual_seed(1)
    kt = torch.randn(3 * BT, HKV, D, generator=g).numpy().astype(np.float32)
    vt = torch.randn(3 * BT, HKV, D, generator=g).numpy().astype(np.float32)
    kp = np.zeros((3, BT, HKV, D), np.uint8)
    vp = np.zeros_like(kp)
    ks = np.zeros((3, BT, HKV), np.float32)
    vs = np.zeros_like(ks)
    for i in range(3):
        r = table[0, i]
        kp[r], ks[r] = O.quantize_per_token(kt[i * BT:(i + 1) * BT])
        vp[r], vs[r] = O.quantize_per_token(vt[i * BT:(i + 1) * BT])
    q = torch.randn(1, HQ, D, generator=g).to(torch.bfloat16)
    dev = lambda a: torch.from_numpy(a).to(cuda_device)  # noqa: E731
    out = F.fp8_paged_decode_attention(q.to(cuda_device), dev(kp), dev(vp), dev(ks), dev(vs),
                                       dev(table), dev(np.array([T], np.int32)))
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    want = O.paged_decode_attention(q.double().numpy(), kp, vp, ks, vs, table, np.array([T]))
    assert_attention_close(np_(out), want, "worked example, per-token scales")


# ---------------------------------------------------------------- scales in a page footer

def _footer_case(B, Hq, Hkv, D, ps, lens, seed, append):
    """K and V pools whose pages carry their tokens' per-token scales as a
    footer (built on the host with the oracle's per-token quantizer), a
    permuted block table, q and the new token."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens)
    npg = (lens + (1 if append else 0) + ps - 1) // ps
    P = int(npg.sum()) + 2
    perm = rng.permutation(P)
    table = np.full((B, int(npg.max())), -1, np.int32)
    off = 0
    for b in range(B):
        table[b, :npg[b]] = perm[off:off + npg[b]]
        off += npg[b]
    g = torch.Generator().manual_seed(seed)
    pools = []
    for _ in range(2):
        pool, codes, scales = footer_pool(P, ps, Hkv, D)
        x = torch.randn(P, ps, Hkv, D, generator=g) * (0.1 + 4 * torch.rand(P, ps, Hkv, 1, generator=g))
        c, s = O.quantize_per_token(x.numpy())
        codes.copy_(torch.from_numpy(c))
        scales.copy_(torch.from_numpy(s))
        pools.append(pool)
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16)
    return dict(pools=pools, P=P, table=table, lens=lens, q=q, kn=kn, vn=vn)


@pytest.mark.parametrize("shape", [(3, 16, 1, 64, 64), (3, 8, 2, 64, 16), (2, 16, 2, 128, 32)],
                         ids=["4352-byte-pages", "p1-rows-16x2x64", "ps32-D128"])
def test_scales_in_page_footer(F, cuda_device, shape):
    """Per-token scales stored after the codes of each page (DeepGEMM's
    64 x (64 + 4) = 4352-byte pages; the solution page's packed 16-token
    rows): the scale tensors are float32 views into the pool itself."""
    B, Hq, Hkv, D, ps = shape
    c = _footer_case(B, Hq, Hkv, D, ps, [5, 700, 1500][:B], 70 + D + ps, append=False)
    dev_pools = [p.to(cuda_device) for p in c["pools"]]
    (kc, ks), (vc, vs) = (footer_views(p, c["P"], ps, Hkv, D) for p in dev_pools)
    out = F.fp8_paged_decode_attention(c["q"].to(cuda_device), kc, vc, ks, vs,
                                       torch.from_numpy(c["table"]).to(cuda_device),
                                       torch.from_numpy(c["lens"].astype(np.int32)).to(cuda_device))
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    (hkc, hks), (hvc, hvs) = (footer_views(p, c["P"], ps, Hkv, D) for p in c["pools"])
    want = O.paged_decode_attention(c["q"].double().numpy(), hkc.numpy(), hvc.numpy(), hks.numpy(),
                                    hvs.numpy(), c["table"], c["lens"])
    assert_attention_close(np_(out), want, f"footer {shape}")


def test_fused_append_into_page_footer(F, cuda_device):
    """The fused call writes the new token's codes and its own scale into the
    page and the page's footer: the whole pool, bytes and all, as the
    oracle's append leaves it."""
    B, Hq, Hkv, D, ps = 3, 16, 1, 64, 64
    c = _footer_case(B, Hq, Hkv, D, ps, [63, 64, 900], 90, append=True)
    dev_pools = [p.to(cuda_device) for p in c["pools"]]
    (kc, ks), (vc, vs) = (footer_views(p, c["P"], ps, Hkv, D) for p in dev_pools)
    pos = c["lens"].astype(np.int32)
    out = F.fp8_paged_decode_append_attention(
        c["q"].to(cuda_device), c["kn"].to(cuda_device), c["vn"].to(cuda_device), kc, vc, ks, vs,
        torch.from_numpy(c["table"]).to(cuda_device), torch.from_numpy(pos).to(cuda_device))
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    (hkc, hks), (hvc, hvs) = (footer_views(p, c["P"], ps, Hkv, D) for p in c["pools"])
    views = [t.numpy() for t in (hkc, hvc, hks, hvs)]      # numpy views: the append writes the pools
    O.kv_append(np_(c["kn"]), np_(c["vn"]), *views, c["table"], pos)
    for got, want in zip(dev_pools, c["pools"]):
        assert torch.equal(got.cpu(), want)
    want = O.paged_decode_attention(c["q"].double().numpy(), *views, c["table"], pos + 1)
    assert_attention_close(np_(out), want, "fused footer")
