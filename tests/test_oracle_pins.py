"""Pins for the float64 CPU oracle, checked against things other than itself:
the E4M3 format's published limits, a library implementation of the format
(PyTorch ``float8_e4m3fn``), brute force, a library attention routine
(``scaled_dot_product_attention`` in float64), closed forms and invariants.
"""

import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _anchors():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_anchors.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            c, v = line.split()
            rows.append((int(c, 16), float(v)))
    return rows


# ---------------------------------------------------------------- E4M3 decode

def test_decode_anchor_values():
    for code, want in _anchors():
        got = O.e4m3_decode(np.array([code]))[0]
        if math.isnan(want):
            assert math.isnan(got), hex(code)
        else:
            assert got == want, (hex(code), got, want)
            assert math.copysign(1.0, got) == math.copysign(1.0, want), hex(code)


def test_decode_matches_library_float8_for_all_256_codes():
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    ours = O.e4m3_decode(codes)
    assert np.array_equal(ours, lib, equal_nan=True)


def test_decode_structure():
    v = O.e4m3_decode(np.arange(256, dtype=np.uint8))
    pos = v[:0x7F]
    assert np.all(np.diff(pos) > 0)                       # strictly increasing 0x00..0x7E
    assert np.array_equal(v[0x80:0xFF], -pos)             # sign symmetry
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert np.isfinite(v).sum() == 254
    # constant spacing inside each binade: 2^-9 for subnormals and [2^-6, 2^-5)
    for e in range(-6, 9):
        inb = pos[(pos >= 2.0 ** e) & (pos < 2.0 ** (e + 1))]
        assert np.allclose(np.diff(inb), 2.0 ** (e - 3), rtol=0, atol=0)
    sub = pos[pos < 2.0 ** -6]
    assert np.array_equal(sub, np.arange(8) * 2.0 ** -9)


# ---------------------------------------------------------------- E4M3 encode

def test_encode_roundtrip_finite_codes():
    codes = np.arange(256, dtype=np.uint8)
    v = O.e4m3_decode(codes)
    fin = np.isfinite(v)
    assert np.array_equal(O.e4m3_encode(v[fin]), codes[fin])


def test_encode_midpoints_go_to_even_mantissa():
    pos = O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2
    got = O.e4m3_encode(mids)
    lower = np.arange(0x7E)
    want = np.where(lower % 2 == 0, lower, lower + 1)
    assert np.array_equal(got, want.astype(np.uint8))
    # a hair either side of every midpoint goes to the nearer neighbour
    eps = np.spacing(mids) * 4
    assert np.array_equal(O.e4m3_encode(mids - eps), lower.astype(np.uint8))
    assert np.array_equal(O.e4m3_encode(mids + eps), (lower + 1).astype(np.uint8))
    assert np.array_equal(O.e4m3_encode(-mids), (want | 0x80).astype(np.uint8))


def test_encode_special_values():
    cases = [
        (448.0, 0x7E), (449.0, 0x7E), (464.0, 0x7E), (465.0, 0x7E), (1e30, 0x7E), (math.inf, 0x7E),
        (-math.inf, 0xFE), (-1e30, 0xFE), (0.0, 0x00), (-0.0, 0x80),
        (2.0 ** -10, 0x00),            # tie between 0 and 2^-9 -> even (0)
        (3 * 2.0 ** -11, 0x01),        # nearer 2^-9
        (2.0 ** -12, 0x00),
        (-(2.0 ** -9), 0x81),
    ]
    got = O.e4m3_encode(np.array([x for x, _ in cases]))
    assert [int(g) for g in got] == [c for _, c in cases]
    n = O.e4m3_encode(np.array([math.nan, -math.nan]))
    assert n[0] == 0x7F and n[1] == 0xFF


def test_encode_matches_brute_force_nearest():
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 1e-1, 1.0, 30.0, 150.0)])
    x = x[np.abs(x) < 448]
    grid = O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    got = O.e4m3_encode(x)
    for xi, gi in zip(x[:5000], got[:5000]):
        a = abs(xi)
        d = np.abs(grid - a)
        best = np.flatnonzero(d == d.min())
        code = best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]
        if xi < 0 or (xi == 0 and math.copysign(1, xi) < 0):
            code |= 0x80
        assert gi == code, (xi, gi, code)


def test_encode_matches_library_float8_for_float32_inputs():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(200000) * s for s in (1e-4, 1e-2, 1.0, 100.0)])
    x = x.astype(np.float32)
    x = x[np.abs(x) <= 464]
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(x.astype(np.float64)), lib)


def test_quantize_all_bf16_inputs_match_library_path():
    """Every bf16 bit pattern, several scales: float32 division, then E4M3.
    The library path (torch float32 division, float8 cast) agrees wherever the
    quotient is <= 464; above that the library gives NaN where E4M3
    quantization saturates to +-448."""
    bits = np.arange(65536, dtype=np.uint32) << 16
    x = bits.view(np.float32)
    for scale in (1.0, 0.5, 4.0 / 448, 3.0 / 448, 1e-3, 2.0 ** -20, 1e6, 37.0 / 448):
        s = np.float32(scale)
        ours = O.quantize(x, s)
        xt = torch.from_numpy(x.copy())
        quot = (xt / torch.tensor(s)).numpy()
        lib = torch.from_numpy(quot).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        ok = np.isfinite(quot) & (np.abs(quot) <= 464)
        assert np.array_equal(ours[ok], lib[ok]), scale
        big = np.isfinite(quot) & (np.abs(quot) > 464) | np.isinf(quot)
        assert np.all((ours[big] & 0x7F) == 0x7E)
        assert np.all((ours[np.isnan(quot)] & 0x7F) == 0x7F)


def test_quantize_divides_in_float32():
    """The code is a function of the float32 quotient: aim x / s just below a
    midpoint whose lower neighbour has an odd mantissa. In float64 the quotient
    rounds down; in float32 it rounds onto the midpoint, which then goes to the
    even (upper) code. The oracle must give the float32 answer."""
    pos = O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    rng = np.random.default_rng(3)
    found = 0
    for c in range(9, 0x7D, 2):                      # odd lower neighbour
        m = (pos[c] + pos[c + 1]) / 2
        for s in rng.uniform(0.001, 0.05, 400).astype(np.float32):
            x = np.float32(m * float(s))
            q64 = float(x) / float(s)
            q32 = float(np.float32(x) / s)
            if q32 == m and q64 < m:
                assert O.e4m3_encode(np.array([q64]))[0] == c
                assert O.quantize(np.array([x]), s)[0] == c + 1
                found += 1
                break
    assert found > 20


# ---------------------------------------------------------------- attention

def _dense_case(rng, B=2, Hq=8, Hkv=2, D=16, ps=16, L=(37, 50), scale_mode="page",
                permute=True, extra_pages=3):
    lens = np.array([L[b % len(L)] for b in range(B)])
    npg = (lens + ps - 1) // ps
    total = int(npg.sum()) + extra_pages
    perm = rng.permutation(total) if permute else np.arange(total)
    table = np.full((B, npg.max()), -1, np.int32)
    off = 0
    for b in range(B):
        table[b, :npg[b]] = perm[off:off + npg[b]]
        off += npg[b]
    k = rng.integers(0, 256, size=(total, ps, Hkv, D)).astype(np.uint8)
    v = rng.integers(0, 256, size=(total, ps, Hkv, D)).astype(np.uint8)
    k[(k & 0x7F) == 0x7F] = 0x10                                 # no NaN codes
    v[(v & 0x7F) == 0x7F] = 0x21
    if scale_mode == "page":
        ks = rng.uniform(0.001, 0.02, size=(total, Hkv)).astype(np.float32)
        vs = rng.uniform(0.001, 0.02, size=(total, Hkv)).astype(np.float32)
    elif scale_mode == "token":
        ks = rng.uniform(0.001, 0.02, size=(total, ps, Hkv)).astype(np.float32)
        vs = rng.uniform(0.001, 0.02, size=(total, ps, Hkv)).astype(np.float32)
    else:
        ks = rng.uniform(0.001, 0.02, size=Hkv).astype(np.float32)
        vs = rng.uniform(0.001, 0.02, size=Hkv).astype(np.float32)
    q = torch.randn(B, Hq, D, generator=torch.Generator().manual_seed(int(rng.integers(1 << 30))))
    q = q.to(torch.bfloat16).double().numpy()
    return dict(q=q, k=k, v=v, ks=ks, vs=vs, table=table, lens=lens)


def _scale_rows(sc, phys, slots, h):
    if sc.ndim == 3:
        return sc[phys, slots, h]
    return sc[phys, h] if sc.ndim == 2 else np.full(len(phys), sc[h])


def _sdpa_reference(c, window, sinks, sm_scale):
    """Library attention (torch SDPA, float64) over the dequantized keys,
    with KV heads repeated G times, the window as an additive mask, and a
    sink as one extra key with a zero value and logit = sink."""
    q, k, v, ks, vs, table, lens = (c[n] for n in ("q", "k", "v", "ks", "vs", "table", "lens"))
    B, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    ps = k.shape[1]
    out = np.zeros((B, Hq, D))
    for b in range(B):
        L = int(lens[b])
        t = np.arange(L)
        phys = table[b][t // ps]
        K = np.zeros((Hq, L + 1, D))
        V = np.zeros((Hq, L + 1, D))
        for hq in range(Hq):
            h = hq // G
            kscale = _scale_rows(ks, phys, t % ps, h)
            vscale = _scale_rows(vs, phys, t % ps, h)
            K[hq, :L] = torch.from_numpy(k[phys, t % ps, h]).view(torch.float8_e4m3fn).double().numpy() \
                * kscale[:, None]
            V[hq, :L] = torch.from_numpy(v[phys, t % ps, h]).view(torch.float8_e4m3fn).double().numpy() \
                * vscale[:, None]
        mask = np.zeros((Hq, 1, L + 1))
        if window > 0:
            mask[:, :, :max(0, L - window)] = -np.inf
        mask[:, :, L] = -np.inf if sinks is None else sinks[:, None]
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b][:, None, :]), torch.from_numpy(K), torch.from_numpy(V),
            attn_mask=torch.from_numpy(mask), scale=float(np.float32(sm_scale)))
        out[b] = o[:, 0, :].numpy()
    return out


def _run(c, **kw):
    return O.paged_decode_attention(c["q"], c["k"], c["v"], c["ks"], c["vs"], c["table"],
                                    c["lens"], **kw)


@pytest.mark.parametrize("window,with_sinks,scale_mode",
                         [(0, False, "page"), (0, True, "head"), (20, False, "head"), (7, True, "page"),
                          (0, False, "token"), (9, True, "token")])
def test_attention_matches_library_sdpa(window, with_sinks, scale_mode):
    rng = np.random.default_rng(100 + window)
    c = _dense_case(rng, scale_mode=scale_mode)
    sinks = rng.standard_normal(8).astype(np.float32) if with_sinks else None
    sm = 0.3
    got = _run(c, window=window, sinks=sinks, sm_scale=sm)
    want = _sdpa_reference(c, window, sinks, sm)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_paged_equals_contiguous():
    rng = np.random.default_rng(7)
    c = _dense_case(rng, B=1, L=(53,), permute=True, extra_pages=0)
    # contiguous copy: logical page i stored at physical page i
    ps = c["k"].shape[1]
    n = c["table"].shape[1]
    k2 = c["k"][c["table"][0]]
    v2 = c["v"][c["table"][0]]
    ks2 = c["ks"][c["table"][0]]
    vs2 = c["vs"][c["table"][0]]
    c2 = dict(c, k=k2, v=v2, ks=ks2, vs=vs2, table=np.arange(n, dtype=np.int32)[None])
    a = _run(c, window=0)
    b = _run(c2, window=0)
    assert np.array_equal(a, b)
    assert ps == 16


def test_gqa_equals_repeated_kv_heads():
    rng = np.random.default_rng(8)
    c = _dense_case(rng, Hq=8, Hkv=2)
    G = 4
    rep = dict(c, k=np.repeat(c["k"], G, axis=2), v=np.repeat(c["v"], G, axis=2),
               ks=np.repeat(c["ks"], G, axis=1), vs=np.repeat(c["vs"], G, axis=1))
    assert np.array_equal(_run(c, window=0), _run(rep, window=0))


def test_minus_inf_sink_equals_no_sink_and_infinite_window_equals_full():
    rng = np.random.default_rng(9)
    c = _dense_case(rng)
    base = _run(c, window=0)
    assert np.array_equal(_run(c, window=0, sinks=np.full(8, -np.inf, np.float32)), base)
    assert np.array_equal(_run(c, window=int(c["lens"].max())), base)
    assert np.array_equal(_run(c, window=10 ** 6), base)


def test_closed_forms_zero_query_and_single_key():
    rng = np.random.default_rng(10)
    c = _dense_case(rng, scale_mode="head")
    c0 = dict(c, q=np.zeros_like(c["q"]))
    ps = c["k"].shape[1]
    G = 4
    for window, sinks in ((0, None), (9, np.linspace(-1, 1, 8).astype(np.float32))):
        got = _run(c0, window=window, sinks=sinks)
        for b in range(2):
            L = int(c["lens"][b])
            lo = max(0, L - window) if window else 0
            t = np.arange(lo, L)
            phys = c["table"][b][t // ps]
            for hq in range(8):
                h = hq // G
                V = O.e4m3_decode(c["v"][phys, t % ps, h]) * float(c["vs"][h])
                den = len(t) + (0.0 if sinks is None else math.exp(float(sinks[hq])))
                assert np.allclose(got[b, hq], V.sum(0) / den, rtol=1e-13, atol=1e-15)
    c1 = dict(c, lens=np.array([1, 1]))
    got = _run(c1, window=0)
    for b in range(2):
        p = c["table"][b][0]
        for hq in range(8):
            assert np.array_equal(got[b, hq], O.e4m3_decode(c["v"][p, 0, hq // G]) * float(c["vs"][hq // G]))


def test_empty_sequence_gives_zero():
    rng = np.random.default_rng(12)
    c = dict(_dense_case(rng), lens=np.array([0, 0]))
    assert np.array_equal(_run(c, window=0), np.zeros((2, 8, 16)))
    assert np.array_equal(_run(c, window=0, sinks=np.ones(8, np.float32)), np.zeros((2, 8, 16)))


def test_brute_force_tiny_inputs():
    """Naive softmax without max subtraction, in pure Python, on tiny inputs."""
    rng = np.random.default_rng(13)
    for trial in range(20):
        D = int(rng.integers(1, 9))
        L = int(rng.integers(1, 9))
        c = _dense_case(rng, B=1, Hq=2, Hkv=1, D=D, ps=16, L=(L,), scale_mode="page")
        window = int(rng.integers(0, L + 2))
        sinks = rng.standard_normal(2).astype(np.float32) if trial % 2 else None
        sm = float(np.float32(rng.uniform(0.05, 0.5)))
        got = _run(c, window=window, sinks=sinks, sm_scale=sm)
        for hq in range(2):
            lo = max(0, L - window) if window else 0
            num = [0.0] * D
            den = 0.0 if sinks is None else math.exp(float(sinks[hq]))
            for t in range(lo, L):
                p = int(c["table"][0][t // 16])
                kv = [e4m3(int(c["k"][p, t % 16, 0, d])) * float(c["ks"][p, 0]) for d in range(D)]
                vv = [e4m3(int(c["v"][p, t % 16, 0, d])) * float(c["vs"][p, 0]) for d in range(D)]
                s = sm * sum(float(c["q"][0, hq, d]) * kv[d] for d in range(D))
                w = math.exp(s)
                den += w
                for d in range(D):
                    num[d] += w * vv[d]
            want = [x / den for x in num] if den > 0 else [0.0] * D
            assert np.allclose(got[0, hq], want, rtol=1e-12, atol=1e-14)


def e4m3(code: int) -> float:
    """Tiny independent E4M3 reading through the library float8 type."""
    return float(torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).double()[0])


def test_page1_worked_example_shape():
    """The paged oracle reproduces plain softmax attention over dequantized
    K/V for the worked example's shape (16-token blocks, GQA 2:1, 40 tokens,
    block table [2, 0, 1]); per-(page, head) scales from the oracle quantizer."""
    spec = {}
    with open(os.path.join(GOLDEN, "page1_worked_example.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, *v = line.split()
                spec[k] = v
    BT, HKV, HQ, D, T = (int(spec[k][0]) for k in
                         ("block_tokens", "n_kv_heads", "n_q_heads", "head_dim", "live_tokens"))
    table = np.array([[int(x) for x in spec["block_table"]]], np.int32)
    n_blk = (T + BT - 1) // BT
    g = torch.Generator().manual_seed(0)
    kt = torch.randn(n_blk * BT, HKV, D, generator=g).numpy().astype(np.float32)
    vt = torch.randn(n_blk * BT, HKV, D, generator=g).numpy().astype(np.float32)
    kp = np.zeros((n_blk, BT, HKV, D), np.uint8)
    vp = np.zeros_like(kp)
    ks = np.zeros((n_blk, HKV), np.float32)
    vs = np.zeros_like(ks)
    for i in range(n_blk):
        r = table[0, i]
        blk_k, blk_v = kt[i * BT:(i + 1) * BT], vt[i * BT:(i + 1) * BT]
        ks[r] = np.abs(blk_k).max(axis=(0, 2)) / np.float32(448)
        vs[r] = np.abs(blk_v).max(axis=(0, 2)) / np.float32(448)
        kp[r] = O.quantize(blk_k, ks[r][None, :, None])
        vp[r] = O.quantize(blk_v, vs[r][None, :, None])
    q = torch.randn(1, HQ, D, generator=g).to(torch.bfloat16).double().numpy()
    out = O.paged_decode_attention(q, kp, vp, ks, vs, table, np.array([T]), window=0)
    # plain attention over the dequantized values, in logical order
    kd = np.concatenate([O.e4m3_decode(kp[table[0, i]]) * ks[table[0, i]][None, :, None]
                         for i in range(n_blk)])[:T].transpose(1, 0, 2)
    vd = np.concatenate([O.e4m3_decode(vp[table[0, i]]) * vs[table[0, i]][None, :, None]
                         for i in range(n_blk)])[:T].transpose(1, 0, 2)
    qq = q[0].reshape(HKV, HQ // HKV, D)
    w = torch.softmax(torch.einsum("hgd,htd->hgt", torch.from_numpy(qq), torch.from_numpy(kd)) * D ** -0.5,
                      dim=-1)
    want = torch.einsum("hgt,htd->hgd", w, torch.from_numpy(vd)).reshape(1, HQ, D).numpy()
    assert np.allclose(out, want, rtol=1e-12, atol=1e-12)
    # the dequantized values are within E4M3 rounding of the originals
    assert np.all(np.abs(kd.transpose(1, 0, 2) - kt[:T]) <= np.abs(kt[:T]) / 16 + 2.0 ** -10)
    assert float(spec["tolerance"][0]) == 1e-2


def test_page1_worked_example_per_token_scales():
    """The worked example as the page writes it: each 16-token block goes
    through the per-token-per-head quantizer (one scale per token and KV
    head) into its permuted page; the paged oracle then reproduces plain
    softmax attention over the dequantized values."""
    spec = {}
    with open(os.path.join(GOLDEN, "page1_worked_example.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, *v = line.split()
                spec[k] = v
    BT, HKV, HQ, D, T = (int(spec[k][0]) for k in
                         ("block_tokens", "n_kv_heads", "n_q_heads", "head_dim", "live_tokens"))
    table = np.array([[int(x) for x in spec["block_table"]]], np.int32)
    n_blk = (T + BT - 1) // BT
    g = torch.Generator().manual_seed(1)
    kt = torch.randn(n_blk * BT, HKV, D, generator=g).numpy().astype(np.float32)
    vt = torch.randn(n_blk * BT, HKV, D, generator=g).numpy().astype(np.float32)
    kp = np.zeros((n_blk, BT, HKV, D), np.uint8)
    vp = np.zeros_like(kp)
    ks = np.zeros((n_blk, BT, HKV), np.float32)
    vs = np.zeros_like(ks)
    kd, vd = [], []
    for i in range(n_blk):
        r = table[0, i]
        kp[r], ks[r] = O.quantize_per_token(kt[i * BT:(i + 1) * BT])
        vp[r], vs[r] = O.quantize_per_token(vt[i * BT:(i + 1) * BT])
        # dequantized through the library float8 type, not the oracle's table
        f8 = lambda c: torch.from_numpy(c).view(torch.float8_e4m3fn).double().numpy()  # noqa: E731
        kd.append(f8(kp[r]) * ks[r][..., None])
        vd.append(f8(vp[r]) * vs[r][..., None])
    kd = np.concatenate(kd)[:T].transpose(1, 0, 2)
    vd = np.concatenate(vd)[:T].transpose(1, 0, 2)
    q = torch.randn(1, HQ, D, generator=g).to(torch.bfloat16).double().numpy()
    out = O.paged_decode_attention(q, kp, vp, ks, vs, table, np.array([T]), window=0)
    qq = q[0].reshape(HKV, HQ // HKV, D)
    w = torch.softmax(torch.einsum("hgd,htd->hgt", torch.from_numpy(qq), torch.from_numpy(kd)) * D ** -0.5,
                      dim=-1)
    want = torch.einsum("hgt,htd->hgd", w, torch.from_numpy(vd)).reshape(1, HQ, D).numpy()
    assert np.allclose(out, want, rtol=1e-12, atol=1e-12)
    # per-token scales keep every value within half an E4M3 step of its row
    ks_rows = np.concatenate([ks[table[0, i]] for i in range(n_blk)])[:T][..., None]
    assert np.all(np.abs(kd.transpose(1, 0, 2) - kt[:T]) <= np.abs(kt[:T]) / 16 + 2.0 ** -10 * ks_rows)


# ---------------------------------------------------------------- append

def test_append_writes_only_the_new_slot():
    rng = np.random.default_rng(14)
    num_pages, ps, Hkv, D, B = 12, 16, 2, 32, 3
    kp = rng.integers(0, 256, (num_pages, ps, Hkv, D)).astype(np.uint8)
    vp = rng.integers(0, 256, (num_pages, ps, Hkv, D)).astype(np.uint8)
    k0, v0 = kp.copy(), vp.copy()
    table = rng.permutation(num_pages)[:B * 4].reshape(B, 4).astype(np.int32)
    pos = np.array([0, 17, 63])
    ks = rng.uniform(0.005, 0.02, (num_pages, Hkv)).astype(np.float32)
    vs = rng.uniform(0.005, 0.02, Hkv).astype(np.float32)
    g = torch.Generator().manual_seed(14)
    kn = (torch.randn(B, Hkv, D, generator=g) * 3).to(torch.bfloat16).float().numpy()
    vn = (torch.randn(B, Hkv, D, generator=g) * 3).to(torch.bfloat16).float().numpy()
    O.kv_append(kn, vn, kp, vp, ks, vs, table, pos)
    touched = np.zeros((num_pages, ps), bool)
    for b in range(B):
        p, s = table[b, pos[b] // ps], pos[b] % ps
        touched[p, s] = True
        for h in range(Hkv):
            for got, x, sc in ((kp[p, s, h], kn[b, h], ks[p, h]), (vp[p, s, h], vn[b, h], vs[h])):
                quot = (torch.from_numpy(x) / torch.tensor(sc)).numpy()
                lib = torch.from_numpy(quot).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
                small = np.abs(quot) <= 464          # the library cast agrees up to here
                assert np.array_equal(got[small], lib[small])
                assert np.all((got[~small] & 0x7F) == 0x7E)   # beyond it E4M3 saturates
    assert np.array_equal(kp[~touched], k0[~touched])
    assert np.array_equal(vp[~touched], v0[~touched])


# ---------------------------------------------------------------- per-token scales

def test_token_scale_matches_library_amax_over_448():
    g = torch.Generator().manual_seed(21)
    x = (torch.randn(64, 4, 96, generator=g) * torch.rand(64, 4, 1, generator=g) * 50).to(torch.bfloat16).float()
    want = (x.abs().amax(-1) / torch.tensor(448.0)).numpy()        # float32 IEEE division
    got = O.token_scale(x.numpy())
    assert got.dtype == np.float32 and np.array_equal(got, want)


def test_token_scale_special_rows():
    rows = np.array([[0.0, -0.0, 0.0, 0.0],            # all zero -> 1
                     [np.nan, 2.0, -3.0, 1.0],          # NaN skipped -> 3 / 448
                     [-896.0, 1.0, 0.5, 0.0]], np.float32)
    s = O.token_scale(rows)
    assert s[0] == 1.0
    assert s[1] == np.float32(3.0) / np.float32(448.0)
    assert s[2] == 2.0
    codes, _ = O.quantize_per_token(rows[[0, 2]])
    assert list(codes[0]) == [0x00, 0x80, 0x00, 0x00]
    assert codes[1][0] == 0xFE                          # -448: the row's maximum


def test_quantize_per_token_maximum_maps_to_448_and_error_bound():
    """Every row's largest magnitude lands on code 0x7E / 0xFE (448), and the
    dequantized value is within half an E4M3 step: 2^-4 relative in the
    normal range, 2^-10 * scale below it (P1 "Supported scope")."""
    rng = np.random.default_rng(22)
    x = (rng.standard_normal((200, 3, 64)) * rng.uniform(1e-3, 1e3, (200, 3, 1))).astype(np.float32)
    codes, s = O.quantize_per_token(x)
    idx = np.abs(x).argmax(-1)
    top = np.take_along_axis(codes, idx[..., None], -1)[..., 0]
    assert np.all((top & 0x7F) == 0x7E)
    deq = O.e4m3_decode(codes) * s[..., None].astype(np.float64)
    err = np.abs(deq - x.astype(np.float64))
    normal = np.abs(x) / s[..., None] >= 2.0 ** -6
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(x[normal]) * (1 + 1e-6))
    sub = np.broadcast_to(s[..., None], x.shape)[~normal].astype(np.float64)
    assert np.all(err[~normal] <= 2.0 ** -10 * sub * (1 + 1e-6))


def test_per_token_scale_constant_over_slots_equals_per_page():
    rng = np.random.default_rng(23)
    c = _dense_case(rng, scale_mode="page")
    ps = c["k"].shape[1]
    c3 = dict(c, ks=np.repeat(c["ks"][:, None, :], ps, 1), vs=np.repeat(c["vs"][:, None, :], ps, 1))
    for w in (0, 11):
        assert np.array_equal(_run(c, window=w, sm_scale=0.2), _run(c3, window=w, sm_scale=0.2))


def _logical_scale_case(B=3, Hq=4, Hkv=2, D=8, ps=16, lens=(5, 40, 33), seed=24):
    """Every K and V code is 0x38 (1.0); scales are set per logical position
    t of each sequence through a permuted block table."""
    rng = np.random.default_rng(seed)
    lens = np.array(lens)
    npg = (lens + ps - 1) // ps
    total = int(npg.sum()) + 2
    perm = rng.permutation(total)
    table = np.full((B, npg.max()), -1, np.int32)
    off = 0
    for b in range(B):
        table[b, :npg[b]] = perm[off:off + npg[b]]
        off += npg[b]
    k = np.full((total, ps, Hkv, D), 0x38, np.uint8)
    v = np.full((total, ps, Hkv, D), 0x38, np.uint8)
    return table, k, v, lens, total


def test_per_token_v_scale_closed_form():
    """Scores all 0 (q = 0): out = mean over the attended keys of the V scale
    of each key, which is set to 1 + t + 1000 h at logical position t; the
    mean of an arithmetic series is 1 + 1000 h + (lo + L - 1) / 2."""
    B, Hq, Hkv, D, ps = 3, 4, 2, 8, 16
    table, k, v, lens, total = _logical_scale_case(B, Hq, Hkv, D, ps)
    ks = np.ones((total, ps, Hkv), np.float32)
    vs = np.zeros((total, ps, Hkv), np.float32)
    for b in range(B):
        for t in range(lens[b]):
            vs[table[b, t // ps], t % ps, :] = 1 + t + 1000 * np.arange(Hkv)
    q = np.zeros((B, Hq, D))
    for window in (0, 4, 100):
        out = O.paged_decode_attention(q, k, v, ks, vs, table, lens, window=window, sm_scale=0.5)
        for b in range(B):
            lo, L = max(0, lens[b] - window) if window else 0, lens[b]
            for hq in range(Hq):
                h = hq // (Hq // Hkv)
                assert np.allclose(out[b, hq], 1 + 1000 * h + (lo + L - 1) / 2, rtol=1e-13)


def test_per_token_k_scale_closed_form():
    """q = 1 everywhere, K scale a * t and V scale t at logical position t:
    the weights are r^t with r = exp(sm * D * a), so out is the r-weighted
    mean of t over the attended keys."""
    B, Hq, Hkv, D, ps = 3, 4, 2, 8, 16
    table, k, v, lens, total = _logical_scale_case(B, Hq, Hkv, D, ps, seed=25)
    a, sm = 0.01, 0.5
    ks = np.zeros((total, ps, Hkv), np.float32)
    vs = np.zeros((total, ps, Hkv), np.float32)
    for b in range(B):
        for t in range(lens[b]):
            ks[table[b, t // ps], t % ps, :] = np.float32(a * t)
            vs[table[b, t // ps], t % ps, :] = t
    q = np.ones((B, Hq, D))
    out = O.paged_decode_attention(q, k, v, ks, vs, table, lens, sm_scale=sm)
    for b in range(B):
        t = np.arange(lens[b])
        w = np.exp(sm * D * np.float32(a * t).astype(np.float64) * 1.0)
        want = (w * t).sum() / w.sum()
        assert np.allclose(out[b], want, rtol=1e-12)


def test_append_per_token_writes_its_scale_and_codes():
    rng = np.random.default_rng(26)
    num_pages, ps, Hkv, D, B = 10, 16, 2, 64, 3
    kp = rng.integers(0, 256, (num_pages, ps, Hkv, D)).astype(np.uint8)
    vp = kp.copy()
    ks = rng.uniform(0.01, 0.02, (num_pages, ps, Hkv)).astype(np.float32)
    vs = ks.copy()
    k0, v0, ks0, vs0 = kp.copy(), vp.copy(), ks.copy(), vs.copy()
    table = rng.permutation(num_pages)[:B * 3].reshape(B, 3).astype(np.int32)
    pos = np.array([0, 20, 47])
    g = torch.Generator().manual_seed(26)
    kn = (torch.randn(B, Hkv, D, generator=g) * 7).to(torch.bfloat16).float()
    vn = (torch.randn(B, Hkv, D, generator=g) * 0.01).to(torch.bfloat16).float()
    O.kv_append(kn.numpy(), vn.numpy(), kp, vp, ks, vs, table, pos)
    touched = np.zeros((num_pages, ps), bool)
    for b in range(B):
        p, s = table[b, pos[b] // ps], pos[b] % ps
        touched[p, s] = True
        for pages, scales, x in ((kp, ks, kn[b]), (vp, vs, vn[b])):
            lib_s = (x.abs().amax(-1) / torch.tensor(448.0)).numpy()
            assert np.array_equal(scales[p, s], lib_s)
            quot = x / torch.from_numpy(lib_s)[:, None]
            lib = quot.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(pages[p, s], lib)
    assert np.array_equal(kp[~touched], k0[~touched]) and np.array_equal(vp[~touched], v0[~touched])
    assert np.array_equal(ks[~touched], ks0[~touched]) and np.array_equal(vs[~touched], vs0[~touched])


# ---------------------------------------------------------------- sub-row key groups

def test_group_scale_matches_library():
    g = torch.Generator().manual_seed(31)
    x = (torch.randn(40, 2, 128, generator=g) * 9).to(torch.bfloat16).float()
    for G in (1, 2, 4, 8):
        want = (x.view(40, 2, G, 128 // G).abs().amax(-1) / torch.tensor(448.0)).numpy()
        got = O.group_scale(x.numpy(), G)
        assert got.shape == (40, 2, G) and np.array_equal(got, want)
    assert np.array_equal(O.group_scale(x.numpy(), 1)[..., 0], O.token_scale(x.numpy()))


def test_one_group_equals_per_token():
    rng = np.random.default_rng(32)
    c = _dense_case(rng, scale_mode="token")
    c4 = dict(c, ks=c["ks"][..., None])
    for w in (0, 13):
        assert np.array_equal(_run(c, window=w, sm_scale=0.3), _run(c4, window=w, sm_scale=0.3))


def test_grouped_key_scales_match_library_sdpa():
    """K scales per (token, KV head, group of D/4 entries), dequantized here
    by index arithmetic of the test's own, against torch SDPA."""
    rng = np.random.default_rng(33)
    c = _dense_case(rng, scale_mode="token")
    total, ps, Hkv = c["ks"].shape
    G, D = 4, c["k"].shape[-1]
    ks4 = rng.uniform(0.001, 0.05, size=(total, ps, Hkv, G)).astype(np.float32)
    sinks = rng.standard_normal(8).astype(np.float32)
    got = _run(dict(c, ks=ks4), window=9, sinks=sinks, sm_scale=0.4)
    # fold each group's scale into the codes' values: a per-token K scale of 1
    # and K values decoded by the library, times the group scale per entry
    kval = torch.from_numpy(c["k"]).view(torch.float8_e4m3fn).double().numpy()
    kval = kval * np.stack([ks4[..., d * G // D] for d in range(D)], axis=-1)
    q, B = c["q"], c["q"].shape[0]
    out = np.zeros_like(got)
    for b in range(B):
        L = int(c["lens"][b])
        t = np.arange(L)
        phys, slot = c["table"][b][t // ps], t % ps
        for hq in range(q.shape[1]):
            h = hq // (q.shape[1] // Hkv)
            K = torch.from_numpy(kval[phys, slot, h])[None]
            V = torch.from_numpy(torch.from_numpy(c["v"][phys, slot, h]).view(torch.float8_e4m3fn)
                                 .double().numpy() * c["vs"][phys, slot, h][:, None])[None]
            K = torch.cat([K, torch.zeros(1, 1, D, dtype=K.dtype)], 1)
            V = torch.cat([V, torch.zeros(1, 1, D, dtype=V.dtype)], 1)
            mask = np.zeros((1, 1, L + 1))
            mask[..., :max(0, L - 9)] = -np.inf
            mask[..., L] = sinks[hq]
            o = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[b, hq])[None, None], K, V, attn_mask=torch.from_numpy(mask),
                scale=float(np.float32(0.4)))
            out[b, hq] = o[0, 0].numpy()
    assert np.allclose(got, out, rtol=1e-12, atol=1e-12)


def test_grouped_key_scale_closed_form():
    """q is 1 on the entries of group 2 and 0 elsewhere, every code is 0x38
    (1.0); group 2's K scale is a * t at logical position t, the other groups'
    scales are huge. The scores are sm * (D/4) * a * t, so out is the r^t
    weighted mean of the V scale t, whatever the other groups hold."""
    B, Hq, Hkv, D, ps = 3, 4, 2, 16, 16
    table, k, v, lens, total = _logical_scale_case(B, Hq, Hkv, D, ps, seed=34)
    a, sm, G = 0.01, 0.5, 4
    ks = np.full((total, ps, Hkv, G), 1e6, np.float32)
    vs = np.zeros((total, ps, Hkv), np.float32)
    for b in range(B):
        for t in range(lens[b]):
            ks[table[b, t // ps], t % ps, :, 2] = np.float32(a * t)
            vs[table[b, t // ps], t % ps, :] = t
    q = np.zeros((B, Hq, D))
    q[:, :, 2 * D // G:3 * D // G] = 1.0
    out = O.paged_decode_attention(q, k, v, ks, vs, table, lens, sm_scale=sm)
    for b in range(B):
        t = np.arange(lens[b])
        w = np.exp(sm * (D // G) * np.float32(a * t).astype(np.float64))
        assert np.allclose(out[b], (w * t).sum() / w.sum(), rtol=1e-12)


def test_append_grouped_key_scales():
    rng = np.random.default_rng(35)
    num_pages, ps, Hkv, D, B, G = 8, 16, 2, 64, 3, 4
    kp = rng.integers(0, 256, (num_pages, ps, Hkv, D)).astype(np.uint8)
    vp = kp.copy()
    ks = rng.uniform(0.01, 0.02, (num_pages, ps, Hkv, G)).astype(np.float32)
    vs = rng.uniform(0.01, 0.02, (num_pages, ps, Hkv)).astype(np.float32)
    k0, ks0 = kp.copy(), ks.copy()
    table = rng.permutation(num_pages)[:B * 2].reshape(B, 2).astype(np.int32)
    pos = np.array([3, 16, 31])
    g = torch.Generator().manual_seed(35)
    kn = (torch.randn(B, Hkv, D, generator=g) * torch.tensor([1e-3, 1.0, 30.0, 0.1]).repeat_interleave(D // G)
          ).to(torch.bfloat16).float()
    vn = torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16).float()
    O.kv_append(kn.numpy(), vn.numpy(), kp, vp, ks, vs, table, pos)
    touched = np.zeros((num_pages, ps), bool)
    for b in range(B):
        p, s = table[b, pos[b] // ps], pos[b] % ps
        touched[p, s] = True
        lib_s = (kn[b].view(Hkv, G, D // G).abs().amax(-1) / torch.tensor(448.0))
        assert np.array_equal(ks[p, s], lib_s.numpy())
        quot = kn[b] / lib_s.repeat_interleave(D // G, dim=-1)
        assert np.array_equal(kp[p, s], quot.to(torch.float8_e4m3fn).view(torch.uint8).numpy())
    assert np.array_equal(kp[~touched], k0[~touched]) and np.array_equal(ks[~touched], ks0[~touched])


# ------------------------------------------------------ window boundary pins
# The window is defined in words on the pages: the solution page's "Expected
# result" keeps "the last W keys", and the gpt-oss workload keeps the keys at
# positions greater than cur_pos - W, cur_pos = L - 1 being the query's own
# position. The pins below derive the attended set from those words with a
# per-position predicate (never from the oracle's lower bound) and read the
# set the oracle actually used off its output.

def _marker_case(L: int, ps: int = 16, Hq: int = 2, Hkv: int = 1, seed: int = 31):
    """One sequence of L keys whose value at logical position t is the unit
    vector e_t (code 0x38 = 1.0 at dim t, scale 1) and whose keys are
    random: with q = 0 every attended key gets the same weight, so the
    output is 1/n on exactly the attended positions and 0 elsewhere."""
    rng = np.random.default_rng(seed)
    D = L
    npg = (L + ps - 1) // ps
    perm = rng.permutation(npg + 2)
    table = perm[:npg].astype(np.int32)[None]
    k = rng.integers(0, 0x70, size=(npg + 2, ps, Hkv, D)).astype(np.uint8)
    v = np.zeros((npg + 2, ps, Hkv, D), np.uint8)
    for t in range(L):
        v[table[0, t // ps], t % ps, :, t] = 0x38
    ones = np.ones(Hkv, np.float32)
    return dict(q=np.zeros((1, Hq, D)), k=k, v=v, ks=ones, vs=ones, table=table,
                lens=np.array([L]))


def _last_w_keys(L: int, W: int) -> list:
    """Positions t in [0, L) with t > cur_pos - W, cur_pos = L - 1; every key
    when W = 0 (no window)."""
    cur = L - 1
    return [t for t in range(L) if W == 0 or t > cur - W]


@pytest.mark.parametrize("L", [1, 2, 17, 40])
def test_window_keeps_exactly_the_last_w_keys(L):
    c = _marker_case(L)
    for W in sorted({0, 1, 2, 3, L - 1, L, L + 1, 2 * L + 5}):
        got = _run(c, window=W)[0]
        want_set = _last_w_keys(L, W)
        assert len(want_set) == (min(L, W) if W > 0 else L)
        support = [t for t in range(L) if got[0, t] != 0.0]
        assert support == want_set, (L, W, support)
        assert np.allclose(got[:, want_set], 1.0 / len(want_set), rtol=0, atol=1e-15)


def test_window_one_is_the_current_key_alone():
    """W = 1: only the query's own position is attended, so the output is
    that key's value exactly; with a sink s (no value) the weight of the one
    key is e^score / (e^score + e^s)."""
    rng = np.random.default_rng(41)
    c = _dense_case(rng, B=2, scale_mode="page", L=(37, 50))
    ps = c["k"].shape[1]
    G = 4
    got = _run(c, window=1, sm_scale=0.3)
    sinks = np.linspace(-1.5, 2.0, 8).astype(np.float32)
    got_s = _run(c, window=1, sinks=sinks, sm_scale=0.3)
    for b in range(2):
        t = int(c["lens"][b]) - 1
        p = int(c["table"][b][t // ps])
        for hq in range(8):
            h = hq // G
            kv = O.e4m3_decode(c["k"][p, t % ps, h]) * float(c["ks"][p, h])
            vv = O.e4m3_decode(c["v"][p, t % ps, h]) * float(c["vs"][p, h])
            assert np.array_equal(got[b, hq], vv)
            s = float(np.float32(0.3)) * float(kv @ c["q"][b, hq])
            w = math.exp(s) / (math.exp(s) + math.exp(float(sinks[hq])))
            assert np.allclose(got_s[b, hq], w * vv, rtol=1e-13, atol=1e-16)


def test_window_two_is_the_two_key_softmax():
    """W = 2: the keys at positions L-2 and L-1, a two-term softmax written
    out by hand."""
    rng = np.random.default_rng(42)
    c = _dense_case(rng, B=2, scale_mode="token", L=(33, 16))
    ps = c["k"].shape[1]
    G = 4
    sm = float(np.float32(0.25))
    got = _run(c, window=2, sm_scale=0.25)
    for b in range(2):
        L = int(c["lens"][b])
        for hq in range(8):
            h = hq // G
            s, vals = [], []
            for t in (L - 2, L - 1):
                p = int(c["table"][b][t // ps])
                kv = O.e4m3_decode(c["k"][p, t % ps, h]) * float(c["ks"][p, t % ps, h])
                vals.append(O.e4m3_decode(c["v"][p, t % ps, h]) * float(c["vs"][p, t % ps, h]))
                s.append(sm * float(kv @ c["q"][b, hq]))
            e0, e1 = math.exp(s[0] - max(s)), math.exp(s[1] - max(s))
            want = (e0 * vals[0] + e1 * vals[1]) / (e0 + e1)
            assert np.allclose(got[b, hq], want, rtol=1e-13, atol=1e-16)


def test_window_of_all_but_one_drops_key_zero():
    """W = L - 1 equals full attention over the sequence with its first key
    removed: the same keys re-stored, one position earlier, in a fresh pool
    (key 0 is left out by slicing the data, not by a window)."""
    rng = np.random.default_rng(43)
    ps, Hkv, D, L = 16, 2, 16, 45
    K = rng.integers(0, 0x70, size=(L, Hkv, D)).astype(np.uint8) | \
        (rng.integers(0, 2, size=(L, Hkv, D)).astype(np.uint8) << 7)
    V = rng.integers(0, 0x70, size=(L, Hkv, D)).astype(np.uint8)
    ks = np.array([0.01, 0.02], np.float32)
    vs = np.array([0.03, 0.005], np.float32)
    q = torch.randn(1, 8, D, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    q = q.double().numpy()

    def paged(keys, vals):
        n = keys.shape[0]
        npg = (n + ps - 1) // ps
        perm = rng.permutation(npg)
        kp = np.zeros((npg, ps, Hkv, D), np.uint8)
        vp = np.zeros((npg, ps, Hkv, D), np.uint8)
        for t in range(n):
            kp[perm[t // ps], t % ps] = keys[t]
            vp[perm[t // ps], t % ps] = vals[t]
        return dict(q=q, k=kp, v=vp, ks=ks, vs=vs, table=perm.astype(np.int32)[None],
                    lens=np.array([n]))

    full = paged(K, V)
    trimmed = paged(K[1:], V[1:])
    sinks = np.linspace(-1, 1, 8).astype(np.float32)
    for sk in (None, sinks):
        a = _run(full, window=L - 1, sinks=sk, sm_scale=0.2)
        b = _run(trimmed, window=0, sinks=sk, sm_scale=0.2)
        assert np.allclose(a, b, rtol=1e-13, atol=1e-16)
        assert not np.allclose(a, _run(full, window=0, sinks=sk, sm_scale=0.2), rtol=1e-6, atol=0)


# ------------------------------------------------- fp8 compute path (opt-in)
# The solution page's "Two compute paths" table and "Limitations": the fp8
# path adds one E4M3 rounding on q and one on p, and is held to 1.5e-1.

def _torch_e4m3(x) -> np.ndarray:
    return torch.tensor(np.asarray(x, dtype=np.float64)).float().to(torch.float8_e4m3fn) \
        .double().numpy()


def test_fp8_query_rounding_matches_library_float8():
    rng = np.random.default_rng(51)
    for trial in range(200):
        row = rng.standard_normal(64) * 10.0 ** rng.uniform(-6, 6)
        row = torch.tensor(row).to(torch.bfloat16).double().numpy()
        amax = np.abs(row).max()
        k = 7 - math.floor(math.log2(amax))           # 2^7 <= amax * 2^k < 2^8
        assert 128 <= amax * 2.0 ** k < 256
        want = _torch_e4m3(row * 2.0 ** k) * 2.0 ** -k
        assert np.array_equal(O.fp8_compute_query(row), want)
    assert np.array_equal(O.fp8_compute_query(np.zeros(8)), np.zeros(8))


def test_fp8_compute_equals_f32_where_nothing_rounds():
    """q = 0 (every weight is exactly 1), a single key (one weight of 1, the
    value alone) and W = 1 give the f32 result exactly."""
    rng = np.random.default_rng(52)
    c = _dense_case(rng, scale_mode="page")
    c0 = dict(c, q=np.zeros_like(c["q"]))
    sinks = np.linspace(-1, 1, 8).astype(np.float32)     # above and below the scores
    for kw in (dict(window=0), dict(window=9, sinks=sinks)):
        assert np.allclose(_run(c0, compute="fp8", **kw), _run(c0, **kw), rtol=1e-14, atol=1e-16)
    c1 = dict(c, lens=np.array([1, 1]))
    assert np.array_equal(_run(c1, compute="fp8"), _run(c1))
    assert np.array_equal(_run(c, window=1, compute="fp8"), _run(c, window=1))


def test_fp8_compute_brute_force_tiny_inputs():
    """Pure-Python softmax with the two roundings done by the library float8
    type: q per row after the power-of-two scale, each weight as w * 2^8."""
    rng = np.random.default_rng(53)
    for trial in range(20):
        D = int(rng.integers(1, 9))
        L = int(rng.integers(2, 9))
        c = _dense_case(rng, B=1, Hq=2, Hkv=1, D=D, ps=16, L=(L,), scale_mode="page")
        sinks = rng.standard_normal(2).astype(np.float32) if trial % 2 else None
        sm = float(np.float32(rng.uniform(0.05, 0.5)))
        got = _run(c, sinks=sinks, sm_scale=sm, compute="fp8")
        for hq in range(2):
            row = c["q"][0, hq]
            amax = float(np.abs(row).max())
            k = 7 - math.floor(math.log2(amax))
            qr = [float(x) for x in _torch_e4m3(row * 2.0 ** k) * 2.0 ** -k]
            s = []
            vals = []
            for t in range(L):
                p = int(c["table"][0][t // 16])
                kv = [e4m3(int(c["k"][p, t % 16, 0, d])) * float(c["ks"][p, 0]) for d in range(D)]
                vals.append([e4m3(int(c["v"][p, t % 16, 0, d])) * float(c["vs"][p, 0]) for d in range(D)])
                s.append(sm * sum(qr[d] * kv[d] for d in range(D)))
            M = max(s)                              # weights against the largest score
            w = [math.exp(x - M) for x in s]
            den = sum(w) + (0.0 if sinks is None else math.exp(float(sinks[hq]) - M))
            wr = [float(_torch_e4m3([x * 256.0])[0]) / 256.0 for x in w]
            want = [sum(wr[t] * vals[t][d] for t in range(L)) / den for d in range(D)]
            assert np.allclose(got[0, hq], want, rtol=1e-12, atol=1e-14)


def test_fp8_compute_stays_within_the_pages_tolerance_of_f32():
    """Serving-like data (K and V drawn N(0,1), quantized with amax / 448
    scales per KV head, q N(0,1) in bf16, sm_scale = D^-0.5): the fp8 path
    is within the page's 1.5e-1 of the f32 path, and differs from it."""
    rng = np.random.default_rng(54)
    for D, L, window, with_sinks in ((64, 300, 0, True), (128, 173, 40, False), (128, 1000, 0, False)):
        B, Hq, Hkv, ps = 2, 8, 2, 16
        npg = (L + ps - 1) // ps
        x = rng.standard_normal((2, B * npg, ps, Hkv, D))
        amax = np.abs(x).max(axis=(1, 2, 4))                       # [2, Hkv]
        sc = (amax / 448.0).astype(np.float32)
        k = O.quantize(x[0], sc[0][None, None, :, None])
        v = O.quantize(x[1], sc[1][None, None, :, None])
        table = rng.permutation(B * npg).astype(np.int32).reshape(B, npg)
        q = torch.randn(B, Hq, D, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16)
        c = dict(q=q.double().numpy(), k=k, v=v, ks=sc[0], vs=sc[1], table=table,
                 lens=np.array([L, L - 7]))
        sinks = rng.standard_normal(Hq).astype(np.float32) if with_sinks else None
        f32 = _run(c, window=window, sinks=sinks, sm_scale=D ** -0.5)
        f8 = _run(c, window=window, sinks=sinks, sm_scale=D ** -0.5, compute="fp8")
        err = np.abs(f8 - f32) / np.maximum(1.0, np.abs(f32))
        assert err.max() <= 1.5e-1, err.max()
        assert err.max() > 0.0                      # the roundings do change the result


# ------------------------------------------- context-parallel partials + combine
# Splitting a sequence's keys over GPUs and merging the slices' partial
# results must give the attention over all keys (the log-sum-exp combine of
# splits). The pins check the oracle's partial and combine against the full
# attention (pinned above), not against themselves.

def _partition(rng, L, R, ps, aligned=True):
    """R contiguous slices covering [0, L): page-aligned cut points, or
    arbitrary ones; some slices may be empty."""
    cuts = rng.integers(0, L + 1, size=R - 1)
    if aligned:
        cuts = (cuts // ps) * ps
    cuts = np.sort(np.concatenate([[0], cuts, [L]]))
    return [(int(cuts[i]), int(cuts[i + 1])) for i in range(R)]


@pytest.mark.parametrize("window,with_sinks", [(0, False), (0, True), (50, True), (7, False)])
def test_combined_partials_over_any_partition_equal_full_attention(window, with_sinks):
    rng = np.random.default_rng(61 + window)
    c = _dense_case(rng, B=3, L=(120, 77, 33), scale_mode="page")
    sinks = rng.standard_normal(8).astype(np.float32) if with_sinks else None
    want = _run(c, window=window, sinks=sinks, sm_scale=0.3)
    for R, aligned in ((1, True), (2, True), (3, False), (8, True), (8, False)):
        ranges = [_partition(rng, int(L), R, 16, aligned) for L in c["lens"]]
        parts = [O.paged_decode_partial(c["q"], c["k"], c["v"], c["ks"], c["vs"], c["table"],
                                        c["lens"], np.array([ranges[b][r] for b in range(3)]),
                                        window=window, sm_scale=0.3) for r in range(R)]
        got = O.combine_partials(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]),
                                 sinks)
        assert np.allclose(got, want, rtol=1e-12, atol=1e-14), (R, aligned)


def test_partial_closed_forms():
    """q = 0: every score is 0, so m = 0, l = the slice's key count and o the
    plain sum of its values; an empty slice gives (-inf, 0, 0) and adds
    nothing to a combine."""
    rng = np.random.default_rng(62)
    c = _dense_case(rng, B=2, L=(90, 40), scale_mode="head")
    c0 = dict(c, q=np.zeros_like(c["q"]))
    kr = np.array([[16, 70], [0, 40]])
    o, ml = O.paged_decode_partial(c0["q"], c0["k"], c0["v"], c0["ks"], c0["vs"], c0["table"],
                                   c0["lens"], kr)
    G, ps = 4, 16
    for b in range(2):
        t = np.arange(kr[b][0], kr[b][1])
        phys = c["table"][b][t // ps]
        for hq in range(8):
            V = O.e4m3_decode(c["v"][phys, t % ps, hq // G]) * float(c["vs"][hq // G])
            assert ml[b, hq, 0] == 0.0 and ml[b, hq, 1] == len(t)
            assert np.allclose(o[b, hq], V.sum(0), rtol=1e-13, atol=1e-15)
    o_e, ml_e = O.paged_decode_partial(c["q"], c["k"], c["v"], c["ks"], c["vs"], c["table"],
                                       c["lens"], np.array([[5, 5], [40, 90]]))
    assert np.all(ml_e[:, :, 0] == -np.inf) and np.all(ml_e[:, :, 1] == 0) and np.all(o_e == 0)
    full = O.paged_decode_partial(c["q"], c["k"], c["v"], c["ks"], c["vs"], c["table"], c["lens"])
    both = O.combine_partials(np.stack([full[0], o_e]), np.stack([full[1], ml_e]))
    assert np.array_equal(both, O.combine_partials(full[0][None], full[1][None]))


# ------------------------------------------------------------------ MXFP8
# The OCP microscaling reading of the MXFP8 cache: E4M3 elements in blocks of
# 32 entries sharing one E8M0 scale. Pins: the library's own E8M0 and E4M3
# types, the scale rule written out from its definition, and attention over
# values dequantized through the library types.

def test_e8m0_decode_matches_library_type_on_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e8m0fnu).double().numpy()
    assert np.array_equal(O.e8m0_decode(codes), lib, equal_nan=True)
    assert O.e8m0_decode(127) == 1.0 and O.e8m0_decode(0) == 2.0 ** -127
    assert np.isnan(O.e8m0_decode(255))


def test_mx_quantize_matches_the_library_casts():
    """Scale: the block's largest magnitude, divided by the scale, lies in
    [2^8, 2^9) (2^8 = E4M3's largest binade); codes: the library's E4M3 cast of
    the clamped quotient."""
    rng = np.random.default_rng(81)
    for trial in range(40):
        D = int(rng.choice([32, 64, 128, 256, 512]))
        x = (rng.standard_normal((3, D)) * 10.0 ** rng.uniform(-8, 8)).astype(np.float32)
        x[0, :32] *= 0                                       # an all-zero block
        codes, sc = O.mx_quantize(x)
        assert sc.shape == (3, D // 32) and sc.dtype == np.uint8
        assert sc[0, 0] == 127
        scale = torch.from_numpy(sc).view(torch.float8_e8m0fnu).double().numpy()
        blocks = x.astype(np.float64).reshape(3, D // 32, 32)
        amax = np.abs(blocks).max(-1)
        nz = amax > 0
        ratio = amax[nz] / scale[nz]
        assert np.all((ratio >= 256) & (ratio < 512))
        q = np.clip(blocks / scale[..., None], -448, 448).reshape(3, D)
        want = torch.from_numpy(q).float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(codes, want)


@pytest.mark.parametrize("window,with_sinks", [(0, False), (40, True)])
def test_mx_attention_matches_library_sdpa(window, with_sinks):
    """K and V in MXFP8 (codes and E8M0 block scales, as mx_quantize writes
    them): the oracle against torch SDPA over values dequantized with the
    library's float8 types, one scale per 32-entry block."""
    rng = np.random.default_rng(82)
    B, Hq, Hkv, D, ps = 2, 8, 2, 64, 16
    lens = np.array([70, 33])
    npg = (lens + ps - 1) // ps
    total = int(npg.sum()) + 2
    perm = rng.permutation(total)
    table = np.full((B, npg.max()), -1, np.int32)
    off = 0
    for b in range(B):
        table[b, :npg[b]] = perm[off:off + npg[b]]
        off += npg[b]
    xk = rng.standard_normal((total, ps, Hkv, D)) * np.exp(rng.uniform(-3, 3, (total, ps, Hkv, 1)))
    xv = rng.standard_normal((total, ps, Hkv, D)) * np.exp(rng.uniform(-3, 3, (total, ps, Hkv, 1)))
    k, ks = O.mx_quantize(xk)
    v, vs = O.mx_quantize(xv)
    q = torch.randn(B, Hq, D, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).double()
    sinks = rng.standard_normal(Hq).astype(np.float32) if with_sinks else None
    sm = 0.15
    got = O.paged_decode_attention(q.numpy(), k, v, ks, vs, table, lens, window=window,
                                   sinks=sinks, sm_scale=sm)
    deq = lambda c, s: (torch.from_numpy(c).view(torch.float8_e4m3fn).double() *  # noqa: E731
                        torch.from_numpy(s).view(torch.float8_e8m0fnu).double()
                        .repeat_interleave(32, dim=-1))
    K, V = deq(k, ks), deq(v, vs)
    G = Hq // Hkv
    for b in range(B):
        L = int(lens[b])
        lo = max(0, L - window) if window else 0
        t = np.arange(L)
        phys = table[b][t // ps]
        Kb = K[phys, t % ps].permute(1, 0, 2).repeat_interleave(G, 0)   # [Hq, L, D]
        Vb = V[phys, t % ps].permute(1, 0, 2).repeat_interleave(G, 0)
        mask = torch.zeros(Hq, 1, L + 1, dtype=torch.float64)
        mask[:, :, :lo] = -math.inf
        mask[:, :, L] = -math.inf if sinks is None else torch.from_numpy(sinks).double()[:, None]
        Kb = torch.cat([Kb, torch.zeros(Hq, 1, D, dtype=torch.float64)], 1)
        Vb = torch.cat([Vb, torch.zeros(Hq, 1, D, dtype=torch.float64)], 1)
        o = torch.nn.functional.scaled_dot_product_attention(q[b][:, None, :], Kb, Vb,
                                                             attn_mask=mask,
                                                             scale=float(np.float32(sm)))
        assert np.allclose(got[b], o[:, 0].numpy(), rtol=1e-12, atol=1e-12)


def test_mx_append_writes_the_tokens_block_scales_and_codes():
    rng = np.random.default_rng(83)
    B, Hkv, D, ps, P = 3, 2, 128, 16, 9
    kp = rng.integers(0, 256, (P, ps, Hkv, D)).astype(np.uint8)
    vp = kp.copy()
    ks = rng.integers(0, 255, (P, ps, Hkv, D // 32)).astype(np.uint8)
    vs = ks.copy()
    table = rng.permutation(P)[:B * 3].reshape(B, 3).astype(np.int32)
    pos = np.array([5, 16, 47])
    kn = torch.randn(B, Hkv, D).to(torch.bfloat16).double().numpy() * 3
    vn = torch.randn(B, Hkv, D).to(torch.bfloat16).double().numpy() * 1e-3
    kp0, vp0, ks0, vs0 = kp.copy(), vp.copy(), ks.copy(), vs.copy()
    O.kv_append(kn, vn, kp, vp, ks, vs, table, pos)
    touched = np.zeros((P, ps), bool)
    for b in range(B):
        page, slot = table[b][pos[b] // ps], pos[b] % ps
        touched[page, slot] = True
        for new, pages, sc in ((kn, kp, ks), (vn, vp, vs)):
            c, s = O.mx_quantize(new[b])
            assert np.array_equal(pages[page, slot], c) and np.array_equal(sc[page, slot], s)
    for a, a0 in ((kp, kp0), (vp, vp0), (ks, ks0), (vs, vs0)):
        assert np.array_equal(a[~touched], a0[~touched])
