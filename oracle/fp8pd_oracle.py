"""Plain CPU oracle for FP8 (E4M3) paged decode attention and KV append.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module:
only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` call it. It shares no code with the
CUDA library; it is a slow, literal restatement of what the method computes.

Sources (the pages this restates):

* P1 = "How do I run paged decode attention over an FP8 KV cache for a
  quantized MoE serving path, with sliding windows, attention sinks and a
  custom scale?" (cerinamroth.com solution page for ``fp8_paged_decode_attention``).
* P2 = "Lecture 8 -- Inference Path: KV Cache, Decode, RoPE, GQA, Paged KV"
  (FlashAttention Course).
* E4M3 itself is only named by the pages; its values are those of the OCP
  8-bit floating point format E4M3 (1 sign bit, 4 exponent bits with bias 7,
  3 mantissa bits, subnormals, no infinities, S.1111.111 is NaN).

Arithmetic is float64 except where the method fixes the precision: the
quantizer divides in IEEE float32 (the stored code is a function of the
float32 quotient), then rounds that quotient to the E4M3 grid exactly.

Readings of the pages (each is listed with its reason in the design notes):

* window W > 0 keeps the last W keys, i.e. positions t with t > (L-1) - W;
  W = 0 keeps all keys (P1 "Expected result": ``window=W`` restricts each
  query to the last W keys).
* a sink is one extra logit per query head, in the same units as the scaled
  scores, added to the softmax denominator with no value (P1 "Expected
  result", the gpt-oss ``s_aux`` convention).
* ``sm_scale`` multiplies q.k and replaces D**-0.5 (P1 "Expected result").
* query head h uses KV head h // G, G = Hq / Hkv (P1 "Smallest correct
  example", ``q.view(H_KV, H_Q // H_KV, D)``; P2 "MQA / GQA").
* token t of sequence b lives in physical page block_table[b, t // ps] at
  slot t % ps (P2 "Paged KV cache").
* a K/V scale is indexed by the physical page id and the KV head; a
  per-KV-head scale is the same array broadcast over pages. The
  per-token-per-head form (P1 "Supported scope", ``quantize_kv_fp8``) keeps
  one scale per stored (page, slot, KV head), shaped like the cache without
  its last axis, and is max|x| / 448 of that token and head in float32 (an
  all-zero row takes scale 1); the append writes it with the codes. Sub-row
  groups (P1 "Supported scope", ``k_groups``) add a last axis of ``groups``
  scales, group g covering entries [g D/groups, (g+1) D/groups).
* empty attention (no keys, no sink) returns 0.
* MXFP8 (P3, "Attention MXFP8 TKG", decode attention over an MXFP8 KV
  cache; the page names the format without spelling it out): the OCP
  microscaling format, E4M3 elements in blocks of 32 consecutive entries
  that share one E8M0 scale 2^(c - 127) (c = 255 is NaN). A cache row of D
  entries per (token, KV head) has D / 32 scale bytes, stored as a uint8
  array [num_pages, ps, Hkv, D / 32] beside the codes. A block's scale is
  2^(floor(log2 max|x|) - 8) (8 = E4M3's largest exponent; all-zero block:
  2^0), clamped to the E8M0 range, and its codes are E4M3 of x / scale,
  saturating at 448.
* the opt-in "fp8 compute" path (P1 "Two compute paths", ``compute="fp8"``,
  and "Limitations": it adds one E4M3 rounding on q and on p) rounds each
  query row to E4M3 after a power-of-two scale that puts its largest
  magnitude in [2^7, 2^8), and each softmax weight p_t = exp(s_t - M_s)
  taken against the largest score M_s (at most 1) to E4M3 as p_t * 2^8, in
  the weighted sum of values only; the denominator sums the unrounded
  weights and the sink's exp(sink - M_s).
"""

from __future__ import annotations

import math

import numpy as np

E4M3_MAX = 448.0
E4M3_NAN_CODE = 0x7F


# ---------------------------------------------------------------------------
# E4M3 codec
# ---------------------------------------------------------------------------

def e4m3_code_value(code: int) -> float:
    """Value of one E4M3 code from the format's closed form (OCP E4M3).

    sign s = bit 7, exponent e = bits 6..3 (bias 7), mantissa m = bits 2..0:
      e == 0            -> (-1)^s * (m / 8) * 2^(1 - 7)      (subnormal)
      e == 15, m == 7   -> NaN
      otherwise         -> (-1)^s * (1 + m / 8) * 2^(e - 7)
    """
    s = (code >> 7) & 1
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        mag = (m / 8.0) * 2.0 ** (1 - 7)
    else:
        mag = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


#: float64 value of every code 0..255 (NaN for 0x7F and 0xFF).
E4M3_TABLE = np.array([e4m3_code_value(c) for c in range(256)], dtype=np.float64)

#: the 127 non-negative finite values, codes 0x00..0x7E, strictly increasing.
_E4M3_POS = E4M3_TABLE[:0x7F].copy()


def e4m3_decode(codes) -> np.ndarray:
    """Decode uint8 E4M3 codes to float64 values."""
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(values) -> np.ndarray:
    """Round real values to E4M3 codes: nearest grid value, ties to an even
    mantissa, saturating to +-448.

    The grid in the binade [2^e, 2^(e+1)) for e >= -6 has spacing 2^(e-3);
    below 2^-6 (subnormals) the spacing is 2^-9, the same as the e = -6
    binade, so the spacing is 2^(max(e, -6) - 3) everywhere. A value divided
    by its spacing is exact (power of two), and rounding that quotient to the
    nearest integer with ties to even picks the neighbour whose code has an
    even mantissa. A result above 448 (including +-Inf) saturates to 448.
    NaN maps to the NaN code with the input's sign; -0 keeps its sign.
    """
    v = np.asarray(values, dtype=np.float64)
    flat = v.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint8)
    sign = np.signbit(flat)
    a = np.abs(flat)
    is_nan = np.isnan(flat)
    finite = np.isfinite(a)

    mag = np.full(flat.shape, E4M3_MAX)          # Inf and huge values saturate
    af = np.where(finite & ~is_nan, a, 0.0)
    _, ex = np.frexp(af)                          # af = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)                    # binade exponent, floored at -6
    spacing = np.ldexp(1.0, e - 3)
    r = np.rint(af / spacing)                     # round half to even
    rounded = r * spacing
    sel = finite & ~is_nan
    mag[sel] = np.minimum(rounded[sel], E4M3_MAX)

    idx = np.searchsorted(_E4M3_POS, mag)
    idx = np.minimum(idx, 0x7E)
    if not np.all(_E4M3_POS[idx[sel | ~finite]] == mag[sel | ~finite]):
        raise AssertionError("e4m3_encode: rounded value is not on the grid")
    out[:] = idx.astype(np.uint8)
    out[is_nan] = E4M3_NAN_CODE
    out |= (sign.astype(np.uint8) << 7)
    return out.reshape(v.shape)


def quantize(x, scale) -> np.ndarray:
    """E4M3 code of x / scale, the quotient taken in IEEE float32.

    ``x`` holds bf16 or float32 values (exact in float32); ``scale`` is a
    float32 array broadcastable to ``x``. The division is float32
    round-to-nearest (numpy float32 division; no flush to zero), then the
    float32 quotient is rounded to E4M3 exactly by :func:`e4m3_encode`.
    """
    x32 = np.asarray(x, dtype=np.float32)
    s32 = np.asarray(scale, dtype=np.float32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        quot = np.divide(x32, s32, dtype=np.float32)
    return e4m3_encode(quot.astype(np.float64))


def token_scale(x) -> np.ndarray:
    """Per-token-per-head scale of ``x`` [..., D]: max_d |x| / 448 in float32.

    P1 "Supported scope" names ``quantize_kv_fp8`` as per-token-per-head E4M3
    with an fp32 scale; the scale that maps each row's largest magnitude onto
    the largest finite E4M3 value (448) is the plainest reading. The maximum
    skips NaN entries; a row whose maximum is 0 takes scale 1 (its codes are
    then signed zeros). The division is IEEE float32.
    """
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.fmax.reduce(np.abs(x32), axis=-1)          # fmax: NaN entries are skipped
    amax = np.where(np.isnan(amax), np.float32(0.0), amax).astype(np.float32)
    with np.errstate(over="ignore"):
        s = np.divide(amax, np.float32(E4M3_MAX), dtype=np.float32)
    return np.where(amax == 0, np.float32(1.0), s).astype(np.float32)


def quantize_per_token(x) -> tuple[np.ndarray, np.ndarray]:
    """(codes, scales) of ``x`` [..., D] with one scale per row (token, head):
    scales = :func:`token_scale`, codes = :func:`quantize` of x / scale."""
    s = token_scale(x)
    return quantize(x, s[..., None]), s


def group_scale(x, groups: int) -> np.ndarray:
    """Sub-row scales of ``x`` [..., D]: the D values of a row cut into
    ``groups`` equal runs of D / groups consecutive entries, each with its own
    :func:`token_scale`. Returns [..., groups] (P1 "Supported scope":
    ``k_groups`` sub-row key scales, ``quantize_kv_fp8`` with sub-row groups).
    """
    x32 = np.asarray(x, dtype=np.float32)
    D = x32.shape[-1]
    if groups < 1 or D % groups:
        raise ValueError("groups must divide the head dim")
    return token_scale(x32.reshape(*x32.shape[:-1], groups, D // groups))


MX_BLOCK = 32


def e8m0_decode(codes) -> np.ndarray:
    """E8M0 scale codes to float64: 2^(c - 127), NaN for 255."""
    c = np.asarray(codes, dtype=np.int64)
    return np.where(c == 255, np.nan, np.exp2((c - 127).astype(np.float64)))


def mx_scale_code(block) -> int:
    """E8M0 code of one block's shared scale: c = floor(log2 max|x|) - 8 +
    127, clamped to [0, 254]; NaN entries are skipped and an all-zero block
    takes c = 127 (scale 1)."""
    a = np.abs(np.asarray(block, dtype=np.float64))
    a = a[~np.isnan(a)]
    amax = float(a.max()) if a.size else 0.0
    if amax == 0.0:
        return 127
    if not math.isfinite(amax):
        return 254
    _, e = math.frexp(amax)            # amax in [2^(e-1), 2^e)
    return int(min(254, max(0, (e - 1) - 8 + 127)))


def mx_quantize(x) -> tuple[np.ndarray, np.ndarray]:
    """MXFP8 quantization of rows x [..., D] (D a multiple of 32): returns
    (E4M3 codes [..., D], E8M0 scale codes [..., D / 32]). Each element is
    E4M3(x / 2^(c - 127)) of float32 x, the division by a power of two exact
    in float64, rounded to nearest even and saturated at 448."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    D = x.shape[-1]
    if D % MX_BLOCK:
        raise ValueError("D must be a multiple of 32")
    blocks = x.reshape(x.shape[:-1] + (D // MX_BLOCK, MX_BLOCK))
    sc = np.zeros(blocks.shape[:-1], dtype=np.uint8)
    for idx in np.ndindex(*sc.shape):
        sc[idx] = mx_scale_code(blocks[idx])
    scale = np.exp2(sc.astype(np.float64) - 127.0)[..., None]
    codes = e4m3_encode(blocks / scale).reshape(x.shape)
    return codes, sc


def expand_groups(scales: np.ndarray, D: int) -> np.ndarray:
    """[..., groups] sub-row scales -> [..., D]: entry d takes the scale of its
    group d // (D / groups)."""
    scales = np.asarray(scales)
    return np.repeat(scales, D // scales.shape[-1], axis=-1)


# ---------------------------------------------------------------------------
# Paged gather, attention and append
# ---------------------------------------------------------------------------

def _scale_of(scale: np.ndarray, page: np.ndarray, slot: np.ndarray, head: int) -> np.ndarray:
    """Scale of the token stored at (physical page, slot) for KV head ``head``:
    ``scale`` is [Hkv] (per KV head), [num_pages, Hkv] (per physical page and
    KV head) or [num_pages, ps, Hkv] (per stored token and KV head). With
    [num_pages, ps, Hkv, groups] (sub-row groups) the result has a trailing
    axis of the token's group scales."""
    scale = np.asarray(scale)
    if scale.dtype == np.uint8:  # MXFP8: E8M0 block scales [num_pages, ps, Hkv, D / 32]
        return e8m0_decode(scale[page, slot, head, :])
    if scale.ndim == 1:
        return np.full(np.shape(page), np.float64(scale[head]))
    if scale.ndim == 2:
        return scale[page, head].astype(np.float64)
    if scale.ndim == 3:
        return scale[page, slot, head].astype(np.float64)
    return scale[page, slot, head, :].astype(np.float64)


def _dequantize(codes: np.ndarray, scale: np.ndarray, page, slot, head: int) -> np.ndarray:
    """Values of the codes [n, D] of KV head ``head`` stored at (page, slot):
    decode(code) times the scale of each entry (a group scale, when the scale
    array has sub-row groups, covers its run of D / groups entries)."""
    s = _scale_of(scale, page, slot, head)
    D = codes.shape[-1]
    s = expand_groups(s, D) if np.ndim(scale) == 4 else s[..., None]
    return e4m3_decode(codes) * s


def gather_tokens(pages: np.ndarray, block_table_row: np.ndarray, positions: np.ndarray,
                  head: int) -> tuple[np.ndarray, np.ndarray]:
    """Codes of KV head ``head`` at logical token ``positions`` of one sequence.

    ``pages`` is the layer's view [num_pages, ps, Hkv, D] of the pool (any
    strides). Token t is in physical page block_table_row[t // ps], slot
    t % ps. Returns (codes [n, D] uint8, physical page of each token [n]).
    """
    ps = pages.shape[1]
    phys = np.asarray(block_table_row)[positions // ps].astype(np.int64)
    slots = positions % ps
    return pages[phys, slots, head, :], phys


def attended_range(seq_len: int, window: int) -> tuple[int, int]:
    """Keys [lo, L) a decode query at position L-1 attends to."""
    L = int(seq_len)
    lo = max(0, L - int(window)) if window > 0 else 0
    return lo, L


def e4m3_round(x) -> np.ndarray:
    """x rounded to the nearest E4M3 value (ties to an even mantissa,
    saturating to +-448), as float64."""
    return e4m3_decode(e4m3_encode(x))


def fp8_compute_query(q_row) -> np.ndarray:
    """One E4M3 rounding of a query row (the fp8 compute path): scaled by
    2^k so that its largest magnitude lies in [2^7, 2^8), rounded, scaled
    back. A zero row stays zero."""
    q_row = np.asarray(q_row, dtype=np.float64)
    amax = float(np.max(np.abs(q_row))) if q_row.size else 0.0
    if amax == 0.0 or not math.isfinite(amax):
        return q_row.copy()
    _, e = math.frexp(amax)                 # amax in [2^(e-1), 2^e)
    k = 8 - e
    return e4m3_round(q_row * 2.0 ** k) * 2.0 ** -k


def paged_decode_attention(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens,
                           window: int = 0, sinks=None, sm_scale: float | None = None,
                           batch_heads=None, compute: str = "f32") -> np.ndarray:
    """Single-query attention over a paged E4M3 KV cache, float64.

    q [B, Hq, D] (bf16 values given as floats), k_pages / v_pages
    [num_pages, ps, Hkv, D] uint8 codes, k_scale / v_scale [Hkv],
    [num_pages, Hkv] or [num_pages, ps, Hkv] float32, or
    [num_pages, ps, Hkv, groups] (sub-row groups of D / groups entries),
    block_table [B, max_pages] int32, seq_lens [B] = number of keys 0..L-1 visible to the query,
    sinks [Hq] float32 or None. Returns out [B, Hq, D] float64.

    For each (b, hq), with h = hq // G and keys t in [lo, L):
      s_t  = sm_scale * sum_d q[b,hq,d] * K(t,d)
      M    = max(max_t s_t, sink)
      out  = sum_t exp(s_t - M) V(t) / (sum_t exp(s_t - M) + exp(sink - M))
    where K(t,d) = decode(code) * k_scale(page(t), slot(t), h[, d // (D / groups)]). This is plain softmax
    attention over the dequantized values (P1 "Smallest correct example"),
    with the window, sinks and scale of P1 "Expected result".

    ``batch_heads``: optional list of (b, hq) pairs; only those outputs are
    computed (the others stay 0), for sampled checks at full size.

    ``compute="fp8"`` is P1's fp8 compute path: q is replaced by
    :func:`fp8_compute_query` of its row, the weights are taken against the
    largest score, w_t = exp(s_t - max_t s_t), and in the numerator each is
    replaced by E4M3(w_t * 2^8) / 2^8; the denominator is
    sum_t w_t + exp(sink - max_t s_t).
    """
    if compute not in ("f32", "fp8"):
        raise ValueError(compute)
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    Hkv = k_pages.shape[2]
    G = Hq // Hkv
    if sm_scale is None:
        sm_scale = D ** -0.5
    sm = float(np.float32(sm_scale))
    out = np.zeros((B, Hq, D), dtype=np.float64)
    if batch_heads is None:
        wanted = {(b, hq) for b in range(B) for hq in range(Hq)}
    else:
        wanted = {(int(b), int(hq)) for b, hq in batch_heads}
    for b in range(B):
        lo, L = attended_range(int(seq_lens[b]), int(window))
        positions = np.arange(lo, L, dtype=np.int64)
        for h in range(Hkv):
            heads = [h * G + g for g in range(G) if (b, h * G + g) in wanted]
            if not heads:
                continue
            kc, phys = gather_tokens(k_pages, block_table[b], positions, h)
            vc, _ = gather_tokens(v_pages, block_table[b], positions, h)
            slots = positions % k_pages.shape[1]
            K = _dequantize(kc, k_scale, phys, slots, h)
            V = _dequantize(vc, v_scale, phys, slots, h)
            for hq in heads:
                qrow = fp8_compute_query(q[b, hq]) if compute == "fp8" else q[b, hq]
                s = sm * (K @ qrow)
                sink = None if sinks is None else float(sinks[hq])
                m_keys = s.max() if s.size else -math.inf
                M = m_keys if sink is None else max(m_keys, sink)
                if compute == "fp8" and s.size:
                    M = m_keys  # the rounded weights are taken against the largest score
                if M == -math.inf:
                    continue                       # no keys and no finite sink: 0
                w = np.exp(s - M)
                den = w.sum() + (0.0 if sink is None else math.exp(sink - M))
                wv = e4m3_round(w * 2.0 ** 8) * 2.0 ** -8 if compute == "fp8" else w
                if den > 0.0:
                    out[b, hq] = (wv @ V) / den
    return out


LOG2E = 1.0 / math.log(2.0)


def paged_decode_partial(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens,
                         key_ranges=None, window: int = 0, sm_scale: float | None = None):
    """Unnormalized attention over a slice of each sequence's keys (one GPU's
    share of a context-parallel split), float64.

    Keys: the window's range [lo, L) of :func:`attended_range` cut to
    [key_ranges[b, 0], key_ranges[b, 1]) (all of it when key_ranges is None).
    With s_t the scaled scores of those keys (as in
    :func:`paged_decode_attention`, no sink) and m = max_t s_t:
      ml[b, hq] = (m * log2(e), sum_t exp(s_t - m)),  o[b, hq] = sum_t exp(s_t - m) V(t);
    (-inf, 0) and 0 with no keys. Returns (o [B, Hq, D], ml [B, Hq, 2]).
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    Hkv = k_pages.shape[2]
    G = Hq // Hkv
    if sm_scale is None:
        sm_scale = D ** -0.5
    sm = float(np.float32(sm_scale))
    o = np.zeros((B, Hq, D))
    ml = np.zeros((B, Hq, 2))
    ml[:, :, 0] = -math.inf
    for b in range(B):
        lo, L = attended_range(int(seq_lens[b]), int(window))
        if key_ranges is not None:
            lo, L = max(lo, int(key_ranges[b][0])), min(L, int(key_ranges[b][1]))
        if L <= lo:
            continue
        positions = np.arange(lo, L, dtype=np.int64)
        for h in range(Hkv):
            kc, phys = gather_tokens(k_pages, block_table[b], positions, h)
            vc, _ = gather_tokens(v_pages, block_table[b], positions, h)
            slots = positions % k_pages.shape[1]
            K = _dequantize(kc, k_scale, phys, slots, h)
            V = _dequantize(vc, v_scale, phys, slots, h)
            for hq in range(h * G, (h + 1) * G):
                s = sm * (K @ q[b, hq])
                m = s.max()
                w = np.exp(s - m)
                o[b, hq] = w @ V
                ml[b, hq] = (m * LOG2E, w.sum())
    return o, ml


def combine_partials(part_o, part_ml, sinks=None) -> np.ndarray:
    """The log-sum-exp combine of R partials (as :func:`paged_decode_partial`
    writes them) into the attention output, the sink added once:
    M = max(max_r m_r, sink log2 e), den = sum_r l_r 2^(m_r - M) + 2^(sink log2 e - M),
    out = sum_r o_r 2^(m_r - M) / den, 0 when den is 0. part_o [R, B, Hq, D],
    part_ml [R, B, Hq, 2]."""
    part_o = np.asarray(part_o, dtype=np.float64)
    part_ml = np.asarray(part_ml, dtype=np.float64)
    R, B, Hq, D = part_o.shape
    out = np.zeros((B, Hq, D))
    for b in range(B):
        for hq in range(Hq):
            m = part_ml[:, b, hq, 0]
            sl = -math.inf if sinks is None else float(sinks[hq]) * LOG2E
            M = max(float(m.max()), sl)
            if M == -math.inf:
                continue
            w = np.where(m == -math.inf, 0.0, np.exp2(np.where(m == -math.inf, 0.0, m) - M))
            den = float((w * part_ml[:, b, hq, 1]).sum()) + (0.0 if sinks is None else 2.0 ** (sl - M))
            if den > 0.0:
                out[b, hq] = (w[:, None] * part_o[:, b, hq]).sum(0) / den
    return out


def kv_append(k_new, v_new, k_pages, v_pages, k_scale, v_scale, block_table, positions) -> None:
    """Quantize one new token per sequence and store it in its page, in place.

    k_new / v_new [B, Hkv, D] (bf16 values as floats), pages
    [num_pages, ps, Hkv, D] uint8 (numpy arrays, written in place), scales
    [Hkv], [num_pages, Hkv], [num_pages, ps, Hkv] or
    [num_pages, ps, Hkv, groups] float32, positions [B].
    Token position p of sequence b goes to page block_table[b, p // ps], slot
    p % ps, as code = E4M3(float32(x) / scale) (P1 "Supported scope", the
    one-launch T=1 append; P2 "In-kernel KV cache update"). A per-head or
    per-page scale is read only. A per-token scale is the new token's own
    (:func:`token_scale` of its D values, per KV head) and is written to
    ``scale[page, slot, h]`` with the codes; with sub-row groups each group's
    scale (:func:`group_scale`) is written to ``scale[page, slot, h, g]`` and
    quantizes its run of entries.
    """
    B, Hkv, _ = np.shape(k_new)
    ps = k_pages.shape[1]
    for b in range(B):
        p = int(positions[b])
        page = int(block_table[b][p // ps])
        slot = p % ps
        for h in range(Hkv):
            for x, pages, scale in ((k_new[b][h], k_pages, k_scale), (v_new[b][h], v_pages, v_scale)):
                x32 = np.asarray(x, np.float32)
                if np.asarray(scale).dtype == np.uint8:   # MXFP8: the token's own block scales
                    codes, sc = mx_quantize(x32)
                    scale[page, slot, h, :] = sc
                    pages[page, slot, h, :] = codes
                    continue
                if np.ndim(scale) == 4:
                    scale[page, slot, h, :] = group_scale(x32, np.shape(scale)[3])
                    s = expand_groups(np.asarray(scale[page, slot, h, :], np.float32), x32.shape[-1])
                    pages[page, slot, h, :] = quantize(x32, s)
                    continue
                if np.ndim(scale) == 3:
                    scale[page, slot, h] = token_scale(x32)
                s = np.float32(_scale_of(scale, np.array(page), np.array(slot), h))
                pages[page, slot, h, :] = quantize(x32, s)
