"""Seeded synthetic workloads for FP8 paged decode attention.

This module is shared by the tests, the benchmark and the oracle checks, and
holds none of the attention method's arithmetic: it draws random numbers,
lays out block tables and pools, applies each workload's scale recipe
(amax / 448 per KV head, or per physical page and KV head) and stores the
cache contents with PyTorch's own ``float8_e4m3fn`` conversion, a library
routine. The K/V codes it produces are *inputs* to the attention under test;
the append under test quantizes the new token itself.

The workloads follow the serving shapes the method is used for (the
"FP8 paged attention for MoE serving" solution page names Granite, Gemma-4
sliding + full layers sharing one pool, and gpt-oss with sinks; the
"Lecture 8 -- Inference Path" page gives the GQA Llama-style shape and
16-token pages). No dataset is involved; every value is drawn here.
"""

from __future__ import annotations

import dataclasses

from dataclasses import dataclass, field

import numpy as np
import torch

E4M3_MAX = 448.0


@dataclass(frozen=True)
class LayerSpec:
    """One attention layer reading the pool: heads, head dim, window."""
    Hq: int
    Hkv: int
    D: int
    window: int = 0
    sm_scale: float | None = None      # None -> D ** -0.5


@dataclass(frozen=True)
class Spec:
    name: str
    B: int
    ps: int
    layers: tuple                       # tuple[LayerSpec, ...]; >1 = layers sharing one pool
    seq_len: int | tuple = 256          # int, or (lo, hi) inclusive uniform range per sequence
    scale_mode: str = "head"            # "head": [Hkv]; "page": [num_pages, Hkv]; "token": [num_pages, ps, Hkv];
                                        # "mx": MXFP8, uint8 E8M0 [num_pages, ps, Hkv, D / 32] for K and V
    k_groups: int = 1                   # "token" only: K scales [num_pages, ps, Hkv, k_groups] when > 1
    dist: str = "normal"                # "normal": N(0,1); "normal2_outliers": N(0,2), 1% x20
    sinks: bool = False
    append: bool = False                # one new token per sequence at position seq_len
    pool_pages: int | None = None       # pool size; None -> exactly the pages the tables use
    seed: int = 0


SPECS: dict[str, Spec] = {
    # B=1, Hq=8, Hkv=2, D=64, 16-token pages, 256 tokens on 16 of 32 pages.
    "tiny": Spec("tiny", B=1, ps=16, layers=(LayerSpec(8, 2, 64, 0, 1 / 8),),
                 seq_len=256, scale_mode="head", pool_pages=32, seed=1),
    # Llama-3-8B-like layer: GQA 32/8, D=128, lengths U[512, 4096], per-page scales, append.
    "llama": Spec("llama", B=32, ps=16, layers=(LayerSpec(32, 8, 128, 0, 128 ** -0.5),),
                  seq_len=(512, 4096), scale_mode="page", append=True, seed=2),
    # gpt-oss-like: 64/8 heads, D=64, 8192 tokens, sinks; window 128 and full.
    "gptoss_w128": Spec("gptoss_w128", B=64, ps=16, layers=(LayerSpec(64, 8, 64, 128, 1 / 8),),
                        seq_len=8192, scale_mode="head", sinks=True, seed=3),
    "gptoss_full": Spec("gptoss_full", B=64, ps=16, layers=(LayerSpec(64, 8, 64, 0, 1 / 8),),
                        seq_len=8192, scale_mode="head", sinks=True, seed=3),
    # Gemma-like mixed pool: a sliding layer and a full layer share one pool of
    # 32-token pages whose stride is the larger layer's page (65,536 bytes).
    "mixed": Spec("mixed", B=16, ps=32,
                  layers=(LayerSpec(16, 8, 256, 1024, 1 / 128), LayerSpec(16, 2, 512, 0, 1 / 128)),
                  seq_len=(2048, 16384), scale_mode="page", dist="normal2_outliers", seed=4),
    # Long context, split-KV: 131,072 tokens, 64-token pages, append.
    "long_b1": Spec("long_b1", B=1, ps=64, layers=(LayerSpec(64, 8, 128, 0, 128 ** -0.5),),
                    seq_len=131072, scale_mode="head", append=True, seed=5),
    "long_b8": Spec("long_b8", B=8, ps=64, layers=(LayerSpec(64, 8, 128, 0, 128 ** -0.5),),
                    seq_len=131072, scale_mode="head", append=True, seed=5),
}


@dataclass
class LayerCase:
    """Inputs of one attention call (one layer) over the shared pool."""
    spec: LayerSpec
    q: torch.Tensor                     # [B, Hq, D] bf16
    k_pages: torch.Tensor               # [num_pages, ps, Hkv, D] uint8 view of the K pool
    v_pages: torch.Tensor
    k_scale: torch.Tensor               # [Hkv], [num_pages, Hkv] or [num_pages, ps, Hkv] float32
    v_scale: torch.Tensor
    block_table: torch.Tensor           # [B, max_pages] int32 (-1 = unused entry)
    sinks: torch.Tensor | None          # [Hq] float32
    k_new: torch.Tensor | None          # [B, Hkv, D] bf16 (append only)
    v_new: torch.Tensor | None
    window: int = 0
    sm_scale: float = 1.0


@dataclass
class Case:
    spec: Spec
    k_pool: torch.Tensor                # flat uint8 pool (all layers)
    v_pool: torch.Tensor
    page_stride: int                    # bytes between consecutive pages
    cache_lens: torch.Tensor            # [B] int32, tokens stored before the step
    attend_lens: torch.Tensor           # [B] int32, keys visible to the query
    positions: torch.Tensor | None      # [B] int32 append positions (= cache_lens)
    layers: list = field(default_factory=list)   # list[LayerCase]

    @property
    def B(self) -> int:
        return self.spec.B


def spec_with(name_or_spec, **overrides) -> Spec:
    spec = SPECS[name_or_spec] if isinstance(name_or_spec, str) else name_or_spec
    return dataclasses.replace(spec, **overrides) if overrides else spec


def _lengths(spec: Spec, rng: np.random.Generator) -> np.ndarray:
    if isinstance(spec.seq_len, tuple):
        lo, hi = spec.seq_len
        return rng.integers(lo, hi + 1, size=spec.B).astype(np.int64)
    return np.full(spec.B, int(spec.seq_len), dtype=np.int64)


def _tables(spec: Spec, n_pages: np.ndarray, rng: np.random.Generator, n_layers: int):
    """Disjoint physical pages for every (layer, sequence), drawn from one
    shuffled pool; the logical order inside a sequence is the draw order."""
    need = int(n_pages.sum()) * n_layers
    total = spec.pool_pages if spec.pool_pages is not None else need
    if total < need:
        raise ValueError(f"pool of {total} pages cannot hold {need}")
    perm = rng.permutation(total)
    max_pages = int(n_pages.max()) if n_pages.size else 0
    tables, off = [], 0
    for _ in range(n_layers):
        t = np.full((spec.B, max(max_pages, 1)), -1, dtype=np.int32)
        for b in range(spec.B):
            t[b, :n_pages[b]] = perm[off:off + n_pages[b]]
            off += int(n_pages[b])
        tables.append(t)
    return tables, total


def _raw(gen: torch.Generator, shape, dist: str, device) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if dist == "normal2_outliers":
        x = x * 2.0
        hit = torch.rand(shape, generator=gen, device=device) < 0.01
        x = torch.where(hit, x * 20.0, x)
    elif dist != "normal":
        raise ValueError(dist)
    return x


def make_case(name_or_spec, device="cpu", chunk_pages: int = 1024, **overrides) -> Case:
    """Build one workload on ``device`` (deterministic for a device type).

    Lengths, block tables and permutations come from numpy ``default_rng``
    (identical on every device); q, sinks and K/V values from a seeded
    ``torch.Generator`` on ``device``. Pages are filled in chunks so the
    float32 draws never need the whole pool at once.
    """
    spec = spec_with(name_or_spec, **overrides)
    device = torch.device(device)
    rng = np.random.default_rng(spec.seed)
    cache_lens = _lengths(spec, rng)
    extra = 1 if spec.append else 0
    stored = cache_lens + extra                       # tokens that will live in the pool
    n_pages = (stored + spec.ps - 1) // spec.ps
    n_layers = len(spec.layers)
    tables, total_pages = _tables(spec, n_pages, rng, n_layers)
    page_bytes = [spec.ps * L.Hkv * L.D for L in spec.layers]
    page_stride = max(page_bytes)
    k_pool = torch.zeros(total_pages * page_stride, dtype=torch.uint8, device=device)
    v_pool = torch.zeros_like(k_pool)
    gen = torch.Generator(device=device)

    case = Case(spec=spec, k_pool=k_pool, v_pool=v_pool, page_stride=page_stride,
                cache_lens=torch.tensor(cache_lens, dtype=torch.int32, device=device),
                attend_lens=torch.tensor(cache_lens + extra, dtype=torch.int32, device=device),
                positions=(torch.tensor(cache_lens, dtype=torch.int32, device=device)
                           if spec.append else None))

    for li, L in enumerate(spec.layers):
        seed = spec.seed * 1000 + li * 7
        gen.manual_seed(seed)
        q = torch.randn(spec.B, L.Hq, L.D, generator=gen, device=device).to(torch.bfloat16)
        sinks = (torch.randn(L.Hq, generator=gen, device=device, dtype=torch.float32)
                 if spec.sinks else None)
        table = tables[li]
        # page -> (sequence, index of the page in that sequence), for validity.
        owner = np.full(total_pages, -1, dtype=np.int64)
        pidx = np.zeros(total_pages, dtype=np.int64)
        for b in range(spec.B):
            owner[table[b, :n_pages[b]]] = b
            pidx[table[b, :n_pages[b]]] = np.arange(n_pages[b])
        valid = np.where(owner >= 0, np.clip(stored[np.maximum(owner, 0)] - pidx * spec.ps, 0, spec.ps), 0)
        append_page = np.full(spec.B, -1, dtype=np.int64)
        if spec.append:
            for b in range(spec.B):
                append_page[b] = table[b, cache_lens[b] // spec.ps]

        def page_values(p0: int, p1: int, which: int) -> torch.Tensor:
            g = torch.Generator(device=device)
            g.manual_seed(seed * 7919 + which * 104729 + p0)
            x = _raw(g, (p1 - p0, spec.ps, L.Hkv, L.D), spec.dist, device)
            slot = torch.arange(spec.ps, device=device).view(1, spec.ps, 1, 1)
            nv = torch.tensor(valid[p0:p1], device=device).view(-1, 1, 1, 1)
            x = torch.where(slot < nv, x, torch.zeros((), device=device))
            # the token about to be appended is a bf16 value
            return x

        def page_values_bf16_new(x: torch.Tensor, p0: int, p1: int) -> torch.Tensor:
            if not spec.append:
                return x
            for b in range(spec.B):
                p = int(append_page[b])
                if p0 <= p < p1:
                    s = int(cache_lens[b] % spec.ps)
                    x[p - p0, s] = x[p - p0, s].to(torch.bfloat16).float()
            return x

        views, scales, news = [], [], []
        for which, pool in ((0, k_pool), (1, v_pool)):
            # pass 1: scales from the values (including the token to append)
            G = spec.k_groups if (spec.scale_mode == "token" and which == 0) else 1
            if spec.scale_mode == "mx":
                # MXFP8: per 32-entry block, 2^(floor(log2 amax) - 8) as an E8M0 code
                # (127 for an all-zero block), codes the clamped E4M3 cast of x / scale
                view = torch.as_strided(pool, (total_pages, spec.ps, L.Hkv, L.D),
                                        (page_stride, L.Hkv * L.D, L.D, 1))
                codes_sc = torch.full((total_pages, spec.ps, L.Hkv, L.D // 32), 127,
                                      dtype=torch.uint8, device=device)
                new = torch.zeros(spec.B, L.Hkv, L.D, dtype=torch.bfloat16, device=device)
                for p0 in range(0, total_pages, chunk_pages):
                    p1 = min(total_pages, p0 + chunk_pages)
                    x = page_values_bf16_new(page_values(p0, p1, which), p0, p1)
                    xb = x.view(p1 - p0, spec.ps, L.Hkv, L.D // 32, 32)
                    amax = xb.abs().amax(dim=-1)
                    e = torch.frexp(amax).exponent.to(torch.int32) - 1 - 8 + 127
                    c = torch.where(amax > 0, e.clamp(0, 254), torch.full_like(e, 127))
                    sc = torch.pow(2.0, (c - 127).to(torch.float64)).float()
                    quot = (xb / sc[..., None]).clamp(-E4M3_MAX, E4M3_MAX).reshape(x.shape)
                    codes = quot.to(torch.float8_e4m3fn).view(torch.uint8)
                    if spec.append:
                        for b in range(spec.B):
                            p = int(append_page[b])
                            if p0 <= p < p1:
                                s = int(cache_lens[b] % spec.ps)
                                new[b] = x[p - p0, s].to(torch.bfloat16)
                                codes[p - p0, s] = 0
                    view[p0:p1] = codes
                    codes_sc[p0:p1] = c.to(torch.uint8)
                views.append(view)
                scales.append(codes_sc)
                news.append(new if spec.append else None)
                continue
            if spec.scale_mode == "head":
                amax = torch.zeros(L.Hkv, device=device)
            elif spec.scale_mode == "token" and G > 1:
                amax = torch.zeros(total_pages, spec.ps, L.Hkv, G, device=device)
            elif spec.scale_mode == "token":
                amax = torch.zeros(total_pages, spec.ps, L.Hkv, device=device)
            else:
                amax = torch.zeros(total_pages, L.Hkv, device=device)
            for p0 in range(0, total_pages, chunk_pages):
                p1 = min(total_pages, p0 + chunk_pages)
                x = page_values_bf16_new(page_values(p0, p1, which), p0, p1)
                if spec.scale_mode == "token" and G > 1:          # [pages, ps, Hkv, G]
                    amax[p0:p1] = x.view(p1 - p0, spec.ps, L.Hkv, G, L.D // G).abs().amax(dim=4)
                    continue
                if spec.scale_mode == "token":
                    amax[p0:p1] = x.abs().amax(dim=3)             # [pages, ps, Hkv]
                    continue
                a = x.abs().amax(dim=(1, 3))                      # [pages, Hkv]
                if spec.scale_mode == "head":
                    amax = torch.maximum(amax, a.amax(dim=0))
                else:
                    amax[p0:p1] = a
            scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones((), device=device)).float()
            # pass 2: codes of the stored tokens; the append slot stays 0
            view = torch.as_strided(pool, (total_pages, spec.ps, L.Hkv, L.D),
                                    (page_stride, L.Hkv * L.D, L.D, 1))
            new = torch.zeros(spec.B, L.Hkv, L.D, dtype=torch.bfloat16, device=device)
            for p0 in range(0, total_pages, chunk_pages):
                p1 = min(total_pages, p0 + chunk_pages)
                x = page_values_bf16_new(page_values(p0, p1, which), p0, p1)
                if spec.scale_mode == "head":
                    sc = scale.view(1, 1, L.Hkv, 1)
                elif spec.scale_mode == "token" and G > 1:
                    sc = scale[p0:p1].repeat_interleave(L.D // G, dim=3)
                elif spec.scale_mode == "token":
                    sc = scale[p0:p1].view(-1, spec.ps, L.Hkv, 1)
                else:
                    sc = scale[p0:p1].view(-1, 1, L.Hkv, 1)
                codes = (x / sc).to(torch.float8_e4m3fn).view(torch.uint8)
                if spec.append:
                    for b in range(spec.B):
                        p = int(append_page[b])
                        if p0 <= p < p1:
                            s = int(cache_lens[b] % spec.ps)
                            new[b] = x[p - p0, s].to(torch.bfloat16)
                            codes[p - p0, s] = 0
                view[p0:p1] = codes
            views.append(view)
            scales.append(scale)
            news.append(new if spec.append else None)
        sm = L.sm_scale if L.sm_scale is not None else L.D ** -0.5
        case.layers.append(LayerCase(
            spec=L, q=q, k_pages=views[0], v_pages=views[1], k_scale=scales[0], v_scale=scales[1],
            block_table=torch.tensor(table, dtype=torch.int32, device=device), sinks=sinks,
            k_new=news[0], v_new=news[1], window=L.window, sm_scale=float(sm)))
    return case


def algorithmic_bytes(case: Case, layer: int = 0) -> int:
    """Bytes a decode step must read for one layer: the attended K and V bytes
    (window-limited, once per KV head), q, and the block-table entries of the
    attended pages; with per-token scales also the attended tokens' K and V
    scales (4 bytes each per KV head and sub-row group). Per-head and per-page scales, the
    output and split partials are not counted."""
    L = case.layers[layer]
    lens = case.attend_lens.cpu().numpy().astype(np.int64)
    ps = case.spec.ps
    kv = 0
    tbl = 0
    for Lb in lens:
        lo = max(0, Lb - L.window) if L.window > 0 else 0
        n = max(0, Lb - lo)
        kv += 2 * n * L.spec.Hkv * L.spec.D
        if n > 0:
            tbl += 4 * ((Lb - 1) // ps - lo // ps + 1)
    q = L.q.numel() * 2
    # per-token scales: 4 bytes per attended token, KV head and group, for K and for V
    # (MXFP8: one byte per 32-entry block)
    tok_scales = sum(kv // L.spec.D // 2 * (sc.shape[3] if sc.dim() == 4 else 1) *
                     (1 if sc.dtype == torch.uint8 else 4)
                     for sc in (L.k_scale, L.v_scale) if sc.dim() >= 3)
    return int(kv + q + tbl + tok_scales)


def describe(spec: Spec) -> str:
    parts = [f"B={spec.B}", f"ps={spec.ps}"]
    for L in spec.layers:
        parts.append(f"[Hq={L.Hq},Hkv={L.Hkv},D={L.D},W={L.window}]")
    parts.append(f"L={spec.seq_len}")
    return " ".join(parts)


__all__ = ["Spec", "LayerSpec", "SPECS", "Case", "LayerCase", "make_case", "spec_with",
           "algorithmic_bytes", "describe", "E4M3_MAX"]

