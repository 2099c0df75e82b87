"""Shared helpers for the GPU parity tests: run the CUDA library and the
float64 oracle on the same seeded inputs and compare them."""

from __future__ import annotations

import numpy as np
import torch

import oracle as O

#: attention tolerance: max |got - ref| <= ATOL_REL * max(1, |ref|), element-wise
ATOL_REL = 1e-3


def np_(t: torch.Tensor | None):
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        return t.detach().float().cpu().numpy().astype(np.float64)
    return t.detach().cpu().numpy()


def oracle_attention(layer, lens, batch_heads=None, pages=None, compute="f32") -> np.ndarray:
    """Oracle output for one layer of a workload (inputs copied to the host)."""
    return O.paged_decode_attention(
        np_(layer.q), np_(layer.k_pages if pages is None else pages[0]),
        np_(layer.v_pages if pages is None else pages[1]),
        np_(layer.k_scale), np_(layer.v_scale), np_(layer.block_table), np_(lens),
        window=layer.window, sinks=np_(layer.sinks), sm_scale=layer.sm_scale,
        batch_heads=batch_heads, compute=compute)


def gpu_attention(F, layer, lens, out=None):
    return F.fp8_paged_decode_attention(
        layer.q, layer.k_pages, layer.v_pages, layer.k_scale, layer.v_scale, layer.block_table,
        lens, window=layer.window, sinks=layer.sinks, sm_scale=layer.sm_scale, out=out)


def assert_attention_close(got, want, where: str = "", mask=None) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    if mask is not None:
        got, want = got[mask], want[mask]
    assert np.all(np.isfinite(got)), f"{where}: non-finite output"
    err = np.abs(got - want) / np.maximum(1.0, np.abs(want))
    worst = float(err.max()) if err.size else 0.0
    assert worst <= ATOL_REL, f"{where}: max scaled error {worst:.3e} > {ATOL_REL}"
    return worst


def footer_pool(num_pages: int, ps: int, hkv: int, d: int, device="cpu"):
    """One pool whose pages hold the E4M3 codes of ps tokens x hkv heads x d,
    then one float32 scale per (token, head) as a page footer: the packed
    pages of the solution page's pack_kv_block rows and of DeepGEMM's
    64 x (64 + 4) = 4352-byte index pages. Returns (pool bytes, codes view
    [num_pages, ps, hkv, d], scales view [num_pages, ps, hkv]); the views
    alias the pool."""
    page = ps * hkv * d + 4 * ps * hkv
    pool = torch.zeros(num_pages * page, dtype=torch.uint8, device=device)
    return (pool, *footer_views(pool, num_pages, ps, hkv, d))


def footer_views(pool: torch.Tensor, num_pages: int, ps: int, hkv: int, d: int):
    """(codes, scales) views of a footer pool made by :func:`footer_pool`."""
    code_bytes = ps * hkv * d
    page = code_bytes + 4 * ps * hkv
    assert page % 16 == 0 and code_bytes % 4 == 0 and pool.numel() == num_pages * page
    codes = torch.as_strided(pool, (num_pages, ps, hkv, d), (page, hkv * d, d, 1))
    scales = torch.as_strided(pool.view(torch.float32), (num_pages, ps, hkv), (page // 4, hkv, 1),
                              code_bytes // 4)
    return codes, scales
