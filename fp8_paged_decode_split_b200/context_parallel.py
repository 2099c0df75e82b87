"""Context-parallel split-KV decode attention across GPUs.

One long sequence's keys do not fit one GPU's time budget, so its pages are
spread over the ranks of a process group (one process per GPU): rank r holds
the pages of its key slice of every sequence, attends that slice with
``fp8_paged_decode_attention_partial`` (an unnormalized (O, m, l) per
sequence and query head), the ranks exchange those partials with one NCCL
all-gather (B x Hq x (D + 2) floats per rank: 33 KB for one sequence of 64
query heads at D = 128), and every rank merges them with
``fp8pd_combine_partials``, adding the sink once. This is the split-KV of the
solution page's "Why it happens" (a grid over sequence, KV head and split)
taken across GPUs, with the log-sum-exp combine of the splits.

The slicing (:func:`key_slices`) and the exchange (:func:`gather_partials`)
are host logic; the attention and the combine run in the library's kernels.
"""

from __future__ import annotations

import numpy as np
import torch

from . import fp8_paged_decode_attention_partial, fp8pd_combine_partials


def key_slices(seq_lens, page_size: int, world: int) -> np.ndarray:
    """Contiguous, page-aligned key slices of each sequence for ``world``
    ranks: int32 [world, B, 2] (begin, end). Rank r gets pages
    [floor(r P / world), floor((r+1) P / world)) of a sequence of P pages
    (the last page may be partial), so the slices cover [0, L) exactly, each
    page belongs to one rank and the ranks' page counts differ by at most one."""
    lens = np.asarray(seq_lens, dtype=np.int64).reshape(-1)
    if world < 1 or page_size < 1:
        raise ValueError("world and page_size must be >= 1")
    pages = (lens + page_size - 1) // page_size
    out = np.zeros((world, lens.size, 2), dtype=np.int32)
    for r in range(world):
        p0 = (r * pages) // world
        p1 = ((r + 1) * pages) // world
        out[r, :, 0] = np.minimum(p0 * page_size, lens)
        out[r, :, 1] = np.minimum(p1 * page_size, lens)
    return out


def gather_partials(part_o: torch.Tensor, part_ml: torch.Tensor, group=None):
    """All-gathers every rank's partials over the process group (NCCL for
    CUDA tensors): returns ([R, B, Hq, D], [R, B, Hq, 2]) in rank order. With
    no initialized group, or a group of one, the local partials alone."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return part_o.unsqueeze(0), part_ml.unsqueeze(0)
    world = dist.get_world_size(group)
    # concatenated along the batch (the form every backend takes), then viewed per rank
    all_o = torch.empty((world * part_o.shape[0],) + tuple(part_o.shape[1:]), dtype=part_o.dtype,
                        device=part_o.device)
    all_ml = torch.empty((world * part_ml.shape[0],) + tuple(part_ml.shape[1:]),
                         dtype=part_ml.dtype, device=part_ml.device)
    dist.all_gather_into_tensor(all_o, part_o.contiguous(), group=group)
    dist.all_gather_into_tensor(all_ml, part_ml.contiguous(), group=group)
    return all_o.view((world,) + tuple(part_o.shape)), all_ml.view((world,) + tuple(part_ml.shape))


def attention(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens, key_ranges,
              window: int = 0, sinks=None, sm_scale: float | None = None, group=None,
              out=None, stream=None) -> torch.Tensor:
    """Decode attention of the whole sequences from this rank's slice:
    ``key_ranges`` (int32 [B, 2] on the device) is this rank's slice of each
    sequence (see :func:`key_slices`), ``block_table`` maps the sequence's
    logical pages to this rank's pool (entries outside the slice are never
    read), ``seq_lens`` are the full lengths. Every rank returns the full
    output [B, Hq, D]."""
    part_o, part_ml = fp8_paged_decode_attention_partial(
        q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens, key_ranges,
        window=window, sm_scale=sm_scale, stream=stream)
    all_o, all_ml = gather_partials(part_o, part_ml, group)
    return fp8pd_combine_partials(all_o, all_ml, sinks=sinks, out=out, stream=stream)


__all__ = ["key_slices", "gather_partials", "attention"]
