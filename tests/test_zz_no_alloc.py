"""GPU: the attention entry point that allocates nothing.

Some callers cannot allocate device memory where they run attention (an
allocator-free runtime, a memory manager that owns the whole device, code that
must not synchronize the device with cudaMalloc). For them the library offers
fp8_paged_decode_attention_noalloc, which keeps its split scratch in a fixed
array inside the library instead of an allocated workspace. These checks call
it through the C ABI and compare it with fp8_paged_decode_attention on the same
inputs, twice in a row (the array keeps the previous call's contents), within
the tolerance of the other attention tests. This file is collected last.
"""

import numpy as np
import pytest
import torch

import workloads as W
from tests._common import ATOL_REL, np_, oracle_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F(cuda_device):
    import fp8_paged_decode_split_b200 as F
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)
    yield F
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)


def _both(F, layer, lens):
    ref = F.fp8_paged_decode_attention(layer.q, layer.k_pages, layer.v_pages, layer.k_scale,
                                       layer.v_scale, layer.block_table, lens, window=layer.window,
                                       sinks=layer.sinks, sm_scale=layer.sm_scale)
    outs = []
    for _ in range(2):   # twice in a row: the shared scratch keeps the last call's contents
        out = torch.full_like(ref, float("nan"))
        F.fp8_paged_decode_attention_noalloc(layer.q, layer.k_pages, layer.v_pages, layer.k_scale,
                                             layer.v_scale, layer.block_table, lens,
                                             window=layer.window, sinks=layer.sinks,
                                             sm_scale=layer.sm_scale, out=out)
        outs.append(out)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    return np_(ref), [np_(o) for o in outs]


@pytest.mark.parametrize("name,overrides,splits,schedule", [
    ("llama", dict(B=6, seq_len=(40, 700)), 0, 1),        # ragged lengths, per-page scales
    ("long_b1", dict(seq_len=20000), 0, 1),               # many splits, two-level merge
    ("long_b1", dict(seq_len=20000), 5, 1),               # a single merge group
    ("gptoss_full", dict(B=3, seq_len=1000), 0, 1),       # sinks
    ("llama", dict(B=6, seq_len=(40, 700)), 0, 3),        # proportional splits
    ("long_b1", dict(seq_len=60000), 0, 3),               # proportional, two-level merge
])
def test_noalloc_matches_the_allocating_entry_point(F, cuda_device, name, overrides, splits,
                                                    schedule):
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, splits)
    F.fp8pd_set_option(F.OPT_SCHEDULE, schedule)
    try:
        case = W.make_case(name, cuda_device, **overrides)
        ref, outs = _both(F, case.layers[0], case.attend_lens)
    finally:
        F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)
        F.fp8pd_set_option(F.OPT_SCHEDULE, 0)
    want = oracle_attention(case.layers[0], case.attend_lens)
    report = {}
    for label, arr in [("allocating", ref), ("noalloc 1", outs[0]), ("noalloc 2", outs[1])]:
        e = np.abs(arr - want) / np.maximum(1.0, np.abs(want))
        bad = np.argwhere(~(e <= ATOL_REL))
        report[label] = (float(np.nanmax(e)) if np.isfinite(e).any() else float("nan"),
                         sorted({(int(b), int(h)) for b, h, _ in bad})[:8])
    for got in outs:
        assert np.all(np.isfinite(got)), report
        err = np.abs(got - ref) / np.maximum(1.0, np.abs(ref))
        assert err.max() <= ATOL_REL, report
    assert report["allocating"][0] <= ATOL_REL, report


def test_noalloc_refuses_a_call_whose_scratch_exceeds_its_array(F, cuda_device):
    """A call whose plan needs more than the 8 MiB array is refused with
    FP8PD_ERR_TOO_LARGE and launches nothing."""
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 256)
    try:
        case = W.make_case("gptoss_full", cuda_device, B=64, seq_len=1000)
        L = case.layers[0]
        out = torch.full(L.q.shape, 7.0, device=cuda_device)
        with pytest.raises(F.Fp8pdError) as e:
            F.fp8_paged_decode_attention_noalloc(L.q, L.k_pages, L.v_pages, L.k_scale, L.v_scale,
                                                 L.block_table, case.attend_lens, window=0,
                                                 sinks=L.sinks, sm_scale=L.sm_scale, out=out)
        assert e.value.status == -10
        torch.cuda.synchronize()
        assert torch.all(out == 7.0)
    finally:
        F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)
