"""GPU: every workload at full size, in the launch configuration the benchmark
times, against the oracle on sampled outputs.

The benchmark's step is used as is (bench.Step): the planner's default
schedule, the hardware decode of K and V, and, where the workload has an
append, the fused append + attention launch (and, as a second case, the
append and attention calls on their own). The oracle cannot afford every
output at these sizes, so a few sequences are sampled (first, last and one
drawn from a seeded generator), and for each the pages it uses are gathered
into a small pool that the oracle reads in full: all query heads of the
sampled sequences are checked element by element. The append is checked
bit-exactly over the same pages, before-and-after against the oracle's own
append.
"""

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from tests._common import ATOL_REL, np_

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def F(cuda_device):
    import fp8_paged_decode_split_b200 as F
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)
    F.fp8pd_set_option(F.OPT_SCHEDULE, 0)
    F.fp8pd_set_option(F.OPT_K_DECODE, 1)     # the benchmark's default decodes
    F.fp8pd_set_option(F.OPT_V_DECODE, 1)
    return F


def _sampled_sequences(B: int, seed: int) -> list:
    rng = np.random.default_rng(seed)
    return sorted({0, B - 1, int(rng.integers(0, B))})


def _sub_pool(layer, b: int, n_pages: int):
    """The pages sequence b uses, gathered in logical order, with a matching
    identity table and the scales that travel with them."""
    ids = layer.block_table[b, :n_pages].long()
    kp = layer.k_pages[ids].contiguous()
    vp = layer.v_pages[ids].contiguous()
    ks = layer.k_scale[ids] if layer.k_scale.dim() == 2 else layer.k_scale
    vs = layer.v_scale[ids] if layer.v_scale.dim() == 2 else layer.v_scale
    return kp, vp, ks, vs


@pytest.mark.parametrize("name,fused", [("llama", True), ("llama", False), ("gptoss_w128", True),
                                        ("gptoss_full", True), ("mixed", True),
                                        ("long_b1", True), ("long_b1", False),
                                        ("long_b8", True)])
def test_full_size_step_matches_oracle_on_sampled_sequences(F, cuda_device, name, fused):
    import bench
    case = W.make_case(name, cuda_device)
    spec = case.spec
    seqs = _sampled_sequences(spec.B, 1000 + spec.seed)
    lens = case.attend_lens.cpu().numpy()
    ps = spec.ps
    n_pages = {b: (int(lens[b]) + ps - 1) // ps for b in seqs}

    before = {}
    for li, layer in enumerate(case.layers):
        if spec.append:
            before[li] = {b: tuple(np_(t).copy() for t in _sub_pool(layer, b, n_pages[b])[:2])
                          for b in seqs}

    for layer in case.layers:
        layer.out = torch.empty(layer.q.shape, dtype=torch.float32, device=cuda_device)
    step = bench.Step(F, case, fused)          # the benchmark's step, every layer
    step.run()
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    assert step.fused == (fused and spec.append)
    outs = [layer.out for layer in case.layers]

    worst = 0.0
    for li, layer in enumerate(case.layers):
        got = np_(outs[li])
        for b in seqs:
            kp, vp, ks, vs = _sub_pool(layer, b, n_pages[b])
            kp, vp, ks, vs = np_(kp), np_(vp), np_(ks), np_(vs)
            table = np.arange(n_pages[b], dtype=np.int32)[None, :]
            if spec.append:
                kp0, vp0 = before[li][b]
                pos = np.array([int(case.positions[b])])
                O.kv_append(np_(layer.k_new[b:b + 1]), np_(layer.v_new[b:b + 1]), kp0, vp0,
                            ks, vs, table, pos)
                assert np.array_equal(kp, kp0) and np.array_equal(vp, vp0), \
                    f"{name} layer {li} seq {b}: append not bit-exact"
            want = O.paged_decode_attention(
                np_(layer.q[b:b + 1]), kp, vp, ks, vs, table, lens[b:b + 1],
                window=layer.window, sinks=np_(layer.sinks), sm_scale=layer.sm_scale)[0]
            err = np.abs(got[b] - want) / np.maximum(1.0, np.abs(want))
            assert np.all(np.isfinite(got[b]))
            assert err.max() <= ATOL_REL, f"{name} layer {li} seq {b}: max rel err {err.max():.3g}"
            worst = max(worst, float(err.max()))
    print(f"{name} fused={step.fused}: sequences {seqs}, worst error {worst:.3g}")
