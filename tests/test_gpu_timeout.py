"""GPU: the bounded waits of the attention kernel, made to run out on purpose.

Every wait on a tile copy's barrier gives up after a bounded number of polls,
sets FP8PD_FLAG_TIMEOUT in the device error word and leaves that warp's keys
out, so a lost copy can never hang the GPU. The test hook FP8PD_OPT_TEST_STALL
makes warp 0 of the launch's first block post its first copy's bytes on the
barrier without issuing the copy: that one wait runs out (after a short poll
limit set with FP8PD_OPT_WAIT_POLLS), with no copy in flight on the stalled
stage, and the launch ends normally. The tests check the flag, the documented
output and that the next call, without the hook, is exact again.
"""

import dataclasses

import numpy as np
import pytest
import torch

import workloads as W
from tests._common import assert_attention_close, gpu_attention, np_, oracle_attention

pytestmark = pytest.mark.gpu


@pytest.fixture
def F(cuda_device):
    import fp8_paged_decode_split_b200 as F
    yield F
    F.fp8pd_set_option(F.OPT_TEST_STALL, 0)
    F.fp8pd_set_option(F.OPT_WAIT_POLLS, 1 << 17)
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)
    F.fp8pd_set_option(F.OPT_SCHEDULE, 0)
    F.fp8pd_check_errors()


def _case(cuda_device, seq_len=64, D=64):
    spec = W.Spec("stall", B=2, ps=16, layers=(W.LayerSpec(8, 1, D, 0, 0.125),),
                  seq_len=seq_len, scale_mode="page", seed=91)
    return W.make_case(spec, cuda_device)


@pytest.mark.parametrize("D", [64, 512])
def test_a_wait_that_runs_out_drops_that_warps_keys_and_sets_the_flag(F, cuda_device, D):
    """One block per sequence (one split), 64 keys: tile stream w attends tile
    w, so the stalled warp 0 of sequence 0's block drops keys 0..15. Sequence
    0's output is then attention over its last 48 keys; sequence 1 is
    untouched. At D = 512 stream 0 is two or four warps, each on its part of
    the head dim: the stalled warp's partners learn of the lost copy when the
    score parts meet, and all leave the tile stream."""
    case = _case(cuda_device, D=D)
    layer = case.layers[0]
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 1)
    F.fp8pd_set_option(F.OPT_SCHEDULE, 1)
    F.fp8pd_set_option(F.OPT_WAIT_POLLS, 32)
    F.fp8pd_set_option(F.OPT_TEST_STALL, 1)
    got = np_(gpu_attention(F, layer, case.attend_lens))
    torch.cuda.synchronize()
    flags = F.fp8pd_check_errors()
    assert flags & F.FLAG_TIMEOUT
    assert flags & ~F.FLAG_TIMEOUT == 0
    run = F.fp8pd_last_run_info()
    assert run["num_splits"] == 1 and run["schedule"] == 1
    assert (run["dim_split"] in (2, 4)) if D == 512 else run["dim_split"] == 1
    full = oracle_attention(layer, case.attend_lens)
    last48 = dataclasses.replace(layer, window=48)
    want0 = oracle_attention(last48, case.attend_lens)[0]
    assert_attention_close(got[0], want0, "stalled sequence")
    assert_attention_close(got[1], full[1], "other sequence")
    assert not np.allclose(got[0], full[0], rtol=1e-3, atol=1e-3)

    # the context is usable and the next call, without the hook, is exact
    F.fp8pd_set_option(F.OPT_TEST_STALL, 0)
    again = np_(gpu_attention(F, layer, case.attend_lens))
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    assert_attention_close(again, full, "after the stall")


@pytest.mark.parametrize("schedule", [1, 3])
def test_a_stall_in_a_split_sequence_is_reported_and_bounded(F, cuda_device, schedule):
    """Several blocks per sequence (uniform or proportional splits) merged
    through the ticket counters: the stalled warp's keys are left out of
    sequence 0's first split, so the test checks the flag, finite output, the
    untouched second sequence (other blocks), and exact calls afterwards, whose
    tickets the stalled call's merges put back to zero."""
    case = _case(cuda_device, seq_len=3000)
    layer = case.layers[0]
    F.fp8pd_set_option(F.OPT_SCHEDULE, schedule)
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 4 if schedule == 1 else 0)
    F.fp8pd_set_option(F.OPT_WAIT_POLLS, 32)
    F.fp8pd_set_option(F.OPT_TEST_STALL, 1)
    got = np_(gpu_attention(F, layer, case.attend_lens))
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() & F.FLAG_TIMEOUT
    assert np.all(np.isfinite(got))
    full = oracle_attention(layer, case.attend_lens)
    assert_attention_close(got[1], full[1], "other sequence")
    F.fp8pd_set_option(F.OPT_TEST_STALL, 0)
    for _ in range(2):
        again = np_(gpu_attention(F, layer, case.attend_lens))
        torch.cuda.synchronize()
        assert F.fp8pd_check_errors() == 0
        assert_attention_close(again, full, "after the stall")
