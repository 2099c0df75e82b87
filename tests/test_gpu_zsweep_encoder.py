"""GPU: the library's E4M3 encoder (fp8pd_e4m3_encode, the cvt.rn.satfinite
rounding the append uses) against the oracle on every float32 bit pattern.
Collected after the other parity files: it holds several GB of device memory
per chunk of the sweep."""

import numpy as np
import pytest
import torch

import oracle as O
from tests.test_gpu_append import _nan_class

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F(cuda_device):
    import fp8_paged_decode_split_b200 as F
    return F


def test_encoder_matches_oracle_on_every_float32(F, cuda_device):
    """fp8pd_e4m3_encode (the cvt.rn.satfinite the append uses) on all 2^32
    float32 bit patterns against the oracle's encoder. The GPU codes, taken
    in bit-pattern order and with the two NaN bytes as one class, fall into
    runs of equal code; the oracle must give each run's code at both ends of
    the run. The oracle's code is monotone in the magnitude within each sign
    (pinned on the CPU), so it then equals the GPU's on every pattern."""
    chunk = 1 << 28
    starts, codes = [], []
    last = None
    for c0 in range(0, 1 << 32, chunk):
        v = torch.arange(c0, c0 + chunk, dtype=torch.int64, device=cuda_device)
        v = torch.where(v >= 1 << 31, v - (1 << 32), v).to(torch.int32)
        out = F.fp8pd_e4m3_encode(v.view(torch.float32))
        out = torch.where((out & 0x7F) == 0x7F, torch.full_like(out, 0x7F), out)
        if last is None or int(out[0]) != last:
            starts.append(c0)
            codes.append(int(out[0]))
        chg = torch.nonzero(out[1:] != out[:-1]).flatten() + 1
        starts += (chg + c0).tolist()
        codes += out[chg].tolist()
        last = int(out[-1])
        del v, out, chg
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    ends = [s - 1 for s in starts[1:]] + [(1 << 32) - 1]
    as_f32 = lambda b: np.array(b, dtype=np.uint64).astype(np.uint32).view(np.float32)  # noqa: E731
    want = np.array(codes, dtype=np.uint8)
    for edge in (starts, ends):
        got = _nan_class(O.e4m3_encode(as_f32(edge).astype(np.float64)))
        assert np.array_equal(got, want)
    # +0 .. +448, +NaN, -0 .. -448, -NaN: one run per code
    assert len(codes) == 256
