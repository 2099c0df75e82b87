"""GPU: fp8_kv_append is bit-exact against the oracle's quantizer and writes
nothing but the new token's slots."""

import numpy as np
import pytest
import torch

import oracle as O
from tests._common import np_

pytestmark = pytest.mark.gpu


def _nan_class(codes: np.ndarray) -> np.ndarray:
    """E4M3 has two NaN bytes (0x7F, 0xFF); a NaN input may map to either
    (the sign of a NaN carries no value), so compare NaN codes as a class.
    Every other byte must match exactly."""
    c = codes.copy()
    c[(c & 0x7F) == 0x7F] = 0x7F
    return c


@pytest.fixture(scope="module")
def F(cuda_device):
    import fp8_paged_decode_split_b200 as F
    return F


def _append_case(dev, scale, per_page_v, seed):
    g = torch.Generator().manual_seed(seed)
    B, Hkv, D, ps, npages = 64, 4, 256, 16, 80
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    k_new = bits.reshape(B, Hkv, D)
    v_new = torch.roll(bits, 12345).reshape(B, Hkv, D)
    perm = torch.randperm(npages, generator=g)
    table = perm[: B * 1].reshape(B, 1).to(torch.int32)
    positions = (torch.arange(B) * 7 % ps).to(torch.int32)
    kp = torch.randint(0, 256, (npages, ps, Hkv, D), generator=g, dtype=torch.uint8)
    vp = torch.randint(0, 256, (npages, ps, Hkv, D), generator=g, dtype=torch.uint8)
    ks = torch.full((Hkv,), scale, dtype=torch.float32)
    if per_page_v:
        vs = (torch.rand(npages, Hkv, generator=g) * 2 + 0.25) * scale
        vs = vs.float()
    else:
        vs = torch.full((Hkv,), scale, dtype=torch.float32)
    return [t.to(dev) for t in (k_new, v_new, kp, vp, ks, vs, table, positions)]


@pytest.mark.parametrize("scale", [1.0, 0.5, 4.0 / 448, 3.0 / 448, 1e-3, 2.0 ** -20, 1e6,
                                   37.0 / 448, 2.0 ** -30])
def test_append_every_bf16_pattern_bit_exact(F, cuda_device, scale):
    k_new, v_new, kp, vp, ks, vs, table, pos = _append_case(cuda_device, scale, scale < 1, 7)
    kp0, vp0 = np_(kp).copy(), np_(vp).copy()
    F.fp8_kv_append(k_new, v_new, kp, vp, ks, vs, table, pos)
    torch.cuda.synchronize()
    assert F.fp8pd_check_errors() == 0
    O.kv_append(np_(k_new), np_(v_new), kp0, vp0, np_(ks), np_(vs), np_(table), np_(pos))
    got_k, got_v = np_(kp), np_(vp)
    assert np.array_equal(_nan_class(got_k), _nan_class(kp0))
    assert np.array_equal(_nan_class(got_v), _nan_class(vp0))
    # non-NaN inputs: the exact byte, sign included
    nn = ~np.isnan(np_(k_new))
    b_idx = np.arange(64)[:, None, None]
    page = np_(table)[:, 0][b_idx]
    slot = np_(pos)[b_idx]
    h = np.arange(4)[None, :, None]
    d = np.arange(256)[None, None, :]
    assert np.array_equal(got_k[page, slot, h, d][nn], kp0[page, slot, h, d][nn])


def test_append_into_strided_shared_pool(F, cuda_device):
    """Two layers with different geometry share one pool (page stride wider
    than a layer's page); appends to one layer leave the other untouched."""
    g = torch.Generator().manual_seed(3)
    npages, ps, stride = 12, 32, 32 * 8 * 256
    pool_k = torch.randint(0, 256, (npages * stride,), generator=g, dtype=torch.uint8).to(cuda_device)
    pool_v = torch.randint(0, 256, (npages * stride,), generator=g, dtype=torch.uint8).to(cuda_device)
    before_k, before_v = np_(pool_k).copy(), np_(pool_v).copy()
    Hkv, D = 2, 512
    kview = torch.as_strided(pool_k, (npages, ps, Hkv, D), (stride, Hkv * D, D, 1))
    vview = torch.as_strided(pool_v, (npages, ps, Hkv, D), (stride, Hkv * D, D, 1))
    B = 5
    table = torch.tensor([[3, 7], [1, 0], [11, 2], [5, 6], [9, 8]], dtype=torch.int32, device=cuda_device)
    pos = torch.tensor([0, 33, 31, 63, 40], dtype=torch.int32, device=cuda_device)
    k_new = torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16).to(cuda_device) * 3
    v_new = torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16).to(cuda_device)
    ks = (torch.rand(npages, Hkv, generator=g) * 0.02 + 0.001).to(cuda_device)
    vs = torch.tensor([0.004, 0.01], device=cuda_device)
    F.fp8_kv_append(k_new, v_new, kview, vview, ks, vs, table, pos)
    torch.cuda.synchronize()
    kv_np = np.lib.stride_tricks.as_strided(before_k, (npages, ps, Hkv, D), (stride, Hkv * D, D, 1))
    vv_np = np.lib.stride_tricks.as_strided(before_v, (npages, ps, Hkv, D), (stride, Hkv * D, D, 1))
    O.kv_append(np_(k_new), np_(v_new), kv_np, vv_np, np_(ks), np_(vs), np_(table), np_(pos))
    assert np.array_equal(np_(pool_k), before_k)
    assert np.array_equal(np_(pool_v), before_v)


def test_append_out_of_range_is_flagged_not_written(F, cuda_device):
    ps, Hkv, D = 16, 2, 64
    kp = torch.zeros(4, ps, Hkv, D, dtype=torch.uint8, device=cuda_device)
    vp = torch.zeros_like(kp)
    ks = torch.ones(Hkv, device=cuda_device)
    kn = torch.ones(3, Hkv, D, dtype=torch.bfloat16, device=cuda_device)
    table = torch.tensor([[0, 1], [2, 9], [3, 3]], dtype=torch.int32, device=cuda_device)
    pos = torch.tensor([32, 20, -1], dtype=torch.int32, device=cuda_device)  # beyond table, bad page, <0
    assert F.fp8pd_check_errors() == 0
    F.fp8_kv_append(kn, kn, kp, vp, ks, ks, table, pos)
    flags = F.fp8pd_check_errors()
    assert flags & F.FLAG_POS_OOB and flags & F.FLAG_PAGE_OOB
    assert int(kp.sum()) == 0 and int(vp.sum()) == 0
    assert F.fp8pd_check_errors() == 0


def test_append_many_tokens_of_one_sequence_with_broadcast_table_row(F, cuda_device):
    """block_table stride 0 over the batch: one call writes T tokens of one
    sequence (a prefill-style fill through the same entry point)."""
    g = torch.Generator().manual_seed(5)
    ps, Hkv, D, T = 16, 2, 128, 70
    npages = 8
    kp = torch.zeros(npages, ps, Hkv, D, dtype=torch.uint8, device=cuda_device)
    vp = torch.zeros_like(kp)
    row = torch.tensor([5, 2, 7, 0, 3], dtype=torch.int32, device=cuda_device)
    table = row.view(1, -1).expand(T, -1)
    assert table.stride(0) == 0
    pos = torch.arange(T, dtype=torch.int32, device=cuda_device)
    kn = torch.randn(T, Hkv, D, generator=g).to(torch.bfloat16).to(cuda_device)
    vn = torch.randn(T, Hkv, D, generator=g).to(torch.bfloat16).to(cuda_device)
    ks = torch.tensor([0.01, 0.02], device=cuda_device)
    vs = torch.tensor([0.015, 0.005], device=cuda_device)
    k0, v0 = np_(kp).copy(), np_(vp).copy()
    F.fp8_kv_append(kn, vn, kp, vp, ks, vs, table, pos)
    O.kv_append(np_(kn), np_(vn), k0, v0, np_(ks), np_(vs), np.broadcast_to(np_(row), (T, 5)), np_(pos))
    assert np.array_equal(np_(kp), k0) and np.array_equal(np_(vp), v0)

