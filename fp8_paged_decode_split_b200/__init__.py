"""FP8 (E4M3) paged split-KV decode attention for NVIDIA B200 (sm_100a).

A thin ctypes binding over the C ABI in ``include/fp8pd.h``: it turns torch
tensors into descriptors (pointer, dtype, shape, strides) and calls the
library on the current CUDA stream. Every step of the computation runs in
the library's CUDA kernels; there is no Python or CPU fallback. If the
library is missing, importing this package raises ``ImportError``.

Entry points (same names as the C ABI):

* :func:`fp8_paged_decode_attention` -- decode attention over a paged E4M3
  KV cache with GQA, an optional sliding window, optional sink logits and a
  caller softmax scale.
* :func:`fp8_kv_append` -- quantize one new bf16 K/V token per sequence to
  E4M3 and store it in its page.
* :func:`fp8_paged_decode_append_attention` -- both in one launch: the
  append, then the attention over the updated cache.
"""

from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "fp8_paged_decode_attention", "fp8_paged_decode_attention_noalloc", "fp8_kv_append",
    "fp8_paged_decode_append_attention",
    "fp8pd_plan", "fp8pd_reserve_workspace", "fp8pd_e4m3_encode",
    "fp8pd_check_errors", "fp8pd_set_option", "fp8pd_get_option", "fp8pd_last_run_info",
    "fp8pd_timing_enable", "fp8pd_timing_collect", "Fp8pdError", "lib", "LIB_PATH",
    "fp8_paged_decode_attention_partial", "fp8pd_combine_partials",
    "FLAG_PAGE_OOB", "FLAG_SEQLEN_OOB", "FLAG_POS_OOB", "FLAG_INTERNAL", "OPT_NUM_SPLITS",
    "OPT_SCHEDULE", "OPT_K_DECODE", "OPT_V_DECODE", "OPT_WAIT_POLLS",
    "OPT_TEST_STALL", "OPT_COMPUTE", "OPT_KERNEL", "FLAG_TIMEOUT",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libfp8pd.so")

DTYPE_U8, DTYPE_I32, DTYPE_F32, DTYPE_BF16 = 1, 2, 3, 4
FLAG_PAGE_OOB, FLAG_SEQLEN_OOB, FLAG_POS_OOB, FLAG_INTERNAL, FLAG_TIMEOUT = 1, 2, 4, 8, 16
OPT_NUM_SPLITS, OPT_SCHEDULE, OPT_K_DECODE, OPT_V_DECODE = 1, 2, 3, 4
OPT_WAIT_POLLS, OPT_TEST_STALL, OPT_COMPUTE, OPT_KERNEL = 6, 7, 8, 9
_DTYPES = {torch.uint8: DTYPE_U8, torch.int32: DTYPE_I32, torch.float32: DTYPE_F32,
           torch.bfloat16: DTYPE_BF16}


class Tensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class Scales(ctypes.Structure):
    _fields_ = [("k_scale", Tensor), ("v_scale", Tensor)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("num_splits", ctypes.c_int32), ("head_groups", ctypes.c_int32),
                ("grid_blocks", ctypes.c_int32), ("combine", ctypes.c_int32),
                ("workspace_bytes", ctypes.c_uint64), ("schedule", ctypes.c_int32),
                ("warps", ctypes.c_int32)]


class RunInfo(ctypes.Structure):
    _fields_ = [("schedule", ctypes.c_int32), ("num_splits", ctypes.c_int32),
                ("head_groups", ctypes.c_int32), ("grid_blocks", ctypes.c_int32),
                ("combine", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("calls", ctypes.c_int64), ("appends", ctypes.c_int64),
                ("kernel_launches", ctypes.c_int64), ("compute", ctypes.c_int32),
                ("kernel", ctypes.c_int32), ("dim_split", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python fp8_paged_decode_split_b200/_build.py` "
            "(nvcc, sm_100a). There is no fallback implementation.")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    T = P(Tensor)
    i32, f32, vp = ctypes.c_int32, ctypes.c_float, ctypes.c_void_p
    lib.fp8_paged_decode_attention.argtypes = [T, T, T, T, T, T, T, i32, T, f32, T, vp]
    lib.fp8_paged_decode_attention_noalloc.argtypes = [T, T, T, T, T, T, T, i32, T, f32, T, vp]
    lib.fp8_kv_append.argtypes = [T, T, T, T, P(Scales), T, T, vp]
    lib.fp8_paged_decode_attention_partial.argtypes = [T, T, T, T, T, T, T, T, i32, f32, T, T, vp]
    lib.fp8pd_combine_partials.argtypes = [T, T, T, T, vp]
    lib.fp8_paged_decode_append_attention.argtypes = [T, T, T, T, T, T, T, T, T, i32, T, f32, T, vp]
    lib.fp8pd_plan.argtypes = [T, T, T, i32, P(PlanInfo)]
    lib.fp8pd_reserve_workspace.argtypes = [ctypes.c_uint64]
    lib.fp8pd_e4m3_encode.argtypes = [T, T, vp]
    lib.fp8pd_check_errors.argtypes = [vp, P(ctypes.c_uint32)]
    lib.fp8pd_set_option.argtypes = [i32, ctypes.c_int64]
    lib.fp8pd_get_option.argtypes = [i32]
    lib.fp8pd_get_option.restype = ctypes.c_int64
    lib.fp8pd_last_run_info.argtypes = [P(RunInfo)]
    lib.fp8pd_timing_enable.argtypes = [i32]
    lib.fp8pd_timing_collect.argtypes = [P(ctypes.c_double), P(i32), P(ctypes.c_double), P(i32)]
    lib.fp8pd_status_string.argtypes = [i32]
    lib.fp8pd_status_string.restype = ctypes.c_char_p
    lib.fp8pd_last_cuda_error.restype = i32
    lib.fp8pd_version.restype = i32
    for name in ("fp8_paged_decode_attention", "fp8_paged_decode_attention_noalloc",
                 "fp8_kv_append", "fp8_paged_decode_append_attention", "fp8pd_plan",
                 "fp8pd_reserve_workspace", "fp8pd_check_errors", "fp8pd_set_option",
                 "fp8pd_last_run_info", "fp8pd_timing_enable", "fp8pd_timing_collect"):
        getattr(lib, name).restype = i32
    return lib


lib = _load()


class Fp8pdError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib.fp8pd_status_string(status).decode()
        if status == -9:
            msg += f" (cudaError {lib.fp8pd_last_cuda_error()})"
        super().__init__(f"{where}: status {status}: {msg}")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != 0:
        raise Fp8pdError(status, where)


def describe(t: torch.Tensor | None) -> Tensor | None:
    """Descriptor of a torch tensor (no copy; the tensor must outlive the call)."""
    if t is None:
        return None
    if t.dim() > 4:
        raise ValueError("at most 4 dimensions")
    d = Tensor()
    d.data = t.data_ptr()
    d.dtype = _DTYPES.get(t.dtype, 0)
    d.ndim = t.dim()
    for i, (s, st) in enumerate(zip(t.shape, t.stride())):
        d.shape[i] = s
        d.stride[i] = st
    return d


def _same_device(*ts) -> None:
    """All tensors on one CUDA device, or all on the host (which the library
    then refuses during validation, before any CUDA call)."""
    devs = {t.device for t in ts if t is not None}
    if len(devs) > 1:
        raise ValueError(f"tensors on different devices: {sorted(map(str, devs))}")


def _ref(d: Tensor | None):
    return ctypes.byref(d) if d is not None else None


def _stream(stream, like: torch.Tensor | None = None) -> int:
    if stream is None:
        if like is not None and like.device.type != "cuda":
            return 0  # host tensors: the library refuses them before any CUDA call
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def fp8_paged_decode_attention(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens,
                               window: int = 0, sinks=None, sm_scale: float | None = None,
                               out=None, stream=None) -> torch.Tensor:
    """Decode attention over a paged E4M3 KV cache (see include/fp8pd.h).

    q [B, Hq, D] bf16; k_pages / v_pages [num_pages, ps, Hkv, D] uint8 views
    (any page stride that is a multiple of 16 bytes); k_scale / v_scale
    float32 [Hkv], [num_pages, Hkv] or [num_pages, ps, Hkv] (per stored
    token and KV head; K also [num_pages, ps, Hkv, G], one scale per run of
    D / G head-dim entries); block_table int32 [B, max_pages];
    seq_lens int32 [B] (keys visible to the query); sinks float32 [Hq] or
    None; sm_scale defaults to D ** -0.5. Returns out [B, Hq, D] float32.
    """
    if sm_scale is None:
        sm_scale = q.shape[-1] ** -0.5
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    _same_device(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens, sinks, out)
    ds = [describe(t) for t in (q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens)]
    ds_sinks, ds_out = describe(sinks), describe(out)
    st = lib.fp8_paged_decode_attention(*[_ref(d) for d in ds], int(window), _ref(ds_sinks),
                                        float(sm_scale), _ref(ds_out), _stream(stream, q))
    _check(st, "fp8_paged_decode_attention")
    return out


def fp8_paged_decode_attention_noalloc(q, k_pages, v_pages, k_scale, v_scale, block_table,
                                       seq_lens, window: int = 0, sinks=None,
                                       sm_scale: float | None = None, out=None,
                                       stream=None) -> torch.Tensor:
    """Same as :func:`fp8_paged_decode_attention`, for callers that cannot
    allocate device memory during the call: the split scratch is a fixed
    8 MiB array inside the library instead of an allocated workspace, so the
    library allocates nothing (``out`` must then be supplied by such a caller;
    when it is None this wrapper creates it with torch). Calls on one device
    share that array and must not overlap on the GPU."""
    if sm_scale is None:
        sm_scale = q.shape[-1] ** -0.5
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    _same_device(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens, sinks, out)
    ds = [describe(t) for t in (q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens)]
    ds_sinks, ds_out = describe(sinks), describe(out)
    st = lib.fp8_paged_decode_attention_noalloc(*[_ref(d) for d in ds], int(window),
                                                _ref(ds_sinks), float(sm_scale), _ref(ds_out),
                                                _stream(stream, q))
    _check(st, "fp8_paged_decode_attention_noalloc")
    return out


def fp8_paged_decode_attention_partial(q, k_pages, v_pages, k_scale, v_scale, block_table,
                                       seq_lens, key_ranges=None, window: int = 0,
                                       sm_scale: float | None = None, part_o=None, part_ml=None,
                                       stream=None):
    """Unnormalized decode attention over the keys [key_ranges[b, 0],
    key_ranges[b, 1]) of each sequence's window (all of it when key_ranges is
    None), for context-parallel split-KV. Returns (part_o [B, Hq, D],
    part_ml [B, Hq, 2]): the numerator, and the maximum score in log2 units
    with its sum of exponentials; no sink (fp8pd_combine_partials adds it)."""
    if sm_scale is None:
        sm_scale = q.shape[-1] ** -0.5
    if part_o is None:
        part_o = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    if part_ml is None:
        part_ml = torch.empty(q.shape[0], q.shape[1], 2, dtype=torch.float32, device=q.device)
    _same_device(q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens, key_ranges,
                 part_o, part_ml)
    ds = [describe(t) for t in (q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens,
                                key_ranges)]
    d_o, d_ml = describe(part_o), describe(part_ml)
    st = lib.fp8_paged_decode_attention_partial(*[_ref(d) for d in ds], int(window),
                                                float(sm_scale), _ref(d_o), _ref(d_ml),
                                                _stream(stream, q))
    _check(st, "fp8_paged_decode_attention_partial")
    return part_o, part_ml


def fp8pd_combine_partials(part_o, part_ml, sinks=None, out=None, stream=None) -> torch.Tensor:
    """Merges R partial results (part_o [R, B, Hq, D], part_ml [R, B, Hq, 2])
    into the attention output [B, Hq, D], adding the sink once."""
    if out is None:
        out = torch.empty(part_o.shape[1:], dtype=torch.float32, device=part_o.device)
    _same_device(part_o, part_ml, sinks, out)
    d = [describe(t) for t in (part_o, part_ml, sinks, out)]
    st = lib.fp8pd_combine_partials(*[_ref(x) for x in d], _stream(stream, part_o))
    _check(st, "fp8pd_combine_partials")
    return out


def fp8_kv_append(k_new, v_new, k_pages, v_pages, k_scale, v_scale, block_table, positions,
                  stream=None) -> None:
    """Quantize k_new / v_new [B, Hkv, D] bf16 to E4M3 and write them at
    positions[b] of each sequence's pages (see include/fp8pd.h). Scales of
    shape [num_pages, ps, Hkv] are per token: the new token's own
    max|x| / 448 is written with its codes."""
    _same_device(k_new, v_new, k_pages, v_pages, k_scale, v_scale, block_table, positions)
    sc = Scales()
    sc.k_scale = describe(k_scale)
    sc.v_scale = describe(v_scale)
    ds = [describe(t) for t in (k_new, v_new, k_pages, v_pages)]
    dt, dp = describe(block_table), describe(positions)
    st = lib.fp8_kv_append(*[_ref(d) for d in ds], ctypes.byref(sc), _ref(dt), _ref(dp),
                           _stream(stream, k_new))
    _check(st, "fp8_kv_append")


def fp8_paged_decode_append_attention(q, k_new, v_new, k_pages, v_pages, k_scale, v_scale,
                                      block_table, positions, window: int = 0, sinks=None,
                                      sm_scale: float | None = None, out=None,
                                      stream=None) -> torch.Tensor:
    """:func:`fp8_kv_append` of k_new / v_new at ``positions`` followed by
    :func:`fp8_paged_decode_attention` over ``positions + 1`` keys, in one
    launch (see include/fp8pd.h). The pools are written. Returns out
    [B, Hq, D] float32."""
    if sm_scale is None:
        sm_scale = q.shape[-1] ** -0.5
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    _same_device(q, k_new, v_new, k_pages, v_pages, k_scale, v_scale, block_table, positions,
                 sinks, out)
    ds = [describe(t) for t in (q, k_new, v_new, k_pages, v_pages, k_scale, v_scale, block_table,
                                positions)]
    ds_sinks, ds_out = describe(sinks), describe(out)
    st = lib.fp8_paged_decode_append_attention(*[_ref(d) for d in ds], int(window),
                                               _ref(ds_sinks), float(sm_scale), _ref(ds_out),
                                               _stream(stream, q))
    _check(st, "fp8_paged_decode_append_attention")
    return out


def fp8pd_e4m3_encode(x, out=None, stream=None) -> torch.Tensor:
    """E4M3 codes (uint8) of a 1-D float32 tensor with the append's rounding:
    nearest even, saturating to +-448, NaN to the NaN code (see
    include/fp8pd.h)."""
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _same_device(x, out)
    dx, do = describe(x), describe(out)
    _check(lib.fp8pd_e4m3_encode(_ref(dx), _ref(do), _stream(stream, x)), "fp8pd_e4m3_encode")
    return out


def fp8pd_plan(q, k_pages, block_table, window: int = 0) -> dict:
    info = PlanInfo()
    dq, dk, dt = describe(q), describe(k_pages), describe(block_table)
    _check(lib.fp8pd_plan(_ref(dq), _ref(dk), _ref(dt), int(window), ctypes.byref(info)),
           "fp8pd_plan")
    return {f: getattr(info, f) for f, _ in PlanInfo._fields_}


def fp8pd_reserve_workspace(nbytes: int) -> None:
    _check(lib.fp8pd_reserve_workspace(int(nbytes)), "fp8pd_reserve_workspace")


def fp8pd_check_errors(stream=None) -> int:
    flags = ctypes.c_uint32(0)
    _check(lib.fp8pd_check_errors(_stream(stream), ctypes.byref(flags)), "fp8pd_check_errors")
    return int(flags.value)


def fp8pd_set_option(option: int, value: int) -> None:
    _check(lib.fp8pd_set_option(int(option), int(value)), "fp8pd_set_option")


def fp8pd_get_option(option: int) -> int:
    return int(lib.fp8pd_get_option(int(option)))


def fp8pd_last_run_info() -> dict:
    info = RunInfo()
    _check(lib.fp8pd_last_run_info(ctypes.byref(info)), "fp8pd_last_run_info")
    return {f: getattr(info, f) for f, _ in RunInfo._fields_}


def fp8pd_timing_enable(on: bool) -> None:
    _check(lib.fp8pd_timing_enable(1 if on else 0), "fp8pd_timing_enable")


def fp8pd_timing_collect() -> dict:
    a, b = ctypes.c_double(), ctypes.c_double()
    na, nb = ctypes.c_int32(), ctypes.c_int32()
    _check(lib.fp8pd_timing_collect(ctypes.byref(a), ctypes.byref(na), ctypes.byref(b),
                                    ctypes.byref(nb)), "fp8pd_timing_collect")
    return {"attention_ms": a.value, "attention_launches": na.value, "append_ms": b.value,
            "append_launches": nb.value}
