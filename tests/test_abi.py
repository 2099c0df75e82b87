"""CPU-only checks of the C ABI: the library loads, exports every function
include/fp8pd.h declares, refuses bad arguments with the documented status
before touching CUDA, and plans splits as documented."""

import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def F():
    import __graft_entry__
    __graft_entry__.build()
    import fp8_paged_decode_split_b200 as F
    return F


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "fp8pd.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b((?:fp8_|fp8pd_)\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("fp8_paged_decode_attention", "fp8_kv_append",
                     "fp8_paged_decode_append_attention", "fp8pd_check_errors",
                     "fp8pd_reserve_workspace", "fp8pd_plan", "fp8pd_status_string"):
        assert required in names


def test_library_exports_every_declared_function(F):
    lib = ctypes.CDLL(F.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_version_and_status_strings(F):
    assert F.lib.fp8pd_version() == 1
    for code in range(0, -11, -1):
        assert F.lib.fp8pd_status_string(code).decode() != "unknown status"
    assert F.lib.fp8pd_status_string(-99).decode() == "unknown status"


def _args(**over):
    a = dict(
        q=torch.zeros(2, 8, 128, dtype=torch.bfloat16),
        k=torch.zeros(6, 16, 2, 128, dtype=torch.uint8),
        v=torch.zeros(6, 16, 2, 128, dtype=torch.uint8),
        ks=torch.ones(2), vs=torch.ones(6, 2),
        table=torch.zeros(2, 3, dtype=torch.int32), lens=torch.zeros(2, dtype=torch.int32),
        window=0, sinks=None, sm_scale=0.1, out=torch.zeros(2, 8, 128),
    )
    a.update(over)
    return a


def _call(F, a):
    try:
        F.fp8_paged_decode_attention(a["q"], a["k"], a["v"], a["ks"], a["vs"], a["table"], a["lens"],
                                     window=a["window"], sinks=a["sinks"], sm_scale=a["sm_scale"],
                                     out=a["out"], stream=0)
    except F.Fp8pdError as e:
        return e.status
    return 0


@pytest.mark.parametrize("over,status", [
    (dict(q=torch.zeros(2, 8, 128)), -2),                                    # q not bf16
    (dict(q=torch.zeros(2, 8, 96, dtype=torch.bfloat16),
          out=torch.zeros(2, 8, 96)), -3),                                   # pool D != q D
    (dict(k=torch.zeros(6, 16, 2, 96, dtype=torch.uint8), v=torch.zeros(6, 16, 2, 96, dtype=torch.uint8),
          q=torch.zeros(2, 8, 96, dtype=torch.bfloat16), out=torch.zeros(2, 8, 96)), -5),  # D=96
    (dict(k=torch.zeros(6, 8, 2, 128, dtype=torch.uint8), v=torch.zeros(6, 8, 2, 128, dtype=torch.uint8)), -5),
    (dict(q=torch.zeros(2, 6, 128, dtype=torch.bfloat16), out=torch.zeros(2, 6, 128),
          k=torch.zeros(6, 16, 4, 128, dtype=torch.uint8), v=torch.zeros(6, 16, 4, 128, dtype=torch.uint8),
          ks=torch.ones(4), vs=torch.ones(4)), -5),                           # Hq % Hkv
    (dict(window=-1), -6),
    (dict(sm_scale=0.0), -6),
    (dict(sm_scale=float("nan")), -6),
    (dict(ks=torch.ones(3)), -3),
    (dict(vs=torch.ones(5, 2)), -3),
    (dict(ks=torch.ones(6, 8, 2)), -3),                                      # per-token: ps
    (dict(vs=torch.ones(5, 16, 2)), -3),                                     # per-token: pages
    (dict(ks=torch.ones(6, 16, 3)), -3),                                     # per-token: Hkv
    (dict(vs=torch.ones(())), -3),                                           # 0-D scale
    (dict(ks=torch.ones(6, 16, 2, dtype=torch.float64)), -2),
    (dict(ks=torch.ones(6, 16, 2, 16)), -5),                                 # D / groups < 16
    (dict(ks=torch.ones(6, 16, 2, 3)), -5),                                  # groups not a power of 2
    (dict(vs=torch.ones(6, 16, 2, 2)), -5),                                  # V sub-row groups
    (dict(ks=torch.ones(6, 16, 3, 2)), -3),
    (dict(ks=torch.zeros(6, 16, 2, 5, dtype=torch.uint8)), -3),             # MX: D / 32 blocks
    (dict(vs=torch.zeros(6, 16, 2, dtype=torch.uint8)), -3),                 # MX: 4-D only
    (dict(vs=torch.zeros(6, 8, 2, 4, dtype=torch.uint8)), -3),               # MX: ps
    (dict(sinks=torch.zeros(7)), -3),
    (dict(table=torch.zeros(3, 3, dtype=torch.int32)), -3),
    (dict(lens=torch.zeros(2, dtype=torch.int64)), -2),
    (dict(out=torch.zeros(2, 8, 128, dtype=torch.bfloat16)), -2),
    (dict(out=torch.zeros(2, 8, 256)[:, :, ::2]), -4),                       # out not contiguous in d
    (dict(k=torch.zeros(6, 16, 2, 136, dtype=torch.uint8)[..., :128]), -4),  # strides not 16 B multiples
    (dict(k=torch.zeros(6 * 16 * 2 * 128 + 8, dtype=torch.uint8)[8:].view(6, 16, 2, 128)), -4),  # base
])
def test_validation_refuses_before_any_launch(F, over, status):
    assert _call(F, _args(**over)) == status


def test_null_descriptors(F):
    st = F.lib.fp8_paged_decode_attention(None, None, None, None, None, None, None, 0, None, 1.0,
                                          None, None)
    assert st == -1
    st = F.lib.fp8_kv_append(None, None, None, None, None, None, None, None)
    assert st == -1


def test_fused_append_attention_validation(F):
    """The fused call checks everything the attention call checks, then the
    new token's dtype and shape, before any launch."""
    a = _args()
    kn = torch.zeros(2, 2, 128, dtype=torch.bfloat16)

    def fused(**over):
        b = dict(a, kn=kn, vn=kn)
        b.update(over)
        try:
            F.fp8_paged_decode_append_attention(
                b["q"], b["kn"], b["vn"], b["k"], b["v"], b["ks"], b["vs"], b["table"], b["lens"],
                window=b["window"], sinks=b["sinks"], sm_scale=b["sm_scale"], out=b["out"],
                stream=0)
        except F.Fp8pdError as e:
            return e.status
        return 0

    assert fused(kn=kn.float()) == -2
    assert fused(vn=kn.float()) == -2
    assert fused(kn=torch.zeros(2, 3, 128, dtype=torch.bfloat16)) == -3
    assert fused(vn=torch.zeros(2, 2, 64, dtype=torch.bfloat16)) == -3
    assert fused(window=-1) == -6
    assert fused(k=torch.zeros(6, 16, 2, 136, dtype=torch.uint8)[..., :128]) == -4
    st = F.lib.fp8_paged_decode_append_attention(None, None, None, None, None, None, None, None,
                                                 None, 0, None, 1.0, None, None)
    assert st == -1


def test_append_validation(F):
    kn = torch.zeros(2, 2, 64, dtype=torch.bfloat16)
    kp = torch.zeros(4, 16, 2, 64, dtype=torch.uint8)
    ks = torch.ones(2)
    tbl = torch.zeros(2, 2, dtype=torch.int32)
    pos = torch.zeros(2, dtype=torch.int32)
    with pytest.raises(F.Fp8pdError) as e:
        F.fp8_kv_append(kn.float(), kn, kp, kp, ks, ks, tbl, pos, stream=0)
    assert e.value.status == -2
    with pytest.raises(F.Fp8pdError) as e:
        F.fp8_kv_append(kn, kn, kp, kp, torch.ones(3), ks, tbl, pos, stream=0)
    assert e.value.status == -3
    with pytest.raises(F.Fp8pdError) as e:
        F.fp8_kv_append(kn, kn, kp, kp, ks, ks, tbl, torch.zeros(3, dtype=torch.int32), stream=0)
    assert e.value.status == -3
    with pytest.raises(F.Fp8pdError) as e:                  # per-token scale with the wrong ps
        F.fp8_kv_append(kn, kn, kp, kp, torch.ones(4, 8, 2), ks, tbl, pos, stream=0)
    assert e.value.status == -3
    with pytest.raises(F.Fp8pdError) as e:                  # 32 groups: more than 16
        F.fp8_kv_append(kn, kn, kp, kp, torch.ones(4, 16, 2, 32), ks, tbl, pos, stream=0)
    assert e.value.status == -5


def test_encode_validation(F):
    x = torch.zeros(8)
    c = torch.zeros(8, dtype=torch.uint8)
    for bad, status in ((dict(x=x.double()), -2), (dict(c=c.to(torch.int32)), -2),
                        (dict(c=torch.zeros(7, dtype=torch.uint8)), -3),
                        (dict(x=torch.zeros(2, 4)), -3)):
        a = dict(x=x, c=c)
        a.update(bad)
        with pytest.raises(F.Fp8pdError) as e:
            F.fp8pd_e4m3_encode(a["x"], out=a["c"], stream=0)
        assert e.value.status == status
    assert F.lib.fp8pd_e4m3_encode(None, None, None) == -1


def test_options_roundtrip(F):
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 7)
    assert F.fp8pd_get_option(F.OPT_NUM_SPLITS) == 7
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)
    F.fp8pd_set_option(F.OPT_SCHEDULE, 3)
    assert F.fp8pd_get_option(F.OPT_SCHEDULE) == 3
    F.fp8pd_set_option(F.OPT_SCHEDULE, 0)
    for bad in (2, 5, -1):
        with pytest.raises(F.Fp8pdError):
            F.fp8pd_set_option(F.OPT_SCHEDULE, bad)
    assert F.fp8pd_get_option(F.OPT_SCHEDULE) == 0
    assert F.fp8pd_get_option(F.OPT_WAIT_POLLS) == 1 << 17
    F.fp8pd_set_option(F.OPT_WAIT_POLLS, 64)
    assert F.fp8pd_get_option(F.OPT_WAIT_POLLS) == 64
    F.fp8pd_set_option(F.OPT_WAIT_POLLS, 1 << 17)
    for opt, bad in ((F.OPT_WAIT_POLLS, 0), (F.OPT_WAIT_POLLS, (1 << 20) + 1),
                     (F.OPT_TEST_STALL, 2), (F.OPT_TEST_STALL, -1)):
        with pytest.raises(F.Fp8pdError):
            F.fp8pd_set_option(opt, bad)
    assert F.fp8pd_get_option(F.OPT_TEST_STALL) == 0
    assert F.fp8pd_get_option(F.OPT_COMPUTE) == 0
    F.fp8pd_set_option(F.OPT_COMPUTE, 1)
    assert F.fp8pd_get_option(F.OPT_COMPUTE) == 1
    F.fp8pd_set_option(F.OPT_COMPUTE, 0)
    for bad in (2, -1):
        with pytest.raises(F.Fp8pdError):
            F.fp8pd_set_option(F.OPT_COMPUTE, bad)
    F.fp8pd_set_option(F.OPT_K_DECODE, 2)
    assert F.fp8pd_get_option(F.OPT_K_DECODE) == 2
    F.fp8pd_set_option(F.OPT_K_DECODE, 1)
    with pytest.raises(F.Fp8pdError):
        F.fp8pd_set_option(F.OPT_K_DECODE, 3)
    assert F.fp8pd_get_option(F.OPT_KERNEL) == 0
    for k in (1, 2, 0):
        F.fp8pd_set_option(F.OPT_KERNEL, k)
        assert F.fp8pd_get_option(F.OPT_KERNEL) == k
    for bad in (3, -1):
        with pytest.raises(F.Fp8pdError):
            F.fp8pd_set_option(F.OPT_KERNEL, bad)
    with pytest.raises(F.Fp8pdError):
        F.fp8pd_set_option(99, 1)
    with pytest.raises(F.Fp8pdError):
        F.fp8pd_set_option(F.OPT_NUM_SPLITS, -1)


def _plan(F, B, Hq, Hkv, D, ps, max_pages, window=0):
    q = torch.zeros(B, Hq, D, dtype=torch.bfloat16)
    k = torch.zeros(1, ps, Hkv, D, dtype=torch.uint8).expand(2, ps, Hkv, D)
    k = torch.as_strided(torch.zeros(ps * Hkv * D, dtype=torch.uint8), (2, ps, Hkv, D), (0, Hkv * D, D, 1))
    t = torch.as_strided(torch.zeros(1, dtype=torch.int32), (B, max_pages), (0, 0))
    return F.fp8pd_plan(q, k, t, window)


@pytest.fixture
def split_schedule(F):
    F.fp8pd_set_option(F.OPT_SCHEDULE, 1)
    yield
    F.fp8pd_set_option(F.OPT_SCHEDULE, 0)


def test_planner_fills_the_device_with_enough_work_per_split(F, split_schedule):
    # long context, one sequence: many splits, each >= 256 keys
    p = _plan(F, 1, 64, 8, 128, 64, 2049)
    assert p["num_splits"] > 16 and p["combine"] == 1
    assert 2049 / p["num_splits"] >= 4
    S = p["num_splits"]
    assert p["workspace_bytes"] >= 1 * 64 * S * (128 + 2) * 4 + 8 * 4
    NG = (S + 7) // 8
    assert p["workspace_bytes"] <= 64 * (S + NG) * (128 + 2) * 4 + 8 * (1 + NG) * 4 + 5 * 256
    # no split may cover more than 8,192 keys: 1 Mi keys on 16-token pages
    p = _plan(F, 64, 64, 8, 64, 16, 65537)
    assert p["num_splits"] >= 129 and 65537 * 16 / p["num_splits"] <= 8192 + 16
    assert p["num_splits"] <= 256
    # more than 256 splits of 8,192 keys in one sequence is refused
    with pytest.raises(F.Fp8pdError) as e:
        _plan(F, 1, 8, 8, 128, 16, 256 * 512 + 1)
    assert e.value.status == -10
    assert _plan(F, 1, 8, 8, 128, 16, 256 * 512 + 1, window=4096)["num_splits"] >= 1
    # short window: one split, no combine, no workspace
    p = _plan(F, 64, 64, 8, 64, 16, 513, window=128)
    assert p["num_splits"] == 1 and p["combine"] == 0 and p["workspace_bytes"] == 0
    # head groups of at most 8 query heads
    assert _plan(F, 2, 32, 2, 128, 16, 10)["head_groups"] == 2
    assert _plan(F, 2, 24, 2, 128, 16, 10)["head_groups"] == 2
    assert _plan(F, 2, 8, 8, 128, 16, 10)["head_groups"] == 1
    # forced split count, capped by the pages there are
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, 5)
    try:
        assert _plan(F, 4, 32, 8, 128, 16, 100)["num_splits"] == 5
        assert _plan(F, 4, 32, 8, 128, 16, 3)["num_splits"] == 3
        assert _plan(F, 4, 32, 8, 128, 16, 6000)["num_splits"] == 12   # raised: <= 8,192 keys each
        F.fp8pd_set_option(F.OPT_NUM_SPLITS, 1000)
        assert 240 <= _plan(F, 4, 32, 8, 128, 16, 5000)["num_splits"] <= 256  # capped
    finally:
        F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)


def test_planner_default_schedule(F):
    """The planner's own choice: proportional splits for full attention and
    long windows with enough work when their grid is one wave, uniform splits
    otherwise. Without a GPU it assumes
    148 SMs and the launch-bound blocks per SM."""
    assert _plan(F, 32, 32, 8, 128, 16, 257)["schedule"] == 3           # Llama-like
    assert _plan(F, 1, 64, 8, 128, 64, 2049)["schedule"] == 3           # one 131k-key sequence
    assert _plan(F, 16, 16, 2, 512, 32, 513)["schedule"] == 3           # any head dim
    assert _plan(F, 64, 64, 8, 64, 16, 513)["schedule"] == 1            # gpt-oss-like: two waves
    assert _plan(F, 64, 64, 8, 64, 16, 513, window=4096)["schedule"] == 1
    assert _plan(F, 8, 64, 8, 128, 64, 2049)["schedule"] == 1           # 8 x 131k keys: > 1 wave
    assert _plan(F, 64, 64, 8, 64, 16, 513, window=128)["schedule"] == 1
    assert _plan(F, 1, 8, 2, 64, 16, 16)["schedule"] == 1               # too little work
    assert _plan(F, 1025, 8, 8, 128, 16, 400)["schedule"] == 1          # more than 1,024 sequences


def test_planner_proportional_splits(F):
    """Schedule 3: one wave of split-kernel blocks per KV head x head group
    (148 SMs x the split kernel's blocks per SM without a GPU), shared among
    the sequences in the kernel."""
    F.fp8pd_set_option(F.OPT_SCHEDULE, 3)
    try:
        p = _plan(F, 32, 32, 8, 128, 16, 257)
        assert p["schedule"] == 3 and p["combine"] == 1 and p["num_splits"] == 0
        assert p["grid_blocks"] % 8 == 0 and p["grid_blocks"] >= 8 * 32
        # every sequence needs room for splits of at most 8,192 keys
        p = _plan(F, 4, 8, 8, 128, 64, 2049)                       # 131,136 keys: 17 splits each
        assert p["schedule"] == 3 and p["grid_blocks"] >= 8 * 4 * 17
        assert _plan(F, 1025, 8, 8, 128, 16, 4)["schedule"] == 1    # more than 1,024 sequences
        F.fp8pd_set_option(F.OPT_NUM_SPLITS, 2)
        assert _plan(F, 32, 32, 8, 128, 16, 257)["schedule"] == 1   # a forced split count wins
    finally:
        F.fp8pd_set_option(F.OPT_NUM_SPLITS, 0)
        F.fp8pd_set_option(F.OPT_SCHEDULE, 0)


def test_planner_plans_for_the_kernel_that_runs(F):
    """With the tensor-memory kernel requested (head dim 64 / 128), the plan
    counts that kernel's blocks per SM (one without a GPU, against four or
    five for the split kernel), so it plans fewer blocks; head dims it does not
    take plan as before."""
    try:
        F.fp8pd_set_option(F.OPT_KERNEL, 1)
        split = _plan(F, 8, 64, 8, 128, 64, 2049)
        d256 = _plan(F, 4, 16, 8, 256, 32, 200)
        F.fp8pd_set_option(F.OPT_KERNEL, 2)
        umma = _plan(F, 8, 64, 8, 128, 64, 2049)
        assert umma["grid_blocks"] < split["grid_blocks"]
        assert umma["warps"] == umma["grid_blocks"] * 10
        assert _plan(F, 4, 16, 8, 256, 32, 200) == d256
    finally:
        F.fp8pd_set_option(F.OPT_KERNEL, 0)


def test_planner_counts_the_head_dim_split_warps(F):
    """At head dim 512 (page or head scales, the default f32 compute and
    decodes) a tile stream is two warps, each on half of the head dim: the
    plan's warps are a multiple of twice its blocks and more than the four
    whole-width warps per block; other head dims keep four warps per block."""
    d512 = _plan(F, 16, 16, 2, 512, 32, 513)
    wpb, rem = divmod(d512["warps"], d512["grid_blocks"])
    assert rem == 0 and wpb % 2 == 0 and wpb > 4
    for D in (64, 128, 256):
        p = _plan(F, 8, 16, 2, D, 32, 200)
        assert p["warps"] == p["grid_blocks"] * 4, D


def test_partial_and_combine_validation(F):
    """The context-parallel entry points refuse bad arguments before any
    launch: the partial call as the attention call plus its own outputs and
    key ranges; the combine call its shapes, layout and rank count."""
    a = _args()
    kw = dict(window=0, sm_scale=0.1, stream=0)

    def partial(**over):
        b = dict(a, kr=torch.zeros(2, 2, dtype=torch.int32), po=torch.zeros(2, 8, 128),
                 pml=torch.zeros(2, 8, 2))
        b.update(over)
        try:
            F.fp8_paged_decode_attention_partial(b["q"], b["k"], b["v"], b["ks"], b["vs"], b["table"],
                                                 b["lens"], b["kr"], part_o=b["po"],
                                                 part_ml=b["pml"], **kw)
        except F.Fp8pdError as e:
            return e.status
        return 0
    assert partial(kr=torch.zeros(2, 3, dtype=torch.int32)) == -3
    assert partial(kr=torch.zeros(2, 2, dtype=torch.int64)) == -2
    assert partial(pml=torch.zeros(2, 8, 3)) == -3
    assert partial(po=torch.zeros(2, 16, 128)[:, ::2]) == -4          # not contiguous
    assert partial(q=torch.zeros(2, 8, 128)) == -2

    def combine(o, ml, sinks=None, out=None):
        try:
            F.fp8pd_combine_partials(o, ml, sinks=sinks, out=out, stream=0)
        except F.Fp8pdError as e:
            return e.status
        return 0
    o, ml = torch.zeros(3, 2, 8, 128), torch.zeros(3, 2, 8, 2)
    assert combine(o, ml[:2]) == -3
    assert combine(o, ml, out=torch.zeros(2, 8, 64)) == -3
    assert combine(o, ml, sinks=torch.zeros(5)) == -3
    assert combine(o.double(), ml) == -2
    assert combine(o[:, :, :, :126], ml) == -5                        # D % 4
    assert combine(torch.zeros(1025, 1, 1, 4), torch.zeros(1025, 1, 1, 2)) == -10
    assert F.lib.fp8pd_combine_partials(None, None, None, None, None) == -1
