"""CPU: the host logic of context-parallel split-KV, with gloo ranks.

The GPU path is: each rank attends its key slice (kernel), the ranks
all-gather their (O, m, l) partials (NCCL), every rank combines them
(kernel). Without a GPU the two host steps are checked as they run there --
the slicing (``key_slices``) and the exchange (``gather_partials``, on two
gloo ranks) -- with the partials and the combine supplied by the oracle.
"""

import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_key_slices_cover_each_sequence_in_page_aligned_balanced_runs():
    from fp8_paged_decode_split_b200.context_parallel import key_slices
    rng = np.random.default_rng(71)
    for trial in range(50):
        B = int(rng.integers(1, 6))
        ps = int(rng.choice([16, 32, 64]))
        world = int(rng.integers(1, 9))
        lens = rng.integers(0, 5000, size=B)
        ks = key_slices(lens, ps, world)
        assert ks.shape == (world, B, 2) and ks.dtype == np.int32
        for b in range(B):
            L = int(lens[b])
            assert ks[0, b, 0] == 0 and ks[-1, b, 1] == L
            for r in range(world - 1):
                assert ks[r, b, 1] == ks[r + 1, b, 0]                 # contiguous
                assert ks[r, b, 1] % ps == 0 or ks[r, b, 1] == L     # page-aligned cuts
            pages = [-(-int(e) // ps) - int(s) // ps if e > s else 0 for s, e in ks[:, b]]
            assert sum(pages) == -(-L // ps)                           # each page once
            assert max(pages) - min(pages) <= 1                       # balanced


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    """A small seeded case (two long sequences) the oracle can afford."""
    rng = np.random.default_rng(72)
    B, Hq, Hkv, D, ps = 2, 8, 2, 32, 16
    lens = np.array([700, 333])
    npg = (lens + ps - 1) // ps
    total = int(npg.sum())
    perm = rng.permutation(total)
    table = np.full((B, npg.max()), -1, np.int32)
    off = 0
    for b in range(B):
        table[b, :npg[b]] = perm[off:off + npg[b]]
        off += npg[b]
    k = rng.integers(0, 0x70, size=(total, ps, Hkv, D)).astype(np.uint8)
    v = rng.integers(0, 0x70, size=(total, ps, Hkv, D)).astype(np.uint8) | \
        (rng.integers(0, 2, size=(total, ps, Hkv, D)).astype(np.uint8) << 7)
    ks = rng.uniform(0.001, 0.01, size=(total, Hkv)).astype(np.float32)
    vs = rng.uniform(0.001, 0.01, size=(total, Hkv)).astype(np.float32)
    q = torch.randn(B, Hq, D, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    sinks = rng.standard_normal(Hq).astype(np.float32)
    return dict(q=q.double().numpy(), k=k, v=v, ks=ks, vs=vs, table=table, lens=lens, ps=ps,
                sinks=sinks)


def _worker(rank: int, world: int, port: int, out_dir: str, window: int):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import oracle as O
    from fp8_paged_decode_split_b200.context_parallel import gather_partials, key_slices
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        c = _case()
        kr = key_slices(c["lens"], c["ps"], world)[rank]
        o, ml = O.paged_decode_partial(c["q"], c["k"], c["v"], c["ks"], c["vs"], c["table"],
                                       c["lens"], kr, window=window, sm_scale=0.2)
        all_o, all_ml = gather_partials(torch.from_numpy(o), torch.from_numpy(ml))
        got = O.combine_partials(all_o.numpy(), all_ml.numpy(), c["sinks"])
        want = O.paged_decode_attention(c["q"], c["k"], c["v"], c["ks"], c["vs"], c["table"],
                                        c["lens"], window=window, sinks=c["sinks"], sm_scale=0.2)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"err": float(np.abs(got - want).max()),
                       "order": [float(x) for x in all_ml.numpy()[:, 0, 0, 1]],
                       "mine": float(ml[0, 0, 1]), "shape": list(all_o.shape)}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("window", [0, 300])
def test_two_gloo_ranks_gather_and_combine_to_the_full_attention(tmp_path, window):
    mp.start_processes(_worker, args=(2, _free_port(), str(tmp_path), window), nprocs=2,
                       join=True, start_method="spawn")
    rows = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for r, row in enumerate(rows):
        assert row["err"] < 1e-12
        assert row["shape"] == [2, 2, 8, 32]
        assert row["order"][r] == row["mine"]          # gathered in rank order
    assert rows[0]["order"] == rows[1]["order"]


def test_gather_without_a_group_is_the_local_partial():
    from fp8_paged_decode_split_b200.context_parallel import gather_partials
    assert not dist.is_initialized()
    o, ml = torch.ones(2, 3, 4), torch.zeros(2, 3, 2)
    go, gml = gather_partials(o, ml)
    assert go.shape == (1, 2, 3, 4) and gml.shape == (1, 2, 3, 2)
    assert torch.equal(go[0], o)
