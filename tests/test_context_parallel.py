"""Context-parallel decode on the host: shard planning and the exchange of
partials over two gloo ranks (CPU).

Each rank attends to its shard of every sequence's rows, the ranks all-gather
their partials with context_parallel.gather_partials, and the log-sum-exp
merge of the gathered partials must be the attention over all rows.  The
partial attentions and the merge are the fp64 oracle's here (the library's
kernels need a GPU; tests/test_gpu_parity.py runs them), so this checks the
shard plan and the exchange: which rows each rank takes and that every rank
ends with every rank's partial in rank order.
"""
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from head_latent_attention_03_b200.context_parallel import shard_ranges  # noqa: E402


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_ranges_cover_each_sequence_in_tiles(world):
    kv = [1, 127, 128, 129, 1000, 8193, 131073]
    r = shard_ranges(kv, world)
    assert r.shape == (world, len(kv), 2)
    for b, L in enumerate(kv):
        assert r[0, b, 0] == 0 and r[-1, b, 1] == L
        for k in range(world):
            lo, hi = r[k, b]
            assert 0 <= lo <= hi <= L and lo % 128 == 0
            if k:
                assert lo == r[k - 1, b, 1]  # contiguous, in rank order
        sizes = [int(-(-(r[k, b, 1] - r[k, b, 0]) // 128)) for k in range(world)]
        assert max(sizes) - min(sizes) <= 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    from head_latent_attention_03_b200.inputs import LayerDims
    D = LayerDims(d=32, n_h=3, d_h=8, d_c=16, d_cq=0, d_hr=4, dtype="f32")
    rng = np.random.default_rng(7)
    kv = [300, 90, 513]
    rows = [rng.standard_normal((L, D.row)) for L in kv]
    q_lat = rng.standard_normal((len(kv), D.n_h, D.d_c))
    q_r = rng.standard_normal((len(kv), D.n_h, D.d_hr))
    W = {"w_uv": rng.standard_normal((D.n_h * D.d_h, D.d_c)), "w_o": rng.standard_normal((D.d, D.n_h * D.d_h))}
    return D, W, kv, rows, q_lat, q_r


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from head_latent_attention_03_b200.context_parallel import gather_partials
    from oracle import mla_oracle as O
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        D, W, kv, rows, q_lat, q_r = _problem()
        rng_ = shard_ranges(kv, world)[rank]
        o_part = torch.zeros((len(kv), D.n_h, D.d_c), dtype=torch.float64)
        lse_part = torch.full((len(kv), D.n_h), -float("inf"), dtype=torch.float64)
        for b in range(len(kv)):
            lo, hi = rng_[b]
            if hi > lo:
                o, l, _ = O.attend_absorbed(D, W, q_lat[b], q_r[b], rows[b][lo:hi])
                o_part[b] = torch.from_numpy(o)
                lse_part[b] = torch.from_numpy(l)
        o_all, l_all = gather_partials(o_part, lse_part)
        assert o_all.shape == (world,) + tuple(o_part.shape)
        merged = [O.merge_partials([o_all[k, b].numpy() for k in range(world)],
                                   [l_all[k, b].numpy() for k in range(world)]) for b in range(len(kv))]
        np.save(os.path.join(out_dir, f"o_{rank}.npy"), np.stack([m[0] for m in merged]))
        np.save(os.path.join(out_dir, f"l_{rank}.npy"), np.stack([m[1] for m in merged]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_merge_to_the_full_attention(tmp_path):
    from oracle import mla_oracle as O
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn", join=True)
    D, W, kv, rows, q_lat, q_r = _problem()
    for r in range(world):
        o, l = np.load(tmp_path / f"o_{r}.npy"), np.load(tmp_path / f"l_{r}.npy")
        for b in range(len(kv)):
            fo, fl, _ = O.attend_absorbed(D, W, q_lat[b], q_r[b], rows[b])
            assert np.max(np.abs(o[b] - fo)) <= 1e-12 * np.max(np.abs(fo))
            assert np.max(np.abs(l[b] - fl)) <= 1e-12 * np.max(np.abs(fl))
