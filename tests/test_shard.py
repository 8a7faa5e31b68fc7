"""Multi-process CPU tests of the head-sharded and sequence-sharded paths
(block_sparse_attention_coarse_b200.shard) on gloo ranks.

Each rank is a separate `python tests/shard_worker.py` process on
127.0.0.1; the per-head computation is the fp64 oracle, so the tests check
the data movement only: every rank's result must equal, bit for bit, the
matching slice of one single-process oracle run over all heads, and the
regrouped layout must equal a direct slice of the full inputs.
"""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_coarse_b200 import shard

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
import shard_worker as W  # noqa: E402


@pytest.mark.parametrize("n", range(0, 23))
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_head_range_is_a_balanced_partition(n, world):
    ranges = [shard.head_range(n, r, world) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == n
    for (lo, hi), (lo2, _) in zip(ranges, ranges[1:]):
        assert hi == lo2
    sizes = [hi - lo for lo, hi in ranges]
    assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1
    assert sizes == sorted(sizes, reverse=True)


def test_head_range_rejects_bad_rank():
    for rank, world in ((2, 2), (-1, 2), (0, 0)):
        with pytest.raises(ValueError):
            shard.head_range(8, rank, world)


def free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def single_process(rope_base=None):
    q, k, v = W.inputs()
    return W.oracle_compute(rope_base)(q, k, v, W.B, W.H).numpy()


@pytest.mark.parametrize("world", [2, 4])
def test_ranks_match_single_process(tmp_path, world):
    port = str(free_port())
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", OMP_NUM_THREADS="1")
    procs = [subprocess.Popen([sys.executable, os.path.join(HERE, "shard_worker.py"), str(r), str(world), port,
                               str(tmp_path)], env=env, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)
             for r in range(world)]
    logs = []
    try:
        for p in procs:
            out, _ = p.communicate(timeout=300)
            logs.append(out.decode(errors="replace")[-2000:])
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
    assert all(p.returncode == 0 for p in procs), logs

    q, _, _ = (t.numpy() for t in W.inputs())
    full = single_process()
    full_rope = single_process(500.0)
    assert not np.array_equal(full, full_rope)
    L = W.L_SRC + W.L_CTX
    Lc, Hl = L // world, W.H // world
    covered = []
    for r in range(world):
        res = np.load(tmp_path / f"rank{r}.npz")
        seq = slice(r * Lc, (r + 1) * Lc)
        # sequence chunks of every head -> full sequences of heads [r*H/N, (r+1)*H/N)
        np.testing.assert_array_equal(res["heads"], q[:, r * Hl:(r + 1) * Hl])
        np.testing.assert_array_equal(res["back"], q[:, :, seq])
        np.testing.assert_array_equal(res["out_seq"], full[:, :, seq])
        np.testing.assert_array_equal(res["out_rope"], full_rope[:, :, seq])
        lo, hi = int(res["lo"]), int(res["hi"])
        assert (lo, hi) == shard.head_range(W.B * W.H, r, world)
        np.testing.assert_array_equal(res["out_heads"], full.reshape(W.B * W.H, L, W.D)[lo:hi])
        covered.extend(range(lo, hi))
    assert covered == list(range(W.B * W.H))


def test_sequence_chunks_must_cover_the_sequence():
    """The length check runs before any communication (world size 1, no
    process group needed for the shape check to fire)."""
    class P:
        D, L_src, L_ctx = 16, 40, 24
    if not torch.distributed.is_initialized():
        torch.distributed.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{free_port()}", rank=0,
                                             world_size=1)
    try:
        x = torch.zeros(1, 2, 63, 16, dtype=torch.float64)
        with pytest.raises(ValueError):
            shard.isa_attention_seq_sharded(x, x, x, P, compute=lambda *a: None)
        y = torch.zeros(1, 2, 64, 16, dtype=torch.float64)
        out = shard.isa_attention_seq_sharded(y, y, y, P, compute=lambda q, k, v, b, h: q + 1)
        assert torch.equal(out, y + 1)
    finally:
        torch.distributed.destroy_process_group()


def test_oracle_compute_of_a_head_subset_is_the_subset():
    """Per-head independence the sharding relies on: the oracle forward of a
    subset of heads equals that subset of the all-heads forward."""
    q, k, v = W.inputs()
    full = single_process()
    sub = W.oracle_compute()(q[:, 1:3].contiguous(), k[:, 1:3].contiguous(), v[:, 1:3].contiguous(), 1, 2).numpy()
    np.testing.assert_array_equal(sub, full[:, 1:3])
    p = O.Params(D=W.D, L_src=W.L_SRC, L_ctx=W.L_CTX, block=W.BLOCK, alpha_s=0.5, alpha_f=0.5, alpha_ns=0.25)
    assert len(O.isa_forward(q.numpy(), k.numpy(), v.numpy(), p)[2]) == W.B * W.H
