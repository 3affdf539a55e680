"""Head / sequence sharding of a batch over several GPUs (paged_kv_attention_verify_b200.shard;
no exchange inside attention). CPU checks: the layout (tp x sp = world, KV heads never split),
exact coverage of every (query head, sequence) by one rank, and, with gloo ranks on CPU,
that each rank's shard computed alone (the float64 oracle standing in for the GPU) gathers
into the whole batch's result."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import workloads as W
from paged_kv_attention_verify_b200 import shard as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("world, hkv, expect", [(1, 8, (1, 1)), (2, 8, (2, 1)), (8, 8, (8, 1)),
                                                (8, 4, (4, 2)), (4, 2, (2, 2)), (3, 8, (1, 3)),
                                                (6, 4, (2, 3)), (8, 1, (1, 8))])
def test_layout(world, hkv, expect):
    tp, sp = S.shard_layout(world, hkv)
    assert (tp, sp) == expect and tp * sp == world and hkv % tp == 0


@pytest.mark.parametrize("world, hq, hkv, nseq", [(2, 32, 8, 5), (8, 28, 4, 7), (4, 16, 16, 3), (6, 8, 2, 2)])
def test_every_head_and_sequence_once(world, hq, hkv, nseq):
    seen = {}
    for r in range(world):
        tpr, spr, tp, sp = S.shard_coords(r, world, hkv)
        kv0, kv1, q0, q1 = S.head_range(tpr, tp, hq, hkv)
        for h in range(q0, q1):
            assert kv0 <= h // (hq // hkv) < kv1              # a query head travels with its KV head
            for s in S.sequence_subset(nseq, spr, sp):
                seen[(h, s)] = seen.get((h, s), 0) + 1
    assert seen == {(h, s): 1 for h in range(hq) for s in range(nseq)}


def _assemble(b, world, runner):
    """Run each rank's shard with `runner(shard) -> [rows, heads, d]` and put its rows and
    head columns back where they belong in the whole batch's output."""
    out = np.zeros((b.total_q, b.num_q_heads, b.head_dim))
    qo = b.q_offsets()
    for r in range(world):
        part = W.shard_batch(b, r, world)
        tpr, spr, tp, sp = S.shard_coords(r, world, b.num_kv_heads)
        kv0, kv1, q0, q1 = S.head_range(tpr, tp, b.num_q_heads, b.num_kv_heads)
        res = runner(part)
        row = 0
        for s in S.sequence_subset(len(b.seqs), spr, sp):
            T = b.seqs[s].query_len
            out[qo[s]:qo[s] + T, q0:q1] = res[row:row + T]
            row += T
    return out


def _oracle_all(b):
    return oracle.attention([np.asarray(b.seq_q(s).double()) for s in range(len(b.seqs))],
                            [np.asarray(b.seq_kv(s)[0].double()) for s in range(len(b.seqs))],
                            [np.asarray(b.seq_kv(s)[1].double()) for s in range(len(b.seqs))],
                            b.query_lens, b.mask_kinds, [sp.parents or None for sp in b.seqs])


@pytest.mark.parametrize("world", [2, 3, 8])
def test_shards_gather_into_the_whole_batch(world):
    b = W.random_small(41, num_seqs=5, Hq=16, Hkv=4, d=32, max_ctx=40, max_q=6, tree_frac=0.4)
    got = _assemble(b, world, lambda part: _oracle_all(part) if part.seqs else np.zeros((0, part.num_q_heads, 32)))
    assert np.allclose(got, _oracle_all(b), atol=1e-12, rtol=0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    b = W.random_small(42, num_seqs=4, Hq=8, Hkv=2, d=16, max_ctx=30, max_q=4)
    part = W.shard_batch(b, rank, world)
    mine = torch.from_numpy(_oracle_all(part))
    parts = [None] * world
    dist.all_gather_object(parts, (rank, mine))            # test harness only: the path needs none
    if rank == 0:
        got = _assemble(b, world, lambda p, it=iter(sorted(parts, key=lambda x: x[0])): next(it)[1].numpy())
        q.put(float(np.abs(got - _oracle_all(b)).max()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_each_compute_their_shard():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    err = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert err < 1e-12
