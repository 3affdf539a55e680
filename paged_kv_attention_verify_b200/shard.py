"""Splitting one batch's attention over several GPUs (one process per GPU).

Attention has no exchange between KV heads or between sequences, so a batch splits over P
GPUs with no collective inside the path: tp KV-head groups x sp sequence subsets, tp * sp = P.
Each GPU holds the KV cache of its KV heads only and computes the query heads of those KV
heads for its sequences; its output columns are already where a row-parallel output
projection of the surrounding model wants them.

Arctic Inference with Shift Parallelism (arXiv 2507.11830), review page, section 3: the KV
cache keeps one layout when sequence parallelism x tensor parallelism equals the GPU count
(SP x TP = P); here tp takes the largest share the KV-head count allows and sp the rest.
"""
from __future__ import annotations

from math import gcd
from typing import List, Tuple


def shard_layout(world: int, num_kv_heads: int) -> Tuple[int, int]:
    """(tp, sp) with tp * sp == world: tp is the largest divisor of ``world`` that also divides
    ``num_kv_heads`` (KV heads are never split), sp the rest (sequences split sp ways)."""
    if world < 1 or num_kv_heads < 1:
        raise ValueError("world and num_kv_heads must be >= 1")
    tp = gcd(world, num_kv_heads)
    return tp, world // tp


def shard_coords(rank: int, world: int, num_kv_heads: int) -> Tuple[int, int, int, int]:
    """(tp_rank, sp_rank, tp, sp) of ``rank``: ranks tp_rank = rank % tp share a KV-head group."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    tp, sp = shard_layout(world, num_kv_heads)
    return rank % tp, rank // tp, tp, sp


def head_range(tp_rank: int, tp: int, num_q_heads: int, num_kv_heads: int) -> Tuple[int, int, int, int]:
    """(kv0, kv1, q0, q1): the KV heads [kv0, kv1) of KV-head group ``tp_rank`` and the query
    heads [q0, q1) that read them (query head h reads KV head h // (Hq / Hkv))."""
    if num_kv_heads % tp or num_q_heads % num_kv_heads:
        raise ValueError("tp must divide num_kv_heads, and num_kv_heads must divide num_q_heads")
    per = num_kv_heads // tp
    G = num_q_heads // num_kv_heads
    kv0 = tp_rank * per
    return kv0, kv0 + per, kv0 * G, (kv0 + per) * G


def sequence_subset(num_seqs: int, sp_rank: int, sp: int) -> List[int]:
    """The sequences of subset ``sp_rank``: every sp-th sequence (round robin)."""
    return list(range(sp_rank, num_seqs, sp))
