"""Shared helpers for the GPU parity tests: run the float64 oracle on chosen rows of a
batch and compare bf16 results against it under the stated tolerance."""
import numpy as np
import torch

import oracle
import workloads as W

# tolerance of the bf16-in / fp32-accumulate / bf16-out path against the float64 oracle
TOL_MAX_ABS = 2e-2
TOL_MEAN_ABS = 2e-3


def np64(t):
    return t.detach().to(torch.float64).cpu().numpy()


def oracle_rows(batch, seq_ids=None, token_picker=None):
    """Expected outputs (float64) for the chosen sequences / tokens.

    Returns (row_index_list, expected [n_rows, Hq, D]) where row indices address the
    packed q/out layout of the batch.
    """
    seq_ids = range(len(batch.seqs)) if seq_ids is None else seq_ids
    qoff = batch.q_offsets()
    rows, exp = [], []
    for s in seq_ids:
        sp = batch.seqs[s]
        toks = list(range(sp.query_len)) if token_picker is None else token_picker(sp)
        k, v = batch.seq_kv(s)
        q = np64(batch.seq_q(s)[toks])
        scale = oracle.default_scale(batch.head_dim)
        exp.append(oracle.attend_rows(q, np64(k), np64(v), sp.seq_len, sp.query_len, toks,
                                      sp.mask_kind, sp.parents or None, scale))
        rows.extend(qoff[s] + t for t in toks)
    return rows, np.concatenate(exp, axis=0)


def errors(got, exp):
    d = np.abs(np64(got) - exp)
    return float(d.max()), float(d.mean())


def assert_close(got, exp, what=""):
    mx, mean = errors(got, exp)
    assert np.isfinite(mx), f"{what}: non-finite output"
    assert mx <= TOL_MAX_ABS and mean <= TOL_MEAN_ABS, f"{what}: max abs {mx:.3e}, mean abs {mean:.3e}"
    return mx, mean


def tc_verify_seqs():
    """Decode steps beside verify trees and short causal chunks that run as tensor-core tasks
    (16 query / 4 KV heads: 20 to 128 packed rows per KV head, at least 512 keys)."""
    gen = torch.Generator().manual_seed(12)
    return [W.SeqSpec(3000 + 7 * i, 1, W.CAUSAL, []) for i in range(6)] + [
        W.SeqSpec(640 + 7, 7, W.TREE, W.random_tree(gen, 7)),       # new keys start a KV tile
        W.SeqSpec(766 + 6, 6, W.TREE, W.random_tree(gen, 6)),       # new keys cross a tile boundary
        W.SeqSpec(4100, 5, W.TREE, W.random_tree(gen, 5)),          # two chunks of KV tiles
        W.SeqSpec(1000 + 20, 20, W.CAUSAL, []),                     # a short causal chunk: 80 rows
        W.SeqSpec(2500, 30, W.CAUSAL, []),                          # 120 rows
        W.SeqSpec(513, 8, W.TREE, W.random_tree(gen, 8)),           # one key past the threshold
        W.SeqSpec(128 * 5 + 1, 1, W.CAUSAL, []),
        W.SeqSpec(600, 32, W.TREE, W.random_tree(gen, 32)),         # 128 rows: a full tile
    ]


def tc_verify_wide_seqs():
    """Decode steps beside tensor-core verify units at their row limit (8 query / 4 KV heads:
    64-node trees = 128 packed rows, a 63-token causal chunk = 126 rows, a 40-node chain)."""
    gen = torch.Generator().manual_seed(21)
    return [W.SeqSpec(2000 + 9 * i, 1, W.CAUSAL, []) for i in range(12)] + [
        W.SeqSpec(700 + 64, 64, W.TREE, W.random_tree(gen, 64)),
        W.SeqSpec(740 + 64, 64, W.TREE, W.random_tree(gen, 64)),       # new keys 740..803 cross 768
        W.SeqSpec(4500 + 63, 63, W.CAUSAL, []),                         # 36 KV tiles: two chunks
        W.SeqSpec(1000 + 40, 40, W.TREE, list(range(-1, 39))),          # a chain
    ]
