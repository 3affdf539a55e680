"""Shared helpers for the GPU parity tests: run the float64 oracle on chosen rows of a
batch and compare bf16 results against it under the stated tolerance."""
import numpy as np
import torch

import oracle

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
