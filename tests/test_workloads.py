"""Host checks of the seeded input generator's batch splitting: the per-class parts of a
mixed batch (prefill chunks, decode steps, verify trees) that the benchmark times alone."""
import numpy as np
import torch

import oracle
import workloads as W


def mixed_batch():
    seqs = [W.SeqSpec(40, 40, W.CAUSAL, []),                 # prefill chunk, no prefix
            W.SeqSpec(77, 1, W.CAUSAL, []),                  # decode
            W.SeqSpec(53, 5, W.TREE, [-1, 0, 0, 1, -1]),     # verify tree
            W.SeqSpec(120, 24, W.CAUSAL, []),                # prefill chunk on a prefix
            W.SeqSpec(16, 1, W.CAUSAL, []),                  # decode, one full page
            W.SeqSpec(33, 3, W.TREE, [-1, 0, 1])]            # verify chain
    return W.build_batch("mixed", seqs, 8, 2, 16, seed=7, bt_extra=1)


def test_classes_partition_the_sequences():
    b = mixed_batch()
    parts = W.class_batches(b)
    assert sorted(parts) == ["decode", "prefill", "verify"]
    assert [len(parts[c].seqs) for c in ("prefill", "decode", "verify")] == [2, 2, 2]
    assert sum(p.total_q for p in parts.values()) == b.total_q
    for cls, p in parts.items():
        assert all(W.seq_class(s) == cls for s in p.seqs)
        assert p.k_cache is b.k_cache and p.v_cache is b.v_cache
        assert p.block_table.shape == (len(p.seqs), b.block_table.shape[1])


def test_parts_keep_each_sequences_rows_and_pages():
    b = mixed_batch()
    ids = {c: [i for i, s in enumerate(b.seqs) if W.seq_class(s) == c] for c in W.SEQUENCE_CLASSES}
    for cls, p in W.class_batches(b).items():
        for j, i in enumerate(ids[cls]):
            assert torch.equal(p.seq_q(j), b.seq_q(i))
            k, v = p.seq_kv(j)
            k0, v0 = b.seq_kv(i)
            assert torch.equal(k, k0) and torch.equal(v, v0)
            # the part's block table addresses the same pages of the shared pool
            L = p.seqs[j].seq_len
            row = p.block_table[j].tolist()
            kc = p.k_cache.to(torch.float64).numpy()
            assert np.array_equal(oracle.gather_paged(kc, row, L), k0.to(torch.float64).numpy())


def test_oracle_on_the_parts_equals_the_whole_batch():
    b = mixed_batch()
    f64 = lambda t: t.to(torch.float64).numpy()

    def run(batch):
        kv = [batch.seq_kv(i) for i in range(len(batch.seqs))]
        return oracle.attention([f64(batch.seq_q(i)) for i in range(len(batch.seqs))],
                                [f64(k) for k, _ in kv], [f64(v) for _, v in kv],
                                batch.query_lens, batch.mask_kinds,
                                [s.parents for s in batch.seqs])
    whole = run(b)
    qo = b.q_offsets()
    for cls, p in W.class_batches(b).items():
        rows = [r for i, s in enumerate(b.seqs) if W.seq_class(s) == cls
                for r in range(qo[i], qo[i] + s.query_len)]
        assert np.array_equal(run(p), whole[rows])
