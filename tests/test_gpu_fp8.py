"""GPU parity of the FP8 (E4M3) KV cache path (attn_plan_kv + attn_run_fp8) against the
float64 oracle over the decoded codes (oracle.dequantize_kv: code value x per-head scale).

The decode/verify tasks decode every code exactly and compute in f16 with fp32
accumulation; the tensor-core (prefill) tasks read exact bf16 copies of the codes staged
before the launch and apply the scales in fp32. So the same tolerance as the bf16 path
applies (max abs <= 2e-2, mean abs <= 2e-3). Codes in the slots past each sequence's end
are random bytes, NaN codes included.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_attention_verify_b200 as pk
import workloads as W
from _util import assert_close, np64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def fp8_oracle_rows(b, f, seq_ids=None, token_picker=None):
    seq_ids = range(len(b.seqs)) if seq_ids is None else seq_ids
    qoff, kvoff = b.q_offsets(), b.kv_offsets()
    ks, vs = f.k_scale.cpu().numpy(), f.v_scale.cpu().numpy()
    rows, exp = [], []
    for s in seq_ids:
        sp = b.seqs[s]
        toks = list(range(sp.query_len)) if token_picker is None else token_picker(sp)
        o = kvoff[s]
        k = oracle.dequantize_kv(f.k_codes[o:o + sp.seq_len].cpu().numpy(), ks)
        v = oracle.dequantize_kv(f.v_codes[o:o + sp.seq_len].cpu().numpy(), vs)
        q = np64(b.seq_q(s)[toks])
        exp.append(oracle.attend_rows(q, k, v, sp.seq_len, sp.query_len, toks, sp.mask_kind,
                                      sp.parents or None, oracle.default_scale(b.head_dim)))
        rows.extend(qoff[s] + t for t in toks)
    return rows, np.concatenate(exp, axis=0)


def run_fp8(b, f):
    plan = pk.plan_for_batch(b, kv_fp8=True)
    out = plan.run_fp8(b.q, f.k_cache, f.v_cache_t, f.k_scale, f.v_scale)
    assert plan.check() == 0
    return out, plan


SMALL = [
    dict(seed=31, Hq=8, Hkv=2, d=64, max_ctx=80, max_q=9),
    dict(seed=32, Hq=8, Hkv=2, d=128, max_ctx=300, max_q=20),
    dict(seed=33, Hq=28, Hkv=4, d=128, max_ctx=500, max_q=6, tree_frac=0.6),
    dict(seed=34, Hq=16, Hkv=16, d=128, max_ctx=200, max_q=33),
    dict(seed=35, Hq=32, Hkv=2, d=64, max_ctx=700, max_q=5, tree_frac=0.5),
    dict(seed=36, Hq=4, Hkv=1, d=128, max_ctx=40, max_q=64, tree_frac=0.5, max_draft=64),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: f"seed{c['seed']}_H{c['Hq']}x{c['Hkv']}_d{c['d']}")
def test_fp8_small_batches_all_rows(cfg):
    cfg = dict(cfg)
    b = W.random_small(cfg.pop("seed"), device=DEV, bt_extra=2, **cfg)
    f = W.fp8_kv(b)
    out, plan = run_fp8(b, f)
    rows, exp = fp8_oracle_rows(b, f)
    assert_close(out[rows], exp, "fp8 small batch")
    plan.close()


def test_fp8_prefill_chunks_run_on_tensor_cores():
    """Long causal chunks over FP8 caches run as tensor-core tasks on bf16 staging copies:
    no prefix, a prefix that ends inside a page, a multi-tile chunk on a long prefix, and a
    decode step beside them. Every row against the oracle."""
    seqs = [W.SeqSpec(300, 300, W.CAUSAL, []), W.SeqSpec(133 + 200, 200, W.CAUSAL, []),
            W.SeqSpec(1500 + 384, 384, W.CAUSAL, []), W.SeqSpec(900, 1, W.CAUSAL, [])]
    b = W.build_batch("fp8_prefill", seqs, 16, 2, 128, seed=37, device=DEV)
    f = W.fp8_kv(b)
    out, plan = run_fp8(b, f)
    info = plan.info()
    assert info["num_prefill_items"] > 0 and info["num_decode_items"] > 0
    rows, exp = fp8_oracle_rows(b, f)
    assert_close(out[rows], exp, "fp8 prefill chunks")
    # the same batch again (staging pages rewritten, nothing carried over)
    out2 = plan.run_fp8(b.q, f.k_cache, f.v_cache_t, f.k_scale, f.v_scale)
    assert plan.check() == 0
    assert torch.equal(out, out2)
    plan.close()


def _sample(sp):
    return sorted({0, sp.query_len // 2, sp.query_len - 1})


@pytest.mark.parametrize("name", ["llama3_8b_decode", "long_ctx_split", "qwen2_7b_unified", "llama33_70b_prefill"])
def test_fp8_configs_full_size(name):
    b = W.make_config(name, device=DEV)
    f = W.fp8_kv(b)
    out, plan = run_fp8(b, f)
    seq_ids = list(range(0, len(b.seqs), max(1, len(b.seqs) // 12)))
    rows, exp = fp8_oracle_rows(b, f, seq_ids=seq_ids, token_picker=_sample)
    assert_close(out[rows], exp, f"fp8 {name}")
    # the FP8 plan reads half the bytes of the bf16 one
    bf = pk.plan_for_batch(b)
    assert plan.info()["kv_bytes"] * 2 == bf.info()["kv_bytes"]
    bf.close()
    plan.close()


def test_fp8_plan_and_run_mismatches_are_rejected():
    b = W.random_small(38, num_seqs=2, d=64, device=DEV)
    f = W.fp8_kv(b)
    p8 = pk.plan_for_batch(b, kv_fp8=True)
    with pytest.raises(pk.PkvaError) as ei:
        p8.run(b.q, b.k_cache, b.v_cache)
    assert ei.value.code == -1
    pb = pk.plan_for_batch(b)
    with pytest.raises(pk.PkvaError) as ei:
        pb.run_fp8(b.q, f.k_cache, f.v_cache_t, f.k_scale, f.v_scale)
    assert ei.value.code == -1
    L = pk.lib()
    rc = L.attn_run_fp8(p8._handle, b.q.data_ptr(), f.k_cache.data_ptr(), f.v_cache_t.data_ptr(), None,
                        f.v_scale.data_ptr(), b.q.data_ptr(), None)
    assert rc == -1
    p8.close()
    pb.close()


def _fp8_append_case(b, expect_prefill=False):
    """Append into FP8 caches: the new tokens' slots start as NaN codes; afterwards they hold
    E4M3(float32(x) / scale) of the dense input (oracle.e4m3_encode, bit for bit) and every
    other byte is unchanged; the output matches the oracle over those codes."""
    f = W.fp8_kv(b)
    k_new, v_new = W.new_token_kv(b)
    pg, sl = W.new_token_slots(b)
    ks, vs = f.k_scale.cpu().numpy(), f.v_scale.cpu().numpy()
    k_enc = oracle.e4m3_encode((k_new.float().cpu().numpy() / ks[None, :, None]).astype(np.float32))
    v_enc = oracle.e4m3_encode((v_new.float().cpu().numpy() / vs[None, :, None]).astype(np.float32))
    exp_k, exp_vt = f.k_cache.clone(), f.v_cache_t.clone()
    exp_k[pg, :, sl] = torch.from_numpy(k_enc).to(DEV)
    exp_vt[pg, :, :, sl] = torch.from_numpy(v_enc).to(DEV)
    kc, vct = f.k_cache.clone(), f.v_cache_t.clone()
    kc[pg, :, sl] = 0x7F
    vct[pg, :, :, sl] = 0x7F
    plan = pk.plan_for_batch(b, kv_fp8=True)
    if expect_prefill:
        assert plan.info()["num_prefill_items"] > 0
    out = plan.run_fp8_append(b.q, k_new, v_new, kc, vct, f.k_scale, f.v_scale)
    assert plan.check() == 0
    assert torch.equal(kc, exp_k), "k_cache codes after append"
    assert torch.equal(vct, exp_vt), "v_cache_t codes after append"
    # the oracle over the codes the caches now hold (the contiguous codes with the new ones)
    kc_codes, vc_codes = f.k_codes.clone(), f.v_codes.clone()
    kvo, qo = b.kv_offsets(), b.q_offsets()
    for s, sp in enumerate(b.seqs):
        T, L = sp.query_len, sp.seq_len
        kc_codes[kvo[s] + L - T:kvo[s] + L] = torch.from_numpy(k_enc[qo[s]:qo[s] + T]).to(DEV)
        vc_codes[kvo[s] + L - T:kvo[s] + L] = torch.from_numpy(v_enc[qo[s]:qo[s] + T]).to(DEV)
    f.k_codes, f.v_codes = kc_codes, vc_codes
    rows, exp = fp8_oracle_rows(b, f)
    assert_close(out[rows], exp, "fp8 append output")
    plan.close()


@pytest.mark.parametrize("seed, d", [(51, 64), (52, 128)])
def test_fp8_append_small(seed, d):
    b = W.random_small(seed, num_seqs=6, Hq=16, Hkv=4, d=d, max_ctx=300, max_q=40, tree_frac=0.4, device=DEV)
    _fp8_append_case(b)


def test_fp8_append_with_prefill_chunks():
    """Append over FP8 caches when long chunks run as tensor-core tasks: the staging pass
    writes those sequences' new codes into the caches, the decode tasks write theirs."""
    seqs = [W.SeqSpec(200, 200, W.CAUSAL, []), W.SeqSpec(77 + 150, 150, W.CAUSAL, []),
            W.SeqSpec(640, 1, W.CAUSAL, []), W.SeqSpec(400 + 5, 5, W.TREE, [-1, 0, 0, 1, 2]),
            W.SeqSpec(1024 + 256, 256, W.CAUSAL, [])]
    b = W.build_batch("fp8_append_prefill", seqs, 16, 4, 128, seed=54, device=DEV)
    _fp8_append_case(b, expect_prefill=True)


def test_fp8_append_rejects_bf16_paths():
    b = W.random_small(53, num_seqs=2, d=64, device=DEV)
    k_new, v_new = W.new_token_kv(b)
    p8 = pk.plan_for_batch(b, kv_fp8=True)
    with pytest.raises(pk.PkvaError):
        p8.run_append(b.q, k_new, v_new, b.k_cache, b.v_cache)
    p8.close()


@pytest.mark.parametrize("seed, heads", [(0, (16, 4)), (1, (28, 4)), (3, (64, 2)), (4, (32, 1))])
def test_fp8_shared_prefix_small_all_rows(seed, heads):
    """Shared-prefix groups over FP8 caches (attn_plan_shared_kv): the cascade tasks read bf16
    copies of the shared pages, the members' own keys stay E4M3. Every row against the oracle
    over the decoded codes; a second run is bitwise the same (arrival counters reset)."""
    b = W.random_shared_small(seed, *heads, device=DEV)
    f = W.fp8_kv(b)
    plan = pk.plan_for_batch(b, kv_fp8=True)
    assert plan.info()["num_cascade_items"] > 0
    out = plan.run_fp8(b.q, f.k_cache, f.v_cache_t, f.k_scale, f.v_scale)
    assert plan.check() == 0
    rows, exp = fp8_oracle_rows(b, f)
    assert_close(out[rows], exp, f"fp8 shared prefix seed {seed}")
    again = plan.run_fp8(b.q, f.k_cache, f.v_cache_t, f.k_scale, f.v_scale)
    assert plan.check() == 0
    assert torch.equal(out, again)
    plan.close()


def test_fp8_shared_prefix_config_full_size():
    b = W.make_shared_config("llama3_8b_shared_prefix", device=DEV)
    f = W.fp8_kv(b)
    plan = pk.plan_for_batch(b, kv_fp8=True)
    assert plan.info()["num_cascade_items"] == 4 * 8 * 2
    out = plan.run_fp8(b.q, f.k_cache, f.v_cache_t, f.k_scale, f.v_scale)
    assert plan.check() == 0
    rows, exp = fp8_oracle_rows(b, f, seq_ids=list(range(0, len(b.seqs), 5)),
                                token_picker=lambda sp: sorted({0, sp.query_len - 1}))
    assert_close(out[rows], exp, "fp8 llama3_8b_shared_prefix")
    plan.close()


def test_fp8_shared_prefix_with_fused_append():
    _fp8_append_case(W.random_shared_small(5, 16, 4, device=DEV), expect_prefill=True)


def _large_tree_seqs():
    gen = torch.Generator().manual_seed(9)
    return [W.SeqSpec(3000 + 7 * i, 1, W.CAUSAL, []) for i in range(8)] + \
        [W.SeqSpec(12000 + 5, 5, W.TREE, W.random_tree(gen, 5)), W.SeqSpec(600 + 5, 5, W.TREE, W.random_tree(gen, 5)),
         W.SeqSpec(37 + 6, 6, W.TREE, W.random_tree(gen, 6))]


@pytest.mark.parametrize("Hq, Hkv, d", [(28, 4, 128), (32, 2, 128), (32, 2, 64)])
def test_fp8_large_verify_trees_all_rows(Hq, Hkv, d):
    """Verify trees of 35 to 96 packed rows per KV head among decode steps, over FP8 caches (the
    planner keeps 16-row tasks there: row-split tasks measured slower over E4M3 pages). Every row
    against the oracle over the codes, and a second run is bitwise the same."""
    b = W.build_batch("large_trees_fp8", _large_tree_seqs(), Hq, Hkv, d, seed=92, device=DEV)
    items = pk.inspect(b.seq_lens, b.query_lens, b.mask_kinds, b.parents_flat, num_q_heads=Hq,
                       num_kv_heads=Hkv, head_dim=d, num_pages=b.k_cache.shape[0],
                       bt_stride=b.block_table.shape[1],
                       num_sms=torch.cuda.get_device_properties(0).multi_processor_count, ctas_per_sm=3)
    assert any(it["row_count"] > 16 for it in items)
    f = W.fp8_kv(b)
    out, plan = run_fp8(b, f)
    rows, exp = fp8_oracle_rows(b, f)
    assert_close(out[rows], exp, f"fp8 large trees Hq={Hq} Hkv={Hkv} d={d}")
    again = plan.run_fp8(b.q, f.k_cache, f.v_cache_t, f.k_scale, f.v_scale)
    assert plan.check() == 0
    assert torch.equal(out, again)
    plan.close()


@pytest.mark.parametrize("d", [64, 128])
def test_fp8_append_with_large_verify_trees(d):
    b = W.build_batch("large_trees_fp8_append", _large_tree_seqs(), 28, 4, d, seed=93, device=DEV)
    _fp8_append_case(b)


def test_fp8_head_dim_64_keeps_tensor_core_tasks_off():
    """Over FP8 caches the tensor-core tasks run at head_dim 128 only (their staging copies are
    head_dim 128): a head_dim 64 causal chunk runs as decode tasks, and a shared-prefix group
    at head_dim 64 is refused with PKVA_EUNSUPPORTED."""
    b = W.build_batch("fp8_d64_chunk", [W.SeqSpec(40 + 300, 300, W.CAUSAL, [])], 16, 4, 64, seed=5, device=DEV)
    f = W.fp8_kv(b)
    out, plan = run_fp8(b, f)
    assert plan.info()["num_prefill_items"] == 0
    rows, exp = fp8_oracle_rows(b, f)
    assert_close(out[rows], exp, "fp8 head_dim 64 chunk")
    plan.close()
    sb = W.random_shared_small(0, 16, 4, device=DEV, d=64)
    with pytest.raises(pk.PkvaError) as ei:
        pk.plan_for_batch(sb, kv_fp8=True)
    assert ei.value.code == -2
