"""Pins for the float64 oracle: facts fixed by the definition of softmax attention and
by the problem statement, each checked against something other than the oracle itself.

Pins (every one runs on CPU):
  1  softmax rows sum to 1 (weights directly, and output = 1 when V = 1)
  2  a single allowed key returns its V exactly (row 0 of a prefill with no prefix)
  3  identical keys return the mean of V over the allowed set (checks the mask's set)
  4  a chain-shaped draft tree gives the causal result
  5  decoding one token at a time reproduces the rows of one full prefill
  6  any page permutation of the block table gives identical output
  7  brute force with pure-Python loops on tiny inputs
  8  torch's float64 scaled_dot_product_attention with an explicit boolean mask
  9  the split-KV log-sum-exp merge equals the unsplit result

``test_planted_mistakes_are_caught`` swaps plausible mistakes into the oracle (on the
CPU) and checks that at least one pin fails for each, so the pins are known to bite.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W


# ----------------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------------

def np64(t):
    return t.detach().to(torch.float64).cpu().numpy()


def batch_lists(b):
    qs, ks, vs = [], [], []
    for i in range(len(b.seqs)):
        k, v = b.seq_kv(i)
        qs.append(np64(b.seq_q(i)))
        ks.append(np64(k))
        vs.append(np64(v))
    return qs, ks, vs


def run_oracle(b, scale=None):
    qs, ks, vs = batch_lists(b)
    return oracle.attention(qs, ks, vs, b.query_lens, b.mask_kinds,
                            [s.parents for s in b.seqs], scale)


def rng_arrays(seed, T, L, Hq, Hkv, d):
    r = np.random.default_rng(seed)
    return (r.standard_normal((T, Hq, d)), r.standard_normal((L, Hkv, d)),
            r.standard_normal((L, Hkv, d)))


def brute_force(q, k, v, L, T, mask_kind, parents, scale):
    """Pure-Python triple loop, written independently of the oracle."""
    Tq, Hq, d = len(q), len(q[0]), len(q[0][0])
    Hkv = len(k[0])
    G = Hq // Hkv
    prefix = L - T
    anc = []
    for i in range(T):
        s = {i}
        if mask_kind == W.TREE:
            a = parents[i]
            while a != -1:
                s.add(a)
                a = parents[a]
        anc.append(s)
    out = [[[0.0] * d for _ in range(Hq)] for _ in range(T)]
    for i in range(T):
        for h in range(Hq):
            g = h // G
            keys = []
            for j in range(L):
                if mask_kind == W.CAUSAL:
                    ok = j <= prefix + i
                else:
                    ok = j < prefix or (j - prefix) in anc[i]
                if ok:
                    keys.append(j)
            sc = []
            for j in keys:
                acc = 0.0
                for c in range(d):
                    acc += q[i][h][c] * k[j][g][c]
                sc.append(acc * scale)
            mx = max(sc)
            e = [math.exp(x - mx) for x in sc]
            z = sum(e)
            for c in range(d):
                out[i][h][c] = sum(e[n] * v[keys[n]][g][c] for n in range(len(keys))) / z
    return out


# ----------------------------------------------------------------------------------
# the pins, written as checks so the planted-mistake test can run them again
# ----------------------------------------------------------------------------------

def pin1_rows_sum_to_one():
    q, k, v = rng_arrays(1, 6, 30, 4, 2, 8)
    for mk, par in ((W.CAUSAL, None), (W.TREE, [-1, 0, 0, 1, -1, 4])):
        al = oracle.allowed_mask(30, 6, mk, par)
        w = oracle.attention_weights(q, k, al, 0.3)
        assert np.allclose(w.sum(axis=2), 1.0, atol=1e-12)
        assert np.all(w[~np.broadcast_to(al[:, None, :], w.shape)] == 0.0)
        out = oracle.attend_seq(q, k, np.ones_like(v), al, 0.3)
        assert np.allclose(out, 1.0, atol=1e-12)


def pin2_single_key():
    q, k, v = rng_arrays(2, 5, 5, 4, 2, 8)
    out = oracle.attention([q], [k], [v], [5], [W.CAUSAL], [[]], 0.5)
    for h in range(4):
        assert np.array_equal(out[0, h], v[0, h // 2])


def pin3_identical_keys_give_mean():
    L, T, Hq, Hkv, d = 23, 6, 6, 3, 8
    q, k, v = rng_arrays(3, T, L, Hq, Hkv, d)
    k[:] = k[0:1]
    par = [-1, 0, 1, 0, -1, 4]
    for mk in (W.CAUSAL, W.TREE):
        out = oracle.attention([q], [k], [v], [T], [mk], [par if mk == W.TREE else []], 0.7)
        prefix = L - T
        for i in range(T):
            if mk == W.CAUSAL:
                keys = list(range(prefix + i + 1))
            else:
                keys = list(range(prefix)) + [prefix + a for a in {0: [0], 1: [0, 1], 2: [0, 1, 2],
                                                                  3: [0, 3], 4: [4], 5: [4, 5]}[i]]
            for h in range(Hq):
                assert np.allclose(out[i, h], v[keys, h // (Hq // Hkv)].mean(axis=0), atol=1e-12)


def pin4_chain_tree_is_causal():
    L, T = 40, 7
    q, k, v = rng_arrays(4, T, L, 8, 2, 16)
    chain = [-1] + list(range(T - 1))
    a = oracle.attention([q], [k], [v], [T], [W.TREE], [chain], 0.25)
    c = oracle.attention([q], [k], [v], [T], [W.CAUSAL], [[]], 0.25)
    assert np.allclose(a, c, atol=1e-13, rtol=0)


def pin5_decode_steps_match_prefill():
    L, T = 37, 12
    q, k, v = rng_arrays(5, T, L, 4, 1, 8)
    full = oracle.attention([q], [k], [v], [T], [W.CAUSAL], [[]], 0.4)
    for i in range(T):
        Li = L - T + i + 1
        step = oracle.attention([q[i:i + 1]], [k[:Li]], [v[:Li]], [1], [W.CAUSAL], [[]], 0.4)
        assert np.allclose(step[0], full[i], atol=1e-13, rtol=0)


def pin6_page_permutation_invariance():
    b1 = W.random_small(11, num_seqs=3, max_ctx=50, max_q=20)
    b2 = W.repage(b1, perm_seed=999)
    assert not torch.equal(b1.block_table, b2.block_table)
    outs = []
    for b in (b1, b2):
        qs, ks, vs = [], [], []
        kc, vc = np64(b.k_cache), np64(b.v_cache)
        for i, s in enumerate(b.seqs):
            row = b.block_table[i].tolist()
            ks.append(oracle.gather_paged(kc, row, s.seq_len))
            vs.append(oracle.gather_paged(vc, row, s.seq_len))
            qs.append(np64(b.seq_q(i)))
        outs.append(oracle.attention(qs, ks, vs, b.query_lens, b.mask_kinds,
                                     [s.parents for s in b.seqs]))
    assert np.array_equal(outs[0], outs[1])
    # and the paged gather reproduces the contiguous copy the generator kept
    assert np.array_equal(outs[0], run_oracle(b1))


def pin7_brute_force():
    for seed in range(3):
        b = W.random_small(100 + seed, num_seqs=3, Hq=4, Hkv=2, d=8, max_ctx=20, max_q=8,
                           tree_frac=0.5, max_draft=6)
        got = run_oracle(b, scale=0.37)
        off = 0
        for i, s in enumerate(b.seqs):
            k, v = b.seq_kv(i)
            ref = brute_force(np64(b.seq_q(i)).tolist(), np64(k).tolist(), np64(v).tolist(),
                              s.seq_len, s.query_len, s.mask_kind, s.parents, 0.37)
            assert np.allclose(got[off:off + s.query_len], np.array(ref), atol=1e-12, rtol=0)
            off += s.query_len


def pin8_sdpa():
    for seed in range(3):
        b = W.random_small(200 + seed, num_seqs=4, Hq=8, Hkv=2, d=32, max_ctx=60, max_q=30)
        got = run_oracle(b)
        off = 0
        for i, s in enumerate(b.seqs):
            k, v = b.seq_kv(i)
            q = b.seq_q(i).to(torch.float64)
            G = b.num_q_heads // b.num_kv_heads
            kk = k.to(torch.float64).repeat_interleave(G, dim=1)       # [L, Hq, d]
            vv = v.to(torch.float64).repeat_interleave(G, dim=1)
            L, T = s.seq_len, s.query_len
            prefix = L - T
            mask = torch.zeros(T, L, dtype=torch.bool)
            if s.mask_kind == W.CAUSAL:
                mask = torch.ones(T, L, dtype=torch.bool).tril(diagonal=prefix)
            else:
                mask[:, :prefix] = True
                for r in range(T):
                    a = r
                    while a != -1:
                        mask[r, prefix + a] = True
                        a = s.parents[a]
            ref = torch.nn.functional.scaled_dot_product_attention(
                q.transpose(0, 1), kk.transpose(0, 1), vv.transpose(0, 1), attn_mask=mask)
            assert np.allclose(got[off:off + T], ref.transpose(0, 1).numpy(), atol=1e-12, rtol=0)
            off += T


def pin9_split_merge():
    L, T = 90, 5
    q, k, v = rng_arrays(9, T, L, 4, 2, 16)
    k[::7] *= 8.0                                      # outlier keys, as in the long-context batch
    for mk, par in ((W.CAUSAL, None), (W.TREE, [-1, 0, -1, 2, 1])):
        al = oracle.allowed_mask(L, T, mk, par)
        full = oracle.attend_seq(q, k, v, al, 0.3)
        for cuts in ([0, 90], [0, 30, 60, 90], [0, 1, 50, 86, 90], [0, 85, 86, 87, 88, 89, 90]):
            parts = [oracle.attend_partial(q, k, v, al, slice(a, b), 0.3)
                     for a, b in zip(cuts[:-1], cuts[1:])]
            assert np.allclose(oracle.lse_merge(parts), full, atol=1e-12, rtol=0)


def pin10_e4m3_codes():
    """FP8 E4M3 decoding against values the format's definition fixes in closed form."""
    d = oracle.e4m3_decode
    fixed = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 / 8 * 2.0 ** -6, 0x08: 2.0 ** -6, 0x30: 0.5,
             0x38: 1.0, 0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x44: 3.0, 0x70: 128.0, 0x78: 256.0,
             0x7E: 448.0, 0xB8: -1.0, 0xC0: -2.0, 0xFE: -448.0, 0x81: -(2.0 ** -9)}
    for c, val in fixed.items():
        assert d(np.array([c]))[0] == val, hex(c)
    assert np.signbit(d(np.array([0x80]))[0]) and d(np.array([0x80]))[0] == 0.0
    assert np.isnan(d(np.array([0x7F, 0xFF]))).all()
    pos = d(np.arange(0x00, 0x7F))
    assert np.all(np.diff(pos) > 0)                        # codes 0..126 strictly increase
    assert np.array_equal(d(np.arange(0x80, 0xFF)), -pos)  # the sign bit only negates
    # consecutive normal codes in one binade are 1/8 of the binade apart
    for e in range(1, 16):
        base = 2.0 ** (e - 7)
        vals = d(np.arange(e * 8, e * 8 + (7 if e == 15 else 8)))
        assert np.allclose(np.diff(vals), base / 8, rtol=0, atol=0)
    # dequantisation multiplies by the KV head's own scale
    codes = np.array([[[0x38, 0x40]], [[0xC0, 0x08]]], dtype=np.uint8).repeat(2, axis=1)
    deq = oracle.dequantize_kv(codes, np.array([0.5, 3.0]))
    assert deq[0, 0, 0] == 0.5 and deq[0, 1, 0] == 3.0 and deq[1, 1, 0] == -6.0


def pin11_e4m3_encode():
    """Rounding into E4M3: every finite code round-trips; halfway values go to the even
    mantissa; values past 448 clamp; the subnormal binade has quantum 2^-9; and the
    encoding agrees with torch's float8_e4m3fn conversion (a library special case) on a
    dense grid of values below 448."""
    enc, dec = oracle.e4m3_encode, oracle.e4m3_decode
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.int64)
    assert np.array_equal(enc(dec(finite)), finite.astype(np.uint8))
    # halfway between 1.0 (0x38, even) and 1.125 (0x39): to 0x38; between 1.125 and 1.25: to 0x3A
    assert enc(np.array([1.0625]))[0] == 0x38 and enc(np.array([1.1875]))[0] == 0x3A
    assert enc(np.array([1.0624]))[0] == 0x38 and enc(np.array([1.0626]))[0] == 0x39
    assert enc(np.array([448.0, 449.0, 1e6, -500.0])).tolist() == [0x7E, 0x7E, 0x7E, 0xFE]
    assert enc(np.array([2.0 ** -10, 1.5 * 2.0 ** -9, 2.0 ** -11]))[:].tolist() == [0x00, 0x02, 0x00]
    assert enc(np.array([np.nan]))[0] == 0x7F
    assert enc(np.array([-0.0]))[0] == 0x80
    import torch
    grid = np.concatenate([np.linspace(-447.9, 447.9, 20001), np.linspace(-0.05, 0.05, 20001)]).astype(np.float32)
    ref = torch.from_numpy(grid).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(enc(grid), ref)


PINS = [pin1_rows_sum_to_one, pin2_single_key, pin3_identical_keys_give_mean,
        pin4_chain_tree_is_causal, pin5_decode_steps_match_prefill,
        pin6_page_permutation_invariance, pin7_brute_force, pin8_sdpa, pin9_split_merge,
        pin10_e4m3_codes, pin11_e4m3_encode]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_oracle_rejects_bad_inputs():
    with pytest.raises(ValueError):
        oracle.allowed_mask(5, 0, W.CAUSAL)
    with pytest.raises(ValueError):
        oracle.allowed_mask(5, 6, W.CAUSAL)
    with pytest.raises(ValueError):
        oracle.allowed_mask(9, 3, W.TREE, [-1, 2, 0])     # parent after child
    with pytest.raises(ValueError):
        oracle.attention_weights(np.zeros((1, 3, 4)), np.zeros((2, 2, 4)),
                                 np.ones((1, 2), bool), 1.0)


def test_attend_rows_matches_full():
    q, k, v = rng_arrays(12, 9, 41, 4, 2, 8)
    par = [-1, 0, 0, 2, -1, 4, 5, 1, 3]
    full = oracle.attend_seq(q, k, v, oracle.allowed_mask(41, 9, W.TREE, par), 0.2)
    rows = [0, 3, 8]
    got = oracle.attend_rows(q[rows], k, v, 41, 9, rows, W.TREE, par, 0.2)
    assert np.array_equal(got, full[rows])


# ----------------------------------------------------------------------------------
# planted mistakes: each must make at least one pin fail
# ----------------------------------------------------------------------------------

def _mut_gqa_modulo(orig):
    def attention_weights(q, k, allowed, scale):
        q = np.asarray(q, np.float64); k = np.asarray(k, np.float64)
        T, Hq, d = q.shape; Hkv = k.shape[1]
        w = np.zeros((T, Hq, k.shape[0]))
        for h in range(Hq):
            s = np.where(allowed, scale * (q[:, h] @ k[:, h % Hkv].T), -np.inf)
            e = np.where(allowed, np.exp(s - s.max(1, keepdims=True)), 0)
            w[:, h] = e / e.sum(1, keepdims=True)
        return w
    return {"attention_weights": attention_weights}


def _mut_causal_excludes_diagonal(orig):
    def allowed_mask(L, T, mk, parents=None):
        m = orig.allowed_mask(L, T, mk, parents)
        if mk == W.CAUSAL:
            for i in range(T):
                if L - T + i > 0:
                    m[i, L - T + i] = False
        return m
    return {"allowed_mask": allowed_mask}


def _mut_tree_self_only(orig):
    def allowed_mask(L, T, mk, parents=None):
        if mk == W.TREE:
            m = np.zeros((T, L), bool)
            m[:, :L - T] = True
            for i in range(T):
                m[i, L - T + i] = True
            return m
        return orig.allowed_mask(L, T, mk, parents)
    return {"allowed_mask": allowed_mask}


def _mut_tree_parent_not_ancestors(orig):
    def allowed_mask(L, T, mk, parents=None):
        if mk == W.TREE:
            m = np.zeros((T, L), bool)
            m[:, :L - T] = True
            for i in range(T):
                m[i, L - T + i] = True
                if parents[i] >= 0:
                    m[i, L - T + parents[i]] = True
            return m
        return orig.allowed_mask(L, T, mk, parents)
    return {"allowed_mask": allowed_mask}


def _mut_no_max_subtraction_scale(orig):
    def attention_weights(q, k, allowed, scale):
        return orig.attention_weights(q, k, allowed, 1.0)      # scale dropped
    return {"attention_weights": attention_weights}


def _mut_top_left_causal(orig):
    def allowed_mask(L, T, mk, parents=None):
        if mk == W.CAUSAL:
            m = np.zeros((T, L), bool)
            for i in range(T):
                m[i, :i + 1] = True
            return m
        return orig.allowed_mask(L, T, mk, parents)
    return {"allowed_mask": allowed_mask}


def _mut_transposed_value(orig):
    def attend_seq(q, k, v, allowed, scale):
        w = orig.attention_weights(q, k, allowed, scale)
        v = np.asarray(v, np.float64)
        G = q.shape[1] // v.shape[1]
        out = np.empty((w.shape[0], w.shape[1], v.shape[2]))
        for h in range(w.shape[1]):
            out[:, h] = w[:, h] @ v[:, (h // G + 1) % v.shape[1]]  # wrong V head
        return out
    return {"attend_seq": attend_seq}


def _mut_merge_unweighted(orig):
    def lse_merge(parts):
        ms = np.stack([p[1] for p in parts]); mstar = ms.max(0)
        num = sum(np.exp(np.where(np.isfinite(m), m, -np.inf) - mstar)[..., None] * o for o, m, l in parts)
        den = sum(np.exp(np.where(np.isfinite(m), m, -np.inf) - mstar) for o, m, l in parts)
        return num / den[..., None]                              # l_i weights dropped
    return {"lse_merge": lse_merge}


def _mut_e4m3_bias_8(orig):
    def e4m3_decode(codes):
        return orig.e4m3_decode(codes) / 2.0                  # exponent bias 8 instead of 7
    return {"e4m3_decode": e4m3_decode}


def _mut_e4m3_no_subnormals(orig):
    def e4m3_decode(codes):
        c = np.asarray(codes).astype(np.int64) & 0xFF
        v = orig.e4m3_decode(codes)
        return np.where(((c >> 3) & 0xF) == 0, np.where(c & 0x80, -0.0, 0.0), v)   # flushed to zero
    return {"e4m3_decode": e4m3_decode}


def _mut_e4m3_ieee_style_inf(orig):
    def e4m3_decode(codes):
        c = np.asarray(codes).astype(np.int64) & 0xFF
        v = orig.e4m3_decode(codes)
        return np.where(((c >> 3) & 0xF) == 15, np.where(c & 7, np.nan, np.inf), v)   # top binade reserved
    return {"e4m3_decode": e4m3_decode}


def _mut_dequant_wrong_head(orig):
    def dequantize_kv(codes, scale):
        return orig.e4m3_decode(codes) * np.asarray(scale, np.float64)[::-1][None, :, None]
    return {"dequantize_kv": dequantize_kv}


def _mut_e4m3_round_half_up(orig):
    def e4m3_encode(x):
        x = np.asarray(x, np.float64)
        return orig.e4m3_encode(np.nextafter(x, np.sign(x) * np.inf))     # ties pushed away from zero
    return {"e4m3_encode": e4m3_encode}


def _mut_e4m3_no_saturation(orig):
    def e4m3_encode(x):
        c = orig.e4m3_encode(x)
        big = np.abs(np.asarray(x, np.float64)) > 464.0
        return np.where(big, (c & 0x80) | 0x7F, c).astype(np.uint8)      # overflow to NaN
    return {"e4m3_encode": e4m3_encode}


MUTANTS = [_mut_gqa_modulo, _mut_causal_excludes_diagonal, _mut_tree_self_only,
           _mut_tree_parent_not_ancestors, _mut_no_max_subtraction_scale,
           _mut_top_left_causal, _mut_transposed_value, _mut_merge_unweighted,
           _mut_e4m3_bias_8, _mut_e4m3_no_subnormals, _mut_e4m3_ieee_style_inf,
           _mut_dequant_wrong_head, _mut_e4m3_round_half_up, _mut_e4m3_no_saturation]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda f: f.__name__)
def test_planted_mistakes_are_caught(mutant, monkeypatch):
    import copy
    import types
    orig = types.SimpleNamespace(**{n: getattr(oracle, n) for n in dir(oracle) if not n.startswith("__")})
    for name, fn in mutant(orig).items():
        monkeypatch.setattr(oracle, name, fn)
    failed = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, ValueError, ZeroDivisionError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught {mutant.__name__}"
