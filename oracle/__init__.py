"""Float64 CPU oracle for paged-KV attention over a mixed prefill / decode / verify batch.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package. The product path
(``paged_kv_attention_verify_b200``) never calls it, and shares no code with it: this
module is plain NumPy in float64 with no blocking, fusion or reordering beyond the
definition it writes out.

What it computes (exact softmax attention, written out as its definition):

  For each sequence s with total KV length L and T new query tokens, query row i
  sits at absolute position p_i = L - T + i. For each query head h, with KV head
  g = h // (Hq / Hkv) (grouped-query attention: consecutive query heads share one
  KV head),

      score_ij = scale * <q_ih, k_jg>          for every allowed key j
      w_ij     = exp(score_ij - max_j score) / sum_j exp(score_ij - max_j score)
      out_ih   = sum_j w_ij v_jg

  Allowed keys (the row-wise mask):
    CAUSAL (a prefill chunk on a cached prefix, or a decode step, T = 1):
        j <= p_i                              (bottom-right aligned causal mask)
    TREE (speculative-decoding verify of T draft tokens in a tree):
        j <  L - T                            (the whole committed prefix), or
        j == L - T + a  with a = i or a an ancestor of i under ``parents``.

Passages followed:
  * XY-Serve (arXiv 2412.18106), verdict page, ``pith_extraction.forward_implications[2]``:
    a single attention kernel, choosing the visible keys row by row, covers prefill,
    decode and verify rows; ``core_discovery``: chunked prefill, prefix caching and a
    paged block cache are all cases of one tiled attention; ``referee_report.significance``:
    verify runs over a tree of draft tokens; supporting citation [1]: FlashAttention's
    QK / softmax / SV pattern.
  * Understanding Inference Scaling for LLMs (arXiv 2605.19775), reference list:
    PagedAttention and grouped-query attention (the GQA head grouping).

Readings where the pages are silent (each listed in the design notes):
  * scale defaults to 1/sqrt(d);
  * causal masks are bottom-right aligned (the new tokens' K/V are already cached);
  * a tree is a parent array with parents[i] in {-1} U [0, i); -1 hangs the node off
    the committed prefix, so forests are allowed; every node sees itself;
  * no row is ever fully masked (query_len >= 1 and each row sees itself).

Parity status: every function here is pinned by CPU tests (invariants, closed forms,
brute force and a library special case); none is pinned to a worked example printed
on the pages, because the pages print none.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

CAUSAL = 0
TREE = 1


def ancestors_or_self(parents: Sequence[int]) -> List[List[int]]:
    """For each draft node i, the sorted list {i} U ancestors(i) under the parent array.

    Tree encoding (a reading of the draft tree of speculative decoding, XY-Serve verdict
    page, ``referee_report.significance``): parents[i] is -1 or an earlier node index.
    """
    out = []
    for i in range(len(parents)):
        chain = [i]
        a = parents[i]
        while a != -1:
            if not (0 <= a < chain[-1]):
                raise ValueError(f"parents[{chain[-1]}] = {a} is not -1 or an earlier node")
            chain.append(a)
            a = parents[a]
        out.append(sorted(chain))
    return out


def allowed_mask(seq_len: int, query_len: int, mask_kind: int,
                 parents: Optional[Sequence[int]] = None) -> np.ndarray:
    """Boolean [T, L]: which keys each new query row may attend to.

    XY-Serve verdict page, ``forward_implications[2]`` (the visible keys are chosen per
    row, for prefill, decode and verify rows alike).
    """
    L, T = seq_len, query_len
    if not (1 <= T <= L):
        raise ValueError("need 1 <= query_len <= seq_len")
    prefix = L - T
    m = np.zeros((T, L), dtype=bool)
    if mask_kind == CAUSAL:
        for i in range(T):
            m[i, :prefix + i + 1] = True
    elif mask_kind == TREE:
        if parents is None or len(parents) != T:
            raise ValueError("TREE rows need one parent per draft token")
        m[:, :prefix] = True
        for i, anc in enumerate(ancestors_or_self(parents)):
            for a in anc:
                m[i, prefix + a] = True
    else:
        raise ValueError(f"unknown mask kind {mask_kind}")
    return m


def _group_size(num_q_heads: int, num_kv_heads: int) -> int:
    if num_q_heads % num_kv_heads != 0:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    return num_q_heads // num_kv_heads


def attention_weights(q: np.ndarray, k: np.ndarray, allowed: np.ndarray,
                      scale: float) -> np.ndarray:
    """Softmax weights [T, Hq, L] (float64) for one sequence.

    q: [T, Hq, d], k: [L, Hkv, d]; allowed: [T, L]. Masked weights are exactly 0.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    T, Hq, d = q.shape
    L, Hkv, _ = k.shape
    G = _group_size(Hq, Hkv)
    w = np.zeros((T, Hq, L), dtype=np.float64)
    for h in range(Hq):
        g = h // G
        s = scale * (q[:, h, :] @ k[:, g, :].T)            # [T, L]
        s = np.where(allowed, s, -np.inf)
        mx = s.max(axis=1, keepdims=True)
        e = np.where(allowed, np.exp(s - mx), 0.0)
        w[:, h, :] = e / e.sum(axis=1, keepdims=True)
    return w


def attend_seq(q: np.ndarray, k: np.ndarray, v: np.ndarray, allowed: np.ndarray,
               scale: float) -> np.ndarray:
    """out[T, Hq, d] = softmax-weighted sum of V over the allowed keys, per query head."""
    v = np.asarray(v, dtype=np.float64)
    w = attention_weights(q, k, allowed, scale)
    T, Hq, L = w.shape
    Hkv = v.shape[1]
    G = _group_size(Hq, Hkv)
    out = np.empty((T, Hq, v.shape[2]), dtype=np.float64)
    for h in range(Hq):
        out[:, h, :] = w[:, h, :] @ v[:, h // G, :]
    return out


def default_scale(head_dim: int) -> float:
    """1/sqrt(d): the pages never state the softmax scale; this is the standard one."""
    return 1.0 / math.sqrt(head_dim)


def attention(q_seqs: Sequence[np.ndarray], k_seqs: Sequence[np.ndarray],
              v_seqs: Sequence[np.ndarray], query_lens: Sequence[int],
              mask_kinds: Sequence[int], parents: Sequence[Sequence[int]],
              scale: Optional[float] = None) -> np.ndarray:
    """Whole-batch oracle: concatenated [sum T, Hq, d] float64 output.

    Each sequence's K/V arrive contiguous and un-paged ([L, Hkv, d]), so the oracle
    never touches a block table.
    """
    outs = []
    for q, k, v, T, mk, par in zip(q_seqs, k_seqs, v_seqs, query_lens, mask_kinds, parents):
        L = k.shape[0]
        sc = default_scale(q.shape[2]) if scale is None else scale
        outs.append(attend_seq(q, k, v, allowed_mask(L, T, mk, par), sc))
    return np.concatenate(outs, axis=0)


def attend_rows(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, seq_len: int,
                query_len: int, row_ids: Sequence[int], mask_kind: int,
                parents: Optional[Sequence[int]], scale: float) -> np.ndarray:
    """Outputs for selected query rows only (sampled parity at full sizes).

    q_rows: [len(row_ids), Hq, d] — the queries of rows ``row_ids`` of one sequence.
    """
    allowed = allowed_mask(seq_len, query_len, mask_kind, parents)[list(row_ids)]
    return attend_seq(q_rows, k, v, allowed, scale)


# -------------------------------------------------------------------------------------
# Split-KV (flash-decoding) partials and their log-sum-exp merge.
# The benchmark spec of the path asks for a split-KV combine for long contexts;
# the merge below is the algebraic identity that makes the split exact.
# -------------------------------------------------------------------------------------

def attend_partial(q: np.ndarray, k: np.ndarray, v: np.ndarray, allowed: np.ndarray,
                   cols: slice, scale: float) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Attention restricted to the key range ``cols``: (o, m, l) with
    m = max allowed score (-inf if none), l = sum exp(score - m), o = normalized output
    (zeros where l = 0). Shapes: o [T, Hq, d], m and l [T, Hq]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)[cols]
    v = np.asarray(v, dtype=np.float64)[cols]
    al = allowed[:, cols]
    T, Hq, d = q.shape
    G = _group_size(Hq, k.shape[1])
    o = np.zeros((T, Hq, d))
    m = np.full((T, Hq), -np.inf)
    l = np.zeros((T, Hq))
    for h in range(Hq):
        s = scale * (q[:, h, :] @ k[:, h // G, :].T)
        s = np.where(al, s, -np.inf)
        mh = s.max(axis=1) if s.shape[1] else np.full(T, -np.inf)
        ref = np.where(np.isfinite(mh), mh, 0.0)
        e = np.where(al, np.exp(s - ref[:, None]), 0.0)
        lh = e.sum(axis=1)
        with np.errstate(invalid="ignore", divide="ignore"):
            oh = np.where(lh[:, None] > 0, (e @ v[:, h // G, :]) / lh[:, None], 0.0)
        o[:, h, :], m[:, h], l[:, h] = oh, mh, lh
    return o, m, l


def lse_merge(parts: Sequence[Tuple[np.ndarray, np.ndarray, np.ndarray]]) -> np.ndarray:
    """Merge split partials: m* = max_i m_i; out = sum_i e^(m_i-m*) l_i o_i / sum_i e^(m_i-m*) l_i."""
    ms = np.stack([p[1] for p in parts])                    # [S, T, Hq]
    mstar = ms.max(axis=0)
    num = 0.0
    den = 0.0
    for o, m, l in parts:
        wgt = np.where(np.isfinite(m), np.exp(np.where(np.isfinite(m), m, 0.0) - mstar), 0.0) * l
        num = num + wgt[..., None] * o
        den = den + wgt
    return num / den[..., None]


# -------------------------------------------------------------------------------------
# Paged layout helper, used only by the page-permutation invariance pin.
# -------------------------------------------------------------------------------------

def gather_paged(cache: np.ndarray, block_table_row: Sequence[int], seq_len: int) -> np.ndarray:
    """Contiguous [L, Hkv, d] from a paged pool [num_pages, Hkv, P, d] through one
    block-table row (PagedAttention-style block cache)."""
    P = cache.shape[2]
    rows = []
    for pos in range(seq_len):
        page = block_table_row[pos // P]
        rows.append(cache[page, :, pos % P, :])
    return np.stack(rows)


# -------------------------------------------------------------------------------------
# FP8 (E4M3) KV cache: decoding of the stored codes. The attention itself is unchanged:
# the oracle decodes every code exactly (float64) and multiplies by the per-KV-head scale,
# then runs the definition above on those values.
# -------------------------------------------------------------------------------------

def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """float64 value of each FP8 E4M3 code (one byte each).

    The format, written out: bit 7 is the sign; bits 6..3 are a biased exponent e (bias 7);
    bits 2..0 a mantissa m. e = 0 encodes subnormals m/8 * 2^-6; e in 1..15 encodes
    (1 + m/8) * 2^(e-7), except e = 15 with m = 7, which is NaN. There are no infinities,
    so the largest finite magnitude is (1 + 6/8) * 2^8 = 448.

    Reading: the pages name FP8 and quantised KV-cache formats without fixing one (Arctic
    Inference review page, section 3 comments); E4M3 of this form is taken as the FP8 KV
    format, the plainest common choice.
    """
    c = np.asarray(codes).astype(np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def dequantize_kv(codes: np.ndarray, scale_per_head: np.ndarray) -> np.ndarray:
    """Values [L, Hkv, d] of an FP8 K or V tensor [L, Hkv, d] with one scale per KV head:
    value = e4m3_decode(code) * scale[head]."""
    s = np.asarray(scale_per_head, dtype=np.float64)
    return e4m3_decode(codes) * s[None, :, None]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """FP8 E4M3 code (uint8) of each value, rounded to the nearest representable value with
    ties to the even mantissa, magnitudes beyond the largest finite value (448) clamped to
    it, NaN to the NaN code 0x7F; the sign of a zero is kept.

    Reading: quantising a value into an E4M3 cache rounds to nearest-even and saturates
    (the format has no infinities); the value quantised is float32(x) / float32(scale),
    the division correctly rounded in float32 (the caller does that division).
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros(x.shape, dtype=np.uint8)
    for idx, v in np.ndenumerate(x):
        if np.isnan(v):
            out[idx] = 0x7F
            continue
        sign = 0x80 if np.signbit(v) else 0x00
        a = abs(v)
        if a >= 448.0:
            out[idx] = sign | 0x7E
            continue
        if a < 2.0 ** -6:                              # subnormal binade: quantum 2^-9
            m = int(np.rint(a / 2.0 ** -9))            # ties to even (exact in float64)
            out[idx] = sign | m                        # m = 8 is the smallest normal, 0x08
            continue
        e = int(np.floor(np.log2(a)))
        if 2.0 ** e > a:                               # guard against log2 rounding
            e -= 1
        elif 2.0 ** (e + 1) <= a:
            e += 1
        m = int(np.rint(a / 2.0 ** (e - 3)))           # 8 .. 16
        if m == 16:
            e, m = e + 1, 8
        code = ((e + 7) << 3) | (m - 8)
        out[idx] = sign | min(code, 0x7E)              # 480 would round past 448: clamp
    return out
