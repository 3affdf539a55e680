"""Seeded synthetic batches for paged-KV attention (inputs only, no attention arithmetic).

This module is the single source of inputs for both sides of every parity check: the
float64 CPU oracle (``oracle/``) and the CUDA path (``paged_kv_attention_verify_b200``).
It holds no part of the attention computation itself: it draws lengths, draft-tree
parent arrays, Q/K/V values and a page permutation, then lays K/V out twice — once
contiguous per sequence (what the oracle reads) and once scattered into a pool of
fixed-size pages addressed through a block table (what the kernels read).

Workload shapes follow the five batches the pages' problem is benchmarked on
(decode on a Llama-3-8B-shaped cache, chunked prefill on a Llama-3.3-70B-shaped
cache, a unified prefill/decode/verify batch on a Qwen2-7B-shaped cache, and a
long-context decode with outlier keys). XY-Serve (arXiv 2412.18106, verdict page,
``core_discovery``) names the mixed prefill / decode / verify batch over a
PagedAttention-style block cache; the sizes are those of the benchmark configs.

Randomness recipe (stated once, used everywhere):
  * sequence lengths and draft trees come from a CPU ``torch.Generator`` seeded with
    the config seed (the config's index, 0..4);
  * the page permutation comes from a CPU generator seeded with ``seed + 1000``, so
    structure is identical whatever device the values are drawn on;
  * bulk values (Q, K, V, outlier flags, page-tail filler) come from a generator on
    the target device seeded with ``seed + 1001``; values are N(0,1) rounded to bf16
    (a CPU draw and a CUDA draw of the same seed differ; each test feeds both sides
    from one draw);
  * page slots past a sequence's length are filled with finite values of large
    magnitude (N(0,1) x 50) so that any failure to mask them shows up in parity.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import torch

CAUSAL = 0
TREE = 1


@dataclasses.dataclass
class SeqSpec:
    seq_len: int          # total KV length including the new tokens
    query_len: int        # number of new query tokens (their K/V are already cached)
    mask_kind: int        # CAUSAL or TREE
    parents: List[int]    # TREE only: parents[i] in {-1} U [0, i)


@dataclasses.dataclass
class Batch:
    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    seqs: List[SeqSpec]
    q: torch.Tensor                  # [sum T, Hq, d] bf16
    k: Optional[torch.Tensor]        # [sum L, Hkv, d] bf16, contiguous per sequence
    v: Optional[torch.Tensor]
    k_cache: torch.Tensor            # [num_pages, Hkv, page_size, d] bf16
    v_cache: torch.Tensor
    block_table: torch.Tensor        # [B, max_pages] int32, -1 = unused slot
    page_perm: torch.Tensor          # [num_pages] int64 (CPU): logical page -> physical page
    seed: int = 0
    outlier_frac: float = 0.0
    # shared-prefix groups: prefix_group[s] in {-1} U [0, G); the first prefix_len[g] keys of
    # every member of group g are the same values on the same physical pages
    prefix_group: Optional[List[int]] = None
    prefix_len: Optional[List[int]] = None

    # -- convenience views (layout only) ---------------------------------------------
    @property
    def seq_lens(self) -> List[int]:
        return [s.seq_len for s in self.seqs]

    @property
    def query_lens(self) -> List[int]:
        return [s.query_len for s in self.seqs]

    @property
    def mask_kinds(self) -> List[int]:
        return [s.mask_kind for s in self.seqs]

    @property
    def parents_flat(self) -> List[int]:
        out: List[int] = []
        for s in self.seqs:
            if s.mask_kind == TREE:
                out.extend(s.parents)
        return out

    def q_offsets(self) -> List[int]:
        off, acc = [], 0
        for s in self.seqs:
            off.append(acc)
            acc += s.query_len
        return off

    def kv_offsets(self) -> List[int]:
        off, acc = [], 0
        for s in self.seqs:
            off.append(acc)
            acc += s.seq_len
        return off

    def seq_q(self, i: int) -> torch.Tensor:
        o = self.q_offsets()[i]
        return self.q[o:o + self.seqs[i].query_len]

    def seq_kv(self, i: int):
        if self.k is None:
            raise ValueError("contiguous K/V were dropped for this batch")
        o = self.kv_offsets()[i]
        L = self.seqs[i].seq_len
        return self.k[o:o + L], self.v[o:o + L]

    @property
    def total_q(self) -> int:
        return sum(s.query_len for s in self.seqs)

    @property
    def total_kv(self) -> int:
        return sum(s.seq_len for s in self.seqs)


# ---------------------------------------------------------------------------------
# Named configurations (sizes of the five benchmark batches)
# ---------------------------------------------------------------------------------

CONFIG_NAMES = [
    "tiny_decode",          # 4 seqs, ctx {17,64,100,255}, 8q/2kv, d64
    "llama3_8b_decode",     # 128 seqs, ctx U[512,8192], 32q/8kv, d128
    "llama33_70b_prefill",  # 8 seqs x 2048-token chunk on ctx U[0,16384], 64q/8kv, d128
    "qwen2_7b_unified",     # 4x512 prefill + 192 decode + 32 verify(5-node tree), 28q/4kv
    "long_ctx_split",       # 16 seqs, ctx U[32768,131072], 128q/8kv, 1% outlier keys x8
]


def _randint(gen: torch.Generator, lo: int, hi: int, n: int) -> List[int]:
    """n integers uniform on [lo, hi] inclusive."""
    return torch.randint(lo, hi + 1, (n,), generator=gen).tolist()


def random_tree(gen: torch.Generator, n: int) -> List[int]:
    """Parent array of a random draft tree: parents[0] = -1, parents[i] ~ U{-1..i-1}."""
    par = [-1]
    for i in range(1, n):
        par.append(int(torch.randint(-1, i, (1,), generator=gen).item()))
    return par


def config_seqs(name: str, gen: torch.Generator) -> tuple:
    """(seqs, Hq, Hkv, d, outlier_frac) for a named configuration."""
    if name == "tiny_decode":
        seqs = [SeqSpec(L, 1, CAUSAL, []) for L in (17, 64, 100, 255)]
        return seqs, 8, 2, 64, 0.0
    if name == "llama3_8b_decode":
        seqs = [SeqSpec(L, 1, CAUSAL, []) for L in _randint(gen, 512, 8192, 128)]
        return seqs, 32, 8, 128, 0.0
    if name == "llama33_70b_prefill":
        seqs = [SeqSpec(c + 2048, 2048, CAUSAL, []) for c in _randint(gen, 0, 16384, 8)]
        return seqs, 64, 8, 128, 0.0
    if name == "qwen2_7b_unified":
        seqs = [SeqSpec(512, 512, CAUSAL, []) for _ in range(4)]
        seqs += [SeqSpec(L, 1, CAUSAL, []) for L in _randint(gen, 256, 4096, 192)]
        for ctx in _randint(gen, 256, 4096, 32):
            seqs.append(SeqSpec(ctx + 5, 5, TREE, random_tree(gen, 5)))
        return seqs, 28, 4, 128, 0.0
    if name == "long_ctx_split":
        seqs = [SeqSpec(L, 1, CAUSAL, []) for L in _randint(gen, 32768, 131072, 16)]
        return seqs, 128, 8, 128, 0.01
    raise KeyError(name)


SHARED_CONFIG_NAMES = [
    "llama3_8b_shared_prefix",   # 4 groups x 32 seqs on a shared 4096-key prefix, 32q/8kv, d128
]


def shared_config(name: str, gen: torch.Generator) -> tuple:
    """(seqs, prefix_group, prefix_len, Hq, Hkv, d) for a named shared-prefix batch."""
    if name == "llama3_8b_shared_prefix":
        seqs, group = [], []
        for g in range(4):
            for i in range(32):
                own = int(torch.randint(0, 1025, (1,), generator=gen).item())
                if i % 4 == 3:          # every fourth member verifies a 5-node draft tree
                    seqs.append(SeqSpec(4096 + own + 5, 5, TREE, random_tree(gen, 5)))
                else:
                    seqs.append(SeqSpec(4096 + own + 1, 1, CAUSAL, []))
                group.append(g)
        return seqs, group, [4096] * 4, 32, 8, 128
    raise KeyError(name)


def build_shared_batch(name: str, seqs: Sequence[SeqSpec], prefix_group: Sequence[int],
                       prefix_len: Sequence[int], num_q_heads: int, num_kv_heads: int,
                       head_dim: int, seed: int, device="cpu", page_size: int = 16,
                       keep_contiguous: bool = True, bt_extra: int = 0) -> Batch:
    """Like ``build_batch``, but the members of each group share the values and the physical
    pages of their first ``prefix_len[g]`` keys (a common prompt held once in the cache).

    Seeding as in ``build_batch``; the shared keys of group g are drawn once, after the
    per-sequence values."""
    device = torch.device(device)
    sgen = torch.Generator().manual_seed(seed)
    vgen = torch.Generator(device=device).manual_seed(seed + 1)
    Hq, Hkv, d, P = num_q_heads, num_kv_heads, head_dim, page_size
    B = len(seqs)
    for s, g in zip(seqs, prefix_group):
        if g >= 0 and (prefix_len[g] % P or prefix_len[g] > s.seq_len - s.query_len):
            raise ValueError("a shared prefix must be page-aligned and within the committed prefix")

    def randn_bf16(*shape):
        return torch.randn(*shape, generator=vgen, device=device,
                           dtype=torch.float32).to(torch.bfloat16)

    total_q = sum(s.query_len for s in seqs)
    total_kv = sum(s.seq_len for s in seqs)
    q = randn_bf16(total_q, Hq, d)
    k = randn_bf16(total_kv, Hkv, d)
    v = randn_bf16(total_kv, Hkv, d)
    shared_k = [randn_bf16(n, Hkv, d) for n in prefix_len]
    shared_v = [randn_bf16(n, Hkv, d) for n in prefix_len]

    # logical pages: each group's shared pages once, then every sequence's own pages
    shared_pages = [n // P for n in prefix_len]
    own_pages = [(s.seq_len + P - 1) // P - (shared_pages[g] if g >= 0 else 0)
                 for s, g in zip(seqs, prefix_group)]
    num_pages = sum(shared_pages) + sum(own_pages)
    perm = torch.randperm(num_pages, generator=sgen)
    group_first = []
    acc = 0
    for n in shared_pages:
        group_first.append(acc)
        acc += n
    max_pages = max((s.seq_len + P - 1) // P for s in seqs) + bt_extra
    block_table = torch.full((B, max_pages), -1, dtype=torch.int32)
    tok_page, tok_slot = [], []
    kv_off = 0
    for i, (s, g) in enumerate(zip(seqs, prefix_group)):
        ns = shared_pages[g] if g >= 0 else 0
        logical = list(range(group_first[g], group_first[g] + ns)) if g >= 0 else []
        logical += list(range(acc, acc + own_pages[i]))
        acc += own_pages[i]
        block_table[i, :len(logical)] = perm[logical].to(torch.int32)
        pos = torch.arange(s.seq_len)
        tok_page.append(torch.tensor(logical, dtype=torch.long)[pos // P])
        tok_slot.append(pos % P)
        if g >= 0:
            n = prefix_len[g]
            k[kv_off:kv_off + n] = shared_k[g]
            v[kv_off:kv_off + n] = shared_v[g]
        kv_off += s.seq_len
    tok_phys = perm[torch.cat(tok_page)].to(device)
    tok_slot = torch.cat(tok_slot).to(device)
    k_cache = (randn_bf16(num_pages, Hkv, P, d).float() * 50.0).to(torch.bfloat16)
    v_cache = (randn_bf16(num_pages, Hkv, P, d).float() * 50.0).to(torch.bfloat16)
    k_cache[tok_phys, :, tok_slot] = k
    v_cache[tok_phys, :, tok_slot] = v
    del tok_phys, tok_slot
    return Batch(name=name, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=d, page_size=P,
                 seqs=list(seqs), q=q, k=k if keep_contiguous else None,
                 v=v if keep_contiguous else None, k_cache=k_cache, v_cache=v_cache,
                 block_table=block_table.to(device), page_perm=perm, seed=seed,
                 prefix_group=list(prefix_group), prefix_len=list(prefix_len))


def random_shared_small(seed: int, Hq: int = 16, Hkv: int = 4, device="cpu", d: int = 128) -> Batch:
    """A small shared-prefix batch (head_dim d): group 0 has six decode / verify members on
    48 shared keys; one sequence belongs to no group; group 1 has three members on 160
    shared keys, one of them a 100-token causal chunk (which runs as a prefill task)."""
    gen = torch.Generator().manual_seed(seed)
    seqs, group = [], []
    for i in range(6):
        own = int(torch.randint(0, 40, (1,), generator=gen).item())
        T = 1 if i % 3 else 4
        seqs.append(SeqSpec(48 + own + T, T, TREE if T == 4 else CAUSAL,
                            random_tree(gen, 4) if T == 4 else []))
        group.append(0)
    seqs.append(SeqSpec(70, 2, CAUSAL, []))
    group.append(-1)
    for T in (3, 100, 1):
        seqs.append(SeqSpec(160 + 20 + T, T, CAUSAL, []))
        group.append(1)
    return build_shared_batch(f"shared_small_{seed}", seqs, group, [48, 160], Hq, Hkv, d, seed=seed,
                              device=device)


def make_shared_config(name: str, device="cpu", seed: Optional[int] = None,
                       keep_contiguous: bool = True) -> Batch:
    """A named shared-prefix batch (seeded by 100 + its index unless ``seed`` is given)."""
    if seed is None:
        seed = 100 + SHARED_CONFIG_NAMES.index(name)
    sgen = torch.Generator().manual_seed(seed)
    seqs, group, plen, Hq, Hkv, d = shared_config(name, sgen)
    return build_shared_batch(name, seqs, group, plen, Hq, Hkv, d, seed=seed + 1000, device=device,
                              keep_contiguous=keep_contiguous)


def build_batch(name: str, seqs: Sequence[SeqSpec], num_q_heads: int, num_kv_heads: int,
                head_dim: int, seed: int, device="cpu", page_size: int = 16,
                outlier_frac: float = 0.0, outlier_scale: float = 8.0,
                keep_contiguous: bool = True, bt_extra: int = 0,
                perm_seed: Optional[int] = None) -> Batch:
    """Draw Q/K/V for ``seqs`` and lay K/V out in a shuffled paged pool.

    ``seed`` seeds the page permutation (CPU) and ``seed + 1`` the values (device);
    ``perm_seed`` overrides the permutation seed alone, keeping the values.
    ``bt_extra`` adds unused (-1) columns to the block table to exercise a stride
    larger than the longest sequence needs.
    """
    device = torch.device(device)
    sgen = torch.Generator().manual_seed(seed if perm_seed is None else perm_seed)
    vgen = torch.Generator(device=device).manual_seed(seed + 1)     # bulk values
    Hq, Hkv, d, P = num_q_heads, num_kv_heads, head_dim, page_size
    B = len(seqs)
    total_q = sum(s.query_len for s in seqs)
    total_kv = sum(s.seq_len for s in seqs)

    def randn_bf16(*shape):
        return torch.randn(*shape, generator=vgen, device=device,
                           dtype=torch.float32).to(torch.bfloat16)

    q = randn_bf16(total_q, Hq, d)
    k = randn_bf16(total_kv, Hkv, d)
    v = randn_bf16(total_kv, Hkv, d)
    if outlier_frac > 0:
        flags = torch.rand(total_kv, Hkv, 1, generator=vgen, device=device) < outlier_frac
        k = torch.where(flags, (k.float() * outlier_scale).to(torch.bfloat16), k)

    pages_per_seq = [(s.seq_len + P - 1) // P for s in seqs]
    num_pages = sum(pages_per_seq)
    max_pages = max(pages_per_seq) + bt_extra
    perm = torch.randperm(num_pages, generator=sgen)                # logical -> physical

    block_table = torch.full((B, max_pages), -1, dtype=torch.int32)
    page_off = 0
    tok_page = []      # per token: logical global page index
    tok_slot = []
    for i, s in enumerate(seqs):
        n = pages_per_seq[i]
        block_table[i, :n] = perm[page_off:page_off + n].to(torch.int32)
        pos = torch.arange(s.seq_len)
        tok_page.append(page_off + pos // P)
        tok_slot.append(pos % P)
        page_off += n
    tok_phys = perm[torch.cat(tok_page)].to(device)
    tok_slot = torch.cat(tok_slot).to(device)

    # page-tail filler: finite, large, so an unmasked tail slot ruins parity
    k_cache = (randn_bf16(num_pages, Hkv, P, d).float() * 50.0).to(torch.bfloat16)
    v_cache = (randn_bf16(num_pages, Hkv, P, d).float() * 50.0).to(torch.bfloat16)
    k_cache[tok_phys, :, tok_slot] = k
    v_cache[tok_phys, :, tok_slot] = v
    del tok_phys, tok_slot

    return Batch(name=name, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=d, page_size=P,
                 seqs=list(seqs), q=q, k=k if keep_contiguous else None,
                 v=v if keep_contiguous else None, k_cache=k_cache, v_cache=v_cache,
                 block_table=block_table.to(device), page_perm=perm,
                 seed=seed, outlier_frac=outlier_frac)


def new_token_slots(batch: Batch):
    """Physical (page, slot) of every new token, in q's token order (positions
    L - T .. L - 1 of each sequence through its block table)."""
    bt = batch.block_table.cpu()
    pages, slots = [], []
    for i, s in enumerate(batch.seqs):
        pos = torch.arange(s.seq_len - s.query_len, s.seq_len)
        pages.append(bt[i, pos // batch.page_size].long())
        slots.append(pos % batch.page_size)
    dev = batch.k_cache.device
    return torch.cat(pages).to(dev), torch.cat(slots).to(dev)


def tail_slots(batch: Batch):
    """Physical (page, slot) of the unused slots past L in each sequence's last page."""
    bt = batch.block_table.cpu()
    pages, slots = [], []
    for i, s in enumerate(batch.seqs):
        n = (-s.seq_len) % batch.page_size
        if n:
            pos = torch.arange(s.seq_len, s.seq_len + n)
            pages.append(bt[i, pos // batch.page_size].long())
            slots.append(pos % batch.page_size)
    dev = batch.k_cache.device
    if not pages:
        return torch.zeros(0, dtype=torch.long, device=dev), torch.zeros(0, dtype=torch.long, device=dev)
    return torch.cat(pages).to(dev), torch.cat(slots).to(dev)


def new_token_kv(batch: Batch):
    """The new tokens' K and V as dense [sum T, Hkv, d] tensors in q's token order (the
    inputs of a fused cache append), read from the cache where the batch placed them."""
    pg, sl = new_token_slots(batch)
    return batch.k_cache[pg, :, sl].contiguous(), batch.v_cache[pg, :, sl].contiguous()


@dataclasses.dataclass
class Fp8KV:
    """A batch's K/V as FP8 (E4M3) codes with one scale per KV head.

    k_codes, v_codes  [sum L, Hkv, d] uint8, contiguous per sequence (what the oracle
                      decodes); k_scale, v_scale [Hkv] float32;
    k_cache           [num_pages, Hkv, page_size, d] uint8 (the batch's paging);
    v_cache_t         [num_pages, Hkv, d, page_size] uint8: each page block transposed,
                      the layout the FP8 kernels read V in.
    Unused slots past a sequence's end hold random bytes (NaN codes included)."""
    k_codes: torch.Tensor
    v_codes: torch.Tensor
    k_scale: torch.Tensor
    v_scale: torch.Tensor
    k_cache: torch.Tensor
    v_cache_t: torch.Tensor


def fp8_kv(batch: Batch, seed: int = 0) -> Fp8KV:
    """Quantise a batch's K/V to FP8 E4M3 per KV head (scale = max |x| / 448 over the head;
    round to nearest with torch's float8_e4m3fn conversion) and lay the codes out paged.
    Inputs only: the oracle decodes the codes itself."""
    if batch.k is None:
        raise ValueError("fp8_kv needs the batch's contiguous K/V")
    dev = batch.k.device
    P = batch.page_size

    def quant(x):
        amax = x.float().abs().amax(dim=(0, 2)).clamp_min(1e-30)          # [Hkv]
        scale = amax / 448.0
        codes = (x.float() / scale[None, :, None]).to(torch.float8_e4m3fn).view(torch.uint8)
        return codes, scale.to(torch.float32)

    kc, ks = quant(batch.k)
    vc, vs = quant(batch.v)
    gen = torch.Generator(device=dev).manual_seed(seed + 4242)
    num_pages, Hkv, _, d = batch.k_cache.shape
    k_cache = torch.randint(0, 256, (num_pages, Hkv, P, d), generator=gen, device=dev, dtype=torch.int32).to(torch.uint8)
    v_cache = torch.randint(0, 256, (num_pages, Hkv, P, d), generator=gen, device=dev, dtype=torch.int32).to(torch.uint8)
    bt = batch.block_table.cpu()
    pages, slots = [], []
    for i, sp in enumerate(batch.seqs):
        pos = torch.arange(sp.seq_len)
        pages.append(bt[i, pos // P].long())
        slots.append(pos % P)
    pg = torch.cat(pages).to(dev)
    sl = torch.cat(slots).to(dev)
    k_cache[pg, :, sl] = kc
    v_cache[pg, :, sl] = vc
    return Fp8KV(k_codes=kc, v_codes=vc, k_scale=ks, v_scale=vs, k_cache=k_cache,
                 v_cache_t=v_cache.transpose(2, 3).contiguous())


def shard_batch(batch: Batch, rank: int, world: int) -> Batch:
    """The part of ``batch`` one of ``world`` GPUs holds (paged_kv_attention_verify_b200.shard):
    its KV heads' cache and queries for its sequences. The page pool keeps its size (the
    block table still addresses it); only the sequences' rows are taken."""
    from paged_kv_attention_verify_b200 import shard as S
    tp_rank, sp_rank, tp, sp = S.shard_coords(rank, world, batch.num_kv_heads)
    kv0, kv1, q0, q1 = S.head_range(tp_rank, tp, batch.num_q_heads, batch.num_kv_heads)
    seqs = S.sequence_subset(len(batch.seqs), sp_rank, sp)
    qo, ko = batch.q_offsets(), batch.kv_offsets()
    empty = torch.zeros(0, dtype=torch.long)
    qrows = torch.cat([empty] + [torch.arange(qo[s], qo[s] + batch.seqs[s].query_len) for s in seqs]).to(batch.q.device)
    k = v = None
    if batch.k is not None:
        krows = torch.cat([empty] + [torch.arange(ko[s], ko[s] + batch.seqs[s].seq_len) for s in seqs]).to(batch.k.device)
        k = batch.k[krows, kv0:kv1].contiguous()
        v = batch.v[krows, kv0:kv1].contiguous()
    return Batch(name=f"{batch.name}[rank {rank}/{world}]", num_q_heads=q1 - q0, num_kv_heads=kv1 - kv0,
                 head_dim=batch.head_dim, page_size=batch.page_size, seqs=[batch.seqs[s] for s in seqs],
                 q=batch.q[qrows, q0:q1].contiguous(), k=k, v=v,
                 k_cache=batch.k_cache[:, kv0:kv1].contiguous(), v_cache=batch.v_cache[:, kv0:kv1].contiguous(),
                 block_table=batch.block_table[torch.tensor(seqs, dtype=torch.long,
                                                            device=batch.block_table.device)].contiguous(),
                 page_perm=batch.page_perm, seed=batch.seed, outlier_frac=batch.outlier_frac)


SEQUENCE_CLASSES = ("prefill", "decode", "verify")


def seq_class(spec: SeqSpec) -> str:
    """prefill: a causal chunk of several new tokens; decode: one new token; verify: a draft tree."""
    if spec.mask_kind == TREE:
        return "verify"
    return "decode" if spec.query_len == 1 else "prefill"


def class_batches(batch: Batch) -> dict:
    """The batch's sequences split by class (prefill / decode / verify): each part keeps the
    same page pool, caches and query values, and takes only its sequences' query rows and
    block-table rows. Classes with no sequence are left out."""
    qo = batch.q_offsets()
    parts = {}
    for cls in SEQUENCE_CLASSES:
        seqs = [i for i, sp in enumerate(batch.seqs) if seq_class(sp) == cls]
        if not seqs:
            continue
        qrows = torch.cat([torch.arange(qo[i], qo[i] + batch.seqs[i].query_len) for i in seqs]).to(batch.q.device)
        k = v = None
        if batch.k is not None:
            ko = batch.kv_offsets()
            krows = torch.cat([torch.arange(ko[i], ko[i] + batch.seqs[i].seq_len) for i in seqs]).to(batch.k.device)
            k, v = batch.k[krows], batch.v[krows]
        sel = torch.tensor(seqs, dtype=torch.long, device=batch.block_table.device)
        parts[cls] = Batch(name=f"{batch.name}[{cls}]", num_q_heads=batch.num_q_heads,
                           num_kv_heads=batch.num_kv_heads, head_dim=batch.head_dim,
                           page_size=batch.page_size, seqs=[batch.seqs[i] for i in seqs],
                           q=batch.q[qrows].contiguous(), k=k, v=v,
                           k_cache=batch.k_cache, v_cache=batch.v_cache,
                           block_table=batch.block_table[sel].contiguous(),
                           page_perm=batch.page_perm, seed=batch.seed, outlier_frac=batch.outlier_frac)
    return parts


def make_config(name: str, device="cpu", seed: Optional[int] = None,
                keep_contiguous: bool = True, max_seqs: Optional[int] = None) -> Batch:
    """One of the five named batches, seeded by its index unless ``seed`` is given.

    ``max_seqs`` keeps only the first sequences (smaller cases of the same shape, e.g.
    for profiler captures)."""
    if seed is None:
        seed = CONFIG_NAMES.index(name)
    sgen = torch.Generator().manual_seed(seed)
    seqs, Hq, Hkv, d, outl = config_seqs(name, sgen)
    if max_seqs is not None:
        seqs = seqs[:max_seqs]
    # structure draws above advance sgen; build_batch re-seeds its own structure stream
    return build_batch(name, seqs, Hq, Hkv, d, seed=seed + 1000, device=device,
                       outlier_frac=outl, keep_contiguous=keep_contiguous)


def repage(batch: Batch, perm_seed: int) -> Batch:
    """Same Q/K/V values, a different random page permutation (for invariance tests)."""
    return build_batch(batch.name, batch.seqs, batch.num_q_heads, batch.num_kv_heads,
                       batch.head_dim, seed=batch.seed, device=batch.q.device,
                       page_size=batch.page_size, perm_seed=perm_seed,
                       outlier_frac=batch.outlier_frac)


def random_small(seed: int, num_seqs: int = 4, Hq: int = 8, Hkv: int = 2, d: int = 64,
                 max_ctx: int = 80, max_q: int = 40, tree_frac: float = 0.3,
                 max_draft: int = 8, device="cpu", bt_extra: int = 0) -> Batch:
    """A small mixed batch: causal chunks of random length on random prefixes, decode
    steps, and verify rows on random draft trees; sized for the CPU oracle."""
    gen = torch.Generator().manual_seed(seed)
    seqs = []
    for _ in range(num_seqs):
        r = torch.rand((), generator=gen).item()
        prefix = int(torch.randint(0, max_ctx + 1, (1,), generator=gen).item())
        if r < tree_frac:
            T = int(torch.randint(1, max_draft + 1, (1,), generator=gen).item())
            seqs.append(SeqSpec(prefix + T, T, TREE, random_tree(gen, T)))
        else:
            T = int(torch.randint(1, max_q + 1, (1,), generator=gen).item())
            seqs.append(SeqSpec(prefix + T, T, CAUSAL, []))
    return build_batch(f"random_small_{seed}", seqs, Hq, Hkv, d, seed=seed + 7,
                       device=device, bt_extra=bt_extra)
