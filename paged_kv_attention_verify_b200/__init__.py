"""Paged-KV attention for unified prefill / decode / verify batches on B200 (sm_100a).

Thin ctypes binding over the C ABI in ``include/pkva.h`` (library: ``lib/libpkva.so``,
built in-tree by ``python -m paged_kv_attention_verify_b200.build``). This module only
marshals arguments: host integer arrays go in as int32 buffers, device tensors as raw
pointers, the stream as a ``cudaStream_t``. Every step of the computation runs in the
library's kernels; there is no fallback of any kind, so a missing library is an error.

    plan = Plan(seq_lens, query_lens, block_table, mask_kind, parents,
                num_q_heads=32, num_kv_heads=8, head_dim=128, num_pages=P)
    out = plan.run(q, k_cache, v_cache)        # q, caches, out: bf16 CUDA tensors
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libpkva.so")

CAUSAL = 0
TREE = 1

PKVA_OK = 0
STATUS_NAMES = {0: "PKVA_OK", -1: "PKVA_EINVAL", -2: "PKVA_EUNSUPPORTED", -3: "PKVA_ECUDA",
                -4: "PKVA_ENOMEM", -5: "PKVA_EDEVICE"}
KV_BF16 = 0
KV_FP8_E4M3 = 1
DEVERR_BAD_PAGE = 0x1
DEVERR_TIMEOUT = 0x2

# every entry point that include/pkva.h declares
EXPORTED = ["attn_plan", "attn_plan_shared", "attn_plan_kv", "attn_plan_shared_kv", "attn_run", "attn_run_fp8", "attn_run_fp8_append",
            "attn_run_host_async", "attn_host_wait", "attn_run_append", "attn_run_host", "attn_check", "attn_plan_destroy",
            "attn_last_error", "attn_plan_get_info", "attn_plan_inspect", "attn_run_static",
            "pkva_selftest_wait_timeout"]


class PkvaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


class PlanInfo(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("num_decode_items", ctypes.c_int32),
                ("num_prefill_items", ctypes.c_int32), ("num_split_units", ctypes.c_int32),
                ("num_partial_slots", ctypes.c_int32), ("decode_rows", ctypes.c_int32),
                ("kv_bytes", ctypes.c_int64), ("attn_flops", ctypes.c_int64),
                ("scratch_bytes", ctypes.c_int64), ("num_cascade_items", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class WorkDesc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("seq", ctypes.c_int32), ("kv_head", ctypes.c_int32),
                ("q_head", ctypes.c_int32), ("row_begin", ctypes.c_int32), ("row_count", ctypes.c_int32),
                ("key_begin", ctypes.c_int32), ("key_end", ctypes.c_int32),
                ("split", ctypes.c_int32), ("num_splits", ctypes.c_int32)]


_lib = None
_i32p = ctypes.POINTER(ctypes.c_int32)
_vp = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    """Load the in-tree library (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m paged_kv_attention_verify_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    L.attn_plan.argtypes = [ctypes.POINTER(_vp), ctypes.c_int, _i32p, _i32p, _vp, ctypes.c_int,
                            ctypes.c_int, _i32p, _i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                            ctypes.c_int, ctypes.c_float]
    L.attn_plan_shared.argtypes = L.attn_plan.argtypes + [_i32p, _i32p, ctypes.c_int]
    L.attn_plan_kv.argtypes = L.attn_plan.argtypes + [ctypes.c_int]
    L.attn_plan_shared_kv.argtypes = L.attn_plan_shared.argtypes + [ctypes.c_int]
    L.attn_run_fp8.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    L.attn_run_fp8_append.argtypes = [_vp] * 10
    L.attn_run.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp]
    L.attn_run_append.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    L.attn_run_host.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp]
    L.attn_run_host_async.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp]
    L.attn_host_wait.argtypes = [_vp, _vp]
    L.attn_check.argtypes = [_vp, _vp, _i32p]
    L.attn_plan_destroy.argtypes = [_vp]
    L.attn_plan_destroy.restype = None
    L.attn_last_error.restype = ctypes.c_char_p
    L.attn_plan_get_info.argtypes = [_vp, ctypes.POINTER(PlanInfo)]
    L.attn_plan_inspect.argtypes = [ctypes.c_int, _i32p, _i32p, ctypes.c_int, ctypes.c_int, _i32p,
                                    _i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    _i32p, _i32p, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ctypes.POINTER(WorkDesc),
                                    ctypes.c_int, _i32p]
    L.attn_run_static.argtypes = [ctypes.c_int, _i32p, _i32p, _vp, ctypes.c_int, ctypes.c_int, _i32p,
                                  _i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_float, _vp, _vp, _vp, _vp, _vp]
    L.pkva_selftest_wait_timeout.argtypes = [ctypes.c_longlong, _i32p]
    for name in ("attn_plan", "attn_plan_shared", "attn_plan_kv", "attn_plan_shared_kv", "attn_run_fp8", "attn_run_fp8_append",
                 "attn_run_host_async", "attn_host_wait", "attn_run", "attn_run_append", "attn_run_host", "attn_check", "attn_plan_get_info",
                 "attn_plan_inspect", "attn_run_static", "pkva_selftest_wait_timeout"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _check(rc: int):
    if rc != PKVA_OK:
        raise PkvaError(rc, lib().attn_last_error().decode())


def _i32(values) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(values, dtype=np.int32).reshape(-1))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_i32p) if a.size else None


def _stream_handle(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _host_arrays(seq_lens, query_lens, mask_kind, parents):
    """The per-sequence host arrays as int32 buffers, one entry per sequence each."""
    sl, ql, mk = _i32(seq_lens), _i32(query_lens), _i32(mask_kind)
    par = _i32(parents if parents is not None else [])
    if len(sl) != len(ql) or len(sl) != len(mk):
        raise ValueError("seq_lens, query_lens and mask_kind must have one entry per sequence")
    return sl, ql, mk, par


def _block_table_arg(block_table, num_seqs: int):
    """(device pointer, bt_stride) of a contiguous int32 CUDA block table [num_seqs, stride]."""
    import torch
    if not num_seqs:
        return None, 0
    if not (isinstance(block_table, torch.Tensor) and block_table.is_cuda
            and block_table.dtype == torch.int32 and block_table.dim() == 2
            and block_table.is_contiguous() and block_table.shape[0] == num_seqs):
        raise ValueError("block_table must be a contiguous int32 CUDA tensor [num_seqs, bt_stride]")
    return block_table.data_ptr(), block_table.shape[1]


def _check_bf16_tensors(q, k_cache, v_cache, out, total_q, Hq, Hkv, D, num_pages, page_size):
    """q / out bf16 [total_q, Hq, D] and the caches bf16 [num_pages, Hkv, page_size, D], all
    contiguous CUDA tensors."""
    import torch
    for name, t, shape in (("q", q, (total_q, Hq, D)), ("out", out, (total_q, Hq, D)),
                           ("k_cache", k_cache, (num_pages, Hkv, page_size, D)),
                           ("v_cache", v_cache, (num_pages, Hkv, page_size, D))):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be a bf16 CUDA tensor")
        if tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous with shape {shape}, got {tuple(t.shape)}")


class Plan:
    """A planned batch (``attn_plan``); run it any number of times with ``run``."""

    def __init__(self, seq_lens: Sequence[int], query_lens: Sequence[int], block_table,
                 mask_kind: Sequence[int], parents: Optional[Sequence[int]] = None, *,
                 num_q_heads: int, num_kv_heads: int, head_dim: int, num_pages: int,
                 page_size: int = 16, sm_scale: Optional[float] = None,
                 prefix_group: Optional[Sequence[int]] = None,
                 prefix_len: Optional[Sequence[int]] = None, kv_fp8: bool = False):
        """``attn_plan``; with ``prefix_group`` / ``prefix_len`` (shared-prefix groups),
        ``attn_plan_shared``; with ``kv_fp8``, ``attn_plan_kv`` (or ``attn_plan_shared_kv``
        with groups) for FP8 E4M3 caches."""
        self._handle = None
        sl, ql, mk, par = _host_arrays(seq_lens, query_lens, mask_kind, parents)
        bt_ptr, bt_stride = _block_table_arg(block_table, len(sl))
        self.block_table = block_table          # keep the caller's table alive with the plan
        self.num_q_heads, self.num_kv_heads, self.head_dim = num_q_heads, num_kv_heads, head_dim
        self.num_pages, self.page_size = num_pages, page_size
        self.total_q = int(ql.sum()) if len(ql) else 0
        h = _vp()
        args = (ctypes.byref(h), len(sl), _ptr(sl), _ptr(ql), bt_ptr, bt_stride, num_pages, _ptr(mk),
                _ptr(par), num_q_heads, num_kv_heads, head_dim, page_size,
                float(sm_scale) if sm_scale else 0.0)
        self.kv_fp8 = kv_fp8
        if prefix_group is None:
            _check(lib().attn_plan_kv(*args, KV_FP8_E4M3) if kv_fp8 else lib().attn_plan(*args))
        else:
            pg, pl = _i32(prefix_group), _i32(prefix_len if prefix_len is not None else [])
            if len(pg) != len(sl):
                raise ValueError("prefix_group must have one entry per sequence")
            if kv_fp8:
                _check(lib().attn_plan_shared_kv(*args, _ptr(pg), _ptr(pl), len(pl), KV_FP8_E4M3))
            else:
                _check(lib().attn_plan_shared(*args, _ptr(pg), _ptr(pl), len(pl)))
        self._handle = h

    # -- marshalling checks (shapes, dtypes, devices) ---------------------------------
    def _check_tensors(self, q, k_cache, v_cache, out):
        _check_bf16_tensors(q, k_cache, v_cache, out, self.total_q, self.num_q_heads, self.num_kv_heads,
                            self.head_dim, self.num_pages, self.page_size)

    def run(self, q, k_cache, v_cache, out=None, stream=None):
        """out = attention(q, paged K/V); asynchronous on ``stream`` (default: current)."""
        import torch
        if out is None:
            out = torch.empty_like(q)
        self._check_tensors(q, k_cache, v_cache, out)
        _check(lib().attn_run(self._handle, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                              out.data_ptr(), _stream_handle(stream)))
        return out

    def run_append(self, q, k_new, v_new, k_cache, v_cache, out=None, stream=None):
        """Write the new tokens' K/V (``k_new``/``v_new`` [sum T, Hkv, D]) into the cache and
        compute the attention, in one launch (``attn_run_append``)."""
        import torch
        if out is None:
            out = torch.empty_like(q)
        self._check_tensors(q, k_cache, v_cache, out)
        shape = (self.total_q, self.num_kv_heads, self.head_dim)
        for name, t in (("k_new", k_new), ("v_new", v_new)):
            if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16 \
                    or tuple(t.shape) != shape or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor {shape}")
        _check(lib().attn_run_append(self._handle, q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(),
                                     k_cache.data_ptr(), v_cache.data_ptr(), out.data_ptr(),
                                     _stream_handle(stream)))
        return out

    def run_fp8(self, q, k_cache, v_cache_t, k_scale, v_scale, out=None, stream=None, _new=None):
        """``attn_run_fp8``: E4M3 codes (uint8) in ``k_cache`` [pages, Hkv, 16, D] and, each
        page block transposed, ``v_cache_t`` [pages, Hkv, D, 16]; float32 scales [Hkv]."""
        import torch
        if out is None:
            out = torch.empty_like(q)
        D, Hq, Hkv = self.head_dim, self.num_q_heads, self.num_kv_heads
        checks = (("q", q, (self.total_q, Hq, D), torch.bfloat16), ("out", out, (self.total_q, Hq, D), torch.bfloat16),
                  ("k_cache", k_cache, (self.num_pages, Hkv, self.page_size, D), torch.uint8),
                  ("v_cache_t", v_cache_t, (self.num_pages, Hkv, D, self.page_size), torch.uint8),
                  ("k_scale", k_scale, (Hkv,), torch.float32), ("v_scale", v_scale, (Hkv,), torch.float32))
        for name, t, shape, dt in checks:
            if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != dt or tuple(t.shape) != shape \
                    or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous {dt} CUDA tensor {shape}")
        if _new is None:
            _check(lib().attn_run_fp8(self._handle, q.data_ptr(), k_cache.data_ptr(), v_cache_t.data_ptr(),
                                      k_scale.data_ptr(), v_scale.data_ptr(), out.data_ptr(), _stream_handle(stream)))
        else:
            _check(lib().attn_run_fp8_append(self._handle, q.data_ptr(), _new[0].data_ptr(), _new[1].data_ptr(),
                                             k_cache.data_ptr(), v_cache_t.data_ptr(), k_scale.data_ptr(),
                                             v_scale.data_ptr(), out.data_ptr(), _stream_handle(stream)))
        return out

    def run_fp8_append(self, q, k_new, v_new, k_cache, v_cache_t, k_scale, v_scale, out=None, stream=None):
        """``attn_run_fp8_append``: quantise the new tokens' K/V (bf16 [sum T, Hkv, D]) into the
        FP8 caches at their slots and compute the attention (one launch; with tensor-core
        tasks, the staging launch before it appends their sequences' rows)."""
        import torch
        if out is None:
            out = torch.empty_like(q)
        shape = (self.total_q, self.num_kv_heads, self.head_dim)
        for name, t in (("k_new", k_new), ("v_new", v_new)):
            if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16 \
                    or tuple(t.shape) != shape or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor {shape}")
        self.run_fp8(q, k_cache, v_cache_t, k_scale, v_scale, out=out, stream=stream, _new=(k_new, v_new))
        return out

    def run_host(self, q_host, k_cache, v_cache, out_host, stream=None):
        """End-to-end call: q and out in (pinned) host memory; copies ride on ``stream``."""
        import torch
        for name, t in (("q_host", q_host), ("out_host", out_host)):
            if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or \
                    tuple(t.shape) != (self.total_q, self.num_q_heads, self.head_dim):
                raise ValueError(f"{name} must be a contiguous bf16 host tensor "
                                 f"[{self.total_q}, {self.num_q_heads}, {self.head_dim}]")
        _check(lib().attn_run_host(self._handle, q_host.data_ptr(), k_cache.data_ptr(),
                                   v_cache.data_ptr(), out_host.data_ptr(), _stream_handle(stream)))
        return out_host

    def run_host_async(self, q_host, k_cache, v_cache, out_host, stream=None):
        """``attn_run_host_async``: as ``run_host`` with the copy out on the plan's own stream;
        ``out_host`` is complete once ``stream`` has passed ``host_wait`` (then synchronize)."""
        import torch
        for name, t in (("q_host", q_host), ("out_host", out_host)):
            if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or \
                    tuple(t.shape) != (self.total_q, self.num_q_heads, self.head_dim):
                raise ValueError(f"{name} must be a contiguous bf16 host tensor "
                                 f"[{self.total_q}, {self.num_q_heads}, {self.head_dim}]")
        _check(lib().attn_run_host_async(self._handle, q_host.data_ptr(), k_cache.data_ptr(),
                                         v_cache.data_ptr(), out_host.data_ptr(), _stream_handle(stream)))
        return out_host

    def host_wait(self, stream=None):
        """``attn_host_wait``: order ``stream`` after every copy out issued so far."""
        _check(lib().attn_host_wait(self._handle, _stream_handle(stream)))

    def check(self, stream=None) -> int:
        """Synchronize and return the device error bits (0 if none); raises on CUDA errors."""
        err = ctypes.c_int32(0)
        rc = lib().attn_check(self._handle, _stream_handle(stream), ctypes.byref(err))
        if rc not in (PKVA_OK, -5):
            _check(rc)
        return int(err.value)

    def info(self) -> Dict[str, int]:
        inf = PlanInfo()
        _check(lib().attn_plan_get_info(self._handle, ctypes.byref(inf)))
        return {f: getattr(inf, f) for f, _ in PlanInfo._fields_}

    def close(self):
        if self._handle:
            lib().attn_plan_destroy(self._handle)
            self._handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def inspect(seq_lens, query_lens, mask_kind, parents=None, *, num_q_heads: int,
            num_kv_heads: int, head_dim: int, num_pages: int, bt_stride: int,
            num_sms: int = 148, ctas_per_sm: int = 2, page_size: int = 16,
            prefix_group=None, prefix_len=None) -> List[Dict[str, int]]:
    """Host-only planner run (``attn_plan_inspect``): the tile tasks in launch order."""
    sl, ql, mk = _i32(seq_lens), _i32(query_lens), _i32(mask_kind)
    par = _i32(parents if parents is not None else [])
    pg = _i32(prefix_group if prefix_group is not None else [])
    pl = _i32(prefix_len if prefix_len is not None else [])
    n = ctypes.c_int32(0)
    args = (len(sl), _ptr(sl), _ptr(ql), bt_stride, num_pages, _ptr(mk), _ptr(par), num_q_heads,
            num_kv_heads, head_dim, page_size, _ptr(pg), _ptr(pl), len(pl) if prefix_group is not None else 0,
            num_sms, ctas_per_sm)
    _check(lib().attn_plan_inspect(*args, None, 0, ctypes.byref(n)))
    arr = (WorkDesc * max(1, n.value))()
    _check(lib().attn_plan_inspect(*args, arr, n.value, ctypes.byref(n)))
    return [{f: getattr(arr[i], f) for f, _ in WorkDesc._fields_} for i in range(n.value)]


def run_static(seq_lens, query_lens, block_table, mask_kind, parents, q, k_cache, v_cache, out, *,
               num_q_heads: int, num_kv_heads: int, head_dim: int, num_pages: int,
               page_size: int = 16, sm_scale: Optional[float] = None, stream=None):
    """``attn_run_static``: plan and run in one call without allocating device memory.

    For callers that cannot allocate where they need attention; ``out`` must be
    allocated by the caller beforehand. The library keeps the call's tables and split
    scratch in a fixed array it reserves per GPU, so overlapping calls race (serialize
    them), and batches beyond that array's limits raise PKVA_EUNSUPPORTED.

    Every tensor must be on the current CUDA device: the call reaches the scratch of that
    device and launches there."""
    import torch
    sl, ql, mk, par = _host_arrays(seq_lens, query_lens, mask_kind, parents)
    bt_ptr, bt_stride = _block_table_arg(block_table, len(sl))
    total_q = int(ql.sum()) if len(ql) else 0
    _check_bf16_tensors(q, k_cache, v_cache, out, total_q, num_q_heads, num_kv_heads, head_dim, num_pages,
                        page_size)
    dev = torch.cuda.current_device()
    for name, t in (("block_table", block_table), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                    ("out", out)):
        if (name != "block_table" or len(sl)) and t.device.index != dev:
            raise ValueError(f"{name} is on {t.device}, not on the current device cuda:{dev}")
    _check(lib().attn_run_static(len(sl), _ptr(sl), _ptr(ql), bt_ptr,
                                 bt_stride, num_pages, _ptr(mk), _ptr(par), num_q_heads, num_kv_heads,
                                 head_dim, page_size, float(sm_scale) if sm_scale else 0.0,
                                 q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), out.data_ptr(),
                                 _stream_handle(stream)))
    return out


def selftest_wait_timeout(limit_ns: int = 20_000_000) -> int:
    """Run the bounded-wait self-test; returns the device error bits it reported."""
    err = ctypes.c_int32(0)
    _check(lib().pkva_selftest_wait_timeout(int(limit_ns), ctypes.byref(err)))
    return int(err.value)


def plan_for_batch(batch, sm_scale: Optional[float] = None, shared: bool = True, kv_fp8: bool = False) -> Plan:
    """Plan a ``workloads.Batch`` (a convenience for tests and the benchmark); a batch with
    shared-prefix groups is planned with them unless ``shared`` is False; ``kv_fp8`` plans
    for FP8 caches."""
    groups = getattr(batch, "prefix_group", None) if shared else None
    return Plan(batch.seq_lens, batch.query_lens, batch.block_table, batch.mask_kinds,
                batch.parents_flat, num_q_heads=batch.num_q_heads, num_kv_heads=batch.num_kv_heads,
                head_dim=batch.head_dim, num_pages=batch.k_cache.shape[0],
                page_size=batch.page_size, sm_scale=sm_scale,
                prefix_group=groups, prefix_len=batch.prefix_len if groups is not None else None,
                kv_fp8=kv_fp8)
