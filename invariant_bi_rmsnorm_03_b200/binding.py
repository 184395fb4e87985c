"""Thin ctypes binding of the C ABI (include/bi.h), taking torch tensors.

Each method marshals its arguments (device pointers, sizes, the current CUDA
stream) and calls the C entry point of the same name; every step of the
computation runs in the library's CUDA kernels.  torch provides device
memory and streams only.  There is no fallback: if the library is missing or
cannot be loaded, :func:`load` raises.
"""
from __future__ import annotations

import ctypes
import enum
import math
import os
from dataclasses import dataclass

import torch

LIBDIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib")
PAGE_SIZE = 16
SPLIT_KEYS = 256
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024  # BI_NOALLOC_SCRATCH_BYTES of include/bi.h


class Status(enum.IntEnum):
    OK = 0
    INVALID = 1
    UNSUPPORTED = 2
    CUDA = 3
    TIMEOUT = 4
    WORKSPACE = 5
    DEVICE_INDEX = 6


class BIError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__("%s failed: %s (%d)" % (fn, text, status))
        self.status = Status(status)


class _PagedKV(ctypes.Structure):
    _fields_ = [("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("max_pages_per_seq", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


@dataclass
class PagedKV:
    """A paged KV cache on the device: ``k_cache``/``v_cache`` bf16 tensors
    of shape ``[num_pages, Hkv, 16, d]`` holding one 16 x d block per (page,
    kv head), each block stored in the tensor core's core-matrix order (see
    ``include/bi.h``; ``bi_kv_write`` produces it), and ``block_table`` int32
    ``[num_seqs, max_pages]``.  The caller owns the tensors."""

    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_table: torch.Tensor

    def c_struct(self) -> _PagedKV:
        k, v, bt = self.k_cache, self.v_cache, self.block_table
        if k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16 or bt.dtype != torch.int32:
            raise TypeError("k_cache/v_cache must be bfloat16 and block_table int32")
        if k.shape != v.shape or k.dim() != 4 or k.shape[2] != PAGE_SIZE:
            raise ValueError("cache tensors must be [num_pages, Hkv, 16, d]")
        for t in (k, v, bt):
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError("cache tensors must be contiguous CUDA tensors")
        return _PagedKV(k.data_ptr(), v.data_ptr(), bt.data_ptr(), bt.shape[1], k.shape[0],
                        PAGE_SIZE, k.shape[1], k.shape[3])

    @property
    def num_kv_heads(self) -> int:
        return self.k_cache.shape[1]

    @property
    def head_dim(self) -> int:
        return self.k_cache.shape[3]


_DT = {torch.bfloat16: 0, torch.float32: 1}


def _stream(stream=None) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


class Library:
    """One loaded build of the library (invariant or variant-off)."""

    SYMBOLS = ("bi_rmsnorm", "bi_matmul", "bi_matmul_workspace_bytes", "bi_kv_write",
               "bi_attention_decode", "bi_attention_decode_workspace_bytes",
               "bi_attention_prefill", "bi_attention_prefill_workspace_bytes",
               "bi_status_string", "bi_build_invariant", "bi_device_status",
               "bi_debug_bounded_wait", "bi_add_rmsnorm", "bi_embedding", "bi_rope_kv_write",
               "bi_swiglu", "bi_argmax", "bi_sample", "bi_moe_route", "bi_moe_dispatch",
               "bi_moe_combine", "bi_matmul_grouped", "bi_fold_norm_weight",
               "bi_rmsnorm_matmul", "bi_matmul_residual", "bi_rope_table",
               "bi_rmsnorm_matmul_rope_kv", "bi_rmsnorm_backward",
               "bi_rmsnorm_backward_workspace_bytes", "bi_transpose", "bi_matmul_backward",
               "bi_matmul_backward_workspace_bytes", "bi_swiglu_backward", "bi_rope_backward",
               "bi_attention_backward", "bi_attention_backward_workspace_bytes",
               "bi_rmsnorm_matmul_workspace_bytes")

    def __init__(self, path: str):
        if not os.path.exists(path):
            raise ImportError("CUDA library %s is missing: build it with "
                              "`python -m invariant_bi_rmsnorm_03_b200.build`" % path)
        self.path = path
        L = ctypes.CDLL(path)
        P, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
        sz, st = ctypes.c_size_t, ctypes.c_int
        kvp = ctypes.POINTER(_PagedKV)
        L.bi_rmsnorm.argtypes = [P, P, P, i64, i64, f32, st, P]
        L.bi_matmul.argtypes = [P, P, P, i64, i64, i64, st, P, sz, P]
        L.bi_matmul_workspace_bytes.argtypes = [i64, i64, i64]
        L.bi_matmul_workspace_bytes.restype = sz
        L.bi_kv_write.argtypes = [kvp, P, P, P, i64, P]
        L.bi_attention_decode.argtypes = [kvp, P, P, P, P, i32, i32, i32, f32, i32, P, sz, P]
        L.bi_attention_decode_workspace_bytes.argtypes = [kvp, i32, i32, i32, i32]
        L.bi_attention_decode_workspace_bytes.restype = sz
        L.bi_attention_prefill.argtypes = [kvp, P, P, P, P, P, i32, i32, i64, i32, f32, P, sz, P]
        L.bi_attention_prefill_workspace_bytes.argtypes = [kvp, i32, i32, i32]
        L.bi_attention_prefill_workspace_bytes.restype = sz
        L.bi_status_string.argtypes = [st]
        L.bi_status_string.restype = ctypes.c_char_p
        L.bi_build_invariant.restype = ctypes.c_int
        L.bi_device_status.argtypes = [P]
        L.bi_debug_bounded_wait.argtypes = [ctypes.c_uint64, P]
        L.bi_attention_decode_noalloc.argtypes = [kvp, P, P, P, P, i32, i32, i32, f32, i32, P]
        L.bi_attention_decode_noalloc.restype = st
        L.bi_add_rmsnorm.argtypes = [P, P, P, P, i64, i64, f32, st, P]
        L.bi_embedding.argtypes = [P, i64, i64, P, P, i64, P]
        L.bi_rope_kv_write.argtypes = [kvp, P, P, P, P, i64, i32, f32, P]
        L.bi_swiglu.argtypes = [P, P, i64, i64, P]
        L.bi_argmax.argtypes = [P, i64, i64, P, P]
        L.bi_sample.argtypes = [P, i64, i64, P, P, P, P, P, P]
        L.bi_moe_route.argtypes = [P, i64, i32, i32, P, P, P]
        L.bi_moe_dispatch.argtypes = [P, i64, i32, i32, P, P, P, P, P]
        L.bi_moe_combine.argtypes = [P, P, P, i64, i32, i64, P, P]
        L.bi_matmul_grouped.argtypes = [P, P, P, P, i32, i64, i64, i64, st, P]
        L.bi_fold_norm_weight.argtypes = [P, P, P, i64, i64, P]
        L.bi_rmsnorm_matmul.argtypes = [P, P, P, i64, i64, i64, f32, st, P, sz, P]
        L.bi_rmsnorm_matmul_workspace_bytes.argtypes = [i64]
        L.bi_rmsnorm_matmul_workspace_bytes.restype = sz
        L.bi_matmul_residual.argtypes = [P, P, P, P, i64, i64, i64, P]
        L.bi_rope_table.argtypes = [P, i32, i32, f32, P]
        L.bi_rmsnorm_matmul_rope_kv.argtypes = [P, P, f32, kvp, P, i32, P, P, P, i64, i64, i32, P,
                                                sz, P]
        L.bi_rmsnorm_backward_workspace_bytes.argtypes = [i64, i64]
        L.bi_rmsnorm_backward_workspace_bytes.restype = sz
        L.bi_rmsnorm_backward.argtypes = [P, P, P, P, P, i64, i64, f32, st, P, sz, P]
        L.bi_transpose.argtypes = [P, P, i64, i64, i64, P]
        L.bi_matmul_backward_workspace_bytes.argtypes = [i64, i64, i64]
        L.bi_matmul_backward_workspace_bytes.restype = sz
        L.bi_matmul_backward.argtypes = [P, P, P, P, P, i64, i64, i64, st, P, sz, P]
        L.bi_swiglu_backward.argtypes = [P, P, P, i64, i64, st, P]
        L.bi_rope_backward.argtypes = [P, i64, P, P, i64, i64, i32, i32, f32, st, P]
        L.bi_attention_backward.argtypes = [kvp, P, P, P, P, P, P, i32, i32, i64, i32, i32, f32,
                                            P, P, P, P, sz, P]
        L.bi_attention_backward_workspace_bytes.argtypes = [i32, i64]
        L.bi_attention_backward_workspace_bytes.restype = sz
        for name in ("bi_rmsnorm", "bi_matmul", "bi_kv_write", "bi_attention_decode",
                     "bi_attention_prefill", "bi_device_status", "bi_debug_bounded_wait",
                     "bi_add_rmsnorm", "bi_embedding", "bi_rope_kv_write", "bi_swiglu",
                     "bi_argmax", "bi_sample", "bi_moe_route", "bi_moe_dispatch",
                     "bi_moe_combine", "bi_matmul_grouped", "bi_fold_norm_weight",
                     "bi_rmsnorm_matmul", "bi_matmul_residual", "bi_rope_table",
                     "bi_rmsnorm_matmul_rope_kv", "bi_rmsnorm_backward", "bi_transpose",
                     "bi_matmul_backward", "bi_swiglu_backward", "bi_rope_backward",
                     "bi_attention_backward"):
            getattr(L, name).restype = st
        self.lib = L

    # ------------------------------------------------------------ helpers
    def _check(self, fn: str, status: int):
        if status != 0:
            raise BIError(fn, status, self.lib.bi_status_string(status).decode())

    def bi_build_invariant(self) -> int:
        return int(self.lib.bi_build_invariant())

    def bi_status_string(self, status: int) -> str:
        return self.lib.bi_status_string(int(status)).decode()

    def bi_device_status(self, stream=None) -> Status:
        return Status(self.lib.bi_device_status(_stream(stream)))

    def bi_debug_bounded_wait(self, timeout_ns: int, stream=None) -> None:
        self._check("bi_debug_bounded_wait",
                    self.lib.bi_debug_bounded_wait(int(timeout_ns), _stream(stream)))

    # ------------------------------------------------------------ RMSNorm
    def bi_rmsnorm(self, x: torch.Tensor, w: torch.Tensor, eps: float = 1e-6, out=None,
                   out_dtype=torch.bfloat16, stream=None) -> torch.Tensor:
        _need(x, "x", torch.bfloat16)
        M, H = x.shape
        _need(w, "w", torch.bfloat16, (H,))
        if out is None:
            out = torch.empty((M, H), dtype=out_dtype, device=x.device)
        _need(out, "out", out_dtype, (M, H))
        self._check("bi_rmsnorm", self.lib.bi_rmsnorm(_ptr(x), _ptr(w), _ptr(out), M, H,
                                                      float(eps), _DT[out_dtype], _stream(stream)))
        return out

    def bi_add_rmsnorm(self, x: torch.Tensor, delta: torch.Tensor, w: torch.Tensor,
                       eps: float = 1e-6, out=None, out_dtype=torch.bfloat16,
                       stream=None) -> torch.Tensor:
        """x <- round(x + delta) in place; returns RMSNorm(x) * w."""
        _need(x, "x", torch.bfloat16)
        M, H = x.shape
        _need(delta, "delta", torch.bfloat16, (M, H))
        _need(w, "w", torch.bfloat16, (H,))
        if out is None:
            out = torch.empty((M, H), dtype=out_dtype, device=x.device)
        _need(out, "out", out_dtype, (M, H))
        self._check("bi_add_rmsnorm", self.lib.bi_add_rmsnorm(
            _ptr(x), _ptr(delta), _ptr(w), _ptr(out), M, H, float(eps), _DT[out_dtype],
            _stream(stream)))
        return out

    # ------------------------------------------------------------ matmul
    def bi_matmul_workspace_bytes(self, M: int, N: int, K: int) -> int:
        return int(self.lib.bi_matmul_workspace_bytes(M, N, K))

    def bi_matmul(self, a: torch.Tensor, w: torch.Tensor, out=None, out_dtype=torch.bfloat16,
                  ws=None, stream=None) -> torch.Tensor:
        """C = a @ w.T with a [M, K] and w [N, K] (bf16)."""
        _need(a, "a", torch.bfloat16)
        M, K = a.shape
        _need(w, "w", torch.bfloat16)
        N = w.shape[0]
        if w.shape[1] != K:
            raise ValueError("w must be [N, K] with K = %d" % K)
        if out is None:
            out = torch.empty((M, N), dtype=out_dtype, device=a.device)
        _need(out, "out", out_dtype, (M, N))
        need = self.bi_matmul_workspace_bytes(M, N, K)
        if need and (ws is None or ws.numel() * ws.element_size() < need):
            ws = torch.empty(need, dtype=torch.uint8, device=a.device)
        nbytes = 0 if ws is None else ws.numel() * ws.element_size()
        self._check("bi_matmul", self.lib.bi_matmul(_ptr(a), _ptr(w), _ptr(out), M, N, K,
                                                    _DT[out_dtype], _ptr(ws), nbytes,
                                                    _stream(stream)))
        return out

    def bi_fold_norm_weight(self, W: torch.Tensor, w: torch.Tensor, out=None,
                            stream=None) -> torch.Tensor:
        """wf = round(W * w[None, :]) for W [N, K] and w [K] (bf16)."""
        _need(W, "W", torch.bfloat16)
        N, K = W.shape
        _need(w, "w", torch.bfloat16, (K,))
        if out is None:
            out = torch.empty_like(W)
        _need(out, "out", torch.bfloat16, (N, K))
        self._check("bi_fold_norm_weight",
                    self.lib.bi_fold_norm_weight(_ptr(W), _ptr(w), _ptr(out), N, K,
                                                 _stream(stream)))
        return out

    def bi_rmsnorm_matmul(self, x: torch.Tensor, wf: torch.Tensor, eps: float, out=None,
                          out_dtype=torch.bfloat16, ws=None, stream=None) -> torch.Tensor:
        """C = RMSNorm(x) @ wf.T; x [M, K], wf [N, K] the weight with the norm
        weight folded in (bi_fold_norm_weight).  `ws` (uint8, optional): the
        workspace for the M row statistics."""
        _need(x, "x", torch.bfloat16)
        M, K = x.shape
        _need(wf, "wf", torch.bfloat16)
        N = wf.shape[0]
        if wf.shape[1] != K:
            raise ValueError("wf must be [N, K] with K = %d" % K)
        if out is None:
            out = torch.empty((M, N), dtype=out_dtype, device=x.device)
        _need(out, "out", out_dtype, (M, N))
        ws = self._norm_ws(M, x.device, ws)
        self._check("bi_rmsnorm_matmul",
                    self.lib.bi_rmsnorm_matmul(_ptr(x), _ptr(wf), _ptr(out), M, N, K, float(eps),
                                               _DT[out_dtype], _ptr(ws), ws.numel(),
                                               _stream(stream)))
        return out

    def _norm_ws(self, M: int, device, ws=None) -> torch.Tensor:
        """The fused norm forms' workspace (M row statistics): the caller's
        `ws` if it is large enough, else a new one."""
        need = max(int(self.lib.bi_rmsnorm_matmul_workspace_bytes(M)), 16)
        if ws is None or ws.numel() * ws.element_size() < need:
            ws = torch.empty(need, dtype=torch.uint8, device=device)
        return ws

    def bi_matmul_residual(self, a: torch.Tensor, w: torch.Tensor, r: torch.Tensor, out=None,
                           stream=None) -> torch.Tensor:
        """C = round(r + round(a @ w.T)); a [M, K], w [N, K], r [M, N] (bf16).
        ``out`` may be ``r`` (in place); by default the result goes to a new
        tensor."""
        _need(a, "a", torch.bfloat16)
        M, K = a.shape
        _need(w, "w", torch.bfloat16)
        N = w.shape[0]
        if w.shape[1] != K:
            raise ValueError("w must be [N, K] with K = %d" % K)
        _need(r, "r", torch.bfloat16, (M, N))
        if out is None:
            out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
        _need(out, "out", torch.bfloat16, (M, N))
        self._check("bi_matmul_residual",
                    self.lib.bi_matmul_residual(_ptr(a), _ptr(w), _ptr(r), _ptr(out), M, N, K,
                                                _stream(stream)))
        return out

    def bi_matmul_grouped(self, a: torch.Tensor, w: torch.Tensor, offsets: torch.Tensor,
                          out=None, out_dtype=torch.bfloat16, stream=None) -> torch.Tensor:
        """Rows offsets[g]..offsets[g+1]-1 of a [rows, K] times w[g] ([G, N, K]
        bf16, stacked) -> c [rows, N]; offsets int64 [G + 1] on the device."""
        _need(a, "a", torch.bfloat16)
        rows, K = a.shape
        _need(w, "w", torch.bfloat16)
        G, N, K2 = w.shape
        if K2 != K:
            raise ValueError("w must be [groups, N, K] with K = %d" % K)
        _need(offsets, "offsets", torch.int64, (G + 1,))
        if out is None:
            out = torch.empty((rows, N), dtype=out_dtype, device=a.device)
        _need(out, "out", out_dtype, (rows, N))
        self._check("bi_matmul_grouped", self.lib.bi_matmul_grouped(
            _ptr(a), _ptr(w), _ptr(out), _ptr(offsets), G, rows, N, K, _DT[out_dtype],
            _stream(stream)))
        return out

    # ------------------------------------------------------------ KV cache
    def bi_kv_write(self, kv: PagedKV, k_new: torch.Tensor, v_new: torch.Tensor,
                    slot_mapping: torch.Tensor, stream=None) -> None:
        T = k_new.shape[0]
        shape = (T, kv.num_kv_heads, kv.head_dim)
        _need(k_new, "k_new", torch.bfloat16, shape)
        _need(v_new, "v_new", torch.bfloat16, shape)
        _need(slot_mapping, "slot_mapping", torch.int64, (T,))
        c = kv.c_struct()
        self._check("bi_kv_write", self.lib.bi_kv_write(ctypes.byref(c), _ptr(k_new), _ptr(v_new),
                                                        _ptr(slot_mapping), T, _stream(stream)))

    # ------------------------------------------------------------ decoder glue
    def bi_embedding(self, table: torch.Tensor, ids: torch.Tensor, out=None,
                     stream=None) -> torch.Tensor:
        """Rows ``table[ids]`` ([V, H] bf16, int32 ids [T]) -> [T, H]."""
        _need(table, "table", torch.bfloat16)
        V, H = table.shape
        _need(ids, "ids", torch.int32)
        T = ids.shape[0]
        if out is None:
            out = torch.empty((T, H), dtype=torch.bfloat16, device=table.device)
        _need(out, "out", torch.bfloat16, (T, H))
        self._check("bi_embedding", self.lib.bi_embedding(_ptr(table), V, H, _ptr(ids), _ptr(out),
                                                          T, _stream(stream)))
        return out

    def bi_rope_kv_write(self, kv: PagedKV, qkv: torch.Tensor, positions: torch.Tensor,
                         slot_mapping: torch.Tensor, Hq: int, theta: float = 10000.0,
                         q_out=None, stream=None) -> torch.Tensor:
        """Rotate q and k of ``qkv`` [T, (Hq + 2 Hkv) d]; k and v go to the
        cache at ``slot_mapping``; returns the rotated q [T, Hq, d]."""
        _need(qkv, "qkv", torch.bfloat16)
        T = qkv.shape[0]
        d, Hkv = kv.head_dim, kv.num_kv_heads
        _need(qkv, "qkv", torch.bfloat16, (T, (Hq + 2 * Hkv) * d))
        _need(positions, "positions", torch.int32, (T,))
        _need(slot_mapping, "slot_mapping", torch.int64, (T,))
        if q_out is None:
            q_out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device=qkv.device)
        _need(q_out, "q_out", torch.bfloat16, (T, Hq, d))
        c = kv.c_struct()
        self._check("bi_rope_kv_write", self.lib.bi_rope_kv_write(
            ctypes.byref(c), _ptr(qkv), _ptr(positions), _ptr(slot_mapping), _ptr(q_out), T, Hq,
            float(theta), _stream(stream)))
        return q_out

    def bi_rope_table(self, max_pos: int, head_dim: int, theta: float = 10000.0, device="cuda",
                      stream=None) -> torch.Tensor:
        """(cos, sin) of p theta^(-2i/d) as fp32 [max_pos, d/2, 2], the same floats
        bi_rope_kv_write evaluates."""
        table = torch.empty((max_pos, head_dim // 2, 2), dtype=torch.float32, device=device)
        self._check("bi_rope_table", self.lib.bi_rope_table(_ptr(table), int(max_pos),
                                                            int(head_dim), float(theta),
                                                            _stream(stream)))
        return table

    def bi_rmsnorm_matmul_rope_kv(self, x: torch.Tensor, wf: torch.Tensor, eps: float,
                                  kv: PagedKV, rope_table: torch.Tensor, positions: torch.Tensor,
                                  slot_mapping: torch.Tensor, Hq: int, q_out=None, ws=None,
                                  stream=None) -> torch.Tensor:
        """RMSNorm(x) @ wf.T, then RoPE and the cache write of k and v in the
        matmul's epilogue (bit for bit bi_rmsnorm_matmul + bi_rope_kv_write);
        returns the rotated q [T, Hq, d]."""
        _need(x, "x", torch.bfloat16)
        T, K = x.shape
        d, Hkv = kv.head_dim, kv.num_kv_heads
        _need(wf, "wf", torch.bfloat16, ((Hq + 2 * Hkv) * d, K))
        _need(rope_table, "rope_table", torch.float32)
        if rope_table.dim() != 3 or rope_table.shape[1:] != (d // 2, 2):
            raise ValueError("rope_table must be [max_pos, %d, 2]" % (d // 2))
        _need(positions, "positions", torch.int32, (T,))
        _need(slot_mapping, "slot_mapping", torch.int64, (T,))
        if q_out is None:
            q_out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device=x.device)
        _need(q_out, "q_out", torch.bfloat16, (T, Hq, d))
        c = kv.c_struct()
        ws = self._norm_ws(T, x.device, ws)
        self._check("bi_rmsnorm_matmul_rope_kv", self.lib.bi_rmsnorm_matmul_rope_kv(
            _ptr(x), _ptr(wf), float(eps), ctypes.byref(c), _ptr(rope_table),
            int(rope_table.shape[0]), _ptr(positions), _ptr(slot_mapping), _ptr(q_out), T, K, Hq,
            _ptr(ws), ws.numel(), _stream(stream)))
        return q_out

    # ------------------------------------------------------------ backward
    def bi_rmsnorm_backward(self, x: torch.Tensor, w: torch.Tensor, dy: torch.Tensor,
                            eps: float = 1e-6, out_dtype=torch.bfloat16, stream=None):
        """(dx [M, H], dw [H]) of y = RMSNorm(x) * w for the upstream gradient dy."""
        _need(x, "x", torch.bfloat16)
        M, H = x.shape
        _need(w, "w", torch.bfloat16, (H,))
        _need(dy, "dy", torch.bfloat16, (M, H))
        dx = torch.empty((M, H), dtype=out_dtype, device=x.device)
        dw = torch.empty((H,), dtype=out_dtype, device=x.device)
        need = int(self.lib.bi_rmsnorm_backward_workspace_bytes(M, H))
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
        self._check("bi_rmsnorm_backward", self.lib.bi_rmsnorm_backward(
            _ptr(x), _ptr(w), _ptr(dy), _ptr(dx), _ptr(dw), M, H, float(eps), _DT[out_dtype],
            _ptr(ws), ws.numel(), _stream(stream)))
        return dx, dw

    def bi_transpose(self, a: torch.Tensor, ld_out: int | None = None, stream=None) -> torch.Tensor:
        """a.T for bf16 a [R, C], as [C, ld_out] with the columns past R zero."""
        _need(a, "a", torch.bfloat16)
        R, C = a.shape
        ld = R if ld_out is None else int(ld_out)
        out = torch.empty((C, ld), dtype=torch.bfloat16, device=a.device)
        self._check("bi_transpose", self.lib.bi_transpose(_ptr(a), _ptr(out), R, C, ld,
                                                          _stream(stream)))
        return out

    def bi_matmul_backward(self, dc: torch.Tensor, a: torch.Tensor, w: torch.Tensor,
                           out_dtype=torch.bfloat16, want_da: bool = True, want_dw: bool = True,
                           stream=None):
        """(dA, dW) for C = a @ w.T: dA = dc @ w [M, K], dW = dc.T @ a [N, K]."""
        _need(dc, "dc", torch.bfloat16)
        M, N = dc.shape
        _need(a, "a", torch.bfloat16)
        K = a.shape[1]
        _need(a, "a", torch.bfloat16, (M, K))
        _need(w, "w", torch.bfloat16, (N, K))
        da = torch.empty((M, K), dtype=out_dtype, device=dc.device) if want_da else None
        dw = torch.empty((N, K), dtype=out_dtype, device=dc.device) if want_dw else None
        need = int(self.lib.bi_matmul_backward_workspace_bytes(M, N, K))
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dc.device)
        self._check("bi_matmul_backward", self.lib.bi_matmul_backward(
            _ptr(dc), _ptr(a), _ptr(w), _ptr(da), _ptr(dw), M, N, K, _DT[out_dtype], _ptr(ws),
            ws.numel(), _stream(stream)))
        return da, dw

    def bi_swiglu_backward(self, gu: torch.Tensor, dout: torch.Tensor, out=None,
                           out_dtype=torch.bfloat16, stream=None) -> torch.Tensor:
        """[dgate | dup] [T, 2F] of out = silu(gate) * up for the upstream dout [T, F]."""
        _need(gu, "gu", torch.bfloat16)
        T, F2 = gu.shape
        _need(dout, "dout", torch.bfloat16, (T, F2 // 2))
        if out is None:
            out = torch.empty((T, F2), dtype=out_dtype, device=gu.device)
        _need(out, "out", out_dtype, (T, F2))
        self._check("bi_swiglu_backward", self.lib.bi_swiglu_backward(
            _ptr(gu), _ptr(dout), _ptr(out), T, F2 // 2, _DT[out_dtype], _stream(stream)))
        return out

    def bi_rope_backward(self, dy: torch.Tensor, positions: torch.Tensor, theta: float = 10000.0,
                         out=None, out_dtype=torch.bfloat16, stream=None) -> torch.Tensor:
        """Gradient of the rotary rotation's input for the upstream dy [T, nh, d]
        (dy and out may be column slices of wider rows, e.g. of a q/k/v gradient)."""
        if dy.dtype != torch.bfloat16 or dy.dim() != 3 or dy.stride(2) != 1 or \
                dy.stride(1) != dy.shape[2] or not dy.is_cuda:
            raise ValueError("dy: bf16 [T, nh, d] with dense heads")
        T, nh, d = dy.shape
        _need(positions, "positions", torch.int32, (T,))
        if out is None:
            out = torch.empty((T, nh, d), dtype=out_dtype, device=dy.device)
        if out.dtype != out_dtype or tuple(out.shape) != (T, nh, d) or out.stride(2) != 1 or \
                out.stride(1) != d:
            raise ValueError("out: [T, nh, d] of out_dtype with dense heads")
        self._check("bi_rope_backward", self.lib.bi_rope_backward(
            ctypes.c_void_p(dy.data_ptr()), dy.stride(0), _ptr(positions),
            ctypes.c_void_p(out.data_ptr()), out.stride(0), T, nh, d, float(theta),
            _DT[out_dtype], _stream(stream)))
        return out

    def bi_swiglu(self, gu: torch.Tensor, out=None, stream=None) -> torch.Tensor:
        """silu(gate) * up of gu [T, 2F] = [gate | up] -> [T, F]."""
        _need(gu, "gu", torch.bfloat16)
        T, F2 = gu.shape
        if out is None:
            out = torch.empty((T, F2 // 2), dtype=torch.bfloat16, device=gu.device)
        _need(out, "out", torch.bfloat16, (T, F2 // 2))
        self._check("bi_swiglu", self.lib.bi_swiglu(_ptr(gu), _ptr(out), T, F2 // 2,
                                                    _stream(stream)))
        return out

    def bi_argmax(self, logits: torch.Tensor, out=None, stream=None) -> torch.Tensor:
        """Lowest index of each row's maximum; logits [T, V] fp32 -> int32 [T]."""
        _need(logits, "logits", torch.float32)
        T, V = logits.shape
        if out is None:
            out = torch.empty((T,), dtype=torch.int32, device=logits.device)
        _need(out, "out", torch.int32, (T,))
        self._check("bi_argmax", self.lib.bi_argmax(_ptr(logits), T, V, _ptr(out),
                                                    _stream(stream)))
        return out

    def bi_sample(self, logits: torch.Tensor, temperature, top_p, seed, offset, out=None,
                  stream=None) -> torch.Tensor:
        """One token per row of fp32 logits [T, V]; temperature, top_p (fp32),
        seed and offset (int64/uint64 bit patterns) are per-row tensors [T]
        on the device, or Python scalars broadcast to every row."""
        _need(logits, "logits", torch.float32)
        T, V = logits.shape
        dev = logits.device

        def col(x, dtype, name):
            if not isinstance(x, torch.Tensor):
                x = torch.full((T,), x, dtype=dtype, device=dev)
            _need(x, name, dtype, (T,))
            return x

        temperature = col(temperature, torch.float32, "temperature")
        top_p = col(top_p, torch.float32, "top_p")
        seed = col(seed, torch.int64, "seed")        # uint64 bits
        offset = col(offset, torch.int64, "offset")
        if out is None:
            out = torch.empty((T,), dtype=torch.int32, device=dev)
        _need(out, "out", torch.int32, (T,))
        self._check("bi_sample", self.lib.bi_sample(
            _ptr(logits), T, V, _ptr(temperature), _ptr(top_p), _ptr(seed), _ptr(offset), _ptr(out),
            _stream(stream)))
        return out

    # ------------------------------------------------------------ mixture of experts
    def bi_moe_route(self, logits: torch.Tensor, k: int, stream=None):
        """(experts int32 [T, k], weights fp32 [T, k]) from fp32 router logits [T, E]."""
        _need(logits, "logits", torch.float32)
        T, E = logits.shape
        ex = torch.empty((T, k), dtype=torch.int32, device=logits.device)
        w = torch.empty((T, k), dtype=torch.float32, device=logits.device)
        self._check("bi_moe_route", self.lib.bi_moe_route(_ptr(logits), T, E, k, _ptr(ex), _ptr(w),
                                                          _stream(stream)))
        return ex, w

    def bi_moe_dispatch(self, experts: torch.Tensor, E: int, stream=None):
        """(offsets [E+1], order [T*k], pos [T*k], token_sorted [T*k]) grouping by expert."""
        _need(experts, "experts", torch.int32)
        T, k = experts.shape
        dev = experts.device
        off = torch.empty((E + 1,), dtype=torch.int64, device=dev)
        order = torch.empty((T * k,), dtype=torch.int64, device=dev)
        pos = torch.empty((T * k,), dtype=torch.int64, device=dev)
        tok = torch.empty((T * k,), dtype=torch.int32, device=dev)
        self._check("bi_moe_dispatch", self.lib.bi_moe_dispatch(
            _ptr(experts), T, k, E, _ptr(off), _ptr(order), _ptr(pos), _ptr(tok), _stream(stream)))
        return off, order, pos, tok

    def bi_moe_combine(self, y: torch.Tensor, pos: torch.Tensor, weights: torch.Tensor, out=None,
                       stream=None) -> torch.Tensor:
        """Gate-weighted sum in rank order: y [T*k, H] bf16 (dispatch order) -> [T, H]."""
        _need(weights, "weights", torch.float32)
        T, k = weights.shape
        _need(y, "y", torch.bfloat16)
        H = y.shape[1]
        _need(y, "y", torch.bfloat16, (T * k, H))
        _need(pos, "pos", torch.int64, (T * k,))
        if out is None:
            out = torch.empty((T, H), dtype=torch.bfloat16, device=y.device)
        _need(out, "out", torch.bfloat16, (T, H))
        self._check("bi_moe_combine", self.lib.bi_moe_combine(
            _ptr(y), _ptr(pos), _ptr(weights), T, k, H, _ptr(out), _stream(stream)))
        return out

    # ------------------------------------------------------------ attention
    def bi_attention_decode_workspace_bytes(self, kv: PagedKV, B: int, Hq: int, max_seq_len: int,
                                            splits_per_cta: int = 0) -> int:
        c = kv.c_struct()
        return int(self.lib.bi_attention_decode_workspace_bytes(ctypes.byref(c), B, Hq,
                                                                max_seq_len, splits_per_cta))

    def bi_attention_decode(self, kv: PagedKV, q: torch.Tensor, seq_lens: torch.Tensor,
                            max_seq_len: int, scale: float | None = None, want_lse: bool = False,
                            splits_per_cta: int = 0, out=None, lse=None, ws=None, stream=None):
        """One query token per sequence: q [B, Hq, d] -> o [B, Hq, d] (and lse [B, Hq])."""
        _need(q, "q", torch.bfloat16)
        B, Hq, d = q.shape
        _need(seq_lens, "seq_lens", torch.int32, (B,))
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        if out is None:
            out = torch.empty_like(q)
        _need(out, "out", torch.bfloat16, (B, Hq, d))
        if want_lse and lse is None:
            lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        if lse is not None:
            _need(lse, "lse", torch.float32, (B, Hq))
        c = kv.c_struct()
        need = int(self.lib.bi_attention_decode_workspace_bytes(ctypes.byref(c), B, Hq,
                                                                max_seq_len, splits_per_cta))
        if need and (ws is None or ws.numel() * ws.element_size() < need):
            ws = torch.empty(need, dtype=torch.uint8, device=q.device)
        nbytes = 0 if ws is None else ws.numel() * ws.element_size()
        self._check("bi_attention_decode", self.lib.bi_attention_decode(
            ctypes.byref(c), _ptr(q), _ptr(out), _ptr(lse), _ptr(seq_lens), B, Hq,
            int(max_seq_len), float(scale), int(splits_per_cta), _ptr(ws), nbytes,
            _stream(stream)))
        return (out, lse) if want_lse else out

    def bi_attention_decode_noalloc(self, kv: PagedKV, q: torch.Tensor, seq_lens: torch.Tensor,
                                    max_seq_len: int, scale: float | None = None,
                                    want_lse: bool = False, splits_per_cta: int = 0, out=None,
                                    lse=None, stream=None):
        """bi_attention_decode with its scratch in the library's fixed array
        (no workspace, no device allocation by the library).  `out` and
        `lse` are the caller's; pass them to avoid any allocation here."""
        _need(q, "q", torch.bfloat16)
        B, Hq, d = q.shape
        _need(seq_lens, "seq_lens", torch.int32, (B,))
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        if out is None:
            out = torch.empty_like(q)
        _need(out, "out", torch.bfloat16, (B, Hq, d))
        if want_lse and lse is None:
            lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        if lse is not None:
            _need(lse, "lse", torch.float32, (B, Hq))
        c = kv.c_struct()
        self._check("bi_attention_decode_noalloc", self.lib.bi_attention_decode_noalloc(
            ctypes.byref(c), _ptr(q), _ptr(out), _ptr(lse), _ptr(seq_lens), B, Hq,
            int(max_seq_len), float(scale), int(splits_per_cta), _stream(stream)))
        return (out, lse) if want_lse else out

    def bi_attention_backward(self, kv: PagedKV, q: torch.Tensor, o: torch.Tensor,
                              dout: torch.Tensor, lse: torch.Tensor, cu_q: torch.Tensor,
                              ctx_lens: torch.Tensor, max_q_len: int, max_kv_len: int,
                              scale: float | None = None, dk=None, dv=None, stream=None):
        """(dq [T, Hq, d], dk, dv) of bi_attention_prefill's output o (with its
        lse) for the upstream gradient dout.  dk and dv are shaped like the
        caches; they start as zeros unless given (pages no sequence of the
        call owns are not written)."""
        _need(q, "q", torch.bfloat16)
        T, Hq, d = q.shape
        B = ctx_lens.shape[0]
        _need(o, "o", torch.bfloat16, (T, Hq, d))
        _need(dout, "dout", torch.bfloat16, (T, Hq, d))
        _need(lse, "lse", torch.float32, (T, Hq))
        _need(cu_q, "cu_q", torch.int32, (B + 1,))
        _need(ctx_lens, "ctx_lens", torch.int32, (B,))
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        dq = torch.empty_like(q)
        if dk is None:
            dk = torch.zeros_like(kv.k_cache)
        if dv is None:
            dv = torch.zeros_like(kv.v_cache)
        _need(dk, "dk", torch.bfloat16, tuple(kv.k_cache.shape))
        _need(dv, "dv", torch.bfloat16, tuple(kv.v_cache.shape))
        need = int(self.lib.bi_attention_backward_workspace_bytes(Hq, T))
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
        c = kv.c_struct()
        self._check("bi_attention_backward", self.lib.bi_attention_backward(
            ctypes.byref(c), _ptr(q), _ptr(o), _ptr(dout), _ptr(lse), _ptr(cu_q), _ptr(ctx_lens),
            B, Hq, T, int(max_q_len), int(max_kv_len), float(scale), _ptr(dq), _ptr(dk), _ptr(dv),
            _ptr(ws), ws.numel(), _stream(stream)))
        return dq, dk, dv

    def bi_attention_prefill(self, kv: PagedKV, q: torch.Tensor, cu_q: torch.Tensor,
                             ctx_lens: torch.Tensor, max_q_len: int, scale: float | None = None,
                             want_lse: bool = False, out=None, lse=None, stream=None):
        """Causal prompt chunks: q [T_total, Hq, d] packed by cu_q -> o (and lse [T_total, Hq])."""
        _need(q, "q", torch.bfloat16)
        T, Hq, d = q.shape
        B = ctx_lens.shape[0]
        _need(cu_q, "cu_q", torch.int32, (B + 1,))
        _need(ctx_lens, "ctx_lens", torch.int32, (B,))
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        if out is None:
            out = torch.empty_like(q)
        _need(out, "out", torch.bfloat16, (T, Hq, d))
        if want_lse and lse is None:
            lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
        if lse is not None:
            _need(lse, "lse", torch.float32, (T, Hq))
        c = kv.c_struct()
        self._check("bi_attention_prefill", self.lib.bi_attention_prefill(
            ctypes.byref(c), _ptr(q), _ptr(out), _ptr(lse), _ptr(cu_q), _ptr(ctx_lens), B, Hq, T,
            int(max_q_len), float(scale), None, 0, _stream(stream)))
        return (out, lse) if want_lse else out


_LIBS: dict = {}


def load(variant: bool = False) -> Library:
    """The invariant library (default) or the variant-off build."""
    name = "libbi_variant.so" if variant else "libbi.so"
    if name not in _LIBS:
        _LIBS[name] = Library(os.path.join(LIBDIR, name))
    return _LIBS[name]
