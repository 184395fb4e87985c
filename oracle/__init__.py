"""fp64 CPU oracle for the batch-invariant forward path (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path never does.

The arithmetic lives in ``oracle.c`` (plain C, fp64); this module compiles it
with gcc (OpenMP over independent rows) and marshals numpy arrays into it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile ``oracle.c`` (or another copy of it) into a shared library
    with gcc -O2 -fopenmp."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".tmp%d" % os.getpid()
        # -ffp-contract=off: no fused multiply-add, so every product and sum
        # rounds exactly as written in the source.
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", src, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bfloat16 inputs are passed as uint16 bit patterns"
    return a


class Oracle:
    """The oracle's entry points, bound to one build of ``oracle.c``."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        lib.oracle_rmsnorm.argtypes = [P, P, i64, i64, f64, P]
        lib.oracle_matmul.argtypes = [P, P, i64, i64, i64, P]
        lib.oracle_kv_write.argtypes = [P, P, i32, i32, P, P, P, i64]
        lib.oracle_attention.argtypes = [P, i64, i32, P, P, P, i32, P, P, i32, P, i32, f64, P, P]
        lib.oracle_embedding.argtypes = [P, i64, i64, P, i64, P]
        lib.oracle_rope.argtypes = [P, i64, i32, i32, P, f64, P]
        lib.oracle_swiglu.argtypes = [P, i64, i64, P]
        lib.oracle_add_rmsnorm.argtypes = [P, P, P, i64, i64, f64, P, P]
        lib.oracle_argmax.argtypes = [P, i64, i64, P]
        lib.oracle_philox4x32_10.argtypes = [P, P, P]
        lib.oracle_sample.argtypes = [P, i64, i64, P, P, P, P, P, P, P]
        lib.oracle_moe_route.argtypes = [P, i64, i32, i32, P, P]
        lib.oracle_moe_dispatch.argtypes = [P, i64, i32, P, P, P]
        lib.oracle_moe_combine.argtypes = [P, P, P, i64, i32, i64, P]
        lib.oracle_fold_norm_weight.argtypes = [P, P, i64, i64, P]
        lib.oracle_rmsnorm_matmul.argtypes = [P, P, i64, i64, i64, f64, P]
        lib.oracle_matmul_residual.argtypes = [P, P, P, i64, i64, i64, P]
        lib.oracle_rope_angles.argtypes = [i32, i32, f64, P]
        lib.oracle_rmsnorm_backward.argtypes = [P, P, P, i64, i64, f64, P, P]
        lib.oracle_swiglu_backward.argtypes = [P, P, i64, i64, P]
        lib.oracle_rope_backward.argtypes = [P, i64, i32, i32, P, f64, P]
        lib.oracle_attention_backward.argtypes = [P, P, i64, i32, P, P, P, i32, P, P, i32, i32,
                                                  P, i32, f64, P, P, P]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        self.lib = lib

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(int(n))

    def rmsnorm(self, x, w, eps: float) -> np.ndarray:
        """y = x / sqrt(mean(x^2) + eps) * w per row; x [M, H], w [H] (bf16 bits)."""
        x, w = _u16(x), _u16(w)
        M, H = x.shape
        y = np.empty((M, H), dtype=np.float64)
        self.lib.oracle_rmsnorm(_p(x), _p(w), M, H, float(eps), _p(y))
        return y

    def matmul(self, a, w) -> np.ndarray:
        """C = A @ W.T; a [M, K], w [N, K] (bf16 bits) -> C [M, N] float64."""
        a, w = _u16(a), _u16(w)
        M, K = a.shape
        N, K2 = w.shape
        assert K == K2
        c = np.empty((M, N), dtype=np.float64)
        self.lib.oracle_matmul(_p(a), _p(w), M, N, K, _p(c))
        return c

    def kv_write(self, k_cache, v_cache, k_new, v_new, slots) -> None:
        """Scatter new tokens into the paged cache in place (bit copy)."""
        k_cache, v_cache = _u16(k_cache), _u16(v_cache)
        k_new, v_new = _u16(k_new), _u16(v_new)
        slots = np.ascontiguousarray(slots, dtype=np.int64)
        _, Hkv, page, d = k_cache.shape
        assert page == 16
        T = k_new.shape[0]
        self.lib.oracle_kv_write(_p(k_cache), _p(v_cache), Hkv, d, _p(k_new), _p(v_new),
                                 _p(slots), T)

    def attention(self, q_rows, row_seq, row_head, row_pos, Hq: int, k_cache, v_cache,
                  block_table, scale: float | None = None, want_lse: bool = False):
        """Causal softmax attention of query rows over a paged cache.

        ``q_rows`` [R, d] bf16 bits; row r is head ``row_head[r]`` of sequence
        ``row_seq[r]`` at absolute position ``row_pos[r]`` (it sees keys
        ``0..row_pos[r]``).  Returns ``o`` [R, d] float64 (and ``lse`` [R]).
        """
        q_rows = _u16(q_rows)
        k_cache, v_cache = _u16(k_cache), _u16(v_cache)
        R, d = q_rows.shape
        _, Hkv, page, d2 = k_cache.shape
        assert page == 16 and d2 == d and Hq % Hkv == 0
        bt = np.ascontiguousarray(block_table, dtype=np.int32)
        rs = np.ascontiguousarray(row_seq, dtype=np.int32)
        rh = np.ascontiguousarray(row_head, dtype=np.int32)
        rp = np.ascontiguousarray(row_pos, dtype=np.int32)
        assert rs.shape == rh.shape == rp.shape == (R,)
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        o = np.empty((R, d), dtype=np.float64)
        lse = np.empty((R,), dtype=np.float64)
        self.lib.oracle_attention(_p(q_rows), R, d, _p(rs), _p(rh), _p(rp), Hq, _p(k_cache),
                                  _p(v_cache), Hkv, _p(bt), bt.shape[1], float(scale), _p(o),
                                  _p(lse))
        return (o, lse) if want_lse else o

    # ---------------------------------------------------------- decoder glue

    def embedding(self, table, ids) -> np.ndarray:
        """Rows of ``table`` [V, H] (bf16 bits) at ``ids`` [T] -> [T, H] bits."""
        table = _u16(table)
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        V, H = table.shape
        out = np.zeros((ids.shape[0], H), dtype=np.uint16)
        self.lib.oracle_embedding(_p(table), V, H, _p(ids), ids.shape[0], _p(out))
        return out

    def rope(self, x, pos, theta: float = 10000.0) -> np.ndarray:
        """Rotary embedding (rotate-half pairs) of x [T, nh, d] at positions
        ``pos`` [T] -> float64 [T, nh, d]."""
        x = _u16(x)
        T, nh, d = x.shape
        pos = np.ascontiguousarray(pos, dtype=np.int32)
        assert pos.shape == (T,) and d % 2 == 0
        out = np.empty((T, nh, d), dtype=np.float64)
        self.lib.oracle_rope(_p(x), T, nh, d, _p(pos), float(theta), _p(out))
        return out

    def rope_angles(self, P: int, d: int, theta: float = 10000.0) -> np.ndarray:
        """(cos, sin) of p * theta^(-2i/d) -> float64 [P, d/2, 2]."""
        out = np.empty((P, d // 2, 2), dtype=np.float64)
        self.lib.oracle_rope_angles(int(P), int(d), float(theta), _p(out))
        return out

    def swiglu(self, gu) -> np.ndarray:
        """silu(gate) * up of gu [T, 2F] = [gate | up] -> float64 [T, F]."""
        gu = _u16(gu)
        T, F2 = gu.shape
        assert F2 % 2 == 0
        out = np.empty((T, F2 // 2), dtype=np.float64)
        self.lib.oracle_swiglu(_p(gu), T, F2 // 2, _p(out))
        return out

    def add_rmsnorm(self, x, delta, w, eps: float):
        """(s, y): s = x + delta, y = RMSNorm(s) * w, all rows; float64."""
        x, delta, w = _u16(x), _u16(delta), _u16(w)
        M, H = x.shape
        assert delta.shape == (M, H) and w.shape == (H,)
        s = np.empty((M, H), dtype=np.float64)
        y = np.empty((M, H), dtype=np.float64)
        self.lib.oracle_add_rmsnorm(_p(x), _p(delta), _p(w), M, H, float(eps), _p(s), _p(y))
        return s, y

    def argmax(self, logits) -> np.ndarray:
        """Lowest index of each row's maximum; logits [T, V] float32."""
        logits = np.ascontiguousarray(logits, dtype=np.float32)
        T, V = logits.shape
        out = np.empty((T,), dtype=np.int32)
        self.lib.oracle_argmax(_p(logits), T, V, _p(out))
        return out

    # ---------------------------------------------------------- sampling

    def philox4x32_10(self, ctr, key) -> np.ndarray:
        """Philox4x32-10 of a 4-word counter and a 2-word key -> 4 words."""
        c = np.ascontiguousarray(ctr, dtype=np.uint32)
        k = np.ascontiguousarray(key, dtype=np.uint32)
        assert c.shape == (4,) and k.shape == (2,)
        out = np.empty(4, dtype=np.uint32)
        self.lib.oracle_philox4x32_10(_p(c), _p(k), _p(out))
        return out

    def sample(self, logits, temperature, top_p, seed, offset, details: bool = False):
        """One token per row of fp32 logits [T, V] (temperature 0: greedy;
        else softmax at that temperature, nucleus top_p, the draw from
        Philox4x32-10 keyed by the row's seed at counter ``offset``).
        With ``details``, also (r, zk): the draw and the kept mass as
        fractions of the total weight."""
        logits = np.ascontiguousarray(logits, dtype=np.float32)
        T, V = logits.shape
        temp = np.ascontiguousarray(np.broadcast_to(temperature, (T,)), dtype=np.float32)
        tp = np.ascontiguousarray(np.broadcast_to(top_p, (T,)), dtype=np.float32)
        sd = np.ascontiguousarray(np.broadcast_to(seed, (T,)), dtype=np.uint64)
        off = np.ascontiguousarray(np.broadcast_to(offset, (T,)), dtype=np.uint64)
        out = np.empty((T,), dtype=np.int32)
        r = np.empty((T,), dtype=np.float64)
        zk = np.empty((T,), dtype=np.float64)
        self.lib.oracle_sample(_p(logits), T, V, _p(temp), _p(tp), _p(sd), _p(off), _p(out),
                               _p(r), _p(zk))
        return (out, r, zk) if details else out

    # ---------------------------------------------------------- mixture of experts

    def moe_route(self, logits, k: int):
        """(experts [T, k] int32, weights [T, k] float64) from fp32 router logits [T, E]."""
        logits = np.ascontiguousarray(logits, dtype=np.float32)
        T, E = logits.shape
        ex = np.empty((T, k), dtype=np.int32)
        w = np.empty((T, k), dtype=np.float64)
        self.lib.oracle_moe_route(_p(logits), T, E, k, _p(ex), _p(w))
        return ex, w

    def moe_dispatch(self, experts, E: int):
        """(offsets [E+1], order [N], pos [N]) grouping the flat entries by expert."""
        ex = np.ascontiguousarray(experts, dtype=np.int32).ravel()
        N = ex.shape[0]
        off = np.empty(E + 1, dtype=np.int64)
        order = np.empty(N, dtype=np.int64)
        pos = np.empty(N, dtype=np.int64)
        self.lib.oracle_moe_dispatch(_p(ex), N, E, _p(off), _p(order), _p(pos))
        return off, order, pos

    def moe_combine(self, y, pos, weights) -> np.ndarray:
        """Gate-weighted sum of each token's expert rows; y [N, H] bf16 bits."""
        y = _u16(y)
        w = np.ascontiguousarray(weights, dtype=np.float64)
        T, k = w.shape
        ps = np.ascontiguousarray(pos, dtype=np.int64)
        H = y.shape[1]
        out = np.empty((T, H), dtype=np.float64)
        self.lib.oracle_moe_combine(_p(y), _p(ps), _p(w), T, k, H, _p(out))
        return out

    # ---------------------------------------------------------- backward

    def rmsnorm_backward(self, x, w, dy, eps: float):
        """(dx [M, H], dw [H]) of y = RMSNorm(x) * w for upstream dy; float64."""
        x, w, dy = _u16(x), _u16(w), _u16(dy)
        M, H = x.shape
        assert w.shape == (H,) and dy.shape == (M, H)
        dx = np.empty((M, H), dtype=np.float64)
        dw = np.empty((H,), dtype=np.float64)
        self.lib.oracle_rmsnorm_backward(_p(x), _p(w), _p(dy), M, H, float(eps), _p(dx), _p(dw))
        return dx, dw

    def swiglu_backward(self, gu, dout) -> np.ndarray:
        """[dgate | dup] [T, 2F] of swiglu for the upstream gradient dout [T, F]."""
        gu, dout = _u16(gu), _u16(dout)
        T, F2 = gu.shape
        assert dout.shape == (T, F2 // 2)
        out = np.empty((T, F2), dtype=np.float64)
        self.lib.oracle_swiglu_backward(_p(gu), _p(dout), T, F2 // 2, _p(out))
        return out

    def rope_backward(self, dy, pos, theta: float = 10000.0) -> np.ndarray:
        """Gradient of rope's input for the upstream gradient dy [T, nh, d]."""
        dy = _u16(dy)
        T, nh, d = dy.shape
        pos = np.ascontiguousarray(pos, dtype=np.int32)
        out = np.empty((T, nh, d), dtype=np.float64)
        self.lib.oracle_rope_backward(_p(dy), T, nh, d, _p(pos), float(theta), _p(out))
        return out

    def attention_backward(self, q_rows, dout_rows, row_seq, row_head, row_pos, Hq: int,
                           k_cache, v_cache, block_table, scale: float | None = None):
        """(dq [R, d], dk, dv [num_pages, Hkv, 16, d]) of ``attention`` for the
        upstream gradients ``dout_rows`` [R, d] (bf16 bits); float64."""
        q_rows, dout_rows = _u16(q_rows), _u16(dout_rows)
        k_cache, v_cache = _u16(k_cache), _u16(v_cache)
        R, d = q_rows.shape
        num_pages, Hkv, page, d2 = k_cache.shape
        assert page == 16 and d2 == d and Hq % Hkv == 0 and dout_rows.shape == (R, d)
        bt = np.ascontiguousarray(block_table, dtype=np.int32)
        rs = np.ascontiguousarray(row_seq, dtype=np.int32)
        rh = np.ascontiguousarray(row_head, dtype=np.int32)
        rp = np.ascontiguousarray(row_pos, dtype=np.int32)
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        dq = np.empty((R, d), dtype=np.float64)
        dk = np.empty(k_cache.shape, dtype=np.float64)
        dv = np.empty(k_cache.shape, dtype=np.float64)
        self.lib.oracle_attention_backward(_p(q_rows), _p(dout_rows), R, d, _p(rs), _p(rh),
                                           _p(rp), Hq, _p(k_cache), _p(v_cache), Hkv, num_pages,
                                           _p(bt), bt.shape[1], float(scale), _p(dq), _p(dk),
                                           _p(dv))
        return dq, dk, dv

    # ---------------------------------------------------------- fused matmuls

    def fold_norm_weight(self, W, w) -> np.ndarray:
        """wf[n, k] = W[n, k] * w[k]; W [N, K], w [K] (bf16 bits) -> float64."""
        W, w = _u16(W), _u16(w)
        N, K = W.shape
        assert w.shape == (K,)
        out = np.empty((N, K), dtype=np.float64)
        self.lib.oracle_fold_norm_weight(_p(W), _p(w), N, K, _p(out))
        return out

    def rmsnorm_matmul(self, x, wf, eps: float) -> np.ndarray:
        """C = RMSNorm(x) @ wf.T with the norm weight already in wf; x [M, K],
        wf [N, K] (bf16 bits) -> float64 [M, N]."""
        x, wf = _u16(x), _u16(wf)
        M, K = x.shape
        N, K2 = wf.shape
        assert K == K2
        c = np.empty((M, N), dtype=np.float64)
        self.lib.oracle_rmsnorm_matmul(_p(x), _p(wf), M, N, K, float(eps), _p(c))
        return c

    def matmul_residual(self, r, a, w) -> np.ndarray:
        """C = R + A @ W.T; r [M, N], a [M, K], w [N, K] (bf16 bits) -> float64."""
        r, a, w = _u16(r), _u16(a), _u16(w)
        M, K = a.shape
        N, K2 = w.shape
        assert K == K2 and r.shape == (M, N)
        c = np.empty((M, N), dtype=np.float64)
        self.lib.oracle_matmul_residual(_p(r), _p(a), _p(w), M, N, K, _p(c))
        return c


def default() -> Oracle:
    global _lib
    if _lib is None:
        _lib = Oracle(build())
    return _lib


def num_threads() -> int:
    return default().num_threads()


def set_num_threads(n: int) -> None:
    default().set_num_threads(n)


def rmsnorm(x, w, eps: float) -> np.ndarray:
    return default().rmsnorm(x, w, eps)


def matmul(a, w) -> np.ndarray:
    return default().matmul(a, w)


def kv_write(k_cache, v_cache, k_new, v_new, slots) -> None:
    default().kv_write(k_cache, v_cache, k_new, v_new, slots)


def attention(q_rows, row_seq, row_head, row_pos, Hq: int, k_cache, v_cache, block_table,
              scale: float | None = None, want_lse: bool = False):
    return default().attention(q_rows, row_seq, row_head, row_pos, Hq, k_cache, v_cache,
                               block_table, scale=scale, want_lse=want_lse)


def embedding(table, ids) -> np.ndarray:
    return default().embedding(table, ids)


def rope(x, pos, theta: float = 10000.0) -> np.ndarray:
    return default().rope(x, pos, theta)


def rope_angles(P: int, d: int, theta: float = 10000.0) -> np.ndarray:
    return default().rope_angles(P, d, theta)


def swiglu(gu) -> np.ndarray:
    return default().swiglu(gu)


def add_rmsnorm(x, delta, w, eps: float):
    return default().add_rmsnorm(x, delta, w, eps)


def argmax(logits) -> np.ndarray:
    return default().argmax(logits)


def philox4x32_10(ctr, key) -> np.ndarray:
    return default().philox4x32_10(ctr, key)


def sample(logits, temperature, top_p, seed, offset, details: bool = False):
    return default().sample(logits, temperature, top_p, seed, offset, details)


def moe_route(logits, k: int):
    return default().moe_route(logits, k)


def moe_dispatch(experts, E: int):
    return default().moe_dispatch(experts, E)


def moe_combine(y, pos, weights) -> np.ndarray:
    return default().moe_combine(y, pos, weights)


def fold_norm_weight(W, w) -> np.ndarray:
    return default().fold_norm_weight(W, w)


def rmsnorm_backward(x, w, dy, eps: float):
    return default().rmsnorm_backward(x, w, dy, eps)


def swiglu_backward(gu, dout) -> np.ndarray:
    return default().swiglu_backward(gu, dout)


def rope_backward(dy, pos, theta: float = 10000.0) -> np.ndarray:
    return default().rope_backward(dy, pos, theta)


def attention_backward(q_rows, dout_rows, row_seq, row_head, row_pos, Hq: int, k_cache,
                       v_cache, block_table, scale: float | None = None):
    return default().attention_backward(q_rows, dout_rows, row_seq, row_head, row_pos, Hq,
                                        k_cache, v_cache, block_table, scale)


def rmsnorm_matmul(x, wf, eps: float) -> np.ndarray:
    return default().rmsnorm_matmul(x, wf, eps)


def matmul_residual(r, a, w) -> np.ndarray:
    return default().matmul_residual(r, a, w)


def decode_rows(q, seq_lens, heads=None):
    """Rows for a decode step: every head of every request at position L-1.
    ``q`` [B, Hq, d].  Returns (q_rows, row_seq, row_head, row_pos)."""
    B, Hq, d = q.shape
    heads = range(Hq) if heads is None else heads
    heads = list(heads)
    rs, rh, rp, rows = [], [], [], []
    for b in range(B):
        for h in heads:
            rs.append(b)
            rh.append(h)
            rp.append(int(seq_lens[b]) - 1)
            rows.append(q[b, h])
    return np.stack(rows), np.array(rs), np.array(rh), np.array(rp)
