"""CPU oracle for the MoE layer forward -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package.  The library path never touches it: the CUDA path and the oracle
share no code.  The arithmetic lives in ``moe_oracle.c`` (plain C, IEEE double,
plain loops); this module compiles it with gcc and wraps it with numpy.

Every function cites the passage it follows in the C source.  Inputs are numpy
arrays: bf16 tensors are passed as their uint16 bit patterns (dtype code 0),
fp32 tensors as float32 (dtype code 1).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

BF16, FP32 = 0, 1


def build(force: bool = False) -> str:
    """Compile liboracle.so from moe_oracle.c (gcc, OpenMP)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        L.oracle_router_logits.argtypes = [i, i, i, i, P, P, P]
        L.oracle_topk.argtypes = [i, i, i, P, P]
        L.oracle_topk_k.argtypes = [i, i, i, P, P, P]
        L.oracle_topk_k.restype = ctypes.c_int
        L.oracle_gate_weights.argtypes = [i, i, i, i, i, P, P, P]
        L.oracle_align.argtypes = [i, i, i, i, i, P, ctypes.c_int64, P, P, P, P, P, P, P]
        L.oracle_swiglu_ffn.argtypes = [i, i, i, P, P, P, P]
        L.oracle_permute.argtypes = [i, i, i, P, P, i, P]
        L.oracle_combine.argtypes = [i, i, i, i, P, P, P, P, P]
        L.oracle_dense_ffn.argtypes = [i, i, i, i, P, P, P, P, i]
        L.oracle_moe_layer.argtypes = [i, i, i, i, i, i, i, i, i, P, P, P, P, P, P, P, P, P, i, P, P, P, i]
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_quantize_fp8.argtypes = [i, i, i, P, P, P]
        L.oracle_quantize_fp8.restype = ctypes.c_int
        L.oracle_moe_layer_fp8.argtypes = [i, i, i, i, i, i, i, i, i, P, P, P, P, P, P, P, P, P, P, P, P, P, i,
                                           P, i]
        L.oracle_moe_layer_fp8.restype = ctypes.c_int
        for f in (L.oracle_router_logits, L.oracle_topk, L.oracle_gate_weights, L.oracle_align,
                  L.oracle_swiglu_ffn, L.oracle_dense_ffn, L.oracle_moe_layer, L.oracle_permute,
                  L.oracle_combine):
            f.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _typed(a):
    """Return (contiguous array, dtype code) for a bf16-as-uint16 or fp32 array."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return a, BF16
    if a.dtype == np.float32:
        return a, FP32
    raise TypeError(f"oracle inputs are uint16 (bf16 bits) or float32, got {a.dtype}")


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its input (rc={rc})")


def nthreads_default() -> int:
    return max(1, os.cpu_count() or 1)


def router_logits(x, w_r):
    """logits[T,E] (float64) = x . W_r^T."""
    x, dt = _typed(x)
    w_r, dt2 = _typed(w_r)
    assert dt == dt2
    T, H = x.shape
    E = w_r.shape[0]
    out = np.empty((T, E), np.float64)
    _check(lib().oracle_router_logits(T, H, E, dt, _ptr(x), _ptr(w_r), _ptr(out)), "router_logits")
    return out


def topk(logits, K, k=None):
    """ids[T,K] int32: K largest fp32 logits per token, lower index on ties.
    With k (int32 [T], 0 <= k[t] <= K) token t takes its k[t] largest and the
    slots from k[t] on hold -1 (per-token dynamic K)."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    ids = np.empty((T, K), np.int32)
    kk = None if k is None else np.ascontiguousarray(k, dtype=np.int32)
    _check(lib().oracle_topk_k(T, E, K, _ptr(kk), _ptr(logits), _ptr(ids)), "topk")
    return ids


def gate_weights(logits, ids, score_fn=0, renorm=1):
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, E = logits.shape
    K = ids.shape[1]
    w = np.empty((T, K), np.float64)
    _check(lib().oracle_gate_weights(T, E, K, score_fn, renorm, _ptr(logits), _ptr(ids), _ptr(w)),
           "gate_weights")
    return w


def expected_active(E: int, K: int, m: int) -> float:
    """E[E_active] = E * (1 - (1 - K/E)^m): expected number of experts that
    receive at least one of m tokens under uniform top-K routing (talk notes,
    "Balls-Bins-Buckets" model construction)."""
    return E * (1.0 - (1.0 - K / E) ** m)


def p_max(T, K, E, B, mode=0):
    """Upper bound on padded rows.  Block-wise (mode 0): A + min(E, A) * (B - 1),
    A = T*K.  Max-value (mode 1): E * ceil(min(T, A) / B) * B (an expert holds at
    most one assignment per token)."""
    A = T * K
    if mode == 1:
        return E * ((min(T, A) + B - 1) // B) * B
    return A + min(E, A) * (B - 1)


def align(ids, E, B, P_max=None, mode=0):
    """Alignment of the assignments with block-wise (mode 0) or max-value
    (mode 1) padding; returns a dict of int32 arrays."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, K = ids.shape
    if P_max is None:
        P_max = p_max(T, K, E, B, mode)
    nblk = (P_max + B - 1) // B
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    sorted_ids = np.empty(max(P_max, 1), np.int32)
    block_expert = np.empty(max(nblk, 1), np.int32)
    pos = np.empty(max(T * K, 1), np.int32)
    P = np.zeros(1, np.int32)
    ea = np.zeros(1, np.int32)
    _check(lib().oracle_align(T, K, E, B, mode, _ptr(ids), P_max, _ptr(counts), _ptr(offsets),
                              _ptr(sorted_ids), _ptr(block_expert), _ptr(pos), _ptr(P), _ptr(ea)),
           "align")
    return dict(counts=counts, offsets=offsets, sorted_ids=sorted_ids[:P_max],
                block_expert=block_expert[:nblk], pos=pos[:T * K], P=int(P[0]), E_active=int(ea[0]))


def permute(x, sorted_ids, K, P):
    """x_perm[P,H] (float64): row p is x[sorted_ids[p] // K], zero for -1."""
    x, dt = _typed(x)
    sid = np.ascontiguousarray(sorted_ids, dtype=np.int32)
    H = x.shape[1]
    out = np.empty((P, H), np.float64)
    _check(lib().oracle_permute(H, K, dt, _ptr(x), _ptr(sid), P, _ptr(out)), "permute")
    return out


def combine(y, pos, w, shared=None):
    """out[T,H] (float64) = sum_k w[t,k] * y[pos[t*K+k]] (+ shared[t])."""
    y, dt = _typed(y)
    pos = np.ascontiguousarray(pos, dtype=np.int32).ravel()
    w = np.ascontiguousarray(w, dtype=np.float64)
    T, K = w.shape
    H = y.shape[1]
    sh = None
    if shared is not None:
        sh, d2 = _typed(shared)
        assert d2 == dt
    out = np.empty((T, H), np.float64)
    _check(lib().oracle_combine(T, H, K, dt, _ptr(y), _ptr(pos), _ptr(w), _ptr(sh), _ptr(out)), "combine")
    return out


def swiglu_ffn(x_row, w13, w2):
    """y[H] for one token through one SwiGLU expert (w13 [2I,H], w2 [H,I])."""
    x_row, dt = _typed(x_row)
    w13, _ = _typed(w13)
    w2, _ = _typed(w2)
    H = x_row.shape[-1]
    I = w2.shape[1]
    y = np.empty(H, np.float64)
    _check(lib().oracle_swiglu_ffn(H, I, dt, _ptr(x_row), _ptr(w13), _ptr(w2), _ptr(y)), "swiglu_ffn")
    return y


def dense_ffn(x, w13, w2, nthreads=None):
    """out[T,H] (float64) of a dense SwiGLU FFN (DenseFA / DensePA / shared)."""
    x, dt = _typed(x)
    w13, _ = _typed(w13)
    w2, _ = _typed(w2)
    T, H = x.shape
    I = w2.shape[1]
    out = np.empty((T, H), np.float64)
    _check(lib().oracle_dense_ffn(T, H, I, dt, _ptr(x), _ptr(w13), _ptr(w2), _ptr(out),
                                  nthreads or nthreads_default()), "dense_ffn")
    return out


def moe_layer(x, w_r, w13, w2, K, score_fn=0, renorm=1, w13_sh=None, w2_sh=None,
              logits=None, tokens=None, nthreads=None, return_routing=False, k=None):
    """MoE layer output rows (float64) for the listed tokens (all if None).

    w13 / w2: either stacked arrays [E,2I,H] / [E,H,I], or lists of per-expert
    arrays (None allowed for experts that no listed token selects).
    """
    x, dt = _typed(x)
    T, H = x.shape
    if isinstance(w13, np.ndarray):
        E = w13.shape[0]
        w13_list = [np.ascontiguousarray(w13[e]) for e in range(E)]
        w2_list = [np.ascontiguousarray(w2[e]) for e in range(E)]
    else:
        w13_list, w2_list = list(w13), list(w2)
        E = len(w13_list)
    I = next(w.shape[1] for w in w2_list if w is not None)
    keep = []
    p13 = (ctypes.c_void_p * E)()
    p2 = (ctypes.c_void_p * E)()
    for e in range(E):
        for arr, tab in ((w13_list[e], p13), (w2_list[e], p2)):
            if arr is None:
                tab[e] = None
            else:
                a, d = _typed(arr)
                assert d == dt
                keep.append(a)
                tab[e] = a.ctypes.data
    w_r_c = None
    if w_r is not None:
        w_r_c, d = _typed(w_r)
        assert d == dt
    I_sh = 0
    if w13_sh is not None:
        w13_sh, _ = _typed(w13_sh)
        w2_sh, _ = _typed(w2_sh)
        I_sh = w2_sh.shape[1]
    lg = None
    if logits is not None:
        lg = np.ascontiguousarray(logits, dtype=np.float32)
    elif w_r_c is None:
        raise ValueError("need router weights or logits")
    tok = None
    n = T
    if tokens is not None:
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        n = tok.shape[0]
    out = np.empty((n, H), np.float64)
    ids = np.empty((n, K), np.int32)
    w = np.empty((n, K), np.float64)
    kk = None if k is None else np.ascontiguousarray(k, dtype=np.int32)
    rc = lib().oracle_moe_layer(T, H, E, K, I, I_sh, score_fn, renorm, dt, _ptr(x), _ptr(w_r_c),
                                p13, p2, _ptr(w13_sh), _ptr(w2_sh), _ptr(lg), _ptr(kk), _ptr(tok), n,
                                _ptr(out), _ptr(ids), _ptr(w), nthreads or nthreads_default())
    _check(rc, "moe_layer")
    if return_routing:
        return out, ids, w
    return out


# ------------------------------------------------------------- FP8 weights

def e4m3_value(codes):
    """Values (float64) of E4M3 codes (uint8 array), from the format definition."""
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([lib().oracle_e4m3_value(c) for c in range(256)], np.float64)
    return table[codes]


def e4m3_encode(v):
    """Nearest E4M3 codes (ties to even, saturating at +-448) of fp32 values."""
    v = np.asarray(v, dtype=np.float32)
    f = lib().oracle_e4m3_encode
    return np.array([f(float(a)) for a in v.ravel()], np.uint8).reshape(v.shape)


def quantize_fp8(w):
    """Row-wise FP8 quantisation of a 2-D weight matrix (bf16 as uint16 bit
    patterns, or fp32): returns (codes uint8 [rows, cols], scales fp32 [rows])."""
    w, dt = _typed(w)
    rows, cols = w.shape
    q = np.empty((rows, cols), np.uint8)
    sc = np.empty(rows, np.float32)
    _check(lib().oracle_quantize_fp8(rows, cols, dt, _ptr(w), _ptr(q), _ptr(sc)), "quantize_fp8")
    return q, sc


def moe_layer_fp8(x, w_r, q13, s13, q2, s2, K, score_fn=0, renorm=1, q13_sh=None, s13_sh=None, q2_sh=None,
                  s2_sh=None, logits=None, tokens=None, k=None, nthreads=None):
    """MoE layer output rows (float64) with FP8 expert weights: q13 [E,2I,H] /
    q2 [E,H,I] uint8 codes, s13 [E,2I] / s2 [E,H] fp32 row scales (shared FFN
    likewise, optional); x (and w_r) bf16 bit patterns or fp32."""
    x, dt = _typed(x)
    T, H = x.shape
    E = q13.shape[0]
    I = q2.shape[2]
    keep = []

    def table(arrs, ctype=ctypes.c_void_p):
        tab = (ctype * E)()
        for e in range(E):
            a = np.ascontiguousarray(arrs[e])
            keep.append(a)
            tab[e] = a.ctypes.data
        return tab

    p13, p2 = table(q13), table(q2)
    ps13, ps2 = table(np.asarray(s13, np.float32)), table(np.asarray(s2, np.float32))
    w_r_c = None
    if w_r is not None:
        w_r_c, d = _typed(w_r)
        assert d == dt
    I_sh = 0 if q13_sh is None else q2_sh.shape[1]
    sh = [None if a is None else np.ascontiguousarray(a) for a in (q13_sh, q2_sh)]
    ssh = [None if a is None else np.ascontiguousarray(a, np.float32) for a in (s13_sh, s2_sh)]
    lg = None if logits is None else np.ascontiguousarray(logits, dtype=np.float32)
    if lg is None and w_r_c is None:
        raise ValueError("need router weights or logits")
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    n = T if tok is None else tok.shape[0]
    kk = None if k is None else np.ascontiguousarray(k, dtype=np.int32)
    out = np.empty((n, H), np.float64)
    _check(lib().oracle_moe_layer_fp8(T, H, E, K, I, I_sh, score_fn, renorm, dt, _ptr(x), _ptr(w_r_c), p13, p2,
                                      ps13, ps2, _ptr(sh[0]), _ptr(sh[1]), _ptr(ssh[0]), _ptr(ssh[1]), _ptr(lg),
                                      _ptr(kk), _ptr(tok), n, _ptr(out), nthreads or nthreads_default()),
           "moe_layer_fp8")
    return out


# ------------------------------------------------ tensor parallelism over I

def tp_shard(w13, w2, rank, n_ranks):
    """Rank `rank` of `n_ranks` of a layer split over the expert intermediate
    dimension I (talk notes, "Demystifying the Mixture of Experts Serving
    Tax", "Balls-Bins-Buckets framework": under TP the buckets are the n_tp
    GPUs, each holding a share of every expert).  Reading: every GPU holds,
    for every expert, the gate rows [r*I/n, (r+1)*I/n) of W1, the same rows of
    W3 (rows I + that range of the packed [2I, H] matrix) and the same columns
    of W2, so the FFN of the slice yields W2[:, slice] (silu(W1[slice] x) *
    W3[slice] x), and the slices' outputs sum to the expert's output.

    w13 [E, 2I, H] / w2 [E, H, I] (or one dense FFN [2I, H] / [H, I]);
    returns (w13 slice [E, 2I/n, H], w2 slice [E, H, I/n]) as new arrays."""
    w13 = np.asarray(w13)
    w2 = np.asarray(w2)
    I = w2.shape[-1]
    if n_ranks < 1 or not 0 <= rank < n_ranks or I % n_ranks:
        raise ValueError("I must split evenly over the ranks")
    n = I // n_ranks
    lo, hi = rank * n, (rank + 1) * n
    g = w13[..., lo:hi, :]
    u = w13[..., I + lo:I + hi, :]
    return np.ascontiguousarray(np.concatenate([g, u], axis=-2)), np.ascontiguousarray(w2[..., lo:hi])


def moe_layer_tp(x, w_r, w13, w2, K, n_ranks, score_fn=0, renorm=1, w13_sh=None, w2_sh=None, logits=None,
                 tokens=None, k=None, nthreads=None, partials=False):
    """The layer under TP over I: every rank routes the same tokens the same
    way (the router weights are whole on every rank), runs its slice of every
    expert and of the shared FFN and combines with the gate weights; the
    all-reduce (talk notes, "Key findings" 3: the AllReduce after the MoE
    block under TP) sums the ranks' outputs, here in rank order in float64.
    Returns the sum [n, H], or the list of the ranks' outputs if `partials`."""
    parts = []
    for r in range(n_ranks):
        a13, a2 = tp_shard(w13, w2, r, n_ranks)
        s13, s2 = (None, None) if w13_sh is None else tp_shard(w13_sh, w2_sh, r, n_ranks)
        parts.append(moe_layer(x, w_r, a13, a2, K, score_fn=score_fn, renorm=renorm, w13_sh=s13, w2_sh=s2,
                               logits=logits, tokens=tokens, k=k, nthreads=nthreads))
    if partials:
        return parts
    out = np.zeros_like(parts[0])
    for p in parts:
        out += p
    return out
