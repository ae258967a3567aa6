"""ctypes binding of the fp64 CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product path never does.

Every function takes numpy arrays (any float dtype is upcast to float64,
which is exact for fp32 and bf16 values) and returns numpy arrays.  The
arithmetic lives in ``lsh_oracle.cpp``; this file only marshals arguments and
builds that file with the host C++ compiler when its library is missing or
older than the source.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lsh_oracle.cpp")
_LIB = os.path.join(_HERE, "liblsh_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile lsh_oracle.cpp into liblsh_oracle.so (plain -O2, no fast-math)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-fno-fast-math",
                               _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_lsh_hash.argtypes = [I, I, I, I, I, I, P, P, P, P, P]
        lib.oracle_lsh_sort.argtypes = [I, I, P, P]
        lib.oracle_lsh_attend_fwd.argtypes = [I, I, I, I, I, I, I, P, P, P, P, P, P]
        lib.oracle_lsh_attend_fwd_range.argtypes = [I, I, I, I, I, I, I, P, P, P, P, I, I, P, P]
        lib.oracle_lsh_combine.argtypes = [I, I, I, I, I, P, P, P, P]
        lib.oracle_lsh_attend_bwd.argtypes = [I, I, I, I, I, I, I, P, P, P, P, P, P, P]
        lib.oracle_ffn_forward.argtypes = [I, I, I, I, P, P, P, P, P, P]
        lib.oracle_ffn_backward.argtypes = [I, I, I, I, P, P, P, P, P, P, P, P, P, P]
        for f in (lib.oracle_lsh_hash, lib.oracle_lsh_sort, lib.oracle_lsh_attend_fwd,
                  lib.oracle_lsh_attend_fwd_range,
                  lib.oracle_lsh_combine, lib.oracle_lsh_attend_bwd, lib.oracle_ffn_forward,
                  lib.oracle_ffn_backward):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, name: str):
    if rc != 0:
        raise ValueError(f"{name}: invalid argument (status {rc})")


def lsh_hash(Q, rot, n_buckets: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Q [B,H,L,d], rot [R,d,nb/2] -> keys u32, buckets i32, near_tie u8, each [R,B,H,L]."""
    Q = _f64(Q)
    rot = _f64(rot)
    B, H, L, d = Q.shape
    R = rot.shape[0]
    keys = np.zeros((R, B, H, L), np.uint32)
    buckets = np.zeros((R, B, H, L), np.int32)
    tie = np.zeros((R, B, H, L), np.uint8)
    rc = _load().oracle_lsh_hash(B, H, L, d, n_buckets, R, _ptr(Q), _ptr(rot), _ptr(keys),
                                 _ptr(buckets), _ptr(tie))
    _check(rc, "oracle_lsh_hash")
    return keys, buckets, tie


def lsh_sort(keys: np.ndarray) -> np.ndarray:
    """keys [..., L] u32 (bucket*L + position) -> perm [..., L] i32."""
    keys = np.ascontiguousarray(keys, dtype=np.uint32)
    L = keys.shape[-1]
    rows = keys.size // L if L else 0
    perm = np.zeros(keys.shape, np.int32)
    _check(_load().oracle_lsh_sort(rows, L, _ptr(keys), _ptr(perm)), "oracle_lsh_sort")
    return perm


def lsh_attend_fwd(Q, V, keys, perm, chunk: int, causal: bool):
    """-> o_part [R,B,H,L,d] and lse_r [R,B,H,L], both float64."""
    Q = _f64(Q)
    V = _f64(V)
    keys = np.ascontiguousarray(keys, dtype=np.uint32)
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    B, H, L, d = Q.shape
    R = keys.shape[0]
    o_part = np.zeros((R, B, H, L, d))
    lse_r = np.zeros((R, B, H, L))
    rc = _load().oracle_lsh_attend_fwd(B, H, L, d, R, chunk, int(bool(causal)), _ptr(Q), _ptr(V),
                                       _ptr(keys), _ptr(perm), _ptr(o_part), _ptr(lse_r))
    _check(rc, "oracle_lsh_attend_fwd")
    return o_part, lse_r


def lsh_attend_fwd_range(Q, V, keys, perm, chunk: int, causal: bool, chunk_begin: int,
                         chunk_end: int):
    """lsh_attend_fwd restricted to the queries of chunks [chunk_begin, chunk_end)
    of every row; other positions of the outputs stay zero."""
    Q = _f64(Q)
    V = _f64(V)
    keys = np.ascontiguousarray(keys, dtype=np.uint32)
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    B, H, L, d = Q.shape
    R = keys.shape[0]
    o_part = np.zeros((R, B, H, L, d))
    lse_r = np.zeros((R, B, H, L))
    rc = _load().oracle_lsh_attend_fwd_range(B, H, L, d, R, chunk, int(bool(causal)), _ptr(Q),
                                             _ptr(V), _ptr(keys), _ptr(perm), chunk_begin,
                                             chunk_end, _ptr(o_part), _ptr(lse_r))
    _check(rc, "oracle_lsh_attend_fwd_range")
    return o_part, lse_r


def lsh_combine(o_part, lse_r):
    """o_part [R,B,H,L,d], lse_r [R,B,H,L] -> O [B,H,L,d], lse [B,H,L]."""
    o_part = _f64(o_part)
    lse_r = _f64(lse_r)
    R, B, H, L, d = o_part.shape
    O = np.zeros((B, H, L, d))
    lse = np.zeros((B, H, L))
    rc = _load().oracle_lsh_combine(R, B, H, L, d, _ptr(o_part), _ptr(lse_r), _ptr(O), _ptr(lse))
    _check(rc, "oracle_lsh_combine")
    return O, lse


def lsh_attend_bwd(Q, V, dO, keys, perm, chunk: int, causal: bool):
    """Gradients of sum(dO * O) with buckets frozen -> dQ, dV [B,H,L,d] float64."""
    Q = _f64(Q)
    V = _f64(V)
    dO = _f64(dO)
    keys = np.ascontiguousarray(keys, dtype=np.uint32)
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    B, H, L, d = Q.shape
    R = keys.shape[0]
    dQ = np.zeros_like(Q)
    dV = np.zeros_like(V)
    rc = _load().oracle_lsh_attend_bwd(B, H, L, d, R, chunk, int(bool(causal)), _ptr(Q), _ptr(V),
                                       _ptr(dO), _ptr(keys), _ptr(perm), _ptr(dQ), _ptr(dV))
    _check(rc, "oracle_lsh_attend_bwd")
    return dQ, dV


def lsh_forward(Q, V, rot, n_buckets: int, chunk: int, causal: bool):
    """The whole forward: hash -> sort -> attend -> combine.  Returns a dict of arrays."""
    keys, buckets, tie = lsh_hash(Q, rot, n_buckets)
    perm = lsh_sort(keys)
    o_part, lse_r = lsh_attend_fwd(Q, V, keys, perm, chunk, causal)
    O, lse = lsh_combine(o_part, lse_r)
    return {"keys": keys, "buckets": buckets, "near_tie": tie, "perm": perm,
            "o_part": o_part, "lse_r": lse_r, "O": O, "lse": lse}


def ffn_forward(X, W1, b1, W2, b2, chunk: int):
    """Chunked feed-forward: X [T, d_model] -> Y [T, d_model] float64."""
    X, W1, b1, W2, b2 = (_f64(a) for a in (X, W1, b1, W2, b2))
    T, d_model = X.shape
    d_ff = W1.shape[0]
    Y = np.zeros((T, d_model))
    rc = _load().oracle_ffn_forward(T, d_model, d_ff, chunk, _ptr(X), _ptr(W1), _ptr(b1),
                                    _ptr(W2), _ptr(b2), _ptr(Y))
    _check(rc, "oracle_ffn_forward")
    return Y


def ffn_backward(X, W1, b1, W2, dY, chunk: int):
    """Gradients of sum(dY * Y) -> dX, dW1, db1, dW2, db2 (float64)."""
    X, W1, b1, W2, dY = (_f64(a) for a in (X, W1, b1, W2, dY))
    T, d_model = X.shape
    d_ff = W1.shape[0]
    dX = np.zeros_like(X)
    dW1, db1 = np.zeros_like(W1), np.zeros(d_ff)
    dW2, db2 = np.zeros_like(W2), np.zeros(d_model)
    rc = _load().oracle_ffn_backward(T, d_model, d_ff, chunk, _ptr(X), _ptr(W1), _ptr(b1),
                                     _ptr(W2), _ptr(dY), _ptr(dX), _ptr(dW1), _ptr(db1),
                                     _ptr(dW2), _ptr(db2))
    _check(rc, "oracle_ffn_backward")
    return dX, dW1, db1, dW2, db2


# ---------------------------------------------------------------------------
# reversible residual block around LSH attention (composition of the above)
# ---------------------------------------------------------------------------

def _heads(x, H):
    """[B, L, H*d] (token-major) -> [B, H, L, d]."""
    B, L, D = x.shape
    return np.ascontiguousarray(x.reshape(B, L, H, D // H).transpose(0, 2, 1, 3))


def _tokens(x):
    """[B, H, L, d] -> [B, L, H*d]."""
    B, H, L, d = x.shape
    return np.ascontiguousarray(x.transpose(0, 2, 1, 3).reshape(B, L, H * d))


def rev_attention(x, keys, perm, H, chunk, causal):
    """F(x): LSH attention with the token's own features as query (= key)
    and value, head by head: [B, L, H*d] -> [B, L, H*d], buckets given."""
    q = _heads(_f64(x), H)
    o_part, lse_r = lsh_attend_fwd(q, q, keys, perm, chunk, causal)
    O, _ = lsh_combine(o_part, lse_r)
    return _tokens(O)


def rev_forward(X1, X2, rot, n_buckets, H, chunk, causal, W1, b1, W2, b2, ffn_chunk):
    """Reversible block (RevNet residuals, as the Reformer abstract and the
    explainer describe): Y1 = X1 + F(X2), Y2 = X2 + G(Y1), with F = LSH
    attention of X2 and G the chunked feed-forward.  Returns Y1, Y2 and the
    keys and permutations of X2's hash, which the backward holds constant."""
    X1, X2 = _f64(X1), _f64(X2)
    B, L, D = X2.shape
    keys, _, _ = lsh_hash(_heads(X2, H), rot, n_buckets)
    perm = lsh_sort(keys)
    Y1 = X1 + rev_attention(X2, keys, perm, H, chunk, causal)
    Y2 = X2 + ffn_forward(Y1.reshape(B * L, D), W1, b1, W2, b2, ffn_chunk).reshape(B, L, D)
    return Y1, Y2, keys, perm


def rev_backward(Y1, Y2, dY1, dY2, keys, perm, H, chunk, causal, W1, b1, W2, b2, ffn_chunk,
                 g_input=None, f_upstream=None):
    """Backward of the reversible block from its outputs alone: the inputs
    are recomputed (X2 = Y2 - G(Y1), X1 = Y1 - F(X2)), not stored.  With the
    buckets held constant:
      dY1' = dY1 + G'(Y1)^T dY2,   dX2 = dY2 + F'(X2)^T dY1',   dX1 = dY1',
    and the feed-forward's weight and bias gradients.  F'(x)^T g is the sum
    of the attention's query and value gradients (both are x).  `g_input`
    (default Y1) is the input G is evaluated at, for a comparison with an
    implementation that feeds G a rounded copy of Y1: G's max(0, .) then
    takes the same decisions on both sides; `f_upstream` (default dY1') is the
    upstream gradient F's backward is given, likewise.
    Returns X1, X2, dX1, dX2, dW1, db1, dW2, db2."""
    Y1, Y2, dY1, dY2 = (_f64(a) for a in (Y1, Y2, dY1, dY2))
    B, L, D = Y1.shape
    T = B * L
    gin = (Y1 if g_input is None else _f64(g_input)).reshape(T, D)
    X2 = Y2 - ffn_forward(gin, W1, b1, W2, b2, ffn_chunk).reshape(B, L, D)
    gY1, dW1, db1, dW2, db2 = ffn_backward(gin, W1, b1, W2, dY2.reshape(T, D), ffn_chunk)
    dY1p = dY1 + gY1.reshape(B, L, D)
    X1 = Y1 - rev_attention(X2, keys, perm, H, chunk, causal)
    q = _heads(X2, H)
    up = dY1p if f_upstream is None else _f64(f_upstream)
    dQ, dV = lsh_attend_bwd(q, q, _heads(up, H), keys, perm, chunk, causal)
    dX2 = dY2 + _tokens(dQ + dV)
    return X1, X2, dY1p, dX2, dW1, db1, dW2, db2
