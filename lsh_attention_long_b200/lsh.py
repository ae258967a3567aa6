"""Python binding of the C ABI in include/lsh.h (argument marshalling only).

Every function here checks tensor shapes, allocates missing outputs with
torch on the inputs' device, and calls the same-named entry point of
``liblsh.so`` through ctypes on the current CUDA stream.  All arithmetic runs
in the library's CUDA kernels; there is no CPU path.  Importing works without
a GPU, and a missing library raises instead of falling back.
"""

from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblsh.so")

LSH_F32, LSH_BF16 = 0, 1
STATUS = {0: "LSH_OK", 1: "LSH_ERR_INVALID_ARG", 2: "LSH_ERR_UNSUPPORTED", 3: "LSH_ERR_CUDA",
          4: "LSH_ERR_WORKSPACE", 5: "LSH_ERR_TIMEOUT", 6: "LSH_ERR_BAD_KEYS",
          7: "LSH_ERR_SCRATCH_LIMIT"}

EXPORTS = ("lsh_workspace_size", "lsh_hash", "lsh_sort", "lsh_attend_fwd", "lsh_combine",
           "lsh_forward", "lsh_forward_host", "lsh_forward_host_ws_size", "lsh_attend_bwd",
           "lsh_device_status", "lsh_status_string", "lsh_attend_fwd_static", "lsh_set_wait_test",
           "lsh_ffn_ws_size", "lsh_ffn_forward", "lsh_ffn_bwd_ws_size", "lsh_ffn_backward",
           "lsh_rev_ws_size", "lsh_rev_forward", "lsh_rev_backward")


class LshError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "H", "L", "d", "n_buckets", "n_rounds", "chunk", "causal", "dtype")]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load liblsh.so (built by ``python -m lsh_attention_long_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is missing; build it with "
                           "`python -m lsh_attention_long_b200.build`")
    lib = ctypes.CDLL(path)
    P, S = ctypes.c_void_p, ctypes.POINTER(Shape)
    sz = ctypes.c_size_t
    sig = {
        "lsh_workspace_size": ([S], sz),
        "lsh_hash": ([S, P, P, P, P, P], ctypes.c_int),
        "lsh_sort": ([S, P, P, P, sz, P], ctypes.c_int),
        "lsh_attend_fwd": ([S, P, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "lsh_combine": ([S, P, P, P, P, P], ctypes.c_int),
        "lsh_forward": ([S, P, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "lsh_forward_host_ws_size": ([S], sz),
        "lsh_forward_host": ([S, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "lsh_attend_bwd": ([S, P, P, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "lsh_device_status": ([P], ctypes.c_int),
        "lsh_attend_fwd_static": ([S, P, P, P, P, P, P, P], ctypes.c_int),
        "lsh_set_wait_test": ([ctypes.c_int32, ctypes.c_int64], ctypes.c_int),
        "lsh_ffn_ws_size": ([ctypes.c_int32] * 4, sz),
        "lsh_ffn_forward": ([ctypes.c_int32] * 4 + [P] * 7 + [sz, P], ctypes.c_int),
        "lsh_ffn_bwd_ws_size": ([ctypes.c_int32] * 4, sz),
        "lsh_ffn_backward": ([ctypes.c_int32] * 4 + [P] * 12 + [sz, P], ctypes.c_int),
        "lsh_rev_ws_size": ([S, ctypes.c_int32, ctypes.c_int32], sz),
        "lsh_rev_forward": ([S, ctypes.c_int32, ctypes.c_int32] + [P] * 12 + [sz, P],
                            ctypes.c_int),
        "lsh_rev_backward": ([S, ctypes.c_int32, ctypes.c_int32] + [P] * 19 + [sz, P],
                             ctypes.c_int),
        "lsh_status_string": ([ctypes.c_int], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return LSH_F32
    if t == torch.bfloat16:
        return LSH_BF16
    raise TypeError(f"unsupported dtype {t}; use float32 or bfloat16")


def make_shape(B, H, L, d, n_buckets, n_rounds, chunk, causal, dtype: torch.dtype) -> Shape:
    return Shape(B, H, L, d, n_buckets, n_rounds, chunk, int(bool(causal)), _dtype_code(dtype))


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the LSH library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _call(name: str, *args):
    rc = getattr(load_library(), name)(*args)
    if rc != 0:
        raise LshError(name, rc)


def _qshape(Q: torch.Tensor):
    if not isinstance(Q, torch.Tensor) or Q.dim() != 4:
        raise ValueError("Q must be a [B, H, L, d] tensor")
    return tuple(Q.shape)


def _validate(specs, device=None):
    """Checks (name, tensor, shape, dtype, on_device) entries before any call:
    the library takes plain pointers, so a wrong size, type or memory space
    would otherwise reach the kernels.  Shapes and types are checked for every
    entry first, then where each tensor lives (CUDA tensors on one device;
    host tensors for the host-buffer forward).  None tensors are skipped."""
    for name, t, shape, dtype, _ in specs:
        if t is None:
            continue
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if dtype is not None and t.dtype != dtype:
            raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    for name, t, _, _, on_device in specs:
        if t is None:
            continue
        if on_device and not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not on_device and t.is_cuda:
            raise ValueError(f"{name} must be a host tensor")
        if on_device:
            if device is None:
                device = t.device
            elif t.device != device:
                raise ValueError(f"{name} is on {t.device}, expected {device}")


def _rot_spec(rot, R, d, n_buckets, dtype, on_device=True):
    """The rotation is read only when n_buckets > 1: [R, d, n_buckets/2]."""
    if n_buckets > 1:
        return ("rot", rot, (R, d, n_buckets // 2), dtype, on_device)
    return ("rot", None, None, None, on_device)


def lsh_workspace_size(shape: Shape) -> int:
    return int(load_library().lsh_workspace_size(ctypes.byref(shape)))


def workspace(shape: Shape, device) -> torch.Tensor:
    """A byte tensor large enough for any call on this shape."""
    return torch.empty(max(lsh_workspace_size(shape), 16), dtype=torch.uint8, device=device)


def lsh_hash(Q, rot, n_buckets: int, *, keys=None, buckets=None, want_buckets=True, stream=None):
    """Step 1: keys [R,B,H,L] u32 (as int32 storage) and bucket ids [R,B,H,L] i32."""
    B, H, L, d = _qshape(Q)
    R = rot.shape[0]
    shape = make_shape(B, H, L, d, n_buckets, R, 1, False, Q.dtype)
    rows = (R, B, H, L)
    _validate([("Q", Q, None, None, True), _rot_spec(rot, R, d, n_buckets, Q.dtype),
               ("keys", keys, rows, torch.int32, True),
               ("buckets", buckets, rows, torch.int32, True)])
    if keys is None:
        keys = torch.empty((R, B, H, L), dtype=torch.int32, device=Q.device)
    if buckets is None and want_buckets:
        buckets = torch.empty((R, B, H, L), dtype=torch.int32, device=Q.device)
    _call("lsh_hash", ctypes.byref(shape), _ptr(Q), _ptr(rot) if n_buckets > 1 else None,
          _ptr(keys), _ptr(buckets), _stream(stream))
    return keys, buckets


def lsh_sort(keys, n_buckets: int, *, perm=None, stream=None):
    """Step 2: perm [R,B,H,L] i32 (original position at each sorted slot)."""
    if not isinstance(keys, torch.Tensor) or keys.dim() != 4:
        raise ValueError("keys must be a [R, B, H, L] tensor")
    R, B, H, L = keys.shape
    shape = make_shape(B, H, L, 64, n_buckets, R, 1, False, torch.float32)
    _validate([("keys", keys, None, torch.int32, True),
               ("perm", perm, (R, B, H, L), torch.int32, True)])
    if perm is None:
        perm = torch.empty_like(keys, dtype=torch.int32)
    _call("lsh_sort", ctypes.byref(shape), _ptr(keys), _ptr(perm), None, 0, _stream(stream))
    return perm


def lsh_attend_fwd(Q, V, keys, perm, n_buckets: int, chunk: int, causal: bool, *,
                   o_part=None, lse_r=None, O=None, lse=None, combine=True, ws=None,
                   stream=None):
    """Steps 3-5.  Returns (O, lse, o_part, lse_r); O/lse are None when combine=False."""
    B, H, L, d = _qshape(Q)
    R = keys.shape[0]
    shape = make_shape(B, H, L, d, n_buckets, R, chunk, causal, Q.dtype)
    rows = (R, B, H, L)
    _validate([("Q", Q, None, None, True), ("V", V, Q.shape, Q.dtype, True),
               ("keys", keys, rows, torch.int32, True), ("perm", perm, rows, torch.int32, True),
               ("o_part", o_part, rows + (d,), torch.float32, True),
               ("lse_r", lse_r, rows, torch.float32, True),
               ("O", O, Q.shape, Q.dtype, True), ("lse", lse, (B, H, L), torch.float32, True),
               ("ws", ws, None, None, True)])
    if combine:
        if O is None:
            O = torch.empty_like(Q)
        if lse is None:
            lse = torch.empty((B, H, L), dtype=torch.float32, device=Q.device)
    else:
        if o_part is None:
            o_part = torch.empty((R, B, H, L, d), dtype=torch.float32, device=Q.device)
        if lse_r is None:
            lse_r = torch.empty((R, B, H, L), dtype=torch.float32, device=Q.device)
    if ws is None:
        ws = workspace(shape, Q.device)
    _call("lsh_attend_fwd", ctypes.byref(shape), _ptr(Q), _ptr(V), _ptr(keys), _ptr(perm),
          _ptr(o_part), _ptr(lse_r), _ptr(O) if combine else None,
          _ptr(lse) if combine else None, _ptr(ws), 0 if ws is None else ws.numel(),
          _stream(stream))
    return O, lse, o_part, lse_r


def lsh_combine(o_part, lse_r, dtype: torch.dtype, *, O=None, lse=None, stream=None):
    """Step 5 alone: O [B,H,L,d] in dtype and lse [B,H,L] fp32."""
    if not isinstance(o_part, torch.Tensor) or o_part.dim() != 5:
        raise ValueError("o_part must be a [R, B, H, L, d] tensor")
    R, B, H, L, d = o_part.shape
    shape = make_shape(B, H, L, d, 2, R, 1, False, dtype)
    _validate([("o_part", o_part, None, torch.float32, True),
               ("lse_r", lse_r, (R, B, H, L), torch.float32, True),
               ("O", O, (B, H, L, d), dtype, True), ("lse", lse, (B, H, L), torch.float32, True)])
    if O is None:
        O = torch.empty((B, H, L, d), dtype=dtype, device=o_part.device)
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=o_part.device)
    _call("lsh_combine", ctypes.byref(shape), _ptr(o_part), _ptr(lse_r), _ptr(O), _ptr(lse),
          _stream(stream))
    return O, lse


def lsh_forward(Q, V, rot, n_buckets: int, chunk: int, causal: bool, *, out=None, ws=None,
                want_buckets=False, stream=None) -> Dict[str, torch.Tensor]:
    """Whole forward (hash -> sort -> attend with fused combine) in one C call.

    ``out`` may hold preallocated tensors under the keys returned."""
    B, H, L, d = _qshape(Q)
    R = rot.shape[0]
    shape = make_shape(B, H, L, d, n_buckets, R, chunk, causal, Q.dtype)
    o = dict(out or {})
    rows = (R, B, H, L)
    _validate([("Q", Q, None, None, True), ("V", V, Q.shape, Q.dtype, True),
               _rot_spec(rot, R, d, n_buckets, Q.dtype),
               ("out['keys']", o.get("keys"), rows, torch.int32, True),
               ("out['perm']", o.get("perm"), rows, torch.int32, True),
               ("out['buckets']", o.get("buckets"), rows, torch.int32, True),
               ("out['O']", o.get("O"), Q.shape, Q.dtype, True),
               ("out['lse']", o.get("lse"), (B, H, L), torch.float32, True),
               ("ws", ws, None, None, True)])
    dev = Q.device
    o.setdefault("keys", torch.empty((R, B, H, L), dtype=torch.int32, device=dev))
    o.setdefault("perm", torch.empty((R, B, H, L), dtype=torch.int32, device=dev))
    o.setdefault("O", torch.empty_like(Q))
    o.setdefault("lse", torch.empty((B, H, L), dtype=torch.float32, device=dev))
    if want_buckets:
        o.setdefault("buckets", torch.empty((R, B, H, L), dtype=torch.int32, device=dev))
    if ws is None:
        ws = workspace(shape, dev)
    _call("lsh_forward", ctypes.byref(shape), _ptr(Q), _ptr(V),
          _ptr(rot) if n_buckets > 1 else None, _ptr(o["keys"]), _ptr(o.get("buckets")),
          _ptr(o["perm"]), _ptr(o["O"]), _ptr(o["lse"]), _ptr(ws), ws.numel(), _stream(stream))
    return o


def forward_host_workspace(shape: Shape, device) -> torch.Tensor:
    """Device scratch for lsh_forward_host on this shape."""
    n = load_library().lsh_forward_host_ws_size(ctypes.byref(shape))
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def lsh_forward_host(Q, V, rot, n_buckets: int, chunk: int, causal: bool, *, O=None, lse=None,
                     ws=None, device=None, stream=None):
    """Whole forward from host tensors (page-locked for overlapped copies):
    returns host O [B,H,L,d] and lse [B,H,L].  The library pipelines the
    copies and kernels over groups of heads; the call returns once they are
    queued on ``stream`` (synchronise it before reading O)."""
    B, H, L, d = _qshape(Q)
    R = rot.shape[0]
    shape = make_shape(B, H, L, d, n_buckets, R, chunk, causal, Q.dtype)
    _validate([("Q", Q, None, None, False), ("V", V, Q.shape, Q.dtype, False),
               _rot_spec(rot, R, d, n_buckets, Q.dtype, on_device=False),
               ("O", O, Q.shape, Q.dtype, False), ("lse", lse, (B, H, L), torch.float32, False),
               ("ws", ws, None, None, True)])
    if O is None:
        O = torch.empty_like(Q, pin_memory=True)
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, pin_memory=True)
    if ws is None:
        ws = forward_host_workspace(shape, device or torch.device("cuda", torch.cuda.current_device()))
    _call("lsh_forward_host", ctypes.byref(shape), _ptr(Q), _ptr(V),
          _ptr(rot) if n_buckets > 1 else None, _ptr(O), _ptr(lse), _ptr(ws), ws.numel(),
          _stream(stream))
    return O, lse


def lsh_attend_bwd(Q, V, O, dO, keys, perm, lse, n_buckets: int, chunk: int, causal: bool, *,
                   dQ=None, dV=None, ws=None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Backward with buckets frozen: (dQ, dV) in Q's dtype."""
    B, H, L, d = _qshape(Q)
    R = keys.shape[0]
    shape = make_shape(B, H, L, d, n_buckets, R, chunk, causal, Q.dtype)
    rows = (R, B, H, L)
    _validate([("Q", Q, None, None, True), ("V", V, Q.shape, Q.dtype, True),
               ("O", O, Q.shape, Q.dtype, True), ("dO", dO, Q.shape, Q.dtype, True),
               ("keys", keys, rows, torch.int32, True), ("perm", perm, rows, torch.int32, True),
               ("lse", lse, (B, H, L), torch.float32, True),
               ("dQ", dQ, Q.shape, Q.dtype, True), ("dV", dV, Q.shape, Q.dtype, True),
               ("ws", ws, None, None, True)])
    if dQ is None:
        dQ = torch.empty_like(Q)
    if dV is None:
        dV = torch.empty_like(V)
    if ws is None:
        ws = workspace(shape, Q.device)
    _call("lsh_attend_bwd", ctypes.byref(shape), _ptr(Q), _ptr(V), _ptr(O), _ptr(dO),
          _ptr(keys), _ptr(perm), _ptr(lse), _ptr(dQ), _ptr(dV), _ptr(ws), ws.numel(),
          _stream(stream))
    return dQ, dV


def ffn_workspace(tokens: int, d_model: int, d_ff: int, chunk: int, device) -> torch.Tensor:
    """Device scratch for lsh_ffn_forward: one chunk's hidden activation."""
    n = load_library().lsh_ffn_ws_size(tokens, d_model, d_ff, chunk)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def lsh_ffn_forward(X, W1, b1, W2, b2, chunk: int, *, Y=None, ws=None, stream=None):
    """Chunked feed-forward: Y = W2 max(0, W1 x + b1) + b2 per position of X
    [..., d_model] (bf16), `chunk` positions at a time."""
    if not isinstance(X, torch.Tensor) or X.dim() < 2:
        raise ValueError("X must be a [..., d_model] tensor")
    d_model = X.shape[-1]
    tokens = X.numel() // d_model if d_model else 0
    d_ff = W1.shape[0] if isinstance(W1, torch.Tensor) and W1.dim() == 2 else -1
    bf = torch.bfloat16
    _validate([("X", X, None, bf, True), ("W1", W1, (d_ff, d_model), bf, True),
               ("b1", b1, (d_ff,), bf, True), ("W2", W2, (d_model, d_ff), bf, True),
               ("b2", b2, (d_model,), bf, True), ("Y", Y, X.shape, bf, True),
               ("ws", ws, None, None, True)])
    if Y is None:
        Y = torch.empty_like(X)
    if ws is None:
        ws = ffn_workspace(tokens, d_model, d_ff, chunk, X.device)
    _call("lsh_ffn_forward", tokens, d_model, d_ff, chunk, _ptr(X), _ptr(W1), _ptr(b1), _ptr(W2),
          _ptr(b2), _ptr(Y), _ptr(ws), ws.numel(), _stream(stream))
    return Y


def lsh_ffn_backward(X, W1, b1, W2, dY, chunk: int, *, R=None, dX=None, grads=None, ws=None,
                     stream=None):
    """Backward of the chunked feed-forward: returns dX (fp32, plus R when
    given) and the fp32 gradients dW1, db1, dW2, db2 (in ``grads`` when given)."""
    if not isinstance(X, torch.Tensor) or X.dim() < 2:
        raise ValueError("X must be a [..., d_model] tensor")
    d_model = X.shape[-1]
    tokens = X.numel() // d_model if d_model else 0
    d_ff = W1.shape[0] if isinstance(W1, torch.Tensor) and W1.dim() == 2 else -1
    bf, f32 = torch.bfloat16, torch.float32
    g = dict(grads or {})
    _validate([("X", X, None, bf, True), ("W1", W1, (d_ff, d_model), bf, True),
               ("b1", b1, (d_ff,), bf, True), ("W2", W2, (d_model, d_ff), bf, True),
               ("dY", dY, X.shape, bf, True), ("R", R, X.shape, f32, True),
               ("dX", dX, X.shape, f32, True), ("dW1", g.get("dW1"), (d_ff, d_model), f32, True),
               ("db1", g.get("db1"), (d_ff,), f32, True),
               ("dW2", g.get("dW2"), (d_model, d_ff), f32, True),
               ("db2", g.get("db2"), (d_model,), f32, True), ("ws", ws, None, None, True)])
    dev = X.device
    if dX is None:
        dX = torch.empty(X.shape, dtype=f32, device=dev)
    g.setdefault("dW1", torch.empty((d_ff, d_model), dtype=f32, device=dev))
    g.setdefault("db1", torch.empty((d_ff,), dtype=f32, device=dev))
    g.setdefault("dW2", torch.empty((d_model, d_ff), dtype=f32, device=dev))
    g.setdefault("db2", torch.empty((d_model,), dtype=f32, device=dev))
    if ws is None:
        n = load_library().lsh_ffn_bwd_ws_size(tokens, d_model, d_ff, chunk)
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
    _call("lsh_ffn_backward", tokens, d_model, d_ff, chunk, _ptr(X), _ptr(W1), _ptr(b1), _ptr(W2),
          _ptr(dY), _ptr(R), _ptr(dX), _ptr(g["dW1"]), _ptr(g["db1"]), _ptr(g["dW2"]),
          _ptr(g["db2"]), _ptr(ws), ws.numel(), _stream(stream))
    return dX, g


def _rev_shape(X, H, n_buckets, n_rounds, chunk, causal):
    if not isinstance(X, torch.Tensor) or X.dim() != 3 or X.shape[2] % H:
        raise ValueError("X must be a [B, L, H * 64] tensor")
    B, Lx, D = X.shape
    return make_shape(B, H, Lx, D // H, n_buckets, n_rounds, chunk, causal, torch.bfloat16)


def rev_workspace(shape: Shape, d_ff: int, ffn_chunk: int, device) -> torch.Tensor:
    n = load_library().lsh_rev_ws_size(ctypes.byref(shape), d_ff, ffn_chunk)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def lsh_rev_forward(X1, X2, rot, W1, b1, W2, b2, H: int, n_buckets: int, chunk: int,
                    causal: bool, ffn_chunk: int, *, ws=None, stream=None):
    """Reversible block: Y1 = X1 + F(X2), Y2 = X2 + G(Y1) (F: LSH attention,
    G: chunked feed-forward).  X1, X2 fp32 [B, L, H*64].  Returns Y1, Y2 and
    the keys and permutations of X2's hash."""
    R = rot.shape[0]
    shape = _rev_shape(X2, H, n_buckets, R, chunk, causal)
    B, Lx, D = X2.shape
    d_ff = W1.shape[0] if isinstance(W1, torch.Tensor) and W1.dim() == 2 else -1
    f32, bf = torch.float32, torch.bfloat16
    _validate([("X1", X1, X2.shape, f32, True), ("X2", X2, None, f32, True),
               _rot_spec(rot, R, 64, n_buckets, bf), ("W1", W1, (d_ff, D), bf, True),
               ("b1", b1, (d_ff,), bf, True), ("W2", W2, (D, d_ff), bf, True),
               ("b2", b2, (D,), bf, True), ("ws", ws, None, None, True)])
    dev = X2.device
    Y1, Y2 = torch.empty_like(X2), torch.empty_like(X2)
    keys = torch.empty((R, B, H, Lx), dtype=torch.int32, device=dev)
    perm = torch.empty_like(keys)
    if ws is None:
        ws = rev_workspace(shape, d_ff, ffn_chunk, dev)
    _call("lsh_rev_forward", ctypes.byref(shape), d_ff, ffn_chunk, _ptr(X1), _ptr(X2),
          _ptr(rot) if n_buckets > 1 else None, _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), _ptr(Y1),
          _ptr(Y2), _ptr(keys), _ptr(perm), _ptr(ws), ws.numel(), _stream(stream))
    return Y1, Y2, keys, perm


def lsh_rev_backward(Y1, Y2, dY1, dY2, keys, perm, W1, b1, W2, b2, H: int, n_buckets: int,
                     chunk: int, causal: bool, ffn_chunk: int, *, ws=None, stream=None):
    """Backward of the reversible block from its outputs: returns the
    recomputed X1, X2, the input gradients dX1, dX2 (fp32) and G's parameter
    gradients {dW1, db1, dW2, db2} (fp32)."""
    R = keys.shape[0]
    shape = _rev_shape(Y2, H, n_buckets, R, chunk, causal)
    B, Lx, D = Y2.shape
    d_ff = W1.shape[0] if isinstance(W1, torch.Tensor) and W1.dim() == 2 else -1
    f32, bf = torch.float32, torch.bfloat16
    rows = (R, B, H, Lx)
    _validate([("Y1", Y1, Y2.shape, f32, True), ("Y2", Y2, None, f32, True),
               ("dY1", dY1, Y2.shape, f32, True), ("dY2", dY2, Y2.shape, f32, True),
               ("keys", keys, rows, torch.int32, True), ("perm", perm, rows, torch.int32, True),
               ("W1", W1, (d_ff, D), bf, True), ("b1", b1, (d_ff,), bf, True),
               ("W2", W2, (D, d_ff), bf, True), ("b2", b2, (D,), bf, True),
               ("ws", ws, None, None, True)])
    dev = Y2.device
    X1, X2, dX1, dX2 = (torch.empty_like(Y2) for _ in range(4))
    g = {"dW1": torch.empty((d_ff, D), dtype=f32, device=dev),
         "db1": torch.empty((d_ff,), dtype=f32, device=dev),
         "dW2": torch.empty((D, d_ff), dtype=f32, device=dev),
         "db2": torch.empty((D,), dtype=f32, device=dev)}
    if ws is None:
        ws = rev_workspace(shape, d_ff, ffn_chunk, dev)
    _call("lsh_rev_backward", ctypes.byref(shape), d_ff, ffn_chunk, _ptr(Y1), _ptr(Y2), _ptr(dY1),
          _ptr(dY2), _ptr(keys), _ptr(perm), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), _ptr(X1),
          _ptr(X2), _ptr(dX1), _ptr(dX2), _ptr(g["dW1"]), _ptr(g["db1"]), _ptr(g["dW2"]),
          _ptr(g["db2"]), _ptr(ws), ws.numel(), _stream(stream))
    return X1, X2, dX1, dX2, g


def lsh_set_wait_test(hold_tile: int = -1, wait_cycles: int = 0) -> None:
    """Test hook of the bounded device waits (see include/lsh.h): a clock-cycle
    limit for the tensor-core attention kernel's waits (0 = default) and a tile
    its producers withhold (-1 = none).  Process-wide."""
    _call("lsh_set_wait_test", int(hold_tile), int(wait_cycles))


def lsh_device_status(stream=None) -> int:
    """Synchronise and return (and clear) the first device-side error code."""
    return int(load_library().lsh_device_status(_stream(stream)))
