"""Host-side checks of the C ABI: the library loads without a GPU, exports
every entry point the headers declare, and rejects bad arguments before any
launch (these calls never reach the device)."""

import ctypes
import glob
import os
import re
import subprocess

import pytest

import lsh_attention_long_b200 as L
from lsh_attention_long_b200 import build as B
from lsh_attention_long_b200.lsh import Shape

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load_library()


def declared_symbols():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names += re.findall(r"LSH_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return sorted(set(names))


def test_headers_declare_the_five_steps():
    names = declared_symbols()
    for n in ("lsh_hash", "lsh_sort", "lsh_attend_fwd", "lsh_attend_bwd", "lsh_combine"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", B.LIB], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in declared_symbols():
        assert n in exported, n
        assert hasattr(lib, n)


def test_library_is_built_for_sm100a():
    assert "arch=compute_100a,code=sm_100a" in " ".join(B.NVCC_FLAGS)


def _shape(**kw):
    base = dict(B=1, H=2, L=256, d=64, n_buckets=16, n_rounds=2, chunk=64, causal=1, dtype=1)
    base.update(kw)
    return Shape(*[base[k] for k in ("B", "H", "L", "d", "n_buckets", "n_rounds", "chunk",
                                     "causal", "dtype")])


def test_status_strings(lib):
    for code in range(8):
        assert lib.lsh_status_string(code)
    assert lib.lsh_status_string(6) == b"keys are not bucket*L + position"


@pytest.mark.parametrize("kw,expect", [
    (dict(d=32), 2), (dict(chunk=48), 1), (dict(n_buckets=3), 1), (dict(n_buckets=0), 1),
    (dict(n_rounds=0), 1), (dict(dtype=7), 1), (dict(chunk=128, L=256), 2),
    (dict(B=-1), 1), (dict(n_buckets=65536), 2), (dict(L=1 << 20, n_buckets=4096), 2),
    (dict(B=1, H=4096, n_rounds=16), 2),                        # 65 536 rows > 65 535
    (dict(B=1, H=512, L=65536, n_buckets=2, n_rounds=64), 2),   # B*H*L*R = 2^31
])
def test_invalid_shapes_are_rejected_before_launch(lib, kw, expect):
    s = _shape(**kw)
    fake = ctypes.c_void_p(256)  # never dereferenced: the shape check fails first
    rc = lib.lsh_hash(ctypes.byref(s), fake, fake, fake, None, None)
    assert rc == expect
    assert lib.lsh_workspace_size(ctypes.byref(s)) == 0


def test_null_and_misaligned_pointers_are_rejected(lib):
    s = _shape()
    fake = ctypes.c_void_p(256)
    assert lib.lsh_hash(ctypes.byref(s), None, fake, fake, None, None) == 1
    assert lib.lsh_hash(ctypes.byref(s), ctypes.c_void_p(258), fake, fake, None, None) == 1
    assert lib.lsh_sort(ctypes.byref(s), fake, None, None, 0, None) == 1
    assert lib.lsh_attend_fwd(ctypes.byref(s), fake, fake, fake, fake, None, None, None, None,
                              None, 0, None) == 1
    assert lib.lsh_attend_bwd(ctypes.byref(s), fake, fake, fake, fake, fake, fake, fake, fake,
                              None, None, 0, None) == 1
    assert lib.lsh_hash(None, fake, fake, fake, None, None) == 1


def test_host_forward_checks_arguments_before_any_copy(lib):
    s = _shape(B=1, H=4, L=1024, n_buckets=16, n_rounds=2)
    host = ctypes.c_void_p(4096)  # never dereferenced: every call below fails its checks first
    need = lib.lsh_forward_host_ws_size(ctypes.byref(s))
    # two head groups in flight: at least twice one group's q, v, o and keys
    assert need >= 2 * 2 * (1024 * 64 * 2 * 3 + 2 * 1024 * 8)
    assert lib.lsh_forward_host(ctypes.byref(s), None, host, host, host, None, host, need,
                                None) == 1
    assert lib.lsh_forward_host(ctypes.byref(s), host, host, host, host, None, None, need,
                                None) == 1
    assert lib.lsh_forward_host(ctypes.byref(s), host, host, host, host, None,
                                ctypes.c_void_p(4096), need - 1, None) == 4  # LSH_ERR_WORKSPACE
    empty = _shape(B=0)
    assert lib.lsh_forward_host(ctypes.byref(empty), None, None, None, None, None, None, 0,
                                None) == 0
    assert lib.lsh_forward_host_ws_size(ctypes.byref(empty)) == 0


def test_empty_shapes_are_no_ops(lib):
    for kw in (dict(B=0), dict(H=0), dict(L=0)):
        s = _shape(**kw)
        assert lib.lsh_hash(ctypes.byref(s), None, None, None, None, None) == 0
        assert lib.lsh_forward(ctypes.byref(s), None, None, None, None, None, None, None, None,
                               None, 0, None) == 0
        assert lib.lsh_workspace_size(ctypes.byref(s)) == 0


def test_workspace_size_covers_partials_and_gradients(lib):
    n_tok = 2 * 8 * 16384
    bwd = n_tok * 4 + 3 * n_tok * 64 * 4
    # tensor-core path (bf16, chunk 64): key scales, fp16 values and every
    # round's fp16 output and fp32 logsumexp
    s = _shape(B=2, H=8, L=16384, n_buckets=256, n_rounds=4)
    fwd = n_tok * 4 + n_tok * 128 + 4 * n_tok * (64 * 2 + 4)
    assert lib.lsh_workspace_size(ctypes.byref(s)) >= max(fwd, bwd)
    # CUDA-core path (f32): fp32 partials of the first R-1 rounds
    s = _shape(B=2, H=8, L=16384, n_buckets=256, n_rounds=4, dtype=0)
    fwd = 3 * n_tok * 65 * 4
    assert lib.lsh_workspace_size(ctypes.byref(s)) >= max(fwd, bwd)


def test_missing_library_fails_loudly(tmp_path):
    import lsh_attention_long_b200.lsh as mod
    saved = mod._lib
    mod._lib = None
    try:
        with pytest.raises(RuntimeError):
            mod.load_library(str(tmp_path / "absent.so"))
    finally:
        mod._lib = saved


def _align(x):
    return (x + 255) // 256 * 256


def _tc_need(n, R):
    """Tensor-core path: key scales and fp16 values, then (R > 1) every
    round's fp16 output and fp32 logsumexp."""
    base = _align(n * 4) + _align(n * 128)
    return base if R == 1 else base + _align(R * n * 128) + _align(R * n * 4)


@pytest.mark.parametrize("Lx,R,chunk,dtype,need", [
    # tensor-core path (bf16, chunk 64), two rounds, either side of 64 MiB
    (169408, 2, 64, 1, _tc_need(169408, 2)),
    (169472, 2, 64, 1, _tc_need(169472, 2)),
    # one round: only the key scales and fp16 values
    (508352, 1, 64, 1, _tc_need(508352, 1)),
    (508416, 1, 64, 1, _tc_need(508416, 1)),
    # CUDA-core path (f32), two rounds: one round of fp32 partials (256 + 4 B)
    (258048, 2, 64, 0, _align(258048 * 256) + _align(258048 * 4)),
    (258112, 2, 64, 0, _align(258112 * 256) + _align(258112 * 4)),
    # one problem (L=98304, R=4) on each path: 64.9 MB on the tensor-core
    # path, 76.7 MB on the CUDA-core path (chunk 32)
    (98304, 4, 64, 1, _tc_need(98304, 4)),
    (98304, 4, 32, 1, _align(3 * 98304 * 256) + _align(3 * 98304 * 4)),
])
def test_static_scratch_limit_follows_the_path(lib, Lx, R, chunk, dtype, need):
    """lsh_attend_fwd_static refuses exactly the problems whose need, on the
    path they take, exceeds its 64 MiB array.  An accepted problem goes on to
    look up the array, which fails on a machine without a GPU (LSH_ERR_CUDA),
    so it is probed only there."""
    P = ctypes.c_void_p
    lib.lsh_attend_fwd_static.argtypes = [ctypes.POINTER(Shape), P, P, P, P, P, P, P]
    lib.lsh_attend_fwd_static.restype = ctypes.c_int
    s = _shape(B=1, H=1, L=Lx, n_buckets=2, n_rounds=R, chunk=chunk, dtype=dtype)
    fake = ctypes.c_void_p(256)
    limit = 64 << 20
    if need > limit:
        assert lib.lsh_attend_fwd_static(ctypes.byref(s), fake, fake, fake, fake, fake, None,
                                         None) == 7
        return
    import torch
    if torch.cuda.is_available():
        pytest.skip("an accepted problem would launch on these placeholder pointers")
    assert lib.lsh_attend_fwd_static(ctypes.byref(s), fake, fake, fake, fake, fake, None,
                                     None) == 3


def test_ffn_checks_arguments_before_any_launch(lib):
    fake = ctypes.c_void_p(256)  # never dereferenced: every call below fails its checks first
    args = [fake] * 6
    assert lib.lsh_ffn_forward(128, 200, 512, 128, *args, fake, 1 << 20, None) == 2   # d_model % 256
    assert lib.lsh_ffn_forward(100, 256, 512, 128, *args, fake, 1 << 20, None) == 2   # tokens % 128
    assert lib.lsh_ffn_forward(128, 256, 512, 0, *args, fake, 1 << 20, None) == 1     # chunk
    assert lib.lsh_ffn_forward(128, 256, 512, 128, None, *args[1:], fake, 1 << 20, None) == 1
    assert lib.lsh_ffn_forward(128, 256, 512, 128, ctypes.c_void_p(264), *args[1:], fake,
                               1 << 20, None) == 1                                    # misaligned
    need = lib.lsh_ffn_ws_size(256, 256, 512, 128)
    assert need >= 128 * 512 * 2
    assert lib.lsh_ffn_forward(256, 256, 512, 128, *args, fake, need - 1, None) == 4  # workspace
    assert lib.lsh_ffn_forward(0, 256, 512, 128, None, None, None, None, None, None, None, 0,
                               None) == 0                                             # empty
