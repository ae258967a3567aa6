"""lsh_attend_fwd_static: the forward attention entry point that allocates nothing.

Some callers cannot allocate device memory when they run attention: a host
framework whose planner owns every buffer, a plugin executing inside another
runtime, or a latency-critical loop where cudaMalloc would synchronise the
device.  For them the library keeps its scratch in a built-in device array of
fixed size.  These tests call that entry point through the C ABI and check it
against lsh_attend_fwd with a caller-provided workspace on two calls in a row
that take the same kernel path (the second call finds the first one's state
in the shared array), and check the size limit with the need of the path a
case actually takes.

The file is named so that pytest collects it last.
"""

import ctypes

import pytest
import torch

import lsh_attention_long_b200 as L
from lsh_attention_long_b200 import workloads as W
from lsh_attention_long_b200.lsh import Shape

pytestmark = pytest.mark.gpu

STATIC_BYTES = 64 << 20


def _align(x):
    return (x + 255) // 256 * 256


def static_need(B, H, Lx, R, chunk, dtype):
    """Scratch bytes the header documents for lsh_attend_fwd_static."""
    n = B * H * Lx
    if dtype == torch.bfloat16 and chunk == 64:  # tensor-core path
        base = _align(n * 4) + _align(n * 64 * 2)  # key scales, fp16 values
        if R == 1:
            return base
        return base + _align(R * n * 64 * 2) + _align(R * n * 4)
    if R == 1:  # CUDA-core path
        return 0
    return _align((R - 1) * n * 64 * 4) + _align((R - 1) * n * 4)


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from lsh_attention_long_b200 import build
    build.build()
    lib = L.load_library()
    P = ctypes.c_void_p
    lib.lsh_attend_fwd_static.argtypes = [ctypes.POINTER(Shape), P, P, P, P, P, P, P]
    lib.lsh_attend_fwd_static.restype = ctypes.c_int
    return lib


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_static(lib, shape, Q, V, keys, perm, O, lse):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.lsh_attend_fwd_static(ctypes.byref(shape), _p(Q), _p(V), _p(keys), _p(perm),
                                     _p(O), _p(lse), stream)


def _same_as_workspace_call(lib, B, H, Lx, nb, R, chunk, causal, dtype, seed):
    """Runs both entry points on one problem; their O and lse must be equal
    bit for bit (the same kernels, only the scratch differs)."""
    assert static_need(B, H, Lx, R, chunk, dtype) <= STATIC_BYTES
    inp = W.make_random(B, H, Lx, 64, nb, R, dtype, seed=seed)
    Q, V, rot = (inp[k].cuda() for k in ("Q", "V", "rot"))
    keys, _ = L.lsh_hash(Q, rot, nb, want_buckets=False)
    perm = L.lsh_sort(keys, nb)
    O_ref, lse_ref, _, _ = L.lsh_attend_fwd(Q, V, keys, perm, nb, chunk, causal)
    shape = L.make_shape(B, H, Lx, 64, nb, R, chunk, causal, Q.dtype)
    O = torch.full_like(Q, float("nan"))
    lse = torch.full((B, H, Lx), float("nan"), dtype=torch.float32, device=Q.device)
    rc = _call_static(lib, shape, Q, V, keys, perm, O, lse)
    assert rc == 0, L.lsh.STATUS.get(rc, rc)
    torch.cuda.synchronize()
    assert L.lsh_device_status() == 0
    assert torch.equal(O, O_ref)
    assert torch.equal(lse, lse_ref)


@pytest.mark.parametrize("dtype,chunk2", [(torch.bfloat16, 64), (torch.float32, 32)])
def test_static_scratch_matches_workspace_entry_point(lib, dtype, chunk2):
    """Two calls in a row on one path: a larger problem leaves its per-round
    partials in the shared array, then a smaller one must not read any of
    them."""
    _same_as_workspace_call(lib, 2, 4, 2048, 64, 4, 64, True, dtype, seed=11)
    _same_as_workspace_call(lib, 1, 3, 320, 16, 3, chunk2, False, dtype, seed=12)


def test_static_scratch_capacity_follows_the_path(lib):
    """Problems that fit one path's formula but not the other's.  B=1 H=2
    L=49152 R=4: the tensor-core path (bf16, chunk 64) needs 64.9 MB and runs,
    the CUDA-core path (f32, or bf16 with chunk 32) needs 76.7 MB and is
    refused.  B=1 H=1 L=254976 R=2: the CUDA-core path needs 66.3 MB and runs,
    the tensor-core path needs 101 MB and is refused."""
    fake = ctypes.c_void_p(256)  # never dereferenced: the size check fails first
    refused = [(1, 2, 49152, 4, 64, torch.float32), (1, 2, 49152, 4, 32, torch.bfloat16),
               (1, 1, 254976, 2, 64, torch.bfloat16)]
    for B, H, Lx, R, chunk, dtype in refused:
        assert static_need(B, H, Lx, R, chunk, dtype) > STATIC_BYTES
        shape = L.make_shape(B, H, Lx, 64, 64, R, chunk, True, dtype)
        rc = lib.lsh_attend_fwd_static(ctypes.byref(shape), fake, fake, fake, fake, fake, None,
                                       None)
        assert rc == 7
    assert lib.lsh_status_string(7).startswith(b"problem exceeds")
    _same_as_workspace_call(lib, 1, 2, 49152, 64, 4, 64, True, torch.bfloat16, seed=21)
    _same_as_workspace_call(lib, 1, 1, 254976, 64, 2, 64, True, torch.float32, seed=22)
    _same_as_workspace_call(lib, 1, 4, 65536, 64, 1, 64, True, torch.bfloat16, seed=23)
