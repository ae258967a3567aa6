"""lsh_attend_fwd_static: the forward attention entry point that allocates nothing.

Some callers cannot allocate device memory when they run attention: a host
framework whose planner owns every buffer, a plugin executing inside another
runtime, or a latency-critical loop where cudaMalloc would synchronise the
device.  For them the library keeps its scratch in a built-in device array of
fixed size; this test calls that entry point through the C ABI and checks it
against lsh_attend_fwd with a caller-provided workspace, on two calls in a
row (different inputs), plus the size limit.

The file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

import lsh_attention_long_b200 as L
from lsh_attention_long_b200 import workloads as W
from lsh_attention_long_b200.lsh import Shape

pytestmark = pytest.mark.gpu

STATIC_BYTES = 64 << 20


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


def _run_static(lib, Q, V, keys, perm, nb, chunk, causal):
    B, H, Lx, d = Q.shape
    shape = L.make_shape(B, H, Lx, d, nb, keys.shape[0], chunk, causal, Q.dtype)
    O = torch.full_like(Q, float("nan"))
    lse = torch.full((B, H, Lx), float("nan"), dtype=torch.float32, device=Q.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.lsh_attend_fwd_static(ctypes.byref(shape), _p(Q), _p(V), _p(keys), _p(perm), _p(O),
                                   _p(lse), stream)
    assert rc == 0, L.lsh.STATUS.get(rc, rc)
    return O, lse


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_static_scratch_matches_workspace_entry_point(lib, dtype):
    cases = [  # two calls in a row on different problems; the second reuses the array
        (2, 4, 1024, 64, 4, 64, True, 11),
        (1, 3, 320, 16, 3, 32, False, 12),
    ]
    tol = 2e-2 if dtype == torch.bfloat16 else 2e-3
    for B, H, Lx, nb, R, chunk, causal, seed in cases:
        inp = W.make_random(B, H, Lx, 64, nb, R, dtype, seed=seed)
        Q, V, rot = (inp[k].cuda() for k in ("Q", "V", "rot"))
        keys, _ = L.lsh_hash(Q, rot, nb, want_buckets=False)
        perm = L.lsh_sort(keys, nb)
        O_ref, lse_ref, _, _ = L.lsh_attend_fwd(Q, V, keys, perm, nb, chunk, causal)
        O, lse = _run_static(lib, Q, V, keys, perm, nb, chunk, causal)
        torch.cuda.synchronize()
        assert L.lsh_device_status() == 0
        np.testing.assert_allclose(O.float().cpu().numpy(), O_ref.float().cpu().numpy(),
                                   rtol=0, atol=tol)
        np.testing.assert_allclose(lse.cpu().numpy(), lse_ref.cpu().numpy(), rtol=1e-6, atol=tol)


def test_static_scratch_rejects_problems_beyond_its_size(lib):
    # (R-1) * B*H*L * 65 floats: 1 * 8*8*4096 * 260 B = 68 MB > 64 MiB
    B, H, Lx, R = 8, 8, 4096, 2
    shape = L.make_shape(B, H, Lx, 64, 64, R, 64, True, torch.bfloat16)
    fake = ctypes.c_void_p(256)  # never dereferenced: the size check fails first
    rc = lib.lsh_attend_fwd_static(ctypes.byref(shape), fake, fake, fake, fake, fake, None, None)
    assert rc == 7
    assert lib.lsh_status_string(7).startswith(b"problem exceeds")
    assert (R - 1) * B * H * Lx * 65 * 4 > STATIC_BYTES
