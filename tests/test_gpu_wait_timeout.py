"""Failure detection on the device: a bounded wait that runs out.

Every wait in the kernels gives up after a limit of clock cycles, records
LSH_ERR_TIMEOUT in the device status word, lets its thread block finish its
in-flight copies and tensor-core operations, frees tensor memory and returns.
Here the tensor-core attention kernel's producers are told to stop before the
first tile of every thread block (a slot that nothing fills) with a limit of
about a millisecond: the call must report the timeout quickly, and the next
normal call must run green with the same results as before.  Nothing here
faults, traps or hangs the GPU.
"""

import time

import pytest
import torch

import lsh_attention_long_b200 as L
from lsh_attention_long_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from lsh_attention_long_b200 import build
    build.build()
    L.load_library()


def test_attention_wait_timeout_is_reported_and_recovered():
    B, H, Lx, nb, R = 1, 4, 2048, 32, 3
    inp = W.make_random(B, H, Lx, 64, nb, R, torch.bfloat16, seed=41)
    Q, V, rot = (inp[k].cuda() for k in ("Q", "V", "rot"))
    keys, _ = L.lsh_hash(Q, rot, nb, want_buckets=False)
    perm = L.lsh_sort(keys, nb)
    O_ref, lse_ref, _, _ = L.lsh_attend_fwd(Q, V, keys, perm, nb, 64, True)
    assert L.lsh_device_status() == 0
    L.lsh_set_wait_test(hold_tile=0, wait_cycles=2_000_000)  # ~1 ms at 2 GHz
    try:
        t0 = time.perf_counter()
        L.lsh_attend_fwd(Q, V, keys, perm, nb, 64, True)
        status = L.lsh_device_status()
        elapsed = time.perf_counter() - t0
    finally:
        L.lsh_set_wait_test(-1, 0)
    assert status == 5  # LSH_ERR_TIMEOUT
    # the short limit decided it, not the default one (about 2 s)
    assert elapsed < 1.0
    O, lse, _, _ = L.lsh_attend_fwd(Q, V, keys, perm, nb, 64, True)
    assert L.lsh_device_status() == 0
    assert torch.equal(O, O_ref)
    assert torch.equal(lse, lse_ref)


def test_wait_test_hook_rejects_a_negative_limit():
    with pytest.raises(L.LshError):
        L.lsh_set_wait_test(-1, -5)
