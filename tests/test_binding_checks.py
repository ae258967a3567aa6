"""The Python binding rejects tensors of the wrong shape, type or memory
space before anything reaches the library (which takes plain pointers and
could not tell).  These run on the CPU: every check fires before a call."""
import pytest
import torch

import lsh_attention_long_b200 as L

B, H, N, D, NB, R = 1, 2, 128, 64, 16, 2


def _inputs(dtype=torch.bfloat16):
    Q = torch.zeros(B, H, N, D, dtype=dtype)
    return Q, torch.zeros_like(Q), torch.zeros(R, D, NB // 2, dtype=dtype)


def test_host_tensors_are_refused_where_device_memory_is_expected():
    Q, V, rot = _inputs()
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        L.lsh_forward(Q, V, rot, NB, 64, True)
    keys = torch.zeros(R, B, H, N, dtype=torch.int32)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        L.lsh_sort(keys, NB)


def test_mismatched_shapes_are_refused():
    Q, V, rot = _inputs()
    with pytest.raises(ValueError, match="V has shape"):
        L.lsh_forward(Q, V[:, :, :64], rot, NB, 64, True)
    with pytest.raises(ValueError, match="rot has shape"):
        L.lsh_forward(Q, V, rot[:, :, :4], NB, 64, True)
    keys = torch.zeros(R, B, H, N, dtype=torch.int32)
    with pytest.raises(ValueError, match="perm has shape"):
        L.lsh_attend_fwd(Q, V, keys, keys[:, :, :1], NB, 64, True)
    with pytest.raises(ValueError, match="lse has shape"):
        L.lsh_attend_bwd(Q, V, Q, Q, keys, keys, torch.zeros(B, H, N + 1), NB, 64, True)


def test_wrong_types_are_refused():
    Q, V, rot = _inputs()
    with pytest.raises(ValueError, match="V has dtype"):
        L.lsh_forward(Q, V.float(), rot, NB, 64, True)
    with pytest.raises(ValueError, match="keys has dtype"):
        L.lsh_sort(torch.zeros(R, B, H, N, dtype=torch.int64), NB)
    keys = torch.zeros(R, B, H, N, dtype=torch.int32)
    with pytest.raises(ValueError, match="dO has dtype"):
        L.lsh_attend_bwd(Q, V, Q, Q.float(), keys, keys, torch.zeros(B, H, N), NB, 64, True)
    with pytest.raises(ValueError, match="o_part has dtype"):
        L.lsh_combine(torch.zeros(R, B, H, N, D, dtype=torch.float64), torch.zeros(R, B, H, N),
                      torch.bfloat16)


def test_non_contiguous_tensors_are_refused():
    Q, V, rot = _inputs()
    with pytest.raises(ValueError, match="must be contiguous"):
        L.lsh_forward(Q.transpose(1, 2).contiguous().transpose(1, 2), V, rot, NB, 64, True)


def test_one_bucket_does_not_read_the_rotation():
    Q, V, _ = _inputs()
    # any rotation tensor is accepted (it is never read); the device check still fires
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        L.lsh_forward(Q, V, torch.zeros(R, 1, 1, dtype=torch.float64), 1, 64, True)


def test_host_buffer_forward_wants_host_inputs_and_a_device_workspace():
    Q, V, rot = _inputs()
    with pytest.raises(ValueError, match="O has shape"):
        L.lsh_forward_host(Q, V, rot, NB, 64, True, O=torch.zeros(B, H, N, D + 1,
                                                                   dtype=Q.dtype))
    with pytest.raises(ValueError, match="ws must be a CUDA tensor"):
        L.lsh_forward_host(Q, V, rot, NB, 64, True, ws=torch.zeros(16, dtype=torch.uint8))


def test_binding_argument_counts_match_the_header():
    """Every entry point's ctypes signature has as many arguments as its
    declaration in include/lsh.h (the C functions take plain pointers, so a
    miscounted signature would pass the wrong value to the library)."""
    import os
    import re
    from lsh_attention_long_b200 import lsh as M
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    text = open(os.path.join(root, "include", "lsh.h")).read()
    decls = {m.group(1): m.group(2) for m in
             re.finditer(r"LSH_API\s+[\w\s\*]+?\b(\w+)\s*\(([^)]*)\)", text)}
    lib = M.load_library() if os.path.exists(M.LIB_PATH) else None
    if lib is None:
        pytest.skip("library not built")
    for name, params in decls.items():
        n = 0 if params.strip() in ("", "void") else params.count(",") + 1
        assert len(getattr(lib, name).argtypes or []) == n, name
