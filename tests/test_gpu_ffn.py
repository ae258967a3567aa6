"""GPU parity of the chunked feed-forward (lsh_ffn_forward) against the fp64 oracle.

Y = W2 max(0, W1 x + b1) + b2 per position, `chunk` positions at a time
("Reformer explainer", single section; "Reformer Language Models (Korean)",
Reformer overview).  bf16 inputs with fp32 accumulation: max-abs 2e-2.
"""

import numpy as np
import pytest
import torch

import lsh_attention_long_b200 as L
from lsh_attention_long_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from lsh_attention_long_b200 import build
    build.build()
    L.load_library()


def _np(t):
    return t.detach().float().cpu().numpy()


def _run(inp, chunk):
    t = {k: v.cuda() for k, v in inp.items()}
    Y = L.lsh_ffn_forward(t["X"], t["W1"], t["b1"], t["W2"], t["b2"], chunk)
    torch.cuda.synchronize()
    assert L.lsh_device_status() == 0
    return Y


@pytest.mark.parametrize("tokens,d_model,d_ff,chunk", [
    (128, 256, 256, 128),     # one tile, one chunk
    (512, 256, 512, 128),     # four chunks
    (1024, 512, 2048, 384),   # chunks of 384, 384, 256 (a ragged last chunk)
    (640, 768, 1024, 640),    # five token tiles, three output tiles
])
def test_ffn_matches_the_oracle(oracle, tokens, d_model, d_ff, chunk):
    inp = W.ffn_inputs(tokens, d_model, d_ff, seed=tokens + d_ff)
    Y = _run(inp, chunk)
    ref = oracle.ffn_forward(*(_np(inp[k]) for k in ("X", "W1", "b1", "W2", "b2")), chunk)
    np.testing.assert_allclose(_np(Y), ref, rtol=0, atol=TOL)


def test_chunking_does_not_change_the_device_result():
    """Every output row is computed by the same tiles whatever the chunk, so
    the result is bit-identical across chunk sizes."""
    inp = W.ffn_inputs(1024, 512, 2048, seed=3)
    Y1 = _run(inp, 128)
    Y2 = _run(inp, 1024)
    assert torch.equal(Y1, Y2)


def test_ffn_workload_at_full_size(oracle, parity_record):
    """The benchmarked workload (65 536 positions, 512 -> 2048 -> 512, chunks
    of 8192): 512 sampled positions, spread over every chunk, against the
    oracle."""
    w = W.FFN_WORKLOADS["ffn_bf16_L65536"]
    inp = W.ffn_inputs(w.tokens, w.d_model, w.d_ff)
    Y = _run(inp, w.chunk)
    rows = np.random.default_rng(0).choice(w.tokens, 512, replace=False)
    ref = oracle.ffn_forward(_np(inp["X"])[rows], *(_np(inp[k]) for k in ("W1", "b1", "W2", "b2")),
                             128)
    err = float(np.abs(_np(Y)[rows] - ref).max())
    parity_record.append({"workload": w.name, "positions_checked": len(rows), "max_abs": {"Y": err},
                          "tol": TOL})
    assert err <= TOL


def test_ffn_rejects_unsupported_shapes_and_empty_input_is_a_no_op():
    inp = W.ffn_inputs(128, 256, 256, seed=1)
    t = {k: v.cuda() for k, v in inp.items()}
    with pytest.raises(L.LshError):  # chunk not a multiple of 128
        L.lsh_ffn_forward(t["X"], t["W1"], t["b1"], t["W2"], t["b2"], 100)
    empty = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    Y = L.lsh_ffn_forward(empty, t["W1"], t["b1"], t["W2"], t["b2"], 128)
    assert Y.numel() == 0
    assert L.lsh_device_status() == 0


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------

def _run_bwd(inp, chunk, with_residual):
    t = {k: v.cuda() for k, v in inp.items()}
    R = torch.randn(t["X"].shape, generator=torch.Generator().manual_seed(9)).cuda() \
        if with_residual else None
    dX, g = L.lsh_ffn_backward(t["X"], t["W1"], t["b1"], t["W2"], t["dY"], chunk, R=R)
    torch.cuda.synchronize()
    assert L.lsh_device_status() == 0
    return dX, g, R


@pytest.mark.parametrize("tokens,d_model,d_ff,chunk,with_residual", [
    (128, 256, 256, 128, False),
    (512, 256, 512, 128, True),
    (1024, 512, 2048, 384, True),   # a ragged last chunk
])
def test_ffn_backward_matches_the_oracle(oracle, tokens, d_model, d_ff, chunk, with_residual):
    inp = W.ffn_inputs(tokens, d_model, d_ff, seed=7 * tokens + d_ff, backward=True)
    dX, g, R = _run_bwd(inp, chunk, with_residual)
    ref = oracle.ffn_backward(*(_np(inp[k]) for k in ("X", "W1", "b1", "W2", "dY")), chunk)
    rdX = ref[0] + (_np(R) if R is not None else 0.0)
    np.testing.assert_allclose(_np(dX), rdX, rtol=0, atol=TOL)
    # parameter gradients sum over every position: compare relative to their
    # scale (bf16 operands, fp32 accumulation)
    for name, r in zip(("dW1", "db1", "dW2", "db2"), ref[1:]):
        scale = max(1.0, float(np.abs(r).max()))
        np.testing.assert_allclose(_np(g[name]), r, rtol=0, atol=TOL * scale, err_msg=name)


def test_ffn_backward_at_full_size(oracle, parity_record):
    """The workload's backward: dX on 256 sampled positions and the bias
    gradients in full (they sum every position) against the oracle."""
    w = W.FFN_WORKLOADS["ffn_bf16_L65536"]
    inp = W.ffn_inputs(w.tokens, w.d_model, w.d_ff, backward=True)
    dX, g, _ = _run_bwd(inp, w.chunk, False)
    rows = np.random.default_rng(1).choice(w.tokens, 256, replace=False)
    ref = oracle.ffn_backward(_np(inp["X"])[rows], *(_np(inp[k]) for k in ("W1", "b1", "W2")),
                              _np(inp["dY"])[rows], 128)
    err = float(np.abs(_np(dX)[rows] - ref[0]).max())
    db2 = _np(inp["dY"]).astype(np.float64).sum(0)
    scale = max(1.0, float(np.abs(db2).max()))
    err_db2 = float(np.abs(_np(g["db2"]) - db2).max())
    parity_record.append({"workload": w.name + " (backward)", "positions_checked": len(rows),
                          "max_abs": {"dX": err, "db2": err_db2}, "tol": TOL})
    assert err <= TOL
    assert err_db2 <= TOL * scale


def test_back_to_back_chunks_are_ordered():
    """Consecutive GEMM launches overlap their set-up with the previous
    product's last tiles, and a later chunk's hidden product loads and
    multiplies before the previous output product has finished.  Repeated
    runs of eight chunks, with one workspace reused and nothing in between,
    must give bit-identical outputs (forward Y, backward dX: neither is
    accumulated with atomics), so no chunk reads or overwrites the hidden
    activation out of order."""
    inp = W.ffn_inputs(1024, 512, 2048, seed=21, backward=True)
    t = {k: v.cuda() for k, v in inp.items()}
    ws = L.ffn_workspace(1024, 512, 2048, 128, t["X"].device)
    first = None
    for _ in range(20):
        Y = L.lsh_ffn_forward(t["X"], t["W1"], t["b1"], t["W2"], t["b2"], 128, ws=ws)
        if first is None:
            first = Y.clone()
        else:
            assert torch.equal(Y, first)
    torch.cuda.synchronize()
    assert L.lsh_device_status() == 0
    dX0 = None
    for _ in range(10):
        dX, _ = L.lsh_ffn_backward(t["X"], t["W1"], t["b1"], t["W2"], t["dY"], 128)
        if dX0 is None:
            dX0 = dX.clone()
        else:
            assert torch.equal(dX, dX0)
    torch.cuda.synchronize()
    assert L.lsh_device_status() == 0
