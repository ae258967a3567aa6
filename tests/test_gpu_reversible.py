"""GPU parity of the reversible residual block around LSH attention.

Y1 = X1 + F(X2), Y2 = X2 + G(Y1), with F the LSH attention of X2 (its own
query = key and value, H heads of 64) and G the chunked feed-forward; the
backward recomputes X2 = Y2 - G(Y1) and X1 = Y1 - F(X2) from the outputs
alone (the Reformer abstract: reversible residual layers store activations
once; the explainer: activations recomputed in the backward pass).  The
buckets of X2's hash are held constant in the backward.

Each sublayer is compared with the fp64 oracle fed the input the GPU used
(the GPU's buckets for F, the bf16 copy of Y1 for G), so that a near-tie
bucket flip or a bf16 rounding upstream cannot masquerade as an error of the
sublayer: G's max(0, .) is a decision floating point takes, and a
pre-activation within a bf16 rounding of zero would otherwise switch a
hidden unit's whole gradient on one side only.  F's backward likewise gets
the bf16 copy of dX1 that the GPU's attention backward consumes.  bf16 sublayers with fp32 accumulation: max-abs 2e-2; parameter
gradients (sums over every position) relative to their largest entry.
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
    return t.detach().double().cpu().numpy()


def _case(B, Lx, H, nb, R, d_ff, seed):
    D = H * 64
    g = torch.Generator().manual_seed(seed)
    # residual-stream inputs that bf16 represents exactly, so F sees X2 itself
    X1 = torch.randn(B, Lx, D, generator=g).to(torch.bfloat16).float()
    X2 = torch.randn(B, Lx, D, generator=g).to(torch.bfloat16).float()
    dY1 = torch.randn(B, Lx, D, generator=g)
    dY2 = torch.randn(B, Lx, D, generator=g)
    rot = torch.randn(R, 64, nb // 2, generator=g).to(torch.bfloat16)
    ffn = W.ffn_inputs(B * Lx, D, d_ff, seed=seed + 100)
    return dict(X1=X1, X2=X2, dY1=dY1, dY2=dY2, rot=rot,
                **{k: ffn[k] for k in ("W1", "b1", "W2", "b2")})


def _check(oracle, c, H, nb, chunk, causal, fchunk, parity_record=None, name=None):
    t = {k: v.cuda() for k, v in c.items()}
    w = (t["W1"], t["b1"], t["W2"], t["b2"])
    Y1, Y2, keys, perm = L.lsh_rev_forward(t["X1"], t["X2"], t["rot"], *w, H, nb, chunk, causal,
                                           fchunk)
    X1r, X2r, dX1, dX2, g = L.lsh_rev_backward(Y1, Y2, t["dY1"], t["dY2"], keys, perm, *w, H, nb,
                                               chunk, causal, fchunk)
    torch.cuda.synchronize()
    assert L.lsh_device_status() == 0
    B, Lx, D = c["X1"].shape
    W1, b1, W2, b2 = (_np(c[k]) for k in ("W1", "b1", "W2", "b2"))
    keys_np = keys.cpu().numpy().view(np.uint32)
    perm_np = perm.cpu().numpy()
    X1, X2 = _np(c["X1"]), _np(c["X2"])
    # the hash of X2: bucket ids bit-exact outside near ties
    _, ob, tie = oracle.lsh_hash(oracle._heads(X2, H), _np(c["rot"]), nb)
    gb = keys_np // np.uint32(Lx)
    assert not ((gb != ob) & (tie == 0)).any()
    assert np.array_equal(perm_np, oracle.lsh_sort(keys_np))
    err = {}
    # forward: F with the GPU's buckets; G of the bf16 Y1 the GPU fed it
    Y1_ref = X1 + oracle.rev_attention(X2, keys_np, perm_np, H, chunk, causal)
    err["Y1"] = float(np.abs(_np(Y1) - Y1_ref).max())
    y1b = _np(Y1.to(torch.bfloat16)).reshape(B * Lx, D)
    Y2_ref = X2 + oracle.ffn_forward(y1b, W1, b1, W2, b2, fchunk).reshape(B, Lx, D)
    err["Y2"] = float(np.abs(_np(Y2) - Y2_ref).max())
    # backward from the GPU's outputs, the oracle in fp64, G evaluated at the
    # bf16 copy of Y1 the GPU fed it (its max(0, .) mask is decided there)
    ref = oracle.rev_backward(_np(Y1), _np(Y2), _np(c["dY1"]), _np(c["dY2"]), keys_np, perm_np,
                              H, chunk, causal, W1, b1, W2, b2, fchunk,
                              g_input=y1b.reshape(B, Lx, D),
                              f_upstream=_np(dX1.to(torch.bfloat16)))
    err["X1"] = float(np.abs(_np(X1r) - X1).max())
    err["X2"] = float(np.abs(_np(X2r) - X2).max())
    err["dX1"] = float(np.abs(_np(dX1) - ref[2]).max())
    err["dX2"] = float(np.abs(_np(dX2) - ref[3]).max())
    rel = {}
    for name_, r in zip(("dW1", "db1", "dW2", "db2"), ref[4:]):
        rel[name_] = float(np.abs(_np(g[name_]) - r).max() / max(1.0, np.abs(r).max()))
    if parity_record is not None:
        parity_record.append({"workload": name, "max_abs": err, "max_rel_param_grads": rel,
                              "near_ties": int(tie.sum()), "tol": TOL})
    for k, e in err.items():
        assert e <= TOL, (k, e)
    for k, e in rel.items():
        assert e <= TOL, (k, e)


@pytest.mark.parametrize("B,Lx,H,nb,R,d_ff,chunk,causal,fchunk", [
    (1, 512, 4, 16, 2, 512, 64, True, 128),
    (2, 256, 4, 8, 3, 256, 64, False, 384),    # a ragged last feed-forward chunk
    (1, 1024, 8, 32, 2, 1024, 32, True, 512),  # the CUDA-core attention path (chunk 32)
])
def test_reversible_block_matches_the_oracle(oracle, B, Lx, H, nb, R, d_ff, chunk, causal, fchunk):
    _check(oracle, _case(B, Lx, H, nb, R, d_ff, seed=Lx + H + R), H, nb, chunk, causal, fchunk)


def test_reversible_block_at_a_larger_size(oracle, parity_record):
    """L=4096, 8 heads (d_model 512), 256 buckets, 4 rounds, causal, d_ff 2048,
    feed-forward chunks of 1024."""
    _check(oracle, _case(1, 4096, 8, 256, 4, 2048, seed=5), 8, 256, 64, True, 1024,
           parity_record, "rev_bf16_L4096")
