"""GPU parity: every step of the CUDA path against the fp64 CPU oracle.

Bit-exact for integers (bucket ids away from near ties, keys, permutations);
max-abs 2e-3 (f32 inputs) or 2e-2 (bf16 inputs, fp32 accumulation) for
outputs, logsumexps and gradients.  The oracle is fed the GPU's own keys and
permutations so that a legitimate near-tie flip cannot cause a tolerance
failure; near ties (top two rotated projections within 1e-5 relative) are
counted and reported.
"""

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import lsh_attention_long_b200 as L
from lsh_attention_long_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 2e-3, torch.bfloat16: 2e-2}
# host threads for the oracle over independent (b, h) heads; its C routines
# release the GIL
WORKERS = max(1, min(16, os.cpu_count() or 1))


def _pmap(fn, items):
    with ThreadPoolExecutor(max_workers=WORKERS) as ex:
        return list(ex.map(fn, items))


def _heads(B, H):
    return [(b, h) for b in range(B) for h in range(H)]


def _err(got, ref, atol, rtol=0.0):
    """(largest |got - ref|, whether every element is within atol + rtol |ref|)."""
    if got.size == 0:
        return 0.0, True
    d = np.abs(got.astype(np.float64) - ref)
    return float(d.max()), bool((d <= atol + rtol * np.abs(ref)).all())


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from lsh_attention_long_b200 import build
    build.build()
    L.load_library()


def _np(t):
    return t.detach().float().cpu().numpy()


def _check_status():
    assert L.lsh_device_status() == 0


def check_hash(oracle, Q, rot, nb, keys, buckets, sample=None):
    """Bucket ids bit-exact except near ties; keys = bucket*L + position."""
    Qn = _np(Q)
    Ln = Q.shape[2]
    kb = buckets.cpu().numpy()
    kk = keys.cpu().numpy().view(np.uint32)
    pos = np.arange(Ln, dtype=np.uint64)
    assert np.array_equal(kk.astype(np.uint64), kb.astype(np.uint64) * Ln + pos)
    if sample is not None:
        flat = Qn.reshape(-1, Qn.shape[-1])
        idx = np.random.default_rng(0).choice(flat.shape[0], size=min(sample, flat.shape[0]),
                                              replace=False)
        _, ob, tie = oracle.lsh_hash(flat[idx][None, None], _np(rot), nb)
        gb = kb.reshape(kb.shape[0], -1)[:, idx]
        ob, tie = ob[:, 0, 0], tie[:, 0, 0]
    else:
        _, ob, tie = oracle.lsh_hash(Qn, _np(rot), nb)
        gb = kb
    bad = (gb != ob) & (tie == 0)
    assert not bad.any(), f"{int(bad.sum())} bucket mismatches outside near ties"
    return int(tie.sum())


def hash_every_token(oracle, Q, rot, nb, keys):
    """Every token's bucket id in every round against the oracle, head by
    head over host threads.  Returns the near-tie count and how many near
    ties the GPU resolved the other way; any other mismatch fails."""
    Qn, rotn = _np(Q), _np(rot)
    B, H, Ln = Qn.shape[:3]
    kk = keys.cpu().numpy().view(np.uint32)
    gb = (kk // np.uint32(Ln)).astype(np.int64)
    assert np.array_equal(kk % np.uint32(Ln),
                          np.broadcast_to(np.arange(Ln, dtype=np.uint32), kk.shape))

    def one(bh):
        b, h = bh
        _, ob, tie = oracle.lsh_hash(Qn[b:b + 1, h:h + 1], rotn, nb)
        diff = gb[:, b:b + 1, h:h + 1] != ob
        return int((diff & (tie == 0)).sum()), int(tie.sum()), int((diff & (tie != 0)).sum())

    res = _pmap(one, _heads(B, H))
    bad = sum(r[0] for r in res)
    assert bad == 0, f"{bad} bucket mismatches outside near ties"
    return sum(r[1] for r in res), sum(r[2] for r in res)


def attention_every_head(oracle, Q, V, keys, perm, chunk, causal, O, lse, o_part=None,
                         lse_r=None):
    """O and lse (and, when given, the per-round o_part and lse_r) of every
    (b, h) head against the oracle fed the GPU's keys and permutations, head
    by head over host threads.  Returns the largest error of each output."""
    tol = TOL[Q.dtype]
    Qn, Vn = _np(Q), _np(V)
    keys_np = keys.cpu().numpy().view(np.uint32)
    perm_np = perm.cpu().numpy()
    gO, glse = _np(O), _np(lse)
    gop = None if o_part is None else _np(o_part)
    glr = None if lse_r is None else _np(lse_r)

    def one(bh):
        b, h = bh
        op, lr = oracle.lsh_attend_fwd(Qn[b:b + 1, h:h + 1], Vn[b:b + 1, h:h + 1],
                                       keys_np[:, b:b + 1, h:h + 1],
                                       perm_np[:, b:b + 1, h:h + 1], chunk, causal)
        Oo, lo = oracle.lsh_combine(op, lr)
        e = {"O": _err(gO[b, h], Oo[0, 0], tol), "lse": _err(glse[b, h], lo[0, 0], tol, 1e-6)}
        if gop is not None:
            e["o_part"] = _err(gop[:, b, h], op[:, 0, 0], tol)
            e["lse_r"] = _err(glr[:, b, h], lr[:, 0, 0], tol, 1e-6)
        return bh, e

    return _collect(_pmap(one, _heads(*Qn.shape[:2])))


def _collect(per_head):
    """Largest error per output over heads; fails naming the first head out
    of tolerance."""
    worst = {}
    for bh, e in per_head:
        for k, (m, ok) in e.items():
            assert ok, f"{k} of head {bh} differs from the oracle by {m}"
            worst[k] = max(worst.get(k, 0.0), m)
    return worst


def run_steps(inp, nb, chunk, causal):
    Q, V, rot = (inp[k].cuda() for k in ("Q", "V", "rot"))
    keys, buckets = L.lsh_hash(Q, rot, nb)
    perm = L.lsh_sort(keys, nb)
    _, _, o_part, lse_r = L.lsh_attend_fwd(Q, V, keys, perm, nb, chunk, causal, combine=False)
    O, lse, _, _ = L.lsh_attend_fwd(Q, V, keys, perm, nb, chunk, causal)
    torch.cuda.synchronize()
    _check_status()
    return dict(Q=Q, V=V, rot=rot, keys=keys, buckets=buckets, perm=perm, o_part=o_part,
                lse_r=lse_r, O=O, lse=lse)


def check_all(oracle, inp, nb, chunk, causal, heads=None):
    g = run_steps(inp, nb, chunk, causal)
    tol = TOL[inp["Q"].dtype]
    check_hash(oracle, g["Q"], g["rot"], nb, g["keys"], g["buckets"])
    keys_np = g["keys"].cpu().numpy().view(np.uint32)
    assert np.array_equal(g["perm"].cpu().numpy(), oracle.lsh_sort(keys_np))
    Qn, Vn = _np(g["Q"]), _np(g["V"])
    perm_np = g["perm"].cpu().numpy()
    if heads is not None:  # restrict the attention comparison to some (b, h)
        b, h = heads
        Qn, Vn = Qn[b:b + 1, h:h + 1], Vn[b:b + 1, h:h + 1]
        keys_np = keys_np[:, b:b + 1, h:h + 1]
        perm_np = perm_np[:, b:b + 1, h:h + 1]
        sl = (slice(b, b + 1), slice(h, h + 1))
    else:
        sl = (slice(None), slice(None))
    o_part, lse_r = oracle.lsh_attend_fwd(Qn, Vn, keys_np, perm_np, chunk, causal)
    O, lse = oracle.lsh_combine(o_part, lse_r)
    np.testing.assert_allclose(_np(g["o_part"])[:, sl[0], sl[1]], o_part, rtol=0, atol=tol)
    np.testing.assert_allclose(_np(g["lse_r"])[:, sl[0], sl[1]], lse_r, rtol=1e-6, atol=tol)
    np.testing.assert_allclose(_np(g["O"])[sl], O, rtol=0, atol=tol)
    np.testing.assert_allclose(_np(g["lse"])[sl], lse, rtol=1e-6, atol=tol)
    # standalone combine of the GPU partials equals the fused / online combine
    # up to one output ulp (two fp32 summation orders can round to adjacent
    # bf16 values: 2^-7 relative)
    Oc, lsec = L.lsh_combine(g["o_part"], g["lse_r"], g["Q"].dtype)
    torch.cuda.synchronize()
    ulp = 2.0 ** -7 if g["Q"].dtype == torch.bfloat16 else 2.0 ** -20
    np.testing.assert_allclose(_np(Oc), _np(g["O"]), rtol=ulp, atol=tol / 4)
    np.testing.assert_allclose(_np(lsec), _np(g["lse"]), rtol=1e-6, atol=1e-5)
    return g


CASES = [
    # B, H, L, nb, R, chunk, causal
    (1, 3, 320, 16, 2, 64, True),     # 5 chunks (odd), ragged hash tiles
    (2, 1, 96, 6, 3, 32, False),      # nb/2 = 3, three chunks
    (1, 2, 64, 8, 2, 64, True),       # one chunk: window is the chunk once
    (1, 2, 128, 4, 2, 64, False),     # two chunks: each sees the whole row
    (1, 1, 256, 1, 2, 64, True),      # one bucket
    (1, 2, 256, 2, 3, 16, False),     # hyperplane hash, small chunks
    (1, 1, 256, 1024, 1, 64, False),  # more buckets than tokens: lone tokens
    (1, 2, 64, 4, 1, 4, True),        # tiny chunks
    (1, 1, 512, 32768, 1, 64, True),  # the largest bucket count
    (1, 2, 384, 8, 5, 64, True),      # five rounds of fp16 partials, combined
    (2, 1, 256, 4, 8, 64, False),     # eight rounds, non-causal
    (1, 2, 384, 8, 3, 64, True),      # three rounds (each round count has its own combine)
    (1, 1, 512, 16, 4, 64, False),    # four rounds
    (1, 2, 256, 8, 6, 64, True),      # six rounds
    (1, 1, 320, 16, 7, 64, False),    # seven rounds, ragged last tile
    (1, 1, 256, 96, 2, 64, True),     # nb/2 = 48, not a power of two: CUDA-core hash
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,H,Lx,nb,R,chunk,causal", CASES)
def test_small_shapes(oracle, dtype, B, H, Lx, nb, R, chunk, causal):
    inp = W.make_random(B, H, Lx, 64, nb, R, dtype, seed=Lx + nb + R)
    check_all(oracle, inp, nb, chunk, causal)


def test_workload_fwd_f32_L1024(oracle, parity_record):
    w = W.WORKLOADS["fwd_f32_L1024"]
    g = check_all(oracle, W.make_inputs(w), w.n_buckets, w.chunk, w.causal)
    ties, flips = hash_every_token(oracle, g["Q"], g["rot"], w.n_buckets, g["keys"])
    worst = attention_every_head(oracle, g["Q"], g["V"], g["keys"], g["perm"], w.chunk, w.causal,
                                 g["O"], g["lse"], g["o_part"], g["lse_r"])
    parity_record.append({"workload": w.name, "heads": 1, "tokens_hashed": w.L,
                          "near_ties": ties, "near_tie_flips": flips, "rows_sorted": 1,
                          "max_abs": worst, "tol": TOL[torch.float32]})


@pytest.mark.parametrize("name", ["fwd_bf16_L4096", "fwd_bf16_L16384_clustered"])
def test_workload_bf16_every_head(oracle, parity_record, name):
    """Every step of the forward on every (b, h) head of the workload: bucket
    ids of every token, permutations of every row, per-round partials and the
    combined O and lse."""
    w = W.WORKLOADS[name]
    g = run_steps(W.make_inputs(w), w.n_buckets, w.chunk, w.causal)
    ties, flips = hash_every_token(oracle, g["Q"], g["rot"], w.n_buckets, g["keys"])
    keys_np = g["keys"].cpu().numpy().view(np.uint32)
    assert np.array_equal(g["perm"].cpu().numpy(), oracle.lsh_sort(keys_np))
    worst = attention_every_head(oracle, g["Q"], g["V"], g["keys"], g["perm"], w.chunk, w.causal,
                                 g["O"], g["lse"], g["o_part"], g["lse_r"])
    parity_record.append({"workload": name, "heads": w.B * w.H, "tokens_hashed": w.B * w.H * w.L,
                          "near_ties": ties, "near_tie_flips": flips, "rows_sorted":
                          w.n_rounds * w.B * w.H, "max_abs": worst, "tol": TOL[g["Q"].dtype]})


def test_workload_L65536_as_benchmarked(oracle, parity_record):
    """The benchmarked forward (one lsh_forward call, the online combine) at
    full size: every token's bucket ids in all 8 rounds, every row's
    permutation, O and lse of all 8 heads."""
    w = W.WORKLOADS["fwd_bf16_L65536"]
    inp = W.make_inputs(w)
    Q, V, rot = (inp[k].cuda() for k in ("Q", "V", "rot"))
    out = L.lsh_forward(Q, V, rot, w.n_buckets, w.chunk, w.causal, want_buckets=True)
    torch.cuda.synchronize()
    _check_status()
    assert torch.equal(out["keys"] // w.L, out["buckets"])
    ties, flips = hash_every_token(oracle, Q, rot, w.n_buckets, out["keys"])
    keys_np = out["keys"].cpu().numpy().view(np.uint32)
    assert np.array_equal(out["perm"].cpu().numpy(), oracle.lsh_sort(keys_np))
    worst = attention_every_head(oracle, Q, V, out["keys"], out["perm"], w.chunk, w.causal,
                                 out["O"], out["lse"])
    parity_record.append({"workload": w.name, "heads": w.B * w.H,
                          "tokens_hashed": w.B * w.H * w.L, "near_ties": ties,
                          "near_tie_flips": flips, "rows_sorted": w.n_rounds * w.B * w.H,
                          "max_abs": worst, "tol": 2e-2})


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,H,Lx,nb,R,causal", [(2, 3, 1024, 16, 2, True),
                                                 (1, 1, 512, 8, 3, False),
                                                 (1, 8, 4096, 64, 2, True),
                                                 (1, 5, 2048, 32, 2, False)])
def test_host_buffer_forward_equals_device_forward(dtype, B, H, Lx, nb, R, causal):
    """lsh_forward_host (pinned host buffers, head groups pipelined through
    the device) gives exactly lsh_forward's O and lse."""
    inp = W.make_random(B, H, Lx, 64, nb, R, dtype, seed=Lx + H)
    host = {k: inp[k].pin_memory() for k in ("Q", "V", "rot")}
    ref = L.lsh_forward(*(host[k].cuda() for k in ("Q", "V", "rot")), nb, 64, causal)
    O, lse = L.lsh_forward_host(host["Q"], host["V"], host["rot"], nb, 64, causal)
    torch.cuda.synchronize()
    _check_status()
    assert torch.equal(O, ref["O"].cpu())
    assert torch.equal(lse, ref["lse"].cpu())


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------

def check_bwd(oracle, inp, nb, chunk, causal, heads=None):
    dtype = inp["Q"].dtype
    Q, V, rot, dO = (inp[k].cuda() for k in ("Q", "V", "rot", "dO"))
    out = L.lsh_forward(Q, V, rot, nb, chunk, causal)
    dQ, dV = L.lsh_attend_bwd(Q, V, out["O"], dO, out["keys"], out["perm"], out["lse"], nb,
                              chunk, causal)
    torch.cuda.synchronize()
    _check_status()
    keys_np = out["keys"].cpu().numpy().view(np.uint32)
    perm_np = out["perm"].cpu().numpy()
    Qn, Vn, dOn = _np(Q), _np(V), _np(dO)
    gQ, gV = _np(dQ), _np(dV)
    if heads is not None:
        b, h = heads
        Qn, Vn, dOn = (x[b:b + 1, h:h + 1] for x in (Qn, Vn, dOn))
        keys_np, perm_np = keys_np[:, b:b + 1, h:h + 1], perm_np[:, b:b + 1, h:h + 1]
        gQ, gV = gQ[b:b + 1, h:h + 1], gV[b:b + 1, h:h + 1]
    rQ, rV = oracle.lsh_attend_bwd(Qn, Vn, dOn, keys_np, perm_np, chunk, causal)
    tol = TOL[dtype]
    np.testing.assert_allclose(gV, rV, rtol=0, atol=tol)
    np.testing.assert_allclose(gQ, rQ, rtol=0, atol=tol)


def check_bwd_every_head(oracle, w, inp):
    """Forward and backward of a full-size workload, every (b, h) head: the
    hash of every token, every row's permutation, O and lse, dQ and dV."""
    Q, V, rot, dO = (inp[k].cuda() for k in ("Q", "V", "rot", "dO"))
    out = L.lsh_forward(Q, V, rot, w.n_buckets, w.chunk, w.causal)
    dQ, dV = L.lsh_attend_bwd(Q, V, out["O"], dO, out["keys"], out["perm"], out["lse"],
                              w.n_buckets, w.chunk, w.causal)
    torch.cuda.synchronize()
    _check_status()
    ties, flips = hash_every_token(oracle, Q, rot, w.n_buckets, out["keys"])
    keys_np = out["keys"].cpu().numpy().view(np.uint32)
    perm_np = out["perm"].cpu().numpy()
    assert np.array_equal(perm_np, oracle.lsh_sort(keys_np))
    worst = attention_every_head(oracle, Q, V, out["keys"], out["perm"], w.chunk, w.causal,
                                 out["O"], out["lse"])
    tol = TOL[Q.dtype]
    Qn, Vn, dOn, gQ, gV = (_np(t) for t in (Q, V, dO, dQ, dV))

    def one(bh):
        b, h = bh
        rQ, rV = oracle.lsh_attend_bwd(Qn[b:b + 1, h:h + 1], Vn[b:b + 1, h:h + 1],
                                       dOn[b:b + 1, h:h + 1], keys_np[:, b:b + 1, h:h + 1],
                                       perm_np[:, b:b + 1, h:h + 1], w.chunk, w.causal)
        return bh, {"dQ": _err(gQ[b, h], rQ[0, 0], tol), "dV": _err(gV[b, h], rV[0, 0], tol)}

    worst.update(_collect(_pmap(one, _heads(w.B, w.H))))
    return {"heads": w.B * w.H, "tokens_hashed": w.B * w.H * w.L, "near_ties": ties,
            "near_tie_flips": flips, "rows_sorted": w.n_rounds * w.B * w.H, "max_abs": worst,
            "tol": tol}


BWD_CASES = [
    (1, 3, 320, 16, 2, 64, True),
    (2, 1, 96, 6, 3, 32, False),
    (1, 2, 64, 8, 2, 64, True),
    (1, 2, 128, 4, 2, 64, False),
    (1, 1, 256, 1, 2, 64, True),
    (1, 1, 256, 1024, 2, 64, False),
    (1, 2, 64, 4, 1, 4, True),
    (2, 2, 1024, 64, 3, 64, False),   # sixteen chunks, several tiles per row
    (1, 2, 1088, 32, 2, 64, True),    # seventeen chunks: last tile has one query chunk
    (1, 1, 256, 1, 2, 64, False),     # one bucket, non-causal
    (1, 2, 384, 8, 5, 64, True),      # five rounds
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,H,Lx,nb,R,chunk,causal", BWD_CASES)
def test_backward_small_shapes(oracle, dtype, B, H, Lx, nb, R, chunk, causal):
    inp = W.make_random(B, H, Lx, 64, nb, R, dtype, seed=7 * Lx + nb, backward=True)
    check_bwd(oracle, inp, nb, chunk, causal)


def test_backward_workload_L16384_every_head(oracle, parity_record):
    w = W.WORKLOADS["fwdbwd_bf16_L16384"]
    rec = check_bwd_every_head(oracle, w, W.make_inputs(w))
    parity_record.append({"workload": w.name + " (fwd+bwd)", **rec})


def test_backward_L65536_every_head(oracle, parity_record):
    """The backward at the headline size (8 rounds, 1024 buckets), every head
    against the oracle, with dO ~ N(0, 1) from seed 2."""
    w = W.WORKLOADS["fwd_bf16_L65536"]
    inp = W.make_inputs(w)
    inp["dO"] = W.gaussian(tuple(inp["Q"].shape), 2, inp["Q"].dtype)
    rec = check_bwd_every_head(oracle, w, inp)
    parity_record.append({"workload": w.name + " (fwd+bwd)", **rec})


# ---------------------------------------------------------------------------
# edge cases of the ABI on the device
# ---------------------------------------------------------------------------

def test_malformed_keys_are_reported():
    """Keys that are not bucket*L + position (here two rows swapped) are
    detected by the sort kernel's own check; every access stays in bounds."""
    inp = W.make_random(1, 1, 256, 64, 16, 1, torch.bfloat16, seed=3)
    Q, rot = inp["Q"].cuda(), inp["rot"].cuda()
    keys, _ = L.lsh_hash(Q, rot, 16)
    bad = keys.clone()
    bad[0, 0, 0, 0], bad[0, 0, 0, 1] = keys[0, 0, 0, 1], keys[0, 0, 0, 0]
    L.lsh_sort(bad, 16)
    assert L.lsh_device_status() == 6
    L.lsh_sort(keys, 16)
    assert L.lsh_device_status() == 0


def test_empty_batch_is_a_no_op():
    Q = torch.empty((0, 2, 64, 64), dtype=torch.bfloat16, device="cuda")
    rot = torch.randn(1, 64, 4, device="cuda").to(torch.bfloat16)
    out = L.lsh_forward(Q, Q, rot, 8, 64, True)
    assert out["O"].numel() == 0
    assert L.lsh_device_status() == 0


# ---------------------------------------------------------------------------
# tensor-core hash: shapes that exercise its round grouping and N-tiling
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("B,H,Lx,nb,R", [
    (1, 3, 320, 32, 3),     # nb/2 = 16: 16-column chunks, ragged token tiles
    (2, 2, 256, 64, 5),     # five rounds in one group (5 * 32 = 160 columns)
    (1, 2, 512, 256, 3),    # 3 * 128 columns: groups of two rounds, then one
    (1, 1, 384, 512, 9),    # 9 * 256: one round per N-tile, two groups
    (1, 1, 256, 2048, 2),   # nb/2 = 1024: four N-tiles per round
    (2, 2, 256, 256, 4),    # nb/2 = 128, even rounds: four epilogue warpgroups, a round each
    (1, 3, 320, 256, 2),    # the same kernel, one round pair, ragged token tiles
    (1, 1, 256, 256, 10),   # the same kernel, groups of eight rounds and of two
    (1, 3, 320, 512, 5),    # nb/2 = 256: a round shared by a pair of warpgroups, groups of 4 and 1
    (1, 3, 320, 1024, 2),   # nb/2 = 512: a round shared by all four warpgroups, ragged token tiles
])
def test_tensor_core_hash_shapes(oracle, B, H, Lx, nb, R):
    inp = W.make_random(B, H, Lx, 64, nb, R, torch.bfloat16, seed=nb + R)
    Q, rot = inp["Q"].cuda(), inp["rot"].cuda()
    keys, buckets = L.lsh_hash(Q, rot, nb)
    torch.cuda.synchronize()
    _check_status()
    check_hash(oracle, Q, rot, nb, keys, buckets)


def test_tensor_core_hash_exact_ties_take_lowest_index():
    """Duplicated and negated rotation columns make exact ties in the GPU's own
    arithmetic; the first index of [p ; -p] must win."""
    nb, half = 64, 32
    g = torch.Generator().manual_seed(5)
    base = torch.randn(64, half, generator=g)
    base[:, 1] = base[:, 0]        # p_1 == p_0
    base[:, 3] = -base[:, 2]       # p_3 == -p_2
    rot = base[None].to(torch.bfloat16).cuda()
    Q = torch.randn(1, 1, 1024, 64, generator=g).to(torch.bfloat16).cuda()
    _, b = L.lsh_hash(Q, rot, nb)
    torch.cuda.synchronize()
    b = b.cpu().numpy().ravel()
    assert not np.isin(b, [1, half + 1]).any()       # column 0 always beats its copy
    # p_3 == -p_2: z_3 ties z_{half+2} and z_2 ties z_{half+3}; the lower index wins
    assert not np.isin(b, [half + 2, half + 3]).any()
    assert np.isin(b, [0, half, 2, 3]).any()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_zero_queries(oracle, dtype):
    """Rows of Q that are exactly zero: bucket 0 (every entry of [p ; -p] is
    zero, the first index wins), a zero unit key (scores 0 against them), and
    no gradient through the normalisation of a zero row."""
    inp = W.make_random(1, 2, 320, 64, 16, 2, dtype, seed=91, backward=True)
    zero = [0, 5, 63, 64, 77, 200, 201, 319]
    inp["Q"][0, 0, zero] = 0
    inp["Q"][0, 1, 100:164] = 0          # a whole chunk's worth of zero rows
    check_all(oracle, inp, 16, 64, True)
    check_bwd(oracle, inp, 16, 64, True)
    _, buckets = L.lsh_hash(inp["Q"].cuda(), inp["rot"].cuda(), 16)
    assert (buckets[:, 0, 0, zero] == 0).all()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("chunk,causal", [(2, False), (2, True), (1, False)])
def test_hand_worked_bucket_pairs_on_the_device(dtype, chunk, causal):
    """The hand-worked example of tests/golden/attention_pairs.txt, padded
    from d = 2 to d = 64 with zeros (the rotation's two columns are the first
    two axes): each output is one named token's value (up to fp32 rounding)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "attention_pairs.txt")
    rows = [line.split() for line in open(path) if line.strip() and not line.startswith("#")]
    n = len(rows)
    Q = torch.zeros(1, 1, n, 64)
    Q[0, 0, :, 0] = torch.tensor([float(r[1]) for r in rows])
    Q[0, 0, :, 1] = torch.tensor([float(r[2]) for r in rows])
    V = torch.zeros(1, 1, n, 64)
    V[0, 0, :, 0] = torch.arange(n, dtype=torch.float32)
    V[0, 0, :, 1] = 10 + torch.arange(n, dtype=torch.float32)
    rot = torch.zeros(1, 64, 2)
    rot[0, 0, 0] = rot[0, 1, 1] = 1
    Q, V, rot = (t.to(dtype).cuda() for t in (Q, V, rot))
    out = L.lsh_forward(Q, V, rot, 4, chunk, causal)
    torch.cuda.synchronize()
    _check_status()
    O, lse = out["O"].float().cpu(), out["lse"].cpu()
    for i, r in enumerate(rows):
        mate = r[5] if chunk == 1 else (r[4] if causal else r[3])
        j = i if mate == "self" else int(mate)
        # the mate's weight is p / p in fp32: equal to 1 up to rounding
        assert torch.allclose(O[0, 0, i], V[0, 0, j].float().cpu(), rtol=0, atol=1e-5)
        if mate == "self":
            assert abs(lse[0, 0, i].item() + 1e5) < 0.05


def test_largest_row_count(oracle):
    """n_rounds * B * H = 65 535 rows, the most the launch grid takes."""
    inp = W.make_random(1, 4369, 64, 64, 4, 15, torch.bfloat16, seed=5)
    check_all(oracle, inp, 4, 64, False, heads=(0, 4368))


@pytest.mark.parametrize("causal", [True, False])
def test_large_norm_queries_take_the_exact_softmax(oracle, causal):
    """Queries scaled by 100 (score bound |q|/sqrt(d) ~ 100): the tensor-core
    softmax leaves the bound-referenced fast path for the exact two-pass one."""
    inp = W.make_random(1, 2, 320, 64, 16, 2, torch.bfloat16, seed=77)
    inp["Q"] = (inp["Q"].float() * 100).to(torch.bfloat16)
    check_all(oracle, inp, 16, 64, causal)
