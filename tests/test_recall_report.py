"""The recall report's window enumeration and recall figure (CPU).

`bench.py --recall` measures how much of full shared-QK attention's
probability mass LSH attention can see ("Reformer explainer",
akshathtiwari.co.in/blog/reformer: more hash rounds raise the chance that
similar tokens share a bucket).  The pages print no recall value, so the
report is unpinned as a number; these tests pin the computation itself:
a single bucket and a single chunk must see everything (recall 1), and the
attended sets must equal a brute-force enumeration over the oracle's keys
and sort.
"""

import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _keys_perm(oracle, Q, nb, R, seed):
    rng = np.random.default_rng(seed)
    rot = rng.standard_normal((R, Q.shape[-1], max(nb // 2, 1)))
    keys, _, _ = oracle.lsh_hash(Q, rot, nb)
    perm = oracle.lsh_sort(keys)
    return (torch.from_numpy(keys.astype(np.int64)), torch.from_numpy(perm.astype(np.int64)))


@pytest.mark.parametrize("causal", [False, True])
def test_one_bucket_one_chunk_sees_everything(oracle, causal):
    rng = np.random.default_rng(0)
    L = 96
    Q = rng.standard_normal((1, 1, L, 64))
    keys, perm = _keys_perm(oracle, Q, 1, 2, 1)
    rows = torch.arange(L)
    rec = bench.full_attention_recall(torch.from_numpy(Q), keys, perm, L, causal, rows, 0, 0)
    np.testing.assert_allclose(rec.numpy(), 1.0, rtol=0, atol=1e-12)
    assert rec.numel() == (L - 1 if causal else L)  # causal: position 0 has no key


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("L,chunk,nb,R", [(256, 32, 8, 2), (128, 64, 4, 3), (64, 64, 4, 1)])
def test_attended_sets_match_brute_force(oracle, causal, L, chunk, nb, R):
    rng = np.random.default_rng(L + nb)
    Q = rng.standard_normal((1, 2, L, 64))
    keys, perm = _keys_perm(oracle, Q, nb, R, L)
    rows = torch.arange(0, L, 3)
    h = 1
    got = bench.attended_mask(keys, perm, L, chunk, causal, rows, 0, h).numpy()
    nch = L // chunk
    want = np.zeros_like(got)
    for qi, i in enumerate(rows.tolist()):
        for r in range(R):
            k = keys[r, 0, h].numpy() & 0xFFFFFFFF
            p = perm[r, 0, h].numpy()
            slot = int(np.nonzero(p == i)[0][0])
            c = slot // chunk
            chunks = [c] if nch == 1 else [(c - 1) % nch, c]
            for cc in chunks:
                for j in p[cc * chunk:(cc + 1) * chunk]:
                    if j == i or k[j] // L != k[i] // L or (causal and j > i):
                        continue
                    want[qi, j] = True
    assert np.array_equal(got, want)


def test_topk_recall_one_bucket_one_chunk_is_one(oracle):
    rng = np.random.default_rng(3)
    L = 128
    Q = rng.standard_normal((1, 1, L, 64))
    keys, perm = _keys_perm(oracle, Q, 1, 1, 2)
    rec = bench.full_attention_recall(torch.from_numpy(Q), keys, perm, L, False,
                                      torch.arange(L), 0, 0, topk=16)
    np.testing.assert_allclose(rec.numpy(), 1.0, rtol=0, atol=0)


def test_topk_recall_counts_the_top_keys(oracle):
    # top-k recall equals the share of each query's k best keys in its
    # attended set, computed here directly from the mask and the scores
    rng = np.random.default_rng(4)
    L, k = 256, 8
    Q = rng.standard_normal((1, 1, L, 64))
    keys, perm = _keys_perm(oracle, Q, 16, 2, 6)
    rows = torch.arange(L)
    got = bench.full_attention_recall(torch.from_numpy(Q), keys, perm, 32, False, rows, 0, 0,
                                      topk=k).numpy()
    mask = bench.attended_mask(keys, perm, L, 32, False, rows, 0, 0).numpy()
    q = Q[0, 0]
    khat = q / np.linalg.norm(q, axis=1, keepdims=True)
    s = q @ khat.T
    np.fill_diagonal(s, -np.inf)
    want = np.array([mask[i, np.argsort(-s[i])[:k]].mean() for i in range(L)])
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_recall_is_a_share_of_the_mass(oracle):
    rng = np.random.default_rng(5)
    L = 256
    Q = rng.standard_normal((1, 1, L, 64))
    keys, perm = _keys_perm(oracle, Q, 16, 2, 9)
    rec = bench.full_attention_recall(torch.from_numpy(Q), keys, perm, 32, False,
                                      torch.arange(L), 0, 0).numpy()
    assert np.all(rec >= 0.0) and np.all(rec <= 1.0 + 1e-12)
    assert 0.0 < rec.mean() < 1.0


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_attended_sets_on_the_device_match_brute_force(causal):
    """The recall report as the bench runs it: keys and permutations from the
    CUDA path (clustered queries, several chunks and rounds), the attended
    sets computed from device tensors, against a brute-force enumeration of
    the same keys and permutations on the host."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import lsh_attention_long_b200 as L
    from lsh_attention_long_b200 import build
    from lsh_attention_long_b200 import workloads as W
    build.build()
    L.load_library()
    Lx, chunk, nb, R = 1024, 64, 16, 3
    inp = W.make_random(1, 2, Lx, 64, nb, R, torch.bfloat16, seed=29)
    Q, V, rot = (inp[k].cuda() for k in ("Q", "V", "rot"))
    out = L.lsh_forward(Q, V, rot, nb, chunk, causal)
    torch.cuda.synchronize()
    assert L.lsh_device_status() == 0
    rows = torch.arange(0, Lx, 7, device="cuda")
    got = bench.attended_mask(out["keys"].to(torch.int64), out["perm"].to(torch.int64), Lx,
                              chunk, causal, rows, 0, 1).cpu().numpy()
    keys = out["keys"].cpu().numpy().view(np.uint32)
    perm = out["perm"].cpu().numpy()
    nch = Lx // chunk
    want = np.zeros_like(got)
    for qi, i in enumerate(rows.tolist()):
        for r in range(R):
            k, p = keys[r, 0, 1], perm[r, 0, 1]
            c = int(np.nonzero(p == i)[0][0]) // chunk
            for cc in ([c] if nch == 1 else [(c - 1) % nch, c]):
                for j in p[cc * chunk:(cc + 1) * chunk]:
                    if j != i and k[j] // Lx == k[i] // Lx and not (causal and j > i):
                        want[qi, j] = True
    assert np.array_equal(got, want)
    rec = bench.full_attention_recall(Q.float(), out["keys"].to(torch.int64),
                                      out["perm"].to(torch.int64), chunk, causal, rows, 0, 1)
    assert torch.all((rec >= 0) & (rec <= 1 + 1e-9))
