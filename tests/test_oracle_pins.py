"""Pins of the fp64 CPU oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something it does not compute by its own
code path: a probability the Reformer explainer states (collision rate
1 - theta/pi for angular LSH), exact symmetries of the hash, library routines
on special cases that reduce to dense attention, brute-force enumeration of
bucket-mates on tiny inputs, closed forms (constant values, lone tokens,
repeated rounds) and finite differences of the forward.
"""

import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------
# hash
# ---------------------------------------------------------------------------

def test_collision_probability_matches_one_minus_theta_over_pi(oracle):
    """Reformer explainer, angular LSH: two vectors at angle theta share a
    bucket with probability 1 - theta/pi (hyperplane case, n_buckets = 2)."""
    d = 64
    rounds = 100_000
    thetas = np.linspace(0.15, math.pi - 0.15, 12)
    rng = _rng(11)
    basis, _ = np.linalg.qr(rng.standard_normal((d, d)))
    e0, e1 = basis[:, 0], basis[:, 1]
    vecs = []
    for th in thetas:
        vecs.append(3.0 * e0)
        vecs.append(0.5 * (math.cos(th) * e0 + math.sin(th) * e1))
    Q = np.stack(vecs)[None, None]  # [1, 1, 24, d]
    rot = rng.standard_normal((rounds, d, 1))
    _, buckets, _ = oracle.lsh_hash(Q, rot, 2)
    b = buckets[:, 0, 0, :]  # [rounds, 24]
    for a, th in enumerate(thetas):
        rate = np.mean(b[:, 2 * a] == b[:, 2 * a + 1])
        assert abs(rate - (1.0 - th / math.pi)) < 0.01, (th, rate)


@pytest.mark.parametrize("nb", [4, 16, 64, 1024])
def test_hash_antipodal_symmetry(oracle, nb):
    """Negating x negates every projection, so its sector is the opposite one:
    bucket(-x) = (bucket(x) + nb/2) mod nb whenever there is no near tie."""
    rng = _rng(nb)
    x = rng.standard_normal((1, 1, 200, 64))
    Q = np.concatenate([x, -x], axis=2)
    rot = rng.standard_normal((3, 64, nb // 2))
    _, b, tie = oracle.lsh_hash(Q, rot, nb)
    bp, bn = b[..., :200], b[..., 200:]
    ok = (tie[..., :200] == 0) & (tie[..., 200:] == 0)
    assert ok.mean() > 0.95
    assert np.array_equal(bn[ok], (bp[ok] + nb // 2) % nb)


@pytest.mark.parametrize("nb", [2, 6, 32, 256])
def test_hash_brute_force_over_sector_directions(oracle, nb):
    """Brute force: enumerate the nb directions +R_j and -R_j as explicit
    vectors and take the first direction of largest projection."""
    rng = _rng(100 + nb)
    Q = rng.standard_normal((2, 3, 50, 64))
    rot = rng.standard_normal((2, 64, nb // 2))
    keys, b, tie = oracle.lsh_hash(Q, rot, nb)
    for r in range(2):
        dirs = np.concatenate([rot[r], -rot[r]], axis=1)  # [d, nb] sector directions
        proj = np.einsum("bhld,dn->bhln", Q, dirs)
        expect = np.argmax(proj, axis=-1)  # first index of the maximum
        ok = tie[r] == 0
        assert np.array_equal(b[r][ok], expect[ok])
    L = Q.shape[2]
    pos = np.arange(L, dtype=np.uint64)
    assert np.array_equal(keys.astype(np.uint64), b.astype(np.uint64) * L + pos)


def test_hash_exact_ties_take_the_lowest_index(oracle):
    """Duplicated or negated rotation columns make exact ties; the first index
    of [p ; -p] wins and the tie is flagged."""
    rng = _rng(5)
    Q = rng.standard_normal((1, 1, 40, 16))
    # columns 0 and 1 identical, column 2 much shorter: max |p| sits at 0 == 1
    r = rng.standard_normal((16, 1))
    rot = np.concatenate([r, r, 1e-3 * rng.standard_normal((16, 1))], axis=1)[None]
    _, b, tie = oracle.lsh_hash(Q, rot, 6)
    p0 = Q[0, 0] @ r[:, 0]
    expect = np.where(p0 >= 0, 0, 3)
    assert np.array_equal(b[0, 0, 0], expect)
    assert np.all(tie == 1)
    # column 1 = -column 0: z = (p, -p, -p, p); the first half wins the tie
    rot2 = np.concatenate([r, -r], axis=1)[None]
    _, b2, tie2 = oracle.lsh_hash(Q, rot2, 4)
    assert np.array_equal(b2[0, 0, 0], np.where(p0 >= 0, 0, 1))
    assert np.all(tie2 == 1)


def test_hash_hand_worked_axis_sectors(oracle):
    """The worked example in tests/golden/hash_axis_sectors.txt: with the
    identity as rotation, each bucket is a signed coordinate axis, derived by
    hand (including the lowest-index rule on exact ties)."""
    path = os.path.join(os.path.dirname(__file__), "golden", "hash_axis_sectors.txt")
    rows = [line.split() for line in open(path) if line.strip() and not line.startswith("#")]
    for d in sorted({int(r[0]) for r in rows}):
        sel = [r for r in rows if int(r[0]) == d]
        X = np.array([[float(v) for v in r[1:1 + d]] for r in sel])
        want = np.array([int(r[1 + d]) for r in sel])
        L = len(sel)
        keys, buckets, _ = oracle.lsh_hash(X[None, None], np.eye(d)[None], 2 * d)
        np.testing.assert_array_equal(buckets[0, 0, 0], want)
        np.testing.assert_array_equal(keys[0, 0, 0], want * L + np.arange(L))


def test_hash_one_bucket_ignores_rotation(oracle):
    rng = _rng(6)
    Q = rng.standard_normal((2, 2, 32, 64))
    keys, b, tie = oracle.lsh_hash(Q, np.zeros((3, 64, 0)), 1)
    assert np.all(b == 0) and np.all(tie == 0)
    assert np.array_equal(keys, np.broadcast_to(np.arange(32, dtype=np.uint32), keys.shape))


# ---------------------------------------------------------------------------
# sort
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("nb,L", [(2, 64), (8, 256), (64, 1000), (1024, 4096)])
def test_sort_is_stable_bucket_order(oracle, nb, L):
    rng = _rng(L)
    buckets = rng.integers(0, nb, size=(3, L)).astype(np.uint64)
    keys = (buckets * L + np.arange(L, dtype=np.uint64)).astype(np.uint32)
    perm = oracle.lsh_sort(keys)
    for row in range(3):
        p = perm[row]
        assert np.array_equal(np.sort(p), np.arange(L))
        assert np.all(np.diff(keys[row][p].astype(np.int64)) > 0)
        assert np.array_equal(p, np.lexsort((np.arange(L), buckets[row])))


# ---------------------------------------------------------------------------
# attention and combine
# ---------------------------------------------------------------------------

def _dense_reference(Q, V, causal, same_bucket=None):
    """Dense shared-QK attention through torch's SDPA in float64: keys are the
    unit queries, the diagonal gets -1e5, future positions -inf."""
    q = torch.from_numpy(Q)
    v = torch.from_numpy(V)
    k = q / q.norm(dim=-1, keepdim=True)
    L = q.shape[-2]
    mask = torch.zeros(L, L, dtype=torch.float64)
    if causal:
        mask = mask.masked_fill(torch.ones(L, L, dtype=torch.bool).triu(1), float("-inf"))
    mask = mask.expand(q.shape[0], q.shape[1], L, L).clone()
    if same_bucket is not None:
        mask = mask.masked_fill(~torch.from_numpy(same_bucket), float("-inf"))
    mask = mask + torch.diag(torch.full((L,), -1e5, dtype=torch.float64))
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=1.0 / math.sqrt(Q.shape[-1]))
    return o.numpy()


@pytest.mark.parametrize("causal", [False, True])
def test_one_bucket_one_chunk_is_full_attention(oracle, causal):
    """With one bucket and c = L, LSH attention is dense shared-QK attention
    with the self mask."""
    rng = _rng(7 + causal)
    Q = rng.standard_normal((2, 3, 48, 64))
    V = rng.standard_normal((2, 3, 48, 64))
    out = oracle.lsh_forward(Q, V, np.zeros((1, 64, 0)), 1, 48, causal)
    ref = _dense_reference(Q, V, causal)
    np.testing.assert_allclose(out["O"], ref, rtol=0, atol=1e-12)
    # lse: the library logsumexp of the scores with the diagonal replaced
    q = torch.from_numpy(Q)
    s = q @ (q / q.norm(dim=-1, keepdim=True)).transpose(-1, -2) / 8.0
    s = s.clone()
    s.diagonal(dim1=-2, dim2=-1).fill_(-1e5)
    if causal:
        s = s.masked_fill(torch.ones(48, 48, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(out["lse"], torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-9)


@pytest.mark.parametrize("causal", [False, True])
def test_two_chunks_see_the_whole_row(oracle, causal):
    """With two chunks, chunk 0's previous chunk is chunk 1 and vice versa, so
    every query sees every same-bucket key: dense attention under a
    bucket-equality mask."""
    rng = _rng(17 + causal)
    Q = rng.standard_normal((1, 2, 64, 64))
    V = rng.standard_normal((1, 2, 64, 64))
    rot = rng.standard_normal((1, 64, 2))
    out = oracle.lsh_forward(Q, V, rot, 4, 32, causal)
    b = out["buckets"][0]
    same = b[..., :, None] == b[..., None, :]
    ref = _dense_reference(Q, V, causal, same_bucket=same)
    np.testing.assert_allclose(out["O"], ref, rtol=0, atol=1e-12)


def _brute_force(Q, V, buckets, chunk, causal):
    """Per query, enumerate the same-bucket keys whose sorted chunk is the
    query's own or the one before it (a set, wrapping), then take one
    softmax per round and one over all rounds together."""
    R = buckets.shape[0]
    B, H, L, d = Q.shape
    n_c = L // chunk
    o_r = np.zeros((R, B, H, L, d))
    lse_r = np.zeros((R, B, H, L))
    O = np.zeros((B, H, L, d))
    lse = np.zeros((B, H, L))
    for b in range(B):
        for h in range(H):
            q = Q[b, h]
            nrm = np.linalg.norm(q, axis=1)
            all_s = [[] for _ in range(L)]
            all_v = [[] for _ in range(L)]
            for r in range(R):
                bk = buckets[r, b, h]
                order = np.lexsort((np.arange(L), bk))
                slot = np.empty(L, int)
                slot[order] = np.arange(L)
                ch = slot // chunk
                for i in range(L):
                    allowed = {ch[i], (ch[i] - 1) % n_c}
                    s, vs = [], []
                    for j in range(L):
                        if bk[j] != bk[i] or ch[j] not in allowed:
                            continue
                        if causal and j > i:
                            continue
                        sc = -1e5 if j == i else float(q[i] @ q[j]) / (nrm[j] * math.sqrt(d))
                        s.append(sc)
                        vs.append(V[b, h, j])
                    s = np.array(s)
                    m = s.max()
                    l = m + math.log(np.exp(s - m).sum())
                    lse_r[r, b, h, i] = l
                    o_r[r, b, h, i] = (np.exp(s - l)[:, None] * np.array(vs)).sum(0)
                    all_s[i].extend(s)
                    all_v[i].extend(vs)
            for i in range(L):
                s = np.array(all_s[i])
                m = s.max()
                l = m + math.log(np.exp(s - m).sum())
                lse[b, h, i] = l
                O[b, h, i] = (np.exp(s - l)[:, None] * np.array(all_v[i])).sum(0)
    return o_r, lse_r, O, lse


@pytest.mark.parametrize("L,chunk,nb,R,causal", [
    (8, 4, 2, 1, False), (16, 4, 4, 2, True), (32, 8, 8, 3, False),
    (48, 16, 4, 2, True), (24, 8, 2, 2, True), (40, 8, 6, 1, False),
])
def test_brute_force_bucket_mates(oracle, L, chunk, nb, R, causal):
    rng = _rng(L * 31 + nb)
    Q = rng.standard_normal((1, 2, L, 16))
    V = rng.standard_normal((1, 2, L, 16))
    rot = rng.standard_normal((R, 16, nb // 2))
    out = oracle.lsh_forward(Q, V, rot, nb, chunk, causal)
    o_r, lse_r, O, lse = _brute_force(Q, V, out["buckets"], chunk, causal)
    np.testing.assert_allclose(out["o_part"], o_r, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["lse_r"], lse_r, rtol=1e-12, atol=1e-9)
    np.testing.assert_allclose(out["O"], O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["lse"], lse, rtol=1e-12, atol=1e-9)


@pytest.mark.parametrize("chunk,causal", [(2, False), (2, True), (1, False), (1, True)])
def test_hand_worked_bucket_pairs(oracle, chunk, causal):
    """tests/golden/attention_pairs.txt: every query has at most one
    bucket-mate in its window, so the output is that mate's value exactly,
    or the token's own value with lse = -1e5 when causality masks the mate."""
    path = os.path.join(os.path.dirname(__file__), "golden", "attention_pairs.txt")
    rows = [line.split() for line in open(path) if line.strip() and not line.startswith("#")]
    L = len(rows)
    Q = np.array([[float(r[1]), float(r[2])] for r in rows])[None, None]
    V = np.array([[i, 10.0 + i] for i in range(L)])[None, None]
    out = oracle.lsh_forward(Q, V, np.eye(2)[None], 4, chunk, causal)
    for i, r in enumerate(rows):
        mate = r[5] if chunk == 1 else (r[4] if causal else r[3])
        if mate == "self":
            np.testing.assert_array_equal(out["O"][0, 0, i], V[0, 0, i])
            assert out["lse"][0, 0, i] == -1e5
        else:
            j = int(mate)
            np.testing.assert_array_equal(out["O"][0, 0, i], V[0, 0, j])
            s_ij = Q[0, 0, i] @ Q[0, 0, j] / (np.linalg.norm(Q[0, 0, j]) * math.sqrt(2))
            assert abs(out["lse"][0, 0, i] - s_ij) < 1e-12


def test_constant_values_give_constant_output(oracle):
    rng = _rng(9)
    Q = rng.standard_normal((1, 2, 64, 64))
    V = np.full((1, 2, 64, 64), 3.25)
    out = oracle.lsh_forward(Q, V, rng.standard_normal((3, 64, 4)), 8, 16, True)
    np.testing.assert_allclose(out["O"], 3.25, rtol=0, atol=1e-12)


def test_lone_token_returns_its_own_value(oracle):
    """A token with no bucket-mate in its window attends only to itself:
    o_r = v and lse_r = -1e5 exactly."""
    rng = _rng(10)
    L, c = 32, 4
    Q = rng.standard_normal((1, 1, L, 64))
    V = rng.standard_normal((1, 1, L, 64))
    out = oracle.lsh_forward(Q, V, rng.standard_normal((1, 64, 32)), 64, c, False)
    bk = out["buckets"][0, 0, 0]
    perm = out["perm"][0, 0, 0]
    slot = np.empty(L, int)
    slot[perm] = np.arange(L)
    n_c = L // c
    lone = 0
    for i in range(L):
        chs = {slot[i] // c, (slot[i] // c - 1) % n_c}
        mates = [j for j in range(L) if j != i and bk[j] == bk[i] and slot[j] // c in chs]
        if not mates:
            lone += 1
            assert out["lse_r"][0, 0, 0, i] == -1e5
            np.testing.assert_array_equal(out["o_part"][0, 0, 0, i], V[0, 0, i])
    assert lone > 5


def test_identical_rounds_equal_one_round(oracle):
    """R copies of one rotation: the combine averages R equal results, so O is
    the one-round output and lse grows by ln R."""
    rng = _rng(12)
    Q = rng.standard_normal((1, 2, 64, 64))
    V = rng.standard_normal((1, 2, 64, 64))
    r1 = rng.standard_normal((1, 64, 8))
    one = oracle.lsh_forward(Q, V, r1, 16, 16, True)
    four = oracle.lsh_forward(Q, V, np.repeat(r1, 4, axis=0), 16, 16, True)
    np.testing.assert_allclose(four["O"], one["O"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(four["lse"], one["lse"] + math.log(4), rtol=1e-12, atol=1e-9)


def test_combine_of_one_round_is_identity(oracle):
    rng = _rng(13)
    o = rng.standard_normal((1, 2, 3, 8, 16))
    l = rng.standard_normal((1, 2, 3, 8))
    O, lse = oracle.lsh_combine(o, l)
    np.testing.assert_allclose(O, o[0], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, l[0], rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("L,chunk,nb,R,causal", [(16, 4, 4, 2, True), (32, 8, 2, 3, False),
                                                  (24, 8, 4, 1, True)])
def test_backward_matches_finite_differences(oracle, L, chunk, nb, R, causal):
    """Central differences of sum(dO * O) in fp64 with buckets frozen."""
    rng = _rng(L + 1000 * R)
    d = 8
    Q = rng.standard_normal((1, 2, L, d))
    V = rng.standard_normal((1, 2, L, d))
    dO = rng.standard_normal((1, 2, L, d))
    rot = rng.standard_normal((R, d, nb // 2))
    keys, _, _ = oracle.lsh_hash(Q, rot, nb)
    perm = oracle.lsh_sort(keys)
    dQ, dV = oracle.lsh_attend_bwd(Q, V, dO, keys, perm, chunk, causal)

    def loss(Qx, Vx):
        o_part, lse_r = oracle.lsh_attend_fwd(Qx, Vx, keys, perm, chunk, causal)
        O, _ = oracle.lsh_combine(o_part, lse_r)
        return float((dO * O).sum())

    h = 1e-5
    idx = [tuple(rng.integers(0, s) for s in Q.shape) for _ in range(40)]
    for ix in idx:
        for X, G, name in ((Q, dQ, "dQ"), (V, dV, "dV")):
            Xp = X.copy(); Xp[ix] += h
            Xm = X.copy(); Xm[ix] -= h
            fd = (loss(Xp, V) - loss(Xm, V)) / (2 * h) if name == "dQ" else \
                 (loss(Q, Xp) - loss(Q, Xm)) / (2 * h)
            assert abs(fd - G[ix]) <= 1e-6 * max(1.0, abs(fd)), (name, ix, fd, G[ix])


@pytest.mark.parametrize("causal", [False, True])
def test_backward_one_bucket_matches_autograd(oracle, causal):
    """nb = 1 and c = L: dense shared-QK attention, differentiated by torch
    autograd in float64 (key normalisation included)."""
    rng = _rng(21 + causal)
    L, d = 32, 16
    Q = rng.standard_normal((1, 2, L, d))
    V = rng.standard_normal((1, 2, L, d))
    dO = rng.standard_normal((1, 2, L, d))
    keys, _, _ = oracle.lsh_hash(Q, np.zeros((1, d, 0)), 1)
    perm = oracle.lsh_sort(keys)
    dQ, dV = oracle.lsh_attend_bwd(Q, V, dO, keys, perm, L, causal)
    q = torch.from_numpy(Q).requires_grad_(True)
    v = torch.from_numpy(V).requires_grad_(True)
    k = q / q.norm(dim=-1, keepdim=True)
    mask = torch.zeros(L, L, dtype=torch.float64)
    if causal:
        mask = mask.masked_fill(torch.ones(L, L, dtype=torch.bool).triu(1), float("-inf"))
    mask = mask + torch.diag(torch.full((L,), -1e5, dtype=torch.float64))
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=1.0 / math.sqrt(d))
    (o * torch.from_numpy(dO)).sum().backward()
    np.testing.assert_allclose(dQ, q.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dV, v.grad.numpy(), rtol=0, atol=1e-10)


def test_chunk_range_restricts_the_full_computation(oracle):
    """The chunk-range entry point (used to time bounded samples) computes the
    same values as the full call on the queries of those chunks, nothing else."""
    rng = _rng(31)
    Q = rng.standard_normal((1, 2, 128, 16))
    V = rng.standard_normal((1, 2, 128, 16))
    keys, _, _ = oracle.lsh_hash(Q, rng.standard_normal((2, 16, 4)), 8)
    perm = oracle.lsh_sort(keys)
    full_o, full_l = oracle.lsh_attend_fwd(Q, V, keys, perm, 16, True)
    o, l = oracle.lsh_attend_fwd_range(Q, V, keys, perm, 16, True, 2, 5)
    slots = perm[..., 32:80]  # queries of chunks 2..4
    mask = np.zeros(l.shape, bool)
    for r in range(2):
        for h in range(2):
            mask[r, 0, h, slots[r, 0, h]] = True
    np.testing.assert_array_equal(l[mask], full_l[mask])
    np.testing.assert_array_equal(o[mask], full_o[mask])
    assert np.all(l[~mask] == 0) and np.all(o[~mask] == 0)


# ---------------------------------------------------------------------------
# chunked feed-forward (the companion op of LSH attention in a Reformer layer)
# ---------------------------------------------------------------------------

def _ffn_golden():
    path = os.path.join(os.path.dirname(__file__), "golden", "ffn_small.txt")
    vals = {}
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            name, *nums = line.split()
            vals[name] = np.array([float(x) for x in nums])
    shapes = {"W1": (3, 2), "b1": (3,), "W2": (2, 3), "b2": (2,), "X": (3, 2), "Y": (3, 2),
              "dY": (3, 2), "dX": (3, 2), "dW1": (3, 2), "db1": (3,), "dW2": (2, 3),
              "db2": (2,)}
    return {k: vals[k].reshape(s) for k, s in shapes.items()}


def test_ffn_hand_worked_example(oracle):
    g = _ffn_golden()
    for chunk in (1, 2, 3):
        Y = oracle.ffn_forward(g["X"], g["W1"], g["b1"], g["W2"], g["b2"], chunk)
        np.testing.assert_array_equal(Y, g["Y"])
        dX, dW1, db1, dW2, db2 = oracle.ffn_backward(g["X"], g["W1"], g["b1"], g["W2"], g["dY"],
                                                     chunk)
        for got, name in ((dX, "dX"), (dW1, "dW1"), (db1, "db1"), (dW2, "dW2"), (db2, "db2")):
            np.testing.assert_array_equal(got, g[name], err_msg=name)


def test_ffn_identity_weights_give_relu(oracle):
    rng = np.random.default_rng(1)
    X = rng.standard_normal((37, 8))
    I = np.eye(8)
    Y = oracle.ffn_forward(X, I, np.zeros(8), I, np.zeros(8), 5)
    np.testing.assert_array_equal(Y, np.maximum(X, 0.0))


def test_ffn_zero_second_layer_gives_its_bias(oracle):
    rng = np.random.default_rng(2)
    X = rng.standard_normal((9, 4))
    b2 = rng.standard_normal(4)
    Y = oracle.ffn_forward(X, rng.standard_normal((16, 4)), rng.standard_normal(16),
                           np.zeros((4, 16)), b2, 4)
    np.testing.assert_array_equal(Y, np.broadcast_to(b2, Y.shape))


def test_ffn_chunking_does_not_change_the_result(oracle):
    rng = np.random.default_rng(3)
    T, dm, dff = 50, 16, 64
    X, W1, b1 = rng.standard_normal((T, dm)), rng.standard_normal((dff, dm)), rng.standard_normal(dff)
    W2, b2 = rng.standard_normal((dm, dff)), rng.standard_normal(dm)
    dY = rng.standard_normal((T, dm))
    whole = oracle.ffn_forward(X, W1, b1, W2, b2, T)
    gw = oracle.ffn_backward(X, W1, b1, W2, dY, T)
    for chunk in (1, 7, 16, 49):
        np.testing.assert_array_equal(oracle.ffn_forward(X, W1, b1, W2, b2, chunk), whole)
        for a, b in zip(oracle.ffn_backward(X, W1, b1, W2, dY, chunk), gw):
            np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-12)


def test_ffn_matches_library_matmuls(oracle):
    rng = np.random.default_rng(4)
    T, dm, dff = 33, 24, 96
    X, W1, b1 = rng.standard_normal((T, dm)), rng.standard_normal((dff, dm)), rng.standard_normal(dff)
    W2, b2 = rng.standard_normal((dm, dff)), rng.standard_normal(dm)
    ref = np.maximum(X @ W1.T + b1, 0.0) @ W2.T + b2
    np.testing.assert_allclose(oracle.ffn_forward(X, W1, b1, W2, b2, 8), ref, rtol=1e-12,
                               atol=1e-12)


def test_ffn_backward_matches_finite_differences(oracle):
    rng = np.random.default_rng(5)
    T, dm, dff = 6, 5, 7
    X, W1, b1 = rng.standard_normal((T, dm)), rng.standard_normal((dff, dm)), rng.standard_normal(dff)
    W2, b2 = rng.standard_normal((dm, dff)), rng.standard_normal(dm)
    dY = rng.standard_normal((T, dm))
    grads = dict(zip(("X", "W1", "b1", "W2", "b2"),
                     oracle.ffn_backward(X, W1, b1, W2, dY, 4)))
    params = {"X": X, "W1": W1, "b1": b1, "W2": W2, "b2": b2}
    eps = 1e-6

    def loss():
        return float((dY * oracle.ffn_forward(params["X"], params["W1"], params["b1"],
                                              params["W2"], params["b2"], 4)).sum())

    for name, p in params.items():
        num = np.zeros_like(p)
        for idx in np.ndindex(p.shape):
            keep = p[idx]
            p[idx] = keep + eps
            up = loss()
            p[idx] = keep - eps
            down = loss()
            p[idx] = keep
            num[idx] = (up - down) / (2 * eps)
        np.testing.assert_allclose(grads[name], num, rtol=1e-6, atol=1e-7, err_msg=name)


# ---------------------------------------------------------------------------
# reversible residual block (Y1 = X1 + F(X2), Y2 = X2 + G(Y1); F = LSH
# attention of X2 with its buckets held constant, G = chunked feed-forward)
# ---------------------------------------------------------------------------

def _rev_case(seed, B=1, L=16, H=1, d=64, dff=32, nb=4, R=2):
    rng = np.random.default_rng(seed)
    D = H * d
    return dict(X1=rng.standard_normal((B, L, D)), X2=rng.standard_normal((B, L, D)),
                rot=rng.standard_normal((R, d, nb // 2)), nb=nb, H=H,
                W1=rng.standard_normal((dff, D)) / np.sqrt(D), b1=0.1 * rng.standard_normal(dff),
                W2=rng.standard_normal((D, dff)) / np.sqrt(dff), b2=0.1 * rng.standard_normal(D),
                dY1=rng.standard_normal((B, L, D)), dY2=rng.standard_normal((B, L, D)))


def test_reversible_block_reconstructs_its_inputs(oracle):
    """The RevNet property: the backward recovers X1 and X2 from Y1 and Y2."""
    c = _rev_case(1, L=64, H=2)
    Y1, Y2, keys, perm = oracle.rev_forward(c["X1"], c["X2"], c["rot"], c["nb"], c["H"], 8, True,
                                            c["W1"], c["b1"], c["W2"], c["b2"], 16)
    X1, X2 = oracle.rev_backward(Y1, Y2, c["dY1"][:, :64], c["dY2"][:, :64], keys, perm,
                                 c["H"], 8, True, c["W1"], c["b1"], c["W2"], c["b2"], 16)[:2]
    np.testing.assert_allclose(X1, c["X1"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(X2, c["X2"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_reversible_block_gradients_match_finite_differences(oracle, causal):
    """Gradients of sum(dY1 * Y1 + dY2 * Y2), buckets held at those of the
    unperturbed X2, against central differences in fp64."""
    c = _rev_case(2 + causal)
    chunk, fchunk = 4, 8
    Y1, Y2, keys, perm = oracle.rev_forward(c["X1"], c["X2"], c["rot"], c["nb"], c["H"], chunk,
                                            causal, c["W1"], c["b1"], c["W2"], c["b2"], fchunk)
    got = dict(zip(("X1", "X2", "dX1", "dX2", "W1", "b1", "W2", "b2"),
                   oracle.rev_backward(Y1, Y2, c["dY1"], c["dY2"], keys, perm, c["H"], chunk,
                                       causal, c["W1"], c["b1"], c["W2"], c["b2"], fchunk)))
    grads = {"X1": got["dX1"], "X2": got["dX2"], "W1": got["W1"], "b1": got["b1"],
             "W2": got["W2"], "b2": got["b2"]}
    p = {k: c[k].copy() for k in ("X1", "X2", "W1", "b1", "W2", "b2")}
    B, L, D = p["X1"].shape

    def loss():
        y1 = p["X1"] + oracle.rev_attention(p["X2"], keys, perm, c["H"], chunk, causal)
        y2 = p["X2"] + oracle.ffn_forward(y1.reshape(B * L, D), p["W1"], p["b1"], p["W2"],
                                          p["b2"], fchunk).reshape(B, L, D)
        return float((c["dY1"] * y1).sum() + (c["dY2"] * y2).sum())

    rng = np.random.default_rng(7)
    eps = 1e-6
    for name, arr in p.items():
        flat = arr.reshape(-1)
        for idx in rng.choice(flat.size, size=min(24, flat.size), replace=False):
            keep = flat[idx]
            flat[idx] = keep + eps
            up = loss()
            flat[idx] = keep - eps
            down = loss()
            flat[idx] = keep
            num = (up - down) / (2 * eps)
            ana = grads[name].reshape(-1)[idx]
            assert abs(ana - num) <= 1e-6 * max(1.0, abs(num)), (name, idx, ana, num)
