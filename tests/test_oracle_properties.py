"""Randomised properties of the fp64 oracle over many small shapes
(hypothesis): invariants that any correct implementation of the method
satisfies, whatever the buckets come out as.

- keys are bucket * L + position, and perm sorts them (a permutation);
- every round's output is a convex combination of value rows, so each
  coordinate lies between that coordinate's minimum and maximum over V;
- a round's lse is at least the token's own score -1e5;
- the combined lse is the logsumexp of the round lse, and the combined
  output a convex combination of the round outputs;
- permuting the batch and head order permutes the outputs the same way."""
import math

import numpy as np
import pytest
from hypothesis import given, settings, HealthCheck
from hypothesis import strategies as st

from oracle import oracle as cpu_oracle


@pytest.fixture(scope="module", autouse=True)
def _build():
    cpu_oracle.build()


shapes = st.tuples(
    st.integers(1, 2),                      # B
    st.integers(1, 2),                      # H
    st.sampled_from([(8, 4), (16, 4), (16, 8), (24, 8), (32, 16), (12, 12)]),  # L, chunk
    st.sampled_from([1, 2, 4, 6, 8]),       # n_buckets
    st.integers(1, 3),                      # rounds
    st.booleans(),                          # causal
    st.integers(0, 2 ** 31 - 1),            # seed
)


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(shapes)
def test_forward_invariants(case):
    B, H, (L, chunk), nb, R, causal, seed = case
    d = 8
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, H, L, d))
    V = rng.standard_normal((B, H, L, d))
    rot = rng.standard_normal((R, d, nb // 2))
    out = cpu_oracle.lsh_forward(Q, V, rot, nb, chunk, causal)
    keys, perm, buckets = out["keys"], out["perm"], out["buckets"]
    pos = np.arange(L)
    assert np.array_equal(keys.astype(np.int64), buckets.astype(np.int64) * L + pos)
    assert (buckets >= 0).all() and (buckets < nb).all()
    assert np.array_equal(np.sort(perm, axis=-1), np.broadcast_to(pos, perm.shape))
    assert (np.diff(np.take_along_axis(keys.astype(np.int64), perm, -1), axis=-1) > 0).all()

    # slack: a lone token's lse is about -1e5, where an fp64 ulp (1.5e-11)
    # perturbs its combine weight by that much relative
    lo = V.min(axis=2, keepdims=True) - 1e-10
    hi = V.max(axis=2, keepdims=True) + 1e-10
    assert ((out["o_part"] >= lo) & (out["o_part"] <= hi)).all()
    assert ((out["O"] >= lo) & (out["O"] <= hi)).all()
    assert (out["lse_r"] >= -1e5 - 1e-6).all()

    m = out["lse_r"].max(axis=0)
    lse = m + np.log(np.exp(out["lse_r"] - m).sum(axis=0))
    np.testing.assert_allclose(out["lse"], lse, rtol=1e-12, atol=1e-9)
    w = np.exp(out["lse_r"] - out["lse"])
    np.testing.assert_allclose(w.sum(axis=0), 1.0, rtol=1e-9)
    np.testing.assert_allclose(out["O"], (w[..., None] * out["o_part"]).sum(axis=0),
                               rtol=1e-9, atol=1e-10)


@settings(max_examples=20, deadline=None)
@given(st.integers(0, 2 ** 31 - 1), st.booleans())
def test_heads_are_independent(seed, causal):
    rng = np.random.default_rng(seed)
    B, H, L, d, nb, R, chunk = 2, 3, 16, 8, 4, 2, 4
    Q = rng.standard_normal((B, H, L, d))
    V = rng.standard_normal((B, H, L, d))
    rot = rng.standard_normal((R, d, nb // 2))
    a = cpu_oracle.lsh_forward(Q, V, rot, nb, chunk, causal)
    pb, ph = rng.permutation(B), rng.permutation(H)
    b = cpu_oracle.lsh_forward(Q[pb][:, ph], V[pb][:, ph], rot, nb, chunk, causal)
    np.testing.assert_array_equal(b["O"], a["O"][pb][:, ph])
    np.testing.assert_array_equal(b["perm"], a["perm"][:, pb][:, :, ph])
