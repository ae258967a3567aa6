"""The seeded synthetic inputs follow their stated recipe: shapes, dtypes,
seeds, rotation rounding, and the clustered query structure."""
import torch

from lsh_attention_long_b200 import workloads as W

SHAPES = {  # B, H, L, n_buckets, n_rounds, dtype
    "fwd_f32_L1024": (1, 1, 1024, 32, 1, torch.float32),
    "fwd_bf16_L4096": (8, 8, 4096, 64, 2, torch.bfloat16),
    "fwd_bf16_L16384_clustered": (2, 8, 16384, 256, 4, torch.bfloat16),
    "fwd_bf16_L65536": (1, 8, 65536, 1024, 8, torch.bfloat16),
    "fwdbwd_bf16_L16384": (2, 8, 16384, 256, 4, torch.bfloat16),
}


def test_every_workload_has_its_stated_shape_and_dtype():
    assert set(W.WORKLOADS) == set(SHAPES)
    for name, (B, H, L, nb, R, dt) in SHAPES.items():
        w = W.WORKLOADS[name]
        assert (w.B, w.H, w.L, w.d, w.n_buckets, w.n_rounds, w.chunk) == (B, H, L, 64, nb, R, 64)
        if L > 16384:
            continue  # shapes above are enough; the large draw is covered by the bench
        t = W.make_inputs(w)
        assert t["Q"].shape == t["V"].shape == (B, H, L, 64)
        assert t["rot"].shape == (R, 64, nb // 2)
        assert t["Q"].dtype == t["V"].dtype == t["rot"].dtype == dt
        assert ("dO" in t) == w.backward


def test_inputs_are_reproducible_and_seeded_as_stated():
    w = W.WORKLOADS["fwd_f32_L1024"]
    a, b = W.make_inputs(w), W.make_inputs(w)
    for k in a:
        assert torch.equal(a[k], b[k])
    g = torch.Generator().manual_seed(0)
    q = torch.randn(1, 1, 1024, 64, generator=g)
    v = torch.randn(1, 1, 1024, 64, generator=g)
    assert torch.equal(a["Q"], q) and torch.equal(a["V"], v)  # one stream, Q first
    r = torch.randn(1, 64, 16, generator=torch.Generator().manual_seed(1))
    assert torch.equal(a["rot"], r)


def test_rotations_are_rounded_once_to_the_input_dtype():
    r32 = W.rotations(2, 64, 64, 1, torch.float32)
    r16 = W.rotations(2, 64, 64, 1, torch.bfloat16)
    assert torch.equal(r16, r32.to(torch.bfloat16))
    assert W.rotations(3, 64, 1, 1, torch.float32).shape == (3, 64, 0)


def test_clustered_queries_sit_near_unit_centres():
    q = W.clustered_queries(1, 2, 4096, 64, 512, 0.05, 3, 4, 5, torch.float32)
    # |centre + noise|^2 = 1 + 64 * 0.05^2 on average
    msq = (q.norm(dim=-1) ** 2).mean().item()
    assert abs(msq - (1 + 64 * 0.0025)) < 0.01
    # tokens of one cluster differ by their noise only: a query's nearest other
    # query lies about sqrt(2 * 64) * 0.05 = 0.57 away, a random pair about
    # sqrt(2 + 0.32) = 1.52 (4096 tokens over 512 centres: ~8 per cluster)
    d2 = torch.cdist(q[0, 0], q[0, 0])
    d2.fill_diagonal_(float("inf"))
    nearest = d2.min(dim=1).values.median().item()
    assert abs(nearest - (2 * 64) ** 0.5 * 0.05) < 0.08
    assert abs(d2[d2.isfinite()].median().item() - 2.32 ** 0.5) < 0.08
