"""The bench's CPU baselines: the oracle timed single-threaded and with the
independent heads spread over host threads.  The threaded run must compute
what the serial one computes (the oracle's C routines hold no shared state),
and both report a positive rate."""
import os
import sys
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from lsh_attention_long_b200 import workloads as W  # noqa: E402
from oracle import oracle as cpu_oracle  # noqa: E402


def test_threaded_heads_equal_serial_heads():
    w = W.make_random(1, 4, 256, 64, 16, 2, torch.float32, seed=11)
    Q, V, rot = w["Q"].numpy(), w["V"].numpy(), w["rot"].numpy()
    heads = range(Q.shape[1])
    serial = [cpu_oracle.lsh_forward(Q[:, h:h + 1], V[:, h:h + 1], rot, 16, 32, True)
              for h in heads]
    with ThreadPoolExecutor(max_workers=4) as pool:
        threaded = list(pool.map(
            lambda h: cpu_oracle.lsh_forward(Q[:, h:h + 1], V[:, h:h + 1], rot, 16, 32, True),
            heads))
    for a, b in zip(serial, threaded):
        assert np.array_equal(a["perm"], b["perm"])
        assert np.array_equal(a["O"], b["O"]) and np.array_equal(a["lse"], b["lse"])


def test_baseline_records():
    w = W.WORKLOADS["fwd_f32_L1024"]
    one = bench.run_cpu_baseline(w)
    many = bench.run_cpu_baseline_threads(w)
    for r in (one, many):
        assert r["kind"] == "oracle" and r["unit"] == "tokens/s" and r["value"] > 0
        assert r["nproc"] >= r["cores"] and r["cpu_model"]
    assert one["cores"] == 1
    assert 1 <= many["cores"] <= w.B * w.H
