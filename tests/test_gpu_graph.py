"""The whole forward (hash, sort, attention with the fused combine) captured
once into a CUDA graph and replayed: the replay gives exactly the eager
results, and replaying after new inputs are copied into the captured buffers
gives exactly the eager results on those inputs."""
import pytest
import torch

import lsh_attention_long_b200 as L
from lsh_attention_long_b200 import workloads as W

pytestmark = pytest.mark.gpu

NB, CHUNK, CAUSAL = 64, 64, True


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from lsh_attention_long_b200 import build
    build.build()
    L.load_library()


def _inputs(seed):
    inp = W.make_random(1, 4, 1024, 64, NB, 3, torch.bfloat16, seed=seed)
    return [inp[k].cuda() for k in ("Q", "V", "rot")]


def test_forward_replays_from_a_cuda_graph():
    Q, V, rot = _inputs(21)
    shape = L.make_shape(1, 4, 1024, 64, NB, 3, CHUNK, CAUSAL, Q.dtype)
    ws = L.workspace(shape, Q.device)
    out = L.lsh_forward(Q, V, rot, NB, CHUNK, CAUSAL, ws=ws)  # eager, also sets up the library
    torch.cuda.synchronize()
    assert L.lsh_device_status() == 0
    ref = {k: v.clone() for k, v in out.items()}

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        L.lsh_forward(Q, V, rot, NB, CHUNK, CAUSAL, out=out, ws=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        L.lsh_forward(Q, V, rot, NB, CHUNK, CAUSAL, out=out, ws=ws)
    for t in out.values():
        t.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert L.lsh_device_status() == 0
    for k in ref:
        assert torch.equal(out[k], ref[k]), k

    Q2, V2, _ = _inputs(22)
    eager2 = L.lsh_forward(Q2, V2, rot, NB, CHUNK, CAUSAL)
    Q.copy_(Q2)
    V.copy_(V2)
    graph.replay()
    torch.cuda.synchronize()
    assert L.lsh_device_status() == 0
    for k in ref:
        assert torch.equal(out[k], eager2[k]), k
    del graph
