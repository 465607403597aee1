"""A DiT block's linear layers (adaptive-norm modulation on AWQ W4A16, the
fused QKV projection, the attention output projection and the GELU MLP) run
eagerly, replayed from a CUDA graph, and with programmatic dependent launch
switched off: the results must not depend on how the launches were issued.
The layers that have no atomic sums (everything except the MLP's low-rank
activation) must agree bit for bit."""
import os

import pytest
import torch

import bench
import workloads as wl

pytestmark = pytest.mark.gpu


def _snapshot(out):
    return {k: v.clone() for k, v in out.items()}


def _assert_same(a, b, what):
    for k in ("mod", "qkv", "attn_out"):
        assert torch.equal(a[k], b[k]), f"{what}: {k} differs"
    d = (a["mlp"].float() - b["mlp"].float()).abs().max().item()
    assert d <= 2e-2 * a["mlp"].float().abs().max().item(), f"{what}: mlp differs by {d}"


@pytest.mark.parametrize("M", [384, 129])
def test_block_graph_and_pdl_invariance(M):
    import bit_w4a4_diffusion_b200 as B
    run, out, _ = bench.block_layers(B, wl, torch.device("cuda:0"), M)
    run()
    torch.cuda.synchronize()
    eager = _snapshot(out)
    for v in out.values():
        v.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            run()
    torch.cuda.current_stream().wait_stream(s)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    _assert_same(eager, _snapshot(out), "graph replay")
    os.environ["SVDQ_PDL"] = "0"
    try:
        for v in out.values():
            v.zero_()
        run()
        torch.cuda.synchronize()
    finally:
        os.environ.pop("SVDQ_PDL", None)
    _assert_same(eager, _snapshot(out), "without PDL")
    del g
