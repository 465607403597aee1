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


@pytest.mark.parametrize("M", [129, 384])
def test_block_layers_match_oracle(M):
    """Each layer of the graph-replayed block against its oracle: the AWQ
    modulation, the QKV projection with RMSNorm and RoPE and the attention
    output projection within the layer bound; the MLP with the bounds of the
    GELU-MLP tests (its hidden decisions are read back from the workspace,
    where the MLP, the block's last layer, left them)."""
    import numpy as np
    import bit_w4a4_diffusion_b200 as B
    from oracle import awq as OA
    from oracle import calibrate as OC
    from oracle import qkv as OQ
    from oracle import svdq as O
    from tests.helpers import assert_output_close
    from tests.test_gpu_mlp import _assert_mlp_output, _check_hidden

    run, out, _ = bench.block_layers(B, wl, torch.device("cuda:0"), M, calibrate=OC.calibrate)
    inp = run.inputs
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            run()
    torch.cuda.current_stream().wait_stream(s)
    for v in out.values():
        v.zero_()
    g.replay()
    torch.cuda.synchronize()
    got = {k: v.float().cpu().numpy() for k, v in out.items()}

    a = inp["awq"]
    q4, sc, z = OA.awq_quantize(a.W)
    assert_output_close(got["mod"], OA.awq_linear(a.x, q4, sc, z)[1], "block: AWQ modulation")

    q = inp["qkv"]
    pw = O.pack_weights("nvfp4", q.W, q.lam, q.L1, q.L2)
    act = O.quantize_activations("nvfp4", q.x, pw["inv_lam"], np.float32(q.act_scale))
    gq, gk, cos, sin = inp["rope"]
    ref = OQ.qkv_layer_f64(act, pw, q.L1, q.L2, q.bias, gq, gk, cos, sin, inp["heads"])
    assert_output_close(got["qkv"], ref, "block: QKV + RMSNorm + RoPE")

    o = inp["attn_out"]
    pw = O.pack_weights("nvfp4", o.W, o.lam, o.L1, o.L2)
    act = O.quantize_activations("nvfp4", o.x, pw["inv_lam"], np.float32(o.act_scale))
    assert_output_close(got["attn_out"], O.linear_f64("nvfp4", act, pw, o.L1, o.L2, o.bias), "block: attn out")

    iu, idn = inp["mlp_up"], inp["mlp_down"]
    K, N = iu.case.K, iu.case.N
    pk_u = B.svdq_pack_weights("nvfp4", iu.W_bits, iu.lam, iu.L1_bits, iu.L2_bits)
    pk_d = B.svdq_pack_weights("nvfp4", idn.W_bits, idn.lam, idn.L1_bits, idn.L2_bits)
    ws = inp["workspace"]
    # the MLP's workspace: [up layer's | down layer's | work]
    base = B.workspace_bytes("nvfp4", M, N, K)
    oh = B.workspace_offsets("nvfp4", M, K, N)
    hc = ws[base + oh[1]:base + oh[1] + M * N // 2].view(M, N // 2)
    hs = ws[base + oh[2]:base + oh[2] + B.act_scale_bytes("nvfp4", M, N)]
    hl = ws[base + oh[3]:base + oh[3] + M * 128].view(torch.bfloat16).view(M, 64)
    v, h = _check_hidden(iu, idn, pk_u, pk_d, hc, hs, hl)
    ref_d = O.pack_weights("nvfp4", idn.W, idn.lam, idn.L1, idn.L2)
    y64 = O.linear_f64("nvfp4", h, ref_d, idn.L1, idn.L2, idn.bias)
    # 12288 hidden codes per row: most rows carry a few flipped decisions, so
    # the layer bound applies to the (few) rows that carry none.
    _assert_mlp_output(got["mlp"], y64, hc, hs, h, M, N, "block: GELU MLP")
    del g
