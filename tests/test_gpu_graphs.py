"""The entry points are asynchronous on their stream and allocate nothing, so a sequence of
them can be captured into a CUDA graph once and replayed: prefill, split-KV decode, paged
decode, the backward pass and the FP8 quantizer plus prefill are captured together, and
every replay must give bit for bit what eager calls give on the same inputs -- also after
the inputs were overwritten in place between replays."""
import numpy as np
import pytest
import torch

import workloads
from io_aware_softmax_b200 import (attn_bwd, attn_decode, attn_decode_paged, attn_fwd,
                                   attn_fwd_fp8, bwd_workspace_bytes, decode_workspace_bytes,
                                   device_status, quantize_fp8)

pytestmark = pytest.mark.gpu


def _inputs(seed):
    g = {}
    g["q"], g["k"], g["v"], g["do"] = (workloads.randn_bf16((1, 4, 300, 128), seed, i).cuda()
                                       for i in range(4))
    g["qd"] = workloads.randn_bf16((2, 8, 1, 128), seed, 4).cuda()
    g["kc"] = workloads.randn_bf16((2, 2, 700, 128), seed, 5).cuda()
    g["vc"] = workloads.randn_bf16((2, 2, 700, 128), seed, 6).cuda()
    g["kp"] = workloads.randn_bf16((12, 2, 64, 128), seed, 7).cuda()
    g["vp"] = workloads.randn_bf16((12, 2, 64, 128), seed, 8).cuda()
    return g


def _run(g, o):
    """Every call writes into preallocated outputs; returns nothing (graph-safe)."""
    attn_fwd(g["q"], g["k"], g["v"], mask="causal", out=o["o"], lse=o["lse"])
    attn_bwd(g["q"], g["k"], g["v"], o["o"], o["lse"], g["do"], mask="causal", dq=o["dq"],
             dk=o["dk"], dv=o["dv"], workspace=o["wsb"])
    attn_decode(g["qd"], g["kc"], g["vc"], num_splits=3, workspace=o["wsd"], out=o["od"],
                lse=o["ld"])
    attn_decode_paged(g["qd"], g["kp"], g["vp"], o["table"], o["lens"], num_splits=3,
                      workspace=o["wsp"], out=o["op"], lse=o["lp"])


def _outputs():
    o = {"o": torch.empty((1, 4, 300, 128), dtype=torch.bfloat16, device="cuda"),
         "lse": torch.empty((1, 4, 300), dtype=torch.float32, device="cuda")}
    for n in ("dq", "dk", "dv"):
        o[n] = torch.empty((1, 4, 300, 128), dtype=torch.bfloat16, device="cuda")
    o["wsb"] = torch.empty(bwd_workspace_bytes(1, 4, 300), dtype=torch.uint8, device="cuda")
    o["wsd"] = torch.empty(decode_workspace_bytes(2, 8, 128, 3), dtype=torch.uint8, device="cuda")
    o["wsp"] = torch.empty(decode_workspace_bytes(2, 8, 128, 3), dtype=torch.uint8, device="cuda")
    for n, l in (("od", "ld"), ("op", "lp")):
        o[n] = torch.empty((2, 8, 1, 128), dtype=torch.bfloat16, device="cuda")
        o[l] = torch.empty((2, 8, 1), dtype=torch.float32, device="cuda")
    o["table"] = torch.from_numpy(np.random.default_rng(1).permutation(12).astype(np.int32)
                                  .reshape(2, 6)).cuda()
    o["lens"] = torch.tensor([350, 129], dtype=torch.int32, device="cuda")
    return o


def test_capture_and_replay_matches_eager_bit_for_bit():
    g = _inputs(31)
    eager = _outputs()
    _run(g, eager)
    torch.cuda.synchronize()
    assert device_status() == 0
    cap = _outputs()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        _run(g, cap)                      # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        _run(g, cap)
    for n in cap:
        if n not in ("table", "lens") and not n.startswith("ws"):
            cap[n].zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert device_status() == 0
    for n in ("o", "lse", "dq", "dk", "dv", "od", "ld", "op", "lp"):
        assert torch.equal(cap[n], eager[n]), n
    # new inputs in place: the replay reads them, as eager calls would
    g2 = _inputs(32)
    for n in g:
        g[n].copy_(g2[n])
    eager2 = _outputs()
    _run(g2, eager2)
    graph.replay()
    torch.cuda.synchronize()
    assert device_status() == 0
    for n in ("o", "lse", "dq", "dk", "dv", "od", "ld", "op", "lp"):
        assert torch.equal(cap[n], eager2[n]), n
        assert not torch.equal(cap[n], eager[n]), n


def test_fp8_quantize_and_prefill_capture():
    q, k, v = (workloads.randn_bf16((1, 2, 260, 128), 40, i).cuda() for i in range(3))
    signs = torch.from_numpy(np.random.default_rng(4).choice([-1.0, 1.0], 128)
                             .astype(np.float32)).cuda()

    def run():
        q8, qs = quantize_fp8(q, block_rows=128, signs=signs)
        k8, ks = quantize_fp8(k, block_rows=128, signs=signs)
        vt8, vs = quantize_fp8(v, block_rows=260, transpose=True)
        return attn_fwd_fp8(q8, qs, k8, ks, vt8, vs[:, :, 0], mask="causal")

    o_ref, l_ref = run()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        o_cap, l_cap = run()
    graph.replay()
    torch.cuda.synchronize()
    assert device_status() == 0
    assert torch.equal(o_cap, o_ref) and torch.equal(l_cap, l_ref)
