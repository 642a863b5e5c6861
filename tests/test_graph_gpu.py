"""The device entry points inside a CUDA graph: captured once, replayed, same bits as eager calls.

A model loop or a serving path replays its work from a CUDA graph to amortise launch latency
(the 20x20 YOLO call is launch-bound).  The entry points allocate nothing per call and never
synchronise, so after one eager call (which sets the kernels' shared-memory attribute) they can
be captured; these tests capture the forward (16-bit, split mode and e4m3), the backward and
the attention block, replay the graph on new inputs copied into the captured buffers, and
require the results of eager calls on the same inputs bit for bit.
"""
import math

import pytest
import torch

import exact_attention_153_b200 as A
from exact_attention_153_b200 import build_lib
from seeded_inputs import make_block_inputs, make_fp8_qkv, make_grad_out, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build_lib.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()  # eager warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


@pytest.mark.parametrize("B,H,N,d,dtype,causal", [(1, 2, 400, 64, "fp16", False),
                                                  (2, 2, 700, 128, "bf16", True),
                                                  (1, 1, 2000, 64, "fp16", True)])
def test_forward_graph_replay(B, H, N, d, dtype, causal):
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, N, d, dtype, seed=N + d))
    ws = A.workspace_for(q, k, causal)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    g = _capture(lambda: A.forward(q, k, v, causal=causal, out=o, lse=lse, workspace=ws))
    q2, k2, v2 = (t.cuda() for t in make_qkv(B, H, N, N, d, dtype, seed=N + d + 1))
    q.copy_(q2), k.copy_(k2), v.copy_(v2)
    g.replay()
    torch.cuda.synchronize()
    o_ref, l_ref = A.forward(q2, k2, v2, causal=causal, workspace=A.workspace_for(q2, k2, causal))
    torch.cuda.synchronize()
    assert A.attn_get_device_status()[0] == 0
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


def test_fp8_forward_graph_replay():
    q8, k8, vt8, ds = (x.cuda() if hasattr(x, "cuda") else x
                       for x in make_fp8_qkv(1, 2, 1000, 1024, 128, seed=5))
    o = torch.empty((1, 2, 1000, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 2, 1000), dtype=torch.float32, device="cuda")
    g = _capture(lambda: A.forward_fp8(q8, k8, vt8, ds, causal=True, out=o, lse=lse))
    g.replay()
    torch.cuda.synchronize()
    o_ref, l_ref = A.forward_fp8(q8, k8, vt8, ds, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


def test_backward_graph_replay():
    B, H, N, d = 1, 2, 500, 64
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, N, d, "fp16", seed=9))
    do = make_grad_out(B, H, N, d, "fp16", seed=9).cuda()
    o, lse = A.forward(q, k, v, causal=True)
    ws = torch.empty(A.attn_bwd_workspace_size(B, H, N, N, d), dtype=torch.uint8, device="cuda")
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    g = _capture(lambda: A.backward(q, k, v, o, lse, do, causal=True, workspace=ws, out=grads))
    g.replay()
    torch.cuda.synchronize()
    dq, dk, dv = A.backward(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    # dK and dV come from one CTA each and are deterministic; dQ sums key tiles in any order
    assert torch.equal(grads[1], dk) and torch.equal(grads[2], dv)
    assert float((grads[0].float() - dq.float()).abs().max()) <= 1e-3 * float(dq.float().abs().max())


def test_block_graph_replay():
    B, N, H, d = 2, 400, 4, 64
    x, w_qkv, b_qkv, w_o, b_o = (t.cuda() if t is not None else None
                                 for t in make_block_inputs(B, N, H, d, H * d, "bf16", 3))
    out = {}

    def run():
        out["y"] = A.block_forward(x, w_qkv, b_qkv, w_o, b_o, H)[0]

    run()
    torch.cuda.synchronize()
    y_ref = out["y"].clone()
    g = _capture(run)
    g.replay()
    torch.cuda.synchronize()
    y_graph = out["y"]
    assert torch.equal(y_graph, y_ref)
