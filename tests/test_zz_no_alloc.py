"""attn_fwd_noalloc: the allocation-free entry point, on the GPU.

Some callers cannot allocate device memory (a plugin whose host framework
owns all device memory, a fixed memory plan, a path that cannot afford
cudaMalloc's device-wide synchronisation); attn_fwd_noalloc serves them by
taking its split-mode scratch from a fixed array inside the library.  These
tests call it through the C ABI and compare it with attn_fwd_ws (the same
kernel with a caller workspace) on two calls in a row, within the parity
tolerances.  This file is collected last so that a failure here leaves every
other test already run; it passes alone in a fresh process as well.
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_153_b200 as A
from exact_attention_153_b200 import build_lib
from seeded_inputs import make_qkv

pytestmark = pytest.mark.gpu

TOL = {"fp16": 4e-3, "bf16": 2e-2}
LSE_TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def built():
    build_lib.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _call_noalloc(q, k, v, o, lse, causal, scale, dtype_code):
    B, H, Nq, d = q.shape
    st = A.attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                            lse.data_ptr(), B, H, Nq, k.shape[2], d, scale, causal, dtype_code,
                            torch.cuda.current_stream().cuda_stream)
    return st


@pytest.mark.parametrize("B,H,Nq,Nk,d,dtype", [
    (1, 1, 2000, 2000, 64, "fp16"),   # split mode over 128 CTAs, 16 pieces per unit
    (1, 2, 300, 4000, 64, "bf16"),    # split mode, empty second tile in the last pair
    (16, 4, 1600, 1600, 64, "fp16"),  # 40x40 YOLO shape: unit mode (dual units), no scratch
    (1, 2, 400, 400, 64, "fp16"),     # 20x20 YOLO shape: unit mode, no scratch
])
def test_noalloc_matches_workspace_entry(B, H, Nq, Nk, d, dtype):
    q, k, v = (t.cuda() for t in make_qkv(B, H, Nq, Nk, d, dtype, seed=Nq + Nk))
    scale = 1.0 / math.sqrt(d)
    code = A.ATTN_BF16 if dtype == "bf16" else A.ATTN_FP16
    ws = A.workspace_for(q, k, False)
    o_ref, l_ref = A.forward(q, k, v, causal=False, scale=scale, workspace=ws)
    for _ in range(2):  # two calls in a row share (and must clear) the fixed scratch
        o = torch.full_like(q, float("nan"))
        lse = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device="cuda")
        assert _call_noalloc(q, k, v, o, lse, False, scale, code) == 0
        torch.cuda.synchronize()
        assert A.attn_get_device_status()[0] == 0
        eo = float((o.double() - o_ref.double()).abs().max())
        el = float((lse.double() - l_ref.double()).abs().max())
        assert eo <= TOL[dtype] and el <= LSE_TOL, (eo, el)


@pytest.mark.parametrize("B,H,N,split", [(1, 2, 2000, True), (16, 4, 700, False)])
def test_noalloc_causal(B, H, N, split):
    """Causal shapes: a small grid takes split mode from the fixed scratch and gives the bits of
    attn_fwd_ws; a full grid needs no scratch and gives the bits of attn_fwd."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert A.attn_plan(B, H, N, N, 64, 1, sms)["split"] == int(split)
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, N, 64, "fp16", seed=3))
    ws = A.workspace_for(q, k, True)
    assert (ws is not None) == split
    o_ref, l_ref = A.forward(q, k, v, causal=True, workspace=ws)
    for _ in range(2):  # two calls in a row share (and must clear) the fixed scratch
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
        assert _call_noalloc(q, k, v, o, lse, True, 0.125, A.ATTN_FP16) == 0
        torch.cuda.synchronize()
        assert A.attn_get_device_status()[0] == 0
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


def test_noalloc_rejects_plans_beyond_its_scratch():
    # d = 128 split over 148 CTAs needs ~39 MB of scratch: more than the fixed 24 MiB
    B, H, Nq, Nk, d = 2, 2, 512, 8192, 128
    plan = A.attn_plan(B, H, Nq, Nk, d, 0, torch.cuda.get_device_properties(0).multi_processor_count)
    assert plan["split"] == 1 and plan["workspace_bytes"] > (24 << 20)
    q, k, v = (t.cuda() for t in make_qkv(B, H, Nq, Nk, d, "bf16", seed=4))
    o = torch.zeros_like(q)
    lse = torch.zeros((B, H, Nq), dtype=torch.float32, device="cuda")
    assert _call_noalloc(q, k, v, o, lse, False, 1 / math.sqrt(d), A.ATTN_BF16) == 10
    torch.cuda.synchronize()
    assert int(o.abs().sum()) == 0  # nothing was launched
