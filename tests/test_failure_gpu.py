"""Failure detection on the GPU without a GPU fault.

Every wait inside the kernel is bounded (about one second of %globaltimer).
The test hook attn_fwd_stall_test points one wait at a barrier nothing ever
arrives on; the kernel must then record a timeout in its status word, let
every role leave its loop, wait for its own loads and MMAs, free tensor
memory and return.  The host reads ATTN_ERR_DEVICE_TIMEOUT, and the same
CUDA context then computes a correct result.  Nothing here traps, faults or
hangs the GPU: the stall ends by its time limit.
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_153_b200 as A
import oracle
from exact_attention_153_b200 import build_lib
from seeded_inputs import make_qkv

pytestmark = pytest.mark.gpu

TIMEOUT = 9
INJECTED = 0x8000000A


@pytest.fixture(scope="module", autouse=True)
def built():
    build_lib.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


CASES = [
    # (stall site, split mode, d)
    (1, False, 64), (2, False, 64), (3, False, 64), (2, False, 128), (1, False, 128),
    (1, True, 64), (2, True, 64), (4, True, 64), (4, True, 128),
]


@pytest.mark.parametrize("site,split,d", CASES)
def test_injected_stall_times_out_and_context_recovers(site, split, d):
    dtype = "fp16" if d == 64 else "bf16"
    code = A.ATTN_FP16 if d == 64 else A.ATTN_BF16
    if split:  # shapes for which attn_fwd_ws takes split mode
        B, H, N, Nk = (1, 1, 2000, 2000) if d == 64 else (2, 2, 512, 8192)
    else:
        B, H, N = 1, 2, 300
        Nk = N if d == 64 else 1700
    q, k, v = make_qkv(B, H, N, Nk, d, dtype, seed=site * 10 + d)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    ws = A.workspace_for(qd, kd, False) if split else None
    if split:
        assert ws is not None
    scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream().cuda_stream
    st = A.attn_fwd_stall_test(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(),
                               lse.data_ptr(), B, H, N, Nk, d, scale, 0, code,
                               ws.data_ptr() if ws is not None else None,
                               ws.numel() if ws is not None else 0, site, stream)
    assert st == 0
    status, word = A.attn_get_device_status()
    assert status == TIMEOUT, (status, hex(word))
    assert word & 0x80000000
    # The injected wait normally expires first; a role that was waiting on it
    # may time out in the same instant, so any timeout site is accepted.
    assert (word & 0xFF) in range(1, 11)
    # The status word was cleared by the read, and the context still works.
    assert A.attn_get_device_status() == (0, 0)
    if ws is not None:
        ws.zero_()  # a timed-out split call may leave piece counters set
    o2, l2 = A.forward(qd, kd, vd, causal=False, scale=scale, workspace=ws)
    torch.cuda.synchronize()
    assert A.attn_get_device_status()[0] == 0
    o_ref, l_ref = oracle.attention_f64(q, k, v, scale, False)
    tol = 4e-3 if dtype == "fp16" else 2e-2
    assert float(np.max(np.abs(o2.cpu().double().numpy() - o_ref))) <= tol
    assert float(np.max(np.abs(l2.cpu().double().numpy() - l_ref))) <= 1e-3


def test_stall_hook_rejects_unknown_site():
    q = torch.zeros(1, 1, 8, 64, dtype=torch.float16, device="cuda")
    p = q.data_ptr()
    st = A.attn_fwd_stall_test(p, p, p, p, None, 1, 1, 8, 8, 64, 0.125, 0, 0, None, 0, 7,
                               torch.cuda.current_stream().cuda_stream)
    assert st == 2
