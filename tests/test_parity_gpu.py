"""GPU parity: the sm_100a kernel against the float64 CPU oracle.

Bar (fixed for every case): max |O_gpu - O_oracle| <= 4e-3 for fp16 and 2e-2
for bf16; max |lse_gpu - lse_oracle| <= 1e-3.  Inputs are the seeded
workloads; the oracle sees exactly the fp16 / bf16 values the GPU sees.
Every case compares every element of O and lse, the five full-size
workloads included (the three large ones with the oracle spread over a
process pool, one (batch, head) slice per task).
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_153_b200 as A
import oracle
from exact_attention_153_b200 import build_lib
from seeded_inputs import WORKLOADS, make_qkv, make_workload_qkv

pytestmark = pytest.mark.gpu

TOL = {"fp16": 4e-3, "bf16": 2e-2}
LSE_TOL = 1e-3
SENTINEL = 0x7E01  # a NaN pattern in fp16 and bf16 alike; the kernel never writes it


@pytest.fixture(scope="module", autouse=True)
def built():
    build_lib.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _run(q, k, v, causal, scale):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = A.forward(qd, kd, vd, causal=causal, scale=scale)
    torch.cuda.synchronize()
    st, word = A.attn_get_device_status()
    assert st == 0, f"device status {word:#x}"
    return o.cpu(), lse.cpu()


def _err(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))))


def _check_full(q, k, v, causal, scale, dtype):
    o, lse = _run(q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attention_f64(q, k, v, scale, causal)
    eo = _err(o.double().numpy(), o_ref)
    el = _err(lse.double().numpy(), lse_ref)
    assert eo <= TOL[dtype], f"O err {eo:.3e}"
    assert el <= LSE_TOL, f"lse err {el:.3e}"
    return eo, el


SQUARE = [1, 7, 127, 128, 129, 255, 256, 257, 400, 1000]


@pytest.mark.parametrize("N", SQUARE)
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
def test_square_shapes(N, d, dtype, causal):
    q, k, v = make_qkv(2, 3, N, N, d, dtype, seed=N * 10 + d + (dtype == "bf16"))
    _check_full(q, k, v, causal, 1.0 / math.sqrt(d), dtype)


@pytest.mark.parametrize("Nq,Nk", [(100, 300), (300, 100), (513, 129), (1, 1000), (1000, 1),
                                   (129, 700), (640, 257)])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_rectangular_shapes(Nq, Nk, d, causal):
    dtype = "fp16" if d == 64 else "bf16"
    q, k, v = make_qkv(1, 2, Nq, Nk, d, dtype, seed=Nq + 7 * Nk + d)
    _check_full(q, k, v, causal, 1.0 / math.sqrt(d), dtype)


@pytest.mark.parametrize("scale", [0.01, 0.3, 1.0])
def test_other_scales(scale):
    q, k, v = make_qkv(1, 2, 300, 300, 64, "fp16", seed=5)
    _check_full(q, k, v, True, scale, "fp16")


def test_many_units_persistent_loop():
    """More work units than SMs: every CTA loops over several units."""
    q, k, v = make_qkv(8, 40, 257, 257, 64, "bf16", seed=11)
    _check_full(q, k, v, True, 0.125, "bf16")
    _check_full(q, k, v, False, 0.125, "bf16")


# ------------------------------------------------------------ the five workloads

@pytest.mark.parametrize("idx", [0, 1])
def test_workload_full_compare(idx):
    import time
    w = WORKLOADS[idx]
    q, k, v = make_workload_qkv(w)
    t0 = time.perf_counter()
    eo, el = _check_full(q, k, v, w.causal, w.scale, w.dtype)
    dt = time.perf_counter() - t0
    print(f"\nPARITY {w.name}: max|dO| {eo:.3e} (tol {TOL[w.dtype]}), "
          f"max|dlse| {el:.3e} (tol {LSE_TOL}), {w.B * w.H} (batch, head) slices, "
          f"oracle and GPU {dt:.1f} s in one process")


@pytest.mark.parametrize("idx", [2, 3, 4])
def test_workload_full_parity(idx):
    """Every element of O and lse of the three large workloads against the oracle.

    The oracle runs one (batch, head) slice per task in a spawn-started process
    pool; the GPU output is compared element by element, with the same bar as
    every other case.
    """
    from tests.oracle_pool import compare_all_slices
    import time
    from tests.oracle_pool import workers
    w = WORKLOADS[idx]
    q, k, v = make_workload_qkv(w)
    o, lse = _run(q, k, v, w.causal, w.scale)
    t0 = time.perf_counter()
    worst_o, worst_l, per_slice = compare_all_slices(q, k, v, o, lse, w.scale, w.causal)
    dt = time.perf_counter() - t0
    assert len(per_slice) == w.B * w.H
    print(f"\nPARITY {w.name}: max|dO| {worst_o:.3e} (tol {TOL[w.dtype]}), "
          f"max|dlse| {worst_l:.3e} (tol {LSE_TOL}), {len(per_slice)} (batch, head) slices, "
          f"oracle {dt:.1f} s on {workers()} processes")
    assert worst_o <= TOL[w.dtype], f"O err {worst_o:.3e}"
    assert worst_l <= LSE_TOL, f"lse err {worst_l:.3e}"


# ------------------------------------------------------------ invariants on the GPU

@pytest.mark.parametrize("causal", [False, True])
def test_constant_v(causal):
    q, k, _ = make_qkv(2, 2, 300, 300, 64, "fp16", seed=21)
    r = torch.randn(64, generator=torch.Generator().manual_seed(3)).half()
    v = r.expand(2, 2, 300, 64).contiguous()
    o, _ = _run(q, k, v, causal, 0.125)
    assert _err(o.double().numpy(), np.broadcast_to(r.double().numpy(), o.shape)) <= TOL["fp16"]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_q_zero_closed_form(causal, d):
    N = 333
    _, k, v = make_qkv(1, 2, N, N, d, "bf16", seed=22)
    q = torch.zeros(1, 2, N, d, dtype=torch.bfloat16)
    o, lse = _run(q, k, v, causal, 1.0 / math.sqrt(d))
    vf = v.double().numpy()
    if causal:
        mean = np.cumsum(vf, axis=2) / np.arange(1, N + 1)[None, None, :, None]
        lse_ref = np.broadcast_to(np.log(np.arange(1, N + 1)), (1, 2, N))
    else:
        mean = np.broadcast_to(vf.mean(axis=2, keepdims=True), vf.shape)
        lse_ref = np.full((1, 2, N), math.log(N))
    assert _err(o.double().numpy(), mean) <= TOL["bf16"]
    assert _err(lse.double().numpy(), lse_ref) <= LSE_TOL


def test_causal_row0_is_v0():
    q, k, v = make_qkv(2, 4, 500, 500, 128, "bf16", seed=23)
    o, lse = _run(q, k, v, True, 1.0 / math.sqrt(128))
    assert torch.equal(o[:, :, 0], v[:, :, 0])
    s00 = (q[:, :, 0].double() * k[:, :, 0].double()).sum(-1) / math.sqrt(128)
    assert _err(lse[:, :, 0].double().numpy(), s00.numpy()) <= LSE_TOL


def test_single_key():
    q, k, v = make_qkv(1, 3, 200, 1, 64, "fp16", seed=24)
    o, _ = _run(q, k, v, False, 0.125)
    assert torch.equal(o, v.expand_as(o))


def test_dominant_key():
    q, k, v = make_qkv(1, 1, 256, 256, 64, "fp16", seed=25)
    i, j = 77, 200
    qi = q[0, 0, i].double()
    k[0, 0, j] = (30.0 * qi / qi.norm()).half()  # gap of ~30 / sqrt(64) * |q_i| in the exponent
    o, _ = _run(q, k, v, False, 1.0)
    assert _err(o[0, 0, i].double().numpy(), v[0, 0, j].double().numpy()) <= TOL["fp16"]


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_late_keys_raise_the_running_max(dtype):
    """Keys in later tiles whose scores exceed every earlier score by 12, 20 and 40 (base 2):
    12 stays on the stale-max path (P up to 2^12), 20 and 40 force the row max and a raise."""
    q, k, v = make_qkv(1, 2, 600, 900, 64, dtype, seed=26)
    scale = 0.125
    log2e = 1.4426950408889634
    for n, (row, key, gap) in enumerate([(5, 300, 12.0), (130, 520, 20.0), (257, 777, 40.0),
                                         (400, 899, 20.0), (599, 640, 12.0)]):
        qi = q[0, n % 2, row].double()
        # score of (row, key) = scale * |q_row| * a, in base 2: gap above the row's other scores
        a = (gap / log2e + 4.0) / (scale * float(qi.norm()))
        k[0, n % 2, key] = (a * qi / qi.norm()).to(k.dtype)
    _check_full(q, k, v, False, scale, dtype)


# Keys 0-7, 32-39, 64-71 and 96-103 of a 128-key tile take 2^x from the FMA-pipe polynomial on the
# d = 64 stale-max path; a key there whose base-2 score lies 150-300 above the running max must
# still win its row (the dominant-key invariant), not wrap to a tiny or negative weight.
POLY_COLUMNS = [0, 33, 70, 101]


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
def test_dominant_key_in_polynomial_slots(dtype, causal):
    N, d, scale = 640, 64, 0.125
    log2e = 1.4426950408889634
    q, k, v = make_qkv(1, 2, N, N, d, dtype, seed=41 + causal)
    if causal:
        plants = [(300, 128 + 0, 150.0), (301, 128 + 33, 200.0), (450, 384 + 33, 300.0),
                  (600, 384 + 70, 150.0), (602, 384 + 101, 250.0), (260, 128 + 101, 300.0)]
    else:
        plants = [(5, 128 + 0, 150.0), (130, 128 + 33, 200.0), (7, 384 + 70, 300.0),
                  (250, 384 + 101, 150.0), (131, 384 + 0, 250.0), (600, 128 + 70, 300.0)]
    for n, (row, key, gap) in enumerate(plants):
        h = n % 2
        qi = q[0, h, row].double()
        qn = float(qi.norm())
        s_other = float((k[0, h].double() @ qi).abs().max()) * scale
        # base-2 score of (row, key): gap above every other score of the row
        a = (gap / log2e + s_other) / (scale * qn)
        k[0, h, key] = (a * qi / qn).to(k.dtype)
    o, lse = _run(q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attention_f64(q, k, v, scale, causal)
    for n, (row, key, _) in enumerate(plants):
        assert _err(o_ref[0, n % 2, row], v[0, n % 2, key].double().numpy()) <= 1e-6
    assert _err(o.double().numpy(), o_ref) <= TOL[dtype]
    assert _err(lse.double().numpy(), lse_ref) <= LSE_TOL


# ------------------------------------------------------------ memory safety, determinism

@pytest.mark.parametrize("Nq,d,dtype", [(400, 64, "fp16"), (129, 128, "bf16"), (1, 64, "bf16")])
def test_canary_bands(Nq, d, dtype):
    """Rows past Nq, and memory around O and lse, are never written."""
    B, H = 2, 3
    q, k, v = make_qkv(B, H, Nq, 300, d, dtype, seed=26)
    t = q.dtype
    pad = 4096
    n_o = B * H * Nq * d
    o_buf = torch.full((n_o + 2 * pad,), 0, dtype=torch.int16, device="cuda")
    o_buf.fill_(SENTINEL)
    o_buf = o_buf.view(t)
    l_buf = torch.full((B * H * Nq + 2 * pad,), float("nan"), dtype=torch.float32, device="cuda")
    o = o_buf[pad:pad + n_o].view(B, H, Nq, d)
    lse = l_buf[pad:pad + B * H * Nq].view(B, H, Nq)
    A.forward(q.cuda(), k.cuda(), v.cuda(), causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    ob = o_buf.view(torch.int16).cpu()
    assert (ob[:pad] == SENTINEL).all() and (ob[pad + n_o:] == SENTINEL).all()
    lb = l_buf.cpu()
    assert torch.isnan(lb[:pad]).all() and torch.isnan(lb[pad + B * H * Nq:]).all()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    o_ref, l_ref = oracle.attention_f64(q, k, v, 1.0 / math.sqrt(d), True)
    assert _err(o.cpu().double().numpy(), o_ref) <= TOL[dtype]
    assert _err(lse.cpu().double().numpy(), l_ref) <= LSE_TOL


def test_lse_null_skips_lse():
    q, k, v = make_qkv(1, 2, 200, 200, 64, "fp16", seed=27)
    o, lse = A.forward(q.cuda(), k.cuda(), v.cuda(), causal=False, return_lse=False)
    assert lse is None
    o2, _ = A.forward(q.cuda(), k.cuda(), v.cuda(), causal=False)
    assert torch.equal(o, o2)


@pytest.mark.parametrize("idx", [1, 3])
def test_deterministic(idx):
    w = WORKLOADS[idx]
    q, k, v = (t.cuda() for t in make_workload_qkv(w))
    o1, l1 = A.forward(q, k, v, causal=w.causal)
    o2, l2 = A.forward(q, k, v, causal=w.causal)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_host_entry_matches_device_entry():
    w = WORKLOADS[0]
    q, k, v = make_workload_qkv(w)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32).pin_memory()
    qd, kd, vd = (torch.empty_like(t, device="cuda") for t in (q, k, v))
    od = torch.empty_like(qd)
    ld = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device="cuda")
    A.forward_host(qh, kh, vh, oh, lh, qd, kd, vd, od, ld, causal=w.causal)
    torch.cuda.synchronize()
    o, lse = A.forward(q.cuda(), k.cuda(), v.cuda(), causal=w.causal)
    torch.cuda.synchronize()
    assert torch.equal(oh, o.cpu()) and torch.equal(lh, lse.cpu())


def test_device_errors_do_not_launch():
    q = torch.zeros(1, 1, 8, 64, dtype=torch.float16, device="cuda")
    base = q.data_ptr()
    st = A.attn_fwd(base + 2, base, base, base, None, 1, 1, 8, 8, 64, 0.1, 0, 0, 0)
    assert st == 5
    st = A.attn_fwd(base, base, base, base, None, 1, 1, 8, 8, 80, 0.1, 0, 0, 0)
    assert st == 3
    assert A.attn_get_device_status()[0] == 0


# ------------------------------------------------------------ split mode (attn_fwd_ws)

def _run_ws(q, k, v, causal, scale):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ws = A.workspace_for(qd, kd, causal)
    o, lse = A.forward(qd, kd, vd, causal=causal, scale=scale, workspace=ws)
    torch.cuda.synchronize()
    st, word = A.attn_get_device_status()
    assert st == 0, f"device status {word:#x}"
    return o.cpu(), lse.cpu(), ws


def test_small_workloads_take_unit_mode():
    """The YOLO 20x20 workload (4 units of 4 key tiles) is faster without split pieces."""
    w = WORKLOADS[0]
    q, k, v = make_workload_qkv(w)
    o, lse, ws = _run_ws(q, k, v, w.causal, w.scale)
    assert ws is None
    o_ref, l_ref = oracle.attention_f64(q, k, v, w.scale, w.causal)
    assert _err(o.double().numpy(), o_ref) <= TOL[w.dtype]
    assert _err(lse.double().numpy(), l_ref) <= LSE_TOL


@pytest.mark.parametrize("B,H,Nq,Nk,d,dtype", [
    (1, 1, 2000, 2000, 64, "fp16"),    # 8 units x 16 key tiles on 128 CTAs: 16 pieces per unit
    (1, 1, 3000, 3000, 64, "bf16"),    # 2 or 3 steps per CTA: pieces start mid-unit, ragged keys
    (1, 2, 300, 4000, 64, "bf16"),     # odd query tiles: tile 1 of the last pair is empty
    (2, 2, 512, 8192, 128, "fp16"),    # d = 128, 148 CTAs, ~19 pieces per unit
])
def test_split_many_pieces(B, H, Nq, Nk, d, dtype):
    q, k, v = make_qkv(B, H, Nq, Nk, d, dtype, seed=Nq + Nk + d)
    scale = 1.0 / math.sqrt(d)
    o, lse, ws = _run_ws(q, k, v, False, scale)
    assert ws is not None
    o_ref, l_ref = oracle.attention_f64(q, k, v, scale, False)
    assert _err(o.double().numpy(), o_ref) <= TOL[dtype]
    assert _err(lse.double().numpy(), l_ref) <= LSE_TOL


@pytest.mark.parametrize("B,H,Nq,Nk,d,dtype", [
    (1, 1, 4096, 4096, 64, "fp16"),    # 8 causal units -> 272 key-tile steps on 148 CTAs
    (1, 1, 2000, 2000, 64, "bf16"),    # 72 steps: first tiles of late pieces see no key
    (1, 2, 4096, 4096, 128, "fp16"),   # d = 128, 544 steps on 148 CTAs
    (1, 4, 2048, 2048, 64, "fp16"),
    (1, 1, 3000, 1000, 64, "bf16"),    # Nq > Nk: later pairs see every key tile
    (1, 1, 2500, 8000, 64, "bf16"),    # Nq < Nk: most key tiles hidden from every query
])
def test_split_causal(B, H, Nq, Nk, d, dtype):
    assert A.attn_plan(B, H, Nq, Nk, d, 1, torch.cuda.get_device_properties(0).multi_processor_count)["split"] == 1
    q, k, v = make_qkv(B, H, Nq, Nk, d, dtype, seed=Nq + 3 * Nk + d)
    scale = 1.0 / math.sqrt(d)
    o, lse, ws = _run_ws(q, k, v, True, scale)
    assert ws is not None
    o_ref, l_ref = oracle.attention_f64(q, k, v, scale, True)
    assert _err(o.double().numpy(), o_ref) <= TOL[dtype]
    assert _err(lse.double().numpy(), l_ref) <= LSE_TOL
    # a second call on the same workspace gives the same bits (the counters were reset)
    o2, lse2, _ = _run_ws(q, k, v, True, scale)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_split_workspace_reuse_is_deterministic():
    """Reusing one workspace gives the same bits: each call leaves the counters at zero."""
    q, k, v = (t.cuda() for t in make_qkv(1, 2, 1500, 1500, 64, "fp16", seed=31))
    ws = A.workspace_for(q, k, False)
    o1, l1 = A.forward(q, k, v, workspace=ws)
    o2, l2 = A.forward(q, k, v, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o3, l3 = A.forward(q, k, v)  # unsplit
    torch.cuda.synchronize()
    n_units = A.attn_plan(1, 2, 1500, 1500, 64, 0, 148)["split_units"]
    counters = ws[-(n_units * 4 + 16):-16].view(torch.int32)
    assert int(counters.abs().sum()) == 0
    assert _err(o1.cpu().double().numpy(), o3.cpu().double().numpy()) <= TOL["fp16"]
    assert _err(l1.cpu().double().numpy(), l3.cpu().double().numpy()) <= LSE_TOL


def test_split_small_workspace_falls_back_to_units():
    """A workspace that is too small is ignored (same as attn_fwd), not overrun."""
    assert A.attn_plan(1, 1, 2000, 2000, 64, 0, 148)["split"] == 1
    q, k, v = (t.cuda() for t in make_qkv(1, 1, 2000, 2000, 64, "fp16", seed=32))
    small = torch.zeros(64, dtype=torch.uint8, device="cuda")
    o1, l1 = A.forward(q, k, v, workspace=small)
    o2, l2 = A.forward(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert int(small.sum()) == 0


def test_host_entry_with_workspace():
    w = WORKLOADS[1]
    q, k, v = make_workload_qkv(w)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32).pin_memory()
    qd, kd, vd = (torch.empty_like(t, device="cuda") for t in (q, k, v))
    od = torch.empty_like(qd)
    ld = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device="cuda")
    ws = A.workspace_for(qd, kd, w.causal)
    A.forward_host(qh, kh, vh, oh, lh, qd, kd, vd, od, ld, causal=w.causal, workspace=ws)
    torch.cuda.synchronize()
    o, lse = A.forward(q.cuda(), k.cuda(), v.cuda(), causal=w.causal, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(oh, o.cpu()) and torch.equal(lh, lse.cpu())


# ------------------------------------------------------------ dual units (unit mode)

@pytest.mark.parametrize("B,H,Nq,Nk,d,dtype", [
    (1, 5, 300, 300, 64, "fp16"),     # odd head count: the last dual unit has one tile
    (2, 3, 1100, 700, 128, "bf16"),   # ragged last query tile, d = 128 (in-order issue)
    (4, 4, 100, 333, 64, "bf16"),     # one query tile per head: every unit is dual
    (3, 3, 850, 1000, 64, "fp16"),
])
def test_dual_units(B, H, Nq, Nk, d, dtype):
    """Odd query-tile counts pair the last tiles of two heads in one unit."""
    assert A.attn_plan(B, H, Nq, Nk, d, 0, 148)["dual_units"] == (B * H + 1) // 2
    q, k, v = make_qkv(B, H, Nq, Nk, d, dtype, seed=B * H + Nq + Nk)
    _check_full(q, k, v, False, 1.0 / math.sqrt(d), dtype)


def test_yolo_40x40_uses_dual_units_not_split():
    w = WORKLOADS[1]
    p = A.attn_plan(w.B, w.H, w.Nq, w.Nk, w.d, int(w.causal),
                    torch.cuda.get_device_properties(0).multi_processor_count)
    assert p["dual_units"] == 32 and p["num_units"] == 416 and p["split"] == 0


# ------------------------------------------------------------ pipelined host entry

@pytest.mark.parametrize("B,H,N,d,dtype,causal,with_lse", [
    (4, 8, 2048, 64, "fp16", True, True),     # 25 MB in: 8 chunks of 4 heads
    (1, 13, 1000, 128, "bf16", False, False),  # 13 heads: 7 chunks, the last with one head
    (16, 4, 1600, 64, "fp16", False, True),   # the 40x40 YOLO shape (dual units per chunk)
])
def test_host_entry_pipelined_matches_device_entry(B, H, N, d, dtype, causal, with_lse):
    """Chunked copies and forwards on library streams give the bits of attn_fwd, ordered on the
    caller's stream: earlier work on it finishes first, later work sees the results."""
    q, k, v = make_qkv(B, H, N, N, d, dtype, seed=B * H + N + d)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((B, H, N), dtype=torch.float32).pin_memory() if with_lse else None
    qd, kd, vd = (torch.empty_like(t, device="cuda") for t in (q, k, v))
    od = torch.empty_like(qd)
    ld = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        od.fill_(7.0)  # earlier work on the caller's stream
        torch.cuda._sleep(1_000_000)
        A.forward_host(qh, kh, vh, oh, lh, qd, kd, vd, od, ld, causal=causal, stream=side)
        o_after = od.clone()  # later work on the caller's stream
    side.synchronize()
    o, lse = A.forward(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(oh, o.cpu())
    assert torch.equal(o_after, o)
    if with_lse:
        assert torch.equal(lh, lse.cpu())
    assert A.attn_get_device_status()[0] == 0


@pytest.mark.parametrize("dtype,causal", [("bf16", True), ("fp16", False)])
def test_128k_context_sampled(dtype, causal):
    """The longest context the pages speak of (128K tokens, FA3 on a 70B model): one
    (batch, head) pair per head of B = 1, H = 2, N = 131072, d = 128, Q and K x 0.5 like the
    long-context workload.  The first, 32 seeded and the last 32 query rows of each head against
    all 131072 keys, within the forward's bars."""
    B, H, N, d = 1, 2, 131072, 128
    q, k, v = make_qkv(B, H, N, N, d, dtype, seed=131, qk_scale=0.5)
    scale = 1.0 / math.sqrt(d)
    o, lse = _run(q, k, v, causal, scale)
    rng = np.random.default_rng(131)
    rows = np.unique(np.concatenate([np.arange(32), rng.integers(32, N - 32, 32), np.arange(N - 32, N)]))
    for h in range(H):
        o_ref, l_ref = oracle.attention_head_rows(q[0, h, rows], k[0, h], v[0, h], scale, causal, rows)
        assert _err(o[0, h, rows].double().numpy(), o_ref) <= TOL[dtype]
        assert _err(lse[0, h, rows].double().numpy(), l_ref) <= LSE_TOL
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
