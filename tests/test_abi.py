"""Host-side tests of the C ABI (no GPU needed).

* the library loads and exports every function ``include/attn.h`` declares;
* argument validation returns the documented code before any CUDA call;
* ``attn_plan`` gives the launch geometry the kernel uses;
* without a usable device a valid call fails loudly (ATTN_ERR_CUDA) -- there
  is no CPU fallback.
"""
import ctypes
import os
import re
import subprocess

import pytest

import exact_attention_153_b200 as A
from exact_attention_153_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    build_lib.build()


def header_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    assert header_functions() == sorted([
        "attn_fwd", "attn_fwd_ws", "attn_workspace_size", "attn_fwd_noalloc", "attn_fwd_host",
        "attn_fwd_stall_test", "attn_plan", "attn_get_device_status", "attn_strerror",
        "attn_version", "attn_bwd", "attn_bwd_workspace_size", "attn_qkv_proj", "attn_out_proj",
        "attn_block_fwd", "attn_fwd_fp8"])


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(A.library_path())
    for name in header_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", A.library_path()], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r"\bT (attn_\w+)", out))
    assert set(header_functions()) <= exported


def test_status_enum_matches_header():
    text = open(HEADER, encoding="utf-8").read()
    for code, name in A.STATUS_NAMES.items():
        assert re.search(rf"\b{name}\s*=\s*{code}\b", text), name


def test_strerror_and_version():
    for code in range(12):
        assert A.attn_strerror(code) != "unknown status"
    assert A.attn_strerror(1234) == "unknown status"
    assert A.attn_version() == 100


GOOD = dict(q=0x10000, k=0x20000, v=0x30000, o=0x40000, lse=0x50000, B=1, H=2, Nq=400, Nk=400,
            d=64, scale=0.125, causal=0, dtype=A.ATTN_FP16, stream=None)


def call(**kw):
    a = dict(GOOD)
    a.update(kw)
    return A.attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Nq"], a["Nk"],
                      a["d"], a["scale"], a["causal"], a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(k=None), 1), (dict(v=None), 1), (dict(o=None), 1),
    (dict(dtype=2), 4), (dict(dtype=-1), 4),
    (dict(d=32), 3), (dict(d=96), 3), (dict(d=256), 3),
    (dict(B=0), 2), (dict(H=0), 2), (dict(Nq=0), 2), (dict(Nk=0), 2), (dict(Nk=-5), 2),
    (dict(B=1 << 16, H=1 << 15), 2),
    (dict(q=0x10008), 5), (dict(o=0x40004), 5), (dict(lse=0x50002), 5),
    (dict(scale=0.0), 6), (dict(scale=-1.0), 6), (dict(scale=float("nan")), 6),
    (dict(scale=float("inf")), 6),
])
def test_argument_errors(kw, code):
    assert call(**kw) == code


def test_error_order_null_first():
    assert call(q=None, d=7, dtype=9) == 1
    assert call(dtype=9, d=7) == 4
    assert call(d=7, B=0) == 3


def test_lse_may_be_null():
    # With valid arguments the next step needs a device; this host has none
    # (or it is not an sm_100 part): the call must fail, not compute elsewhere.
    st = call(lse=None)
    assert st in (0, 7, 8)


def test_no_silent_fallback_without_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; covered by the gpu tests")
    assert call() == 8
    assert A.attn_get_device_status(0)[0] == 8


def test_host_entry_argument_errors():
    base = [0x1000] * 10 + [None, 0]
    args = dict(B=1, H=1, Nq=8, Nk=8, d=64, scale=0.125, causal=0, dtype=0, stream=None)
    assert A.attn_fwd_host(None, *base[1:], *args.values()) == 1
    ptrs = list(base)
    ptrs[5] = None  # q_dev
    assert A.attn_fwd_host(*ptrs, *args.values()) == 1
    args["d"] = 80
    assert A.attn_fwd_host(*base, *args.values()) == 3


def test_workspace_entry_argument_errors():
    a = dict(GOOD)
    assert A.attn_fwd_ws(None, a["k"], a["v"], a["o"], a["lse"], 1, 2, 400, 400, 64, 0.125, 0, 0,
                         0x60000, 1 << 20, None) == 1
    assert A.attn_fwd_ws(a["q"], a["k"], a["v"], a["o"], a["lse"], 1, 2, 400, 400, 96, 0.125, 0,
                         0, 0x60000, 1 << 20, None) == 3
    with pytest.raises(A.AttnError) as e:
        A.attn_workspace_size(1, 2, 400, 400, 80, 0)
    assert e.value.status == 3


def test_plan_geometry():
    p = A.attn_plan(1, 2, 400, 400, 64, 0, 148)
    assert (p["num_q_tiles"], p["num_q_pairs"], p["num_kv_tiles"], p["num_units"]) == (4, 2, 4, 4)
    # 4 units of 4 key tiles: splitting saves 3 serial steps, less than it costs to merge
    # 4 pieces per unit, so unit mode
    assert p["split"] == 0 and p["workspace_bytes"] == 0 and p["split_grid"] == 16
    ps = A.attn_plan(1, 1, 2000, 2000, 64, 0, 148)
    # 8 units of 16 key tiles: 16 serial steps per CTA against 1 step and 16-piece merges
    assert (ps["split"], ps["split_grid"], ps["split_units"]) == (1, 128, 8)
    assert ps["workspace_bytes"] == 128 * 2 * 2 * 128 * 65 * 4 + 8 * 4 + 16
    assert A.attn_plan(1, 4, 1000, 1000, 64, 0, 148)["split"] == 0  # 7 steps saved, 8 pieces
    pd = A.attn_plan(2, 2, 512, 8192, 128, 0, 148)  # d = 128: 64 steps against 4 + 19 pieces
    assert (pd["split"], pd["split_grid"]) == (1, 148)
    assert p["grid"] == 4 and p["block"] == 384
    assert p["qk_tile_products"] == 2 * 4 * 4
    p = A.attn_plan(16, 4, 1600, 1600, 64, 0, 148)
    # 13 query tiles per head: 6 full pairs per head, and the 64 lone last tiles
    # paired across heads in 32 dual units -> 416 units, at most 3 per SM: unit mode
    assert (p["num_q_tiles"], p["num_q_pairs"], p["units_per_head"], p["dual_units"],
            p["num_units"], p["grid"]) == (13, 7, 6, 32, 416, 148)
    assert p["split"] == 0 and p["workspace_bytes"] == 0
    assert p["split_units"] == 64 * 7  # what split mode would share out (plain units)
    p3 = A.attn_plan(16, 4, 6400, 6400, 64, 0, 148)  # 1600 units: 98 % even already
    assert p3["split"] == 0 and p3["workspace_bytes"] == 0 and p3["dual_units"] == 0
    p4 = A.attn_plan(1, 3, 300, 300, 64, 0, 148)
    assert (p4["units_per_head"], p4["dual_units"], p4["num_units"]) == (1, 2, 5)
    assert (p4["split"], p4["split_units"], p4["split_grid"]) == (0, 6, 18)
    # dual units in unit mode, but split mode (over the plain units) when it pays
    p5 = A.attn_plan(1, 2, 300, 4000, 64, 0, 148)
    assert (p5["dual_units"], p5["num_units"], p5["split_units"]) == (1, 3, 4)
    assert (p5["split"], p5["split_grid"]) == (1, 128)
    assert p5["workspace_bytes"] == 128 * 2 * 2 * 128 * 65 * 4 + 4 * 4 + 16
    # no dual units for causal problems or a single head
    assert A.attn_plan(4, 4, 300, 300, 64, 1, 148)["dual_units"] == 0
    assert A.attn_plan(1, 1, 300, 300, 64, 0, 148)["dual_units"] == 0
    assert p["smem_bytes"] <= 232448
    p = A.attn_plan(32, 16, 2048, 2048, 64, 1, 148)
    assert p["split"] == 0  # causal work is balanced by the mirror pairing instead
    # causal: a unit is a heavy query pair with its mirror (8 pairs -> 4 units per head)
    assert (p["num_q_pairs"], p["units_per_head"], p["num_units"]) == (8, 4, 32 * 16 * 4)
    # causal: query tile i visits key tiles 0..i
    assert p["qk_tile_products"] == 32 * 16 * sum(range(1, 17))
    p = A.attn_plan(1, 32, 32768, 32768, 128, 1, 148)
    assert p["stages"] == 5 and p["smem_bytes"] <= 232448  # 3 K + 2 V slots at d=128
    assert (p["num_q_pairs"], p["units_per_head"]) == (128, 64)
    p2 = A.attn_plan(1, 1, 3 * 256, 3 * 256, 64, 1, 148)  # odd pair count: middle pair alone
    assert (p2["num_q_pairs"], p2["units_per_head"], p2["num_units"]) == (3, 2, 2)
    assert p["qk_tile_products"] == 32 * sum(range(1, 257))
    # ragged causal with Nq != Nk (top-left): rows past Nk see every key
    p = A.attn_plan(1, 1, 300, 200, 64, 1, 148)
    assert p["qk_tile_products"] == 1 + 2 + 2


@pytest.mark.parametrize("kw,code", [
    (dict(d=48), 3), (dict(B=0), 2), (dict(num_sms=0), 2)])
def test_plan_errors(kw, code):
    a = dict(B=1, H=1, Nq=10, Nk=10, d=64, causal=0, num_sms=148)
    a.update(kw)
    with pytest.raises(A.AttnError) as e:
        A.attn_plan(*a.values())
    assert e.value.status == code


# ------------------------------------------------------------------ backward arguments

BWD = dict(q=0x10000, k=0x20000, v=0x30000, o=0x40000, lse=0x50000, do=0x60000, dq=0x70000,
           dk=0x80000, dv=0x90000, B=1, H=2, Nq=400, Nk=300, d=64, scale=0.125, causal=0,
           dtype=A.ATTN_FP16, ws=0xA0000, ws_bytes=1 << 30)


def call_bwd(**kw):
    a = dict(BWD)
    a.update(kw)
    return A.attn_bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["do"], a["dq"], a["dk"],
                      a["dv"], a["B"], a["H"], a["Nq"], a["Nk"], a["d"], a["scale"], a["causal"],
                      a["dtype"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(lse=None), 1), (dict(do=None), 1), (dict(dq=None), 1),
    (dict(dk=None), 1), (dict(dv=None), 1),
    (dict(dtype=3), 4), (dict(d=96), 3), (dict(Nq=0), 2), (dict(Nk=0), 2),
    (dict(do=0x60002), 5), (dict(dq=0x70008), 5), (dict(dk=0x80004), 5), (dict(dv=0x90001), 5),
    (dict(scale=0.0), 6),
    (dict(ws=None), 11), (dict(ws=0xA0004), 11), (dict(ws_bytes=1000), 11),
])
def test_bwd_argument_errors(kw, code):
    assert call_bwd(**kw) == code


def test_bwd_workspace_size():
    # fp32 dQ accumulator plus two padded per-row vectors
    n = A.attn_bwd_workspace_size(2, 3, 200, 77, 64)
    assert n == 2 * 3 * 200 * 64 * 4 + 2 * 2 * 3 * 256 * 4
    assert A.attn_bwd_workspace_size(1, 1, 128, 1, 128) == 128 * 128 * 4 + 2 * 128 * 4
    with pytest.raises(A.AttnError):
        A.attn_bwd_workspace_size(1, 1, 128, 1, 80)


# ------------------------------------------------------------------ e4m3 forward arguments

FP8 = dict(q=0x10000, k=0x20000, vt=0x30000, o=0x40000, lse=None, B=1, H=2, Nq=300, Nk=512,
           d=128, scale=0.088, qs=0.01, ks=0.02, vs=0.03, causal=0, ws=None, ws_bytes=0)


def call_fp8(**kw):
    a = dict(FP8)
    a.update(kw)
    return A.attn_fwd_fp8(a["q"], a["k"], a["vt"], a["o"], a["lse"], a["B"], a["H"], a["Nq"],
                          a["Nk"], a["d"], a["scale"], a["qs"], a["ks"], a["vs"], a["causal"],
                          a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(vt=None), 1), (dict(o=None), 1),
    (dict(d=64), 3), (dict(d=256), 3),
    (dict(Nq=0), 2), (dict(Nk=0), 2), (dict(Nk=500), 2), (dict(B=0), 2),
    (dict(qs=0.0), 6), (dict(ks=-1.0), 6), (dict(vs=float("nan")), 6), (dict(qs=float("inf")), 6),
    (dict(scale=0.0), 6), (dict(scale=1e-20, qs=1e-10, ks=1e-10), 6),
    (dict(q=0x10008), 5), (dict(vt=0x30004), 5), (dict(o=0x40002), 5), (dict(lse=0x50002), 5),
    (dict(), 8),  # valid arguments, no usable device here: ATTN_ERR_CUDA, never a CPU path
])
def test_fp8_argument_errors(kw, code):
    import torch
    if code == 8 and torch.cuda.is_available():
        pytest.skip("a device is present")
    assert call_fp8(**kw) == code


# ------------------------------------------------------------------ projection arguments

def test_proj_argument_errors():
    good = dict(x=0x10000, w=0x20000, b=None, q=0x30000, k=0x40000, v=0x50000)
    def qkv(**kw):
        a = dict(good, B=1, N=100, H=2, d=64, dtype=A.ATTN_FP16)
        a.update(kw)
        return A.attn_qkv_proj(a["x"], a["w"], a["b"], a["q"], a["k"], a["v"], a["B"], a["N"],
                               a["H"], a["d"], a["dtype"], None)
    assert qkv(x=None) == 1 and qkv(v=None) == 1
    assert qkv(dtype=5) == 4 and qkv(d=32) == 3 and qkv(N=0) == 2 and qkv(H=0) == 2
    assert qkv(x=0x10008) == 5 and qkv(b=0x60002) == 5
    def outp(**kw):
        a = dict(o=0x10000, w=0x20000, b=None, y=0x30000, B=1, N=100, H=2, d=64, C_out=128,
                 dtype=A.ATTN_BF16)
        a.update(kw)
        return A.attn_out_proj(a["o"], a["w"], a["b"], a["y"], a["B"], a["N"], a["H"], a["d"],
                               a["C_out"], a["dtype"], None)
    assert outp(y=None) == 1 and outp(C_out=100) == 2 and outp(C_out=0) == 2
    assert outp(o=0x10004) == 5 and outp(d=100) == 3
    assert A.attn_block_fwd(0x10000, 0x20000, None, 0x30000, None, 0x40000, 0x50000, 0x60000,
                            0x70000, None, 0x80000, 1, 64, 2, 64, 128, 0.0, 0, 0, None) == 6
