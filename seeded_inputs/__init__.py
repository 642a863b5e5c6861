"""Seeded synthetic workloads for the attention forward.

This module is shared by the CPU oracle's tests and by the CUDA path's
tests and benchmark.  It holds only the workload shapes and the random
input recipe: none of the attention arithmetic lives here.

Workload shapes follow the pages:

* YOLO11 x FlashAttention-2 (kwkr.cn/news/620085), section 1.1: C2PSA
  feature maps of 20x20 / 40x40 / 80x80 flatten to sequence lengths
  400 / 1600 / 6400; section 3.1: batch 16 at 640x640.
* "FlashAttention 深度解读" (coreui.cn), section "怎么用": q/k/v of shape
  [32, 2048, 1024] in fp16 with causal=True, read as B=32, H=16, d=64.
* "一个反直觉的事实：大模型推理的瓶颈不是计算，而是显存" (ai2ai.xin),
  section "Self-Attention的计算瓶颈": long contexts, here capped at 32768.

Input recipe (the pages give distributions but no seeds):

* one CPU ``torch.Generator`` per workload, seeded ``1000 + index`` with
  index 1..5 for the five workloads below;
* draw Q, then K, then V, each standard normal float32 in [B, H, N, d];
* optionally multiply Q and K by ``qk_scale`` in float32 before the cast
  (0.5 for the long-context workload);
* cast to fp16 / bf16 with round-to-nearest-even.  The oracle sees the
  cast values, upcast exactly.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

__all__ = ["Workload", "WORKLOADS", "workload", "make_qkv", "dtype_of", "make_grad_out",
           "make_workload_qkv", "make_block_inputs", "make_fp8_qkv"]

_DTYPES = {"fp16": torch.float16, "bf16": torch.bfloat16}


def dtype_of(name: str) -> torch.dtype:
    """Map 'fp16' / 'bf16' to the torch dtype."""
    return _DTYPES[name]


@dataclass(frozen=True)
class Workload:
    """One attention-forward workload: shapes, dtype, mask and input seed."""

    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    dtype: str
    causal: bool
    seed: int
    qk_scale: float = 1.0
    note: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        """Softmax scale 1/sqrt(d), the default of the pages' SDPA call."""
        return 1.0 / float(self.d) ** 0.5

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs of the two contractions, halved when causal."""
        f = 4.0 * self.B * self.H * self.Nq * self.Nk * self.d
        return f / 2.0 if self.causal else f

    @property
    def bytes(self) -> float:
        """Algorithmic HBM bytes: read Q, K, V once and write O once."""
        return 2.0 * self.B * self.H * (2 * self.Nq + 2 * self.Nk) * self.d

    @property
    def lse_bytes(self) -> float:
        return 4.0 * self.B * self.H * self.Nq

    def as_config(self) -> dict:
        return {
            "workload": self.name, "B": self.B, "H": self.H, "Nq": self.Nq,
            "Nk": self.Nk, "d": self.d, "dtype": self.dtype,
            "causal": self.causal, "seed": self.seed, "qk_scale": self.qk_scale,
        }


WORKLOADS = [
    Workload("yolo_c2psa_20x20", 1, 2, 400, 400, 64, "fp16", False, 1001,
             note="C2PSA attention on a 20x20 feature map"),
    Workload("yolo_neck_40x40_b16", 16, 4, 1600, 1600, 64, "fp16", False, 1002,
             note="neck attention at 40x40, batch 16"),
    Workload("yolo_highres_80x80_b16", 16, 4, 6400, 6400, 64, "bf16", False, 1003,
             note="high-resolution attention at 80x80, batch 16"),
    Workload("llm_causal_2048", 32, 16, 2048, 2048, 64, "fp16", True, 1004,
             note="hidden 1024 split into 16 heads, causal"),
    Workload("long_context_32k", 1, 32, 32768, 32768, 128, "bf16", True, 1005,
             qk_scale=0.5, note="long-context causal, Q and K scaled by 0.5"),
]


def workload(name_or_index) -> Workload:
    """Look a workload up by name or by 0-based index."""
    if isinstance(name_or_index, int):
        return WORKLOADS[name_or_index]
    for w in WORKLOADS:
        if w.name == name_or_index:
            return w
    raise KeyError(name_or_index)


def make_qkv(B: int, H: int, Nq: int, Nk: int, d: int, dtype: str, seed: int,
             qk_scale: float = 1.0):
    """Draw Q, K, V on the CPU from one seeded generator.

    Returns contiguous CPU tensors of ``dtype_of(dtype)`` with shapes
    [B,H,Nq,d], [B,H,Nk,d], [B,H,Nk,d].
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn((B, H, Nq, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, H, Nk, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, H, Nk, d), generator=g, dtype=torch.float32)
    if qk_scale != 1.0:
        q.mul_(qk_scale)
        k.mul_(qk_scale)
    t = dtype_of(dtype)
    return q.to(t).contiguous(), k.to(t).contiguous(), v.to(t).contiguous()


def make_grad_out(B: int, H: int, Nq: int, dv: int, dtype: str, seed: int):
    """A seeded output gradient dO [B, H, Nq, dv], N(0,1) drawn on the CPU."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 7919)
    return torch.randn((B, H, Nq, dv), generator=g, dtype=torch.float32).to(dtype_of(dtype)).contiguous()


def make_workload_qkv(w: Workload):
    """Inputs of a named workload."""
    return make_qkv(w.B, w.H, w.Nq, w.Nk, w.d, w.dtype, w.seed, w.qk_scale)


def make_block_inputs(B: int, N: int, H: int, d: int, C_out: int, dtype: str, seed: int,
                      qkv_bias: bool = False):
    """Seeded input and weights of an attention block: x [B, N, C] N(0,1), W_qkv [3C, C] and
    W_o [C_out, C] N(0, 1/C) (the scale of a default-initialised Linear), b_o [C_out] fp32
    N(0, 0.1^2), and b_qkv [3C] fp32 likewise when ``qkv_bias`` (the page's qkv Linear has
    none).  Returns (x, w_qkv, b_qkv or None, w_o, b_o)."""
    C = H * d
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 104729)
    t = dtype_of(dtype)
    x = torch.randn((B, N, C), generator=g, dtype=torch.float32).to(t).contiguous()
    w_qkv = (torch.randn((3 * C, C), generator=g, dtype=torch.float32) / C ** 0.5).to(t).contiguous()
    w_o = (torch.randn((C_out, C), generator=g, dtype=torch.float32) / C ** 0.5).to(t).contiguous()
    b_o = 0.1 * torch.randn((C_out,), generator=g, dtype=torch.float32)
    b_qkv = 0.1 * torch.randn((3 * C,), generator=g, dtype=torch.float32) if qkv_bias else None
    return x, w_qkv, b_qkv, w_o, b_o


def make_fp8_qkv(B: int, H: int, Nq: int, Nk: int, d: int, seed: int, qk_scale: float = 1.0):
    """Seeded e4m3 inputs with one scale factor per tensor.

    Q, K, V are drawn as in ``make_qkv`` (float32, Q and K times
    ``qk_scale``); each tensor x is stored as the e4m3 codes of
    x * (448 / max|x|) (torch's round-to-nearest-even cast, so the largest
    magnitude lands on 448, the format's largest finite value) with descale
    max|x| / 448, which turns codes back into values.  V is stored
    transposed, [B, H, d, Nk].  Returns CPU tensors
    (q8 [B,H,Nq,d], k8 [B,H,Nk,d], vt8 [B,H,d,Nk]) of torch.float8_e4m3fn
    and the descales (q_descale, k_descale, v_descale) as Python floats.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn((B, H, Nq, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, H, Nk, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, H, Nk, d), generator=g, dtype=torch.float32)
    if qk_scale != 1.0:
        q.mul_(qk_scale)
        k.mul_(qk_scale)

    def quantize(x):
        amax = float(x.abs().max())
        amax = amax if amax > 0 else 1.0
        return (x * (448.0 / amax)).to(torch.float8_e4m3fn).contiguous(), amax / 448.0

    q8, qs = quantize(q)
    k8, ks = quantize(k)
    vt8, vs = quantize(v.transpose(-1, -2).contiguous())
    return q8, k8, vt8, (qs, ks, vs)
