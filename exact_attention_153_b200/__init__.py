"""Python binding of the sm_100a exact attention forward (libattn_sm100.so).

Argument marshalling only: every step of the computation runs in the CUDA
library.  PyTorch supplies device memory and streams.  If the library is not
built the import still works, but every call raises -- there is no CPU or
PyTorch fallback.

    from exact_attention_153_b200 import forward
    o, lse = forward(q, k, v, causal=True)          # q, k, v: [B, H, N, d] cuda fp16/bf16

The C entry points are mirrored one to one (``attn_fwd``, ``attn_fwd_host``,
``attn_plan``, ``attn_get_device_status``, ``attn_strerror``,
``attn_version``) for callers that manage raw pointers.
"""
from __future__ import annotations

import ctypes
import math
import os

__all__ = [
    "ATTN_FP16", "ATTN_BF16", "AttnError", "lib", "library_path", "attn_fwd", "attn_fwd_host",
    "attn_plan", "attn_get_device_status", "attn_strerror", "attn_version", "forward",
    "forward_host", "STATUS_NAMES", "attn_fwd_ws", "attn_workspace_size", "workspace_for",
    "attn_fwd_noalloc", "attn_bwd", "attn_bwd_workspace_size", "backward",
    "attn_qkv_proj", "attn_out_proj", "attn_block_fwd", "qkv_proj", "out_proj", "block_forward",
    "attn_fwd_fp8", "forward_fp8",
]

ATTN_FP16 = 0
ATTN_BF16 = 1
STATUS_NAMES = {
    0: "ATTN_OK", 1: "ATTN_ERR_NULL", 2: "ATTN_ERR_SHAPE", 3: "ATTN_ERR_HEAD_DIM",
    4: "ATTN_ERR_DTYPE", 5: "ATTN_ERR_ALIGN", 6: "ATTN_ERR_SCALE", 7: "ATTN_ERR_ARCH",
    8: "ATTN_ERR_CUDA", 9: "ATTN_ERR_DEVICE_TIMEOUT", 10: "ATTN_ERR_SCRATCH_LIMIT",
    11: "ATTN_ERR_WORKSPACE",
}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libattn_sm100.so"
_lib = None


def library_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


class AttnError(RuntimeError):
    """A non-zero status from the C library."""

    def __init__(self, status: int, where: str = "attn_fwd"):
        self.status = int(status)
        name = STATUS_NAMES.get(self.status, str(status))
        super().__init__(f"{where} failed: {name}: {attn_strerror(self.status)}")


class _Plan(ctypes.Structure):
    _fields_ = [("num_q_tiles", ctypes.c_int), ("num_q_pairs", ctypes.c_int),
                ("num_kv_tiles", ctypes.c_int), ("units_per_head", ctypes.c_int),
                ("num_units", ctypes.c_int), ("dual_units", ctypes.c_int),
                ("grid", ctypes.c_int), ("block", ctypes.c_int), ("smem_bytes", ctypes.c_int),
                ("stages", ctypes.c_int), ("qk_tile_products", ctypes.c_longlong),
                ("split", ctypes.c_int), ("split_grid", ctypes.c_int),
                ("split_units", ctypes.c_int), ("workspace_bytes", ctypes.c_longlong),
                ("split_steps", ctypes.c_longlong)]


def lib() -> ctypes.CDLL:
    """Load the in-tree library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m exact_attention_153_b200.build_lib` "
                "(there is no fallback implementation)")
        L = ctypes.CDLL(path)
        vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
        L.attn_fwd.restype = i
        L.attn_fwd_ws.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, ctypes.c_size_t,
                                  vp]
        L.attn_fwd_ws.restype = i
        L.attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, f, f, f, i, vp,
                                   ctypes.c_size_t, vp]
        L.attn_fwd_fp8.restype = i
        L.attn_workspace_size.argtypes = [i, i, i, i, i, i, ctypes.POINTER(ctypes.c_size_t)]
        L.attn_workspace_size.restype = i
        L.attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
        L.attn_fwd_noalloc.restype = i
        L.attn_fwd_stall_test.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp,
                                          ctypes.c_size_t, i, vp]
        L.attn_fwd_stall_test.restype = i
        L.attn_fwd_host.argtypes = [vp] * 11 + [ctypes.c_size_t, i, i, i, i, i, f, i, i, vp]
        L.attn_fwd_host.restype = i
        L.attn_bwd.argtypes = [vp] * 9 + [i, i, i, i, i, f, i, i, vp, ctypes.c_size_t, vp]
        L.attn_bwd.restype = i
        L.attn_bwd_workspace_size.argtypes = [i, i, i, i, i, ctypes.POINTER(ctypes.c_size_t)]
        L.attn_bwd_workspace_size.restype = i
        L.attn_qkv_proj.argtypes = [vp] * 6 + [i, i, i, i, i, vp]
        L.attn_qkv_proj.restype = i
        L.attn_out_proj.argtypes = [vp] * 4 + [i, i, i, i, i, i, vp]
        L.attn_out_proj.restype = i
        L.attn_block_fwd.argtypes = [vp] * 11 + [i, i, i, i, i, f, i, i, vp]
        L.attn_block_fwd.restype = i
        L.attn_plan.argtypes = [i, i, i, i, i, i, i, ctypes.POINTER(_Plan)]
        L.attn_plan.restype = i
        L.attn_get_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint)]
        L.attn_get_device_status.restype = i
        L.attn_strerror.argtypes = [i]
        L.attn_strerror.restype = ctypes.c_char_p
        L.attn_version.argtypes = []
        L.attn_version.restype = i
        _lib = L
    return _lib


# ----------------------------------------------------------------- raw entry points

def attn_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, dtype, stream) -> int:
    """Raw ``attn_fwd``: pointers and the stream handle as Python ints."""
    return lib().attn_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, float(scale), int(causal), dtype, stream)


def attn_fwd_ws(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, dtype, workspace, ws_bytes,
                stream) -> int:
    """Raw ``attn_fwd_ws``: attn_fwd with a device workspace (split mode)."""
    return lib().attn_fwd_ws(q, k, v, o, lse, B, H, Nq, Nk, d, float(scale), int(causal), dtype,
                             workspace, ws_bytes, stream)


def attn_fwd_fp8(q, k, vt, o, lse, B, H, Nq, Nk, d, scale, q_descale, k_descale, v_descale,
                 causal, workspace, ws_bytes, stream) -> int:
    """Raw ``attn_fwd_fp8``: e4m3 q, k and transposed v with per-tensor descales, bf16 o."""
    return lib().attn_fwd_fp8(q, k, vt, o, lse, B, H, Nq, Nk, d, float(scale), float(q_descale),
                              float(k_descale), float(v_descale), int(causal), workspace,
                              ws_bytes, stream)


def attn_fwd_noalloc(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, dtype, stream) -> int:
    """Raw ``attn_fwd_noalloc``: split mode with the library's fixed scratch, no allocation.

    For callers that cannot allocate device memory themselves (see include/attn.h).
    """
    return lib().attn_fwd_noalloc(q, k, v, o, lse, B, H, Nq, Nk, d, float(scale), int(causal),
                                  dtype, stream)


def attn_fwd_stall_test(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, dtype, workspace,
                        ws_bytes, stall_site, stream) -> int:
    """Raw ``attn_fwd_stall_test``: the failure-path test hook (see include/attn.h)."""
    return lib().attn_fwd_stall_test(q, k, v, o, lse, B, H, Nq, Nk, d, float(scale),
                                     int(causal), dtype, workspace, ws_bytes, stall_site, stream)


def attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, Nq, Nk, d, scale, causal, dtype, workspace,
             ws_bytes, stream) -> int:
    """Raw ``attn_bwd``: pointers and the stream handle as Python ints."""
    return lib().attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, Nq, Nk, d, float(scale),
                          int(causal), dtype, workspace, ws_bytes, stream)


def attn_bwd_workspace_size(B, H, Nq, Nk, d) -> int:
    """Workspace bytes ``attn_bwd`` needs for these sizes."""
    n = ctypes.c_size_t(0)
    st = lib().attn_bwd_workspace_size(B, H, Nq, Nk, d, ctypes.byref(n))
    if st != 0:
        raise AttnError(st, "attn_bwd_workspace_size")
    return n.value


def attn_qkv_proj(x, w_qkv, b_qkv, q, k, v, B, N, H, d, dtype, stream) -> int:
    """Raw ``attn_qkv_proj``: pointers and the stream handle as Python ints."""
    return lib().attn_qkv_proj(x, w_qkv, b_qkv, q, k, v, B, N, H, d, dtype, stream)


def attn_out_proj(o, w_o, b_o, y, B, N, H, d, C_out, dtype, stream) -> int:
    """Raw ``attn_out_proj``."""
    return lib().attn_out_proj(o, w_o, b_o, y, B, N, H, d, C_out, dtype, stream)


def attn_block_fwd(x, w_qkv, b_qkv, w_o, b_o, q, k, v, o, lse, y, B, N, H, d, C_out, scale,
                   causal, dtype, stream) -> int:
    """Raw ``attn_block_fwd``."""
    return lib().attn_block_fwd(x, w_qkv, b_qkv, w_o, b_o, q, k, v, o, lse, y, B, N, H, d, C_out,
                                float(scale), int(causal), dtype, stream)


def attn_workspace_size(B, H, Nq, Nk, d, causal) -> int:
    """Workspace bytes attn_fwd_ws uses for these sizes on the current device."""
    n = ctypes.c_size_t(0)
    st = lib().attn_workspace_size(B, H, Nq, Nk, d, int(causal), ctypes.byref(n))
    if st != 0:
        raise AttnError(st, "attn_workspace_size")
    return n.value


def attn_fwd_host(q_h, k_h, v_h, o_h, lse_h, q_d, k_d, v_d, o_d, lse_d, workspace, ws_bytes, B,
                  H, Nq, Nk, d, scale, causal, dtype, stream) -> int:
    """Raw ``attn_fwd_host``: host and device pointers as Python ints."""
    return lib().attn_fwd_host(q_h, k_h, v_h, o_h, lse_h, q_d, k_d, v_d, o_d, lse_d, workspace,
                               ws_bytes, B, H, Nq, Nk, d, float(scale), int(causal), dtype,
                               stream)


def attn_plan(B, H, Nq, Nk, d, causal, num_sms) -> dict:
    """Launch geometry for these sizes on a GPU with ``num_sms`` SMs."""
    p = _Plan()
    st = lib().attn_plan(B, H, Nq, Nk, d, int(causal), num_sms, ctypes.byref(p))
    if st != 0:
        raise AttnError(st, "attn_plan")
    return {name: getattr(p, name) for name, _ in _Plan._fields_}


def attn_get_device_status(stream=None):
    """(status, raw word) after synchronising ``stream``."""
    word = ctypes.c_uint(0)
    st = lib().attn_get_device_status(_stream_handle(stream), ctypes.byref(word))
    return st, word.value


def attn_strerror(status: int) -> str:
    return lib().attn_strerror(int(status)).decode()


def attn_version() -> int:
    return lib().attn_version()


# ----------------------------------------------------------------- torch helpers

def _stream_handle(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float16:
        return ATTN_FP16
    if t.dtype == torch.bfloat16:
        return ATTN_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: fp16 or bf16 only")


def forward(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
            return_lse: bool = True, stream=None, workspace=None):
    """Attention forward on CUDA tensors [B, H, N, d]; returns (o, lse).

    ``scale`` defaults to 1/sqrt(d), the default of the pages' SDPA call
    (YOLO11 x FlashAttention-2, kwkr.cn, section 2.2).  Inputs must be
    contiguous (the page's transposed views need ``.contiguous()``).
    """
    import torch
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if k.shape != (B, H, Nk, d) or v.shape != (B, H, Nk, d):
        raise ValueError(f"shape mismatch: q {tuple(q.shape)} k {tuple(k.shape)} v {tuple(v.shape)}")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors (no CPU path exists)")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    code = _dtype_code(q)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, Nq, d), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    if workspace is None:
        st = attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                      lse.data_ptr() if lse is not None else None, B, H, Nq, Nk, d, scale, causal,
                      code, _stream_handle(stream))
    else:
        st = attn_fwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                         lse.data_ptr() if lse is not None else None, B, H, Nq, Nk, d, scale,
                         causal, code, workspace.data_ptr(),
                         workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if st != 0:
        raise AttnError(st)
    return out, lse


def forward_fp8(q8, k8, vt8, descales, causal: bool = False, scale: float | None = None,
                out=None, lse=None, return_lse: bool = True, stream=None, workspace=None):
    """FP8 attention forward: e4m3 q8 [B, H, Nq, 128], k8 [B, H, Nk, 128] and V transposed,
    vt8 [B, H, 128, Nk] (Nk a multiple of 16), with ``descales`` = (q, k, v) factors that turn
    codes into values.  Returns (o bf16 [B, H, Nq, 128], lse fp32 [B, H, Nq]).

    The FP8 path of FlashAttention-3 ("一个反直觉的事实", ai2ai.xin, section
    "FlashAttention-3的进一步增强", item 2).
    """
    import torch
    if q8.dim() != 4 or k8.dim() != 4 or vt8.dim() != 4:
        raise ValueError("q8, k8 must be [B, H, N, d] and vt8 [B, H, d, Nk]")
    B, H, Nq, d = q8.shape
    Nk = k8.shape[2]
    if k8.shape != (B, H, Nk, d) or vt8.shape != (B, H, d, Nk):
        raise ValueError(f"shape mismatch: q8 {tuple(q8.shape)} k8 {tuple(k8.shape)} "
                         f"vt8 {tuple(vt8.shape)}")
    if not (q8.is_cuda and k8.is_cuda and vt8.is_cuda):
        raise ValueError("q8, k8, vt8 must be CUDA tensors (no CPU path exists)")
    for name, t in (("q8", q8), ("k8", k8), ("vt8", vt8)):
        if t.dtype != torch.float8_e4m3fn:
            raise TypeError(f"{name} must be torch.float8_e4m3fn")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=q8.device)
    if lse is None and return_lse:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q8.device)
    qs, ks, vs = descales
    st = attn_fwd_fp8(q8.data_ptr(), k8.data_ptr(), vt8.data_ptr(), out.data_ptr(),
                      lse.data_ptr() if lse is not None else None, B, H, Nq, Nk, d, scale,
                      qs, ks, vs, causal,
                      workspace.data_ptr() if workspace is not None else None,
                      workspace.numel() * workspace.element_size() if workspace is not None else 0,
                      _stream_handle(stream))
    if st != 0:
        raise AttnError(st, "attn_fwd_fp8")
    return out, lse


def workspace_for(q, k, causal: bool = False):
    """A zero-filled device workspace sized for attn_fwd_ws on these inputs (or None)."""
    import torch
    B, H, Nq, d = q.shape
    n = attn_workspace_size(B, H, Nq, k.shape[2], d, causal)
    if n == 0:
        return None
    return torch.zeros(n, dtype=torch.uint8, device=q.device)


def forward_host(q_h, k_h, v_h, o_h, lse_h, q_d, k_d, v_d, o_d, lse_d, causal=False, scale=None,
                 stream=None, workspace=None):
    """End-to-end call from (pinned) host tensors through caller-owned device buffers."""
    B, H, Nq, d = q_h.shape
    Nk = k_h.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    st = attn_fwd_host(q_h.data_ptr(), k_h.data_ptr(), v_h.data_ptr(), o_h.data_ptr(),
                       lse_h.data_ptr() if lse_h is not None else None,
                       q_d.data_ptr(), k_d.data_ptr(), v_d.data_ptr(), o_d.data_ptr(),
                       lse_d.data_ptr() if lse_d is not None else None,
                       workspace.data_ptr() if workspace is not None else None,
                       workspace.numel() * workspace.element_size() if workspace is not None else 0,
                       B, H, Nq, Nk, d, scale, causal, _dtype_code(q_h), _stream_handle(stream))
    if st != 0:
        raise AttnError(st, "attn_fwd_host")


def backward(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
             stream=None, workspace=None, out=None):
    """Gradients (dq, dk, dv) of the forward for the output gradient ``dout``.

    ``o`` and ``lse`` are the forward's outputs for these inputs.  A workspace
    of ``attn_bwd_workspace_size`` bytes is allocated when none is given.
    """
    import torch
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout), ("lse", lse)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if workspace is None:
        workspace = torch.empty(attn_bwd_workspace_size(B, H, Nq, Nk, d), dtype=torch.uint8,
                                device=q.device)
    dq, dk, dv = out if out is not None else (torch.empty_like(q), torch.empty_like(k),
                                              torch.empty_like(v))
    st = attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                  dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, Nq, Nk, d,
                  scale, causal, _dtype_code(q), workspace.data_ptr(),
                  workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if st != 0:
        raise AttnError(st, "attn_bwd")
    return dq, dk, dv


def _ptr(t):
    return t.data_ptr() if t is not None else None


def qkv_proj(x, w_qkv, b_qkv, H: int, stream=None, out=None):
    """q, k, v [B, H, N, d] = the head split of x W_qkv^T (+ b_qkv), x [B, N, C]."""
    import torch
    B, N, C = x.shape
    d = C // H
    if d * H != C:
        raise ValueError("C must be H * d")
    q, k, v = out if out is not None else tuple(
        torch.empty((B, H, N, d), dtype=x.dtype, device=x.device) for _ in range(3))
    st = attn_qkv_proj(x.data_ptr(), w_qkv.data_ptr(), _ptr(b_qkv), q.data_ptr(), k.data_ptr(),
                       v.data_ptr(), B, N, H, d, _dtype_code(x), _stream_handle(stream))
    if st != 0:
        raise AttnError(st, "attn_qkv_proj")
    return q, k, v


def out_proj(o, w_o, b_o, stream=None, out=None):
    """y [B, N, C_out] = o' W_o^T (+ b_o), o' the [B, N, H d] view of o [B, H, N, d]."""
    import torch
    B, H, N, d = o.shape
    C_out = w_o.shape[0]
    y = out if out is not None else torch.empty((B, N, C_out), dtype=o.dtype, device=o.device)
    st = attn_out_proj(o.data_ptr(), w_o.data_ptr(), _ptr(b_o), y.data_ptr(), B, N, H, d, C_out,
                       _dtype_code(o), _stream_handle(stream))
    if st != 0:
        raise AttnError(st, "attn_out_proj")
    return y


def block_forward(x, w_qkv, b_qkv, w_o, b_o, H: int, causal: bool = False, scale=None,
                  stream=None):
    """The attention block: returns (y, q, k, v, o, lse)."""
    import torch
    B, N, C = x.shape
    d = C // H
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    q, k, v, o = (torch.empty((B, H, N, d), dtype=x.dtype, device=x.device) for _ in range(4))
    lse = torch.empty((B, H, N), dtype=torch.float32, device=x.device)
    C_out = w_o.shape[0]
    y = torch.empty((B, N, C_out), dtype=x.dtype, device=x.device)
    st = attn_block_fwd(x.data_ptr(), w_qkv.data_ptr(), _ptr(b_qkv), w_o.data_ptr(), _ptr(b_o),
                        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                        y.data_ptr(), B, N, H, d, C_out, scale, causal, _dtype_code(x),
                        _stream_handle(stream))
    if st != 0:
        raise AttnError(st, "attn_block_fwd")
    return y, q, k, v, o, lse
