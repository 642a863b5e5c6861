"""Run the float64 oracle over many (batch, head) slices in parallel processes.

Test infrastructure for the full-size parity tests.  The pool is started with
the ``spawn`` method, so the workers are fresh interpreters that import only
numpy and ``oracle`` (never CUDA), which is safe after the parent process has
used the GPU.  Each task is one (batch, head): the worker computes that
slice's O and lse with ``oracle.attention_f64`` (the plain definition, S
materialised in row blocks) and returns the largest absolute differences
from the GPU's output, so only two numbers per slice travel back.
"""
from __future__ import annotations

import multiprocessing
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np

_THREAD_VARS = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS",
                "NUMEXPR_NUM_THREADS")


def _slice_errors(task):
    """Max |O_gpu - O_ref| and max |lse_gpu - lse_ref| for one (batch, head)."""
    import oracle
    bh, q, k, v, o_gpu, lse_gpu, scale, causal = task
    o_ref, lse_ref = oracle.attention_f64(q[None, None], k[None, None], v[None, None], scale,
                                          causal)
    eo = float(np.max(np.abs(o_gpu.astype(np.float64) - o_ref[0, 0])))
    el = float(np.max(np.abs(lse_gpu.astype(np.float64) - lse_ref[0, 0])))
    return bh, eo, el


def workers() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def compare_all_slices(q, k, v, o, lse, scale: float, causal: bool, n_workers: int | None = None):
    """Compare every element of O [B,H,Nq,d] and lse [B,H,Nq] (CPU torch tensors) with the oracle.

    q, k, v are the fp16 / bf16 inputs the GPU saw; they travel as float32,
    which holds every fp16 and bf16 value exactly.  Returns (max O error, max
    lse error, per-slice list of (index, O error, lse error)).
    """
    import torch
    B, H = q.shape[0], q.shape[1]

    def exact(t):  # float32 holds fp16 / bf16 / fp32 values exactly; float64 stays float64
        return t.numpy() if t.dtype == torch.float64 else t.float().numpy()

    def tasks():
        for b in range(B):
            for h in range(H):
                yield (b * H + h, exact(q[b, h]), exact(k[b, h]), exact(v[b, h]), exact(o[b, h]),
                       exact(lse[b, h]), float(scale), bool(causal))

    n = n_workers or workers()
    saved = {name: os.environ.get(name) for name in _THREAD_VARS}
    for name in _THREAD_VARS:  # one BLAS thread per worker; the pool supplies the parallelism
        os.environ[name] = "1"
    try:
        # a worker that dies raises BrokenProcessPool here instead of leaving the map waiting
        ctx = multiprocessing.get_context("spawn")
        with ProcessPoolExecutor(max_workers=min(n, B * H), mp_context=ctx) as pool:
            per_slice = sorted(pool.map(_slice_errors, tasks()))
    finally:
        for name, val in saved.items():
            if val is None:
                os.environ.pop(name, None)
            else:
                os.environ[name] = val
    worst_o = max(e for _, e, _ in per_slice)
    worst_l = max(e for _, _, e in per_slice)
    return worst_o, worst_l, per_slice
