"""KDA oracle (test infrastructure only).

This package is the correctness oracle for the CUDA path.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it.  It shares no code with ``gated_delta_rule_124_b200`` and imports nothing
from it; the library never imports this package.

Contents
--------
* ``kda_oracle.c`` -- the fp64 token-by-token recurrence (the definition), built
  into ``libkda_oracle.so`` by :func:`build` with gcc + OpenMP.
* :func:`forward` / :func:`decode_step` -- ctypes wrappers around it.
* :mod:`oracle.chunkwise` -- an fp64 numpy restatement of the chunkwise WY/UT
  form, used to check the GPU path's per-chunk intermediates.  It is itself
  checked against :func:`forward` by the CPU tests.

The recurrence (Kimi Linear, aiwiki.ai, sections "Kimi Delta Attention" and
"The constrained DPLR form and the chunkwise algorithm"): per (sequence, head),
``S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T`` and
``o_t = S_t^T q_t`` with ``alpha_t = exp(g_t)`` per channel.

Pins (all in ``tests/test_oracle.py``, run with ``-m "not gpu"``): explicit
products of the dense dk x dk transition matrices; the DeltaNet (alpha = 1),
Gated DeltaNet (head-uniform alpha) and pure-decay (beta = 0) special cases;
exact overwrite retrieval with orthonormal keys; a hand-worked example in
``tests/golden/``; varlen / split / decode composition.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` into ``libkda_oracle.so`` (gcc, -O2, OpenMP).

    No fast-math: the oracle keeps IEEE fp64 semantics.
    """
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int32)
            lib.kda_ref_forward.argtypes = [dp, dp, dp, dp, dp, dp, ip, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, dp, dp, ctypes.c_int]
            lib.kda_ref_forward.restype = ctypes.c_int
            lib.kda_ref_decode_step.argtypes = [dp, dp, dp, dp, dp, dp, dp, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int]
            lib.kda_ref_decode_step.restype = ctypes.c_int
            lib.kda_ref_max_threads.argtypes = []
            lib.kda_ref_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Widen to a C-contiguous float64 array (exact for bf16 / fp32 inputs)."""
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu")
        import torch  # local: only when handed torch tensors
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    return int(_load().kda_ref_max_threads())


def forward(q, k, v, g, beta, initial_state=None, cu_seqlens=None, num_threads: int = 0):
    """fp64 token recurrence over packed sequences.

    Shapes: q, k, g ``[T, H, dk]``; v ``[T, H, dv]``; beta ``[T, H]``;
    initial_state ``[N, H, dk, dv]`` or None (zeros); cu_seqlens ``[N + 1]`` or
    None (one sequence of length T).  A leading batch dimension ``[B, T, ...]``
    is accepted for q/k/v/g/beta and means B equal-length sequences.

    Returns ``(o [T, H, dv] (or [B, T, H, dv]), final_state [N, H, dk, dv])``
    as float64 numpy arrays.
    """
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    batched = q.ndim == 4
    if batched:
        B, T = q.shape[:2]
        if cu_seqlens is not None:
            raise ValueError("cu_seqlens with batched [B, T, ...] inputs")
        cu = np.arange(0, (B + 1) * T, T, dtype=np.int32)
        q, k, g = (x.reshape(B * T, *x.shape[2:]) for x in (q, k, g))
        v = v.reshape(B * T, *v.shape[2:])
        beta = beta.reshape(B * T, -1)
    else:
        cu = (np.array([0, q.shape[0]], dtype=np.int32) if cu_seqlens is None
              else np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32)))
    total, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or g.shape != q.shape or v.shape != (total, H, dv) \
            or beta.shape != (total, H):
        raise ValueError("shape mismatch")
    N = cu.shape[0] - 1
    h0 = None if initial_state is None else _f64(initial_state)
    if h0 is not None and h0.shape != (N, H, dk, dv):
        raise ValueError(f"initial_state must be {(N, H, dk, dv)}, got {h0.shape}")
    o = np.zeros((total, H, dv), dtype=np.float64)
    hN = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load().kda_ref_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                 cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), N, total,
                                 H, dk, dv, _ptr(o), _ptr(hN), int(num_threads))
    if rc != 0:
        raise ValueError(f"kda_ref_forward failed with code {rc}")
    if batched:
        o = o.reshape(B, T, H, dv)
    return o, hN


def decode_step(q, k, v, g, beta, state, num_threads: int = 0):
    """One fp64 recurrent step per (sequence, head).

    q, k, g ``[N, H, dk]``; v ``[N, H, dv]``; beta ``[N, H]``; state
    ``[N, H, dk, dv]``.  Returns ``(o [N, H, dv], new_state)``; the input state
    is not modified.
    """
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    st = _f64(state).copy()
    N, H, dk = q.shape
    dv = v.shape[-1]
    if st.shape != (N, H, dk, dv):
        raise ValueError("state shape mismatch")
    o = np.zeros((N, H, dv), dtype=np.float64)
    rc = _load().kda_ref_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(st),
                                     _ptr(o), N, H, dk, dv, int(num_threads))
    if rc != 0:
        raise ValueError(f"kda_ref_decode_step failed with code {rc}")
    return o, st
