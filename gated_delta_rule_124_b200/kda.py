"""Thin ctypes binding of libkda.so (see include/kda.h).

Argument marshalling only: every function here passes device pointers, sizes
and the current CUDA stream to the C ABI, and every step of the computation
runs in the library's CUDA kernels.  There is no CPU fallback: if libkda.so
cannot be loaded, every call raises :class:`KdaError`.

Functions with the C names take tensors that are already allocated (device
tensors from PyTorch) and return the status code, raising :class:`KdaError`
on anything but ``KDA_OK`` unless ``check=False``.  :func:`chunk_fwd` and
:func:`decode_step` are convenience wrappers that allocate outputs and the
workspace with PyTorch and then make the same calls.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkda.so")

KDA_OK = 0
KDA_ERR_INVALID_ARG = 1
KDA_ERR_UNSUPPORTED = 2
KDA_ERR_CUDA = 3
KDA_ERR_TIMEOUT = 4
KDA_ERR_WORKSPACE = 5
KDA_ERR_BAD_SEQLENS = 6

KDA_DTYPE_F32 = 0
KDA_DTYPE_BF16 = 1

# Every symbol include/kda.h declares.
EXPORTS = (
    "kda_status_string", "kda_chunk_fwd_workspace_size", "kda_chunk_fwd",
    "kda_num_chunks_upper_bound", "kda_chunk_gate_cumsum", "kda_chunk_intra",
    "kda_chunk_inter", "kda_chunk_output", "kda_decode_step", "kda_get_device_status",
    "kda_chunk_fwd_noalloc", "kda_chunk_split_workspace_size", "kda_chunk_split_intra",
    "kda_chunk_split_chain", "kda_chunk_fwd_plan", "kda_qkv_conv_norm",
    "kda_output_norm_gate", "kda_gdn_chunk_fwd_workspace_size", "kda_gdn_chunk_fwd",
    "kda_gdn_decode_step", "kda_chunk_bwd_workspace_size", "kda_chunk_bwd",
    "kda_gdn_chunk_bwd_workspace_size", "kda_gdn_chunk_bwd", "kda_qkv_conv_norm_step",
    "kda_chunk_fwd_with_plan", "kda_chunk_fwd_plan_workspace_size",
    "kda_test_overlap_flag_timeout", "kda_layer_decode_step", "kda_layer_chunk_fwd",
    "kda_layer_chunk_fwd_workspace_size", "kda_chunk_state_maps", "kda_fold_segment_states",
)


class KdaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        super().__init__(f"{what}: {status_string(status)}" if what else status_string(status))


_lib = None
_lock = threading.Lock()

_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_SIGS = {
    "kda_status_string": ([_i], ctypes.c_char_p),
    "kda_chunk_fwd_workspace_size": ([_i, _i, _i, _i, _i, _i, _i], _sz),
    "kda_num_chunks_upper_bound": ([_i, _i, _i], _i),
    "kda_chunk_fwd": ([_vp] * 7 + [_i] * 8 + [_vp, _vp, _vp, _sz, _vp], _i),
    "kda_chunk_gate_cumsum": ([_vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _sz, _vp], _i),
    "kda_chunk_intra": ([_vp] * 5 + [_i] * 8 + [_vp, _vp, _vp, _sz, _vp], _i),
    "kda_chunk_inter": ([_vp] * 6 + [_i] * 8 + [_vp, _vp, _vp, _sz, _vp], _i),
    "kda_chunk_output": ([_vp] * 6 + [_i] * 8 + [_vp, _vp, _sz, _vp], _i),
    "kda_decode_step": ([_vp] * 7 + [_i] * 5 + [_vp], _i),
    "kda_get_device_status": ([_vp, _vp], _i),
    "kda_chunk_fwd_noalloc": ([_vp] * 7 + [_i] * 8 + [_vp, _vp, _vp], _i),
    "kda_chunk_split_workspace_size": ([_i, _i, _i], _sz),
    "kda_chunk_fwd_plan": ([_i] * 8, _i),
    "kda_chunk_fwd_with_plan": ([_i] + [_vp] * 7 + [_i] * 8 + [_vp, _vp, _vp, _sz, _vp], _i),
    "kda_chunk_fwd_plan_workspace_size": ([_i] * 8, _sz),
    "kda_test_overlap_flag_timeout": ([_vp] * 7 + [_i] * 4 + [_vp] * 3 + [_sz, _i, _i,
                                      ctypes.c_ulonglong, _vp], _i),
    "kda_qkv_conv_norm": ([_vp] * 7 + [_i] * 7 + [ctypes.c_float] + [_vp] * 4, _i),
    "kda_output_norm_gate": ([_vp] * 3 + [_i] * 4 + [ctypes.c_float] + [_vp] * 2, _i),
    "kda_gdn_chunk_fwd_workspace_size": ([_i] * 7, _sz),
    "kda_gdn_chunk_fwd": ([_vp] * 7 + [_i] * 8 + [_vp, _vp, _vp, _sz, _vp], _i),
    "kda_gdn_decode_step": ([_vp] * 7 + [_i] * 5 + [_vp], _i),
    "kda_chunk_bwd_workspace_size": ([_i] * 5, _sz),
    "kda_chunk_bwd": ([_vp] * 9 + [_i] * 7 + [_vp] * 7 + [_sz, _vp], _i),
    "kda_gdn_chunk_bwd_workspace_size": ([_i] * 5, _sz),
    "kda_gdn_chunk_bwd": ([_vp] * 9 + [_i] * 7 + [_vp] * 7 + [_sz, _vp], _i),
    "kda_qkv_conv_norm_step": ([_vp] * 9 + [_i] * 5 + [ctypes.c_float] + [_vp] * 4, _i),
    "kda_chunk_split_intra": ([_vp] * 5 + [_i] * 4 + [_vp, _sz, _vp], _i),
    "kda_layer_decode_step": ([_vp] * 14 + [_i] * 5 + [ctypes.c_float] * 2 + [_vp, _vp], _i),
    "kda_layer_chunk_fwd": ([_vp] * 10 + [_i] * 8 + [_vp, _vp] + [ctypes.c_float] * 2 +
                            [_vp, _vp, _vp, _sz, _vp], _i),
    "kda_layer_chunk_fwd_workspace_size": ([_i] * 7, _sz),
    "kda_chunk_state_maps": ([_vp] * 6 + [_i] * 4 + [_vp, _vp, _vp, _sz, _vp], _i),
    "kda_fold_segment_states": ([_vp] * 3 + [_i] * 6 + [_vp, _vp, _vp], _i),
    "kda_chunk_split_chain": ([_vp] * 3 + [_i] * 4 + [_vp, _vp, _vp, _sz, _vp], _i),
}

# Size of the library's built-in scratch used by kda_chunk_fwd_noalloc.
KDA_NOALLOC_SCRATCH_BYTES = 64 << 20


def load(path: str = LIB_PATH):
    """Load libkda.so (once).  Raises KdaError if it is missing."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise KdaError(KDA_ERR_CUDA, f"libkda.so not found at {path}; run "
                               "`python -m gated_delta_rule_124_b200.build`")
            lib = ctypes.CDLL(path)
            for name, (args, res) in _SIGS.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = res
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    try:
        return load().kda_status_string(int(status)).decode()
    except KdaError:
        return f"status {status}"


def _p(t) -> int | None:
    """Device pointer of a tensor (or None for NULL); a plain int is passed
    through as a raw address."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


_TORCH_OF = {KDA_DTYPE_F32: torch.float32, KDA_DTYPE_BF16: torch.bfloat16}


def _check(what, dtype=None, typed=(), f32=(), i32=(), raw=()):
    """Reject tensors the C ABI would misread, before any pointer is passed:
    every tensor must be contiguous and on one device; `typed` tensors (q, k,
    v, o, dout ...) must have the call's dtype, `f32` ones (g, beta, states,
    gradients) float32, `i32` ones (cu_seqlens) int32; `raw` ones (workspaces)
    only contiguous.  Plain ints (raw addresses) and None are not checked."""
    want = None if dtype is None else _TORCH_OF[dtype_code(dtype)]
    dev = None
    for group, need in ((typed, want), (f32, torch.float32), (i32, torch.int32), (raw, None)):
        for t in group:
            if t is None or isinstance(t, int):
                continue
            if not isinstance(t, torch.Tensor):
                raise ValueError(f"{what}: expected a tensor, got {type(t).__name__}")
            if not t.is_contiguous():
                raise ValueError(f"{what}: every tensor must be contiguous (got strides "
                                 f"{tuple(t.stride())} for shape {tuple(t.shape)})")
            if need is not None and t.dtype != need:
                raise ValueError(f"{what}: expected {need}, got {t.dtype}")
            if dev is None:
                dev = t.device
            elif t.device != dev:
                raise ValueError(f"{what}: tensors on {dev} and {t.device}")


def _stream(stream) -> int | None:
    if stream is None:
        if not torch.cuda.is_available():
            return None
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def dtype_code(dtype) -> int:
    if dtype in (torch.bfloat16, "bf16", KDA_DTYPE_BF16):
        return KDA_DTYPE_BF16
    if dtype in (torch.float32, "f32", KDA_DTYPE_F32):
        return KDA_DTYPE_F32
    raise ValueError(f"unsupported dtype {dtype}")


def _ret(st: int, what: str, check: bool) -> int:
    if check and st != KDA_OK:
        raise KdaError(st, what)
    return st


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


# ------------------------------------------------------------- C-named calls

def kda_chunk_fwd_workspace_size(total_tokens, num_seqs, H, dk, dv, chunk, dtype) -> int:
    return int(load().kda_chunk_fwd_workspace_size(total_tokens, num_seqs, H, dk, dv, chunk,
                                                   dtype_code(dtype)))


KDA_PLAN_SIMT, KDA_PLAN_SPLIT, KDA_PLAN_OVERLAP = 0, 2, 3
PLAN_NAMES = {KDA_PLAN_SIMT: "simt", KDA_PLAN_SPLIT: "split", KDA_PLAN_OVERLAP: "overlap"}
PLAN_CODES = {v: k for k, v in PLAN_NAMES.items()}


def plan_code(plan) -> int:
    return PLAN_CODES[plan] if isinstance(plan, str) else int(plan)


def kda_chunk_fwd_plan(total_tokens, num_seqs, H, dk, dv, chunk, dtype, packed=False) -> int:
    return int(load().kda_chunk_fwd_plan(total_tokens, num_seqs, int(bool(packed)), H, dk, dv,
                                         chunk, dtype_code(dtype)))


def kda_num_chunks_upper_bound(total_tokens, num_seqs, chunk) -> int:
    return int(load().kda_num_chunks_upper_bound(total_tokens, num_seqs, chunk))


def kda_chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, B, T, num_seqs, H, dk, dv,
                  chunk, dtype, o, final_state, workspace, workspace_bytes=None, stream=None,
                  check=True) -> int:
    _check("kda_chunk_fwd", dtype, typed=(q, k, v, o), f32=(g, beta, initial_state, final_state),
           i32=(cu_seqlens,), raw=(workspace,))
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().kda_chunk_fwd(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(initial_state),
                              _p(cu_seqlens), B, T, num_seqs, H, dk, dv, chunk,
                              dtype_code(dtype), _p(o), _p(final_state), _p(workspace), wb,
                              _stream(stream))
    return _ret(st, "kda_chunk_fwd", check)


def kda_chunk_fwd_plan_workspace_size(plan, total_tokens, num_seqs, H, dk, dv, chunk,
                                      dtype) -> int:
    return int(load().kda_chunk_fwd_plan_workspace_size(plan_code(plan), total_tokens, num_seqs,
                                                        H, dk, dv, chunk, dtype_code(dtype)))


def kda_chunk_fwd_with_plan(plan, q, k, v, g, beta, initial_state, cu_seqlens, B, T, num_seqs, H,
                            dk, dv, chunk, dtype, o, final_state, workspace, workspace_bytes=None,
                            stream=None, check=True) -> int:
    """kda_chunk_fwd on an explicitly chosen plan ('simt', 'split', 'overlap'
    or its KDA_PLAN_* code); KDA_ERR_UNSUPPORTED where it cannot run."""
    _check("kda_chunk_fwd_with_plan", dtype, typed=(q, k, v, o),
           f32=(g, beta, initial_state, final_state), i32=(cu_seqlens,), raw=(workspace,))
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().kda_chunk_fwd_with_plan(plan_code(plan), _p(q), _p(k), _p(v), _p(g), _p(beta),
                                        _p(initial_state), _p(cu_seqlens), B, T, num_seqs, H,
                                        dk, dv, chunk, dtype_code(dtype), _p(o),
                                        _p(final_state), _p(workspace), wb, _stream(stream))
    return _ret(st, "kda_chunk_fwd_with_plan", check)


def kda_test_overlap_flag_timeout(q, k, v, g, beta, initial_state, cu_seqlens, B, T, num_seqs,
                                  H, o, final_state, workspace, withheld_chunk, withheld_head,
                                  flag_wait_ns, workspace_bytes=None, stream=None,
                                  check=True) -> int:
    """The overlap plan with one chunk's ready flag withheld and the chains'
    flag waits bounded by flag_wait_ns: exercises the bounded-wait error path
    (kda_get_device_status then reports KDA_ERR_TIMEOUT).  Testing only."""
    _check("kda_test_overlap_flag_timeout", "bf16", typed=(q, k, v, o),
           f32=(g, beta, initial_state, final_state), i32=(cu_seqlens,), raw=(workspace,))
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().kda_test_overlap_flag_timeout(_p(q), _p(k), _p(v), _p(g), _p(beta),
                                              _p(initial_state), _p(cu_seqlens), B, T, num_seqs,
                                              H, _p(o), _p(final_state), _p(workspace), wb,
                                              withheld_chunk, withheld_head, flag_wait_ns,
                                              _stream(stream))
    return _ret(st, "kda_test_overlap_flag_timeout", check)


def kda_chunk_gate_cumsum(g, cu_seqlens, B, T, num_seqs, H, dk, chunk, G, workspace,
                          workspace_bytes=None, stream=None, check=True) -> int:
    _check("kda_chunk_gate_cumsum", None, f32=(g, G), i32=(cu_seqlens,), raw=(workspace,))
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().kda_chunk_gate_cumsum(_p(g), _p(cu_seqlens), B, T, num_seqs, H, dk, chunk,
                                      _p(G), _p(workspace), wb, _stream(stream))
    return _ret(st, "kda_chunk_gate_cumsum", check)


def kda_chunk_intra(k, v, G, beta, cu_seqlens, B, T, num_seqs, H, dk, dv, chunk, dtype, W, Ut,
                    workspace, workspace_bytes=None, stream=None, check=True) -> int:
    _check("kda_chunk_intra", dtype, typed=(k, v), f32=(G, beta, W, Ut), i32=(cu_seqlens,),
           raw=(workspace,))
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().kda_chunk_intra(_p(k), _p(v), _p(G), _p(beta), _p(cu_seqlens), B, T, num_seqs,
                                H, dk, dv, chunk, dtype_code(dtype), _p(W), _p(Ut),
                                _p(workspace), wb, _stream(stream))
    return _ret(st, "kda_chunk_intra", check)


def kda_chunk_inter(k, G, W, U, initial_state, cu_seqlens, B, T, num_seqs, H, dk, dv, chunk,
                    dtype, chunk_states, final_state, workspace, workspace_bytes=None,
                    stream=None, check=True) -> int:
    _check("kda_chunk_inter", dtype, typed=(k,), f32=(G, W, U, initial_state, chunk_states,
           final_state), i32=(cu_seqlens,), raw=(workspace,))
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().kda_chunk_inter(_p(k), _p(G), _p(W), _p(U), _p(initial_state), _p(cu_seqlens),
                                B, T, num_seqs, H, dk, dv, chunk, dtype_code(dtype),
                                _p(chunk_states), _p(final_state), _p(workspace), wb,
                                _stream(stream))
    return _ret(st, "kda_chunk_inter", check)


def kda_chunk_output(q, k, G, U, chunk_states, cu_seqlens, B, T, num_seqs, H, dk, dv, chunk,
                     dtype, o, workspace, workspace_bytes=None, stream=None,
                     check=True) -> int:
    _check("kda_chunk_output", dtype, typed=(q, k, o), f32=(G, U, chunk_states),
           i32=(cu_seqlens,), raw=(workspace,))
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().kda_chunk_output(_p(q), _p(k), _p(G), _p(U), _p(chunk_states), _p(cu_seqlens),
                                 B, T, num_seqs, H, dk, dv, chunk, dtype_code(dtype), _p(o),
                                 _p(workspace), wb, _stream(stream))
    return _ret(st, "kda_chunk_output", check)


def kda_chunk_split_workspace_size(total_tokens, num_seqs, H) -> int:
    return int(load().kda_chunk_split_workspace_size(total_tokens, num_seqs, H))


def kda_chunk_split_intra(q, k, g, beta, cu_seqlens, B, T, num_seqs, H, workspace,
                          workspace_bytes=None, stream=None, check=True) -> int:
    _check("kda_chunk_split_intra", "bf16", typed=(q, k), f32=(g, beta), i32=(cu_seqlens,),
           raw=(workspace,))
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().kda_chunk_split_intra(_p(q), _p(k), _p(g), _p(beta), _p(cu_seqlens), B, T,
                                      num_seqs, H, _p(workspace), wb, _stream(stream))
    return _ret(st, "kda_chunk_split_intra", check)


def kda_chunk_split_chain(v, initial_state, cu_seqlens, B, T, num_seqs, H, o, final_state,
                          workspace, workspace_bytes=None, stream=None, check=True) -> int:
    _check("kda_chunk_split_chain", "bf16", typed=(v, o), f32=(initial_state, final_state),
           i32=(cu_seqlens,), raw=(workspace,))
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().kda_chunk_split_chain(_p(v), _p(initial_state), _p(cu_seqlens), B, T,
                                      num_seqs, H, _p(o), _p(final_state), _p(workspace), wb,
                                      _stream(stream))
    return _ret(st, "kda_chunk_split_chain", check)


def kda_gdn_chunk_fwd_workspace_size(total_tokens, num_seqs, H, dk, dv, chunk, dtype) -> int:
    return int(load().kda_gdn_chunk_fwd_workspace_size(total_tokens, num_seqs, H, dk, dv, chunk,
                                                       dtype_code(dtype)))


def kda_gdn_chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, B, T, num_seqs, H, dk, dv,
                      chunk, dtype, o, final_state, workspace, workspace_bytes=None, stream=None,
                      check=True) -> int:
    _check("kda_gdn_chunk_fwd", dtype, typed=(q, k, v, o), f32=(g, beta, initial_state,
           final_state), i32=(cu_seqlens,), raw=(workspace,))
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().kda_gdn_chunk_fwd(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(initial_state),
                                  _p(cu_seqlens), B, T, num_seqs, H, dk, dv, chunk,
                                  dtype_code(dtype), _p(o), _p(final_state), _p(workspace), wb,
                                  _stream(stream))
    return _ret(st, "kda_gdn_chunk_fwd", check)


def kda_gdn_decode_step(q, k, v, g, beta, state, o, N, H, dk, dv, dtype, stream=None,
                        check=True) -> int:
    _check("kda_gdn_decode_step", dtype, typed=(q, k, v, o), f32=(g, beta, state))
    st = load().kda_gdn_decode_step(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(state), _p(o), N,
                                    H, dk, dv, dtype_code(dtype), _stream(stream))
    return _ret(st, "kda_gdn_decode_step", check)


def kda_chunk_bwd_workspace_size(total_tokens, num_seqs, H, dk, dv) -> int:
    return int(load().kda_chunk_bwd_workspace_size(total_tokens, num_seqs, H, dk, dv))


def kda_chunk_bwd(q, k, v, g, beta, initial_state, dout, dfinal_state, cu_seqlens, B, T,
                  num_seqs, H, dk, dv, dtype, dq, dk_out, dv_out, dg, dbeta, dinitial_state,
                  workspace, workspace_bytes=None, stream=None, check=True) -> int:
    _check("kda_chunk_bwd", dtype, typed=(q, k, v, dout), f32=(g, beta, initial_state,
           dfinal_state, dq, dk_out, dv_out, dg, dbeta, dinitial_state), i32=(cu_seqlens,),
           raw=(workspace,))
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().kda_chunk_bwd(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(initial_state),
                              _p(dout), _p(dfinal_state), _p(cu_seqlens), B, T, num_seqs, H, dk,
                              dv, dtype_code(dtype), _p(dq), _p(dk_out), _p(dv_out), _p(dg),
                              _p(dbeta), _p(dinitial_state), _p(workspace), wb,
                              _stream(stream))
    return _ret(st, "kda_chunk_bwd", check)


def kda_gdn_chunk_bwd_workspace_size(total_tokens, num_seqs, H, dk, dv) -> int:
    return int(load().kda_gdn_chunk_bwd_workspace_size(total_tokens, num_seqs, H, dk, dv))


def kda_gdn_chunk_bwd(q, k, v, g, beta, initial_state, dout, dfinal_state, cu_seqlens, B, T,
                      num_seqs, H, dk, dv, dtype, dq, dk_out, dv_out, dg, dbeta, dinitial_state,
                      workspace, workspace_bytes=None, stream=None, check=True) -> int:
    _check("kda_gdn_chunk_bwd", dtype, typed=(q, k, v, dout), f32=(g, beta, initial_state,
           dfinal_state, dq, dk_out, dv_out, dg, dbeta, dinitial_state), i32=(cu_seqlens,),
           raw=(workspace,))
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().kda_gdn_chunk_bwd(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(initial_state),
                                  _p(dout), _p(dfinal_state), _p(cu_seqlens), B, T, num_seqs, H,
                                  dk, dv, dtype_code(dtype), _p(dq), _p(dk_out), _p(dv_out),
                                  _p(dg), _p(dbeta), _p(dinitial_state), _p(workspace), wb,
                                  _stream(stream))
    return _ret(st, "kda_gdn_chunk_bwd", check)


def kda_qkv_conv_norm_step(xq, xk, xv, wq, wk, wv, conv_q, conv_k, conv_v, N, H, dk, dv,
                           dtype, eps, q, k, v, stream=None, check=True) -> int:
    _check("kda_qkv_conv_norm_step", dtype, typed=(xq, xk, xv, conv_q, conv_k, conv_v, q, k, v),
           f32=(wq, wk, wv))
    st = load().kda_qkv_conv_norm_step(_p(xq), _p(xk), _p(xv), _p(wq), _p(wk), _p(wv),
                                       _p(conv_q), _p(conv_k), _p(conv_v), N, H, dk, dv,
                                       dtype_code(dtype), eps, _p(q), _p(k), _p(v),
                                       _stream(stream))
    return _ret(st, "kda_qkv_conv_norm_step", check)


def kda_qkv_conv_norm(xq, xk, xv, wq, wk, wv, cu_seqlens, B, T, num_seqs, H, dk, dv, dtype,
                      eps, q, k, v, stream=None, check=True) -> int:
    _check("kda_qkv_conv_norm", dtype, typed=(xq, xk, xv, q, k, v), f32=(wq, wk, wv),
           i32=(cu_seqlens,))
    st = load().kda_qkv_conv_norm(_p(xq), _p(xk), _p(xv), _p(wq), _p(wk), _p(wv),
                                  _p(cu_seqlens), B, T, num_seqs, H, dk, dv, dtype_code(dtype),
                                  float(eps), _p(q), _p(k), _p(v), _stream(stream))
    return _ret(st, "kda_qkv_conv_norm", check)


def kda_output_norm_gate(o, gate, w, total_tokens, H, dv, dtype, eps, y, stream=None,
                         check=True) -> int:
    _check("kda_output_norm_gate", dtype, typed=(o, gate, y), f32=(w,))
    st = load().kda_output_norm_gate(_p(o), _p(gate), _p(w), total_tokens, H, dv,
                                     dtype_code(dtype), float(eps), _p(y), _stream(stream))
    return _ret(st, "kda_output_norm_gate", check)


def kda_chunk_state_maps(q, k, v, g, beta, cu_seqlens, B, T, num_seqs, H, M, Bm, workspace,
                         workspace_bytes=None, stream=None, check=True) -> int:
    _check("kda_chunk_state_maps", "bf16", typed=(q, k, v), f32=(g, beta, M, Bm),
           i32=(cu_seqlens,), raw=(workspace,))
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().kda_chunk_state_maps(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(cu_seqlens), B, T,
                                     num_seqs, H, _p(M), _p(Bm), _p(workspace), wb,
                                     _stream(stream))
    return _ret(st, "kda_chunk_state_maps", check)


def kda_fold_segment_states(M, Bm, S0, R, N, H, dk, dv, reverse, each, final_state, stream=None,
                            check=True) -> int:
    _check("kda_fold_segment_states", None, f32=(M, Bm, S0, each, final_state))
    st = load().kda_fold_segment_states(_p(M), _p(Bm), _p(S0), R, N, H, dk, dv, int(bool(reverse)),
                                        _p(each), _p(final_state), _stream(stream))
    return _ret(st, "kda_fold_segment_states", check)


def kda_layer_chunk_fwd_workspace_size(total_tokens, num_seqs, H, dk, dv, chunk, dtype) -> int:
    return int(load().kda_layer_chunk_fwd_workspace_size(total_tokens, num_seqs, H, dk, dv, chunk,
                                                         dtype_code(dtype)))


def kda_layer_chunk_fwd(xq, xk, xv, wq, wk, wv, g, beta, initial_state, cu_seqlens, B, T,
                        num_seqs, H, dk, dv, chunk, dtype, gate, w_norm, l2_eps, rms_eps, y,
                        final_state, workspace, workspace_bytes=None, stream=None,
                        check=True) -> int:
    _check("kda_layer_chunk_fwd", dtype, typed=(xq, xk, xv, gate, y),
           f32=(wq, wk, wv, g, beta, initial_state, w_norm, final_state), i32=(cu_seqlens,),
           raw=(workspace,))
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().kda_layer_chunk_fwd(_p(xq), _p(xk), _p(xv), _p(wq), _p(wk), _p(wv), _p(g),
                                    _p(beta), _p(initial_state), _p(cu_seqlens), B, T, num_seqs,
                                    H, dk, dv, chunk, dtype_code(dtype), _p(gate), _p(w_norm),
                                    float(l2_eps), float(rms_eps), _p(y), _p(final_state),
                                    _p(workspace), wb, _stream(stream))
    return _ret(st, "kda_layer_chunk_fwd", check)


def kda_layer_decode_step(xq, xk, xv, wq, wk, wv, conv_q, conv_k, conv_v, g, beta, state, gate,
                          w_norm, N, H, dk, dv, dtype, l2_eps, rms_eps, y, stream=None,
                          check=True) -> int:
    _check("kda_layer_decode_step", dtype, typed=(xq, xk, xv, conv_q, conv_k, conv_v, gate, y),
           f32=(wq, wk, wv, g, beta, state, w_norm))
    st = load().kda_layer_decode_step(_p(xq), _p(xk), _p(xv), _p(wq), _p(wk), _p(wv),
                                      _p(conv_q), _p(conv_k), _p(conv_v), _p(g), _p(beta),
                                      _p(state), _p(gate), _p(w_norm), N, H, dk, dv,
                                      dtype_code(dtype), float(l2_eps), float(rms_eps), _p(y),
                                      _stream(stream))
    return _ret(st, "kda_layer_decode_step", check)


def kda_decode_step(q, k, v, g, beta, state, o, N, H, dk, dv, dtype, stream=None,
                    check=True) -> int:
    _check("kda_decode_step", dtype, typed=(q, k, v, o), f32=(g, beta, state))
    st = load().kda_decode_step(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(state), _p(o), N, H,
                                dk, dv, dtype_code(dtype), _stream(stream))
    return _ret(st, "kda_decode_step", check)


def kda_chunk_fwd_noalloc(q, k, v, g, beta, initial_state, cu_seqlens, B, T, num_seqs, H, dk,
                          dv, chunk, dtype, o, final_state, stream=None, check=True) -> int:
    """kda_chunk_fwd without a workspace: for callers that may not allocate
    device memory.  The library's own static scratch array is used instead;
    see include/kda.h for its size limit and sharing rules."""
    _check("kda_chunk_fwd_noalloc", dtype, typed=(q, k, v, o), f32=(g, beta, initial_state,
           final_state), i32=(cu_seqlens,))
    st = load().kda_chunk_fwd_noalloc(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(initial_state),
                                      _p(cu_seqlens), B, T, num_seqs, H, dk, dv, chunk,
                                      dtype_code(dtype), _p(o), _p(final_state),
                                      _stream(stream))
    return _ret(st, "kda_chunk_fwd_noalloc", check)


def kda_get_device_status(workspace, stream=None) -> int:
    _check("kda_get_device_status", None, raw=(workspace,))
    return int(load().kda_get_device_status(_p(workspace), _stream(stream)))


# ------------------------------------------------------- allocating wrappers

def alloc_workspace(total_tokens, num_seqs, H, dk, dv, chunk, dtype, device="cuda"):
    n = kda_chunk_fwd_workspace_size(total_tokens, num_seqs, H, dk, dv, chunk, dtype)
    if n == 0:
        raise KdaError(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def chunk_fwd(q, k, v, g, beta, initial_state=None, cu_seqlens=None, chunk=64,
              output_final_state=True, workspace=None, stream=None):
    """KDA chunkwise forward.  q, k [B, T, H, dk] or [T_total, H, dk] (packed with
    cu_seqlens); v likewise with dv; g like q (fp32); beta [.., H] (fp32).
    Returns (o, final_state or None).  All tensors on the current CUDA device."""
    packed = q.dim() == 3
    if packed:
        total, H, dk = q.shape
        B, T = 1, total
        N = (cu_seqlens.numel() - 1) if cu_seqlens is not None else 1
        if cu_seqlens is None:
            B, T = 1, total
    else:
        B, T, H, dk = q.shape
        total, N = B * T, B
        if cu_seqlens is not None:
            raise ValueError("cu_seqlens needs packed [T_total, H, d] inputs")
    dv = v.shape[-1]
    o = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    hN = (torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
          if output_final_state else None)
    if workspace is None:
        workspace = alloc_workspace(total, N, H, dk, dv, chunk, q.dtype, q.device)
    kda_chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, B, T, N, H, dk, dv, chunk,
                  q.dtype, o, hN, workspace, stream=stream)
    return o, hN


def chunk_bwd(q, k, v, g, beta, dout, initial_state=None, dfinal_state=None, cu_seqlens=None,
              head_gate=False, workspace=None, stream=None):
    """Gradients of sum(o * dout) + sum(final_state * dfinal_state) for
    chunk_fwd's inputs: returns (dq, dk, dv, dg, dbeta, dinitial_state), fp32,
    shaped like the inputs (dinitial_state [N, H, dk, dv]).  head_gate=True:
    g and dg are [.., H] (Gated DeltaNet)."""
    packed = q.dim() == 3
    if packed:
        total, H, dk = q.shape
        B, T = 1, total
        N = (cu_seqlens.numel() - 1) if cu_seqlens is not None else 1
    else:
        B, T, H, dk = q.shape
        total, N = B * T, B
        if cu_seqlens is not None:
            raise ValueError("cu_seqlens needs packed [T_total, H, d] inputs")
    dv = v.shape[-1]
    f32 = dict(dtype=torch.float32, device=q.device)
    dq = torch.empty(q.shape, **f32)
    dk_ = torch.empty(k.shape, **f32)
    dv_ = torch.empty(v.shape, **f32)
    dg = torch.empty(g.shape, **f32)
    db = torch.empty(beta.shape, **f32)
    dh0 = torch.empty(N, H, dk, dv, **f32)
    size = (kda_gdn_chunk_bwd_workspace_size if head_gate else kda_chunk_bwd_workspace_size)(
        total, N, H, dk, dv)
    if workspace is None:
        workspace = torch.empty(size, dtype=torch.uint8, device=q.device)
    call = kda_gdn_chunk_bwd if head_gate else kda_chunk_bwd
    call(q, k, v, g, beta, initial_state, dout, dfinal_state, cu_seqlens, B, T, N, H, dk, dv,
         q.dtype, dq, dk_, dv_, dg, db, dh0, workspace, stream=stream)
    return dq, dk_, dv_, dg, db, dh0


class ChunkKDA(torch.autograd.Function):
    """Differentiable KDA prefill: forward = chunk_fwd, backward = chunk_bwd (which
    recomputes the forward's per-chunk quantities, so only the inputs are
    saved).  Gradients of q, k, v are returned in their dtype."""

    @staticmethod
    def forward(ctx, q, k, v, g, beta, initial_state, cu_seqlens, head_gate):
        if head_gate:
            packed = q.dim() == 3
            H, dk = q.shape[-2], q.shape[-1]
            B, T = (1, q.shape[0]) if packed else (q.shape[0], q.shape[1])
            total = B * T
            N = (cu_seqlens.numel() - 1) if cu_seqlens is not None else B
            dv = v.shape[-1]
            o = torch.empty(v.shape, dtype=v.dtype, device=v.device)
            hN = torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
            ws = torch.empty(kda_gdn_chunk_fwd_workspace_size(total, N, H, dk, dv, 64, q.dtype),
                             dtype=torch.uint8, device=q.device)
            kda_gdn_chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, B, T, N, H, dk, dv, 64,
                              q.dtype, o, hN, ws)
        else:
            o, hN = chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens=cu_seqlens, chunk=64)
        ctx.save_for_backward(q, k, v, g, beta, initial_state, cu_seqlens)
        ctx.head_gate = head_gate
        return o, hN

    @staticmethod
    def backward(ctx, do, dhN):
        q, k, v, g, beta, h0, cu = ctx.saved_tensors
        do = torch.zeros_like(v) if do is None else do.to(v.dtype).contiguous()
        dhN = None if dhN is None else dhN.float().contiguous()
        dq, dk, dv, dg, db, dh0 = chunk_bwd(q, k, v, g, beta, do, h0, dhN, cu,
                                            head_gate=ctx.head_gate)
        return (dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype), dg, db,
                dh0 if h0 is not None else None, None, None)


def chunk_kda(q, k, v, g, beta, initial_state=None, cu_seqlens=None, head_gate=False):
    """Differentiable prefill: (o, final_state); see ChunkKDA."""
    return ChunkKDA.apply(q, k, v, g, beta, initial_state, cu_seqlens, head_gate)


def decode_step(q, k, v, g, beta, state, o=None, stream=None):
    """One recurrent step.  q, k, g [N, H, dk]; v [N, H, dv]; beta [N, H];
    state [N, H, dk, dv] fp32, updated in place.  Returns o [N, H, dv]."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty(N, H, dv, dtype=v.dtype, device=v.device)
    kda_decode_step(q, k, v, g, beta, state, o, N, H, dk, dv, q.dtype, stream=stream)
    return o
