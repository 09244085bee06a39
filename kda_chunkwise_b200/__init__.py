"""kda_chunkwise_b200 — Python binding of libkda (the KDA gated delta-rule recurrence on B200).

Argument marshalling only: every step of the recurrence runs in the CUDA kernels of libkda.so,
reached through its C ABI (include/kda.h).  PyTorch provides device memory and streams.  There is
no CPU or PyTorch fallback: importing this package without the built library raises ImportError.

Entry points (same names as the C ABI):
  kda_chunk_fwd(q, k, v, a, beta, A_log, cu_seqlens, ...)  prefill, chunkwise form
  kda_chunk_fwd_host(...)                                   the same prefill on host tensors, the copies
                                                            overlapped with the compute piece by piece
  kda_decode_step(q, k, v, a, beta, A_log, state, ...)      one recurrent step, state in place
  kda_decode_verify / kda_decode_commit                     K proposed tokens, then the accepted prefix
  kda_short_conv, kda_output_norm_gate                      the module's short convolution and
                                                            pre-gate normalisation + output gate
  kda_segment_maps, kda_state_combine,                      context-parallel prefill: a sequence split
  kda_context_parallel_fwd                                  into segments over the ranks of a group
  kda_chunk_bwd                                             gradients of the prefill (chunkwise=True: the
                                                            chunkwise form, kda_chunk_bwd_chunkwise)
  chunk_kda(...)                                            the prefill as a torch.autograd function: its
                                                            forward is kda_chunk_fwd, its backward kda_chunk_bwd
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

import torch

__all__ = ["kda_chunk_fwd", "kda_decode_step", "kda_chunk_fwd_workspace_size",
           "kda_chunk_fwd_workspace_min", "kda_sync_check", "kda_status_string", "KDAError",
           "kda_launch_count", "kda_chunk_fwd_noalloc", "kda_inject_stall",
           "kda_decode_verify", "kda_decode_commit", "kda_short_conv", "kda_output_norm_gate",
           "kda_state_combine", "kda_segment_maps", "context_parallel_states", "kda_context_parallel_fwd",
           "kda_chunk_bwd", "kda_chunk_bwd_workspace_size", "kda_chunk_fwd_host",
           "kda_chunk_fwd_host_buffer_size", "chunk_kda",
           "LIB_PATH", "lib"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkda.so")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_TIMEOUT, KDA_ERR_RANGE = range(6)
KDA_DTYPE_BF16, KDA_DTYPE_F32 = 0, 1
_OUT_DTYPES = {torch.bfloat16: KDA_DTYPE_BF16, torch.float32: KDA_DTYPE_F32}


class KDAError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = f"{where}: {kda_status_string(status)}"
        super().__init__(msg + (f" ({detail})" if detail else ""))


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkda.so is not built ({LIB_PATH}); run `python "
                          "kda_chunkwise_b200/csrc/build.py` (nvcc 12.9, sm_100a) first")
    L = ctypes.CDLL(LIB_PATH)
    vp, fp, i32, i64, sz, f32 = (ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                 ctypes.c_int64, ctypes.c_size_t, ctypes.c_float)
    L.kda_chunk_fwd.argtypes = [vp, vp, vp, vp, fp, vp, fp, vp, i32, i64, i32, i32, i32, i32, f32,
                                fp, fp, vp, ctypes.c_int, vp, sz, vp]
    L.kda_chunk_fwd.restype = ctypes.c_int
    L.kda_chunk_fwd_noalloc.argtypes = [vp, vp, vp, vp, fp, vp, fp, vp, i32, i64, i32, i32, i32,
                                        i32, f32, fp, fp, vp, ctypes.c_int, vp]
    L.kda_chunk_fwd_noalloc.restype = ctypes.c_int
    L.kda_chunk_fwd_workspace_size.argtypes = [i64, i32, i32, i32, i32, i32]
    L.kda_chunk_fwd_workspace_size.restype = sz
    L.kda_chunk_fwd_workspace_min.argtypes = [i64, i32, i32, i32, i32, i32]
    L.kda_chunk_fwd_workspace_min.restype = sz
    L.kda_decode_step.argtypes = [vp, vp, vp, vp, fp, vp, fp, fp, vp, ctypes.c_int, i32, i32, i32,
                                  i32, f32, vp]
    L.kda_decode_step.restype = ctypes.c_int
    L.kda_status_string.argtypes = [ctypes.c_int]
    L.kda_status_string.restype = ctypes.c_char_p
    L.kda_sync_check.argtypes = [vp]
    L.kda_sync_check.restype = ctypes.c_int
    L.kda_last_error.argtypes = []
    L.kda_last_error.restype = ctypes.c_char_p
    L.kda_launch_count.argtypes = []
    L.kda_launch_count.restype = ctypes.c_uint64
    L.kda_decode_verify.argtypes = [vp, vp, vp, vp, fp, vp, fp, fp, fp, vp, ctypes.c_int, i32, i32, i32,
                                    i32, i32, f32, vp]
    L.kda_decode_verify.restype = ctypes.c_int
    L.kda_decode_commit.argtypes = [vp, vp, fp, vp, fp, fp, i32, i32, i32, i32, i32, vp]
    L.kda_decode_commit.restype = ctypes.c_int
    L.kda_short_conv.argtypes = [vp, fp, vp, i32, i64, i32, i32, i32, i32, vp, vp]
    L.kda_short_conv.restype = ctypes.c_int
    L.kda_output_norm_gate.argtypes = [fp, vp, fp, i64, i32, i32, f32, vp, ctypes.c_int, vp]
    L.kda_output_norm_gate.restype = ctypes.c_int
    L.kda_state_combine.argtypes = [fp, fp, fp, fp, i32, i32, i32, vp]
    L.kda_state_combine.restype = ctypes.c_int
    L.kda_chunk_bwd.argtypes = [vp, vp, vp, vp, fp, vp, fp, vp, i32, i64, i32, i32, i32, f32, fp, fp, fp,
                                fp, fp, fp, fp, fp, fp, fp, fp, vp, sz, vp]
    L.kda_chunk_bwd.restype = ctypes.c_int
    L.kda_chunk_bwd_workspace_size.argtypes = [i64, i32, i32, i32, i32]
    L.kda_chunk_bwd_workspace_size.restype = sz
    L.kda_chunk_bwd_chunkwise.argtypes = L.kda_chunk_bwd.argtypes
    L.kda_chunk_bwd_chunkwise.restype = ctypes.c_int
    L.kda_chunk_bwd_chunkwise_workspace_size.argtypes = [i64, i32, i32, i32, i32]
    L.kda_chunk_bwd_chunkwise_workspace_size.restype = sz
    L.kda_chunk_fwd_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, f32, vp, vp, vp,
                                     ctypes.c_int, i64, vp, sz, vp]
    L.kda_chunk_fwd_host.restype = ctypes.c_int
    L.kda_chunk_fwd_host_buffer_size.argtypes = [vp, i32, i64, i32, i32, i32, ctypes.c_int, i64]
    L.kda_chunk_fwd_host_buffer_size.restype = sz
    L.kda_inject_stall.argtypes = [i32, ctypes.c_uint64]
    L.kda_inject_stall.restype = ctypes.c_int
    L.kda_set_prefill_path.argtypes = [i32]
    L.kda_set_prefill_path.restype = ctypes.c_int
    L.kda_prefill_path.argtypes = [i64, i32, i32]
    L.kda_prefill_path.restype = i32
    L.kda_segment_maps.argtypes = [vp, vp, vp, vp, fp, fp, vp, i32, i64, i32, i32, i32, f32, fp, fp, vp, sz, vp]
    L.kda_segment_maps.restype = ctypes.c_int
    L.kda_segment_maps_workspace_size.argtypes = [i64, i32, i32, i32]
    L.kda_segment_maps_workspace_size.restype = sz
    return L


lib = _load()


def kda_status_string(status: int) -> str:
    return lib.kda_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != KDA_OK:
        raise KDAError(status, where, lib.kda_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype, shape, device):
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def kda_chunk_fwd_workspace_size(total_tokens, num_seqs, max_seqlen, H, d_k, d_v) -> int:
    return int(lib.kda_chunk_fwd_workspace_size(total_tokens, num_seqs, max_seqlen, H, d_k, d_v))


def kda_chunk_fwd_workspace_min(total_tokens, num_seqs, max_seqlen, H, d_k, d_v) -> int:
    return int(lib.kda_chunk_fwd_workspace_min(total_tokens, num_seqs, max_seqlen, H, d_k, d_v))


def kda_chunk_fwd(q, k, v, a, beta, A_log, cu_seqlens, gate=None, initial_state=None,
                  output_final_state: bool = True, scale: float = 1.0, max_seqlen: int | None = None,
                  out=None, final_state=None, workspace=None, stream=None,
                  out_dtype=torch.bfloat16):
    """Chunkwise prefill over packed sequences (see include/kda.h for the full contract).

    q, k, a [T, H, d_k] bf16; v, gate [T, H, d_v] bf16; beta [T, H] fp32; A_log [H] fp32;
    cu_seqlens [N+1] int32 (device); initial_state [N, H, d_k, d_v] fp32 or None.
    max_seqlen: longest sequence (None: computed from cu_seqlens with one device->host copy).
    out_dtype: storage of the output, torch.bfloat16 or torch.float32 (taken from ``out`` if given).
    Returns (out [T, H, d_v], final_state [N, H, d_k, d_v] fp32 or None).
    """
    dev = q.device
    T, H, d_k = q.shape
    d_v = v.shape[-1]
    N = cu_seqlens.numel() - 1
    bf = torch.bfloat16
    for name, t, shp in (("q", q, (T, H, d_k)), ("k", k, (T, H, d_k)), ("a", a, (T, H, d_k)),
                         ("v", v, (T, H, d_v))):
        _need(t, name, bf, shp, dev)
    _need(beta, "beta", torch.float32, (T, H), dev)
    _need(A_log, "A_log", torch.float32, (H,), dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,), dev)
    if gate is not None:
        _need(gate, "gate", bf, (T, H, d_v), dev)
    if initial_state is not None:
        _need(initial_state, "initial_state", torch.float32, (N, H, d_k, d_v), dev)
    if out is None:
        out = torch.empty((T, H, d_v), dtype=out_dtype, device=dev)
    if out.dtype not in _OUT_DTYPES:
        raise TypeError("out must be bfloat16 or float32")
    _need(out, "out", out.dtype, (T, H, d_v), dev)
    if output_final_state and final_state is None:
        final_state = torch.empty((N, H, d_k, d_v), dtype=torch.float32, device=dev)
    if final_state is not None:
        _need(final_state, "final_state", torch.float32, (N, H, d_k, d_v), dev)
    if max_seqlen is None:
        max_seqlen = int((cu_seqlens[1:] - cu_seqlens[:-1]).max().item()) if N > 0 else 0
    if workspace is None:
        nbytes = kda_chunk_fwd_workspace_size(T, N, max_seqlen, H, d_k, d_v)
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    st = lib.kda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta), _ptr(gate),
                           _ptr(A_log), _ptr(cu_seqlens), N, T, int(max_seqlen), H, d_k, d_v,
                           float(scale), _ptr(initial_state), _ptr(final_state), _ptr(out),
                           _OUT_DTYPES[out.dtype], _ptr(workspace), workspace.numel() * workspace.element_size(),
                           _stream_handle(stream, dev))
    _check(st, "kda_chunk_fwd")
    return out, final_state


def kda_chunk_fwd_host_buffer_size(cu_seqlens, H, d_k, d_v, out_dtype=torch.bfloat16, piece_tokens: int = 0) -> int:
    """Device bytes kda_chunk_fwd_host needs; cu_seqlens is a host int32 tensor."""
    N = cu_seqlens.numel() - 1
    T = int(cu_seqlens[-1]) if N >= 0 else 0
    return int(lib.kda_chunk_fwd_host_buffer_size(_ptr(cu_seqlens), N, T, H, d_k, d_v, _OUT_DTYPES[out_dtype],
                                                  int(piece_tokens)))


def kda_chunk_fwd_host(q, k, v, a, beta, A_log, cu_seqlens, gate=None, initial_state=None, out=None,
                       final_state=None, out_dtype=torch.bfloat16, scale: float = 1.0, piece_tokens: int = 0,
                       device_buffer=None, device=None, stream=None):
    """Prefill of a batch held in host memory (see include/kda.h): every tensor, A_log and cu_seqlens
    included, is on the CPU (page-locked tensors let the copies overlap the compute).  The outputs
    ``out`` and ``final_state`` (host tensors; allocated page-locked when not given) hold the result
    once ``stream`` has reached the end of the call.  device_buffer: a CUDA uint8 tensor of
    kda_chunk_fwd_host_buffer_size(...) bytes (allocated when not given).
    Returns (out, final_state)."""
    cpu = torch.device("cpu")
    T, H, d_k = q.shape
    d_v = v.shape[-1]
    N = cu_seqlens.numel() - 1
    bf = torch.bfloat16
    for name, t, shp in (("q", q, (T, H, d_k)), ("k", k, (T, H, d_k)), ("a", a, (T, H, d_k)),
                         ("v", v, (T, H, d_v))):
        _need(t, name, bf, shp, cpu)
    _need(beta, "beta", torch.float32, (T, H), cpu)
    _need(A_log, "A_log", torch.float32, (H,), cpu)
    _need(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,), cpu)
    if gate is not None:
        _need(gate, "gate", bf, (T, H, d_v), cpu)
    if initial_state is not None:
        _need(initial_state, "initial_state", torch.float32, (N, H, d_k, d_v), cpu)
    for name, t in (("q", q), ("k", k), ("a", a), ("v", v), ("beta", beta), ("gate", gate),
                    ("initial_state", initial_state), ("A_log", A_log), ("cu_seqlens", cu_seqlens)):
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if out is None:
        out = torch.empty((T, H, d_v), dtype=out_dtype, pin_memory=True)
    if out.dtype not in _OUT_DTYPES:
        raise TypeError("out must be bfloat16 or float32")
    _need(out, "out", out.dtype, (T, H, d_v), cpu)
    if final_state is None:
        final_state = torch.empty((N, H, d_k, d_v), dtype=torch.float32, pin_memory=True)
    _need(final_state, "final_state", torch.float32, (N, H, d_k, d_v), cpu)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if device_buffer is None:
        nbytes = kda_chunk_fwd_host_buffer_size(cu_seqlens, H, d_k, d_v, out.dtype, piece_tokens)
        device_buffer = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    st = lib.kda_chunk_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta), _ptr(gate), _ptr(A_log),
                                _ptr(cu_seqlens), N, T, H, d_k, d_v, float(scale), _ptr(initial_state),
                                _ptr(final_state), _ptr(out), _OUT_DTYPES[out.dtype], int(piece_tokens),
                                _ptr(device_buffer), device_buffer.numel(), _stream_handle(stream, dev))
    _check(st, "kda_chunk_fwd_host")
    return out, final_state


def kda_chunk_fwd_noalloc(q, k, v, a, beta, A_log, cu_seqlens, max_seqlen: int, gate=None,
                          initial_state=None, scale: float = 1.0, out=None, final_state=None,
                          stream=None):
    """kda_chunk_fwd on the library's built-in 32 MiB scratch instead of a workspace.

    For callers that cannot allocate device memory on this path: it allocates nothing (the
    caller passes ``out`` and ``final_state`` if it wants them; ``out`` is required and its dtype,
    bfloat16 or float32, selects the output storage).  Calls on one device share the scratch:
    keep them on one stream.  max_seqlen must be given (no device-to-host read is made).
    """
    dev = q.device
    T, H, d_k = q.shape
    d_v = v.shape[-1]
    N = cu_seqlens.numel() - 1
    bf = torch.bfloat16
    for name, t, shp in (("q", q, (T, H, d_k)), ("k", k, (T, H, d_k)), ("a", a, (T, H, d_k)),
                         ("v", v, (T, H, d_v))):
        _need(t, name, bf, shp, dev)
    _need(beta, "beta", torch.float32, (T, H), dev)
    _need(A_log, "A_log", torch.float32, (H,), dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,), dev)
    if gate is not None:
        _need(gate, "gate", bf, (T, H, d_v), dev)
    if initial_state is not None:
        _need(initial_state, "initial_state", torch.float32, (N, H, d_k, d_v), dev)
    if out is None or out.dtype not in _OUT_DTYPES:
        raise ValueError("out (bfloat16 or float32, [T, H, d_v]) is required")
    _need(out, "out", out.dtype, (T, H, d_v), dev)
    if final_state is not None:
        _need(final_state, "final_state", torch.float32, (N, H, d_k, d_v), dev)
    st = lib.kda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta), _ptr(gate),
                                   _ptr(A_log), _ptr(cu_seqlens), N, T, int(max_seqlen), H, d_k,
                                   d_v, float(scale), _ptr(initial_state), _ptr(final_state),
                                   _ptr(out), _OUT_DTYPES[out.dtype], _stream_handle(stream, dev))
    _check(st, "kda_chunk_fwd_noalloc")
    return out, final_state


def kda_decode_step(q, k, v, a, beta, A_log, state, gate=None, scale: float = 1.0, out=None,
                    stream=None, out_dtype=torch.bfloat16):
    """One recurrent step for N sequences; ``state`` [N, H, d_k, d_v] fp32 is updated in place.

    q, k, a [N, H, d_k] bf16; v, gate [N, H, d_v] bf16; beta [N, H] fp32; A_log [H] fp32.
    Returns out [N, H, d_v] (bfloat16 or float32, see kda_chunk_fwd).
    """
    dev = q.device
    N, H, d_k = q.shape
    d_v = v.shape[-1]
    bf = torch.bfloat16
    for name, t, shp in (("q", q, (N, H, d_k)), ("k", k, (N, H, d_k)), ("a", a, (N, H, d_k)),
                         ("v", v, (N, H, d_v))):
        _need(t, name, bf, shp, dev)
    _need(beta, "beta", torch.float32, (N, H), dev)
    _need(A_log, "A_log", torch.float32, (H,), dev)
    _need(state, "state", torch.float32, (N, H, d_k, d_v), dev)
    if gate is not None:
        _need(gate, "gate", bf, (N, H, d_v), dev)
    if out is None:
        out = torch.empty((N, H, d_v), dtype=out_dtype, device=dev)
    if out.dtype not in _OUT_DTYPES:
        raise TypeError("out must be bfloat16 or float32")
    _need(out, "out", out.dtype, (N, H, d_v), dev)
    st = lib.kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta), _ptr(gate),
                             _ptr(A_log), _ptr(state), _ptr(out), _OUT_DTYPES[out.dtype], N, H,
                             d_k, d_v, float(scale),
                             _stream_handle(stream, dev))
    _check(st, "kda_decode_step")
    return out


def kda_decode_verify(q, k, v, a, beta, A_log, state, gate=None, scale: float = 1.0, u=None, out=None,
                      stream=None, out_dtype=torch.bfloat16):
    """Run K proposed tokens of N sequences from ``state`` without changing it.

    q, k, a [N, K, H, d_k] bf16; v, gate [N, K, H, d_v] bf16; beta [N, K, H] fp32; A_log [H];
    state [N, H, d_k, d_v] fp32 (read only).  Returns (out [N, K, H, d_v], u [N, H, K, d_v] fp32);
    pass u to kda_decode_commit.
    """
    dev = q.device
    N, K, H, d_k = q.shape
    d_v = v.shape[-1]
    bf = torch.bfloat16
    for name, t, shp in (("q", q, (N, K, H, d_k)), ("k", k, (N, K, H, d_k)), ("a", a, (N, K, H, d_k)),
                         ("v", v, (N, K, H, d_v))):
        _need(t, name, bf, shp, dev)
    _need(beta, "beta", torch.float32, (N, K, H), dev)
    _need(A_log, "A_log", torch.float32, (H,), dev)
    _need(state, "state", torch.float32, (N, H, d_k, d_v), dev)
    if gate is not None:
        _need(gate, "gate", bf, (N, K, H, d_v), dev)
    if u is None:
        u = torch.empty((N, H, K, d_v), dtype=torch.float32, device=dev)
    _need(u, "u", torch.float32, (N, H, K, d_v), dev)
    if out is None:
        out = torch.empty((N, K, H, d_v), dtype=out_dtype, device=dev)
    if out.dtype not in _OUT_DTYPES:
        raise TypeError("out must be bfloat16 or float32")
    _need(out, "out", out.dtype, (N, K, H, d_v), dev)
    st = lib.kda_decode_verify(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta), _ptr(gate), _ptr(A_log),
                               _ptr(state), _ptr(u), _ptr(out), _OUT_DTYPES[out.dtype], N, K, H, d_k, d_v,
                               float(scale), _stream_handle(stream, dev))
    _check(st, "kda_decode_verify")
    return out, u


def kda_decode_commit(k, a, A_log, accepted, u, state, stream=None):
    """Advance each state by its accepted[n] verified tokens (int32 [N] on the device); in place."""
    dev = k.device
    N, K, H, d_k = k.shape
    d_v = u.shape[-1]
    _need(k, "k", torch.bfloat16, (N, K, H, d_k), dev)
    _need(a, "a", torch.bfloat16, (N, K, H, d_k), dev)
    _need(A_log, "A_log", torch.float32, (H,), dev)
    _need(accepted, "accepted", torch.int32, (N,), dev)
    _need(u, "u", torch.float32, (N, H, K, d_v), dev)
    _need(state, "state", torch.float32, (N, H, d_k, d_v), dev)
    st = lib.kda_decode_commit(_ptr(k), _ptr(a), _ptr(A_log), _ptr(accepted), _ptr(u), _ptr(state),
                               N, K, H, d_k, d_v, _stream_handle(stream, dev))
    _check(st, "kda_decode_commit")
    return state


def kda_short_conv(x, w, cu_seqlens, l2norm: bool = False, out=None, stream=None):
    """Causal depthwise convolution over time per packed sequence (bf16 [T, H, d] in and out),
    optionally L2-normalising every (token, head) row.  w: fp32 [H, d, width], width <= 4."""
    dev = x.device
    T, H, d = x.shape
    width = w.shape[-1]
    _need(x, "x", torch.bfloat16, (T, H, d), dev)
    _need(w, "w", torch.float32, (H, d, width), dev)
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.device != dev or cu_seqlens.dim() != 1:
        raise TypeError("cu_seqlens must be int32 [num_seqs + 1] on the device")
    if out is None:
        out = torch.empty_like(x)
    _need(out, "out", torch.bfloat16, (T, H, d), dev)
    st = lib.kda_short_conv(_ptr(x), _ptr(w), _ptr(cu_seqlens), cu_seqlens.numel() - 1, T, H, d, width,
                            1 if l2norm else 0, _ptr(out), _stream_handle(stream, dev))
    _check(st, "kda_short_conv")
    return out


def kda_output_norm_gate(o, gate, w, eps: float = 1e-6, out=None, stream=None, out_dtype=torch.bfloat16):
    """out = sigmoid(gate) * RMSNorm(o) * w per (token, head) row; o fp32 [T, H, d_v], gate bf16 or
    None, w fp32 [d_v]."""
    dev = o.device
    T, H, d_v = o.shape
    _need(o, "o", torch.float32, (T, H, d_v), dev)
    _need(w, "w", torch.float32, (d_v,), dev)
    if gate is not None:
        _need(gate, "gate", torch.bfloat16, (T, H, d_v), dev)
    if out is None:
        out = torch.empty((T, H, d_v), dtype=out_dtype, device=dev)
    if out.dtype not in _OUT_DTYPES:
        raise TypeError("out must be bfloat16 or float32")
    _need(out, "out", out.dtype, (T, H, d_v), dev)
    st = lib.kda_output_norm_gate(_ptr(o), _ptr(gate), _ptr(w), T, H, d_v, float(eps), _ptr(out),
                                  _OUT_DTYPES[out.dtype], _stream_handle(stream, dev))
    _check(st, "kda_output_norm_gate")
    return out


def kda_state_combine(M, S_in, B, out=None, stream=None):
    """S_out = M S_in + B per (sequence, head): M fp32 [..., d_k, d_k], S_in and B [..., d_k, d_v]."""
    dev = M.device
    d_k, d_v = B.shape[-2], B.shape[-1]
    lead = tuple(B.shape[:-2])
    units = int(np.prod(lead)) if lead else 1
    _need(M, "M", torch.float32, lead + (d_k, d_k), dev)
    _need(S_in, "S_in", torch.float32, lead + (d_k, d_v), dev)
    _need(B, "B", torch.float32, lead + (d_k, d_v), dev)
    if out is None:
        out = torch.empty_like(B)
    _need(out, "out", torch.float32, lead + (d_k, d_v), dev)
    st = lib.kda_state_combine(_ptr(M), _ptr(S_in), _ptr(B), _ptr(out), units, d_k, d_v,
                               _stream_handle(stream, dev))
    _check(st, "kda_state_combine")
    return out


def kda_segment_maps(q, k, v, a, beta, A_log, cu_seqlens, scale: float = 1.0, max_seqlen=None, stream=None,
                     single_pass: bool | None = None):
    """The affine map S -> M S + B of each (sequence, head) over the tokens given: B is the final
    state from S = 0, M the final state of the homogeneous recurrence (v = 0) from S = I.  Returns
    (M [N, H, d_k, d_k], B [N, H, d_k, d_v]).

    single_pass: one pass of the cluster kernel over value columns [0 | v] from [I | 0]
    (kda_segment_maps; d_k = d_v only), which shares the chunk-local work of both maps but needs
    2 d / 32 CTAs per unit; or two kda_chunk_fwd calls.  None: one pass when every unit's cluster
    fits the GPU at once (then it takes the time of one of the two calls), else two calls (the same
    SM time, and with many units kda_chunk_fwd's per-unit kernel is the faster one)."""
    N = cu_seqlens.numel() - 1
    T, H, d_k = q.shape
    d_v = v.shape[-1]
    dev = q.device
    if single_pass is None:
        sms = torch.cuda.get_device_properties(dev).multi_processor_count if dev.type == "cuda" else 0
        single_pass = N * H * (2 * d_k // 32) <= sms
    if single_pass and d_k == d_v:
        for name, t in (("q", q), ("k", k), ("v", v), ("a", a)):
            _need(t, name, torch.bfloat16, (T, H, d_k), dev)
        _need(beta, "beta", torch.float32, (T, H), dev)
        _need(A_log, "A_log", torch.float32, (H,), dev)
        _need(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,), dev)
        if max_seqlen is None:
            max_seqlen = int((cu_seqlens[1:] - cu_seqlens[:-1]).max().item()) if N > 0 else 0
        M = torch.empty((N, H, d_k, d_k), dtype=torch.float32, device=dev)
        B = torch.empty((N, H, d_k, d_k), dtype=torch.float32, device=dev)
        ws = torch.empty(max(int(lib.kda_segment_maps_workspace_size(T, N, H, d_k)), 1), dtype=torch.uint8, device=dev)
        st = lib.kda_segment_maps(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta), _ptr(A_log), _ptr(cu_seqlens), N, T,
                                  max_seqlen, H, d_k, scale, _ptr(M), _ptr(B), _ptr(ws), ws.numel(),
                                  _stream_handle(stream, dev))
        _check(st, "kda_segment_maps")
        return M, B
    _, B = kda_chunk_fwd(q, k, v, a, beta, A_log, cu_seqlens, gate=None, initial_state=None, scale=scale,
                         max_seqlen=max_seqlen, stream=stream, out_dtype=torch.bfloat16)
    v0 = torch.zeros((T, H, d_k), dtype=torch.bfloat16, device=q.device)
    eye = torch.eye(d_k, dtype=torch.float32, device=q.device).expand(N, H, d_k, d_k).contiguous()
    _, M = kda_chunk_fwd(q, k, v0, a, beta, A_log, cu_seqlens, gate=None, initial_state=eye, scale=scale,
                         max_seqlen=max_seqlen, stream=stream, out_dtype=torch.bfloat16)
    return M, B


def context_parallel_states(M, B, S0, group=None, combine=None):
    """Incoming state of this rank's segments: gather every rank's (M, B) over the process group and
    fold the maps of the ranks before this one, in rank order, starting from S0.  ``combine(M, S, B)``
    applies one map (kda_state_combine unless given)."""
    import torch.distributed as dist
    combine = combine or (lambda m, s, b: kda_state_combine(m, s, b))
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    S = S0.clone() if S0 is not None else torch.zeros_like(B)
    if world == 1:
        return S
    rank = dist.get_rank(group)

    # NCCL gathers device tensors directly; gloo (CPU ranks, or ranks sharing one GPU) goes through
    # host copies
    via_host = M.is_cuda and dist.get_backend(group) == "gloo"

    def gather(x):   # every rank's x, stacked in rank order
        src = x.contiguous().cpu() if via_host else x.contiguous()
        flat = torch.empty((world * src.shape[0],) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
        dist.all_gather_into_tensor(flat, src, group=group)
        flat = flat.to(x.device) if via_host else flat
        return flat.view((world,) + tuple(x.shape))

    Ms, Bs = gather(M), gather(B)
    for r in range(rank):
        S = combine(Ms[r], S, Bs[r])
    return S


def kda_context_parallel_fwd(q, k, v, a, beta, A_log, cu_seqlens, gate=None, initial_state=None,
                             scale: float = 1.0, group=None, max_seqlen=None, stream=None,
                             out_dtype=torch.bfloat16):
    """Prefill of sequences split along time over the ranks of ``group``: this rank holds segment
    `rank` of every sequence (the same sequences, in the same order, on every rank; segments in
    rank order).  ``initial_state`` is the sequences' initial state (the same on every rank).
    Returns (out of this segment, state after this segment): on the last rank, the final states."""
    M, B = kda_segment_maps(q, k, v, a, beta, A_log, cu_seqlens, scale=scale, max_seqlen=max_seqlen,
                            stream=stream)
    S_in = context_parallel_states(M, B, initial_state, group=group)
    return kda_chunk_fwd(q, k, v, a, beta, A_log, cu_seqlens, gate=gate, initial_state=S_in, scale=scale,
                         max_seqlen=max_seqlen, stream=stream, out_dtype=out_dtype)


def kda_chunk_bwd_workspace_size(total_tokens, num_seqs, H, d_k, d_v) -> int:
    return int(lib.kda_chunk_bwd_workspace_size(total_tokens, num_seqs, H, d_k, d_v))


def kda_chunk_bwd_chunkwise_workspace_size(total_tokens, num_seqs, H, d_k, d_v) -> int:
    return int(lib.kda_chunk_bwd_chunkwise_workspace_size(total_tokens, num_seqs, H, d_k, d_v))


def kda_chunk_bwd(q, k, v, a, beta, A_log, cu_seqlens, dout, gate=None, initial_state=None,
                  dfinal_state=None, scale: float = 1.0, workspace=None, stream=None, chunkwise: bool = False):
    """Gradients of kda_chunk_fwd's outputs (and final states) with respect to its inputs.

    dout fp32 [T, H, d_v]; dfinal_state fp32 [N, H, d_k, d_v] or None.  Returns a dict of fp32
    tensors: dq, dk, da [T, H, d_k]; dv, dgate [T, H, d_v] (dgate None without a gate); dbeta
    [T, H]; dA_log [H]; dinitial_state [N, H, d_k, d_v] (None without an initial state).
    chunkwise: run kda_chunk_bwd_chunkwise (the chunkwise form) instead of the token-level kernel;
    the gradients agree to rounding.
    """
    dev = q.device
    T, H, d_k = q.shape
    d_v = v.shape[-1]
    N = cu_seqlens.numel() - 1
    bf, f32 = torch.bfloat16, torch.float32
    for name, t, shp in (("q", q, (T, H, d_k)), ("k", k, (T, H, d_k)), ("a", a, (T, H, d_k)),
                         ("v", v, (T, H, d_v))):
        _need(t, name, bf, shp, dev)
    _need(beta, "beta", f32, (T, H), dev)
    _need(A_log, "A_log", f32, (H,), dev)
    _need(dout, "dout", f32, (T, H, d_v), dev)
    if gate is not None:
        _need(gate, "gate", bf, (T, H, d_v), dev)
    if initial_state is not None:
        _need(initial_state, "initial_state", f32, (N, H, d_k, d_v), dev)
    if dfinal_state is not None:
        _need(dfinal_state, "dfinal_state", f32, (N, H, d_k, d_v), dev)
    g = dict(dq=torch.empty((T, H, d_k), dtype=f32, device=dev), dk=torch.empty((T, H, d_k), dtype=f32, device=dev),
             da=torch.empty((T, H, d_k), dtype=f32, device=dev), dv=torch.empty((T, H, d_v), dtype=f32, device=dev),
             dbeta=torch.empty((T, H), dtype=f32, device=dev), dA_log=torch.empty((H,), dtype=f32, device=dev),
             dgate=None if gate is None else torch.empty((T, H, d_v), dtype=f32, device=dev),
             dinitial_state=None if initial_state is None else torch.empty((N, H, d_k, d_v), dtype=f32, device=dev))
    need = (kda_chunk_bwd_chunkwise_workspace_size if chunkwise else kda_chunk_bwd_workspace_size)(T, N, H, d_k, d_v)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    fn = lib.kda_chunk_bwd_chunkwise if chunkwise else lib.kda_chunk_bwd
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(beta), _ptr(gate), _ptr(A_log),
                           _ptr(cu_seqlens), N, T, H, d_k, d_v, float(scale), _ptr(initial_state), _ptr(dout),
                           _ptr(dfinal_state), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["da"]),
                           _ptr(g["dbeta"]), _ptr(g["dgate"]), _ptr(g["dA_log"]), _ptr(g["dinitial_state"]),
                           _ptr(workspace), workspace.numel() * workspace.element_size(), _stream_handle(stream, dev))
    _check(st, "kda_chunk_bwd_chunkwise" if chunkwise else "kda_chunk_bwd")
    return g


class _ChunkKDA(torch.autograd.Function):
    """kda_chunk_fwd forward, kda_chunk_bwd backward (both through the C ABI); the gradients come
    back in fp32 and are cast to each input's dtype."""

    @staticmethod
    def forward(ctx, q, k, v, a, beta, A_log, gate, initial_state, cu_seqlens, scale, out_dtype):
        out, S = kda_chunk_fwd(q, k, v, a, beta, A_log, cu_seqlens, gate=gate, initial_state=initial_state,
                               scale=scale, out_dtype=out_dtype)
        ctx.save_for_backward(q, k, v, a, beta, A_log, gate, initial_state, cu_seqlens)
        ctx.scale = scale
        return out, S

    @staticmethod
    def backward(ctx, dout, dS):
        q, k, v, a, beta, A_log, gate, initial_state, cu_seqlens = ctx.saved_tensors
        if dout is None:
            dout = torch.zeros((q.shape[0], q.shape[1], v.shape[-1]), dtype=torch.float32, device=q.device)
        g = kda_chunk_bwd(q, k, v, a, beta, A_log, cu_seqlens, dout.to(torch.float32).contiguous(), gate=gate,
                          initial_state=initial_state, dfinal_state=None if dS is None else dS.contiguous(),
                          scale=ctx.scale)
        like = lambda x, ref: None if x is None or ref is None else x.to(ref.dtype)
        return (like(g["dq"], q), like(g["dk"], k), like(g["dv"], v), like(g["da"], a), g["dbeta"], g["dA_log"],
                like(g["dgate"], gate), g["dinitial_state"], None, None, None)


def chunk_kda(q, k, v, a, beta, A_log, cu_seqlens, gate=None, initial_state=None, scale: float = 1.0,
              out_dtype=torch.bfloat16):
    """The prefill (kda_chunk_fwd) as a differentiable function of q, k, v, a, beta, A_log, gate and
    initial_state.  Returns (out [T, H, d_v], final_state [N, H, d_k, d_v] fp32); a loss on either
    or both reaches the inputs through kda_chunk_bwd."""
    return _ChunkKDA.apply(q, k, v, a, beta, A_log, gate, initial_state, cu_seqlens, float(scale), out_dtype)


def kda_launch_count() -> int:
    """Kernels launched through libkda by this process so far."""
    return int(lib.kda_launch_count())


def kda_set_prefill_path(path: int) -> None:
    """Which prefill kernel kda_chunk_fwd runs for d_k = d_v = 128: 0 chosen from the shapes,
    1 the cluster kernel (chunk records in the workspace), 2 one CTA per (sequence, head)."""
    _check(lib.kda_set_prefill_path(int(path)), "kda_set_prefill_path")


def kda_prefill_path(num_units: int, d_k: int, d_v: int) -> int:
    """The kernel kda_chunk_fwd would run now for num_units units: 1 (cluster) or 2 (per unit)."""
    return int(lib.kda_prefill_path(int(num_units), int(d_k), int(d_v)))


def kda_inject_stall(enable: bool, wait_limit_ns: int = 0) -> None:
    """Failure injection for tests: while enabled, prefill launches withhold chunk 0 and every
    device-side wait gives up after wait_limit_ns (the next kda_sync_check raises a timeout)."""
    _check(lib.kda_inject_stall(1 if enable else 0, int(wait_limit_ns)), "kda_inject_stall")


def kda_sync_check(stream=None, device=None) -> None:
    """Synchronise the stream and raise KDAError if a kernel recorded a device-side error."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    _check(lib.kda_sync_check(_stream_handle(stream, dev)), "kda_sync_check")
