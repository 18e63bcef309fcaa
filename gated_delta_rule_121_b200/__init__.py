"""Python binding of libkda.so, the B200 (sm_100a) KDA forward library.

Argument marshalling only: every step of the forward pass runs in the CUDA
kernels behind the C ABI (include/kda.h).  PyTorch supplies device memory
and streams.  There is no CPU fallback: if the shared library cannot be
loaded, every call raises.

Functions mirror the C entry points:
  kda_fwd(q, k, v, log_alpha, beta, ...)        chunked prefill
  kda_fwd_noalloc(...)                           the same, scratch in a fixed library array
  kda_fwd_checkpoints(..., interval)             prefill plus the state every `interval` tokens
  kda_segment_fwd(...)                           zero-start outputs/state and transition of segments
  kda_state_compose(...), kda_output_correct(...)   prefix composition, output correction
  kda_fwd_cp(..., n_seg)                         prefill with every sequence split over the SMs
  kda_decode_step(q, k, v, log_alpha, beta, state, ...)   in-place decode
  kda_decode_step_gated(q, k, v, z, A_log, beta, state, ...)   the same with the input prologue
  kda_decode_spec(prev, n_accepted, cur, state, ...)   speculative verification with state replay
  kda_fwd_workspace_size(...), kda_workspace_status(ws), kda_status_string(s)
and ``kda_fwd_host`` runs kda_fwd on host (pinned) tensors through the C
entry point of the same name, which copies inputs in and outputs back on the
given stream.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkda.so")

(KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_WORKSPACE, KDA_ERR_CUDA, KDA_ERR_TIMEOUT,
 KDA_ERR_RANGE) = range(7)
KDA_F32, KDA_BF16 = 0, 1
_DT = {torch.float32: KDA_F32, torch.bfloat16: KDA_BF16}

_lib = None
_vp, _fp, _i32p = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p


class KdaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {kda_status_string(code)}")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libkda.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m gated_delta_rule_121_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.kda_version.restype = ctypes.c_int
        L.kda_status_string.restype = ctypes.c_char_p
        L.kda_status_string.argtypes = [ctypes.c_int]
        L.kda_fwd_workspace_size.restype = ctypes.c_size_t
        L.kda_fwd_workspace_size.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int]
        fwd_args = [_vp, _vp, _vp, _fp, _fp, _fp, _vp, _fp, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                    ctypes.c_int, ctypes.c_int, _i32p, _vp, ctypes.c_int, _vp, ctypes.c_size_t]
        L.kda_fwd.restype = ctypes.c_int
        L.kda_fwd.argtypes = fwd_args
        L.kda_testing_fwd.restype = ctypes.c_int
        L.kda_testing_fwd.argtypes = fwd_args + [_fp, ctypes.c_uint64, ctypes.c_int]
        L.kda_testing_debug_floats.restype = ctypes.c_int
        L.kda_testing_fwd_path.restype = ctypes.c_int
        L.kda_testing_fwd_path.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.kda_fwd_noalloc.restype = ctypes.c_int
        L.kda_fwd_noalloc.argtypes = fwd_args[:-2]
        L.kda_fwd_noalloc_status.restype = ctypes.c_int
        L.kda_fwd_noalloc_status.argtypes = [_vp]
        L.kda_decode_step.restype = ctypes.c_int
        L.kda_decode_step.argtypes = [_vp, _vp, _vp, _fp, _fp, _fp, _vp, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_int, _vp, ctypes.c_int]
        L.kda_fwd_host.restype = ctypes.c_int
        L.kda_fwd_host.argtypes = [_vp, _vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   _vp, ctypes.c_int, _vp, ctypes.c_size_t]
        L.kda_fwd_checkpoints_workspace_size.restype = ctypes.c_size_t
        L.kda_fwd_checkpoints_workspace_size.argtypes = L.kda_fwd_workspace_size.argtypes
        L.kda_fwd_checkpoints.restype = ctypes.c_int
        L.kda_fwd_checkpoints.argtypes = fwd_args[:-2] + [_fp, ctypes.c_int, ctypes.c_int64, _vp, ctypes.c_size_t]
        L.kda_segment_fwd.restype = ctypes.c_int
        L.kda_segment_fwd.argtypes = [_vp, _vp, _vp, _fp, _fp, _fp, _fp, _fp, _fp, ctypes.c_int, ctypes.c_int64,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32p, _vp, ctypes.c_int, _vp,
                                      ctypes.c_size_t]
        L.kda_state_compose.restype = ctypes.c_int
        L.kda_state_compose.argtypes = [_fp, _fp, _fp, _fp, _fp] + [ctypes.c_int] * 6 + [_vp]
        L.kda_output_correct.restype = ctypes.c_int
        L.kda_output_correct.argtypes = [_fp, _fp, _fp, _vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, _i32p, _vp, ctypes.c_int]
        L.kda_fwd_cp_workspace_size.restype = ctypes.c_size_t
        L.kda_fwd_cp_workspace_size.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.kda_cp_segments.restype = ctypes.c_int
        L.kda_cp_segments.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int]
        L.kda_fwd_cp.restype = ctypes.c_int
        L.kda_fwd_cp.argtypes = fwd_args[:-2] + [ctypes.c_int, _vp, ctypes.c_size_t]
        L.kda_fwd_gated.restype = ctypes.c_int
        L.kda_fwd_gated.argtypes = [_vp, _vp, _vp, _vp, _fp, ctypes.c_float] + fwd_args[4:]
        L.kda_decode_step_gated.restype = ctypes.c_int
        L.kda_decode_step_gated.argtypes = [_vp, _vp, _vp, _vp, _fp, ctypes.c_float, _fp, _fp, _vp, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, ctypes.c_int]
        spec = [_vp] * 5 + [_i32p] + [_vp] * 5
        tail = [_fp, _vp] + [ctypes.c_int] * 6 + [_vp, ctypes.c_int]
        L.kda_decode_spec.restype = ctypes.c_int
        L.kda_decode_spec.argtypes = spec + tail
        L.kda_decode_spec_gated.restype = ctypes.c_int
        L.kda_decode_spec_gated.argtypes = spec + [_fp, ctypes.c_float] + tail
        L.kda_workspace_status.restype = ctypes.c_int
        L.kda_workspace_status.argtypes = [_vp, _vp]
        _lib = L
    return _lib


def kda_status_string(code: int) -> str:
    return lib().kda_status_string(int(code)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(code, what):
    if code != KDA_OK:
        raise KdaError(code, what)


def kda_fwd_workspace_size(B, T, H, dk, dv, dtype=torch.bfloat16) -> int:
    return int(lib().kda_fwd_workspace_size(B, T, H, dk, dv, _DT[dtype]))


def alloc_workspace(B, T, H, dk, dv, dtype=torch.bfloat16, device="cuda") -> torch.Tensor:
    n = kda_fwd_workspace_size(B, T, H, dk, dv, dtype)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def kda_workspace_status(workspace: torch.Tensor, stream=None) -> int:
    return int(lib().kda_workspace_status(_ptr(workspace), _stream_ptr(stream)))


def _shapes(q, v, cu_seqlens):
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, dk]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is not None:
        if B != 1:
            raise ValueError("packed (cu_seqlens) inputs must have batch dimension 1")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    return B, T, H, dk, dv, N


def kda_fwd(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, out=None, final_state=None,
            output_final_state=True, workspace=None, stream=None, _debug=None, _wait_ns=None, _inject_stuck=False):
    """KDA forward over whole sequences (see include/kda.h, kda_fwd).

    q, k, log_alpha: [B,T,H,dk]; v: [B,T,H,dv]; beta: [B,T,H]; q/k/v share a
    dtype (bf16 or fp32); log_alpha, beta and states are fp32.  Returns
    ``(out, final_state)``; final_state is None when not requested.
    """
    B, T, H, dk, dv, N = _shapes(q, v, cu_seqlens)
    dt = _DT[q.dtype]
    for name, t, dtype in (("k", k, q.dtype), ("v", v, q.dtype), ("log_alpha", log_alpha, torch.float32),
                           ("beta", beta, torch.float32)):
        if t.dtype != dtype or not t.is_contiguous() or t.device != q.device:
            raise ValueError(f"{name}: expected contiguous {dtype} on {q.device}")
    if init_state is not None and (init_state.dtype != torch.float32 or not init_state.is_contiguous()
                                   or tuple(init_state.shape) != (N, H, dk, dv)):
        raise ValueError("init_state must be contiguous fp32 [N, H, dk, dv]")
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(N, B * T, H, dk, dv, q.dtype, q.device)
    # packed: T is the total token count, the per-sequence length otherwise
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(init_state), _ptr(out),
            _ptr(final_state), N, T, H, dk, dv, _ptr(cu_seqlens), _stream_ptr(stream), dt,
            _ptr(workspace), workspace.numel())
    if _debug is None and _wait_ns is None and not _inject_stuck:
        code = lib().kda_fwd(*args)
    else:
        code = lib().kda_testing_fwd(*args, _ptr(_debug), int(_wait_ns if _wait_ns is not None else 2_000_000_000),
                                     int(bool(_inject_stuck)))
    _check(code, "kda_fwd")
    return out, final_state


def _check_inputs(q, k, v, log_alpha, beta, init_state, cu_seqlens, N, H, dk, dv):
    for name, t, dtype in (("k", k, q.dtype), ("v", v, q.dtype), ("log_alpha", log_alpha, torch.float32),
                           ("beta", beta, torch.float32)):
        if t.dtype != dtype or not t.is_contiguous() or t.device != q.device:
            raise ValueError(f"{name}: expected contiguous {dtype} on {q.device}")
    if init_state is not None and (init_state.dtype != torch.float32 or not init_state.is_contiguous()
                                   or tuple(init_state.shape) != (N, H, dk, dv)):
        raise ValueError("init_state must be contiguous fp32 [N, H, dk, dv]")
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")


def kda_fwd_checkpoints(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, interval=512, capacity=None,
                        out=None, final_state=None, checkpoints=None, workspace=None, stream=None):
    """kda_fwd plus the state after every whole multiple of ``interval`` tokens
    of each sequence (include/kda.h, kda_fwd_checkpoints).  ``capacity`` (the
    number of checkpoint slots) defaults to the exact count, which for packed
    batches is computed from ``cu_seqlens`` on the host (one small copy).
    Returns ``(out, final_state, checkpoints [capacity, H, dk, dv])``."""
    B, T, H, dk, dv, N = _shapes(q, v, cu_seqlens)
    _check_inputs(q, k, v, log_alpha, beta, init_state, cu_seqlens, N, H, dk, dv)
    if capacity is None:
        if cu_seqlens is None:
            capacity = N * (T // interval)
        else:
            lens = (cu_seqlens[1:] - cu_seqlens[:-1]).cpu()
            capacity = int((lens // interval).sum())
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    if checkpoints is None:
        checkpoints = torch.empty((max(capacity, 0), H, dk, dv), dtype=torch.float32, device=q.device)
    if workspace is None:
        n = int(lib().kda_fwd_checkpoints_workspace_size(N, B * T, H, dk, dv, _DT[q.dtype]))
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    code = lib().kda_fwd_checkpoints(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(init_state),
                                     _ptr(out), _ptr(final_state), N, T, H, dk, dv, _ptr(cu_seqlens),
                                     _stream_ptr(stream), _DT[q.dtype], _ptr(checkpoints), int(interval),
                                     int(capacity), _ptr(workspace), workspace.numel())
    _check(code, "kda_fwd_checkpoints")
    return out, final_state, checkpoints


def kda_segment_fwd(q, k, v, log_alpha, beta, cu_seqlens=None, workspace=None, stream=None):
    """Pieces of every sequence taken as one segment (include/kda.h,
    kda_segment_fwd).  Returns ``(out_zero, state_zero, qhat, transition)``,
    all fp32: zero-start outputs [B,T,H,dv] and final states [N,H,dk,dv], and
    qhat [B,T,H,dk] with the segment transitions [N,H,dk,dk]."""
    B, T, H, dk, dv, N = _shapes(q, v, cu_seqlens)
    _check_inputs(q, k, v, log_alpha, beta, None, cu_seqlens, N, H, dk, dv)
    dev = q.device
    out_zero = torch.empty((B, T, H, dv), dtype=torch.float32, device=dev)
    qhat = torch.empty((B, T, H, dk), dtype=torch.float32, device=dev)
    state_zero = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    transition = torch.empty((N, H, dk, dk), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = alloc_workspace(N, B * T, H, dk, dv, q.dtype, dev)
    code = lib().kda_segment_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(out_zero),
                                 _ptr(state_zero), _ptr(qhat), _ptr(transition), N, T, H, dk, dv,
                                 _ptr(cu_seqlens), _stream_ptr(stream), _DT[q.dtype], _ptr(workspace),
                                 workspace.numel())
    _check(code, "kda_segment_fwd")
    return out_zero, state_zero, qhat, transition


def kda_state_compose(transition, state_zero, R, init_state=None, rank_major=False, state_in=None,
                      final_state=None, stream=None):
    """Incoming state of every piece and the final state of N sequences cut
    into R pieces (include/kda.h, kda_state_compose).  transition
    [R*N,H,dk,dk] and state_zero [R*N,H,dk,dv] fp32 on the device.  Returns
    ``(state_in [R*N,H,dk,dv], final_state [N,H,dk,dv])``."""
    P, H, dk, dv = state_zero.shape
    if P % R:
        raise ValueError("the piece count must be a multiple of R")
    N = P // R
    for t in (transition, state_zero, init_state):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous()):
            raise ValueError("states must be contiguous fp32")
    if state_in is None:
        state_in = torch.empty_like(state_zero)
    if final_state is None:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=state_zero.device)
    code = lib().kda_state_compose(_ptr(transition), _ptr(state_zero), _ptr(init_state), _ptr(state_in),
                                   _ptr(final_state), R, N, H, dk, dv, int(bool(rank_major)), _stream_ptr(stream))
    _check(code, "kda_state_compose")
    return state_in, final_state


def kda_output_correct(out_zero, qhat, state_in, cu_seqlens=None, dtype=torch.bfloat16, out=None, stream=None):
    """out_t = out_zero_t + S_in^T qhat_t with S_in = state_in[sequence of t]
    (include/kda.h, kda_output_correct).  Returns ``out`` in ``dtype``."""
    B, T, H, dv = out_zero.shape
    dk = qhat.shape[-1]
    N = cu_seqlens.numel() - 1 if cu_seqlens is not None else B
    if tuple(state_in.shape) != (N, H, dk, dv):
        raise ValueError("state_in must be [N, H, dk, dv]")
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=dtype, device=out_zero.device)
    code = lib().kda_output_correct(_ptr(out_zero), _ptr(qhat), _ptr(state_in), _ptr(out), N, T, H, dk, dv,
                                    _ptr(cu_seqlens), _stream_ptr(stream), _DT[out.dtype])
    _check(code, "kda_output_correct")
    return out


def kda_cp_segments(N, tokens_per_sequence, H, sm_count=None) -> int:
    """Segments per sequence suggested for kda_fwd_cp on this device."""
    if sm_count is None:
        sm_count = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return int(lib().kda_cp_segments(N, tokens_per_sequence, H, sm_count))


def kda_fwd_cp(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, n_seg=None, out=None,
               final_state=None, workspace=None, stream=None):
    """kda_fwd with every sequence split into ``n_seg`` segments that run on
    separate SMs (include/kda.h, kda_fwd_cp).  ``n_seg`` defaults to
    kda_cp_segments(...).  Returns ``(out, final_state)``."""
    B, T, H, dk, dv, N = _shapes(q, v, cu_seqlens)
    _check_inputs(q, k, v, log_alpha, beta, init_state, cu_seqlens, N, H, dk, dv)
    if n_seg is None:
        n_seg = kda_cp_segments(N, (B * T) // max(N, 1), H)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_cp_workspace(N, B * T, H, dk, dv, n_seg, q.dtype, q.device)
    code = lib().kda_fwd_cp(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(init_state), _ptr(out),
                            _ptr(final_state), N, T, H, dk, dv, _ptr(cu_seqlens), _stream_ptr(stream),
                            _DT[q.dtype], int(n_seg), _ptr(workspace), workspace.numel())
    _check(code, "kda_fwd_cp")
    return out, final_state


def alloc_cp_workspace(N, T_total, H, dk, dv, n_seg, dtype=torch.bfloat16, device="cuda"):
    n = int(lib().kda_fwd_cp_workspace_size(N, T_total, H, dk, dv, _DT[dtype], n_seg))
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def kda_fwd_noalloc(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, out=None, final_state=None,
                    stream=None):
    """kda_fwd without a caller workspace (see include/kda.h, kda_fwd_noalloc):
    the library's fixed device array serves as scratch, nothing is allocated
    by the library.  Returns ``(out, final_state)``."""
    B, T, H, dk, dv, N = _shapes(q, v, cu_seqlens)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    code = lib().kda_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(init_state),
                                 _ptr(out), _ptr(final_state), N, T, H, dk, dv, _ptr(cu_seqlens),
                                 _stream_ptr(stream), _DT[q.dtype])
    _check(code, "kda_fwd_noalloc")
    return out, final_state


def kda_fwd_noalloc_status(stream=None) -> int:
    """Device status of the last kda_fwd_noalloc call on the current device
    (synchronises the stream)."""
    return int(lib().kda_fwd_noalloc_status(_stream_ptr(stream)))


def kda_decode_step(q, k, v, log_alpha, beta, state, out=None, stream=None):
    """One decode step; ``state`` [B,H,dk,dv] fp32 is updated in place.
    q,k,log_alpha: [B,H,dk]; v: [B,H,dv]; beta: [B,H].  Returns out [B,H,dv]."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    if state.dtype != torch.float32 or not state.is_contiguous() or tuple(state.shape) != (B, H, dk, dv):
        raise ValueError("state must be contiguous fp32 [B, H, dk, dv]")
    for name, t in (("k", k), ("v", v), ("log_alpha", log_alpha), ("beta", beta)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    code = lib().kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(state), _ptr(out),
                                 B, H, dk, dv, _stream_ptr(stream), _DT[q.dtype])
    _check(code, "kda_decode_step")
    return out


class _FwdTensors(ctypes.Structure):
    """kda_fwd_tensors_t: the pointers of one kda_fwd call."""
    _fields_ = [(n, ctypes.c_void_p) for n in ("q", "k", "v", "log_alpha", "beta", "init_state", "cu_seqlens",
                                                 "out", "final_state")]


def _tensors(d):
    return _FwdTensors(*[None if d.get(n) is None else d[n].data_ptr() for n, _ in _FwdTensors._fields_])


G_MIN = -5.0  # the model's lower bound of the log decay


def kda_fwd_gated(q, k, v, z, A_log, beta, init_state=None, cu_seqlens=None, g_min=G_MIN, out=None,
                  final_state=None, workspace=None, stream=None):
    """kda_fwd on the model's raw prologue inputs (include/kda.h,
    kda_fwd_gated): q, k unnormalised [B,T,H,dk], z the decay logits (dtype of
    q), A_log [H] fp32.  Returns ``(out, final_state)``."""
    B, T, H, dk, dv, N = _shapes(q, v, cu_seqlens)
    for name, t, dtype in (("k", k, q.dtype), ("v", v, q.dtype), ("z", z, q.dtype), ("beta", beta, torch.float32)):
        if t.dtype != dtype or not t.is_contiguous() or t.device != q.device:
            raise ValueError(f"{name}: expected contiguous {dtype} on {q.device}")
    if tuple(z.shape) != tuple(q.shape):
        raise ValueError("z must be shaped like q")
    if init_state is not None and (init_state.dtype != torch.float32 or not init_state.is_contiguous()
                                   or tuple(init_state.shape) != (N, H, dk, dv)):
        raise ValueError("init_state must be contiguous fp32 [N, H, dk, dv]")
    if A_log.dtype != torch.float32 or tuple(A_log.shape) != (H,):
        raise ValueError("A_log must be fp32 [H]")
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(N, B * T, H, dk, dv, q.dtype, q.device)
    code = lib().kda_fwd_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(A_log), float(g_min), _ptr(beta),
                               _ptr(init_state), _ptr(out), _ptr(final_state), N, T, H, dk, dv, _ptr(cu_seqlens),
                               _stream_ptr(stream), _DT[q.dtype], _ptr(workspace), workspace.numel())
    _check(code, "kda_fwd_gated")
    return out, final_state


def kda_decode_step_gated(q, k, v, z, A_log, beta, state, g_min=G_MIN, out=None, stream=None):
    """One decode step on raw prologue inputs (include/kda.h,
    kda_decode_step_gated): q, k unnormalised, z the decay logits [B,H,dk]
    (dtype of q), A_log [H] fp32.  ``state`` is updated in place."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    if state.dtype != torch.float32 or not state.is_contiguous() or tuple(state.shape) != (B, H, dk, dv):
        raise ValueError("state must be contiguous fp32 [B, H, dk, dv]")
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    code = lib().kda_decode_step_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(A_log), float(g_min), _ptr(beta),
                                       _ptr(state), _ptr(out), B, H, dk, dv, _stream_ptr(stream), _DT[q.dtype])
    _check(code, "kda_decode_step_gated")
    return out


def kda_decode_spec(prev, n_accepted, cur, state, A_log=None, g_min=G_MIN, out=None, stream=None):
    """Speculative verification with state replay (include/kda.h,
    kda_decode_spec): ``prev`` (or None) and ``cur`` are dicts of q, k, v, g,
    beta shaped [B, W, H, *] (g = the log-decay, or the decay logits when
    ``A_log`` is given: the gated variant, q and k then unnormalised);
    ``n_accepted`` int32 [B] on the device.  ``state`` [B,H,dk,dv] is updated
    to the state after the accepted drafts and the bonus token cur[:, 0].
    Returns the outputs of ``cur`` [B, W, H, dv]."""
    B, W, H, dk = cur["q"].shape
    dv = cur["v"].shape[-1]
    Wp = 0 if prev is None else prev["q"].shape[1]
    if state.dtype != torch.float32 or not state.is_contiguous() or tuple(state.shape) != (B, H, dk, dv):
        raise ValueError("state must be contiguous fp32 [B, H, dk, dv]")
    for src in (prev, cur):
        if src is not None:
            for n in ("q", "k", "v", "g", "beta"):
                if not src[n].is_contiguous():
                    raise ValueError(f"{n} must be contiguous")
    if out is None:
        out = torch.empty((B, W, H, dv), dtype=cur["q"].dtype, device=cur["q"].device)
    p = (lambda n: None) if prev is None else (lambda n: _ptr(prev[n]))
    head = [p("q"), p("k"), p("v"), p("g"), p("beta"), _ptr(n_accepted) if Wp else None,
            _ptr(cur["q"]), _ptr(cur["k"]), _ptr(cur["v"]), _ptr(cur["g"]), _ptr(cur["beta"])]
    tail = [_ptr(state), _ptr(out), B, Wp, W, H, dk, dv, _stream_ptr(stream), _DT[cur["q"].dtype]]
    if A_log is None:
        code = lib().kda_decode_spec(*head, *tail)
    else:
        code = lib().kda_decode_spec_gated(*head, _ptr(A_log), float(g_min), *tail)
    _check(code, "kda_decode_spec")
    return out


def kda_fwd_host(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, device="cuda", stream=None,
                 dev_buffers=None, output_final_state=True):
    """kda_fwd on host tensors through the C entry point kda_fwd_host: one call
    enqueues the host-to-device copies of the inputs (pinned memory makes them
    asynchronous), the forward, and the copies of ``out`` and the final state
    back.  ``dev_buffers`` (a dict returned by a previous call) holds the
    device buffers and the pinned host outputs for repeated calls.  Returns
    (out_host, final_host, dev_buffers) (final_host None without
    ``output_final_state``); synchronise the stream before reading the host
    outputs."""
    s = stream if stream is not None else torch.cuda.current_stream(device)
    B, T, H, dk, dv, N = _shapes(q, v, cu_seqlens)
    host_in = dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, init_state=init_state, cu_seqlens=cu_seqlens)
    if dev_buffers is None:
        dev_buffers = {}
    if dev_buffers.get("_shape") != (B, T, H, dk, dv, N, q.dtype):
        dev_buffers.clear()
        dev_buffers["_shape"] = (B, T, H, dk, dv, N, q.dtype)
        dev = {n: (None if t is None else torch.empty(t.shape, dtype=t.dtype, device=device))
               for n, t in host_in.items()}
        dev["out"] = torch.empty((B, T, H, dv), dtype=q.dtype, device=device)
        dev["final_state"] = torch.empty((N, H, dk, dv), dtype=torch.float32, device=device)
        dev_buffers["dev"] = dev
        dev_buffers["ws"] = alloc_workspace(N, B * T, H, dk, dv, q.dtype, device)
        dev_buffers["out_h"] = torch.empty((B, T, H, dv), dtype=q.dtype, pin_memory=True)
        dev_buffers["fin_h"] = torch.empty((N, H, dk, dv), dtype=torch.float32, pin_memory=True)
    fin_h = dev_buffers["fin_h"] if output_final_state else None
    host = dict(host_in, out=dev_buffers["out_h"], final_state=fin_h)
    dev = dict(dev_buffers["dev"]) if output_final_state else dict(dev_buffers["dev"], final_state=None)
    for n, t in host_in.items():
        if t is not None and (t.device.type != "cpu" or not t.is_contiguous()):
            raise ValueError(f"{n}: expected a contiguous host tensor")
    ws = dev_buffers["ws"]
    code = lib().kda_fwd_host(ctypes.byref(_tensors(host)), ctypes.byref(_tensors(dev)), N, T, H,
                              dk, dv, ctypes.c_void_p(s.cuda_stream), _DT[q.dtype], _ptr(ws), ws.numel())
    _check(code, "kda_fwd_host")
    return dev_buffers["out_h"], fin_h, dev_buffers
