"""fp64 CPU oracle for the KDA forward pass.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The CUDA library never
imports, links or calls anything here, and nothing here imports the library.

The arithmetic lives in ``kda_oracle.c`` (plain C, fp64, token-by-token
recurrence).  It follows the Kimi K3 technical-report digest
(discuss.pytorch.kr), section "Kimi Delta Attention: delta rule with a
per-channel forget gate", state-update equation
``S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T``,
``o_t = S_t^T q_t``, with ``alpha_t = exp(g_t)`` from the "Bounded decay"
section.  This module only marshals arrays: it converts inputs to fp64
exactly (bf16 and fp32 values are representable in fp64) and calls C.

Every function is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile the C oracle in place (gcc, -O3, portable x86-64 code)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O3", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.kda_oracle_fwd.restype = ctypes.c_int
        lib.kda_oracle_fwd.argtypes = [_dp] * 8 + [ctypes.c_int, _i64p] + [ctypes.c_int] * 4
        lib.kda_oracle_decode_step.restype = None
        lib.kda_oracle_decode_step.argtypes = [_dp] * 7 + [ctypes.c_int] * 4
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor: exact widening on the host
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def default_threads() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


def fwd(q, k, v, g, beta, init_state=None, cu_seqlens=None, nthreads: int | None = None,
        want_out: bool = True):
    """Token-by-token fp64 KDA forward.

    Shapes follow the library's layout: q,k,g ``[B,T,H,dk]``, v ``[B,T,H,dv]``,
    beta ``[B,T,H]``, init_state ``[N,H,dk,dv]`` or None (zeros).  With
    ``cu_seqlens`` (N+1 offsets) the tensors are packed ``[1,T_total,H,*]``
    and each sequence starts from its own ``init_state[n]``.

    Returns ``(out [B,T,H,dv], final_state [N,H,dk,dv])`` as float64 arrays.
    """
    lib = _load()
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        offsets = np.arange(B + 1, dtype=np.int64) * T
    else:
        offsets = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
        assert B == 1, "packed inputs have batch dimension 1"
    N = len(offsets) - 1
    init = None if init_state is None else _f64(init_state)
    out = np.zeros((B, T, H, dv), np.float64) if want_out else None
    fin = np.zeros((N, H, dk, dv), np.float64)
    lib.kda_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(init), _ptr(out),
                       _ptr(fin), N, offsets.ctypes.data_as(_i64p), H, dk, dv,
                       int(nthreads or default_threads()))
    return out, fin


def decode_step(q, k, v, g, beta, state):
    """One in-place decode step on an fp64 state ``[B,H,dk,dv]`` (modified).

    q,k,g ``[B,H,dk]``, v ``[B,H,dv]``, beta ``[B,H]``.  Returns out ``[B,H,dv]``.
    """
    lib = _load()
    assert state.dtype == np.float64 and state.flags.c_contiguous
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    B, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((B, H, dv), np.float64)
    lib.kda_oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state),
                               _ptr(out), B, H, dk, dv)
    return out


def transition(q, k, g, beta, cu_seqlens=None, nthreads: int | None = None):
    """Segment transition of every (sequence, head) and the transformed queries.

    The KCP paragraph of the digest's co-design section writes the recurrence
    as ``S_t = M_t S_{t-1} + beta_t k_t v_t^T`` with
    ``M_t = (I - beta_t k_t k_t^T) Diag(alpha_t)``; the transition of a
    segment is ``M = M_last ... M_first``.  With every value zero the
    recurrence is ``S_t = M_t S_{t-1}``, so starting from ``S_0 = I`` it gives
    ``S_t = M_t ... M_first`` and reads ``o_t = S_t^T q_t``.  Returns
    ``(qhat [B,T,H,dk], M [N,H,dk,dk])`` as float64 arrays, where qhat_t is
    that read: the transition through token t applied to q_t.
    """
    q64 = _f64(q)
    B, T, H, dk = q64.shape
    N = B if cu_seqlens is None else (len(cu_seqlens) - 1 if not hasattr(cu_seqlens, "numel")
                                       else cu_seqlens.numel() - 1)
    zeros_v = np.zeros((B, T, H, dk), np.float64)
    eye = np.broadcast_to(np.eye(dk), (N, H, dk, dk)).copy()
    return fwd(q64, k, zeros_v, g, beta, eye, cu_seqlens, nthreads=nthreads)


# -- the model's input prologue (digest: "Kimi Delta Attention" section, q and
#    k L2-normalised, decay logits with a per-head bias/scale; "Bounded decay"
#    section, g = g_min * sigmoid(exp(A_h) * z) with g_min = -5) ---------------
G_MIN = -5.0
L2NORM_EPS = 1e-6


def gate(z, A_log, g_min=G_MIN):
    """Log-decay from decay logits z [..., H, dk] and per-head log scales A_log
    [H]: g = g_min * sigmoid(exp(A_h) * z), in fp64."""
    z = _f64(z)
    a = np.exp(_f64(A_log))[:, None]          # [H, 1], broadcast over the key channels
    return g_min / (1.0 + np.exp(-a * z))


def l2norm(x, eps=L2NORM_EPS):
    """x / sqrt(|x|^2 + eps) over the last axis, in fp64."""
    x = _f64(x)
    return x / np.sqrt((x * x).sum(-1, keepdims=True) + eps)


def fwd_gated(q, k, v, z, A_log, beta, init_state=None, cu_seqlens=None, g_min=G_MIN, nthreads=None):
    """The forward with the prologue: normalise q and k, map z to g, then the
    token-by-token recurrence (``fwd``)."""
    return fwd(l2norm(q), l2norm(k), v, gate(z, A_log, g_min), beta, init_state, cu_seqlens, nthreads=nthreads)


def decode_step_gated(q, k, v, z, A_log, beta, state, g_min=G_MIN):
    """``decode_step`` with the prologue applied to the token's raw inputs."""
    return decode_step(l2norm(q), l2norm(k), v, gate(z, A_log, g_min), beta, state)


def spec_decode(prev, n_accepted, cur, state):
    """Speculative-decode verification with state replay (digest, serving
    section, "speculative decoding and KDA state rewind"), as a plain loop of
    decode steps.  ``prev`` and ``cur`` are dicts of q, k, v, g, beta shaped
    [B, W, H, *] (``prev`` may be None when nothing was drafted);
    ``n_accepted`` [B].  For every sequence b: the first n_accepted[b] tokens
    of ``prev`` are applied to the state (no outputs), then every token of
    ``cur`` with its output; the state kept is the one after ``cur``'s first
    token (or after the replay when ``cur`` is empty).  ``state`` (fp64
    [B, H, dk, dv]) is updated in place to that kept state.  Returns the
    outputs [B, W, H, dv]."""
    B, W, H = cur["q"].shape[:3]
    dv = state.shape[-1]
    out = np.zeros((B, W, H, dv), np.float64)
    na = np.asarray(_f64(n_accepted)).astype(np.int64) if n_accepted is not None else np.zeros(B, np.int64)
    for b in range(B):
        S = np.ascontiguousarray(state[b:b + 1])
        one = lambda src, t: {n: _f64(src[n])[b:b + 1, t] for n in ("q", "k", "v", "g", "beta")}
        for t in range(int(na[b]) if prev is not None else 0):
            x = one(prev, t)
            decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S)
        keep = S.copy()
        for t in range(W):
            x = one(cur, t)
            out[b, t] = decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S)[0]
            if t == 0:
                keep = S.copy()
        state[b] = keep[0]
    return out
