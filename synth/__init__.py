"""Seeded synthetic inputs for the KDA forward pass.

Shared by the tests, the benchmark and the smoke check; holds none of the
method's arithmetic (no recurrence, no decay products, no chunk algebra).  It
draws the tensors that the KDA layers of the Kimi K3 model would feed the
recurrence: per-token L2-normalised q and k (the digest's KDA section says
the model normalises them), Gaussian v, a log-decay g squashed into a
bounded range, a write strength beta in (0, 1) and an optional Gaussian
initial state.

Recipe (one ``torch.Generator`` seeded with ``seed`` on the target device;
tensors drawn in this order, each in token slabs of ``SLAB`` tokens):
  q, k ~ N(0,1) in fp32, then divided by their per-token, per-head L2 norm;
  v ~ N(0,1);
  g = -g_scale * sigmoid(z),  z ~ N(0,1)   (g_scale = 5/64, or 5 for stress);
  beta = sigmoid(N(0,1));
  init_state ~ N(0, 0.01), i.e. standard deviation 0.1 (variance 0.01).
q, k, v are then cast to the requested I/O dtype; g, beta and states stay fp32.
Packed variable-length batches draw sequence lengths log-uniformly from
``numpy.random.default_rng(seed)`` until the running total reaches the
target, truncating the last length so the total is exact.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

SLAB = 1 << 16  # tokens drawn per randn call (bounds temporary memory)


@dataclasses.dataclass(frozen=True)
class PrefillSpec:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: torch.dtype
    seed: int
    g_scale: float = 5.0 / 64.0
    init: bool = False
    varlen: tuple | None = None  # (total_tokens, min_len, max_len)


@dataclasses.dataclass(frozen=True)
class DecodeSpec:
    name: str
    B: int
    H: int
    dk: int
    dv: int
    dtype: torch.dtype
    seed: int
    steps: int
    g_scale: float = 5.0 / 64.0


# The workloads: a tiny fp32 case, a mid prefill, the model-shaped 64K
# pretraining prefill (H=96 heads of 128x128 state), a packed 1M-token
# variable-length batch, the B=512 decode, and a model-range decay stress case.
TINY = PrefillSpec("tiny_fp32_B1_H2_T64_d16", 1, 64, 2, 16, 16, torch.float32, 0)
MID = PrefillSpec("mid_bf16_B2_H16_T4096_d128", 2, 4096, 16, 128, 128, torch.bfloat16, 1, init=True)
PRETRAIN = PrefillSpec("prefill_bf16_B1_H96_T65536_d128", 1, 65536, 96, 128, 128, torch.bfloat16, 2)
VARLEN = PrefillSpec("varlen_bf16_H32_T1048576_d128", 1, 1 << 20, 32, 128, 128, torch.bfloat16, 3,
                     init=True, varlen=(1 << 20, 1024, 262144))
STRESS = PrefillSpec("stress_bf16_B2_H16_T1024_d128_gmin5", 2, 1024, 16, 128, 128, torch.bfloat16, 5,
                     g_scale=5.0, init=True)
DECODE = DecodeSpec("decode_bf16_B512_H96_d128", 512, 96, 128, 128, torch.bfloat16, 4, 256)
# One tensor-parallel rank's share of the 64K prefill: 4 of the model's 96 heads
# (24-way head split), the case where the chains are far fewer than the SMs.
TP4 = PrefillSpec("tp4_bf16_B1_H4_T65536_d128", 1, 65536, 4, 128, 128, torch.bfloat16, 6)

# The 64K prefill with decays in the model's whole range (g = -5 sigmoid(z)):
# every chunk takes the bounded-decay (general) path.
PRETRAIN_MODEL_RANGE = PrefillSpec("prefill_bf16_B1_H96_T65536_d128_gmin5", 1, 65536, 96, 128, 128, torch.bfloat16, 7,
                                   g_scale=5.0)

PREFILL_SPECS = {s.name: s for s in (TINY, MID, PRETRAIN, VARLEN, STRESS, TP4, PRETRAIN_MODEL_RANGE)}


def varlen_lengths(total: int, lo: int, hi: int, seed: int) -> list[int]:
    rng = np.random.default_rng(seed)
    out, acc = [], 0
    while acc < total:
        L = int(math.floor(math.exp(rng.uniform(math.log(lo), math.log(hi)))))
        L = min(L, total - acc)
        out.append(L)
        acc += L
    return out


def _randn(gen, shape, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _slabbed(gen, T, rest, device, fn):
    """Draw a [T, *rest] tensor slab by slab, applying fn to each fp32 slab."""
    if T == 0:
        return fn(_randn(gen, (0,) + tuple(rest), device))
    parts = []
    for t0 in range(0, T, SLAB):
        parts.append(fn(_randn(gen, (min(SLAB, T - t0),) + tuple(rest), device)))
    return torch.cat(parts, 0) if len(parts) > 1 else parts[0]


def _unit_rows(x):
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def draw_tokens(gen, T, H, dk, dv, io_dtype, g_scale, device):
    """q, k, v, g, beta for T tokens (token-major [T,H,*])."""
    q = _slabbed(gen, T, (H, dk), device, lambda x: _unit_rows(x).to(io_dtype))
    k = _slabbed(gen, T, (H, dk), device, lambda x: _unit_rows(x).to(io_dtype))
    v = _slabbed(gen, T, (H, dv), device, lambda x: x.to(io_dtype))
    g = _slabbed(gen, T, (H, dk), device, lambda x: torch.sigmoid(x).mul_(-g_scale))
    beta = _slabbed(gen, T, (H,), device, torch.sigmoid)
    return q, k, v, g, beta


def make_prefill(spec: PrefillSpec, device="cpu", T: int | None = None, B: int | None = None,
                 H: int | None = None, lengths: list[int] | None = None):
    """Inputs for one prefill call.  T/B/H/lengths override the spec's sizes
    (parity tests use shortened versions of the big workloads)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(spec.seed)
    H = H or spec.H
    if spec.varlen is not None or lengths is not None:
        if lengths is None:
            total, lo, hi = spec.varlen
            lengths = varlen_lengths(T or total, lo, hi, spec.seed)
        Ttot = int(sum(lengths))
        q, k, v, g, beta = draw_tokens(gen, Ttot, H, spec.dk, spec.dv, spec.dtype, spec.g_scale, device)
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device=device)
        N, Bx, Tx = len(lengths), 1, Ttot
    else:
        B = B or spec.B
        T = T if T is not None else spec.T
        q, k, v, g, beta = draw_tokens(gen, B * T, H, spec.dk, spec.dv, spec.dtype, spec.g_scale, device)
        cu, N, Bx, Tx = None, B, B, T
    init = None
    if spec.init:
        init = (_randn(gen, (N, H, spec.dk, spec.dv), device) * 0.1).contiguous()
    shp = lambda x, d: x.reshape(Bx, Tx, H, d) if d else x.reshape(Bx, Tx, H)
    return dict(q=shp(q, spec.dk), k=shp(k, spec.dk), v=shp(v, spec.dv), g=shp(g, spec.dk),
                beta=shp(beta, 0), init_state=init, cu_seqlens=cu)


def make_decode_state(spec: DecodeSpec, device="cpu", B: int | None = None, H: int | None = None):
    gen = torch.Generator(device=device)
    gen.manual_seed(spec.seed)
    B, H = B or spec.B, H or spec.H
    return (_randn(gen, (B, H, spec.dk, spec.dv), device) * 0.1).contiguous()


def make_decode_step(spec: DecodeSpec, step: int, device="cpu", B: int | None = None,
                     H: int | None = None):
    """Per-step decode inputs, shaped [B,H,*]: one token per sequence."""
    gen = torch.Generator(device=device)
    gen.manual_seed(spec.seed * 1_000_003 + 1 + step)
    B, H = B or spec.B, H or spec.H
    q, k, v, g, beta = draw_tokens(gen, B, H, spec.dk, spec.dv, spec.dtype, spec.g_scale, device)
    return dict(q=q, k=k, v=v, g=g, beta=beta)


# -- raw inputs of the model's prologue (for the fused-prologue entry points) --
def draw_prologue_tokens(gen, T, H, dk, dv, io_dtype, z_shift, device):
    """Unnormalised q, k ~ N(0,1) (scaled per token by a factor in [0.5, 2) so
    the normalisation matters), v ~ N(0,1), decay logits z ~ N(z_shift, 1) in
    the I/O dtype, beta = sigmoid(N(0,1)); all token-major [T,H,*]."""
    def scaled(x):
        s = torch.rand(x.shape[:-1] + (1,), generator=gen, device=device) * 1.5 + 0.5
        return (x * s).to(io_dtype)
    q = _slabbed(gen, T, (H, dk), device, scaled)
    k = _slabbed(gen, T, (H, dk), device, scaled)
    v = _slabbed(gen, T, (H, dv), device, lambda x: x.to(io_dtype))
    z = _slabbed(gen, T, (H, dk), device, lambda x: (x + z_shift).to(io_dtype))
    beta = _slabbed(gen, T, (H,), device, torch.sigmoid)
    return q, k, v, z, beta


def make_prologue_prefill(spec: PrefillSpec, device="cpu", T: int | None = None, B: int | None = None,
                          H: int | None = None, lengths: list[int] | None = None, z_shift: float = -5.0,
                          a_std: float = 0.5):
    """Raw prologue inputs for one prefill call: q, k, v, z (decay logits), beta,
    A_log [H] ~ N(0, a_std^2), init_state, cu_seqlens.  With A_log = 0
    (a_std = 0), z_shift = -5 gives per-token log-decays g = -5 sigmoid(z) of
    about -0.01 to -0.09 (the mild regime of the benchmark generators); a
    spread of A_log moves some heads into strong decay; z_shift = 0 gives the
    model's full range down to -5."""
    gen = torch.Generator(device=device)
    gen.manual_seed(spec.seed + 1000)
    H = H or spec.H
    if lengths is not None or spec.varlen is not None:
        if lengths is None:
            total, lo, hi = spec.varlen
            lengths = varlen_lengths(T or total, lo, hi, spec.seed)
        Ttot = int(sum(lengths))
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device=device)
        N, Bx, Tx = len(lengths), 1, Ttot
    else:
        B = B or spec.B
        T = T if T is not None else spec.T
        cu, N, Bx, Tx, Ttot = None, B, B, T, B * T
    q, k, v, z, beta = draw_prologue_tokens(gen, Ttot, H, spec.dk, spec.dv, spec.dtype, z_shift, device)
    A_log = (_randn(gen, (H,), device) * a_std).contiguous()
    init = (_randn(gen, (N, H, spec.dk, spec.dv), device) * 0.1).contiguous() if spec.init else None
    shp = lambda x, d: x.reshape(Bx, Tx, H, d) if d else x.reshape(Bx, Tx, H)
    return dict(q=shp(q, spec.dk), k=shp(k, spec.dk), v=shp(v, spec.dv), z=shp(z, spec.dk), beta=shp(beta, 0),
                A_log=A_log, init_state=init, cu_seqlens=cu)


def make_spec_window(spec: DecodeSpec, step: int, W: int, device="cpu", B: int | None = None,
                     H: int | None = None, prologue: bool = False, z_shift: float = -5.0):
    """One window of W tokens per sequence for speculative decoding, shaped
    [B, W, H, *]: q, k, v, g (log-decay) and beta, or with ``prologue`` the
    raw q, k and the decay logits z (as key "g") of the prologue."""
    gen = torch.Generator(device=device)
    gen.manual_seed(spec.seed * 1_000_003 + 7919 * (step + 1) + W)
    B, H = B or spec.B, H or spec.H
    if prologue:
        q, k, v, g, beta = draw_prologue_tokens(gen, B * W, H, spec.dk, spec.dv, spec.dtype, z_shift, device)
    else:
        q, k, v, g, beta = draw_tokens(gen, B * W, H, spec.dk, spec.dv, spec.dtype, spec.g_scale, device)
    r = lambda x: x.reshape((B, W) + tuple(x.shape[1:])).contiguous()
    return dict(q=r(q), k=r(k), v=r(v), g=r(g), beta=r(beta))
