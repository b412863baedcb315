"""Seeded synthetic inputs for the KDA hot path.

This module only draws random numbers with the shapes, distributions and
seeds of the workloads; it holds none of the method's arithmetic beyond the
stated sampling recipes.  Both the CUDA-path tests/benchmark and the oracle
tests take their inputs from here, and from nowhere else.

Workloads (d = dk = dv):

=========  ==================================================================
tiny       B=1, T=256, H=2, d=64, fp32.  q,k,v ~ N(0,1); z ~ N(0,1);
           A_h ~ U(-1,0); g = -5*sigmoid(exp(A_h) z); beta = sigmoid(N(0,1));
           S0 = 0.  Seed 0.
prefill    B=1, T=4096, H=16, d=128, bf16 q/k/v/g/beta, same distributions,
           S0 ~ N(0, 0.01) fp32 (0.01 read as the standard deviation).
sweep      B=1, H=96, d=128, T in {2048, 8192, 32768, 65536}, bf16, raw
           pre-conv q,k,v ~ N(0,1); conv weights ~ U(-0.5,0.5) [3, H*d, 4];
           z ~ N(0,1); A_h ~ U(-1,0); beta logits ~ N(0,1) fp32;
           S0 ~ N(0, 0.01).  Seed T.
decode     N=256 sequences, H=96, d=128, 64 steps.  S ~ N(0, 0.05) fp32;
           per step fresh q,k,v,z ~ N(0,1) bf16, g from z as above,
           beta = sigmoid(N(0,1)).  Seed 0 for S, 1+step for each step.
ckda       B=8, T=8192, H=32, d=128, bf16.  alpha = tanh(N(0,1)) with its
           magnitude clamped to >= exp(-5), sign kept; beta = 2*sigmoid(N(0,1));
           q,k,v ~ N(0,1); S0 ~ N(0, 0.01) (not stated by the workload; chosen
           so that the S0 path is exercised).  Seed 0.
softplus   any of the above with Kimi Linear's gate (``gate="softplus"``):
           g = -exp(A_h) softplus(z), z ~ N(0,1), A_h = log U(1,16) (the
           A_log initialisation printed on the Kimi K3 page); g is unbounded
           below (typically -0.7 x [1, 16], tail far below -5).
=========  ==================================================================

Tensors are drawn in fp32 on the CPU from one ``torch.Generator`` and then
cast to the run dtype; consumers widen the cast tensors, so input rounding is
never counted as error.
"""
from __future__ import annotations

import math

import torch

SWEEP_T = (2048, 8192, 32768, 65536)

WORKLOADS = {
    "tiny": dict(B=1, T=256, H=2, dk=64, dv=64, dtype=torch.float32, S0_std=0.0, seed=0),
    "prefill": dict(B=1, T=4096, H=16, dk=128, dv=128, dtype=torch.bfloat16, S0_std=0.01, seed=0),
    "ckda": dict(B=8, T=8192, H=32, dk=128, dv=128, dtype=torch.bfloat16, S0_std=0.01, seed=0),
}
DECODE = dict(N=256, H=96, dk=128, dv=128, steps=64, S_std=0.05, dtype=torch.bfloat16)
SWEEP = dict(B=1, H=96, dk=128, dv=128, dtype=torch.bfloat16, S0_std=0.01)

LOG_DECAY_FLOOR = -5.0


_DEVICE = "cpu"


def set_device(device: str) -> None:
    """Draw on another device (the benchmark draws its timing-only inputs on
    the GPU to save host time; every parity test draws on the CPU)."""
    global _DEVICE
    _DEVICE = device


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device=_DEVICE)
    g.manual_seed(int(seed))
    return g


def _randn(shape, gen):
    return torch.randn(shape, generator=gen, dtype=torch.float32, device=gen.device)


def _uniform(shape, lo, hi, gen):
    return torch.rand(shape, generator=gen, dtype=torch.float32, device=gen.device) * (hi - lo) + lo


def _sampled_log_decay(z, A):
    # the workloads' stated sampling recipe for g (pushforward of z and A_h)
    return LOG_DECAY_FLOOR * torch.sigmoid(torch.exp(A)[:, None] * z)


def _sampled_softplus_decay(z, A):
    # the softplus workloads' sampling recipe for g (pushforward of z and A_h)
    return -torch.exp(A)[:, None] * torch.nn.functional.softplus(z)


def _log_scale(H, gen, gate):
    # A_h ~ U(-1, 0) for the bounded gate; log U(1, 16) for Kimi Linear's softplus gate
    if gate == "softplus":
        return torch.log(_uniform((H,), 1.0, 16.0, gen))
    if gate != "bounded":
        raise ValueError(f"unknown gate {gate!r}")
    return _uniform((H,), -1.0, 0.0, gen)


def chunk_inputs(B, T, H, dk, dv, *, dtype=torch.bfloat16, S0_std=0.01, seed=0,
                 complex_gate=False, gate="bounded"):
    """Inputs of ``kda_chunk_fwd``: q, k, v, g, beta (run dtype), S0 (fp32 or None).

    Unsigned KDA: g is the log-decay in (-5, 0).  Complex-KDA: g holds the
    signed gate alpha in [-1, 1] with |alpha| >= exp(-5), beta in [0, 2].
    """
    gen = _gen(seed)
    q = _randn((B, T, H, dk), gen)
    k = _randn((B, T, H, dk), gen)
    v = _randn((B, T, H, dv), gen)
    if complex_gate:
        a = torch.tanh(_randn((B, T, H, dk), gen))
        sgn = torch.where(a < 0, -1.0, 1.0)
        g = sgn * torch.clamp(a.abs(), min=math.exp(LOG_DECAY_FLOOR))
        beta = 2.0 * torch.sigmoid(_randn((B, T, H), gen))
    else:
        z = _randn((B, T, H, dk), gen)
        A = _log_scale(H, gen, gate)
        g = _sampled_log_decay(z, A) if gate == "bounded" else _sampled_softplus_decay(z, A)
        beta = torch.sigmoid(_randn((B, T, H), gen))
    S0 = None
    if S0_std > 0:
        S0 = _randn((B, H, dk, dv), gen) * S0_std
    cast = lambda x: x.to(dtype).contiguous()
    if complex_gate:
        g = cast(g)
        # keep |alpha| >= exp(-5) after rounding to the run dtype
        floor = torch.tensor(math.exp(LOG_DECAY_FLOOR), dtype=dtype, device=g.device)
        g = torch.where(g.abs() < floor, torch.where(g < 0, -floor, floor), g).contiguous()
    else:
        g = cast(g)
    return dict(q=cast(q), k=cast(k), v=cast(v), g=g, beta=cast(beta), S0=S0)


def workload_inputs(name, **overrides):
    cfg = dict(WORKLOADS[name])
    cfg.update(overrides)
    return chunk_inputs(cfg["B"], cfg["T"], cfg["H"], cfg["dk"], cfg["dv"], dtype=cfg["dtype"],
                        S0_std=cfg["S0_std"], seed=cfg["seed"],
                        complex_gate=(name == "ckda") or overrides.get("complex_gate", False))


def prologue_inputs(B, T, H, dk, dv, *, dtype=torch.bfloat16, S0_std=0.01, seed=0,
                    gate="bounded"):
    """Raw inputs of ``kda_chunk_fwd_prologue`` (sweep recipe; ``gate`` picks A_h's law)."""
    gen = _gen(seed)
    q_pre = _randn((B, T, H, dk), gen)
    k_pre = _randn((B, T, H, dk), gen)
    v_pre = _randn((B, T, H, dv), gen)
    conv_w = _uniform((3, H * dk, 4), -0.5, 0.5, gen)
    z = _randn((B, T, H, dk), gen)
    A = _log_scale(H, gen, gate)
    b_logit = _randn((B, T, H), gen)
    S0 = _randn((B, H, dk, dv), gen) * S0_std if S0_std > 0 else None
    cast = lambda x: x.to(dtype).contiguous()
    return dict(q_pre=cast(q_pre), k_pre=cast(k_pre), v_pre=cast(v_pre), conv_w=cast(conv_w),
                z=cast(z), A=A.contiguous(), b_logit=b_logit.contiguous(), S0=S0)


def sweep_inputs(T, **kw):
    return prologue_inputs(SWEEP["B"], T, SWEEP["H"], SWEEP["dk"], SWEEP["dv"],
                           dtype=SWEEP["dtype"], S0_std=SWEEP["S0_std"], seed=kw.get("seed", T))


def decode_state(N, H, dk, dv, *, S_std=0.05, seed=0):
    return _randn((N, H, dk, dv), _gen(seed)) * S_std


def decode_log_scale(H, *, seed=0):
    """Per-head A_h ~ U(-1, 0) of the decode workload (fixed across steps)."""
    return _uniform((H,), -1.0, 0.0, _gen(10_000 + seed))


def decode_prologue_params(H, d, *, dtype=torch.bfloat16, seed=0):
    """Per-head parameters of the decode prologue: conv taps [3, H*d, 4] ~ U(-0.5, 0.5)
    (the sweep recipe) and A [H] ~ U(-1, 0) FP32."""
    gen = _gen(500 + seed)
    conv_w = _uniform((3, H * d, 4), -0.5, 0.5, gen).to(dtype).contiguous()
    A = _uniform((H,), -1.0, 0.0, gen).contiguous()
    return dict(conv_w=conv_w, A=A)


def decode_prologue_step_inputs(N, H, d, step, *, dtype=torch.bfloat16):
    """One decode token's raw prologue inputs: q_pre, k_pre, v_pre, z [N, H, d] ~ N(0,1) in
    the run dtype, beta logits [N, H] ~ N(0,1) FP32."""
    gen = _gen(700 + step)
    cast = lambda x: x.to(dtype).contiguous()
    q_pre, k_pre, v_pre, z = (cast(_randn((N, H, d), gen)) for _ in range(4))
    return dict(q_pre=q_pre, k_pre=k_pre, v_pre=v_pre, z=z, b_logit=_randn((N, H), gen).contiguous())


def decode_step_inputs(N, H, dk, dv, step, *, A=None, dtype=torch.bfloat16):
    """One decode step's token: q, k, v [N, H, d], g [N, H, dk], beta [N, H]."""
    if A is None:
        A = decode_log_scale(H)
    gen = _gen(1 + step)
    q = _randn((N, H, dk), gen)
    k = _randn((N, H, dk), gen)
    v = _randn((N, H, dv), gen)
    z = _randn((N, H, dk), gen)
    g = _sampled_log_decay(z, A)
    beta = torch.sigmoid(_randn((N, H), gen))
    cast = lambda x: x.to(dtype).contiguous()
    return dict(q=cast(q), k=cast(k), v=cast(v), g=cast(g), beta=cast(beta))


def grad_inputs(B, T, H, dk, dv, *, dtype=torch.bfloat16, dST_std=0.01, seed=0):
    """Upstream gradients of the backward workloads: dout ~ N(0,1) [B,T,H,dv] in the run
    dtype and dS_T ~ N(0, dST_std) [B,H,dk,dv] FP32 (None when dST_std is 0)."""
    gen = _gen(20_000 + seed)
    dout = _randn((B, T, H, dv), gen).to(dtype).contiguous()
    dST = _randn((B, H, dk, dv), gen) * dST_std if dST_std > 0 else None
    return dict(dout=dout, dS_T=dST)
