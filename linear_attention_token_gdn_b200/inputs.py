"""Seeded synthetic inputs for the GDN mixer workloads.

This module only draws random numbers in the shapes, value distributions and
layouts of the five workloads below.  It holds none of the method's arithmetic
(the recurrence, the short convolution, the norms); the one place where a
formula appears is the recipe that *draws* the decay input, which the workload
definition states as alpha = exp(-exp(A) * softplus(u)) with u ~ N(0,1) and
exp(A) uniform.  Both the CUDA path and the fp64 oracle read the tensors made
here, byte for byte.

Workloads (every tensor is token-major: [N, H, d] with d contiguous):

0. tiny: B=1, H=2, T=64, dk=dv=16, fp32 q/k/v; S0 = 0.
1. prefill: B=2, H=16, T=4096, dk=dv=128, bf16 q/k/v, fp32 g/beta, S0 = 0, chunk 64.
2. long prefill: B=1, H=32, T=32768, dk=dv=128, bf16; exp(A) ~ U(1,64);
   S0 ~ N(0, 0.02) (standard deviation), output y and S_T.
3. decode: 256 sequences x H=32, dk=dv=128, fp32 state ~ N(0, 0.05), fresh
   bf16 q/k/v and fp32 g/beta at each of 100 steps.
4. full mixer: 4 packed sequences with lengths ~ U{1024..8192}, H=16, d=128,
   bf16 projection outputs ~ N(0,1), conv taps ~ N(0, 0.5) width 4, beta/alpha
   logits ~ N(0,1), A = log U(1,16), b_alpha ~ N(0, 0.5), z ~ N(0,1),
   norm weight ~ N(0, 0.02), eps 1e-6.
5. input projections + prep: the mixer's lengths, H=16, d=128, from the normalised
   residual stream x ~ N(0,1) of width D = H*d = 2048 (bf16) and the stacked weight rows
   [W_q; W_k; W_v; W_z; W_beta; W_alpha] ~ N(0, 1/D) (standard deviation D^-1/2, so each
   projection output is about N(0,1), the mixer's distribution), conv taps, A and b_alpha
   as in the mixer.

q and k are drawn N(0,1) and scaled to unit L2 norm per head (in fp32) before
the cast to the storage dtype; v ~ N(0,1); beta = sigmoid(N(0,1)).
"""
from __future__ import annotations

import numpy as np
import torch

SEED_BASE = 20261202

# workload keys (each workload's seed is SEED_BASE + its key)
TINY, PREFILL, LONG_PREFILL, DECODE, MIXER, INPROJ = 0, 1, 2, 3, 4, 5

WORKLOAD_SPECS = {
    TINY: dict(name="tiny_fp32_B1_H2_T64_d16", kind="prefill", B=1, H=2, T=64, d=16, dtype=torch.float32,
            expA=(1.0, 16.0), S0_std=0.0, chunk=0),
    PREFILL: dict(name="prefill_B2_H16_T4096_d128", kind="prefill", B=2, H=16, T=4096, d=128,
            dtype=torch.bfloat16, expA=(1.0, 16.0), S0_std=0.0, chunk=64),
    LONG_PREFILL: dict(name="prefill_B1_H32_T32768_d128", kind="prefill", B=1, H=32, T=32768, d=128,
            dtype=torch.bfloat16, expA=(1.0, 64.0), S0_std=0.02, chunk=64),
    DECODE: dict(name="decode_B256_H32_d128_x100", kind="decode", B=256, H=32, d=128, dtype=torch.bfloat16,
            expA=(1.0, 16.0), state_std=0.05, steps=100),
    MIXER: dict(name="mixer_4seq_H16_d128_N<=32768", kind="mixer", nseq=4, H=16, d=128, L=(1024, 8192),
            dtype=torch.bfloat16, W=4, conv_std=0.5, norm_std=0.02, expA=(1.0, 16.0), ba_std=0.5,
            eps=1e-6),
    INPROJ: dict(name="inproj_prep_4seq_H16_d128_D2048", kind="inproj", nseq=4, H=16, d=128, D=2048,
            L=(1024, 8192), dtype=torch.bfloat16, W=4, conv_std=0.5, expA=(1.0, 16.0), ba_std=0.5, eps=1e-6),
}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def unit_rows(n, H, d, gen, device, dtype):
    """N(0,1) rows scaled to unit L2 norm per (token, head), then cast to ``dtype``."""
    x = torch.randn(n, H, d, generator=gen, device=device, dtype=torch.float32)
    x = x / x.norm(dim=-1, keepdim=True).clamp_min(1e-20)
    return x.to(dtype)


def decay_and_write_gates(n, H, expA_range, gen, device):
    """g = log(alpha) with alpha = exp(-exp(A) softplus(u)), u ~ N(0,1), exp(A) ~ U(lo, hi) per head;
    beta = sigmoid(N(0,1)).  Returned in fp32, shape [n, H]."""
    lo, hi = expA_range
    expA = torch.empty(H, device=device, dtype=torch.float64).uniform_(lo, hi, generator=gen)
    u = torch.randn(n, H, generator=gen, device=device, dtype=torch.float64)
    g = -(expA[None, :] * torch.nn.functional.softplus(u))
    beta = torch.sigmoid(torch.randn(n, H, generator=gen, device=device, dtype=torch.float64))
    return g.to(torch.float32), beta.to(torch.float32)


def make_prefill(cfg=PREFILL, device="cpu", seed=None, **over):
    """Inputs of a prefill workload.  Keyword overrides: B, T, H, d (or dk/dv), dtype,
    S0_std, expA, lengths (packed variable lengths; overrides B and T)."""
    c = dict(WORKLOAD_SPECS[cfg])
    c.update(over)
    dk = c.get("dk", c["d"])
    dv = c.get("dv", c["d"])
    H = c["H"]
    gen = _gen(device, SEED_BASE + cfg if seed is None else seed)
    if c.get("lengths") is not None:
        lengths = [int(x) for x in c["lengths"]]
        cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
        num_seqs = len(lengths)
    else:
        num_seqs = c["B"]
        cu = (np.arange(num_seqs + 1) * c["T"]).astype(np.int32)
    N = int(cu[-1])
    q = unit_rows(N, H, dk, gen, device, c["dtype"])
    k = unit_rows(N, H, dk, gen, device, c["dtype"])
    v = torch.randn(N, H, dv, generator=gen, device=device, dtype=torch.float32).to(c["dtype"])
    g, beta = decay_and_write_gates(N, H, c["expA"], gen, device)
    S0 = None
    if c["S0_std"] > 0:
        S0 = torch.randn(num_seqs, H, dk, dv, generator=gen, device=device, dtype=torch.float32) * c["S0_std"]
    return dict(q=q, k=k, v=v, g=g, beta=beta, S0=S0,
                cu_seqlens=torch.from_numpy(cu).to(device), num_seqs=num_seqs, N=N, H=H, dk=dk, dv=dv,
                chunk=c.get("chunk", 64))


def make_decode_state(cfg=DECODE, device="cpu", seed=None, **over):
    c = dict(WORKLOAD_SPECS[cfg])
    c.update(over)
    dk = c.get("dk", c["d"])
    dv = c.get("dv", c["d"])
    gen = _gen(device, (SEED_BASE + cfg if seed is None else seed) * 7 + 1)
    slots = c.get("slots", c["B"])
    return torch.randn(slots, c["H"], dk, dv, generator=gen, device=device, dtype=torch.float32) * c["state_std"]


def make_decode_step(cfg=DECODE, device="cpu", step=0, seed=None, **over):
    """Fresh one-token inputs for decode step ``step``."""
    c = dict(WORKLOAD_SPECS[cfg])
    c.update(over)
    dk = c.get("dk", c["d"])
    dv = c.get("dv", c["d"])
    B, H = c["B"], c["H"]
    gen = _gen(device, (SEED_BASE + cfg if seed is None else seed) * 1000 + 17 + step)
    q = unit_rows(B, H, dk, gen, device, c["dtype"])
    k = unit_rows(B, H, dk, gen, device, c["dtype"])
    v = torch.randn(B, H, dv, generator=gen, device=device, dtype=torch.float32).to(c["dtype"])
    g, beta = decay_and_write_gates(B, H, c["expA"], gen, device)
    return dict(q=q, k=k, v=v, g=g, beta=beta)


def mixer_lengths(cfg=MIXER, seed=None, nseq=None, L=None):
    c = WORKLOAD_SPECS[cfg]
    rng = np.random.Generator(np.random.PCG64(SEED_BASE + cfg if seed is None else seed))
    lo, hi = c["L"] if L is None else L
    return [int(x) for x in rng.integers(lo, hi + 1, size=c["nseq"] if nseq is None else nseq)]


def make_mixer(cfg=MIXER, device="cpu", seed=None, lengths=None, **over):
    """Raw (post-projection) inputs of the full mixer workload."""
    c = dict(WORKLOAD_SPECS[cfg])
    c.update(over)
    H, d, W = c["H"], c["d"], c["W"]
    if lengths is None:
        lengths = mixer_lengths(cfg, seed)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    N = int(cu[-1])
    gen = _gen(device, SEED_BASE + cfg if seed is None else seed)
    dt = c["dtype"]

    def randn(*shape, std=1.0):
        return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32) * std

    lo, hi = c["expA"]
    expA = torch.empty(H, device=device, dtype=torch.float64).uniform_(lo, hi, generator=gen)
    return dict(
        x_q=randn(N, H, d).to(dt), x_k=randn(N, H, d).to(dt), x_v=randn(N, H, d).to(dt),
        w_q=randn(H * d, W, std=c["conv_std"]), w_k=randn(H * d, W, std=c["conv_std"]),
        w_v=randn(H * d, W, std=c["conv_std"]),
        beta_logit=randn(N, H).to(dt), alpha_logit=randn(N, H).to(dt),
        A_log=torch.log(expA).to(torch.float32), alpha_bias=randn(H, std=c["ba_std"]),
        z=randn(N, H, d).to(dt), norm_w=randn(d, std=c["norm_std"]),
        cu_seqlens=torch.from_numpy(cu).to(device), num_seqs=len(lengths), N=N, H=H, d=d, W=W,
        eps=c["eps"], lengths=list(lengths))


def make_inproj(cfg=INPROJ, device="cpu", seed=None, lengths=None, **over):
    """Residual-stream rows x [N, D] and the stacked projection weights w [4*H*d + 2*H, D] with
    the prep parameters, for the fused input projections."""
    c = dict(WORKLOAD_SPECS[cfg])
    c.update(over)
    H, d, D, W = c["H"], c["d"], c["D"], c["W"]
    if lengths is None:
        lengths = mixer_lengths(MIXER, seed)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    N = int(cu[-1])
    gen = _gen(device, SEED_BASE + cfg if seed is None else seed)
    dt = c["dtype"]

    def randn(*shape, std=1.0):
        return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32) * std

    lo, hi = c["expA"]
    expA = torch.empty(H, device=device, dtype=torch.float64).uniform_(lo, hi, generator=gen)
    return dict(
        x=randn(N, D).to(dt), w=randn(4 * H * d + 2 * H, D, std=D ** -0.5).to(dt),
        conv_q=randn(H * d, W, std=c["conv_std"]), conv_k=randn(H * d, W, std=c["conv_std"]),
        conv_v=randn(H * d, W, std=c["conv_std"]),
        A_log=torch.log(expA).to(torch.float32), alpha_bias=randn(H, std=c["ba_std"]),
        cu_seqlens=torch.from_numpy(cu).to(device), num_seqs=len(lengths), N=N, H=H, d=d, D=D, W=W,
        eps=c["eps"], lengths=list(lengths))
