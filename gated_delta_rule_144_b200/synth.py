"""Seeded synthetic inputs for the KDA workloads (shared by the tests, the oracle checks and the bench).

This module draws random numbers and casts them to the dtypes the library consumes. It holds
none of the recurrence's arithmetic: q and k are L2-normalised here because the workloads
specify inputs that arrive already normalised; the library itself never normalises.

Workloads (names follow the shapes they describe):
  tiny-fp32        B=1, T=64, H=2, dk=dv=32, fp32 everything, zero initial state
  prefill-t4096    B=1, T=4096, H=16, dk=dv=128, bf16 q/k/v/beta, fp32 log g, zero state
  packed-8docs     8 documents, lengths U[512, 8192] (integers, whole set redrawn until the total
                   is <= 32768), one packed row described by int32 cu_seqlens, H=32, d=128, bf16
  decode-n256      N=256 sequences, one token each, H=32, d=128, fp32 state S ~ N(0, 0.02^2)
  long-t65536      B=2, T=65536, H=32, d=128, bf16, h0 ~ N(0, 0.02^2), log g = -softplus(N(2, 1))
  long-t65536-slow same with log g = -softplus(N(-2, 1)) (slow decay; reported, not a target)

Distributions: q, k ~ N(0, 1) then L2-normalised per (token, head) vector; v ~ N(0, 1);
log g = -softplus(N(mu, 1)) per key channel (mu = 0 unless stated); beta = sigmoid(N(0, 1)).
Seeds: workload i uses seed 1000 + i. Values are drawn in float32 with a torch.Generator on the
device the tensors are made on (the stream therefore depends on the device, the distribution
does not), then cast.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    kind: str                 # "prefill" or "decode"
    B: int = 1
    T: int = 0
    H: int = 1
    dk: int = 128
    dv: int = 128
    dtype: str = "bf16"       # dtype of q, k, v, beta and o
    decay_mu: float = 0.0
    h0_std: float = 0.0       # 0 = zero initial state
    chunk_size: int = 0
    docs: int = 0             # > 0: packed variable-length row with this many documents
    doc_len: tuple = (512, 8192)
    max_total: int = 32768
    N: int = 0                # decode: number of sequences
    state_std: float = 0.0    # decode: std of the state
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "tiny-fp32": Workload("tiny-fp32", 0, "prefill", B=1, T=64, H=2, dk=32, dv=32, dtype="f32",
                          chunk_size=16),
    "prefill-t4096": Workload("prefill-t4096", 1, "prefill", B=1, T=4096, H=16),
    "packed-8docs": Workload("packed-8docs", 2, "prefill", B=1, H=32, docs=8),
    "decode-n256": Workload("decode-n256", 3, "decode", N=256, H=32, state_std=0.02),
    "long-t65536": Workload("long-t65536", 4, "prefill", B=2, T=65536, H=32, decay_mu=2.0,
                            h0_std=0.02),
    "long-t65536-slow": Workload("long-t65536-slow", 4, "prefill", B=2, T=65536, H=32,
                                 decay_mu=-2.0, h0_std=0.02),
    # several rows per sequence against the decode state (verify rows of batched decoding):
    # the decode workload's sequences and distributions with T = 4 rows each
    "decode-rows-n256-t4": Workload("decode-rows-n256-t4", 3, "decode", N=256, T=4, H=32,
                                    state_std=0.02),
}

_TORCH_DTYPE = {"bf16": torch.bfloat16, "f32": torch.float32}


def doc_lengths(num_docs: int, lo: int, hi: int, max_total: int, seed: int) -> list[int]:
    """Integer lengths uniform on [lo, hi]; the whole set is redrawn until its sum <= max_total."""
    rng = np.random.default_rng(seed)
    while True:
        lens = rng.integers(lo, hi, size=num_docs, endpoint=True)
        if int(lens.sum()) <= max_total:
            return [int(x) for x in lens]


def cu_seqlens_from_lengths(lengths, device="cpu") -> torch.Tensor:
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return torch.tensor(cu, dtype=torch.int32, device=device)


def _normal(gen, shape, device, mean=0.0, std=1.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if mean != 0.0:
        x.add_(mean)
    return x


def _unit_rows(gen, shape, device, dtype):
    x = _normal(gen, shape, device)
    x.div_(torch.linalg.vector_norm(x, dim=-1, keepdim=True).clamp_min(1e-30))
    return x.to(dtype)


def _gate(gen, shape, device, mu):
    # log g = -softplus(N(mu, 1)), kept in float32
    return F.softplus(_normal(gen, shape, device, mean=mu)).neg_()


def prefill_inputs(w: Workload | str, device="cpu", *, B=None, T=None, H=None, lengths=None,
                   seed=None, dtype=None, dk=None, dv=None, decay_mu=None, h0_std=None):
    """Make the inputs of one prefill call. Overrides shrink or reshape a workload for tests.

    Returns a dict with q, k, v (dtype), log_g (f32), beta (dtype), h0 (f32 or None),
    cu_seqlens (int32 or None), lengths (list or None) and the resolved sizes.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    dt = _TORCH_DTYPE[dtype or w.dtype]
    H = H or w.H
    dk = dk or w.dk
    dv = dv or w.dv
    seed = 1000 + w.index if seed is None else seed
    mu = w.decay_mu if decay_mu is None else decay_mu
    hstd = w.h0_std if h0_std is None else h0_std
    cu = None
    if lengths is None and w.docs > 0:
        lengths = doc_lengths(w.docs, w.doc_len[0], w.doc_len[1], w.max_total, seed)
    if lengths is not None:
        B = 1
        T = int(sum(lengths))
        cu = cu_seqlens_from_lengths(lengths, device)
        N = len(lengths)
    else:
        B = B or w.B
        T = w.T if T is None else T
        N = B
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = _unit_rows(gen, (B, T, H, dk), device, dt)
    k = _unit_rows(gen, (B, T, H, dk), device, dt)
    v = _normal(gen, (B, T, H, dv), device).to(dt)
    log_g = _gate(gen, (B, T, H, dk), device, mu)
    beta = torch.sigmoid(_normal(gen, (B, T, H), device)).to(dt)
    h0 = _normal(gen, (N, H, dk, dv), device, std=hstd) if hstd > 0 else None
    return dict(q=q, k=k, v=v, log_g=log_g, beta=beta, h0=h0, cu_seqlens=cu, lengths=lengths,
                B=B, T=T, H=H, dk=dk, dv=dv, N=N, dtype=dtype or w.dtype, seed=seed)


def decode_tokens_inputs(w: Workload | str = "decode-rows-n256-t4", device="cpu", *, N=None,
                         T=None, H=None, seed=None, dtype=None, dk=None, dv=None,
                         decay_mu=None, state_std=None):
    """Inputs of T decode rows per sequence: q, k, log_g [N, T, H, dk], v [N, T, H, dv],
    beta [N, T, H] (drawn like a prefill batch of N sequences) and the fp32 state S [N, H, dk, dv]
    ~ N(0, state_std^2)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    N = N or w.N
    T = w.T if T is None else T
    H = H or w.H
    seed = 1000 + w.index + 50 if seed is None else seed
    sstd = w.state_std if state_std is None else state_std
    p = prefill_inputs("prefill-t4096", device, B=N, T=T, H=H, seed=seed,
                       dtype=dtype or w.dtype, dk=dk or w.dk, dv=dv or w.dv,
                       decay_mu=w.decay_mu if decay_mu is None else decay_mu, h0_std=sstd)
    S = p["h0"] if p["h0"] is not None else torch.zeros(
        (N, H, p["dk"], p["dv"]), dtype=torch.float32, device=device)
    return dict(q=p["q"], k=p["k"], v=p["v"], log_g=p["log_g"], beta=p["beta"], S=S, N=N, T=T,
                H=H, dk=p["dk"], dv=p["dv"], dtype=dtype or w.dtype, seed=seed)


def decode_inputs(w: Workload | str = "decode-n256", device="cpu", *, N=None, H=None, seed=None,
                  dtype=None, dk=None, dv=None, decay_mu=None, state_std=None):
    """Inputs of one decode step: q, k, v, log_g, beta per sequence and the fp32 state S."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    dt = _TORCH_DTYPE[dtype or w.dtype]
    N = N or w.N
    H = H or w.H
    dk = dk or w.dk
    dv = dv or w.dv
    seed = 1000 + w.index if seed is None else seed
    mu = w.decay_mu if decay_mu is None else decay_mu
    sstd = w.state_std if state_std is None else state_std
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = _unit_rows(gen, (N, H, dk), device, dt)
    k = _unit_rows(gen, (N, H, dk), device, dt)
    v = _normal(gen, (N, H, dv), device).to(dt)
    log_g = _gate(gen, (N, H, dk), device, mu)
    beta = torch.sigmoid(_normal(gen, (N, H), device)).to(dt)
    S = _normal(gen, (N, H, dk, dv), device, std=sstd)
    return dict(q=q, k=k, v=v, log_g=log_g, beta=beta, S=S, N=N, H=H, dk=dk, dv=dv,
                dtype=dtype or w.dtype, seed=seed)
