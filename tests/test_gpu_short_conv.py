"""GPU parity of kda_short_conv (the input prologue: short causal convolution with packed-document
resets, optional SiLU, optional per-group L2 norm) against the float64 oracle
(oracle/short_conv.py, pinned in tests/test_oracle_short_conv.py).

Metric: relative L2 over all elements, bound 1e-5 for fp32 and 5e-3 for bf16 (the kernel sums the
W taps in fp32 from the values it reads; the bf16 bound covers the output rounding). Also the
prologue followed by kda_fwd against the oracle's prologue followed by the oracle's recurrence.
"""

import numpy as np
import pytest
import torch

import gated_delta_rule_144_b200 as kda
from gated_delta_rule_144_b200 import synth
from kda_testutil import TOL_BF16, TOL_F32, host, oracle_fwd, rel_l2, require_cuda
from oracle.short_conv import short_conv as oracle_conv

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _cuda():
    require_cuda()
    yield


def _inputs(B, T, C, W, dtype, seed, lengths=None):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((B, T, C), generator=g).to(dtype)
    w = torch.randn((C, W), generator=g) / np.sqrt(W)
    cu = None
    if lengths is not None:
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    return x, w, cu


@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, TOL_BF16), (torch.float32, TOL_F32)],
                         ids=["bf16", "fp32"])
@pytest.mark.parametrize("act,group", [("none", 0), ("silu", 0), ("silu", 128), ("none", 32)])
@pytest.mark.parametrize("W", [1, 4, 8])
def test_packed_documents_against_the_oracle(dtype, tol, act, group, W):
    """Packed documents of 1, 0, 5, 17, 33 and 40 tokens (resets inside warps' token runs, an
    empty document), 3 heads of 128 channels."""
    lengths = [1, 0, 5, 17, 33, 40]
    x, w, cu = _inputs(1, sum(lengths), 384, W, dtype, 100 + W, lengths)
    y = kda.short_conv(x.to(DEV), w.to(DEV), cu.to(DEV), activation=act, norm_group=group)
    torch.cuda.synchronize()
    assert kda.get_device_error() == 0
    ref = oracle_conv(host(x), host(w), cu.numpy(), activation=act, norm_group=group)
    err = rel_l2(host(y), ref)
    assert err <= tol, err


@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, TOL_BF16), (torch.float32, TOL_F32)],
                         ids=["bf16", "fp32"])
def test_batch_rows_and_a_partial_channel_warp(dtype, tol):
    """B = 3 rows of 50 tokens (each row one document; 50 is not a multiple of the 16-token runs),
    C = 96 channels (one warp with lanes past C), L2 norm over groups of 32."""
    x, w, _ = _inputs(3, 50, 96, 3, dtype, 7)
    y = kda.short_conv(x.to(DEV), w.to(DEV), activation="silu", norm_group=32)
    torch.cuda.synchronize()
    ref = oracle_conv(host(x), host(w), None, activation="silu", norm_group=32)
    assert rel_l2(host(y), ref) <= tol


@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, TOL_BF16), (torch.float32, TOL_F32)],
                         ids=["bf16", "fp32"])
def test_partial_warp_span_and_one_lane_groups(dtype, tol):
    """C = 100 channels (a warp's 128-channel span is partly idle) and a norm group of 4 (one lane
    per group, no shuffles); packed documents, W = 2."""
    lengths = [9, 30, 1, 20]
    x, w, cu = _inputs(1, sum(lengths), 100, 2, dtype, 9, lengths)
    y = kda.short_conv(x.to(DEV), w.to(DEV), cu.to(DEV), activation="silu", norm_group=4)
    torch.cuda.synchronize()
    assert kda.get_device_error() == 0
    ref = oracle_conv(host(x), host(w), cu.numpy(), activation="silu", norm_group=4)
    assert rel_l2(host(y), ref) <= tol


def test_packed_8docs_shape_full_size():
    """The packed 8-document workload's q shape (28937 tokens, 32 heads x 128 channels), W = 4,
    SiLU and a per-head L2 norm, every element against the oracle."""
    inp = synth.prefill_inputs("packed-8docs")
    T = inp["T"]
    x, w, _ = _inputs(1, T, 32 * 128, 4, torch.bfloat16, 8)
    cu = inp["cu_seqlens"]
    y = kda.short_conv(x.to(DEV), w.to(DEV), cu.to(DEV), activation="silu", norm_group=128)
    torch.cuda.synchronize()
    assert kda.get_device_error() == 0
    ref = oracle_conv(host(x), host(w), cu.numpy(), activation="silu", norm_group=128)
    err = rel_l2(host(y), ref)
    print("rel-L2 %.3e" % err)
    assert err <= TOL_BF16


def test_prologue_then_recurrence():
    """Projections of q, k, v (random) through the prologue (SiLU; q and k L2-normalised per head)
    and then kda_fwd, against the oracle's prologue followed by the oracle's recurrence, on packed
    documents; each side rounds the prologue's outputs to bf16 as the recurrence reads them."""
    H, d, W = 4, 128, 4
    lengths = [70, 1, 130, 33]
    T = sum(lengths)
    base = synth.prefill_inputs("packed-8docs", lengths=lengths, H=H, h0_std=0.05, seed=61)
    cu = base["cu_seqlens"]
    xs = {n: _inputs(1, T, H * d, W, torch.bfloat16, 62 + i)[:2] for i, n in enumerate("qkv")}
    gpu = {}
    ref = {}
    for n, (x, w) in xs.items():
        grp = d if n in "qk" else 0
        gpu[n] = kda.short_conv(x.to(DEV), w.to(DEV), cu.to(DEV), activation="silu",
                                norm_group=grp).view(1, T, H, d)
        r = oracle_conv(host(x), host(w), cu.numpy(), activation="silu", norm_group=grp)
        ref[n] = torch.from_numpy(r).float().to(torch.bfloat16).view(1, T, H, d)
    g = {k: base[k].to(DEV) if base[k] is not None else None
         for k in ("log_g", "beta", "h0", "cu_seqlens")}
    o, hT = kda.fwd(gpu["q"], gpu["k"], gpu["v"], g["log_g"], g["beta"], h0=g["h0"],
                    cu_seqlens=g["cu_seqlens"])
    torch.cuda.synchronize()
    assert kda.get_device_error() == 0
    o_ref, h_ref = oracle_fwd(dict(q=ref["q"], k=ref["k"], v=ref["v"], log_g=base["log_g"],
                                   beta=base["beta"], h0=base["h0"], cu_seqlens=cu))
    eo, eh = rel_l2(host(o), o_ref), rel_l2(host(hT), h_ref)
    print("rel-L2 o %.3e hT %.3e" % (eo, eh))
    assert eo <= TOL_BF16 and eh <= TOL_BF16
