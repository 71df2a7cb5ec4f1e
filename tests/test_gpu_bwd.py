"""GPU parity of kda_bwd (gradients of the recurrence, for training) against the float64 oracle
(oracle/backward.py, pinned in tests/test_oracle_backward.py).

Metric: relative L2 over all elements of each gradient (dq, dk, dv, dlog_g, dbeta, dh0). Bound
1e-4 for bf16 and fp32 inputs alike: the kernel computes every gradient in fp32 from the exact
values it reads (the oracle gets the same values), so only fp32 rounding separates them. A
gradient element sums up to 128 x 128 products per token through a reverse chain whose decays
are below one; with unit roundoff 6e-8 that is about sqrt(128 * T) * 6e-8, under 1e-5 for these
sizes, and the bound keeps ten times that.
"""

import numpy as np
import pytest
import torch

import gated_delta_rule_144_b200 as kda
from gated_delta_rule_144_b200 import synth
from kda_testutil import host, rel_l2, require_cuda, to
from oracle.backward import kda_bwd as oracle_bwd

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TOL_BWD = 1e-4
NAMES = ("dq", "dk", "dv", "dlog_g", "dbeta", "dh0")


@pytest.fixture(autouse=True)
def _cuda():
    require_cuda()
    yield


def _check(inp, seed, with_dhT=True):
    g = to(inp, DEV)
    B, T, H, _ = g["q"].shape
    N = inp["N"]
    gen = torch.Generator().manual_seed(seed)
    do = torch.randn(tuple(g["v"].shape), generator=gen).to(g["v"].dtype).to(DEV)
    dhT = (torch.randn((N, H, 128, 128), generator=gen) * 0.5).to(DEV) if with_dhT else None
    cu = g.get("cu_seqlens")
    grads = kda.bwd(g["q"], g["k"], g["v"], g["log_g"], g["beta"], do, h0=g.get("h0"), dhT=dhT,
                    cu_seqlens=cu)
    torch.cuda.synchronize()
    assert kda.get_device_error() == 0
    ref = oracle_bwd(host(g["q"]), host(g["k"]), host(g["v"]), host(g["log_g"]),
                     host(g["beta"]), host(do), dhT=host(dhT), h0=host(g.get("h0")),
                     cu_seqlens=None if cu is None else cu.cpu().numpy())
    errs = {n: rel_l2(host(x), r) for n, x, r in zip(NAMES, grads, ref)}
    print(" ".join("%s %.2e" % kv for kv in errs.items()))
    assert all(e <= TOL_BWD for e in errs.values()), errs


def test_bwd_fp32_batch_partial_chunks():
    """fp32 inputs, B=2 sequences of 150 tokens (chunks of 64, 64 and 22), h0 and dhT."""
    _check(synth.prefill_inputs("prefill-t4096", B=2, T=150, H=2, dtype="f32", h0_std=0.1,
                                seed=31), seed=1)


def test_bwd_bf16_packed_with_empty_document():
    """bf16 packed documents of 70, 0 and 130 tokens, h0 and dhT per document."""
    _check(synth.prefill_inputs("packed-8docs", lengths=[70, 0, 130], H=2, h0_std=0.05,
                                seed=32), seed=2)


def test_bwd_bf16_one_chunk_no_initial_or_final_state():
    """One full chunk, no h0 and no dhT (both zero)."""
    inp = synth.prefill_inputs("prefill-t4096", B=1, T=64, H=1, seed=33)
    inp["h0"] = None
    _check(inp, seed=3, with_dhT=False)


def test_bwd_without_tokens_passes_the_final_state_gradient_through():
    """T = 0: the final state is h0, so dh0 = dhT."""
    z = lambda *s: torch.zeros(s, dtype=torch.bfloat16, device=DEV)
    dhT = torch.randn((2, 3, 128, 128), device=DEV)
    grads = kda.bwd(z(2, 0, 3, 128), z(2, 0, 3, 128), z(2, 0, 3, 128),
                    torch.zeros((2, 0, 3, 128), device=DEV), z(2, 0, 3), z(2, 0, 3, 128),
                    dhT=dhT)
    torch.cuda.synchronize()
    assert torch.equal(grads[5], dhT)


def test_bwd_at_the_benched_size_sampled_heads():
    """The T=4096, H=16 bf16 workload that the benchmark times, with the benchmark's seeds: the GPU
    computes every gradient of all 16 heads; the oracle recomputes four heads end to end (every
    token's dq, dk, dv, dlog_g, dbeta and the head's dh0) and each is compared element by
    element."""
    inp = synth.prefill_inputs("prefill-t4096", device=DEV, seed=1001)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(1095)
    do = torch.randn(inp["v"].shape, generator=gen, device=DEV).to(inp["v"].dtype)
    dhT = torch.randn((inp["N"], inp["H"], 128, 128), generator=gen, device=DEV)
    grads = kda.bwd(inp["q"], inp["k"], inp["v"], inp["log_g"], inp["beta"], do, h0=inp["h0"],
                    dhT=dhT)
    torch.cuda.synchronize()
    assert kda.get_device_error() == 0
    worst = dict.fromkeys(NAMES, 0.0)
    for h in (0, 5, 10, 15):
        sl = lambda t: host(t[:, :, h:h + 1])
        ref = oracle_bwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["log_g"]),
                         sl(inp["beta"]), sl(do), dhT=host(dhT[:, h:h + 1]),
                         h0=None if inp["h0"] is None else host(inp["h0"][:, h:h + 1]))
        got = [sl(x) for x in grads[:5]] + [host(grads[5][:, h:h + 1])]
        for n, x, r in zip(NAMES, got, ref):
            worst[n] = max(worst[n], rel_l2(x, r))
    print("worst head: " + " ".join("%s %.2e" % kv for kv in worst.items()))
    assert all(e <= TOL_BWD for e in worst.values()), worst
