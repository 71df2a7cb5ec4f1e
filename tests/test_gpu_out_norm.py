"""The gated per-head RMSNorm of the output on the GPU, against the float64 oracle.

The reference is oracle.out_norm.out_norm_gated applied to the oracle's prefill output.

Bounds (relative L2 over all elements):
- the norm alone, on exact inputs: 5e-3 for bf16 (rounding of y), 1e-5 for fp32;
- the whole prefill followed by the norm: 1e-2 for bf16. The norm rescales every (token, head)
  vector to unit RMS, and dy = (dx - x (x . dx) / (D rms^2)) / rms * w * sigmoid(g), so
  |dy| <= 2 |dx| / rms: each vector's relative error at most doubles, and the vectors now count
  equally instead of by their size. Twice the prefill's own bound on o (5e-3) covers it;
  the final states keep the prefill's 5e-3.
"""

import pytest
import torch

import gated_delta_rule_144_b200 as kda
from gated_delta_rule_144_b200 import synth
from kda_testutil import TOL_BF16, TOL_F32, host, oracle_fwd, rel_l2, require_cuda, to

TOL_NORMED_BF16 = 2 * TOL_BF16   # the prefill's bound on o, through the per-vector norm
from oracle.out_norm import out_norm_gated

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
EPS = 1e-6


@pytest.fixture(autouse=True)
def _cuda():
    require_cuda()
    yield


def _gate_weight(shape, dtype, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    gate = torch.randn(shape, generator=g, device=DEV).to(dtype)
    w = torch.rand(shape[-1], generator=g, device=DEV) + 0.5
    return gate, w


@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, TOL_BF16), (torch.float32, TOL_F32)])
@pytest.mark.parametrize("dv", [128, 64, 40])
def test_standalone_norm_matches_the_oracle(dtype, tol, dv):
    g = torch.Generator(device=DEV)
    g.manual_seed(90 + dv)
    x = (torch.randn((3, 70, 5, dv), generator=g, device=DEV) * 2).to(dtype)
    gate, w = _gate_weight(x.shape, dtype, 91 + dv)
    y = kda.out_norm_gated(x, gate, w, EPS)
    ref = out_norm_gated(host(x), host(gate), host(w), EPS)
    assert rel_l2(host(y), ref) <= tol
    x2 = x.clone()
    kda.out_norm_gated(x2, gate, w, EPS, y=x2)   # in place
    assert torch.equal(x2, y)


CASES = [
    ("partial chunks with h0", lambda: synth.prefill_inputs("prefill-t4096", B=2, T=200, H=3,
                                                            h0_std=0.1, seed=92)),
    ("packed edge documents", lambda: synth.prefill_inputs(
        "packed-8docs", lengths=[1, 63, 64, 65, 0, 130, 7, 200], H=4, h0_std=0.05, seed=93)),
    ("one sequence, several chunks", lambda: synth.prefill_inputs("long-t65536", B=1, T=513,
                                                                  H=2, seed=94)),
    # 71 chunks: the split path runs two chunk segments, each state pass applying the norm (the
    # plain state pass: with 4 chains the default plan would take the two-level one)
    ("two chunk segments", lambda: synth.prefill_inputs("long-t65536", B=2, T=64 * 70 + 9, H=2,
                                                        h0_std=0.05, seed=98), "0"),
    # the two-level state pass, 4 segments: segment 0 and the last phase apply the norm
    ("two-level state pass", lambda: synth.prefill_inputs("long-t65536", B=2, T=64 * 20 + 9,
                                                          H=2, h0_std=0.05, decay_mu=-3.0,
                                                          seed=99), "4"),
]


@pytest.mark.parametrize("path", ["split", "fused", "per-token"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_fwd_normed_matches_the_oracle(case, path, monkeypatch):
    if len(case) > 2:   # the state-pass plan this case is about
        monkeypatch.setenv("KDA_SCAN_SEGMENTS", case[2])
    inp = case[1]()
    g = to(inp, DEV)
    B, T, H = g["B"], g["T"], g["H"]
    gate, w = _gate_weight((B, T, H, 128), torch.bfloat16, 95)
    y, hT = kda.fwd(g["q"], g["k"], g["v"], g["log_g"], g["beta"], h0=g.get("h0"),
                    cu_seqlens=g.get("cu_seqlens"), chunk_size=1 if path == "per-token" else 0,
                    fused=path == "fused", out_norm=(gate, w, EPS))
    torch.cuda.synchronize()
    assert kda.get_device_error() == 0
    o_ref, h_ref = oracle_fwd(inp)
    y_ref = out_norm_gated(o_ref, host(gate), host(w), EPS)
    ey, eh = rel_l2(host(y), y_ref), rel_l2(host(hT), h_ref)
    print("%s %s: rel-L2 y %.3e hT %.3e" % (case[0], path, ey, eh))
    assert ey <= TOL_NORMED_BF16 and eh <= TOL_BF16, (ey, eh)


@pytest.mark.parametrize("fused", [False, True], ids=["split", "fused"])
def test_normed_call_equals_fwd_then_norm(fused):
    """kda_fwd_normed is the plain prefill followed by the norm on the same bf16 output: the
    fused kernel runs the norm as a pass over its output, the split path's state pass applies it
    to each output tile before storing it, in the same arithmetic, so both are bit-identical to
    the plain call followed by kda_out_norm_gated."""
    inp = synth.prefill_inputs("packed-8docs", lengths=[700, 64, 1300, 1, 300], H=8, seed=96,
                               device=DEV)
    gate, w = _gate_weight((1, inp["T"], 8, 128), torch.bfloat16, 97)
    y, _ = kda.fwd(inp["q"], inp["k"], inp["v"], inp["log_g"], inp["beta"],
                   cu_seqlens=inp["cu_seqlens"], out_norm=(gate, w, EPS), fused=fused)
    o, _ = kda.fwd(inp["q"], inp["k"], inp["v"], inp["log_g"], inp["beta"],
                   cu_seqlens=inp["cu_seqlens"], fused=fused)
    y2 = kda.out_norm_gated(o, gate, w, EPS)
    torch.cuda.synchronize()
    assert kda.get_device_error() == 0
    assert torch.equal(y, y2), rel_l2(host(y), host(y2))


def test_normed_call_equals_fwd_then_norm_two_level(monkeypatch):
    """The same identity on the two-level state pass (5 segments forced): segment 0 and the last
    phase's segments apply the norm to their output tiles; the maps launch writes no output."""
    monkeypatch.setenv("KDA_SCAN_SEGMENTS", "5")
    inp = synth.prefill_inputs("long-t65536", B=2, T=64 * 25 + 3, H=3, h0_std=0.05, seed=100,
                               device=DEV)
    B, T = inp["B"], inp["T"]
    assert kda.fwd_scan_segments(B, T, 3, 128, 128, B) == 5
    gate, w = _gate_weight((B, T, 3, 128), torch.bfloat16, 101)
    y, h1 = kda.fwd(inp["q"], inp["k"], inp["v"], inp["log_g"], inp["beta"], h0=inp["h0"],
                    out_norm=(gate, w, EPS))
    o, h2 = kda.fwd(inp["q"], inp["k"], inp["v"], inp["log_g"], inp["beta"], h0=inp["h0"])
    y2 = kda.out_norm_gated(o, gate, w, EPS)
    torch.cuda.synchronize()
    assert kda.get_device_error() == 0
    assert torch.equal(y, y2), rel_l2(host(y), host(y2))
    assert torch.equal(h1, h2)
