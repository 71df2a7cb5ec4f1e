"""GPU parity: libkda.so (through its C ABI) against the float64 oracle on the same inputs.

Metric: relative L2 error over all elements of o and of the final state, bound 1e-5 for fp32
inputs and 5e-3 for bf16 inputs.
"""

import numpy as np
import pytest
import torch

import gated_delta_rule_144_b200 as kda
from gated_delta_rule_144_b200 import synth
from kda_testutil import (TOL_BF16, TOL_F32, host, oracle_decode, oracle_fwd, rel_l2,
                          require_cuda, to)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _cuda():
    require_cuda()
    yield
    # no test may leave a device error behind
    assert kda.get_device_error() == 0


def _check_fwd(inp, tol, chunk_size=0):
    g = to(inp, DEV)
    o, hT = kda.fwd(g["q"], g["k"], g["v"], g["log_g"], g["beta"], h0=g.get("h0"),
                    cu_seqlens=g.get("cu_seqlens"), chunk_size=chunk_size)
    torch.cuda.synchronize()
    o_ref, h_ref = oracle_fwd(inp)
    eo, eh = rel_l2(host(o), o_ref), rel_l2(host(hT), h_ref)
    assert eo <= tol and eh <= tol, (eo, eh)
    return eo, eh


# ---------------------------------------------------------------- per-token (exact) path

def test_tiny_fp32_workload():
    """The fp32 workload: B=1, T=64, H=2, dk=dv=32, zero initial state, 1e-5."""
    inp = synth.prefill_inputs("tiny-fp32")
    _check_fwd(inp, TOL_F32, chunk_size=16)


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 48), (128, 128), (200, 20), (256, 8)])
def test_per_token_fp32_shapes(dk, dv):
    inp = synth.prefill_inputs("tiny-fp32", T=37, H=3, dk=dk, dv=dv, h0_std=0.3, seed=5)
    _check_fwd(inp, TOL_F32, chunk_size=1)


def test_per_token_bf16_t4096_h16():
    """The T=4096, H=16 bf16 workload through the per-token walk."""
    inp = synth.prefill_inputs("prefill-t4096")
    _check_fwd(inp, TOL_BF16, chunk_size=1)


def test_per_token_packed_with_empty_and_unit_documents():
    lengths = [37, 0, 1, 130, 64, 0]
    inp = synth.prefill_inputs("packed-8docs", lengths=lengths, H=4, h0_std=0.1, seed=9)
    _check_fwd(inp, TOL_BF16, chunk_size=1)
    inp32 = synth.prefill_inputs("packed-8docs", lengths=lengths, H=4, h0_std=0.1, seed=9,
                                 dtype="f32")
    _check_fwd(inp32, TOL_F32, chunk_size=1)


def test_zero_length_is_a_copy_of_h0():
    inp = synth.prefill_inputs("tiny-fp32", T=0, H=2, h0_std=0.5, seed=3)
    g = to(inp, DEV)
    o, hT = kda.fwd(g["q"], g["k"], g["v"], g["log_g"], g["beta"], h0=g["h0"])
    torch.cuda.synchronize()
    assert o.numel() == 0
    np.testing.assert_array_equal(host(hT), host(g["h0"]))


def test_bad_cu_seqlens_reported_by_device():
    inp = synth.prefill_inputs("packed-8docs", lengths=[4, 4], H=1, seed=2)
    g = to(inp, DEV)
    bad = torch.tensor([0, 6, 3], dtype=torch.int32, device=DEV)  # not monotone
    kda.fwd(g["q"], g["k"], g["v"], g["log_g"], g["beta"], cu_seqlens=bad, chunk_size=1)
    assert kda.get_device_error() == 5
    bad_end = torch.tensor([0, 4, 7], dtype=torch.int32, device=DEV)  # last != T
    kda.fwd(g["q"], g["k"], g["v"], g["log_g"], g["beta"], cu_seqlens=bad_end, chunk_size=1)
    assert kda.get_device_error() == 5


# ---------------------------------------------------------------- decode

def test_decode_n256_h32_full():
    """Decode workload at full size (256 sequences x 32 heads, fp32 state in place)."""
    inp = synth.decode_inputs("decode-n256", device=DEV)
    S_before = inp["S"].clone()
    o = kda.decode_step(inp["q"], inp["k"], inp["v"], inp["log_g"], inp["beta"], inp["S"])
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_decode(inp, S_before)
    eo, es = rel_l2(host(o), o_ref), rel_l2(host(inp["S"]), S_ref)
    assert eo <= TOL_BF16 and es <= TOL_BF16, (eo, es)
    # the state is fp32 and the math fp32: far tighter than the bf16 bound
    assert es <= 1e-5, es


@pytest.mark.parametrize("dtype,dk,dv", [("f32", 128, 128), ("f32", 64, 32), ("bf16", 96, 128),
                                         ("f32", 256, 256)])
def test_decode_shapes(dtype, dk, dv):
    inp = synth.decode_inputs("decode-n256", device=DEV, N=5, H=3, dk=dk, dv=dv, dtype=dtype,
                              seed=77)
    S_before = inp["S"].clone()
    o = kda.decode_step(inp["q"], inp["k"], inp["v"], inp["log_g"], inp["beta"], inp["S"])
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_decode(inp, S_before)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert rel_l2(host(o), o_ref) <= tol
    assert rel_l2(host(inp["S"]), S_ref) <= TOL_F32


def test_decode_equals_prefill_of_one_token():
    inp = synth.decode_inputs("decode-n256", device=DEV, N=8, H=4, dtype="f32", seed=4)
    S0 = inp["S"].clone()
    o_d = kda.decode_step(inp["q"], inp["k"], inp["v"], inp["log_g"], inp["beta"], inp["S"])
    o_p, hT = kda.fwd(inp["q"][:, None], inp["k"][:, None], inp["v"][:, None],
                      inp["log_g"][:, None], inp["beta"][:, None], h0=S0, chunk_size=1)
    torch.cuda.synchronize()
    assert rel_l2(host(o_d), host(o_p[:, 0])) <= 1e-6
    assert rel_l2(host(inp["S"]), host(hT)) <= 1e-6
