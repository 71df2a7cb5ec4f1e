"""kda_fwd_no_alloc against kda_fwd, through the C ABI, on the GPU.

kda_fwd_no_alloc serves callers that cannot allocate device memory when they run the prefill:
engines that reserve all device memory at start-up and hand kernels fixed buffers, plugin hosts
with no allocator, serving loops where an allocation could synchronise the device or fail. It
takes the scratch kda_fwd gets from a workspace (the longest-first order of packed documents)
from a static device array instead and runs the fused chunked kernel, so it must give bit for bit
what kda_fwd gives on that path (fused=True), and agree with the float64 oracle within the bf16
bound. Two calls in a row with different document counts also check that the shared array's
leftover contents never leak into the next call.

This file is collected last on purpose, so that a failure here comes after every other test.
"""

import ctypes

import pytest
import torch

import gated_delta_rule_144_b200 as kda
from gated_delta_rule_144_b200 import synth
from kda_testutil import TOL_BF16, host, oracle_fwd, rel_l2, require_cuda

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _regular(inp):
    """kda_fwd on the path the no-alloc entry point takes: the fused chunked kernel."""
    o, hT = kda.fwd(inp["q"], inp["k"], inp["v"], inp["log_g"], inp["beta"], h0=inp["h0"],
                    cu_seqlens=inp["cu_seqlens"], fused=True)
    return o, hT


def _check_against_oracle(inp, o, hT):
    o_ref, h_ref = oracle_fwd(inp)
    eo, eh = rel_l2(host(o), o_ref), rel_l2(host(hT), h_ref)
    assert eo <= TOL_BF16 and eh <= TOL_BF16, (eo, eh)


def _no_alloc_via_c_abi(inp):
    L = kda.lib()
    B, T, H, dk = inp["q"].shape
    dv = inp["v"].shape[3]
    N = inp["cu_seqlens"].numel() - 1 if inp["cu_seqlens"] is not None else B
    # caller-owned outputs, allocated up front by the test (the entry point allocates nothing)
    o = torch.empty((B, T, H, dv), dtype=inp["q"].dtype, device=DEV)
    hT = torch.empty((N, H, dk, dv), dtype=torch.float32, device=DEV)
    desc = kda.FwdDesc(B, T, H, dk, dv, N, kda.KDA_BF16, 0)
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = L.kda_fwd_no_alloc(ctypes.byref(desc), P(inp["q"]), P(inp["k"]), P(inp["v"]),
                            P(inp["log_g"]), P(inp["beta"]), P(inp["h0"]),
                            P(inp["cu_seqlens"]), P(o), P(hT), stream)
    assert st == 0, L.kda_last_error()
    return o, hT


def test_no_alloc_matches_kda_fwd_on_two_calls_in_a_row():
    require_cuda()
    first = synth.prefill_inputs("packed-8docs", lengths=[700, 64, 1300, 1, 300], H=8,
                                 h0_std=0.05, seed=21, device=DEV)
    second = synth.prefill_inputs("packed-8docs", lengths=[90, 500, 2], H=8, seed=22,
                                  device=DEV)
    for inp in (first, second):
        o_ref, h_ref = _regular(inp)
        o, hT = _no_alloc_via_c_abi(inp)
        torch.cuda.synchronize()
        assert kda.get_device_error() == 0
        assert torch.equal(o, o_ref) and torch.equal(hT, h_ref)
        _check_against_oracle(inp, o, hT)


def test_python_wrapper_of_the_no_alloc_entry_point():
    require_cuda()
    inp = synth.prefill_inputs("packed-8docs", lengths=[257, 1024, 33], H=4, seed=23, device=DEV)
    o_ref, h_ref = _regular(inp)
    o = torch.empty_like(o_ref)
    hT = torch.empty_like(h_ref)
    kda.fwd_no_alloc(inp["q"], inp["k"], inp["v"], inp["log_g"], inp["beta"], inp["h0"],
                     inp["cu_seqlens"], o, hT)
    torch.cuda.synchronize()
    assert kda.get_device_error() == 0
    assert torch.equal(o, o_ref) and torch.equal(hT, h_ref)
    _check_against_oracle(inp, o, hT)
