"""kda_decode_tokens on the GPU: T rows per sequence against the decode state, in place.

The oracle is the float64 prefill from h0 = S (T tokens of each of N sequences), whose final
state is the new S. Bound: relative L2 over all elements of o and of S, 5e-3 for bf16 inputs and
1e-5 for fp32 (bf16 o is rounded, so its fp32-input bound applies to S and the fp32 o only).
"""

import pytest
import torch

import gated_delta_rule_144_b200 as kda
import oracle
from gated_delta_rule_144_b200 import synth
from kda_testutil import TOL_BF16, TOL_F32, host, rel_l2, require_cuda

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _cuda():
    require_cuda()
    yield


def _oracle(inp, S_before):
    return oracle.kda_fwd(host(inp["q"]), host(inp["k"]), host(inp["v"]), host(inp["log_g"]),
                          host(inp["beta"]), h0=host(S_before))


def _run(inp):
    S = inp["S"].clone()
    o = kda.decode_tokens(inp["q"], inp["k"], inp["v"], inp["log_g"], inp["beta"], S)
    torch.cuda.synchronize()
    assert kda.get_device_error() == 0
    return o, S


@pytest.mark.parametrize("T", [1, 2, 4, 7, 8, 9, 20])
@pytest.mark.parametrize("dtype,tol", [("bf16", TOL_BF16), ("f32", TOL_F32)])
def test_rows_match_the_oracle(T, dtype, tol):
    """T up to 8 arrives with the state (prefetched rows); 9 and 20 add groups read later."""
    inp = synth.decode_tokens_inputs(N=6, T=T, H=3, dtype=dtype, seed=60 + T, device=DEV)
    o, S = _run(inp)
    o_ref, S_ref = _oracle(inp, inp["S"])
    eo, es = rel_l2(host(o), o_ref), rel_l2(host(S), S_ref)
    assert eo <= tol and es <= tol, (eo, es)


@pytest.mark.parametrize("dk,dv", [(64, 32), (256, 128)])
def test_general_head_sizes_take_the_per_token_walk(dk, dv):
    inp = synth.decode_tokens_inputs(N=4, T=3, H=2, dtype="f32", dk=dk, dv=dv, seed=70,
                                     device=DEV)
    o, S = _run(inp)
    o_ref, S_ref = _oracle(inp, inp["S"])
    assert rel_l2(host(o), o_ref) <= TOL_F32 and rel_l2(host(S), S_ref) <= TOL_F32


@pytest.mark.parametrize("T,N,H", [(5, 8, 4), (11, 40, 8)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_rows_equal_successive_decode_steps_bit_for_bit(dtype, T, N, H):
    """T rows in one call = T calls of kda_decode_step: the state stays fp32 in registers between
    rows exactly as it would in memory, and each row's arithmetic runs in the same order. 40 x 8
    units exceed the persistent grid, so blocks walk several units with prefetched rows."""
    inp = synth.decode_tokens_inputs(N=N, T=T, H=H, dtype=dtype, seed=80, device=DEV)
    o, S = _run(inp)
    S2 = inp["S"].clone()
    for t in range(T):
        sl = lambda x: x[:, t].contiguous()
        o_t = kda.decode_step(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["log_g"]),
                              sl(inp["beta"]), S2)
        assert torch.equal(o_t, o[:, t]), t
    torch.cuda.synchronize()
    assert torch.equal(S, S2)


def test_zero_rows_leave_the_state_alone():
    inp = synth.decode_tokens_inputs(N=3, T=0, H=2, seed=81, device=DEV)
    o, S = _run(inp)
    assert o.numel() == 0 and torch.equal(S, inp["S"])


def test_decode_rows_n256_t4_full():
    """The 256-sequence, 32-head workload with 4 rows each, every element against the oracle."""
    inp = synth.decode_tokens_inputs("decode-rows-n256-t4", device=DEV)
    o, S = _run(inp)
    o_ref, S_ref = _oracle(inp, inp["S"])
    eo, es = rel_l2(host(o), o_ref), rel_l2(host(S), S_ref)
    print("rel-L2 o %.3e S %.3e" % (eo, es))
    assert eo <= TOL_BF16 and es <= TOL_BF16, (eo, es)
