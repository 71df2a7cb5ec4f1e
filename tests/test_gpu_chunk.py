"""GPU parity of the chunked tcgen05 prefill (bf16, dk = dv = 128) against the float64 oracle.

Both chunked paths are checked: the split path (intra-chunk kernel over all chunks, then the
state pass; what kda_fwd runs with a full workspace) and the fused kernel (what it runs with the
minimum workspace). Sizes escalate from one chunk to the full workloads. Metric: relative L2 over
all elements of o and of the final states, bound 5e-3 (bf16 inputs).
"""

import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import gated_delta_rule_144_b200 as kda
import oracle
from gated_delta_rule_144_b200 import synth
from kda_testutil import TOL_BF16, host, oracle_fwd, rel_l2, require_cuda, to

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _cuda():
    require_cuda()
    yield


PATHS = pytest.mark.parametrize("fused", [False, True], ids=["split", "fused"])


def _run(inp, chunk_size=64, fused=False, workspace=None):
    g = to(inp, DEV)
    o, hT = kda.fwd(g["q"], g["k"], g["v"], g["log_g"], g["beta"], h0=g.get("h0"),
                    cu_seqlens=g.get("cu_seqlens"), chunk_size=chunk_size, fused=fused,
                    workspace=workspace)
    torch.cuda.synchronize()
    st = kda.get_device_error()
    return o, hT, st


def _check(inp, tol=TOL_BF16, fused=False):
    o, hT, st = _run(inp, fused=fused)
    assert st == 0, "device error %d" % st
    o_ref, h_ref = oracle_fwd(inp)
    eo, eh = rel_l2(host(o), o_ref), rel_l2(host(hT), h_ref)
    print("rel-L2 o %.3e hT %.3e" % (eo, eh))
    assert eo <= tol and eh <= tol, (eo, eh)
    return eo, eh


def test_chunk_path_is_selected():
    assert kda.fwd_algorithm(1, 64, 1, 128, 128, 1) == kda.CHUNK_64


@PATHS
def test_one_full_chunk(fused):
    _check(synth.prefill_inputs("prefill-t4096", T=64, H=1, seed=11), fused=fused)


@PATHS
def test_partial_chunks_batch_and_h0(fused):
    _check(synth.prefill_inputs("prefill-t4096", B=2, T=200, H=3, h0_std=0.1, seed=12), fused=fused)


@pytest.mark.parametrize("T", [1, 63, 65, 127, 129, 333])
@PATHS
def test_ragged_lengths(T, fused):
    _check(synth.prefill_inputs("long-t65536", B=1, T=T, H=2, seed=13 + T), fused=fused)


@pytest.mark.parametrize("B,T,H", [(4, 200, 64), (2, 129, 128)])
@PATHS
def test_many_chains_take_the_full_width_path(B, T, H, fused):
    """With more (sequence, head) chains than half the SMs, one CTA owns all 128 value columns
    of a chain; check that variant with h0, batches and ragged lengths."""
    _check(synth.prefill_inputs("prefill-t4096", B=B, T=T, H=H, h0_std=0.05, seed=17 + T),
           fused=fused)


@PATHS
def test_prefill_t4096_h16_full(fused):
    """The T=4096, H=16 bf16 workload at full size."""
    _check(synth.prefill_inputs("prefill-t4096"), fused=fused)


@PATHS
def test_packed_edge_documents(fused):
    lengths = [1, 63, 64, 65, 0, 130, 7, 200]
    _check(synth.prefill_inputs("packed-8docs", lengths=lengths, H=4, h0_std=0.05, seed=14),
           fused=fused)


@PATHS
def test_packed_documents_scheduled_longest_first(fused):
    """Documents in increasing length: the scheduling permutation is far from the identity."""
    _check(synth.prefill_inputs("packed-8docs", lengths=[50, 100, 700, 1300, 2, 1301], H=8,
                                h0_std=0.05, seed=18), fused=fused)


@PATHS
def test_packed_8docs_full(fused):
    """The packed 8-document workload (H = 32) at full size, every token and state."""
    _check(synth.prefill_inputs("packed-8docs"), fused=fused)


def test_chunked_equals_per_token_path():
    inp = synth.prefill_inputs("packed-8docs", lengths=[300, 17, 129], H=8, h0_std=0.02,
                               seed=15)
    o1, h1, st1 = _run(inp, 64)
    o2, h2, st2 = _run(inp, 1)
    assert st1 == 0 and st2 == 0
    assert rel_l2(host(o1), host(o2)) <= TOL_BF16
    assert rel_l2(host(h1), host(h2)) <= TOL_BF16


@pytest.mark.parametrize("name", ["long-t65536", "long-t65536-slow"])
def test_long_context_full_size_every_chain(name):
    """B=2, T=65536, H=32 with h0, at full size on both chunked paths: every one of the 64
    (sequence, head) chains is recomputed by the oracle end to end (every token's output and the
    final state) and compared element by element. The bound holds per chain, which is stricter
    than the relative L2 over the whole tensor (reported too). The oracle runs eight heads of one
    sequence at a time to bound host memory."""
    inp = synth.prefill_inputs(name, device=DEV)
    outs = {}
    for fused in (False, True):
        o, hT, st = _run(inp, fused=fused)
        assert st == 0, "device error %d" % st
        outs["fused" if fused else "split"] = (o, hT)
    f = lambda t: t.float().cpu().numpy()
    B, T, H = inp["q"].shape[:3]
    worst = {p: (0.0, 0.0, None) for p in outs}
    sq = {p: [0.0, 0.0] for p in outs}   # squared error over the whole tensor, per path
    ref_sq = [0.0, 0.0]
    group = 8
    for n in range(B):
        for h0_ in range(0, H, group):
            hs = slice(h0_, h0_ + group)
            o_ref, h_ref = oracle.kda_fwd(f(inp["q"][n:n + 1, :, hs]), f(inp["k"][n:n + 1, :, hs]),
                                          f(inp["v"][n:n + 1, :, hs]),
                                          f(inp["log_g"][n:n + 1, :, hs]),
                                          f(inp["beta"][n:n + 1, :, hs]),
                                          h0=f(inp["h0"][n:n + 1, hs]))
            ref_sq[0] += float(np.sum(o_ref ** 2))
            ref_sq[1] += float(np.sum(h_ref ** 2))
            for path, (o, hT) in outs.items():
                og = f(o[n:n + 1, :, hs]).astype(np.float64)
                hg = f(hT[n:n + 1, hs]).astype(np.float64)
                sq[path][0] += float(np.sum((og - o_ref) ** 2))
                sq[path][1] += float(np.sum((hg - h_ref) ** 2))
                for j in range(group):
                    eo = rel_l2(og[:, :, j], o_ref[:, :, j])
                    eh = rel_l2(hg[:, j], h_ref[:, j])
                    w = worst[path]
                    worst[path] = (max(w[0], eo), max(w[1], eh),
                                   (n, h0_ + j) if eo > w[0] else w[2])
    for path in outs:
        whole = (np.sqrt(sq[path][0] / ref_sq[0]), np.sqrt(sq[path][1] / ref_sq[1]))
        print("%s %s: worst chain rel-L2 o %.3e (chain %s) hT %.3e; whole tensor o %.3e hT %.3e"
              % (name, path, worst[path][0], worst[path][2], worst[path][1], *whole))
        assert worst[path][0] <= TOL_BF16 and worst[path][1] <= TOL_BF16, (path, worst[path])


def test_segmented_split_path_uneven_segments(monkeypatch):
    """Equal-length sequences of 101 chunks (the last one partial) run the split path in three
    chunk segments of 33, 34 and 34 chunks, the state crossing each boundary through the
    workspace: o and hT against the oracle. (The plain state pass: with 4 chains the default
    plan would take the two-level one.)"""
    monkeypatch.setenv("KDA_SCAN_SEGMENTS", "0")
    assert kda.fwd_split_segments(2, 64 * 100 + 17, 2, 128, 128, 2) == 3
    _check(synth.prefill_inputs("long-t65536", B=2, T=64 * 100 + 17, H=2, h0_std=0.05, seed=23))


def test_segment_count_does_not_change_the_result(monkeypatch):
    """The state crosses segment boundaries in fp32 and every chunk runs the same code, so any
    segment count gives bit-identical o and hT."""
    inp = to(synth.prefill_inputs("long-t65536", B=1, T=64 * 70 + 5, H=3, h0_std=0.05, seed=29),
             DEV)
    monkeypatch.setenv("KDA_SCAN_SEGMENTS", "0")   # the plain state pass, in chunk segments
    outs = []
    for segs in ("1", "2", "5", "8"):
        monkeypatch.setenv("KDA_SPLIT_SEGMENTS", segs)
        o, hT = kda.fwd(inp["q"], inp["k"], inp["v"], inp["log_g"], inp["beta"], h0=inp["h0"])
        torch.cuda.synchronize()
        outs.append((o.clone(), hT.clone()))
    assert kda.get_device_error() == 0
    for o, hT in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(hT, outs[0][1])


@pytest.mark.parametrize("P,expect", [("3", 3), ("4", 4), ("7", 7), ("32", 14)])
def test_two_level_state_pass_against_the_oracle(P, expect, monkeypatch):
    """The two-level state pass, forced to P segments (KDA_SCAN_SEGMENTS), on 2 sequences of
    14 chunks (the last one partial) x 3 heads with h0: segment 0 from h0, the transition maps
    and zero-start states of the inner segments, their fp32 chain, then the other segments at
    once; o and hT against the oracle. 32 asked gives one chunk per segment (14 segments). The
    gates decay slowly (log g = -softplus(N(-5, 1)): the median channel keeps about 0.65 of its
    state over a chunk), so every segment's initial state weighs on its outputs."""
    monkeypatch.setenv("KDA_SCAN_SEGMENTS", P)
    inp = synth.prefill_inputs("prefill-t4096", B=2, T=64 * 13 + 29, H=3, h0_std=0.05,
                               decay_mu=-5.0, seed=31)
    assert kda.fwd_scan_segments(2, inp["T"], 3, 128, 128, 2) == expect
    _check(inp)


@pytest.mark.parametrize("P", ["0", "4", "13"])
def test_two_level_state_pass_carries_h0_exactly_without_writes(P, monkeypatch):
    """beta = 0: every chunk's map is the pure decay (W = U~ = 0 exactly), so the final state is
    diag(prod_t g_t) h0 in closed form (the oracle pin beta = 0 => S_T = diag(prod g) S_0). The
    two-level pass carries h0 through the transition maps alone (A_p = the segment's decay
    product, B_p = 0, the fp32 chain of the segments' initial states): hT must meet the closed
    form to fp32 rounding, like the plain pass (P = 0); o against the oracle. The bound, 2e-4,
    allows for the chunk decays being products of 64 fp32 exponentials each (839 tokens); a
    segment's decay lost or applied twice would be off by about 45 %."""
    monkeypatch.setenv("KDA_SCAN_SEGMENTS", P)
    inp = synth.prefill_inputs("prefill-t4096", B=2, T=64 * 13 + 7, H=2, h0_std=1.0,
                               decay_mu=-5.0, seed=34)
    inp["beta"] = torch.zeros_like(inp["beta"])
    o, hT, st = _run(inp)
    assert st == 0
    total = inp["log_g"].double().sum(dim=1)                       # [B, H, dk]
    closed = torch.exp(total)[..., None] * inp["h0"].double()      # [B, H, dk, dv]
    eh = rel_l2(host(hT), closed.numpy())
    o_ref, _ = oracle_fwd(inp)
    eo = rel_l2(host(o), o_ref)
    print("P %s: hT vs closed form %.3e, o %.3e" % (P, eh, eo))
    assert eh <= 2e-4 and eo <= TOL_BF16


def test_two_level_state_pass_weak_writes_slow_decay(monkeypatch):
    """beta scaled by 0.05 and slow gates (log g = -softplus(N(-6, 1))): the state persists over
    many chunks, so the segments' initial states (the transition maps and zero-start states of
    the inner segments and their chain) carry most of hT. Forced 5 segments against the oracle and
    against the plain pass."""
    inp = synth.prefill_inputs("prefill-t4096", B=1, T=64 * 30 + 11, H=3, h0_std=0.5,
                               decay_mu=-6.0, seed=35)
    inp["beta"] = (inp["beta"].float() * 0.05).to(inp["beta"].dtype)
    monkeypatch.setenv("KDA_SCAN_SEGMENTS", "5")
    eo, eh = _check(inp)
    o2, h2, st = _run(inp)
    monkeypatch.setenv("KDA_SCAN_SEGMENTS", "0")
    o1, h1, st1 = _run(inp)
    assert st == 0 and st1 == 0
    d_o, d_h = rel_l2(host(o2), host(o1)), rel_l2(host(h2), host(h1))
    print("two-level vs plain: o %.3e hT %.3e" % (d_o, d_h))
    assert d_o <= TOL_BF16 and d_h <= TOL_BF16


def test_two_level_and_plain_state_pass_slow_decay(monkeypatch):
    """Slow gates (log g = -softplus(N(-6, 1))) over 40 chunks x 4 chains: the two-level pass
    (default plan) and the plain pass both meet the oracle, and differ from each other only by
    rounding."""
    monkeypatch.delenv("KDA_SCAN_SEGMENTS", raising=False)
    inp = synth.prefill_inputs("prefill-t4096", B=1, T=64 * 40, H=4, h0_std=0.05,
                               decay_mu=-6.0, seed=33)
    assert kda.fwd_scan_segments(1, inp["T"], 4, 128, 128, 1) >= 3
    _check(inp)
    o2, h2, st = _run(inp)
    assert st == 0
    monkeypatch.setenv("KDA_SCAN_SEGMENTS", "0")
    _check(inp)
    o1, h1, st = _run(inp)
    assert st == 0
    assert not torch.equal(h1, h2)   # the two passes round differently
    assert rel_l2(host(o2), host(o1)) <= TOL_BF16 and rel_l2(host(h2), host(h1)) <= TOL_BF16


def test_two_level_state_pass_without_final_state_and_with_steep_decays(monkeypatch):
    """Forced two-level pass (5 segments) with output_final_state=False (only o is written; the
    segments' states stay in the workspace), and with log g = -30 everywhere (every chunk takes
    the direct path; the transition maps are then all but zero)."""
    monkeypatch.setenv("KDA_SCAN_SEGMENTS", "5")
    inp = synth.prefill_inputs("long-t65536", B=1, T=64 * 10, H=2, h0_std=0.05, decay_mu=-5.0,
                               seed=32)
    g = to(inp, DEV)
    o, hT = kda.fwd(g["q"], g["k"], g["v"], g["log_g"], g["beta"], h0=g["h0"],
                    output_final_state=False)
    torch.cuda.synchronize()
    assert hT is None and kda.get_device_error() == 0
    o_ref, _ = oracle_fwd(inp)
    assert rel_l2(host(o), o_ref) <= TOL_BF16
    inp["log_g"] = torch.full_like(inp["log_g"], -30.0)
    _check(inp)


def test_prefill_t4096_two_level_and_plain_state_pass(monkeypatch):
    """The T=4096, H=16 workload at full size: the default plan takes the two-level state pass
    (16 chains); it and the plain pass (KDA_SCAN_SEGMENTS=0) both meet the oracle."""
    monkeypatch.delenv("KDA_SCAN_SEGMENTS", raising=False)
    inp = synth.prefill_inputs("prefill-t4096")
    assert kda.fwd_scan_segments(1, 4096, 16, 128, 128, 1) >= 3
    o_ref, h_ref = oracle_fwd(inp)
    res = {}
    for plan in ("default", "0"):
        if plan == "0":
            monkeypatch.setenv("KDA_SCAN_SEGMENTS", "0")
        o, hT, st = _run(inp)
        assert st == 0
        res[plan] = (rel_l2(host(o), o_ref), rel_l2(host(hT), h_ref))
        print(plan, "rel-L2 o %.3e hT %.3e" % res[plan])
        assert res[plan][0] <= TOL_BF16 and res[plan][1] <= TOL_BF16


def test_workspace_size_selects_the_path():
    """A workspace below kda_fwd_workspace_size (but covering the minimum) runs the fused kernel:
    bit-identical to fused=True; the full size runs the split path, which agrees within the
    tolerance (it stores the factors in bf16)."""
    inp = synth.prefill_inputs("packed-8docs", lengths=[300, 65, 1000], H=4, h0_std=0.02,
                               seed=19)
    T, N = inp["T"], inp["N"]
    full = kda.fwd_workspace_size(1, T, 4, 128, 128, N)
    small = kda.fwd_workspace_size_min(1, T, 4, 128, 128, N)
    assert 0 < small < full
    ws_small = torch.empty(full - 256, dtype=torch.uint8, device=DEV)
    o1, h1, st1 = _run(inp, workspace=ws_small)
    o2, h2, st2 = _run(inp, fused=True)
    o3, h3, st3 = _run(inp)
    assert st1 == st2 == st3 == 0
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
    assert rel_l2(host(o3), host(o2)) <= TOL_BF16 and rel_l2(host(h3), host(h2)) <= TOL_BF16


@PATHS
def test_steep_decay_everywhere(fused):
    """log g = -30 per token: every chunk's decay over 8 rows leaves the anchored factors' float32
    range, so every chunk takes the direct path; o and hT against the oracle."""
    inp = synth.prefill_inputs("prefill-t4096", B=2, T=200, H=2, h0_std=0.05, seed=16)
    inp["log_g"] = torch.full_like(inp["log_g"], -30.0)
    _check(inp, fused=fused)


@PATHS
def test_steep_and_gentle_chunks_in_one_chain(fused):
    """Ordinary gates with a few steep rows (log g from -40 to -200 in scattered rows and
    channels): the chunks that hold them take the direct path, the others the anchored factors,
    within one chain and one launch; packed documents, one of them ending inside a steep chunk."""
    inp = synth.prefill_inputs("packed-8docs", lengths=[64 * 5 + 17, 70, 300], H=3, h0_std=0.05,
                               seed=26)
    g = torch.Generator().manual_seed(27)
    lg = inp["log_g"]
    T = lg.shape[1]
    rows = torch.randint(0, T, (12,), generator=g)
    for r in rows.tolist():
        ch = torch.randint(0, 128, (8,), generator=g)
        lg[0, r, :, ch] = -40.0 - 160.0 * torch.rand((lg.shape[2], 8), generator=g)
    _check(inp, fused=fused)


def test_direct_path_forced_on_ordinary_inputs():
    """KDA_DEBUG_FORCE_DIRECT=1 sends every chunk of both chunked paths through the steep-decay
    path: on ordinary inputs (packed documents with h0, and a batch ending in a partial chunk) it
    must meet the oracle like the anchored factors do. Runs in a child process (the hook is read
    once per process)."""
    code = (
        "import torch, gated_delta_rule_144_b200 as kda, sys\n"
        "sys.path.insert(0, 'tests')\n"
        "from gated_delta_rule_144_b200 import synth\n"
        "from kda_testutil import oracle_fwd, rel_l2, host, to\n"
        "cases = [synth.prefill_inputs('packed-8docs', lengths=[700, 1, 64, 300], H=4,\n"
        "                              h0_std=0.05, seed=24),\n"
        "         synth.prefill_inputs('long-t65536', B=2, T=64 * 9 + 5, H=2, seed=25)]\n"
        "worst = 0.0\n"
        "for inp in cases:\n"
        "    o_ref, h_ref = oracle_fwd(inp)\n"
        "    g = to(inp, 'cuda:0')\n"
        "    for fused in (False, True):\n"
        "        o, hT = kda.fwd(g['q'], g['k'], g['v'], g['log_g'], g['beta'], h0=g['h0'],\n"
        "                        cu_seqlens=g['cu_seqlens'], fused=fused)\n"
        "        torch.cuda.synchronize()\n"
        "        assert kda.get_device_error() == 0\n"
        "        worst = max(worst, rel_l2(host(o), o_ref), rel_l2(host(hT), h_ref))\n"
        "print('WORST', worst)\n")
    env = dict(os.environ, KDA_DEBUG_FORCE_DIRECT="1")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], env=env, cwd=root, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    worst = float([x for x in r.stdout.splitlines() if x.startswith("WORST")][-1].split()[1])
    print("direct path, worst rel-L2 %.3e" % worst)
    assert worst <= TOL_BF16


def test_expired_wait_reports_timeout_and_context_survives():
    """Failure injection: with KDA_DEBUG_STALL_WAIT set, every CTA of the split path's two
    kernels waits (bounded by a 2M-cycle budget, about a millisecond) on a barrier that nothing
    signals; the state pass has its first record copies in flight at that point. Each kernel
    must report KDA_ERR_TIMEOUT, drain its own copies, free TMEM and return; the context must
    stay usable. Runs in a child process: the hooks are read once per process."""
    code = (
        "import torch, gated_delta_rule_144_b200 as kda\n"
        "from gated_delta_rule_144_b200 import synth\n"
        "inp = synth.prefill_inputs('prefill-t4096', T=512, H=2, device='cuda:0')\n"
        "kda.fwd(inp['q'], inp['k'], inp['v'], inp['log_g'], inp['beta'], chunk_size=64)\n"
        "st = kda.get_device_error()\n"
        "o, hT = kda.fwd(inp['q'], inp['k'], inp['v'], inp['log_g'], inp['beta'], chunk_size=1)\n"
        "torch.cuda.synchronize()\n"
        "print('STATUS', st, int(kda.get_device_error()))\n")
    env = dict(os.environ, KDA_DEBUG_WAIT_CYCLES="2000000", KDA_DEBUG_STALL_WAIT="1")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], env=env, cwd=root, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [x for x in r.stdout.splitlines() if x.startswith("STATUS")][-1]
    st, after = map(int, line.split()[1:])
    assert st == 4
    assert after == 0        # the context stays usable: the exact path runs clean afterwards


@pytest.mark.parametrize("plan", ["segments", "two-level"])
def test_split_call_replays_in_a_cuda_graph(plan, monkeypatch):
    """The split path's fork and join (state passes on the library's side stream) are event
    records and waits, so a call can be captured in a CUDA graph. The replay must equal the
    eager call bit for bit. Chunk segments overlapping the intra-chunk kernel (plain state pass,
    3 segments) and the two-level state pass (4 segments). The eager call also creates the
    library's side stream, events and kernel attributes before the capture."""
    if plan == "segments":
        monkeypatch.setenv("KDA_SCAN_SEGMENTS", "0")
        inp = synth.prefill_inputs("long-t65536", B=2, T=64 * 100 + 17, H=2, h0_std=0.05,
                                   seed=36, device=DEV)
    else:
        monkeypatch.setenv("KDA_SCAN_SEGMENTS", "4")
        inp = synth.prefill_inputs("prefill-t4096", B=1, T=64 * 20 + 5, H=3, h0_std=0.05,
                                   decay_mu=-3.0, seed=37, device=DEV)
    B, T, H = inp["B"], inp["T"], inp["H"]
    if plan == "segments":
        assert kda.fwd_split_segments(B, T, H, 128, 128, B) == 3
    else:
        assert kda.fwd_scan_segments(B, T, H, 128, 128, B) == 4
    args = (inp["q"], inp["k"], inp["v"], inp["log_g"], inp["beta"])
    ws = torch.empty(kda.fwd_workspace_size(B, T, H, 128, 128, B), dtype=torch.uint8,
                     device=DEV)
    o_ref, h_ref = kda.fwd(*args, h0=inp["h0"], workspace=ws)
    torch.cuda.synchronize()
    o = torch.empty_like(o_ref)
    hT = torch.empty_like(h_ref)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        kda.fwd(*args, h0=inp["h0"], o=o, hT=hT, workspace=ws)
    o.zero_()
    hT.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert kda.get_device_error() == 0
    assert torch.equal(o, o_ref) and torch.equal(hT, h_ref)
    del graph
