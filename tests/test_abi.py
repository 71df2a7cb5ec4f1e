"""C-ABI checks that need no GPU: the library loads, exports what include/kda.h declares, and
rejects bad arguments on the host before any launch.

Every call here fails host-side validation (NULL, misaligned or inconsistent arguments), so these
tests launch nothing even when a GPU is present; fake pointers are never dereferenced.
"""

import ctypes
import re
from pathlib import Path

import pytest

import gated_delta_rule_144_b200 as kda
from gated_delta_rule_144_b200 import build as kbuild

ROOT = Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    return kda.lib()


def _declared_functions():
    text = (ROOT / "include" / "kda.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for must in ("kda_fwd", "kda_decode_step", "kda_decode_tokens", "kda_get_device_error",
                 "kda_status_string",
                 "kda_fwd_workspace_size", "kda_last_error", "kda_version"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    for name in _declared_functions():
        assert hasattr(L, name), name


def test_status_strings_and_version(L):
    assert L.kda_version() >= 100
    for code in range(7):
        assert L.kda_status_string(code)
    assert L.kda_status_string(99) == b"unknown status"


def _desc(**kw):
    d = dict(B=1, T=64, H=2, dk=128, dv=128, num_seqs=1, dtype=kda.KDA_BF16, chunk_size=0)
    d.update(kw)
    return kda.FwdDesc(**d)


FAKE = 0x100000  # aligned fake address: only ever passed alongside an argument that fails


def _fwd(L, desc, q=FAKE, k=FAKE, v=FAKE, g=FAKE, b=FAKE, h0=None, cu=None, o=FAKE, hT=None):
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return L.kda_fwd(None if desc is None else ctypes.byref(desc), P(q), P(k), P(v), P(g),
                     P(b), P(h0), P(cu), P(o), P(hT), None, 0, None)


@pytest.mark.parametrize("case", [
    ("null desc", None, {}),
    ("negative T", _desc(T=-1), {}),
    ("zero heads", _desc(H=0), {}),
    ("N != B without cu_seqlens", _desc(B=2, num_seqs=1), {}),
    ("cu_seqlens with B > 1", _desc(B=2, num_seqs=2), {"cu": FAKE}),
    ("bad dtype", _desc(dtype=7), {}),
    ("null q", _desc(), {"q": None}),
    ("null beta", _desc(), {"b": None}),
    ("null o", _desc(), {"o": None}),
    ("misaligned k", _desc(), {"k": FAKE + 2}),
    ("misaligned h0", _desc(), {"h0": FAKE + 8}),
    ("misaligned cu_seqlens", _desc(num_seqs=1), {"cu": FAKE + 4, "q": FAKE + 1}),
], ids=lambda c: c[0])
def test_fwd_rejects_on_host(L, case):
    _, desc, kw = case
    st = _fwd(L, desc, **kw)
    assert st == 1, (st, L.kda_last_error())
    assert L.kda_last_error()


def test_fwd_unsupported_combinations(L):
    # chunked tensor-core path is bf16 with dk = dv = 128 only
    assert _fwd(L, _desc(dk=64, chunk_size=64), q=None) in (1, 2)
    assert _fwd(L, _desc(chunk_size=48), q=FAKE + 1) in (1, 2)
    st = _fwd(L, _desc(dk=64, dv=64, chunk_size=64))
    assert st == 2
    st = _fwd(L, _desc(dk=512, dv=64, chunk_size=1))
    assert st == 2


def test_decode_rejects_on_host(L):
    P = ctypes.c_void_p
    args = lambda **kw: [kw.get(n, P(FAKE)) for n in ("q", "k", "v", "g", "b", "S", "o")]
    assert L.kda_decode_step(-1, 1, 128, 128, 1, *args(), None) == 1
    assert L.kda_decode_step(1, 0, 128, 128, 1, *args(), None) == 1
    assert L.kda_decode_step(1, 1, 128, 128, 5, *args(), None) == 1
    assert L.kda_decode_step(1, 1, 512, 128, 1, *args(), None) == 2
    assert L.kda_decode_step(1, 1, 128, 128, 1, *args(S=None), None) == 1
    assert L.kda_decode_step(1, 1, 128, 128, 1, *args(o=P(FAKE + 4)), None) == 1


def _split_bytes(B, T, H, N, packed):
    """Split-path workspace: per (64-token chunk record, head) 32 KiB of [W; Q+], 2 x 16 KiB of
    K_end and U~, 8 KiB of A_qk and 512 B of decay; 256 B of record counters (one per chunk
    segment, at most 16); the record map and document order when packed, else one fp32 128 x 128
    state per (sequence, head) carried between chunk segments."""
    up = lambda x: (x + 255) // 256 * 256
    ncT = (T + 63) // 64
    G = ncT + N if packed else B * ncT
    R = G * H
    order = up(4 * N) if packed and 2 <= N <= 2048 else 0
    state = 0 if packed else N * H * 128 * 128 * 4
    return (order + (up(4 * G) if packed else 0) + up(8 * 16) + state + up(512 * R) +
            R * (32768 + 2 * 16384 + 8192))


def test_decode_tokens_rejects_on_host(L):
    P = ctypes.c_void_p
    args = lambda **kw: [kw.get(n, P(FAKE)) for n in ("q", "k", "v", "g", "b", "S", "o")]
    assert L.kda_decode_tokens(1, 1, -1, 128, 128, 1, *args(), None) == 1
    assert L.kda_decode_tokens(1, 0, 4, 128, 128, 1, *args(), None) == 1
    assert L.kda_decode_tokens(1, 1, 4, 128, 128, 9, *args(), None) == 1
    assert L.kda_decode_tokens(1, 1, 4, 512, 128, 1, *args(), None) == 2
    assert L.kda_decode_tokens(1, 1, 4, 128, 128, 1, *args(S=None), None) == 1
    assert L.kda_decode_tokens(1, 1, 4, 128, 128, 1, *args(q=P(FAKE + 2)), None) == 1
    # nothing to do: no pointer is needed
    assert L.kda_decode_tokens(1, 1, 0, 128, 128, 1, None, None, None, None, None, None, None,
                               None) == 0


def test_out_norm_rejects_on_host(L):
    P = ctypes.c_void_p
    d = _desc()
    nrm = kda.OutNorm(FAKE, FAKE, 1e-6)
    call = lambda desc, norm: L.kda_fwd_normed(ctypes.byref(desc), P(FAKE), P(FAKE), P(FAKE),
                                               P(FAKE), P(FAKE), None, None, norm, P(FAKE), None,
                                               None, 0, None)
    assert call(d, None) == 1                                     # no norm
    assert call(_desc(dv=512, dtype=kda.KDA_F32), ctypes.byref(nrm)) == 2   # dv > 256
    bad = kda.OutNorm(FAKE, FAKE, -1.0)
    assert call(d, ctypes.byref(bad)) == 1                        # eps < 0
    bad = kda.OutNorm(None, FAKE, 1e-6)
    assert call(d, ctypes.byref(bad)) == 1                        # no gate
    assert L.kda_out_norm_gated(4, 300, 1, P(FAKE), P(FAKE), P(FAKE), 1e-6, P(FAKE), None) == 2
    assert L.kda_out_norm_gated(4, 128, 1, P(FAKE), None, P(FAKE), 1e-6, P(FAKE), None) == 1
    assert L.kda_out_norm_gated(4, 128, 1, P(FAKE + 2), P(FAKE), P(FAKE), 1e-6, P(FAKE),
                                None) == 1
    assert L.kda_out_norm_gated(0, 128, 1, None, None, None, 1e-6, None, None) == 0


def test_workspace_size_is_host_only(L):
    # minimum (fused chunked path): only packed documents need scratch, one int32 each
    d = _desc()
    assert L.kda_fwd_workspace_size_min(ctypes.byref(d)) == 0
    d = _desc(num_seqs=8)
    assert L.kda_fwd_workspace_size_min(ctypes.byref(d)) == 256
    d = _desc(num_seqs=300)
    assert L.kda_fwd_workspace_size_min(ctypes.byref(d)) == 1280
    # preferred (split chunked path): the stored WY factors of every chunk record and head
    for kw, packed in (({}, True), ({"num_seqs": 8}, True), ({"num_seqs": 300}, True),
                       ({"B": 2, "num_seqs": 2, "T": 4096, "H": 16}, False)):
        d = _desc(**kw)
        want = _split_bytes(d.B, d.T, d.H, d.num_seqs, packed)
        assert L.kda_fwd_workspace_size(ctypes.byref(d)) == want, kw
    # the exact path needs none
    d = _desc(num_seqs=8, chunk_size=1)
    assert L.kda_fwd_workspace_size(ctypes.byref(d)) == 0
    assert L.kda_fwd_workspace_size_min(ctypes.byref(d)) == 0


def test_split_segments_rule(L, monkeypatch):
    """Equal-length sequences of more than 64 chunks run in segments of at least 32 chunks, at
    most 12; packed documents, sequences of up to 64 chunks and the per-token path in one; the
    environment override is capped at 16 and at the chunk count."""
    L.kda_fwd_split_segments.restype = ctypes.c_int
    seg = lambda T, varlen=0, **kw: L.kda_fwd_split_segments(ctypes.byref(_desc(T=T, **kw)),
                                                             varlen)
    monkeypatch.delenv("KDA_SPLIT_SEGMENTS", raising=False)
    monkeypatch.setenv("KDA_SCAN_SEGMENTS", "0")   # the plain state pass (no two-level plan)
    assert seg(64 * 63) == 1 and seg(64 * 64) == 1 and seg(64 * 64 + 1) == 2
    assert seg(64 * 101) == 3 and seg(65536) == 12 and seg(1 << 20) == 12
    assert seg(65536, varlen=1, B=1, num_seqs=4) == 1
    assert seg(65536, chunk_size=1) == 1
    monkeypatch.setenv("KDA_SPLIT_SEGMENTS", "40")
    assert seg(65536) == 16 and seg(64 * 3) == 3
    monkeypatch.setenv("KDA_SPLIT_SEGMENTS", "1")
    assert seg(65536) == 1


def test_bwd_workspace_size_and_host_rejections(L):
    """kda_bwd: per (sequence or document, head) one 64 KiB state per 64 tokens plus one, a
    64-token chunk of states and 64 x 2 x 128 fp32 read-outs; dk = dv = 128 only; missing
    pointers and a short workspace are rejected before any launch."""
    L.kda_bwd_workspace_size.restype = ctypes.c_size_t
    for kw in (dict(B=2, T=150, H=2, num_seqs=2), dict(B=1, T=200, H=2, num_seqs=3),
               dict(B=1, T=64, H=1, num_seqs=1)):
        d = _desc(**kw)
        chains = kw["num_seqs"] * kw["H"]
        nck = (kw["T"] + 63) // 64 + 1
        want = chains * ((nck + 64) * 128 * 128 + 64 * 2 * 128) * 4
        assert L.kda_bwd_workspace_size(ctypes.byref(d)) == want, kw
    assert L.kda_bwd_workspace_size(ctypes.byref(_desc(dk=64))) == 0
    P = ctypes.c_void_p
    F = P(FAKE)

    def bwd(desc, dout=F, ws=F, ws_bytes=1 << 40):
        return L.kda_bwd(ctypes.byref(desc), F, F, F, F, F, None, None, dout, None, F, F, F, F,
                         F, None, ws, ctypes.c_size_t(ws_bytes), None)
    assert bwd(_desc(dk=64)) == 2
    assert bwd(_desc(dv=64)) == 2
    assert bwd(_desc(), dout=None) == 1 and b"do" in L.kda_last_error()
    assert bwd(_desc(), ws=None) == 1 and b"workspace" in L.kda_last_error()
    assert bwd(_desc(), ws_bytes=1024) == 1
    assert bwd(_desc(), dout=P(FAKE + 4)) == 1   # misaligned


def test_packed_chunked_call_without_workspace_is_rejected_on_host(L):
    P = ctypes.c_void_p
    d = _desc(num_seqs=8)
    st = L.kda_fwd(ctypes.byref(d), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), None, P(FAKE),
                   P(FAKE), None, None, 0, None)
    assert st == 1 and b"workspace" in L.kda_last_error()
    st = L.kda_fwd(ctypes.byref(d), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), None, P(FAKE),
                   P(FAKE), None, P(FAKE + 8), 4096, None)   # misaligned workspace
    assert st == 1 and b"workspace" in L.kda_last_error()


def test_no_alloc_entry_rejects_more_documents_than_its_scratch_on_host(L):
    P = ctypes.c_void_p
    d = _desc(num_seqs=2049)
    st = L.kda_fwd_no_alloc(ctypes.byref(d), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), None,
                            P(FAKE), P(FAKE), None, None)
    assert st == 1 and b"2048" in L.kda_last_error()


def test_python_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 4, 1, 8)
    with pytest.raises(ValueError, match="CUDA tensor"):
        kda.fwd(q, q, q, q, torch.zeros(1, 4, 1))
    with pytest.raises(ValueError, match="CUDA tensor"):
        kda.decode_step(q[0], q[0], q[0], q[0], torch.zeros(4, 1), torch.zeros(4, 1, 8, 8))


def test_no_alloc_binding_checks_shapes_before_any_launch():
    """fwd_no_alloc reads v, o and hT with the sizes taken from q: a v shorter in T or H, an o or
    hT of the wrong shape, or a malformed cu_seqlens must raise before the library is called."""
    import torch
    B, T, H, d = 1, 8, 2, 16
    q = torch.zeros(B, T, H, d, dtype=torch.bfloat16)
    g = torch.zeros(B, T, H, d)
    beta = torch.zeros(B, T, H, dtype=torch.bfloat16)
    o = torch.zeros(B, T, H, d, dtype=torch.bfloat16)
    hT = torch.zeros(B, H, d, d)
    short_t = torch.zeros(B, T - 1, H, d, dtype=torch.bfloat16)
    short_h = torch.zeros(B, T, H - 1, d, dtype=torch.bfloat16)
    for v in (short_t, short_h, torch.zeros(T, H, d, dtype=torch.bfloat16)):
        with pytest.raises(ValueError, match="v must be"):
            kda.fwd_no_alloc(q, q, v, g, beta, None, None, o, hT)
    with pytest.raises(ValueError, match="q must be"):
        kda.fwd_no_alloc(q[0], q, q, g, beta, None, None, o, hT)
    with pytest.raises(ValueError, match="o must have shape"):
        kda.fwd_no_alloc(q, q, q, g, beta, None, None, o[:, :4], hT)
    with pytest.raises(ValueError, match="hT must have shape"):
        kda.fwd_no_alloc(q, q, q, g, beta, None, None, o, hT[:, :1])
    with pytest.raises(ValueError, match="cu_seqlens"):
        kda.fwd_no_alloc(q, q, q, g, beta, None, torch.zeros((2, 2), dtype=torch.int32), o, None)


def test_short_conv_rejects_on_host(L):
    P = ctypes.c_void_p
    ok = dict(B=1, T=16, C=256, W=4, dtype=kda.KDA_BF16, x=P(FAKE), w=P(FAKE), cu=None, N=1,
              act=0, group=128, eps=1e-6, y=P(FAKE + 0x100000))

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return L.kda_short_conv(a["B"], a["T"], a["C"], a["W"], a["dtype"], a["x"], a["w"],
                                a["cu"], a["N"], a["act"], a["group"], a["eps"], a["y"], None)

    assert call(W=0) == 2 and call(W=9) == 2
    assert call(C=258) == 2                      # not a multiple of 4
    assert call(group=12) == 2 and call(group=256) == 2 and call(C=192, group=128) == 2
    assert call(act=3) == 1
    assert call(eps=-1.0) == 1
    assert call(x=None) == 1 and call(x=P(FAKE + 4)) == 1
    assert call(y=P(FAKE + 64)) == 1             # overlaps x
    assert b"overlaps" in L.kda_last_error()
    assert call(B=2, cu=P(FAKE)) == 1            # cu_seqlens needs B == 1
    assert call(T=0) == 0                        # no tokens: nothing to do


def test_scan_segments_rule(L, monkeypatch):
    """Host plan of the two-level state pass: few chains of many chunks take it, many chains or
    short sequences the plain pass; KDA_SCAN_SEGMENTS overrides (capped by the chunks, no empty
    segment); its states grow the workspace; the split path then runs one chunk segment."""
    monkeypatch.delenv("KDA_SCAN_SEGMENTS", raising=False)

    def plan(B, T, H, cu=0, **kw):
        return L.kda_fwd_scan_segments(ctypes.byref(_desc(B=B, T=T, H=H, num_seqs=B, **kw)), cu)

    assert plan(1, 4096, 16) >= 3              # 16 chains of 64 chunks
    assert plan(2, 65536, 32) == 1             # 64 chains: chunk segments overlap instead
    assert plan(4, 4096, 16) == 1              # 64 chains
    assert plan(1, 200, 3) == 1                # 4 chunks
    assert plan(1, 4096, 16, cu=1) == 1        # packed documents
    assert plan(1, 4096, 16, chunk_size=1) == 1
    assert plan(1, 4096, 16, dtype=7) < 0      # rejected description
    d = _desc(B=1, T=4096, H=16, num_seqs=1)
    assert L.kda_fwd_split_segments(ctypes.byref(d), 0) == 1
    ws_two_level = L.kda_fwd_workspace_size(ctypes.byref(d))
    for v, want in (("0", 1), ("1", 1), ("2", 1), ("3", 3), ("5", 5), ("40", 32)):
        monkeypatch.setenv("KDA_SCAN_SEGMENTS", v)
        assert plan(1, 4096, 16) == want, v
    assert plan(1, 64 * 13 + 29, 3) == 14      # 14 chunks: one per segment
    assert plan(1, 64 * 9, 3) == 9
    monkeypatch.setenv("KDA_SCAN_SEGMENTS", "7")
    assert plan(1, 64 * 10, 3) == 5            # 7 asked: segments of 2 chunks, 5 of them
    monkeypatch.setenv("KDA_SCAN_SEGMENTS", "0")
    ws_plain = L.kda_fwd_workspace_size(ctypes.byref(d))
    assert ws_two_level > ws_plain
