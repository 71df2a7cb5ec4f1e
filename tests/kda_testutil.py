"""Helpers shared by the GPU parity tests: relative-L2 metric and oracle calls on GPU inputs."""

import numpy as np
import torch

import oracle

# Tolerances (relative L2 over all elements of a tensor).
TOL_F32 = 1e-5   # fp32 inputs
TOL_BF16 = 5e-3  # bf16 inputs


def rel_l2(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    return float(np.linalg.norm((x - ref).ravel()) / max(den, 1e-300))


def host(t):
    return None if t is None else t.detach().float().cpu().numpy()


def oracle_fwd(inp, num_threads=0):
    cu = inp.get("cu_seqlens")
    return oracle.kda_fwd(host(inp["q"]), host(inp["k"]), host(inp["v"]), host(inp["log_g"]),
                          host(inp["beta"]), h0=host(inp.get("h0")),
                          cu_seqlens=None if cu is None else cu.cpu().numpy(),
                          num_threads=num_threads)


def oracle_decode(inp, S_before):
    return oracle.kda_decode(host(inp["q"]), host(inp["k"]), host(inp["v"]), host(inp["log_g"]),
                             host(inp["beta"]), host(S_before))


def to(inp, device):
    out = dict(inp)
    for key in ("q", "k", "v", "log_g", "beta", "h0", "cu_seqlens", "S"):
        if out.get(key) is not None:
            out[key] = out[key].to(device)
    return out


def require_cuda():
    import pytest
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
