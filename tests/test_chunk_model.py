"""The float64 model of the chunked prefill (tests/chunk_model.py) equals the pinned per-token
oracle: the chunk algebra the tcgen05 kernels follow (block-midpoint anchored factors, the UT
transform, the WY factors and the state pass) is the recurrence, up to float64 rounding. Sequences
end in a partial chunk; the state starts from h0."""

import numpy as np
import pytest

import oracle
from chunk_model import chunk_forward


@pytest.mark.parametrize("T,mu", [(64, 0.0), (150, 0.0), (200, 2.0)])
def test_chunk_model_equals_the_oracle(T, mu):
    rng = np.random.default_rng(40 + T)
    d = 16
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q = unit(rng.standard_normal((1, T, 1, d))).astype(np.float32)
    k = unit(rng.standard_normal((1, T, 1, d))).astype(np.float32)
    v = rng.standard_normal((1, T, 1, d)).astype(np.float32)
    lg = (-np.logaddexp(0.0, rng.standard_normal((1, T, 1, d)) + mu)).astype(np.float32)
    beta = (1.0 / (1.0 + np.exp(-rng.standard_normal((1, T, 1))))).astype(np.float32)
    h0 = (rng.standard_normal((1, 1, d, d)) * 0.1).astype(np.float32)
    o_ref, h_ref = oracle.kda_fwd(q, k, v, lg, beta, h0=h0)
    o, S = chunk_forward(q[0, :, 0], k[0, :, 0], v[0, :, 0], lg[0, :, 0], beta[0, :, 0],
                         h0[0, 0])
    eo = np.linalg.norm(o - o_ref[0, :, 0]) / np.linalg.norm(o_ref[0, :, 0])
    eh = np.linalg.norm(S - h_ref[0, 0]) / np.linalg.norm(h_ref[0, 0])
    assert eo < 1e-12 and eh < 1e-12, (eo, eh)
