"""The gradients of the chunked form (tests/chunk_bwd_model.py) equal the pinned per-token gradient
oracle in float64: the algebra a chunked backward kernel would follow is right before any such
kernel exists. Chunk sizes 16 and 64, sequences that end in a partial chunk, with and without
initial and final states."""

import numpy as np
import pytest

from chunk_bwd_model import chunked_bwd
from oracle.backward import kda_bwd

NAMES = ("dq", "dk", "dv", "dlog_g", "dbeta", "dh0")


def _case(seed, B, T, H, dk, dv, states=True):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q = rng.standard_normal((B, T, H, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    return dict(q=q, k=k, v=rng.standard_normal((B, T, H, dv)),
                log_g=-np.logaddexp(0.0, rng.standard_normal((B, T, H, dk)) - 1.0),
                beta=1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H)))),
                do=rng.standard_normal((B, T, H, dv)),
                h0=rng.standard_normal((B, H, dk, dv)) * 0.3 if states else None,
                dhT=rng.standard_normal((B, H, dk, dv)) if states else None)


@pytest.mark.parametrize("C,T,states", [(16, 50, True), (16, 64, False), (64, 150, True),
                                        (64, 40, True)])
def test_chunked_gradients_equal_the_oracle(C, T, states):
    c = _case(100 + C + T, B=2, T=T, H=2, dk=8, dv=6, states=states)
    args = (c["q"], c["k"], c["v"], c["log_g"], c["beta"], c["do"])
    got = chunked_bwd(*args, dhT=c["dhT"], h0=c["h0"], C=C)
    ref = kda_bwd(*args, dhT=c["dhT"], h0=c["h0"])
    for name, x, r in zip(NAMES, got, ref):
        err = np.linalg.norm(x - r) / max(np.linalg.norm(r), 1e-300)
        assert err < 1e-10, (name, err)
