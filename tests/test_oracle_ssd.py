"""Pins of the structured-state-space-duality (Mamba-2) oracle.

CPU only.  The SSD recurrence (a scalar A per head, an N x P state, B and C
shared by the heads of a group) is checked against the pinned Mamba-1
oracle (each of a head's P channels is a selective SSM whose N states share
the head's decay), against the materialised 1-semiseparable matrix, against
the chunked algorithm the pages describe (quadratic within chunks, linear
recurrence across them), and against causal linear attention (no decay).
"""
import numpy as np
import pytest

import oracle
from oracle import scans


def _ssd_inputs(seed, batch=2, L=24, H=4, P=3, G=2, N=5):
    rng = np.random.default_rng(seed)
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    return dict(x=f(batch, L, H, P), dt=(0.5 * f(batch, L, H)).astype(np.float32),
                A=(-rng.uniform(0.2, 2.0, H)).astype(np.float32), B=f(batch, L, G, N), C=f(batch, L, G, N),
                D=f(H), z=f(batch, L, H, P), dt_bias=(0.3 * f(H)).astype(np.float32))


def test_ssd_head_is_mamba1_channels_sharing_the_decay():
    """A head's channel p is a Mamba-1 channel with input x[..., p], the head's
    step size and A_n = A_h for every state: the two oracles agree bitwise
    (same operations in the same order)."""
    inp = _ssd_inputs(200)
    h0 = np.random.default_rng(201).standard_normal((2, 4, 5, 3))
    y, last = oracle.ssd_fwd(**inp, initial_state=h0)
    batch, L, H, P = inp["x"].shape
    G, N = inp["B"].shape[2:]
    for h in range(H):
        g = h // (H // G)
        for p in range(P):
            y1, last1 = oracle.scan_fwd(
                u=np.ascontiguousarray(inp["x"][:, :, h, p])[:, None, :],
                delta=np.ascontiguousarray(inp["dt"][:, :, h])[:, None, :],
                A=np.full((1, N), inp["A"][h], dtype=np.float32),
                B=np.ascontiguousarray(np.transpose(inp["B"][:, :, g, :], (0, 2, 1))),
                C=np.ascontiguousarray(np.transpose(inp["C"][:, :, g, :], (0, 2, 1))),
                D=inp["D"][h:h + 1], z=np.ascontiguousarray(inp["z"][:, :, h, p])[:, None, :],
                delta_bias=inp["dt_bias"][h:h + 1], initial_state=np.ascontiguousarray(h0[:, h, :, p])[:, None, :])
            assert np.array_equal(y1[:, 0, :], y[:, :, h, p])
            assert np.array_equal(last1[:, 0, :], last[:, h, :, p])


def _head(inp, b, h):
    """One head's a, delta, B, C, X as fp64 (no bias/softplus: dt used as is)."""
    G = inp["B"].shape[2]
    g = h // (inp["x"].shape[2] // G)
    delta = inp["dt"][b, :, h].astype(np.float64)
    a = np.exp(delta * float(inp["A"][h]))
    return (a, delta, inp["B"][b, :, g].astype(np.float64), inp["C"][b, :, g].astype(np.float64),
            inp["x"][b, :, h].astype(np.float64))


def test_ssd_is_the_semiseparable_matrix():
    inp = _ssd_inputs(202)
    inp["dt"] = np.abs(inp["dt"]) + np.float32(0.05)
    y, _ = oracle.ssd_fwd(**{k: v for k, v in inp.items() if k not in ("D", "z", "dt_bias")}, softplus_flag=False)
    for b in range(2):
        for h in range(4):
            a, delta, B, C, X = _head(inp, b, h)
            np.testing.assert_allclose(y[b, :, h], scans.ssd_matrix(a, delta, B, C) @ X, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("chunk", [1, 5, 8, 24, 100])
def test_ssd_chunked_algorithm(chunk):
    """Quadratic within chunks plus the recurrence of chunk states gives the
    recurrence, including the final state, for any chunk size."""
    inp = _ssd_inputs(203)
    inp["dt"] = np.abs(inp["dt"]) + np.float32(0.05)
    y, last = oracle.ssd_fwd(**{k: v for k, v in inp.items() if k not in ("D", "z", "dt_bias")},
                             softplus_flag=False)
    for b in range(2):
        for h in range(4):
            a, delta, B, C, X = _head(inp, b, h)
            Yc, S = scans.ssd_chunked(a, delta, B, C, X, chunk)
            np.testing.assert_allclose(Yc, y[b, :, h], rtol=1e-11, atol=1e-11)
            np.testing.assert_allclose(S, last[b, h], rtol=1e-11, atol=1e-11)


def test_ssd_without_decay_is_causal_linear_attention():
    """With A = 0 (Abar = I) and unit steps the map is causal linear attention:
    y_t = sum_{i <= t} (C_t . B_i) x_i."""
    inp = _ssd_inputs(204, G=1)
    inp["A"] = np.zeros(4, dtype=np.float32)
    inp["dt"] = np.ones_like(inp["dt"])
    y, _ = oracle.ssd_fwd(x=inp["x"], dt=inp["dt"], A=inp["A"], B=inp["B"], C=inp["C"], softplus_flag=False)
    for b in range(2):
        scores = np.tril(inp["C"][b, :, 0].astype(np.float64) @ inp["B"][b, :, 0].astype(np.float64).T)
        for h in range(4):
            np.testing.assert_allclose(y[b, :, h], scores @ inp["x"][b, :, h].astype(np.float64), rtol=1e-12,
                                       atol=1e-12)
