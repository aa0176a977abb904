"""The seeded input generator: determinism, bf16 rounding, value ranges."""
import numpy as np
import torch

from selective_state_space_mss_b200 import inputs


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.0078125 + 2**-9, 3.0e38, 1e-40],
                                 dtype=np.float32)])
    bits = inputs.to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)
    back = inputs.bf16_bits_to_f32(bits)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_generator_is_deterministic_and_in_range():
    a = inputs.scan_inputs(2, 8, 16, 64, "bf16", 1234, "normal")
    b = inputs.scan_inputs(2, 8, 16, 64, "bf16", 1234, "normal")
    for k in ("u", "delta", "z", "B", "C"):
        assert np.array_equal(a[k].stored, b[k].stored)
        assert a[k].stored.dtype == np.uint16
        assert np.array_equal(inputs.bf16_bits_to_f32(a[k].stored), a[k].values)
    assert np.array_equal(a["A"], -np.tile(np.arange(1, 17, dtype=np.float32), (8, 1)))
    # softplus(bias) lies in [1e-3, 1e-1]: check with the exact inverse relation
    dt = np.log1p(np.exp(a["delta_bias"].astype(np.float64)))
    assert np.all(dt > 0.9e-3) and np.all(dt < 1.1e-1)
    c = inputs.scan_inputs(2, 8, 16, 64, "bf16", 1235, "normal")
    assert not np.array_equal(a["u"].stored, c["u"].stored)


def test_workload_table():
    w = inputs.WORKLOADS[inputs.BENCH_WORKLOAD]
    assert (w.batch, w.dim, w.dstate, w.seqlen, w.dtype) == (4, 4096, 16, 4096, "bf16")
    assert inputs.WORKLOADS["s6-fwd-fp32-b1-d16-n4-l256"].dtype == "f32"
    small = inputs.workload_inputs("s6-fwd-fp32-b1-d16-n4-l256")
    assert small["u"].stored.dtype == np.float32 and small["u"].values.shape == (1, 16, 256)
    s = inputs.decode_step_inputs(4, 8, 16, "bf16", 1005, 3)
    assert s["B"].values.shape == (4, 16) and s["u"].values.shape == (4, 8)


def test_a_recipes():
    n = np.arange(1, 17, dtype=np.float32)
    for recipe in inputs.A_RECIPES:
        A = inputs.a_matrix(40, 16, recipe, 77)
        assert A.shape == (40, 16) and A.dtype == np.float32 and np.all(A < 0)
        geo = np.array([np.array_equal(A[d], (n * A[d, 0]).astype(np.float32)) for d in range(40)])
        if recipe in ("s4d-real", "scaled"):
            assert geo.all()
        elif recipe == "random":
            assert not geo.any() and A.min() >= -20.0 and A.max() <= -0.1
            assert len(np.unique(A[:, 0])) == 40
        else:
            # every 16 consecutive channels hold S4D-Real, random and scaled rows
            for d0 in range(0, 40 - 16 + 1):
                kinds = {0 if np.array_equal(A[d], -n) else (2 if geo[d] else 1) for d in range(d0, d0 + 16)}
                assert kinds == {0, 1, 2}
        if recipe == "scaled":
            assert len(np.unique(A[:, 0])) == 40
    # the A recipe leaves the other draws unchanged
    a = inputs.scan_inputs(2, 8, 16, 32, "bf16", 5, "normal")
    b = inputs.scan_inputs(2, 8, 16, 32, "bf16", 5, "normal", a_init="random")
    assert np.array_equal(a["D"], b["D"]) and np.array_equal(a["delta_bias"], b["delta_bias"])
    assert np.array_equal(a["u"].stored, b["u"].stored) and not np.array_equal(a["A"], b["A"])
