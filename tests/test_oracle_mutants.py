"""The pins must catch plausible mistakes in the oracle.

Each case copies oracle/mss_oracle.c, plants one mistake (a dropped term, a
wrong sign, a swapped operand, a wrong index or order), builds the copy and
runs the pin tests against it in a subprocess.  The pins must fail for every
mutant and pass for the unmodified source.  CPU only; nothing here touches
the CUDA path.
"""
import concurrent.futures
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "mss_oracle.c")

MUTANTS = {
    "drop_input_term": ("h[n] = abar[n] * h[n] + bx[n];", "h[n] = abar[n] * h[n];"),
    "exponent_sign": ("abar[n] = exp(dt * a);", "abar[n] = exp(-dt * a);"),
    "readout_before_update": (
        "h[n] = abar[n] * h[n] + bx[n];\n        acc += c[n] * h[n];",
        "acc += c[n] * h[n];\n        h[n] = abar[n] * h[n] + bx[n];"),
    "B_and_C_swapped": ("bx[n] = w * (double)B_bt[n * L] * u;", "bx[n] = w * (double)C_bt[n * L] * u;"),
    "input_rule_without_step": ("expm1(dt * a) / a : dt;", "expm1(dt * a) / a : 1.0;"),
    "zoh_ignored": ("? expm1(dt * a) / a : dt;", "? dt : dt;"),
    "zoh_second_order_sign": ("? expm1(dt * a) / a : dt;", "? -expm1(-dt * a) / a : dt;"),
    "zoh_zero_A_limit": ("(zoh_input && a != 0.0) ? expm1(dt * a) / a : dt;",
                         "zoh_input ? (a != 0.0 ? expm1(dt * a) / a : 0.0) : dt;"),
    "softplus_drops_one": ("return log1p(exp(s));", "return log(exp(s));"),
    "softplus_positive_branch": ("return s + log1p(exp(-s));", "return log1p(exp(-s));"),
    "bias_dropped": ("double s = delta_raw + bias;", "double s = delta_raw;"),
    "skip_dropped": ("double out = recurrence_step(h, abar, bx, c, N) + Dd * ut;",
                     "double out = recurrence_step(h, abar, bx, c, N);"),
    "gate_is_sigmoid": ("return z / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(-z));"),
    "state_not_reset_per_row": ("        for (int64_t n = 0; n < N; ++n)\n            h[n] = j->initial_state ? j->initial_state[row * N + n] : 0.0;\n        for (int64_t t = 0; t < L; ++t) {\n            const double ut = K",
                                "        for (int64_t t = 0; t < L; ++t) {\n            const double ut = K"),
    "initial_state_ignored": ("h[n] = j->initial_state ? j->initial_state[row * N + n] : 0.0;\n        for (int64_t t = 0; t < L; ++t) {\n            const double ut = K",
                              "h[n] = 0.0;\n        for (int64_t t = 0; t < L; ++t) {\n            const double ut = K"),
    "bwd_initial_state_ignored": ("h[n] = j->initial_state ? j->initial_state[row * N + n] : 0.0;\n        for (int64_t t = 0; t < L; ++t) {\n            const double s =",
                                  "h[n] = 0.0;\n        for (int64_t t = 0; t < L; ++t) {\n            const double s ="),
    "decode_B_token_stride": ("j->B + b * N, j->C + b * N, 1, N,", "j->B + b * N, j->C + b * N, N, N,"),
    "B_batch_index": ("const float *B_b = j->B + b * N * L;", "const float *B_b = j->B;"),
    "conv_taps_reversed": ("acc += (double)w[k] * ext[t + k];", "acc += (double)w[K - 1 - k] * ext[t + k];"),
    "conv_bias_dropped": ("        double acc = cb;\n", "        double acc = 0.0;\n"),
    "conv_without_silu": ("uc[t] = mss_oracle_silu(uc[t]);", "uc[t] = uc[t];"),
    "conv_state_out_offset": ("j->conv_state_out[row * (K - 1) + k] = ext[L + k];",
                              "j->conv_state_out[row * (K - 1) + k] = ext[L + k - 1];"),
    "conv_decode_no_shift": ("                cs[k] = cs[k + 1];\n", "                cs[k] = cs[k];\n"),
    "bwd_no_state_propagation": ("gh[n] *= atn; /* dLoss/dh_{t-1} */", "gh[n] *= 1.0;"),
    "bwd_softplus_derivative": ("ddt * (j->softplus_flag ? sigmoid(ss[t]) : 1.0)",
                                "ddt * (j->softplus_flag ? sigmoid(-ss[t]) : 1.0)"),
    "bwd_dB_without_u": ("j->dB[(b * N + n) * L + t] += gh[n] * wtn * ut;", "j->dB[(b * N + n) * L + t] += gh[n] * wtn;"),
    "bwd_dC_previous_state": ("j->dC[(b * N + n) * L + t] += dr * h[(t + 1) * N + n];",
                              "j->dC[(b * N + n) * L + t] += dr * h[t * N + n];"),
    "bwd_zoh_dA_sign": ("(dt * atn - wtn) / An", "(dt * atn + wtn) / An"),
    "bwd_gate_derivative": ("(sg + zt * sg * (1.0 - sg))", "(sg + zt * sg * sg)"),
    "ssd_group_index": ("g = h / (H / G);", "g = h % G;"),
    "ssd_no_decay": ("S[n * P + p] = a * S[n * P + p] + delta", "S[n * P + p] = S[n * P + p] + delta"),
    "ssd_input_without_step": ("+ delta * (double)Bt[n] * (double)xt[p];", "+ (double)Bt[n] * (double)xt[p];"),
    "ssd_state_layout": ("acc += (double)Ct[n] * S[n * P + p];", "acc += (double)Ct[n] * S[p * N + n];"),
    "ssd_bias_dropped": ("const double bias = j->bias ? (double)j->bias[h] : 0.0;", "const double bias = 0.0;"),
    "ssd_skip_dropped": ("double out = acc + Dh * (double)xt[p];", "double out = acc;"),
    "ssd_gate_dropped": ("out *= mss_oracle_silu((double)j->z[((b * L + t) * H + h) * P + p]);", "out *= 1.0;"),
    "ssd_initial_state_ignored": ("S[k] = j->initial_state ? j->initial_state[row * N * P + k] : 0.0;",
                                  "S[k] = 0.0;"),
    "ssd_last_state_row": ("j->last_state[row * N * P + k] = S[k];", "j->last_state[k] = S[k];"),
    "ssd_x_head_index": ("const float *xt = j->x + ((b * L + t) * H + h) * P;",
                         "const float *xt = j->x + ((b * L + t) * H) * P;"),
}


def _run_pins(lib_path):
    env = dict(os.environ, MSS_ORACLE_LIB=lib_path)
    return subprocess.run(
        [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
         os.path.join(ROOT, "tests", "test_oracle_pins.py"), os.path.join(ROOT, "tests", "test_oracle_ssd.py")],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


# mutant builds stay inside the repository (a git-ignored build folder)
BUILD_DIR = os.path.join(ROOT, "oracle", "_build", "mutants")


def _build(src_text, name):
    os.makedirs(BUILD_DIR, exist_ok=True)
    c = os.path.join(BUILD_DIR, f"{name}.{os.getpid()}.c")
    so = os.path.join(BUILD_DIR, f"{name}.{os.getpid()}.so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-fno-fast-math", "-ffp-contract=off",
                           "-fPIC", "-shared", "-o", so, c, "-lm", "-lpthread"])
    return so


def _pins_on(src_text, name):
    so = _build(src_text, name)
    try:
        return _run_pins(so)
    finally:
        for path in (so, so[:-3] + ".c"):
            if os.path.exists(path):
                os.remove(path)


@pytest.fixture(scope="module")
def pin_runs():
    """The pin run of the unmodified source and of every mutant whose site is
    found exactly once, run side by side (one subprocess per core)."""
    with open(SRC) as f:
        text = f.read()
    jobs = {"original": text}
    for name, (old, new) in MUTANTS.items():
        if text.count(old) == 1:
            jobs[name] = text.replace(old, new)
    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        futures = {name: ex.submit(_pins_on, src, name) for name, src in jobs.items()}
        return {name: fut.result() for name, fut in futures.items()}


def test_unmodified_source_passes(pin_runs):
    r = pin_runs["original"]
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, pin_runs):
    old, _ = MUTANTS[name]
    with open(SRC) as f:
        text = f.read()
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    r = pin_runs[name]
    assert r.returncode != 0, f"pins did not catch mutant {name}"
