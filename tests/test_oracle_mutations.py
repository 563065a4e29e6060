"""Planted mistakes: each plausible error in a copy of the oracle must fail a pin.

The copy is built on the CPU from gdn_oracle.c with one textual change, and the pin suite
runs against it in a subprocess.  The committed oracle is never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gdn_oracle.c")

MUTATIONS = {
    "error_sign": ("e[i] = beta * (v[i] - vhat[i]);", "e[i] = beta * (v[i] + vhat[i]);"),
    "no_decay": ("S[(size_t)i * dk + j] *= alpha;", "S[(size_t)i * dk + j] *= 1.0;"),
    "read_before_decay": ("acc += S[(size_t)i * dk + j] * k[j];",
                          "acc += S[(size_t)i * dk + j] * k[j] / alpha;"),
    "transposed_write": ("S[(size_t)i * dk + j] += e[i] * k[j];",
                         "S[(size_t)i * dk + j] += e[j % dv] * k[i % dk];"),
    "read_before_write": ("acc += S[(size_t)i * dk + j] * (q_scale * q[j]);",
                          "acc += (S[(size_t)i * dk + j] - e[i] * k[j]) * (q_scale * q[j]);"),
    "conv_taps_reversed": ("acc += w[i] * xv;", "acc += w[3 - i] * xv;"),
    "no_silu_after_conv": ("out[t * stride] = oracle_silu(acc);", "out[t * stride] = acc;"),
    "softplus_wrong": ("log1p(exp(-fabs(x)))", "log1p(exp(-x))"),
    "rms_sum_not_mean": ("1.0 / sqrt(ss / dv + eps)", "1.0 / sqrt(ss + eps)"),
    "chunk_drops_diagonal": ("for (int s = 0; s <= t; ++s) {", "for (int s = 0; s < t; ++s) {"),
    "head_map_modulo": ("const int j = h / (hv / hq);", "const int j = h % hq;"),
    "k_channel_block": ("(long)hq * dk + (long)j * dk,", "(long)j * dk + 0 * (long)hq,"),
    "beta_from_a": ("beta[t] = oracle_sigmoid((double)b[", "beta[t] = oracle_sigmoid((double)a["),
    "conv_shift_wrong": ("o[0 * cconv + c] = or_load(conv_state, ((size_t)n * 3 + 1)",
                         "o[0 * cconv + c] = or_load(conv_state, ((size_t)n * 3 + 0)"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor for {name} not unique"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(text.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", str(lib),
                           str(mutant), "-lm"])
    env = dict(os.environ, GDN_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"planted mistake {name!r} passed every pin:\n{r.stdout[-2000:]}"
