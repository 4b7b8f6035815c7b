"""Plant plausible mistakes in a copy of the oracle's C source and check that the
pin suite catches every one of them (no GPU).

Each mutant is built from a textual edit of ``oracle/gdn_oracle.c`` into a
temporary directory and exercised in a child process, so a mutant that reads
out of bounds cannot take the test process down with it."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gdn_oracle.c")

MUTANTS = {
    "decay_dropped": ("const double alpha = exp(g[t * HV + h]);", "const double alpha = 1.0;"),
    "decay_after_read": ("- alpha * bt * Sk[r] * kh[c]", "- bt * Sk[r] * kh[c]"),
    "write_sign": ("+ bt * vt[r] * kh[c];", "- bt * vt[r] * kh[c];"),
    "erase_missing": ("- alpha * bt * Sk[r] * kh[c]", "- 0.0 * Sk[r] * kh[c]"),
    "output_transposed_read": ("acc += S[r * Dk + c] * qh[c];", "acc += S[c * Dk + r] * qh[c];"),
    "read_with_query": ("acc += S[r * Dk + c] * kh[c];\n                Sk[r] = acc;",
                        "acc += S[r * Dk + c] * qh[c];\n                Sk[r] = acc;"),
    "beta_complement": ("const double bt = beta[t * HV + h];", "const double bt = 1.0 - beta[t * HV + h];"),
    "gate_no_exp": ("g[i] = -exp(A_log[h]) *", "g[i] = -A_log[h] *"),
    "softplus_sign": ("log1p(exp(-fabs(x)))", "log1p(exp(fabs(x)))"),
    "sigmoid_sign": ("1.0 / (1.0 + exp(-x))", "1.0 / (1.0 + exp(x))"),
    "gqa_round_robin": ("const int64_t hk = h / group;", "const int64_t hk = h % HK;"),
    "h0_transposed": ("h0[((n * HV + h) * Dk + c) * Dv + r]", "h0[((n * HV + h) * Dv + r) * Dk + c]"),
    "l2norm_eps_outside": ("1.0 / sqrt(ss + 1e-6)", "1.0 / (sqrt(ss) + 1e-6)"),
    "scale_dropped": ("ot[r] = scale * acc;", "ot[r] = acc;"),
    "conv_taps_reversed": ("acc += w[c * 4 + i] * win[i];", "acc += w[c * 4 + 3 - i] * win[i];"),
    "conv_state_not_shifted": ("win[1] = win[2];", "win[1] = win[3];"),
    "conv_silu_sign": ("acc * oracle_sigmoid(acc)", "acc * oracle_sigmoid(-acc)"),
    "norm_eps_outside": ("1.0 / sqrt(ss / (double)D + eps)", "1.0 / (sqrt(ss / (double)D) + eps)"),
    "norm_sum_not_mean": ("1.0 / sqrt(ss / (double)D + eps)", "1.0 / sqrt(ss + eps)"),
    "norm_weight_not_centred": ("* (1.0 + w[j]) *", "* w[j] *"),
    "gate_sign": ("oracle_sigmoid(z[r * D + j])", "oracle_sigmoid(-z[r * D + j])"),
}

_CHILD = r"""
import json, sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import oracle, pins
orc = oracle.OracleLib({lib!r})
failed = []
for p in pins.ALL_PINS:
    try:
        p(orc)
    except AssertionError:
        failed.append(p.__name__)
    except Exception as e:
        failed.append(p.__name__ + ':' + type(e).__name__)
print(json.dumps(failed))
"""


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    import oracle
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/found"
    msrc = tmp_path / "mutant.c"
    msrc.write_text(src.replace(old, new))
    lib = oracle.build(str(msrc), str(tmp_path / "libmutant.so"), force=True)
    code = _CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), lib=lib)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    if r.returncode != 0:
        return  # the mutant crashed the pin suite: caught
    failed = json.loads(r.stdout.strip().splitlines()[-1])
    assert failed, f"no pin caught mutant {name}"
