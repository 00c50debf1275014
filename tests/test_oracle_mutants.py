"""Plants plausible mistakes in a temporary copy of the oracle's C source and
checks that the pin suite (test_oracle_pins.py) fails for each one: evidence
that the pins would notice a dropped term, a wrong sign, index or operand.
CPU only; the product path is not involved."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = open(os.path.join(ROOT, "oracle", "gdn_oracle.c")).read()

_DECAY = ("for (int i = 0; i < dk; ++i)\n                    for (int j = 0; j < dv; ++j) S[i * dv + j] *= al;\n")
_M = ("for (int j = 0; j < dv; ++j) {\n                    m[j] = 0.0;\n"
      "                    for (int i = 0; i < dk; ++i) m[j] += S[i * dv + j] * kk[i];\n                }\n")
_UPD = "for (int i = 0; i < dk; ++i)\n                    for (int j = 0; j < dv; ++j) S[i * dv + j] += kk[i] * d[j];\n"
_RD = ("for (int j = 0; j < dv; ++j) {\n                    double acc = 0.0;\n"
       "                    for (int i = 0; i < dk; ++i) acc += S[i * dv + j] * qq[i];\n"
       "                    o[(row * Hv + h) * dv + j] = acc;\n                }\n")
_IND = "                "

MUTANTS = {
    "key read before the decay": (_DECAY + _IND + _M, _M + _IND + _DECAY),
    "readout on the old state": (_UPD + _IND + _RD, _RD + _IND + _UPD),
    "wrong sign in delta": ("d[j] = be * (vv[j] - m[j]);", "d[j] = be * (vv[j] + m[j]);"),
    "outer product transposed": ("S[i * dv + j] += kk[i] * d[j];", "S[i * dv + j] += kk[j % dk] * d[i % dv];"),
    "GQA map h % Hk": ("k + (row * Hk + h / G) * dk;\n                const double* qq = q + (row * Hk + h / G) * dk;\n                const double* vv = v + (row * Hv + h) * dv;\n                const double al = alpha[row * Hv + h], be = beta[row * Hv + h];\n                double* S = state_pool + ((size_t)slots[b] * Hv + h) * dk * dv;\n                for (int i = 0; i < dk; ++i)\n                    for (int j = 0; j < dv; ++j) S[i * dv + j] *= al;",
                       "k + (row * Hk + h % Hk) * dk;\n                const double* qq = q + (row * Hk + h % Hk) * dk;\n                const double* vv = v + (row * Hv + h) * dv;\n                const double al = alpha[row * Hv + h], be = beta[row * Hv + h];\n                double* S = state_pool + ((size_t)slots[b] * Hv + h) * dk * dv;\n                for (int i = 0; i < dk; ++i)\n                    for (int j = 0; j < dv; ++j) S[i * dv + j] *= al;"),
    "conv taps reversed": ("conv_w[(size_t)ch * W + j]", "conv_w[(size_t)ch * W + (W - 1 - j)]"),
    "conv history not rolled": ("for (int r = 0; r < W - 1; ++r) st[(size_t)r * C + ch] = hist[T + r];", "(void)0;"),
    "conv roll off by one": ("st[(size_t)r * C + ch] = hist[T + r];", "st[(size_t)r * C + ch] = hist[T - 1 + r];"),
    "no SiLU on V": ("s[(size_t)t * C + ch] = silu(u);", "s[(size_t)t * C + ch] = ch < 2 * Hk * dk ? silu(u) : u;"),
    "Q and K blocks swapped": ("const double* st_q = s + (size_t)t * C;\n            const double* st_k = st_q + Hk * dk;",
                               "const double* st_k = s + (size_t)t * C;\n            const double* st_q = st_k + Hk * dk;"),
    "L2 eps outside the root": ("nq = 1.0 / sqrt(sq + c->l2_eps), nk = 1.0 / sqrt(sk + c->l2_eps);",
                                "nq = 1.0 / fmax(sqrt(sq), c->l2_eps), nk = 1.0 / fmax(sqrt(sk), c->l2_eps);"),
    "q scale dropped": ("st_q[h * dk + i] * nq * qs;", "st_q[h * dk + i] * nq;"),
    "softplus replaced by exp": ("softplus(from_bf16(a[i]) + (double)dt_bias[h])", "exp(from_bf16(a[i]) + (double)dt_bias[h])"),
    "gate sign flipped": ("const double g = -exp((double)A_log[h])", "const double g = exp(-(double)A_log[h])"),
    "beta of -b": ("beta[i] = sigmoid(from_bf16(b[i]));", "beta[i] = sigmoid(-from_bf16(b[i]));"),
    "RMS over the sum": ("sqrt(ss / dv + c->rms_eps)", "sqrt(ss + c->rms_eps)"),
    "norm weight dropped": ("o[i] * inv * from_bf16(norm_w[j]) * silu", "o[i] * inv * silu"),
    "sigmoid gate instead of SiLU": ("* silu(from_bf16(z[i]));", "* sigmoid(from_bf16(z[i]));"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    assert SRC.count(old) >= 1, f"mutation site for {name!r} no longer in the oracle source"
    shutil.copytree(os.path.join(ROOT, "oracle"), tmp_path / "oracle",
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    pkg = tmp_path / "gated_delta_rule_102_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "gated_delta_rule_102_b200", "synth.py"), pkg / "synth.py")
    (pkg / "__init__.py").write_text("")
    (tmp_path / "tests").mkdir()
    for f in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), tmp_path / "tests" / f)
    (tmp_path / "oracle" / "gdn_oracle.c").write_text(SRC.replace(old, new, 1))
    # the mutant must compile, so that a failing pin run means a caught mistake
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o",
                           str(tmp_path / "oracle" / "liboracle.so"),
                           str(tmp_path / "oracle" / "gdn_oracle.c"), "-lm"])
    p = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_oracle_pins.py"], cwd=tmp_path, capture_output=True, text=True,
                       timeout=300)
    assert p.returncode == 1, f"pins did not catch {name!r}:\n{p.stdout[-2000:]}"
