"""Plant plausible mistakes in private copies of the plain C oracle's source
(on the CPU), compile each copy and check that at least one pin fails for it:
the pins catch a dropped scale, a wrong sign, a swapped or misindexed operand
and a mis-decoded input in the C statement too."""
import shutil
import subprocess

import pytest

from oracle import build_oracle, lora_oracle_c
from tests import oracle_pins

SRC = build_oracle.SRC

# (name, text in the source, its replacement); the first occurrence is replaced
MUTATIONS = [
    ("drop_scale", "Z[i] = Z[i] + s * bax[i];", "Z[i] = Z[i] + bax[i];"),
    ("sigmoid_sign", "return 1.0 / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(z));"),
    ("silu_grad_sign", "return g * (1.0 + z * (1.0 - g));", "return g * (1.0 - z * (1.0 - g));"),
    ("dx_sign", "const double g = dzw[i] + s * ua[i];", "const double g = dzw[i] - s * ua[i];"),
    ("dA_no_scale", "for (int64_t i = 0; i < r * d_in; ++i) dA[i] = s * dA[i];", ""),
    ("dB_wrong_operand", "matmul_tn(dZ, T, dB, M, d_out, r);", "matmul_tn(dZ, U, dB, M, d_out, r);"),
    ("swiglu_swapped", "else Y[i] = silu(Z[i]) * Z_up[i];", "else Y[i] = silu(Z_up[i]) * Z[i];"),
    ("swiglu_up_grad", "dZ_up[i] = dY[i] * silu(Z[i]);", "dZ_up[i] = dY[i] * Z[i];"),
    ("swiglu_dx_not_summed", "dX[i] = add ? dX[i] + g : g;", "dX[i] = g;"),
    ("bf16_shift15", "(uint32_t)bits[i] << 16", "(uint32_t)bits[i] << 15"),
    ("linear_reversed_k", "acc += q->a[m * q->K + k] * q->b[n * q->K + k];",
     "acc += q->a[m * q->K + k] * q->b[n * q->K + (q->K - 1 - k)];"),
    ("matmul_tn_transposed", "const double a = q->a[k * q->M + m];", "const double a = q->a[m * q->K + k];"),
]


def _build_variant(tmp_path, name, text):
    src = tmp_path / f"{name}.c"
    src.write_text(text)
    lib = tmp_path / f"lib{name}.so"
    cc = shutil.which("gcc") or shutil.which("cc")
    subprocess.run([cc, "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", str(src), "-o", str(lib), "-lm"],
                   check=True)
    return lora_oracle_c.COracle(str(lib))


def test_unmodified_copy_passes(tmp_path):
    o = _build_variant(tmp_path, "unmodified", open(SRC).read())
    assert oracle_pins.run_all(o) == []


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_in_c_oracle_is_caught(tmp_path, name, old, new):
    text = open(SRC).read()
    assert old in text, f"mutation site of {name} not found in the C oracle"
    o = _build_variant(tmp_path, name, text.replace(old, new, 1))
    assert oracle_pins.run_all(o), f"no pin caught {name}"

