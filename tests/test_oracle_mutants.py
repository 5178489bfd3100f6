"""Plant plausible mistakes in a COPY of the oracle (on the CPU) and require
each one to trip at least one pin. This is what shows the pins would catch a
dropped term, a wrong sign, a wrong divisor, a wrong index or a swapped
operand in the oracle."""
import os

import pytest

import oracle
import oracle_pins
from oracle import build as oracle_build

with open(oracle_build.SOURCE) as _f:
    SOURCE = _f.read()

MUTANTS = {
    "rms divisor D-1": ("double mean_sq = sum_sq / (double)dim;",
                        "double mean_sq = sum_sq / (double)(dim - 1);"),
    "rms divisor D+1": ("double mean_sq = sum_sq / (double)dim;",
                        "double mean_sq = sum_sq / (double)(dim + 1);"),
    "rms drops eps": ("sqrt(mean_sq + eps)", "sqrt(mean_sq)"),
    "rms eps outside sqrt": ("sqrt(mean_sq + eps)", "(sqrt(mean_sq) + eps)"),
    "rms drops weight": ("y_row[j] = v / rms * weight;", "y_row[j] = v / rms;"),
    "rms squares weight": ("y_row[j] = v / rms * weight;",
                           "y_row[j] = v / rms * weight * weight;"),
    "rms multiplies by rms": ("y_row[j] = v / rms * weight;",
                              "y_row[j] = v * rms * weight;"),
    "rms sums |x| not x^2": ("sum_sq += v * v;", "sum_sq += fabs(v);"),
    "rms ignores row offset": (
        "double v = decode_element(x, dtype, first + j);\n        double weight = (w != NULL) ? decode_element(w, dtype, j) : 1.0;\n        y_row[j] = v / rms",
        "double v = decode_element(x, dtype, j);\n        double weight = (w != NULL) ? decode_element(w, dtype, j) : 1.0;\n        y_row[j] = v / rms"),
    "rms weight reversed": (
        "double weight = (w != NULL) ? decode_element(w, dtype, j) : 1.0;\n        y_row[j] = v / rms",
        "double weight = (w != NULL) ? decode_element(w, dtype, dim - 1 - j) : 1.0;\n        y_row[j] = v / rms"),
    "row stride ignored": ("const int64_t first = row * row_stride;\n    double sum_sq",
                           "const int64_t first = row * dim;\n    double sum_sq"),
    "ln mean divisor D-1": ("double mean = sum / (double)dim;",
                            "double mean = sum / (double)(dim - 1);"),
    "ln sample variance": ("double var = sum_dev_sq / (double)dim;",
                           "double var = sum_dev_sq / (double)(dim - 1);"),
    "ln raw second moment": ("double dev = decode_element(x, dtype, first + i) - mean;",
                             "double dev = decode_element(x, dtype, first + i);"),
    "ln output misses mean": ("y_row[j] = (v - mean) / denom * weight + bias;",
                              "y_row[j] = v / denom * weight + bias;"),
    "ln output adds mean": ("y_row[j] = (v - mean) / denom * weight + bias;",
                            "y_row[j] = (v + mean) / denom * weight + bias;"),
    "ln bias sign": ("y_row[j] = (v - mean) / denom * weight + bias;",
                     "y_row[j] = (v - mean) / denom * weight - bias;"),
    "ln bias scaled by weight": ("y_row[j] = (v - mean) / denom * weight + bias;",
                                 "y_row[j] = ((v - mean) / denom + bias) * weight;"),
    "ln drops eps": ("double denom = sqrt(var + eps);", "double denom = sqrt(var);"),
    "ln eps outside sqrt": ("double denom = sqrt(var + eps);", "double denom = sqrt(var) + eps;"),
    "ln weight and bias swapped": (
        "double weight = (w != NULL) ? decode_element(w, dtype, j) : 1.0;\n        double bias = (b != NULL) ? decode_element(b, dtype, j) : 0.0;",
        "double weight = (b != NULL) ? decode_element(b, dtype, j) : 1.0;\n        double bias = (w != NULL) ? decode_element(w, dtype, j) : 0.0;"),
    "dual query uses key weight": (
        "oracle_rms_norm(q, dtype, q_rows, q_dim, q_stride, wq, eps, yq,",
        "oracle_rms_norm(q, dtype, q_rows, q_dim, q_stride, wk, eps, yq,"),
    "bf16 decoded with wrong shift": ("(uint32_t)half << 16", "(uint32_t)half << 15"),
    "add stores the unrounded sum": ("h_row[i] = store_round(s, dtype);", "h_row[i] = s;"),
    "add ignores the residual": (
        "double s = decode_element(x, dtype, row * x_stride + i) +\n"
        "                   decode_element(r, dtype, row * r_stride + i);",
        "double s = decode_element(x, dtype, row * x_stride + i);"),
    "add subtracts the residual": (
        "double s = decode_element(x, dtype, row * x_stride + i) +\n",
        "double s = decode_element(x, dtype, row * x_stride + i) -\n"),
    "add residual read with x stride": ("decode_element(r, dtype, row * r_stride + i)",
                                        "decode_element(r, dtype, row * x_stride + i)"),
    "bf16 store truncates": (
        "if (dropped > 0x8000u || (dropped == 0x8000u && kept_lsb)) u += 0x10000u;", ""),
    "bf16 store ties away from zero": (
        "if (dropped > 0x8000u || (dropped == 0x8000u && kept_lsb)) u += 0x10000u;",
        "if (dropped >= 0x8000u) u += 0x10000u;"),
    "add rms divisor D-1": ("double mean_h2 = sum_h2 / (double)dim;",
                            "double mean_h2 = sum_h2 / (double)(dim - 1);"),
    "add rms drops weight": ("y_row[j] = h_row[j] / rms_h * weight;",
                             "y_row[j] = h_row[j] / rms_h;"),
    "gated silu sign": ("double silu = gate / (1.0 + exp(-gate));",
                        "double silu = gate / (1.0 + exp(gate));"),
    "gated sigmoid only": ("double silu = gate / (1.0 + exp(-gate));",
                           "double silu = 1.0 / (1.0 + exp(-gate));"),
    "gated drops eps": ("double rms_x = sqrt(mean_x2 + eps);", "double rms_x = sqrt(mean_x2);"),
    "gated gate read with x stride": ("decode_element(z, dtype, row * z_stride + j)",
                                      "decode_element(z, dtype, row * x_stride + j)"),
    "gated drops weight": ("y_row[j] = xv / rms_x * weight * silu;",
                           "y_row[j] = xv / rms_x * silu;"),
    "rope sign flipped": ("y_row[a] = n_row[a] * c - n_row[b] * s;",
                          "y_row[a] = n_row[a] * c + n_row[b] * s;"),
    "rope cos and sin swapped": ("double c = cos(theta), s = sin(theta);",
                                 "double c = sin(theta), s = cos(theta);"),
    "rope exponent without 2": ("pow(base, -2.0 * (double)i / (double)dims)",
                                "pow(base, -(double)i / (double)dims)"),
    "rope position per row not token": ("double pos = (double)(offset + r / heads);",
                                        "double pos = (double)(offset + r);"),
    "rope ignores offset": ("double pos = (double)(offset + r / heads);",
                            "double pos = (double)(r / heads);"),
    "rope ignores scale": ("double theta = pos * scale * f;", "double theta = pos * f;"),
    "rope partner off by one": ("int64_t b = traditional ? 2 * i + 1 : i + half;",
                                "int64_t b = traditional ? 2 * i + 1 : i + half - 1;"),
    "rope ignores the layout flag": ("int64_t a = traditional ? 2 * i : i;\n"
                                     "        int64_t b = traditional ? 2 * i + 1 : i + half;",
                                     "int64_t a = i;\n        int64_t b = i + half;"),
    "rope rotates the whole row": ("const int64_t half = dims / 2;",
                                   "const int64_t half = dim / 2;"),
    "rope ignores the frequency table": (
        "double f = (inv_freq != NULL) ? (double)inv_freq[i]\n"
        "                                      : pow(",
        "double f = (inv_freq != NULL && 0) ? (double)inv_freq[i]\n"
        "                                      : pow("),
    "rope key rows use query heads": (
        "return rms_rope_rows(k, dtype, k_rows, k_dim, k_stride, wk, (double)eps, heads_k,",
        "return rms_rope_rows(k, dtype, k_rows, k_dim, k_stride, wk, (double)eps, heads_q,"),
}


def _mutant(tmp_path_factory, name):
    old, new = MUTANTS[name]
    assert SOURCE.count(old) == 1, f"mutation site for {name!r} must be unique"
    d = tmp_path_factory.mktemp("mutant")
    src = os.path.join(d, "mutant.c")
    with open(src, "w") as f:
        f.write(SOURCE.replace(old, new))
    return oracle.Oracle(oracle_build.compile_source(src, os.path.join(d, "libmutant.so")))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path_factory, name):
    orc = _mutant(tmp_path_factory, name)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError, FloatingPointError, ZeroDivisionError) as e:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name!r}"
