"""Plant plausible mistakes in copies of the oracle source and show the pins catch each.

Every mutant is compiled from a copy of ``oracle/vla_attn_oracle.cpp`` in a
temporary directory (the real oracle is never touched) and run through the pin
suite; the test passes only if at least one pin fails for every mutant.
"""
import os
import shutil
import subprocess

import pytest

import oracle
from oracle import build as oracle_build
from oracle_pins import ALL_PINS

# (name, original text, replacement) -- each a mistake someone could plausibly make.
MUTANTS = [
    ("scale_dropped", "s[j] = scale * dot;", "s[j] = dot;"),
    ("scale_squared", "s[j] = scale * dot;", "s[j] = scale * scale * dot;"),
    ("key_index_is_query_index", "const double* kj = k + j * tok_stride;",
     "const double* kj = k + (j == 0 ? 0 : j - 1) * tok_stride;"),
    ("no_normalisation", "oi[c] = acc / l;", "oi[c] = acc;"),
    ("value_channels_reversed", "acc += s[j] * v[j * tok_stride + c];",
     "acc += s[j] * v[j * tok_stride + (d - 1 - c)];"),
    ("last_key_dropped_from_softmax", "for (int j = 0; j < N; ++j) {\n    s[j] = std::exp(s[j] - m);",
     "for (int j = 0; j < N - 1; ++j) {\n    s[j] = std::exp(s[j] - m);"),
    ("no_max_subtraction", "s[j] = std::exp(s[j] - m);", "s[j] = std::exp(s[j]);"),
    ("sign_flip_logits", "s[j] = scale * dot;", "s[j] = -scale * dot;"),
    ("k_and_v_slots_swapped", "k[static_cast<size_t>(n) * d + c] = widen_bf16(row[hd + c]);",
     "k[static_cast<size_t>(n) * d + c] = widen_bf16(row[2 * hd + c]);"),
    ("head_offset_ignored", "const uint16_t* row = qkv + (b * N + n) * tok + h * d;",
     "const uint16_t* row = qkv + (b * N + n) * tok;"),
    ("weights_not_exponentiated_in_probs", "for (int j = 0; j < N; ++j) probs[j] = s[j] / l;",
     "for (int j = 0; j < N; ++j) probs[j] = s[j];"),
    ("ln_unbiased_variance", "const double var = ss / W;", "const double var = ss / (W - 1);"),
    ("ln_eps_dropped", "const double rstd = 1.0 / std::sqrt(var + eps);",
     "const double rstd = 1.0 / std::sqrt(var);"),
    ("ln_beta_dropped",
     "ym[i] = (widen_bf16(xm[i]) - mu) * rstd * widen_bf16(gamma[i]) + widen_bf16(beta[i]);",
     "ym[i] = (widen_bf16(xm[i]) - mu) * rstd * widen_bf16(gamma[i]);"),
    ("ln_mean_not_subtracted",
     "ym[i] = (widen_bf16(xm[i]) - mu) * rstd * widen_bf16(gamma[i]) + widen_bf16(beta[i]);",
     "ym[i] = widen_bf16(xm[i]) * rstd * widen_bf16(gamma[i]) + widen_bf16(beta[i]);"),
    ("linear_weight_transposed",
     "const uint16_t* wn = w + n * static_cast<std::ptrdiff_t>(K);\n      double acc = 0.0;\n"
     "      for (int k = 0; k < K; ++k) acc += xm[k] * widen_bf16(wn[k]);",
     "double acc = 0.0;\n"
     "      for (int k = 0; k < K; ++k) acc += xm[k] * widen_bf16(w[k * static_cast<std::ptrdiff_t>(N) + n]);"),
    ("linear_bias_dropped", "if (bias != nullptr) acc += widen_bf16(bias[n]);", ""),
    ("linear_last_k_dropped", "for (int k = 0; k < K; ++k) acc += xm[k] * widen_bf16(wn[k]);",
     "for (int k = 0; k < K - 1; ++k) acc += xm[k] * widen_bf16(wn[k]);"),
    ("linear_residual_dropped",
     "if (res != nullptr) acc += widen_bf16(res[m * static_cast<std::ptrdiff_t>(N) + n]);", ""),
    ("round_toward_zero", "std::nearbyint(std::ldexp(v, -q))", "std::trunc(std::ldexp(v, -q))"),
    ("round_ties_away", "std::nearbyint(std::ldexp(v, -q))", "std::round(std::ldexp(v, -q))"),
    ("round_seven_bits", "const int q = std::max(e - 8, -133);",
     "const int q = std::max(e - 7, -133);"),
    ("round_subnormals_flushed", "const int q = std::max(e - 8, -133);",
     "const int q = std::max(e - 8, -126);"),
    ("add_ln_residual_dropped",
     "s[off + i] = round_bf16(widen_bf16(x[off + i]) + widen_bf16(r[off + i]));",
     "s[off + i] = round_bf16(widen_bf16(x[off + i]));"),
    ("add_ln_normalises_x_not_stream",
     "return oracle_layernorm_bf16(s, gamma, beta, y, M, W, eps, nthreads);",
     "return oracle_layernorm_bf16(x, gamma, beta, y, M, W, eps, nthreads);"),
    ("gelu_cubic_sign", "a + 0.044715 * a * a * a", "a - 0.044715 * a * a * a"),
    ("gelu_half_dropped", "y[i] = 0.5 * a * (1.0 + std::tanh(", "y[i] = a * (1.0 + std::tanh("),
    ("gelu_sqrt_two_over_pi_wrong", "std::sqrt(2.0 / 3.14159265358979323846)",
     "std::sqrt(1.0 / 3.14159265358979323846)"),
    ("gelu_bias_ignored", "oracle_linear_bf16(x, w, bias, nullptr, y, M, K, N, nthreads)",
     "oracle_linear_bf16(x, w, nullptr, nullptr, y, M, K, N, nthreads)"),
    ("gelu_is_sigmoid_form", "std::tanh(c * (a + 0.044715 * a * a * a))",
     "std::tanh(0.851 * a)"),
]


@pytest.fixture(scope="module")
def source():
    with open(oracle.SOURCE) as f:
        return f.read()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, source, name, old, new):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    assert old in source, f"mutation site for {name} no longer in the oracle source"
    src = tmp_path / f"mutant_{name}.cpp"
    src.write_text(source.replace(old, new, 1))
    lib_path = str(tmp_path / f"libmutant_{name}.so")
    try:
        oracle_build.compile_source(str(src), lib_path)
    except subprocess.CalledProcessError:
        pytest.fail(f"mutant {name} does not compile")
    lib = oracle.OracleLib(lib_path)
    failed = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError, FloatingPointError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught mutant {name}"
    os.remove(lib_path)
