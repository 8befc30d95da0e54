"""Plant plausible mistakes in copies of the oracle and require the pins to
catch every one.  Each mutant is the oracle source with one textual change,
compiled on the CPU into a temporary library; the real oracle is untouched.
"""
import os
import subprocess
import tempfile

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.cpp")

MUTANTS = {
    "swigluoai_drops_plus_one": ("* (u + 1.0);", "* (u);"),
    "gelu_drops_cubic_term": ("(g + 0.044715 * g * g * g)", "(g)"),
    "sink_selects_on_raw_logit": ("float sig = static_cast<float>(1.0 / (1.0 + std::exp(-z)));",
                                  "float sig = static_cast<float>(z);"),
    "sink_weights_skip_log_sigmoid": ("v[j] = log_sigmoid(", "v[j] = ("),
    "sink_bias_enters_weights": ("for (int j = 0; j < k; ++j) v[j] = log_sigmoid(logit_at(logits, logits_is_bf16, t, stride, idx[t * k + j]));",
                                 "for (int j = 0; j < k; ++j) v[j] = log_sigmoid(logit_at(logits, logits_is_bf16, t, stride, idx[t * k + j]) + (bias ? bias[idx[t * k + j]] : 0.0f));"),
    "ties_to_highest_index": ("return key[a] > key[b]; });", "return key[a] > key[b] || (key[a] == key[b] && a > b); });"),
    "softmax_normalises_over_all_experts": ("for (int j = 0; j < k; ++j) sum += std::exp(z[idx[t * k + j]] - m);",
                                            "for (int j = 0; j < E; ++j) sum += std::exp(z[j] - m);"),
    "csr_not_stable": ("for (int64_t s = 0; s < R; ++s) {\n    int32_t pos", "for (int64_t s = R - 1; s >= 0; --s) {\n    int32_t pos"),
    "interleaved_gate_up_swapped": ("double g = gate_up_format == 0 ? a[i] : a[2 * i];",
                                    "double g = gate_up_format == 0 ? a[i] : a[2 * i + 1];"),
    "gate_up_bias_dropped": ("a[n] = b_gu ? bf16_bits_to_double(b_gu[e * N1 + n]) : 0.0;", "a[n] = 0.0;"),
    "down_weight_transposed": ("ys[c] += hi * bf16_bits_to_double(row[c]);", "ys[c] += hi * bf16_bits_to_double(Wd[c * D + i]);"),
    "router_weight_not_applied": ("o[c] += wj * ys[c];", "o[c] += ys[c];"),
    "up_clamp_sign": ("u = std::min(std::max(u, -limit), limit);\n      }\n      return g / (1.0",
                      "u = std::min(std::max(u, limit), limit);\n      }\n      return g / (1.0"),
    "swigluoai_alpha_ignored": ("std::exp(-alpha * g)", "std::exp(-g)"),
    "weight_first_ignored": ("const double in_scale = weight_first ? w[t * k + s % k] : 1.0;",
                             "const double in_scale = 1.0;"),
    "weight_first_also_weights_output": ("const double wj = weight_first ? 1.0 : w[t * k + j];",
                                         "const double wj = w[t * k + j];"),
    "mask_ignored": ("      if (token_mask && token_mask[t] == 0) continue;\n", ""),
    "sink_global_scale_dropped": ("double scale = route_scale * global_scale;", "double scale = route_scale;"),
    "sink_lanes_read_from_column_zero": ("log_sigmoid(logit_at(logits, logits_is_bf16, t, stride, E + i))",
                                         "log_sigmoid(logit_at(logits, logits_is_bf16, t, stride, i))"),
    "silu_applied_to_up": ("return g / (1.0 + std::exp(-g)) * u;", "return u / (1.0 + std::exp(-u)) * g;"),
    "gelu_drops_one_half": ("return 0.5 * g * (1.0 + std::tanh(inner)) * u;", "return g * (1.0 + std::tanh(inner)) * u;"),
    "silu_gate_clamped_from_below": ("g = std::min(g, limit);\n        u = std::min(std::max(u, -limit), limit);\n      }\n      return g / (1.0",
                                     "g = std::min(std::max(g, -limit), limit);\n        u = std::min(std::max(u, -limit), limit);\n      }\n      return g / (1.0"),
    "down_bias_dropped": ("ys[c] = b_d ? bf16_bits_to_double(b_d[static_cast<int64_t>(e) * H + c]) : 0.0;", "ys[c] = 0.0;"),
    "csr_inverse_off_by_one": ("if (inv) inv[s] = pos;", "if (inv) inv[s] = pos + 1;"),
    "softmax_weights_not_normalised": ("w[t * k + j] = std::exp(z[idx[t * k + j]] - m) / sum;",
                                       "w[t * k + j] = std::exp(z[idx[t * k + j]] - m);"),
    "interleaved_up_is_gate": ("double u = gate_up_format == 0 ? a[D + i] : a[2 * i + 1];",
                               "double u = gate_up_format == 0 ? a[D + i] : a[2 * i];"),
    "concatenated_up_is_gate": ("double u = gate_up_format == 0 ? a[D + i] : a[2 * i + 1];",
                                "double u = gate_up_format == 0 ? a[i] : a[2 * i + 1];"),
}


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutated = source.replace(old, new)
    src = tmp_path / "mutant.cpp"
    src.write_text(mutated)
    lib = tmp_path / "libmutant.so"
    subprocess.run(["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                    str(src), "-o", str(lib)], check=True)
    real = oracle._load()
    import ctypes
    mutant = ctypes.CDLL(str(lib))
    for fn in ("oracle_activation", "oracle_route_softmax_topk", "oracle_route_sigmoid_sink",
               "oracle_create_indices", "oracle_expert_ffn", "oracle_expert_ffn_ex", "oracle_num_threads"):
        getattr(mutant, fn).restype = getattr(real, fn).restype
        getattr(mutant, fn).argtypes = getattr(real, fn).argtypes
    caught = []
    oracle._lib = mutant
    try:
        for pin in pins.ALL_PINS:
            try:
                pin()
            except Exception as exc:  # an assertion or a rejected result
                caught.append((pin.__name__, type(exc).__name__))
    finally:
        oracle._lib = real
    assert caught, f"no pin catches the planted mistake {name}"
