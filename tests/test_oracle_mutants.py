"""The oracle's pins must catch plausible mistakes planted in the oracle itself.

Each mutant is a copy of oracle/gdn_oracle.c with one textual change (a dropped term,
a flipped sign, a wrong operand or order), compiled on the CPU into a temporary
library. The pin suite of test_oracle_pins.py is run against it and at least one
pin must fail. This shows that the pins constrain every step of the oracle.
"""
import ctypes
import os
import subprocess
import types

import pytest

import oracle
from tests import test_oracle_backward as bpins
from tests import test_oracle_featurize as fpins
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")

MUTANTS = {
    # error formed against the undecayed state (decay moved after the error)
    "decay_after_error": [("        for (int a = 0; a < dk * dv; ++a)\n            S[a] *= alpha;\n"
                           "        /* e = v - S~^T k",
                           "        /* e = v - S~^T k"),
                          ("        /* S = S~ + beta k e^T */\n",
                           "        for (int a = 0; a < dk * dv; ++a)\n            S[a] *= alpha;\n"
                           "        /* S = S~ + beta k e^T */\n")],
    "error_sign": [("e[b] = vt[b] - acc;\n        }\n        /* S = S~",
                    "e[b] = vt[b] + acc;\n        }\n        /* S = S~")],
    "decode_error_sign": [("e[b] = vt[b] - acc;\n        }\n        for (int a = 0; a < dk; ++a)\n"
                           "            for (int b = 0; b < dv; ++b)\n                S[a * dv + b] += beta",
                           "e[b] = vt[b] + acc;\n        }\n        for (int a = 0; a < dk; ++a)\n"
                           "            for (int b = 0; b < dv; ++b)\n                S[a * dv + b] += beta")],
    "dropped_beta": [("S[a * dv + b] += beta * kt[a] * e[b];\n        /* y",
                      "S[a * dv + b] += kt[a] * e[b];\n        /* y")],
    "read_before_write": [("        /* S = S~ + beta k e^T */\n        for (int a = 0; a < dk; ++a)\n"
                           "            for (int b = 0; b < dv; ++b)\n"
                           "                S[a * dv + b] += beta * kt[a] * e[b];\n",
                           ""),
                          ("            yt[b] = acc;\n        }\n    }\n    if (A->S_T)",
                           "            yt[b] = acc;\n        }\n        for (int a = 0; a < dk; ++a)\n"
                           "            for (int b = 0; b < dv; ++b)\n"
                           "                S[a * dv + b] += beta * kt[a] * e[b];\n    }\n"
                           "    if (A->S_T)")],
    "error_uses_query": [("acc += S[a * dv + b] * kt[a];\n            e[b] = vt[b] - acc;\n        }\n"
                          "        /* S = S~",
                          "acc += S[a * dv + b] * qt[a];\n            e[b] = vt[b] - acc;\n        }\n"
                          "        /* S = S~")],
    "scale_on_state": [("qs[a] = A->scale * qt[a];", "qs[a] = qt[a];"),
                       ("yt[b] = acc;\n        }\n    }\n    if (A->S_T)",
                        "yt[b] = acc;\n        }\n        for (int a = 0; a < dk * dv; ++a) S[a] *= A->scale;\n"
                        "    }\n    if (A->S_T)")],
    "decode_no_decay": [("        for (int a = 0; a < dk * dv; ++a)\n            S[a] *= alpha;\n"
                         "        for (int b = 0; b < dv; ++b) {",
                         "        for (int b = 0; b < dv; ++b) {")],
    "norm_weight_not_centred": [("* (1.0 + w[j]);", "* w[j];")],
    "norm_mean_off_by_one": [("sqrt(ss / dv + eps)", "sqrt(ss / (dv - 1) + eps)")],
    "gate_silu": [("const double gate = 1.0 / (1.0 + exp(-zr[j]));",
                   "const double gate = zr[j] / (1.0 + exp(-zr[j]));")],
    # featurisation: taps in the wrong order, a window that crosses sequence starts, no
    # SiLU, v normalised too, the decay bias dropped, the decay rate not exponentiated
    "conv_taps_reversed": [("acc += w[j] * x[((size_t)s * H + h) * d + c];",
                            "acc += w[W - 1 - j] * x[((size_t)s * H + h) * d + c];")],
    "conv_crosses_sequences": [("if (s >= cu[i])\n", "if (s >= 0)\n")],
    "no_silu": [("o[c] = acc / (1.0 + exp(-acc));", "o[c] = acc;")],
    "v_normalised": [("featurize_stream(xv, conv_v, W, cu, n_seq, H, dv, 0, eps, v);",
                      "featurize_stream(xv, conv_v, W, cu, n_seq, H, dv, 1, eps, v);")],
    "decay_bias_dropped": [("softplus(alpha_logit[e] + b_alpha[h]);", "softplus(alpha_logit[e]);")],
    "decay_rate_not_exp": [("log_alpha[e] = -exp(A[h]) * softplus", "log_alpha[e] = -A[h] * softplus")],
    # gradients: the output term dropped from the state adjoint, the error term's sign, the
    # decay gradient against the new state, the decay missing from the carried adjoint, the
    # key gradient's error part dropped
    "bwd_no_output_term": [("                            G[a * dv + b] += scale * qt[a] * dyt[b];\n", "")],
    "bwd_error_term_sign": [("Gt[a * dv + b] -= kt[a] * de[b];", "Gt[a * dv + b] += kt[a] * de[b];")],
    "bwd_dalpha_new_state": [("dal += Gt[a] * Sp[a];", "dal += Gt[a] * St[a];")],
    "bwd_carry_without_decay": [("G[a] = alpha * Gt[a];", "G[a] = Gt[a];")],
    "bwd_dk_error_part_dropped": [("                        dkt[a] -= sd;\n", "")],
}

PIN_TESTS = [
    lambda m: [pins.test_equivalent_form(m, *p) for p in [(5, 3, (7, 1, 0, 12), 2), (4, 6, (3, 9), 1)]],
    lambda m: [pins.test_brute_force_products(m, T) for T in (2, 5)],
    pins.test_noop_gates,
    pins.test_orthonormal_retrieval,
    pins.test_readback_identity,
    pins.test_linearity_in_values_and_state,
    pins.test_split_sequence,
    pins.test_hand_example,
    pins.test_decode_step_matches_one_token_recurrence,
    pins.test_gate_norm_closed_forms,
] + fpins.PINS + bpins.PINS


def _mutant_module(tmp_path, name, edits):
    src = open(SRC).read()
    for old, new in edits:
        assert src.count(old) == 1, (name, old)
        src = src.replace(old, new)
    c_path = tmp_path / f"{name}.c"
    so_path = tmp_path / f"lib{name}.so"
    c_path.write_text(src)
    subprocess.run(["gcc", "-O2", "-std=c99", "-shared", "-fPIC", "-o", str(so_path),
                    str(c_path), "-lm", "-lpthread"], check=True)
    lib = oracle._configure(ctypes.CDLL(str(so_path)))
    mod = types.SimpleNamespace()
    for fn in ("recurrent", "decode_step", "gate_norm", "featurize", "backward"):
        f = getattr(oracle, fn)

        def wrapped(*a, _f=f, **kw):
            saved = oracle._lib
            oracle._lib = lib
            try:
                return _f(*a, **kw)
            finally:
                oracle._lib = saved
        setattr(mod, fn, wrapped)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, oracle_mod, name):
    mod = _mutant_module(tmp_path, name, MUTANTS[name])
    failed = 0
    for t in PIN_TESTS:
        try:
            t(mod)
        except AssertionError:
            failed += 1
    assert failed >= 1, f"no pin caught mutant {name}"


def test_unmutated_copy_passes_all_pins(tmp_path, oracle_mod):
    mod = _mutant_module(tmp_path, "identity", [])
    for t in PIN_TESTS:
        t(mod)
