"""Planted mistakes: each mutant is a copy of the oracle source with one plausible
slip (wrong scale, sign, index, window edge, operand stride, dropped term). It is
compiled on the CPU into a temporary library and run through the pins of
``test_oracle_pins``; every mutant must fail at least one pin. Nothing here
touches a GPU or the committed oracle.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdla_oracle.c")

MUTANTS = {
    "scale_multiplied": ("s = s / root;", "s = s * root;"),
    "subtract_sign": ("const double dd = hs[d] - l * hn[d];", "const double dd = hs[d] + l * hn[d];"),
    "gate_sign": ("dd / (1.0 + exp(-g))", "dd / (1.0 + exp(g))"),
    "window_off_by_one": ("if (J->window > 0 && t - J->window + 1 > 0) lo = t - J->window + 1;\n"
                          "        const long nkeys = (long)(t - lo + 1);\n"
                          "        const long kstride = (long)J->hkv * DQK, vstride = (long)J->hkv * DV;\n"
                          "        const uint16_t *krow = J->k + (s0 + lo) * kstride",
                          "if (J->window > 0 && t - J->window + 2 > 0) lo = t - J->window + 2;\n"
                          "        const long nkeys = (long)(t - lo + 1);\n"
                          "        const long kstride = (long)J->hkv * DQK, vstride = (long)J->hkv * DV;\n"
                          "        const uint16_t *krow = J->k + (s0 + lo) * kstride"),
    "noise_group_index": ("const uint16_t *qn = J->q_noise + (n * J->hkv + j) * DQK;",
                          "const uint16_t *qn = J->q_noise + (n * J->hkv + (J->hkv - 1 - j)) * DQK;"),
    "lambda_per_group": ("const float *lam = J->lambda + n * hs + GROUP * j;",
                         "const float *lam = J->lambda + n * hs + j;"),
    "normalisation_dropped": ("for (int d = 0; d < DV; ++d) h[d] /= den;", ""),
    "value_head_index": ("const uint16_t *vrow = J->v + (s0 + lo) * vstride + (long)j * DV;",
                         "const uint16_t *vrow = J->v + (s0 + lo) * vstride;"),
    "key_stride_transposed": ("const uint16_t *kr = k_rows + u * kstride;",
                              "const uint16_t *kr = k_rows + u * vstride;"),
    "gate_head_index": ("bf16_to_double(gate[(long)i * DV + d])", "bf16_to_double(gate[d])"),
    "signal_query_head": ("attend(qs + (long)i * DQK,", "attend(qs,"),
}

PINS = [
    (P.test_full_output_against_library_attention, {"window": 0}),
    (P.test_full_output_against_library_attention, {"window": 3}),
    (P.test_window_one_closed_form, {}),
    (P.test_identical_paths_with_lambda_one_cancel_exactly, {}),
    (P.test_identical_paths_cancel_only_in_their_own_group, {}),
    (P.test_gate_zero_halves_gate_open_exactly, {}),
    (P.test_uniform_scores_give_running_mean, {}),
    (P.test_decode_equals_last_prefill_row, {"window": 2}),
]


# Mutant builds stay inside the repository, in its (git-ignored) build folder.
MUTANT_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "_build", "oracle_mutants")


def _build_mutant(name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    os.makedirs(MUTANT_DIR, exist_ok=True)
    path = os.path.join(MUTANT_DIR, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new, 1))   # first site: the prefill path
    lib = os.path.join(MUTANT_DIR, f"lib{name}.so")
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", str(lib),
                           str(path), "-lm"], env={**os.environ, "TMPDIR": MUTANT_DIR})
    return str(lib)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    old, new = MUTANTS[name]
    path = _build_mutant(name, old, new)
    real = oracle._load()
    lib = ctypes.CDLL(path)
    for fn in ("gdla_oracle_prefill", "gdla_oracle_decode"):
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        getattr(lib, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", lib)
    caught = []
    for pin, kwargs in PINS:
        try:
            pin(**kwargs)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"


# Slips in the decode path's own code (the prefill path untouched): each must break
# "decode equals the last prefill row".
DECODE_MUTANTS = {
    "decode_window_off_by_one": (
        "const int64_t t = len - 1;              /* the query's own position */\n        int64_t lo = 0;\n"
        "        if (J->window > 0 && t - J->window + 1 > 0) lo = t - J->window + 1;",
        "const int64_t t = len - 1;              /* the query's own position */\n        int64_t lo = 0;\n"
        "        if (J->window > 0 && t - J->window + 2 > 0) lo = t - J->window + 2;"),
    "decode_query_position": ("const int64_t t = len - 1;              /* the query's own position */",
                              "const int64_t t = len - 2;              /* the query's own position */"),
    "decode_noise_group_index": ("const uint16_t *qn = J->q_noise + (b * J->hkv + j) * DQK;",
                                 "const uint16_t *qn = J->q_noise + (b * J->hkv + (J->hkv - 1 - j)) * DQK;"),
    "decode_lambda_index": ("const float *lam = J->lambda + b * hs + GROUP * j;",
                            "const float *lam = J->lambda + b * hs + j;"),
    "decode_gate_group": ("const uint16_t *gate = J->gate + (b * hs + (long)GROUP * j) * DV;",
                          "const uint16_t *gate = J->gate + (b * hs) * DV;"),
    "decode_sequence_offset_dropped": ("const uint16_t *krow = J->k + (s0 + lo) * kstride + (long)j * DQK;\n"
                                       "        const uint16_t *vrow = J->v + (s0 + lo) * vstride + (long)j * DV;\n"
                                       "        const uint16_t *qs = J->q_sig + (b * hs",
                                       "const uint16_t *krow = J->k + lo * kstride + (long)j * DQK;\n"
                                       "        const uint16_t *vrow = J->v + lo * vstride + (long)j * DV;\n"
                                       "        const uint16_t *qs = J->q_sig + (b * hs"),
}


@pytest.mark.parametrize("name", sorted(DECODE_MUTANTS))
def test_decode_mutant_is_caught(name, monkeypatch):
    old, new = DECODE_MUTANTS[name]
    assert open(SRC).read().count(old) == 1, name
    path = _build_mutant(name, old, new)
    real = oracle._load()
    lib = ctypes.CDLL(path)
    for fn in ("gdla_oracle_prefill", "gdla_oracle_decode"):
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        getattr(lib, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", lib)
    caught = []
    for window in (0, 2, 300):
        try:
            P.test_decode_equals_last_prefill_row(window)
        except AssertionError:
            caught.append(window)
    assert caught, f"decode mutant {name} passed every pin"
