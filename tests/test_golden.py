"""Golden fixtures: the constants the pages print, and the oracle regression file."""
import os
import re

import pytest

import gdla_inputs as gi
import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _paper_constants():
    vals = {}
    with open(os.path.join(HERE, "golden", "paper_constants.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                name, value = line.split()
                vals[name] = int(value)
    return vals


def test_printed_head_arithmetic_is_consistent():
    c = _paper_constants()
    g = c["group_ratio"]
    assert c["noise_heads"] == c["query_heads"] // (g + 1)
    assert c["signal_heads"] == g * c["noise_heads"]
    assert c["signal_heads"] + c["noise_heads"] == c["query_heads"]
    assert c["noise_heads"] == c["kv_heads"]          # one noise head per KV head
    assert c["rotary_dim"] < c["dqk"]


def test_oracle_constants_match_pages():
    c = _paper_constants()
    src = open(os.path.join(ROOT, "oracle", "gdla_oracle.c")).read()
    defines = dict(re.findall(r"#define\s+(\w+)\s+(\d+)", src))
    assert int(defines["GROUP"]) == c["group_ratio"]
    assert int(defines["DQK"]) == c["dqk"]
    assert int(defines["DV"]) == c["dv"]


def test_header_constants_match_pages():
    c = _paper_constants()
    hdr = open(os.path.join(ROOT, "include", "gdla.h")).read()
    defines = dict(re.findall(r"#define\s+(GDLA_\w+)\s+(\d+)", hdr))
    assert int(defines["GDLA_GROUP"]) == c["group_ratio"]
    assert int(defines["GDLA_DQK"]) == c["dqk"]
    assert int(defines["GDLA_DV"]) == c["dv"]
    assert int(defines["GDLA_MAX_KV_HEADS"]) >= c["kv_heads"]


def test_workloads_follow_pages():
    c = _paper_constants()
    for w in (gi.PREFILL_FULL, gi.SWA, *gi.HYBRID_LAYERS, gi.DECODE_FULL, gi.DECODE_W128):
        assert w.num_kv_heads == c["kv_heads"]
    assert gi.SWA.window == c["window"] == gi.DECODE_W128.window
    modes = [l.window for l in gi.HYBRID_LAYERS]
    assert modes.count(0) == c["hybrid_full"] and modes.count(c["window"]) == c["hybrid_swa"]


def test_oracle_regression_fixture():
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_oracle_regression",
                                                  os.path.join(HERE, "golden", "make_oracle_regression.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    res = mod.compute()
    n_checked = 0
    with open(os.path.join(HERE, "golden", "oracle_regression_T12_H2.txt")) as f:
        for line in f:
            if line.startswith("#"):
                continue
            w, n, h, d, val = line.split()
            assert res[int(w)][int(n), int(h), int(d)] == pytest.approx(float(val), rel=1e-13, abs=1e-15)
            n_checked += 1
    assert n_checked > 300
