"""The benchmark's accounting on CPU: algorithmic flops and bytes of the workloads
(closed forms), the comment-insensitive source hash that ties a profile summary
to the code it was taken of, and the traffic lookup that depends on it."""
import os

import pytest

import bench
import gdla_inputs as gi


def test_full_causal_flops_closed_form():
    # T(T+1)/2 visible pairs x 80 heads x (2*192 + 2*128) flops
    T = 4096
    assert bench.prefill_flops(gi.PREFILL_FULL) == T * (T + 1) // 2 * 80 * 640 == 429601587200


def test_window_pairs_closed_form():
    # per sequence: 1 + 2 + ... + 128 for the first 128 queries, then 128 each
    w = gi.SWA
    per_seq = 128 * 129 // 2 + (32768 - 128) * 128
    assert w.visible_pairs() == 2 * per_seq == 8372352
    assert bench.prefill_flops(w) == 2 * per_seq * 80 * 640


def test_bytes_per_token_and_per_key():
    # prefill: q_sig 24,576 + q_noise 6,144 + k 6,144 + v 4,096 + lambda 256 + gate 16,384 + out 16,384
    assert bench.prefill_bytes(gi.PREFILL_FULL) == 4096 * 73984
    # decode: 16 groups x (192 + 128) x 2 B per visible key, 63,744 B per query token
    assert bench.decode_bytes([1000, 3000], 16, 0) == 4000 * 10240 + 2 * 63744
    assert bench.decode_bytes([1000, 100], 16, 128) == (128 + 100) * 10240 + 2 * 63744


def test_latent_decode_accounting():
    # 1,152 B per visible key (576 bf16, shared by all 80 heads); per query 80 x 576 absorbed query
    # dims, 64 x 128 gate and output (bf16) and 64 lambdas; W^UV (16 x 128 x 512 bf16) once
    per_query = 2 * (80 * 576 + 64 * 128 + 64 * 128) + 4 * 64
    assert bench.latent_bytes([1000, 3000], 16, 0) == 4000 * 1152 + 2 * per_query + 16 * 128 * 512 * 2
    assert bench.latent_bytes([1000, 100], 16, 128) == 228 * 1152 + 2 * per_query + 16 * 128 * 512 * 2
    # flops: 80 heads x (576 score + 512 value) x 2 per key, 80 x 128 x 512 x 2 up-projection per query
    assert bench.latent_flops([1000], 16, 0) == 1000 * 80 * 1088 * 2 + 80 * 128 * 512 * 2


def test_code_only_ignores_comments_and_blank_lines():
    a = "int f(int x) {  // doubles\n    /* the\n       body */\n    return 2 * x;\n}\n\n"
    b = "int f(int x) {\n\n    return 2 * x;   // twice x\n}\n"
    c = "int f(int x) {\n    return 3 * x;\n}\n"
    assert bench._code_only(a) == bench._code_only(b) == "int f(int x) {\n    return 2 * x;\n}"
    assert bench._code_only(c) != bench._code_only(a)


def test_profiled_traffic_follows_the_source_hash(monkeypatch):
    kernel, workload = bench.PREFILL_KERNEL, gi.PREFILL_FULL.name
    path = os.path.join(bench.ROOT, "profiles", f"{kernel}__{workload}.txt")
    if not os.path.exists(path):
        pytest.skip("no profile summary for the headline kernel")
    text = open(path).read()
    recorded = [line.split()[1] for line in text.splitlines() if line.startswith("kernel_sources_sha256_16:")][0]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda k: recorded)
    assert bench.profiled_traffic(kernel, workload) > 0
    monkeypatch.setattr(bench, "kernel_source_hash", lambda k: "0" * 16)
    assert bench.profiled_traffic(kernel, workload) is None


def test_peaks_fall_back_when_unmeasured(monkeypatch):
    # a root with no MEASURED_PEAKS.json (the directory does not exist; nothing is created)
    monkeypatch.setattr(bench, "ROOT", os.path.join(bench.ROOT, "no_such_directory"))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS
