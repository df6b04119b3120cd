"""Writes oracle_regression_T12_H2.txt: oracle outputs for a small seeded case.

Calls only ``oracle`` (and the seeded input generator). The file guards the
oracle against unintended edits of its arithmetic; it is not a pin (the pins
are in tests/test_oracle_pins.py). Rerun only when a change to the oracle's
arithmetic is justified by a passage of the pages, and name it in the commit.
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import gdla_inputs as gi  # noqa: E402
import oracle  # noqa: E402

SEQLENS = (5, 7)
HKV = 2
SEED = 77
WINDOWS = (0, 3)


def compute():
    t = gi.make_prefill_inputs(SEQLENS, HKV, SEED, device="cpu")
    args = [gi.bf16_bits(t["q_sig"]), gi.bf16_bits(t["q_noise"]), gi.bf16_bits(t["k"]),
            gi.bf16_bits(t["v"]), t["lam"].numpy(), gi.bf16_bits(t["gate"])]
    return {w: oracle.prefill(*args, SEQLENS, w) for w in WINDOWS}


def main():
    res = compute()
    path = os.path.join(HERE, "oracle_regression_T12_H2.txt")
    with open(path, "w") as f:
        f.write(f"# seqlens {SEQLENS} hkv {HKV} seed {SEED}; rows: window token head d value (repr of fp64)\n")
        for w, out in res.items():
            # every 61st element keeps the file small
            for idx in range(0, out.size, 61):
                n, h, d = np.unravel_index(idx, out.shape)
                f.write(f"{w} {n} {h} {d} {float(out[n, h, d])!r}\n")


if __name__ == "__main__":
    main()
