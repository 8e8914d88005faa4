"""Write tests/golden/input_sha256.txt: the SHA-256 of every workload's
seeded inputs (seed 0) as ternary_weight_selective_b200.synthetic draws them,
so that a change of draw order or distribution is caught.  It reads only the
input generator (no method arithmetic, no CUDA path).

    python tests/golden/make_input_sha256.py
"""

from __future__ import annotations

import hashlib
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from ternary_weight_selective_b200 import synthetic as S  # noqa: E402

FIELDS = ("W_in", "W_dt_down", "W_B", "W_C", "W_dt_up", "W_out", "A", "D", "dt_bias",
          "W_z", "conv_w", "conv_b")


def digests(wl):
    x, layers = S.make_inputs(wl, seed=0)
    hx = hashlib.sha256(np.ascontiguousarray(x, np.float32).tobytes()).hexdigest()
    hw = hashlib.sha256()
    for lw in layers:
        for f in FIELDS:
            a = getattr(lw, f)
            if a is not None:
                hw.update(np.ascontiguousarray(a, np.float32).tobytes())
    return hx, hw.hexdigest()


def main():
    lines = ["# workload  sha256(x float32 bytes)  sha256(weights float32 bytes, per layer in field order)"]
    for name, wl in S.WORKLOADS.items():
        hx, hw = digests(wl)
        lines.append(f"{name} {hx} {hw}")
    with open(os.path.join(HERE, "input_sha256.txt"), "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
