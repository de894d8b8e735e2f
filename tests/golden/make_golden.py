"""Writes the stored expected values under tests/golden/ from the CPU oracle only.

visible_pairs.json: visible (query, key) pairs per window step, per prefill and
per verify call of each synthetic workload, counted on the oracle's dense mask.
Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

from oracle.stream_oracle import ViewMajorWindow, visible_mask  # noqa: E402

SHAPES = {  # views, frames, tok_per_frame, text_len (the five synthetic workloads)
    "1": (2, 2, 16, 8),
    "2": (4, 4, 64, 32),
    "3": (4, 4, 180, 256),
    "4": (7, 8, 256, 512),
    "5": (4, 4, 64, 32),
}
VERIFY_TOKENS = 8


def main():
    out = {}
    for k, (V, T, n, X) in SHAPES.items():
        w = ViewMajorWindow(V, T, n, X)
        kpos = w.key_positions()
        L = w.window_len
        step = int(visible_mask(w.step_query_positions(), kpos).sum())
        pre = int(visible_mask(kpos, kpos).sum())
        kx = np.arange(L + VERIFY_TOKENS)
        ver = int(visible_mask(np.arange(L, L + VERIFY_TOKENS), kx).sum())
        out[k] = dict(window_len=L, step_queries=int(w.step_tokens), step_pairs=step,
                      prefill_pairs=pre, verify_pairs=ver)
    with open(os.path.join(HERE, "visible_pairs.json"), "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)
        f.write("\n")


if __name__ == "__main__":
    main()
