"""Writes tiny_redraws.txt: the redraw indices that the tiny configuration's
input rule assigns to the benchmark's decode steps.

The tiny configuration (hidden 256, 16 experts, top-4, 4 tokens per step,
seed 0) redraws a token's hidden row while the gap between consecutive
logits among its top k + 1 is below 1e-3 (reading of the configuration's
rule: the gap is taken in fp64, and the redraw is the next independent
draw).  Deciding it needs the router, so the decision is made here, once,
with the fp64 oracle, and stored: the benchmark then builds its inputs from
the seeded generator and this table alone.

    python tests/golden/make_tiny_redraws.py [steps]

Each line: stream token draw -- the hidden row of `token` at `stream` is the
generator's draw number `draw` (0: the step's own row; d > 0: the row
gen_hidden(..., draw=d * 65536 + token + 1)).
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from int4_routed_expert_02_b200 import synth  # noqa: E402

FIRST_STREAM = 10_000   # the benchmark's decode streams: 10_000 + step
GAP = 1e-3


def min_gap(row, k):
    srt = np.sort(row)[::-1][: k + 1]
    return float(np.min(srt[:-1] - srt[1:]))


def main(steps=600):
    cfg = synth.CONFIGS[0]
    w = {n: v.cpu() for n, v in synth.gen_layer(cfg, 0, 0).items()}
    L = oracle.OracleLayer(w, cfg.H, cfg.E, cfg.k, cfg.I, cfg.Is)
    lines = []
    for step in range(steps):
        stream = FIRST_STREAM + step
        h = synth.gen_hidden(cfg, 0, stream, cfg.T)
        for t in range(cfg.T):
            d, row = 0, h[t:t + 1]
            while min_gap(oracle.router(L, row)[0][0], cfg.k) < GAP:
                d += 1
                row = synth.gen_hidden(cfg, 0, stream, 1, draw=d * 65536 + t + 1)
            if d:
                lines.append(f"{stream} {t} {d}")
    with open(os.path.join(HERE, "tiny_redraws.txt"), "w") as f:
        f.write("# tiny configuration (seed 0, layer 0): stream token draw for every decode row of streams "
                f"{FIRST_STREAM}..{FIRST_STREAM + steps - 1} whose top-(k+1) logit gap is below {GAP}\n")
        f.write("# written by tests/golden/make_tiny_redraws.py with the fp64 oracle; rows not listed keep draw 0\n")
        f.write(f"# steps {steps}\n")
        for ln in lines:
            f.write(ln + "\n")
    print(f"{len(lines)} redrawn rows in {steps} steps")


if __name__ == "__main__":
    main(int(sys.argv[1]) if len(sys.argv) > 1 else 600)
