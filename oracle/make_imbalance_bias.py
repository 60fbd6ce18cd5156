"""Find the router-bias constants of the load-imbalanced workload.

Bisects, on the seed-0 inputs of the 8 x 4096-token workload (d_model 1024,
8 experts, top-1), an additive bias b_0 > 0 on expert 0 so that about 40 % of
the tokens pick expert 0, and b_7 < 0 on expert 7 so that it receives about
1.5 % (under 2 %). Each bias moves the other's share, so the two searches
alternate twice. Routing decisions come from the oracle's router only. The
values are rounded to a multiple of 2^-10 and printed, to be pasted into
mixture_experts_projections_b200/inputs.py.
"""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from mixture_experts_projections_b200.inputs import make_block_inputs  # noqa: E402
from oracle.rom_oracle import route  # noqa: E402


def share(x, w_r, b, e):
    idx = route(x, w_r, 1, bias=b)["topk_idx"][:, 0]
    return float(np.mean(idx == e))


def main():
    inp = make_block_inputs(8 * 4096, 1024, 1, 8, seed=0)  # De does not affect routing
    x, w_r = inp["x"], inp["w_r"]
    b = np.zeros(8)
    for _ in range(2):
        lo, hi = 0.0, 4.0
        for _ in range(16):
            b[0] = 0.5 * (lo + hi)
            lo, hi = (b[0], hi) if share(x, w_r, b, 0) < 0.40 else (lo, b[0])
        b[0] = round(0.5 * (lo + hi) * 1024) / 1024
        lo, hi = -6.0, 0.0
        for _ in range(16):
            b[7] = 0.5 * (lo + hi)
            lo, hi = (b[7], hi) if share(x, w_r, b, 7) < 0.015 else (lo, b[7])
        b[7] = round(0.5 * (lo + hi) * 1024) / 1024
    idx = route(x, w_r, 1, bias=b)["topk_idx"][:, 0]
    print("IMBALANCE_BIAS_E0 =", float(b[0]))
    print("IMBALANCE_BIAS_E7 =", float(b[7]))
    print("load:", np.round(np.bincount(idx, minlength=8) / idx.size, 4))


if __name__ == "__main__":
    main()
