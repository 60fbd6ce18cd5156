"""Write the oracle regression fixtures in this folder.

Calls only the CPU oracle (oracle/) on seeded inputs from the input module.
The fixtures freeze the oracle's float64 results on tiny cases so that an
unintended change of its arithmetic shows up as a test failure; a deliberate
change regenerates them and names, in its commit message, the passage of the
pages that justifies it.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from mixture_experts_projections_b200.inputs import (make_block_inputs, make_core_params,  # noqa
                                                     make_inproj_inputs)
from oracle import rom_oracle as orc  # noqa: E402

CASES = [
    # name, T, Dm, De, E, k, renorm
    ("block_T8_Dm4_De6_E3_k1", 8, 4, 6, 3, 1, False),
    ("block_T8_Dm4_De6_E3_k2_renorm", 8, 4, 6, 3, 2, True),
]


def main():
    out = {"source": "oracle/rom_oracle.py (RoM page, Knowl 1, 4 and 9; Swimba page, Extended "
                     "abstract; the Mamba recurrence for the core)",
           "cases": {}}
    for name, T, Dm, De, E, k, renorm in CASES:
        inp = make_block_inputs(T, Dm, De, E, seed=123, router_std=0.5, with_dout=True)
        fw = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"],
                               k=k, renorm=renorm)
        bw = orc.block_backward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"],
                                inp["w_out"], inp["dout"], k=k, renorm=renorm)
        out["cases"][name] = dict(T=T, Dm=Dm, De=De, E=E, k=k, renorm=renorm, seed=123,
                                  router_std=0.5, topk_idx=fw["topk_idx"].tolist(),
                                  topk_w=fw["topk_w"].tolist(), O=fw["O"].tolist(),
                                  dX=bw["dX"].tolist(), dlogits=bw["dlogits"].tolist())
    inp = make_inproj_inputs(6, 8, 5, 4, seed=123, router_std=0.5)
    s = orc.inproj_forward(inp["x"], inp["w_r"], inp["w"], k=1)
    out["cases"]["inproj_T6_Dm8_N5_E4_k1"] = dict(T=6, Dm=8, N=5, E=4, k=1, seed=123,
                                                 router_std=0.5, S=s["S"].tolist(),
                                                 topk_idx=s["topk_idx"].tolist())
    # independently routed projections (RoM page, Knowl 4)
    inp = make_block_inputs(8, 4, 6, 3, seed=123, router_std=0.5, extra_routers=True)
    v = orc.variant_block_forward(inp["x"], inp["w_conv"], inp["w_gate"], inp["w_out"], 1,
                                  {"conv": inp["w_r"], "gate": inp["w_r_gate"],
                                   "out": inp["w_r_out"]},
                                  {"conv": True, "gate": True, "out": True})
    out["cases"]["independent_T8_Dm4_De6_E3_k1"] = dict(T=8, Dm=4, De=6, E=3, k=1, seed=123,
                                                       router_std=0.5, O=v["O"].tolist())
    # the block with the dense core over two sequences (Knowl 1 Y_t, Knowl 9)
    inp = make_block_inputs(12, 8, 16, 3, seed=123, router_std=0.5)
    core = make_core_params(16, 8, seed=123, N=4, K=3)
    c = orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"], 1,
                          core=core, seq_len=6)
    out["cases"]["core_T12_Dm8_De16_E3_k1_L6"] = dict(T=12, Dm=8, De=16, E=3, k=1, seed=123,
                                                     router_std=0.5, N=4, K=3, seq_len=6,
                                                     O=c["O"].tolist(), Y=c["Y"].tolist())
    with open(os.path.join(HERE, "oracle_regression.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
