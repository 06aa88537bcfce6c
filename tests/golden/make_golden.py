"""Write tests/golden/tiny_layer.json: the fp64 oracle's results on the tiny
fp32 layer (routing, forward, backward, warehouse cells) for fixed seeded
inputs. Calls only the oracle and the seeded input generator.

The pages print no worked numerical example of the operator, so these are
not page values: they are regression fixtures that make any change to the
oracle's arithmetic visible (a deliberate change regenerates them, and its
commit names the passage or reading that justifies it); the pins in
tests/test_oracle_*.py are what tie the oracle to the pages.

Usage: python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from dynamic_convolution_b200 import synth  # noqa: E402


def compute():
    cfg = synth.CONFIGS["tiny_fp32"]
    inp = synth.make_inputs(cfg, seed=0, structured=1.0)
    _, dy = synth.make_upstream_grad(cfg, seed=1)
    alpha = oracle.route(inp.x_f64, inp.Wr, inp.br, cfg.mode, cfg.tau)
    y = oracle.forward(inp.x_f64, inp.experts_f64, alpha, inp.bias, stride=cfg.stride,
                       pad=cfg.pad, groups=cfg.groups)
    g = oracle.backward(inp.x_f64, dy, inp.experts_f64, alpha, inp.bias, inp.Wr, cfg.mode, cfg.tau,
                        stride=cfg.stride, pad=cfg.pad, groups=cfg.groups)
    ci = synth.make_cell_inputs(cfg, 4, 6, seed=0)
    a_cells = oracle.route_cells(ci.x_f64, ci.Wr, ci.br, 4, cfg.mode, cfg.tau)
    y_cells = oracle.forward_cells(ci.x_f64, ci.warehouse_f64, a_cells, ci.bias, cfg.C_out,
                                   cfg.KH, cfg.KW, cfg.stride, cfg.pad, cfg.groups)
    out = {"alpha": alpha, "y": y, "alpha_cells": a_cells, "y_cells": y_cells}
    out.update({k: v for k, v in g.items() if v is not None})
    return {k: np.asarray(v).tolist() for k, v in out.items()}


if __name__ == "__main__":
    data = {"source": "fp64 oracle on the tiny_fp32 layer (synth.make_inputs seed 0, "
                      "structured 1.0; dy seed 1; cells: 4 cells, warehouse of 6, seed 0); "
                      "written by tests/golden/make_golden.py",
            "values": compute()}
    with open(os.path.join(HERE, "tiny_layer.json"), "w") as f:
        json.dump(data, f)
    print("wrote", os.path.join(HERE, "tiny_layer.json"))
