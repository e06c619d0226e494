"""Small hand-built cases for pinning the oracle (no CUDA, no product code)."""
import copy
import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        g = json.load(f)
    case = {
        "activations": {k: np.array(v, dtype=np.float64) for k, v in g["activations"].items()},
        "parameters": {k: np.array(v, dtype=np.float64) for k, v in g["parameters"].items()},
        "masks": {k: np.array(v, dtype=bool) for k, v in g["masks"].items()},
        "structure": {k: np.array(v, dtype=np.int64) for k, v in g["structure"].items()},
        "eps": g["eps"], "style": g["style"], "stage": g["stage"], "radius": g["radius"],
    }
    return g, case


def clone(case):
    return copy.deepcopy(case)


def run(oracle, case, **kw):
    args = dict(eps=case["eps"], style=case["style"], stage=case["stage"], radius=case["radius"])
    args.update(kw)
    return oracle.windowed_atom_attention(case["activations"], case["parameters"], case["masks"],
                                          case["structure"], **args)


def ln2(v, eps):
    """Population LayerNorm of a 2-vector in closed form: [delta, -delta]."""
    half = (v[0] - v[1]) / 2.0
    dlt = half / math.sqrt(half * half + eps)
    return np.array([dlt, -dlt])


def rms2(v, eps):
    return np.asarray(v, dtype=np.float64) / math.sqrt((v[0] ** 2 + v[1] ** 2) / 2.0 + eps)


def from_workload(w):
    """Float64 copy of a workloads.make_inputs() dict in the oracle's case form."""
    spec = w["spec"]
    return {
        "activations": {k: v.astype(np.float64) for k, v in w["activations"].items()},
        "parameters": {k: v.astype(np.float64) for k, v in w["parameters"].items()},
        "masks": {k: v.copy() for k, v in w["masks"].items()},
        "structure": {k: v.copy() for k, v in w["structure"].items()},
        "eps": spec.eps, "style": spec.style, "stage": spec.stage, "radius": spec.radius,
    }
