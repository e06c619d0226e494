"""Helpers shared by the GPU parity tests: move a seeded workload to the device, run
the CUDA library through its C ABI, run the oracle on the same values, compare."""
import numpy as np
import torch

import oracle
from sparse_windowed_atom_b200 import atomenc, workloads
from tests.oracle_cases import from_workload

TOL = {"float32": 2e-4, "bfloat16": 2e-2}   # max|err| <= tol * (1 + |ref|)


def to_torch(w, device="cuda"):
    spec = w["spec"]
    fdt = torch.bfloat16 if spec.dtype == "bfloat16" else torch.float32

    def f(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=fdt)

    act = {k: f(v) for k, v in w["activations"].items()}
    prm = {k: f(v) for k, v in w["parameters"].items()}
    msk = {k: torch.from_numpy(np.ascontiguousarray(v)).to(device) for k, v in w["masks"].items()}
    st = {k: torch.from_numpy(np.ascontiguousarray(v)).to(device) for k, v in w["structure"].items()}
    return act, prm, msk, st


def run_cuda(w, device="cuda", **over):
    spec = w["spec"]
    act, prm, msk, st = to_torch(w, device)
    args = dict(eps=spec.eps, style=spec.style, stage=spec.stage, radius=spec.radius)
    args.update(over)
    out = atomenc.windowed_atom_attention(act, prm, msk, st, **args)
    torch.cuda.synchronize()
    return {k: v.float().cpu().numpy().astype(np.float64) for k, v in out.items()}


def run_oracle(w, query_select=None, **over):
    case = from_workload(w)
    args = dict(eps=case["eps"], style=case["style"], stage=case["stage"], radius=case["radius"])
    args.update(over)
    return oracle.windowed_atom_attention(case["activations"], case["parameters"], case["masks"],
                                          case["structure"], query_select=query_select, **args)


def compare(got, ref, dtype, what=""):
    """Elementwise |got - ref| <= tol (1 + |ref|) over every element the oracle wrote."""
    tol = TOL[dtype]
    for k, r in ref.items():
        g = got[k]
        assert g.shape == r.shape, (k, g.shape, r.shape)
        m = ~np.isnan(r)
        assert np.all(np.isfinite(g[m])), f"{what} {k}: non-finite output"
        err = np.abs(g[m] - r[m])
        bound = tol * (1.0 + np.abs(r[m]))
        bad = err > bound
        if bad.any():
            i = np.argmax(err / bound)
            raise AssertionError(
                f"{what} {k}: {bad.sum()} of {m.sum()} elements out of tolerance; worst "
                f"got {g[m][i]!r} ref {r[m][i]!r} (err {err[i]:.3g} > {bound[i]:.3g})")


def exact_zero_pattern(got, ref):
    """Masking decisions are exact: an entry the oracle sets to exactly 0 by a mask or an
    empty row is exactly 0 on the GPU too (attention, hidden rows, position updates)."""
    for k in ("attention", "hidden", "position_update"):
        if k in ref:
            m = ref[k] == 0.0
            assert np.all(got[k][m] == 0.0), f"{k}: nonzero where the oracle is exactly zero"


def sample_queries(spec, w, frac=0.01, seed=1):
    """A seeded sample of whole tokens (all their atoms) plus scattered atoms."""
    rng = np.random.default_rng(seed)
    att = w["structure"]["atom_to_token"]
    sel = np.zeros((spec.B, spec.A), bool)
    for b in range(spec.B):
        toks = rng.choice(spec.T, size=max(1, int(spec.T * frac)), replace=False)
        sel[b] = np.isin(att[b], toks)
        sel[b, rng.choice(spec.A, size=max(1, int(spec.A * frac)), replace=False)] = True
        sel[b, :2] = True
        sel[b, -2:] = True
    return sel
