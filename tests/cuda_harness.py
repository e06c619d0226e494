"""Helpers shared by the GPU parity tests: move a seeded workload to the device, run
the CUDA library through its C ABI, run the oracle on the same values, compare."""
import os

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
    # check_status (the default) raises if a bounded wait of the pass gave up
    out = atomenc.windowed_atom_attention(act, prm, msk, st, check_status=True, **args)
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
        # ATOMENC_MARGIN_LOG=<file>: append the largest error and its share of the bound
        log = os.environ.get("ATOMENC_MARGIN_LOG")
        if log and err.size:
            with open(log, "a") as f:
                f.write(f"{what} {k} n={err.size} max_err={err.max():.3e} "
                        f"max_err_over_bound={(err / bound).max():.4f}\n")
        if bad.any():
            i = np.argmax(err / bound)
            raise AssertionError(
                f"{what} {k}: {bad.sum()} of {m.sum()} elements out of tolerance; worst "
                f"got {g[m][i]!r} ref {r[m][i]!r} (err {err[i]:.3g} > {bound[i]:.3g})")


UNDERFLOW_FLOOR = 1e-30   # weights this small may round to zero in float32 / bf16


def exact_zero_pattern(got, ref):
    """Masking and eligibility decisions are exact, in both directions.

    attention, per entry: exactly 0 on the GPU wherever the oracle is exactly 0 (a slot
    that is not permitted, an empty row), and nonzero wherever the oracle's weight is
    above the float32 underflow floor (a permitted slot the GPU wrongly denied shows up
    here even when its weight is far below the numeric tolerance).
    hidden, position_update and token_output, per row: a row is all zero on the GPU iff
    it is all zero in the oracle (unusable atoms, tokens without usable atoms)."""
    if "attention" in ref:
        r, g = ref["attention"], got["attention"]
        m = ~np.isnan(r)
        zero_ref = m & (r == 0.0)
        assert np.all(g[zero_ref] == 0.0), "attention: nonzero where the oracle is exactly zero"
        live_ref = m & (np.abs(r) > UNDERFLOW_FLOOR)
        denied = live_ref & (g == 0.0)
        assert not denied.any(), (
            f"attention: {int(denied.sum())} permitted slots are exactly zero on the GPU "
            f"(first at {tuple(int(i[0]) for i in np.nonzero(denied))})")
    for k in ("hidden", "position_update", "token_output"):
        if k not in ref:
            continue
        r, g = ref[k], got[k]
        rows_r = r.reshape(-1, r.shape[-1])
        rows_g = g.reshape(-1, g.shape[-1])
        m = ~np.isnan(rows_r).any(axis=1)
        zr = np.all(rows_r[m] == 0.0, axis=1)
        zg = np.all(rows_g[m] == 0.0, axis=1)
        assert np.array_equal(zr, zg), (
            f"{k}: {int((zr != zg).sum())} rows differ in being all zero "
            f"(oracle zero, GPU not: {int((zr & ~zg).sum())}; GPU zero, oracle not: "
            f"{int((zg & ~zr).sum())})")


def assert_status_clean(ws, what=""):
    """No bounded wait of the pass gave up (status bit 4 clear)."""
    st = atomenc.atomenc_get_status(ws)
    assert not st & atomenc.STATUS_WAIT_TIMEOUT, f"{what}: device status {st:#x} (bit 4: invalid)"


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
