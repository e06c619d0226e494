"""GPU parity of the attention core's gradient (atomenc_attention_backward) against the
float64 oracle (orc_attention_core_backward, pinned by finite differences).

Inputs are seeded and synthetic: q, k, v, value-gate logits ~ N(0, 1) (bf16 cases
rounded to bf16 once, so both sides see the same values), key ids drawn as the
workloads draw them (blocked windows, or random within +-w of the query) with
duplicated slots inside one row and keys shared by many queries, missing and
out-of-range ids, unusable atoms, window masks, radius windows, empty rows. Tolerance
as in the forward parity tests: |err| <= tol (1 + |ref|), 2e-4 float32, 2e-2 bf16."""
import numpy as np
import pytest
import torch

import oracle
from sparse_windowed_atom_b200 import atomenc
from sparse_windowed_atom_b200.workloads import round_to_bf16

pytestmark = pytest.mark.gpu
TOL = {"float32": 2e-4, "bfloat16": 2e-2}


def _case(style, dtype, seed, B=2, A=300, K=40, H=4, D=32, P=16, keys="random", radius=-1):
    rng = np.random.default_rng(seed)
    HD = H * D
    f = (lambda x: round_to_bf16(x.astype(np.float32))) if dtype == "bfloat16" else \
        (lambda x: x.astype(np.float32))
    core = {n: f(rng.normal(size=(B, A, HD))) for n in ("q", "k", "v", "g")}
    a = np.arange(A)[:, None]
    if keys == "blocked":
        kid = (a // 16) * 16 - 8 + np.arange(K)[None, :]
        kid = np.where((kid >= 0) & (kid < A), kid, -1)
        kid = np.broadcast_to(kid, (B, A, K)).copy()
    else:
        kid = a[None] + rng.integers(-25, 26, size=(B, A, K))
    kid[:, :, 3] = kid[:, :, 2]                     # a duplicated slot in every row
    kid[:, ::7, 5] = -1                             # missing
    kid[:, ::11, 6] = A + 3                         # out of range
    core["key_index"] = kid.astype(np.int64)
    core["window_mask"] = rng.random((B, A, K)) < 0.9
    core["usable"] = rng.random((B, A)) < 0.92
    core["window_mask"][:, 17] = False             # an empty row
    if style == "af3":
        core["pair"] = f(rng.normal(size=(B, A, K, P)))
        core["pair_scale"] = f(1 + 0.1 * rng.normal(size=P))
        core["w_pair"] = f(rng.normal(size=(P, H)) / np.sqrt(P))
    d_out = f(rng.normal(size=(B, A, HD)))
    d_att = f(rng.normal(size=(B, H, A, K)))
    return core, d_out, d_att


def _run_gpu(core, H, d_out, d_att, style, dtype, radius):
    fdt = torch.bfloat16 if dtype == "bfloat16" else torch.float32
    dev = "cuda"
    t = {}
    for n, v in core.items():
        if v.dtype in (np.float32, np.float64):
            t[n] = torch.from_numpy(np.ascontiguousarray(v)).to(dev, dtype=fdt)
        else:
            t[n] = torch.from_numpy(np.ascontiguousarray(v)).to(dev)
    dO = torch.from_numpy(d_out).to(dev, dtype=fdt)
    dA = None if d_att is None else torch.from_numpy(d_att).to(dev, dtype=fdt)
    g = atomenc.attention_backward(t, H, dO, dA, style=style, radius=radius)
    torch.cuda.synchronize()
    return {k: v.double().cpu().numpy() for k, v in g.items()}


def _compare(got, ref, dtype, what):
    tol = TOL[dtype]
    for k, r in ref.items():
        g = got[k]
        assert g.shape == r.shape, (k, g.shape, r.shape)
        err = np.abs(g - r)
        bound = tol * (1.0 + np.abs(r))
        bad = err > bound
        assert not bad.any(), (f"{what} {k}: {int(bad.sum())} of {r.size} out of tolerance; "
                               f"worst err {float((err / bound).max()):.3g} x bound")


@pytest.mark.parametrize("style", ["af3", "esmfold2"])
@pytest.mark.parametrize("dtype", ["float32", "bfloat16"])
@pytest.mark.parametrize("keys,radius", [("random", -1), ("random", 9), ("blocked", -1)])
def test_core_gradient_matches_oracle(style, dtype, keys, radius):
    H, D = (4, 32) if style == "af3" else (8, 16)
    core, d_out, d_att = _case(style, dtype, seed=51 + radius, H=H, D=D, keys=keys)
    got = _run_gpu(core, H, d_out, d_att, style, dtype, radius)
    ref = oracle.attention_core_backward(core, H, d_out, d_att, style=style, radius=radius)
    _compare(got, ref, dtype, f"{style}/{dtype}/{keys}/{radius}")


@pytest.mark.parametrize("D,H", [(16, 2), (64, 2), (8, 4)])
def test_core_gradient_head_widths_and_no_weight_gradient(D, H):
    core, d_out, _ = _case("esmfold2", "float32", seed=61, A=150, K=24, H=H, D=D)
    got = _run_gpu(core, H, d_out, None, "esmfold2", "float32", -1)
    ref = oracle.attention_core_backward(core, H, d_out, None, style="esmfold2")
    _compare(got, ref, "float32", f"D={D}")


def test_core_gradient_is_deterministic():
    """Keys shared by many slots: the fixed-point sums give bit-identical gradients on
    every run."""
    core, d_out, d_att = _case("af3", "float32", seed=71, A=400, K=64)
    a = _run_gpu(core, 4, d_out, d_att, "af3", "float32", -1)
    b = _run_gpu(core, 4, d_out, d_att, "af3", "float32", -1)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
