"""Pins of the single-to-pair oracle (page "ESMFold Single-to-Pair Features",
esmfold_single_to_pair): the printed worked example, library reductions, masking and
NaN isolation, the optional output LayerNorm."""
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "single_to_pair_worked_example.json")


def _case(seed, B=2, N=7, C=12, H=3, Dp=5, p_present=0.75):
    rng = np.random.default_rng(seed)
    act = {"x": rng.normal(size=(B, N, C))}
    prm = {"weight": rng.normal(size=(C, 2 * H)) / np.sqrt(C), "bias": 0.1 * rng.normal(size=2 * H),
           "norm_scale": 1 + 0.1 * rng.normal(size=C), "norm_bias": 0.1 * rng.normal(size=C),
           "out_weight": rng.normal(size=(2 * H, Dp)) / np.sqrt(2 * H),
           "out_bias": 0.1 * rng.normal(size=Dp),
           "output_scale": 1 + 0.1 * rng.normal(size=Dp), "output_bias": 0.1 * rng.normal(size=Dp)}
    msk = {"mask": rng.random((B, N)) < p_present}
    msk["mask"][:, 0] = True
    return act, prm, msk


def test_worked_example():
    g = json.load(open(GOLDEN))
    pf, out = oracle.single_to_pair({k: np.array(v) for k, v in g["activations"].items()},
                                    {k: np.array(v) for k, v in g["parameters"].items()},
                                    {k: np.array(v) for k, v in g["masks"].items()},
                                    eps=g["eps"], output_norm=g["output_norm"])
    np.testing.assert_allclose(pf, np.array(g["expected"]["pair_features"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(out, np.array(g["expected"]["output"]), rtol=0, atol=1e-15)


@pytest.mark.parametrize("output_norm", [False, True])
def test_library_reduction(output_norm):
    """torch layer_norm / linear on the present tokens reproduce every present pair."""
    act, prm, msk = _case(3)
    eps = 1e-3
    pf, out = oracle.single_to_pair(act, prm, msk, eps=eps, output_norm=output_norm)
    t = {k: torch.tensor(v) for k, v in prm.items()}
    x = torch.tensor(act["x"])
    C = x.shape[-1]
    qk = torch.nn.functional.layer_norm(x, (C,), t["norm_scale"], t["norm_bias"], eps) @ t["weight"] + t["bias"]
    H = qk.shape[-1] // 2
    q, k = qk[..., :H], qk[..., H:]
    prod = torch.einsum("bih,bjh->bijh", k, q)                 # k_i * q_j
    diff = q[:, None, :, :] - k[:, :, None, :]                 # q_j - k_i
    f = torch.cat([prod, diff], dim=-1)
    o = torch.nn.functional.linear(f, t["out_weight"].T, t["out_bias"])
    if output_norm:
        o = torch.nn.functional.layer_norm(o, (o.shape[-1],), t["output_scale"], t["output_bias"], eps)
    m = torch.tensor(msk["mask"])
    both = (m[:, :, None] & m[:, None, :]).numpy()
    np.testing.assert_allclose(pf[both], f.numpy()[both], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out[both], o.numpy()[both], rtol=1e-12, atol=1e-12)


def test_absent_endpoints_give_exact_zeros_and_isolate_nan():
    act, prm, msk = _case(5)
    x = act["x"].copy()
    x[~msk["mask"]] = np.nan
    x[0, np.where(~msk["mask"][0])[0][:1]] = np.inf if (~msk["mask"][0]).any() else x[0, :0]
    pf, out = oracle.single_to_pair({"x": x}, prm, msk, output_norm=True)
    pf0, out0 = oracle.single_to_pair(act, prm, msk, output_norm=True)
    m = msk["mask"]
    both = m[:, :, None] & m[:, None, :]
    assert np.all(pf[~both] == 0.0) and np.all(out[~both] == 0.0)
    assert np.array_equal(pf, pf0) and np.array_equal(out, out0)


def test_direction_matters_and_product_is_symmetric_in_q_k_swap():
    """pair(i, j) and pair(j, i) share nothing in general, but with weight columns such
    that k = q the product channels agree both ways and the differences are opposite."""
    act, prm, msk = _case(7, B=1, N=5)
    msk["mask"][:] = True
    pf, _ = oracle.single_to_pair(act, prm, msk)
    H = pf.shape[-1] // 2
    assert not np.allclose(pf[0, 1, 2], pf[0, 2, 1])
    w = prm["weight"].copy()
    w[:, H:] = w[:, :H]
    b = prm["bias"].copy()
    b[H:] = b[:H]
    pf2, _ = oracle.single_to_pair(act, dict(prm, weight=w, bias=b), msk)
    np.testing.assert_allclose(pf2[0, 1, 2, :H], pf2[0, 2, 1, :H], rtol=1e-14)
    np.testing.assert_allclose(pf2[0, 1, 2, H:], -pf2[0, 2, 1, H:], rtol=1e-14)
    np.testing.assert_allclose(pf2[0, 3, 3, H:], 0.0, atol=1e-15)
