"""Single-to-pair features (page "ESMFold Single-to-Pair Features"): host-side argument
checks of the C ABI (no GPU needed) and parity of the CUDA pass with the oracle (gpu)."""
import ctypes
import json
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_windowed_atom_b200 import atomenc

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "single_to_pair_worked_example.json")
TOL = {torch.float32: 2e-4, torch.bfloat16: 2e-2}


def _case(seed, B=2, N=37, C=64, H=16, Dp=48, p_present=0.8, poison=True):
    rng = np.random.default_rng(seed)
    act = {"x": rng.normal(size=(B, N, C))}
    prm = {"weight": rng.normal(size=(C, 2 * H)) / np.sqrt(C), "bias": 0.1 * rng.normal(size=2 * H),
           "norm_scale": 1 + 0.1 * rng.normal(size=C), "norm_bias": 0.1 * rng.normal(size=C),
           "out_weight": rng.normal(size=(2 * H, Dp)) / np.sqrt(2 * H),
           "out_bias": 0.1 * rng.normal(size=Dp),
           "output_scale": 1 + 0.1 * rng.normal(size=Dp), "output_bias": 0.1 * rng.normal(size=Dp)}
    msk = {"mask": rng.random((B, N)) < p_present}
    if poison:
        act["x"][~msk["mask"]] = np.nan
    return act, prm, msk


def _torch(d, dtype, device):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).to(device=device, dtype=dtype)
            for k, v in d.items()}


def _structs(act, prm, msk, pf, out):
    return atomenc._s2p_structs(act, prm, msk, {"pair_features": pf, "output": out})


def _rc(act, prm, msk, pf, out, eps=1e-5, onorm=0, ws=None, nbytes=1 << 20):
    ins, p, o = _structs(act, prm, msk, pf, out)
    lib = atomenc.load_library()
    buf = ws if ws is not None else torch.empty(nbytes + 256, dtype=torch.uint8)
    ptr = (buf.data_ptr() + 255) // 256 * 256 if ws is None else 0
    return lib.atomenc_single_to_pair(ctypes.byref(ins), ctypes.byref(p), eps, onorm, ctypes.byref(o),
                                      ptr, nbytes if ws is None else 0, None)


def test_argument_errors_are_decided_on_the_host():
    a, p, m = _case(1, B=1, N=4, C=8, H=2, Dp=3)
    act, prm = _torch(a, torch.float32, "cpu"), _torch(p, torch.float32, "cpu")
    msk = {"mask": torch.from_numpy(m["mask"])}
    pf, out = torch.empty(1, 4, 4, 4), torch.empty(1, 4, 4, 3)
    assert _rc(act, prm, {"mask": msk["mask"].to(torch.int64)}, pf, out) == -3      # mask dtype
    assert _rc(act, dict(prm, weight=prm["weight"][:, :3].contiguous()), msk, pf, out) == -4  # odd 2H
    assert _rc(act, prm, msk, torch.empty(1, 4, 4, 5), out) == -4                    # output shape
    assert _rc(act, prm, msk, pf, out, eps=0.0) == -6                                # eps
    big = {"weight": torch.zeros(8, 258), "bias": torch.zeros(258)}
    assert _rc(act, dict(prm, **big, out_weight=torch.zeros(258, 3)), msk,
               torch.empty(1, 4, 4, 258), out) == -9                                 # 2H > 256
    assert _rc(act, dict(prm, output_scale=None), msk, pf, out, onorm=1) == -1      # missing tensor
    assert _rc(act, prm, msk, pf, out, ws=torch.empty(0)) == -10                    # workspace


def _check(seed, dtype, output_norm, **kw):
    a, p, m = _case(seed, **kw)
    eps = 1e-4
    act, prm = _torch(a, dtype, "cuda"), _torch(p, dtype, "cuda")
    # the oracle sees the values the GPU sees (bf16 rounding of every float input)
    a64 = {k: v.double().cpu().numpy() for k, v in act.items()}
    p64 = {k: v.double().cpu().numpy() for k, v in prm.items()}
    ref_pf, ref_out = oracle.single_to_pair(a64, p64, m, eps=eps, output_norm=output_norm)
    msk = {"mask": torch.from_numpy(m["mask"]).cuda()}
    pf, out = atomenc.single_to_pair(act, prm, msk, eps=eps, output_norm=output_norm)
    torch.cuda.synchronize()
    tol = TOL[dtype]
    for got, ref in ((pf, ref_pf), (out, ref_out)):
        g = got.double().cpu().numpy()
        assert np.all(np.isfinite(g))
        err = np.abs(g - ref)
        assert np.all(err <= tol * (1 + np.abs(ref))), float((err / (1 + np.abs(ref))).max())
        both = m["mask"][:, :, None] & m["mask"][:, None, :]
        assert np.all(g[~both] == 0.0)                    # absent endpoints: exact zeros


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("output_norm", [False, True])
def test_parity(dtype, output_norm):
    _check(11, dtype, output_norm)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("output_norm", [False, True])
@pytest.mark.parametrize("kw", [dict(B=2, N=150, C=64, H=32, Dp=128), dict(B=1, N=130, C=96, H=64, Dp=96),
                                dict(B=1, N=40, C=32, H=16, Dp=256)])
def test_parity_tensor_core_readout(dtype, output_norm, kw):
    """2H and D multiples of 32 (2H <= 128, D <= 256): the tensor-core readout, with a
    ragged last tile of pairs, two k chunks (2H = 128), a padded output tile (D = 96) and
    two output tiles (D = 256)."""
    _check(17, dtype, output_norm, **kw)


@pytest.mark.gpu
@pytest.mark.parametrize("kw", [dict(B=1, N=1, C=5, H=1, Dp=3), dict(B=3, N=33, C=130, H=128, Dp=64),
                                dict(B=1, N=65, C=96, H=32, Dp=256), dict(B=2, N=20, p_present=0.0)])
def test_shapes_and_edges(kw):
    _check(12, torch.float32, True, **kw)


@pytest.mark.gpu
def test_worked_example_on_gpu():
    g = json.load(open(GOLDEN))
    f = lambda d: {k: torch.tensor(v, dtype=torch.float32, device="cuda") for k, v in d.items()}
    pf, out = atomenc.single_to_pair(f(g["activations"]), f(g["parameters"]),
                                     {"mask": torch.tensor(g["masks"]["mask"], device="cuda")},
                                     eps=g["eps"], output_norm=g["output_norm"])
    np.testing.assert_allclose(pf.cpu().numpy(), np.array(g["expected"]["pair_features"]), atol=1e-6)
    np.testing.assert_allclose(out.cpu().numpy(), np.array(g["expected"]["output"]), atol=1e-6)


@pytest.mark.gpu
def test_full_size_sampled():
    """B=1, N=384, C=128, 2H=64, Dp=128: every pair of 24 sampled rows i against the oracle
    run on those rows' tokens and all columns."""
    a, p, m = _case(13, B=1, N=384, C=128, H=32, Dp=128)
    act, prm = _torch(a, torch.float32, "cuda"), _torch(p, torch.float32, "cuda")
    pf, out = atomenc.single_to_pair(act, prm, {"mask": torch.from_numpy(m["mask"]).cuda()},
                                     eps=1e-5, output_norm=True)
    torch.cuda.synchronize()
    ref_pf, ref_out = oracle.single_to_pair(a, p, m, eps=1e-5, output_norm=True)
    rows = np.random.default_rng(0).choice(384, 24, replace=False)
    for got, ref in ((pf, ref_pf), (out, ref_out)):
        g = got.cpu().numpy()[:, rows]
        r = ref[:, rows]
        assert np.all(np.abs(g - r) <= 2e-4 * (1 + np.abs(r)))
