"""GPU parity: the CUDA library against the float64 oracle, element by element.

Tolerance (max |err| <= tol (1 + |ref|)): 2e-4 for float32 storage, 2e-2 for bf16
storage. Masking, eligibility and empty-row decisions are exact (zeros match exactly).
"""
import numpy as np
import pytest
import torch

from sparse_windowed_atom_b200 import atomenc, workloads
from tests.cuda_harness import (TOL, assert_status_clean, compare, exact_zero_pattern, run_cuda,
                                run_oracle, sample_queries, to_torch)
from tests.oracle_cases import load_golden

pytestmark = pytest.mark.gpu

COMBOS = [(s, g, d) for s in ("af3", "esmfold2") for g in ("encoder", "decoder")
          for d in ("float32", "bfloat16")]


def _check(w, what, **over):
    got = run_cuda(w, **over)
    ref = run_oracle(w, **over)
    compare(got, ref, w["spec"].dtype, what)
    exact_zero_pattern(got, ref)
    return got, ref


@pytest.mark.parametrize("style,stage,dtype", COMBOS)
def test_tiny_parity(style, stage, dtype):
    """Several query tiles plus a ragged tail, duplicates, missing ids, NaN payloads."""
    w = workloads.make_inputs(workloads.tiny_spec(style, stage, dtype), seed=3)
    _check(w, f"{style}/{stage}/{dtype}")


@pytest.mark.parametrize("style", ["af3", "esmfold2"])
@pytest.mark.parametrize("radius", [0, 3, 17])
def test_radius_window(style, radius):
    w = workloads.make_inputs(workloads.tiny_spec(style, "encoder", radius=radius), seed=4)
    _check(w, f"radius {radius}")


@pytest.mark.parametrize("style", ["af3", "esmfold2"])
def test_empty_windows_and_all_invalid(style):
    w = workloads.make_inputs(workloads.tiny_spec(style, "encoder", window_p=0.0), seed=5)
    got, _ = _check(w, "empty windows")
    assert np.all(got["attention"] == 0.0)
    w = workloads.make_inputs(workloads.tiny_spec(style, "decoder", valid_p=0.0), seed=5)
    got, _ = _check(w, "all invalid")
    assert np.all(got["hidden"] == 0.0) and np.all(got["position_update"] == 0.0)


@pytest.mark.parametrize("style", ["af3", "esmfold2"])
def test_single_atom(style):
    spec = workloads.tiny_spec(style, "encoder", B=1, A=1, T=1, K=1, keys=("blocked", 1, 0),
                               tokens=("fixed", 1), valid_p=1.0, token_valid_p=1.0, window_p=1.0,
                               dup_p=0.0, miss_p=0.0, poison_invalid=False)
    got, _ = _check(workloads.make_inputs(spec, seed=6), "single atom")
    assert np.all(got["attention"] == 1.0)


def test_wide_random_keys_take_the_unstaged_path():
    """Keys spread over +-1500 atoms exceed the shared-memory stage; the kernel gathers
    them from L2 instead, with the same result."""
    spec = workloads.tiny_spec("esmfold2", "encoder", A=3000, T=400, K=40, keys=("random", 1500),
                               D=32, H=4)
    w = workloads.make_inputs(spec, seed=7)
    act, prm, msk, st = to_torch(w)
    outs = {k: torch.empty(s, device="cuda") for k, s in
            atomenc.output_shapes("esmfold2", "encoder", {**act, **msk, **st}, prm).items()}
    ws = torch.empty(atomenc.atomenc_workspace_size("esmfold2", "encoder", {**act, **msk, **st},
                                                    prm, outs), dtype=torch.uint8, device="cuda")
    atomenc.atomenc_forward("esmfold2", "encoder", {**act, **msk, **st}, prm, spec.eps,
                            spec.radius, outs, ws)
    assert atomenc.atomenc_get_status(ws) & 1
    assert_status_clean(ws, "unstaged keys")
    _check(w, "unstaged keys")


def test_unsorted_atom_to_token():
    spec = workloads.tiny_spec("af3", "encoder")
    w = workloads.make_inputs(spec, seed=8)
    rng = np.random.default_rng(0)
    for b in range(spec.B):
        w["structure"]["atom_to_token"][b] = rng.permutation(w["structure"]["atom_to_token"][b])
    _check(w, "unsorted tokens")


@pytest.mark.parametrize("D,H", [(5, 3), (8, 2), (64, 2)])
def test_af3_head_widths(D, H):
    spec = workloads.tiny_spec("af3", "encoder", D=D, H=H, K=70, P=7)
    _check(workloads.make_inputs(spec, seed=9), f"D={D}")


@pytest.mark.parametrize("D,H", [(2, 4), (8, 4), (16, 8), (64, 2)])
def test_esmfold2_head_widths(D, H):
    spec = workloads.tiny_spec("esmfold2", "decoder", D=D, H=H, K=150)
    _check(workloads.make_inputs(spec, seed=10), f"D={D}")


@pytest.mark.parametrize("dtype,A,radius,valid_p", [("float32", 900, 64, 1.0), ("float32", 700, 64, 0.9),
                                                   ("bfloat16", 611, -1, 1.0)])
def test_blocked_windows_with_shared_rows(dtype, A, radius, valid_p):
    """128 slots in blocked windows: queries whose slots name the same key rows are
    processed in pairs (each with its own mask), tiles whose pairs differ and odd tails
    one query at a time."""
    spec = workloads.tiny_spec("esmfold2", "encoder", dtype=dtype, A=A, T=120, K=128,
                               keys=("blocked", 32, 48), radius=radius, dup_p=0.0, miss_p=0.0,
                               window_p=1.0 if valid_p == 1.0 else 0.9, valid_p=valid_p)
    _check(workloads.make_inputs(spec, seed=23), f"blocked A={A}")


@pytest.mark.parametrize("style,stage", [("af3", "encoder"), ("esmfold2", "decoder")])
@pytest.mark.parametrize("dtype", ["float32", "bfloat16"])
@pytest.mark.parametrize("C,S", [(24, 40), (20, 36), (10, 8)])
def test_operand_widths_off_the_vector_path(style, stage, dtype, C, S):
    """Channel widths below one 64-wide k chunk: K a multiple of 8 takes the pipelined
    operand loads with a partial chunk (k past K clamped and zeroed), K not a multiple of
    8 the per-element loads; C != 128 also runs the tail unfused. C = 2 mod 4 puts the
    last eight-column group of a 2C-wide gate row past the row's end."""
    spec = workloads.tiny_spec(style, stage, dtype, C=C, S=S, H=2, D=8, M=40, U=28, V=20)
    _check(workloads.make_inputs(spec, seed=31), f"C={C} S={S}")


@pytest.mark.parametrize("style,C,S", [("esmfold2", 24, 36), ("af3", 40, 24)])
def test_persistent_products_with_odd_widths(style, C, S):
    """448 row blocks of bf16 rows (every product on the persistent kernel, formed
    operands included) with widths whose operands take the pipelined loads with a partial
    k chunk and the per-element loads; a seeded sample of whole tokens checked against the
    oracle."""
    spec = workloads.tiny_spec(style, "encoder", "bfloat16", B=1, A=448 * 128, T=7000, K=24,
                               C=C, S=S, H=2, D=8, M=40, U=28, keys=("random", 64),
                               tokens=("ragged", 16), radius=-1)
    w = workloads.make_inputs(spec, seed=37)
    got = run_cuda(w)
    ref = run_oracle(w, query_select=sample_queries(spec, w, frac=0.01))
    compare(got, ref, spec.dtype, f"persistent {style} C={C} S={S}")
    exact_zero_pattern(got, ref)


@pytest.mark.parametrize("style,stage", [("af3", "encoder"), ("esmfold2", "decoder")])
def test_unaligned_atom_and_condition_rows(style, stage):
    """atom and condition views that start one element into their storage (dense, but not
    16-byte aligned) take the general row-preparation kernel; same results."""
    w = workloads.make_inputs(workloads.tiny_spec(style, stage), seed=29)
    ref = run_oracle(w)
    act, prm, msk, st = to_torch(w)
    for k in ("atom", "condition"):
        v = act[k]
        buf = torch.empty(v.numel() + 1, dtype=v.dtype, device=v.device)
        view = buf[1:].view(v.shape)
        view.copy_(v)
        assert view.data_ptr() % 16 != 0
        act[k] = view
    spec = w["spec"]
    out = atomenc.windowed_atom_attention(act, prm, msk, st, eps=spec.eps, style=style,
                                          stage=stage, radius=spec.radius)
    torch.cuda.synchronize()
    got = {k: v.float().cpu().numpy().astype(np.float64) for k, v in out.items()}
    compare(got, ref, spec.dtype, "unaligned rows")
    exact_zero_pattern(got, ref)


@pytest.mark.parametrize("eps", [1.0, 1e-3])
def test_eps(eps):
    w = workloads.make_inputs(workloads.tiny_spec("af3", "decoder"), seed=11)
    _check(w, f"eps {eps}", eps=eps)


@pytest.mark.parametrize("name,style", [("af3_encoder_worked_example.json", "af3"),
                                        ("esmfold2_encoder_worked_example.json", "esmfold2")])
def test_worked_examples_on_gpu(name, style):
    g, case = load_golden(name)
    dev = "cuda"
    f = lambda v: torch.tensor(v, dtype=torch.float32, device=dev)
    act = {k: f(v) for k, v in case["activations"].items()}
    prm = {k: f(v) for k, v in case["parameters"].items()}
    msk = {k: torch.tensor(v, device=dev) for k, v in case["masks"].items()}
    st = {k: torch.tensor(v, device=dev) for k, v in case["structure"].items()}
    out = atomenc.windowed_atom_attention(act, prm, msk, st, eps=case["eps"], style=style,
                                          stage="encoder")
    import math
    if style == "af3":
        p = 1 / (1 + math.exp(-0.25 / math.sqrt(2)))
        d = (2 * p - 1) / 16
        exp_tok0 = ((1 - d) + (4 + 1 / 16)) / 2
    else:
        l, h = 1.0, 3.0
        r = math.sqrt((l * l + h * h) / 2 + 1)
        p = 1 / (1 + math.exp(-2 * l * l / ((l * l + h * h + 1) * math.sqrt(2))))
        exp_tok0 = (l + (p * l + (1 - p) * h) / (2 * r) + h + h / (2 * r)) / 2
    att = out["attention"].cpu().double().numpy()
    assert abs(att[0, 0, 0, 0] - p) < 2e-6
    assert att[0, 0, 1, 0] == 0.0 and att[0, 0, 1, 1] == 1.0
    assert abs(out["token_output"][0, 0, 0].item() - exp_tok0) < 2e-5


def test_deterministic_and_inputs_untouched():
    w = workloads.make_inputs(workloads.tiny_spec("af3", "encoder", A=700, T=90), seed=12)
    act, prm, msk, st = to_torch(w)
    before = {k: v.clone() for d in (act, prm, msk, st) for k, v in d.items()}
    o1 = atomenc.windowed_atom_attention(act, prm, msk, st, style="af3", stage="encoder")
    o2 = atomenc.windowed_atom_attention(act, prm, msk, st, style="af3", stage="encoder")
    torch.cuda.synchronize()
    for k in o1:
        assert torch.equal(o1[k], o2[k]), k
    for d in (act, prm, msk, st):
        for k, v in d.items():
            assert torch.equal(v, before[k]) or (torch.isnan(v) == torch.isnan(before[k])).all() \
                and torch.equal(torch.nan_to_num(v), torch.nan_to_num(before[k])), k


@pytest.mark.parametrize("style", ["af3", "esmfold2"])
def test_prepared_forward_matches_the_plain_call(style):
    """atomenc.Forward (descriptors built once) gives bit-identical results to
    atomenc_forward, call after call."""
    w = workloads.make_inputs(workloads.tiny_spec(style, "encoder", A=500, T=64), seed=21)
    act, prm, msk, st = to_torch(w)
    spec = w["spec"]
    ref = atomenc.windowed_atom_attention(act, prm, msk, st, style=style, stage="encoder",
                                          eps=spec.eps, radius=spec.radius)
    inputs = {**act, **msk, **st}
    outs = {k: torch.empty_like(v) for k, v in ref.items()}
    ws = torch.empty(atomenc.atomenc_workspace_size(style, "encoder", inputs, prm, outs),
                     dtype=torch.uint8, device="cuda")
    fwd = atomenc.Forward(style, "encoder", inputs, prm, spec.eps, spec.radius, outs, ws)
    for _ in range(2):
        for v in outs.values():
            v.fill_(7.0)
        fwd()
        torch.cuda.synchronize()
        assert_status_clean(ws, "prepared forward")
        for k in ref:
            assert torch.equal(outs[k], ref[k]), k


def test_argument_errors_are_reported():
    w = workloads.make_inputs(workloads.tiny_spec("esmfold2", "encoder"), seed=13)
    act, prm, msk, st = to_torch(w)
    with pytest.raises(atomenc.AtomencError):
        atomenc.windowed_atom_attention(act, prm, msk, st, eps=0.0, style="esmfold2",
                                        stage="encoder")
    with pytest.raises(atomenc.AtomencError):
        atomenc.windowed_atom_attention(act, prm, msk, st, radius=-3, style="esmfold2",
                                        stage="encoder")
    bad = dict(act)
    bad["rope_cos"] = act["rope_cos"][..., :-1].contiguous()
    with pytest.raises((atomenc.AtomencError, ValueError)):
        atomenc.windowed_atom_attention(bad, prm, msk, st, style="esmfold2", stage="encoder")


# ------------------------------------------------------------------ full-size workloads

@pytest.mark.parametrize("name", workloads.WORKLOAD_ORDER)
def test_reference_workload_sampled(name):
    """Each reference workload at full size, in the launch configuration the benchmark
    times; the oracle computes a seeded sample of whole tokens and scattered atoms."""
    spec = workloads.WORKLOADS[name]
    w = workloads.make_inputs(spec, seed=0)
    got = run_cuda(w)
    sel = sample_queries(spec, w, frac=0.01 if spec.A > 4096 else 1.0)
    ref = run_oracle(w, query_select=sel)
    compare(got, ref, spec.dtype, name)
    exact_zero_pattern(got, ref)
    # properties that hold everywhere: rows sum to 1 or are empty; masked rows zero
    att = got["attention"]
    s = att.sum(-1)
    assert np.all((np.abs(s - 1) < 50 * TOL[spec.dtype]) | (s == 0))
