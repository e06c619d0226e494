"""Invariants of the block that hold at any size, checked on the oracle with random
tiny workloads (brute-force style: every property follows from the page text)."""
import numpy as np
import pytest

import oracle
from sparse_windowed_atom_b200 import workloads
from tests.oracle_cases import clone, from_workload, run

COMBOS = [("af3", "encoder"), ("af3", "decoder"), ("esmfold2", "encoder"), ("esmfold2", "decoder")]


def small(style, stage, seed=0, **kw):
    spec = workloads.tiny_spec(style, stage, "float32", B=2, A=40, T=8, K=10, C=16, S=8, H=2,
                               D=8, P=4, M=16, U=12, V=10, keys=("blocked", 8, 4), **kw)
    return from_workload(workloads.make_inputs(spec, seed=seed))


@pytest.mark.parametrize("style,stage", COMBOS)
def test_outputs_finite_and_masked(style, stage):
    case = small(style, stage)
    out = run(oracle, case)
    use = oracle.usable(case["activations"], case["parameters"], case["masks"], case["structure"],
                        style=style, stage=stage)
    for v in out.values():
        assert np.all(np.isfinite(v))
    assert np.all(out["hidden"][~use] == 0.0)
    att = out["attention"]                                        # [B,H,A,K]
    rows = att.sum(-1)
    pm = oracle.permitted(case["activations"], case["parameters"], case["masks"],
                          case["structure"], radius=case["radius"], style=style, stage=stage)
    has = pm.any(-1)                                              # [B,A]
    for h in range(att.shape[1]):
        np.testing.assert_allclose(rows[:, h][has], 1.0, rtol=0, atol=1e-14)
        assert np.all(att[:, h][~has] == 0.0)                     # empty rows: exact zero
        assert np.all(att[:, h][~pm] == 0.0)
    if stage == "decoder":
        assert np.all(out["position_update"][~use] == 0.0)


@pytest.mark.parametrize("style,stage", COMBOS)
def test_slot_permutation(style, stage):
    """Permuting the slots of every row permutes the attention rows and leaves the
    rest unchanged (slots are an unordered set of softmax entries)."""
    case = small(style, stage, seed=1)
    out = run(oracle, case)
    K = case["structure"]["key_index"].shape[-1]
    perm = np.random.default_rng(3).permutation(K)
    c2 = clone(case)
    c2["structure"]["key_index"] = case["structure"]["key_index"][..., perm]
    c2["masks"]["window_mask"] = case["masks"]["window_mask"][..., perm]
    if style == "af3":
        c2["activations"]["pair"] = case["activations"]["pair"][:, :, perm]
    out2 = run(oracle, c2)
    np.testing.assert_allclose(out2["attention"], out["attention"][..., perm], rtol=1e-12, atol=1e-14)
    for k in out:
        if k != "attention":
            np.testing.assert_allclose(out2[k], out[k], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("style,stage", COMBOS)
def test_batch_independence(style, stage):
    """Key ids are within one batch element: no batch mixing."""
    case = small(style, stage, seed=2)
    out = run(oracle, case)
    for b in range(2):
        cb = clone(case)
        for grp in ("activations", "masks", "structure"):
            cb[grp] = {k: v[b:b + 1] for k, v in case[grp].items()}
        ob = run(oracle, cb)
        for k in out:
            np.testing.assert_array_equal(ob[k][0], out[k][b])


def test_duplicate_slots_are_separate_entries():
    """A key listed twice gets two equal entries; together they weigh as one entry
    whose logit is raised by ln 2."""
    case = small("af3", "encoder", seed=4, dup_p=0.0, miss_p=0.0, window_p=1.0, valid_p=1.0,
                 token_valid_p=1.0, poison_invalid=False, tokens=("fixed", 5))
    kid = case["structure"]["key_index"]
    a = 20
    row = kid[0, a].copy()
    assert len(set(row[row >= 0])) == len(row[row >= 0])
    c2 = clone(case)
    c2["structure"]["key_index"][0, a, 1] = row[0]                # slot 1 := slot 0
    c2["activations"]["pair"][0, a, 1] = case["activations"]["pair"][0, a, 0]
    out2 = run(oracle, c2)
    w = out2["attention"][0, :, a]                                # [H, K]
    np.testing.assert_allclose(w[:, 0], w[:, 1], rtol=1e-14, atol=0)
    # reference row: slot 1 masked, slot 0 logit + ln 2 is the same as doubling its weight
    c3 = clone(c2)
    c3["masks"]["window_mask"][0, a, 1] = False
    w3 = run(oracle, c3)["attention"][0, :, a]
    e0 = w3[:, 0] / (1.0 - w3[:, 0])                              # odds of slot 0 vs the rest
    combined = 2 * e0 / (1 + 2 * e0)
    np.testing.assert_allclose(w[:, 0] + w[:, 1], combined, rtol=1e-12)


@pytest.mark.parametrize("radius", [0, 1, 3, 6])
def test_radius_is_index_window(radius):
    case = small("esmfold2", "encoder", seed=5, radius=radius)
    out = run(oracle, case)
    c2 = clone(case)
    c2["radius"] = -1
    A = case["structure"]["key_index"].shape[1]
    far = np.abs(case["structure"]["key_index"] - np.arange(A)[None, :, None]) > radius
    c2["masks"]["window_mask"] = case["masks"]["window_mask"] & ~far
    out2 = run(oracle, c2)
    for k in out:
        np.testing.assert_array_equal(out[k], out2[k])


@pytest.mark.parametrize("style,stage", COMBOS)
def test_unusable_payloads_are_sanitised(style, stage):
    """NaN / Inf payloads on unusable atoms change nothing: replacing them with any
    finite values gives identical outputs."""
    case = small(style, stage, seed=6)
    use = oracle.usable(case["activations"], case["parameters"], case["masks"], case["structure"],
                        style=style, stage=stage)
    assert not np.all(np.isfinite(case["activations"]["atom"]))
    out = run(oracle, case)
    c2 = clone(case)
    rng = np.random.default_rng(0)
    for name in ("atom", "condition", "rope_cos", "rope_sin"):
        if name in c2["activations"]:
            arr = c2["activations"][name]
            arr[~use] = rng.normal(size=arr[~use].shape)
    if style == "af3":
        arr = c2["activations"]["pair"]
        arr[~use] = rng.normal(size=arr[~use].shape)
    out2 = run(oracle, c2)
    for k in out:
        np.testing.assert_array_equal(out[k], out2[k])


def test_pooling_counts_usable_atoms_only():
    case = small("af3", "encoder", seed=7)
    out = run(oracle, case)
    use = oracle.usable(case["activations"], case["parameters"], case["masks"], case["structure"])
    att = case["structure"]["atom_to_token"]
    T = case["masks"]["token_valid"].shape[1]
    w_pool = case["parameters"]["w_pool"]
    for b in range(2):
        for t in range(T):
            members = np.where(use[b] & (att[b] == t))[0]
            if len(members) == 0:
                assert np.all(out["token_output"][b, t] == 0.0)
            else:
                # ReLU(hidden @ w_pool) mean with numpy on the oracle's own hidden rows
                ref = np.maximum(out["hidden"][b, members] @ w_pool, 0).mean(0)
                np.testing.assert_allclose(out["token_output"][b, t], ref, rtol=1e-12, atol=1e-14)
    assert (~use).any()


@pytest.mark.parametrize("style", ["af3", "esmfold2"])
def test_decoder_with_zero_token_projection_matches_encoder(style):
    enc = small(style, "encoder", seed=8)
    dec = small(style, "decoder", seed=8)
    for grp in ("activations", "masks", "structure"):
        for k, v in enc[grp].items():
            if k in dec[grp]:
                dec[grp][k] = v.copy()
    for k, v in enc["parameters"].items():
        if k in dec["parameters"]:
            dec["parameters"][k] = v.copy()
    dec["parameters"]["w_token"][:] = 0.0
    oe, od = run(oracle, enc), run(oracle, dec)
    np.testing.assert_array_equal(oe["hidden"], od["hidden"])
    np.testing.assert_array_equal(oe["attention"], od["attention"])


@pytest.mark.parametrize("style,stage", COMBOS)
def test_query_select_matches_full(style, stage):
    case = small(style, stage, seed=9)
    full = run(oracle, case)
    sel = np.zeros(case["masks"]["valid"].shape, bool)
    sel[:, ::3] = True
    part = run(oracle, case, query_select=sel)
    A = sel.shape[1]
    for b in range(2):
        for a in range(A):
            if sel[b, a]:
                np.testing.assert_array_equal(part["hidden"][b, a], full["hidden"][b, a])
                np.testing.assert_array_equal(part["attention"][b, :, a], full["attention"][b, :, a])
            else:
                assert np.all(np.isnan(part["hidden"][b, a]))
    if stage == "encoder":
        ok = ~np.isnan(part["token_output"][..., 0])
        np.testing.assert_array_equal(part["token_output"][ok], full["token_output"][ok])


def test_argument_errors():
    case = small("esmfold2", "encoder")
    with pytest.raises(oracle.OracleError):
        run(oracle, case, eps=0.0)
    with pytest.raises(oracle.OracleError):
        run(oracle, case, eps=float("nan"))
    with pytest.raises(oracle.OracleError):
        run(oracle, case, radius=-2)
