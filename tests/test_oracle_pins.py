"""Pins of the CPU float64 oracle to the pages, closed forms and library routines.

Each test fixes a value that the pages or the mathematics decide, so that a
plausible slip in the oracle (a dropped term, a wrong stage or head index, a
transposed weight, a sign) fails one of them.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle
from tests.oracle_cases import clone, ln2, load_golden, rms2, run, sig

pytestmark = pytest.mark.filterwarnings("ignore")


# --------------------------------------------------------------- worked examples

def test_af3_worked_example():
    """AlphaFold 3 Atom Attention Encoder, Worked example: p = sigmoid(0.25/sqrt 2)
    ~ 0.544079, update [-d, d] with d = (2p-1)/16, query 1 update [1/16, -1/16],
    pooled channel 0 = ((1-d) + (4+1/16))/2."""
    g, case = load_golden("af3_encoder_worked_example.json")
    out = run(oracle, case)
    p = sig(0.25 / math.sqrt(2.0))
    assert abs(p - g["page_values"]["first_key_weight_p"]) < 5e-7
    d = (2 * p - 1) / 16
    att = out["attention"]
    np.testing.assert_allclose(att[0, 0, 0], [p, 1 - p], rtol=0, atol=1e-15)
    assert att[0, 0, 1, 0] == 0.0 and att[0, 0, 1, 1] == 1.0     # single permitted slot
    np.testing.assert_allclose(out["hidden"][0, 0], [1 - d, 3 + d], rtol=0, atol=1e-14)
    np.testing.assert_allclose(out["hidden"][0, 1] - case["activations"]["atom"][0, 1],
                               g["page_values"]["query1_update"], rtol=0, atol=1e-15)
    assert abs(out["token_output"][0, 0, 0] - ((1 - d) + (4 + 1 / 16)) / 2) < 1e-14
    # channel 1 by the same algebra (both hidden channels are positive, ReLU keeps them)
    assert abs(out["token_output"][0, 0, 1] - ((3 + d) + (2 - 1 / 16)) / 2) < 1e-14


def test_esmfold2_worked_example():
    """ESMFold 2 Atom Attention Encoder, Worked example: self weight
    p = sigmoid(2 l^2 / ((l^2+h^2+1) sqrt 2)), hidden channel 0 = l + [p l + (1-p) h]/(2r),
    r = sqrt((l^2+h^2)/2 + 1); query 1 uses only its own key; mean pooling."""
    g, case = load_golden("esmfold2_encoder_worked_example.json")
    out = run(oracle, case)
    l, h = g["page_values"]["l"], g["page_values"]["h"]
    r = math.sqrt((l * l + h * h) / 2 + 1)
    p = sig(2 * l * l / ((l * l + h * h + 1) * math.sqrt(2.0)))
    np.testing.assert_allclose(out["attention"][0, 0, 0], [p, 1 - p], rtol=0, atol=1e-15)
    assert out["attention"][0, 0, 1, 0] == 0.0 and out["attention"][0, 0, 1, 1] == 1.0
    hid = out["hidden"][0]
    assert abs(hid[0, 0] - (l + (p * l + (1 - p) * h) / (2 * r))) < 1e-14
    assert abs(hid[0, 1] - (h + (p * h + (1 - p) * l) / (2 * r))) < 1e-14
    np.testing.assert_allclose(hid[1], [h + h / (2 * r), l + l / (2 * r)], rtol=0, atol=1e-14)
    np.testing.assert_allclose(out["token_output"][0, 0], hid.mean(axis=0), rtol=0, atol=1e-14)


# --------------------------------------------------------------- row helpers vs library

@pytest.mark.parametrize("n,eps", [(1, 1e-5), (2, 3.0), (7, 1e-5), (128, 1e-5), (33, 0.5)])
def test_layer_norm_matches_torch(n, eps):
    v = np.random.default_rng(n).normal(size=n) * 3 + 1.5
    ref = F.layer_norm(torch.tensor(v, dtype=torch.float64), (n,), eps=eps).numpy()
    np.testing.assert_allclose(oracle.layer_norm(v, eps), ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("n,eps", [(1, 1e-5), (2, 1.0), (16, 1e-5), (128, 1e-6)])
def test_rms_norm_matches_torch(n, eps):
    v = np.random.default_rng(n + 100).normal(size=n) * 2 - 0.5
    ref = F.rms_norm(torch.tensor(v, dtype=torch.float64), (n,), eps=eps).numpy()
    np.testing.assert_allclose(oracle.rms_norm(v, eps), ref, rtol=1e-12, atol=1e-13)


def test_sigmoid_silu_match_scipy_including_subnormal_tail():
    zs = [-700.0, -30.0, -1.0, 0.0, 0.3, 5.0, 40.0, 800.0]
    for z in zs:
        assert oracle.sigmoid(z) == pytest.approx(scipy.special.expit(z), rel=1e-14, abs=0)
        assert oracle.silu(z) == pytest.approx(z * scipy.special.expit(z), rel=1e-14, abs=0)
    # a representable subnormal tail is kept, not flushed (windowed page, last bullet):
    # for z << 0, sigmoid(z) = e^z / (1 + e^z) and 1 + e^z rounds to 1
    for z in (-740.0, -744.0):
        assert oracle.sigmoid(z) == math.exp(z) and 0.0 < oracle.sigmoid(z) < 1e-300
        assert oracle.silu(z) == z * math.exp(z)


@pytest.mark.parametrize("D", [2, 4, 16, 32])
def test_rope_is_complex_rotation(D):
    """With one angle per dim pair (d, d+D/2), q*cos + rotate_half(q)*sin turns each
    pair (q_d, q_{d+D/2}) as the complex number q_d + i q_{d+D/2} times e^{i theta}."""
    rng = np.random.default_rng(D)
    q = rng.normal(size=D)
    th = rng.uniform(0, 2 * np.pi, size=D // 2)
    cos = np.concatenate([np.cos(th), np.cos(th)])
    sin = np.concatenate([np.sin(th), np.sin(th)])
    out = oracle.rope_half_split(q, cos, sin)
    z = (q[: D // 2] + 1j * q[D // 2:]) * np.exp(1j * th)
    np.testing.assert_allclose(out, np.concatenate([z.real, z.imag]), rtol=0, atol=1e-14)
    assert np.linalg.norm(out) == pytest.approx(np.linalg.norm(q), rel=1e-14)
    back = oracle.rope_half_split(out, cos, -sin)      # rotate back by -theta
    np.testing.assert_allclose(back, q, rtol=0, atol=1e-14)


def test_masked_softmax_matches_scipy():
    rng = np.random.default_rng(5)
    lg = rng.normal(size=12) * 4
    pm = rng.random(12) < 0.6
    pm[3] = True
    out = oracle.masked_softmax(lg, pm)
    ref = np.zeros(12)
    ref[pm] = scipy.special.softmax(lg[pm])
    np.testing.assert_allclose(out, ref, rtol=1e-14, atol=1e-16)
    assert np.all(out[~pm] == 0.0)
    # shift invariance, large logits stay finite (stabilised)
    np.testing.assert_allclose(oracle.masked_softmax(lg + 900.0, pm), ref, rtol=1e-12, atol=1e-15)
    # empty row: exact zeros; single permitted slot: exactly one
    assert np.all(oracle.masked_softmax(lg, np.zeros(12, bool)) == 0.0)
    one = np.zeros(12, bool)
    one[7] = True
    s = oracle.masked_softmax(lg, one)
    assert s[7] == 1.0 and np.all(np.delete(s, 7) == 0.0)


# --------------------------------------------------------------- eligibility brute force

def _tiny_structure(rng, B=2, A=9, K=6, T=4):
    kid = rng.integers(-8, A + 7, size=(B, A, K))
    kid[0, 0, :4] = [-1, -7, A, A + 5]
    masks = {"valid": rng.random((B, A)) < 0.8, "token_valid": rng.random((B, T)) < 0.8,
             "window_mask": rng.random((B, A, K)) < 0.8}
    structure = {"key_index": kid, "atom_to_token": rng.integers(-2, T + 2, size=(B, A))}
    act = {"atom": np.zeros((B, A, 2)), "condition": np.zeros((B, A, 1)),
           "pair": np.zeros((B, A, K, 1))}
    prm = {"w_q": np.zeros((2, 2)), "w_pair": np.zeros((1, 1)), "w_ff_gate": np.zeros((2, 1)),
           "w_pool": np.zeros((2, 2))}
    return act, prm, masks, structure


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_usable_and_permitted_brute_force(seed):
    rng = np.random.default_rng(seed)
    act, prm, masks, st = _tiny_structure(rng)
    B, A = masks["valid"].shape
    T = masks["token_valid"].shape[1]
    K = st["key_index"].shape[2]
    use = oracle.usable(act, prm, masks, st)
    for b in range(B):
        for a in range(A):
            t = st["atom_to_token"][b, a]
            exp = bool(masks["valid"][b, a]) and 0 <= t < T and bool(masks["token_valid"][b, t])
            assert use[b, a] == exp
    for radius in (-1, 0, 1, 2, 3, 100):
        pm = oracle.permitted(act, prm, masks, st, radius=radius)
        for b in range(B):
            for a in range(A):
                for k in range(K):
                    j = st["key_index"][b, a, k]
                    exp = 0 <= j < A and use[b, a] and use[b, j] and masks["window_mask"][b, a, k]
                    if radius >= 0:
                        exp = exp and abs(j - a) <= radius
                    assert pm[b, a, k] == exp, (radius, b, a, k)


# --------------------------------------------------------------- closed forms, C = 2

def _af3_base():
    return load_golden("af3_encoder_worked_example.json")[1]


def _attention_closed_form(case, q0, K0, K1, V0, V1, gate0, vgate0):
    """Query 0 of the two-atom example: both slots, one head, D = 2."""
    lg0, lg1 = q0 @ K0 / math.sqrt(2), q0 @ K1 / math.sqrt(2)
    p = sig(lg0 - lg1)
    o = p * V0 + (1 - p) * V1
    return p, o


def test_af3_bq_and_projection_orientation():
    """Q = A_0(x) @ w_q + b_q (only Q has a bias), K = A_1(x) @ w_k; weights are [in,out]."""
    case = _af3_base()
    prm = case["parameters"]
    prm["w_q"] = np.array([[2.0, 0.5], [0.0, 1.0]])
    prm["b_q"] = np.array([0.3, -0.1])
    prm["w_k"] = np.array([[1.0, 0.0], [0.5, 2.0]])
    out = run(oracle, case)
    eps = case["eps"]
    f = [ln2(case["activations"]["atom"][0, a], eps) * 0.5 for a in range(2)]   # sigmoid(0)=1/2
    q0 = f[0] @ prm["w_q"] + prm["b_q"]
    K0, K1 = f[0] @ prm["w_k"], f[1] @ prm["w_k"]
    p = sig((q0 @ K0 - q0 @ K1) / math.sqrt(2))
    np.testing.assert_allclose(out["attention"][0, 0, 0], [p, 1 - p], rtol=0, atol=1e-14)
    o = p * f[0] + (1 - p) * f[1]                       # V = A_1(x) @ I
    np.testing.assert_allclose(out["hidden"][0, 0], case["activations"]["atom"][0, 0] + o / 4,
                               rtol=0, atol=1e-14)


def test_af3_stage_indices_and_shift():
    """Stage 0 normalises queries, stage 1 keys/values, stage 2 the transition; shifts
    come from LN(condition) * cond_scale[j] @ w_shift[j]."""
    case = _af3_base()
    act, prm, eps = case["activations"], case["parameters"], case["eps"]
    act["condition"] = np.array([[[0.7, -0.4], [1.2, 2.0]]])          # S = 2
    prm["cond_scale"] = np.array([[1.0, 1.0], [0.5, 2.0], [1.5, -1.0]])
    prm["w_scale"] = np.zeros((3, 2, 2))
    prm["b_scale"] = np.array([[0.4, 0.4], [-0.7, -0.7], [1.1, 1.1]])
    prm["w_shift"] = np.zeros((3, 2, 2))
    prm["w_shift"][1] = [[0.2, -0.1], [0.05, 0.3]]
    prm["w_residual_gate"] = np.zeros((2, 2, 2))
    out = run(oracle, case)
    c = [ln2(act["condition"][0, a], eps) for a in range(2)]
    x = act["atom"][0]
    A0 = [ln2(x[a], eps) * sig(0.4) for a in range(2)]
    A1 = [ln2(x[a], eps) * sig(-0.7) + (c[a] * prm["cond_scale"][1]) @ prm["w_shift"][1]
          for a in range(2)]
    q0 = A0[0]
    p = sig((q0 @ A1[0] - q0 @ A1[1]) / math.sqrt(2))
    np.testing.assert_allclose(out["attention"][0, 0, 0], [p, 1 - p], rtol=0, atol=1e-14)
    o0 = p * A1[0] + (1 - p) * A1[1]
    np.testing.assert_allclose(out["hidden"][0, 0], x[0] + o0 / 4, rtol=0, atol=1e-14)
    np.testing.assert_allclose(out["hidden"][0, 1], x[1] + A1[1] / 4, rtol=0, atol=1e-14)


def test_af3_residual_gate_uses_raw_condition():
    case = _af3_base()
    act, prm = case["activations"], case["parameters"]
    act["condition"] = np.array([[[2.0], [-1.0]]])
    prm["w_residual_gate"] = np.array([[[0.5, -0.25]], [[0.0, 0.0]]])
    prm["b_residual_gate"] = np.array([[0.1, 0.2], [0.0, 0.0]])
    out = run(oracle, case)
    p = sig(0.25 / math.sqrt(2.0))
    o0 = np.array([-0.25, 0.25]) * (2 * p - 1)
    g0 = np.array([sig(2.0 * 0.5 + 0.1), sig(-2.0 * 0.25 + 0.2)])
    np.testing.assert_allclose(out["hidden"][0, 0], act["atom"][0, 0] + g0 * o0 / 2,
                               rtol=0, atol=1e-14)
    g1 = np.array([sig(-0.5 + 0.1), sig(0.25 + 0.2)])
    np.testing.assert_allclose(out["hidden"][0, 1],
                               act["atom"][0, 1] + g1 * np.array([0.25, -0.25]) / 2,
                               rtol=0, atol=1e-14)


def test_af3_pair_bias_per_head():
    """Logit bias (LN(pair) * pair_scale) @ w_pair, one value per head, added after
    the 1/sqrt(D) scaling."""
    case = _af3_base()
    act, prm, eps = case["activations"], case["parameters"], case["eps"]
    act["pair"] = np.array([[[[1.0, 2.0], [0.5, -1.5]], [[3.0, 0.0], [-2.0, 1.0]]]])   # P = 2
    prm["pair_scale"] = np.array([1.5, 0.5])
    prm["w_pair"] = np.array([[1.0, -2.0], [0.5, 3.0]])                 # H = 2, D = 1
    out = run(oracle, case)
    q = np.array([-0.25, 0.25])                                        # heads of query 0
    Kk = [np.array([-0.25, 0.25]), np.array([0.25, -0.25])]
    for h in range(2):
        beta = [(ln2(act["pair"][0, 0, k], eps) * prm["pair_scale"]) @ prm["w_pair"][:, h]
                for k in range(2)]
        lg = [q[h] * Kk[k][h] / 1.0 + beta[k] for k in range(2)]
        p = sig(lg[0] - lg[1])
        np.testing.assert_allclose(out["attention"][0, h, 0], [p, 1 - p], rtol=0, atol=1e-14)
    assert np.all(out["attention"][0, :, 1] == [[0.0, 1.0], [0.0, 1.0]])


def test_af3_value_gate_and_transition_on_new_state():
    case = _af3_base()
    act, prm, eps = case["activations"], case["parameters"], case["eps"]
    prm["w_value_gate"] = np.array([[0.5, -1.0], [2.0, 0.25]])
    prm["b_scale"] = np.array([[0.0, 0.0], [0.0, 0.0], [0.2, -0.3]])
    prm["b_residual_gate"] = np.array([[0.0, 0.0], [0.4, -0.6]])
    prm["w_ff_gate"] = np.array([[0.3], [-0.2]])
    prm["w_ff_up"] = np.array([[0.5], [0.1]])
    prm["w_ff_out"] = np.array([[1.5, -0.5]])
    out = run(oracle, case)
    x = act["atom"][0]
    f = [ln2(x[a], eps) * 0.5 for a in range(2)]
    p = sig(0.25 / math.sqrt(2.0))
    o = [p * f[0] + (1 - p) * f[1], f[1]]
    for a in range(2):
        G = f[a] @ prm["w_value_gate"]
        xn = x[a] + 0.5 * (o[a] * np.array([sig(G[0]), sig(G[1])]))
        z = ln2(xn, eps) * np.array([sig(0.2), sig(-0.3)])
        ga, gb = z @ prm["w_ff_gate"][:, 0], z @ prm["w_ff_up"][:, 0]
        ff = ga * sig(ga) * gb * prm["w_ff_out"][0]
        hid = xn + np.array([sig(0.4), sig(-0.6)]) * ff
        np.testing.assert_allclose(out["hidden"][0, a], hid, rtol=0, atol=1e-14)


@pytest.mark.parametrize("style", ["af3", "esmfold2"])
def test_decoder_start_and_readout(style):
    """Decoder: x = skip + gather(token @ w_token); readout (LN(hidden) * scale [+ bias])
    @ w_readout, masked to zero for unusable atoms."""
    case = _af3_base()
    act, prm, msk, st, eps = (case["activations"], case["parameters"], case["masks"],
                              case["structure"], case["eps"])
    case["stage"], case["style"] = "decoder", style
    act["token"] = np.array([[[0.5, -1.0, 2.0], [1.0, 1.0, 1.0]]])
    msk["token_valid"] = np.array([[True, True]])
    st["atom_to_token"] = np.array([[1, 0]])
    msk["window_mask"][:] = False                     # no attention update
    prm["w_token"] = np.array([[1.0, 0.5], [-1.0, 2.0], [0.25, 0.0]])
    prm["readout_scale"] = np.array([1.5, -0.5])
    prm["readout_bias"] = np.array([0.2, 0.1])
    prm["w_readout"] = np.array([[1.0, 0.0, 2.0], [0.5, -1.0, 0.0]])
    del prm["w_pool"]
    if style == "esmfold2":
        for k in ("cond_scale", "w_scale", "b_scale", "w_shift", "w_residual_gate",
                  "b_residual_gate", "b_q", "pair_scale", "w_pair"):
            prm.pop(k)
        del act["pair"]
        prm["w_mod"] = np.zeros((1, 6, 2))
        act["rope_cos"] = np.ones((1, 2, 2))
        act["rope_sin"] = np.zeros((1, 2, 2))
    msk2 = clone(case)
    msk2["masks"]["valid"] = np.array([[True, False]])
    for c, n_ok in ((case, 2), (msk2, 1)):
        out = run(oracle, c)
        for a in range(2):
            if a >= n_ok:
                assert np.all(out["hidden"][0, a] == 0.0)
                assert np.all(out["position_update"][0, a] == 0.0)
                continue
            x = act["atom"][0, a] + act["token"][0, st["atom_to_token"][0, a]] @ prm["w_token"]
            np.testing.assert_allclose(out["hidden"][0, a], x, rtol=0, atol=1e-14)
            y = ln2(x, eps) * prm["readout_scale"]
            if style == "esmfold2":
                y = y + prm["readout_bias"]
            np.testing.assert_allclose(out["position_update"][0, a], y @ prm["w_readout"],
                                       rtol=0, atol=1e-14)
        assert np.all(out["attention"] == 0.0)


def test_esmfold2_six_vector_order():
    """SiLU(condition) @ w_mod gives attention shift, scale, gate; transition shift,
    scale, gate in that order; gates are raw."""
    c0 = 0.8
    s = c0 * sig(c0)
    m = np.array([[0.1, -0.2], [0.3, 0.05], [0.7, -1.1], [-0.15, 0.25], [0.4, -0.35], [1.3, 0.6]])
    case = {
        "activations": {"atom": np.array([[[1.0, -2.0]]]), "condition": np.array([[[c0]]]),
                        "rope_cos": np.ones((1, 1, 2)), "rope_sin": np.zeros((1, 1, 2))},
        "parameters": {"w_mod": (m / s)[None], "w_q": np.eye(2), "w_k": np.eye(2),
                       "w_v": np.array([[1.0, 0.5], [-0.5, 2.0]]),
                       "w_value_gate": np.array([[0.3, 0.0], [0.1, -0.4]]),
                       "w_attention_out": np.array([[1.0, 0.2], [0.0, 1.0]]),
                       "w_ff_gate": np.array([[0.3], [-0.2]]), "w_ff_up": np.array([[0.5], [0.1]]),
                       "w_ff_out": np.array([[1.5, -0.5]]), "w_pool": np.eye(2)},
        "masks": {"valid": np.array([[True]]), "token_valid": np.array([[True]]),
                  "window_mask": np.array([[[True]]])},
        "structure": {"key_index": np.array([[[0]]]), "atom_to_token": np.array([[0]])},
        "eps": 0.5, "style": "esmfold2", "stage": "encoder", "radius": -1,
    }
    out = run(oracle, case)
    eps, prm = 0.5, case["parameters"]
    x = case["activations"]["atom"][0, 0]
    a_shift, a_scale, a_gate, t_shift, t_scale, t_gate = m
    u = rms2(x, eps) * (1 + a_scale) + a_shift
    V, G = u @ prm["w_v"], u @ prm["w_value_gate"]
    xn = x + a_gate * ((V * np.array([sig(G[0]), sig(G[1])])) @ prm["w_attention_out"])
    z = rms2(xn, eps) * (1 + t_scale) + t_shift
    ga, gb = z @ prm["w_ff_gate"][:, 0], z @ prm["w_ff_up"][:, 0]
    hid = xn + t_gate * (ga * sig(ga) * gb * prm["w_ff_out"][0])
    assert out["attention"][0, 0, 0, 0] == 1.0
    np.testing.assert_allclose(out["hidden"][0, 0], hid, rtol=0, atol=1e-13)
    np.testing.assert_allclose(out["token_output"][0, 0], np.maximum(hid, 0), rtol=0, atol=1e-13)


# --------------------------------------------------------------- dense-attention reductions

def _dense_case(style, rng, A=6, C=8, S=5, H=2, D=4, P=3, M=6, U=5):
    HD = H * D
    act = {"atom": rng.normal(size=(1, A, C)), "condition": rng.normal(size=(1, A, S))}
    prm = {"w_q": rng.normal(size=(C, HD)) / 3, "w_k": rng.normal(size=(C, HD)) / 3,
           "w_v": rng.normal(size=(C, HD)), "w_value_gate": rng.normal(size=(C, HD)),
           "w_attention_out": rng.normal(size=(HD, C)) / 3, "w_ff_gate": rng.normal(size=(C, M)),
           "w_ff_up": rng.normal(size=(C, M)), "w_ff_out": rng.normal(size=(M, C)) / 3,
           "w_pool": rng.normal(size=(C, U))}
    if style == "af3":
        act["pair"] = rng.normal(size=(1, A, A, P))
        prm.update(cond_scale=1 + 0.1 * rng.normal(size=(3, S)),
                   w_scale=rng.normal(size=(3, S, C)) / 2, b_scale=0.1 * rng.normal(size=(3, C)),
                   w_shift=rng.normal(size=(3, S, C)) / 2,
                   w_residual_gate=rng.normal(size=(2, S, C)) / 2,
                   b_residual_gate=0.1 * rng.normal(size=(2, C)), b_q=0.1 * rng.normal(size=HD),
                   pair_scale=1 + 0.1 * rng.normal(size=P), w_pair=rng.normal(size=(P, H)))
    else:
        th = rng.uniform(0, 2 * np.pi, size=(1, A, D // 2))
        th = np.concatenate([th, th], axis=-1)
        act["rope_cos"], act["rope_sin"] = np.cos(th), np.sin(th)
        prm["w_mod"] = rng.normal(size=(S, 6, C)) * 0.3
    masks = {"valid": np.ones((1, A), bool), "token_valid": np.ones((1, 2), bool),
             "window_mask": np.ones((1, A, A), bool)}
    st = {"key_index": np.broadcast_to(np.arange(A), (1, A, A)).copy(),
          "atom_to_token": (np.arange(A) * 2 // A)[None].astype(np.int64)}
    return {"activations": act, "parameters": prm, "masks": masks, "structure": st,
            "eps": 1e-5, "style": style, "stage": "encoder", "radius": -1}


@pytest.mark.parametrize("style", ["af3", "esmfold2"])
def test_dense_window_reduces_to_library_attention(style):
    """All slots permitted with key_index = 0..A-1: the block is dense softmax
    attention with an additive bias, computed here with torch float64 library
    routines (layer_norm, rms_norm, softmax, scaled_dot_product_attention)."""
    rng = np.random.default_rng(11 if style == "af3" else 12)
    case = _dense_case(style, rng)
    out = run(oracle, case)
    t = {k: torch.tensor(v) for k, v in {**case["activations"], **case["parameters"]}.items()}
    eps = case["eps"]
    A, C = case["activations"]["atom"].shape[1:]
    S = case["activations"]["condition"].shape[2]
    H, D = 2, 4
    x, c = t["atom"][0], t["condition"][0]
    if style == "af3":
        lc = F.layer_norm(c, (S,), eps=eps)
        lx = F.layer_norm(x, (C,), eps=eps)
        cj = [lc * t["cond_scale"][j] for j in range(3)]
        feat = [lx * torch.sigmoid(cj[j] @ t["w_scale"][j] + t["b_scale"][j]) + cj[j] @ t["w_shift"][j]
                for j in range(2)]
        q = feat[0] @ t["w_q"] + t["b_q"]
        k, v, g = feat[1] @ t["w_k"], feat[1] @ t["w_v"], feat[0] @ t["w_value_gate"]
        pn = F.layer_norm(t["pair"][0], (t["pair"].shape[-1],), eps=eps) * t["pair_scale"]
        bias = (pn @ t["w_pair"]).permute(2, 0, 1)                       # [H, A, A]
        g0 = torch.sigmoid(c @ t["w_residual_gate"][0] + t["b_residual_gate"][0])
    else:
        mod = (F.silu(c) @ t["w_mod"].reshape(S, 6 * C)).reshape(A, 6, C)
        u = F.rms_norm(x, (C,), eps=eps) * (1 + mod[:, 1]) + mod[:, 0]
        qh = F.rms_norm((u @ t["w_q"]).reshape(A, H, D), (D,), eps=eps)
        kh = F.rms_norm((u @ t["w_k"]).reshape(A, H, D), (D,), eps=eps)
        th = torch.atan2(t["rope_sin"][0, :, : D // 2], t["rope_cos"][0, :, : D // 2])[:, None]
        rot = lambda z: torch.view_as_real(torch.complex(z[..., : D // 2], z[..., D // 2:])
                                           * torch.exp(1j * th)).permute(0, 1, 3, 2).reshape(A, H, D)
        q, k = rot(qh).reshape(A, H * D), rot(kh).reshape(A, H * D)
        v, g = u @ t["w_v"], u @ t["w_value_gate"]
        bias = torch.zeros(H, A, A, dtype=torch.float64)
        g0 = mod[:, 2]
    qh, kh, vh = (z.reshape(A, H, D).permute(1, 0, 2) for z in (q, k, v))
    att = torch.softmax(qh @ kh.transpose(1, 2) / math.sqrt(D) + bias, dim=-1)
    np.testing.assert_allclose(out["attention"][0], att.numpy(), rtol=1e-11, atol=1e-13)
    o = F.scaled_dot_product_attention(qh[None], kh[None], vh[None], attn_mask=bias[None])[0]
    o = o.permute(1, 0, 2).reshape(A, H * D) * torch.sigmoid(g)
    xn = x + g0 * (o @ t["w_attention_out"])
    assert np.all(np.isfinite(out["hidden"]))
    # the attention update alone: compare x' through a zero transition
    case2 = clone(case)
    case2["parameters"]["w_ff_out"] = np.zeros_like(case2["parameters"]["w_ff_out"])
    out2 = run(oracle, case2)
    np.testing.assert_allclose(out2["hidden"][0], xn.numpy(), rtol=1e-10, atol=1e-11)
