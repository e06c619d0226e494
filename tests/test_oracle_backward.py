"""Pins of the attention core's float64 forward and gradient in the oracle.

The forward (orc_attention_core) is pinned to torch float64 attention on a dense
window; the gradient (orc_attention_core_backward) to central finite differences of
that forward for every input, with duplicated keys (in one query and across queries),
missing ids, unusable atoms, a radius window and empty rows in the data, so that a
dropped term, a wrong sign or an index slip fails here.
Pages: "Local atom attention, encoder pooling and decoder skip/readout", Required
behavior (slot permission and radius, logits and masked softmax, repeated slots as
separate entries whose gradients accumulate, value gate)."""
import numpy as np
import pytest
import torch

import oracle


def _core(style, seed, B=2, A=7, K=5, H=2, D=3, P=3, dup=True):
    rng = np.random.default_rng(seed)
    c = {n: rng.normal(size=(B, A, H * D)) for n in ("q", "k", "v", "g")}
    kid = rng.integers(-2, A + 2, size=(B, A, K))     # includes missing and out-of-range ids
    if dup:
        kid[:, :, 1] = kid[:, :, 0]                     # the same key twice in one row
        kid[:, 2, 3] = 4                                # key 4 from several queries
        kid[:, 3, 2] = 4
        kid[:, 5, 0] = 4
    c["key_index"] = kid
    c["window_mask"] = rng.random((B, A, K)) < 0.85
    c["usable"] = rng.random((B, A)) < 0.85
    c["usable"][:, 4] = True
    c["window_mask"][:, 6] = False                      # an empty row
    if style == "af3":
        c["pair"] = rng.normal(size=(B, A, K, P))
        c["pair_scale"] = 1 + 0.2 * rng.normal(size=P)
        c["w_pair"] = rng.normal(size=(P, H))
    return c


def _loss(core, H, style, radius, R_out, R_att):
    att, out = oracle.attention_core(core, H, style=style, radius=radius)
    return float((out * R_out).sum() + (att * R_att).sum())


@pytest.mark.parametrize("style", ["af3", "esmfold2"])
@pytest.mark.parametrize("radius", [-1, 2])
def test_gradient_matches_central_differences(style, radius):
    H = 2
    core = _core(style, seed=3 + radius)
    rng = np.random.default_rng(11)
    att, out = oracle.attention_core(core, H, style=style, radius=radius)
    R_out = rng.normal(size=out.shape)
    R_att = rng.normal(size=att.shape)
    grads = oracle.attention_core_backward(core, H, R_out, R_att, style=style, radius=radius)
    names = [("q", "d_q"), ("k", "d_k"), ("v", "d_v"), ("g", "d_g")]
    if style == "af3":
        names += [("pair", "d_pair"), ("pair_scale", "d_pair_scale"), ("w_pair", "d_w_pair")]
    h = 1e-6
    for x, dx in names:
        base = core[x]
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            plus = {**core, x: base.copy()}
            minus = {**core, x: base.copy()}
            plus[x][idx] += h
            minus[x][idx] -= h
            fd[idx] = (_loss(plus, H, style, radius, R_out, R_att) -
                       _loss(minus, H, style, radius, R_out, R_att)) / (2 * h)
        np.testing.assert_allclose(grads[dx], fd, rtol=1e-5, atol=1e-7, err_msg=f"{style} {dx}")


def test_repeated_keys_accumulate_and_empty_rows_vanish():
    """A key named by two slots of one query receives both slots' value gradients;
    a row with no permitted slot gives no gradient to its query."""
    H = 1
    core = _core("esmfold2", seed=5, B=1, H=1, D=2)
    kid = core["key_index"]
    kid[0, 0] = [3, 3, -1, -1, -1]
    core["window_mask"][0, 0] = True
    core["usable"][0, [0, 3]] = True
    d_out = np.zeros((1, 7, 2))
    d_out[0, 0] = [1.0, 0.0]
    g = oracle.attention_core_backward(core, H, d_out, style="esmfold2")
    att, out = oracle.attention_core(core, H, style="esmfold2")
    s = 1 / (1 + np.exp(-core["g"][0, 0, 0]))
    # both slots select key 3 with equal weight 1/2: d_v[3] = (w0 + w1) * d_o = 1 * s
    assert att[0, 0, 0, 0] == pytest.approx(0.5) and att[0, 0, 0, 1] == pytest.approx(0.5)
    assert g["d_v"][0, 3, 0] == pytest.approx(s, rel=1e-12)
    assert np.all(g["d_q"][0, 6] == 0.0) and np.all(att[0, :, 6] == 0.0)


@pytest.mark.parametrize("style", ["af3", "esmfold2"])
def test_dense_window_forward_equals_torch_attention(style):
    """Every slot permitted with key_index = 0..A-1: the core is dense softmax attention
    (plus the LayerNorm pair bias in AF3 style), gated by sigmoid(g)."""
    B, A, H, D, P = 2, 6, 2, 4, 5
    rng = np.random.default_rng(21)
    core = {n: rng.normal(size=(B, A, H * D)) for n in ("q", "k", "v", "g")}
    core["key_index"] = np.broadcast_to(np.arange(A), (B, A, A)).copy()
    core["window_mask"] = np.ones((B, A, A), bool)
    core["usable"] = np.ones((B, A), bool)
    eps = 1e-5
    t = lambda x: torch.tensor(x, dtype=torch.float64)
    q = t(core["q"]).view(B, A, H, D).transpose(1, 2)
    k = t(core["k"]).view(B, A, H, D).transpose(1, 2)
    v = t(core["v"]).view(B, A, H, D).transpose(1, 2)
    logits = q @ k.transpose(-1, -2) / np.sqrt(D)
    if style == "af3":
        core["pair"] = rng.normal(size=(B, A, A, P))
        core["pair_scale"] = 1 + 0.2 * rng.normal(size=P)
        core["w_pair"] = rng.normal(size=(P, H))
        ln = torch.nn.functional.layer_norm(t(core["pair"]), (P,), eps=eps)
        beta = (ln * t(core["pair_scale"])) @ t(core["w_pair"])      # [B, A, K, H]
        logits = logits + beta.permute(0, 3, 1, 2)
    w = torch.softmax(logits, dim=-1)
    o = (w @ v).transpose(1, 2).reshape(B, A, H * D) * torch.sigmoid(t(core["g"]))
    att, out = oracle.attention_core(core, H, eps=eps, style=style)
    np.testing.assert_allclose(att, w.numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(out, o.numpy(), rtol=1e-12, atol=1e-14)
