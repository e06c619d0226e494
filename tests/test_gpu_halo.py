"""Halo sharding on the GPU: a problem split into token-aligned shards (owned atoms plus
the key halo, sparse_windowed_atom_b200/halo.py), each shard's extended problem run
through the CUDA forward, gives the outputs of the whole problem's CUDA forward (every
query's and every token's arithmetic is the same), and agrees with the float64 oracle
within the parity tolerance. One GPU runs the shards one after another; the exchange
itself is covered on gloo ranks in test_halo_cpu.py."""
import numpy as np
import pytest
import torch

import oracle
from sparse_windowed_atom_b200 import atomenc, halo, workloads

pytestmark = pytest.mark.gpu
TOL = {"float32": 2e-4, "bfloat16": 2e-2}


def _to(x, dev, fdt):
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(dev, dtype=fdt) if t.is_floating_point() else t.to(dev)


@pytest.mark.parametrize("style,stage,dtype,kw", [
    ("af3", "encoder", "bfloat16", dict(keys=("blocked", 16, 8))),
    ("esmfold2", "encoder", "bfloat16", dict(keys=("random", 48), radius=24)),
    ("af3", "decoder", "float32", dict(keys=("blocked", 16, 8))),
    ("esmfold2", "decoder", "float32", dict(keys=("random", 48), radius=-1)),
])
def test_shards_on_gpu_equal_the_whole_problem(style, stage, dtype, kw):
    spec = workloads.tiny_spec(style, stage, dtype, B=1, A=900, T=110, K=32, **kw)
    w = workloads.make_inputs(spec, seed=21)
    dev, fdt = "cuda", torch.bfloat16 if dtype == "bfloat16" else torch.float32
    act = {k: _to(v, dev, fdt) for k, v in w["activations"].items()}
    msk = {k: _to(v, dev, fdt) for k, v in w["masks"].items()}
    st = {k: _to(v, dev, fdt) for k, v in w["structure"].items()}
    prm = {k: _to(v, dev, fdt) for k, v in w["parameters"].items()}
    full = atomenc.windowed_atom_attention(act, prm, msk, st, spec.eps, style, stage, spec.radius)
    shards = halo.plan(w["structure"], w["masks"], spec.T, 3, spec.radius)
    parts = []
    for (sh,) in shards:
        key_rows = {k: act[k][0, sh.e0:sh.e1] for k in ("atom", "condition", "rope_cos", "rope_sin") if k in act}
        key_rows["valid"] = msk["valid"][0, sh.e0:sh.e1]
        key_rows["atom_to_token"] = st["atom_to_token"][0, sh.e0:sh.e1]
        query_rows = {"key_index": st["key_index"][0, sh.a0:sh.a1],
                      "window_mask": msk["window_mask"][0, sh.a0:sh.a1]}
        if "pair" in act:
            query_rows["pair"] = act["pair"][0, sh.a0:sh.a1]
        tokens = {"token_valid": msk["token_valid"][0]}
        if "token" in act:
            tokens["token"] = act["token"][0]
        a, m, s = halo.local_problem(key_rows, query_rows, tokens, sh, spec.T)
        out = atomenc.windowed_atom_attention(a, prm, m, s, spec.eps, style, stage, spec.radius)
        parts.append((sh, halo.owned_outputs(out, sh)))
    asm = halo.assemble(parts, spec.B, spec.A, spec.T)
    torch.cuda.synchronize()
    for k in full:
        assert torch.equal(asm[k], full[k]), k
    ref = oracle.windowed_atom_attention(w["activations"], w["parameters"], w["masks"], w["structure"],
                                         eps=spec.eps, style=style, stage=stage, radius=spec.radius)
    for k, r in ref.items():
        g = asm[k].double().cpu().numpy()
        bad = np.abs(g - r) > TOL[dtype] * (1 + np.abs(r))
        assert not bad.any(), (k, int(bad.sum()))
