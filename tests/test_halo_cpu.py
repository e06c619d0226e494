"""Halo sharding of one problem across ranks (sparse_windowed_atom_b200/halo.py), on CPU.

The decomposition is checked against the float64 oracle: every shard's extended
problem (owned atoms plus the key halo) run through the oracle, with the owned outputs
assembled, equals the oracle on the whole problem exactly, since every query sees the
same key rows and every token the same atoms in the same order (page "Local atom
attention, encoder pooling and decoder skip/readout", Required behavior, bullets 4-6,
15, 16, 19). The row exchange runs on two gloo ranks."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from sparse_windowed_atom_b200 import halo, workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = [
    ("af3", "encoder", dict(keys=("blocked", 16, 8))),
    ("af3", "decoder", dict(keys=("blocked", 16, 8))),
    ("esmfold2", "encoder", dict(keys=("random", 40), radius=20, P=0)),
    ("esmfold2", "decoder", dict(keys=("random", 40), radius=-1, P=0)),
]


def _spec(style, stage, kw, B=1):
    base = dict(B=B, A=220, T=30, K=20, C=16, S=8, H=2, D=8, M=16, U=12, V=10)
    base.update(kw)
    if style == "af3":
        base.setdefault("P", 4)
    return workloads.tiny_spec(style, stage, **base)


def _t(x):
    return None if x is None else torch.from_numpy(np.ascontiguousarray(x))


def _oracle(act, msk, st, spec, style, stage):
    a = {k: v.numpy() for k, v in act.items()}
    m = {k: v.numpy() for k, v in msk.items()}
    s = {k: v.numpy() for k, v in st.items()}
    out = oracle.windowed_atom_attention(a, _params(spec), m, s, eps=spec.eps, style=style,
                                         stage=stage, radius=spec.radius)
    return {k: torch.from_numpy(v) for k, v in out.items()}


_PARAMS = {}


def _params(spec):
    return _PARAMS[spec.name]


def _shard_inputs(w, sh: halo.Shard):
    act, msk, st = w["activations"], w["masks"], w["structure"]
    b = sh.b
    key_rows = {"atom": _t(act["atom"][b, sh.e0:sh.e1]), "condition": _t(act["condition"][b, sh.e0:sh.e1]),
                "valid": _t(msk["valid"][b, sh.e0:sh.e1]),
                "atom_to_token": _t(st["atom_to_token"][b, sh.e0:sh.e1])}
    for k in ("rope_cos", "rope_sin"):
        if k in act:
            key_rows[k] = _t(act[k][b, sh.e0:sh.e1])
    query_rows = {"key_index": _t(st["key_index"][b, sh.a0:sh.a1]),
                  "window_mask": _t(msk["window_mask"][b, sh.a0:sh.a1])}
    if "pair" in act:
        query_rows["pair"] = _t(act["pair"][b, sh.a0:sh.a1])
    tokens = {"token_valid": _t(msk["token_valid"][b])}
    if "token" in act:
        tokens["token"] = _t(act["token"][b])
    return key_rows, query_rows, tokens


def test_partition_is_token_aligned_and_covers_everything():
    rng = np.random.default_rng(3)
    for trial in range(40):
        T = int(rng.integers(1, 40))
        counts = rng.integers(0, 9, size=T)
        att = np.repeat(np.arange(T), counts)
        att = np.concatenate([att, np.full(int(rng.integers(0, 5)), T)])   # unmapped tail
        if att.size == 0:
            continue
        for parts in (1, 2, 3, 5):
            cuts = halo.partition(att, T, parts)
            assert cuts[0][0] == 0 and cuts[-1][1] == att.size
            assert cuts[0][2] == 0 and cuts[-1][3] == T
            for (a0, a1, t0, t1), (b0, b1, u0, u1) in zip(cuts, cuts[1:]):
                assert a1 == b0 and t1 == u0
            for (a0, a1, t0, t1) in cuts:
                inr = att[a0:a1][(att[a0:a1] >= 0) & (att[a0:a1] < T)]
                assert np.all((inr >= t0) & (inr < t1))            # a token is never split
    with pytest.raises(ValueError):
        halo.partition(np.array([0, 1, 0]), 2, 2)


def test_halo_extent_is_the_span_of_permitted_keys():
    rng = np.random.default_rng(5)
    A, K = 60, 7
    kid = rng.integers(-5, A + 5, size=(A, K))
    win = rng.random((A, K)) < 0.7
    for radius in (-1, 0, 3, 10):
        for a0, a1 in ((0, 20), (20, 41), (41, 60)):
            e0, e1 = halo.halo_extent(kid[a0:a1], win[a0:a1], a0, a1, A, radius)
            need = [int(j) for a in range(a0, a1) for j, w in zip(kid[a], win[a])
                    if w and 0 <= j < A and (radius < 0 or abs(j - a) <= radius)]
            assert e0 == min([a0] + need) and e1 == max([a1] + [j + 1 for j in need])


@pytest.mark.parametrize("style,stage,kw", CASES)
@pytest.mark.parametrize("parts", [2, 3])
def test_shards_reproduce_the_whole_problem(style, stage, kw, parts):
    spec = _spec(style, stage, kw, B=2)
    w = workloads.make_inputs(spec, seed=11)
    _PARAMS[spec.name] = w["parameters"]
    full = _oracle({k: _t(v) for k, v in w["activations"].items()},
                   {k: _t(v) for k, v in w["masks"].items()},
                   {k: _t(v) for k, v in w["structure"].items()}, spec, style, stage)
    shards = halo.plan(w["structure"], w["masks"], spec.T, spec.B * parts, spec.radius)
    assert len(shards) == spec.B * parts
    got = []
    for (sh,) in shards:
        assert sh.e0 <= sh.a0 <= sh.a1 <= sh.e1
        key_rows, query_rows, tokens = _shard_inputs(w, sh)
        act, msk, st = halo.local_problem(key_rows, query_rows, tokens, sh, spec.T)
        got.append((sh, halo.owned_outputs(_oracle(act, msk, st, spec, style, stage), sh)))
    asm = halo.assemble(got, spec.B, spec.A, spec.T)
    for k, ref in full.items():
        np.testing.assert_array_equal(asm[k].numpy(), ref.numpy(), err_msg=k)


def test_whole_batch_elements_per_rank_when_ranks_are_few():
    spec = _spec("af3", "encoder", dict(keys=("blocked", 16, 8)), B=3)
    w = workloads.make_inputs(spec, seed=2)
    per = halo.plan(w["structure"], w["masks"], spec.T, 2, -1)
    owned = sorted(sh.b for shs in per for sh in shs)
    assert owned == [0, 1, 2]
    assert all(sh.a0 == 0 and sh.a1 == spec.A and sh.e0 == 0 and sh.e1 == spec.A
               for shs in per for sh in shs)


# ------------------------------------------------------------------ two gloo ranks

def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, style, stage, kw, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    from sparse_windowed_atom_b200 import halo as hl, workloads as wl
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    spec = _spec(style, stage, kw, B=1)
    w = wl.make_inputs(spec, seed=13)
    _PARAMS[spec.name] = w["parameters"]
    shards = [s[0] for s in hl.plan(w["structure"], w["masks"], spec.T, world, spec.radius)]
    me = shards[rank]
    # this rank holds only its own atoms' rows
    own = hl.Shard(me.b, me.a0, me.a1, me.t0, me.t1, me.a0, me.a1)
    owned_keys, query_rows, tokens = _shard_inputs(w, own)
    key_rows = hl.exchange(owned_keys, shards, rank)
    act, msk, st = hl.local_problem(key_rows, query_rows, tokens, me, spec.T)
    out = hl.owned_outputs(_oracle(act, msk, st, spec, style, stage), me)
    q.put((rank, me, {k: v.numpy() for k, v in out.items()}))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("style,stage,kw", [CASES[0], CASES[2], CASES[3]])
def test_exchange_over_two_gloo_ranks(style, stage, kw):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, style, stage, kw, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    spec = _spec(style, stage, kw, B=1)
    w = workloads.make_inputs(spec, seed=13)
    _PARAMS[spec.name] = w["parameters"]
    full = _oracle({k: _t(v) for k, v in w["activations"].items()},
                   {k: _t(v) for k, v in w["masks"].items()},
                   {k: _t(v) for k, v in w["structure"].items()}, spec, style, stage)
    parts = [(sh, {k: torch.from_numpy(v) for k, v in o.items()}) for _, sh, o in sorted(res, key=lambda r: r[0])]
    assert any(sh.e0 < sh.a0 or sh.e1 > sh.a1 for sh, _ in parts)   # a real halo was exchanged
    asm = halo.assemble(parts, spec.B, spec.A, spec.T)
    for k, ref in full.items():
        np.testing.assert_array_equal(asm[k].numpy(), ref.numpy(), err_msg=k)
