"""Halo sharding of one problem's atoms across ranks (one process per GPU).

Page "Local atom attention, encoder pooling and decoder skip/readout", Required
behavior: every query's output depends on its own rows and on the K/V rows of the keys
its slots name (bullets 4-6, 8, 13-16), and a token's pooled output on the token's own
atoms (bullet 19). So a problem too large for one GPU splits into contiguous atom
ranges cut at token boundaries; each rank owns the queries and tokens of its range and
needs, besides its own rows, the key-side rows of the atoms its slots name outside the
range (the halo). The key-side rows of an atom (atom or skip, condition, rope rows,
valid flag, token id) are exchanged between ranks once, before the forward pass; every
rank then runs the single-GPU forward on its extended range (owned atoms plus halo) and
keeps the outputs of what it owns. Halo atoms only serve as keys: their own query rows
are left empty and their outputs are dropped. Token-level tensors (token_valid, the
decoder's token features) are small and replicated on every rank.

This module holds the host logic: the token-aligned partition, the halo extents, the
row exchange over torch.distributed (NCCL between GPUs, gloo on CPU), the extended
local problem and the assembly of owned outputs. All arithmetic of the block stays in
the forward pass each rank runs.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

# per-atom rows a key needs (exchanged for the halo); per-query rows (owned only)
KEY_ROWS = ("atom", "condition", "rope_cos", "rope_sin", "valid", "atom_to_token")
QUERY_ROWS = ("key_index", "window_mask", "pair")


@dataclass(frozen=True)
class Shard:
    """One rank's part of batch element b: owned atoms [a0, a1), owned tokens [t0, t1)
    and the extended atom range [e0, e1) (owned atoms plus the key halo)."""
    b: int
    a0: int
    a1: int
    t0: int
    t1: int
    e0: int = -1
    e1: int = -1


def _np(x):
    return x.detach().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x)


def partition(atom_to_token, T: int, parts: int) -> list[tuple[int, int, int, int]]:
    """Split the atoms of one batch element into `parts` contiguous ranges cut at token
    boundaries, as evenly as the boundaries allow. Needs the atoms grouped by token
    (atom_to_token non-decreasing; ids outside [0, T) count as one more token after the
    last). Returns (a0, a1, t0, t1) per part: owned atoms and owned tokens; every token
    is owned by exactly one part (a token without atoms by the part whose range of ids
    holds it)."""
    att = _np(atom_to_token).astype(np.int64).reshape(-1)
    A = att.shape[0]
    key = np.where((att >= 0) & (att < T), att, T)
    if np.any(np.diff(key) < 0):
        raise ValueError("a token-aligned partition needs the atoms grouped by token "
                         "(atom_to_token non-decreasing)")
    cuts = [0]
    for p in range(1, parts):
        a = max(int(round(p * A / parts)), cuts[-1])
        # move the cut to the next token boundary
        while 0 < a < A and key[a] == key[a - 1]:
            a += 1
        cuts.append(min(a, A))
    cuts.append(A)
    out = []
    for p in range(parts):
        a0, a1 = cuts[p], cuts[p + 1]
        t0 = 0 if p == 0 else (int(min(key[a0], T)) if a0 < A else T)
        t1 = T if p == parts - 1 else (int(min(key[a1], T)) if a1 < A else T)
        out.append((a0, a1, t0, max(t0, t1)))
    return out


def halo_extent(key_index, window_mask, a0: int, a1: int, A: int, radius: int = -1) -> tuple[int, int]:
    """Extended range [e0, e1) of the owned queries [a0, a1): the owned atoms plus every
    key that one of their slots could permit (id in [0, A), window bit set, within the
    radius when there is one); key_index / window_mask are the owned rows [a1-a0, K]."""
    kid = _np(key_index).astype(np.int64)
    win = _np(window_mask).astype(bool)
    a = np.arange(a0, a1, dtype=np.int64)[:, None]
    ok = win & (kid >= 0) & (kid < A)
    if radius >= 0:
        ok &= np.abs(kid - a) <= radius
    e0, e1 = a0, a1
    if ok.any():
        e0 = min(e0, int(kid[ok].min()))
        e1 = max(e1, int(kid[ok].max()) + 1)
    return e0, e1


def plan(structure: dict, masks: dict, T: int, world: int, radius: int = -1) -> list[Shard]:
    """Shards of a batch of B problems over `world` ranks: by batch first (world <= B:
    rank r owns whole batch elements, no halo), then by token-aligned atom ranges
    (world = B * parts: each batch element split over `parts` consecutive ranks).
    Returns one list of shards per rank."""
    att = _np(structure["atom_to_token"])
    kid = _np(structure["key_index"])
    win = _np(masks["window_mask"])
    B, A = att.shape
    if world <= B:
        per = [[] for _ in range(world)]
        for b in range(B):
            r = b * world // B
            per[r].append(Shard(b, 0, A, 0, T, 0, A))
        return per
    if world % B:
        raise ValueError(f"{world} ranks do not split {B} batch elements evenly")
    parts = world // B
    per = []
    for b in range(B):
        for (a0, a1, t0, t1) in partition(att[b], T, parts):
            e0, e1 = halo_extent(kid[b, a0:a1], win[b, a0:a1], a0, a1, A, radius)
            per.append([Shard(b, a0, a1, t0, t1, e0, e1)])
    return per


def _tokens(att_ext: np.ndarray, T: int, t0: int, t1: int):
    """Local token ids of an extended range: owned tokens first (t - t0), then every
    other in-range token its halo atoms name, in increasing order; ids outside [0, T)
    stay outside (-> the local count). Returns (local ids, global ids of the local
    tokens)."""
    att_ext = att_ext.astype(np.int64)
    inr = (att_ext >= 0) & (att_ext < T)
    extra = np.unique(att_ext[inr & ((att_ext < t0) | (att_ext >= t1))])
    glob = np.concatenate([np.arange(t0, t1, dtype=np.int64), extra])
    Tl = glob.shape[0]
    loc = np.full(att_ext.shape, Tl, dtype=np.int64)
    own = inr & (att_ext >= t0) & (att_ext < t1)
    loc[own] = att_ext[own] - t0
    if extra.size:
        pos = np.searchsorted(extra, att_ext[inr & ~own])
        loc[inr & ~own] = (t1 - t0) + pos
    return loc, glob


def local_problem(key_rows: dict, query_rows: dict, tokens: dict, shard: Shard, T: int):
    """The extended problem of one shard, as B = 1 tensors: key_rows are the key-side
    per-atom rows of [e0, e1) ([e1-e0, ...], atom_to_token with global token ids),
    query_rows the owned rows [a1-a0, ...] (key_index with global atom ids), tokens the
    replicated token-level tensors of this batch element (token_valid [T], token
    [T, V] for the decoder). Halo query rows are empty (all slots masked). Returns
    (activations, masks, structure) of the local problem."""
    e0, e1, a0, a1 = shard.e0, shard.e1, shard.a0, shard.a1
    Ae, Ao = e1 - e0, a1 - a0
    ref = key_rows["atom"]
    dev = ref.device

    att_ext = _np(key_rows["atom_to_token"])
    loc, glob = _tokens(att_ext, T, shard.t0, shard.t1)
    glob_t = torch.as_tensor(glob, device=dev)

    act = {k: key_rows[k].unsqueeze(0) for k in ("atom", "condition", "rope_cos", "rope_sin")
           if key_rows.get(k) is not None}
    kid = query_rows["key_index"].to(torch.int64)
    K = kid.shape[-1]
    inside = (kid >= e0) & (kid < e1)
    kid_l = torch.full((Ae, K), -1, dtype=torch.int64, device=dev)
    kid_l[a0 - e0:a1 - e0] = torch.where(inside, kid - e0, torch.full_like(kid, -1))
    win_l = torch.zeros((Ae, K), dtype=torch.bool, device=dev)
    win_l[a0 - e0:a1 - e0] = query_rows["window_mask"].to(torch.bool)
    if query_rows.get("pair") is not None:
        pr = query_rows["pair"]
        pair_l = torch.zeros((Ae,) + tuple(pr.shape[1:]), dtype=pr.dtype, device=dev)
        pair_l[a0 - e0:a1 - e0] = pr
        act["pair"] = pair_l.unsqueeze(0)
    if tokens.get("token") is not None:
        act["token"] = tokens["token"].index_select(0, glob_t).unsqueeze(0)
    masks = {"valid": key_rows["valid"].to(torch.bool).unsqueeze(0),
             "token_valid": tokens["token_valid"].to(torch.bool).index_select(0, glob_t).unsqueeze(0),
             "window_mask": win_l.unsqueeze(0)}
    structure = {"key_index": kid_l.unsqueeze(0),
                 "atom_to_token": torch.as_tensor(loc, device=dev).unsqueeze(0)}
    return act, masks, structure


def owned_outputs(out: dict, shard: Shard) -> dict:
    """The owned part of a local forward's outputs: hidden / position_update rows and
    attention rows of the owned queries, token_output rows of the owned tokens."""
    lo, hi = shard.a0 - shard.e0, shard.a1 - shard.e0
    res = {"hidden": out["hidden"][0, lo:hi], "attention": out["attention"][0, :, lo:hi]}
    if "token_output" in out:
        res["token_output"] = out["token_output"][0, :shard.t1 - shard.t0]
    if "position_update" in out:
        res["position_update"] = out["position_update"][0, lo:hi]
    return res


def assemble(parts: list[tuple[Shard, dict]], B: int, A: int, T: int) -> dict:
    """Full-problem outputs from every shard's owned outputs (a test and gather helper)."""
    first = parts[0][1]
    like = first["hidden"]
    C = like.shape[-1]
    H, K = first["attention"].shape[0], first["attention"].shape[-1]
    res = {"hidden": torch.zeros((B, A, C), dtype=like.dtype, device=like.device),
           "attention": torch.zeros((B, H, A, K), dtype=like.dtype, device=like.device)}
    if "token_output" in first:
        res["token_output"] = torch.zeros((B, T, first["token_output"].shape[-1]),
                                          dtype=like.dtype, device=like.device)
    if "position_update" in first:
        res["position_update"] = torch.zeros((B, A, 3), dtype=like.dtype, device=like.device)
    for sh, o in parts:
        res["hidden"][sh.b, sh.a0:sh.a1] = o["hidden"]
        res["attention"][sh.b, :, sh.a0:sh.a1] = o["attention"]
        if "token_output" in o:
            res["token_output"][sh.b, sh.t0:sh.t1] = o["token_output"]
        if "position_update" in o:
            res["position_update"][sh.b, sh.a0:sh.a1] = o["position_update"]
    return res


def exchange(owned_key_rows: dict, shards: list[Shard], rank: int, group=None) -> dict:
    """Key-side rows of this rank's extended range [e0, e1), from its owned rows
    [a0, a1) and the other ranks' (point-to-point over torch.distributed: each rank
    sends every other rank of the same batch element the rows of its range that the
    other's halo covers, and receives the rows its own halo lacks). `shards` lists every
    rank's shard (one per rank, halo split only). Every rank makes the same sends and
    receives in the same order."""
    import torch.distributed as dist
    me = shards[rank]
    out, was_bool = {}, set()
    for name, t in owned_key_rows.items():
        if t is None:
            continue
        if t.dtype == torch.bool:        # moved as bytes (not every backend sends bool)
            t = t.to(torch.uint8)
            was_bool.add(name)
        full = torch.zeros((me.e1 - me.e0,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
        full[me.a0 - me.e0:me.a1 - me.e0] = t
        out[name] = full
    ops = []
    for other, sh in enumerate(shards):
        if other == rank or sh.b != me.b:
            continue
        # rows of mine that the other's halo covers
        s0, s1 = max(sh.e0, me.a0), min(sh.e1, me.a1)
        if s0 < s1:
            for name in sorted(out):
                ops.append(dist.P2POp(dist.isend, out[name][s0 - me.e0:s1 - me.e0].contiguous(), other, group))
        # rows of the other's range that my halo covers
        r0, r1 = max(me.e0, sh.a0), min(me.e1, sh.a1)
        if r0 < r1:
            for name in sorted(out):
                buf = torch.empty_like(out[name][r0 - me.e0:r1 - me.e0])
                ops.append((dist.P2POp(dist.irecv, buf, other, group), name, r0, r1, buf))
    plain = [op if isinstance(op, dist.P2POp) else op[0] for op in ops]
    if plain:
        for req in dist.batch_isend_irecv(plain):
            req.wait()
    for op in ops:
        if not isinstance(op, dist.P2POp):
            _, name, r0, r1, buf = op
            out[name][r0 - me.e0:r1 - me.e0] = buf
    for name in was_bool:
        out[name] = out[name].to(torch.bool)
    return out


def forward_rank(owned_key_rows: dict, query_rows: dict, tokens: dict, shards: list[Shard],
                 rank: int, parameters: dict, T: int, eps: float = 1e-5, style: str = "af3",
                 stage: str = "decoder", radius: int = -1, group=None) -> dict:
    """One rank's forward of a halo-sharded problem: exchange the key-side rows, build
    the extended problem, run the CUDA forward (atomenc.windowed_atom_attention) on it
    and return the owned outputs. owned_key_rows / query_rows are this rank's own atoms'
    rows (CUDA tensors; key_index and atom_to_token with global ids), tokens the
    replicated token-level tensors of its batch element."""
    from . import atomenc
    me = shards[rank]
    key_rows = exchange(owned_key_rows, shards, rank, group)
    act, msk, st = local_problem(key_rows, query_rows, tokens, me, T)
    out = atomenc.windowed_atom_attention(act, parameters, msk, st, eps, style, stage, radius)
    return owned_outputs(out, me)
