"""Seeded synthetic inputs for the windowed atom attention block.

This module draws random numbers and builds index structure; it holds none of the
block's arithmetic. Both the CUDA path (tests, benchmark) and the CPU oracle take
their inputs from here, so the two sides always see identical values.

Arrays are numpy: floats as float32 whose values are already rounded to the
workload's storage dtype (bf16 values are exactly representable in float32),
indices int64, masks bool. Dictionary keys follow the names the pages use in their
formulas (the pages print no key table).

Recipe (names and sizes of the five reference workloads are in ``WORKLOADS``):
  * activations atom / condition / pair / token ~ N(0, 1);
  * weight matrices ~ N(0, 1/fan_in), fan_in = contraction width; w_mod ~ N(0, 0.02^2);
  * cond_scale, pair_scale, readout_scale = 1 + 0.1 N(0, 1);
    b_q, b_scale, b_residual_gate, readout_bias = 0.1 N(0, 1);
  * masks Bernoulli with the workload's rates;
  * rope: cos/sin of uniform(0, 2 pi) angles, one angle per (atom, dim pair), the
    pair being dims d and d + D/2;
  * keys "blocked": query block b = a // block uses ids block*b - offset + k,
    out-of-range ids become -1; keys "random": a + uniform{-w..w}, out-of-range ids
    kept as drawn (the block treats them as missing);
  * slot corruption: a fraction of slots copies another slot of the same row
    (duplicates), another fraction becomes -1;
  * ragged tokens: per-token counts uniform{1..n}; atom a maps to
    searchsorted(cumsum(counts), a, 'right'); atoms past the total map to T (out of
    range, hence unusable) and trailing tokens may get no atom;
  * invalid atoms may carry NaN / +Inf / -Inf payloads in atom, condition, rope and
    (AF3) the pair rows of their query slots.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class WorkloadSpec:
    name: str
    style: str            # 'af3' | 'esmfold2'
    stage: str            # 'encoder' | 'decoder'
    dtype: str            # 'float32' | 'bfloat16'
    B: int
    A: int
    T: int
    K: int
    C: int = 128
    S: int = 128
    H: int = 4
    D: int = 32
    P: int = 16
    M: int = 256
    U: int = 384
    V: int = 384
    keys: tuple = ("blocked", 32, 48)      # ('blocked', block, offset) | ('random', half_width)
    tokens: tuple = ("fixed", 8)           # ('fixed', atoms_per_token) | ('ragged', max_per_token)
    valid_p: float = 1.0
    token_valid_p: float = 1.0
    window_p: float = 1.0
    dup_p: float = 0.0
    miss_p: float = 0.0
    poison_invalid: bool = False
    radius: int = -1
    eps: float = 1e-5
    description: str = ""

    @property
    def entries(self) -> int:
        """Attention entries B*A*H*K (one per query atom, head and key slot)."""
        return self.B * self.A * self.H * self.K

    @property
    def atoms(self) -> int:
        return self.B * self.A

    def replace(self, **kw) -> "WorkloadSpec":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "af3_encoder_fp32_a256": WorkloadSpec(
        name="af3_encoder_fp32_a256", style="af3", stage="encoder", dtype="float32",
        B=1, A=256, T=32, K=32, C=128, S=64, H=4, D=32, P=16, M=256, U=384,
        keys=("blocked", 16, 8), tokens=("fixed", 8), valid_p=0.95, window_p=0.90,
        description="AF3 encoder, fp32, B=1 A=256 T=32, blocked keys K=32"),
    "esm_encoder_fp32_a4096": WorkloadSpec(
        name="esm_encoder_fp32_a4096", style="esmfold2", stage="encoder", dtype="float32",
        B=1, A=4096, T=512, K=128, C=128, S=128, H=4, D=32, P=0, M=256, U=384,
        keys=("blocked", 32, 48), tokens=("fixed", 8), valid_p=0.97, window_p=0.95,
        radius=64, description="ESMFold2 encoder, fp32, B=1 A=4096 T=512, K=128, radius 64"),
    "af3_encoder_bf16_b4_a8192": WorkloadSpec(
        name="af3_encoder_bf16_b4_a8192", style="af3", stage="encoder", dtype="bfloat16",
        B=4, A=8192, T=1024, K=128, C=128, S=128, H=4, D=32, P=16, M=256, U=384,
        keys=("blocked", 32, 48), tokens=("ragged", 15), valid_p=0.95, dup_p=0.02,
        miss_p=0.03, poison_invalid=True,
        description="AF3 encoder, bf16, B=4 A=8192 T=1024 ragged, K=128, dup/missing slots"),
    "af3_decoder_fp32_a24576": WorkloadSpec(
        name="af3_decoder_fp32_a24576", style="af3", stage="decoder", dtype="float32",
        B=1, A=24576, T=3072, K=128, C=128, S=128, H=4, D=32, P=16, M=256, V=384,
        keys=("blocked", 32, 48), tokens=("fixed", 8), token_valid_p=0.98,
        description="AF3 decoder, fp32, B=1 A=24576 T=3072, K=128"),
    "esm_encoder_bf16_b2_a32768": WorkloadSpec(
        name="esm_encoder_bf16_b2_a32768", style="esmfold2", stage="encoder", dtype="bfloat16",
        B=2, A=32768, T=4096, K=128, C=128, S=256, H=8, D=16, P=0, M=256, U=384,
        keys=("random", 256), tokens=("ragged", 16), valid_p=0.90, window_p=0.90,
        poison_invalid=True, radius=128,
        description="ESMFold2 encoder, bf16, B=2 A=32768 T=4096 ragged, random keys +-256"),
}

WORKLOAD_ORDER = list(WORKLOADS)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), kept as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    nan = np.isnan(x)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    r = ((u + bias) & np.uint32(0xFFFF0000)).astype(np.uint32)
    r = np.where(nan, np.uint32(0x7FC00000), r)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are exactly bf16."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32)
    return round_to_bf16(x) if dtype == "bfloat16" else np.ascontiguousarray(x)


def _key_index(rng, spec: WorkloadSpec) -> np.ndarray:
    B, A, K = spec.B, spec.A, spec.K
    a = np.arange(A, dtype=np.int64)[:, None]
    k = np.arange(K, dtype=np.int64)[None, :]
    if spec.keys[0] == "blocked":
        _, block, offset = spec.keys
        ids = (a // block) * block - offset + k
        ids = np.where((ids >= 0) & (ids < A), ids, -1)
        kid = np.broadcast_to(ids, (B, A, K)).copy()
    elif spec.keys[0] == "random":
        _, w = spec.keys
        kid = a[None] + rng.integers(-w, w + 1, size=(B, A, K), dtype=np.int64)
    else:
        raise ValueError(spec.keys)
    if spec.dup_p > 0:
        dup = rng.random((B, A, K)) < spec.dup_p
        other = (k[None] + rng.integers(1, K, size=(B, A, K))) % K if K > 1 else \
            np.zeros((B, A, K), dtype=np.int64)
        src = np.take_along_axis(kid, other, axis=2)
        kid = np.where(dup, src, kid)
    if spec.miss_p > 0:
        kid = np.where(rng.random((B, A, K)) < spec.miss_p, -1, kid)
    return np.ascontiguousarray(kid, dtype=np.int64)


def _atom_to_token(rng, spec: WorkloadSpec) -> np.ndarray:
    B, A, T = spec.B, spec.A, spec.T
    if spec.tokens[0] == "fixed":
        n = spec.tokens[1]
        att = np.minimum(np.arange(A, dtype=np.int64) // n, T)
        return np.broadcast_to(att, (B, A)).copy()
    n = spec.tokens[1]
    out = np.empty((B, A), dtype=np.int64)
    for b in range(B):
        counts = rng.integers(1, n + 1, size=T)
        ends = np.cumsum(counts)
        out[b] = np.searchsorted(ends, np.arange(A), side="right")
    return out


def make_inputs(spec: WorkloadSpec, seed: int = 0) -> dict:
    """Draw one workload; returns {'activations','parameters','masks','structure',
    'spec'} with numpy arrays."""
    rng = np.random.default_rng(seed)
    B, A, T, K, C, S, H, D, P, M, U, V = (spec.B, spec.A, spec.T, spec.K, spec.C, spec.S,
                                          spec.H, spec.D, spec.P, spec.M, spec.U, spec.V)
    HD = H * D
    dt = spec.dtype
    af3, enc = spec.style == "af3", spec.stage == "encoder"

    def normal(*shape, std=1.0):
        return rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)

    masks = {
        "valid": rng.random((B, A)) < spec.valid_p,
        "token_valid": rng.random((B, T)) < spec.token_valid_p,
        "window_mask": rng.random((B, A, K)) < spec.window_p,
    }
    structure = {"key_index": _key_index(rng, spec), "atom_to_token": _atom_to_token(rng, spec)}

    act = {"atom": normal(B, A, C), "condition": normal(B, A, S)}
    if af3:
        act["pair"] = normal(B, A, K, P)
    else:
        theta = rng.uniform(0.0, 2.0 * np.pi, size=(B, A, D // 2))
        theta = np.concatenate([theta, theta], axis=-1)
        act["rope_cos"] = np.cos(theta).astype(np.float32)
        act["rope_sin"] = np.sin(theta).astype(np.float32)
    if not enc:
        act["token"] = normal(B, T, V)

    if spec.poison_invalid:
        bad = ~masks["valid"]
        pool = np.array([np.nan, np.inf, -np.inf], dtype=np.float32)
        for name in ("atom", "condition", "rope_cos", "rope_sin"):
            if name in act:
                arr = act[name]
                pick = pool[rng.integers(0, 3, size=arr.shape)]
                poison = bad[..., None] & (rng.random(arr.shape) < 0.5)
                act[name] = np.where(poison, pick, arr).astype(np.float32)
        if af3:
            arr = act["pair"]
            poison = bad[..., None, None] & (rng.random(arr.shape) < 0.5)
            act["pair"] = np.where(poison, np.float32(np.nan), arr).astype(np.float32)

    p = {}

    def w(*shape, fan_in):
        return normal(*shape, std=1.0 / np.sqrt(fan_in))

    if af3:
        p["cond_scale"] = 1.0 + 0.1 * normal(3, S)
        p["w_scale"] = w(3, S, C, fan_in=S)
        p["b_scale"] = 0.1 * normal(3, C)
        p["w_shift"] = w(3, S, C, fan_in=S)
        p["w_residual_gate"] = w(2, S, C, fan_in=S)
        p["b_residual_gate"] = 0.1 * normal(2, C)
    else:
        p["w_mod"] = normal(S, 6, C, std=0.02)
    p["w_q"] = w(C, HD, fan_in=C)
    if af3:
        p["b_q"] = 0.1 * normal(HD)
    p["w_k"] = w(C, HD, fan_in=C)
    p["w_v"] = w(C, HD, fan_in=C)
    p["w_value_gate"] = w(C, HD, fan_in=C)
    if af3:
        p["pair_scale"] = 1.0 + 0.1 * normal(P)
        p["w_pair"] = w(P, H, fan_in=P)
    p["w_attention_out"] = w(HD, C, fan_in=HD)
    p["w_ff_gate"] = w(C, M, fan_in=C)
    p["w_ff_up"] = w(C, M, fan_in=C)
    p["w_ff_out"] = w(M, C, fan_in=M)
    if enc:
        p["w_pool"] = w(C, U, fan_in=C)
    else:
        p["w_token"] = w(V, C, fan_in=V)
        p["readout_scale"] = 1.0 + 0.1 * normal(C)
        if not af3:
            p["readout_bias"] = 0.1 * normal(C)
        p["w_readout"] = w(C, 3, fan_in=C)

    act = {k: _store(v, dt) for k, v in act.items()}
    p = {k: _store(v, dt) for k, v in p.items()}
    return {"activations": act, "parameters": p, "masks": masks, "structure": structure,
            "spec": spec}


def tiny_spec(style="af3", stage="encoder", dtype="float32", **kw) -> WorkloadSpec:
    """A small workload for parity cases (several tiles plus a ragged tail)."""
    base = dict(name=f"tiny_{style}_{stage}_{dtype}", style=style, stage=stage, dtype=dtype,
                B=2, A=300, T=40, K=24, C=128, S=64, H=4, D=32, P=16 if style == "af3" else 0,
                M=256, U=384, V=96, keys=("blocked", 16, 8), tokens=("ragged", 12),
                valid_p=0.9, token_valid_p=0.95, window_p=0.85, dup_p=0.05, miss_p=0.05,
                poison_invalid=True, radius=-1)
    base.update(kw)
    return WorkloadSpec(**base)
