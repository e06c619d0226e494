"""CPU float64 oracle of the windowed atom attention block (test infrastructure).

This package is the correctness reference for the CUDA library and nothing else:
only the tests, the package smoke check and the benchmark's CPU-baseline leg may
import it. The arithmetic lives in ``oracle.c`` (plain C, float64, straight loops
in the order the pages give the steps); this module only builds it with gcc and
marshals numpy arrays through ctypes. It shares no code with the CUDA path.

Sources: "Local atom attention, encoder pooling and decoder skip/readout"
(windowed_atom_attention), "AlphaFold 3 Atom Attention Encoder" and "ESMFold 2
Atom Attention Encoder", sections Required behavior and Worked example.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_HDR = os.path.join(_HERE, "oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")

STYLES = {"af3": 0, "esmfold2": 1}
STAGES = {"decoder": 0, "encoder": 1}


_LIB_OMP = os.path.join(_HERE, "liboracle_omp.so")


def _compile(lib: str, extra: list, force: bool) -> str:
    stale = not os.path.exists(lib) or any(
        os.path.getmtime(f) > os.path.getmtime(lib) for f in (_SRC, _HDR))
    if force or stale:
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared",
                               "-fno-fast-math", *extra, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, lib)
    return lib


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so beside it (gcc, -O2, no fast-math), and the
    same source with -fopenmp into liboracle_omp.so (per-atom loops on all host cores,
    each atom's arithmetic unchanged; used to time the oracle as a CPU baseline)."""
    _compile(_LIB_OMP, ["-fopenmp"], force)
    return _compile(_LIB, [], force)


_i64 = ctypes.c_int64
_pd = ctypes.POINTER(ctypes.c_double)
_pu8 = ctypes.POINTER(ctypes.c_uint8)
_pi64 = ctypes.POINTER(ctypes.c_int64)


class _Dims(ctypes.Structure):
    _fields_ = [(n, _i64) for n in "B A T K C S H D P M U V".split()]


class _Inputs(ctypes.Structure):
    _fields_ = [("atom", _pd), ("condition", _pd), ("pair", _pd), ("token", _pd),
                ("rope_cos", _pd), ("rope_sin", _pd), ("valid", _pu8),
                ("token_valid", _pu8), ("window_mask", _pu8), ("key_index", _pi64),
                ("atom_to_token", _pi64)]


_PARAM_NAMES = ["cond_scale", "w_scale", "b_scale", "w_shift", "w_residual_gate",
                "b_residual_gate", "w_mod", "w_q", "b_q", "w_k", "w_v", "w_value_gate",
                "pair_scale", "w_pair", "w_attention_out", "w_ff_gate", "w_ff_up",
                "w_ff_out", "w_pool", "w_token", "readout_scale", "readout_bias",
                "w_readout"]


class _Params(ctypes.Structure):
    _fields_ = [(n, _pd) for n in _PARAM_NAMES] + [("value_gate_per_head", ctypes.c_int32)]


class _CoreInputs(ctypes.Structure):
    _fields_ = [("q", _pd), ("k", _pd), ("v", _pd), ("g", _pd), ("pair", _pd),
                ("pair_scale", _pd), ("w_pair", _pd), ("key_index", _pi64),
                ("window_mask", _pu8), ("usable", _pu8)]


class _Outputs(ctypes.Structure):
    _fields_ = [("hidden", _pd), ("attention", _pd), ("token_output", _pd),
                ("position_update", _pd)]


_libs = {}


def _load(threads: str = "one"):
    """The oracle library: threads="one" (the checker) or "all" (OpenMP build)."""
    if threads not in _libs:
        build()
        lib = ctypes.CDLL(_LIB if threads == "one" else _LIB_OMP)
        lib.orc_sigmoid.restype = ctypes.c_double
        lib.orc_sigmoid.argtypes = [ctypes.c_double]
        lib.orc_silu.restype = ctypes.c_double
        lib.orc_silu.argtypes = [ctypes.c_double]
        for fn in (lib.orc_layer_norm, lib.orc_rms_norm):
            fn.restype = None
            fn.argtypes = [_pd, _i64, ctypes.c_double, _pd]
        lib.orc_rope_half_split.restype = None
        lib.orc_rope_half_split.argtypes = [_pd, _pd, _pd, _i64, _pd]
        lib.orc_masked_softmax.restype = None
        lib.orc_masked_softmax.argtypes = [_pd, _pu8, _i64, _pd]
        lib.orc_usable.restype = None
        lib.orc_usable.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Inputs), _pu8]
        lib.orc_permitted.restype = None
        lib.orc_permitted.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Inputs),
                                      _pu8, _i64, _pu8]
        lib.orc_forward.restype = ctypes.c_int
        lib.orc_forward.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(_Dims),
                                    ctypes.POINTER(_Inputs), ctypes.POINTER(_Params),
                                    ctypes.c_double, _i64, _pu8, ctypes.POINTER(_Outputs)]
        lib.orc_single_to_pair.restype = ctypes.c_int
        lib.orc_single_to_pair.argtypes = [_i64, _i64, _i64, _i64, _i64, _pd, _pu8] + [_pd] * 8 + [
            ctypes.c_double, ctypes.c_int, _pd, _pd]
        lib.orc_attention_core.restype = ctypes.c_int
        lib.orc_attention_core.argtypes = [ctypes.c_int] + [_i64] * 6 + [
            ctypes.POINTER(_CoreInputs), ctypes.c_double, _i64, _pd, _pd]
        lib.orc_attention_core_backward.restype = ctypes.c_int
        lib.orc_attention_core_backward.argtypes = [ctypes.c_int] + [_i64] * 6 + [
            ctypes.POINTER(_CoreInputs), ctypes.c_double, _i64, _pd, _pd] + [_pd] * 7
        lib.orc_threads.restype = ctypes.c_int
        lib.orc_threads.argtypes = []
        _libs[threads] = lib
    return _libs[threads]


def threads_used(threads: str = "all") -> int:
    """Host threads the per-atom loops of the chosen build run on."""
    return int(_load(threads).orc_threads())


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(arr, typ):
    return arr.ctypes.data_as(typ) if arr is not None else ctypes.cast(None, typ)


# ---------------------------------------------------------------- row helpers

def sigmoid(z: float) -> float:
    return _load().orc_sigmoid(float(z))


def silu(z: float) -> float:
    return _load().orc_silu(float(z))


def layer_norm(v, eps: float) -> np.ndarray:
    v = _f64(v)
    out = np.empty_like(v)
    _load().orc_layer_norm(_ptr(v, _pd), v.size, eps, _ptr(out, _pd))
    return out


def rms_norm(v, eps: float) -> np.ndarray:
    v = _f64(v)
    out = np.empty_like(v)
    _load().orc_rms_norm(_ptr(v, _pd), v.size, eps, _ptr(out, _pd))
    return out


def rope_half_split(q, cos, sin) -> np.ndarray:
    q, cos, sin = _f64(q), _f64(cos), _f64(sin)
    out = np.empty_like(q)
    _load().orc_rope_half_split(_ptr(q, _pd), _ptr(cos, _pd), _ptr(sin, _pd), q.size,
                                _ptr(out, _pd))
    return out


def masked_softmax(logits, permitted) -> np.ndarray:
    lg = _f64(logits)
    pm = np.ascontiguousarray(np.asarray(permitted, dtype=np.uint8))
    out = np.empty_like(lg)
    _load().orc_masked_softmax(_ptr(lg, _pd), _ptr(pm, _pu8), lg.size, _ptr(out, _pd))
    return out


# ---------------------------------------------------------------- full forward

def _u8(x):
    return None if x is None else np.ascontiguousarray(np.asarray(x).astype(np.uint8))


def _i64a(x):
    return None if x is None else np.ascontiguousarray(np.asarray(x, dtype=np.int64))


def _opt64(x):
    return None if x is None else _f64(x)


def infer_dims(style, stage, activations, parameters, masks, structure):
    """Dimensions from the shapes (the pages print no shape table; see oracle.h)."""
    atom = np.asarray(activations["atom"])
    B, A, C = atom.shape
    S = np.asarray(activations["condition"]).shape[-1]
    K = np.asarray(structure["key_index"]).shape[-1]
    T = np.asarray(masks["token_valid"]).shape[-1]
    HD = np.asarray(parameters["w_q"]).shape[-1]
    if style == "af3":
        H = np.asarray(parameters["w_pair"]).shape[-1]
        D = HD // H
        P = np.asarray(activations["pair"]).shape[-1]
    else:
        D = np.asarray(activations["rope_cos"]).shape[-1]
        H = HD // D
        P = 0
    M = np.asarray(parameters["w_ff_gate"]).shape[-1]
    U = np.asarray(parameters["w_pool"]).shape[-1] if stage == "encoder" else 0
    V = np.asarray(activations["token"]).shape[-1] if stage == "decoder" else 0
    return dict(B=B, A=A, T=T, K=K, C=C, S=S, H=H, D=D, P=P, M=M, U=U, V=V)


class OracleError(RuntimeError):
    pass


def windowed_atom_attention(activations, parameters, masks, structure, eps=1e-5,
                            style="af3", stage="decoder", radius=-1, query_select=None,
                            threads="one"):
    """Float64 forward pass; returns a dict of float64 numpy arrays.

    Returns hidden [B,A,C] and attention [B,H,A,K] plus token_output [B,T,U]
    (encoder) or position_update [B,A,3] (decoder). With ``query_select`` only the
    selected query atoms (and tokens all of whose usable atoms are selected) are
    computed; everything else is NaN. ``threads="all"`` runs the OpenMP build of the
    same source (identical per-atom arithmetic) on every host core.
    """
    lib = _load(threads)
    dm = infer_dims(style, stage, activations, parameters, masks, structure)
    dims = _Dims(**dm)
    keep = {}

    def hold(name, arr):
        keep[name] = arr
        return arr

    act = {k: hold("a_" + k, _opt64(activations.get(k))) for k in
           ("atom", "condition", "pair", "token", "rope_cos", "rope_sin")}
    msk = {k: hold("m_" + k, _u8(masks.get(k))) for k in ("valid", "token_valid", "window_mask")}
    st = {k: hold("s_" + k, _i64a(structure.get(k))) for k in ("key_index", "atom_to_token")}
    inputs = _Inputs(atom=_ptr(act["atom"], _pd), condition=_ptr(act["condition"], _pd),
                     pair=_ptr(act["pair"], _pd), token=_ptr(act["token"], _pd),
                     rope_cos=_ptr(act["rope_cos"], _pd), rope_sin=_ptr(act["rope_sin"], _pd),
                     valid=_ptr(msk["valid"], _pu8), token_valid=_ptr(msk["token_valid"], _pu8),
                     window_mask=_ptr(msk["window_mask"], _pu8),
                     key_index=_ptr(st["key_index"], _pi64),
                     atom_to_token=_ptr(st["atom_to_token"], _pi64))
    prm = {n: hold("p_" + n, _opt64(parameters.get(n))) for n in _PARAM_NAMES}
    per_head = 0
    if prm["w_value_gate"] is not None and dm["D"] > 1 and \
            prm["w_value_gate"].shape[-1] == dm["H"]:
        per_head = 1
    params = _Params(**{n: _ptr(prm[n], _pd) for n in _PARAM_NAMES},
                     value_gate_per_head=per_head)
    B, A, T, K, C, H, U = (dm[k] for k in "B A T K C H U".split())
    res = {"hidden": np.full((B, A, C), np.nan), "attention": np.full((B, H, A, K), np.nan)}
    if stage == "encoder":
        res["token_output"] = np.full((B, T, U), np.nan)
    else:
        res["position_update"] = np.full((B, A, 3), np.nan)
    outs = _Outputs(hidden=_ptr(res["hidden"], _pd), attention=_ptr(res["attention"], _pd),
                    token_output=_ptr(res.get("token_output"), _pd),
                    position_update=_ptr(res.get("position_update"), _pd))
    sel = _u8(query_select)
    rc = lib.orc_forward(STYLES[style], STAGES[stage], ctypes.byref(dims), ctypes.byref(inputs),
                         ctypes.byref(params), float(eps), int(radius), _ptr(sel, _pu8),
                         ctypes.byref(outs))
    if rc != 0:
        raise OracleError(f"orc_forward failed with code {rc}")
    return res


def usable(activations, parameters, masks, structure, style="af3", stage="encoder"):
    dm = infer_dims(style, stage, activations, parameters, masks, structure)
    msk = {k: _u8(masks.get(k)) for k in ("valid", "token_valid", "window_mask")}
    st = {k: _i64a(structure.get(k)) for k in ("key_index", "atom_to_token")}
    inputs = _Inputs(valid=_ptr(msk["valid"], _pu8), token_valid=_ptr(msk["token_valid"], _pu8),
                     window_mask=_ptr(msk["window_mask"], _pu8),
                     key_index=_ptr(st["key_index"], _pi64),
                     atom_to_token=_ptr(st["atom_to_token"], _pi64))
    out = np.zeros((dm["B"], dm["A"]), dtype=np.uint8)
    _load().orc_usable(ctypes.byref(_Dims(**dm)), ctypes.byref(inputs), _ptr(out, _pu8))
    return out.astype(bool)


def permitted(activations, parameters, masks, structure, radius=-1, style="af3",
              stage="encoder"):
    dm = infer_dims(style, stage, activations, parameters, masks, structure)
    msk = {k: _u8(masks.get(k)) for k in ("valid", "token_valid", "window_mask")}
    st = {k: _i64a(structure.get(k)) for k in ("key_index", "atom_to_token")}
    inputs = _Inputs(valid=_ptr(msk["valid"], _pu8), token_valid=_ptr(msk["token_valid"], _pu8),
                     window_mask=_ptr(msk["window_mask"], _pu8),
                     key_index=_ptr(st["key_index"], _pi64),
                     atom_to_token=_ptr(st["atom_to_token"], _pi64))
    use = np.zeros((dm["B"], dm["A"]), dtype=np.uint8)
    dims = _Dims(**dm)
    _load().orc_usable(ctypes.byref(dims), ctypes.byref(inputs), _ptr(use, _pu8))
    out = np.zeros((dm["B"], dm["A"], dm["K"]), dtype=np.uint8)
    _load().orc_permitted(ctypes.byref(dims), ctypes.byref(inputs), _ptr(use, _pu8),
                          int(radius), _ptr(out, _pu8))
    return out.astype(bool)


# ---------------------------------------------------------------- single to pair

def single_to_pair(activations, parameters, masks, eps=1e-5, output_norm=False):
    """Page "ESMFold Single-to-Pair Features" (esmfold_single_to_pair), float64:
    returns (pair_features [B,N,N,2H], output [B,N,N,D]). Keys as the page's worked
    example prints them: x; mask; weight [C,2H], bias, norm_scale, norm_bias,
    out_weight [2H,D], out_bias, and output_scale / output_bias for output_norm."""
    x = _f64(activations["x"])
    B, N, C = x.shape
    mask = _u8(masks["mask"])
    w = _f64(parameters["weight"])
    H2 = w.shape[1]
    if H2 % 2:
        raise OracleError(-2, "weight has an odd number of columns")
    ow = _f64(parameters["out_weight"])
    Dp = ow.shape[1]
    nsc, nbi = _f64(parameters["norm_scale"]), _f64(parameters["norm_bias"])
    b, ob = _f64(parameters["bias"]), _f64(parameters["out_bias"])
    osc = _f64(parameters["output_scale"]) if output_norm else None
    obi = _f64(parameters["output_bias"]) if output_norm else None
    pf = np.zeros((B, N, N, H2))
    out = np.zeros((B, N, N, Dp))
    rc = _load().orc_single_to_pair(B, N, C, H2 // 2, Dp, _ptr(x, _pd), _ptr(mask, _pu8),
                                    _ptr(nsc, _pd), _ptr(nbi, _pd), _ptr(w, _pd), _ptr(b, _pd),
                                    _ptr(ow, _pd), _ptr(ob, _pd), _ptr(osc, _pd), _ptr(obi, _pd),
                                    float(eps), 1 if output_norm else 0, _ptr(pf, _pd),
                                    _ptr(out, _pd))
    if rc != 0:
        raise OracleError(rc, "orc_single_to_pair")
    return pf, out


# ---------------------------------------------------------------- attention core

def _core_struct(core, style):
    keep = {}
    for n in ("q", "k", "v", "g"):
        keep[n] = _f64(core[n])
    for n in ("pair", "pair_scale", "w_pair"):
        keep[n] = _f64(core[n]) if style == "af3" else None
    keep["key_index"] = _i64a(core["key_index"])
    keep["window_mask"] = _u8(core["window_mask"])
    keep["usable"] = _u8(core["usable"])
    st = _CoreInputs(q=_ptr(keep["q"], _pd), k=_ptr(keep["k"], _pd), v=_ptr(keep["v"], _pd),
                     g=_ptr(keep["g"], _pd), pair=_ptr(keep["pair"], _pd),
                     pair_scale=_ptr(keep["pair_scale"], _pd), w_pair=_ptr(keep["w_pair"], _pd),
                     key_index=_ptr(keep["key_index"], _pi64),
                     window_mask=_ptr(keep["window_mask"], _pu8),
                     usable=_ptr(keep["usable"], _pu8))
    return st, keep


def _core_dims(core, style, H):
    B, A, HD = np.asarray(core["q"]).shape
    K = np.asarray(core["key_index"]).shape[-1]
    P = np.asarray(core["pair"]).shape[-1] if style == "af3" else 0
    return B, A, K, H, HD // H, P


def attention_core(core, H, eps=1e-5, style="af3", radius=-1):
    """The attention core alone (float64): core = dict of q, k, v, g [B,A,H*D],
    key_index [B,A,K], window_mask [B,A,K], usable [B,A] and, for AF3, pair [B,A,K,P],
    pair_scale [P], w_pair [P,H]. Returns (attention [B,H,A,K], out [B,A,H*D])."""
    st, keep = _core_struct(core, style)
    B, A, K, H, D, P = _core_dims(core, style, H)
    att = np.zeros((B, H, A, K))
    out = np.zeros((B, A, H * D))
    rc = _load().orc_attention_core(STYLES[style], B, A, K, H, D, P, ctypes.byref(st), float(eps),
                                    int(radius), _ptr(att, _pd), _ptr(out, _pd))
    if rc != 0:
        raise OracleError(f"orc_attention_core failed with code {rc}")
    return att, out


def attention_core_backward(core, H, d_out, d_attention=None, eps=1e-5, style="af3", radius=-1):
    """Gradient of attention_core: returns a dict d_q, d_k, d_v, d_g [B,A,H*D] and for AF3
    d_pair [B,A,K,P], d_pair_scale [P], d_w_pair [P,H]."""
    st, keep = _core_struct(core, style)
    B, A, K, H, D, P = _core_dims(core, style, H)
    dO = _f64(d_out)
    dA = None if d_attention is None else _f64(d_attention)
    res = {n: np.zeros((B, A, H * D)) for n in ("d_q", "d_k", "d_v", "d_g")}
    if style == "af3":
        res.update(d_pair=np.zeros((B, A, K, P)), d_pair_scale=np.zeros(P), d_w_pair=np.zeros((P, H)))
    rc = _load().orc_attention_core_backward(
        STYLES[style], B, A, K, H, D, P, ctypes.byref(st), float(eps), int(radius),
        _ptr(dO, _pd), _ptr(dA, _pd), _ptr(res["d_q"], _pd), _ptr(res["d_k"], _pd),
        _ptr(res["d_v"], _pd), _ptr(res["d_g"], _pd), _ptr(res.get("d_pair"), _pd),
        _ptr(res.get("d_pair_scale"), _pd), _ptr(res.get("d_w_pair"), _pd))
    if rc != 0:
        raise OracleError(f"orc_attention_core_backward failed with code {rc}")
    return res
