"""The C-ABI library loads without a GPU, exports every symbol include/atomenc.h declares,
and rejects bad arguments on the host before any launch (no compute calls here)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

from sparse_windowed_atom_b200 import atomenc, build as cbuild, workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    cbuild.build()
    return atomenc.load_library()


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*[A-Za-z_][\w \*]*?\b(atomenc_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert {"atomenc_forward", "atomenc_workspace_size", "atomenc_get_status",
            "atomenc_strerror"} <= set(names)
    out = subprocess.check_output(["nm", "-D", "--defined-only", atomenc.LIB_PATH], text=True)
    exported = set(re.findall(r"\bT (\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(lib, n)


def test_version_and_strerror(lib):
    assert atomenc.atomenc_version() >= 1
    assert atomenc.atomenc_strerror(0) == "ok"
    for code in range(-1, -12, -1):
        assert atomenc.atomenc_strerror(code) != "unknown atomenc status"


def _host_case(style="af3", stage="encoder", dtype="float32"):
    """Host tensors: the validator only reads shapes, dtypes and strides, never data."""
    spec = workloads.tiny_spec(style, stage, dtype, B=1, A=20, T=4, K=6, C=8, S=4, H=2, D=4,
                               P=3, M=8, U=5, V=6)
    w = workloads.make_inputs(spec, seed=0)
    fdt = torch.bfloat16 if dtype == "bfloat16" else torch.float32
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    inputs = {**{k: t(v).to(fdt) for k, v in w["activations"].items()},
              **{k: t(v) for k, v in w["masks"].items()},
              **{k: t(v) for k, v in w["structure"].items()}}
    params = {k: t(v).to(fdt) for k, v in w["parameters"].items()}
    outs = {k: torch.empty(s, dtype=fdt) for k, s in
            atomenc.output_shapes(style, stage, inputs, params).items()}
    return inputs, params, outs


@pytest.mark.parametrize("style,stage", [("af3", "encoder"), ("af3", "decoder"),
                                         ("esmfold2", "encoder"), ("esmfold2", "decoder")])
def test_workspace_size_validates(lib, style, stage):
    inputs, params, outs = _host_case(style, stage)
    n = atomenc.atomenc_workspace_size(style, stage, inputs, params, outs)
    assert n > 0 and n % 256 == 0


def _forward_rc(style, stage, inputs, params, outs, eps=1e-5, radius=-1, ws_bytes=None):
    ins, prm, out = atomenc._structs(inputs, params, outs)
    ws = ctypes.c_void_p(256 * 1024) if ws_bytes != 0 else ctypes.c_void_p(0)
    return atomenc.load_library().atomenc_forward(
        atomenc.STYLES[style], atomenc.STAGES[stage], ctypes.byref(ins), ctypes.byref(prm),
        eps, radius, ctypes.byref(out), ws, ws_bytes if ws_bytes is not None else 1, None)


def test_host_side_errors(lib):
    inputs, params, outs = _host_case("esmfold2", "encoder")
    # every case below fails validation before any CUDA call
    assert _forward_rc("esmfold2", "encoder", inputs, params, outs, eps=0.0) == -6
    assert _forward_rc("esmfold2", "encoder", inputs, params, outs, eps=float("inf")) == -6
    assert _forward_rc("esmfold2", "encoder", inputs, params, outs, radius=-2) == -7
    assert _forward_rc("esmfold2", "encoder", inputs, params, outs, ws_bytes=0) == -10
    assert _forward_rc("esmfold2", "encoder", inputs, params, outs, ws_bytes=16) == -10
    bad = dict(inputs)
    bad["key_index"] = inputs["key_index"].to(torch.int32)
    assert _forward_rc("esmfold2", "encoder", bad, params, outs) == -3
    bad = dict(inputs)
    bad["window_mask"] = inputs["window_mask"][:, :, :-1]
    assert _forward_rc("esmfold2", "encoder", bad, params, outs) == -4
    bad = dict(inputs)
    bad["condition"] = inputs["condition"].transpose(1, 2).contiguous().transpose(1, 2)
    assert _forward_rc("esmfold2", "encoder", bad, params, outs) == -5
    bad = dict(inputs)
    odd = inputs["rope_cos"][..., :3].contiguous()
    bad["rope_cos"], bad["rope_sin"] = odd, odd
    prm = dict(params)
    for k in ("w_q", "w_k", "w_v", "w_value_gate"):
        prm[k] = params[k][:, :6].contiguous()
    prm["w_attention_out"] = params["w_attention_out"][:6].contiguous()
    assert _forward_rc("esmfold2", "encoder", bad, prm, outs) == -8
    p2 = dict(params)
    del p2["w_mod"]
    assert _forward_rc("esmfold2", "encoder", inputs, p2, outs) == -1
    p3 = {k: v.to(torch.bfloat16) for k, v in params.items()}
    assert _forward_rc("esmfold2", "encoder", inputs, p3, outs) == -3
    ins, prm3, out = atomenc._structs(inputs, params, outs)
    assert atomenc.load_library().atomenc_forward(7, 1, ctypes.byref(ins), ctypes.byref(prm3), 1e-5,
                                                  -1, ctypes.byref(out), None, 0, None) == -2


def test_bf16_eps_that_rounds_to_zero(lib):
    inputs, params, outs = _host_case("af3", "encoder", "bfloat16")
    assert _forward_rc("af3", "encoder", inputs, params, outs, eps=1e-45) == -6
