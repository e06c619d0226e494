"""atomenc_forward_noalloc: the forward pass for callers that may not allocate.

Some callers cannot allocate device memory: code running inside another framework's
stream capture (allocation calls are not allowed there), hosts whose memory pool owns
all device memory, latency-critical loops that cannot take an allocation's implicit
synchronisation. This entry point gives them the same forward pass with its scratch in
a fixed device array inside the library instead of a caller workspace.

The file name makes pytest collect it last, so a run that stops at its first failure
has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_windowed_atom_b200 import atomenc, workloads

CASES = [("af3", "encoder", "float32"), ("esmfold2", "decoder", "bfloat16"),
         ("esmfold2", "encoder", "float32"), ("af3", "decoder", "bfloat16")]
TOL = {"float32": 2e-4, "bfloat16": 2e-2}   # max|err| <= tol * (1 + |ref|), as in the parity tests


def _device_case(style, stage, dtype, device="cuda"):
    spec = workloads.tiny_spec(style, stage, dtype, A=500, T=60)
    w = workloads.make_inputs(spec, seed=21)
    fdt = torch.bfloat16 if dtype == "bfloat16" else torch.float32
    t = lambda a, d=None: torch.from_numpy(np.ascontiguousarray(a)).to(device, dtype=d)
    inputs = {**{k: t(v, fdt) for k, v in w["activations"].items()},
              **{k: t(v) for k, v in w["masks"].items()},
              **{k: t(v) for k, v in w["structure"].items()}}
    params = {k: t(v, fdt) for k, v in w["parameters"].items()}
    return spec, inputs, params


@pytest.mark.gpu
@pytest.mark.parametrize("style,stage,dtype", CASES)
def test_noalloc_matches_workspace_entry_point(style, stage, dtype):
    spec, inputs, params = _device_case(style, stage, dtype)
    shapes = atomenc.output_shapes(style, stage, inputs, params)
    fdt = inputs["atom"].dtype
    ref = {k: torch.empty(s, dtype=fdt, device="cuda") for k, s in shapes.items()}
    need = atomenc.atomenc_workspace_size(style, stage, inputs, params, ref)
    assert need <= atomenc.NOALLOC_SCRATCH_BYTES
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    atomenc.atomenc_forward(style, stage, inputs, params, spec.eps, spec.radius, ref, ws)
    torch.cuda.synchronize()
    assert not atomenc.atomenc_get_status(ws) & atomenc.STATUS_WAIT_TIMEOUT
    tol = TOL[dtype]
    for call in range(2):   # two calls in a row share the library's scratch array
        out = {k: torch.full(s, float("nan"), dtype=fdt, device="cuda") for k, s in shapes.items()}
        atomenc.atomenc_forward_noalloc(style, stage, inputs, params, spec.eps, spec.radius, out)
        torch.cuda.synchronize()
        st = atomenc.atomenc_noalloc_get_status()
        assert not st & atomenc.STATUS_WAIT_TIMEOUT, f"call {call}: device status {st:#x}"
        for k in shapes:
            r, g = ref[k].double(), out[k].double()
            assert torch.isfinite(g).all(), (call, k)
            bad = (g - r).abs() > tol * (1.0 + r.abs())
            assert not bad.any(), f"call {call}, {k}: {int(bad.sum())} elements out of tolerance"


def test_noalloc_rejects_shapes_beyond_its_array():
    """A workload whose scratch exceeds the fixed array is refused on the host with
    ATOMENC_ERR_TOO_LARGE before anything is enqueued (no device needed)."""
    spec = workloads.WORKLOADS["af3_encoder_bf16_b4_a8192"]
    B, A, K, C, S, H, D, P = spec.B, spec.A, spec.K, spec.C, spec.S, spec.H, spec.D, spec.P
    f = lambda *s: torch.empty(s, dtype=torch.bfloat16)
    inputs = {"atom": f(B, A, C), "condition": f(B, A, S), "pair": f(B, A, K, P),
              "valid": torch.empty(B, A, dtype=torch.bool),
              "token_valid": torch.empty(B, spec.T, dtype=torch.bool),
              "window_mask": torch.empty(B, A, K, dtype=torch.bool),
              "key_index": torch.empty(B, A, K, dtype=torch.int64),
              "atom_to_token": torch.empty(B, A, dtype=torch.int64)}
    HD = H * D
    params = {"cond_scale": f(3, S), "w_scale": f(3, S, C), "b_scale": f(3, C),
              "w_shift": f(3, S, C), "w_residual_gate": f(2, S, C), "b_residual_gate": f(2, C),
              "w_q": f(C, HD), "b_q": f(HD), "w_k": f(C, HD), "w_v": f(C, HD),
              "w_value_gate": f(C, HD), "pair_scale": f(P), "w_pair": f(P, H),
              "w_attention_out": f(HD, C), "w_ff_gate": f(C, spec.M), "w_ff_up": f(C, spec.M),
              "w_ff_out": f(spec.M, C), "w_pool": f(C, spec.U)}
    outs = {k: torch.empty(s, dtype=torch.bfloat16) for k, s in
            atomenc.output_shapes("af3", "encoder", inputs, params).items()}
    assert atomenc.atomenc_workspace_size("af3", "encoder", inputs, params, outs) > \
        atomenc.NOALLOC_SCRATCH_BYTES
    ins, prm, out = atomenc._structs(inputs, params, outs)
    rc = atomenc.load_library().atomenc_forward_noalloc(
        atomenc.STYLES["af3"], atomenc.STAGES["encoder"], ctypes.byref(ins), ctypes.byref(prm),
        1e-5, -1, ctypes.byref(out), None)
    assert rc == -12
    assert "64 MiB" in atomenc.atomenc_strerror(rc)
