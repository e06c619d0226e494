"""Thin Python binding of the atomenc C ABI (include/atomenc.h).

Argument marshalling only: every step of the block runs in the CUDA library
libatomenc.so. torch supplies device memory and streams. There is no CPU path: if
the library is missing or no CUDA device is present, the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libatomenc.so")

ATOMENC_F32, ATOMENC_BF16, ATOMENC_I64, ATOMENC_BOOL = 0, 1, 2, 3
STYLES = {"af3": 0, "esmfold2": 1}
STAGES = {"decoder": 0, "encoder": 1}
_DTYPES = {torch.float32: ATOMENC_F32, torch.bfloat16: ATOMENC_BF16,
           torch.int64: ATOMENC_I64, torch.bool: ATOMENC_BOOL}


class AtomencTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 5), ("stride", ctypes.c_int64 * 5)]


INPUT_FIELDS = ["atom", "condition", "pair", "token", "rope_cos", "rope_sin", "valid",
                "token_valid", "window_mask", "key_index", "atom_to_token"]
PARAM_FIELDS = ["cond_scale", "w_scale", "b_scale", "w_shift", "w_residual_gate",
                "b_residual_gate", "w_mod", "w_q", "b_q", "w_k", "w_v", "w_value_gate",
                "pair_scale", "w_pair", "w_attention_out", "w_ff_gate", "w_ff_up", "w_ff_out",
                "w_pool", "w_token", "readout_scale", "readout_bias", "w_readout"]
OUTPUT_FIELDS = ["hidden", "attention", "token_output", "position_update"]


class AtomencInputs(ctypes.Structure):
    _fields_ = [(n, AtomencTensor) for n in INPUT_FIELDS]


class AtomencParams(ctypes.Structure):
    _fields_ = [(n, AtomencTensor) for n in PARAM_FIELDS]


class AtomencOutputs(ctypes.Structure):
    _fields_ = [(n, AtomencTensor) for n in OUTPUT_FIELDS]


S2P_INPUT_FIELDS = ["x", "mask"]
S2P_PARAM_FIELDS = ["norm_scale", "norm_bias", "weight", "bias", "out_weight", "out_bias",
                    "output_scale", "output_bias"]
S2P_OUTPUT_FIELDS = ["pair_features", "output"]


class AtomencS2PInputs(ctypes.Structure):
    _fields_ = [(n, AtomencTensor) for n in S2P_INPUT_FIELDS]


class AtomencS2PParams(ctypes.Structure):
    _fields_ = [(n, AtomencTensor) for n in S2P_PARAM_FIELDS]


class AtomencS2POutputs(ctypes.Structure):
    _fields_ = [(n, AtomencTensor) for n in S2P_OUTPUT_FIELDS]


CORE_BWD_INPUT_FIELDS = ["q", "k", "v", "g", "key_index", "window_mask", "usable", "pair",
                         "pair_scale", "w_pair", "d_out", "d_attention"]
CORE_BWD_OUTPUT_FIELDS = ["d_q", "d_k", "d_v", "d_g", "d_pair", "d_pair_scale", "d_w_pair"]


class AtomencCoreBwdInputs(ctypes.Structure):
    _fields_ = [(n, AtomencTensor) for n in CORE_BWD_INPUT_FIELDS]


class AtomencCoreBwdOutputs(ctypes.Structure):
    _fields_ = [(n, AtomencTensor) for n in CORE_BWD_OUTPUT_FIELDS]


class AtomencError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: atomenc error {code}: {atomenc_strerror(code)}")
        self.code = code


_lib = None


def load_library() -> ctypes.CDLL:
    """Load libatomenc.so; raise if it has not been built (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_windowed_atom_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        lib.atomenc_workspace_size.restype = ctypes.c_size_t
        lib.atomenc_workspace_size.argtypes = [ctypes.c_int, ctypes.c_int, P(AtomencInputs),
                                               P(AtomencParams), P(AtomencOutputs)]
        lib.atomenc_forward.restype = ctypes.c_int
        lib.atomenc_forward.argtypes = [ctypes.c_int, ctypes.c_int, P(AtomencInputs),
                                        P(AtomencParams), ctypes.c_double, ctypes.c_int64,
                                        P(AtomencOutputs), ctypes.c_void_p, ctypes.c_size_t,
                                        ctypes.c_void_p]
        for fn in ("atomenc_weight_image_size", "atomenc_prepared_workspace_size"):
            getattr(lib, fn).restype = ctypes.c_size_t
            getattr(lib, fn).argtypes = lib.atomenc_workspace_size.argtypes
        lib.atomenc_prepare_weights.restype = ctypes.c_int
        lib.atomenc_prepare_weights.argtypes = [ctypes.c_int, ctypes.c_int, P(AtomencInputs),
                                                P(AtomencParams), P(AtomencOutputs),
                                                ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
        lib.atomenc_forward_prepared.restype = ctypes.c_int
        lib.atomenc_forward_prepared.argtypes = [ctypes.c_int, ctypes.c_int, P(AtomencInputs),
                                                 P(AtomencParams), ctypes.c_void_p, ctypes.c_size_t,
                                                 ctypes.c_double, ctypes.c_int64, P(AtomencOutputs),
                                                 ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
        lib.atomenc_forward_profiled.restype = ctypes.c_int
        lib.atomenc_forward_profiled.argtypes = lib.atomenc_forward.argtypes + [
            P(ctypes.c_void_p), ctypes.c_int, P(ctypes.c_int)]
        lib.atomenc_forward_noalloc.restype = ctypes.c_int
        lib.atomenc_forward_noalloc.argtypes = [ctypes.c_int, ctypes.c_int, P(AtomencInputs),
                                                P(AtomencParams), ctypes.c_double, ctypes.c_int64,
                                                P(AtomencOutputs), ctypes.c_void_p]
        lib.atomenc_forward_traced.restype = ctypes.c_int
        lib.atomenc_forward_traced.argtypes = lib.atomenc_forward.argtypes + [
            P(ctypes.c_void_p), ctypes.c_int, P(ctypes.c_int), P(ctypes.c_int)]
        lib.atomenc_get_status.restype = ctypes.c_int
        lib.atomenc_get_status.argtypes = [ctypes.c_void_p, P(ctypes.c_int), ctypes.c_void_p]
        lib.atomenc_noalloc_get_status.restype = ctypes.c_int
        lib.atomenc_noalloc_get_status.argtypes = [P(ctypes.c_int), ctypes.c_void_p]
        lib.atomenc_debug_peer_wait.restype = ctypes.c_int
        lib.atomenc_debug_peer_wait.argtypes = [ctypes.c_uint32, ctypes.c_int]
        lib.atomenc_strerror.restype = ctypes.c_char_p
        lib.atomenc_strerror.argtypes = [ctypes.c_int]
        lib.atomenc_version.restype = ctypes.c_int
        lib.atomenc_version.argtypes = []
        lib.atomenc_attention_backward_workspace_size.restype = ctypes.c_size_t
        lib.atomenc_attention_backward_workspace_size.argtypes = [
            ctypes.c_int, P(AtomencCoreBwdInputs), ctypes.c_int64, P(AtomencCoreBwdOutputs)]
        lib.atomenc_attention_backward.restype = ctypes.c_int
        lib.atomenc_attention_backward.argtypes = [
            ctypes.c_int, P(AtomencCoreBwdInputs), ctypes.c_int64, ctypes.c_double, ctypes.c_int64,
            P(AtomencCoreBwdOutputs), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
        lib.atomenc_s2p_workspace_size.restype = ctypes.c_size_t
        lib.atomenc_s2p_workspace_size.argtypes = [P(AtomencS2PInputs), P(AtomencS2PParams),
                                                   ctypes.c_int, P(AtomencS2POutputs)]
        lib.atomenc_single_to_pair.restype = ctypes.c_int
        lib.atomenc_single_to_pair.argtypes = [P(AtomencS2PInputs), P(AtomencS2PParams),
                                               ctypes.c_double, ctypes.c_int,
                                               P(AtomencS2POutputs), ctypes.c_void_p,
                                               ctypes.c_size_t, ctypes.c_void_p]
        _lib = lib
    return _lib


def describe(t) -> AtomencTensor:
    """atomenc_tensor for a torch tensor (or an empty descriptor for None)."""
    d = AtomencTensor()
    if t is None:
        return d
    if t.dim() > 5:
        raise ValueError("atomenc tensors have at most 5 dims")
    d.data = t.data_ptr()
    d.dtype = _DTYPES.get(t.dtype, 99)      # the library rejects unknown codes
    d.ndim = t.dim()
    for i, (s, st) in enumerate(zip(t.shape, t.stride())):
        d.shape[i] = s
        d.stride[i] = st
    return d


def _structs(inputs: dict, params: dict, outputs: dict):
    ins = AtomencInputs(**{n: describe(inputs.get(n)) for n in INPUT_FIELDS})
    prm = AtomencParams(**{n: describe(params.get(n)) for n in PARAM_FIELDS})
    outs = AtomencOutputs(**{n: describe(outputs.get(n)) for n in OUTPUT_FIELDS})
    return ins, prm, outs


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def atomenc_strerror(code: int) -> str:
    return load_library().atomenc_strerror(int(code)).decode()


def atomenc_version() -> int:
    return load_library().atomenc_version()


def atomenc_workspace_size(style: str, stage: str, inputs: dict, params: dict,
                           outputs: dict) -> int:
    ins, prm, outs = _structs(inputs, params, outputs)
    n = load_library().atomenc_workspace_size(STYLES[style], STAGES[stage], ctypes.byref(ins),
                                              ctypes.byref(prm), ctypes.byref(outs))
    if n == 0:
        raise ValueError("atomenc_workspace_size: the arguments do not validate")
    return int(n)


def atomenc_forward(style: str, stage: str, inputs: dict, params: dict, eps: float,
                    radius: int, outputs: dict, workspace: torch.Tensor, stream=None) -> None:
    ins, prm, outs = _structs(inputs, params, outputs)
    rc = load_library().atomenc_forward(STYLES[style], STAGES[stage], ctypes.byref(ins),
                                        ctypes.byref(prm), float(eps), int(radius),
                                        ctypes.byref(outs), workspace.data_ptr(),
                                        workspace.numel() * workspace.element_size(),
                                        _stream_ptr(stream))
    if rc != 0:
        raise AtomencError(rc, "atomenc_forward")


def _size(fn: str, style, stage, inputs, params, outputs) -> int:
    ins, prm, outs = _structs(inputs, params, outputs)
    n = getattr(load_library(), fn)(STYLES[style], STAGES[stage], ctypes.byref(ins),
                                    ctypes.byref(prm), ctypes.byref(outs))
    if n == 0:
        raise ValueError(f"{fn}: the arguments do not validate")
    return int(n)


def atomenc_weight_image_size(style: str, stage: str, inputs: dict, params: dict, outputs: dict) -> int:
    return _size("atomenc_weight_image_size", style, stage, inputs, params, outputs)


def atomenc_prepared_workspace_size(style: str, stage: str, inputs: dict, params: dict,
                                    outputs: dict) -> int:
    return _size("atomenc_prepared_workspace_size", style, stage, inputs, params, outputs)


def atomenc_prepare_weights(style: str, stage: str, inputs: dict, params: dict, outputs: dict,
                            image: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Build the weight image for these weights (allocated with torch unless given)."""
    need = atomenc_weight_image_size(style, stage, inputs, params, outputs)
    if image is None:
        image = torch.empty(need, dtype=torch.uint8, device=inputs["atom"].device)
    ins, prm, outs = _structs(inputs, params, outputs)
    rc = load_library().atomenc_prepare_weights(STYLES[style], STAGES[stage], ctypes.byref(ins),
                                                ctypes.byref(prm), ctypes.byref(outs),
                                                image.data_ptr(), image.numel() * image.element_size(),
                                                _stream_ptr(stream))
    if rc != 0:
        raise AtomencError(rc, "atomenc_prepare_weights")
    return image


def atomenc_forward_prepared(style: str, stage: str, inputs: dict, params: dict,
                             image: torch.Tensor, eps: float, radius: int, outputs: dict,
                             workspace: torch.Tensor, stream=None) -> None:
    ins, prm, outs = _structs(inputs, params, outputs)
    rc = load_library().atomenc_forward_prepared(
        STYLES[style], STAGES[stage], ctypes.byref(ins), ctypes.byref(prm), image.data_ptr(),
        image.numel() * image.element_size(), float(eps), int(radius), ctypes.byref(outs),
        workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if rc != 0:
        raise AtomencError(rc, "atomenc_forward_prepared")


class Forward:
    """atomenc_forward prepared once for a fixed set of tensors: the descriptors are
    built at construction, so each call is a single C call (no per-call marshalling).
    The tensors must stay alive, in place and unchanged in shape while it is used.
    With `image` (from atomenc_prepare_weights) each call is atomenc_forward_prepared:
    the weight conversion is not repeated."""

    def __init__(self, style: str, stage: str, inputs: dict, params: dict, eps: float,
                 radius: int, outputs: dict, workspace: torch.Tensor, stream=None,
                 image: torch.Tensor | None = None):
        self._ins, self._prm, self._outs = _structs(inputs, params, outputs)
        self._keep = (inputs, params, outputs, workspace, image)
        if image is None:
            self._fn = load_library().atomenc_forward
            self._args = (STYLES[style], STAGES[stage], ctypes.byref(self._ins),
                          ctypes.byref(self._prm), float(eps), int(radius), ctypes.byref(self._outs),
                          workspace.data_ptr(), workspace.numel() * workspace.element_size())
        else:
            self._fn = load_library().atomenc_forward_prepared
            self._args = (STYLES[style], STAGES[stage], ctypes.byref(self._ins),
                          ctypes.byref(self._prm), image.data_ptr(),
                          image.numel() * image.element_size(), float(eps), int(radius),
                          ctypes.byref(self._outs), workspace.data_ptr(),
                          workspace.numel() * workspace.element_size())
        self._stream = None if stream is None else _stream_ptr(stream)

    def __call__(self, stream=None) -> None:
        sp = _stream_ptr(stream) if stream is not None else (
            self._stream if self._stream is not None else _stream_ptr(None))
        rc = self._fn(*self._args, sp)
        if rc != 0:
            raise AtomencError(rc, "atomenc_forward")


NOALLOC_SCRATCH_BYTES = 64 << 20


def atomenc_forward_noalloc(style: str, stage: str, inputs: dict, params: dict, eps: float,
                            radius: int, outputs: dict, stream=None) -> None:
    """Forward pass that allocates nothing: the library's own fixed 64 MiB device
    array is its scratch, so no workspace is passed. For callers that may not allocate
    device memory (inside another framework's stream capture, under a host allocator
    that owns all memory, in latency-critical loops). The first call on a device sets
    the array's address up and should come before any stream capture; calls whose GPU
    work overlaps share the array and race, so order them on one stream."""
    ins, prm, outs = _structs(inputs, params, outputs)
    rc = load_library().atomenc_forward_noalloc(STYLES[style], STAGES[stage], ctypes.byref(ins),
                                                ctypes.byref(prm), float(eps), int(radius),
                                                ctypes.byref(outs), _stream_ptr(stream))
    if rc != 0:
        raise AtomencError(rc, "atomenc_forward_noalloc")


NUM_PHASES = 6
PHASES = ["inputs", "conditioning", "projections", "attention", "transition", "boundary"]


def atomenc_forward_profiled(style: str, stage: str, inputs: dict, params: dict, eps: float,
                             radius: int, outputs: dict, workspace: torch.Tensor, events,
                             stream=None) -> int:
    """atomenc_forward that records events[0] before the first launch and events[i+1]
    after phase i (torch.cuda.Event objects, already recorded once so that they
    exist). Returns the number of kernels launched."""
    ins, prm, outs = _structs(inputs, params, outputs)
    handles = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
    n = ctypes.c_int(0)
    rc = load_library().atomenc_forward_profiled(
        STYLES[style], STAGES[stage], ctypes.byref(ins), ctypes.byref(prm), float(eps),
        int(radius), ctypes.byref(outs), workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream_ptr(stream), handles,
        len(events), ctypes.byref(n))
    if rc != 0:
        raise AtomencError(rc, "atomenc_forward_profiled")
    return n.value


KERNEL_KINDS = ["prep", "gemm", "transition", "attention", "rows", "pool"]
MAX_LAUNCHES = 16


def atomenc_forward_traced(style: str, stage: str, inputs: dict, params: dict, eps: float,
                           radius: int, outputs: dict, workspace: torch.Tensor, events,
                           stream=None) -> list:
    """atomenc_forward with an event after every kernel: events[0] is recorded before
    the first launch and events[i+1] after launch i (torch.cuda.Event objects, already
    recorded once; at least MAX_LAUNCHES + 1 of them). Returns the kernel kinds in
    launch order (names from KERNEL_KINDS)."""
    ins, prm, outs = _structs(inputs, params, outputs)
    handles = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
    kinds = (ctypes.c_int * len(events))()
    n = ctypes.c_int(0)
    rc = load_library().atomenc_forward_traced(
        STYLES[style], STAGES[stage], ctypes.byref(ins), ctypes.byref(prm), float(eps),
        int(radius), ctypes.byref(outs), workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream_ptr(stream), handles,
        len(events), kinds, ctypes.byref(n))
    if rc != 0:
        raise AtomencError(rc, "atomenc_forward_traced")
    return [KERNEL_KINDS[kinds[i]] for i in range(n.value)]


STATUS_L2_FALLBACK = 1     # keys gathered from L2 (same results)
STATUS_WAIT_TIMEOUT = 4    # a bounded wait gave up: the pass's outputs are invalid
STATUS_IMAGE_MISMATCH = 8  # a prepared weight image built for other shapes: outputs invalid


class AtomencStatusError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: device status {status:#x}: a bounded wait inside a kernel "
                         "reached its poll limit; the outputs of this pass are invalid")
        self.status = status


def atomenc_noalloc_get_status(stream=None) -> int:
    """Status word of the last atomenc_forward_noalloc pass on the current device."""
    v = ctypes.c_int(0)
    rc = load_library().atomenc_noalloc_get_status(ctypes.byref(v), _stream_ptr(stream))
    if rc != 0:
        raise AtomencError(rc, "atomenc_noalloc_get_status")
    return v.value


def atomenc_debug_peer_wait(poll_limit: int = 0, withhold_flags: bool = False) -> None:
    """Test hook of the paired transition kernel's bounded wait (0, False restores the
    defaults)."""
    load_library().atomenc_debug_peer_wait(int(poll_limit), 1 if withhold_flags else 0)


def atomenc_get_status(workspace: torch.Tensor, stream=None) -> int:
    v = ctypes.c_int(0)
    rc = load_library().atomenc_get_status(workspace.data_ptr(), ctypes.byref(v),
                                           _stream_ptr(stream))
    if rc != 0:
        raise AtomencError(rc, "atomenc_get_status")
    return v.value


def output_shapes(style: str, stage: str, inputs: dict, params: dict) -> dict:
    B, A, C = inputs["atom"].shape
    K = inputs["key_index"].shape[-1]
    T = inputs["token_valid"].shape[-1]
    HD = params["w_q"].shape[-1]
    H = params["w_pair"].shape[-1] if style == "af3" else HD // inputs["rope_cos"].shape[-1]
    shapes = {"hidden": (B, A, C), "attention": (B, H, A, K)}
    if stage == "encoder":
        shapes["token_output"] = (B, T, params["w_pool"].shape[-1])
    else:
        shapes["position_update"] = (B, A, 3)
    return shapes


def windowed_atom_attention(activations: dict, parameters: dict, masks: dict, structure: dict,
                            eps: float = 1e-5, style: str = "af3", stage: str = "decoder",
                            radius: int = -1, workspace: torch.Tensor | None = None,
                            stream=None, check_status: bool = True) -> dict:
    """Forward pass with the page's signature: dicts of CUDA tensors in, a dict out
    (hidden, attention, and token_output for the encoder or position_update for the
    decoder). Allocates the outputs (and the workspace unless one is given) with torch.
    With check_status (the default) it waits for the pass and raises
    AtomencStatusError if a bounded wait inside a kernel gave up (status bit 4), so that
    invalid outputs are never returned silently; check_status=False keeps the call
    asynchronous (read atomenc_get_status yourself)."""
    inputs = {**activations, **masks, **structure}
    dev = activations["atom"].device
    fdt = activations["atom"].dtype
    outputs = {k: torch.empty(s, dtype=fdt, device=dev)
               for k, s in output_shapes(style, stage, inputs, parameters).items()}
    need = atomenc_workspace_size(style, stage, inputs, parameters, outputs)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    atomenc_forward(style, stage, inputs, parameters, eps, radius, outputs, workspace, stream)
    if check_status:
        st = atomenc_get_status(workspace, stream)
        if st & STATUS_WAIT_TIMEOUT:
            raise AtomencStatusError(st, "windowed_atom_attention")
    return outputs


# ---------------------------------------------------------------- single to pair

def _s2p_structs(activations, parameters, masks, outputs):
    ins = AtomencS2PInputs(x=describe(activations.get("x")), mask=describe(masks.get("mask")))
    prm = AtomencS2PParams(**{n: describe(parameters.get(n)) for n in S2P_PARAM_FIELDS})
    outs = AtomencS2POutputs(**{n: describe(outputs.get(n)) for n in S2P_OUTPUT_FIELDS})
    return ins, prm, outs


def single_to_pair(activations: dict, parameters: dict, masks: dict, eps: float = 1e-5,
                   output_norm: bool = False, workspace: torch.Tensor | None = None,
                   stream=None):
    """Page "ESMFold Single-to-Pair Features" (esmfold_single_to_pair) on the GPU: dicts
    of CUDA tensors in (x; mask; weight, bias, norm_scale, norm_bias, out_weight,
    out_bias, output_scale/output_bias), (pair_features [B,N,N,2H], output [B,N,N,D])
    out. Allocates the outputs (and the workspace unless one is given) with torch."""
    x = activations["x"]
    B, N, _ = x.shape
    H2 = parameters["weight"].shape[1]
    Dp = parameters["out_weight"].shape[1]
    outputs = {"pair_features": torch.empty(B, N, N, H2, dtype=x.dtype, device=x.device),
               "output": torch.empty(B, N, N, Dp, dtype=x.dtype, device=x.device)}
    ins, prm, outs = _s2p_structs(activations, parameters, masks, outputs)
    lib = load_library()
    need = lib.atomenc_s2p_workspace_size(ctypes.byref(ins), ctypes.byref(prm),
                                          1 if output_norm else 0, ctypes.byref(outs))
    if need == 0:
        raise ValueError("atomenc_s2p_workspace_size: the arguments do not validate")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    rc = lib.atomenc_single_to_pair(ctypes.byref(ins), ctypes.byref(prm), float(eps),
                                    1 if output_norm else 0, ctypes.byref(outs),
                                    workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                    _stream_ptr(stream))
    if rc != 0:
        raise AtomencError(rc, "atomenc_single_to_pair")
    return outputs["pair_features"], outputs["output"]


# ---------------------------------------------------------------- attention core gradient

def attention_backward(core: dict, heads: int, d_out: torch.Tensor, d_attention=None,
                       eps: float = 1e-5, style: str = "af3", radius: int = -1,
                       workspace: torch.Tensor | None = None, stream=None) -> dict:
    """Gradient of the slot-gathered attention core on the GPU. core holds CUDA tensors
    q, k, v, g [B,A,H*D], key_index [B,A,K] int64, window_mask [B,A,K] bool, usable [B,A]
    bool and, for AF3, pair [B,A,K,P], pair_scale [P], w_pair [P,H]. Returns d_q, d_k,
    d_v, d_g (and d_pair, d_pair_scale, d_w_pair for AF3), allocated with torch."""
    q = core["q"]
    outs = {n: torch.empty_like(q) for n in ("d_q", "d_k", "d_v", "d_g")}
    if style == "af3":
        outs["d_pair"] = torch.empty_like(core["pair"])
        outs["d_pair_scale"] = torch.empty_like(core["pair_scale"])
        outs["d_w_pair"] = torch.empty_like(core["w_pair"])
    src = {**core, "d_out": d_out, "d_attention": d_attention}
    ins = AtomencCoreBwdInputs(**{n: describe(src.get(n)) for n in CORE_BWD_INPUT_FIELDS})
    out = AtomencCoreBwdOutputs(**{n: describe(outs.get(n)) for n in CORE_BWD_OUTPUT_FIELDS})
    lib = load_library()
    need = lib.atomenc_attention_backward_workspace_size(STYLES[style], ctypes.byref(ins), int(heads),
                                                         ctypes.byref(out))
    if need == 0:
        raise ValueError("atomenc_attention_backward_workspace_size: the arguments do not validate")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    rc = lib.atomenc_attention_backward(STYLES[style], ctypes.byref(ins), int(heads), float(eps),
                                        int(radius), ctypes.byref(out), workspace.data_ptr(),
                                        workspace.numel() * workspace.element_size(),
                                        _stream_ptr(stream))
    if rc != 0:
        raise AtomencError(rc, "atomenc_attention_backward")
    return outs
