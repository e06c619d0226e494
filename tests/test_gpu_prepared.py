"""Prepared weights (atomenc_prepare_weights / atomenc_forward_prepared): the weight
images built once give the same outputs, bit for bit, as the plain forward that builds
them on every call; an image built for other shapes is refused on the device (status
bit 8) instead of being read; short or unaligned images are refused on the host."""
import numpy as np
import pytest
import torch

from sparse_windowed_atom_b200 import atomenc, workloads

pytestmark = pytest.mark.gpu
CASES = [("af3", "encoder", "float32"), ("af3", "decoder", "bfloat16"),
         ("esmfold2", "encoder", "bfloat16"), ("esmfold2", "decoder", "float32")]


def _case(style, stage, dtype, seed=5, **kw):
    spec = workloads.tiny_spec(style, stage, dtype, A=400, T=50, **kw)
    w = workloads.make_inputs(spec, seed=seed)
    fdt = torch.bfloat16 if dtype == "bfloat16" else torch.float32
    t = lambda a, d=None: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dtype=d)
    inputs = {**{k: t(v, fdt) for k, v in w["activations"].items()},
              **{k: t(v) for k, v in w["masks"].items()},
              **{k: t(v) for k, v in w["structure"].items()}}
    params = {k: t(v, fdt) for k, v in w["parameters"].items()}
    shapes = atomenc.output_shapes(style, stage, inputs, params)
    outs = lambda: {k: torch.full(s, float("nan"), dtype=fdt, device="cuda") for k, s in shapes.items()}
    return spec, inputs, params, outs


@pytest.mark.parametrize("style,stage,dtype", CASES)
def test_prepared_forward_equals_the_plain_forward(style, stage, dtype):
    spec, inputs, params, outs = _case(style, stage, dtype)
    ref = outs()
    ws = torch.empty(atomenc.atomenc_workspace_size(style, stage, inputs, params, ref),
                     dtype=torch.uint8, device="cuda")
    atomenc.atomenc_forward(style, stage, inputs, params, spec.eps, spec.radius, ref, ws)
    got = outs()
    image = atomenc.atomenc_prepare_weights(style, stage, inputs, params, got)
    wsp_bytes = atomenc.atomenc_prepared_workspace_size(style, stage, inputs, params, got)
    assert wsp_bytes < ws.numel()
    wsp = torch.empty(wsp_bytes, dtype=torch.uint8, device="cuda")
    # the weights' own tensors may change after preparation: the image keeps what it was
    # built from
    saved = {k: v.clone() for k, v in params.items()}
    for v in params.values():
        v.mul_(3.0)
    for call in range(2):
        atomenc.atomenc_forward_prepared(style, stage, inputs, params, image, spec.eps,
                                         spec.radius, got, wsp)
        torch.cuda.synchronize()
        assert atomenc.atomenc_get_status(wsp) == 0
        for k in ref:
            assert torch.equal(got[k], ref[k]), (call, k)
    for k, v in saved.items():
        params[k].copy_(v)


def test_an_image_for_other_shapes_sets_status_bit_8():
    spec, inputs, params, outs = _case("af3", "encoder", "float32")
    spec2, inputs2, params2, outs2 = _case("af3", "encoder", "float32", U=256)
    image = atomenc.atomenc_prepare_weights("af3", "encoder", inputs2, params2, outs2())
    o = outs()
    ws = torch.empty(atomenc.atomenc_prepared_workspace_size("af3", "encoder", inputs, params, o),
                     dtype=torch.uint8, device="cuda")
    need = atomenc.atomenc_weight_image_size("af3", "encoder", inputs, params, o)
    big = torch.zeros(max(need, image.numel()), dtype=torch.uint8, device="cuda")
    big[:image.numel()] = image
    atomenc.atomenc_forward_prepared("af3", "encoder", inputs, params, big, spec.eps,
                                     spec.radius, o, ws)
    torch.cuda.synchronize()
    assert atomenc.atomenc_get_status(ws) & atomenc.STATUS_IMAGE_MISMATCH
    # an image of the right shapes clears it again
    good = atomenc.atomenc_prepare_weights("af3", "encoder", inputs, params, o)
    atomenc.atomenc_forward_prepared("af3", "encoder", inputs, params, good, spec.eps,
                                     spec.radius, o, ws)
    torch.cuda.synchronize()
    assert atomenc.atomenc_get_status(ws) == 0


def test_short_or_unaligned_images_are_refused_on_the_host():
    spec, inputs, params, outs = _case("esmfold2", "encoder", "bfloat16")
    o = outs()
    need = atomenc.atomenc_weight_image_size("esmfold2", "encoder", inputs, params, o)
    with pytest.raises(atomenc.AtomencError):
        atomenc.atomenc_prepare_weights("esmfold2", "encoder", inputs, params, o,
                                        image=torch.empty(need - 16, dtype=torch.uint8, device="cuda"))
    raw = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
    with pytest.raises(atomenc.AtomencError):
        atomenc.atomenc_prepare_weights("esmfold2", "encoder", inputs, params, o, image=raw[16:16 + need])
    ws = torch.empty(atomenc.atomenc_prepared_workspace_size("esmfold2", "encoder", inputs, params, o),
                     dtype=torch.uint8, device="cuda")
    with pytest.raises(atomenc.AtomencError):
        atomenc.atomenc_forward_prepared("esmfold2", "encoder", inputs, params,
                                         torch.empty(need - 16, dtype=torch.uint8, device="cuda"),
                                         spec.eps, spec.radius, o, ws)
