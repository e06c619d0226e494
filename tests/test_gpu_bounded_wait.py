"""Failure detection without a GPU fault: a bounded wait inside a kernel that runs out
returns an error status the host reads, and the context stays usable.

The paired transition kernel (two CTAs per 128-row block when row blocks are few)
exchanges w_ff_out partials between the two CTAs of a cluster through flags in global
memory, each poll loop bounded. The test hook makes every CTA withhold its flag (a
flag that nothing sets) with a small poll limit: the pass must return, set status
bit 4 (outputs invalid), and the page-signature call must raise instead of returning
the invalid outputs. With the hook cleared, the next pass on the same context is
clean and matches the oracle."""
import pytest
import torch

from sparse_windowed_atom_b200 import atomenc, workloads
from tests.cuda_harness import compare, exact_zero_pattern, run_oracle, to_torch

pytestmark = pytest.mark.gpu


def test_peer_wait_that_runs_out_sets_the_status_and_the_next_pass_is_clean():
    # 600 rows = 5 row blocks: the paired transition mode
    w = workloads.make_inputs(workloads.tiny_spec("esmfold2", "encoder", A=300), seed=41)
    spec = w["spec"]
    act, prm, msk, st = to_torch(w)
    inputs = {**act, **msk, **st}
    outs = {k: torch.empty(s, device="cuda") for k, s in
            atomenc.output_shapes(spec.style, spec.stage, inputs, prm).items()}
    ws = torch.empty(atomenc.atomenc_workspace_size(spec.style, spec.stage, inputs, prm, outs),
                     dtype=torch.uint8, device="cuda")
    try:
        atomenc.atomenc_debug_peer_wait(poll_limit=2000, withhold_flags=True)
        atomenc.atomenc_forward(spec.style, spec.stage, inputs, prm, spec.eps, spec.radius, outs, ws)
        torch.cuda.synchronize()
        assert atomenc.atomenc_get_status(ws) & atomenc.STATUS_WAIT_TIMEOUT
        with pytest.raises(atomenc.AtomencStatusError):
            atomenc.windowed_atom_attention(act, prm, msk, st, eps=spec.eps, style=spec.style,
                                            stage=spec.stage, radius=spec.radius)
    finally:
        atomenc.atomenc_debug_peer_wait(0, False)
    # same context, hook cleared: a clean pass with correct results
    atomenc.atomenc_forward(spec.style, spec.stage, inputs, prm, spec.eps, spec.radius, outs, ws)
    torch.cuda.synchronize()
    assert atomenc.atomenc_get_status(ws) & atomenc.STATUS_WAIT_TIMEOUT == 0
    got = {k: v.double().cpu().numpy() for k, v in outs.items()}
    ref = run_oracle(w)
    compare(got, ref, spec.dtype, "after the hook")
    exact_zero_pattern(got, ref)
