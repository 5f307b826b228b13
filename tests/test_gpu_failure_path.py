"""The failure path of the attention kernel, exercised without faulting or hanging the GPU.

Every wait of the kernel is bounded; a wait that runs out records SAGESLA_ERR_TIMEOUT in the
workspace's status word, sets the CTA's abort flag so that the other roles leave their loops,
and the kernel returns. The test hooks of sagesla_options shorten the limit to a few
milliseconds and make the first CTA skip one tile load (its bytes are never announced, so
nothing is left in flight): the waits for that tile then run out. The call must return, the
status must read TIMEOUT, and a normal call on the same workspace right afterwards must be
correct."""
import time

import pytest
import torch

import sparse_bit_attention_b200 as sba
from sparse_bit_attention_b200 import inputs
from _parity import OUT_TOL, compare_head, gpu_run

pytestmark = pytest.mark.gpu

TIMEOUT = 5   # SAGESLA_ERR_TIMEOUT


@pytest.mark.parametrize("ratio", [0.1, 1.0])
def test_skipped_tile_times_out_and_the_next_call_is_clean(ratio):
    """Ratio 0.1 runs the sparse attention kernel, ratio 1 the dense-mode kernel."""
    q, k, v = (x.cuda() for x in inputs.make_random(1, 2, 2048, 61, k_offset_std=1.0))
    B, H, N, D = q.shape
    ws = sba.alloc_workspace(sba.sagesla_workspace_size(B, H, N, D, ratio))
    out = torch.zeros(q.shape, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    sba.sagesla_forward(q, k, v, ratio, out=out, workspace=ws, debug_spin_limit_us=10000,
                        debug_skip_tile=True)
    status = sba.sagesla_stream_status(None, ws)
    elapsed = time.perf_counter() - t0
    assert status == TIMEOUT, sba.sagesla_status_string(status)
    assert elapsed < 5.0, elapsed               # bounded: a few 10 ms limits, not the 2 s one
    # the CTAs that were not starved wrote their rows: all but the first two query blocks of
    # head 0 (the starved CTA's), whose rows may be left unwritten
    ref = gpu_run(q.cpu(), k.cpu(), v.cpu(), ratio, extras=False)["out"]
    got = out.cpu()
    assert torch.equal(got[:, 0, 128:], ref[:, 0, 128:])
    assert torch.equal(got[:, 1], ref[:, 1])
    # the same workspace, normal call: status clean, output equal to a fresh workspace's
    out2 = sba.sagesla_forward(q, k, v, ratio, workspace=ws)
    assert sba.sagesla_stream_status(None, ws) == 0
    assert torch.equal(out2.cpu(), ref)


def test_short_limit_without_a_fault_completes_normally():
    """A 10 ms limit does not trip on a normal call (every wait ends within microseconds), and
    the result is the ordinary one."""
    q, k, v = inputs.make_random(1, 2, 1500, 62, k_offset_std=1.0)
    res = gpu_run(q, k, v, 0.2)
    out = sba.sagesla_forward(q.cuda(), k.cuda(), v.cuda(), 0.2, workspace=res["ws"],
                              debug_spin_limit_us=10000)
    assert sba.sagesla_stream_status(None, res["ws"]) == 0
    assert torch.equal(out.cpu(), res["out"])
    for h in range(2):
        err, _ = compare_head(q, k, v, 0.2, res, 0, h)
        assert err <= OUT_TOL, err
