"""The debugging aids on the GPU, exercised without faulting or hanging it.

- Workspace canaries (debug_checks): a normal call with them leaves the status word clean and
  the output bit-identical; a canary damaged on purpose by the host (debug_plant = 1) is
  reported as SAGESLA_ERR_CANARY, and the next call on the same workspace is clean.
- The bounds-checking build (libsagesla_checks.so): the same results as the normal build,
  bit for bit (forward in every operand mode, dense mode, backward); an out-of-range kept-list
  entry planted by the host (debug_plant = 2) is caught before any load uses it: the call
  ends with SAGESLA_ERR_BOUNDS, the rows of the CTAs that did not read it are the normal
  ones, and the next call on the same workspace is clean."""
import pytest
import torch

import sparse_bit_attention_b200 as sba
from sparse_bit_attention_b200 import binding, inputs
from sparse_bit_attention_b200.build import build

pytestmark = pytest.mark.gpu

BOUNDS, CANARY = 8, 9

CASES = [((1, 2, 1000, 11), 0.1), ((1, 2, 1088, 12), 0.25), ((2, 1, 1025, 13), 1.0)]


@pytest.fixture(scope="module")
def checks_lib():
    build(checks=True)
    return binding.load_checks_library()


def _inputs(shape):
    B, H, N, seed = shape
    return [x.cuda() for x in inputs.make_random(B, H, N, seed, k_offset_std=1.0)]


def _forward(q, k, v, ratio, ws, **kw):
    out = sba.sagesla_forward(q, k, v, ratio, workspace=ws, **kw)
    return out, sba.sagesla_stream_status(None, ws)


def _workspace(q, ratio, **mode):
    B, H, N, D = q.shape
    return sba.alloc_workspace(sba.sagesla_workspace_size(B, H, N, D, ratio, **mode))


@pytest.mark.parametrize("shape,ratio", CASES)
@pytest.mark.parametrize("mode", [(True, True), (True, False), (False, False)])
def test_canaries_stay_intact_and_change_nothing(shape, ratio, mode):
    q, k, v = _inputs(shape)
    quant, pv_fp8 = mode
    ws = _workspace(q, ratio, quant=quant, pv_fp8=pv_fp8)
    ref, st = _forward(q, k, v, ratio, ws, quant=quant, pv_fp8=pv_fp8)
    assert st == 0
    out, st = _forward(q, k, v, ratio, ws, quant=quant, pv_fp8=pv_fp8, debug_checks=True)
    assert st == 0, sba.sagesla_status_string(st)
    assert torch.equal(out, ref)


def test_damaged_canary_is_reported_and_the_next_call_is_clean():
    q, k, v = _inputs((1, 2, 1000, 21))
    ws = _workspace(q, 0.1)
    ref, st = _forward(q, k, v, 0.1, ws)
    assert st == 0
    out, st = _forward(q, k, v, 0.1, ws, debug_checks=True, debug_plant=1)
    assert st == CANARY, sba.sagesla_status_string(st)
    assert torch.equal(out, ref)              # the damage is in a gap, not in any result
    out, st = _forward(q, k, v, 0.1, ws, debug_checks=True)
    assert st == 0 and torch.equal(out, ref)


@pytest.mark.parametrize("shape,ratio", CASES)
@pytest.mark.parametrize("mode", [(True, True), (False, False)])
def test_checking_build_gives_the_same_results(checks_lib, shape, ratio, mode):
    q, k, v = _inputs(shape)
    quant, pv_fp8 = mode
    ws = _workspace(q, ratio, quant=quant, pv_fp8=pv_fp8)
    ref, st = _forward(q, k, v, ratio, ws, quant=quant, pv_fp8=pv_fp8)
    assert st == 0
    with binding.using_library(checks_lib):
        out, st = _forward(q, k, v, ratio, ws, quant=quant, pv_fp8=pv_fp8, debug_checks=True)
    assert st == 0, sba.sagesla_status_string(st)
    assert torch.equal(out, ref)


def test_checking_build_backward_matches(checks_lib):
    q, k, v = _inputs((1, 2, 1000, 31))
    d_out = torch.randn(q.shape, generator=torch.Generator().manual_seed(3)).to(
        torch.bfloat16).cuda()

    def grads():
        B, H, N, D = q.shape
        ws = sba.alloc_workspace(sba.sagesla_sla_backward_workspace_size(B, H, N, D, 0.2))
        g = [torch.empty(q.shape, dtype=torch.float32, device="cuda") for _ in range(3)]
        sba.sagesla_sla_backward(q, k, v, d_out, 0.2, dq=g[0], dk=g[1], dv=g[2], workspace=ws)
        assert sba.sagesla_stream_status(None, ws) == 0
        return g

    ref = grads()
    with binding.using_library(checks_lib):
        got = grads()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_planted_kept_index_is_caught_by_the_checking_build(checks_lib):
    q, k, v = _inputs((1, 2, 2048, 41))
    ws = _workspace(q, 0.1)
    ref, st = _forward(q, k, v, 0.1, ws)
    assert st == 0
    out = torch.zeros(q.shape, dtype=torch.float32, device="cuda")
    with binding.using_library(checks_lib):
        sba.sagesla_forward(q, k, v, 0.1, out=out, workspace=ws, debug_plant=2,
                            debug_spin_limit_us=10000)
        st = sba.sagesla_stream_status(None, ws)
        assert st == BOUNDS, sba.sagesla_status_string(st)
        # the first kept entry belongs to query block 0 of head 0: only its CTA (query blocks
        # 0 and 1) stops; every other row is the normal one
        assert torch.equal(out[:, 0, 128:], ref[:, 0, 128:])
        assert torch.equal(out[:, 1], ref[:, 1])
        again, st = _forward(q, k, v, 0.1, ws)
        assert st == 0 and torch.equal(again, ref)
