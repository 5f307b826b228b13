"""Host-side checks of the debugging aids (no GPU): the bounds-checking build loads and exports
the same ABI, the workspace plan leaves a 16-byte canary gap after every region, and the
debug options are validated before anything launches."""
import ctypes

import pytest

import sparse_bit_attention_b200 as sba
from sparse_bit_attention_b200 import binding
from sparse_bit_attention_b200.build import build

from test_abi import _header_functions


@pytest.fixture(scope="module", autouse=True)
def built_libraries():
    build()
    build(checks=True)


def test_checking_build_exports_the_same_abi():
    lib = binding.load_checks_library()
    for name in _header_functions():
        assert hasattr(lib, name), name
    assert lib.sagesla_build_checks() == 1
    assert binding.load_library().sagesla_build_checks() == 0


def _region_sizes(B, H, N, r):
    """Bytes of each workspace region, from the shapes include/sagesla.h documents."""
    nb = (N + 63) // 64
    k = sba.sagesla_topk_count(N, r)
    BH = B * H
    n_pairs = (nb + 1) // 2
    n_pad, nbq = 128 * n_pairs, 2 * n_pairs
    ld = (nb + 3) // 4 * 4
    mw = (nb + 31) // 32
    nbk, nbm = (nb + 63) // 64 * 64, (nb + 127) // 128 * 128
    return {
        "status": 4, "q8": BH * n_pad * 128, "k8": BH * n_pad * 128, "v8": BH * n_pad * 128,
        "sq": BH * nbq * 4, "sk": BH * nbq * 4, "s_v": BH * 512, "inv_v": BH * 512,
        "mu": BH * 512, "qbar": BH * nb * 512, "kbar": BH * nb * 512,
        "ksum_part": BH * nb * 1024, "vmax_part": BH * nb * 512, "scores": BH * nb * ld * 4,
        "kept": BH * nb * k * 4, "mask": BH * nb * mw * 4, "amask": BH * nbm * nbk * 2,
        "hflat": BH * nbk * 129 * 128 * 2, "gsum": BH * nbm * 129 * 128 * 2,
    }


@pytest.mark.parametrize("shape", [(1, 2, 1024, 0.1), (1, 3, 1000, 0.25), (2, 1, 65, 1.0),
                                   (1, 40, 75600, 0.1), (1, 1, 1, 0.5)])
def test_every_region_is_followed_by_a_canary_gap(shape):
    lay = sba.sagesla_get_workspace_layout(*shape[:3], 128, shape[3])
    sizes = _region_sizes(*shape)
    order = sorted(sizes, key=lambda f: lay[f])
    ends = [lay[f] for f in order[1:]] + [lay["total_bytes"]]
    for f, nxt in zip(order, ends):
        canary = (lay[f] + sizes[f] + 15) // 16 * 16
        assert canary + 16 <= nxt, (f, lay[f], sizes[f], nxt)


def _layout_status(opt):
    lay = binding.SageslaWorkspaceLayout()
    return binding.load_library().sagesla_get_workspace_layout_ex(
        1, 2, 1000, 128, 0.1, 64, ctypes.byref(opt), ctypes.byref(lay))


def test_debug_options_are_validated():
    opt = binding._options()
    assert opt.debug_checks == 0 and opt.debug_plant == 0
    assert _layout_status(opt) == 0
    opt.debug_checks = 1
    assert _layout_status(opt) == 0
    opt.debug_plant = 1
    assert _layout_status(opt) == 0
    opt.debug_checks = 2
    assert _layout_status(opt) == 1                 # INVALID_ARG
    opt.debug_checks = 0
    assert _layout_status(opt) == 1                 # plant 1 needs the canaries
    opt.debug_plant = 3
    assert _layout_status(opt) == 1
    opt.debug_plant = -1
    assert _layout_status(opt) == 1
    opt.debug_plant = 2                             # only the checking build accepts it
    assert _layout_status(opt) == 2                 # UNSUPPORTED
    with binding.using_library(binding.load_checks_library()):
        assert _layout_status(opt) == 0
    assert binding.load_library() is not binding.load_checks_library()
