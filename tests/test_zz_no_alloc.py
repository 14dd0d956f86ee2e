"""hsa_decode_noalloc, the decode entry point for callers that cannot allocate device memory while
they decode (an engine whose KV-cache pool owns all of HBM, a C caller for whom cudaMalloc/cudaFree
per step would synchronise the device). Its scratch is a fixed array inside the library instead of
a caller workspace. The test calls it through the C ABI twice in a row, with different shapes (the
smaller call first, then the larger, and the other way round, so that a call after a larger one shows
it ignores what that call left in the shared array), and checks each result against hsa_decode on the
same inputs; it also calls it with no selection outputs (the selection then lives in the array), and
checks that a call needing more scratch than the array holds is refused on the host.

This file is collected last on purpose: if it fails, a run that stops at the first failure has
already run every other test.
"""
import ctypes

import pytest
import torch

from ultra_long_context_b200 import hsa, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"
OUT_MAX_ABS = 2e-2      # the output tolerance of the parity tests
W_MAX_ABS = 1e-3


SMALL = dict(B=4, H=4, D=128, Tmax=64 * 3000, lens=[64 * 3000, 64 * 1500 + 9, 100, 64 * 2999], topk=16, seed=71)
LARGE = dict(B=2, H=8, D=64, Tmax=64 * 5000 + 17, lens=[64 * 5000 + 17, 64 * 4000], topk=32, seed=72)


@pytest.mark.parametrize("first,second", [(SMALL, LARGE), (LARGE, SMALL)])
def test_noalloc_decode_matches_workspace_decode_twice_in_a_row(first, second):
    for case in (first, second):
        q, Kc, Vc, Lc, lens, _ = inputs.decode_inputs(case["B"], case["H"], case["lens"], case["D"],
                                                      seed=case["seed"], Tmax=case["Tmax"], device=DEV)
        ref_out, ref_idx, ref_w = hsa.hsa_decode(q, Kc, Vc, Lc, lens, case["topk"])
        out, idx, w = hsa.hsa_decode_noalloc(q, Kc, Vc, Lc, lens, case["topk"])
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert (w - ref_w).abs().max().item() <= W_MAX_ABS
        assert (out.float() - ref_out.float()).abs().max().item() <= OUT_MAX_ABS


def test_noalloc_decode_refuses_calls_beyond_its_scratch():
    B, H, D, Tmax, topk = 64, 64, 128, 64, 64    # partial outputs alone need 64*64*64*128*4 bytes
    q, Kc, Vc, Lc, lens, _ = inputs.decode_inputs(B, H, Tmax, D, seed=73, needle=False, device=DEV)
    with pytest.raises(hsa.HSAError, match="HSA_ERR_UNSUPPORTED.*scratch"):
        hsa.hsa_decode_noalloc(q, Kc, Vc, Lc, lens, topk)


def test_noalloc_decode_without_selection_outputs():
    """NULL sel_idx and sel_w: the selection is kept inside the fixed array; out still matches hsa_decode."""
    c = SMALL
    q, Kc, Vc, Lc, lens, _ = inputs.decode_inputs(c["B"], c["H"], c["lens"], c["D"], seed=c["seed"] + 10,
                                                  Tmax=c["Tmax"], device=DEV)
    ref_out, _, _ = hsa.hsa_decode(q, Kc, Vc, Lc, lens, c["topk"])
    for _ in range(2):
        out = torch.empty_like(q)
        st = hsa.lib().hsa_decode_noalloc(hsa._ptr(q), hsa._ptr(Kc), hsa._ptr(Vc), hsa._ptr(Lc), hsa._ptr(lens),
                                          c["Tmax"], c["B"], c["H"], c["D"], 64, c["topk"], 0.0, hsa._ptr(out), None,
                                          None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, hsa.hsa_last_error()
        torch.cuda.synchronize()
        assert (out.float() - ref_out.float()).abs().max().item() <= OUT_MAX_ABS
