"""awq_score_grid_static_scratch: AWQ candidate scoring with the library's
fixed device scratch instead of a caller-supplied workspace.  It is checked
against the workspace entry point awq_score_grid on the same inputs; that
entry point is itself checked against the oracle in test_gpu_parity.py.

The file is named to be collected last, so the GPU case runs both after the
rest of the suite and, with the file alone, in a fresh process."""
import ctypes
import os

import numpy as np
import pytest

import weight_only_int4_quantize_b200 as w4
from weight_only_int4_quantize_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SCRATCH_BYTES = 32 << 20   # W4_AWQ_STATIC_SCRATCH_BYTES in include/w4.h
A = 0x10000                # aligned fake device addresses: validation touches no device
B = 0x20000


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(w4.LIB_PATH):
        from weight_only_int4_quantize_b200 import build
        build.build()
    return w4.lib()


def test_header_limit_matches():
    src = open(os.path.join(ROOT, "include", "w4.h")).read()
    assert "#define W4_AWQ_STATIC_SCRATCH_BYTES (32u << 20)" in src


def test_refuses_problems_over_the_limit(L):
    """A problem whose workspace exceeds the static scratch is refused with
    W4_ERR_WORKSPACE and a message naming both sizes, before any device call."""
    al = (ctypes.c_float * 20)(*synth.alpha_grid(20))
    sh = (ctypes.c_float * 10)(*synth.shrink_grid(10))
    m, n, k = 2048, 2048, 2048
    need = L.w4_awq_workspace_bytes(m, n, k, 20, 10, 1)
    assert need > SCRATCH_BYTES
    st = L.awq_score_grid_static_scratch(A, m, B, n, k, 128, 0, al, 20, sh, 10, None, 1,
                                         A, B, None)
    assert st == 5
    msg = L.w4_last_error().decode()
    assert str(need) in msg and str(SCRATCH_BYTES) in msg
    # earlier argument errors keep their own status
    assert L.awq_score_grid_static_scratch(A, m, B, n, k, 64, 0, al, 20, sh, 10, None, 1,
                                           A, B, None) == 4
    assert L.awq_score_grid_static_scratch(None, m, B, n, k, 128, 0, al, 20, sh, 10, None, 1,
                                           A, B, None) == 1


@pytest.mark.gpu
@pytest.mark.parametrize("sym,seg", [(False, None), (True, [0, 256, 528, 800])])
def test_matches_workspace_entry_point_twice(sym, seg):
    import torch
    dev = "cuda:0"
    x = synth.student_t_calibration(200, 640, seed=71).to(dev)        # ragged M
    w = synth.normal_weight(800, 640, 0.02, seed=72, n_outliers=4, outlier_scale=20.0).to(dev)
    alphas, shrinks = synth.alpha_grid(20), synth.shrink_grid(10)
    n_seg = 1 if seg is None else len(seg) - 1
    assert w4.awq_workspace_bytes(200, 800, 640, 20, 10, n_seg) <= SCRATCH_BYTES
    ref_sse, ref_arg = w4.awq_score_grid(x, w, alphas, shrinks, sym, seg_offsets=seg)
    ref_sse, ref_arg = ref_sse.cpu().numpy(), ref_arg.cpu().numpy()

    sse = torch.empty((n_seg, 20, 10), dtype=torch.float64, device=dev)
    arg = torch.empty((n_seg + 1, 4), dtype=torch.int32, device=dev)
    for call in range(2):
        sse.fill_(-1.0)
        arg.fill_(-7)
        torch.cuda.synchronize()
        if call == 1:
            free_before = torch.cuda.mem_get_info()[0]
        w4.awq_score_grid_static_scratch(x, w, alphas, shrinks, sym, seg_offsets=seg,
                                         sse_out=sse, argmin_out=arg)
        torch.cuda.synchronize()
        if call == 1:
            # after the first call's set-up, a call takes no device memory
            assert torch.cuda.mem_get_info()[0] == free_before
        got, got_arg = sse.cpu().numpy(), arg.cpu().numpy()
        # The same kernels in the same fixed reduction order as awq_score_grid:
        # the SSE table is bit-identical, not merely within the scorer's error.
        assert np.array_equal(got.view(np.uint64), ref_sse.view(np.uint64)), \
            f"call {call}: SSE differs (max relative {np.max(np.abs(got - ref_sse) / ref_sse):.3e})"
        assert np.array_equal(got_arg, ref_arg), f"call {call}: argmins differ"
    assert w4.device_error(clear=True) == 0
