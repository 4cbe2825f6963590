"""dcn4_backward_noalloc (the backward for callers that cannot allocate
device memory, e.g. inside allocation-free host hooks or plugins whose
framework owns all device memory) against dcn4_backward, called through the
C ABI twice in a row: the second call must not see the first call's
leftovers in the library's shared scratch array."""
import ctypes

import numpy as np
import pytest
import torch

from deformable_convolution_dcn4_b200 import _binding as B
from deformable_convolution_dcn4_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL = 2e-2  # the bf16 gate of the parity tests (scaled max error)


def _scaled(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


def _call_noalloc(lib, desc, d, gin, gow):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.dcn4_backward_noalloc(ctypes.byref(desc), ctypes.c_void_p(d["input"].data_ptr()),
                                   ctypes.c_void_p(d["offset_weight"].data_ptr()),
                                   ctypes.c_void_p(d["grad_out"].data_ptr()),
                                   ctypes.c_void_p(gin.data_ptr()),
                                   ctypes.c_void_p(gow.data_ptr()), stream)
    torch.cuda.synchronize()
    return rc


def test_noalloc_backward_matches_backward_twice_in_a_row():
    lib = B.load()
    # N*H*W*C = 4,194,304 fp32 scratch values = 16 MiB, inside the 32 MiB array
    wl = WORKLOADS["highres_bf16"].replace(N=1)
    d = make_inputs(wl, (wl.H, wl.W), with_grad=True, device="cuda")
    # fp32-weight mode: the mode in which the backward accumulates grad_input
    # in the fp32 scratch (the default 16-bit mode adds into grad_input)
    desc = B.make_desc(wl.N, wl.H, wl.W, wl.C, wl.G, torch.bfloat16, math="f32")
    ref_in, ref_ow = B.dcn4_backward(d["input"], d["offset_weight"], d["grad_out"], group=wl.G,
                                     math="f32")
    torch.cuda.synchronize()
    for call in range(2):
        gin = torch.full_like(d["input"], float("nan"))
        gow = torch.full_like(d["offset_weight"], float("nan"))
        assert _call_noalloc(lib, desc, d, gin, gow) == 0, f"call {call}"
        assert _scaled(gin, ref_in) <= TOL, f"grad_input, call {call}"
        assert _scaled(gow, ref_ow) <= TOL, f"grad_offset_weight, call {call}"
    rc, bits = B.dcn4_last_device_error()
    assert rc == 0 and bits == 0


def test_noalloc_rejects_sizes_beyond_the_scratch():
    lib = B.load()
    # 8 x 128 x 128 x 256 values need 128 MiB of fp32 scratch > 32 MiB
    desc = B.make_desc(8, 128, 128, 256, 16, torch.bfloat16)
    one = ctypes.c_void_p(256)
    rc = lib.dcn4_backward_noalloc(ctypes.byref(desc), one, one, one, one, one,
                                   ctypes.c_void_p(0))
    assert rc == 3  # DCN4_ERR_WORKSPACE, nothing launched
