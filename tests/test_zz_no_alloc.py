"""dcn4_backward_noalloc: the backward for callers that cannot allocate device
memory (allocation-free host hooks, plugins whose framework owns all device
memory, real-time code that cannot take cudaMalloc's implicit
synchronisation). It runs dcn4_backward with the fp32 scratch taken from a
fixed array inside the library, so these tests call it through the C ABI
and check that:
  * it matches dcn4_backward (same math mode) and the CPU oracle on a sampled
    image, on two calls in a row (the second call must not see the first
    call's leftovers in the shared array), for bf16 and fp16 and both math
    modes;
  * a large call followed by a smaller one on the same stream is still right
    (each call clears the part of the array it uses);
  * fp32 calls, which need no scratch, take the direct path;
  * calls beyond the array's size are refused before anything launches.
This file is collected last so that a failure here cannot hide another."""
import ctypes

import pytest
import torch

from deformable_convolution_dcn4_b200 import _binding as B
from deformable_convolution_dcn4_b200.workloads import DTYPES, WORKLOADS, make_inputs

from parity_util import TOL, f32, problem, scaled_err

pytestmark = pytest.mark.gpu


def _call_noalloc(desc, d, gin, gow):
    lib = B.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.dcn4_backward_noalloc(ctypes.byref(desc), ctypes.c_void_p(d["input"].data_ptr()),
                                   ctypes.c_void_p(d["offset_weight"].data_ptr()),
                                   ctypes.c_void_p(d["grad_out"].data_ptr()),
                                   ctypes.c_void_p(gin.data_ptr()),
                                   ctypes.c_void_p(gow.data_ptr()), stream)
    return rc


def _case(wl):
    d = make_inputs(wl, (wl.H, wl.W), with_grad=True, device="cuda")
    desc_kw = dict(kernel_size=(wl.kh, wl.kw), stride=wl.stride, pad=wl.pad,
                   dilation=wl.dilation, offset_scale=wl.offset_scale)
    return d, desc_kw


def _oracle_image(orc, wl, d, n):
    """Oracle grad_input and grad_offset_weight of image n alone."""
    prob = problem(orc, wl, 1)
    return orc.backward(prob, f32(d["input"][n:n + 1]), f32(d["offset_weight"][n:n + 1]),
                        f32(d["grad_out"][n:n + 1]))


def _check_twice(orc, wl, math):
    d, kw = _case(wl)
    desc = B.make_desc(wl.N, wl.H, wl.W, wl.C, wl.G, DTYPES[wl.dtype], math=math, **kw)
    ref_in, ref_ow = B.dcn4_backward(d["input"], d["offset_weight"], d["grad_out"], group=wl.G,
                                     math=math, **kw)
    torch.cuda.synchronize()
    n = wl.N - 1
    rgin, rgow = _oracle_image(orc, wl, d, n)
    tol = TOL[wl.dtype]
    for call in range(2):
        gin = torch.full_like(d["input"], float("nan"))
        gow = torch.full_like(d["offset_weight"], float("nan"))
        assert _call_noalloc(desc, d, gin, gow) == 0, f"call {call}"
        torch.cuda.synchronize()
        assert scaled_err(f32(gin), f32(ref_in)) <= tol, f"grad_input vs dcn4_backward, call {call}"
        assert scaled_err(f32(gow), f32(ref_ow)) <= tol, f"grad_ow vs dcn4_backward, call {call}"
        assert scaled_err(f32(gin[n:n + 1]), rgin) <= tol, f"grad_input vs oracle, call {call}"
        assert scaled_err(f32(gow[n:n + 1]), rgow) <= tol, f"grad_ow vs oracle, call {call}"
    rc, bits = B.dcn4_last_device_error()
    assert rc == 0 and bits == 0


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("math", ["default", "f32"])
def test_noalloc_backward_twice_in_a_row(orc, dtype, math):
    # N*H*W*C = 2 x 128 x 128 x 256 = 8,388,608 fp32 scratch values: exactly
    # the 32 MiB the library holds
    wl = WORKLOADS["highres_bf16"].replace(N=2, dtype=dtype)
    _check_twice(orc, wl, math)


def test_noalloc_backward_fp32_needs_no_scratch(orc):
    # fp32 accumulates in grad_input itself; no size limit applies
    wl = WORKLOADS["internimage_f32"].replace(N=3, H=40, W=40)
    _check_twice(orc, wl, "default")


def test_noalloc_large_then_small_call(orc):
    """A call that fills the whole array followed by a smaller one: the small
    call clears and uses only its own part, so no value of the large call
    leaks into its grad_input."""
    big = WORKLOADS["highres_bf16"].replace(N=2)
    small = WORKLOADS["internimage_bf16"].replace(N=2, H=24, W=24, seed=5)
    db, kb = _case(big)
    ds, ks = _case(small)
    descb = B.make_desc(big.N, big.H, big.W, big.C, big.G, torch.bfloat16, math="f32", **kb)
    descs = B.make_desc(small.N, small.H, small.W, small.C, small.G, torch.bfloat16, math="f32",
                        **ks)
    gb = (torch.empty_like(db["input"]), torch.empty_like(db["offset_weight"]))
    gs = (torch.full_like(ds["input"], float("nan")),
          torch.full_like(ds["offset_weight"], float("nan")))
    assert _call_noalloc(descb, db, *gb) == 0
    assert _call_noalloc(descs, ds, *gs) == 0
    torch.cuda.synchronize()
    ref_in, ref_ow = B.dcn4_backward(ds["input"], ds["offset_weight"], ds["grad_out"],
                                     group=small.G, math="f32", **ks)
    torch.cuda.synchronize()
    assert scaled_err(f32(gs[0]), f32(ref_in)) <= TOL["bf16"]
    assert scaled_err(f32(gs[1]), f32(ref_ow)) <= TOL["bf16"]
    rgin, rgow = _oracle_image(orc, small, ds, 0)
    assert scaled_err(f32(gs[0][:1]), rgin) <= TOL["bf16"]
    assert scaled_err(f32(gs[1][:1]), rgow) <= TOL["bf16"]


def test_noalloc_rejects_sizes_beyond_the_scratch():
    lib = B.load()
    # 8 x 128 x 128 x 256 values need 128 MiB of fp32 scratch > 32 MiB
    desc = B.make_desc(8, 128, 128, 256, 16, torch.bfloat16)
    one = ctypes.c_void_p(256)
    rc = lib.dcn4_backward_noalloc(ctypes.byref(desc), one, one, one, one, one,
                                   ctypes.c_void_p(0))
    assert rc == 3  # DCN4_ERR_WORKSPACE, nothing launched
