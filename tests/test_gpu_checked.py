"""The bounds-checked build (libdcn4_checked.so, compiled with -DDCN4_CHECKED:
every shared- and global-memory access of every kernel is range-checked, a
violation sets the DCN4_ERR_INTERNAL bit of the device error word and skips
the access) on the small and edge parity cases of every kernel: staged,
vectorised and scalar forward and backward, DCNv4 and MSDCN, and both
offset/weight producers. Each case must match the oracle within the usual
gate, give the same forward output bit for bit as the normal build, and leave
the device error word clear. It stands in for compute-sanitizer: the checked
library is how out-of-bounds accesses are caught."""
import os

import pytest
import torch

from deformable_convolution_dcn4_b200 import _binding as B
from deformable_convolution_dcn4_b200 import build as libbuild
from deformable_convolution_dcn4_b200.workloads import (WORKLOADS, make_fused_inputs,
                                                        make_producer_inputs)

from parity_util import (TOL, backward_case, f32, forward_case, gpu_forward, msdcn_backward_case,
                         out_hw, scaled_err)
from deformable_convolution_dcn4_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu

W = WORKLOADS

CASES = {
    "internimage_bf16": W["internimage_bf16"].replace(N=2, H=24, W=20),
    "internimage_f32": W["internimage_f32"].replace(N=1, H=19, W=17),
    "ldm32_f16": W["ldm32_f16"].replace(N=1, H=16, W=12),
    "ragged_bf16": W["internimage_bf16"].replace(name="ragged", N=2, H=37, W=29, C=64, G=4),
    "stride2_pad0_dil2_f16": W["ldm64_f16"].replace(name="s2", N=1, H=33, W=30, C=64, G=4,
                                                    stride=(2, 2), pad=(0, 0), dilation=(2, 2)),
    "far_offsets_bf16": W["internimage_bf16"].replace(name="far", N=1, H=40, W=40,
                                                      offset_dist=("normal", 8.0)),
    "tiny_image_bf16": W["internimage_bf16"].replace(name="t", N=3, H=2, W=3, C=32, G=2),
    "one_pixel_f32": W["tiny_f32"].replace(name="p", N=2, H=1, W=1, C=16, G=4),
    "d64_bf16": W["flowdcn_msdcn_bf16"].replace(name="d64", kind="dcn4", N=1, H=12, W=14,
                                                C=256, G=4, offset_dist=("normal", 2.0)),
    "k5_bf16": W["internimage_bf16"].replace(name="k5b", N=1, H=11, W=9, C=64, G=4, kh=5, kw=5,
                                             pad=(2, 2)),
    "d12_bf16": W["internimage_bf16"].replace(name="d12", N=1, H=14, W=10, C=36, G=3),
    "softmax_bf16": W["internimage_bf16"].replace(name="sm", N=1, H=17, W=21, softmax=True,
                                                  weight_sigma=1.0),
}
MSDCN = {
    "flowdcn_msdcn_bf16": W["flowdcn_msdcn_bf16"].replace(N=1, H=16, W=16),
    "msdcn_d16_bf16": W["internimage_bf16"].replace(name="msd16", N=1, H=20, W=24, kind="msdcn",
                                                    offset_dist=("normal", 1.0), smax=8.0),
    "msdcn_dil_f32": W["internimage_f32"].replace(name="msdil", N=1, H=13, W=17, kind="msdcn",
                                                  offset_dist=("normal", 1.0), smax=3.0,
                                                  msdcn_mode="dilation"),
}


@pytest.fixture(scope="module")
def checked():
    """Switches the binding to the checked build for the module's tests."""
    if not os.path.exists(B.CHECKED_LIBRARY) or not libbuild.up_to_date(B.CHECKED_LIBRARY):
        libbuild.build(checked=True)
    B.load()
    prev = B.use_library(B.CHECKED_LIBRARY)
    torch.cuda.synchronize()
    assert B.dcn4_last_device_error() == (0, 0)
    yield
    torch.cuda.synchronize()
    B.restore_library(prev)


def _clear():
    torch.cuda.synchronize()
    rc, bits = B.dcn4_last_device_error()
    assert rc == 0 and bits == 0, f"checked build reported device error bits {bits}"


@pytest.mark.parametrize("algo", ["auto", "generic", "vector"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_checked_forward(orc, checked, name, algo):
    wl = CASES[name]
    try:
        err = forward_case(orc, wl, algo)
    except B.Dcn4Error as e:
        assert e.code == 2 and algo == "vector"  # the call has no vectorised form
        return
    _clear()
    assert err <= TOL[wl.dtype], f"{name}/{algo}: {err:.3e}"


@pytest.mark.parametrize("name", ["internimage_bf16", "ragged_bf16", "far_offsets_bf16",
                                  "d64_bf16", "internimage_f32"])
def test_checked_forward_bitwise_equal_to_normal_build(checked, name):
    wl = CASES[name]
    data = make_inputs(wl, out_hw(wl))
    got = gpu_forward(wl, data)
    _clear()
    prev = B.use_library(B.LIBRARY)
    try:
        ref = gpu_forward(wl, data)
        torch.cuda.synchronize()
    finally:
        B.restore_library(prev)
    assert torch.equal(got.view(torch.int16 if got.element_size() == 2 else torch.int32),
                       ref.view(torch.int16 if ref.element_size() == 2 else torch.int32))


@pytest.mark.parametrize("math", ["default", "acc16"])
@pytest.mark.parametrize("algo", ["auto", "generic"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_checked_backward(orc, checked, name, algo, math):
    wl = CASES[name]
    if wl.dtype == "f32" and math == "acc16":
        pytest.skip("16-bit accumulation applies to bf16/fp16 only")
    e_in, e_ow = backward_case(orc, wl, algo, math=math)
    _clear()
    tol = TOL[wl.dtype]
    assert e_in <= tol and e_ow <= tol, f"{name}/{algo}/{math}: {e_in:.3e} {e_ow:.3e}"


@pytest.mark.parametrize("algo", ["auto", "generic", "vector"])
@pytest.mark.parametrize("name", sorted(MSDCN))
def test_checked_msdcn(orc, checked, name, algo):
    wl = MSDCN[name]
    err = forward_case(orc, wl, algo)
    _clear()
    assert err <= TOL[wl.dtype], f"{name}/{algo} forward: {err:.3e}"
    errs = msdcn_backward_case(orc, wl, algo)
    _clear()
    assert max(errs) <= TOL[wl.dtype], f"{name}/{algo} backward: {errs}"


@pytest.mark.parametrize("algo", ["auto", "generic"])
@pytest.mark.parametrize("case", [(2, 13, 11, 128, 8, 3, "bf16"), (1, 5, 130, 16, 8, 1, "bf16"),
                                  (1, 8, 8, 320, 20, 3, "f16"), (2, 9, 7, 24, 3, 3, "f32")])
def test_checked_producer(orc, checked, case, algo):
    N, H, Wd, C, G, k, dtype = case
    d = make_producer_inputs(N, H, Wd, C, G, K=k * k, dtype=dtype, seed=3)
    dev = {n: t.cuda() for n, t in d.items()}
    out = B.dcn4_offset_producer(dev["x"], dev["dw_weight"], dev["dw_bias"], dev["lin_weight"],
                                 dev["lin_bias"], group=G, kernel_size=k, pad=(k - 1) // 2,
                                 algo=algo)
    _clear()
    prob = orc.problem(N, H, Wd, C, G, k, k, pad=((k - 1) // 2, (k - 1) // 2))
    ref = orc.offset_producer(prob, f32(d["x"]), f32(d["dw_weight"]), f32(d["dw_bias"]),
                              f32(d["lin_weight"]), f32(d["lin_bias"]))
    assert scaled_err(f32(out), ref) <= TOL[dtype]


@pytest.mark.parametrize("case", [(2, 24, 20, 128, 8, "bf16"), (1, 12, 10, 256, 16, "bf16"),
                                  (3, 2, 3, 64, 4, "f16"), (1, 20, 21, 64, 2, "bf16")])
def test_checked_fused_forward(orc, checked, case):
    """The fused producer + forward kernel (x neighbourhoods, depthwise into
    the MMA operand, lin_w rows, accumulators into the record slots, the
    gathers) through the checked build, against the oracle chain."""
    N, H, Wd, C, G, dtype = case
    d = make_fused_inputs(N, H, Wd, C, G, dtype=dtype, seed=11, offset_sigma=0.5)
    dev = {n: t.cuda() for n, t in d.items()}
    out = B.dcn4_fused_forward(dev["input"], dev["x"], dev["dw_weight"], dev["dw_bias"],
                               dev["lin_weight"], dev["lin_bias"], group=G, algo="halo")
    _clear()
    prob = orc.problem(N, H, Wd, C, G, 3, 3)
    ow = orc.offset_producer(prob, f32(d["x"]), f32(d["dw_weight"]), f32(d["dw_bias"]),
                             f32(d["lin_weight"]), f32(d["lin_bias"]))
    ow = torch.from_numpy(ow).to(d["x"].dtype).float().numpy().reshape(N, H, Wd, G, 9, 3)
    ref = orc.forward(prob, f32(d["input"]), ow)
    assert scaled_err(f32(out), ref) <= TOL[dtype]
