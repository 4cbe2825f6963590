"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs, element by element (scaled max error), for every kernel
variant, the workload shapes (reduced, then full size on sampled images) and
the edge cases."""
import numpy as np
import pytest
import torch

from deformable_convolution_dcn4_b200 import _binding as B
from deformable_convolution_dcn4_b200.workloads import WORKLOADS, make_inputs

from parity_util import (TOL, backward_case, checked_err, desc_kw, msdcn_backward_case, f32,
                         forward_case, gpu_forward, oracle_forward, out_hw, problem,
                         scaled_err)

pytestmark = pytest.mark.gpu

W = WORKLOADS
ALGOS = ["auto", "generic", "halo"]

# Workload shapes at sizes the oracle finishes in seconds (several tiles,
# ragged tails where the sizes allow).
REDUCED = {
    "tiny_f32": W["tiny_f32"],
    "internimage_bf16": W["internimage_bf16"].replace(N=2),
    "internimage_f32": W["internimage_f32"].replace(N=2),
    "ldm64_f16": W["ldm64_f16"].replace(N=1),
    "ldm32_f16": W["ldm32_f16"].replace(N=2),
    "flowdcn_msdcn_bf16": W["flowdcn_msdcn_bf16"].replace(N=2),
    "highres_bf16": W["highres_bf16"].replace(N=1),
}

EDGE = {
    "ragged_bf16": W["internimage_bf16"].replace(name="ragged", N=2, H=37, W=29, C=64, G=4),
    "stride2_pad0_dil2_f16": W["ldm64_f16"].replace(name="s2", N=1, H=33, W=30, C=64, G=4,
                                                    stride=(2, 2), pad=(0, 0), dilation=(2, 2)),
    "stride_mixed_f32": W["tiny_f32"].replace(name="smix", N=2, H=21, W=18, C=32, G=2,
                                              stride=(1, 2), pad=(2, 0), dilation=(1, 2)),
    "offset_scale_bf16": W["internimage_bf16"].replace(name="os", N=1, H=20, W=24,
                                                       offset_scale=0.75),
    "far_offsets_bf16": W["internimage_bf16"].replace(name="far", N=1, H=40, W=40,
                                                      offset_dist=("normal", 8.0)),
    "far_offsets_f32": W["internimage_f32"].replace(name="far32", N=1, H=24, W=32,
                                                    offset_dist=("normal", 6.0)),
    "single_group_f16": W["ldm64_f16"].replace(name="g1", N=2, H=12, W=10, C=16, G=1),
    "tiny_image_bf16": W["internimage_bf16"].replace(name="t", N=3, H=2, W=3, C=32, G=2),
    "one_pixel_f32": W["tiny_f32"].replace(name="p", N=2, H=1, W=1, C=16, G=4),
    "d64_f32": W["tiny_f32"].replace(name="d64", N=1, H=12, W=14, C=128, G=2),
}

GENERIC_ONLY = {
    "k1x1_bf16": W["internimage_bf16"].replace(name="k1", N=1, H=10, W=12, kh=1, kw=1,
                                                pad=(0, 0)),
    "k5x5_f32": W["tiny_f32"].replace(name="k5", N=1, H=11, W=9, kh=5, kw=5, pad=(2, 2)),
    "k3x1_f16": W["ldm64_f16"].replace(name="k31", N=1, H=9, W=8, C=32, G=2, kh=3, kw=1,
                                       pad=(1, 0)),
    "d12_bf16": W["internimage_bf16"].replace(name="d12", N=1, H=14, W=10, C=36, G=3),
    "d6_f32": W["tiny_f32"].replace(name="d6", N=1, H=9, W=9, C=6, G=1),
}


def _halo_supported(wl):
    """The halo kernel stages 128-byte pixels (Gc groups of D channels) and
    needs 3x3 taps and 32-, 64- or 128-byte group slices (16-byte chunks)."""
    eb = 4 if wl.dtype == "f32" else 2
    slice_bytes = wl.D * eb
    if wl.kh != 3 or wl.kw != 3 or slice_bytes not in ((32, 64, 128) if eb == 2 else (64, 128)):
        return False
    return wl.G % (128 // slice_bytes) == 0


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("name", sorted(REDUCED))
def test_forward_reduced(orc, name, algo):
    wl = REDUCED[name]
    err = forward_case(orc, wl, algo)
    assert err <= TOL[wl.dtype], f"{name}/{algo}: {err:.3e}"


@pytest.mark.parametrize("name", [n for n in sorted(REDUCED) if REDUCED[n].dtype != "f32"] +
                         ["ragged_bf16", "stride2_pad0_dil2_f16", "far_offsets_bf16",
                          "offset_scale_bf16"])
@pytest.mark.parametrize("math", ["f32", "mixed16", "packed16"])
def test_forward_math_modes(orc, name, math):
    """fp32 weights, 16-bit weights with the mixed-precision fma (the default
    for 16-bit data) and the packed 16-bit corner blend: all meet the gate."""
    wl = REDUCED.get(name) or EDGE[name]
    data = make_inputs(wl, out_hw(wl))
    dev = "cuda"
    if wl.kind == "msdcn":
        got = B.msdcn_forward(data["input"].to(dev), data["dir_weight"].to(dev),
                              data["scale_raw"].to(dev), data["s0"], wl.smax, group=wl.G,
                              math=math, **_kw(wl))
    else:
        got = B.dcn4_forward(data["input"].to(dev), data["offset_weight"].to(dev), group=wl.G,
                             math=math, **_kw(wl))
    err = checked_err(f32(got), oracle_forward(orc, wl, data), wl.dtype, f"{name}/{math}")
    assert err <= TOL[wl.dtype], f"{name}: {err:.3e}"


def _kw(wl):
    return dict(kernel_size=(wl.kh, wl.kw), stride=wl.stride, pad=wl.pad, dilation=wl.dilation,
                offset_scale=wl.offset_scale)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("name", sorted(EDGE))
def test_forward_edge(orc, name, algo):
    wl = EDGE[name]
    if algo == "halo" and not _halo_supported(wl):
        with pytest.raises(B.Dcn4Error) as e:
            forward_case(orc, wl, algo)
        assert e.value.code == 2
        return
    err = forward_case(orc, wl, algo)
    assert err <= TOL[wl.dtype], f"{name}/{algo}: {err:.3e}"


@pytest.mark.parametrize("name", sorted(GENERIC_ONLY))
def test_forward_generic_shapes(orc, name):
    wl = GENERIC_ONLY[name]
    err = forward_case(orc, wl, "auto")
    assert err <= TOL[wl.dtype], f"{name}: {err:.3e}"
    with pytest.raises(B.Dcn4Error) as e:
        forward_case(orc, wl, "halo")
    assert e.value.code == 2


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("algo", ALGOS)
def test_integer_offsets_gather_exactly(orc, dtype, algo):
    """Integer offsets and one tap with m = 1: the output is a copy of input
    pixels (or zero), so the GPU must equal the oracle bit for bit; this pins
    the corner selection."""
    wl = W["internimage_bf16"].replace(N=2, H=19, W=23, C=64, G=4, dtype=dtype)
    Ho, Wo = out_hw(wl)
    data = make_inputs(wl, (Ho, Wo))
    g = torch.Generator().manual_seed(3)
    ow = torch.zeros((wl.N, Ho, Wo, wl.G, 9, 3))
    ow[..., :2] = torch.randint(-6, 7, (wl.N, Ho, Wo, wl.G, 9, 2), generator=g).float()
    tap = torch.randint(0, 9, (wl.N, Ho, Wo, wl.G), generator=g)
    ow[..., 2].scatter_(-1, tap[..., None], 1.0)
    data["offset_weight"] = ow.to(data["input"].dtype)
    got = f32(gpu_forward(wl, data, algo))
    ref = oracle_forward(orc, wl, data)
    assert np.array_equal(got, ref.astype(np.float32))


@pytest.mark.parametrize("algo", ALGOS)
def test_all_samples_out_of_bounds_give_zero(orc, algo):
    wl = W["internimage_bf16"].replace(N=1, H=16, W=16)
    Ho, Wo = out_hw(wl)
    data = make_inputs(wl, (Ho, Wo))
    ow = data["offset_weight"].float()
    ow[..., 0] = -(wl.W + 5.0)
    data["offset_weight"] = ow.to(torch.bfloat16)
    assert torch.count_nonzero(gpu_forward(wl, data, algo)).item() == 0


def test_nonfinite_offsets_contribute_nothing(orc):
    wl = W["tiny_f32"]
    Ho, Wo = out_hw(wl)
    data = make_inputs(wl, (Ho, Wo))
    ow = data["offset_weight"].clone()
    ow[0, 3, 4, 1, 2, 0] = float("nan")
    ow[0, 5, 6, 2, 7, 1] = float("inf")
    data["offset_weight"] = ow
    for algo in ALGOS:
        got = f32(gpu_forward(wl, data, algo))
        assert scaled_err(got, oracle_forward(orc, wl, data)) <= TOL["f32"]


@pytest.mark.parametrize("algo", ["generic", "halo"])
def test_msdcn_unit_scale_is_dcn4(orc, algo):
    """softplus(30) > Smax = 1 so every scale is exactly 1: MSDCN must equal
    DCNv4 with offsets = directions. The generic kernels must agree bit for
    bit. The halo kernels tile MSDCN and DCNv4 differently, so a sample that
    leaves one window but not the other is summed in another order: there
    almost every element must agree bit for bit and the rest to 1e-2."""
    wl = REDUCED["flowdcn_msdcn_bf16"].replace(N=1, smax=1.0)
    Ho, Wo = out_hw(wl)
    data = make_inputs(wl, (Ho, Wo))
    data["scale_raw"] = torch.full_like(data["scale_raw"], 30.0)
    data["s0"] = torch.ones(wl.G)
    ms = gpu_forward(wl, data, algo)
    dcn = B.dcn4_forward(data["input"].cuda(), data["dir_weight"].cuda(), group=wl.G, algo=algo)
    if algo == "generic":
        assert torch.equal(ms, dcn)
    else:
        same = (ms == dcn).float().mean().item()
        assert same >= 0.99, same
        assert scaled_err(f32(ms), f32(dcn)) <= 1e-2


def test_misaligned_pointers_take_generic_path(orc):
    wl = W["internimage_bf16"].replace(N=1, H=12, W=12)
    Ho, Wo = out_hw(wl)
    data = make_inputs(wl, (Ho, Wo))
    x = torch.empty(data["input"].numel() + 1, dtype=torch.bfloat16, device="cuda")[1:]
    x = x.view(data["input"].shape)
    x.copy_(data["input"])
    assert x.data_ptr() % 16 != 0
    out = B.dcn4_forward(x, data["offset_weight"].cuda(), group=wl.G)
    assert scaled_err(f32(out), oracle_forward(orc, wl, data)) <= TOL["bf16"]
    with pytest.raises(B.Dcn4Error) as e:
        B.dcn4_forward(x, data["offset_weight"].cuda(), group=wl.G, algo="halo")
    assert e.value.code == 2


def test_forward_is_deterministic():
    wl = REDUCED["internimage_bf16"]
    data = make_inputs(wl, out_hw(wl))
    a = gpu_forward(wl, data)
    b = gpu_forward(wl, data)
    assert torch.equal(a, b)


# ---- full sizes, in the bench's launch configuration, sampled images ----
FULL_SAMPLES = {
    "internimage_bf16": [0, 37, 63],
    "internimage_f32": [0, 63],
    "ldm64_f16": [0, 7],
    "ldm32_f16": [0, 5],
    "flowdcn_msdcn_bf16": [0, 31],
    "highres_bf16": [0, 3],
}


@pytest.mark.parametrize("name", sorted(FULL_SAMPLES))
def test_forward_full_size_sampled(orc, name):
    wl = W[name]
    err = forward_case(orc, wl, "auto", images=FULL_SAMPLES[name])
    assert err <= TOL[wl.dtype], f"{name}: {err:.3e}"


# ---- backward ----
BWD = {
    "tiny_f32": W["tiny_f32"],
    "highres_bf16_small": W["highres_bf16"].replace(N=1, H=40, W=36),
    "internimage_bf16": W["internimage_bf16"].replace(N=1),
    "ldm_f16": W["ldm64_f16"].replace(N=1, H=24, W=20),
    "stride2_dil2_f32": W["tiny_f32"].replace(N=2, H=17, W=15, C=32, G=2, stride=(2, 2),
                                              dilation=(2, 2), pad=(2, 1), offset_scale=0.5),
    "k5_f32": W["tiny_f32"].replace(N=1, H=9, W=11, C=8, G=2, kh=5, kw=5, pad=(2, 2)),
    "d12_bf16": W["internimage_bf16"].replace(N=1, H=10, W=9, C=36, G=3),
    "far_bf16": W["internimage_bf16"].replace(N=1, H=24, W=24, offset_dist=("normal", 8.0)),
}


@pytest.mark.parametrize("math", ["default", "acc16"])
@pytest.mark.parametrize("name", sorted(BWD))
def test_backward(orc, name, math):
    """Default: fp32 accumulation of grad_input across CTAs; acc16: each CTA's
    fp32 partial sum added to the 16-bit grad_input directly."""
    wl = BWD[name]
    e_in, e_ow = backward_case(orc, wl, math=math)
    tol = TOL[wl.dtype]
    assert e_in <= tol and e_ow <= tol, f"{name}: grad_input {e_in:.3e} grad_ow {e_ow:.3e}"


@pytest.mark.parametrize("name", ["highres_bf16_small", "ldm_f16", "internimage_bf16"])
def test_backward_f32_weights(orc, name):
    wl = BWD[name]
    e_in, e_ow = backward_case(orc, wl, math="f32")
    tol = TOL[wl.dtype]
    assert e_in <= tol and e_ow <= tol, f"{name}: grad_input {e_in:.3e} grad_ow {e_ow:.3e}"


def test_backward_full_size_sampled(orc):
    wl = W["highres_bf16"]
    e_in, e_ow = backward_case(orc, wl, images=[0, 3])
    assert e_in <= TOL["bf16"] and e_ow <= TOL["bf16"], (e_in, e_ow)


def test_backward_workspace_too_small_is_rejected():
    wl = W["tiny_f32"].replace(dtype="bf16")
    data = make_inputs(wl, out_hw(wl), with_grad=True)
    with pytest.raises(B.Dcn4Error) as e:
        B.dcn4_backward(data["input"].cuda(), data["offset_weight"].cuda(),
                        data["grad_out"].cuda(), group=wl.G,
                        workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.code == 3


def test_no_device_error_left_behind():
    torch.cuda.synchronize()
    rc, bits = B.dcn4_last_device_error()
    assert rc == 0 and bits == 0


def test_bounded_wait_expiry_is_reported_and_context_survives(orc):
    """A barrier that nothing completes: the kernel's wait gives up after 2 ms,
    the host reads DCN4_ERR_TIMEOUT, and the context keeps working."""
    torch.cuda.synchronize()
    B.dcn4_last_device_error()
    B.dcn4_selftest_bounded_wait(2000)
    torch.cuda.synchronize()
    rc, bits = B.dcn4_last_device_error()
    assert rc == 5 and bits & 1, (rc, bits)
    assert B.dcn4_last_device_error() == (0, 0)  # read clears it
    err = forward_case(orc, W["tiny_f32"], "halo")
    assert err <= TOL["f32"]


def test_launch_counter_counts_each_kernel():
    """Forward on the halo path is one kernel, with escape scratch or without;
    the 16-bit backward with 16-bit
    cross-CTA accumulation (acc16) is two (zero grad_input, halo kernel);
    with fp32 accumulation (the default, and f32) it is three (zero
    workspace, halo kernel, convert)."""
    wl = REDUCED["internimage_bf16"]
    data = make_inputs(wl, out_hw(wl), with_grad=True)
    x, ow, go = (data[k].cuda() for k in ("input", "offset_weight", "grad_out"))
    nf = B.dcn4_kernel_launches()
    B.dcn4_forward(x, ow, group=wl.G, algo="halo")
    n0 = B.dcn4_kernel_launches()
    assert n0 - nf == 1
    B.dcn4_forward(x, ow, group=wl.G, algo="halo", defer_escapes=False)
    n1 = B.dcn4_kernel_launches()
    B.dcn4_backward(x, ow, go, group=wl.G, algo="halo", math="acc16")
    n2 = B.dcn4_kernel_launches()
    B.dcn4_backward(x, ow, go, group=wl.G, algo="halo", math="f32")
    n3 = B.dcn4_kernel_launches()
    B.dcn4_backward(x, ow, go, group=wl.G, algo="halo")
    n4 = B.dcn4_kernel_launches()
    torch.cuda.synchronize()
    assert (n1 - n0, n2 - n1, n3 - n2, n4 - n3) == (1, 2, 3, 3)


MSDCN_BWD = {
    "flowdcn_msdcn_bf16": REDUCED["flowdcn_msdcn_bf16"].replace(N=1),
    "msdcn_d16_bf16": W["internimage_bf16"].replace(name="msd16", N=1, H=20, W=24, kind="msdcn",
                                                    offset_dist=("normal", 1.0), smax=8.0),
    "msdcn_d16_f32": W["internimage_f32"].replace(name="msd16f", N=1, H=13, W=17, kind="msdcn",
                                                  offset_dist=("normal", 1.0), smax=3.0),
    "msdcn_stride_f16": W["ldm64_f16"].replace(name="msds", N=2, H=15, W=11, C=32, G=4,
                                               kind="msdcn", offset_dist=("normal", 1.0),
                                               stride=(2, 1), pad=(0, 1), dilation=(1, 2),
                                               offset_scale=0.5, smax=2.0),
}


@pytest.mark.parametrize("name", sorted(MSDCN_BWD))
@pytest.mark.parametrize("math", ["default", "f32", "acc16"])
def test_msdcn_backward(orc, name, math):
    wl = MSDCN_BWD[name]
    errs = msdcn_backward_case(orc, wl, math=math)
    tol = TOL[wl.dtype]
    assert all(e <= tol for e in errs), f"{name}: grad_input/dir/raw errors {errs}"


def test_msdcn_backward_full_size_sampled(orc):
    wl = W["flowdcn_msdcn_bf16"]
    errs = msdcn_backward_case(orc, wl, images=[0, 31])
    assert all(e <= TOL["bf16"] for e in errs), errs


# 64-channel groups (8 16-byte vectors): the staged backward with two lanes
# per (pixel, group), the whole image as its window for MSDCN (FlowDCN token
# grid) and a 4-pixel margin for DCNv4; forced, against the oracle, in all
# three accumulation modes, plus the vectorised kernel on the same shapes
D64_STAGED = {
    "flowdcn_msdcn_bf16": MSDCN_BWD["flowdcn_msdcn_bf16"],
    "flowdcn_msdcn_f16_ragged": W["flowdcn_msdcn_bf16"].replace(name="fd16", N=2, H=21, W=19,
                                                                C=256, G=4, dtype="f16"),
    "msdcn_d32_f32": W["internimage_f32"].replace(name="msd32f", N=1, H=18, W=14, C=64, G=2,
                                                  kind="msdcn", offset_dist=("normal", 1.0),
                                                  smax=4.0),
    "dcn4_d64_bf16": W["internimage_bf16"].replace(name="d64s", N=2, H=23, W=29, C=128, G=2),
}


@pytest.mark.parametrize("math", ["default", "f32", "acc16"])
@pytest.mark.parametrize("name", sorted(D64_STAGED))
def test_backward_staged_wide_groups(orc, name, math):
    wl = D64_STAGED[name]
    if wl.dtype == "f32" and math == "acc16":
        pytest.skip("16-bit accumulation applies to bf16/fp16 only")
    tol = TOL[wl.dtype]
    if wl.kind == "msdcn":
        errs = msdcn_backward_case(orc, wl, algo="halo", math=math)
        assert max(errs) <= tol, f"{name}/{math}: {errs}"
    else:
        e_in, e_ow = backward_case(orc, wl, algo="halo", math=math)
        assert e_in <= tol and e_ow <= tol, f"{name}/{math}: {e_in:.3e} {e_ow:.3e}"


def test_backward_staged_wide_groups_full_size_sampled(orc):
    """The FlowDCN shape (N32 32x32 C1152 G18 bf16) on the staged kernel:
    images 0 and 31 against the oracle."""
    wl = W["flowdcn_msdcn_bf16"]
    errs = msdcn_backward_case(orc, wl, algo="halo", images=[0, 31])
    assert all(e <= TOL["bf16"] for e in errs), errs


# DCNv3 compatibility (softmax over the taps) and the MSDCN scale-as-dilation
# reading, against the oracle's own definitions of both
SOFTMAX = {
    "softmax_bf16": W["internimage_bf16"].replace(name="sm", N=2, H=20, W=24, softmax=True,
                                                  weight_sigma=1.0),
    "softmax_f32": W["internimage_f32"].replace(name="smf", N=1, H=13, W=17, softmax=True,
                                                weight_sigma=1.0),
    "softmax_f16_stride": W["ldm64_f16"].replace(name="sms", N=1, H=15, W=11, C=64, G=4,
                                                 stride=(2, 1), pad=(1, 2), dilation=(1, 2),
                                                 softmax=True, weight_sigma=2.0),
}


@pytest.mark.parametrize("name", sorted(SOFTMAX))
@pytest.mark.parametrize("algo", ["auto", "generic"])
def test_softmax_forward(orc, name, algo):
    wl = SOFTMAX[name]
    err = forward_case(orc, wl, algo)
    assert err <= TOL[wl.dtype], f"{name}/{algo}: {err:.3e}"


@pytest.mark.parametrize("name", sorted(SOFTMAX))
@pytest.mark.parametrize("algo", ["auto", "generic"])
def test_softmax_backward(orc, name, algo):
    wl = SOFTMAX[name]
    e_in, e_ow = backward_case(orc, wl, algo)
    tol = TOL[wl.dtype]
    assert e_in <= tol and e_ow <= tol, f"{name}/{algo}: grad_input {e_in:.3e} grad_ow {e_ow:.3e}"


DILATION = {
    "dil_bf16": MSDCN_BWD["msdcn_d16_bf16"].replace(name="dil16", msdcn_mode="dilation", smax=3.0),
    "dil_f32": MSDCN_BWD["msdcn_d16_f32"].replace(name="dil32", msdcn_mode="dilation", smax=2.5),
    "dil_flowdcn_bf16": REDUCED["flowdcn_msdcn_bf16"].replace(N=1, msdcn_mode="dilation"),
}


@pytest.mark.parametrize("name", sorted(DILATION))
@pytest.mark.parametrize("algo", ["auto", "generic"])
def test_msdcn_dilation_forward(orc, name, algo):
    wl = DILATION[name]
    err = forward_case(orc, wl, algo)
    assert err <= TOL[wl.dtype], f"{name}/{algo}: {err:.3e}"


@pytest.mark.parametrize("name", sorted(DILATION))
def test_msdcn_dilation_backward(orc, name):
    wl = DILATION[name]
    errs = msdcn_backward_case(orc, wl)
    assert all(e <= TOL[wl.dtype] for e in errs), f"{name}: {errs}"


def test_msdcn_rejects_softmax():
    wl = MSDCN_BWD["msdcn_d16_bf16"]
    data = make_inputs(wl, out_hw(wl), with_grad=True)
    desc = B.make_desc(wl.N, wl.H, wl.W, wl.C, wl.G, torch.bfloat16, softmax=True)
    out = torch.empty_like(data["input"]).cuda()
    s0 = (B.ctypes.c_float * wl.G)(*data["s0"].tolist())
    rc = B.load().msdcn_forward(B.ctypes.byref(desc), B._ptr(data["input"].cuda()),
                                B._ptr(data["dir_weight"].cuda()), B._ptr(data["scale_raw"].cuda()),
                                s0, 8.0, B._ptr(out), None)
    assert rc == 2


# Shapes on the global-memory backward kernels: AUTO runs the staged kernel
# where it applies (d64_bf16, softmax_d64_bf16: 64-channel groups), else the
# vectorised global-memory kernel (whole 16-byte vectors per group) or, for
# group widths that are not, the scalar one; "generic" forces the scalar
# kernel, "vector" the vectorised one.
BWD_VEC = {
    "d64_bf16": W["flowdcn_msdcn_bf16"].replace(name="d64", kind="dcn4", N=1, H=12, W=14,
                                                C=256, G=4, offset_dist=("normal", 2.0)),
    "d64_f32": W["tiny_f32"].replace(name="d64f", N=1, H=9, W=10, C=128, G=2),
    "k5_bf16": W["internimage_bf16"].replace(name="k5b", N=1, H=11, W=9, C=64, G=4, kh=5, kw=5,
                                             pad=(2, 2)),
    "k3x1_f16_d8": W["ldm64_f16"].replace(name="k31", N=2, H=9, W=8, C=32, G=4, kh=3, kw=1,
                                          pad=(1, 0)),
    "d12_bf16": BWD["d12_bf16"],
    "softmax_d64_bf16": W["flowdcn_msdcn_bf16"].replace(name="smd64", kind="dcn4", N=1, H=10,
                                                        W=10, C=128, G=2, softmax=True,
                                                        weight_sigma=1.0),
}


@pytest.mark.parametrize("name", sorted(BWD_VEC))
@pytest.mark.parametrize("algo", ["auto", "generic", "vector"])
def test_backward_global_kernels(orc, name, algo):
    wl = BWD_VEC[name]
    vb = wl.D * (4 if wl.dtype == "f32" else 2)
    if algo == "vector" and (vb % 16 or vb > 256 or (vb // 16) & (vb // 16 - 1)):
        pytest.skip("group channels are not whole 16-byte vectors")
    e_in, e_ow = backward_case(orc, wl, algo)
    tol = TOL[wl.dtype]
    assert e_in <= tol and e_ow <= tol, f"{name}/{algo}: grad_input {e_in:.3e} grad_ow {e_ow:.3e}"


# the staged kernel (AUTO picks it for these) and the vectorised one, forced,
# on the same D16 MSDCN shapes (stride, dilation and offset_scale included),
# both readings, both math modes
MSDCN_BWD_HALO = {
    "msdcn_d16_bf16": MSDCN_BWD["msdcn_d16_bf16"],
    "msdcn_d16_f32": MSDCN_BWD["msdcn_d16_f32"],
    "msdcn_stride_bf16": MSDCN_BWD["msdcn_stride_f16"].replace(name="msdsb", dtype="bf16", C=64),
    "dil_bf16": DILATION["dil_bf16"],
    "dil_f32": DILATION["dil_f32"],
    "msdcn_d16_bf16_smax8_far": MSDCN_BWD["msdcn_d16_bf16"].replace(
        name="msdfar", N=2, H=29, W=23, offset_dist=("normal", 2.5)),
}


@pytest.mark.parametrize("name", sorted(MSDCN_BWD_HALO))
@pytest.mark.parametrize("algo", ["halo", "vector"])
@pytest.mark.parametrize("math", ["default", "f32"])
def test_msdcn_backward_staged_and_vector(orc, name, algo, math):
    wl = MSDCN_BWD_HALO[name]
    errs = msdcn_backward_case(orc, wl, algo=algo, math=math)
    tol = TOL[wl.dtype]
    assert all(e <= tol for e in errs), f"{name}/{algo}/{math}: grad_input/dir/raw {errs}"


def test_msdcn_backward_staged_full_size_sampled(orc):
    """The bench's MSDCN shape (N64 56x56 C128 G8 bf16) on the staged kernel;
    images 0 and 63 against the oracle."""
    wl = W["internimage_bf16"].replace(kind="msdcn", offset_dist=("normal", 1.0))
    errs = msdcn_backward_case(orc, wl, algo="halo", images=[0, 63])
    assert all(e <= TOL["bf16"] for e in errs), errs


@pytest.mark.parametrize("name", ["msdcn_d16_bf16", "msdcn_stride_f16"])
def test_msdcn_backward_scalar_kernel(orc, name):
    wl = MSDCN_BWD[name]
    errs = msdcn_backward_case(orc, wl, algo="generic")
    assert all(e <= TOL[wl.dtype] for e in errs), f"{name}: {errs}"


# More edge cases of the later rows: softmax with far offsets (many samples
# take the global escape path of the staged kernels), softmax with fp32 math
# in the backward, MSDCN with a NaN scale and with every scale clamped, and
# the dilation reading at the FlowDCN group width with stride.
EXTRA = {
    "softmax_far_bf16": SOFTMAX["softmax_bf16"].replace(name="smfar", offset_dist=("normal", 8.0)),
    "softmax_ragged_f16": W["ldm64_f16"].replace(name="smr", N=2, H=13, W=11, C=64, G=4,
                                                 softmax=True, weight_sigma=3.0),
}


@pytest.mark.parametrize("name", sorted(EXTRA))
def test_softmax_edge_forward_backward(orc, name):
    wl = EXTRA[name]
    assert forward_case(orc, wl) <= TOL[wl.dtype]
    for math in ("default", "f32"):
        e_in, e_ow = backward_case(orc, wl, math=math)
        assert e_in <= TOL[wl.dtype] and e_ow <= TOL[wl.dtype], (name, math, e_in, e_ow)


def test_msdcn_nan_and_clamped_scales(orc):
    """A NaN raw scale gives no contribution and no gradient for its
    (pixel, group); raw values far above the clamp give s = Smax exactly and
    a zero raw gradient."""
    wl = MSDCN_BWD["msdcn_d16_bf16"].replace(smax=2.0)
    data = make_inputs(wl, out_hw(wl), with_grad=True)
    raw = data["scale_raw"].clone()
    raw[0, 3, 4, 1] = float("nan")
    raw[0, 5, :, :] = 40.0  # every group of row 5 clamped
    data["scale_raw"] = raw
    dev = "cuda"
    out = B.msdcn_forward(data["input"].to(dev), data["dir_weight"].to(dev), raw.to(dev),
                          data["s0"], wl.smax, group=wl.G, **desc_kw(wl))
    gin, gdw, graw = B.msdcn_backward(data["input"].to(dev), data["dir_weight"].to(dev),
                                      raw.to(dev), data["s0"], wl.smax, data["grad_out"].to(dev),
                                      group=wl.G, **desc_kw(wl))
    prob = problem(orc, wl)
    x, dw, go = (f32(data[k]) for k in ("input", "dir_weight", "grad_out"))
    ref = orc.msdcn_forward(prob, x, dw, f32(raw), data["s0"].numpy(), wl.smax)
    rgin, rgdw, rgraw = orc.msdcn_backward(prob, x, dw, f32(raw), data["s0"].numpy(), wl.smax, go)
    got = f32(out)
    # the NaN group's channels are NaN on both sides (m * NaN-position sample
    # is skipped, the oracle skips it too: zero contribution), compare the rest
    assert scaled_err(got, ref) <= TOL["bf16"]
    assert scaled_err(f32(gin), rgin) <= TOL["bf16"]
    assert scaled_err(f32(gdw), rgdw) <= TOL["bf16"]
    g = f32(graw)
    assert np.all(g[0, 5] == 0.0) and np.all(rgraw[0, 5] == 0.0)
    assert g[0, 3, 4, 1] == 0.0 and rgraw[0, 3, 4, 1] == 0.0
    assert scaled_err(g, rgraw) <= TOL["bf16"]


def test_msdcn_dilation_stride_d64(orc):
    wl = REDUCED["flowdcn_msdcn_bf16"].replace(name="dils", N=1, H=15, W=13, C=128, G=2,
                                               stride=(2, 1), pad=(1, 2), dilation=(1, 2),
                                               msdcn_mode="dilation", smax=3.0)
    assert forward_case(orc, wl) <= TOL["bf16"]
    assert all(e <= TOL["bf16"] for e in msdcn_backward_case(orc, wl))


# Forward shapes the staged kernel does not take, on both global-memory
# kernels: AUTO runs the vectorised one (whole 16-byte vectors per group,
# aligned tensors), "generic" the scalar one.
FWD_VEC = {
    "k5_bf16": BWD_VEC["k5_bf16"],
    "k3x1_f16": BWD_VEC["k3x1_f16_d8"],
    "d64_f32": BWD_VEC["d64_f32"],
    "d256_bf16": W["internimage_bf16"].replace(name="d256", N=1, H=9, W=7, C=512, G=2),
    "softmax_k5_f32": W["tiny_f32"].replace(name="smk5", N=1, H=10, W=9, C=32, G=2, kh=5, kw=5,
                                            pad=(2, 2), softmax=True, weight_sigma=1.0),
    "msdcn_k5_bf16": MSDCN_BWD["msdcn_d16_bf16"].replace(name="msk5", H=12, W=11, kh=5, kw=5,
                                                        pad=(2, 2)),
    "msdcn_dil_k5_f32": MSDCN_BWD["msdcn_d16_f32"].replace(name="msdk5", kh=5, kw=5, pad=(2, 2),
                                                          msdcn_mode="dilation", smax=2.0),
}


@pytest.mark.parametrize("name", sorted(FWD_VEC))
@pytest.mark.parametrize("algo", ["auto", "vector", "generic"])
def test_forward_global_kernels(orc, name, algo):
    wl = FWD_VEC[name]
    err = forward_case(orc, wl, algo)
    assert err <= TOL[wl.dtype], f"{name}/{algo}: {err:.3e}"


@pytest.mark.parametrize("name", ["internimage_bf16", "highres_bf16", "flowdcn_msdcn_bf16",
                                  "internimage_f32"])
def test_vector_kernels_on_staged_shapes(orc, name):
    """DCN4_ALGO_VECTOR forces the vectorised global-memory kernels on shapes
    AUTO would stage: same oracle, same gates."""
    wl = REDUCED[name]
    assert forward_case(orc, wl, "vector") <= TOL[wl.dtype]
    if wl.kind == "msdcn":
        errs = msdcn_backward_case(orc, wl.replace(N=1), algo="vector")
        assert all(e <= TOL[wl.dtype] for e in errs), errs
    else:
        e_in, e_ow = backward_case(orc, wl, "vector")
        assert e_in <= TOL[wl.dtype] and e_ow <= TOL[wl.dtype], (e_in, e_ow)


def test_vector_request_on_unaligned_groups_is_unsupported():
    wl = GENERIC_ONLY["d12_bf16"]
    with pytest.raises(B.Dcn4Error) as e:
        forward_case(None, wl, "vector")
    assert e.value.code == 2
