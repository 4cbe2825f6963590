"""Helpers shared by the GPU parity tests: run one case through the C ABI and
through the CPU oracle on the same seeded inputs and compare."""
import numpy as np
import torch

from deformable_convolution_dcn4_b200 import _binding as B
from deformable_convolution_dcn4_b200.workloads import make_inputs

# Gates (scaled error = max |gpu - ref| / max |ref|): fp32 1e-5; bf16/fp16
# outputs are rounded to their 8/11-bit mantissas, gate 2e-2.
TOL = {"f32": 1e-5, "bf16": 2e-2, "f16": 2e-2}

# Second, elementwise gate: max |gpu - ref| / (|ref| + rms(ref)). The scaled
# error measures every element against the largest output, so an error that
# only touches small outputs can hide under it; here each element is measured
# against its own size, floored at the rms so that outputs near zero do not
# turn rounding into a failure. Gates keep a 2-4x margin over the largest
# values seen on B200 (bf16 ~1e-2, 2e-2 with 16-bit accumulation; fp16 ~3e-3;
# fp32 ~6e-7).
FLOOR_TOL = {"f32": 1e-5, "bf16": 5e-2, "f16": 5e-2}


def scaled_err(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite GPU output"
    scale = np.abs(ref).max()
    if scale == 0.0:
        return float(np.abs(got).max())
    return float(np.abs(got - ref).max() / scale)


def rel_err_rms_floor(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    if rms == 0.0:
        return float(np.abs(got).max()) if got.size else 0.0
    return float((np.abs(got - ref) / (np.abs(ref) + rms)).max())


def checked_err(got, ref, dtype, what=""):
    """Scaled error of got against ref, after asserting the elementwise gate."""
    err = scaled_err(got, ref)
    floor = rel_err_rms_floor(got, ref)
    assert floor <= FLOOR_TOL[dtype], f"{what}: elementwise (rms floor) error {floor:.3e}"
    return err


def f32(t):
    return t.float().cpu().numpy()


def desc_kw(wl):
    kw = dict(kernel_size=(wl.kh, wl.kw), stride=wl.stride, pad=wl.pad, dilation=wl.dilation,
              offset_scale=wl.offset_scale)
    if wl.kind == "msdcn":
        kw["msdcn_mode"] = wl.msdcn_mode
    else:
        kw["softmax"] = wl.softmax
    return kw


def out_hw(wl):
    d = B.make_desc(wl.N, wl.H, wl.W, wl.C, wl.G, 0, (wl.kh, wl.kw), wl.stride, wl.pad,
                    wl.dilation, wl.offset_scale)
    return B.dcn4_out_shape(d)


def problem(orc, wl, N=None):
    return orc.problem(N or wl.N, wl.H, wl.W, wl.C, wl.G, wl.kh, wl.kw, wl.stride, wl.pad,
                       wl.dilation, wl.offset_scale, softmax=wl.softmax,
                       msdcn_dilation=wl.msdcn_mode == "dilation")


def gpu_forward(wl, data, algo="auto"):
    dev = "cuda"
    if wl.kind == "msdcn":
        return B.msdcn_forward(data["input"].to(dev), data["dir_weight"].to(dev),
                               data["scale_raw"].to(dev), data["s0"], wl.smax, group=wl.G,
                               algo=algo, **desc_kw(wl))
    return B.dcn4_forward(data["input"].to(dev), data["offset_weight"].to(dev), group=wl.G,
                          algo=algo, **desc_kw(wl))


def oracle_forward(orc, wl, data, images=None):
    """Oracle output for all images, or for the listed images only."""
    sel = slice(None) if images is None else list(images)
    n = wl.N if images is None else len(images)
    prob = problem(orc, wl, n)
    x = f32(data["input"][sel])
    if wl.kind == "msdcn":
        return orc.msdcn_forward(prob, x, f32(data["dir_weight"][sel]),
                                 f32(data["scale_raw"][sel]), data["s0"].numpy(), wl.smax)
    return orc.forward(prob, x, f32(data["offset_weight"][sel]))


def forward_case(orc, wl, algo="auto", images=None):
    data = make_inputs(wl, out_hw(wl))
    got = f32(gpu_forward(wl, data, algo))
    ref = oracle_forward(orc, wl, data, images)
    if images is not None:
        got = got[list(images)]
    return checked_err(got, ref, wl.dtype, "forward")


def backward_case(orc, wl, algo="auto", images=None, math="default"):
    data = make_inputs(wl, out_hw(wl), with_grad=True)
    dev = "cuda"
    gin, gow = B.dcn4_backward(data["input"].to(dev), data["offset_weight"].to(dev),
                               data["grad_out"].to(dev), group=wl.G, algo=algo, math=math,
                               **desc_kw(wl))
    sel = slice(None) if images is None else list(images)
    n = wl.N if images is None else len(images)
    rgin, rgow = orc.backward(problem(orc, wl, n), f32(data["input"][sel]),
                              f32(data["offset_weight"][sel]), f32(data["grad_out"][sel]))
    gin, gow = f32(gin), f32(gow)
    if images is not None:
        gin, gow = gin[list(images)], gow[list(images)]
    return (checked_err(gin, rgin, wl.dtype, "grad_input"),
            checked_err(gow, rgow, wl.dtype, "grad_offset_weight"))


def msdcn_backward_case(orc, wl, algo="auto", images=None, math="default"):
    """Scaled errors of (grad_input, grad_dir_weight, grad_scale_raw)."""
    data = make_inputs(wl, out_hw(wl), with_grad=True)
    dev = "cuda"
    gin, gdw, graw = B.msdcn_backward(data["input"].to(dev), data["dir_weight"].to(dev),
                                      data["scale_raw"].to(dev), data["s0"], wl.smax,
                                      data["grad_out"].to(dev), group=wl.G, algo=algo, math=math,
                                      **desc_kw(wl))
    sel = slice(None) if images is None else list(images)
    n = wl.N if images is None else len(images)
    r = orc.msdcn_backward(problem(orc, wl, n), f32(data["input"][sel]),
                           f32(data["dir_weight"][sel]), f32(data["scale_raw"][sel]),
                           data["s0"].numpy(), wl.smax, f32(data["grad_out"][sel]))
    got = [f32(gin), f32(gdw), f32(graw)]
    if images is not None:
        got = [t[list(images)] for t in got]
    names = ("grad_input", "grad_dir_weight", "grad_scale_raw")
    return tuple(checked_err(a, b, wl.dtype, n) for a, b, n in zip(got, r, names))


def cuda_sync():
    torch.cuda.synchronize()
