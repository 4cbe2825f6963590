"""Runs one operator of the library a few times on a named workload; the
command profilers (ncu) wrap to capture single kernels.

    python -m deformable_convolution_dcn4_b200.run_op --op forward \
        --workload internimage_bf16 --iters 3 [--N 64] [--algo auto] [--math default]

--op: forward, backward, msdcn (MSDCN forward), msdcn_backward, producer, fused.
msdcn / msdcn_backward on a DCNv4 workload use MSDCN inputs of its shape.
--op producer runs the offset/weight producer (depthwise 3x3 + merged linear)
on the workload's N, H, W, C, G with seeded sub-network weights; --op fused
the sub-network fused into the forward (dcn4_fused_forward) on the same shape.
"""
import argparse
import sys

import torch

from . import _binding as B
from .workloads import WORKLOADS, make_fused_inputs, make_inputs, make_producer_inputs


def main(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--op", choices=["forward", "backward", "msdcn", "msdcn_backward", "producer",
                                    "fused"], default="forward")
    p.add_argument("--workload", default="internimage_bf16")
    p.add_argument("--iters", type=int, default=3)
    p.add_argument("--N", type=int, default=None)
    p.add_argument("--algo", default="auto")
    p.add_argument("--math", default="default")
    p.add_argument("--in-place-escapes", action="store_true",
                   help="forward/msdcn: no escape scratch (one kernel)")
    a = p.parse_args(argv)
    wl = WORKLOADS[a.workload]
    if a.N:
        wl = wl.replace(N=a.N)
    if a.op in ("msdcn", "msdcn_backward") and wl.kind != "msdcn":
        wl = wl.replace(kind="msdcn", offset_dist=("normal", 1.0))
    desc = B.make_desc(wl.N, wl.H, wl.W, wl.C, wl.G, 0, (wl.kh, wl.kw), wl.stride, wl.pad,
                       wl.dilation, wl.offset_scale)
    ho, wo = B.dcn4_out_shape(desc)
    if a.op == "producer":
        d = make_producer_inputs(wl.N, wl.H, wl.W, wl.C, wl.G, wl.kh * wl.kw, wl.dtype,
                                 seed=wl.seed, device="cuda")
    elif a.op == "fused":
        d = make_fused_inputs(wl.N, wl.H, wl.W, wl.C, wl.G, wl.dtype, seed=wl.seed, device="cuda")
    else:
        d = make_inputs(wl, (ho, wo), with_grad=a.op in ("backward", "msdcn_backward"),
                        device="cuda")
    kw = dict(group=wl.G, kernel_size=(wl.kh, wl.kw), stride=wl.stride, pad=wl.pad,
              dilation=wl.dilation, offset_scale=wl.offset_scale, algo=a.algo)
    for _ in range(a.iters):
        if a.op == "forward":
            B.dcn4_forward(d["input"], d["offset_weight"],
                           defer_escapes=not a.in_place_escapes, **kw)
        elif a.op == "producer":
            B.dcn4_offset_producer(d["x"], d["dw_weight"], d["dw_bias"], d["lin_weight"],
                                   d["lin_bias"], group=wl.G, kernel_size=(wl.kh, wl.kw),
                                   stride=wl.stride, pad=wl.pad, dilation=wl.dilation,
                                   algo=a.algo)
        elif a.op == "fused":
            B.dcn4_fused_forward(d["input"], d["x"], d["dw_weight"], d["dw_bias"],
                                 d["lin_weight"], d["lin_bias"], math=a.math, **kw)
        elif a.op == "backward":
            B.dcn4_backward(d["input"], d["offset_weight"], d["grad_out"], math=a.math, **kw)
        elif a.op == "msdcn_backward":
            B.msdcn_backward(d["input"], d["dir_weight"], d["scale_raw"], d["s0"], wl.smax,
                             d["grad_out"], math=a.math, **kw)
        else:
            B.msdcn_forward(d["input"], d["dir_weight"], d["scale_raw"], d["s0"], wl.smax,
                            defer_escapes=not a.in_place_escapes, **kw)
    torch.cuda.synchronize()
    rc, bits = B.dcn4_last_device_error()
    print(f"run_op {a.op} {wl.name} N={wl.N} iters={a.iters}: device error bits {bits}")
    return 0 if rc == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
