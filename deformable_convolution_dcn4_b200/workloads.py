"""Seeded synthetic workloads for DCNv4 / MSDCN.

This module only draws random tensors with the shapes and value
distributions of the workloads the pages discuss; it holds none of the
operator's arithmetic (output sizes are passed in by the caller). Both the
CUDA path's tests/benchmark and the CPU oracle consume the tensors it makes.

Workloads (shapes from the pages' model families, distributions fixed here):
  tiny_f32            N1 16x16 C64 G4, the small parity case
  internimage_bf16/f32  N64 56x56 C128 G8 (D16): an InternImage stage
  ldm64_f16 / ldm32_f16 N8 64x64 C320 G20 and N8 32x32 C640 G40: latent-
                      diffusion U-Net levels (the DCNv4-in-U-Net blog swaps
                      3x3 convs of the high-resolution stages)
  flowdcn_msdcn_bf16  N32 32x32 C1152 G18 (D64): FlowDCN-XL token grid,
                      groupwise multi-scale variant
  highres_bf16        N4 128x128 C256 G16: forward + backward case
Draw order (one torch CPU generator per workload, seeded): input, then the
offsets (dx, dy per tap), then the aggregation weights m, then (MSDCN) the
raw scales, then the output gradient.
"""
import dataclasses
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    H: int
    W: int
    C: int
    G: int
    dtype: str
    kh: int = 3
    kw: int = 3
    stride: Tuple[int, int] = (1, 1)
    pad: Tuple[int, int] = (1, 1)
    dilation: Tuple[int, int] = (1, 1)
    offset_scale: float = 1.0
    offset_dist: Tuple[str, float] = ("normal", 2.0)   # ("normal", sigma) | ("uniform", a)
    weight_sigma: float = 0.3
    kind: str = "dcn4"                                   # "dcn4" | "msdcn"
    smax: float = 8.0
    seed: int = 0
    softmax: bool = False                                # DCNv3 weights (DCNv4 kind only)
    msdcn_mode: str = "offset"                           # "offset" | "dilation" (MSDCN only)

    @property
    def D(self):
        return self.C // self.G

    @property
    def K(self):
        return self.kh * self.kw

    def replace(self, **kw):
        return dataclasses.replace(self, **kw)


WORKLOADS = {w.name: w for w in [
    Workload("tiny_f32", 1, 16, 16, 64, 4, "f32", offset_dist=("normal", 1.5), weight_sigma=0.3),
    Workload("internimage_bf16", 64, 56, 56, 128, 8, "bf16"),
    Workload("internimage_f32", 64, 56, 56, 128, 8, "f32"),
    Workload("ldm64_f16", 8, 64, 64, 320, 20, "f16", offset_dist=("uniform", 4.0), weight_sigma=0.2),
    Workload("ldm32_f16", 8, 32, 32, 640, 40, "f16", offset_dist=("uniform", 4.0), weight_sigma=0.2),
    Workload("flowdcn_msdcn_bf16", 32, 32, 32, 1152, 18, "bf16", offset_dist=("normal", 1.0),
             weight_sigma=0.3, kind="msdcn", smax=8.0),
    Workload("highres_bf16", 4, 128, 128, 256, 16, "bf16"),
]}


def msdcn_s0(G):
    """Per-group scale priors 1, 1, 2, 2, ..., G/2, G/2 (a fixed recipe)."""
    return torch.tensor([1.0 + (g // 2) for g in range(G)], dtype=torch.float32)


def make_producer_inputs(N: int, H: int, W: int, C: int, G: int, K: int = 9,
                         dtype: str = "bf16", seed: int = 0, offset_sigma: float = 2.0,
                         device: Optional[str] = None):
    """Feature map and weights of the offset/weight sub-network (depthwise
    3x3 then one linear layer emitting G*K*3 values per pixel).

    Draw order: x [N,H,W,C] ~ N(0,1); dw_weight [3,3,C] ~ N(0, 1/9);
    dw_bias [C] ~ N(0, 0.1^2); lin_weight [G*K*3, C] ~ N(0, offset_sigma^2/C)
    (outputs of about offset_sigma for unit-size features); lin_bias
    [G*K*3] ~ N(0, 0.1^2). All in the storage dtype.
    """
    g = torch.Generator().manual_seed(seed)
    dt = DTYPES[dtype]
    J = G * K * 3
    out = {
        "x": torch.randn((N, H, W, C), generator=g),
        "dw_weight": torch.randn((3, 3, C), generator=g) / 3.0,
        "dw_bias": torch.randn((C,), generator=g) * 0.1,
        "lin_weight": torch.randn((J, C), generator=g) * (offset_sigma / C ** 0.5),
        "lin_bias": torch.randn((J,), generator=g) * 0.1,
    }
    out = {k: v.to(dt) for k, v in out.items()}
    if device is not None:
        out = {k: v.to(device) for k, v in out.items()}
    return out


def make_fused_inputs(N: int, H: int, W: int, C: int, G: int, dtype: str = "bf16",
                      seed: int = 0, offset_sigma: float = 2.0, device: Optional[str] = None):
    """Inputs of the fused call (offset/weight sub-network in front of the
    aggregation): make_producer_inputs(..., seed) for x and the weights, then
    the sampled map input [N,H,W,C] ~ N(0,1) from a generator seeded seed + 1.
    """
    out = make_producer_inputs(N, H, W, C, G, K=9, dtype=dtype, seed=seed,
                               offset_sigma=offset_sigma)
    g = torch.Generator().manual_seed(seed + 1)
    out["input"] = torch.randn((N, H, W, C), generator=g).to(DTYPES[dtype])
    if device is not None:
        out = {k: v.to(device) for k, v in out.items()}
    return out


def make_inputs(wl: Workload, out_hw: Tuple[int, int], with_grad: bool = False,
                device: Optional[str] = None):
    """Returns a dict of tensors in the workload's storage dtype.

    dcn4 : input [N,H,W,C], offset_weight [N,Ho,Wo,G,K,3] = (dx, dy, m)
    msdcn: input, dir_weight [N,Ho,Wo,G,K,3] = (dir_x, dir_y, m),
           scale_raw [N,Ho,Wo,G], s0 [G] (float32, host-side)
    with_grad adds grad_out [N,Ho,Wo,C].
    """
    Ho, Wo = out_hw
    g = torch.Generator().manual_seed(wl.seed)
    dt = DTYPES[wl.dtype]
    inp = torch.randn((wl.N, wl.H, wl.W, wl.C), generator=g)
    shape = (wl.N, Ho, Wo, wl.G, wl.K)
    kind, a = wl.offset_dist
    if kind == "normal":
        off = torch.randn(shape + (2,), generator=g) * a
    elif kind == "uniform":
        off = (torch.rand(shape + (2,), generator=g) * 2.0 - 1.0) * a
    else:
        raise ValueError(kind)
    m = torch.randn(shape + (1,), generator=g) * wl.weight_sigma
    ow = torch.cat([off, m], dim=-1)
    out = {"input": inp.to(dt)}
    if wl.kind == "msdcn":
        out["dir_weight"] = ow.to(dt)
        out["scale_raw"] = torch.randn((wl.N, Ho, Wo, wl.G), generator=g).to(dt)
        out["s0"] = msdcn_s0(wl.G)
    else:
        out["offset_weight"] = ow.to(dt)
    if with_grad:
        out["grad_out"] = torch.randn((wl.N, Ho, Wo, wl.C), generator=g).to(dt)
    if device is not None:
        out = {k: (v if k == "s0" else v.to(device)) for k, v in out.items()}
    return out
