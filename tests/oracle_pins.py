"""Pins that tie the CPU oracle to facts other than itself.

Each pin takes an `oracle.Oracle` and raises AssertionError on a mismatch.
They are run against the committed oracle (test_oracle_pins.py) and against
deliberately broken copies of it (test_oracle_mutants.py), which each must
trip at least one pin.

What pins what (pages cited by title and section):
  pin_conv          zero offsets + per-tap constant weights == depthwise conv
                    (CANN Conv2D article "2.1 标准卷积的数学表达" written out as a
                    brute-force loop, and torch conv2d(groups=C) in float64)
  pin_grid_sample   one tap, m=1 == torch grid_sample(bilinear, zeros,
                    align_corners=True): bilinear weights + per-corner zeros
  pin_gather        integer offsets == exact integer-indexed gathers
                    (also with offset_scale != 1 and dx != dy)
  pin_fractions     dyadic fractions give exact dyadic mixtures
  pin_out_of_bounds samples outside (-1, W) x (-1, H) contribute nothing
  pin_linearity     linear in the input and in the weights m
  pin_equivariance  integer translation of input + offsets translates output
  pin_msdcn         groupwise multi-scale variant (FlowDCN "3.1"): unit scale
                    reduces bit-exactly to DCNv4; clamp at Smax; softplus values
  pin_cost_model    FLOPs 36HWC, ideal 2HWC+27HWG (~3.7HWC), worst 64HWC (17x),
                    ratio 0.6..9.7 (DCNv4 digest "GPU效率的理论分析")
  pin_adjoint       <f(x), g> == <x, grad_input(g)> and <f(m), g> == <m, grad_m(g)>
  pin_unit_columns  grad_input entries == <f(e_q), g> for unit inputs e_q
  pin_finite_diff   grad dx, dy, m == central differences (exact for a
                    piecewise-linear function away from cell edges)
  pin_msdcn_bwd_unit  MSDCN backward at a clamped unit scale == DCNv4 backward
                    bit for bit, and no gradient reaches raw through the clamp
  pin_msdcn_bwd_adjoint  <f(x), g> == <x, grad_input>, <f(m), g> == <m, grad_m>
  pin_msdcn_bwd_dir central differences for dir at a clamped scale s = 2
                    (exact, dyadic positions): the factor s in d/d dir
  pin_msdcn_bwd_raw central differences for raw below the clamp (smooth:
                    softplus scale, positions kept away from cell edges)
  pin_softmax_box   DCNv3 flag, equal logits: weights 1/K, zero offsets ==
                    box filter (torch conv2d, groups=C, float64)
  pin_softmax_shift adding a constant to a pixel-group's logits changes
                    nothing, even at logits of 800 (exp would overflow); one dominant
                    logit == that tap alone (DCNv4 with a one-hot m)
  pin_softmax_bwd   adjoint for grad_input; central differences for the
                    logits (smooth) and the offsets (exact, dyadic)
  pin_msdcn_dilation  scale-as-dilation reading: s = 1 with dyadic dirs ==
                    DCNv4 bit for bit; s = 2, dir = 0 == DCNv4 at twice the
                    dilation (pad + dilation) bit for bit; backward by central
                    differences (dir exact at s = 2; raw smooth)
  pin_producer      offset/weight producer (DCNv4 digest "方法3. DCN模块的微设计优化":
                    depthwise 3x3 + one merged linear): the depthwise part ==
                    torch conv2d(groups=C) in float64, the linear part == a
                    float64 matmul, the composition == conv2d + F.linear, and
                    a constant map through all-ones taps counts the in-image
                    taps exactly (4 at corners, 6 on edges, 9 inside)
"""
import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _ow(o, prob, rng, offsets=None, m=None):
    Ho, Wo = o.out_hw(prob)
    K = prob.kh * prob.kw
    shape = (prob.N, Ho, Wo, prob.G, K)
    ow = np.zeros(shape + (3,), np.float32)
    ow[..., :2] = rng.standard_normal(shape + (2,)) if offsets is None else offsets
    ow[..., 2] = rng.standard_normal(shape) if m is None else m
    return ow


def _close(a, b, rtol, what):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    scale = max(np.abs(b).max(), 1e-300)
    err = np.abs(a - b).max() / scale
    assert err <= rtol, f"{what}: scaled error {err:.3e} > {rtol:.1e}"


CONV_CASES = [
    # N, H, W, C, G, kh, kw, stride, pad, dilation
    (2, 7, 9, 6, 3, 3, 3, (1, 1), (1, 1), (1, 1)),
    (1, 8, 8, 4, 2, 3, 3, (2, 2), (1, 1), (1, 1)),
    (1, 9, 7, 4, 4, 3, 3, (1, 1), (2, 2), (2, 2)),
    (1, 6, 6, 2, 1, 5, 5, (1, 1), (2, 2), (1, 1)),
    (1, 5, 5, 3, 3, 1, 1, (1, 1), (0, 0), (1, 1)),
    (1, 7, 8, 4, 2, 3, 2, (1, 2), (1, 0), (1, 1)),
    (1, 10, 6, 6, 2, 2, 3, (2, 1), (0, 2), (2, 1)),
]


def _conv_bruteforce(x, w, stride, pad, dil):
    """out[y][x][c] = sum_i sum_j in[y*s+i*d-p][x*s+j*d-p][c] * w[i][j][c]."""
    N, H, W, C = x.shape
    kh, kw = w.shape[:2]
    Ho = (H + 2 * pad[0] - dil[0] * (kh - 1) - 1) // stride[0] + 1
    Wo = (W + 2 * pad[1] - dil[1] * (kw - 1) - 1) // stride[1] + 1
    out = np.zeros((N, Ho, Wo, C))
    for n in range(N):
        for yo in range(Ho):
            for xo in range(Wo):
                for i in range(kh):
                    for j in range(kw):
                        yy = yo * stride[0] + i * dil[0] - pad[0]
                        xx = xo * stride[1] + j * dil[1] - pad[1]
                        if 0 <= yy < H and 0 <= xx < W:
                            out[n, yo, xo] += x[n, yy, xx].astype(np.float64) * w[i, j]
    return out


def pin_conv(o):
    for ci, (N, H, W, C, G, kh, kw, st, pd, dl) in enumerate(CONV_CASES):
        rng = _rng(100 + ci)
        prob = o.problem(N, H, W, C, G, kh, kw, st, pd, dl)
        Ho, Wo = o.out_hw(prob)
        D = C // G
        x = rng.standard_normal((N, H, W, C)).astype(np.float32)
        mk = rng.standard_normal((G, kh * kw)).astype(np.float32)
        m = np.broadcast_to(mk, (N, Ho, Wo, G, kh * kw))
        ow = _ow(o, prob, rng, offsets=0.0, m=m)
        got = o.forward(prob, x, ow)
        w = np.zeros((kh, kw, C))
        for c in range(C):
            w[:, :, c] = mk[c // D].reshape(kh, kw)
        _close(got, _conv_bruteforce(x, w, st, pd, dl), 1e-12, f"conv case {ci} vs loop")
        wt = torch.from_numpy(np.ascontiguousarray(w.transpose(2, 0, 1)[:, None]))
        ref = F.conv2d(torch.from_numpy(x.astype(np.float64)).permute(0, 3, 1, 2), wt,
                       stride=st, padding=pd, dilation=dl, groups=C)
        _close(got, ref.permute(0, 2, 3, 1).numpy(), 1e-12, f"conv case {ci} vs torch")


def pin_grid_sample(o):
    rng = _rng(7)
    for (H, W) in [(9, 11), (6, 5)]:
        N, C, G = 2, 6, 3
        D = C // G
        prob = o.problem(N, H, W, C, G, 1, 1, (1, 1), (0, 0), (1, 1))
        x = rng.standard_normal((N, H, W, C)).astype(np.float32)
        offs = rng.uniform(-3, 3, (N, H, W, G, 1, 2)).astype(np.float32)
        ow = _ow(o, prob, rng, offsets=offs, m=1.0)
        got = o.forward(prob, x, ow)
        xs = np.arange(W, dtype=np.float32)[None, None, :, None] + offs[..., 0, 0]
        ys = np.arange(H, dtype=np.float32)[None, :, None, None] + offs[..., 0, 1]
        ref = np.zeros_like(got)
        xt = torch.from_numpy(x.astype(np.float64)).permute(0, 3, 1, 2)
        for g in range(G):
            gx = 2.0 * xs[..., g].astype(np.float64) / (W - 1) - 1.0
            gy = 2.0 * ys[..., g].astype(np.float64) / (H - 1) - 1.0
            grid = torch.from_numpy(np.stack([gx, gy], -1))
            r = F.grid_sample(xt[:, g * D:(g + 1) * D], grid, mode="bilinear",
                              padding_mode="zeros", align_corners=True)
            ref[..., g * D:(g + 1) * D] = r.permute(0, 2, 3, 1).numpy()
        _close(got, ref, 1e-12, f"grid_sample {H}x{W}")


def pin_gather(o):
    for os_ in (1.0, 2.0):
        rng = _rng(11 + int(os_))
        N, H, W, C, G = 2, 8, 10, 8, 4
        D = C // G
        prob = o.problem(N, H, W, C, G, 3, 3, offset_scale=os_)
        Ho, Wo = o.out_hw(prob)
        x = rng.standard_normal((N, H, W, C)).astype(np.float32)
        offs = rng.integers(-3, 4, (N, Ho, Wo, G, 9, 2)).astype(np.float32)
        # (a) one tap with m = 1: an exact copy of a shifted pixel (or zero)
        for tap in (0, 4, 7):
            m = np.zeros((N, Ho, Wo, G, 9), np.float32)
            m[..., tap] = 1.0
            got = o.forward(prob, x, _ow(o, prob, rng, offsets=offs, m=m))
            i, j = divmod(tap, 3)
            ref = np.zeros_like(got)
            for n in range(N):
                for yo in range(Ho):
                    for xo in range(Wo):
                        for g in range(G):
                            yy = yo - 1 + i + int(offs[n, yo, xo, g, tap, 1] * os_)
                            xx = xo - 1 + j + int(offs[n, yo, xo, g, tap, 0] * os_)
                            if 0 <= yy < H and 0 <= xx < W:
                                ref[n, yo, xo, g * D:(g + 1) * D] = x[n, yy, xx, g * D:(g + 1) * D]
            assert np.array_equal(got, ref), f"single-tap integer gather (tap {tap}, os {os_})"
        # (b) all taps, random m: exact integer-indexed weighted sum
        m = rng.standard_normal((N, Ho, Wo, G, 9)).astype(np.float32)
        got = o.forward(prob, x, _ow(o, prob, rng, offsets=offs, m=m))
        ref = np.zeros_like(got)
        for n in range(N):
            for yo in range(Ho):
                for xo in range(Wo):
                    for g in range(G):
                        for k in range(9):
                            i, j = divmod(k, 3)
                            yy = yo - 1 + i + int(offs[n, yo, xo, g, k, 1] * os_)
                            xx = xo - 1 + j + int(offs[n, yo, xo, g, k, 0] * os_)
                            if 0 <= yy < H and 0 <= xx < W:
                                ref[n, yo, xo, g * D:(g + 1) * D] += \
                                    float(m[n, yo, xo, g, k]) * x[n, yy, xx, g * D:(g + 1) * D].astype(np.float64)
        _close(got, ref, 1e-12, f"integer gather, all taps, os {os_}")


def pin_fractions(o):
    """dx = t + 1/4 must give 3/4 of column x0 and 1/4 of column x0+1 (exactly),
    dy = t + 3/4 likewise along H; corners outside the image count as zero."""
    N, H, W, C, G = 1, 6, 7, 2, 1
    prob = o.problem(N, H, W, C, G, 1, 1, (1, 1), (0, 0), (1, 1))
    rng = _rng(5)
    x = rng.integers(-8, 9, (N, H, W, C)).astype(np.float32)
    for fx, fy in [(0.25, 0.0), (0.0, 0.75), (0.25, 0.75), (-0.75, 0.5)]:
        offs = np.zeros((N, H, W, G, 1, 2), np.float32)
        offs[..., 0] = fx
        offs[..., 1] = fy
        got = o.forward(prob, x, _ow(o, prob, rng, offsets=offs, m=1.0))
        ref = np.zeros_like(got)
        for yo in range(H):
            for xo in range(W):
                sx, sy = xo + fx, yo + fy
                x0, y0 = math.floor(sx), math.floor(sy)
                lx, ly = sx - x0, sy - y0
                for a, wy in ((0, 1 - ly), (1, ly)):
                    for b, wx in ((0, 1 - lx), (1, lx)):
                        yy, xx = y0 + a, x0 + b
                        if 0 <= yy < H and 0 <= xx < W:
                            ref[0, yo, xo] += wy * wx * x[0, yy, xx]
        assert np.array_equal(got, ref), f"dyadic fractions ({fx}, {fy})"
    # a sample at x = -0.5 keeps half of column 0
    offs = np.zeros((N, H, W, G, 1, 2), np.float32)
    offs[..., 0] = -0.5 - np.arange(W, dtype=np.float32)[None, None, :, None, None]
    got = o.forward(prob, x, _ow(o, prob, rng, offsets=offs, m=1.0))
    assert np.array_equal(got, 0.5 * np.repeat(x[:, :, :1], W, axis=2)), "x = -0.5"


def pin_out_of_bounds(o):
    N, H, W, C, G = 1, 5, 6, 4, 2
    prob = o.problem(N, H, W, C, G, 3, 3)
    rng = _rng(9)
    x = rng.standard_normal((N, H, W, C)).astype(np.float32)
    offs = np.zeros((N, H, W, G, 9, 2), np.float32)
    offs[..., 0] = -(W + 5)
    got = o.forward(prob, x, _ow(o, prob, rng, offsets=offs))
    assert np.all(got == 0.0), "all samples left of the image must give zero"
    offs[..., 0] = 0.0
    offs[..., 1] = H + 3
    got = o.forward(prob, x, _ow(o, prob, rng, offsets=offs))
    assert np.all(got == 0.0), "all samples below the image must give zero"
    # x = W-1 exactly -> weight 1 on the last column; x = W - 0.5 -> 0.5
    prob1 = o.problem(N, H, W, C, G, 1, 1, (1, 1), (0, 0), (1, 1))
    for frac, wt in ((0.0, 1.0), (0.5, 0.5)):
        offs = np.zeros((N, H, W, G, 1, 2), np.float32)
        offs[..., 0] = (W - 1 + frac) - np.arange(W, dtype=np.float32)[None, None, :, None, None]
        got = o.forward(prob1, x, _ow(o, prob1, rng, offsets=offs, m=1.0))
        assert np.array_equal(got, wt * np.repeat(x[:, :, -1:], W, axis=2)), f"x = W-1+{frac}"


def pin_linearity(o):
    rng = _rng(21)
    prob = o.problem(2, 9, 8, 12, 3, 3, 3)
    # short dyadic values, so alpha*a + beta*b is exact in fp32
    a = (rng.integers(-64, 65, (2, 9, 8, 12)) / 8.0).astype(np.float32)
    b = (rng.integers(-64, 65, (2, 9, 8, 12)) / 8.0).astype(np.float32)
    ow = _ow(o, prob, rng)
    ow[..., :2] *= 2.0
    ow[..., 2] = rng.integers(-64, 65, ow[..., 2].shape) / 16.0
    alpha, beta = 0.5, -2.0
    lhs = o.forward(prob, alpha * a + beta * b, ow)
    rhs = alpha * o.forward(prob, a, ow) + beta * o.forward(prob, b, ow)
    _close(lhs, rhs, 1e-12, "linearity in the input")
    ow2 = ow.copy()
    ow2[..., 2] = rng.integers(-64, 65, ow[..., 2].shape) / 16.0
    ow3 = ow.copy()
    ow3[..., 2] = alpha * ow[..., 2] + beta * ow2[..., 2]
    _close(o.forward(prob, a, ow3),
           alpha * o.forward(prob, a, ow) + beta * o.forward(prob, a, ow2), 1e-12,
           "linearity in m")


def pin_equivariance(o):
    rng = _rng(31)
    N, H, W, C, G = 1, 20, 22, 4, 2
    prob = o.problem(N, H, W, C, G, 3, 3)
    x = rng.standard_normal((N, H, W, C)).astype(np.float32)
    offs = rng.uniform(-1.5, 1.5, (N, H, W, G, 9, 2)).astype(np.float32)
    ow = _ow(o, prob, rng, offsets=offs)
    ty, tx = 3, 2
    xs = np.zeros_like(x)
    xs[:, ty:, tx:] = x[:, :H - ty, :W - tx]
    ows = np.zeros_like(ow)
    ows[:, ty:, tx:] = ow[:, :H - ty, :W - tx]
    y = o.forward(prob, x, ow)
    ys = o.forward(prob, xs, ows)
    m = 5  # margin: samples reach at most 1 + 1.5 + 1 pixels
    _close(ys[:, ty + m:H - m, tx + m:W - m], y[:, m:H - m - ty, m:W - m - tx], 1e-6,
           "translation equivariance")


def pin_msdcn(o):
    rng = _rng(41)
    N, H, W, C, G = 2, 9, 10, 8, 4
    prob = o.problem(N, H, W, C, G, 3, 3)
    Ho, Wo = o.out_hw(prob)
    x = rng.standard_normal((N, H, W, C)).astype(np.float32)
    dw = _ow(o, prob, rng)
    dw[..., :2] *= 1.7
    # unit scale: softplus(30) ~ 30, clamped to Smax = 1 -> exactly DCNv4
    raw = np.full((N, Ho, Wo, G), 30.0, np.float32)
    got = o.msdcn_forward(prob, x, dw, raw, np.ones(G, np.float32), 1.0)
    assert np.array_equal(got, o.forward(prob, x, dw)), "unit scale must reduce to DCNv4"
    # clamp: every scale exceeds Smax = 2.5 -> offsets are fp32(2.5 * dir)
    raw = rng.uniform(2.0, 6.0, (N, Ho, Wo, G)).astype(np.float32)
    s0 = np.full(G, 4.0, np.float32)
    got = o.msdcn_forward(prob, x, dw, raw, s0, 2.5)
    ow = dw.copy()
    ow[..., :2] = (np.float32(2.5) * dw[..., :2]).astype(np.float32)
    assert np.array_equal(got, o.forward(prob, x, ow)), "clamped scale"
    # general scale: s computed here in float64, rounded to fp32
    raw = rng.standard_normal((N, Ho, Wo, G)).astype(np.float32)
    s0 = np.array([1 + g // 2 for g in range(G)], np.float32)
    smax = 2.2
    r = raw.astype(np.float64)
    s = np.minimum(s0.astype(np.float64) * np.log1p(np.exp(r)), smax).astype(np.float32)
    ow = dw.copy()
    ow[..., :2] = (s[..., None, None] * dw[..., :2]).astype(np.float32)
    _close(o.msdcn_forward(prob, x, dw, raw, s0, smax), o.forward(prob, x, ow), 1e-5,
           "general scale")
    # the scale function itself
    assert abs(o.msdcn_scale(0.0, 3.0, 100.0) - 3.0 * math.log(2.0)) < 1e-6
    assert abs(o.msdcn_scale(20.0, 2.0, 100.0) - 40.0) < 1e-5
    assert abs(o.msdcn_scale(-20.0, 1.0, 100.0) / math.exp(-20.0) - 1.0) < 1e-5
    assert abs(o.msdcn_scale(-1.0, 1.0, 100.0) - math.log1p(math.exp(-1.0))) < 1e-6
    assert o.msdcn_scale(5.0, 1.0, 2.0) == 2.0
    assert math.isnan(o.msdcn_scale(float("nan"), 1.0, 8.0))


def pin_cost_model(o):
    with open(os.path.join(GOLDEN, "cost_model.json")) as f:
        page = json.load(f)
    H, W, C = 56, 48, 128
    G = C // 16
    prob = o.problem(1, H, W, C, G, 3, 3)
    HWC = H * W * C
    assert o.flops(prob) == page["flops_per_HWC"] * HWC
    ideal = o.ideal_bytes(prob, 1)
    assert ideal == page["ideal"]["HWC"] * HWC + page["ideal"]["HWG"] * H * W * G
    assert abs(ideal / HWC - page["ideal_at_G_C_over_16_HWC"]) < 0.02
    worst = o.worst_bytes(prob, 1)
    assert worst == page["worst_HWC"] * HWC
    assert round(worst / ideal) == page["worst_over_ideal"]
    lo, hi = page["compute_to_memory_ratio"]
    assert abs(o.flops(prob) / worst - lo) < 0.05
    assert abs(page["flops_per_HWC"] / page["ideal_at_G_C_over_16_HWC"] - hi) < 0.05
    assert o.ideal_bytes(prob, 2) == 2 * ideal  # bytes scale with the element size
    prob5 = o.problem(2, 10, 12, 8, 2, 5, 5, (1, 1), (2, 2), (1, 1))
    assert o.flops(prob5) == 4 * 25 * 2 * 10 * 12 * 8


def _bwd_case(o, seed, os_=1.0, stride=(1, 1), pad=(1, 1), dil=(1, 1), kh=3, kw=3):
    rng = _rng(seed)
    N, H, W, C, G = 2, 7, 8, 6, 3
    prob = o.problem(N, H, W, C, G, kh, kw, stride, pad, dil, offset_scale=os_)
    x = rng.standard_normal((N, H, W, C)).astype(np.float32)
    ow = _ow(o, prob, rng)
    ow[..., :2] *= 2.0
    Ho, Wo = o.out_hw(prob)
    go = rng.standard_normal((N, Ho, Wo, C)).astype(np.float32)
    return prob, x, ow, go


def pin_adjoint(o):
    for seed, kw in ((51, {}), (52, {"os_": 0.5, "stride": (2, 1), "dil": (1, 2)})):
        prob, x, ow, go = _bwd_case(o, seed, **kw)
        gin, gow = o.backward(prob, x, ow, go)
        lhs = float(np.sum(o.forward(prob, x, ow) * go))
        rhs_x = float(np.sum(x.astype(np.float64) * gin))
        rhs_m = float(np.sum(ow[..., 2].astype(np.float64) * gow[..., 2]))
        assert abs(lhs - rhs_x) <= 1e-11 * max(1.0, abs(lhs)), "<f(x), g> vs <x, grad_input>"
        assert abs(lhs - rhs_m) <= 1e-11 * max(1.0, abs(lhs)), "<f(m), g> vs <m, grad_m>"


def pin_unit_columns(o):
    prob, x, ow, go = _bwd_case(o, 61)
    gin, _ = o.backward(prob, x, ow, go)
    rng = _rng(62)
    for _ in range(12):
        q = tuple(int(rng.integers(0, s)) for s in x.shape)
        e = np.zeros_like(x)
        e[q] = 1.0
        col = float(np.sum(o.forward(prob, e, ow) * go))
        assert abs(col - gin[q]) <= 1e-12 * max(1.0, abs(col)), f"grad_input at {q}"


def pin_finite_diff(o):
    """Offsets are odd multiples of 1/512, so x +- 1/1024 stays inside one
    bilinear cell and every position is exact in fp32; the central difference
    of a function linear in x is then exact up to fp64 rounding."""
    for seed, os_ in ((71, 1.0), (72, 0.5)):
        prob, x, ow, go = _bwd_case(o, seed, os_=os_)
        rng = _rng(seed + 100)
        ow[..., :2] = (2 * rng.integers(-900, 900, ow[..., :2].shape) + 1) / 512.0
        gin, gow = o.backward(prob, x, ow, go)
        h = 1.0 / 1024.0
        for _ in range(24):
            idx = tuple(int(rng.integers(0, s)) for s in ow.shape[:-1])
            for comp in range(3):
                hh = h / os_ if comp < 2 else h
                op, om = ow.copy(), ow.copy()
                op[idx + (comp,)] += hh
                om[idx + (comp,)] -= hh
                fd = (np.sum(o.forward(prob, x, op) * go) -
                      np.sum(o.forward(prob, x, om) * go)) / (2 * hh)
                an = gow[idx + (comp,)]
                assert abs(fd - an) <= 1e-8 * max(1.0, abs(an)), \
                    f"finite difference at {idx} comp {comp}: {fd} vs {an}"


def _msdcn_case(o, seed, N=2, H=7, W=8, C=6, G=3, os_=1.0):
    rng = _rng(seed)
    prob = o.problem(N, H, W, C, G, 3, 3, offset_scale=os_)
    Ho, Wo = o.out_hw(prob)
    x = rng.standard_normal((N, H, W, C)).astype(np.float32)
    dw = _ow(o, prob, rng)
    raw = rng.standard_normal((N, Ho, Wo, G)).astype(np.float32)
    go = rng.standard_normal((N, Ho, Wo, C)).astype(np.float32)
    s0 = np.array([1 + g // 2 for g in range(G)], np.float32)
    return prob, x, dw, raw, s0, go


def pin_msdcn_bwd_unit(o):
    """s0 = 1, raw = 30, Smax = 1: s is exactly 1 (clamped), so the MSDCN
    gradients are DCNv4's with offsets = dir, and raw gets none."""
    prob, x, dw, raw, s0, go = _msdcn_case(o, 81, os_=0.75)
    raw[...] = 30.0
    gin, gdw, graw = o.msdcn_backward(prob, x, dw, raw, np.ones(prob.G, np.float32), 1.0, go)
    rgin, rgow = o.backward(prob, x, dw, go)
    assert np.array_equal(gin, rgin), "grad_input at unit scale"
    assert np.array_equal(gdw, rgow), "grad_dir_weight at unit scale"
    assert np.all(graw == 0.0), "no gradient through an active clamp"


def pin_msdcn_bwd_adjoint(o):
    prob, x, dw, raw, s0, go = _msdcn_case(o, 82)
    smax = 2.5
    gin, gdw, _ = o.msdcn_backward(prob, x, dw, raw, s0, smax, go)
    lhs = float(np.sum(o.msdcn_forward(prob, x, dw, raw, s0, smax) * go))
    rhs_x = float(np.sum(x.astype(np.float64) * gin))
    rhs_m = float(np.sum(dw[..., 2].astype(np.float64) * gdw[..., 2]))
    assert abs(lhs - rhs_x) <= 1e-11 * max(1.0, abs(lhs)), "<f(x), g> vs <x, grad_input>"
    assert abs(lhs - rhs_m) <= 1e-11 * max(1.0, abs(lhs)), "<f(m), g> vs <m, grad_m>"


def pin_msdcn_bwd_dir(o):
    """Scale clamped at exactly 2 (s0 = 4, raw >= 1, Smax = 2). dir values are
    odd multiples of 1/1024, so s * dir is an odd multiple of 1/512 and a
    step of 1/2048 in dir moves the sample by 1/1024 inside one bilinear
    cell: the central difference is exact up to fp64 rounding."""
    for seed, os_ in ((83, 1.0), (84, 0.5)):
        prob, x, dw, raw, s0, go = _msdcn_case(o, seed, os_=os_)
        rng = _rng(seed + 100)
        raw = rng.uniform(1.0, 3.0, raw.shape).astype(np.float32)
        s0 = np.full(prob.G, 4.0, np.float32)
        dw[..., :2] = (2 * rng.integers(-900, 900, dw[..., :2].shape) + 1) / 1024.0
        gin, gdw, graw = o.msdcn_backward(prob, x, dw, raw, s0, 2.0, go)
        assert np.all(graw == 0.0)
        h = 1.0 / 2048.0
        for _ in range(20):
            idx = tuple(int(rng.integers(0, s)) for s in dw.shape[:-1])
            for comp in range(3):
                hh = h / os_ if comp < 2 else h
                dp, dm = dw.copy(), dw.copy()
                dp[idx + (comp,)] += hh
                dm[idx + (comp,)] -= hh
                fd = (np.sum(o.msdcn_forward(prob, x, dp, raw, s0, 2.0) * go) -
                      np.sum(o.msdcn_forward(prob, x, dm, raw, s0, 2.0) * go)) / (2 * hh)
                an = gdw[idx + (comp,)]
                assert abs(fd - an) <= 1e-8 * max(1.0, abs(an)), \
                    f"d/d dir at {idx} comp {comp}: {fd} vs {an}"


def pin_msdcn_bwd_raw(o):
    """Below the clamp the loss is a smooth function of raw near the drawn
    point as long as no sample crosses a cell edge. Samples are kept at least
    0.05 px from every edge (directions redrawn until they are), the step is
    1e-3 (moves a sample by < 0.02 px); the central difference then matches
    up to O(h^2) and the fp32 rounding of positions (relative ~1e-4)."""
    prob, x, dw, raw, s0, go = _msdcn_case(o, 85, N=1, H=6, W=6, C=4, G=2)
    Ho, Wo = o.out_hw(prob)
    smax = 50.0
    rng = _rng(185)
    s = np.array([[[[o.msdcn_scale(raw[n, i, j, g], s0[g], smax) for g in range(prob.G)]
                    for j in range(Wo)] for i in range(Ho)] for n in range(prob.N)], np.float64)
    for n in range(prob.N):
        for i in range(Ho):
            for j in range(Wo):
                for g in range(prob.G):
                    for k in range(9):
                        while True:
                            d = rng.standard_normal(2)
                            px = j - 1 + k % 3 + s[n, i, j, g] * d[0]
                            py = i - 1 + k // 3 + s[n, i, j, g] * d[1]
                            fx, fy = px - math.floor(px), py - math.floor(py)
                            if 0.05 < fx < 0.95 and 0.05 < fy < 0.95:
                                break
                        dw[n, i, j, g, k, :2] = d
    _, _, graw = o.msdcn_backward(prob, x, dw, raw, s0, smax, go)
    h = 1e-3
    for idx in np.ndindex(raw.shape):
        rp, rm = raw.copy(), raw.copy()
        rp[idx] += h
        rm[idx] -= h
        fd = (np.sum(o.msdcn_forward(prob, x, dw, rp, s0, smax) * go) -
              np.sum(o.msdcn_forward(prob, x, dw, rm, s0, smax) * go)) / (float(rp[idx]) - float(rm[idx]))
        an = graw[idx]
        assert abs(fd - an) <= 2e-3 * max(1.0, abs(an)), f"d/d raw at {idx}: {fd} vs {an}"


def pin_msdcn_bwd_nan(o):
    """A (pixel, group) whose scale is NaN, and a tap pushed far outside the
    image, contribute nothing (the zero-outside reading applied to the
    FlowDCN "3.1" chain rule): their direction, weight and raw-scale
    gradients are exactly 0, grad_input equals that of the same problem with
    their weights m set to 0, every other gradient is bit-identical to the
    problem without the NaN, and the adjoint identity holds."""
    prob, x, dw, raw, s0, go = _msdcn_case(o, 86)
    smax = 3.0
    nan_at = (1, 2, 3, 1)   # (n, ho, wo, g) with raw = NaN
    far_at = (0, 4, 5, 2)   # (n, ho, wo, g) whose tap 4 leaves the image
    raw[nan_at] = np.nan
    dw[far_at + (4, 0)] = -1000.0
    gin, gdw, graw = o.msdcn_backward(prob, x, dw, raw, s0, smax, go)
    assert np.all(gdw[nan_at] == 0.0), "NaN scale: direction/weight gradients"
    assert graw[nan_at] == 0.0, "NaN scale: raw gradient"
    assert np.all(gdw[far_at + (4,)] == 0.0), "tap outside the image: its gradients"
    assert np.all(np.isfinite(gin)) and np.all(np.isfinite(gdw)) and np.all(np.isfinite(graw))
    # the same problem with the two contributions removed through m = 0
    raw2, dw2 = raw.copy(), dw.copy()
    raw2[nan_at] = 0.25
    dw2[nan_at + (slice(None), 2)] = 0.0
    dw2[far_at + (4, 2)] = 0.0
    rgin, rgdw, rgraw = o.msdcn_backward(prob, x, dw2, raw2, s0, smax, go)
    assert np.array_equal(gin, rgin), "grad_input without the two contributions"
    keep = np.ones(raw.shape, bool)
    keep[nan_at] = False
    assert np.array_equal(graw[keep], rgraw[keep]), "raw gradients of the other pairs"
    assert np.array_equal(gdw[keep], rgdw[keep]), "dir/weight gradients of the other pairs"
    lhs = float(np.sum(o.msdcn_forward(prob, x, dw, raw, s0, smax) * go))
    rhs = float(np.sum(x.astype(np.float64) * gin))
    assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs)), "adjoint with a NaN scale"


def _box(x, K, stride, pad, dil, kh=3, kw=3):
    """Depthwise conv with every weight 1/K (float64, torch)."""
    C = x.shape[-1]
    xt = torch.from_numpy(x.astype(np.float64)).permute(0, 3, 1, 2)
    w = torch.full((C, 1, kh, kw), 1.0 / K, dtype=torch.float64)
    return F.conv2d(xt, w, stride=stride, padding=pad, dilation=dil, groups=C).permute(0, 2, 3, 1).numpy()


def pin_softmax_box(o):
    rng = _rng(91)
    for (N, H, W, C, G, st, pd, dl) in [(2, 7, 9, 6, 3, (1, 1), (1, 1), (1, 1)),
                                        (1, 9, 8, 4, 2, (2, 1), (2, 1), (2, 1))]:
        prob = o.problem(N, H, W, C, G, 3, 3, st, pd, dl, softmax=True)
        x = rng.standard_normal((N, H, W, C)).astype(np.float32)
        Ho, Wo = o.out_hw(prob)
        logit = rng.standard_normal((N, Ho, Wo, G, 1)).astype(np.float32)
        ow = _ow(o, prob, rng, offsets=0.0, m=np.broadcast_to(logit, (N, Ho, Wo, G, 9)))
        _close(o.forward(prob, x, ow), _box(x, 9, st, pd, dl), 1e-12, "softmax of equal logits")


def pin_softmax_shift(o):
    rng = _rng(92)
    N, H, W, C, G = 2, 6, 7, 4, 2
    prob = o.problem(N, H, W, C, G, 3, 3, softmax=True)
    x = rng.standard_normal((N, H, W, C)).astype(np.float32)
    ow = _ow(o, prob, rng)
    ow[..., :2] *= 1.5
    ref = o.forward(prob, x, ow)
    for c in (3.0, 800.0):
        sh = ow.copy()
        sh[..., 2] = (sh[..., 2].astype(np.float64) + c).astype(np.float32)
        got = o.forward(prob, x, sh)
        assert np.all(np.isfinite(got)), f"logits + {c}: overflow"
        # the shifted fp32 logits differ from the originals by rounding, so
        # compare against the softmax weights of the shifted values
        back = sh.copy()
        back[..., 2] = (sh[..., 2].astype(np.float64) - c).astype(np.float32)
        _close(got, o.forward(prob, x, back), 1e-12, f"logits + {c}")
    one = ow.copy()
    k = 4
    one[..., 2] = 0.0
    one[..., k, 2] = 60.0
    hot = ow.copy()
    hot[..., 2] = 0.0
    hot[..., k, 2] = 1.0
    plain = o.problem(N, H, W, C, G, 3, 3)
    _close(o.forward(prob, x, one), o.forward(plain, x, hot), 1e-12, "one dominant logit")


def pin_softmax_bwd(o):
    rng = _rng(93)
    N, H, W, C, G = 2, 7, 8, 6, 3
    prob = o.problem(N, H, W, C, G, 3, 3, softmax=True)
    x = rng.standard_normal((N, H, W, C)).astype(np.float32)
    ow = _ow(o, prob, rng)
    ow[..., :2] = (2 * rng.integers(-900, 900, ow[..., :2].shape) + 1) / 512.0
    Ho, Wo = o.out_hw(prob)
    go = rng.standard_normal((N, Ho, Wo, C)).astype(np.float32)
    gin, gow = o.backward(prob, x, ow, go)
    lhs = float(np.sum(o.forward(prob, x, ow) * go))
    rhs = float(np.sum(x.astype(np.float64) * gin))
    assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs)), "<f(x), g> vs <x, grad_input>"
    # the logit gradients of one pixel-group sum to zero (softmax is shift-invariant)
    assert np.abs(gow[..., 2].sum(axis=-1)).max() <= 1e-12 * max(1.0, np.abs(gow[..., 2]).max())
    for _ in range(20):
        idx = tuple(int(rng.integers(0, s)) for s in ow.shape[:-1])
        for comp, h in ((0, 1.0 / 1024.0), (1, 1.0 / 1024.0), (2, 1e-4)):
            op, om = ow.copy(), ow.copy()
            op[idx + (comp,)] += h
            om[idx + (comp,)] -= h
            step = float(op[idx + (comp,)]) - float(om[idx + (comp,)])
            fd = (np.sum(o.forward(prob, x, op) * go) - np.sum(o.forward(prob, x, om) * go)) / step
            an = gow[idx + (comp,)]
            tol = 1e-8 if comp < 2 else 1e-6
            assert abs(fd - an) <= tol * max(1.0, abs(an)), f"softmax FD at {idx} comp {comp}: {fd} vs {an}"


def pin_msdcn_dilation(o):
    rng = _rng(94)
    N, H, W, C, G = 2, 9, 10, 8, 4
    for st, pd, dl in (((1, 1), (1, 1), (1, 1)), ((2, 1), (2, 1), (1, 2))):
        prob = o.problem(N, H, W, C, G, 3, 3, st, pd, dl, msdcn_dilation=True)
        Ho, Wo = o.out_hw(prob)
        x = rng.standard_normal((N, H, W, C)).astype(np.float32)
        dw = _ow(o, prob, rng)
        dw[..., :2] = rng.integers(-200, 200, dw[..., :2].shape) / 64.0
        ones = np.ones(G, np.float32)
        raw = np.full((N, Ho, Wo, G), 30.0, np.float32)
        got = o.msdcn_forward(prob, x, dw, raw, ones, 1.0)  # s = 1 exactly
        plain = o.problem(N, H, W, C, G, 3, 3, st, pd, dl)
        assert np.array_equal(got, o.forward(plain, x, dw)), "dilation reading at s = 1"
        zero = dw.copy()
        zero[..., :2] = 0.0
        got = o.msdcn_forward(prob, x, zero, raw, np.full(G, 4.0, np.float32), 2.0)  # s = 2
        wide = o.problem(N, H, W, C, G, 3, 3, st, (pd[0] + dl[0], pd[1] + dl[1]),
                         (2 * dl[0], 2 * dl[1]))
        assert o.out_hw(wide) == (Ho, Wo)
        assert np.array_equal(got, o.forward(wide, x, zero)), "s = 2 is twice the dilation"
    # backward: dir by exact central differences at s = 2, raw smoothly
    prob = o.problem(1, 7, 8, 6, 3, 3, 3, msdcn_dilation=True, offset_scale=0.5)
    Ho, Wo = o.out_hw(prob)
    x = rng.standard_normal((1, 7, 8, 6)).astype(np.float32)
    dw = _ow(o, prob, rng)
    dw[..., :2] = (2 * rng.integers(-300, 300, dw[..., :2].shape) + 1) / 512.0
    go = rng.standard_normal((1, Ho, Wo, 6)).astype(np.float32)
    s0 = np.full(3, 4.0, np.float32)
    raw = rng.uniform(1.0, 3.0, (1, Ho, Wo, 3)).astype(np.float32)
    _, gdw, graw = o.msdcn_backward(prob, x, dw, raw, s0, 2.0, go)
    assert np.all(graw == 0.0)
    h = 1.0 / 2048.0
    for _ in range(16):
        idx = tuple(int(rng.integers(0, s)) for s in dw.shape[:-1])
        for comp in range(3):
            hh = h / 0.5 if comp < 2 else h
            dp, dm = dw.copy(), dw.copy()
            dp[idx + (comp,)] += hh
            dm[idx + (comp,)] -= hh
            fd = (np.sum(o.msdcn_forward(prob, x, dp, raw, s0, 2.0) * go) -
                  np.sum(o.msdcn_forward(prob, x, dm, raw, s0, 2.0) * go)) / (2 * hh)
            an = gdw[idx + (comp,)]
            assert abs(fd - an) <= 1e-8 * max(1.0, abs(an)), f"dilation d/d dir {idx} {comp}"
    # raw below the clamp: keep every sample 0.05 px from cell edges
    s0 = np.array([1.0, 1.0, 2.0], np.float32)
    raw = rng.standard_normal((1, Ho, Wo, 3)).astype(np.float32)
    smax = 50.0
    for i in range(Ho):
        for j in range(Wo):
            for g in range(3):
                s = o.msdcn_scale(raw[0, i, j, g], s0[g], smax)
                for k in range(9):
                    while True:
                        d = rng.standard_normal(2)
                        px = j + s * ((k % 3 - 1) + 0.5 * d[0])
                        py = i + s * ((k // 3 - 1) + 0.5 * d[1])
                        fx, fy = px - math.floor(px), py - math.floor(py)
                        if 0.05 < fx < 0.95 and 0.05 < fy < 0.95:
                            break
                    dw[0, i, j, g, k, :2] = d
    _, _, graw = o.msdcn_backward(prob, x, dw, raw, s0, smax, go)
    for idx in np.ndindex(raw.shape):
        rp, rm = raw.copy(), raw.copy()
        rp[idx] += 1e-3
        rm[idx] -= 1e-3
        fd = (np.sum(o.msdcn_forward(prob, x, dw, rp, s0, smax) * go) -
              np.sum(o.msdcn_forward(prob, x, dw, rm, s0, smax) * go)) / (float(rp[idx]) - float(rm[idx]))
        assert abs(fd - graw[idx]) <= 2e-3 * max(1.0, abs(graw[idx])), f"dilation d/d raw {idx}"


def _producer_ref(x, dw_w, dw_b, lin_w, lin_b):
    """torch float64: conv2d(groups=C, padding 1) then F.linear."""
    C = x.shape[-1]
    xt = torch.from_numpy(x.astype(np.float64)).permute(0, 3, 1, 2)
    wt = torch.from_numpy(dw_w.astype(np.float64).transpose(2, 0, 1)[:, None].copy())
    h = F.conv2d(xt, wt, torch.from_numpy(dw_b.astype(np.float64)), padding=1, groups=C)
    h = h.permute(0, 2, 3, 1)
    out = F.linear(h, torch.from_numpy(lin_w.astype(np.float64)),
                   torch.from_numpy(lin_b.astype(np.float64)))
    return h.numpy(), out.numpy()


def pin_producer(o):
    for ci, (N, H, W, C, G, kh, kw) in enumerate([(2, 5, 7, 6, 3, 3, 3), (1, 4, 3, 8, 2, 1, 3),
                                                   (1, 1, 6, 4, 1, 3, 3)]):
        rng = _rng(900 + ci)
        prob = o.problem(N, H, W, C, G, kh, kw, pad=((kh - 1) // 2, (kw - 1) // 2))
        J = G * kh * kw * 3
        x = rng.standard_normal((N, H, W, C)).astype(np.float32)
        dw_w = rng.standard_normal((3, 3, C)).astype(np.float32)
        dw_b = rng.standard_normal(C).astype(np.float32)
        lin_w = rng.standard_normal((J, C)).astype(np.float32)
        lin_b = rng.standard_normal(J).astype(np.float32)
        h_ref, ref = _producer_ref(x, dw_w, dw_b, lin_w, lin_b)
        got = o.offset_producer(prob, x, dw_w, dw_b, lin_w, lin_b).reshape(N, H, W, J)
        _close(got, ref, 1e-12, f"producer case {ci} vs conv2d + linear")
        # selection rows: out[j] = h[j % C] isolates the depthwise part
        sel = np.zeros((J, C), np.float32)
        sel[np.arange(J), np.arange(J) % C] = 1.0
        got = o.offset_producer(prob, x, dw_w, dw_b, sel, np.zeros(J, np.float32))
        _close(got.reshape(N, H, W, J), h_ref[..., np.arange(J) % C], 1e-12,
               f"producer case {ci} depthwise part")
        # identity depthwise (centre tap 1): out = x @ lin_w^T + lin_b
        ident = np.zeros((3, 3, C), np.float32)
        ident[1, 1] = 1.0
        got = o.offset_producer(prob, x, ident, np.zeros(C, np.float32), lin_w, lin_b)
        lin = x.astype(np.float64) @ lin_w.astype(np.float64).T + lin_b
        _close(got.reshape(N, H, W, J), lin, 1e-12, f"producer case {ci} linear part")
        # all-ones taps on a constant map count the in-image taps
        got = o.offset_producer(prob, np.ones_like(x), np.ones((3, 3, C), np.float32),
                                np.zeros(C, np.float32), sel, np.zeros(J, np.float32))
        cnt = np.zeros((H, W))
        for y in range(H):
            for xx in range(W):
                cnt[y, xx] = (min(y + 1, H - 1) - max(y - 1, 0) + 1) * \
                             (min(xx + 1, W - 1) - max(xx - 1, 0) + 1)
        assert np.array_equal(got.reshape(N, H, W, J), np.broadcast_to(
            cnt[None, :, :, None], (N, H, W, J))), f"producer case {ci} tap counts"
    # the counts themselves, written out on a 3 x 3 map
    prob = o.problem(1, 3, 3, 1, 1, 1, 1, pad=(0, 0))
    got = o.offset_producer(prob, np.ones((1, 3, 3, 1), np.float32),
                            np.ones((3, 3, 1), np.float32), np.zeros(1, np.float32),
                            np.ones((3, 1), np.float32), np.zeros(3, np.float32))
    assert np.array_equal(got[0, :, :, 0, 0, 0], [[4, 6, 4], [6, 9, 6], [4, 6, 4]])


ALL_PINS = [pin_conv, pin_grid_sample, pin_gather, pin_fractions, pin_out_of_bounds,
            pin_linearity, pin_equivariance, pin_msdcn, pin_cost_model, pin_adjoint,
            pin_unit_columns, pin_finite_diff, pin_msdcn_bwd_unit, pin_msdcn_bwd_adjoint,
            pin_msdcn_bwd_dir, pin_msdcn_bwd_raw, pin_msdcn_bwd_nan, pin_softmax_box, pin_softmax_shift,
            pin_softmax_bwd, pin_msdcn_dilation, pin_producer]
