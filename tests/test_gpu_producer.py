"""GPU parity of the offset/weight producer (depthwise 3x3 + merged linear,
DCNv4 digest "方法3. DCN模块的微设计优化") through the C ABI against the CPU
oracle on the same seeded inputs: both kernels (tensor-core and generic), the
InternImage shape at full size on sampled images, ragged tails, the shapes
the tensor-core kernel does not take, and the producer feeding dcn4_forward."""
import numpy as np
import pytest
import torch

from deformable_convolution_dcn4_b200 import _binding as B
from deformable_convolution_dcn4_b200.workloads import make_producer_inputs

from parity_util import TOL, checked_err, f32, scaled_err

pytestmark = pytest.mark.gpu

# name: (N, H, W, C, G, k, dtype, tensor-core kernel applies)
CASES = {
    # InternImage stage channels (C128 G8): 286 pixels = 2 full tiles + 30
    "internimage_bf16": (2, 13, 11, 128, 8, 3, "bf16", True),
    "internimage_f16": (1, 17, 19, 128, 8, 3, "f16", True),
    # one K step (C = 16), 1x1 taps (J = 24, N padded to 32), 650 pixels
    "c16_k1_bf16": (1, 5, 130, 16, 8, 1, "bf16", True),
    # C = 256 (16 K steps), 1x1 taps, one ragged tile of 35 pixels
    "c256_k1_bf16": (1, 5, 7, 256, 8, 1, "bf16", True),
    # C = 256 with 3x3 taps: lin_w does not fit next to the tile; the fused
    # kernel's producer steps (4 slices of 2 groups) take it
    "c256_bf16": (1, 5, 7, 256, 8, 3, "bf16", True),
    # the high-resolution stage's channels (C256 G16: J = 432 > 256), 4
    # slices of 108 outputs, tiles 16 x 8 with ragged edges
    "c256_g16_bf16": (2, 19, 13, 256, 16, 3, "bf16", True),
    "c256_g16_f16": (1, 9, 21, 256, 16, 3, "f16", True),
    # not for the tensor cores: fp32; J = 81 (odd 16-byte rows); J = 540 > 256
    "f32_g3": (2, 9, 7, 24, 3, 3, "f32", False),
    "bf16_g3": (1, 10, 12, 48, 3, 3, "bf16", False),
    "ldm_f16": (1, 8, 8, 320, 20, 3, "f16", False),
    # C not a multiple of 16
    "c24_bf16": (1, 6, 9, 24, 8, 3, "bf16", False),
    # the 2-D tiled kernel on an image smaller than one 16 x 8 tile (2 x 4
    # tiles, columns and rows past the image not stored), three images
    "tiny_2d_bf16": (3, 2, 3, 64, 8, 3, "bf16", True),
    # the 2-D tiled kernel over a tall narrow image: 16 x 8 tiles whose
    # columns 5..7 and, in the last tile row, rows 8..15 lie past the image
    "tall_2d_f16": (1, 40, 5, 64, 8, 3, "f16", True),
}


def _inputs(N, H, W, C, G, k, dtype, seed=3):
    return make_producer_inputs(N, H, W, C, G, K=k * k, dtype=dtype, seed=seed)


def _gpu(d, G, k, algo):
    dev = {n: t.cuda() for n, t in d.items()}
    out = B.dcn4_offset_producer(dev["x"], dev["dw_weight"], dev["dw_bias"], dev["lin_weight"],
                                 dev["lin_bias"], group=G, kernel_size=k, pad=(k - 1) // 2,
                                 algo=algo)
    torch.cuda.synchronize()
    assert B.dcn4_last_device_error() == (0, 0)
    return out


def _oracle(orc, d, G, k, images=None):
    x = d["x"] if images is None else d["x"][list(images)]
    N, H, W, C = x.shape
    prob = orc.problem(N, H, W, C, G, k, k, pad=((k - 1) // 2, (k - 1) // 2))
    return orc.offset_producer(prob, f32(x), f32(d["dw_weight"]), f32(d["dw_bias"]),
                               f32(d["lin_weight"]), f32(d["lin_bias"]))


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("algo", ["auto", "generic", "halo"])
def test_producer_parity(orc, name, algo):
    N, H, W, C, G, k, dtype, tc = CASES[name]
    d = _inputs(N, H, W, C, G, k, dtype)
    if algo == "halo" and not tc:
        with pytest.raises(B.Dcn4Error) as e:
            _gpu(d, G, k, algo)
        assert e.value.code == 2
        return
    got = f32(_gpu(d, G, k, algo))
    err = checked_err(got, _oracle(orc, d, G, k), dtype, f"{name} {algo}")
    assert err <= TOL[dtype], f"{name} {algo}: scaled error {err:.2e}"


def test_producer_full_size_internimage(orc):
    """N64 56x56 C128 G8 bf16 on the tensor-core kernel (1568 tiles, tiles
    crossing image boundaries); images 0, 1 and 63 against the oracle."""
    d = _inputs(64, 56, 56, 128, 8, 3, "bf16", seed=0)
    got = f32(_gpu(d, 8, 3, "halo"))
    images = [0, 1, 63]
    err = checked_err(got[images], _oracle(orc, d, 8, 3, images), "bf16", "full size")
    assert err <= TOL["bf16"], f"scaled error {err:.2e}"


def test_producer_full_size_highres(orc):
    """N4 128x128 C256 G16 bf16 (J = 432: the sliced tensor-core path, 4096
    units of 16 x 8 pixels x 4 groups), image 2 against the oracle."""
    d = _inputs(4, 128, 128, 256, 16, 3, "bf16", seed=1)
    got = f32(_gpu(d, 16, 3, "halo"))
    err = checked_err(got[[2]], _oracle(orc, d, 16, 3, [2]), "bf16", "full size")
    assert err <= TOL["bf16"], f"scaled error {err:.2e}"


def test_producer_kernels_agree_closely():
    """Both kernels on the same bf16 inputs: they differ only by the 16-bit
    rounding of h in front of the tensor cores and by summation order."""
    d = _inputs(2, 13, 11, 128, 8, 3, "bf16")
    a = f32(_gpu(d, 8, 3, "halo"))
    b = f32(_gpu(d, 8, 3, "generic"))
    assert scaled_err(a, b) <= 1e-2


def test_producer_feeds_forward(orc):
    """offset_weight from the producer drives dcn4_forward on the GPU; the
    oracle chains its own producer and forward on the same inputs."""
    N, H, W, C, G = 2, 15, 13, 128, 8
    d = _inputs(N, H, W, C, G, 3, "bf16", seed=5)
    ow = _gpu(d, G, 3, "auto")
    got = f32(B.dcn4_forward(d["x"].cuda(), ow, group=G))
    prob = orc.problem(N, H, W, C, G)
    ow_ref = _oracle(orc, d, G, 3)
    ref = orc.forward(prob, f32(d["x"]), ow_ref.astype(np.float32))
    # scaled gate only: the records reach the forward rounded to bf16, which
    # moves a sample by up to half an ulp of its offset, so single outputs
    # near zero can differ by more than the elementwise gate allows
    err = scaled_err(got, ref)
    assert err <= TOL["bf16"], f"scaled error {err:.2e}"


def test_producer_counts_one_launch():
    d = {n: t.cuda() for n, t in _inputs(1, 9, 9, 128, 8, 3, "bf16").items()}
    before = B.dcn4_kernel_launches()
    B.dcn4_offset_producer(d["x"], d["dw_weight"], d["dw_bias"], d["lin_weight"], d["lin_bias"],
                           group=8)
    torch.cuda.synchronize()
    assert B.dcn4_kernel_launches() - before == 1
