"""GPU parity of dcn4_fused_forward, the DCNv4 module's offset/weight
sub-network (depthwise 3x3 + merged linear, DCNv4 digest
"方法3. DCN模块的微设计优化") fused into the aggregation, through the C ABI.

The call stands for the chain producer -> records rounded to the data type ->
forward. Three checks:
  * the aggregation against its records: the fused output against the
    oracle forward (orc_dcn4_forward) run on the records the call used (it
    writes them out on request), at the forward's gate, with offsets of the
    forward workloads' size (N(0, 2^2) pixels); and those records against
    orc_offset_producer at the same gate;
  * end to end against the oracle chain (orc_offset_producer, its fp64
    records rounded to the data type, orc_dcn4_forward) at the same gate,
    with offsets of N(0, 0.5^2) pixels. With 2-pixel offsets the records'
    own 16-bit rounding decides too much: the kernel rounds h to the data
    type before the linear layer, so about 40 % of its records land one
    16-bit step away from the oracle's rounding of the exact value, which
    moves samples by up to 1/16 pixel (scaled error up to ~3.4e-2 by a CPU
    emulation of that arithmetic, ~7e-3 at 0.5 pixel);
  * equality with the library's own two-kernel chain where both take the
    tensor-core producer's arithmetic, and the same output with and without
    the records written out.
Cases: several tiles with ragged edges, both 16-bit types, one and several
group slices, C = 64 .. 256, tiny images, DCNv3 softmax weights, every multiply
mode, the InternImage stage at full size on sampled images, the shapes the
fused kernel does not take (the two-kernel chain through the caller's
scratch), and the refusals (forced variant, missing scratch)."""
import ctypes

import numpy as np
import pytest
import torch

from deformable_convolution_dcn4_b200 import _binding as B
from deformable_convolution_dcn4_b200.workloads import DTYPES, make_fused_inputs

from parity_util import TOL, checked_err, f32, scaled_err

pytestmark = pytest.mark.gpu

# name: (N, H, W, C, G, dtype, the fused kernel applies)
CASES = {
    # InternImage stage channels (C128 G8: two slices of 4 groups); 24 x 20:
    # tiles 16 x 8 with a ragged bottom row and right column
    "internimage_bf16": (2, 24, 20, 128, 8, "bf16", True),
    "internimage_f16": (1, 17, 19, 128, 8, "f16", True),
    # C = 64: one slice, one block of depthwise chunks
    "c64_bf16": (2, 11, 30, 64, 4, "bf16", True),
    # D = 32: 4 chunks per group, 2 groups per slice
    "d32_bf16": (1, 20, 21, 64, 2, "bf16", True),
    # C = 256: 16 MMA K steps, 4 slices; smaller tiles fit shared memory
    "c256_bf16": (1, 12, 10, 256, 16, "bf16", True),
    # smaller than one tile
    "tiny_bf16": (3, 2, 3, 64, 4, "bf16", True),
    "one_pixel_f16": (2, 1, 1, 64, 4, "f16", True),
    # not for the fused kernel: fp32; D = 8 (16-byte groups); C = 24
    "f32": (2, 9, 7, 64, 4, "f32", False),
    "d8_bf16": (1, 10, 12, 64, 8, "bf16", False),
    "c24_bf16": (1, 6, 9, 24, 8, "bf16", False),
}
FUSED = sorted(k for k, v in CASES.items() if v[6])
# fused-kernel shapes where AUTO takes the two-kernel chain when it has room
# for the records: two or more group slices (each slice's CTA repeats the
# depthwise pass) and a shape the 2-D tensor-core producer takes in one
# pass, or four slices and more (the sliced tensor-core producer)
AUTO_CHAIN = {"internimage_bf16", "internimage_f16", "c256_bf16"}


def _inputs(name, seed=7, sigma=2.0):
    N, H, W, C, G, dtype, _ = CASES[name]
    return make_fused_inputs(N, H, W, C, G, dtype=dtype, seed=seed, offset_sigma=sigma)


def _gpu(d, G, algo="auto", math="default", softmax=False, workspace=None, records=False):
    """The fused call's output (and, with records=True, the records it used)."""
    dev = {n: t.cuda() for n, t in d.items()}
    N, H, W, C = d["x"].shape
    rec = torch.full((N, H, W, G, 9, 3), float("nan"), dtype=d["x"].dtype,
                     device="cuda") if records else None
    out = B.dcn4_fused_forward(dev["input"], dev["x"], dev["dw_weight"], dev["dw_bias"],
                               dev["lin_weight"], dev["lin_bias"], group=G, algo=algo, math=math,
                               softmax=softmax, workspace=workspace, offset_weight_out=rec)
    torch.cuda.synchronize()
    assert B.dcn4_last_device_error() == (0, 0)
    return (out, rec) if records else out


def _records(d, G, algo="auto"):
    """The library producer's records for d's x (generic kernel for the
    generic chain, else the tensor-core kernel where it applies)."""
    dev = {n: t.cuda() for n, t in d.items()}
    ow = B.dcn4_offset_producer(dev["x"], dev["dw_weight"], dev["dw_bias"], dev["lin_weight"],
                                dev["lin_bias"], group=G,
                                algo="generic" if algo == "generic" else "auto")
    torch.cuda.synchronize()
    return ow


def _chain(d, G, math="default", softmax=False):
    """The library's two-kernel chain: producer, then dcn4_forward."""
    ow = _records(d, G)
    out = B.dcn4_forward(d["input"].cuda(), ow, group=G, math=math, softmax=softmax)
    torch.cuda.synchronize()
    return out


def _oracle_on(orc, d, G, records, softmax=False, images=None):
    """orc_dcn4_forward on the given records (a tensor [N,H,W,G,9,3])."""
    sel = list(range(d["x"].shape[0])) if images is None else list(images)
    N, H, W, C = d["x"][sel].shape
    prob = orc.problem(N, H, W, C, G, 3, 3, softmax=softmax)
    return orc.forward(prob, f32(d["input"][sel]), f32(records[sel]))


def _oracle(orc, d, G, softmax=False, images=None):
    """orc_offset_producer -> records rounded to the data type ->
    orc_dcn4_forward, on the images listed (all by default)."""
    sel = list(range(d["x"].shape[0])) if images is None else list(images)
    x, inp = d["x"][sel], d["input"][sel]
    N, H, W, C = x.shape
    prob = orc.problem(N, H, W, C, G, 3, 3, softmax=softmax)
    ow = orc.offset_producer(prob, f32(x), f32(d["dw_weight"]), f32(d["dw_bias"]),
                             f32(d["lin_weight"]), f32(d["lin_bias"]))
    ow = torch.from_numpy(ow).to(d["x"].dtype).float().numpy().reshape(N, H, W, G, 9, 3)
    return orc.forward(prob, f32(inp), ow)


def _oracle_records(orc, d, G, images=None):
    sel = list(range(d["x"].shape[0])) if images is None else list(images)
    x = d["x"][sel]
    N, H, W, C = x.shape
    prob = orc.problem(N, H, W, C, G, 3, 3)
    ow = orc.offset_producer(prob, f32(x), f32(d["dw_weight"]), f32(d["dw_bias"]),
                             f32(d["lin_weight"]), f32(d["lin_bias"]))
    return ow.reshape(N, H, W, G, 9, 3)


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("algo", ["auto", "halo", "generic"])
def test_fused_parity(orc, name, algo):
    """The aggregation against the records it used, and those records
    against the oracle's producer (offsets ~2 px)."""
    G, dtype, fused = CASES[name][4], CASES[name][5], CASES[name][6]
    d = _inputs(name)
    if algo == "halo" and not fused:
        with pytest.raises(B.Dcn4Error) as e:
            _gpu(d, G, algo)
        assert e.value.code == 2
        return
    got, rec = _gpu(d, G, algo, records=True)
    err = checked_err(f32(got), _oracle_on(orc, d, G, rec), dtype, "aggregation")
    assert err <= TOL[dtype], f"{name} {algo}: aggregation, scaled error {err:.2e}"
    err = scaled_err(f32(rec), _oracle_records(orc, d, G))
    assert err <= TOL[dtype], f"{name} {algo}: records, scaled error {err:.2e}"


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("algo", ["auto", "generic"])
def test_fused_parity_oracle_chain(orc, name, algo):
    """End to end against the oracle's producer and forward (offsets ~0.5 px)."""
    G, dtype = CASES[name][4], CASES[name][5]
    d = _inputs(name, sigma=0.5)
    err = checked_err(f32(_gpu(d, G, algo)), _oracle(orc, d, G), dtype, "end to end")
    assert err <= TOL[dtype], f"{name} {algo}: scaled error {err:.2e}"


@pytest.mark.parametrize("math", ["f32", "mixed16", "packed16"])
def test_fused_math_modes(orc, math):
    d = _inputs("internimage_bf16")
    got, rec = _gpu(d, 8, "halo", math=math, records=True)
    err = scaled_err(f32(got), _oracle_on(orc, d, 8, rec))
    assert err <= TOL["bf16"], f"{math}: {err:.2e}"


@pytest.mark.parametrize("name", ["internimage_bf16", "c64_bf16"])
def test_fused_softmax_weights(orc, name):
    G, dtype = CASES[name][4], CASES[name][5]
    d = _inputs(name)
    got, rec = _gpu(d, G, "halo", softmax=True, records=True)
    err = scaled_err(f32(got), _oracle_on(orc, d, G, rec, softmax=True))
    assert err <= TOL[dtype], f"{name}: {err:.2e}"


@pytest.mark.parametrize("name", ["internimage_bf16", "internimage_f16"])
def test_fused_matches_two_kernel_chain(name):
    """Where the chain takes the tensor-core producer (whole 16-byte record
    rows, at most 256 outputs) both compute h, the MMA and the records'
    rounding the same way, and the fused kernel runs the forward's own
    gathers: records and output equal the chain's up to the MMA's summation
    order (the fused kernel multiplies one group slice's rows, the producer
    all of them at once)."""
    G = CASES[name][4]
    d = _inputs(name)
    got, rec = _gpu(d, G, "halo", records=True)
    ref_rec = _records(d, G)
    assert float((rec == ref_rec).float().mean()) >= 0.999
    got, ref = f32(got), f32(_chain(d, G))
    assert float(np.mean(got == ref)) >= 0.99
    assert scaled_err(got, ref) <= 1e-2


@pytest.mark.parametrize("name", FUSED)
def test_fused_records_out_changes_nothing(name):
    """Writing the records out is a side copy: the output is bit-identical."""
    G = CASES[name][4]
    d = _inputs(name)
    a = _gpu(d, G, "halo")
    b, _ = _gpu(d, G, "halo", records=True)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_fused_full_size_internimage(orc):
    """N64 56x56 C128 G8 bf16 (the InternImage stage, 3584 units of 16 x 8
    pixels x 4 groups), images 0, 31 and 63: against the oracle forward on the
    records the call used and those against the oracle's producer (offsets
    ~2 px), and end to end against the oracle chain (offsets ~0.5 px)."""
    images = [0, 31, 63]
    d = make_fused_inputs(64, 56, 56, 128, 8, dtype="bf16", seed=0)
    got, rec = _gpu(d, 8, "halo", records=True)
    got = f32(got)
    assert np.isfinite(got).all()
    err = checked_err(got[images], _oracle_on(orc, d, 8, rec.cpu(), images=images), "bf16",
                      "on its records")
    assert err <= TOL["bf16"], f"on its records: {err:.2e}"
    err = scaled_err(f32(rec[images]), _oracle_records(orc, d, 8, images=images))
    assert err <= TOL["bf16"], f"records: {err:.2e}"
    d = make_fused_inputs(64, 56, 56, 128, 8, dtype="bf16", seed=1, offset_sigma=0.5)
    got = f32(_gpu(d, 8, "halo"))
    err = scaled_err(got[images], _oracle(orc, d, 8, images=images))
    assert err <= TOL["bf16"], f"end to end: {err:.2e}"


def test_fused_workspace_size_and_refusal():
    """Shapes on which AUTO runs the fused kernel need no scratch; the others
    (the chain's shapes, and those where AUTO prefers the chain) ask for the
    offset_weight tensor's bytes (rounded to 16) plus the forward's escape
    scratch; the forced fused kernel never does. A chain shape refuses
    scratch smaller than the records before any launch."""
    for name in sorted(CASES):
        N, H, W, C, G, dtype, fused = CASES[name]
        desc = B.make_desc(N, H, W, C, G, DTYPES[dtype])
        need = B.dcn4_fused_forward_workspace_size(desc)
        eb = 4 if dtype == "f32" else 2
        auto_fused = fused and name not in AUTO_CHAIN
        chain = (N * H * W * G * 27 * eb + 15) // 16 * 16 + B.dcn4_forward_workspace_size(desc)
        assert need == (0 if auto_fused else chain), name
        if fused:
            desc = B.make_desc(N, H, W, C, G, DTYPES[dtype], algo="halo")
            assert B.dcn4_fused_forward_workspace_size(desc) == 0, name
    d = {k: v.cuda() for k, v in _inputs("d8_bf16").items()}
    desc = B.make_desc(1, 10, 12, 64, 8, torch.bfloat16)
    out = torch.empty_like(d["input"])
    ws = torch.empty(10 * 12 * 8 * 27 * 2 - 16, dtype=torch.uint8, device="cuda")
    lib = B.load()
    before = B.dcn4_kernel_launches()
    rc = lib.dcn4_fused_forward(ctypes.byref(desc), *(ctypes.c_void_p(d[k].data_ptr()) for k in (
        "input", "x", "dw_weight", "dw_bias", "lin_weight", "lin_bias")),
        ctypes.c_void_p(out.data_ptr()), None, ctypes.c_void_p(ws.data_ptr()), ws.numel(), None)
    assert rc == 3
    assert B.dcn4_kernel_launches() == before


@pytest.mark.parametrize("name", sorted(AUTO_CHAIN))
def test_fused_auto_route(orc, name):
    """AUTO on a shape where the chain is faster: with scratch (or an
    offset_weight_out) it launches the producer and the forward, without it
    the fused kernel; both against the oracle chain."""
    N, H, W, C, G, dtype, _ = CASES[name]
    d = _inputs(name, sigma=0.5)
    ref = _oracle(orc, d, G)
    ws = torch.empty(N * H * W * G * 27 * 2, dtype=torch.uint8, device="cuda")
    for workspace, launches in ((ws, 2), (None, 1)):
        dev = {k: v.cuda() for k, v in d.items()}
        out = torch.empty_like(dev["input"])
        desc = B.make_desc(N, H, W, C, G, DTYPES[dtype])
        before = B.dcn4_kernel_launches()
        rc = B.load().dcn4_fused_forward(
            ctypes.byref(desc), *(ctypes.c_void_p(dev[k].data_ptr()) for k in (
                "input", "x", "dw_weight", "dw_bias", "lin_weight", "lin_bias")),
            ctypes.c_void_p(out.data_ptr()), None,
            None if workspace is None else ctypes.c_void_p(workspace.data_ptr()),
            0 if workspace is None else workspace.numel(), None)
        torch.cuda.synchronize()
        assert rc == 0 and B.dcn4_last_device_error() == (0, 0)
        assert B.dcn4_kernel_launches() - before == launches
        err = scaled_err(f32(out), ref)
        assert err <= TOL[dtype], f"{name} scratch={workspace is not None}: {err:.2e}"


def test_fused_given_workspace(orc):
    """A caller's scratch serves the two-kernel chain (D = 8 bf16)."""
    d = _inputs("d8_bf16", sigma=0.5)
    ws = torch.empty(10 * 12 * 8 * 27 * 2, dtype=torch.uint8, device="cuda")
    err = scaled_err(f32(_gpu(d, 8, "auto", workspace=ws)), _oracle(orc, d, 8))
    assert err <= TOL["bf16"]


def test_fused_unaligned_pointers_take_the_chain(orc):
    """An input and output that start 2 bytes past a 16-byte boundary rule
    the fused kernel out (TMA and 16-byte stores); the call runs the
    two-kernel chain through the scratch it is given and still matches the
    oracle chain, while the forced fused kernel is refused."""
    N, H, W, C, G, dtype, _ = CASES["internimage_bf16"]
    d = _inputs("internimage_bf16", sigma=0.5)
    dev = {k: v.cuda() for k, v in d.items()}
    n = N * H * W * C
    inp_buf = torch.empty(n + 1, dtype=d["input"].dtype, device="cuda")
    inp = inp_buf[1:].view(N, H, W, C)
    inp.copy_(dev["input"])
    out_buf = torch.empty(n + 1, dtype=d["input"].dtype, device="cuda")
    out = out_buf[1:].view(N, H, W, C)
    ws = torch.empty(N * H * W * G * 27 * 2, dtype=torch.uint8, device="cuda")
    B.dcn4_fused_forward(inp, dev["x"], dev["dw_weight"], dev["dw_bias"], dev["lin_weight"],
                         dev["lin_bias"], group=G, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert B.dcn4_last_device_error() == (0, 0)
    err = scaled_err(f32(out), _oracle(orc, d, G))
    assert err <= TOL[dtype], f"scaled error {err:.2e}"
    with pytest.raises(B.Dcn4Error) as e:
        B.dcn4_fused_forward(inp, dev["x"], dev["dw_weight"], dev["dw_bias"],
                             dev["lin_weight"], dev["lin_bias"], group=G, out=out, workspace=ws,
                             algo="halo")
    assert e.value.code == 2


def _random_shapes(count=14, seed=2024):
    """Seeded fused-call shapes: N 1..3, H and W 1..37, C in {64, 96, 128,
    192, 256} with G giving D = 8, 16 or 32 (the fused kernel for D 16/32 with
    whole group slices, the chain for D 8 and for C 96), bf16/fp16."""
    rng = np.random.default_rng(seed)
    shapes = []
    while len(shapes) < count:
        C = int(rng.choice([64, 96, 128, 192, 256]))
        D = int(rng.choice([8, 16, 32]))
        if C % D:
            continue
        shapes.append((int(rng.integers(1, 4)), int(rng.integers(1, 38)),
                       int(rng.integers(1, 38)), C, C // D, str(rng.choice(["bf16", "f16"]))))
    return shapes


@pytest.mark.parametrize("shape", _random_shapes())
def test_fused_random_shapes(orc, shape):
    """End to end against the oracle chain on seeded random shapes (the fused
    kernel where it takes the shape, else the chain through scratch)."""
    N, H, W, C, G, dtype = shape
    d = make_fused_inputs(N, H, W, C, G, dtype=dtype, seed=N * 1000 + H * 37 + W,
                          offset_sigma=0.5)
    err = scaled_err(f32(_gpu(d, G)), _oracle(orc, d, G))
    assert err <= TOL[dtype], f"{shape}: scaled error {err:.2e}"


def test_fused_random_shapes_cover_the_fused_kernel():
    """The sweep above reaches the fused kernel (no scratch needed) and the
    chain (scratch needed) both."""
    kinds = set()
    for N, H, W, C, G, dtype in _random_shapes():
        desc = B.make_desc(N, H, W, C, G, DTYPES[dtype])
        kinds.add(B.dcn4_fused_forward_workspace_size(desc) == 0)
    assert kinds == {True, False}


@pytest.mark.parametrize("algo", ["halo", "generic"])
def test_fused_dilation_and_offset_scale(orc, algo):
    """Dilation 2 with pad 2 keeps the output grid equal to the input grid, so
    the fused call takes it; with offset_scale 0.5 the sampling grid and the
    offsets both differ from the plain case (the depthwise 3x3 of the
    sub-network is unchanged). Against the oracle chain of the same
    geometry."""
    N, H, W, C, G, dtype, _ = CASES["internimage_bf16"]
    d = _inputs("internimage_bf16", sigma=0.5)
    dev = {k: v.cuda() for k, v in d.items()}
    out = B.dcn4_fused_forward(dev["input"], dev["x"], dev["dw_weight"], dev["dw_bias"],
                               dev["lin_weight"], dev["lin_bias"], group=G, pad=2, dilation=2,
                               offset_scale=0.5, algo=algo)
    torch.cuda.synchronize()
    assert B.dcn4_last_device_error() == (0, 0)
    prob = orc.problem(N, H, W, C, G, 3, 3, pad=(2, 2), dilation=(2, 2), offset_scale=0.5)
    rec = orc.offset_producer(prob, f32(d["x"]), f32(d["dw_weight"]), f32(d["dw_bias"]),
                              f32(d["lin_weight"]), f32(d["lin_bias"]))
    rec = torch.from_numpy(rec).to(d["x"].dtype).float().numpy().reshape(N, H, W, G, 9, 3)
    err = scaled_err(f32(out), orc.forward(prob, f32(d["input"]), rec))
    assert err <= TOL[dtype], f"{algo}: scaled error {err:.2e}"


def test_fused_full_size_highres(orc):
    """N4 128x128 C256 G16 bf16 (four group slices, 8 x 8 tiles, 432 outputs
    per pixel: the tensor-core producer of the chain does not take it), image
    3: against the oracle forward on the records the call used, those records
    against the oracle's producer, and end to end against the oracle chain."""
    d = make_fused_inputs(4, 128, 128, 256, 16, dtype="bf16", seed=2)
    got, rec = _gpu(d, 16, "halo", records=True)
    got = f32(got)
    assert np.isfinite(got).all()
    images = [3]
    err = checked_err(got[images], _oracle_on(orc, d, 16, rec.cpu(), images=images), "bf16",
                      "on its records")
    assert err <= TOL["bf16"], f"on its records: {err:.2e}"
    err = scaled_err(f32(rec[images]), _oracle_records(orc, d, 16, images=images))
    assert err <= TOL["bf16"], f"records: {err:.2e}"
    d = make_fused_inputs(4, 128, 128, 256, 16, dtype="bf16", seed=3, offset_sigma=0.5)
    err = scaled_err(f32(_gpu(d, 16, "halo"))[images], _oracle(orc, d, 16, images=images))
    assert err <= TOL["bf16"], f"end to end: {err:.2e}"
