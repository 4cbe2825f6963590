"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, and validates arguments on the host before touching CUDA."""
import ctypes
import re

import pytest
import torch

from deformable_convolution_dcn4_b200 import _binding as B
from deformable_convolution_dcn4_b200 import build as libbuild

HEADER = libbuild.INCLUDE + "/dcn4.h"


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return B.load()


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"DCN4_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_binding_exports():
    assert sorted(declared_symbols()) == sorted(B.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_only_the_abi_is_exported(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIBRARY], capture_output=True,
                         text=True, check=True).stdout
    text_syms = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(declared_symbols()) <= text_syms
    leaked = {s for s in text_syms if s.startswith(("dcn4", "msdcn", "_ZN4dcn4"))} - set(
        declared_symbols())
    assert not leaked, leaked


def test_status_strings(lib):
    for code, name in B.STATUS.items():
        assert B.dcn4_status_string(code) == name
    assert B.dcn4_status_string(99) == "DCN4_UNKNOWN_STATUS"


def _desc(**kw):
    base = dict(N=2, H=9, W=11, C=16, G=4, dtype=0, kernel_size=3, stride=1, pad=1, dilation=1)
    base.update(kw)
    return B.make_desc(base["N"], base["H"], base["W"], base["C"], base["G"], base["dtype"],
                       base["kernel_size"], base["stride"], base["pad"], base["dilation"])


def test_out_shape_matches_oracle(lib, orc):
    cases = [dict(), dict(stride=2), dict(pad=0), dict(dilation=2), dict(kernel_size=5, pad=2),
             dict(kernel_size=1, pad=0), dict(kernel_size=(3, 1), pad=(1, 0)),
             dict(stride=(2, 3), pad=(0, 2), dilation=(2, 1)), dict(H=1, W=1, kernel_size=1, pad=0)]
    for c in cases:
        d = _desc(**c)
        p = orc.problem(d.N, d.H, d.W, d.C, d.G, d.kh, d.kw, (d.stride_h, d.stride_w),
                        (d.pad_h, d.pad_w), (d.dil_h, d.dil_w))
        assert B.dcn4_out_shape(d) == orc.out_hw(p), c


@pytest.mark.parametrize("bad", [dict(C=10, G=4), dict(N=0), dict(G=0), dict(stride=0),
                                 dict(dilation=0), dict(pad=-1), dict(H=2, pad=0),
                                 dict(dtype=7), dict(C=2048, G=2048),
                                 dict(kernel_size=9, pad=4)])
def test_malformed_descriptors_rejected(lib, bad):
    d = _desc(**bad)
    with pytest.raises(B.Dcn4Error) as e:
        B.dcn4_out_shape(d)
    assert e.value.code == 1
    n = ctypes.c_size_t()
    assert lib.dcn4_backward_workspace_size(ctypes.byref(d), ctypes.byref(n)) == 1


def test_bad_enum_fields_rejected(lib):
    for field, val in (("math", 5), ("algo", 9), ("dtype", -1), ("weights", 2),
                       ("msdcn_mode", -1), ("msdcn_mode", 2)):
        d = _desc()
        setattr(d, field, val)
        with pytest.raises(B.Dcn4Error) as e:
            B.dcn4_out_shape(d)
        assert e.value.code == 1


def test_null_pointers_rejected_before_any_launch(lib):
    d = _desc()
    z = ctypes.c_void_p(0)
    one = ctypes.c_void_p(16)
    assert lib.dcn4_forward(ctypes.byref(d), z, one, one, z) == 1
    assert lib.dcn4_forward(ctypes.byref(d), one, z, one, z) == 1
    assert lib.dcn4_forward(ctypes.byref(d), one, one, z, z) == 1
    assert lib.dcn4_forward(None, one, one, one, z) == 1
    s0 = (ctypes.c_float * 4)(1, 1, 2, 2)
    assert lib.msdcn_forward(ctypes.byref(d), one, one, z, s0, 8.0, one, z) == 1
    assert lib.msdcn_forward(ctypes.byref(d), one, one, one, None, 8.0, one, z) == 1
    assert lib.dcn4_backward(ctypes.byref(d), one, one, one, z, one, one, 1 << 30, z) == 1
    # msdcn_backward: every pointer, including the scale gradient and s0
    args = [one, one, one, s0, 8.0, one, one, one, one, one, 1 << 30, z]
    for i in (0, 1, 2, 3, 5, 6, 7, 8):
        bad = list(args)
        bad[i] = None if i == 3 else z
        assert lib.msdcn_backward(ctypes.byref(d), *bad) == 1, i
    assert lib.msdcn_backward(None, *args) == 1


def test_msdcn_rejects_softmax_weights_before_any_launch(lib):
    d = _desc(dtype=1)
    d.weights = 1
    one = ctypes.c_void_p(16)
    z = ctypes.c_void_p(0)
    s0 = (ctypes.c_float * 4)(1, 1, 2, 2)
    assert lib.msdcn_forward(ctypes.byref(d), one, one, one, s0, 8.0, one, z) == 2
    assert lib.msdcn_backward(ctypes.byref(d), one, one, one, s0, 8.0, one, one, one, one, one,
                              1 << 30, z) == 2


def test_workspace_rules(lib):
    d32 = _desc(dtype=0)
    assert B.dcn4_backward_workspace_size(d32) == 0
    d16 = _desc(dtype=1)
    assert B.dcn4_backward_workspace_size(d16) == 2 * 9 * 11 * 16 * 4
    one = ctypes.c_void_p(16)
    z = ctypes.c_void_p(0)
    # too small / missing workspace is reported before anything runs
    assert lib.dcn4_backward(ctypes.byref(d16), one, one, one, one, one, z, 0, z) == 3
    assert lib.dcn4_backward(ctypes.byref(d16), one, one, one, one, one, one, 100, z) == 3


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 8, 8, 16)
    ow = torch.zeros(1, 8, 8, 4, 9, 3)
    with pytest.raises(ValueError):
        B.dcn4_forward(x, ow, group=4)


def test_launch_counter_without_gpu(lib):
    """No kernel has run in this process: the counter reads zero, and a null
    pointer is rejected."""
    assert B.dcn4_kernel_launches() == 0
    assert lib.dcn4_kernel_launches(None) == 1


def test_producer_argument_errors(lib):
    """dcn4_offset_producer rejects null pointers and a strided output grid
    before any launch (no GPU needed)."""
    d = _desc()
    fake = [ctypes.c_void_p(4096)] * 6
    assert lib.dcn4_offset_producer(ctypes.byref(d), None, *fake[:5], None) == 1
    assert lib.dcn4_offset_producer(ctypes.byref(d), *fake[:5], None, None) == 1
    d2 = _desc(stride=2)
    assert lib.dcn4_offset_producer(ctypes.byref(d2), *fake, None) == 2
    bad = _desc(C=10, G=4)
    assert lib.dcn4_offset_producer(ctypes.byref(bad), *fake, None) == 1


def test_fused_forward_argument_errors(lib):
    """dcn4_fused_forward rejects null pointers and a strided output grid, and
    a call that must take the two-kernel chain (fp32 has no fused kernel)
    without scratch is refused with DCN4_ERR_WORKSPACE before any launch."""
    d = _desc()  # fp32, N2 9x11 C16 G4
    fake = [ctypes.c_void_p(4096)] * 7
    n = ctypes.c_size_t()
    assert lib.dcn4_fused_forward_workspace_size(ctypes.byref(d), ctypes.byref(n)) == 0
    assert n.value == 2 * 9 * 11 * 4 * 27 * 4  # the offset_weight tensor, fp32
    assert lib.dcn4_fused_forward_workspace_size(ctypes.byref(d), None) == 1
    assert lib.dcn4_fused_forward(ctypes.byref(d), None, *fake[:6], None, None, 0, None) == 1
    assert lib.dcn4_fused_forward(ctypes.byref(d), *fake[:6], None, None, None, 0, None) == 1
    assert lib.dcn4_fused_forward(ctypes.byref(_desc(stride=2)), *fake, None, None, 0,
                                  None) == 2
    assert lib.dcn4_fused_forward(ctypes.byref(d), *fake, None, None, 0, None) == 3
    assert lib.dcn4_fused_forward(ctypes.byref(d), *fake, None, ctypes.c_void_p(4096),
                                  n.value - 1, None) == 3
    d.algo = B.ALGO_CODE["halo"]  # demands the fused kernel: none for fp32
    assert lib.dcn4_fused_forward(ctypes.byref(d), *fake, None, None, 0, None) == 2


def test_workspace_size_where_it_applies():
    """Scratch only for the staged kernel with one lane per pair: 3x3 taps,
    groups of 32 or 64 bytes (16-bit) or 64 bytes (fp32); AUTO or HALO."""
    def size(C, G, dt, k=3, algo="auto"):
        return B.dcn4_forward_workspace_size(B.make_desc(2, 9, 9, C, G, dt, kernel_size=k,
                                                         pad=(k - 1) // 2, algo=algo))
    npairs = 2 * 9 * 9 * 8
    base = size(128, 8, torch.bfloat16)
    assert base >= (npairs + 3) // 4 * (16 + 4 * 16)
    assert size(128, 4, torch.bfloat16) > 0           # D32 bf16: 4 chunks
    assert size(128, 8, torch.float32) > 0            # D16 fp32: 4 chunks
    assert size(256, 4, torch.bfloat16) == 0          # D64 bf16: two lanes per pair
    assert size(128, 16, torch.bfloat16) == 0         # D8 bf16: 16-byte groups
    assert size(128, 8, torch.bfloat16, k=5) == 0     # 5x5 taps
    assert size(128, 8, torch.bfloat16, algo="generic") == 0
    assert size(128, 8, torch.bfloat16, algo="halo") == base
