"""Thin ctypes binding of libdcn4.so (the C ABI in include/dcn4.h).

Argument marshalling only: tensors come from torch (device memory, the
current stream), every step of the operator runs in the library's CUDA
kernels. There is no CPU fallback: calls raise when the library or a CUDA
device is missing.
"""
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_PKG, "libdcn4.so")
CHECKED_LIBRARY = os.path.join(_PKG, "libdcn4_checked.so")

STATUS = {0: "DCN4_OK", 1: "DCN4_ERR_INVALID_ARG", 2: "DCN4_ERR_UNSUPPORTED",
          3: "DCN4_ERR_WORKSPACE", 4: "DCN4_ERR_CUDA", 5: "DCN4_ERR_TIMEOUT",
          6: "DCN4_ERR_INTERNAL"}
DTYPE_CODE = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}
ALGO_CODE = {"auto": 0, "generic": 1, "halo": 2, "vector": 3}
MATH_CODE = {"default": 0, "f32": 1, "mixed16": 2, "packed16": 3, "acc16": 4}
MSDCN_MODE_CODE = {"offset": 0, "dilation": 1}

# Every symbol include/dcn4.h declares.
EXPORTS = ("dcn4_out_shape", "dcn4_forward", "dcn4_backward_workspace_size", "dcn4_backward",
           "msdcn_forward", "dcn4_status_string", "dcn4_last_device_error",
           "dcn4_backward_noalloc", "dcn4_selftest_bounded_wait", "dcn4_kernel_launches",
           "msdcn_backward", "dcn4_offset_producer", "dcn4_fused_forward_workspace_size",
           "dcn4_fused_forward", "dcn4_forward_workspace_size", "dcn4_forward_ws",
           "msdcn_forward_ws")


class Dcn4Error(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


class Desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("N", "H", "W", "C", "G", "kh", "kw", "stride_h", "stride_w", "pad_h", "pad_w",
                 "dil_h", "dil_w")] + [("offset_scale", ctypes.c_float), ("dtype", ctypes.c_int),
                                       ("algo", ctypes.c_int), ("math", ctypes.c_int),
                                       ("weights", ctypes.c_int), ("msdcn_mode", ctypes.c_int)]


_lib = None


def load(path=LIBRARY):
    """Loads libdcn4.so once; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = _open(path)
    return _lib


def use_library(path):
    """Makes every call of this module go to the library at `path` (e.g. the
    bounds-checked build, libdcn4_checked.so); returns the library used
    before, for restore_library."""
    global _lib
    prev = _lib
    _lib = _open(path)
    return prev


def restore_library(prev):
    global _lib
    _lib = prev


def _open(path):
    if not os.path.exists(path):
        raise RuntimeError(f"{os.path.basename(path)} not built ({path}); run "
                           "`python -m deformable_convolution_dcn4_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(Desc)
    vp, st = ctypes.c_void_p, ctypes.c_int
    lib.dcn4_out_shape.argtypes = [P, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
    lib.dcn4_forward.argtypes = [P, vp, vp, vp, vp]
    lib.dcn4_backward_workspace_size.argtypes = [P, ctypes.POINTER(ctypes.c_size_t)]
    lib.dcn4_backward.argtypes = [P, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.msdcn_backward.argtypes = [P, vp, vp, vp, ctypes.POINTER(ctypes.c_float), ctypes.c_float,
                                   vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.msdcn_forward.argtypes = [P, vp, vp, vp, ctypes.POINTER(ctypes.c_float), ctypes.c_float,
                                  vp, vp]
    lib.dcn4_status_string.argtypes = [st]
    lib.dcn4_status_string.restype = ctypes.c_char_p
    lib.dcn4_last_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint)]
    lib.dcn4_backward_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp]
    lib.dcn4_selftest_bounded_wait.argtypes = [ctypes.c_uint, vp]
    lib.dcn4_kernel_launches.argtypes = [ctypes.POINTER(ctypes.c_ulonglong)]
    lib.dcn4_offset_producer.argtypes = [P, vp, vp, vp, vp, vp, vp, vp]
    lib.dcn4_fused_forward_workspace_size.argtypes = [P, ctypes.POINTER(ctypes.c_size_t)]
    lib.dcn4_fused_forward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t,
                                       vp]
    lib.dcn4_forward_workspace_size.argtypes = [P, ctypes.POINTER(ctypes.c_size_t)]
    lib.dcn4_forward_ws.argtypes = [P, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.msdcn_forward_ws.argtypes = [P, vp, vp, vp, ctypes.POINTER(ctypes.c_float),
                                     ctypes.c_float, vp, vp, ctypes.c_size_t, vp]
    for name in EXPORTS:
        if name != "dcn4_status_string":
            getattr(lib, name).restype = st
    return lib


def _pair(v):
    return (int(v), int(v)) if isinstance(v, (int, float)) else (int(v[0]), int(v[1]))


def make_desc(N, H, W, C, G, dtype, kernel_size=3, stride=1, pad=1, dilation=1,
              offset_scale=1.0, algo="auto", math="default", softmax=False, msdcn_mode="offset"):
    kh, kw = _pair(kernel_size)
    sh, sw = _pair(stride)
    ph, pw = _pair(pad)
    dh, dw = _pair(dilation)
    code = DTYPE_CODE[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    return Desc(N, H, W, C, G, kh, kw, sh, sw, ph, pw, dh, dw, float(offset_scale), code,
                ALGO_CODE[algo], MATH_CODE[math], 1 if softmax else 0,
                MSDCN_MODE_CODE[msdcn_mode])


def _check(fn, rc):
    if rc != 0:
        raise Dcn4Error(fn, rc)


def dcn4_out_shape(desc):
    ho, wo = ctypes.c_int(), ctypes.c_int()
    _check("dcn4_out_shape", load().dcn4_out_shape(ctypes.byref(desc), ctypes.byref(ho),
                                                   ctypes.byref(wo)))
    return ho.value, wo.value


def _stream(t):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _require(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (channel-last)")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _desc_for(inp, group, kernel_size, stride, pad, dilation, offset_scale, algo, math="default",
              softmax=False, msdcn_mode="offset"):
    N, H, W, C = inp.shape
    return make_desc(N, H, W, C, group, inp.dtype, kernel_size, stride, pad, dilation,
                     offset_scale, algo, math, softmax, msdcn_mode)


def dcn4_forward_workspace_size(desc):
    n = ctypes.c_size_t()
    _check("dcn4_forward_workspace_size",
           load().dcn4_forward_workspace_size(ctypes.byref(desc), ctypes.byref(n)))
    return n.value


def _forward_scratch(desc, input, workspace, defer_escapes):
    """(pointer, bytes, tensor) of the escape scratch: the caller's tensor,
    else one from PyTorch's allocator of dcn4_forward_workspace_size bytes
    (the caller keeps the tensor until the launch is issued; the allocator
    reuses it only in stream order after that); None when escapes are to be
    handled in place."""
    if not defer_escapes:
        return None
    if workspace is None:
        need = dcn4_forward_workspace_size(desc)
        if need == 0:
            return (None, 0, None)
        workspace = torch.empty(need, dtype=torch.uint8, device=input.device)
    return (_ptr(workspace), workspace.numel() * workspace.element_size(), workspace)


def dcn4_forward(input, offset_weight, group, kernel_size=3, stride=1, pad=1, dilation=1,
                 offset_scale=1.0, algo="auto", out=None, math="default", softmax=False,
                 workspace=None, defer_escapes=True):
    """DCNv4 forward. input [N,H,W,C]; offset_weight [N,Ho,Wo,G,kh*kw,3].
    softmax=True normalises m over the taps (DCNv3 weights). The staged
    kernel's escaped samples go through scratch (dcn4_forward_ws; `workspace`,
    else one allocated here) unless defer_escapes=False (dcn4_forward)."""
    desc = _desc_for(input, group, kernel_size, stride, pad, dilation, offset_scale, algo, math,
                     softmax)
    ho, wo = dcn4_out_shape(desc)
    N, _, _, C = input.shape
    _require(input, "input", input.dtype)
    _require(offset_weight, "offset_weight", input.dtype,
             (N, ho, wo, group, desc.kh * desc.kw, 3))
    if out is None:
        out = torch.empty((N, ho, wo, C), dtype=input.dtype, device=input.device)
    _require(out, "out", input.dtype, (N, ho, wo, C))
    ws = _forward_scratch(desc, input, workspace, defer_escapes)
    if ws is None:
        _check("dcn4_forward", load().dcn4_forward(ctypes.byref(desc), _ptr(input),
                                                   _ptr(offset_weight), _ptr(out),
                                                   _stream(input)))
    else:
        _check("dcn4_forward_ws", load().dcn4_forward_ws(ctypes.byref(desc), _ptr(input),
                                                         _ptr(offset_weight), _ptr(out), ws[0],
                                                         ws[1], _stream(input)))
    return out


def dcn4_offset_producer(x, dw_weight, dw_bias, lin_weight, lin_bias, group, kernel_size=3,
                         stride=1, pad=1, dilation=1, offset_scale=1.0, algo="auto", out=None):
    """offset_weight [N,H,W,G,kh*kw,3] from the depthwise 3x3 + merged linear
    sub-network: x [N,H,W,C], dw_weight [3,3,C], dw_bias [C],
    lin_weight [G*kh*kw*3, C], lin_bias [G*kh*kw*3], all of x's dtype."""
    desc = _desc_for(x, group, kernel_size, stride, pad, dilation, offset_scale, algo)
    N, H, W, C = x.shape
    J = group * desc.kh * desc.kw * 3
    _require(x, "x", x.dtype)
    _require(dw_weight, "dw_weight", x.dtype, (3, 3, C))
    _require(dw_bias, "dw_bias", x.dtype, (C,))
    _require(lin_weight, "lin_weight", x.dtype, (J, C))
    _require(lin_bias, "lin_bias", x.dtype, (J,))
    shape = (N, H, W, group, desc.kh * desc.kw, 3)
    if out is None:
        out = torch.empty(shape, dtype=x.dtype, device=x.device)
    _require(out, "out", x.dtype, shape)
    _check("dcn4_offset_producer",
           load().dcn4_offset_producer(ctypes.byref(desc), _ptr(x), _ptr(dw_weight), _ptr(dw_bias),
                                       _ptr(lin_weight), _ptr(lin_bias), _ptr(out), _stream(x)))
    return out


def dcn4_fused_forward_workspace_size(desc):
    n = ctypes.c_size_t()
    _check("dcn4_fused_forward_workspace_size",
           load().dcn4_fused_forward_workspace_size(ctypes.byref(desc), ctypes.byref(n)))
    return n.value


def dcn4_fused_forward(input, x, dw_weight, dw_bias, lin_weight, lin_bias, group, kernel_size=3,
                       stride=1, pad=1, dilation=1, offset_scale=1.0, algo="auto", out=None,
                       math="default", softmax=False, workspace=None, offset_weight_out=None):
    """DCNv4 forward with the offset/weight sub-network in front:
    dcn4_forward(input, dcn4_offset_producer(x, ...)) in one call. input and x
    [N,H,W,C]; dw_weight [3,3,C], dw_bias [C], lin_weight [G*kh*kw*3, C],
    lin_bias [G*kh*kw*3]. offset_weight_out [N,Ho,Wo,G,kh*kw,3], when given,
    receives the records the aggregation used. A scratch tensor is allocated
    when the call takes the two-kernel chain and neither it nor
    offset_weight_out is given."""
    desc = _desc_for(input, group, kernel_size, stride, pad, dilation, offset_scale, algo, math,
                     softmax)
    ho, wo = dcn4_out_shape(desc)
    N, H, W, C = input.shape
    J = group * desc.kh * desc.kw * 3
    _require(input, "input", input.dtype)
    _require(x, "x", input.dtype, (N, H, W, C))
    _require(dw_weight, "dw_weight", input.dtype, (3, 3, C))
    _require(dw_bias, "dw_bias", input.dtype, (C,))
    _require(lin_weight, "lin_weight", input.dtype, (J, C))
    _require(lin_bias, "lin_bias", input.dtype, (J,))
    if out is None:
        out = torch.empty((N, ho, wo, C), dtype=input.dtype, device=input.device)
    _require(out, "out", input.dtype, (N, ho, wo, C))
    if offset_weight_out is not None:
        _require(offset_weight_out, "offset_weight_out", input.dtype,
                 (N, ho, wo, group, desc.kh * desc.kw, 3))
    if workspace is None and offset_weight_out is None:
        need = dcn4_fused_forward_workspace_size(desc)
        if need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=input.device)
    ws, nws = (_ptr(workspace), workspace.numel() * workspace.element_size()) \
        if workspace is not None else (None, 0)
    _check("dcn4_fused_forward",
           load().dcn4_fused_forward(ctypes.byref(desc), _ptr(input), _ptr(x), _ptr(dw_weight),
                                     _ptr(dw_bias), _ptr(lin_weight), _ptr(lin_bias), _ptr(out),
                                     None if offset_weight_out is None else _ptr(offset_weight_out),
                                     ws, nws, _stream(input)))
    return out


def dcn4_backward_workspace_size(desc):
    n = ctypes.c_size_t()
    _check("dcn4_backward_workspace_size",
           load().dcn4_backward_workspace_size(ctypes.byref(desc), ctypes.byref(n)))
    return n.value


def dcn4_backward(input, offset_weight, grad_out, group, kernel_size=3, stride=1, pad=1,
                  dilation=1, offset_scale=1.0, algo="auto", workspace=None,
                  grad_input=None, grad_offset_weight=None, math="default", softmax=False):
    """DCNv4 backward -> (grad_input, grad_offset_weight)."""
    desc = _desc_for(input, group, kernel_size, stride, pad, dilation, offset_scale, algo, math,
                     softmax)
    ho, wo = dcn4_out_shape(desc)
    N, H, W, C = input.shape
    _require(input, "input", input.dtype)
    _require(offset_weight, "offset_weight", input.dtype,
             (N, ho, wo, group, desc.kh * desc.kw, 3))
    _require(grad_out, "grad_out", input.dtype, (N, ho, wo, C))
    if grad_input is None:
        grad_input = torch.empty_like(input)
    if grad_offset_weight is None:
        grad_offset_weight = torch.empty_like(offset_weight)
    need = dcn4_backward_workspace_size(desc)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=input.device)
    ws_ptr = _ptr(workspace) if workspace is not None else ctypes.c_void_p(0)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("dcn4_backward", load().dcn4_backward(
        ctypes.byref(desc), _ptr(input), _ptr(offset_weight), _ptr(grad_out), _ptr(grad_input),
        _ptr(grad_offset_weight), ws_ptr, ws_bytes, _stream(input)))
    return grad_input, grad_offset_weight


def dcn4_backward_noalloc(input, offset_weight, grad_out, group, kernel_size=3, stride=1, pad=1,
                          dilation=1, offset_scale=1.0, algo="auto", grad_input=None,
                          grad_offset_weight=None, math="default", softmax=False):
    """dcn4_backward without a caller-supplied workspace: the library's own
    fixed scratch array is used (see include/dcn4.h for its limit)."""
    desc = _desc_for(input, group, kernel_size, stride, pad, dilation, offset_scale, algo, math,
                     softmax)
    ho, wo = dcn4_out_shape(desc)
    N, H, W, C = input.shape
    _require(input, "input", input.dtype)
    _require(offset_weight, "offset_weight", input.dtype,
             (N, ho, wo, group, desc.kh * desc.kw, 3))
    _require(grad_out, "grad_out", input.dtype, (N, ho, wo, C))
    if grad_input is None:
        grad_input = torch.empty_like(input)
    if grad_offset_weight is None:
        grad_offset_weight = torch.empty_like(offset_weight)
    _check("dcn4_backward_noalloc", load().dcn4_backward_noalloc(
        ctypes.byref(desc), _ptr(input), _ptr(offset_weight), _ptr(grad_out), _ptr(grad_input),
        _ptr(grad_offset_weight), _stream(input)))
    return grad_input, grad_offset_weight


def msdcn_forward(input, dir_weight, scale_raw, s0, smax, group, kernel_size=3, stride=1, pad=1,
                  dilation=1, offset_scale=1.0, algo="auto", out=None, math="default",
                  msdcn_mode="offset", workspace=None, defer_escapes=True):
    """MSDCN forward. dir_weight [N,Ho,Wo,G,K,3]; scale_raw [N,Ho,Wo,G]; s0 host floats [G].
    msdcn_mode "offset" (s * dir) or "dilation" (s * (p_k + dir)). Escape
    scratch as in dcn4_forward (msdcn_forward_ws)."""
    desc = _desc_for(input, group, kernel_size, stride, pad, dilation, offset_scale, algo, math,
                     False, msdcn_mode)
    ho, wo = dcn4_out_shape(desc)
    N, _, _, C = input.shape
    _require(input, "input", input.dtype)
    _require(dir_weight, "dir_weight", input.dtype, (N, ho, wo, group, desc.kh * desc.kw, 3))
    _require(scale_raw, "scale_raw", input.dtype, (N, ho, wo, group))
    s0 = [float(v) for v in (s0.tolist() if isinstance(s0, torch.Tensor) else s0)]
    if len(s0) != group:
        raise ValueError("s0 must hold one prior per group")
    s0_arr = (ctypes.c_float * group)(*s0)
    if out is None:
        out = torch.empty((N, ho, wo, C), dtype=input.dtype, device=input.device)
    _require(out, "out", input.dtype, (N, ho, wo, C))
    ws = _forward_scratch(desc, input, workspace, defer_escapes)
    if ws is None:
        _check("msdcn_forward", load().msdcn_forward(
            ctypes.byref(desc), _ptr(input), _ptr(dir_weight), _ptr(scale_raw), s0_arr,
            float(smax), _ptr(out), _stream(input)))
    else:
        _check("msdcn_forward_ws", load().msdcn_forward_ws(
            ctypes.byref(desc), _ptr(input), _ptr(dir_weight), _ptr(scale_raw), s0_arr,
            float(smax), _ptr(out), ws[0], ws[1], _stream(input)))
    return out


def msdcn_backward(input, dir_weight, scale_raw, s0, smax, grad_out, group, kernel_size=3,
                   stride=1, pad=1, dilation=1, offset_scale=1.0, algo="auto", workspace=None,
                   grad_input=None, grad_dir_weight=None, grad_scale_raw=None, math="default",
                   msdcn_mode="offset"):
    """MSDCN backward -> (grad_input, grad_dir_weight, grad_scale_raw)."""
    desc = _desc_for(input, group, kernel_size, stride, pad, dilation, offset_scale, algo, math,
                     False, msdcn_mode)
    ho, wo = dcn4_out_shape(desc)
    N, H, W, C = input.shape
    _require(input, "input", input.dtype)
    _require(dir_weight, "dir_weight", input.dtype, (N, ho, wo, group, desc.kh * desc.kw, 3))
    _require(scale_raw, "scale_raw", input.dtype, (N, ho, wo, group))
    _require(grad_out, "grad_out", input.dtype, (N, ho, wo, C))
    s0 = [float(v) for v in (s0.tolist() if isinstance(s0, torch.Tensor) else s0)]
    if len(s0) != group:
        raise ValueError("s0 must hold one prior per group")
    s0_arr = (ctypes.c_float * group)(*s0)
    if grad_input is None:
        grad_input = torch.empty_like(input)
    if grad_dir_weight is None:
        grad_dir_weight = torch.empty_like(dir_weight)
    if grad_scale_raw is None:
        grad_scale_raw = torch.empty_like(scale_raw)
    need = dcn4_backward_workspace_size(desc)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=input.device)
    ws_ptr = _ptr(workspace) if workspace is not None else ctypes.c_void_p(0)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("msdcn_backward", load().msdcn_backward(
        ctypes.byref(desc), _ptr(input), _ptr(dir_weight), _ptr(scale_raw), s0_arr, float(smax),
        _ptr(grad_out), _ptr(grad_input), _ptr(grad_dir_weight), _ptr(grad_scale_raw), ws_ptr,
        ws_bytes, _stream(input)))
    return grad_input, grad_dir_weight, grad_scale_raw


def dcn4_status_string(code):
    return load().dcn4_status_string(int(code)).decode()


def dcn4_selftest_bounded_wait(timeout_us=2000):
    """Launches the kernel whose bounded wait must expire (see the header)."""
    _check("dcn4_selftest_bounded_wait", load().dcn4_selftest_bounded_wait(
        int(timeout_us), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)))


def dcn4_kernel_launches():
    """Kernels the library has issued in this process (graph captures count
    once, replays not at all)."""
    n = ctypes.c_ulonglong()
    _check("dcn4_kernel_launches", load().dcn4_kernel_launches(ctypes.byref(n)))
    return n.value


def dcn4_last_device_error():
    """(status, raw bits) of the device error word, which it clears."""
    bits = ctypes.c_uint()
    rc = load().dcn4_last_device_error(ctypes.byref(bits))
    return rc, bits.value
