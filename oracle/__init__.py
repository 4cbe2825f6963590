"""ctypes front end of the CPU oracle for DCNv4 / MSDCN.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the package smoke check
and by the benchmark's CPU-baseline leg, never by the product path. Inputs
are float32 numpy arrays holding the values exactly as the device stores them
(bf16/fp16 values widen to float32 exactly); results are float64.
"""
import ctypes
import os

import numpy as np

from . import build as _build


class OrcProblem(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int) for name in
                ("N", "H", "W", "C", "G", "kh", "kw", "sh", "sw", "ph", "pw", "dh", "dw")] + \
               [("offset_scale", ctypes.c_float), ("softmax", ctypes.c_int),
                ("msdcn_dilation", ctypes.c_int)]


_F32P = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_F64P = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")


class Oracle:
    """One loaded copy of the oracle library (the tests may load mutants)."""

    def __init__(self, path=None):
        path = path or _build.build()
        self.path = path
        lib = ctypes.CDLL(path)
        P = ctypes.POINTER(OrcProblem)
        lib.orc_out_hw.argtypes = [P, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
        lib.orc_out_hw.restype = ctypes.c_int
        lib.orc_dcn4_forward.argtypes = [P, _F32P, _F32P, _F64P]
        lib.orc_dcn4_forward.restype = ctypes.c_int
        lib.orc_dcn4_backward.argtypes = [P, _F32P, _F32P, _F32P, _F64P, _F64P]
        lib.orc_dcn4_backward.restype = ctypes.c_int
        lib.orc_msdcn_forward.argtypes = [P, _F32P, _F32P, _F32P, _F32P, ctypes.c_float, _F64P]
        lib.orc_msdcn_forward.restype = ctypes.c_int
        lib.orc_msdcn_backward.argtypes = [P, _F32P, _F32P, _F32P, _F32P, ctypes.c_float, _F32P,
                                           _F64P, _F64P, _F64P]
        lib.orc_msdcn_backward.restype = ctypes.c_int
        lib.orc_offset_producer.argtypes = [P, _F32P, _F32P, _F32P, _F32P, _F32P, _F64P]
        lib.orc_offset_producer.restype = ctypes.c_int
        lib.orc_msdcn_scale.argtypes = [ctypes.c_float, ctypes.c_float, ctypes.c_float]
        lib.orc_msdcn_scale.restype = ctypes.c_float
        for name in ("orc_flops",):
            getattr(lib, name).argtypes = [P]
            getattr(lib, name).restype = ctypes.c_double
        for name in ("orc_ideal_bytes", "orc_worst_bytes"):
            getattr(lib, name).argtypes = [P, ctypes.c_int]
            getattr(lib, name).restype = ctypes.c_double
        self.lib = lib

    def set_threads(self, n):
        """Threads of the oracle's OpenMP loops (a timing knob: the loops are
        parallel over independent outputs, so results do not depend on it)."""
        self.lib.omp_set_num_threads(ctypes.c_int(int(n)))

    # -- problem description -------------------------------------------------
    @staticmethod
    def problem(N, H, W, C, G, kh=3, kw=3, stride=(1, 1), pad=(1, 1), dilation=(1, 1),
                offset_scale=1.0, softmax=False, msdcn_dilation=False):
        return OrcProblem(N, H, W, C, G, kh, kw, stride[0], stride[1], pad[0], pad[1],
                          dilation[0], dilation[1], offset_scale, int(bool(softmax)),
                          int(bool(msdcn_dilation)))

    def out_hw(self, prob):
        ho, wo = ctypes.c_int(), ctypes.c_int()
        if self.lib.orc_out_hw(ctypes.byref(prob), ctypes.byref(ho), ctypes.byref(wo)):
            raise ValueError("malformed problem")
        return ho.value, wo.value

    # -- operators -----------------------------------------------------------
    @staticmethod
    def _f32(a):
        return np.ascontiguousarray(np.asarray(a, dtype=np.float32))

    def forward(self, prob, inp, offset_weight):
        ho, wo = self.out_hw(prob)
        out = np.empty((prob.N, ho, wo, prob.C), np.float64)
        rc = self.lib.orc_dcn4_forward(ctypes.byref(prob), self._f32(inp),
                                       self._f32(offset_weight), out)
        if rc:
            raise ValueError("orc_dcn4_forward failed")
        return out

    def backward(self, prob, inp, offset_weight, grad_out):
        ho, wo = self.out_hw(prob)
        gin = np.empty((prob.N, prob.H, prob.W, prob.C), np.float64)
        gow = np.empty((prob.N, ho, wo, prob.G, prob.kh * prob.kw, 3), np.float64)
        rc = self.lib.orc_dcn4_backward(ctypes.byref(prob), self._f32(inp),
                                        self._f32(offset_weight), self._f32(grad_out), gin, gow)
        if rc:
            raise ValueError("orc_dcn4_backward failed")
        return gin, gow

    def msdcn_forward(self, prob, inp, dir_weight, scale_raw, s0, smax):
        ho, wo = self.out_hw(prob)
        out = np.empty((prob.N, ho, wo, prob.C), np.float64)
        rc = self.lib.orc_msdcn_forward(ctypes.byref(prob), self._f32(inp), self._f32(dir_weight),
                                        self._f32(scale_raw), self._f32(s0), float(smax), out)
        if rc:
            raise ValueError("orc_msdcn_forward failed")
        return out

    def msdcn_backward(self, prob, inp, dir_weight, scale_raw, s0, smax, grad_out):
        ho, wo = self.out_hw(prob)
        gin = np.empty((prob.N, prob.H, prob.W, prob.C), np.float64)
        gdw = np.empty((prob.N, ho, wo, prob.G, prob.kh * prob.kw, 3), np.float64)
        graw = np.empty((prob.N, ho, wo, prob.G), np.float64)
        rc = self.lib.orc_msdcn_backward(ctypes.byref(prob), self._f32(inp), self._f32(dir_weight),
                                         self._f32(scale_raw), self._f32(s0), float(smax),
                                         self._f32(grad_out), gin, gdw, graw)
        if rc:
            raise ValueError("orc_msdcn_backward failed")
        return gin, gdw, graw

    def offset_producer(self, prob, x, dw_weight, dw_bias, lin_weight, lin_bias):
        """offset_weight [N][H][W][G][kh*kw][3] from the depthwise 3x3 + linear
        sub-network (dw_weight [3][3][C], lin_weight [G*kh*kw*3][C])."""
        J = prob.G * prob.kh * prob.kw * 3
        out = np.empty((prob.N, prob.H, prob.W, J), np.float64)
        rc = self.lib.orc_offset_producer(ctypes.byref(prob), self._f32(x), self._f32(dw_weight),
                                          self._f32(dw_bias), self._f32(lin_weight),
                                          self._f32(lin_bias), out)
        if rc:
            raise ValueError("orc_offset_producer failed")
        return out.reshape(prob.N, prob.H, prob.W, prob.G, prob.kh * prob.kw, 3)

    def msdcn_scale(self, raw, s0, smax):
        return self.lib.orc_msdcn_scale(float(raw), float(s0), float(smax))

    # -- cost model ----------------------------------------------------------
    def flops(self, prob):
        return self.lib.orc_flops(ctypes.byref(prob))

    def ideal_bytes(self, prob, elem_bytes):
        return self.lib.orc_ideal_bytes(ctypes.byref(prob), elem_bytes)

    def worst_bytes(self, prob, elem_bytes):
        return self.lib.orc_worst_bytes(ctypes.byref(prob), elem_bytes)


_default = None


def default():
    """The oracle built from the committed source (cached per process)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
