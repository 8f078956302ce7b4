"""Seeded synthetic inputs shared by the tests, the CPU reference checks and the benchmark.

Every element is a pure function of (seed, stream, row, col) defined in
``csa2_synth.h`` and produced bit-identically on the host (``libsynth_host.so``)
and on the device (``libsynth_dev.so``).  The module holds no arithmetic of the
method: it draws numbers only.  Workload shapes live in ``synth.workloads``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(_HERE, "libsynth_host.so")
DEV_LIB = os.path.join(_HERE, "libsynth_dev.so")

S_KIDX, S_KV, S_IQ, S_IW, S_QMAIN, S_SWA = 1, 2, 0x100, 0x200, 0x300, 0x400
KIND_NORMAL, KIND_UNIFORM = 0, 1


class SynTensor(ctypes.Structure):
    _fields_ = [
        ("seed", ctypes.c_uint64),
        ("stream", ctypes.c_uint64),
        ("dim", ctypes.c_int32),
        ("kind", ctypes.c_int32),
        ("outlier", ctypes.c_void_p),
        ("n_needle", ctypes.c_int32),
        ("needle_block", ctypes.c_int32),
        ("needle_blk", ctypes.c_void_p),
        ("needle_dir", ctypes.c_void_p),
        ("needle_shift", ctypes.c_float),
    ]


def _newer(out, *srcs):
    return os.path.exists(out) and all(os.path.getmtime(out) >= os.path.getmtime(s) for s in srcs)


def build(force: bool = False, device: bool = True) -> None:
    hdr = os.path.join(_HERE, "csa2_synth.h")
    src = os.path.join(_HERE, "synth_host.c")
    if force or not _newer(HOST_LIB, hdr, src):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", "-Wall", "-o", HOST_LIB, src])
    dsrc = os.path.join(_HERE, "synth_dev.cu")
    if device and (force or not _newer(DEV_LIB, hdr, dsrc)):
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
                               "-Xcompiler", "-fPIC", "-shared", "-o", DEV_LIB, dsrc])


_host = None
_dev = None


def host_lib():
    global _host
    if _host is None:
        build(device=False)
        L = ctypes.CDLL(HOST_LIB)
        P = ctypes.POINTER(SynTensor)
        L.syn_host_fill_f32.argtypes = [P, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        L.syn_host_fill_rows_f32.argtypes = [P, ctypes.c_uint32, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        L.syn_host_fill_bf16.argtypes = [P, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        L.syn_host_fill_e4m3.argtypes = [P, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_void_p, ctypes.c_void_p]
        L.syn_host_e4m3_code.restype = ctypes.c_uint8
        L.syn_host_e4m3_code.argtypes = [ctypes.c_float]
        L.syn_host_bf16.restype = ctypes.c_uint16
        L.syn_host_bf16.argtypes = [ctypes.c_float]
        L.syn_host_normal.restype = ctypes.c_float
        L.syn_host_normal.argtypes = [ctypes.c_uint64] * 4
        _host = L
    return _host


def dev_lib():
    global _dev
    if _dev is None:
        build()
        L = ctypes.CDLL(DEV_LIB)
        P = ctypes.POINTER(SynTensor)
        L.syn_dev_fill_f32.argtypes = [P, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                       ctypes.c_void_p]
        L.syn_dev_fill_bf16.argtypes = [P, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                        ctypes.c_void_p]
        L.syn_dev_fill_e4m3.argtypes = [P, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        _dev = L
    return _dev


class TensorSpec:
    """One synthetic tensor.  Host-side arrays for outliers/needles are kept
    alive here; ``device()`` returns a copy whose pointers are device memory."""

    def __init__(self, seed, stream, dim, kind=KIND_NORMAL, outlier=None, needle_blk=None,
                 needle_dir=None, needle_shift=2.0, needle_block=8):
        self.seed, self.stream, self.dim, self.kind = int(seed), int(stream), int(dim), int(kind)
        self.outlier = None if outlier is None else np.ascontiguousarray(outlier, np.uint8)
        self.needle_blk = None if needle_blk is None else np.ascontiguousarray(needle_blk, np.int32)
        self.needle_dir = None if needle_dir is None else np.ascontiguousarray(needle_dir, np.float32)
        self.needle_shift = float(needle_shift)
        self.needle_block = int(needle_block)
        self._dev_keep = None

    def _struct(self, outlier_ptr, blk_ptr, dir_ptr):
        n_needle = 0 if self.needle_blk is None else self.needle_blk.shape[1]
        return SynTensor(self.seed, self.stream, self.dim, self.kind, outlier_ptr, n_needle,
                         self.needle_block, blk_ptr, dir_ptr, self.needle_shift)

    def host(self) -> SynTensor:
        return self._struct(
            None if self.outlier is None else self.outlier.ctypes.data,
            None if self.needle_blk is None else self.needle_blk.ctypes.data,
            None if self.needle_dir is None else self.needle_dir.ctypes.data)

    def device(self, torch_device="cuda") -> SynTensor:
        import torch
        keep = []

        def up(a):
            if a is None:
                return None
            t = torch.from_numpy(a).to(torch_device)
            keep.append(t)
            return t.data_ptr()

        s = self._struct(up(self.outlier), up(self.needle_blk), up(self.needle_dir))
        self._dev_keep = keep
        return s

    # --- host fills -------------------------------------------------------
    def rows_f32(self, seq: int, pos0: int, n: int) -> np.ndarray:
        out = np.empty((n, self.dim), np.float32)
        if n:
            st = self.host()
            host_lib().syn_host_fill_f32(ctypes.byref(st), seq, pos0, n, out.ctypes.data)
        return out

    def select_rows_f32(self, seq: int, pos: np.ndarray) -> np.ndarray:
        pos = np.ascontiguousarray(pos, np.int64)
        out = np.empty((len(pos), self.dim), np.float32)
        if len(pos):
            st = self.host()
            host_lib().syn_host_fill_rows_f32(ctypes.byref(st), seq, pos.ctypes.data, len(pos), out.ctypes.data)
        return out

    def rows_bf16_bits(self, seq: int, pos0: int, n: int) -> np.ndarray:
        out = np.empty((n, self.dim), np.uint16)
        if n:
            st = self.host()
            host_lib().syn_host_fill_bf16(ctypes.byref(st), seq, pos0, n, out.ctypes.data)
        return out

    def rows_e4m3(self, seq: int, pos0: int, n: int, ring: int = 0):
        """FP8 rows; with ring > 0 row for position p lands in slot p % ring"""
        m = ring if ring > 0 else n
        codes = np.zeros((m, self.dim), np.uint8)
        scale = np.ones(m, np.float32)
        if n:
            st = self.host()
            host_lib().syn_host_fill_e4m3(ctypes.byref(st), seq, pos0, n, ring, codes.ctypes.data,
                                          scale.ctypes.data)
        return codes, scale

    # --- device fills (torch tensors / raw pointers) ----------------------
    def dev_rows_f32(self, seq, pos0, n, out_ptr, stream_ptr, st=None):
        st = st or self.device()
        rc = dev_lib().syn_dev_fill_f32(ctypes.byref(st), seq, pos0, n, out_ptr, stream_ptr)
        assert rc == 0, f"syn_dev_fill_f32 failed: {rc}"

    def dev_rows_bf16(self, seq, pos0, n, out_ptr, stream_ptr, st=None):
        st = st or self.device()
        rc = dev_lib().syn_dev_fill_bf16(ctypes.byref(st), seq, pos0, n, out_ptr, stream_ptr)
        assert rc == 0, f"syn_dev_fill_bf16 failed: {rc}"

    def dev_rows_e4m3(self, seq, pos0, n, ring, codes_ptr, scale_ptr, stream_ptr, st=None):
        st = st or self.device()
        rc = dev_lib().syn_dev_fill_e4m3(ctypes.byref(st), seq, pos0, n, ring, codes_ptr, scale_ptr, stream_ptr)
        assert rc == 0, f"syn_dev_fill_e4m3 failed: {rc}"


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)
