"""CPU oracle of the BinaryAttention forward pass — test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
import this package. The CUDA library never calls it and shares no code with it.

The arithmetic lives in ``oracle.cpp`` (plain C++17, no CUDA); this module compiles
it with ``g++`` and wraps its ``extern "C"`` functions for numpy arrays. Every
function of ``oracle.cpp`` is pinned by the CPU tests (identities, closed forms,
brute force, statistical laws and a mutation suite); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "oracle.cpp")
_BUILD_DIR = os.path.join(_HERE, "_build")
LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
CXXFLAGS = ["-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
            "-shared", "-fPIC"]

BIAS_NONE, BIAS_DENSE, BIAS_RELPOS2D = 0, 1, 2


def build(source: str = SOURCE, out: str = LIB_PATH, extra_flags: Sequence[str] = ()) -> str:
    """Compile ``source`` into a shared library at ``out`` (skipped when up to date)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if (os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(source)
            and not extra_flags):
        return out
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(["g++", *CXXFLAGS, *extra_flags, source, "-o", tmp], check=True)
    os.replace(tmp, out)
    return out


class _Bias(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("data", ctypes.c_void_p), ("batch_stride", ctypes.c_int64),
                ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int), ("table_h", ctypes.c_int),
                ("table_w", ctypes.c_int), ("n_prefix", ctypes.c_int)]


class _FwdArgs(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("H", ctypes.c_int64), ("N", ctypes.c_int64), ("d", ctypes.c_int),
                ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("bias", _Bias), ("softmax_scale", ctypes.c_float), ("block_c", ctypes.c_int),
                ("rowsum_mode", ctypes.c_int), ("num_threads", ctypes.c_int),
                ("n_rows", ctypes.c_int64), ("rows", ctypes.c_void_p)]


class _FwdDebug(ctypes.Structure):
    _fields_ = [("m_final", ctypes.c_void_p), ("l_final", ctypes.c_void_p), ("p_float", ctypes.c_void_p),
                ("p_u8", ctypes.c_void_p), ("s_logit", ctypes.c_void_p)]


@dataclass
class Bias:
    """Bias description (mirrors the C-ABI's fields; host numpy data)."""
    kind: int = BIAS_NONE
    data: Optional[np.ndarray] = None   # dense [H,N,N] (or [B,H,N,N] with batch_stride) / table [H,T]
    batch_stride: int = 0
    grid_h: int = 0
    grid_w: int = 0
    table_h: int = 0
    table_w: int = 0
    n_prefix: int = 0


def _f32(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """ctypes wrapper around one compiled oracle library."""

    def __init__(self, lib_path: Optional[str] = None):
        path = lib_path or build()
        self.lib = ctypes.CDLL(path)
        L = self.lib
        L.bao_version.restype = ctypes.c_int
        L.bao_pack_signs.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p]
        L.bao_mu.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p]
        L.bao_logits.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                 ctypes.c_int, ctypes.c_void_p]
        L.bao_quant_v.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                  ctypes.c_void_p, ctypes.c_void_p]
        L.bao_bias_materialize.argtypes = [ctypes.POINTER(_Bias), ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_void_p]
        for fn in (L.bao_attention_fwd,):
            fn.argtypes = [ctypes.POINTER(_FwdArgs), ctypes.c_void_p, ctypes.POINTER(_FwdDebug)]
            fn.restype = ctypes.c_int
        for fn in (L.bao_attention_twopass, L.bao_attention_fullprec):
            fn.argtypes = [ctypes.POINTER(_FwdArgs), ctypes.c_void_p]
            fn.restype = ctypes.c_int
        self.version = L.bao_version()

    # ---- step functions -------------------------------------------------------------
    def pack_signs(self, x: np.ndarray) -> np.ndarray:
        """x [..., d] -> uint32 [..., 4]."""
        x = _f32(x)
        d = x.shape[-1]
        rows = int(np.prod(x.shape[:-1]))
        out = np.zeros(x.shape[:-1] + (4,), dtype=np.uint32)
        self.lib.bao_pack_signs(_ptr(x), rows, d, _ptr(out))
        return out

    def mu(self, x: np.ndarray) -> np.ndarray:
        """x [B,H,N,d] -> fp32 [B,H]."""
        x = _f32(x)
        B, H, N, d = x.shape
        out = np.zeros((B, H), dtype=np.float32)
        self.lib.bao_mu(_ptr(x), B * H, N, d, _ptr(out))
        return out

    def logits(self, bq: np.ndarray, bk: np.ndarray, d: int) -> np.ndarray:
        """bits [B,H,N,4] x2 -> int32 [B,H,N,N]."""
        bq = np.ascontiguousarray(bq, dtype=np.uint32)
        bk = np.ascontiguousarray(bk, dtype=np.uint32)
        B, H, N, _ = bq.shape
        out = np.zeros((B, H, N, N), dtype=np.int32)
        self.lib.bao_logits(_ptr(bq), _ptr(bk), B * H, N, d, _ptr(out))
        return out

    def quant_v(self, v: np.ndarray):
        """v [B,H,N,d] -> (int8 [B,H,N,d], fp32 scales [B,H,d])."""
        v = _f32(v)
        B, H, N, d = v.shape
        vq = np.zeros((B, H, N, d), dtype=np.int8)
        sv = np.zeros((B, H, d), dtype=np.float32)
        self.lib.bao_quant_v(_ptr(v), B * H, N, d, _ptr(vq), _ptr(sv))
        return vq, sv

    def bias_materialize(self, bias: Bias, H: int, N: int) -> np.ndarray:
        keep = []
        cb = self._bias_struct(bias, keep)
        out = np.zeros((H, N, N), dtype=np.float32)
        self.lib.bao_bias_materialize(ctypes.byref(cb), H, N, _ptr(out))
        return out

    # ---- forward --------------------------------------------------------------------
    @staticmethod
    def _bias_struct(bias: Optional[Bias], keep: list) -> _Bias:
        cb = _Bias()
        if bias is None or bias.kind == BIAS_NONE:
            cb.kind = 0
            return cb
        data = _f32(bias.data)
        keep.append(data)
        cb.kind = bias.kind
        cb.data = data.ctypes.data
        cb.batch_stride = bias.batch_stride
        cb.grid_h, cb.grid_w = bias.grid_h, bias.grid_w
        cb.table_h, cb.table_w = bias.table_h, bias.table_w
        cb.n_prefix = bias.n_prefix
        return cb

    def _args(self, q, k, v, bias, softmax_scale, block_c, rowsum_mode, num_threads, rows, keep):
        q, k, v = _f32(q), _f32(k), _f32(v)
        keep.extend([q, k, v])
        B, H, N, d = q.shape
        a = _FwdArgs()
        a.B, a.H, a.N, a.d = B, H, N, d
        a.q, a.k, a.v = q.ctypes.data, k.ctypes.data, v.ctypes.data
        a.bias = self._bias_struct(bias, keep)
        a.softmax_scale = float(softmax_scale)
        a.block_c = int(block_c)
        a.rowsum_mode = int(rowsum_mode)
        a.num_threads = int(num_threads)
        if rows is not None:
            r = np.ascontiguousarray(rows, dtype=np.int64)
            keep.append(r)
            a.n_rows, a.rows = len(r), r.ctypes.data
        else:
            a.n_rows, a.rows = N, None
        return a

    def attention_fwd(self, q, k, v, bias: Optional[Bias] = None, softmax_scale: float = 0.0,
                      block_c: int = 128, rowsum_mode: int = 0, num_threads: int = 0,
                      rows: Optional[np.ndarray] = None, debug: bool = False):
        """Blockwise forward. Returns O fp32 [B,H,R,d] (R = N or len(rows)); with debug=True
        also a dict of per-row diagnostics."""
        keep: list = []
        a = self._args(q, k, v, bias, softmax_scale, block_c, rowsum_mode, num_threads, rows, keep)
        R = a.n_rows
        o = np.zeros((a.B, a.H, R, a.d), dtype=np.float32)
        dbg = _FwdDebug()
        extra = {}
        if debug:
            nrow = a.B * a.H * R
            extra = dict(m=np.zeros(nrow, np.float32), l=np.zeros(nrow, np.float64),
                         p=np.zeros((nrow, a.N), np.float32), pu8=np.zeros((nrow, a.N), np.uint8),
                         s=np.zeros((nrow, a.N), np.float32))
            dbg.m_final, dbg.l_final = extra["m"].ctypes.data, extra["l"].ctypes.data
            dbg.p_float, dbg.p_u8, dbg.s_logit = (extra["p"].ctypes.data, extra["pu8"].ctypes.data,
                                                  extra["s"].ctypes.data)
        rc = self.lib.bao_attention_fwd(ctypes.byref(a), _ptr(o), ctypes.byref(dbg) if debug else None)
        if rc != 0:
            raise ValueError(f"oracle rejected the arguments (rc={rc})")
        return (o, extra) if debug else o

    def attention_twopass(self, q, k, v, bias: Optional[Bias] = None, softmax_scale: float = 0.0):
        keep: list = []
        a = self._args(q, k, v, bias, softmax_scale, 1, 0, 1, None, keep)
        o = np.zeros((a.B, a.H, a.N, a.d), dtype=np.float32)
        if self.lib.bao_attention_twopass(ctypes.byref(a), _ptr(o)) != 0:
            raise ValueError("oracle rejected the arguments")
        return o

    def attention_fullprec(self, q, k, v, bias: Optional[Bias] = None, softmax_scale: float = 0.0):
        keep: list = []
        a = self._args(q, k, v, bias, softmax_scale, 1, 0, 1, None, keep)
        o = np.zeros((a.B, a.H, a.N, a.d), dtype=np.float32)
        self.lib.bao_attention_fullprec(ctypes.byref(a), _ptr(o))
        return o


_DEFAULT: Optional[Oracle] = None


def get() -> Oracle:
    """The oracle built from this directory's source (compiled on first use)."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT
