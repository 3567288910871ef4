"""BinaryAttention forward pass for NVIDIA B200 (sm_100a).

Every step of the path runs in the CUDA kernels of the C-ABI library
``libbinattn.so`` (built from ``csrc/`` by ``build.py``). This module only marshals
arguments: it takes torch CUDA tensors, allocates outputs and workspace with torch,
and passes raw device pointers plus the current stream. There is no CPU fallback: if
the library is missing, every call raises.

Functions mirror the C entry points of ``include/binattn.h``:
``pack_signs``, ``quant_v``, ``attention_fwd``, ``attention_fwd_packed``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Tuple

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbinattn.so")

BA_F16, BA_BF16, BA_F32 = 0, 1, 2
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024  # BA_NOALLOC_SCRATCH_BYTES of include/binattn.h
BIAS_NONE, BIAS_DENSE, BIAS_RELPOS2D = 0, 1, 2
IMPL_AUTO, IMPL_SIMT, IMPL_TCGEN05 = 0, 1, 2

STATUS = {0: "BA_OK", 1: "BA_ERR_INVALID_ARG", 2: "BA_ERR_UNSUPPORTED", 3: "BA_ERR_ALIGNMENT",
          4: "BA_ERR_WORKSPACE", 5: "BA_ERR_CUDA", 6: "BA_ERR_TIMEOUT"}


class BinAttnError(RuntimeError):
    def __init__(self, status: int, where: str, cuda_error: int = 0):
        self.status = status
        msg = f"{where}: {STATUS.get(status, status)}"
        if status == 5:
            msg += f" (cudaError {cuda_error})"
        super().__init__(msg)


class CBias(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("data", ctypes.c_void_p), ("batch_stride", ctypes.c_int64),
                ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int), ("table_h", ctypes.c_int),
                ("table_w", ctypes.c_int), ("n_prefix", ctypes.c_int)]


_lib = None

_P, _I, _F, _SZ, _I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_int64
SIGNATURES = {
    "ba_sign_words": (_I, [_I]),
    "ba_v_row_bytes": (_I, [_I]),
    "ba_kv_block": (_I, []),
    "ba_p_code_threshold": (ctypes.c_double, [_I]),
    "ba_prep_fused": (_I, [_I, _I, _I, _I]),
    "ba_pack_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "ba_quant_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "ba_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "ba_pack_signs": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _SZ, _P]),
    "ba_quant_v": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _SZ, _P]),
    "ba_attention_fwd_packed": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, ctypes.POINTER(CBias), _F, _P,
                                     _I, _P, _P]),
    "ba_attention_fwd": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, ctypes.POINTER(CBias), _F, _P, _I, _P, _SZ,
                              _P, _P]),
    "ba_attention_fwd_debug": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, ctypes.POINTER(CBias), _F, _P, _I, _P, _SZ,
                                    _P, _P, _I, _P]),
    "ba_attention_fwd_noalloc": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, ctypes.POINTER(CBias), _F, _P, _I, _P,
                                      _P]),
    "ba_set_attention_impl": (_I, [_I]),
    "ba_get_attention_impl": (_I, []),
    "ba_last_attention_impl": (_I, []),
    "ba_check_device_status": (_I, [_P]),
    "ba_stage_timing": (_I, [_I]),
    "ba_stage_times": (_I, [ctypes.POINTER(ctypes.c_float), _I, ctypes.POINTER(ctypes.c_int)]),
    "ba_status_string": (ctypes.c_char_p, [_I]),
    "ba_last_cuda_error": (_I, []),
}


def lib(path: Optional[str] = None) -> ctypes.CDLL:
    """The loaded C-ABI library. Raises if it has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libbinattn.so not found at {p}: build it with "
                           "`python -m bit_qk_attention_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = L
    return L


def _check(status: int, where: str):
    if status != 0:
        raise BinAttnError(status, where, lib().ba_last_cuda_error())


# ----------------------------------------------------------------------------- helpers
def _torch():
    import torch
    return torch


def _dt(t) -> int:
    torch = _torch()
    if t.dtype == torch.float16:
        return BA_F16
    if t.dtype == torch.bfloat16:
        return BA_BF16
    if t.dtype == torch.float32:
        return BA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _qkv_check(*ts):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [B,H,N,d]")


@dataclass
class Bias:
    """The additive logit bias (see include/binattn.h, ba_bias)."""
    kind: int = BIAS_NONE
    data: Optional[object] = None  # torch fp32 CUDA tensor
    batch_stride: int = 0
    grid_h: int = 0
    grid_w: int = 0
    table_h: int = 0
    table_w: int = 0
    n_prefix: int = 0

    def c(self) -> CBias:
        b = CBias()
        b.kind = self.kind
        b.data = 0 if self.data is None else self.data.data_ptr()
        b.batch_stride = self.batch_stride
        b.grid_h, b.grid_w = self.grid_h, self.grid_w
        b.table_h, b.table_w, b.n_prefix = self.table_h, self.table_w, self.n_prefix
        return b


def sign_words(d: int) -> int:
    return lib().ba_sign_words(d)


def v_row_bytes(d: int) -> int:
    return lib().ba_v_row_bytes(d)


def kv_block() -> int:
    return lib().ba_kv_block()


def p_code_threshold(k: int) -> float:
    """The least d = s - m (double) whose 8-bit P code exceeds k (0 <= k <= 254), else NaN."""
    return lib().ba_p_code_threshold(int(k))


def prep_fused(B: int, H: int, N: int, d: int) -> bool:
    """Whether attention_fwd prepares q, k, v in one launch for this shape (see ba_prep_fused)."""
    return bool(lib().ba_prep_fused(B, H, N, d))


def workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return lib().ba_workspace_bytes(B, H, N, d)


def set_attention_impl(impl: int):
    _check(lib().ba_set_attention_impl(impl), "ba_set_attention_impl")


def get_attention_impl() -> int:
    return lib().ba_get_attention_impl()


def last_attention_impl() -> int:
    return lib().ba_last_attention_impl()


def stage_timing(enable: bool):
    """Turn per-stage CUDA-event timing of attention_fwd on or off (measurement only)."""
    _check(lib().ba_stage_timing(1 if enable else 0), "ba_stage_timing")


def stage_times():
    """(ms per stage summed over calls [stream, finalize, quantise, attention], number of calls)."""
    ms = (ctypes.c_float * 4)()
    calls = ctypes.c_int(0)
    _check(lib().ba_stage_times(ms, 4, ctypes.byref(calls)), "ba_stage_times")
    return [float(x) for x in ms], calls.value


def check_device_status(stream=None):
    _check(lib().ba_check_device_status(_stream(stream)), "ba_check_device_status")


# ----------------------------------------------------------------------------- entry points
def pack_signs(x, stream=None) -> Tuple[object, object]:
    """x [B,H,N,d] fp16/bf16 -> (bits uint32-as-int32 [B,H,N,4], mu fp32 [B,H])."""
    torch = _torch()
    _qkv_check(x)
    B, H, N, d = x.shape
    bits = torch.empty((B, H, N, 4), dtype=torch.int32, device=x.device)
    mu = torch.empty((B, H), dtype=torch.float32, device=x.device)
    nws = lib().ba_pack_workspace_bytes(B, H, N, d)
    nws = 0 if nws == ctypes.c_size_t(-1).value else nws
    ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=x.device)
    _check(lib().ba_pack_signs(_ptr(x), _dt(x), B, H, N, d, _ptr(bits), _ptr(mu), _ptr(ws), nws,
                               _stream(stream)), "ba_pack_signs")
    return bits, mu


def quant_v(v, stream=None) -> Tuple[object, object]:
    """v [B,H,N,d] fp16/bf16 -> (vq int8 [B,H,N,v_row_bytes(d)], v_scale fp32 [B,H,d])."""
    torch = _torch()
    _qkv_check(v)
    B, H, N, d = v.shape
    vq = torch.empty((B, H, N, max(v_row_bytes(d), 1)), dtype=torch.int8, device=v.device)
    vs = torch.empty((B, H, d), dtype=torch.float32, device=v.device)
    nws = lib().ba_quant_workspace_bytes(B, H, N, d)
    nws = 0 if nws == ctypes.c_size_t(-1).value else nws
    ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=v.device)
    _check(lib().ba_quant_v(_ptr(v), _dt(v), B, H, N, d, _ptr(vq), _ptr(vs), _ptr(ws), nws, _stream(stream)),
           "ba_quant_v")
    return vq, vs


def attention_fwd_packed(bits_q, mu_q, bits_k, mu_k, vq, v_scale, d: int, bias: Optional[Bias] = None,
                         softmax_scale: float = 0.0, out=None, out_dtype=None, debug_logits: bool = False,
                         stream=None):
    """Fused step on packed operands. Returns O [B,H,N,d] (and int32 logits [B,H,N,N] if debug_logits)."""
    torch = _torch()
    B, H, N, _ = bits_q.shape
    if out is None:
        out = torch.empty((B, H, N, d), dtype=out_dtype or torch.float32, device=bits_q.device)
    dbg = torch.empty((B, H, N, N), dtype=torch.int32, device=bits_q.device) if debug_logits else None
    cb = (bias or Bias()).c()
    _check(lib().ba_attention_fwd_packed(_ptr(bits_q), _ptr(mu_q), _ptr(bits_k), _ptr(mu_k), _ptr(vq),
                                         _ptr(v_scale), B, H, N, d, ctypes.byref(cb), float(softmax_scale),
                                         _ptr(out), _dt(out), _ptr(dbg), _stream(stream)),
           "ba_attention_fwd_packed")
    return (out, dbg) if debug_logits else out


def attention_fwd(q, k, v, bias: Optional[Bias] = None, softmax_scale: float = 0.0, out=None,
                  out_dtype=None, workspace=None, debug_logits: bool = False, stream=None):
    """The whole forward pass. q, k, v [B,H,N,d] fp16/bf16 CUDA tensors."""
    torch = _torch()
    _qkv_check(q, k, v)
    if q.dtype != k.dtype or q.dtype != v.dtype or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share dtype and shape")
    B, H, N, d = q.shape
    if out is None:
        out = torch.empty((B, H, N, d), dtype=out_dtype or q.dtype, device=q.device)
    nws = lib().ba_workspace_bytes(B, H, N, d)
    if nws == ctypes.c_size_t(-1).value:  # unsupported size: the call below reports it
        nws = 0
    if workspace is None:
        workspace = torch.empty(max(nws, 1), dtype=torch.uint8, device=q.device)
    dbg = torch.empty((B, H, N, N), dtype=torch.int32, device=q.device) if debug_logits else None
    cb = (bias or Bias()).c()
    _check(lib().ba_attention_fwd(_ptr(q), _ptr(k), _ptr(v), _dt(q), B, H, N, d, ctypes.byref(cb),
                                  float(softmax_scale), _ptr(out), _dt(out), _ptr(workspace),
                                  workspace.numel(), _ptr(dbg), _stream(stream)), "ba_attention_fwd")
    return (out, dbg) if debug_logits else out


def attention_fwd_debug(q, k, v, bias: Optional[Bias] = None, softmax_scale: float = 0.0, out_dtype=None,
                        check_all_codes: bool = False, stream=None):
    """The whole forward pass with its debug outputs: (O, int32 logits [B,H,N,N], uint8 P codes
    [B,H,N,N]). check_all_codes recomputes every near-tie code exactly (see ba_attention_fwd_debug)."""
    torch = _torch()
    _qkv_check(q, k, v)
    B, H, N, d = q.shape
    out = torch.empty((B, H, N, d), dtype=out_dtype or q.dtype, device=q.device)
    nws = lib().ba_workspace_bytes(B, H, N, d)
    nws = 0 if nws == ctypes.c_size_t(-1).value else nws
    workspace = torch.empty(max(nws, 1), dtype=torch.uint8, device=q.device)
    dbg = torch.empty((B, H, N, N), dtype=torch.int32, device=q.device)
    dbg_p = torch.empty((B, H, N, N), dtype=torch.uint8, device=q.device)
    cb = (bias or Bias()).c()
    _check(lib().ba_attention_fwd_debug(_ptr(q), _ptr(k), _ptr(v), _dt(q), B, H, N, d, ctypes.byref(cb),
                                        float(softmax_scale), _ptr(out), _dt(out), _ptr(workspace),
                                        workspace.numel(), _ptr(dbg), _ptr(dbg_p), 1 if check_all_codes else 0,
                                        _stream(stream)), "ba_attention_fwd_debug")
    return out, dbg, dbg_p


def bias_from_workload(w, device) -> Optional[Bias]:
    """Device Bias for a workload of bit_qk_attention_b200.inputs."""
    if w.bias_kind == BIAS_NONE or w.bias is None:
        return None
    return Bias(w.bias_kind, w.bias.to(device=device, dtype=_torch().float32).contiguous(), w.batch_stride,
                w.grid_h, w.grid_w, w.table_h, w.table_w, w.n_prefix)
