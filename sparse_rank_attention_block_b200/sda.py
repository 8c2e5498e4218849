"""Python binding of the sda C ABI (include/sda.h).

Argument marshalling only: every step of the path runs in libsda.so's sm_100a
kernels. Functions carry the C names and take torch CUDA tensors (or raw
pointers) plus a stream; `forward` is a convenience wrapper that allocates the
output and the workspace with torch and calls `sda_forward`.

Importing this module does not need a GPU; calling into the library does.
There is no CPU fallback: if libsda.so is missing the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from .synthetic import Workload

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsda.so")

SDA_OK = 0
ERRORS = {-1: "SDA_ERR_NULLPTR", -2: "SDA_ERR_ALIGN", -3: "SDA_ERR_SHAPE", -4: "SDA_ERR_UNSUPPORTED",
          -5: "SDA_ERR_WORKSPACE", -6: "SDA_ERR_LAUNCH", -7: "SDA_ERR_TIMEOUT", -8: "SDA_ERR_DEVICE"}

# every symbol include/sda.h declares
EXPORTS = ["sda_keep_count", "sda_query_blocks", "sda_workspace_size", "sda_workspace_init", "sda_read_status", "sda_block_select",
           "sda_sparse_attn_fwd", "sda_lowrank_fwd", "sda_backward", "sda_backward_workspace_size", "sda_lowrank_fwd_static", "sda_gate_fuse", "sda_qk_prologue", "sda_quant_fp8",
           "sda_forward", "sda_forward_profiled",
           "sda_forward_host_buffer_size", "sda_forward_host", "sda_set_attention_wait_limit_ns",
           "sda_error_string", "sda_last_error_detail", "sda_version"]


class SdaParams(ctypes.Structure):
    """Mirror of `sda_params` (include/sda.h)."""

    _fields_ = [("B", ctypes.c_int32), ("L", ctypes.c_int32), ("H", ctypes.c_int32), ("d", ctypes.c_int32),
                ("grid_t", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
                ("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32), ("sparsity", ctypes.c_double),
                ("rank", ctypes.c_int32), ("pairs_t", ctypes.c_int32), ("pairs_h", ctypes.c_int32),
                ("pairs_w", ctypes.c_int32), ("rope_base", ctypes.c_double), ("rms_eps", ctypes.c_double),
                ("gate_per_head", ctypes.c_int32), ("causal_frames", ctypes.c_int32)]


def params_of(w: Workload) -> SdaParams:
    return SdaParams(B=w.B, L=w.L, H=w.H, d=w.d, grid_t=w.grid_t, grid_h=w.grid_h, grid_w=w.grid_w,
                     block_q=w.block_q, block_k=w.block_k, sparsity=w.sparsity, rank=w.rank,
                     pairs_t=w.pairs_t, pairs_h=w.pairs_h, pairs_w=w.pairs_w, rope_base=w.rope_base,
                     rms_eps=w.rms_eps, gate_per_head=w.gate_per_head, causal_frames=w.causal_frames)


class SdaError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str):
        super().__init__(f"{where}: {ERRORS.get(code, code)}: {detail}")
        self.code = code


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libsda.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python sparse_rank_attention_block_b200/build.py`; there is no fallback")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
        pp = ctypes.POINTER(SdaParams)
        sig = {
            "sda_keep_count": (i32, [pp]),
            "sda_query_blocks": (i32, [pp]),
            "sda_workspace_size": (sz, [pp]),
            "sda_workspace_init": (i32, [vp, sz, vp]),
            "sda_read_status": (i32, [vp, sz, vp]),
            "sda_block_select": (i32, [pp, vp, vp, vp, vp, sz, vp]),
            "sda_sparse_attn_fwd": (i32, [pp, vp, vp, vp, vp, vp, vp, sz, vp]),
            "sda_lowrank_fwd": (i32, [pp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
            "sda_lowrank_fwd_static": (i32, [pp, vp, vp, vp, vp, vp, vp, vp, vp]),
            "sda_gate_fuse": (i32, [pp, vp, vp, vp, vp, vp]),
            "sda_backward_workspace_size": (sz, [pp]),
            "sda_backward": (i32, [pp] + [vp] * 15 + [sz, vp]),
            "sda_quant_fp8": (i32, [pp, vp, vp, vp, vp]),
            "sda_qk_prologue": (i32, [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
            "sda_forward": (i32, [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
            "sda_forward_profiled": (i32, [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, ctypes.POINTER(vp), vp]),
            "sda_forward_host_buffer_size": (sz, [pp]),
            "sda_forward_host": (i32, [pp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
            "sda_set_attention_wait_limit_ns": (ctypes.c_uint64, [ctypes.c_uint64]),
            "sda_error_string": (ctypes.c_char_p, [i32]),
            "sda_last_error_detail": (ctypes.c_char_p, []),
            "sda_version": (ctypes.c_char_p, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(code: int, where: str) -> int:
    if code < 0:
        raise SdaError(code, where, lib().sda_last_error_detail().decode())
    return code


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ---------------------------------------------------------------------------
# thin wrappers with the C names
# ---------------------------------------------------------------------------

def sda_keep_count(p: SdaParams) -> int:
    return _check(lib().sda_keep_count(ctypes.byref(p)), "sda_keep_count")


def sda_query_blocks(p: SdaParams) -> int:
    return _check(lib().sda_query_blocks(ctypes.byref(p)), "sda_query_blocks")


def sda_workspace_size(p: SdaParams) -> int:
    n = lib().sda_workspace_size(ctypes.byref(p))
    if n == 0:
        raise SdaError(-3, "sda_workspace_size", lib().sda_last_error_detail().decode())
    return n


def sda_workspace_init(ws, nbytes: int, stream=None) -> None:
    _check(lib().sda_workspace_init(_ptr(ws), nbytes, _stream(stream)), "sda_workspace_init")


def sda_read_status(ws, nbytes: int, stream=None) -> None:
    _check(lib().sda_read_status(_ptr(ws), nbytes, _stream(stream)), "sda_read_status")


def sda_block_select(p, q, k, block_idx, ws, nbytes, stream=None) -> None:
    _check(lib().sda_block_select(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(block_idx), _ptr(ws), nbytes,
                                  _stream(stream)), "sda_block_select")


def sda_sparse_attn_fwd(p, q, k, v, block_idx, o_s, ws, nbytes, stream=None) -> None:
    _check(lib().sda_sparse_attn_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(block_idx), _ptr(o_s),
                                     _ptr(ws), nbytes, _stream(stream)), "sda_sparse_attn_fwd")


def sda_lowrank_fwd(p, q, k, v, p_q, p_k, o_lr, c_out, ws, nbytes, stream=None) -> None:
    _check(lib().sda_lowrank_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(p_q), _ptr(p_k), _ptr(o_lr),
                                 _ptr(c_out), _ptr(ws), nbytes, _stream(stream)), "sda_lowrank_fwd")


def sda_lowrank_fwd_static(p, q, k, v, p_q, p_k, o_lr, c_out, stream=None) -> None:
    """sda_lowrank_fwd with its scratch in the library's static device array (no workspace)."""
    _check(lib().sda_lowrank_fwd_static(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(p_q), _ptr(p_k),
                                        _ptr(o_lr), _ptr(c_out), _stream(stream)), "sda_lowrank_fwd_static")


def sda_backward_workspace_size(p: SdaParams) -> int:
    n = lib().sda_backward_workspace_size(ctypes.byref(p))
    if n == 0:
        raise SdaError(-4, "sda_backward_workspace_size", lib().sda_last_error_detail().decode())
    return n


def sda_backward(p, q, k, v, p_q, p_k, g, block_idx, d_o, dq, dk, dv, dp_q, dp_k, dg, ws, nbytes,
                 stream=None) -> None:
    args = [_ptr(x) for x in (q, k, v, p_q, p_k, g, block_idx, d_o, dq, dk, dv, dp_q, dp_k, dg, ws)]
    _check(lib().sda_backward(ctypes.byref(p), *args, nbytes, _stream(stream)), "sda_backward")


def sda_gate_fuse(p, o_s, o_lr, g, o, stream=None) -> None:
    _check(lib().sda_gate_fuse(ctypes.byref(p), _ptr(o_s), _ptr(o_lr), _ptr(g), _ptr(o), _stream(stream)),
           "sda_gate_fuse")


def sda_qk_prologue(p, q_raw, k_raw, w_q, w_k, q_norm, k_norm, q_rot, k_rot, stream=None) -> None:
    _check(lib().sda_qk_prologue(ctypes.byref(p), _ptr(q_raw), _ptr(k_raw), _ptr(w_q), _ptr(w_k), _ptr(q_norm),
                                 _ptr(k_norm), _ptr(q_rot), _ptr(k_rot), _stream(stream)), "sda_qk_prologue")


def sda_quant_fp8(p, x, x_q, scale, stream=None) -> None:
    _check(lib().sda_quant_fp8(ctypes.byref(p), _ptr(x), _ptr(x_q), _ptr(scale), _stream(stream)), "sda_quant_fp8")


def sda_forward(p, q, k, v, p_q, p_k, g, o, block_idx_out, ws, nbytes, stream=None) -> None:
    _check(lib().sda_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(p_q), _ptr(p_k), _ptr(g), _ptr(o),
                             _ptr(block_idx_out), _ptr(ws), nbytes, _stream(stream)), "sda_forward")


def sda_forward_profiled(p, q, k, v, p_q, p_k, g, o, block_idx_out, ws, nbytes, events, stream=None) -> None:
    """events: 5 cudaEvent_t handles (ints), recorded around the four stages."""
    arr = (ctypes.c_void_p * 5)(*events)
    _check(lib().sda_forward_profiled(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(p_q), _ptr(p_k), _ptr(g),
                                      _ptr(o), _ptr(block_idx_out), _ptr(ws), nbytes, arr, _stream(stream)),
           "sda_forward_profiled")


def sda_forward_host_buffer_size(p: SdaParams) -> int:
    return lib().sda_forward_host_buffer_size(ctypes.byref(p))


def sda_forward_host(p, q_host, k_host, v_host, p_q_host, p_k_host, g_host, o_host, dev_buf, nbytes,
                     stream=None) -> None:
    _check(lib().sda_forward_host(ctypes.byref(p), _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(p_q_host),
                                  _ptr(p_k_host), _ptr(g_host), _ptr(o_host), _ptr(dev_buf), nbytes,
                                  _stream(stream)), "sda_forward_host")


def sda_set_attention_wait_limit_ns(limit_ns: int) -> int:
    """Failure-path diagnostic: limit of the attention kernel's progress waits; returns the previous one."""
    return lib().sda_set_attention_wait_limit_ns(limit_ns)


def sda_version() -> str:
    return lib().sda_version().decode()


# ---------------------------------------------------------------------------
# convenience
# ---------------------------------------------------------------------------

class Workspace:
    """A caller-owned device workspace (torch allocation) sized for `p`."""

    def __init__(self, p: SdaParams, device=None, stream=None):
        self.nbytes = sda_workspace_size(p)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device or "cuda")
        off = (-self.buf.data_ptr()) % 256
        self.ptr = self.buf.data_ptr() + off
        sda_workspace_init(self.ptr, self.nbytes, stream)

    def check(self, stream=None) -> None:
        sda_read_status(self.ptr, self.nbytes, stream)


def forward(p: SdaParams, q, k, v, p_q, p_k, g, ws: Optional[Workspace] = None, block_idx=None, stream=None):
    """Allocate o (like q), run sda_forward, return o."""
    ws = ws or Workspace(p, device=q.device, stream=stream)
    o = torch.empty_like(q)
    sda_forward(p, q, k, v, p_q, p_k, g, o, block_idx, ws.ptr, ws.nbytes, stream)
    return o
