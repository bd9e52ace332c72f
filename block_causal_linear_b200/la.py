"""ctypes binding of libla_b200.so (the C ABI in include/la.h).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  The raw entry points keep their C names
(``la_workspace_size``, ``la_state_init``, ``la_block_forward``,
``la_full_forward``, ``la_device_status``, ``la_status_string``); the
lower-case wrappers below take torch CUDA tensors, pass their device pointers
and the current CUDA stream, and raise ``LAError`` on a non-zero status.

There is no fallback: if the library is missing or a call fails, this module
raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libla_b200.so")

LA_OK, LA_EINVAL, LA_EUNSUPPORTED, LA_ECUDA, LA_ETIMEOUT, LA_EWORKSPACE = range(6)
LA_F32, LA_BF16 = 0, 1


class LAError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {la_status_string(status)}" if what else la_status_string(status))


class la_rope(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("Hg", ctypes.c_int), ("Wg", ctypes.c_int),
                ("t_offset", ctypes.c_int), ("dt", ctypes.c_int), ("dh", ctypes.c_int),
                ("dw", ctypes.c_int), ("base", ctypes.c_float)]


class la_state(ctypes.Structure):
    _fields_ = [("S", ctypes.c_void_p), ("Z", ctypes.c_void_p), ("B", ctypes.c_int),
                ("H", ctypes.c_int), ("d", ctypes.c_int), ("blocks_committed", ctypes.c_longlong),
                ("t_next", ctypes.c_int)]


class la_state_counters(ctypes.Structure):
    _fields_ = [("blocks_committed", ctypes.c_longlong), ("t_next", ctypes.c_int)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libla_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m block_causal_linear_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, ip, fp, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.la_workspace_size.argtypes = [ip, ip, ip, ip, ip]
        L.la_workspace_size.restype = sz
        L.la_state_init.argtypes = [ctypes.POINTER(la_state), vp, vp, ip, ip, ip, vp]
        L.la_state_init.restype = ip
        L.la_state_save.argtypes = [ctypes.POINTER(la_state), vp, vp, ctypes.POINTER(la_state_counters), vp]
        L.la_state_save.restype = ip
        L.la_state_restore.argtypes = [ctypes.POINTER(la_state), vp, vp, ctypes.POINTER(la_state_counters), vp]
        L.la_state_restore.restype = ip
        L.la_block_forward.argtypes = [vp, vp, vp, vp, ip, ip, ip, ip, ip, ctypes.POINTER(la_state), ip,
                                       ctypes.POINTER(la_rope), fp, vp, sz, vp]
        L.la_block_forward.restype = ip
        L.la_full_forward.argtypes = [vp, vp, vp, vp, ip, ip, ip, ip, ip, ip, ctypes.POINTER(la_rope),
                                      fp, vp, sz, vp]
        L.la_full_forward.restype = ip
        L.la_full_forward_static_ws.argtypes = [vp, vp, vp, vp, ip, ip, ip, ip, ip, ip,
                                                ctypes.POINTER(la_rope), fp, vp]
        L.la_full_forward_static_ws.restype = ip
        L.la_full_forward_e4m3.argtypes = [vp, vp, vp, fp, fp, fp, vp, ip, ip, ip, ip, ip, ctypes.POINTER(la_rope),
                                           fp, vp, sz, vp]
        L.la_full_forward_e4m3.restype = ip
        L.la_block_forward_e4m3.argtypes = [vp, vp, vp, fp, fp, fp, vp, ip, ip, ip, ip, ctypes.POINTER(la_state), ip,
                                            ctypes.POINTER(la_rope), fp, vp, sz, vp]
        L.la_block_forward_e4m3.restype = ip
        L.la_full_forward_nvfp4.argtypes = [vp, vp, vp, vp, vp, vp, fp, fp, fp, vp, ip, ip, ip, ip, ip,
                                            ctypes.POINTER(la_rope), fp, vp, sz, vp]
        L.la_full_forward_nvfp4.restype = ip
        L.la_block_forward_nvfp4.argtypes = [vp, vp, vp, vp, vp, vp, fp, fp, fp, vp, ip, ip, ip, ip,
                                             ctypes.POINTER(la_state), ip, ctypes.POINTER(la_rope), fp, vp, sz, vp]
        L.la_block_forward_nvfp4.restype = ip
        L.la_dwconv3d.argtypes = [vp, vp, ip, ip, ip, ip, ip, ip, ip, ip, ip, vp, vp, vp]
        L.la_dwconv3d.restype = ip
        L.la_split_partial_bytes.argtypes = [ip, ip, ip]
        L.la_split_partial_bytes.restype = sz
        L.la_block_reduce.argtypes = [vp, vp, ip, ip, ip, ip, ip, ctypes.POINTER(la_rope), vp, vp, sz, vp]
        L.la_block_reduce.restype = ip
        L.la_block_apply.argtypes = [vp, vp, ip, ip, ip, ip, ip, vp, ip, ctypes.POINTER(la_state), ip,
                                     ctypes.POINTER(la_rope), fp, vp, sz, vp]
        L.la_block_apply.restype = ip
        L.la_backward_workspace_size.argtypes = [ip, ip, ip, ip, ip]
        L.la_backward_workspace_size.restype = sz
        L.la_full_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, ip, ip, ip, ip, ip, ip,
                                       ctypes.POINTER(la_rope), fp, vp, sz, vp]
        L.la_full_backward.restype = ip
        L.la_device_status.argtypes = [vp]
        L.la_device_status.restype = ip
        L.la_selftest_bounded_wait.argtypes = [vp]
        L.la_selftest_bounded_wait.restype = ip
        L.la_status_string.argtypes = [ip]
        L.la_status_string.restype = ctypes.c_char_p
        L.la_set_stage_events.argtypes = [vp, vp, vp, vp]
        L.la_set_stage_events.restype = None
        L.la_last_launch_count.argtypes = []
        L.la_last_launch_count.restype = ip
        L.la_tc_enabled.argtypes = []
        L.la_tc_enabled.restype = ip
        L.la_last_path.argtypes = []
        L.la_last_path.restype = ctypes.c_char_p
        _lib = L
    return _lib


# ---------------------------------------------------------------- raw C names

def la_workspace_size(B, N, H, d, tokens_per_block) -> int:
    return int(lib().la_workspace_size(B, N, H, d, tokens_per_block))


def la_state_init(st, S, Z, B, H, d, stream) -> int:
    return int(lib().la_state_init(ctypes.byref(st), S, Z, B, H, d, stream))


def la_state_save(st, S_dst, Z_dst, counters, stream) -> int:
    return int(lib().la_state_save(ctypes.byref(st), S_dst, Z_dst,
                                   ctypes.byref(counters) if counters is not None else None, stream))


def la_state_restore(st, S_src, Z_src, counters, stream) -> int:
    return int(lib().la_state_restore(ctypes.byref(st), S_src, Z_src,
                                      ctypes.byref(counters) if counters is not None else None, stream))


def la_block_forward(q, k, v, out, dt, B, N_blk, H, d, st, commit, rope, eps, ws, ws_bytes, stream) -> int:
    return int(lib().la_block_forward(q, k, v, out, dt, B, N_blk, H, d, ctypes.byref(st), commit,
                                      ctypes.byref(rope) if rope is not None else None, eps, ws,
                                      ws_bytes, stream))


def la_full_forward(q, k, v, out, dt, B, N, H, d, tokens_per_block, rope, eps, ws, ws_bytes, stream) -> int:
    return int(lib().la_full_forward(q, k, v, out, dt, B, N, H, d, tokens_per_block,
                                     ctypes.byref(rope) if rope is not None else None, eps, ws,
                                     ws_bytes, stream))


def la_full_forward_static_ws(q, k, v, out, dt, B, N, H, d, tokens_per_block, rope, eps, stream) -> int:
    """la_full_forward with the library's static device scratch (for callers
    that cannot allocate; see include/la.h)."""
    return int(lib().la_full_forward_static_ws(q, k, v, out, dt, B, N, H, d, tokens_per_block,
                                               ctypes.byref(rope) if rope is not None else None,
                                               eps, stream))


LA_STATIC_WS_BYTES = 16 << 20


def la_full_forward_e4m3(q, k, v, sq, sk, sv, out, B, N, H, d, tokens_per_block, rope, eps, ws, ws_bytes,
                         stream) -> int:
    return int(lib().la_full_forward_e4m3(q, k, v, sq, sk, sv, out, B, N, H, d, tokens_per_block,
                                          ctypes.byref(rope) if rope is not None else None, eps, ws, ws_bytes,
                                          stream))


def la_block_forward_e4m3(q, k, v, sq, sk, sv, out, B, N_blk, H, d, st, commit, rope, eps, ws, ws_bytes,
                          stream) -> int:
    return int(lib().la_block_forward_e4m3(q, k, v, sq, sk, sv, out, B, N_blk, H, d, ctypes.byref(st), commit,
                                           ctypes.byref(rope) if rope is not None else None, eps, ws, ws_bytes,
                                           stream))


def la_dwconv3d(x, y, dt, B, T, Hg, Wg, C, kt, kh, kw, weight, bias, stream) -> int:
    return int(lib().la_dwconv3d(x, y, dt, B, T, Hg, Wg, C, kt, kh, kw, weight, bias, stream))


def dwconv3d(x, weight, bias=None, out=None, stream=None):
    """Mix-FFN depthwise convolution: x [B, T, Hg, Wg, C] (bf16 or fp32 CUDA),
    weight [C, kt, kh, kw] fp32 CUDA ((1,3,3) or (3,1,1)), bias [C] or None."""
    if not x.is_cuda or not x.is_contiguous() or x.dim() != 5:
        raise ValueError("x must be a contiguous CUDA tensor [B, T, Hg, Wg, C]")
    if weight.dtype != torch.float32 or not weight.is_cuda or weight.dim() != 4 or not weight.is_contiguous():
        raise ValueError("weight must be a contiguous fp32 CUDA tensor [C, kt, kh, kw]")
    B, T, Hg, Wg, C = x.shape
    out = torch.empty_like(x) if out is None else out
    rc = la_dwconv3d(x.data_ptr(), out.data_ptr(), _dtype_code(x), B, T, Hg, Wg, C, *weight.shape[1:],
                     weight.data_ptr(), None if bias is None else bias.data_ptr(), _stream_ptr(stream))
    if rc != LA_OK:
        raise LAError(rc, "la_dwconv3d")
    return out


def la_split_partial_bytes(B, H, d) -> int:
    return int(lib().la_split_partial_bytes(B, H, d))


def la_block_reduce(k, v, dt, B, N, H, d, rope, partial, ws, ws_bytes, stream) -> int:
    return int(lib().la_block_reduce(k, v, dt, B, N, H, d, ctypes.byref(rope) if rope is not None else None,
                                     partial, ws, ws_bytes, stream))


def la_block_apply(q, out, dt, B, N, H, d, gathered, R, st, commit, rope, eps, ws, ws_bytes, stream) -> int:
    return int(lib().la_block_apply(q, out, dt, B, N, H, d, gathered, R, ctypes.byref(st), commit,
                                    ctypes.byref(rope) if rope is not None else None, eps, ws, ws_bytes, stream))


def block_reduce(k, v, rope=None, ws=None, partial=None, stream=None):
    """This rank's [KV | z] partial sums of a token slice: fp32 [B, H, 1056]."""
    _check_qkv(k, k, v)
    B, N, H, d = k.shape
    if ws is None:
        ws = alloc_workspace(B, N, H, d, N, device=k.device)
    if partial is None:
        partial = torch.empty((B, H, d * d + d), dtype=torch.float32, device=k.device)
    rc = la_block_reduce(k.data_ptr(), v.data_ptr(), _dtype_code(k), B, N, H, d, rope, partial.data_ptr(),
                         ws.data_ptr(), ws.numel() * ws.element_size(), _stream_ptr(stream))
    if rc != LA_OK:
        raise LAError(rc, "la_block_reduce")
    return partial


def block_apply(q, gathered, state: "State", commit=True, rope=None, eps=1e-6, ws=None, out=None, stream=None):
    """out for this rank's token slice from the gathered partials [R, B, H, 1056]
    (rank order) and the state; commits on every rank alike."""
    _check_qkv(q, q, q)
    B, N, H, d = q.shape
    if gathered.dtype != torch.float32 or not gathered.is_contiguous() or gathered.dim() != 4:
        raise ValueError("gathered must be a contiguous fp32 tensor [R, B, H, d*d + d]")
    if ws is None:
        ws = alloc_workspace(B, N, H, d, N, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    rc = la_block_apply(q.data_ptr(), out.data_ptr(), _dtype_code(q), B, N, H, d, gathered.data_ptr(),
                        gathered.shape[0], state.c, int(bool(commit)), rope, float(eps), ws.data_ptr(),
                        ws.numel() * ws.element_size(), _stream_ptr(stream))
    if rc != LA_OK:
        raise LAError(rc, "la_block_apply")
    return out


def la_backward_workspace_size(B, N, H, d, tokens_per_block) -> int:
    return int(lib().la_backward_workspace_size(B, N, H, d, tokens_per_block))


def la_full_backward(q, k, v, dout, dq, dk, dv, dt, B, N, H, d, tokens_per_block, rope, eps, ws, ws_bytes,
                     stream) -> int:
    return int(lib().la_full_backward(q, k, v, dout, dq, dk, dv, dt, B, N, H, d, tokens_per_block,
                                      ctypes.byref(rope) if rope is not None else None, eps, ws,
                                      ws_bytes, stream))


def la_device_status(stream) -> int:
    return int(lib().la_device_status(stream))


def la_status_string(status: int) -> str:
    return lib().la_status_string(int(status)).decode()


def la_set_stage_events(before_reduce, after_reduce, after_finish, after_apply) -> None:
    lib().la_set_stage_events(before_reduce, after_reduce, after_finish, after_apply)


def la_last_launch_count() -> int:
    return int(lib().la_last_launch_count())


def la_last_path() -> str:
    return lib().la_last_path().decode()


def tc_enabled() -> bool:
    """Whether this build routes bf16 (H % 4 == 0) through the tensor-core kernels."""
    return bool(lib().la_tc_enabled())


# ---------------------------------------------------------------- torch wrappers

def _stream_ptr(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return LA_F32
    if t.dtype == torch.bfloat16:
        return LA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check_qkv(q, k, v):
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("q, k, v must be contiguous CUDA tensors [B, N, H, d]")
    if not (q.shape == k.shape == v.shape and q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must agree in shape and dtype")


def make_rope(Hg, Wg, T=0, t_offset=0, dims=(8, 12, 12), base=10000.0) -> la_rope:
    return la_rope(int(T), int(Hg), int(Wg), int(t_offset), int(dims[0]), int(dims[1]), int(dims[2]),
                   float(base))


def workspace_bytes(B, N, H, d=32, tokens_per_block=0) -> int:
    n = la_workspace_size(B, N, H, d, tokens_per_block)
    if n == 0:
        raise LAError(LA_EINVAL, "la_workspace_size")
    return n


def alloc_workspace(B, N, H, d=32, tokens_per_block=0, device=None) -> torch.Tensor:
    """A uint8 CUDA tensor of la_workspace_size bytes (torch allocations are
    256-byte aligned)."""
    return torch.empty(workspace_bytes(B, N, H, d, tokens_per_block), dtype=torch.uint8,
                       device=device or "cuda")


class State:
    """The constant-memory state: S [B,H,d,d] and Z [B,H,d] fp32 CUDA tensors
    bound to a C ``la_state``."""

    def __init__(self, B, H, d=32, device=None, stream=None):
        dev = device or "cuda"
        self.S = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
        self.Z = torch.empty((B, H, d), dtype=torch.float32, device=dev)
        self.c = la_state()
        rc = la_state_init(self.c, self.S.data_ptr(), self.Z.data_ptr(), B, H, d, _stream_ptr(stream))
        if rc != LA_OK:
            raise LAError(rc, "la_state_init")

    @property
    def blocks_committed(self) -> int:
        return int(self.c.blocks_committed)

    @property
    def t_next(self) -> int:
        return int(self.c.t_next)

    def nbytes(self) -> int:
        return self.S.numel() * 4 + self.Z.numel() * 4

    def save(self, S_dst: torch.Tensor, Z_dst: torch.Tensor, stream=None) -> la_state_counters:
        """la_state_save into caller tensors (host, pinned host or device) of
        S's and Z's shapes and dtype; returns the counters."""
        if S_dst.shape != self.S.shape or Z_dst.shape != self.Z.shape or S_dst.dtype != torch.float32 \
                or Z_dst.dtype != torch.float32 or not S_dst.is_contiguous() or not Z_dst.is_contiguous():
            raise ValueError("checkpoint buffers must be contiguous fp32 tensors of S's and Z's shapes")
        c = la_state_counters()
        rc = la_state_save(self.c, S_dst.data_ptr(), Z_dst.data_ptr(), c, _stream_ptr(stream))
        if rc != LA_OK:
            raise LAError(rc, "la_state_save")
        return c

    def restore(self, S_src: torch.Tensor, Z_src: torch.Tensor, counters: la_state_counters, stream=None):
        """la_state_restore from caller tensors saved by ``save``."""
        if S_src.shape != self.S.shape or Z_src.shape != self.Z.shape or S_src.dtype != torch.float32 \
                or Z_src.dtype != torch.float32 or not S_src.is_contiguous() or not Z_src.is_contiguous():
            raise ValueError("checkpoint buffers must be contiguous fp32 tensors of S's and Z's shapes")
        rc = la_state_restore(self.c, S_src.data_ptr(), Z_src.data_ptr(), counters, _stream_ptr(stream))
        if rc != LA_OK:
            raise LAError(rc, "la_state_restore")


def block_forward(q, k, v, state: State, commit=True, rope: Optional[la_rope] = None, eps=1e-6,
                  ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None, stream=None):
    _check_qkv(q, k, v)
    B, N, H, d = q.shape
    if ws is None:
        ws = alloc_workspace(B, N, H, d, N, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    rc = la_block_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _dtype_code(q),
                          B, N, H, d, state.c, int(bool(commit)), rope, float(eps), ws.data_ptr(),
                          ws.numel() * ws.element_size(), _stream_ptr(stream))
    if rc != LA_OK:
        raise LAError(rc, "la_block_forward")
    return out


def full_forward(q, k, v, tokens_per_block=0, rope: Optional[la_rope] = None, eps=1e-6,
                 ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None, stream=None):
    _check_qkv(q, k, v)
    B, N, H, d = q.shape
    if ws is None:
        ws = alloc_workspace(B, N, H, d, tokens_per_block, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    rc = la_full_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _dtype_code(q),
                         B, N, H, d, int(tokens_per_block), rope, float(eps), ws.data_ptr(),
                         ws.numel() * ws.element_size(), _stream_ptr(stream))
    if rc != LA_OK:
        raise LAError(rc, "la_full_forward")
    return out


def _check_codes(q, k, v):
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4 or t.dtype != torch.uint8:
            raise ValueError("E4M3 q, k, v must be contiguous CUDA uint8 tensors [B, N, H, d]")
    if not q.shape == k.shape == v.shape:
        raise ValueError("q, k, v must agree in shape")


def full_forward_e4m3(q, k, v, scales, tokens_per_block=0, eps=1e-6, ws: Optional[torch.Tensor] = None,
                      out: Optional[torch.Tensor] = None, stream=None, rope=None):
    """la_full_forward on FP8 E4M3 codes (uint8 tensors) with per-tensor
    scales (sq, sk, sv), optional 3D RoPE; out is bf16."""
    _check_codes(q, k, v)
    B, N, H, d = q.shape
    if ws is None:
        ws = alloc_workspace(B, N, H, d, tokens_per_block, device=q.device)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    sq, sk, sv = (float(x) for x in scales)
    rc = la_full_forward_e4m3(q.data_ptr(), k.data_ptr(), v.data_ptr(), sq, sk, sv, out.data_ptr(), B, N, H, d,
                              int(tokens_per_block), rope, float(eps), ws.data_ptr(), ws.numel() * ws.element_size(),
                              _stream_ptr(stream))
    if rc != LA_OK:
        raise LAError(rc, "la_full_forward_e4m3")
    return out


def block_forward_e4m3(q, k, v, scales, state: "State", commit=True, eps=1e-6, ws: Optional[torch.Tensor] = None,
                       out: Optional[torch.Tensor] = None, stream=None, rope=None):
    _check_codes(q, k, v)
    B, N, H, d = q.shape
    if ws is None:
        ws = alloc_workspace(B, N, H, d, N, device=q.device)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    sq, sk, sv = (float(x) for x in scales)
    rc = la_block_forward_e4m3(q.data_ptr(), k.data_ptr(), v.data_ptr(), sq, sk, sv, out.data_ptr(), B, N, H, d,
                               state.c, int(bool(commit)), rope, float(eps), ws.data_ptr(),
                               ws.numel() * ws.element_size(), _stream_ptr(stream))
    if rc != LA_OK:
        raise LAError(rc, "la_block_forward_e4m3")
    return out


def la_full_forward_nvfp4(q, k, v, q_sf, k_sf, v_sf, sq, sk, sv, out, B, N, H, d, tokens_per_block, rope, eps, ws,
                          ws_bytes, stream) -> int:
    return int(lib().la_full_forward_nvfp4(q, k, v, q_sf, k_sf, v_sf, sq, sk, sv, out, B, N, H, d, tokens_per_block,
                                           ctypes.byref(rope) if rope is not None else None, eps, ws, ws_bytes,
                                           stream))


def la_block_forward_nvfp4(q, k, v, q_sf, k_sf, v_sf, sq, sk, sv, out, B, N_blk, H, d, st, commit, rope, eps, ws,
                           ws_bytes, stream) -> int:
    return int(lib().la_block_forward_nvfp4(q, k, v, q_sf, k_sf, v_sf, sq, sk, sv, out, B, N_blk, H, d,
                                            ctypes.byref(st), commit,
                                            ctypes.byref(rope) if rope is not None else None, eps, ws, ws_bytes,
                                            stream))


def _check_nvfp4(x):
    """x = (codes uint8 [B, N, H, d/2], block scales uint8 [B, N, H, d/16], scale): returns (B, N, H, d)."""
    codes, sf, _ = x
    for t in (codes, sf):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4 or t.dtype != torch.uint8:
            raise ValueError("NVFP4 codes and block scales must be contiguous CUDA uint8 tensors [B, N, H, *]")
    B, N, H, half = codes.shape
    if tuple(sf.shape) != (B, N, H, half // 8) or half % 8:
        raise ValueError("block scales must be [B, N, H, d/16] for codes [B, N, H, d/2]")
    return B, N, H, 2 * half


def full_forward_nvfp4(q, k, v, tokens_per_block=0, eps=1e-6, ws: Optional[torch.Tensor] = None,
                       out: Optional[torch.Tensor] = None, stream=None, rope=None):
    """la_full_forward on NVFP4 inputs: q, k, v each (codes, block scales,
    per-tensor scale) as synth.to_nvfp4 returns them, optional 3D RoPE; out
    is bf16."""
    shapes = {_check_nvfp4(x) for x in (q, k, v)}
    if len(shapes) != 1:
        raise ValueError("q, k, v must agree in shape")
    B, N, H, d = shapes.pop()
    if ws is None:
        ws = alloc_workspace(B, N, H, d, tokens_per_block, device=q[0].device)
    if out is None:
        out = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=q[0].device)
    rc = la_full_forward_nvfp4(q[0].data_ptr(), k[0].data_ptr(), v[0].data_ptr(), q[1].data_ptr(), k[1].data_ptr(),
                               v[1].data_ptr(), float(q[2]), float(k[2]), float(v[2]), out.data_ptr(), B, N, H, d,
                               int(tokens_per_block), rope, float(eps), ws.data_ptr(),
                               ws.numel() * ws.element_size(), _stream_ptr(stream))
    if rc != LA_OK:
        raise LAError(rc, "la_full_forward_nvfp4")
    return out


def block_forward_nvfp4(q, k, v, state: "State", commit=True, eps=1e-6, ws: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None, stream=None, rope=None):
    shapes = {_check_nvfp4(x) for x in (q, k, v)}
    if len(shapes) != 1:
        raise ValueError("q, k, v must agree in shape")
    B, N, H, d = shapes.pop()
    if ws is None:
        ws = alloc_workspace(B, N, H, d, N, device=q[0].device)
    if out is None:
        out = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=q[0].device)
    rc = la_block_forward_nvfp4(q[0].data_ptr(), k[0].data_ptr(), v[0].data_ptr(), q[1].data_ptr(), k[1].data_ptr(),
                                v[1].data_ptr(), float(q[2]), float(k[2]), float(v[2]), out.data_ptr(), B, N, H, d,
                                state.c, int(bool(commit)), rope, float(eps), ws.data_ptr(),
                                ws.numel() * ws.element_size(), _stream_ptr(stream))
    if rc != LA_OK:
        raise LAError(rc, "la_block_forward_nvfp4")
    return out


def alloc_backward_workspace(B, N, H, d=32, tokens_per_block=0, device=None) -> torch.Tensor:
    n = la_backward_workspace_size(B, N, H, d, tokens_per_block)
    if n == 0:
        raise LAError(LA_EINVAL, "la_backward_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def full_backward(q, k, v, dout, tokens_per_block=0, rope: Optional[la_rope] = None, eps=1e-6,
                  ws: Optional[torch.Tensor] = None, grads=None, stream=None):
    """(dq, dk, dv) of sum(full_forward(q, k, v, ...) * dout)."""
    _check_qkv(q, k, v)
    _check_qkv(q, dout, dout)
    B, N, H, d = q.shape
    if ws is None:
        ws = alloc_backward_workspace(B, N, H, d, tokens_per_block, device=q.device)
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    rc = la_full_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                          dv.data_ptr(), _dtype_code(q), B, N, H, d, int(tokens_per_block), rope, float(eps),
                          ws.data_ptr(), ws.numel() * ws.element_size(), _stream_ptr(stream))
    if rc != LA_OK:
        raise LAError(rc, "la_full_backward")
    return dq, dk, dv


def selftest_bounded_wait(stream=None) -> None:
    """Enqueue the bounded-wait self-test kernel (la_selftest_bounded_wait):
    the next device_status raises LAError(LA_ETIMEOUT)."""
    rc = lib().la_selftest_bounded_wait(_stream_ptr(stream))
    if rc != LA_OK:
        raise LAError(rc, "la_selftest_bounded_wait")


def device_status(stream=None) -> None:
    rc = la_device_status(_stream_ptr(stream))
    if rc != LA_OK:
        raise LAError(rc, "la_device_status")
