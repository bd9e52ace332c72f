"""fp64 CPU oracle for block-causal linear attention (ctypes binding of oracle.c).

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The CUDA library never
imports this package and this package never imports the CUDA library; the two
share nothing but the seeded input generator's tensors.

Every function takes CPU torch tensors laid out ``[B, N, H, d]`` (fp64, fp32 or
bf16 -- bf16 is passed as its bit pattern and widened exactly in C) and returns
fp64 numpy arrays.  What each function computes, with the passages it follows,
is written next to it in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

ORC_F64, ORC_F32, ORC_BF16 = 0, 1, 2


class Rope(ctypes.Structure):
    """3D RoPE description: grid rows Hg, columns Wg, first frame t_offset,
    section dims (dt, dh, dw) for the frame/row/column axes, frequency base."""

    _fields_ = [
        ("enabled", ctypes.c_int),
        ("Hg", ctypes.c_int),
        ("Wg", ctypes.c_int),
        ("t_offset", ctypes.c_int),
        ("dt", ctypes.c_int),
        ("dh", ctypes.c_int),
        ("dw", ctypes.c_int),
        ("base", ctypes.c_double),
    ]


def make_rope(Hg, Wg, t_offset=0, dims=(8, 12, 12), base=10000.0):
    return Rope(1, int(Hg), int(Wg), int(t_offset), int(dims[0]), int(dims[1]), int(dims[2]), float(base))


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (-O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        vp, ip, lp, dp = ctypes.c_void_p, ctypes.c_int, ctypes.c_long, ctypes.c_double
        rp = ctypes.POINTER(Rope)
        L.orc_brute.argtypes = [vp, vp, vp, ip, vp, ip, lp, ip, ip, lp, rp, lp, dp]
        L.orc_block_kv.argtypes = [vp, vp, ip, ip, lp, ip, ip, lp, lp, rp, lp, vp, vp]
        L.orc_apply.argtypes = [vp, ip, ip, lp, ip, ip, vp, vp, vp, lp, rp, lp, dp, vp]
        L.orc_block_forward.argtypes = [vp, vp, vp, ip, vp, ip, lp, ip, ip, vp, vp, ip, rp, lp, dp]
        L.orc_full_forward.argtypes = [vp, vp, vp, ip, vp, ip, lp, ip, ip, lp, rp, dp]
        L.orc_full_backward.argtypes = [vp, vp, vp, vp, ip, vp, vp, vp, ip, lp, ip, ip, lp, rp, dp]
        L.orc_dwconv3d.argtypes = [vp, ip, vp, ip, ip, ip, ip, ip, ip, ip, ip, vp, vp]
        L.orc_set_threads.argtypes = [ip]
        L.orc_get_threads.restype = ip
        for f in ("orc_brute", "orc_block_kv", "orc_apply", "orc_block_forward", "orc_full_forward",
                  "orc_full_backward", "orc_dwconv3d"):
            getattr(L, f).restype = ip
        _lib = L
    return _lib


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def get_threads() -> int:
    return int(lib().orc_get_threads())


def _prep(x: torch.Tensor):
    """Contiguous CPU tensor and its dtype code; bf16 travels as raw bits."""
    x = x.detach()
    if x.device.type != "cpu":
        raise ValueError("the oracle takes CPU tensors only")
    x = x.contiguous()
    if x.dtype == torch.float64:
        return x, ORC_F64
    if x.dtype == torch.float32:
        return x, ORC_F32
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16), ORC_BF16
    raise TypeError(f"unsupported dtype {x.dtype}")


def _shape(q):
    if q.dim() != 4:
        raise ValueError("expected [B, N, H, d]")
    return tuple(int(s) for s in q.shape)


def _rope_ptr(rope):
    return ctypes.byref(rope) if rope is not None else None


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"oracle {name} rejected its arguments")


def brute(q, k, v, tokens_per_block=0, rope=None, eps=1e-6, tok_base=0):
    """Definition form, O(N^2 d): out_i over all j in blocks <= blk(i)."""
    B, N, H, d = _shape(q)
    (qc, dt), (kc, dt2), (vc, dt3) = _prep(q), _prep(k), _prep(v)
    assert dt == dt2 == dt3
    out = np.zeros((B, N, H, d), dtype=np.float64)
    rc = lib().orc_brute(qc.data_ptr(), kc.data_ptr(), vc.data_ptr(), dt, out.ctypes.data,
                         B, N, H, d, int(tokens_per_block), _rope_ptr(rope), int(tok_base), float(eps))
    _check(rc, "brute")
    return out


def block_kv(k, v, t0=0, t1=None, rope=None, tok_base=0):
    """KV_n [B,H,d,d] and z_n [B,H,d] over tokens [t0, t1) of k, v."""
    B, N, H, d = _shape(k)
    t1 = N if t1 is None else t1
    (kc, dt), (vc, dt2) = _prep(k), _prep(v)
    assert dt == dt2
    KV = np.zeros((B, H, d, d), dtype=np.float64)
    z = np.zeros((B, H, d), dtype=np.float64)
    rc = lib().orc_block_kv(kc.data_ptr(), vc.data_ptr(), dt, B, N, H, d, int(t0), int(t1),
                            _rope_ptr(rope), int(tok_base), KV.ctypes.data, z.ctypes.data)
    _check(rc, "block_kv")
    return KV, z


def apply(q, S_eff, Z_eff, toks=None, rope=None, eps=1e-6, tok_base=0):
    """out [B, len(toks), H, d] = psi(q) S_eff / (phi(q).Z_eff + eps) for the listed tokens."""
    B, N, H, d = _shape(q)
    qc, dt = _prep(q)
    toks = np.arange(N, dtype=np.int64) if toks is None else np.ascontiguousarray(toks, dtype=np.int64)
    S = np.ascontiguousarray(S_eff, dtype=np.float64)
    Z = np.ascontiguousarray(Z_eff, dtype=np.float64)
    assert S.shape == (B, H, d, d) and Z.shape == (B, H, d)
    out = np.zeros((B, len(toks), H, d), dtype=np.float64)
    rc = lib().orc_apply(qc.data_ptr(), dt, B, N, H, d, S.ctypes.data, Z.ctypes.data,
                         toks.ctypes.data, len(toks), _rope_ptr(rope), int(tok_base), float(eps),
                         out.ctypes.data)
    _check(rc, "apply")
    return out


class State:
    """The oracle's own fp64 constant-size state: S [B,H,d,d], Z [B,H,d]."""

    def __init__(self, B, H, d):
        self.S = np.zeros((B, H, d, d), dtype=np.float64)
        self.Z = np.zeros((B, H, d), dtype=np.float64)

    def nbytes(self):
        return self.S.nbytes + self.Z.nbytes


def block_forward(q, k, v, state: State, commit=True, rope=None, eps=1e-6, tok_base=0):
    """One streaming block: KV_n, z_n, out with S+KV_n, Z+z_n, commit if asked."""
    B, N, H, d = _shape(q)
    (qc, dt), (kc, _), (vc, _) = _prep(q), _prep(k), _prep(v)
    out = np.zeros((B, N, H, d), dtype=np.float64)
    rc = lib().orc_block_forward(qc.data_ptr(), kc.data_ptr(), vc.data_ptr(), dt, out.ctypes.data,
                                 B, N, H, d, state.S.ctypes.data, state.Z.ctypes.data, int(bool(commit)),
                                 _rope_ptr(rope), int(tok_base), float(eps))
    _check(rc, "block_forward")
    return out


def full_forward(q, k, v, tokens_per_block=0, rope=None, eps=1e-6):
    """Whole sequence from a zero state, block after block (recurrence form)."""
    B, N, H, d = _shape(q)
    (qc, dt), (kc, _), (vc, _) = _prep(q), _prep(k), _prep(v)
    out = np.zeros((B, N, H, d), dtype=np.float64)
    rc = lib().orc_full_forward(qc.data_ptr(), kc.data_ptr(), vc.data_ptr(), dt, out.ctypes.data,
                                B, N, H, d, int(tokens_per_block), _rope_ptr(rope), float(eps))
    _check(rc, "full_forward")
    return out


def full_backward(q, k, v, dout, tokens_per_block=0, rope=None, eps=1e-6):
    """Gradients (dq, dk, dv) of sum(full_forward(q, k, v) * dout), fp64 numpy
    [B, N, H, d] each: the chain rule through the block recurrence (zero
    initial state), ReLU derivative 1[x > 0]."""
    B, N, H, d = _shape(q)
    (qc, dt), (kc, _), (vc, _), (oc, dto) = _prep(q), _prep(k), _prep(v), _prep(dout)
    if dto != dt:
        raise TypeError("dout must have the dtype of q, k, v")
    dq, dk, dv = (np.zeros((B, N, H, d), dtype=np.float64) for _ in range(3))
    rc = lib().orc_full_backward(qc.data_ptr(), kc.data_ptr(), vc.data_ptr(), oc.data_ptr(), dt,
                                 dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, B, N, H, d,
                                 int(tokens_per_block), _rope_ptr(rope), float(eps))
    _check(rc, "full_backward")
    return dq, dk, dv


def e4m3_decode(codes: torch.Tensor, scale: float = 1.0) -> torch.Tensor:
    """fp64 values of FP8 E4M3 codes (uint8) times a per-tensor scale.

    The format (OCP 8-bit floating point, E4M3 variant): 1 sign bit, 4
    exponent bits with bias 7, 3 mantissa bits; exponent field 0 encodes
    subnormals m / 8 * 2^-6; S.1111.111 is NaN and there is no infinity, so
    the largest finite magnitude is 1.75 * 2^8 = 448.  Every value times an
    fp32 scale is exact in fp64 (4 + 24 significant bits)."""
    c = codes.to(torch.int64)
    sign = torch.where(c >= 128, -1.0, 1.0).to(torch.float64)
    e = (c >> 3) & 15
    m = (c & 7).to(torch.float64)
    normal = (1.0 + m / 8.0) * torch.pow(torch.tensor(2.0, dtype=torch.float64), (e - 7).to(torch.float64))
    sub = (m / 8.0) * 2.0 ** -6
    mag = torch.where(e == 0, sub, normal)
    mag = torch.where((e == 15) & ((c & 7) == 7), torch.tensor(float("nan"), dtype=torch.float64), mag)
    return sign * mag * float(scale)


def e2m1_decode(codes: torch.Tensor) -> torch.Tensor:
    """fp64 values of FP4 E2M1 codes (integers 0..15, one code per element).

    The format (OCP Microscaling Formats, FP4 E2M1 element type): bit 3 the
    sign, bits 2..1 the exponent with bias 1, bit 0 the mantissa; exponent
    field 0 encodes the subnormals m * 0.5 (0 and 0.5); no infinity, no NaN,
    so the magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6."""
    c = codes.to(torch.int64)
    sign = torch.where((c & 8) != 0, -1.0, 1.0).to(torch.float64)
    e = (c >> 1) & 3
    m = (c & 1).to(torch.float64)
    normal = (1.0 + m / 2.0) * torch.pow(torch.tensor(2.0, dtype=torch.float64), (e - 1).to(torch.float64))
    mag = torch.where(e == 0, m * 0.5, normal)
    return sign * mag


def nvfp4_decode(codes: torch.Tensor, block_scales: torch.Tensor, scale: float = 1.0) -> torch.Tensor:
    """fp64 values of an NVFP4 tensor: ``codes`` uint8 [..., d/2] holding two
    E2M1 codes per byte (element 2i in the low nibble, 2i+1 in the high
    nibble), ``block_scales`` uint8 [..., d/16] holding one E4M3 scale per 16
    consecutive elements of the last axis, and one fp32 per-tensor scale:
        x[..., i] = e2m1(code i) * e4m3(block_scales[..., i // 16]) * scale.
    Every such product is exact in fp64 (2 + 4 + 24 significant bits)."""
    c = codes.to(torch.int64)
    lo, hi = c & 15, (c >> 4) & 15
    elems = torch.stack((lo, hi), dim=-1).reshape(*c.shape[:-1], 2 * c.shape[-1])
    d = elems.shape[-1]
    if block_scales.shape[-1] * 16 != d or block_scales.shape[:-1] != codes.shape[:-1]:
        raise ValueError("block_scales must be [..., d/16] for codes [..., d/2]")
    sf = e4m3_decode(block_scales).repeat_interleave(16, dim=-1)
    return e2m1_decode(elems) * sf * float(scale)


def dwconv3d(x, weight, bias=None):
    """Depthwise 3D convolution (Mix-FFN): x [B, T, Hg, Wg, C] (fp64/fp32/bf16
    CPU tensor), weight [C, kt, kh, kw], bias [C] or None; zero padding of
    (k-1)/2, fp64 numpy result [B, T, Hg, Wg, C]."""
    if x.dim() != 5:
        raise ValueError("expected [B, T, Hg, Wg, C]")
    B, T, Hg, Wg, C = (int(s_) for s_ in x.shape)
    xc, dt = _prep(x)
    w = np.ascontiguousarray(np.asarray(weight, dtype=np.float64))
    if w.ndim != 4 or w.shape[0] != C:
        raise ValueError("weight must be [C, kt, kh, kw]")
    bb = None if bias is None else np.ascontiguousarray(np.asarray(bias, dtype=np.float64))
    y = np.zeros((B, T, Hg, Wg, C), dtype=np.float64)
    rc = lib().orc_dwconv3d(xc.data_ptr(), dt, y.ctypes.data, B, T, Hg, Wg, C, *(int(k) for k in w.shape[1:]),
                            w.ctypes.data, None if bb is None else bb.ctypes.data)
    _check(rc, "dwconv3d")
    return y
