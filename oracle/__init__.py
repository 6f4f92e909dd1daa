"""fp64 CPU oracle for S^2-Attn and RoPE-PI -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference leg
import this package.  The CUDA library never does, and this package never imports
the CUDA library.  The arithmetic lives in s2attn_oracle.c (plain C, fp64); this
file only marshals numpy arrays into it.

Pinned by tests/test_oracle_pins.py against: textbook causal attention (torch
SDPA in fp64) for G=N without shift; brute force with an explicit N x N mask for
grouped and shifted heads; the shift example of the "LongLoRA paper notes" page
(section 3.3); central finite differences for the gradients; RoPE invariants; for the
decoding step, torch SDPA with an explicit mask, the last rows of full causal
attention, and closed forms.  The LoRA-adapted projection (lora.py, numpy fp64) is pinned
by tests/test_oracle_lora_pins.py.
"""
import ctypes
import numpy as np

from .build import build_oracle

F64, F32, BF16 = 0, 1, 2

_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_oracle())
        vp, ip, dp, llp = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int), ctypes.c_void_p, ctypes.c_void_p
        i = ctypes.c_int
        lib.oracle_s2attn_unit.argtypes = [i, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i,
                                           vp, i, vp, i, dp, dp, dp, dp, dp, llp, llp]
        lib.oracle_s2attn_unit.restype = i
        lib.oracle_s2attn_fwd_full.argtypes = [i, vp, vp, vp, i, i, i, i, i, i, dp, dp]
        lib.oracle_s2attn_fwd_full.restype = i
        lib.oracle_s2attn_bwd_full.argtypes = [i, vp, vp, vp, vp, i, i, i, i, i, i, dp, dp, dp]
        lib.oracle_s2attn_bwd_full.restype = i
        lib.oracle_decode.argtypes = [i, vp, vp, vp, i, i, i, i, i, dp, dp]
        lib.oracle_decode.restype = i
        lib.oracle_rope_pi_f64.argtypes = [vp, vp, i, i, i, i, ctypes.c_double, ctypes.c_double]
        lib.oracle_rope_pi_f64.restype = None
        lib.oracle_rope_pi_f32_bf16.argtypes = [vp, vp, i, i, i, i, ctypes.c_float, ctypes.c_float]
        lib.oracle_rope_pi_f32_bf16.restype = None
        lib.oracle_rope_pi_f32_bf16_at.argtypes = [vp, vp, i, i, i, i, i, ctypes.c_float, ctypes.c_float]
        lib.oracle_rope_pi_f32_bf16_at.restype = None
        _lib = lib
    return _lib


def _dtype_code(a):
    if a.dtype == np.float64:
        return F64
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:  # bf16 bit patterns
        return BF16
    raise TypeError(f"oracle inputs must be float64, float32 or uint16 (bf16 bits), got {a.dtype}")


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _prep(*arrs):
    out = [None if a is None else np.ascontiguousarray(a) for a in arrs]
    codes = {_dtype_code(a) for a in out if a is not None}
    if len(codes) != 1:
        raise TypeError("all oracle inputs must share one dtype")
    return out, codes.pop()


def s2attn_fwd(q, k, v, G, shift_heads):
    """Full forward.  q,k,v: [B,N,H,D].  Returns (o [B,N,H,D] f64, lse [B,H,N] f64)."""
    (q, k, v), code = _prep(q, k, v)
    B, N, H, D = q.shape
    o = np.empty((B, N, H, D), np.float64)
    lse = np.empty((B, H, N), np.float64)
    rc = _load().oracle_s2attn_fwd_full(code, _ptr(q), _ptr(k), _ptr(v), B, N, H, D, G, shift_heads,
                                        _ptr(o), _ptr(lse))
    if rc:
        raise ValueError("oracle: invalid shape")
    return o, lse


def s2attn_bwd(q, k, v, dout, G, shift_heads):
    """Full backward.  Returns (dq, dk, dv), each [B,N,H,D] f64."""
    (q, k, v, dout), code = _prep(q, k, v, dout)
    B, N, H, D = q.shape
    dq, dk, dv = (np.empty((B, N, H, D), np.float64) for _ in range(3))
    rc = _load().oracle_s2attn_bwd_full(code, _ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, N, H, D, G,
                                        shift_heads, _ptr(dq), _ptr(dk), _ptr(dv))
    if rc:
        raise ValueError("oracle: invalid shape")
    return dq, dk, dv


def s2attn_unit(q, k, v, G, shift_heads, b, h, j, qrows=(), krows=(), dout=None):
    """Selected rows of group j of head h (batch b), rows given as rolled-local indices.

    Returns a dict with o [nq,D], lse [nq], dq [nq,D] (if dout), dk/dv [nk,D] (if krows),
    and qtok/ktok: the original token index of each returned row (the un-roll map).
    """
    (q, k, v, dout), code = _prep(q, k, v, dout)
    B, N, H, D = q.shape
    qr = np.ascontiguousarray(np.asarray(qrows, dtype=np.int32))
    kr = np.ascontiguousarray(np.asarray(krows, dtype=np.int32))
    nq, nk = len(qr), len(kr)
    o = np.zeros((max(nq, 1), D)); lse = np.zeros(max(nq, 1))
    dq = np.zeros((max(nq, 1), D)); dk = np.zeros((max(nk, 1), D)); dv = np.zeros((max(nk, 1), D))
    qtok = np.zeros(max(nq, 1), np.int64); ktok = np.zeros(max(nk, 1), np.int64)
    rc = _load().oracle_s2attn_unit(code, _ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, N, H, D, G,
                                    shift_heads, b, h, j, _ptr(qr), nq, _ptr(kr), nk,
                                    _ptr(o), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                                    _ptr(qtok), _ptr(ktok))
    if rc:
        raise ValueError("oracle: invalid arguments")
    out = {"o": o[:nq], "lse": lse[:nq], "qtok": qtok[:nq]}
    if dout is not None:
        out["dq"] = dq[:nq]
    if nk:
        out.update(dk=dk[:nk], dv=dv[:nk], ktok=ktok[:nk])
    return out


def decode(q, k, v):
    """Full causal attention of the last M positions (a decoding step).

    q: [B,M,H,D], query m at position N-M+m; k, v: [B,N,H,D] (all N positions).
    Returns (o [B,M,H,D] f64, lse [B,H,M] f64)."""
    (q, k, v), code = _prep(q, k, v)
    B, M, H, D = q.shape
    N = k.shape[1]
    if k.shape != (B, N, H, D) or v.shape != k.shape:
        raise ValueError("oracle: k and v must be [B,N,H,D] with q's B, H, D")
    o = np.empty((B, M, H, D), np.float64)
    lse = np.empty((B, H, M), np.float64)
    if _load().oracle_decode(code, _ptr(q), _ptr(k), _ptr(v), B, M, N, H, D, _ptr(o), _ptr(lse)):
        raise ValueError("oracle: invalid decode sizes")
    return o, lse


def rope_pi_f64(x, pos_scale, base=10000.0):
    """fp64 RoPE with position interpolation.  x: [B,N,H,D] float64."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    B, N, H, D = x.shape
    _load().oracle_rope_pi_f64(_ptr(x), _ptr(y), B, N, H, D, float(pos_scale), float(base))
    return y


def rope_pi_bf16(x_bits, pos_scale, base=10000.0):
    """fp32 same-operation-order RoPE on bf16 bit patterns (uint16 [B,N,H,D]) -> uint16."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    y = np.empty_like(x)
    B, N, H, D = x.shape
    _load().oracle_rope_pi_f32_bf16(_ptr(x), _ptr(y), B, N, H, D, float(pos_scale), float(base))
    return y


def rope_pi_bf16_at(x_bits, pos0, pos_scale, base=10000.0):
    """As rope_pi_bf16, for a tensor whose row t is the token at position pos0 + t."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    y = np.empty_like(x)
    B, N, H, D = x.shape
    if pos0 < 0:
        raise ValueError("pos0 must be >= 0")
    _load().oracle_rope_pi_f32_bf16_at(_ptr(x), _ptr(y), B, N, H, D, int(pos0), float(pos_scale), float(base))
    return y


from .lora import lora_proj, lora_proj_bwd, rope_pi_bwd_f64  # noqa: E402  (numpy fp64; see lora.py)
