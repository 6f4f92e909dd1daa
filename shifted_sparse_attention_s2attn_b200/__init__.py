"""Python binding of the S^2-Attn C ABI (include/s2attn.h): argument marshalling only.

Every function has the name of the C entry point it calls and takes torch tensors
(device memory, contiguous [B,N,H,D]); shapes are read off the tensors, pointers and
the current CUDA stream are passed through, and a non-zero status raises
S2AttnError.  All arithmetic runs in the CUDA library libs2attn.so; if that library
is missing, every call raises -- there is no fallback.
"""
import ctypes
import os

__all__ = [
    "S2AttnError", "capi", "library_path",
    "s2attn_fwd", "s2attn_bwd", "s2attn_bwd_workspace_bytes", "s2attn_bwd_preprocess", "s2attn_bwd_main",
    "s2attn_bwd_dq_convert", "s2attn_bwd_noalloc", "s2attn_decode", "s2attn_decode_workspace_bytes", "s2attn_fwd_f32", "s2attn_bwd_f32", "rope_pi_apply", "rope_pi_apply_offset",
    "lora_proj_fwd", "lora_proj_workspace_bytes", "lora_proj_bwd", "lora_proj_bwd_workspace_bytes",
    "s2attn_halo_rows", "s2attn_halo_lse",
    "get_device_error", "clear_device_error", "s2attn_selftest_bounded_wait",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
# S2ATTN_LIBRARY selects another build of the library, e.g. libs2attn_debug.so (bounds-checked)
library_path = os.environ.get("S2ATTN_LIBRARY") or os.path.join(_HERE, "libs2attn.so")

STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported shape", -3: "workspace", -4: "CUDA error",
          -5: "device timeout"}


class S2AttnError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} failed: status {status} ({STATUS.get(status, 'unknown')})")
        self.status = status


_lib = None


def capi():
    """The loaded C library (ctypes), with argument types declared."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise RuntimeError(f"CUDA library not built: {library_path} is missing "
                           "(run: python -m shifted_sparse_attention_s2attn_b200._build)")
    lib = ctypes.CDLL(library_path)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "s2attn_version": ([], I),
        "s2attn_status_string": ([I], ctypes.c_char_p),
        "s2attn_fwd": ([P, P, P, P, P, I, I, I, I, I, I, P], I),
        "s2attn_bwd_workspace_bytes": ([I, I, I, I], Z),
        "s2attn_bwd": ([P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, P, Z, P], I),
        "s2attn_bwd_preprocess": ([P, P, P, P, I, I, I, I, P], I),
        "s2attn_bwd_main": ([P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, P], I),
        "s2attn_bwd_dq_convert": ([P, P, I, I, I, I, P], I),
        "s2attn_bwd_noalloc": ([P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, P], I),
        "s2attn_decode_workspace_bytes": ([I, I, I, I, I], Z),
        "s2attn_decode": ([P, P, P, P, P, I, I, I, I, I, P, Z, P], I),
        "s2attn_fwd_f32": ([P, P, P, P, P, I, I, I, I, I, I, P], I),
        "s2attn_bwd_f32": ([P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, P, Z, P], I),
        "rope_pi_apply": ([P, P, I, I, I, I, F, F, P], I),
        "rope_pi_apply_offset": ([P, P, I, I, I, I, I, F, F, P], I),
        "lora_proj_workspace_bytes": ([I, I, I, I, I], Z),
        "lora_proj_fwd": ([P, P, P, P, P, I, I, I, I, I, F, I, I, I, F, F, P, Z, P], I),
        "lora_proj_bwd_workspace_bytes": ([I, I, I, I, I], Z),
        "lora_proj_bwd": ([P, P, P, P, P, P, P, P, I, I, I, I, I, F, P, Z, P], I),
        "s2attn_halo_rows": ([ctypes.POINTER(P), ctypes.POINTER(P), I, I, I, I, I, I, I, I, P], I),
        "s2attn_halo_lse": ([ctypes.POINTER(P), ctypes.POINTER(P), I, I, I, I, I, I, I, P], I),
        "s2attn_get_device_error": ([ctypes.POINTER(I)], I),
        "s2attn_clear_device_error": ([], I),
        "s2attn_selftest_bounded_wait": ([ctypes.c_uint, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, rc):
    if rc != 0:
        raise S2AttnError(fn, rc)


def _bnhd(t, name):
    if t.dim() != 4 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [B,N,H,D] tensor")
    return tuple(t.shape)


# The C entry points see only pointers, so the binding checks every tensor a call reads or
# writes: first that each is contiguous with exactly the elements its role covers and the
# expected dtype (_extent), then that all of them live on a CUDA device (_on_cuda).

def _extent(t, name, numel, dtype):
    if t is None or not t.is_contiguous() or t.numel() != numel or t.dtype != dtype:
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of {numel} elements")


def _on_cuda(**tensors):
    for name, t in tensors.items():
        if t is not None and t.device.type != "cuda":
            raise ValueError(f"{name} must be on a CUDA device")


def _workspace(t):
    if t is None or not t.is_contiguous():
        raise ValueError("workspace must be a contiguous tensor")
    _on_cuda(workspace=t)


def _attn_args(dtype, shape, **tensors):
    """Checks the [B,N,H,D] tensors (q's element count) and the [B,H,N] lse/delta of an
    attention call (dq_acc: fp32 with q's element count), then their device."""
    B, N, H, D = shape
    for name, t in tensors.items():
        if name in ("lse", "delta"):
            _extent(t, name, B * H * N, _torch().float32)
        elif name == "dq_acc":
            _extent(t, name, B * N * H * D, _torch().float32)
        else:
            _extent(t, name, B * N * H * D, dtype)
    _on_cuda(**tensors)


def _torch():
    import torch
    return torch


def s2attn_fwd(q, k, v, o, lse, G, shift_heads, stream=None):
    """bf16 forward: o <- S^2-Attn(q, k, v), lse <- [B,H,N] fp32 log-sum-exp."""
    B, N, H, D = _bnhd(q, "q")
    _attn_args(_torch().bfloat16, (B, N, H, D), q=q, k=k, v=v, o=o, lse=lse)
    _check("s2attn_fwd", capi().s2attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, N, H, D, G,
                                           shift_heads, _stream(stream)))


def s2attn_bwd_workspace_bytes(B, N, H, D):
    return int(capi().s2attn_bwd_workspace_bytes(B, N, H, D))


def s2attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, G, shift_heads, workspace, stream=None):
    """bf16 backward into dq, dk, dv.  workspace: a uint8 device tensor of at least
    s2attn_bwd_workspace_bytes(B,N,H,D) bytes, 256-byte aligned."""
    B, N, H, D = _bnhd(q, "q")
    _attn_args(_torch().bfloat16, (B, N, H, D), q=q, k=k, v=v, o=o, dout=dout, lse=lse, dq=dq, dk=dk, dv=dv)
    _workspace(workspace)
    _check("s2attn_bwd", capi().s2attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                                           _ptr(dk), _ptr(dv), B, N, H, D, G, shift_heads, _ptr(workspace),
                                           workspace.numel() * workspace.element_size(), _stream(stream)))


def s2attn_bwd_preprocess(o, dout, delta, dq_acc, stream=None):
    B, N, H, D = _bnhd(o, "o")
    _attn_args(_torch().bfloat16, (B, N, H, D), o=o, dout=dout, delta=delta, dq_acc=dq_acc)
    _check("s2attn_bwd_preprocess", capi().s2attn_bwd_preprocess(_ptr(o), _ptr(dout), _ptr(delta), _ptr(dq_acc),
                                                                 B, N, H, D, _stream(stream)))


def s2attn_bwd_main(q, k, v, dout, lse, delta, dq_acc, dk, dv, G, shift_heads, stream=None):
    B, N, H, D = _bnhd(q, "q")
    _attn_args(_torch().bfloat16, (B, N, H, D), q=q, k=k, v=v, dout=dout, lse=lse, delta=delta, dq_acc=dq_acc,
               dk=dk, dv=dv)
    _check("s2attn_bwd_main", capi().s2attn_bwd_main(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(lse), _ptr(delta),
                                                     _ptr(dq_acc), _ptr(dk), _ptr(dv), B, N, H, D, G, shift_heads,
                                                     _stream(stream)))


def s2attn_bwd_dq_convert(dq_acc, dq, stream=None):
    B, N, H, D = _bnhd(dq, "dq")
    _attn_args(_torch().bfloat16, (B, N, H, D), dq=dq, dq_acc=dq_acc)
    _check("s2attn_bwd_dq_convert", capi().s2attn_bwd_dq_convert(_ptr(dq_acc), _ptr(dq), B, N, H, D,
                                                                 _stream(stream)))


def s2attn_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, G, shift_heads, stream=None):
    """bf16 backward without a caller workspace: for callers that cannot allocate device
    memory.  Uses the library's fixed device scratch (S2ATTN_NOALLOC_SCRATCH_BYTES per
    device, shared by all calls; overlapping calls race)."""
    B, N, H, D = _bnhd(q, "q")
    _attn_args(_torch().bfloat16, (B, N, H, D), q=q, k=k, v=v, o=o, dout=dout, lse=lse, dq=dq, dk=dk, dv=dv)
    _check("s2attn_bwd_noalloc", capi().s2attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout),
                                                           _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), B, N, H, D, G,
                                                           shift_heads, _stream(stream)))


def _ptr_array(ts):
    return (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])


def s2attn_halo_rows(xs, bufs, to_buf, G, shift_heads, stream=None):
    """Rows [0, G/2) of the shifted heads of each bf16 [B,N,H,D] tensor in xs to (to_buf=True)
    or from (False) the matching contiguous [B, G/2, shift_heads, D] buffer in bufs; one launch."""
    if not xs or len(xs) != len(bufs):
        raise ValueError("xs and bufs must be non-empty lists of equal length")
    B, N, H, D = _bnhd(xs[0], "x")
    bf16 = _torch().bfloat16
    for i, (x, b) in enumerate(zip(xs, bufs)):
        _extent(x, f"x[{i}]", B * N * H * D, bf16)
        _extent(b, f"buf[{i}]", B * (G // 2) * shift_heads * D, bf16)
    for x, b in zip(xs, bufs):
        _on_cuda(x=x, buf=b)
    _check("s2attn_halo_rows", capi().s2attn_halo_rows(_ptr_array(xs), _ptr_array(bufs), len(xs), int(bool(to_buf)),
                                                       B, N, H, D, G, shift_heads, _stream(stream)))


def s2attn_halo_lse(lses, bufs, to_buf, G, shift_heads, stream=None):
    """The same rows of fp32 [B,H,N] tensors (softmax statistics) to or from [B, shift_heads, G/2]
    buffers; one launch."""
    if not lses or len(lses) != len(bufs):
        raise ValueError("lses and bufs must be non-empty lists of equal length")
    if lses[0].dim() != 3:
        raise ValueError("lse must be a [B,H,N] tensor")
    B, H, N = tuple(lses[0].shape)
    f32 = _torch().float32
    for i, (x, b) in enumerate(zip(lses, bufs)):
        _extent(x, f"lse[{i}]", B * H * N, f32)
        _extent(b, f"buf[{i}]", B * shift_heads * (G // 2), f32)
    for x, b in zip(lses, bufs):
        _on_cuda(lse=x, buf=b)
    _check("s2attn_halo_lse", capi().s2attn_halo_lse(_ptr_array(lses), _ptr_array(bufs), len(lses),
                                                     int(bool(to_buf)), B, N, H, G, shift_heads, _stream(stream)))


def s2attn_decode_workspace_bytes(B, M, N, H, D):
    return int(capi().s2attn_decode_workspace_bytes(B, M, N, H, D))


def s2attn_decode(q, k, v, o, lse, workspace, stream=None):
    """Decoding step of full causal attention: q [B,M,H,D] (query m at position N-M+m)
    against k, v [B,N,H,D]; o [B,M,H,D] bf16 and lse [B,H,M] fp32 are written.
    workspace: a uint8 device tensor of at least s2attn_decode_workspace_bytes bytes."""
    B, M, H, D = _bnhd(q, "q")
    Bk, N, Hk, Dk = _bnhd(k, "k")
    if (Bk, Hk, Dk) != (B, H, D):
        raise ValueError("k must be [B,N,H,D] with q's B, H and D")
    bf16 = _torch().bfloat16
    _extent(q, "q", B * M * H * D, bf16)
    _extent(k, "k", B * N * H * D, bf16)
    _extent(v, "v", B * N * H * D, bf16)
    _extent(o, "o", B * M * H * D, bf16)
    _extent(lse, "lse", B * H * M, _torch().float32)
    _on_cuda(q=q, k=k, v=v, o=o, lse=lse)
    _workspace(workspace)
    _check("s2attn_decode", capi().s2attn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, M, N, H, D,
                                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                                 _stream(stream)))


def s2attn_fwd_f32(q, k, v, o, lse, G, shift_heads, stream=None):
    B, N, H, D = _bnhd(q, "q")
    _attn_args(_torch().float32, (B, N, H, D), q=q, k=k, v=v, o=o, lse=lse)
    _check("s2attn_fwd_f32", capi().s2attn_fwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, N, H, D, G,
                                                   shift_heads, _stream(stream)))


def s2attn_bwd_f32(q, k, v, o, dout, lse, dq, dk, dv, G, shift_heads, workspace, stream=None):
    B, N, H, D = _bnhd(q, "q")
    _attn_args(_torch().float32, (B, N, H, D), q=q, k=k, v=v, o=o, dout=dout, lse=lse, dq=dq, dk=dk, dv=dv)
    _workspace(workspace)
    _check("s2attn_bwd_f32", capi().s2attn_bwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                                                   _ptr(dq), _ptr(dk), _ptr(dv), B, N, H, D, G, shift_heads,
                                                   _ptr(workspace), workspace.numel() * workspace.element_size(),
                                                   _stream(stream)))


def rope_pi_apply(q, k, pos_scale, base=10000.0, stream=None):
    """In-place RoPE with position interpolation on bf16 q and/or k ([B,N,H,D])."""
    ref = q if q is not None else k
    B, N, H, D = _bnhd(ref, "q/k")
    for name, t in (("q", q), ("k", k)):
        if t is not None:
            _extent(t, name, B * N * H * D, _torch().bfloat16)
    _on_cuda(q=q, k=k)
    _check("rope_pi_apply", capi().rope_pi_apply(_ptr(q), _ptr(k), B, N, H, D, float(pos_scale), float(base),
                                                 _stream(stream)))


def rope_pi_apply_offset(q, k, pos0, pos_scale, base=10000.0, stream=None):
    """In-place RoPE-PI on bf16 q and/or k whose row t is the token at position pos0 + t."""
    ref = q if q is not None else k
    B, N, H, D = _bnhd(ref, "q/k")
    for name, t in (("q", q), ("k", k)):
        if t is not None:
            _extent(t, name, B * N * H * D, _torch().bfloat16)
    _on_cuda(q=q, k=k)
    _check("rope_pi_apply_offset", capi().rope_pi_apply_offset(_ptr(q), _ptr(k), B, N, H, D, int(pos0),
                                                               float(pos_scale), float(base), _stream(stream)))


def lora_proj_workspace_bytes(T, K, n_out, parts, r):
    return int(capi().lora_proj_workspace_bytes(T, K, n_out, parts, r))


def lora_proj_fwd(x, w, lora_a, lora_b, y, parts, scaling, rope_parts=0, head_dim=128, seq_len=None,
                  pos_scale=1.0, base=10000.0, workspace=None, stream=None):
    """LoRA-adapted projections: y[p] = x W_p^T + scaling (x A_p^T) B_p^T for p < parts, RoPE-PI
    on the first rope_parts parts.  x: [..., K] (T rows), w: [parts*n_out, K], lora_a:
    [parts*r, K] and lora_b: [parts*n_out, r] (both None for r = 0), y: [parts, T, n_out]
    (or any contiguous tensor of that many elements); all bf16 on the device.  workspace:
    uint8 device tensor of lora_proj_workspace_bytes(T, K, n_out, parts, r) bytes (r > 0)."""
    import torch
    if (lora_a is None) != (lora_b is None):
        raise ValueError("lora_a and lora_b are given together (or both None for no adapter)")
    for t, name in ((x, "x"), (w, "w"), (y, "y"), (lora_a, "lora_a"), (lora_b, "lora_b")):
        if t is None:
            continue
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be bf16")
    # The C entry point sees only pointers: every extent it will read or write is checked here.
    K = x.shape[-1]
    T = x.numel() // K
    if parts < 1 or w.dim() != 2 or w.shape[1] != K or w.shape[0] % parts:
        raise ValueError("w must be [parts*n_out, K] with x's K")
    n_out = w.shape[0] // parts
    r = 0
    if lora_a is not None:
        if lora_a.dim() != 2 or lora_a.shape[1] != K or lora_a.shape[0] % parts:
            raise ValueError("lora_a must be [parts*r, K]")
        r = lora_a.shape[0] // parts
        if tuple(lora_b.shape) != (parts * n_out, r):
            raise ValueError("lora_b must be [parts*n_out, r]")
    if y.numel() != parts * T * n_out:
        raise ValueError("y must hold parts * T * n_out elements")
    _on_cuda(x=x, w=w, y=y, lora_a=lora_a, lora_b=lora_b)
    if r > 0:
        _workspace(workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("lora_proj_fwd", capi().lora_proj_fwd(
        _ptr(x), _ptr(w), _ptr(lora_a), _ptr(lora_b), _ptr(y), T, K, n_out, parts, r, float(scaling),
        int(rope_parts), int(head_dim), int(seq_len if seq_len is not None else T), float(pos_scale), float(base),
        _ptr(workspace), ws_bytes, _stream(stream)))


def lora_proj_bwd_workspace_bytes(T, K, n_out, parts, r):
    return int(capi().lora_proj_bwd_workspace_bytes(T, K, n_out, parts, r))


def lora_proj_bwd(x, w, lora_a, lora_b, dy, dx, d_lora_a, d_lora_b, parts, scaling, workspace, stream=None):
    """Backward of lora_proj_fwd (W frozen): dx [T, K], d_lora_a [parts*r, K], d_lora_b
    [parts*n_out, r] from dy [parts, T, n_out] (the gradient before RoPE; rope_pi_apply with
    -pos_scale takes dq, dk back through it)."""
    torch = _torch()
    K = x.shape[-1]
    T = x.numel() // K
    if parts < 1 or w.dim() != 2 or w.shape[1] != K or w.shape[0] % parts:
        raise ValueError("w must be [parts*n_out, K] with x's K")
    n_out = w.shape[0] // parts
    r = 0 if lora_a is None else lora_a.shape[0] // parts
    bf = torch.bfloat16
    _extent(x, "x", T * K, bf)
    _extent(w, "w", parts * n_out * K, bf)
    _extent(dy, "dy", parts * T * n_out, bf)
    _extent(dx, "dx", T * K, bf)
    if r:
        _extent(lora_a, "lora_a", parts * r * K, bf)
        _extent(lora_b, "lora_b", parts * n_out * r, bf)
        _extent(d_lora_a, "d_lora_a", parts * r * K, bf)
        _extent(d_lora_b, "d_lora_b", parts * n_out * r, bf)
    _on_cuda(x=x, w=w, dy=dy, dx=dx, lora_a=lora_a, lora_b=lora_b, d_lora_a=d_lora_a, d_lora_b=d_lora_b)
    _workspace(workspace)
    _check("lora_proj_bwd", capi().lora_proj_bwd(
        _ptr(x), _ptr(w), _ptr(lora_a), _ptr(lora_b), _ptr(dy), _ptr(dx), _ptr(d_lora_a), _ptr(d_lora_b),
        T, K, n_out, parts, r, float(scaling), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def get_device_error():
    """(status, detail) of the current device's error word; synchronize first."""
    d = ctypes.c_int(0)
    rc = capi().s2attn_get_device_error(ctypes.byref(d))
    return rc, d.value


def clear_device_error():
    _check("s2attn_clear_device_error", capi().s2attn_clear_device_error())


def s2attn_selftest_bounded_wait(timeout_us, stream=None):
    """Runs a kernel whose bounded wait must time out (see include/s2attn.h)."""
    _check("s2attn_selftest_bounded_wait", capi().s2attn_selftest_bounded_wait(int(timeout_us), _stream(stream)))
