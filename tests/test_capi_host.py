"""CPU-only checks of the C ABI: the library builds for sm_100a, loads, exports every
function include/s2attn.h declares, and rejects bad arguments on the host (these
calls return before any CUDA work, so no GPU is needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from shifted_sparse_attention_s2attn_b200 import _build, capi
    _build.build()
    return capi()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "s2attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?(?:int|size_t|char\s*\*|const char\s*\*|void)\s*\*?\s*"
                                 r"([a-z_0-9]+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("s2attn_fwd", "s2attn_bwd", "rope_pi_apply", "s2attn_bwd_workspace_bytes",
                     "s2attn_fwd_f32", "s2attn_bwd_f32", "s2attn_get_device_error", "s2attn_decode",
                     "s2attn_decode_workspace_bytes", "lora_proj_fwd", "lora_proj_workspace_bytes"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_version_and_status_strings(lib):
    assert lib.s2attn_version() == 100
    assert lib.s2attn_status_string(0) == b"ok"
    assert lib.s2attn_status_string(-2).startswith(b"unsupported")


def test_workspace_size(lib):
    B, N, H, D = 1, 32768, 32, 128
    acc = B * N * H * D * 4
    delta = B * H * N * 4
    assert lib.s2attn_bwd_workspace_bytes(B, N, H, D) == acc + delta
    assert lib.s2attn_bwd_workspace_bytes(0, N, H, D) == 0


NULL = None


@pytest.mark.parametrize("args,status", [
    ((1, 1000, 2, 128, 300, 0), -1),    # G does not divide N
    ((1, 1024, 2, 128, 512, 3), -1),    # more shifted heads than heads
    ((1, 1024, 2, 128, 0, 0), -1),      # G = 0
    ((0, 1024, 2, 128, 512, 0), -1),    # empty batch
    ((1, 0, 2, 128, 512, 0), -1),       # empty sequence
    ((1, 1024, 2, 64, 512, 0), -2),     # D = 64: fp32 path only
    ((1, 768, 2, 128, 384, 1), -2),     # G/2 not a multiple of the 128-row tile
    ((1, 960, 2, 128, 320, 0), -2),     # G not a multiple of 128
    ((1, 1024, 2, 128, 512, 1), -1),    # valid shape, null pointers
])
def test_fwd_bwd_validation(lib, args, status):
    assert lib.s2attn_fwd(NULL, NULL, NULL, NULL, NULL, *args, NULL) == status
    assert lib.s2attn_bwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, *args, NULL, 0, NULL) == status


def test_misaligned_pointer_rejected(lib):
    p = ctypes.c_void_p(0x1000 + 8)
    assert lib.s2attn_fwd(p, p, p, p, p, 1, 1024, 2, 128, 512, 0, NULL) == -1


def test_f32_validation(lib):
    assert lib.s2attn_fwd_f32(NULL, NULL, NULL, NULL, NULL, 1, 90, 3, 40, 18, 1, NULL) == -1   # null pointers
    assert lib.s2attn_fwd_f32(NULL, NULL, NULL, NULL, NULL, 1, 90, 3, 40, 9, 1, NULL) == -1    # odd G shifted
    assert lib.s2attn_fwd_f32(NULL, NULL, NULL, NULL, NULL, 1, 90, 3, 256, 18, 1, NULL) == -2  # D > 128


def test_rope_offset_validation(lib):
    p = ctypes.c_void_p(0x1000)
    assert lib.rope_pi_apply_offset(p, NULL, 1, 16, 2, 128, -1, 0.5, 10000.0, NULL) == -1        # negative offset
    assert lib.rope_pi_apply_offset(p, NULL, 1, 16, 2, 128, 1 << 24, 0.5, 10000.0, NULL) == -1   # past 2^24
    assert lib.rope_pi_apply_offset(NULL, NULL, 1, 16, 2, 128, 5, 0.5, 10000.0, NULL) == -1      # neither q nor k


def test_rope_validation(lib):
    assert lib.rope_pi_apply(NULL, NULL, 1, 16, 2, 128, 0.5, 10000.0, NULL) == -1   # neither q nor k
    p = ctypes.c_void_p(0x1000)
    assert lib.rope_pi_apply(p, NULL, 1, 16, 2, 100, 0.5, 10000.0, NULL) == -1      # D % 16 != 0
    assert lib.rope_pi_apply(p, NULL, 1, 16, 2, 128, 0.5, -1.0, NULL) == -1         # bad base


@pytest.mark.parametrize("args,status", [
    ((1, 0, 100, 2, 128), -1),     # no query
    ((1, 5, 4, 2, 128), -1),       # more queries than positions
    ((0, 1, 100, 2, 128), -1),     # empty batch
    ((1, 129, 200, 2, 128), -2),   # more than 128 queries
    ((1, 1, 100, 2, 64), -2),      # D = 64
    ((1, 1, 100, 2, 128), -1),     # valid shape, null pointers
])
def test_decode_validation(lib, args, status):
    assert lib.s2attn_decode(NULL, NULL, NULL, NULL, NULL, *args, NULL, 0, NULL) == status


def test_decode_workspace_size(lib):
    # fp32 partials per (b, h, split, query): D output values + (max, sum); at most one split
    # per 64-key tile and at most 64 splits
    B, M, N, H, D = 1, 4, 32768, 32, 128
    assert lib.s2attn_decode_workspace_bytes(B, M, N, H, D) == B * H * 64 * M * (D + 2) * 4
    assert lib.s2attn_decode_workspace_bytes(1, 1, 200, 2, 128) == 2 * 4 * 128 * 4 + 256
    assert lib.s2attn_decode_workspace_bytes(1, 2, 1, 2, 128) == 0
    p = ctypes.c_void_p(0x10000)
    assert lib.s2attn_decode(p, p, p, p, p, B, M, N, H, D, p, 1024, NULL) == -3


def test_workspace_checked_before_launch(lib):
    p = ctypes.c_void_p(0x10000)
    rc = lib.s2attn_bwd(p, p, p, p, p, p, p, p, p, 1, 1024, 2, 128, 512, 0, p, 16, NULL)
    assert rc == -3


def test_lora_workspace_size(lib):
    a256 = lambda n: (n + 255) // 256 * 256
    # u [parts, T, 64] + a_pad [parts*64, K] + b_pad [parts*n_out, 64], bf16, each 256-aligned
    assert lib.lora_proj_workspace_bytes(32768, 4096, 4096, 3, 8) == (
        a256(3 * 32768 * 64 * 2) + a256(3 * 64 * 4096 * 2) + a256(3 * 4096 * 64 * 2))
    assert lib.lora_proj_workspace_bytes(300, 520, 256, 3, 8) == a256(3 * 300 * 128) + a256(3 * 64 * 520 * 2) + 3 * 256 * 128
    assert lib.lora_proj_workspace_bytes(300, 520, 256, 3, 0) == 0      # no adapter: no workspace
    assert lib.lora_proj_workspace_bytes(300, 520, 256, 3, 65) == 0     # rank above 64: invalid
    assert lib.lora_proj_workspace_bytes(0, 520, 256, 3, 8) == 0


_P = 0x10000     # a 256-byte-aligned fake device address: these calls fail before any launch
_WS = 1 << 26


@pytest.mark.parametrize("kw,status", [
    (dict(K=12), -1),                                  # K % 8 != 0
    (dict(K=0), -1),
    (dict(r=65), -1),                                  # rank above 64
    (dict(r=-1), -1),
    (dict(parts=0), -1),
    (dict(x=_P + 8), -1),                              # misaligned x
    (dict(b=None), -1),                                # adapter without its up projection
    (dict(scaling=float("nan")), -1),
    (dict(rope_parts=4), -1),                          # more rotated parts than parts
    (dict(rope_parts=2, head_dim=96), -1),             # head_dim outside {32, 64, 128, 256}
    (dict(rope_parts=2, seq_len=7), -1),               # T not a multiple of seq_len
    (dict(rope_parts=2, base=0.0), -1),
    (dict(n_out=384), -2),                             # n_out not a multiple of the 256-column tile
    (dict(K=56), -2),                                  # K below one 64-column box
    (dict(ws_bytes=1024), -3),                         # workspace too small
    (dict(ws=_P + 16), -3),                            # workspace not 256-byte aligned
    (dict(ws=None), -3),
])
def test_lora_validation(lib, kw, status):
    a = dict(x=_P, w=_P, a=_P, b=_P, y=_P, T=300, K=520, n_out=256, parts=3, r=8, scaling=2.0, rope_parts=0,
             head_dim=128, seq_len=100, pos_scale=0.5, base=10000.0, ws=_P, ws_bytes=_WS)
    a.update(kw)
    vp = lambda v: None if v is None else ctypes.c_void_p(v)
    rc = lib.lora_proj_fwd(vp(a["x"]), vp(a["w"]), vp(a["a"]), vp(a["b"]), vp(a["y"]), a["T"], a["K"], a["n_out"],
                           a["parts"], a["r"], a["scaling"], a["rope_parts"], a["head_dim"], a["seq_len"],
                           a["pos_scale"], a["base"], vp(a["ws"]), a["ws_bytes"], None)
    assert rc == status


def test_binding_fails_loudly_without_library(monkeypatch):
    import shifted_sparse_attention_s2attn_b200 as s2
    monkeypatch.setattr(s2, "_lib", None)
    monkeypatch.setattr(s2, "library_path", "/nonexistent/libs2attn.so")
    with pytest.raises(RuntimeError):
        s2.capi()


def test_plain_c_caller(tmp_path, lib):
    """The boundary is a C ABI: a C99 program built against include/s2attn.h and linked
    with libs2attn.so runs its host-side checks (tests/c_abi/check_boundary.c)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    from shifted_sparse_attention_s2attn_b200 import library_path
    libdir = os.path.dirname(library_path)
    exe = tmp_path / "check_boundary"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi", "check_boundary.c"), "-o", str(exe), "-L", libdir,
                    "-ls2attn", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr


def test_debug_build_exports_the_same_boundary(lib):
    """The bounds-checked build (libs2attn_debug.so, -DS2ATTN_DEBUG) is the same C ABI."""
    from shifted_sparse_attention_s2attn_b200 import _build
    debug = ctypes.CDLL(_build.build(debug=True))
    for name in _declared_functions():
        assert hasattr(debug, name), name
    assert debug.s2attn_version() == 100


def test_lora_binding_checks_extents_before_the_call(lib):
    """The C entry point sees only pointers; the binding rejects tensors whose extents do not
    match before anything is passed on (CPU tensors suffice: nothing reaches the library)."""
    import torch
    import shifted_sparse_attention_s2attn_b200 as s2
    bf = dict(dtype=torch.bfloat16)
    x, w = torch.zeros(300, 520, **bf), torch.zeros(3 * 256, 520, **bf)
    a, b = torch.zeros(3 * 8, 520, **bf), torch.zeros(3 * 256, 8, **bf)
    y = torch.zeros(3, 300, 256, **bf)
    bad = [
        dict(w=torch.zeros(3 * 256, 512, **bf)),         # K differs from x's
        dict(w=torch.zeros(3 * 256 + 1, 520, **bf)),     # rows not a multiple of parts
        dict(a=torch.zeros(3 * 8, 512, **bf)),           # adapter K differs
        dict(b=torch.zeros(3 * 256, 4, **bf)),           # rank differs between A and B
        dict(b=None),                                    # A without B
        dict(y=torch.zeros(3, 299, 256, **bf)),          # output too small
        dict(x=torch.zeros(300, 520)),                   # fp32, not bf16
    ]
    for kw in bad:
        args = dict(x=x, w=w, a=a, b=b, y=y)
        args.update(kw)
        with pytest.raises(ValueError):
            s2.lora_proj_fwd(args["x"], args["w"], args["a"], args["b"], args["y"], 3, 2.0)
