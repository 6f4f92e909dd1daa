"""Seeded synthetic workloads (LLaMA2 layer shapes) shared by the tests, the bench and
the oracle checks.

This module holds no arithmetic of the method: it only names the workloads and
draws their random inputs.  Recipe: for workload index c and tensor id
(q=0, k=1, v=2, dO=3, outlier-row choice=4), numpy.random.default_rng(1000*c + id)
draws standard normals in fp64, rounded to fp32 and then to bf16 (round to nearest
even), or kept in fp32 for the fp32 workload.  For the 100k workload 1% of the
(token, head) rows of K are multiplied by 8 (exact in bf16).  Q and K of the bf16
workloads are then meant to go through RoPE with position interpolation
(pos_scale = L0 / N, L0 = 4096, base 10000) by whoever consumes them.
"""
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    B: int
    N: int
    H: int
    D: int
    G: int
    shift_heads: int
    dtype: str            # "f32" or "bf16"
    rope: bool            # Q/K go through RoPE-PI first
    L0: int = 4096
    base: float = 10000.0
    k_outlier_frac: float = 0.0
    k_outlier_mult: float = 8.0

    @property
    def pos_scale(self) -> float:
        return self.L0 / self.N

    @property
    def groups(self) -> int:
        return self.N // self.G

    def units(self):
        """All (b, h, j) groups of the workload."""
        return [(b, h, j) for b in range(self.B) for h in range(self.H) for j in range(self.groups)]


WORKLOADS = {
    "tiny_fp32": Workload(0, "tiny_fp32", 1, 256, 4, 64, 64, 2, "f32", False),
    "llama2_7b_8k": Workload(1, "llama2_7b_8k", 1, 8192, 32, 128, 2048, 16, "bf16", True),
    "llama2_7b_32k": Workload(2, "llama2_7b_32k", 1, 32768, 32, 128, 8192, 16, "bf16", True),
    "llama2_13b_64k": Workload(3, "llama2_13b_64k", 1, 65536, 40, 128, 16384, 20, "bf16", True),
    "llama2_7b_100k": Workload(4, "llama2_7b_100k", 1, 102400, 32, 128, 25600, 16, "bf16", True,
                               k_outlier_frac=0.01),
}

# Full causal attention at the 32k shape (the inference case: one group, no shift).
FULL_CAUSAL_32K = Workload(2, "llama2_7b_32k_full_causal", 1, 32768, 32, 128, 32768, 0, "bf16", True)

TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "dout": 3, "outlier": 4}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round binary32 values to bf16 (nearest even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal(seed, shape):
    return np.random.default_rng(seed).standard_normal(shape, dtype=np.float64)


def make_tensor(w: Workload, name: str, seed_index: int | None = None) -> np.ndarray:
    """One input tensor [B,N,H,D]: float32 for the fp32 workload, else bf16 bits (uint16)."""
    c = w.index if seed_index is None else seed_index
    x = _normal(1000 * c + TENSOR_IDS[name], (w.B, w.N, w.H, w.D)).astype(np.float32)
    if w.dtype == "f32":
        return x
    bits = f32_to_bf16_bits(x)
    if name == "k" and w.k_outlier_frac > 0:
        rows = outlier_rows(w, seed_index)
        flat = bits.reshape(w.B, w.N * w.H, w.D)
        for b in range(w.B):
            sel = flat[b, rows[b]]
            flat[b, rows[b]] = f32_to_bf16_bits(bf16_bits_to_f32(sel) * np.float32(w.k_outlier_mult))
    return bits


def outlier_rows(w: Workload, seed_index: int | None = None):
    """Per batch entry, round(frac * N * H) distinct (t, h) rows, as flat indices t*H + h."""
    c = w.index if seed_index is None else seed_index
    rng = np.random.default_rng(1000 * c + TENSOR_IDS["outlier"])
    n = int(round(w.k_outlier_frac * w.N * w.H))
    return [np.sort(rng.choice(w.N * w.H, size=n, replace=False)) for _ in range(w.B)]


def make_inputs(w: Workload, names=("q", "k", "v", "dout")):
    return {n: make_tensor(w, n) for n in names}


def scaled(w: Workload, **changes) -> Workload:
    """A smaller copy of a workload (same recipe and seeds) for quick parity cases."""
    d = dict(w.__dict__)
    d.update(changes)
    return Workload(**d)


# ---- LoRA-adapted projections ------------------------------------------------------
# The LLaMA2-7B layer: hidden size 4096 = H*D (32 heads of 128); q, k, v stacked (parts 3)
# and o (parts 1); LoRA rank 8 with alpha 16 (scaling 2), LongLoRA's adapter setting.
LORA_LLAMA2_7B = dict(K=4096, n_out=4096, r=8, scaling=2.0)
LORA_IDS = {"x": 10, "w": 11, "a": 12, "b": 13}


def make_lora_inputs(T, K, n_out, parts, r, seed=0, b_std=0.05):
    """Seeded inputs of a LoRA-adapted projection, as bf16 bit patterns (uint16).

    numpy.random.default_rng(1000*seed + id) draws standard normals in fp32 (ids: x 10,
    W 11, A 12, B 13), scaled and rounded to bf16 (nearest even):
      x [T, K]             ~ N(0, 1)          (a layer's normalised hidden states)
      W [parts*n_out, K]   ~ N(0, 1/K)        (so every output is ~ N(0, 1))
      A [parts*r, K]       ~ N(0, 1/K)
      B [parts*n_out, r]   ~ N(0, b_std^2)    (nonzero, as after some training; LoRA
                                               starts B at zero, which would hide the term)
    Returns (x, W, A, B); A and B are None when r == 0."""
    def draw(name, shape, std):
        rng = np.random.default_rng(1000 * seed + LORA_IDS[name])
        x = rng.standard_normal(shape, dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        return f32_to_bf16_bits(x)
    x = draw("x", (T, K), 1.0)
    w = draw("w", (parts * n_out, K), 1.0 / np.sqrt(K))
    if r == 0:
        return x, w, None, None
    return x, w, draw("a", (parts * r, K), 1.0 / np.sqrt(K)), draw("b", (parts * n_out, r), b_std)
