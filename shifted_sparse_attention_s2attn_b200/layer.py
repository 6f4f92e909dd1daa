"""One LongLoRA attention layer on this library's kernels, forward and backward.

The steps on either side of S^2-Attn in LongLoRA training ("LongLoRA paper notes",
sections 3.2-3.4; nearauto.com article, "long-context LoRA improvement"): the q, k, v
projections with low-rank adapters, RoPE with position interpolation on q and k, S^2-Attn,
and the o projection with its adapter.  W is frozen; the adapters and the layer input get
gradients.  Every step is a C-ABI call of the library:

  forward   lora_proj_fwd (q, k, v stacked; RoPE-PI fused into the epilogue of q and k, so
            there is no separate rotation pass)  ->  s2attn_fwd  ->  lora_proj_fwd (o)
  backward  lora_proj_bwd (o)  ->  s2attn_bwd  ->  rope_pi_apply(dq, dk, -pos_scale) (the
            transposed rotation)  ->  lora_proj_bwd (q, k, v stacked)

Tensors are bf16 on one CUDA device; x is [B*N, K] (K = H*D, the model width) and the layer's
q, k, v live stacked in one [3, B, N, H, D] buffer, so the projection writes them in place
for the attention and the stacked gradient [3, B, N, H, D] feeds the projection backward.
"""
from dataclasses import dataclass

import torch

from . import (lora_proj_bwd, lora_proj_bwd_workspace_bytes, lora_proj_fwd, lora_proj_workspace_bytes,
               rope_pi_apply, s2attn_bwd, s2attn_bwd_workspace_bytes, s2attn_fwd)

__all__ = ["LayerShape", "LayerWeights", "LayerBuffers", "layer_fwd", "layer_bwd"]


@dataclass(frozen=True)
class LayerShape:
    B: int
    N: int
    H: int
    D: int
    G: int
    shift_heads: int
    r: int                  # adapter rank (0: no adapters)
    scaling: float          # alpha / r
    pos_scale: float        # L0 / N
    base: float = 10000.0

    @property
    def T(self):
        return self.B * self.N

    @property
    def width(self):
        return self.H * self.D


@dataclass
class LayerWeights:
    w_qkv: torch.Tensor                 # [3*width, width]
    w_o: torch.Tensor                   # [width, width]
    a_qkv: torch.Tensor = None          # [3*r, width]
    b_qkv: torch.Tensor = None          # [3*width, r]
    a_o: torch.Tensor = None            # [r, width]
    b_o: torch.Tensor = None            # [width, r]


class LayerBuffers:
    """Device buffers of one layer step (activations kept for the backward, gradients and
    the workspaces of the calls), allocated once and reused by every step."""

    def __init__(self, s: LayerShape, device):
        bf, f32 = torch.bfloat16, torch.float32
        T, n, r = s.T, s.width, s.r
        self.qkv = torch.empty((3, s.B, s.N, s.H, s.D), dtype=bf, device=device)
        self.o = torch.empty((s.B, s.N, s.H, s.D), dtype=bf, device=device)
        self.lse = torch.empty((s.B, s.H, s.N), dtype=f32, device=device)
        self.y = torch.empty((1, T, n), dtype=bf, device=device)
        self.do = torch.empty((T, n), dtype=bf, device=device)
        self.dqkv = torch.empty((3, s.B, s.N, s.H, s.D), dtype=bf, device=device)
        self.dx = torch.empty((T, n), dtype=bf, device=device)
        self.da_qkv = torch.empty((3 * r, n), dtype=bf, device=device) if r else None
        self.db_qkv = torch.empty((3 * n, r), dtype=bf, device=device) if r else None
        self.da_o = torch.empty((r, n), dtype=bf, device=device) if r else None
        self.db_o = torch.empty((n, r), dtype=bf, device=device) if r else None

        def ws(nbytes):
            return torch.empty(max(256, nbytes), dtype=torch.uint8, device=device)
        self.ws_fwd_qkv = ws(lora_proj_workspace_bytes(T, n, n, 3, r))
        self.ws_fwd_o = ws(lora_proj_workspace_bytes(T, n, n, 1, r))
        self.ws_attn = ws(s2attn_bwd_workspace_bytes(s.B, s.N, s.H, s.D))
        self.ws_bwd_qkv = ws(lora_proj_bwd_workspace_bytes(T, n, n, 3, r))
        self.ws_bwd_o = ws(lora_proj_bwd_workspace_bytes(T, n, n, 1, r))


def layer_fwd(s: LayerShape, w: LayerWeights, x, buf: LayerBuffers, stream=None):
    """y [1, B*N, width] = o-projection(S^2-Attn(RoPE-PI(q, k), v)) of x [B*N, width].
    Keeps q, k, v, o and lse in `buf` for the backward.  Returns buf.y."""
    lora_proj_fwd(x, w.w_qkv, w.a_qkv, w.b_qkv, buf.qkv, 3, s.scaling, rope_parts=2, head_dim=s.D, seq_len=s.N,
                  pos_scale=s.pos_scale, base=s.base, workspace=buf.ws_fwd_qkv, stream=stream)
    q, k, v = buf.qkv[0], buf.qkv[1], buf.qkv[2]
    s2attn_fwd(q, k, v, buf.o, buf.lse, s.G, s.shift_heads, stream)
    lora_proj_fwd(buf.o.view(s.T, s.width), w.w_o, w.a_o, w.b_o, buf.y, 1, s.scaling, workspace=buf.ws_fwd_o,
                  stream=stream)
    return buf.y


def layer_bwd(s: LayerShape, w: LayerWeights, x, dy, buf: LayerBuffers, stream=None):
    """Gradients of the layer for dy [1, B*N, width]: buf.dx and the adapters' buf.da_qkv,
    buf.db_qkv, buf.da_o, buf.db_o (W frozen).  Needs the activations of layer_fwd in buf."""
    lora_proj_bwd(buf.o.view(s.T, s.width), w.w_o, w.a_o, w.b_o, dy, buf.do, buf.da_o, buf.db_o, 1, s.scaling,
                  buf.ws_bwd_o, stream)
    q, k, v = buf.qkv[0], buf.qkv[1], buf.qkv[2]
    dq, dk, dv = buf.dqkv[0], buf.dqkv[1], buf.dqkv[2]
    s2attn_bwd(q, k, v, buf.o, buf.do.view(s.B, s.N, s.H, s.D), buf.lse, dq, dk, dv, s.G, s.shift_heads,
               buf.ws_attn, stream)
    rope_pi_apply(dq, dk, -s.pos_scale, s.base, stream)
    lora_proj_bwd(x, w.w_qkv, w.a_qkv, w.b_qkv, buf.dqkv, buf.dx, buf.da_qkv, buf.db_qkv, 3, s.scaling,
                  buf.ws_bwd_qkv, stream)
    return buf.dx
