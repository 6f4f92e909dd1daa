"""S^2-Attn with the sequence sharded across ranks (one process per GPU).

The groups of S^2-Attn are independent, so a sequence splits across P ranks with a
single exchange step ("LongLoRA paper notes", section 3.3; nearauto.com, shift short
attention steps (1) and (2)).  Rank p holds the contiguous run of Np = N / P tokens
starting at p * Np (Np a multiple of G):
  * the groups of an unshifted head lie inside one rank;
  * the rolled groups of a shifted head start G/2 tokens into each run, so the last one
    of rank p ends G/2 tokens into rank p+1's run, and rank P-1's wraps round to rank 0's
    (the roll is cyclic).

The library's kernels roll a shifted head cyclically inside the tensors they are given:
on a rank's own run their last rolled group reads the run's tail followed by the run's
rows [0, G/2).  Those rows of the shifted heads are exactly what this rank does not need
(they belong to the previous rank's last group), and the next rank's first G/2 rows (the
halo) are exactly what it lacks.  So each call
  1. copies its rows [0, G/2) of the shifted heads out (halo_rows), sends them to the
     previous rank and receives the next rank's (exchange),
  2. writes the received halo into those rows (put_halo_rows) and runs the unmodified
     kernels with the shift, then writes its own rows back,
  3. copies the results that landed in rows [0, G/2) -- the halo tokens' results -- out,
     sends them to the next rank (their owner) and writes the ones it receives from the
     previous rank into its own rows.
Only G/2 rows of the shifted heads per tensor are copied or sent; no local copy of a whole
tensor is made.  The copies are this library's halo kernels (s2attn_halo_rows and
s2attn_halo_lse), the exchange is torch.distributed point-to-point (NCCL over NVLink
between GPUs; gloo on CPU), received into this rank's memory before a kernel reads it.
Tokens belong to exactly one group per head, so results are moved, never summed.

sharded_fwd and sharded_bwd modify the caller's input tensors (rows [0, G/2) of the
shifted heads) while they run and restore them before they return, on the current
stream: other streams must not read those tensors meanwhile.
"""
import torch
import torch.distributed as dist

__all__ = ["shard_range", "exchange", "halo_rows", "put_halo_rows", "halo_lse", "put_halo_lse",
           "sharded_fwd", "sharded_bwd"]


def shard_range(N, G, world, rank):
    """Tokens [t0, t1) held by `rank` when N tokens are split over `world` ranks."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank or world size")
    if N % world or (N // world) % G:
        raise ValueError("each rank must hold a whole number of groups: (N / world) % G == 0")
    n = N // world
    return rank * n, (rank + 1) * n


def _world(group):
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group), dist.get_rank(group)
    return 1, 0


def exchange(tensors, step, group=None):
    """Sends each tensor to rank (r + step) mod P and returns the tensors received from
    rank (r - step) mod P (same shapes and dtypes).  With one rank the tensors come back."""
    world, rank = _world(group)
    sends = [t.contiguous() for t in tensors]
    if world == 1:
        return sends
    dst, src = (rank + step) % world, (rank - step) % world
    recvs = [torch.empty_like(t) for t in sends]
    ops = []
    for i, (s, r) in enumerate(zip(sends, recvs)):
        ops.append(dist.P2POp(dist.isend, s, dist.get_global_rank(group, dst) if group else dst, group, tag=i))
        ops.append(dist.P2POp(dist.irecv, r, dist.get_global_rank(group, src) if group else src, group, tag=i))
    for w in dist.batch_isend_irecv(ops):
        w.wait()
    return recvs


# ---- the four primitives: the halo copies (library kernels) and the attention calls -----

def _rows_copy(xs, bufs, to_buf, G, shift_heads):
    from . import s2attn_halo_rows
    s2attn_halo_rows(list(xs), list(bufs), to_buf, G, shift_heads)


def _lse_copy(lses, bufs, to_buf, G, shift_heads):
    from . import s2attn_halo_lse
    s2attn_halo_lse(list(lses), list(bufs), to_buf, G, shift_heads)


def _attn_fwd(q, k, v, G, shift_heads):
    from . import s2attn_fwd
    B, N, H, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    s2attn_fwd(q, k, v, o, lse, G, shift_heads)
    return o, lse


def _attn_bwd(q, k, v, o, dout, lse, G, shift_heads):
    from . import s2attn_bwd, s2attn_bwd_workspace_bytes
    B, N, H, D = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(s2attn_bwd_workspace_bytes(B, N, H, D), dtype=torch.uint8, device=q.device)
    s2attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, G, shift_heads, ws)
    return dq, dk, dv


# ---- the halo steps --------------------------------------------------------------------

def halo_rows(xs, G, shift_heads):
    """Rows [0, G/2) of the shifted heads of each [B, Np, H, D] tensor in xs, as new
    contiguous [B, G/2, shift_heads, D] tensors (one library launch)."""
    B, Np, H, D = xs[0].shape
    bufs = [torch.empty((B, G // 2, shift_heads, D), dtype=x.dtype, device=x.device) for x in xs]
    _rows_copy(xs, bufs, True, G, shift_heads)
    return bufs


def put_halo_rows(bufs, xs, G, shift_heads):
    """Writes each [B, G/2, shift_heads, D] buffer into rows [0, G/2) of the shifted heads of
    the matching tensor in xs (one library launch)."""
    _rows_copy(xs, bufs, False, G, shift_heads)


def halo_lse(lses, G, shift_heads):
    """The same rows of [B, H, Np] fp32 statistics, as new [B, shift_heads, G/2] tensors."""
    B, H, Np = lses[0].shape
    bufs = [torch.empty((B, shift_heads, G // 2), dtype=x.dtype, device=x.device) for x in lses]
    _lse_copy(lses, bufs, True, G, shift_heads)
    return bufs


def put_halo_lse(bufs, lses, G, shift_heads):
    _lse_copy(lses, bufs, False, G, shift_heads)


def _check(x, G, shift_heads):
    B, Np, H, D = x.shape
    if Np % G or shift_heads < 0 or shift_heads > H or (shift_heads and G % 2):
        raise ValueError("local run must hold whole groups; G even when heads are shifted")
    return B, Np, H, D


def sharded_fwd(q, k, v, G, shift_heads, group=None):
    """S^2-Attn forward on this rank's run of tokens ([B, Np, H, D] bf16 CUDA tensors).
    Returns this rank's o [B, Np, H, D] and lse [B, H, Np], equal to the rows [t0, t1) of
    the unsharded call (shard_range gives t0, t1).  q, k, v are restored before returning."""
    _check(q, G, shift_heads)
    if shift_heads == 0:
        return _attn_fwd(q, k, v, G, 0)
    xs = [q, k, v]
    own = halo_rows(xs, G, shift_heads)
    halo = exchange(own, -1, group)              # the next rank's first G/2 rows
    put_halo_rows(halo, xs, G, shift_heads)
    try:
        o, lse = _attn_fwd(q, k, v, G, shift_heads)
    finally:
        put_halo_rows(own, xs, G, shift_heads)   # q, k, v as the caller gave them
    # rows [0, G/2) of o and lse hold the halo tokens' results: to their owner, the next rank
    res = halo_rows([o], G, shift_heads) + halo_lse([lse], G, shift_heads)
    back = exchange(res, +1, group)
    put_halo_rows(back[:1], [o], G, shift_heads)
    put_halo_lse(back[1:], [lse], G, shift_heads)
    return o, lse


def sharded_bwd(q, k, v, o, dout, lse, G, shift_heads, group=None):
    """S^2-Attn backward on this rank's run of tokens: dq, dk, dv [B, Np, H, D], equal to
    the rows [t0, t1) of the unsharded backward.  q, k, v, o, dout, lse are restored."""
    _check(q, G, shift_heads)
    if shift_heads == 0:
        return _attn_bwd(q, k, v, o, dout, lse, G, 0)
    xs = [q, k, v, o, dout]
    own = halo_rows(xs, G, shift_heads)
    own_lse = halo_lse([lse], G, shift_heads)
    got = exchange(own + own_lse, -1, group)
    put_halo_rows(got[:len(xs)], xs, G, shift_heads)
    put_halo_lse(got[len(xs):], [lse], G, shift_heads)
    try:
        dq, dk, dv = _attn_bwd(q, k, v, o, dout, lse, G, shift_heads)
    finally:
        put_halo_rows(own, xs, G, shift_heads)
        put_halo_lse(own_lse, [lse], G, shift_heads)
    back = exchange(halo_rows([dq, dk, dv], G, shift_heads), +1, group)
    put_halo_rows(back, [dq, dk, dv], G, shift_heads)
    return dq, dk, dv
