"""S^2-Attn with the sequence sharded across ranks (one process per GPU).

The groups of S^2-Attn are independent, so a sequence splits across P ranks with a
single exchange step ("LongLoRA paper notes", section 3.3; nearauto.com, shift short
attention steps (1) and (2)).  Rank p holds the contiguous run of Np = N / P tokens
starting at p * Np (Np a multiple of G):
  * the groups of an unshifted head lie inside one rank;
  * the rolled groups of a shifted head start G/2 tokens into each run, so the last one
    of rank p ends G/2 tokens into rank p+1's run, and rank P-1's wraps round to rank 0's
    (the roll is cyclic).
Each rank therefore receives the first G/2 rows of the next rank (shifted heads only),
runs the kernels on a local tensor whose shifted heads hold its rows [G/2, Np) followed
by that halo -- so every rolled group is a plain group of the local tensor, computed
with shift_heads = 0 -- and sends the results of the halo rows back to their owner.
Tokens belong to exactly one group per head, so results are moved, never summed.

The exchanges are point-to-point sends and receives between ring neighbours through
torch.distributed (NCCL over NVLink between GPUs; gloo on CPU).  A halo of G/2 rows is
copied into this rank's memory before any kernel reads it.  The steps are public:
to_local (exchange and local layout), the kernels with shift_heads = 0, and to_owner
(un-roll and return of the halo rows); sharded_fwd / sharded_bwd compose them with this
library's CUDA kernels.
"""
import torch
import torch.distributed as dist

__all__ = ["shard_range", "to_local", "to_owner", "sharded_fwd", "sharded_bwd"]


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


def _ring_shift(tensors, step, group):
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


def _check(x, G, shift_heads):
    B, Np, H, D = x.shape
    if Np % G or shift_heads < 0 or shift_heads > H or (shift_heads and G % 2):
        raise ValueError("local run must hold whole groups; G even when heads are shifted")
    return B, Np, H, D


def _to_local(xs, halos, G, hs):
    """The local tensors: shifted heads (index >= hs) hold rows [G/2, Np) then the halo."""
    half = G // 2
    out = []
    for x, halo in zip(xs, halos):
        z = x.clone()
        z[:, : x.shape[1] - half, hs:] = x[:, half:, hs:]
        z[:, x.shape[1] - half:, hs:] = halo
        out.append(z)
    return out


def _lse_to_local(lse, halo, G, hs):
    half = G // 2
    z = lse.clone()
    z[:, hs:, : lse.shape[2] - half] = lse[:, hs:, half:]
    z[:, hs:, lse.shape[2] - half:] = halo
    return z


def _from_local(zs, G, hs, group):
    """Undoes _to_local: local rows [0, Np - G/2) of the shifted heads go back to tokens
    [G/2, Np), and the halo rows' results go to the next rank, which owns those tokens."""
    half = G // 2
    tails = [z[:, z.shape[1] - half:, hs:] for z in zs]
    heads = _ring_shift(tails, +1, group)
    out = []
    for z, head in zip(zs, heads):
        x = z.clone()
        x[:, half:, hs:] = z[:, : z.shape[1] - half, hs:]
        x[:, :half, hs:] = head
        out.append(x)
    return out


def _lse_from_local(lse_z, G, hs, group):
    half = G // 2
    (head,) = _ring_shift([lse_z[:, hs:, lse_z.shape[2] - half:]], +1, group)
    x = lse_z.clone()
    x[:, hs:, half:] = lse_z[:, hs:, : lse_z.shape[2] - half]
    x[:, hs:, :half] = head
    return x


def to_local(xs, G, shift_heads, group=None, lse=None):
    """The local layout of this rank's inputs: the shifted heads of each [B, Np, H, D] tensor
    in `xs` hold rows [G/2, Np) followed by the next rank's first G/2 rows, exchanged here;
    the other heads are unchanged.  With `lse` ([B, H, Np]) its shifted heads are laid out
    the same way.  Returns the list of local tensors (and the local lse when given)."""
    B, Np, H, D = _check(xs[0], G, shift_heads)
    hs, half = H - shift_heads, G // 2
    if shift_heads == 0:
        return (list(xs), lse) if lse is not None else list(xs)
    sends = [x[:, :half, hs:] for x in xs] + ([lse[:, hs:, :half]] if lse is not None else [])
    halos = _ring_shift(sends, -1, group)
    zs = _to_local(xs, halos[: len(xs)], G, hs)
    if lse is None:
        return zs
    return zs, _lse_to_local(lse, halos[len(xs)], G, hs)


def to_owner(zs, G, shift_heads, group=None, lse=None):
    """Undoes to_local for results computed on the local layout: each tensor's shifted heads
    go back to this rank's rows, and the halo rows' results travel to the next rank, which
    owns those tokens.  Returns the list of tensors (and the lse when given)."""
    H = zs[0].shape[2]
    hs = H - shift_heads
    if shift_heads == 0:
        return (list(zs), lse) if lse is not None else list(zs)
    out = _from_local(list(zs), G, hs, group)
    if lse is None:
        return out
    return out, _lse_from_local(lse, G, hs, group)


def _cuda_fwd(q, k, v, G):
    from . import s2attn_fwd
    B, N, H, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    s2attn_fwd(q, k, v, o, lse, G, 0)
    return o, lse


def _cuda_bwd(q, k, v, o, dout, lse, G):
    from . import s2attn_bwd, s2attn_bwd_workspace_bytes
    B, N, H, D = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(s2attn_bwd_workspace_bytes(B, N, H, D), dtype=torch.uint8, device=q.device)
    s2attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, G, 0, ws)
    return dq, dk, dv


def sharded_fwd(q, k, v, G, shift_heads, group=None):
    """S^2-Attn forward on this rank's run of tokens ([B, Np, H, D] bf16 CUDA tensors).
    Returns this rank's o [B, Np, H, D] and lse [B, H, Np], equal to the rows [t0, t1) of
    the unsharded call (shard_range gives t0, t1)."""
    qz, kz, vz = to_local((q, k, v), G, shift_heads, group)
    oz, lse_z = _cuda_fwd(qz, kz, vz, G)
    (o,), lse = to_owner([oz], G, shift_heads, group, lse=lse_z)
    return o, lse


def sharded_bwd(q, k, v, o, dout, lse, G, shift_heads, group=None):
    """S^2-Attn backward on this rank's run of tokens: dq, dk, dv [B, Np, H, D], equal to
    the rows [t0, t1) of the unsharded backward."""
    (qz, kz, vz, oz, dz), lse_z = to_local((q, k, v, o, dout), G, shift_heads, group, lse=lse)
    dqz, dkz, dvz = _cuda_bwd(qz, kz, vz, oz, dz, lse_z, G)
    return tuple(to_owner([dqz, dkz, dvz], G, shift_heads, group))
