"""One prefill (or decode step) split across the ranks of a process group.

Every (b, KV head) group's block selection and attention read only that group's keys and
values ("DashAttention: Making Sparse Attention Fully Differentiable with Adaptive Block
Selection", section "Core Mechanism"), so a prefill splits by KV heads with no exchange on the
data path: rank i computes the query heads of its contiguous range of KV heads on its own GPU
(local memory only), and one all-gather along the head dimension restores the full output on
every rank.  A decode step splits the same way by sequences (the batch dimension).

The per-shard computation is the library's C ABI (`dash_prefill` / `dash_decode` on the
shard's slices) unless the caller passes another callable; the all-gather is the process
group's (NCCL on GPUs, gloo on the CPU).  Shards of unequal size (Hkv or B not divisible by
the world size) are padded to the largest shard for the collective and trimmed after it.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple


def shard_range(n: int, world: int, rank: int) -> Tuple[int, int]:
    """[lo, hi) of `n` units for `rank` of `world`: contiguous, sizes differing by at most one
    (the first n % world ranks take one more)."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def _gather_dim(local, dim: int, sizes, group):
    """All-gather `local` along `dim` when the ranks' sizes along it are `sizes`: pad to the
    largest size, gather, and concatenate the trimmed pieces in rank order."""
    import torch
    import torch.distributed as dist
    world = len(sizes)
    if world == 1:
        return local
    big = max(sizes)
    pad = list(local.shape)
    pad[dim] = big
    buf = torch.zeros(pad, dtype=local.dtype, device=local.device)
    if local.shape[dim] > 0:
        buf.narrow(dim, 0, local.shape[dim]).copy_(local)
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf, group=group)
    return torch.cat([p.narrow(dim, 0, s) for p, s in zip(parts, sizes)], dim=dim)


def _default_prefill(q, k, v, alpha, coarse_scale):
    from . import dash_attn
    out, _ = dash_attn.dash_prefill(q, k, v, alpha=alpha, coarse_scale=coarse_scale)
    return out


def prefill_by_kv_heads(q, k, v, alpha: float, coarse_scale: float, group=None,
                        compute: Optional[Callable] = None, out_dtype=None):
    """Full-output prefill of q [B, Hq, T, d], k, v [B, Hkv, T, d], split by KV heads over the
    ranks of `group` (default: the default process group).  Every rank passes the same full
    tensors (or at least correct values for its own KV heads) and receives the full output.
    compute(q_shard, k_shard, v_shard, alpha, coarse_scale) -> out_shard runs one shard; the
    default is the library's dash_prefill.  out_dtype is the dtype compute returns (default
    q.dtype, which is dash_prefill's); a rank left without KV heads (world > Hkv) contributes
    an empty tensor of that dtype, since every rank of the collective must agree on it."""
    import torch.distributed as dist
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    lo, hi = shard_range(Hkv, world, rank)
    fn = compute or _default_prefill
    if hi > lo:
        out = fn(q[:, lo * G:hi * G].contiguous(), k[:, lo:hi].contiguous(), v[:, lo:hi].contiguous(),
                 alpha, coarse_scale)
    else:
        out = q.new_zeros((B, 0, T, d), dtype=out_dtype or q.dtype)
    sizes = [(shard_range(Hkv, world, r)[1] - shard_range(Hkv, world, r)[0]) * G for r in range(world)]
    return _gather_dim(out, 1, sizes, group)


def _default_decode(q, k_cache, v_cache, ksum, kv_len, alpha, coarse_scale):
    from . import dash_attn
    out, _ = dash_attn.dash_decode(q, k_cache, v_cache, ksum, kv_len, alpha=alpha, coarse_scale=coarse_scale)
    return out


def decode_by_sequences(q, k_cache, v_cache, ksum, kv_len, alpha: float, coarse_scale: float, group=None,
                        compute: Optional[Callable] = None, out_dtype=None):
    """Full-output decode step of q [B, Hq, d] over caches [B, Hkv, Tmax, d] (ksum
    [B, Hkv, Tmax / 64, d], kv_len [B]), split by sequences over the ranks of `group`; every
    rank receives the full output [B, Hq, d].  compute(q, k_cache, v_cache, ksum, kv_len, alpha,
    coarse_scale) -> out runs one shard (default: the library's dash_decode); out_dtype as for
    prefill_by_kv_heads."""
    import torch.distributed as dist
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    B = q.shape[0]
    lo, hi = shard_range(B, world, rank)
    fn = compute or _default_decode
    if hi > lo:
        out = fn(q[lo:hi].contiguous(), k_cache[lo:hi].contiguous(), v_cache[lo:hi].contiguous(),
                 ksum[lo:hi].contiguous(), kv_len[lo:hi].contiguous(), alpha, coarse_scale)
    else:
        out = q.new_zeros((0,) + tuple(q.shape[1:]), dtype=out_dtype or q.dtype)
    sizes = [shard_range(B, world, r)[1] - shard_range(B, world, r)[0] for r in range(world)]
    return _gather_dim(out, 0, sizes, group)
