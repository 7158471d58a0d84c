"""Seeded synthetic inputs for the DashAttention forward pass.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no scores, no entmax, no attention).  Both the CUDA path and the
fp64 oracle are fed from the tensors it returns.

Workloads stand in for the long-context evaluations of "DashAttention and the year
sparse attention became a field" (section "The numbers": 16K-96K context, 75 % and
93.75 % block sparsity), whose datasets and trained models are not available here.
Structure: a set of random topic vectors; every 64-token key block draws one topic and
its keys are 2*topic + N(0, I); every query vector draws its own topic, q = 2*topic +
N(0, I); values are N(0, 1).  The coarse scale that sets the sparsity is calibrated
separately (with the oracle) and stored with the seed.

Generation runs on the CPU with ``torch.Generator`` so the same seed gives the same
bf16 tensors on every machine; draw order is topics, block topics, key noise, query
topics, query noise, values.
"""
from __future__ import annotations

import dataclasses
import hashlib

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str              # "prefill" or "decode"
    B: int
    Hq: int
    Hkv: int
    T: int                 # prefill length, or decode cache length (= kv_len)
    d: int
    block: int
    alpha: float
    n_topics: int          # 0: plain N(0, 1) inputs
    target_sparsity: float | None
    seed: int
    fp32_source: bool = False   # inputs drawn in fp32, rounded once to bf16
    coherent: bool = False      # one query topic per (b, 64-position block), shared by all heads


WORKLOADS = {
    "tiny": Workload("tiny prefill T=512", "prefill", 1, 1, 1, 512, 64, 64, 1.5, 0, None,
                     0xDA5A + 0, fp32_source=True),
    "16k": Workload("16K prefill, 75% block sparsity", "prefill", 1, 16, 2, 16384, 128, 64, 1.5,
                    64, 0.75, 0xDA5A + 1),
    "32k": Workload("32K prefill alpha sweep", "prefill", 1, 16, 2, 32768, 128, 64, 1.5,
                    64, 0.75, 0xDA5A + 2),
    "96k": Workload("96K prefill, 93.75% block sparsity", "prefill", 1, 32, 8, 98304, 128, 64, 1.5,
                    256, 0.9375, 0xDA5A + 3),
    "decode96k": Workload("96K decode, B=8, 93.75% block sparsity", "decode", 8, 32, 8, 98304, 128, 64,
                          1.5, 256, 0.9375, 0xDA5A + 4),
    # not a target workload: query topics shared by the heads and positions of a 64-token
    # block, so the rows of a tile select correlated block sets (little union inflation)
    "16k-coherent": Workload("16K prefill, 75% block sparsity, block-coherent query topics (non-target)",
                             "prefill", 1, 16, 2, 16384, 128, 64, 1.5, 64, 0.75, 0xDA5A + 5,
                             coherent=True),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def topic_prefill(B, Hq, Hkv, T, d, block, n_topics, seed, fp32_source=False, coherent=False):
    """q [B,Hq,T,d], k, v [B,Hkv,T,d] in bf16 (CPU) from the topic generator.

    n_topics == 0 gives plain N(0, 1) q, k, v (drawn in fp32, rounded once to bf16).
    coherent: the query topic is drawn per (b, 64-position block) and shared by every head
    and position of the block (noise stays per query vector)."""
    g = _gen(seed)
    if n_topics == 0:
        q = torch.randn(B, Hq, T, d, generator=g)
        k = torch.randn(B, Hkv, T, d, generator=g)
        v = torch.randn(B, Hkv, T, d, generator=g)
        return q.bfloat16(), k.bfloat16(), v.bfloat16()
    nb = (T + block - 1) // block
    topics = torch.randn(n_topics, d, generator=g)
    blk_topic = torch.randint(0, n_topics, (B, nb), generator=g)
    k = torch.empty(B, Hkv, T, d, dtype=torch.bfloat16)
    for b in range(B):
        tok_topic = blk_topic[b].repeat_interleave(block)[:T]          # [T]
        base = 2.0 * topics[tok_topic]                                  # [T, d]
        for h in range(Hkv):
            k[b, h] = (base + torch.randn(T, d, generator=g)).bfloat16()
    q = torch.empty(B, Hq, T, d, dtype=torch.bfloat16)
    if coherent:
        qb_topic = torch.randint(0, n_topics, (B, nb), generator=g)
        q_topic = qb_topic.repeat_interleave(block, dim=1)[:, :T].unsqueeze(1).expand(B, Hq, T)
    else:
        q_topic = torch.randint(0, n_topics, (B, Hq, T), generator=g)
    for b in range(B):
        for h in range(Hq):
            q[b, h] = (2.0 * topics[q_topic[b, h]] + torch.randn(T, d, generator=g)).bfloat16()
    v = torch.empty(B, Hkv, T, d, dtype=torch.bfloat16)
    for b in range(B):
        for h in range(Hkv):
            v[b, h] = torch.randn(T, d, generator=g).bfloat16()
    return q, k, v


def out_grad(B, Hq, T, d, seed):
    """Upstream gradient d loss / d out [B, Hq, T, d]: N(0, 1) drawn in fp32, rounded to bf16."""
    return torch.randn(B, Hq, T, d, generator=_gen(seed)).bfloat16()


def topic_decode(B, Hq, Hkv, Tmax, d, block, n_topics, seed):
    """Decode step inputs: q [B,Hq,d], caches k, v [B,Hkv,Tmax,d] (bf16, CPU), kv_len [B].

    Every sequence has its own topics, block topics and noise; the cache is full
    (kv_len = Tmax) and already holds the new token."""
    kc = torch.empty(B, Hkv, Tmax, d, dtype=torch.bfloat16)
    vc = torch.empty(B, Hkv, Tmax, d, dtype=torch.bfloat16)
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16)
    for b in range(B):
        qb, kb, vb = topic_prefill_last(1, Hq, Hkv, Tmax, d, block, n_topics, seed * 1000 + b)
        kc[b], vc[b], q[b] = kb[0], vb[0], qb[0]
    kv_len = torch.full((B,), Tmax, dtype=torch.int32)
    return q, kc, vc, kv_len


def topic_prefill_last(B, Hq, Hkv, T, d, block, n_topics, seed):
    """As topic_prefill, but only the query vector at position T-1 is drawn (decode)."""
    g = _gen(seed)
    nb = (T + block - 1) // block
    topics = torch.randn(n_topics, d, generator=g)
    blk_topic = torch.randint(0, n_topics, (B, nb), generator=g)
    k = torch.empty(B, Hkv, T, d, dtype=torch.bfloat16)
    for b in range(B):
        base = 2.0 * topics[blk_topic[b].repeat_interleave(block)[:T]]
        for h in range(Hkv):
            k[b, h] = (base + torch.randn(T, d, generator=g)).bfloat16()
    q_topic = torch.randint(0, n_topics, (B, Hq), generator=g)
    q = (2.0 * topics[q_topic] + torch.randn(B, Hq, d, generator=g)).bfloat16()
    v = torch.empty(B, Hkv, T, d, dtype=torch.bfloat16)
    for b in range(B):
        for h in range(Hkv):
            v[b, h] = torch.randn(T, d, generator=g).bfloat16()
    return q, k, v


def make(name_or_wl, **override):
    """Inputs of a named workload (or a Workload), fields overridable by keyword."""
    wl = WORKLOADS[name_or_wl] if isinstance(name_or_wl, str) else name_or_wl
    if override:
        wl = dataclasses.replace(wl, **override)
    if wl.kind == "decode":
        return wl, topic_decode(wl.B, wl.Hq, wl.Hkv, wl.T, wl.d, wl.block, wl.n_topics, wl.seed)
    return wl, topic_prefill(wl.B, wl.Hq, wl.Hkv, wl.T, wl.d, wl.block, wl.n_topics, wl.seed,
                             wl.fp32_source, wl.coherent)


def sample_rows(B, Hq, T, n, seed, t_fixed=(), t_lo=0):
    """Row triples (b, h, t): stratified positions t_fixed x all heads, plus n uniform draws."""
    g = _gen(seed)
    rows = []
    for t in t_fixed:
        if 0 <= t < T:
            for b in range(B):
                for h in range(Hq):
                    rows.append((b, h, t))
    if n > 0:
        b = torch.randint(0, B, (n,), generator=g)
        h = torch.randint(0, Hq, (n,), generator=g)
        t = torch.randint(t_lo, T, (n,), generator=g)
        rows += list(zip(b.tolist(), h.tolist(), t.tolist()))
    return rows


def sha256(*tensors) -> str:
    h = hashlib.sha256()
    for t in tensors:
        h.update(t.contiguous().view(torch.uint8).numpy().tobytes())
    return h.hexdigest()
