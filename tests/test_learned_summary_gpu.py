"""GPU parity of the learned summary head (Stage 0 as an attention pooling with one query
vector per KV head; "DashAttention and the year sparse attention became a field", section
"What alpha-entmax changes"), through the C ABI, against the fp64 oracle."""
import os
import sys

import numpy as np
import pytest
import torch

sys.path.insert(0, os.path.dirname(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(__file__)))

from sparse_hierarchical_attention_pool_b200 import dash_attn as da  # noqa: E402
from sparse_hierarchical_attention_pool_b200 import inputs  # noqa: E402

import oracle  # noqa: E402
from gpu_helpers import compare_out, rows_of, stratified_rows  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    oracle.build()


def _head(Hkv, d, scale, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(Hkv, d, generator=g) * scale).float()


@pytest.mark.parametrize("d,T", [(128, 1024), (64, 640), (128, 130)])
def test_block_summary_w_vs_oracle(d, T):
    _, (_, k, _) = inputs.make("16k", B=2, Hq=4, Hkv=2, T=T, d=d, n_topics=8, seed=31 + d)
    w = _head(2, d, 0.5, 7)
    got = da.dash_block_summary_w(k.cuda(), w.cuda())
    torch.cuda.synchronize()
    ref = oracle.block_summary(k, 64, w=w.double().numpy())
    err = np.abs(got.cpu().double().numpy()[:, :, :T // 64] - ref)
    assert err.max() <= 2e-5 * max(1.0, np.abs(ref).max()), err.max()
    # the pooling is not the mean for this head
    assert np.abs(ref - oracle.block_summary(k, 64)).max() > 1e-2


def test_zero_head_equals_mean_summary():
    _, (_, k, _) = inputs.make("16k", B=1, Hq=2, Hkv=2, T=512, d=128, n_topics=8, seed=3)
    kd = k.cuda()
    a = da.dash_block_summary_w(kd, torch.zeros(2, 128, device="cuda"))
    b = da.dash_block_summary(kd)
    torch.cuda.synchronize()
    assert (a - b).abs().max().item() <= 1e-6


def test_prefill_w_null_head_is_prefill():
    _, (q, k, v) = inputs.make("16k", B=1, Hq=8, Hkv=1, T=768, d=128, n_topics=8, seed=4)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    a, _ = da.dash_prefill(qd, kd, vd, alpha=1.5, coarse_scale=0.05)
    b, _ = da.dash_prefill_w(qd, kd, vd, None, alpha=1.5, coarse_scale=0.05)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("B,Hq,Hkv,T,d,cs", [(1, 8, 1, 2048, 128, 0.05), (2, 8, 2, 1100, 64, 0.2),
                                              (1, 16, 4, 4096, 128, 0.04)])
def test_prefill_w_vs_oracle(B, Hq, Hkv, T, d, cs):
    _, (q, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, n_topics=16, seed=40 + T)
    w = _head(Hkv, d, 1.0, 11)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out, ws = da.dash_prefill_w(qd, kd, vd, w.cuda(), alpha=1.5, coarse_scale=cs)
    torch.cuda.synchronize()
    assert da.dash_get_device_status(ws) == 0
    rows = stratified_rows(B, Hq, T, 1500, seed=5)
    qr = oracle.gather_q_rows(q, rows)
    ref, tau_ref, nsel = oracle.forward_rows(qr, k, v, rows, Hq, 64, 1.5, cs, w_summary=w.double().numpy())
    mx, mean = compare_out(rows_of(out.float().cpu(), rows).numpy(), ref, f"prefill_w B{B} Hq{Hq} T{T}")
    # thresholds: the learned summaries carry fp32 rounding on top of the hi/lo split
    tau = rows_of(da.dash_prefill_tau(ws, B, Hq, Hkv, T, d).cpu(), rows).numpy()
    past = np.array([t >= 64 for _, _, t in rows])
    kbar = np.abs(oracle.block_summary(k, 64, w=w.double().numpy()))
    qa = np.abs(qr.double().numpy())
    G = Hq // Hkv
    bound = np.array([(qa[i] @ kbar[b, h // G, :max(t // 64, 1)].T).max() if t >= 64 else 0.0
                      for i, (b, h, t) in enumerate(rows)])
    allow = 2.0 ** -14 * 0.5 * cs * bound / np.sqrt(d)
    dt = np.abs(tau - tau_ref)[past]
    assert np.all(dt <= (1e-4 * np.maximum(1.0, np.abs(tau_ref)) + allow)[past])
    # the head matters: with the mean summary the thresholds differ
    _, tau_mean, _ = oracle.forward_rows(qr, k, v, rows, Hq, 64, 1.5, cs)
    assert np.abs(tau_mean - tau_ref)[past].max() > 1e-3
    print("prefill_w", mx, mean, "selected/row", nsel.mean())


def test_decode_with_learned_summaries():
    B, Hq, Hkv, Tmax, d = 2, 8, 2, 5000, 128
    _, (q, kc, vc, _) = inputs.make("decode96k", B=B, Hq=Hq, Hkv=Hkv, T=Tmax, d=d, seed=12)
    lens = [5000, 2113]
    w = _head(Hkv, d, 1.0, 13)
    kcd, vcd = kc.cuda(), vc.cuda()
    ksum = da.dash_block_summary_w(kcd, w.cuda())
    out, ws = da.dash_decode(q.cuda(), kcd, vcd, ksum, torch.tensor(lens, dtype=torch.int32, device="cuda"),
                             alpha=1.5, coarse_scale=0.03)
    torch.cuda.synchronize()
    assert da.dash_get_device_status(ws) == 0
    rows = [(b, h, lens[b] - 1) for b in range(B) for h in range(Hq)]
    qr = torch.stack([q[b, h] for b, h, _ in rows])
    ref, _, _ = oracle.forward_rows(qr, kc, vc, rows, Hq, 64, 1.5, 0.03, w_summary=w.double().numpy())
    got = torch.stack([out[b, h].float().cpu() for b, h, _ in rows]).numpy()
    print("decode learned", compare_out(got, ref, "decode learned head"))


def test_prefill_w_unsupported_on_the_wide_group_path():
    # 32 query heads per KV head: tiles of 4 positions use the CUDA-core path
    _, (q, k, v) = inputs.make("16k", B=1, Hq=32, Hkv=1, T=256, d=64, n_topics=4, seed=2)
    with pytest.raises(da.DashError) as e:
        da.dash_prefill_w(q.cuda(), k.cuda(), v.cuda(), torch.zeros(1, 64, device="cuda"))
    assert e.value.code == -4
