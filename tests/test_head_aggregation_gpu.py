"""GPU parity of head-aggregated selection (entmax head aggregation, "DashAttention and the
year sparse attention became a field", section "Non-dispersive attention at long context"):
the heads of a KV group share the mean of their block weights as prior.  Through the C ABI,
against the fp64 oracle."""
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
from gpu_helpers import calibrated_scale, compare_out, rows_of, stratified_rows  # noqa: E402

pytestmark = pytest.mark.gpu
AGG = da.HEAD_AGGREGATION


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    oracle.build()


@pytest.mark.parametrize("B,Hq,Hkv,T,d,cs", [(1, 8, 1, 2048, 128, 0.05), (2, 8, 2, 1100, 64, 0.2),
                                              (1, 16, 2, 16384, 128, None), (1, 4, 4, 640, 128, 0.1)])
def test_prefill_head_aggregation_vs_oracle(B, Hq, Hkv, T, d, cs):
    if cs is None:
        _, (q, k, v) = inputs.make("16k")
        cs = calibrated_scale("16k")
        rows = stratified_rows(B, Hq, T, 1200, seed=9)
    else:
        _, (q, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, n_topics=16, seed=60 + T)
        rows = stratified_rows(B, Hq, T, 1500, seed=8)
    out, ws = da.dash_prefill_ex(q.cuda(), k.cuda(), v.cuda(), flags=AGG, alpha=1.5, coarse_scale=cs)
    torch.cuda.synchronize()
    assert da.dash_get_device_status(ws) == 0
    ref, nsel = oracle.forward_rows_agg(q, k, v, rows, 64, 1.5, cs)
    mx, mean = compare_out(rows_of(out.float().cpu(), rows).numpy(), ref, f"prefill agg Hq{Hq} Hkv{Hkv} T{T}")
    if Hq > Hkv:
        # aggregation changes the result (the per-head forward is a different function)
        per_head, _, _ = oracle.forward_rows(oracle.gather_q_rows(q, rows), k, v, rows, Hq, 64, 1.5, cs)
        assert np.abs(per_head - ref).max() > 1e-3
    print("prefill agg", mx, mean, "shared support", nsel.mean())


def test_prefill_flags_zero_is_prefill():
    _, (q, k, v) = inputs.make("16k", B=1, Hq=8, Hkv=1, T=700, d=128, n_topics=8, seed=4)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    a, _ = da.dash_prefill(qd, kd, vd, alpha=1.5, coarse_scale=0.05)
    b, _ = da.dash_prefill_ex(qd, kd, vd, flags=0, alpha=1.5, coarse_scale=0.05)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_prefill_aggregation_with_learned_head():
    _, (q, k, v) = inputs.make("16k", B=1, Hq=8, Hkv=2, T=1500, d=128, n_topics=16, seed=5)
    w = (torch.randn(2, 128, generator=torch.Generator().manual_seed(3)) * 0.8).float()
    out, ws = da.dash_prefill_ex(q.cuda(), k.cuda(), v.cuda(), w_summary=w.cuda(), flags=AGG,
                                 alpha=1.5, coarse_scale=0.06)
    torch.cuda.synchronize()
    rows = stratified_rows(1, 8, 1500, 800, seed=6)
    ref, _ = oracle.forward_rows_agg(q, k, v, rows, 64, 1.5, 0.06, w_summary=w.double().numpy())
    compare_out(rows_of(out.float().cpu(), rows).numpy(), ref, "prefill agg learned head")


def test_decode_head_aggregation_vs_oracle():
    wl, (q, kc, vc, kv_len) = inputs.make("decode96k", B=2)
    cs = calibrated_scale("decode96k")
    lens = [98304, 40001]
    kcd, vcd = kc.cuda(), vc.cuda()
    ksum = da.dash_block_summary(kcd)
    out, ws = da.dash_decode_ex(q.cuda(), kcd, vcd, ksum, torch.tensor(lens, dtype=torch.int32, device="cuda"),
                                flags=AGG, alpha=wl.alpha, coarse_scale=cs)
    torch.cuda.synchronize()
    assert da.dash_get_device_status(ws) == 0
    rows = [(b, h, lens[b] - 1) for b in range(2) for h in range(wl.Hq)]
    q4 = q.unsqueeze(2).expand(2, wl.Hq, wl.T, wl.d)     # row (b, h, t) reads q[b, h]
    ref, _ = oracle.forward_rows_agg(q4, kc, vc, rows, 64, wl.alpha, cs)
    got = torch.stack([out[b, h].float().cpu() for b, h, _ in rows]).numpy()
    print("decode agg", compare_out(got, ref, "decode head aggregation"))


def test_aggregation_unsupported_paths():
    _, (q, k, v) = inputs.make("16k", B=1, Hq=32, Hkv=1, T=256, d=64, n_topics=4, seed=2)
    with pytest.raises(da.DashError) as e:
        da.dash_prefill_ex(q.cuda(), k.cuda(), v.cuda(), flags=AGG)
    assert e.value.code == -4
    with pytest.raises(da.DashError) as e:
        da.dash_prefill_ex(q.cuda(), k.cuda(), v.cuda(), flags=2)
    assert e.value.code == -1
    _, (qd, kc, vc, _) = inputs.make("decode96k", B=1, Hq=16, Hkv=1, T=512, d=64)
    ksum = da.dash_block_summary(kc.cuda())
    with pytest.raises(da.DashError) as e:
        da.dash_decode_ex(qd.cuda(), kc.cuda(), vc.cuda(), ksum, torch.tensor([512], dtype=torch.int32, device="cuda"),
                          flags=AGG)
    assert e.value.code == -4
