"""GPU: the block sets and weights the product kernels actually apply, against the oracle,
for the variants the main parity file does not cover (learned summary head, head
aggregation), and the device status path of the threshold solve.

The selection of a prefill is read from the fine stage's own dump variant
(dash_prefill_dump), that of a decode step from the attention kernel (dash_decode_dump):
the same calls that produce the outputs.  Criteria ("DashAttention: Making Sparse Attention
Fully Differentiable with Adaptive Block Selection", Core Mechanism: Stage 1's sparse block
weights are Stage 2's log prior): sets identical outside the 1e-4 band, weights within 1e-4.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_hierarchical_attention_pool_b200 import dash_attn as da
from sparse_hierarchical_attention_pool_b200 import inputs

from gpu_helpers import (calibrated_scale, compare_out, compare_selection, rows_of, score_allowance,  # noqa: E402
                         stratified_rows)

pytestmark = pytest.mark.gpu
AGG = da.HEAD_AGGREGATION
NO_CONVERGE = -7


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_hierarchical_attention_pool_b200 import build
    build.build()
    oracle.build()


def _head(Hkv, d, scale, seed):
    return (torch.randn(Hkv, d, generator=torch.Generator().manual_seed(seed)) * scale).float()


@pytest.mark.parametrize("B,Hq,Hkv,T,d,cs", [(1, 8, 1, 2048, 128, 0.05), (1, 16, 4, 4096, 128, 0.04)])
def test_prefill_learned_head_selection(B, Hq, Hkv, T, d, cs):
    """Learned summary head: the applied weights match the oracle's selection with that head."""
    _, (q, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, n_topics=16, seed=40 + T)
    w = _head(Hkv, d, 1.0, 11)
    rows = stratified_rows(B, Hq, T, 1500, seed=5)
    out, ws, xg, pg = da.dash_prefill_dump(q.cuda(), k.cuda(), v.cuda(), rows, alpha=1.5, coarse_scale=cs,
                                           w_summary=w.cuda())
    torch.cuda.synchronize()
    assert da.dash_get_device_status(ws) == 0
    qr = oracle.gather_q_rows(q, rows)
    wn = w.double().numpy()
    ref, _, _ = oracle.forward_rows(qr, k, v, rows, Hq, 64, 1.5, cs, w_summary=wn)
    compare_out(rows_of(out.float().cpu(), rows).numpy(), ref, "learned head dump")
    sel = oracle.select_rows(qr, k, rows, Hq, 64, 1.5, cs, w_summary=wn)
    # the learned summaries carry fp32 rounding of the softmax pooling on top of the hi/lo
    # split: four times the mean summary's allowance
    allow = 4.0 * score_allowance(qr, k, rows, Hq, 1.5, cs, kbar=oracle.block_summary(k, 64, w=wn))
    res = compare_selection(xg.cpu().numpy(), pg.cpu().numpy(), sel, rows, allow, "learned head")
    assert res["selected"] > 0
    print("learned head selection", res)


@pytest.mark.parametrize("name_or_shape", ["16k", (2, 8, 2, 1100, 64, 0.2)])
def test_prefill_head_aggregation_selection(name_or_shape):
    """Head aggregation: each head's own weights (before the group average) are the oracle's."""
    if name_or_shape == "16k":
        wl, (q, k, v) = inputs.make("16k")
        cs = calibrated_scale("16k")
        B, Hq, Hkv, T = wl.B, wl.Hq, wl.Hkv, wl.T
        rows = stratified_rows(B, Hq, T, 1200, seed=9)
    else:
        B, Hq, Hkv, T, d, cs = name_or_shape
        _, (q, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, n_topics=16, seed=60 + T)
        rows = stratified_rows(B, Hq, T, 1500, seed=8)
    out, ws, xg, pg = da.dash_prefill_dump(q.cuda(), k.cuda(), v.cuda(), rows, alpha=1.5, coarse_scale=cs,
                                           flags=AGG)
    torch.cuda.synchronize()
    assert da.dash_get_device_status(ws) == 0
    ref, _ = oracle.forward_rows_agg(q, k, v, rows, 64, 1.5, cs)
    compare_out(rows_of(out.float().cpu(), rows).numpy(), ref, "aggregation dump")
    qr = oracle.gather_q_rows(q, rows)
    sel = oracle.select_rows(qr, k, rows, Hq, 64, 1.5, cs)
    res = compare_selection(xg.cpu().numpy(), pg.cpu().numpy(), sel, rows,
                            score_allowance(qr, k, rows, Hq, 1.5, cs), "aggregation")
    print("aggregation selection", res)


def test_decode_head_aggregation_selection():
    wl, (q, kc, vc, _) = inputs.make("decode96k", B=2)
    cs = calibrated_scale("decode96k")
    lens = [98304, 40001]
    kcd, vcd = kc.cuda(), vc.cuda()
    ksum = da.dash_block_summary(kcd)
    out, ws, xg, pg, tg = da.dash_decode_dump(q.cuda(), kcd, vcd, ksum, torch.tensor(lens, dtype=torch.int32,
                                                                                     device="cuda"),
                                              alpha=wl.alpha, coarse_scale=cs, flags=AGG)
    torch.cuda.synchronize()
    assert da.dash_get_device_status(ws) == 0
    rows = [(b, h, lens[b] - 1) for b in range(2) for h in range(wl.Hq)]
    qr = torch.stack([q[b, h] for b, h, _ in rows])
    sel = oracle.select_rows(qr, kc, rows, wl.Hq, 64, wl.alpha, cs)
    xg, pg = xg.cpu().numpy(), pg.cpu().numpy()
    res = compare_selection(np.stack([xg[b, h] for b, h, _ in rows]), np.stack([pg[b, h] for b, h, _ in rows]),
                            sel, rows, score_allowance(qr, kc, rows, wl.Hq, wl.alpha, cs), "decode aggregation")
    print("decode aggregation selection", res)


def test_prefill_dump_leaves_outputs_unchanged():
    """The dump variant computes the same outputs and thresholds as dash_prefill."""
    _, (q, k, v) = inputs.make("16k", B=1, Hq=8, Hkv=2, T=1500, d=128, n_topics=16, seed=17)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    a, wa = da.dash_prefill(qd, kd, vd, alpha=1.5, coarse_scale=0.05)
    b, wb, _, _ = da.dash_prefill_dump(qd, kd, vd, [(0, 3, 1400), (0, 0, 70)], alpha=1.5, coarse_scale=0.05)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    ta = da.dash_prefill_tau(wa, 1, 8, 2, 1500, 128)
    tb = da.dash_prefill_tau(wb, 1, 8, 2, 1500, 128)
    assert torch.equal(ta.nan_to_num(), tb.nan_to_num())


def test_dump_unsupported_on_wide_groups():
    """More than 16 query heads per KV head (CUDA-core fine kernel): no dump variant."""
    _, (q, k, v) = inputs.make("16k", B=1, Hq=32, Hkv=1, T=256, d=64, n_topics=4, seed=3)
    with pytest.raises(da.DashError) as e:
        da.dash_prefill_dump(q.cuda(), k.cuda(), v.cuda(), [(0, 0, 100)], alpha=1.5, coarse_scale=0.1)
    assert e.value.code == -4


# ------------------------------------------------------------------ device status of the solve

@pytest.fixture
def solve_cap(monkeypatch):
    """Lower the threshold solve's iteration cap for the calls of one test (read per call)."""
    def set_cap(n):
        monkeypatch.setenv("DASH_DEBUG_SOLVE_CAP", str(n))
    yield set_cap
    monkeypatch.delenv("DASH_DEBUG_SOLVE_CAP", raising=False)


# alpha = 1.25 takes the general Newton iteration (no closed-form finish), whose first pass
# never ends the solve: a cap of one iteration stops every row that has past blocks.

@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (32, 1)])   # tensor-core and CUDA-core coarse kernels
def test_capped_solve_reports_no_converge_prefill(solve_cap, Hq, Hkv):
    wl, (q, k, v) = inputs.make("16k", B=1, Hq=Hq, Hkv=Hkv, T=1024, d=64, n_topics=8, seed=21)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    solve_cap(1)
    _, ws = da.dash_prefill(qd, kd, vd, alpha=1.25, coarse_scale=0.5)
    assert da.dash_get_device_status(ws) == NO_CONVERGE
    assert da.dash_prefill_stats(ws)["status"] & 1
    # the same call with the normal cap is clean: the status comes from the cap alone
    solve_cap(64)
    _, ws = da.dash_prefill(qd, kd, vd, alpha=1.25, coarse_scale=0.5)
    assert da.dash_get_device_status(ws) == 0


def test_capped_solve_reports_no_converge_tiny_config(solve_cap):
    """The tiny configuration, prefill and a decode step over its keys (query at the last
    position): a cap of 1 or 2 iterations is reported, the normal cap is clean."""
    wl, (q, k, v) = inputs.make("tiny")
    cs = calibrated_scale("tiny")
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ksum = da.dash_block_summary(kd)
    lens = torch.tensor([wl.T], dtype=torch.int32, device="cuda")
    qlast = q[:, :, wl.T - 1].contiguous().cuda()
    for cap, want in ((1, NO_CONVERGE), (2, NO_CONVERGE), (64, 0)):
        solve_cap(cap)
        _, ws = da.dash_prefill(qd, kd, vd, alpha=1.25, coarse_scale=cs)
        assert da.dash_get_device_status(ws) == want, f"prefill, cap {cap}"
        _, wsd = da.dash_decode(qlast, kd, vd, ksum, lens, alpha=1.25, coarse_scale=cs)
        assert da.dash_get_device_status(wsd) == want, f"decode, cap {cap}"


def test_capped_solve_reports_no_converge_decode(solve_cap):
    wl, (q, kc, vc, _) = inputs.make("decode96k", B=2, T=8192)
    cs = calibrated_scale("decode96k")
    kcd = kc.cuda()
    ksum = da.dash_block_summary(kcd)
    lens = torch.tensor([8192, 5000], dtype=torch.int32, device="cuda")
    solve_cap(1)
    _, ws = da.dash_decode(q.cuda(), kcd, vc.cuda(), ksum, lens, alpha=1.25, coarse_scale=cs)
    assert da.dash_get_device_status(ws) == NO_CONVERGE
    solve_cap(64)
    _, ws = da.dash_decode(q.cuda(), kcd, vc.cuda(), ksum, lens, alpha=1.25, coarse_scale=cs)
    assert da.dash_get_device_status(ws) == 0


# ------------------------------------------------------------------ histogram-started threshold (F4)

@pytest.fixture
def histogram_start(monkeypatch):
    monkeypatch.setenv("DASH_ENTMAX_INIT", "histogram")
    yield
    monkeypatch.delenv("DASH_ENTMAX_INIT", raising=False)


@pytest.mark.parametrize("name", ["tiny", "ragged", "16k", "96k"])
def test_histogram_start_prefill_vs_oracle(histogram_start, name):
    """The AdaSplash-2 style start (a histogram edge below the root) reaches the oracle's
    thresholds, block sets and weights: register-resident rows (tiny, ragged, 16K) and the
    streamed rows of the 96K workload (more than 512 past blocks)."""
    from gpu_helpers import all_rows, check_prefill
    if name == "tiny":
        wl, (q, k, v) = inputs.make("tiny")
        res, _, _ = check_prefill(q, k, v, 1.5, calibrated_scale("tiny"), all_rows(1, 1, wl.T), "hist tiny")
    elif name == "ragged":
        _, (q, k, v) = inputs.make("16k", B=2, Hq=8, Hkv=2, T=700, d=128, n_topics=16, seed=777)
        res, _, _ = check_prefill(q, k, v, 2.0, 0.1, all_rows(2, 8, 700), "hist ragged alpha=2")
    else:
        wl, (q, k, v) = inputs.make(name)
        rows = stratified_rows(wl.B, wl.Hq, wl.T, 2048 - 17 * wl.Hq, seed=wl.seed + 11)
        res, _, _ = check_prefill(q, k, v, wl.alpha, calibrated_scale(name), rows, f"hist {name}")
    assert res["sel"]["selected"] > 0
    print(name, res)


def test_histogram_start_decode_vs_oracle(histogram_start):
    from gpu_helpers import check_decode
    wl, (q, kc, vc, kv_len) = inputs.make("decode96k")
    res, _, _ = check_decode(q, kc, vc, kv_len.tolist(), wl.alpha, calibrated_scale("decode96k"), "hist decode96k")
    assert res[1] is not None and res[1]["selected"] > 0
    print(res)
