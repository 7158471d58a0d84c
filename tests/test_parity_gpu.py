"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same seeded
inputs.  Small shapes compare every row; the full workload shapes compare >= 2048 sampled
rows (rows are independent, so sampling is exact)."""
import numpy as np
import pytest
import torch

from sparse_hierarchical_attention_pool_b200 import dash_attn as da
from sparse_hierarchical_attention_pool_b200 import inputs

pytestmark = pytest.mark.gpu

import oracle  # noqa: E402

from gpu_helpers import (all_rows, calibrated_scale, check_decode, check_dump, check_prefill,  # noqa: E402
                         compare_out, gpu_prefill, rows_of, stratified_rows)


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_hierarchical_attention_pool_b200 import build
    build.build()
    oracle.build()


# ------------------------------------------------------------------ block summaries

@pytest.mark.parametrize("d,T", [(64, 512), (128, 1000), (128, 63)])
def test_block_summary_vs_oracle(d, T):
    _, (q, k, v) = inputs.make("16k", T=T, d=d, Hq=4, Hkv=2, B=2)
    if T < 64:
        # no complete block: nothing is written (a NaN-filled buffer stays NaN)
        ks = torch.full((2, 2, 1, d), float("nan"), device="cuda")
        da.dash_block_summary(k.cuda(), ks)
        torch.cuda.synchronize()
        assert ks.isnan().all()
        assert oracle.block_summary(k, 64).shape[2] == 0
        return
    ks = da.dash_block_summary(k.cuda()).cpu().double().numpy()
    ref = oracle.block_summary(k, 64)
    assert ks.shape == ref.shape
    assert np.abs(ks - ref).max() <= 1e-6 * max(1.0, np.abs(ref).max())


# ------------------------------------------------------------------ tiny config, every row

def test_tiny_config_all_rows():
    wl, (q, k, v) = inputs.make("tiny")
    res, _, _ = check_prefill(q, k, v, wl.alpha, calibrated_scale("tiny"), all_rows(1, 1, wl.T), "tiny")
    print(res)


@pytest.mark.parametrize("cs", [0.0, 8.0, 32.0, 1e4])
def test_tiny_scales(cs):
    wl, (q, k, v) = inputs.make("tiny")
    # at cs = 1e4 the scores' bf16 hi + lo rounding (A) exceeds 1e-4: band widened by 2 A
    res, _, _ = check_prefill(q, k, v, 1.5, cs, all_rows(1, 1, wl.T), f"tiny cs={cs}", strict_band=cs < 1e3)
    print(cs, res)


@pytest.mark.parametrize("alpha", [1.25, 2.0, 3.0])
def test_tiny_alphas(alpha):
    wl, (q, k, v) = inputs.make("tiny")
    check_prefill(q, k, v, alpha, 8.0, all_rows(1, 1, wl.T), f"tiny alpha={alpha}")


def test_zero_scale_is_uniform_weights():
    wl, (q, k, v) = inputs.make("tiny")
    rows = [(0, 0, t) for t in (64, 200, 511)]
    ksum = da.dash_block_summary(k.cuda())
    idx, p, cnt, tau = da.dash_select_dump(q.cuda(), ksum, rows, 8, 1.5, 0.0, 1)
    for r, (_, _, t) in enumerate(rows):
        bt = t // 64
        assert int(cnt[r]) == bt
        assert torch.allclose(p[r, :bt].cpu(), torch.full((bt,), 1.0 / bt), atol=1e-6)


# ------------------------------------------------------------------ shapes: GQA, ragged, tiny T

@pytest.mark.parametrize("B,Hq,Hkv,T,d,cs", [
    (2, 8, 2, 700, 128, 0.05),    # G = 4, ragged tail
    (1, 16, 2, 1000, 128, 0.05),  # G = 8 (the 16K workload's grouping)
    (1, 6, 2, 333, 64, 0.08),     # G = 3: 32 positions x 3 heads per tile
    (2, 2, 2, 200, 64, 0.1),      # G = 1
    (1, 4, 1, 129, 128, 0.05),    # G = 4, one past block + 1 token
])
def test_shapes_all_rows(B, Hq, Hkv, T, d, cs):
    _, (q, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, n_topics=16, seed=77 + T)
    res, _, _ = check_prefill(q, k, v, 1.5, cs, all_rows(B, Hq, T), f"{(B, Hq, Hkv, T, d)}")
    print(res)


@pytest.mark.parametrize("T", [1, 17, 64, 65, 128])
def test_short_sequences_are_dense_causal(T):
    """At most one past block: weight 1, output = plain causal attention (T <= 2 blocks)."""
    _, (q, k, v) = inputs.make("16k", B=1, Hq=4, Hkv=2, T=T, d=64, n_topics=8, seed=5 + T)
    rows = all_rows(1, 4, T)
    _, _, _, out, _ = gpu_prefill(q, k, v, 1.5, 0.3)
    dense = oracle.dense_causal_rows(oracle.gather_q_rows(q, rows), k, v, rows, 4)
    compare_out(rows_of(out.float().cpu(), rows).numpy(), dense, f"T={T}")


def test_non_dispersive_insertion_on_gpu():
    """Blocks whose keys point away from every query get weight 0; inserting them leaves
    the outputs of later queries unchanged (within bf16 tolerance)."""
    d, T = 64, 384
    g = torch.Generator().manual_seed(3)
    u = torch.randn(d, generator=g)
    u /= u.norm()
    q = (8 * u + 0.3 * torch.randn(1, 1, T, d, generator=g)).bfloat16()
    k = (8 * u + 0.3 * torch.randn(1, 1, T, d, generator=g)).bfloat16()
    v = torch.randn(1, 1, T, d, generator=g).bfloat16()
    bad_k = (-8 * u + 0.3 * torch.randn(1, 1, 128, d, generator=g)).bfloat16()
    bad_v = torch.randn(1, 1, 128, d, generator=g).bfloat16()
    cut = 128
    k2 = torch.cat([k[:, :, :cut], bad_k, k[:, :, cut:]], 2)
    v2 = torch.cat([v[:, :, :cut], bad_v, v[:, :, cut:]], 2)
    q2 = torch.cat([q[:, :, :cut], q[:, :, :128], q[:, :, cut:]], 2)
    _, _, _, o1, _ = gpu_prefill(q, k, v, 1.5, 1.0)
    _, _, _, o2, _ = gpu_prefill(q2, k2, v2, 1.5, 1.0)
    diff = (o1[:, :, cut:].float() - o2[:, :, cut + 128:].float()).abs().max().item()
    assert diff <= 2e-2, diff


def test_host_entry_point_matches_device_path():
    wl, (q, k, v) = inputs.make("16k", T=1024, Hq=8, Hkv=2)
    cs = 0.05
    qd, kd, vd, out, ws = gpu_prefill(q, k, v, 1.5, cs)
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty_like(q).pin_memory()
    da.dash_prefill_host(qh, kh, vh, oh, torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd),
                         torch.empty_like(out), 1.5, cs, ws)
    torch.cuda.synchronize()
    assert torch.equal(oh, out.cpu())


def test_host_entry_point_head_chunks():
    # 4 MiB of queries per head: the host entry point cuts each KV group (4 heads) into chunks
    # of 2 heads, each its own prefill on the group's keys and values; the units run on
    # several compute streams at once
    wl, (q, k, v) = inputs.make("16k", Hq=8, Hkv=2)
    cs = calibrated_scale("16k")
    qd, kd, vd, out, ws = gpu_prefill(q, k, v, 1.5, cs)
    st_dev = da.dash_prefill_stats(ws)
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty_like(q).pin_memory()
    da.dash_prefill_host(qh, kh, vh, oh, torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd),
                         torch.empty_like(out), 1.5, cs, ws)
    torch.cuda.synchronize()
    # the units run on several streams with their own workspace slices; the call's header
    # holds the OR of their status bits and the sums of their statistics
    assert da.dash_get_device_status(ws) == 0
    st = da.dash_prefill_stats(ws)
    assert st["scored_pairs"] == st_dev["scored_pairs"]
    assert st["selected_pairs"] == st_dev["selected_pairs"]
    compare_out(oh.float().numpy(), out.float().cpu().numpy(), "host chunks against the device path")
    rows = stratified_rows(1, 8, wl.T, 512, seed=17)
    ref, _, _ = oracle.forward_rows(oracle.gather_q_rows(q, rows), k, v, rows, 8, 64, 1.5, cs)
    compare_out(rows_of(oh, rows).float().numpy(), ref, "host chunks against the oracle")


@pytest.mark.parametrize("tiles", ["ordered", "positions"])
def test_streamed_tiles_both_tilings(tiles, monkeypatch):
    # T = 40960: tiles past position 32768 have more than 512 past blocks, so their scores are
    # recomputed for every threshold pass (the streamed instantiation of the coarse kernel,
    # four threads per row), with row bitmaps (ordered tiles) or tile lists (position tiles)
    if tiles == "positions":
        monkeypatch.setenv("DASH_TILES", "positions")
    T = 40960
    _, (q, k, v) = inputs.make("16k", T=T, Hq=4, Hkv=1, n_topics=32, seed=77)
    rows = stratified_rows(1, 4, T, 384, seed=5)
    assert sum(t > 32768 for _, _, t in rows) >= 50
    check_prefill(q, k, v, 1.5, calibrated_scale("16k"), rows, f"T={T}, {tiles} tiles")


def test_stats_count_selected_pairs():
    B, Hq, Hkv, T, d = 1, 8, 2, 1000, 128
    _, (q, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, n_topics=16, seed=91)
    _, _, _, _, ws = gpu_prefill(q, k, v, 1.5, 0.05)
    st = da.dash_prefill_stats(ws)
    rows = [r for r in all_rows(B, Hq, T) if r[2] >= 64]
    sel = oracle.select_rows(oracle.gather_q_rows(q, rows), k, rows, Hq, 64, 1.5, 0.05)
    assert st["scored_pairs"] == int(sel["bt"].sum())
    near = int(sum((np.abs(sel["x"][r, :sel["bt"][r]] - sel["tau"][r]) < 1e-4).sum() for r in range(len(rows))))
    assert abs(st["selected_pairs"] - int(sel["nsel"].sum())) <= near
    assert st["status"] == 0 and st["tiles"] > 0
    assert st["union_blocks"] <= st["tiles"] * ((T + 63) // 64)
    assert st["fine_steps"] >= st["union_blocks"]


# ------------------------------------------------------------------ the workloads at full size

@pytest.mark.parametrize("name", ["16k", "96k", "16k-coherent"])
def test_workload_sampled_rows(name):
    wl, (q, k, v) = inputs.make(name)
    cs = calibrated_scale(name)
    rows = stratified_rows(wl.B, wl.Hq, wl.T, 2048 - 17 * wl.Hq, seed=wl.seed + 7)
    res, _, ws = check_prefill(q, k, v, wl.alpha, cs, rows, name)
    st = da.dash_prefill_stats(ws)
    print(name, res, st, "sparsity", 1 - st["selected_pairs"] / st["scored_pairs"])


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_32k_alpha_sweep_sampled_rows(alpha):
    wl, (q, k, v) = inputs.make("32k")
    rows = stratified_rows(wl.B, wl.Hq, wl.T, 2048 - 17 * wl.Hq, seed=wl.seed + int(alpha * 100))
    res, _, _ = check_prefill(q, k, v, alpha, calibrated_scale("32k"), rows, f"32k alpha={alpha}")
    print(alpha, res)


# ------------------------------------------------------------------ decode

def test_decode_small_ragged_lengths():
    B, Hq, Hkv, Tmax, d = 4, 8, 2, 700, 128
    _, (q4, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=Tmax, d=d, n_topics=16, seed=123)
    lens = [700, 333, 64, 1]
    q = torch.stack([q4[b, :, lens[b] - 1] for b in range(B)])
    res, _, _ = check_decode(q, k, v, lens, 1.5, 0.05, "decode small")
    assert res[1] is not None
    print(res)


def test_decode_equals_last_prefill_row():
    B, Hq, Hkv, T, d = 1, 8, 2, 900, 128
    _, (q, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, n_topics=16, seed=9)
    _, _, _, out, _ = gpu_prefill(q, k, v, 1.5, 0.05)
    Tmax = 1024
    kc = torch.zeros(B, Hkv, Tmax, d, dtype=torch.bfloat16)
    vc = torch.zeros(B, Hkv, Tmax, d, dtype=torch.bfloat16)
    kc[:, :, :T], vc[:, :, :T] = k, v
    ksum = da.dash_block_summary(kc.cuda())
    dec, _ = da.dash_decode(q[:, :, T - 1].contiguous().cuda(), kc.cuda(), vc.cuda(), ksum,
                            torch.tensor([T], dtype=torch.int32, device="cuda"), alpha=1.5, coarse_scale=0.05)
    torch.cuda.synchronize()
    diff = (dec.float() - out[:, :, T - 1].float()).abs().max().item()
    assert diff <= 2e-2


def test_decode_invalid_lengths_write_zeros():
    B, Hq, Hkv, Tmax, d = 2, 4, 1, 256, 64
    _, (q4, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=Tmax, d=d, n_topics=4, seed=2)
    q = q4[:, :, -1].contiguous().cuda()
    ksum = da.dash_block_summary(k.cuda())
    out, ws = da.dash_decode(q, k.cuda(), v.cuda(), ksum, torch.tensor([0, Tmax + 5], dtype=torch.int32, device="cuda"),
                             alpha=1.5, coarse_scale=0.1)
    torch.cuda.synchronize()
    assert torch.all(out == 0)
    assert da.dash_get_device_status(ws) == 0


@pytest.mark.parametrize("B,Hq,Hkv,Tmax,d,lens", [
    (2, 2, 2, 400000, 64, [400000, 123457]),   # G = 1: a row longer than the select registers
    (2, 4, 2, 20000, 128, [20000, 4097]),      # G = 2
    (2, 16, 2, 70000, 128, [70000, 65]),       # G = 8, one warp per head, row spills to memory
    (1, 16, 1, 5000, 64, [5000]),              # G = 16: CUDA-core attention path
    (3, 8, 8, 3000, 128, [3000, 64, 129]),     # G = 1, short and block-boundary lengths
])
def test_decode_group_sizes(B, Hq, Hkv, Tmax, d, lens):
    _, (q, kc, vc, _) = inputs.make("decode96k", B=B, Hq=Hq, Hkv=Hkv, T=Tmax, d=d, seed=77 + Hq)
    res, _, ws = check_decode(q, kc, vc, lens, 1.5, calibrated_scale("decode96k"),
                              f"decode G={Hq // Hkv} d={d}")
    print("decode groups", Hq // Hkv, d, res)


def test_decode_96k_workload_all_rows():
    wl, (q, kc, vc, kv_len) = inputs.make("decode96k")
    res, _, ws = check_decode(q, kc, vc, kv_len.tolist(), wl.alpha, calibrated_scale("decode96k"), "decode96k")
    assert res[1] is not None and res[1]["selected"] > 0
    st = da.dash_decode_stats(ws)
    print("decode96k", res, st, "sparsity", 1 - st["selected_pairs"] / st["scored_pairs"])


def test_decode_threshold_start_does_not_change_the_result():
    """The histogram start and the start at u = -1 reach the same thresholds and lists."""
    import os
    wl, (q, kc, vc, kv_len) = inputs.make("decode96k", B=2)
    cs = calibrated_scale("decode96k")
    qd, kcd, vcd, lens = q.cuda(), kc.cuda(), vc.cuda(), kv_len.cuda()
    ksum = da.dash_block_summary(kcd)
    outs, stats = [], []
    for mode in ("newton", "histogram"):
        if mode == "histogram":
            os.environ["DASH_ENTMAX_INIT"] = "histogram"
        try:
            out, ws = da.dash_decode(qd, kcd, vcd, ksum, lens, alpha=wl.alpha, coarse_scale=cs)
            torch.cuda.synchronize()
            assert da.dash_get_device_status(ws) == 0
            outs.append(out.float().cpu())
            stats.append(da.dash_decode_stats(ws))
        finally:
            os.environ.pop("DASH_ENTMAX_INIT", None)
    assert stats[0]["selected_pairs"] == stats[1]["selected_pairs"]
    assert stats[0]["union_blocks"] == stats[1]["union_blocks"]
    assert (outs[0] - outs[1]).abs().max().item() <= 2e-3
