"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI, run the fp64
oracle on the same seeded inputs, and compare with the tolerances of the specification.

Tolerances (bf16 inputs, fp32 accumulation):
  outputs        max-abs <= 2e-2 and mean-abs <= 2e-3 against the fp64 oracle;
  block weights  within 1e-4 absolute;
  block sets     identical except blocks whose (alpha-1) s_j - tau lies within 1e-4 of 0.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle
from sparse_hierarchical_attention_pool_b200 import dash_attn as da
from sparse_hierarchical_attention_pool_b200 import inputs

OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
P_ABS = 1e-4
BAND = 1e-4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "coarse_scale.json")


def calibrated_scale(name):
    with open(GOLDEN) as f:
        return json.load(f)[name]["coarse_scale"]


def all_rows(B, Hq, T):
    return [(b, h, t) for b in range(B) for h in range(Hq) for t in range(T)]


def stratified_rows(B, Hq, T, n_random, seed):
    fixed = sorted({0, 1, 63, 64, 65, 127, 128, 129, 1023, 1024, 4095, 4096, T // 2, T - 65, T - 64, T - 2, T - 1})
    return inputs.sample_rows(B, Hq, T, n_random, seed, t_fixed=fixed)


def gpu_prefill(q, k, v, alpha, cs):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out, ws = da.dash_prefill(qd, kd, vd, alpha=alpha, coarse_scale=cs)
    torch.cuda.synchronize()
    return qd, kd, vd, out, ws


def compare_out(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= OUT_MAX_ABS, f"{what}: max-abs {mx:.3e} > {OUT_MAX_ABS}"
    assert mean <= OUT_MEAN_ABS, f"{what}: mean-abs {mean:.3e} > {OUT_MEAN_ABS}"
    return mx, mean


def rows_of(t4, rows):
    r = torch.as_tensor(np.asarray(rows, dtype=np.int64))
    return t4[r[:, 0], r[:, 1], r[:, 2]]


def score_allowance(q_rows, k, rows, Hq, alpha, cs, kbar=None):
    """Per-row bound A on the error of the tensor-core scores x_j.

    The prefill's scores are products of q with kbar split into bf16 hi + lo parts (2^-17
    relative per element), so x_j, and with it tau, may move by up to
    A = 2^-16 (alpha-1) |cs| max_j sum_i |q_i kbar_ji| / sqrt(d)."""
    if kbar is None:
        kbar = oracle.block_summary(k, 64)                              # [B, Hkv, nbs, d]
    kbar = np.abs(kbar)
    qa = np.abs(q_rows.double().numpy())
    d = qa.shape[1]
    G = Hq // k.shape[1]
    bound = np.array([(qa[i] @ kbar[b, h // G, :max(t // 64, 1)].T).max() if t >= 64 else 0.0
                      for i, (b, h, t) in enumerate(rows)])
    return 2.0 ** -16 * (alpha - 1) * abs(cs) * bound / np.sqrt(d)


def compare_selection(x_gpu, p_gpu, sel, rows, allow, what="", strict_band=True):
    """The block sets and weights a kernel applied against the oracle's (the benchmark spec's criteria).

    x_gpu, p_gpu [n, >= bt]: per row, x_j of every block the kernel listed (NaN when not
    listed) and the weight it applied (0 when not selected or not listed).
      - sets {j : p_j > 0} identical except blocks with |x_ref_j - tau_ref| < 1e-4
        (strict_band) or < 1e-4 + 2 A (score-error allowance, for stress scales);
      - |p_gpu - p_ref| <= 1e-4 for every past block (stress scales: + 4 A, the bound of
        |dp| = e z^(e-1) |dz| for alpha <= 2, z = x - tau <= 1, |dz| <= 2 A);
      - every oracle-selected block outside the band is in the kernel's list;
      - listed x_j within A + 1e-6 max(1, |x|) of the oracle's (auxiliary)."""
    x_gpu = np.asarray(x_gpu, dtype=np.float64)
    p_gpu = np.asarray(p_gpu, dtype=np.float64)
    worst_p, worst_x, n_band, n_pairs, n_sel = 0.0, 0.0, 0, 0, 0
    for r, (b, h, t) in enumerate(rows):
        bt = t // 64
        assert np.all(np.isnan(x_gpu[r, bt:])) and np.all(p_gpu[r, bt:] == 0), \
            f"{what}: row {(b, h, t)} reports blocks at or after its own block"
        if bt == 0:
            continue
        xr, tr, pr = sel["x"][r, :bt], sel["tau"][r], sel["p"][r, :bt]
        band = BAND if strict_band else BAND + 2.0 * allow[r]
        near = np.abs(xr - tr) < band
        s_ref = xr > tr
        s_gpu = p_gpu[r, :bt] > 0
        diff = s_gpu != s_ref
        assert np.all(near[diff]), (f"{what}: row {(b, h, t)} blocks {np.nonzero(diff & ~near)[0][:8]} "
                                    "differ outside the band")
        listed = ~np.isnan(x_gpu[r, :bt])
        assert np.all(listed | ~s_ref | near), f"{what}: row {(b, h, t)}: a selected block is missing from its list"
        n_band += int(diff.sum())
        n_pairs += bt
        n_sel += int(s_ref.sum())
        ptol = P_ABS if strict_band else P_ABS + 4.0 * allow[r]
        worst_p = max(worst_p, float(np.abs(p_gpu[r, :bt] - pr).max()) / ptol * P_ABS)
        if listed.any():
            ex = np.abs(x_gpu[r, :bt][listed] - xr[listed]) / (allow[r] + 1e-6 * np.maximum(1.0, np.abs(xr[listed])))
            worst_x = max(worst_x, float(ex.max()))
    assert worst_p <= P_ABS, f"{what}: block weight error {worst_p:.3e} (scaled to the 1e-4 tolerance) > {P_ABS}"
    assert worst_x <= 1.0, f"{what}: listed x_j off by {worst_x:.3f} x its allowance"
    return {"p_max_err": worst_p, "band_differences": n_band, "pairs": n_pairs, "selected": n_sel,
            "x_err_over_allowance": worst_x}


def prefill_dump_supported(Hq, Hkv):
    P = min(64, 1 << ((128 // (Hq // Hkv)).bit_length() - 1))
    return P >= 8


def check_prefill(q, k, v, alpha, cs, rows, what="", check_selection=True, nthreads=0, strict_band=True):
    """Full parity of one prefill call: outputs, thresholds, and the block sets and weights
    the fine stage applied (read from the same call through dash_prefill_dump)."""
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    use_dump = check_selection and prefill_dump_supported(Hq, Hkv)
    if use_dump:
        out, ws, xg, pg = da.dash_prefill_dump(qd, kd, vd, rows, alpha=alpha, coarse_scale=cs)
    else:
        out, ws = da.dash_prefill(qd, kd, vd, alpha=alpha, coarse_scale=cs)
    torch.cuda.synchronize()
    st = da.dash_get_device_status(ws)
    assert st == 0, f"{what}: device status {st}"
    qr = oracle.gather_q_rows(q, rows)
    ref, tau_ref, nsel_ref = oracle.forward_rows(qr, k, v, rows, Hq, 64, alpha, cs, nthreads)
    got = rows_of(out.float().cpu(), rows).numpy()
    res = {"out": compare_out(got, ref, what)}
    tau_gpu = rows_of(da.dash_prefill_tau(ws, B, Hq, Hkv, T, d).cpu(), rows).numpy()
    has_past = np.array([t >= 64 for _, _, t in rows])
    allow = np.zeros(len(rows))
    if has_past.any():
        # Auxiliary check of tau (the specified checks are the block sets, weights and
        # outputs).  fp32 holds tau to ~1e-7 relative: 1e-4, widened for |tau| > 1, plus the
        # score-error allowance A (score_allowance).
        allow = score_allowance(qr, k, rows, Hq, alpha, cs)
        dt = np.abs(tau_gpu - tau_ref)[has_past]
        lim = (1e-4 * np.maximum(1.0, np.abs(tau_ref)) + allow)[has_past]
        assert np.all(dt <= lim), f"{what}: tau differs by {(dt / lim).max():.3f} x its tolerance"
    assert np.all(np.isnan(tau_gpu[~has_past]))
    if check_selection and has_past.any():
        if use_dump:
            sel = oracle.select_rows(qr, k, rows, Hq, 64, alpha, cs, nthreads)
            res["sel"] = compare_selection(xg.cpu().numpy(), pg.cpu().numpy(), sel, rows, allow, what,
                                           strict_band=strict_band)
        else:
            res["sel"] = check_dump(qd, kd, rows, q, k, alpha, cs, Hkv, tau_gpu, what, tau_allow=allow)
    return res, out, ws


def check_dump(qd, kd, rows, q, k, alpha, cs, Hkv, tau_prefill=None, what="", tau_allow=None):
    """Block sets and weights of dash_select_dump (the independent fp32 recomputation, used
    where the fine stage has no dump variant) against the oracle (band-exempt set parity)."""
    B, Hq, T, d = q.shape
    nbs = T // 64
    ksum = da.dash_block_summary(kd)
    idx, p, cnt, tau = da.dash_select_dump(qd, ksum, rows, max(nbs, 1), alpha, cs, Hkv)
    idx, p, cnt, tau = idx.cpu().numpy(), p.cpu().numpy(), cnt.cpu().numpy(), tau.cpu().numpy()
    sel = oracle.select_rows(oracle.gather_q_rows(q, rows), k, rows, Hq, 64, alpha, cs)
    worst_p, n_band = 0.0, 0
    for r, (b, h, t) in enumerate(rows):
        bt = t // 64
        if bt == 0:
            assert cnt[r] == 0 and np.isnan(tau[r])
            continue
        x, tr = sel["x"][r, :bt], sel["tau"][r]
        s_gpu = set(idx[r, :cnt[r]].tolist())
        s_ref = set(np.nonzero(x > tr)[0].tolist())
        diff = s_gpu ^ s_ref
        for j in diff:
            assert abs(x[j] - tr) < BAND, f"{what}: row {(b, h, t)} block {j} differs outside the band"
        n_band += len(diff)
        pg = np.zeros(bt)
        pg[idx[r, :cnt[r]]] = p[r, :cnt[r]]
        worst_p = max(worst_p, float(np.abs(pg - sel["p"][r, :bt]).max()))
        if tau_prefill is not None:
            # the dump takes fp32 dot products, the prefill tensor-core products of q with
            # kbar's bf16 hi + lo parts: both fp32-accurate, not bit-identical
            extra = 0.0 if tau_allow is None else 2.0 * tau_allow[r]
            assert abs(tau[r] - tau_prefill[r]) <= 1e-4 * max(1.0, abs(tau_prefill[r])) + extra, \
                f"{what}: dump tau {tau[r]} != prefill tau {tau_prefill[r]}"
    assert worst_p <= P_ABS, f"{what}: block weight error {worst_p:.3e}"
    return {"p_max_err": worst_p, "band_differences": n_band}


def check_decode(q, kc, vc, kv_len, alpha, cs, what="", check_selection=True):
    """Decode step on the GPU vs the oracle row t = kv_len - 1 of each sequence: outputs, and
    (groups of at most 8 heads) the thresholds, block sets and weights the attention kernel
    applied, read from the same call through dash_decode_dump."""
    B, Hq, d = q.shape
    Hkv, Tmax = kc.shape[1], kc.shape[2]
    qd, kcd, vcd = q.cuda(), kc.cuda(), vc.cuda()
    lens = torch.as_tensor(kv_len, dtype=torch.int32)
    ksum = da.dash_block_summary(kcd)
    use_dump = check_selection and Hq // Hkv <= 8
    if use_dump:
        out, ws, xg, pg, tg = da.dash_decode_dump(qd, kcd, vcd, ksum, lens.cuda(), alpha=alpha, coarse_scale=cs)
    else:
        out, ws = da.dash_decode(qd, kcd, vcd, ksum, lens.cuda(), alpha=alpha, coarse_scale=cs)
    torch.cuda.synchronize()
    assert da.dash_get_device_status(ws) == 0
    rows = [(b, h, int(lens[b]) - 1) for b in range(B) for h in range(Hq) if 1 <= int(lens[b]) <= Tmax]
    qr = torch.stack([q[b, h] for b, h, _ in rows])
    ref, tau_ref, _ = oracle.forward_rows(qr, kc, vc, rows, Hq, 64, alpha, cs)
    got = torch.stack([out[b, h].float().cpu() for b, h, _ in rows]).numpy()
    res = compare_out(got, ref, what)
    if use_dump:
        xg, pg, tg = xg.cpu().numpy(), pg.cpu().numpy(), tg.cpu().numpy()
        xr = np.stack([xg[b, h] for b, h, _ in rows])
        pr = np.stack([pg[b, h] for b, h, _ in rows])
        tr = np.array([tg[b, h] for b, h, _ in rows])
        has_past = np.array([t >= 64 for _, _, t in rows])
        assert np.all(np.isnan(tr[~has_past])), f"{what}: rows without past blocks must report NaN tau"
        if has_past.any():
            # decode scores are fp32 dot products of d terms with the fp32 summaries; their
            # rounding (d 2^-24 relative to sum |q_i kbar_i|) lies inside the hi/lo bound A
            allow = score_allowance(qr, kc, rows, Hq, alpha, cs)
            dt = np.abs(tr - tau_ref)[has_past]
            lim = (1e-4 * np.maximum(1.0, np.abs(tau_ref)) + allow)[has_past]
            assert np.all(dt <= lim), f"{what}: decode tau differs by {(dt / lim).max():.3f} x its tolerance"
            sel = oracle.select_rows(qr, kc, rows, Hq, 64, alpha, cs)
            selres = compare_selection(xr, pr, sel, rows, allow, what)
            return (res, selres), out, ws
    return (res, None), out, ws
