"""dash_decode_noalloc: the decode step on the library's fixed device scratch array.

This entry point exists for callers that cannot allocate device memory where they decode
(real-time loops that must not synchronise the device through cudaMalloc / cudaFree, or
code whose device memory belongs to a foreign allocator).  Its results must match
dash_decode, which uses a caller-allocated workspace, on consecutive calls: the shared
scratch array keeps the previous call's contents, so a second call with different inputs
shows any state that leaks between calls.  The outputs are also checked against the fp64
oracle, and the device status of the array is read with dash_decode_noalloc_status.

This file is collected last so that a run stopping at its first failure has already run
every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from sparse_hierarchical_attention_pool_b200 import dash_attn as da
from sparse_hierarchical_attention_pool_b200 import inputs

OUT_MAX_ABS = 2e-2      # the output tolerances the parity tests use
OUT_MEAN_ABS = 2e-3


@pytest.fixture(scope="module")
def L():
    from sparse_hierarchical_attention_pool_b200 import build
    build.build()
    oracle.build()
    return da.lib()


def _vs_oracle(q, kc, vc, lens, out, alpha, cs, what):
    """Every valid row of a decode output against the oracle's row t = kv_len - 1."""
    B, Hq, d = q.shape
    qc, kh, vh = q.cpu(), kc.cpu(), vc.cpu()
    rows = [(b, h, int(lens[b]) - 1) for b in range(B) for h in range(Hq)]
    qr = torch.stack([qc[b, h] for b, h, _ in rows])
    ref, _, _ = oracle.forward_rows(qr, kh, vh, rows, Hq, 64, alpha, cs)
    got = torch.stack([out[b, h].float().cpu() for b, h, _ in rows]).double().numpy()
    err = np.abs(got - ref)
    assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS, (what, err.max(), err.mean())


def _decode_inputs(B, Hq, Hkv, Tmax, d, seed, lens):
    _, (q4, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=Tmax, d=d, n_topics=16, seed=seed)
    q = torch.stack([q4[b, :, lens[b] - 1] for b in range(B)]).contiguous()
    return q.cuda(), k.cuda(), v.cuda(), torch.tensor(lens, dtype=torch.int32, device="cuda")


def _via_c_abi(L, q, kc, vc, ksum, lens, out, alpha, cs):
    B, Hq, d = q.shape
    Hkv, Tmax = kc.shape[1], kc.shape[2]
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return L.dash_decode_noalloc(p(q), p(kc), p(vc), p(ksum), p(lens), p(out), B, Hq, Hkv, Tmax, d, 64,
                                 ctypes.c_float(alpha), ctypes.c_float(cs),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.gpu
def test_noalloc_matches_workspace_decode_on_two_calls(L):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cases = [
        (_decode_inputs(4, 8, 2, 1000, 128, 31, [1000, 700, 65, 3]), 0.05),
        (_decode_inputs(4, 8, 2, 1000, 128, 32, [999, 128, 512, 1000]), 0.08),
    ]
    for (q, kc, vc, lens), cs in cases:           # two calls in a row, different inputs
        ksum = da.dash_block_summary(kc)
        ref, _ = da.dash_decode(q, kc, vc, ksum, lens, alpha=1.5, coarse_scale=cs)
        out = torch.full_like(q, float("nan"))
        rc = _via_c_abi(L, q, kc, vc, ksum, lens, out, 1.5, cs)
        assert rc == 0, da.STATUS.get(rc, rc)
        assert L.dash_decode_noalloc_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        diff = (out.float() - ref.float()).abs().max().item()
        assert diff <= OUT_MAX_ABS, diff
        _vs_oracle(q, kc, vc, lens.cpu(), out, 1.5, cs, "noalloc small")


@pytest.mark.gpu
def test_noalloc_full_decode_workload(L):
    """The 96K decode workload itself (B=8, Hq=32, Hkv=8, cache 98304, d=128) runs within
    the fixed scratch: two calls in a row equal dash_decode and the oracle on all 256 rows."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert da.decode_workspace_size(8, 32, 8, 98304, 128) <= 32 << 20
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "coarse_scale.json")) as f:
        cs = json.load(f)["decode96k"]["coarse_scale"]
    wl, (q, kc, vc, kv_len) = inputs.make("decode96k")
    qd, kcd, vcd, lens = q.cuda(), kc.cuda(), vc.cuda(), kv_len.cuda()
    ksum = da.dash_block_summary(kcd)
    ref, _ = da.dash_decode(qd, kcd, vcd, ksum, lens, alpha=wl.alpha, coarse_scale=cs)
    for _ in range(2):
        out = da.dash_decode_noalloc(qd, kcd, vcd, ksum, lens, alpha=wl.alpha, coarse_scale=cs)
        assert da.dash_decode_noalloc_status() == 0
        assert (out.float() - ref.float()).abs().max().item() <= OUT_MAX_ABS
    _vs_oracle(q, kc, vc, kv_len, out, wl.alpha, cs, "noalloc 96K decode")


@pytest.mark.gpu
def test_noalloc_status_reports_a_capped_solve(L, monkeypatch):
    """A threshold solve cut short (debug cap, a normal terminating launch) shows in
    dash_decode_noalloc_status; the next call with the normal cap reads clean."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    q, kc, vc, lens = _decode_inputs(2, 8, 2, 1000, 128, 34, [1000, 700])
    ksum = da.dash_block_summary(kc)
    monkeypatch.setenv("DASH_DEBUG_SOLVE_CAP", "1")
    da.dash_decode_noalloc(q, kc, vc, ksum, lens, alpha=1.25, coarse_scale=0.05)
    assert da.dash_decode_noalloc_status() == -7
    monkeypatch.delenv("DASH_DEBUG_SOLVE_CAP")
    da.dash_decode_noalloc(q, kc, vc, ksum, lens, alpha=1.25, coarse_scale=0.05)
    assert da.dash_decode_noalloc_status() == 0


def test_noalloc_rejects_steps_beyond_the_scratch_limit(L):
    """Checked before any CUDA call: no GPU is needed, nothing is launched."""
    fake = ctypes.c_void_p(1 << 20)
    # 64 sequences x 32 heads at 96K need far more than 32 MiB of scratch
    assert da.decode_workspace_size(64, 32, 8, 98304, 128) > 32 << 20
    rc = L.dash_decode_noalloc(fake, fake, fake, fake, fake, fake, 64, 32, 8, 98304, 128, 64,
                               ctypes.c_float(1.5), ctypes.c_float(0.02), None)
    assert rc == -8
    assert b"SCRATCH" in L.dash_status_string(rc)
    rc = L.dash_decode_noalloc(None, fake, fake, fake, fake, fake, 1, 1, 1, 128, 64, 64,
                               ctypes.c_float(1.5), ctypes.c_float(0.02), None)
    assert rc == -1
