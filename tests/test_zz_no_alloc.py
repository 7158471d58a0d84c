"""dash_decode_noalloc: the decode step on the library's fixed device scratch array.

This entry point exists for callers that cannot allocate device memory where they decode
(inside CUDA graph capture, in real-time loops that must not synchronise the device
through cudaMalloc / cudaFree, or under a foreign allocator).  Its results must match
dash_decode, which uses a caller-allocated workspace, on consecutive calls: the shared
scratch array keeps the previous call's contents, so a second call with different inputs
shows any state that leaks between calls.

This file is collected last so that a run stopping at its first failure has already run
every other test; it also passes on its own in a fresh process.
"""
import ctypes

import pytest
import torch

from sparse_hierarchical_attention_pool_b200 import dash_attn as da
from sparse_hierarchical_attention_pool_b200 import inputs

OUT_MAX_ABS = 2e-2      # the output tolerance the parity tests use


@pytest.fixture(scope="module")
def L():
    from sparse_hierarchical_attention_pool_b200 import build
    build.build()
    return da.lib()


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
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        diff = (out.float() - ref.float()).abs().max().item()
        assert diff <= OUT_MAX_ABS, diff


@pytest.mark.gpu
def test_noalloc_full_decode_workload_shape_fits(L):
    """The 96K decode shape (B=8, Hq=32, Hkv=8, d=128) runs within the fixed scratch."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert da.decode_workspace_size(8, 32, 8, 98304, 128) <= 32 << 20
    B, Hq, Hkv, Tmax, d = 2, 32, 8, 4096, 128
    q, kc, vc, lens = _decode_inputs(B, Hq, Hkv, Tmax, d, 33, [4096, 2049])
    ksum = da.dash_block_summary(kc)
    ref, _ = da.dash_decode(q, kc, vc, ksum, lens, alpha=1.5, coarse_scale=0.05)
    for _ in range(2):
        out = da.dash_decode_noalloc(q, kc, vc, ksum, lens, alpha=1.5, coarse_scale=0.05)
        torch.cuda.synchronize()
        assert (out.float() - ref.float()).abs().max().item() <= OUT_MAX_ABS


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
