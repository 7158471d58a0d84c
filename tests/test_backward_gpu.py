"""GPU parity of the prefill backward (dash_prefill_backward, through the C ABI) against the
fp64 oracle's backward, which differentiates the whole forward: the fine softmax, the log
prior, the alpha-entmax Jacobian on the support, the coarse scores and the mean summaries
("DashAttention: Making Sparse Attention Fully Differentiable with Adaptive Block
Selection", sections "Core Mechanism" and "Key Concepts").

Tolerance.  The kernels round the operands of every product to bf16 (P and dS as well as
q, k, v, dout) and accumulate in fp32; dq, dk and dv are stored in bf16.  A relative
rounding of 2^-8 per operand over sums with mixed signs gives errors that scale with the
size of the gradient, not with 1: each gradient is compared relative to its own largest
entry (max-abs error <= 2e-2 x max |ref|, the output tolerance at unit scale) and relative
to its own norm (||gpu - ref|| <= 1e-2 ||ref||).
"""
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

pytestmark = pytest.mark.gpu

REL_MAX = 2e-2
REL_NORM = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    oracle.build()


def _gpu_grads(q, k, v, dout, alpha, cs):
    qd, kd, vd, gd = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    out, ws = da.dash_prefill(qd, kd, vd, alpha=alpha, coarse_scale=cs)
    dq, dk, dv = da.dash_prefill_backward(qd, kd, vd, out, gd, alpha=alpha, coarse_scale=cs)
    torch.cuda.synchronize()
    return [t.double().cpu().numpy() for t in (dq, dk, dv)]


def _compare(got, ref, what):
    rel = {}
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert np.all(np.isfinite(g)), f"{what} {name}: non-finite"
        err = np.abs(g - r)
        rmax = float(err.max() / max(np.abs(r).max(), 1e-30))
        rnorm = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30))
        rel[name] = (rmax, rnorm)
        assert rmax <= REL_MAX, f"{what} {name}: max-abs error {rmax:.3e} of max |ref|"
        assert rnorm <= REL_NORM, f"{what} {name}: error norm {rnorm:.3e} of ||ref||"
    print(what, {k: f"{a:.2e}/{b:.2e}" for k, (a, b) in rel.items()})
    return rel


# B, Hq, Hkv, T, d, alpha, coarse_scale: tiles of 64, 16, 8 and 4 positions (the last one on
# the CUDA-core coarse stage), ragged tails, both head sizes, alpha 1.5 and 1.25
CASES = [
    (1, 4, 2, 1000, 128, 1.5, 1.0),
    (1, 8, 1, 700, 64, 1.5, 0.3),
    (2, 4, 1, 520, 128, 1.25, 0.3),
    (1, 16, 2, 1024, 128, 1.5, 0.1),
    (1, 32, 1, 300, 64, 1.5, 0.3),
    (1, 4, 2, 1000, 128, 2.0, 0.3),
]


@pytest.mark.parametrize("B,Hq,Hkv,T,d,alpha,cs", CASES)
def test_backward_vs_oracle(B, Hq, Hkv, T, d, alpha, cs):
    _, (q, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, n_topics=8, seed=70 + T + Hq)
    dout = inputs.out_grad(B, Hq, T, d, seed=71 + T)
    got = _gpu_grads(q, k, v, dout, alpha, cs)
    ref = oracle.backward(q, k, v, dout, 64, alpha, cs)
    _compare(got, ref, f"backward B{B} Hq{Hq} Hkv{Hkv} T{T} d{d} a{alpha}")


def test_coarse_path_carries_gradient():
    """The parity cases exercise the selection gradient: the gradient with the prior frozen
    (log p_j held constant; torch autograd in fp64 over the oracle's p) is far from the
    oracle's full gradient, by much more than the tolerance, and the GPU follows the full one."""
    B, Hq, Hkv, T, d, alpha, cs = 1, 4, 2, 1000, 128, 1.5, 3.0
    _, (q, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, n_topics=8, seed=70 + T + Hq)
    dout = inputs.out_grad(B, Hq, T, d, seed=71 + T)
    got = _gpu_grads(q, k, v, dout, alpha, cs)
    full = oracle.backward(q, k, v, dout, 64, alpha, cs)
    rows = [(0, h, t) for h in range(Hq) for t in range(T)]
    sel = oracle.select_rows(oracle.gather_q_rows(q, rows), k, rows, Hq, 64, alpha, cs)
    G, blk = Hq // Hkv, 64
    tok_blk = torch.arange(T) // blk
    prior = torch.full((Hq, T, T), float("-inf"), dtype=torch.float64)
    p = torch.as_tensor(sel["p"]).reshape(Hq, T, -1)
    for h in range(Hq):
        for t in range(T):
            bt = t // blk
            lp = torch.zeros(T, dtype=torch.float64)
            past = tok_blk < bt
            pj = p[h, t][tok_blk[past]]
            lp[past] = torch.where(pj > 0, pj.clamp_min(1e-300).log(), torch.tensor(float("-inf"), dtype=torch.float64))
            lp[t + 1:] = float("-inf")
            prior[h, t] = lp
    qq, kk, vv = (x.double().requires_grad_(True) for x in (q, k, v))
    ke, ve = kk.repeat_interleave(G, dim=1), vv.repeat_interleave(G, dim=1)
    o = torch.softmax(qq @ ke.transpose(-1, -2) / d ** 0.5 + prior.unsqueeze(0), -1) @ ve
    o.backward(dout.double())
    frozen = [x.grad.numpy() for x in (qq, kk)]
    for name, g, r, fz in zip(("dq", "dk"), got[:2], full[:2], frozen):
        gap = np.linalg.norm(fz - r) / np.linalg.norm(r)
        err = np.linalg.norm(g - r) / np.linalg.norm(r)
        assert gap >= 5 * REL_NORM, (name, gap)
        assert err <= REL_NORM, (name, err)


@pytest.mark.parametrize("Hq,Hkv,T,d", [(4, 2, 128, 128), (8, 1, 100, 64), (4, 2, 17, 128), (8, 2, 64, 128),
                                         (2, 1, 65, 64)])
def test_two_blocks_is_dense_causal_backward(Hq, Hkv, T, d):
    """With T <= 128 every row has at most one past block: its entmax weight is 1, the
    prior is log 1 = 0 and a one-element entmax has a zero Jacobian, so the gradients are
    those of dense causal softmax attention (torch autograd in fp64 on the CPU).  Includes
    T < 64 (no complete block), exactly one block, and one block plus a token."""
    B = 1
    _, (q, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, n_topics=8, seed=90 + T)
    dout = inputs.out_grad(B, Hq, T, d, seed=91)
    got = _gpu_grads(q, k, v, dout, 1.5, 0.5)
    qq, kk, vv = (t.double().requires_grad_(True) for t in (q, k, v))
    G = Hq // Hkv
    ke, ve = kk.repeat_interleave(G, dim=1), vv.repeat_interleave(G, dim=1)
    s = qq @ ke.transpose(-1, -2) / d ** 0.5
    s = s.masked_fill(torch.ones(T, T, dtype=torch.bool).triu(1), float("-inf"))
    o = torch.softmax(s, -1) @ ve
    o.backward(dout.double())
    ref = [t.grad.numpy() for t in (qq, kk, vv)]
    _compare(got, ref, f"dense T{T}")


def test_backward_is_deterministic():
    B, Hq, Hkv, T, d = 1, 8, 2, 2048, 128
    _, (q, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, n_topics=16, seed=5)
    dout = inputs.out_grad(B, Hq, T, d, seed=6)
    a = _gpu_grads(q, k, v, dout, 1.5, 0.1)
    b = _gpu_grads(q, k, v, dout, 1.5, 0.1)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_backward_argument_errors():
    q = torch.zeros(1, 2, 128, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(da.DashError):
        da.dash_prefill_backward(q, k, k, q, q, alpha=1.0)
    with pytest.raises(ValueError):
        da.dash_prefill_backward(q, k, k, q[:, :1], q)


def test_mma_sync_backward_matches_oracle():
    """The mma.sync kernels (forced with DASH_BWD_KERNEL=mma, read once per process, hence
    the child process) give the same gradients as the tcgen05 ones, within the tolerance."""
    import json
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = (
        "import sys, json, numpy as np\n"
        f"sys.path.insert(0, {root!r}); sys.path.insert(0, {os.path.join(root, 'tests')!r})\n"
        "import oracle\n"
        "from sparse_hierarchical_attention_pool_b200 import dash_attn as da, inputs\n"
        "_, (q, k, v) = inputs.make('16k', B=1, Hq=8, Hkv=2, T=900, d=128, n_topics=8, seed=17)\n"
        "dout = inputs.out_grad(1, 8, 900, 128, seed=18)\n"
        "out, _ = da.dash_prefill(q.cuda(), k.cuda(), v.cuda(), alpha=1.5, coarse_scale=0.3)\n"
        "g = da.dash_prefill_backward(q.cuda(), k.cuda(), v.cuda(), out, dout.cuda(), alpha=1.5, coarse_scale=0.3)\n"
        "ref = oracle.backward(q, k, v, dout, 64, 1.5, 0.3)\n"
        "print(json.dumps([float(np.linalg.norm(a.double().cpu().numpy() - r) / np.linalg.norm(r))\n"
        "                  for a, r in zip(g, ref)]))\n")
    env = dict(os.environ, DASH_BWD_KERNEL="mma")
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    errs = json.loads(res.stdout.strip().splitlines()[-1])
    assert max(errs) <= REL_NORM, errs


def test_autograd_function_matches_oracle():
    """dash_attention under torch.autograd: a loss of the output back-propagates to q, k, v
    through the library's backward, matching the oracle's gradients."""
    B, Hq, Hkv, T, d, alpha, cs = 1, 8, 2, 640, 128, 1.5, 0.3
    _, (q, k, v) = inputs.make("16k", B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, n_topics=8, seed=23)
    G = inputs.out_grad(B, Hq, T, d, seed=24)
    qd, kd, vd = (t.cuda().requires_grad_(True) for t in (q, k, v))
    out = da.dash_attention(qd, kd, vd, alpha=alpha, coarse_scale=cs)
    (out.float() * G.cuda().float()).sum().backward()
    got = [t.grad.double().cpu().numpy() for t in (qd, kd, vd)]
    ref = oracle.backward(q, k, v, G, 64, alpha, cs)
    _compare(got, ref, "autograd")


def test_full_size_backward_sampled_rows_and_identities():
    """The 16K workload at the bench's shapes and calibrated scale: dq of stratified rows
    against the oracle's per-row backward (a row's dq depends on its own forward only), and
    dk, dv of the whole problem through two exact identities: per KV group the dv rows sum to
    the sum of dout over the group's query rows, and the dk rows sum to zero."""
    from gpu_helpers import calibrated_scale
    wl, (q, k, v) = inputs.make("16k")
    cs = calibrated_scale("16k")
    B, Hq, Hkv, T, d = wl.B, wl.Hq, wl.Hkv, wl.T, wl.d
    dout = inputs.out_grad(B, Hq, T, d, seed=wl.seed + 1)
    qd, kd, vd, gd = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    out, _ = da.dash_prefill(qd, kd, vd, alpha=wl.alpha, coarse_scale=cs)
    dq, dk, dv = da.dash_prefill_backward(qd, kd, vd, out, gd, alpha=wl.alpha, coarse_scale=cs)
    torch.cuda.synchronize()
    rows = [(0, h, t) for h in (0, 7, 8, 15) for t in (0, 63, 64, 1000, 4096, 8191, 12345, T - 1)]
    ref = oracle.backward_dq_rows(q, k, v, dout, rows, 64, wl.alpha, cs)
    got = np.stack([dq[b, h, t].double().cpu().numpy() for b, h, t in rows])
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref)
    assert err.max() <= REL_MAX * np.abs(ref).max(), err.max()
    assert np.linalg.norm(got - ref) <= REL_NORM * np.linalg.norm(ref), np.linalg.norm(got - ref) / np.linalg.norm(ref)
    G = Hq // Hkv
    want = gd.double().reshape(B, Hkv, G, T, d).sum(dim=(2, 3))
    have = dv.double().sum(dim=2)
    assert torch.isfinite(have).all()
    assert (have - want).norm() <= 1e-2 * want.norm(), ((have - want).norm() / want.norm()).item()
    s_dk = dk.double().sum(dim=2)
    scale = dk.double().abs().sum(dim=2)
    assert s_dk.norm() <= 1e-2 * scale.norm(), (s_dk.norm() / scale.norm()).item()
