"""Pins for the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each test checks the oracle against something other than itself: hand-derived values
(tests/golden/worked_example.json), closed forms, a different algorithm (bisection,
brute force over supports), scipy's constrained optimiser on the variational definition
of alpha-entmax, torch's softmax and scaled-dot-product attention as library routines,
and invariants (sum to one, shift and permutation invariance, non-dispersiveness).

Definitions come from "DashAttention: Making Sparse Attention Fully Differentiable with
Adaptive Block Selection", sections "Core Mechanism" and "Key Concepts", and "DashAttention
and the year sparse attention became a field", section "What alpha-entmax changes".
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

GOLD = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")
ALPHAS = [1.25, 1.5, 2.0, 3.0]


@pytest.fixture(scope="module")
def gold():
    with open(GOLD) as f:
        return json.load(f)


# ---------------------------------------------------------------- alpha-entmax

def test_worked_example_exact_values(orc, gold):
    s = gold["scores"]
    p, tau = orc.entmax(s, 1.5)
    assert np.allclose(p, gold["entmax_1_5"]["p"], atol=1e-12)
    assert abs(tau - gold["entmax_1_5"]["tau"]) < 1e-12
    p, tau = orc.entmax(s, 2.0)
    assert np.allclose(p, gold["sparsemax"]["p"], atol=1e-12)
    assert abs(tau - gold["sparsemax"]["tau"]) < 1e-12
    # alpha -> 1 is softmax: compare with the hand-derived values
    p, _ = orc.entmax(s, 1.0 + 1e-7)
    assert np.allclose(p, gold["softmax_exact"]["p"], atol=1e-5)


def test_worked_example_printed_values_are_not_the_definition(orc, gold):
    """The page's printed vectors contradict its own definitions (negative pin)."""
    s = gold["scores"]
    p15, _ = orc.entmax(s, 1.5)
    assert not np.allclose(p15, gold["printed_entmax_1_5"], atol=1e-2)
    sm = torch.softmax(torch.tensor(s, dtype=torch.float64), 0).numpy()
    assert not np.allclose(sm, gold["printed_softmax"], atol=1e-2)


def test_designed_closed_forms(orc, gold):
    for case in gold["designed_cases"]:
        p, tau = orc.entmax(case["scores"], case["alpha"])
        assert np.allclose(p, case["p"], atol=1e-12), case
        assert abs(tau - case["tau"]) < 1e-12


@pytest.mark.parametrize("alpha", ALPHAS)
def test_tau_sort_bisection_bruteforce_agree(orc, alpha):
    rng = np.random.default_rng(int(alpha * 100))
    for _ in range(400):
        n = int(rng.integers(1, 13))
        s = rng.normal(size=n) * rng.uniform(0.05, 6.0)
        if rng.random() < 0.2:            # ties
            s[rng.integers(0, n)] = s[0]
        t_sort = orc.entmax_tau(s, alpha, "sort")
        t_bis = orc.entmax_tau(s, alpha, "bisect")
        t_bru = orc.entmax_tau(s, alpha, "brute")
        assert abs(t_sort - t_bis) < 1e-10
        assert abs(t_sort - t_bru) < 1e-9


@pytest.mark.parametrize("alpha", ALPHAS)
def test_tau_sort_vs_bisection_long_rows(orc, alpha):
    rng = np.random.default_rng(7 + int(alpha * 10))
    for n in (50, 255, 1535):
        s = rng.normal(size=n) * 3
        assert abs(orc.entmax_tau(s, alpha, "sort") - orc.entmax_tau(s, alpha, "bisect")) < 1e-10


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_variational_definition_scipy(orc, alpha):
    """alpha-entmax(s) = argmax_{p in simplex} p.s + (1 - sum p^alpha) / (alpha (alpha - 1))."""
    from scipy.optimize import minimize
    rng = np.random.default_rng(11)
    for _ in range(12):
        n = int(rng.integers(2, 7))
        s = rng.normal(size=n) * 1.5

        def neg(p):
            p = np.clip(p, 0, None)
            return -(p @ s + (1 - np.sum(p ** alpha)) / (alpha * (alpha - 1)))

        res = minimize(neg, np.full(n, 1.0 / n), method="SLSQP", bounds=[(0, 1)] * n,
                       constraints=[{"type": "eq", "fun": lambda p: p.sum() - 1}],
                       options={"ftol": 1e-14, "maxiter": 500})
        p, _ = orc.entmax(s, alpha)
        assert np.allclose(p, res.x, atol=2e-4), (s, p, res.x)


def test_softmax_limit_linear_error(orc):
    rng = np.random.default_rng(3)
    s = rng.normal(size=9)
    sm = torch.softmax(torch.tensor(s), 0).numpy()
    errs = []
    for eps in (1e-2, 1e-3, 1e-4):
        p, _ = orc.entmax(s, 1.0 + eps)
        errs.append(np.abs(p - sm).max())
    assert errs[2] < 1e-3
    assert errs[0] / errs[1] > 5 and errs[1] / errs[2] > 5


@pytest.mark.parametrize("alpha", ALPHAS)
def test_entmax_invariants(orc, alpha):
    rng = np.random.default_rng(5)
    for _ in range(100):
        n = int(rng.integers(1, 40))
        s = rng.normal(size=n) * rng.uniform(0.1, 8)
        p, tau = orc.entmax(s, alpha)
        assert abs(p.sum() - 1) < 1e-12
        x = (alpha - 1) * s
        assert np.all((p == 0) == (x <= tau))
        assert np.all(p >= 0)
        # shift invariance and permutation equivariance
        p2, _ = orc.entmax(s + 3.7, alpha)
        assert np.allclose(p, p2, atol=1e-10)
        perm = rng.permutation(n)
        p3, _ = orc.entmax(s[perm], alpha)
        assert np.allclose(p[perm], p3, atol=1e-12)


def test_support_shrinks_with_alpha(orc):
    """Higher alpha is sparser ("Key Concepts"): checked on random inputs, not assumed."""
    rng = np.random.default_rng(9)
    for _ in range(200):
        s = rng.normal(size=int(rng.integers(2, 30))) * rng.uniform(0.2, 4)
        sizes = [int((orc.entmax(s, a)[0] > 0).sum()) for a in (1.25, 1.5, 2.0, 3.0)]
        assert sizes == sorted(sizes, reverse=True), (s, sizes)


def test_zero_and_huge_scale(orc):
    rng = np.random.default_rng(2)
    s = rng.normal(size=17)
    for a in ALPHAS:
        p, _ = orc.entmax(0 * s, a)
        assert np.allclose(p, 1 / 17, atol=1e-12)
        p, _ = orc.entmax(1e6 * s, a)
        assert p[np.argmax(s)] == 1.0 and p.sum() == 1.0


# ---------------------------------------------------------------- summaries and scores

def _designed_problem(scores, d=4, blk=4, n_diag=2, seed=0):
    """Keys whose block means have first component exactly scores[j]; q = [2, 0, 0, 0]
    so that q . kbar_j / sqrt(d) = scores[j] (d = 4).  Returns q [1,1,T,d], k, v, t."""
    rng = np.random.default_rng(seed)
    nb_past = len(scores)
    T = (nb_past + 1) * blk
    k = rng.normal(size=(1, 1, T, d)).astype(np.float32)
    k -= k.reshape(1, 1, T // blk, blk, d).mean(3).repeat(blk, axis=2)      # zero-mean blocks
    dev = np.array([0.5, -0.5, 0.25, -0.25], dtype=np.float32)              # mean 0, not constant
    for j, sj in enumerate(scores):
        k[0, 0, j * blk:(j + 1) * blk, 0] = sj + dev
    k = k.astype(np.float32)
    v = rng.normal(size=(1, 1, T, d)).astype(np.float32)
    q = np.zeros((1, 1, T, d), dtype=np.float32)
    q[..., 0] = 2.0
    t = nb_past * blk + n_diag - 1
    return q, k, v, t


def test_block_summary_is_numpy_mean(orc):
    rng = np.random.default_rng(1)
    k = rng.normal(size=(2, 3, 200, 8)).astype(np.float32)
    got = orc.block_summary(k, 64)
    ref = k[:, :, :192].astype(np.float64).reshape(2, 3, 3, 64, 8).mean(3)
    assert got.shape == (2, 3, 3, 8)
    assert np.allclose(got, ref, atol=1e-12)


@pytest.mark.parametrize("case_i", [0, 1])
def test_coarse_scores_and_prior_against_sdpa(orc, gold, case_i):
    """Designed keys give the hand-derived block weights; the fine stage then equals torch
    SDPA with an additive mask of log p on past tokens, 0 on the causal own block."""
    case = gold["designed_cases"][case_i]
    alpha, blk, d = case["alpha"], 4, 4
    q, k, v, t = _designed_problem(case["scores"], d=d, blk=blk)
    sel = orc.select_rows(q[0, 0, t][None], k, [(0, 0, t)], 1, blk, alpha, 1.0)
    assert np.allclose(sel["p"][0, :4], case["p"], atol=1e-6)
    assert abs(sel["tau"][0] - case["tau"]) < 1e-6
    out, tau, ns = orc.forward_rows(q[0, 0, t][None], k, v, [(0, 0, t)], 1, blk, alpha, 1.0)
    assert ns[0] == sum(1 for x in case["p"] if x > 0)
    T = k.shape[2]
    bias = np.full(T, -np.inf)
    for i in range(t + 1):
        j = i // blk
        if j == t // blk:
            bias[i] = 0.0
        elif case["p"][j] > 0:
            bias[i] = math.log(case["p"][j])
    qt = torch.tensor(q[0, 0, t], dtype=torch.float64).view(1, 1, 1, d)
    ref = F.scaled_dot_product_attention(qt, torch.tensor(k, dtype=torch.float64),
                                         torch.tensor(v, dtype=torch.float64),
                                         attn_mask=torch.tensor(bias).view(1, 1, 1, T))
    assert np.allclose(out[0], ref.view(d).numpy(), atol=1e-12)


def test_coarse_scale_and_alpha_scaling(orc, gold):
    """Scaling cs by c is scaling the scores by c (checked against the closed form)."""
    case = gold["designed_cases"][0]             # sparsemax case, scores [1, 0.6, -2, -3]
    q, k, v, t = _designed_problem([2 * s for s in case["scores"]])
    sel = orc.select_rows(q[0, 0, t][None], k, [(0, 0, t)], 1, 4, 2.0, 0.5)
    assert np.allclose(sel["p"][0, :4], case["p"], atol=1e-6)


# ---------------------------------------------------------------- whole rows vs dense attention

def _rand_problem(B, Hq, Hkv, T, d, seed, dtype=np.float32):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(B, Hq, T, d)).astype(dtype)
    k = rng.normal(size=(B, Hkv, T, d)).astype(dtype)
    v = rng.normal(size=(B, Hkv, T, d)).astype(dtype)
    return q, k, v


def _sdpa_rows(q, k, v, rows):
    B, Hq, T, d = q.shape
    G = Hq // k.shape[1]
    kk = torch.tensor(k, dtype=torch.float64).repeat_interleave(G, dim=1)
    vv = torch.tensor(v, dtype=torch.float64).repeat_interleave(G, dim=1)
    full = F.scaled_dot_product_attention(torch.tensor(q, dtype=torch.float64), kk, vv, is_causal=True)
    return np.stack([full[b, h, t].numpy() for b, h, t in rows])


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_two_blocks_or_fewer_is_dense_causal(orc, alpha):
    """With T <= 2 blocks a row has at most one past block, whose weight is 1: the output
    is dense causal attention (torch SDPA), for grouped heads too."""
    B, Hq, Hkv, T, d, blk = 2, 4, 2, 128, 16, 64
    q, k, v = _rand_problem(B, Hq, Hkv, T, d, 4)
    rows = [(b, h, t) for b in range(B) for h in range(Hq) for t in range(T)]
    out, _, _ = orc.forward_rows(q.reshape(-1, d), k, v, rows, Hq, blk, alpha, 3.0)
    assert np.allclose(out, _sdpa_rows(q, k, v, rows), atol=1e-12)
    dense = orc.dense_causal_rows(q.reshape(-1, d), k, v, rows, Hq)
    assert np.allclose(dense, out, atol=1e-12)


def test_equal_prior_is_dense_causal(orc):
    B, Hq, Hkv, T, d, blk = 1, 2, 1, 300, 8, 64
    q, k, v = _rand_problem(B, Hq, Hkv, T, d, 8)
    rows = [(0, h, t) for h in range(Hq) for t in range(0, T, 7)]
    qr = np.stack([q[b, h, t] for b, h, t in rows])
    w = np.full((len(rows), T // blk), 0.37)
    out = orc.fine_rows_given_p(qr, k, v, rows, Hq, blk, w, np.full(len(rows), 0.37))
    assert np.allclose(out, _sdpa_rows(q, k, v, rows), atol=1e-12)


def test_zero_scale_weights_are_uniform(orc):
    B, Hq, Hkv, T, d, blk = 1, 2, 2, 640, 8, 64
    q, k, v = _rand_problem(B, Hq, Hkv, T, d, 9)
    rows = [(0, h, t) for h in range(Hq) for t in (64, 200, 639)]
    qr = np.stack([q[b, h, t] for b, h, t in rows])
    sel = orc.select_rows(qr, k, rows, Hq, blk, 1.5, 0.0)
    for r, (b, h, t) in enumerate(rows):
        bt = t // blk
        assert np.allclose(sel["p"][r, :bt], 1.0 / bt, atol=1e-12)


def test_non_dispersive_insertion(orc):
    """Blocks whose weight is zero can be inserted without changing later outputs
    ("Key Concepts", non-dispersive attention)."""
    d, blk, Tb = 16, 64, 6
    rng = np.random.default_rng(12)
    u = rng.normal(size=d); u /= np.linalg.norm(u)
    T = Tb * blk
    q = (8 * u + 0.3 * rng.normal(size=(1, 1, T, d))).astype(np.float32)
    k = (8 * u + 0.3 * rng.normal(size=(1, 1, T, d))).astype(np.float32)
    v = rng.normal(size=(1, 1, T, d)).astype(np.float32)
    ins = 2
    bad = (-8 * u + 0.3 * rng.normal(size=(1, 1, ins * blk, d))).astype(np.float32)
    cut = 2 * blk
    k2 = np.concatenate([k[:, :, :cut], bad, k[:, :, cut:]], axis=2)
    v2 = np.concatenate([v[:, :, :cut], rng.normal(size=(1, 1, ins * blk, d)).astype(np.float32),
                         v[:, :, cut:]], axis=2)
    q2 = np.concatenate([q[:, :, :cut], q[:, :, :ins * blk], q[:, :, cut:]], axis=2)
    ts = list(range(cut, T))
    rows1 = [(0, 0, t) for t in ts]
    rows2 = [(0, 0, t + ins * blk) for t in ts]
    o1, _, _ = orc.forward_rows(q[0, 0, ts], k, v, rows1, 1, blk, 1.5, 1.0)
    sel = orc.select_rows(q2[0, 0, [t + ins * blk for t in ts]], k2, rows2, 1, blk, 1.5, 1.0)
    assert np.all(sel["p"][:, 2:2 + ins] == 0)          # inserted blocks get weight 0
    o2, _, _ = orc.forward_rows(q2[0, 0, [t + ins * blk for t in ts]], k2, v2, rows2, 1, blk, 1.5, 1.0)
    assert np.allclose(o1, o2, atol=1e-12)


def test_decode_reads_nothing_beyond_kv_len(orc):
    """A decode row of a partly filled cache equals the last prefill row; cache slots
    past kv_len hold NaN, so any read of them would show."""
    B, Hq, Hkv, T, d, blk, Tmax = 2, 4, 2, 333, 16, 64, 512
    q, k, v = _rand_problem(B, Hq, Hkv, T, d, 21)
    kc = np.full((B, Hkv, Tmax, d), np.nan, dtype=np.float32)
    vc = np.full((B, Hkv, Tmax, d), np.nan, dtype=np.float32)
    kc[:, :, :T], vc[:, :, :T] = k, v
    rows = [(b, h, T - 1) for b in range(B) for h in range(Hq)]
    qr = np.stack([q[b, h, T - 1] for b, h, _ in rows])
    o_pre, tau_pre, _ = orc.forward_rows(qr, k, v, rows, Hq, blk, 1.5, 4.0)
    o_dec, tau_dec, _ = orc.forward_rows(qr, kc, vc, rows, Hq, blk, 1.5, 4.0)
    assert np.all(np.isfinite(o_dec))
    assert np.array_equal(o_pre, o_dec) and np.array_equal(tau_pre, tau_dec)


def test_bf16_input_path_widens_exactly(orc):
    q, k, v = _rand_problem(1, 2, 1, 200, 8, 30)
    qb, kb, vb = (torch.tensor(a).bfloat16() for a in (q, k, v))
    rows = [(0, h, t) for h in range(2) for t in (10, 70, 199)]
    qr = torch.stack([qb[b, h, t] for b, h, t in rows])
    o1, t1, _ = orc.forward_rows(qr, kb, vb, rows, 2, 64, 1.5, 2.0)
    o2, t2, _ = orc.forward_rows(qr.float().numpy(), kb.float().numpy(), vb.float().numpy(),
                                 rows, 2, 64, 1.5, 2.0)
    assert np.array_equal(o1, o2) and np.array_equal(t1, t2, equal_nan=True)


# ------------------------------------------------------------------ learned summary head
# "DashAttention and the year sparse attention became a field", section "What alpha-entmax
# changes": Stage 0 is a small attention head initialised at zero (mean pooling at zero).

def _keys(B, Hkv, T, d, seed):
    g = np.random.default_rng(seed)
    return g.standard_normal((B, Hkv, T, d)).astype(np.float32)


def test_learned_summary_zero_head_is_the_mean(orc):
    k = _keys(2, 3, 256, 16, 1)
    np.testing.assert_allclose(orc.block_summary(k, 64, w=np.zeros((3, 16))), orc.block_summary(k, 64),
                               rtol=0, atol=1e-12)


def test_learned_summary_two_valued_block_closed_form(orc):
    # a block whose keys take two values a (first 24 keys) and b (40 keys): the pooling
    # weights are proportional to n_a e^{s_a} and n_b e^{s_b}, s = w . key / sqrt(d)
    d = 4
    a = np.array([1.0, -2.0, 0.5, 3.0])
    b = np.array([-1.0, 0.25, 2.0, 0.0])
    w = np.array([[0.3, -0.7, 1.1, 0.2]])
    k = np.zeros((1, 1, 64, d), dtype=np.float32)
    k[0, 0, :24] = a
    k[0, 0, 24:] = b
    sa, sb = w[0] @ a / 2.0, w[0] @ b / 2.0
    wa, wb = 24 * np.exp(sa), 40 * np.exp(sb)
    want = (wa * a + wb * b) / (wa + wb)
    np.testing.assert_allclose(orc.block_summary(k, 64, w=w)[0, 0, 0], want, rtol=0, atol=1e-12)


def test_learned_summary_sharp_head_picks_the_top_key(orc):
    k = _keys(1, 1, 128, 8, 2)
    w = np.zeros((1, 8))
    w[0, 3] = 4000.0
    s = orc.block_summary(k, 64, w=w)
    for j in range(2):
        blk = k[0, 0, 64 * j:64 * (j + 1)].astype(np.float64)
        np.testing.assert_allclose(s[0, 0, j], blk[np.argmax(blk[:, 3])], rtol=0, atol=1e-6)


def test_learned_summary_permutation_and_orthogonal_shift(orc):
    d = 16
    k = _keys(1, 2, 192, d, 3)
    w = np.random.default_rng(4).standard_normal((2, d))
    base = orc.block_summary(k, 64, w=w)
    perm = k.copy()
    for j in range(3):
        idx = np.random.default_rng(10 + j).permutation(64)
        perm[:, :, 64 * j:64 * (j + 1)] = k[:, :, 64 * j + idx]
    np.testing.assert_allclose(orc.block_summary(perm, 64, w=w), base, rtol=0, atol=1e-12)
    # adding c with w_g . c = 0 to every key of head g leaves the weights, and moves kbar by c
    shifted = k.astype(np.float64).copy()
    for g_ in range(2):
        c = np.random.default_rng(20 + g_).standard_normal(d)
        c -= (c @ w[g_]) / (w[g_] @ w[g_]) * w[g_]
        shifted[:, g_] += c
        want = base[:, g_] + c
        got = orc.block_summary(shifted.astype(np.float32), 64, w=w)[:, g_]
        np.testing.assert_allclose(got, want, rtol=0, atol=2e-6)   # float32 inputs


def test_forward_with_zero_head_equals_mean_forward(orc):
    import torch
    B, Hq, Hkv, T, d = 1, 4, 2, 512, 16
    g = torch.Generator().manual_seed(5)
    q = torch.randn(B, Hq, T, d, generator=g).bfloat16()
    k = torch.randn(B, Hkv, T, d, generator=g).bfloat16()
    v = torch.randn(B, Hkv, T, d, generator=g).bfloat16()
    rows = [(0, h, t) for h in range(Hq) for t in (70, 200, 511)]
    qr = orc.gather_q_rows(q, rows)
    o0, t0, _ = orc.forward_rows(qr, k, v, rows, Hq, 64, 1.5, 2.0)
    o1, t1, _ = orc.forward_rows(qr, k, v, rows, Hq, 64, 1.5, 2.0, w_summary=np.zeros((Hkv, d)))
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(t1, t0, rtol=0, atol=1e-12)
    # a learned head changes the selection of some row (it is not silently ignored)
    w = np.random.default_rng(6).standard_normal((Hkv, d)) * 3.0
    o2, t2, _ = orc.forward_rows(qr, k, v, rows, Hq, 64, 1.5, 2.0, w_summary=w)
    assert np.abs(t2 - t0).max() > 1e-6


# ------------------------------------------------------------------ head aggregation
# "DashAttention and the year sparse attention became a field", section "Non-dispersive
# attention at long context" (entmax head aggregation): the heads of a KV group average their
# block distributions and share that prior.

def _agg_inputs(Hq, Hkv, T, d, seed, same_heads=False):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(1, Hq, T, d, generator=g) * 1.5
    if same_heads:
        G = Hq // Hkv
        q = q[:, ::G].repeat_interleave(G, dim=1)
    k = torch.randn(1, Hkv, T, d, generator=g)
    v = torch.randn(1, Hkv, T, d, generator=g)
    return q.bfloat16(), k.bfloat16(), v.bfloat16()


def _agg_rows(Hq, T):
    return [(0, h, t) for h in range(Hq) for t in (0, 63, 64, 200, 450, T - 1)]


def test_aggregation_of_one_head_is_the_per_head_forward(orc):
    q, k, v = _agg_inputs(3, 3, 512, 16, 1)
    rows = _agg_rows(3, 512)
    a, ns_a = orc.forward_rows_agg(q, k, v, rows, 64, 1.5, 3.0)
    b, _, ns_b = orc.forward_rows(orc.gather_q_rows(q, rows), k, v, rows, 3, 64, 1.5, 3.0)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    assert np.array_equal(ns_a, ns_b)


def test_aggregation_of_identical_heads_is_the_per_head_forward(orc):
    q, k, v = _agg_inputs(8, 2, 512, 16, 2, same_heads=True)
    rows = _agg_rows(8, 512)
    a, _ = orc.forward_rows_agg(q, k, v, rows, 64, 1.5, 3.0)
    b, _, _ = orc.forward_rows(orc.gather_q_rows(q, rows), k, v, rows, 8, 64, 1.5, 3.0)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_aggregated_prior_is_the_mean_distribution_and_its_support_the_union(orc):
    Hq, Hkv, T, d, G = 8, 2, 512, 16, 4
    q, k, v = _agg_inputs(Hq, Hkv, T, d, 3)
    rows = [(0, h, t) for h in range(Hq) for t in (130, 300, 511)]
    out, ns = orc.forward_rows_agg(q, k, v, rows, 64, 1.5, 3.0)
    # the same rows through two other routes: every head's selection, then the fine stage
    # with the averaged weights injected
    wts, unions = [], []
    for (b, h, t) in rows:
        grp = [(b, (h // G) * G + i, t) for i in range(G)]
        sel = orc.select_rows(orc.gather_q_rows(q, grp), k, grp, Hq, 64, 1.5, 3.0)
        wts.append(sel["p"].mean(0))
        unions.append(int((sel["p"] > 0).any(0).sum()))
    wts = np.array(wts)
    assert np.allclose(wts.sum(1), 1.0, atol=1e-12)
    assert np.array_equal(ns, np.array(unions))
    ref = orc.fine_rows_given_p(orc.gather_q_rows(q, rows), k, v, rows, Hq, 64, wts, np.ones(len(rows)))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_aggregated_attention_ignores_blocks_outside_the_shared_support(orc):
    # the values of a past block that no head of the group selects never reach the output
    Hq, Hkv, T, d, G = 4, 1, 640, 16, 4
    q, k, v = _agg_inputs(Hq, Hkv, T, d, 4)
    t = 639
    grp = [(0, h, t) for h in range(G)]
    p = orc.select_rows(orc.gather_q_rows(q, grp), k, grp, Hq, 64, 2.0, 6.0)["p"]
    bt = t // 64                           # the own block is always attended
    unused = np.where(~(p[:, :bt] > 0).any(0))[0]
    used = np.where((p[:, :bt] > 0).any(0))[0]
    assert len(unused) > 0 and len(used) > 0
    base, _ = orc.forward_rows_agg(q, k, v, grp, 64, 2.0, 6.0)
    v2 = v.clone()
    for j in unused:
        v2[0, 0, 64 * j:64 * (j + 1)] = (torch.randn(64, d) * 100).bfloat16()
    np.testing.assert_allclose(orc.forward_rows_agg(q, k, v2, grp, 64, 2.0, 6.0)[0], base, rtol=0, atol=1e-12)
    v3 = v.clone()
    v3[0, 0, 64 * used[0]:64 * (used[0] + 1)] += 1.0
    assert np.abs(orc.forward_rows_agg(q, k, v3, grp, 64, 2.0, 6.0)[0] - base).max() > 1e-6


# ------------------------------------------------------------------ backward
# Differentiability is the method's central claim ("DashAttention: Making Sparse Attention Fully
# Differentiable with Adaptive Block Selection", section "Key Concepts"): the oracle backward
# (fine softmax, log prior, alpha-entmax Jacobian, coarse scores, mean summaries) is pinned
# by central finite differences of the fp64 forward.

@pytest.mark.parametrize("alpha,cs,Hq,Hkv,T", [(1.5, 2.0, 2, 1, 448), (2.0, 3.0, 4, 2, 384),
                                               (1.25, 4.0, 2, 2, 320), (3.0, 1.5, 2, 1, 448)])
def test_backward_matches_finite_differences(orc, alpha, cs, Hq, Hkv, T):
    d, B = 8, 1
    rng = np.random.default_rng(int(alpha * 100) + T)
    q = rng.standard_normal((B, Hq, T, d)) * 1.5
    k = rng.standard_normal((B, Hkv, T, d))
    v = rng.standard_normal((B, Hkv, T, d))
    G = rng.standard_normal((B, Hq, T, d))
    rows = [(0, h, t) for h in range(Hq) for t in range(T)]

    def loss(q_, k_, v_):
        out, _, _ = orc.forward_rows(q_.reshape(-1, d), k_, v_, rows, Hq, 64, alpha, cs)
        return float((out * G.reshape(-1, d)).sum())

    dq, dk, dv = orc.backward(q, k, v, G, 64, alpha, cs)
    # the coarse stage is exercised: some rows have a sparse, non-trivial support
    sel = orc.select_rows(q.reshape(-1, d), k, rows, Hq, 64, alpha, cs)
    assert np.any((sel["nsel"] < sel["bt"]) & (sel["nsel"] >= 2))
    h = 1e-6
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, s)) for s in arr.shape)
            args = {"q": q, "k": k, "v": v}
            a = arr.copy(); a[idx] += h; args[name] = a; lp = loss(args["q"], args["k"], args["v"])
            a = arr.copy(); a[idx] -= h; args[name] = a; lm = loss(args["q"], args["k"], args["v"])
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def test_backward_of_dense_rows_is_softmax_attention_backward(orc):
    # T <= 2 blocks: one past block (p = 1, no gradient into the coarse stage) -- plain causal
    # attention, whose gradients torch.autograd gives independently
    B, Hq, Hkv, T, d = 1, 2, 1, 128, 8
    g = torch.Generator().manual_seed(3)
    q = torch.randn(B, Hq, T, d, generator=g, dtype=torch.float64, requires_grad=True)
    k = torch.randn(B, Hkv, T, d, generator=g, dtype=torch.float64, requires_grad=True)
    v = torch.randn(B, Hkv, T, d, generator=g, dtype=torch.float64, requires_grad=True)
    G = torch.randn(B, Hq, T, d, generator=g, dtype=torch.float64)
    kk, vv = k.repeat_interleave(Hq // Hkv, 1), v.repeat_interleave(Hq // Hkv, 1)
    out = F.scaled_dot_product_attention(q, kk, vv, is_causal=True)
    (out * G).sum().backward()
    dq, dk, dv = orc.backward(q.detach(), k.detach(), v.detach(), G, 64, 1.5, 2.0)
    np.testing.assert_allclose(dq, q.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dk, k.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dv, v.grad.numpy(), rtol=0, atol=1e-10)


def test_backward_identities_and_row_dq(orc):
    """Exact identities of the backward, any size: per KV group the dv rows sum to the sum of
    dout over the group's query rows (each row's softmax weights sum to one), and the dk rows
    sum to zero (each row's dS sums to zero over its tokens, and its entmax terms ds_j sum to
    zero over its support).  The rows-only dq equals the full backward's rows."""
    B, Hq, Hkv, T, d, alpha, cs = 1, 4, 2, 384, 8, 1.5, 2.0
    rng = np.random.default_rng(41)
    q = rng.standard_normal((B, Hq, T, d)) * 1.5
    k = rng.standard_normal((B, Hkv, T, d))
    v = rng.standard_normal((B, Hkv, T, d))
    G = rng.standard_normal((B, Hq, T, d))
    dq, dk, dv = orc.backward(q, k, v, G, 64, alpha, cs)
    grp = G.reshape(B, Hkv, Hq // Hkv, T, d).sum(axis=(2, 3))
    np.testing.assert_allclose(dv.sum(axis=2), grp, rtol=0, atol=1e-10 * np.abs(G).sum())
    assert np.abs(dk.sum(axis=2)).max() <= 1e-10 * np.abs(dk).sum()
    # the coarse path is active in this case (sparse, non-trivial supports)
    rows = [(0, h, t) for h in range(Hq) for t in range(T)]
    sel = orc.select_rows(q.reshape(-1, d), k, rows, Hq, 64, alpha, cs)
    assert np.any((sel["nsel"] < sel["bt"]) & (sel["nsel"] >= 2))
    pick = [(0, 1, 383), (0, 3, 200), (0, 0, 64), (0, 2, 5)]
    got = orc.backward_dq_rows(q, k, v, G, pick, 64, alpha, cs)
    ref = np.stack([dq[b, h, t] for b, h, t in pick])
    np.testing.assert_array_equal(got, ref)
