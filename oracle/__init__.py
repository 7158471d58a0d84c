"""fp64 CPU oracle for the DashAttention forward pass and its backward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import this package.  The product path (the CUDA library and its
binding) never does, and shares no code with it.

The arithmetic lives in ``dash_oracle.c`` (plain C, fp64, OpenMP over rows); this file
only builds it with gcc and marshals numpy arrays through ctypes.  What each routine
computes, and which page and section define it, is written at the top of the C file.

Inputs are either float32 arrays or bf16 bit patterns (numpy ``uint16``); both are
widened exactly to double inside the oracle.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dash_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libdash_oracle.so")
_lib = None

_i64 = ctypes.c_longlong
_dbl = ctypes.c_double
_ptr = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile dash_oracle.c into libdash_oracle.so next to it (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        L.oracle_entmax_tau.argtypes = [_ptr, _i64, _dbl, ctypes.c_int, _ptr]
        L.oracle_entmax.argtypes = [_ptr, _i64, _dbl, _ptr, _ptr]
        L.oracle_block_summary.argtypes = [_ptr, ctypes.c_int, _i64, _i64, _i64, _i64, _i64, _ptr]
        L.oracle_block_summary_w.argtypes = [_ptr, ctypes.c_int, _ptr, _i64, _i64, _i64, _i64, _i64, _ptr]
        L.oracle_select_rows_w.argtypes = ([_ptr, ctypes.c_int, _ptr, ctypes.c_int, _ptr]
                                           + [_i64] * 6 + [_dbl, _dbl, _ptr, _i64]
                                           + [_ptr] * 5 + [ctypes.c_int])
        L.oracle_forward_rows_w.argtypes = ([_ptr, ctypes.c_int, _ptr, ctypes.c_int, _ptr, ctypes.c_int, _ptr]
                                            + [_i64] * 6 + [_dbl, _dbl, _ptr, _i64]
                                            + [_ptr] * 3 + [ctypes.c_int])
        L.oracle_select_rows.argtypes = ([_ptr, ctypes.c_int, _ptr, ctypes.c_int]
                                         + [_i64] * 6 + [_dbl, _dbl, _ptr, _i64]
                                         + [_ptr] * 5 + [ctypes.c_int])
        L.oracle_forward_rows.argtypes = ([_ptr, ctypes.c_int, _ptr, ctypes.c_int, _ptr, ctypes.c_int]
                                          + [_i64] * 6 + [_dbl, _dbl, _ptr, _i64]
                                          + [_ptr] * 3 + [ctypes.c_int])
        L.oracle_fine_rows_given_p.argtypes = ([_ptr, ctypes.c_int, _ptr, ctypes.c_int, _ptr, ctypes.c_int]
                                               + [_i64] * 6 + [_ptr, _i64, _ptr, _ptr, _ptr, ctypes.c_int])
        L.oracle_dense_causal_rows.argtypes = ([_ptr, ctypes.c_int, _ptr, ctypes.c_int, _ptr, ctypes.c_int]
                                               + [_i64] * 5 + [_ptr, _i64, _ptr, ctypes.c_int])
        L.oracle_forward_rows_agg.argtypes = ([_ptr, ctypes.c_int, _ptr, ctypes.c_int, _ptr, ctypes.c_int, _ptr]
                                              + [_i64] * 6 + [_dbl, _dbl, _ptr, _i64]
                                              + [_ptr] * 2 + [ctypes.c_int])
        L.oracle_backward.argtypes = ([_ptr, ctypes.c_int] * 4 + [_i64] * 6 + [_dbl, _dbl] + [_ptr] * 3)
        L.oracle_backward_dq_rows.argtypes = ([_ptr, ctypes.c_int] * 4 + [_i64] * 6 + [_dbl, _dbl]
                                              + [_ptr, _i64, _ptr, ctypes.c_int])
        for f in (L.oracle_block_summary_w, L.oracle_select_rows_w, L.oracle_forward_rows_w,
                  L.oracle_forward_rows_agg, L.oracle_backward, L.oracle_backward_dq_rows):
            f.restype = ctypes.c_int
        for f in (L.oracle_entmax_tau, L.oracle_entmax, L.oracle_block_summary, L.oracle_select_rows,
                  L.oracle_forward_rows, L.oracle_fine_rows_given_p, L.oracle_dense_causal_rows):
            f.restype = ctypes.c_int
        _lib = L
    return _lib


def _arr(a):
    """numpy view of an element array: (contiguous array, dtype code 0=f32 / 1=bf16 bits /
    2=f64).  float64 inputs stay float64 (finite-difference checks need them)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype == torch.bfloat16:
                return a.view(torch.int16).numpy().view(np.uint16), 1
            a = a.numpy() if a.dtype == torch.float64 else a.float().numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return a, 1
    if a.dtype == np.float64:
        return a, 2
    return np.ascontiguousarray(a, dtype=np.float32), 0


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"oracle {name} failed with code {rc}")


def entmax_tau(s, alpha, method="sort"):
    """Threshold tau (in x = (alpha-1) s space).  method: 'sort', 'bisect' or 'brute'."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    out = np.zeros(1)
    code = {"sort": 0, "bisect": 1, "brute": 2}[method]
    _check(lib().oracle_entmax_tau(_p(s), s.size, float(alpha), code, _p(out)), "entmax_tau")
    return float(out[0])


def entmax(s, alpha):
    """alpha-entmax of a score vector: returns (p, tau)."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    p = np.zeros_like(s)
    tau = np.zeros(1)
    _check(lib().oracle_entmax(_p(s), s.size, float(alpha), _p(p), _p(tau)), "entmax")
    return p, float(tau[0])


def block_summary(k, blk, w=None):
    """Summary of each complete block of keys: k [B, Hkv, T, d] -> [B, Hkv, T // blk, d] fp64.

    w=None: the mean.  w [Hkv, d]: the learned head, attention pooling of the block's keys
    with softmax(w_g . k_i / sqrt(d)) weights ("DashAttention and the year sparse attention
    became a field", section "What alpha-entmax changes", Stage 0)."""
    ka, kdt = _arr(k)
    B, Hkv, T, d = ka.shape
    out = np.zeros((B, Hkv, T // blk, d))
    if w is None:
        _check(lib().oracle_block_summary(_p(ka), kdt, B, Hkv, T, d, blk, _p(out)), "block_summary")
    else:
        wa = _wsum(w, Hkv, d)
        _check(lib().oracle_block_summary_w(_p(ka), kdt, _p(wa), B, Hkv, T, d, blk, _p(out)), "block_summary_w")
    return out


def _wsum(w, Hkv, d):
    wa = np.ascontiguousarray(np.asarray(w, dtype=np.float64))
    if wa.shape != (Hkv, d):
        raise ValueError(f"summary head weights must be [Hkv, d] = [{Hkv}, {d}], got {wa.shape}")
    return wa


def _rows(rows):
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    return r, r.shape[0]


def select_rows(q_rows, k, rows, Hq, blk, alpha, coarse_scale, nthreads=0, w_summary=None):
    """Coarse stage for rows (b, h, t); q_rows [n, d] holds those rows' query vectors.
    w_summary [Hkv, d]: learned summary head (None: mean pooling).

    Returns dict with x [n, nbs], p [n, nbs], tau [n], bt [n], nsel [n]."""
    qa, qdt = _arr(q_rows)
    ka, kdt = _arr(k)
    B, Hkv, Tk, d = ka.shape
    r, n = _rows(rows)
    nbs = Tk // blk
    x = np.zeros((n, nbs))
    p = np.zeros((n, nbs))
    tau = np.zeros(n)
    bt = np.zeros(n, dtype=np.int64)
    ns = np.zeros(n, dtype=np.int64)
    wa = None if w_summary is None else _wsum(w_summary, Hkv, d)
    _check(lib().oracle_select_rows_w(_p(qa), qdt, _p(ka), kdt, None if wa is None else _p(wa),
                                      B, Hq, Hkv, Tk, d, blk,
                                      float(alpha), float(coarse_scale), _p(r), n,
                                      _p(x), _p(p), _p(tau), _p(bt), _p(ns), int(nthreads)),
           "select_rows")
    return {"x": x, "p": p, "tau": tau, "bt": bt, "nsel": ns}


def forward_rows(q_rows, k, v, rows, Hq, blk, alpha, coarse_scale, nthreads=0, w_summary=None):
    """Full forward for rows (b, h, t): returns (out [n, d] fp64, tau [n], nsel [n]).
    w_summary [Hkv, d]: learned summary head (None: mean pooling)."""
    qa, qdt = _arr(q_rows)
    ka, kdt = _arr(k)
    va, vdt = _arr(v)
    B, Hkv, Tk, d = ka.shape
    r, n = _rows(rows)
    out = np.zeros((n, d))
    tau = np.zeros(n)
    ns = np.zeros(n, dtype=np.int64)
    wa = None if w_summary is None else _wsum(w_summary, Hkv, d)
    _check(lib().oracle_forward_rows_w(_p(qa), qdt, _p(ka), kdt, _p(va), vdt, None if wa is None else _p(wa),
                                       B, Hq, Hkv, Tk, d, blk,
                                       float(alpha), float(coarse_scale), _p(r), n,
                                       _p(out), _p(tau), _p(ns), int(nthreads)),
           "forward_rows")
    return out, tau, ns


def forward_rows_agg(q, k, v, rows, blk, alpha, coarse_scale, nthreads=0, w_summary=None):
    """Head-aggregated forward ("DashAttention and the year sparse attention became a field",
    section "Non-dispersive attention at long context": entmax head aggregation) for rows
    (b, h, t): the KV group's heads average their block distributions and share that prior.
    q is the full [B, Hq, T, d] query tensor (every head of a row's group is needed).
    Returns (out [n, d] fp64, nsel [n] = size of the shared support)."""
    import torch
    B, Hq, T, d = q.shape
    ka, kdt = _arr(k)
    va, vdt = _arr(v)
    Hkv, Tk = ka.shape[1], ka.shape[2]
    G = Hq // Hkv
    r, n = _rows(rows)
    rt = torch.as_tensor(r)
    heads = (rt[:, 1] // G * G).unsqueeze(1) + torch.arange(G).unsqueeze(0)          # [n, G]
    qg = q[rt[:, 0].unsqueeze(1), heads, rt[:, 2].unsqueeze(1)]                      # [n, G, d]
    qa, qdt = _arr(qg.contiguous())
    out = np.zeros((n, d))
    ns = np.zeros(n, dtype=np.int64)
    wa = None if w_summary is None else _wsum(w_summary, Hkv, d)
    _check(lib().oracle_forward_rows_agg(_p(qa), qdt, _p(ka), kdt, _p(va), vdt, None if wa is None else _p(wa),
                                         B, Hq, Hkv, Tk, d, blk, float(alpha), float(coarse_scale),
                                         _p(r), n, _p(out), _p(ns), int(nthreads)),
           "forward_rows_agg")
    return out, ns


def backward(q, k, v, dout, blk, alpha, coarse_scale):
    """Gradients (dq, dk, dv) in fp64 of a scalar loss with d loss / d out = dout, through
    the whole forward: fine softmax, log prior, alpha-entmax (its Jacobian on the support),
    coarse scores and mean summaries.  Every row of the [B, Hq, T, d] problem."""
    qa, qdt = _arr(q)
    ka, kdt = _arr(k)
    va, vdt = _arr(v)
    ga, gdt = _arr(dout)
    B, Hq, T, d = qa.shape
    Hkv = ka.shape[1]
    dq = np.zeros((B, Hq, T, d))
    dk = np.zeros((B, Hkv, T, d))
    dv = np.zeros((B, Hkv, T, d))
    _check(lib().oracle_backward(_p(qa), qdt, _p(ka), kdt, _p(va), vdt, _p(ga), gdt, B, Hq, Hkv, T, d, blk,
                                 float(alpha), float(coarse_scale), _p(dq), _p(dk), _p(dv)), "backward")
    return dq, dk, dv


def backward_dq_rows(q, k, v, dout, rows, blk, alpha, coarse_scale, nthreads=0):
    """dq (fp64 [n, d]) of the listed rows (b, h, t) alone: each row's dq depends only on its
    own forward, so full-size problems can be checked on a sample.  q, dout: [B, Hq, T, d]."""
    qa, qdt = _arr(q)
    ka, kdt = _arr(k)
    va, vdt = _arr(v)
    ga, gdt = _arr(dout)
    B, Hq, T, d = qa.shape
    Hkv = ka.shape[1]
    r, n = _rows(rows)
    out = np.zeros((n, d))
    _check(lib().oracle_backward_dq_rows(_p(qa), qdt, _p(ka), kdt, _p(va), vdt, _p(ga), gdt, B, Hq, Hkv, T, d, blk,
                                         float(alpha), float(coarse_scale), _p(r), n, _p(out), int(nthreads)),
           "backward_dq_rows")
    return out


def fine_rows_given_p(q_rows, k, v, rows, Hq, blk, w_rows, w_diag, nthreads=0):
    """Fine stage with injected block weights w_rows [n, T // blk] and w_diag [n]."""
    qa, qdt = _arr(q_rows)
    ka, kdt = _arr(k)
    va, vdt = _arr(v)
    B, Hkv, Tk, d = ka.shape
    r, n = _rows(rows)
    w = np.ascontiguousarray(w_rows, dtype=np.float64).reshape(n, Tk // blk)
    wd = np.ascontiguousarray(w_diag, dtype=np.float64).reshape(n)
    out = np.zeros((n, d))
    _check(lib().oracle_fine_rows_given_p(_p(qa), qdt, _p(ka), kdt, _p(va), vdt, B, Hq, Hkv, Tk, d, blk,
                                          _p(r), n, _p(w), _p(wd), _p(out), int(nthreads)),
           "fine_rows_given_p")
    return out


def dense_causal_rows(q_rows, k, v, rows, Hq, nthreads=0):
    """Plain causal softmax attention for rows (b, h, t) over tokens 0..t."""
    qa, qdt = _arr(q_rows)
    ka, kdt = _arr(k)
    va, vdt = _arr(v)
    B, Hkv, Tk, d = ka.shape
    r, n = _rows(rows)
    out = np.zeros((n, d))
    _check(lib().oracle_dense_causal_rows(_p(qa), qdt, _p(ka), kdt, _p(va), vdt, B, Hq, Hkv, Tk, d,
                                          _p(r), n, _p(out), int(nthreads)),
           "dense_causal_rows")
    return out


def gather_q_rows(q, rows):
    """Query vectors of rows (b, h, t) from q [B, Hq, T, d] (no arithmetic, a gather)."""
    import torch
    r = torch.as_tensor(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    return q[r[:, 0], r[:, 1], r[:, 2]]
