"""Thin Python binding over libdash_attn.so (the C ABI of include/dash_attn.h).

Every function here only checks tensors and marshals pointers; all computation runs in
the library's CUDA kernels on the current torch stream.  There is no CPU fallback: when
the library is missing or fails to load, the first call raises.

Tensor conventions follow the header: bf16, contiguous, q/out [B, Hq, T, d], k/v
[B, Hkv, T, d], caches [B, Hkv, Tmax, d], block summaries fp32 [B, Hkv, T // 64, d].
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdash_attn.so")

DASH_OK = 0
STATUS = {0: "DASH_OK", -1: "DASH_ERR_ARG", -2: "DASH_ERR_SHAPE", -3: "DASH_ERR_DTYPE",
          -4: "DASH_ERR_UNSUPPORTED", -5: "DASH_ERR_WORKSPACE", -6: "DASH_ERR_CUDA",
          -7: "DASH_ERR_NO_CONVERGE", -8: "DASH_ERR_SCRATCH_LIMIT",
          -9: "DASH_ERR_DEVICE_TIMEOUT", -10: "DASH_ERR_SETUP_IN_CAPTURE"}

EXPORTS = ("dash_status_string", "dash_version", "dash_block_summary", "dash_prefill_workspace_size",
           "dash_prefill", "dash_prefill_host", "dash_prefill_stats", "dash_decode_stats",
           "dash_prefill_tau", "dash_select_dump", "dash_decode_workspace_size", "dash_decode",
           "dash_get_device_status", "dash_prefill_profiled", "dash_decode_profiled",
           "dash_decode_noalloc", "dash_decode_noalloc_status", "dash_block_summary_w", "dash_prefill_w", "dash_prefill_ex",
           "dash_decode_ex", "dash_prefill_backward_workspace_size", "dash_prefill_backward",
           "dash_prefill_dump", "dash_decode_dump")

HEAD_AGGREGATION = 1       # flag of dash_prefill_ex / dash_decode_ex


class DashError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")


class dash_stats(ctypes.Structure):
    _fields_ = [("scored_pairs", ctypes.c_longlong), ("selected_pairs", ctypes.c_longlong),
                ("union_blocks", ctypes.c_longlong), ("tiles", ctypes.c_longlong),
                ("status", ctypes.c_int), ("fine_steps", ctypes.c_longlong)]


_lib = None
_i = ctypes.c_int
_f = ctypes.c_float
_p = ctypes.c_void_p
_sz = ctypes.c_size_t


def lib():
    """Load libdash_attn.so (raises if it is missing: there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libdash_attn.so not found at {LIB_PATH}; build it with "
                           "`python -m sparse_hierarchical_attention_pool_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    L.dash_status_string.restype = ctypes.c_char_p
    L.dash_status_string.argtypes = [_i]
    L.dash_version.restype = _i
    L.dash_block_summary.argtypes = [_p, _p, _i, _i, _i, _i, _i, _p]
    L.dash_block_summary_w.argtypes = [_p, _p, _p, _i, _i, _i, _i, _i, _p]
    L.dash_prefill_w.argtypes = [_p] * 5 + [_i] * 6 + [_f, _f, _p, _sz, _p]
    L.dash_prefill_ex.argtypes = [_p] * 5 + [_i] * 6 + [_f, _f, ctypes.c_uint, _p, _sz, _p]
    L.dash_decode_ex.argtypes = [_p] * 6 + [_i] * 6 + [_f, _f, ctypes.c_uint, _p, _sz, _p]
    L.dash_prefill_workspace_size.argtypes = [_i] * 6
    L.dash_prefill_workspace_size.restype = _sz
    L.dash_prefill_backward_workspace_size.argtypes = [_i] * 6
    L.dash_prefill_backward_workspace_size.restype = _sz
    L.dash_prefill_backward.argtypes = [_p] * 8 + [_i] * 6 + [_f, _f, _p, _sz, _p]
    L.dash_prefill.argtypes = [_p] * 4 + [_i] * 6 + [_f, _f, _p, _sz, _p]
    L.dash_prefill_host.argtypes = [_p] * 8 + [_i] * 6 + [_f, _f, _p, _sz, _p]
    L.dash_prefill_stats.argtypes = [_p, _sz, ctypes.POINTER(dash_stats), _p]
    L.dash_decode_stats.argtypes = [_p, _sz, ctypes.POINTER(dash_stats), _p]
    L.dash_prefill_tau.argtypes = [_p, _sz, _p] + [_i] * 6 + [_p]
    L.dash_select_dump.argtypes = [_p, _p, _p, _i, _i, _p, _p, _p, _p] + [_i] * 6 + [_f, _f, _p]
    L.dash_decode_workspace_size.argtypes = [_i] * 6
    L.dash_decode_workspace_size.restype = _sz
    L.dash_decode.argtypes = [_p] * 6 + [_i] * 6 + [_f, _f, _p, _sz, _p]
    L.dash_get_device_status.argtypes = [_p, _p]
    L.dash_prefill_profiled.argtypes = [_p] * 4 + [_i] * 6 + [_f, _f, _p, _sz, _p, _p]
    L.dash_decode_profiled.argtypes = [_p] * 6 + [_i] * 6 + [_f, _f, _p, _sz, _p, _p]
    L.dash_decode_noalloc.argtypes = [_p] * 6 + [_i] * 6 + [_f, _f, _p]
    L.dash_decode_noalloc_status.argtypes = [_p]
    L.dash_prefill_dump.argtypes = [_p] * 5 + [_i] * 6 + [_f, _f, ctypes.c_uint, _p, _i, _p, _p, _p, _sz, _p]
    L.dash_decode_dump.argtypes = [_p] * 6 + [_i] * 6 + [_f, _f, ctypes.c_uint, _p, _p, _p, _p, _sz, _p]
    for name in EXPORTS:
        if name not in ("dash_status_string", "dash_prefill_workspace_size", "dash_decode_workspace_size",
                        "dash_prefill_backward_workspace_size"):
            getattr(L, name).restype = _i
    _lib = L
    return L


def _check(fn, rc):
    if rc != DASH_OK:
        raise DashError(fn, rc)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def version() -> int:
    return lib().dash_version()


def dash_block_summary(k, ksum=None, block=64, stream=None):
    """Mean of every complete 64-key block: k [B, Hkv, T, d] -> ksum fp32 [B, Hkv, T // 64, d]."""
    B, Hkv, T, d = k.shape
    if ksum is None:
        ksum = torch.empty(B, Hkv, max(T // block, 1), d, device=k.device, dtype=torch.float32)
    _check("dash_block_summary", lib().dash_block_summary(
        _dev(k, torch.bfloat16, "k"), _dev(ksum, torch.float32, "ksum"), B, Hkv, T, d, block, _stream(stream)))
    return ksum


def dash_block_summary_w(k, w, ksum=None, block=64, stream=None):
    """Learned-head summaries: k [B, Hkv, T, d], w fp32 [Hkv, d] -> ksum fp32 [B, Hkv, T // 64, d]."""
    B, Hkv, T, d = k.shape
    if tuple(w.shape) != (Hkv, d):
        raise ValueError("w must be [Hkv, d]")
    if ksum is None:
        ksum = torch.empty(B, Hkv, max(T // block, 1), d, device=k.device, dtype=torch.float32)
    _check("dash_block_summary_w", lib().dash_block_summary_w(
        _dev(k, torch.bfloat16, "k"), _dev(w, torch.float32, "w"), _dev(ksum, torch.float32, "ksum"),
        B, Hkv, T, d, block, _stream(stream)))
    return ksum


def prefill_workspace_size(B, Hq, Hkv, T, d, block=64) -> int:
    n = lib().dash_prefill_workspace_size(B, Hq, Hkv, T, d, block)
    if n == 0:
        raise DashError("dash_prefill_workspace_size", -2)
    return n


def prefill_backward_workspace_size(B, Hq, Hkv, T, d, block=64) -> int:
    n = lib().dash_prefill_backward_workspace_size(B, Hq, Hkv, T, d, block)
    if n == 0:
        raise DashError("dash_prefill_backward_workspace_size", -2)
    return n


def decode_workspace_size(B, Hq, Hkv, Tmax, d, block=64) -> int:
    n = lib().dash_decode_workspace_size(B, Hq, Hkv, Tmax, d, block)
    if n == 0:
        raise DashError("dash_decode_workspace_size", -2)
    return n


def alloc_workspace(nbytes, device="cuda"):
    """A 256-byte aligned uint8 device buffer (torch's caching allocator aligns to 512)."""
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    assert ws.data_ptr() % 256 == 0
    return ws


def dash_prefill(q, k, v, out=None, alpha=1.5, coarse_scale=1.0, workspace=None, block=64, stream=None):
    """Causal DashAttention prefill.  Returns (out, workspace)."""
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, T, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, T, d] matching q")
    if out is None:
        out = torch.empty_like(q)
    need = prefill_workspace_size(B, Hq, Hkv, T, d, block)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    rc = lib().dash_prefill(_dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"),
                            _dev(v, torch.bfloat16, "v"), _dev(out, torch.bfloat16, "out"),
                            B, Hq, Hkv, T, d, block, float(alpha), float(coarse_scale),
                            ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream(stream))
    _check("dash_prefill", rc)
    return out, workspace


def dash_prefill_w(q, k, v, w_summary, out=None, alpha=1.5, coarse_scale=1.0, workspace=None, block=64,
                   stream=None):
    """dash_prefill with a learned summary head w_summary fp32 [Hkv, d] (None: mean pooling)."""
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, T, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, T, d] matching q")
    if w_summary is not None and tuple(w_summary.shape) != (Hkv, d):
        raise ValueError("w_summary must be [Hkv, d]")
    if out is None:
        out = torch.empty_like(q)
    need = prefill_workspace_size(B, Hq, Hkv, T, d, block)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    wp = None if w_summary is None else _dev(w_summary, torch.float32, "w_summary")
    rc = lib().dash_prefill_w(_dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"),
                              _dev(v, torch.bfloat16, "v"), wp, _dev(out, torch.bfloat16, "out"),
                              B, Hq, Hkv, T, d, block, float(alpha), float(coarse_scale),
                              ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream(stream))
    _check("dash_prefill_w", rc)
    return out, workspace


def dash_prefill_ex(q, k, v, w_summary=None, flags=0, out=None, alpha=1.5, coarse_scale=1.0, workspace=None,
                    block=64, stream=None):
    """dash_prefill with options: learned summary head w_summary [Hkv, d] (None: mean) and
    flags (HEAD_AGGREGATION)."""
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, T, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, T, d] matching q")
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(prefill_workspace_size(B, Hq, Hkv, T, d, block), q.device)
    wp = None if w_summary is None else _dev(w_summary, torch.float32, "w_summary")
    rc = lib().dash_prefill_ex(_dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"),
                               _dev(v, torch.bfloat16, "v"), wp, _dev(out, torch.bfloat16, "out"),
                               B, Hq, Hkv, T, d, block, float(alpha), float(coarse_scale), int(flags),
                               ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream(stream))
    _check("dash_prefill_ex", rc)
    return out, workspace


def dash_decode_ex(q, k_cache, v_cache, ksum, kv_len, flags=0, out=None, alpha=1.5, coarse_scale=1.0,
                   workspace=None, block=64, stream=None):
    """dash_decode with flags (HEAD_AGGREGATION)."""
    B, Hq, d = q.shape
    Hkv, Tmax = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(decode_workspace_size(B, Hq, Hkv, Tmax, d, block), q.device)
    rc = lib().dash_decode_ex(_dev(q, torch.bfloat16, "q"), _dev(k_cache, torch.bfloat16, "k_cache"),
                              _dev(v_cache, torch.bfloat16, "v_cache"), _dev(ksum, torch.float32, "ksum"),
                              _dev(kv_len, torch.int32, "kv_len"), _dev(out, torch.bfloat16, "out"),
                              B, Hq, Hkv, Tmax, d, block, float(alpha), float(coarse_scale), int(flags),
                              ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream(stream))
    _check("dash_decode_ex", rc)
    return out, workspace


def _events(evs):
    for e in evs:
        if e.cuda_event == 0:      # torch creates the CUDA event on its first record
            e.record()
    return (ctypes.c_void_p * len(evs))(*[ctypes.c_void_p(e.cuda_event) for e in evs])


def dash_prefill_profiled(q, k, v, out, alpha, coarse_scale, workspace, events, block=64, stream=None):
    """dash_prefill recording torch.cuda.Event objects events[0..3] around its three kernels."""
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    rc = lib().dash_prefill_profiled(_dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"),
                                     _dev(v, torch.bfloat16, "v"), _dev(out, torch.bfloat16, "out"),
                                     B, Hq, Hkv, T, d, block, float(alpha), float(coarse_scale),
                                     ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream(stream),
                                     _events(events))
    _check("dash_prefill_profiled", rc)
    return out


def dash_decode_profiled(q, k_cache, v_cache, ksum, kv_len, out, alpha, coarse_scale, workspace, events,
                         block=64, stream=None):
    """dash_decode recording torch.cuda.Event objects events[0..3]: before the coarse kernels,
    before the attention kernel, after it, and after the merge kernel (if any)."""
    B, Hq, d = q.shape
    Hkv, Tmax = k_cache.shape[1], k_cache.shape[2]
    rc = lib().dash_decode_profiled(_dev(q, torch.bfloat16, "q"), _dev(k_cache, torch.bfloat16, "k_cache"),
                                    _dev(v_cache, torch.bfloat16, "v_cache"), _dev(ksum, torch.float32, "ksum"),
                                    _dev(kv_len, torch.int32, "kv_len"), _dev(out, torch.bfloat16, "out"),
                                    B, Hq, Hkv, Tmax, d, block, float(alpha), float(coarse_scale),
                                    ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream(stream),
                                    _events(events))
    _check("dash_decode_profiled", rc)
    return out


def dash_prefill_host(q_host, k_host, v_host, out_host, q_dev, k_dev, v_dev, out_dev, alpha, coarse_scale,
                      workspace, block=64, stream=None):
    """Prefill from host tensors (pinned for overlap): H2D copies, prefill, D2H copy, async."""
    B, Hq, T, d = q_dev.shape
    Hkv = k_dev.shape[1]
    for name, t in (("q_host", q_host), ("k_host", k_host), ("v_host", v_host), ("out_host", out_host)):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 host tensor")
    rc = lib().dash_prefill_host(
        ctypes.c_void_p(q_host.data_ptr()), ctypes.c_void_p(k_host.data_ptr()),
        ctypes.c_void_p(v_host.data_ptr()), ctypes.c_void_p(out_host.data_ptr()),
        _dev(q_dev, torch.bfloat16, "q_dev"), _dev(k_dev, torch.bfloat16, "k_dev"),
        _dev(v_dev, torch.bfloat16, "v_dev"), _dev(out_dev, torch.bfloat16, "out_dev"),
        B, Hq, Hkv, T, d, block, float(alpha), float(coarse_scale),
        ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream(stream))
    _check("dash_prefill_host", rc)
    return out_host


def _stats(fn, workspace, stream):
    st = dash_stats()
    _check(fn, getattr(lib(), fn)(ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
                                  ctypes.byref(st), _stream(stream)))
    return {f: getattr(st, f) for f, _ in dash_stats._fields_}


def dash_prefill_stats(workspace, stream=None):
    return _stats("dash_prefill_stats", workspace, stream)


def dash_decode_stats(workspace, stream=None):
    return _stats("dash_decode_stats", workspace, stream)


def dash_prefill_tau(workspace, B, Hq, Hkv, T, d, block=64, stream=None):
    tau = torch.empty(B, Hq, T, device=workspace.device, dtype=torch.float32)
    _check("dash_prefill_tau", lib().dash_prefill_tau(
        ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), ctypes.c_void_p(tau.data_ptr()),
        B, Hq, Hkv, T, d, block, _stream(stream)))
    return tau


def dash_select_dump(q, ksum, rows, max_sel, alpha, coarse_scale, Hkv, block=64, stream=None):
    """Selected blocks, weights, support size and tau of rows (b, h, t) [n, 3] int64."""
    B, Hq, T, d = q.shape
    rows = torch.as_tensor(rows, dtype=torch.int64, device=q.device).reshape(-1, 3).contiguous()
    n = rows.shape[0]
    idx = torch.full((n, max(max_sel, 1)), -1, dtype=torch.int32, device=q.device)
    p = torch.zeros((n, max(max_sel, 1)), dtype=torch.float32, device=q.device)
    cnt = torch.zeros(n, dtype=torch.int32, device=q.device)
    tau = torch.zeros(n, dtype=torch.float32, device=q.device)
    _check("dash_select_dump", lib().dash_select_dump(
        _dev(q, torch.bfloat16, "q"), _dev(ksum, torch.float32, "ksum"), ctypes.c_void_p(rows.data_ptr()),
        n, max_sel, ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(p.data_ptr()),
        ctypes.c_void_p(cnt.data_ptr()), ctypes.c_void_p(tau.data_ptr()),
        B, Hq, Hkv, T, d, block, float(alpha), float(coarse_scale), _stream(stream)))
    return idx, p, cnt, tau


def dash_decode(q, k_cache, v_cache, ksum, kv_len, out=None, alpha=1.5, coarse_scale=1.0,
                workspace=None, block=64, stream=None):
    """One decode step.  q [B, Hq, d]; caches [B, Hkv, Tmax, d]; kv_len int32 [B] (device)."""
    B, Hq, d = q.shape
    Hkv, Tmax = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    need = decode_workspace_size(B, Hq, Hkv, Tmax, d, block)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    rc = lib().dash_decode(_dev(q, torch.bfloat16, "q"), _dev(k_cache, torch.bfloat16, "k_cache"),
                           _dev(v_cache, torch.bfloat16, "v_cache"), _dev(ksum, torch.float32, "ksum"),
                           _dev(kv_len, torch.int32, "kv_len"), _dev(out, torch.bfloat16, "out"),
                           B, Hq, Hkv, Tmax, d, block, float(alpha), float(coarse_scale),
                           ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream(stream))
    _check("dash_decode", rc)
    return out, workspace


def dash_decode_noalloc(q, k_cache, v_cache, ksum, kv_len, out=None, alpha=1.5, coarse_scale=1.0,
                        block=64, stream=None):
    """dash_decode on the library's fixed 32 MiB device scratch array, for callers that cannot
    allocate device memory where they decode (real-time loops that must not synchronise the
    device through cudaMalloc / cudaFree, memory owned by a foreign allocator).  No
    workspace; calls that overlap on the GPU race on the shared array.  The device status
    of the call is read with dash_decode_noalloc_status."""
    B, Hq, d = q.shape
    Hkv, Tmax = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    rc = lib().dash_decode_noalloc(_dev(q, torch.bfloat16, "q"), _dev(k_cache, torch.bfloat16, "k_cache"),
                                   _dev(v_cache, torch.bfloat16, "v_cache"), _dev(ksum, torch.float32, "ksum"),
                                   _dev(kv_len, torch.int32, "kv_len"), _dev(out, torch.bfloat16, "out"),
                                   B, Hq, Hkv, Tmax, d, block, float(alpha), float(coarse_scale), _stream(stream))
    _check("dash_decode_noalloc", rc)
    return out


def dash_prefill_dump(q, k, v, rows, alpha=1.5, coarse_scale=1.0, w_summary=None, flags=0, out=None,
                      workspace=None, block=64, stream=None):
    """dash_prefill plus the weights its fine stage applied to the listed rows.

    rows: sequence of (b, h, t).  Returns (out, workspace, x, p) with x, p fp32
    [len(rows), T // 64]: x_j of every block in the row's tile list (NaN when not listed)
    and the applied weight p_j (0 when not selected or not listed)."""
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(prefill_workspace_size(B, Hq, Hkv, T, d, block), q.device)
    # one slot per distinct row (a slot has one writer); repeated rows share their slot's dump
    r = torch.as_tensor([list(x) for x in rows], dtype=torch.long).reshape(-1, 3)
    uniq, inv = torch.unique((r[:, 0] * Hq + r[:, 1]) * T + r[:, 2], return_inverse=True)
    slot = torch.full((B * Hq * T,), -1, dtype=torch.int32)
    slot[uniq] = torch.arange(len(uniq), dtype=torch.int32)
    slot = slot.to(q.device)
    nbs = T // block
    x = torch.empty(max(len(uniq), 1), max(nbs, 1), dtype=torch.float32, device=q.device)
    p = torch.empty_like(x)
    wp = _dev(w_summary, torch.float32, "w_summary") if w_summary is not None else None
    rc = lib().dash_prefill_dump(_dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"),
                                 _dev(v, torch.bfloat16, "v"), wp, _dev(out, torch.bfloat16, "out"),
                                 B, Hq, Hkv, T, d, block, float(alpha), float(coarse_scale), int(flags),
                                 _dev(slot, torch.int32, "row_slot"), len(uniq), _dev(x, torch.float32, "x"),
                                 _dev(p, torch.float32, "p"), ctypes.c_void_p(workspace.data_ptr()),
                                 workspace.numel(), _stream(stream))
    _check("dash_prefill_dump", rc)
    idx = inv.to(q.device)
    return out, workspace, x[:, :nbs][idx], p[:, :nbs][idx]


def dash_decode_dump(q, k_cache, v_cache, ksum, kv_len, alpha=1.5, coarse_scale=1.0, flags=0, out=None,
                     workspace=None, block=64, stream=None):
    """dash_decode plus the weights its attention kernel applied.  Returns (out, workspace,
    x, p, tau): x, p fp32 [B, Hq, Tmax // 64] (NaN / 0 for blocks outside the group's list),
    tau fp32 [B, Hq]."""
    B, Hq, d = q.shape
    Hkv, Tmax = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(decode_workspace_size(B, Hq, Hkv, Tmax, d, block), q.device)
    nbs = Tmax // block
    x = torch.empty(B, Hq, max(nbs, 1), dtype=torch.float32, device=q.device)
    p = torch.empty_like(x)
    tau = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    rc = lib().dash_decode_dump(_dev(q, torch.bfloat16, "q"), _dev(k_cache, torch.bfloat16, "k_cache"),
                                _dev(v_cache, torch.bfloat16, "v_cache"), _dev(ksum, torch.float32, "ksum"),
                                _dev(kv_len, torch.int32, "kv_len"), _dev(out, torch.bfloat16, "out"),
                                B, Hq, Hkv, Tmax, d, block, float(alpha), float(coarse_scale), int(flags),
                                _dev(x, torch.float32, "x"), _dev(p, torch.float32, "p"),
                                _dev(tau, torch.float32, "tau"), ctypes.c_void_p(workspace.data_ptr()),
                                workspace.numel(), _stream(stream))
    _check("dash_decode_dump", rc)
    return out, workspace, x[:, :, :nbs], p[:, :, :nbs], tau


def dash_decode_noalloc_status(stream=None) -> int:
    """Device status of the last dash_decode_noalloc on the current device (syncs the stream)."""
    return lib().dash_decode_noalloc_status(_stream(stream))


def dash_get_device_status(workspace, stream=None) -> int:
    return lib().dash_get_device_status(ctypes.c_void_p(workspace.data_ptr()), _stream(stream))


def dash_prefill_backward(q, k, v, out, dout, alpha=1.5, coarse_scale=1.0, dq=None, dk=None, dv=None,
                          workspace=None, block=64, stream=None):
    """Gradients of dash_prefill: (dq, dk, dv) for d loss / d out = dout.  `out` is the
    forward's output for (q, k, v, alpha, coarse_scale)."""
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, T, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, T, d] matching q")
    if out.shape != q.shape or dout.shape != q.shape:
        raise ValueError("out and dout must be [B, Hq, T, d]")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = prefill_backward_workspace_size(B, Hq, Hkv, T, d, block)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    rc = lib().dash_prefill_backward(
        _dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"), _dev(v, torch.bfloat16, "v"),
        _dev(out, torch.bfloat16, "out"), _dev(dout, torch.bfloat16, "dout"), _dev(dq, torch.bfloat16, "dq"),
        _dev(dk, torch.bfloat16, "dk"), _dev(dv, torch.bfloat16, "dv"), B, Hq, Hkv, T, d, block,
        float(alpha), float(coarse_scale), ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
        _stream(stream))
    _check("dash_prefill_backward", rc)
    return dq, dk, dv


class DashAttentionFunction(torch.autograd.Function):
    """torch.autograd binding of dash_prefill / dash_prefill_backward (mean summaries, per-head
    priors).  The forward saves q, k, v and the output; the backward recomputes the coarse
    stage and the statistics inside dash_prefill_backward."""

    @staticmethod
    def forward(ctx, q, k, v, alpha, coarse_scale):
        out, _ = dash_prefill(q, k, v, alpha=alpha, coarse_scale=coarse_scale)
        ctx.save_for_backward(q, k, v, out)
        ctx.alpha, ctx.coarse_scale = float(alpha), float(coarse_scale)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out = ctx.saved_tensors
        dq, dk, dv = dash_prefill_backward(q, k, v, out, dout.to(torch.bfloat16).contiguous(),
                                           alpha=ctx.alpha, coarse_scale=ctx.coarse_scale)
        return dq, dk, dv, None, None


def dash_attention(q, k, v, alpha=1.5, coarse_scale=1.0):
    """Differentiable causal DashAttention prefill: out [B, Hq, T, d] from bf16 q [B, Hq, T, d]
    and k, v [B, Hkv, T, d]; gradients reach q, k and v through the fine softmax, the log
    prior, the alpha-entmax selection and the block summaries."""
    return DashAttentionFunction.apply(q, k, v, alpha, coarse_scale)

