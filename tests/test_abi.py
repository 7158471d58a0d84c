"""CPU checks of the C ABI: the library builds, loads, exports every declared symbol, and
rejects bad arguments before touching the GPU (no compute call is made here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dash_attn.h")


@pytest.fixture(scope="module")
def L():
    from sparse_hierarchical_attention_pool_b200 import build, dash_attn
    build.build()
    return dash_attn.lib()


def declared():
    src = open(HEADER).read()
    return re.findall(r"DASH_API\s+[\w\s\*]+?\b(dash_\w+)\s*\(", src)


def test_header_declares_entry_points():
    names = declared()
    for n in ("dash_prefill", "dash_decode", "dash_block_summary", "dash_select_dump",
              "dash_prefill_workspace_size", "dash_decode_workspace_size", "dash_get_device_status"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    from sparse_hierarchical_attention_pool_b200 import dash_attn
    for n in declared():
        assert hasattr(L, n), n
    assert set(declared()) == set(dash_attn.EXPORTS)


def test_status_strings(L):
    for code in range(-7, 1):
        assert L.dash_status_string(code)
    assert L.dash_version() >= 100


def test_workspace_sizes(L):
    from sparse_hierarchical_attention_pool_b200 import dash_attn as da
    n16 = da.prefill_workspace_size(1, 16, 2, 16384, 128)
    assert n16 > 16 * 16384 * 4            # at least the per-row thresholds
    assert L.dash_prefill_workspace_size(1, 16, 2, 16384, 128, 32) == 0     # block must be 64
    assert L.dash_prefill_workspace_size(1, 16, 3, 16384, 128, 64) == 0     # Hq % Hkv
    assert L.dash_prefill_workspace_size(1, 16, 2, 16384, 96, 64) == 0      # d
    assert L.dash_prefill_workspace_size(1, 16, 2, 0, 128, 64) == 0         # T
    assert L.dash_prefill_workspace_size(1, 16, 2, (1 << 20) + 1, 128, 64) == 0
    assert da.decode_workspace_size(8, 32, 8, 98304, 128) > 0
    assert L.dash_decode_workspace_size(8, 64, 1, 1024, 128, 64) == 0       # group of 64 heads


def test_argument_errors_return_before_launch(L):
    f = ctypes.c_void_p
    fake = f(1 << 20)         # aligned, never dereferenced: checks fail first
    big = 1 << 30
    # null pointer
    assert L.dash_prefill(None, fake, fake, fake, 1, 1, 1, 128, 64, 64, 1.5, 1.0, fake, big, None) == -1
    # misaligned pointer
    assert L.dash_prefill(f((1 << 20) + 2), fake, fake, fake, 1, 1, 1, 128, 64, 64, 1.5, 1.0, fake, big, None) == -1
    # alpha <= 1, NaN scale
    assert L.dash_prefill(fake, fake, fake, fake, 1, 1, 1, 128, 64, 64, 1.0, 1.0, fake, big, None) == -1
    assert L.dash_prefill(fake, fake, fake, fake, 1, 1, 1, 128, 64, 64, 1.5, float("nan"), fake, big, None) == -1
    # shapes
    assert L.dash_prefill(fake, fake, fake, fake, 1, 3, 2, 128, 64, 64, 1.5, 1.0, fake, big, None) == -2
    assert L.dash_prefill(fake, fake, fake, fake, 1, 1, 1, 128, 80, 64, 1.5, 1.0, fake, big, None) == -2
    assert L.dash_prefill(fake, fake, fake, fake, 1, 1, 1, 128, 64, 128, 1.5, 1.0, fake, big, None) == -2
    # workspace: null, misaligned, too small
    assert L.dash_prefill(fake, fake, fake, fake, 1, 1, 1, 128, 64, 64, 1.5, 1.0, None, big, None) == -5
    assert L.dash_prefill(fake, fake, fake, fake, 1, 1, 1, 128, 64, 64, 1.5, 1.0, f((1 << 20) + 16), big, None) == -5
    assert L.dash_prefill(fake, fake, fake, fake, 1, 1, 1, 128, 64, 64, 1.5, 1.0, fake, 16, None) == -5
    # decode
    assert L.dash_decode(None, fake, fake, fake, fake, fake, 1, 1, 1, 128, 64, 64, 1.5, 1.0, fake, big, None) == -1
    assert L.dash_decode(fake, fake, fake, fake, fake, fake, 1, 1, 1, 128, 64, 64, 0.5, 1.0, fake, big, None) == -1
    assert L.dash_decode(fake, fake, fake, fake, fake, fake, 1, 1, 1, 128, 64, 64, 1.5, 1.0, fake, 8, None) == -5
    # summary and dump
    assert L.dash_block_summary(None, fake, 1, 1, 128, 64, 64, None) == -1
    assert L.dash_block_summary(fake, fake, 1, 1, 128, 64, 32, None) == -2
    assert L.dash_select_dump(fake, fake, fake, -1, 4, fake, fake, fake, fake, 1, 1, 1, 128, 64, 64,
                              1.5, 1.0, None) == -1
    assert L.dash_get_device_status(None, None) == -1
    # host-buffer prefill: host pointers, shape, device pointers, parameters, workspace
    h = lambda *a: L.dash_prefill_host(*a)
    assert h(None, fake, fake, fake, fake, fake, fake, fake, 1, 2, 1, 128, 64, 64, 1.5, 1.0, fake, big, None) == -1
    assert h(fake, fake, fake, None, fake, fake, fake, fake, 1, 2, 1, 128, 64, 64, 1.5, 1.0, fake, big, None) == -1
    assert h(fake, fake, fake, fake, fake, fake, fake, fake, 1, 3, 2, 128, 64, 64, 1.5, 1.0, fake, big, None) == -2
    assert h(fake, fake, fake, fake, fake, fake, fake, fake, 1, 2, 1, 128, 64, 32, 1.5, 1.0, fake, big, None) == -2
    assert h(fake, fake, fake, fake, None, fake, fake, fake, 1, 2, 1, 128, 64, 64, 1.5, 1.0, fake, big, None) == -1
    assert h(fake, fake, fake, fake, fake, fake, fake, fake, 1, 2, 1, 128, 64, 64, 1.0, 1.0, fake, big, None) == -1
    assert h(fake, fake, fake, fake, fake, fake, fake, fake, 1, 2, 1, 128, 64, 64, 1.5, 1.0, None, big, None) == -5
    assert h(fake, fake, fake, fake, fake, fake, fake, fake, 1, 2, 1, 128, 64, 64, 1.5, 1.0, fake, 16, None) == -5


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    from sparse_hierarchical_attention_pool_b200 import dash_attn as da
    monkeypatch.setattr(da, "_lib", None)
    monkeypatch.setattr(da, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not found"):
        da.lib()


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "sparse_hierarchical_attention_pool_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in src and "from oracle" not in src, fn
                assert "dash_oracle" not in src, fn


def test_backward_workspace_and_argument_errors(L):
    from sparse_hierarchical_attention_pool_b200 import dash_attn as da
    B, Hq, Hkv, T, d = 1, 16, 2, 16384, 128
    fwd = da.prefill_workspace_size(B, Hq, Hkv, T, d)
    bwd = da.prefill_backward_workspace_size(B, Hq, Hkv, T, d)
    # the forward's workspace plus three fp32 values per row (D, log-sum-exp, r)
    assert bwd >= fwd + 3 * B * Hq * T * 4
    assert L.dash_prefill_backward_workspace_size(1, 16, 3, 16384, 128, 64) == 0
    assert L.dash_prefill_backward_workspace_size(1, 16, 2, 16384, 128, 32) == 0
    f = ctypes.c_void_p
    fake = f(1 << 20)
    big = 1 << 30
    args = [fake] * 8 + [1, 2, 1, 256, 64, 64, 1.5, 1.0, fake, big, None]

    def call(**over):
        a = list(args)
        for i, v in over.items():
            a[int(i[1:])] = v
        return L.dash_prefill_backward(*a)

    assert call(a4=None) == -1                        # dout null
    assert call(a7=f((1 << 20) + 8)) == -1            # dv misaligned
    assert call(a14=1.0) == -1                        # alpha <= 1
    assert call(a9=3, a10=2) == -2                    # Hq % Hkv
    assert call(a13=32) == -2                         # block
    assert call(a16=None) == -5                       # workspace null
    assert call(a17=16) == -5                         # workspace too small


def test_backward_binding_rejects_bad_shapes_before_any_call():
    import torch
    from sparse_hierarchical_attention_pool_b200 import dash_attn as da
    q = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        da.dash_prefill_backward(q, k, k[:, :, :64], q, q)          # v shape
    with pytest.raises(ValueError):
        da.dash_prefill_backward(q, k, k, q[:, :1], q)              # out shape
    with pytest.raises(ValueError):
        da.dash_prefill_backward(q, k, k, q, q[..., :32])           # dout shape
    with pytest.raises(ValueError):                                 # CPU tensors: no CPU path
        da.dash_prefill_backward(q, k, k, q, q, workspace=torch.zeros(1 << 20, dtype=torch.uint8))
