"""Host-only checks of the C ABI: the library builds, loads, exports every call
include/tokengate.h declares, and rejects bad arguments before any launch.
No GPU is needed: every case here fails validation before the first CUDA call."""
import ctypes
import os
import re

import pytest

from learned_token_pruning_mlp_b200 import build as tgbuild
from learned_token_pruning_mlp_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tokengate.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tg_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    tgbuild.build()
    return _lib.lib()


def test_header_declares_the_four_calls():
    names = _declared()
    for must in ("tg_gate_score", "tg_select_topk", "tg_gather", "tg_gated_attention",
                 "tg_select_topk_varlen", "tg_gated_attention_varlen", "tg_get_device_error"):
        assert must in names


def test_every_declared_symbol_is_exported(L):
    missing = [n for n in _declared() if not hasattr(L, n)]
    assert not missing, missing


def test_library_exports_only_the_declared_calls(L):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if ln.strip()}
    assert exported == set(_declared()), exported ^ set(_declared())


def test_binding_covers_every_declared_symbol():
    assert set(_declared()) <= set(_lib._SIGNATURES)


def test_abi_version_and_status_strings(L):
    assert L.tg_abi_version() == 1
    assert L.tg_status_string(0) == b"TG_OK"
    assert L.tg_status_string(3) == b"TG_ERR_ALIGNMENT"
    assert L.tg_status_string(99) == b"TG_ERR_UNKNOWN"


def _detail(L):
    return L.tg_last_error_detail().decode()


def test_gate_rejects_bad_shapes(L):
    assert L.tg_gate_score(None, 10, 7, None, None, None, None, 64, None, None) == 1          # d % 8
    assert "multiple of 8" in _detail(L)
    assert L.tg_gate_score(None, -1, 64, None, None, None, None, 64, None, None) == 1         # n < 0
    assert L.tg_gate_score(None, 10, 64, None, None, None, None, 48 + 1, None, None) == 2     # h % 16
    assert L.tg_gate_score(None, 10, 64, None, None, None, None, 512, None, None) == 2         # h > 256
    assert L.tg_gate_score(None, 0, 64, None, None, None, None, 64, None, None) == 0          # n = 0: no-op
    assert L.tg_gate_score(None, 10, 64, None, None, None, None, 64, None, None) == 1         # null pointers
    p = ctypes.c_void_p(16 * 1000 + 2)                                                         # misaligned
    assert L.tg_gate_score(p, 10, 64, p, p, p, p, 64, p, None) == 3


def test_topk_rejects_bad_arguments(L):
    one = ctypes.c_void_p(4096)
    assert L.tg_select_topk(one, one, -1, 5, one, 10, one, None) == 1
    assert L.tg_select_topk(one, one, 1 << 31, 5, one, 10, one, None) == 1
    assert L.tg_select_topk(one, one, 10, -1, one, 10, one, None) == 1
    assert L.tg_select_topk(one, one, 10, 5, one, 10, None, None) == 1
    assert L.tg_select_topk(None, one, 10, 5, one, 10, one, None) == 1
    assert L.tg_select_topk_varlen(one, one, one, -1, 10, one, 5, one, 10, one, None) == 1
    assert L.tg_select_topk_varlen(one, one, one, 2, 10, one, 11, one, 10, one, None) == 1  # max_seqlen > total
    assert L.tg_select_topk_varlen(one, one, None, 2, 10, one, 5, one, 10, one, None) == 1


def test_gather_rejects_bad_arguments(L):
    p = ctypes.c_void_p(4096)
    assert L.tg_gather(p, 10, 12, p, 4, None, p, None, None, None) == 1                    # d % 8
    assert L.tg_gather(p, 10, 32768, p, 4, None, p, None, None, None) == 2                 # d too large
    assert L.tg_gather(p, 10, 16, p, 4, None, p, p, None, None) == 1                       # scores without s_k
    assert L.tg_gather(p, 10, 16, p, 0, None, p, None, None, None) == 0                    # nothing to do
    assert L.tg_gather(ctypes.c_void_p(4100), 10, 16, p, 4, None, p, None, None, None) == 3


def test_attention_rejects_bad_arguments(L):
    p = ctypes.c_void_p(4096)
    f = ctypes.c_float(1.0)
    assert L.tg_gated_attention(p, p, p, p, p, f, 10, 6, 4, 128, p, None) == 1             # Hq % Hkv
    assert L.tg_gated_attention(p, p, p, p, p, f, 10, 4, 2, 96, p, None) == 2              # D
    assert L.tg_gated_attention(p, p, p, p, p, ctypes.c_float(float("inf")), 10, 4, 2, 64, p, None) == 1
    assert L.tg_gated_attention(p, p, p, p, p, f, 0, 4, 2, 64, p, None) == 0               # S = 0
    assert L.tg_gated_attention(p, p, p, p, None, f, 10, 4, 2, 64, p, None) == 1            # scores without gain
    assert L.tg_gated_attention(ctypes.c_void_p(4104), p, p, p, p, f, 10, 4, 2, 64, p, None) == 3
    assert L.tg_gated_attention_varlen(p, p, p, p, p, f, None, 2, 10, 5, 4, 2, 64, p, None) == 1
    assert L.tg_gated_attention_varlen(p, p, p, p, p, f, p, 2, 10, 11, 4, 2, 64, p, None) == 1


def test_projections_reject_bad_arguments(L):
    p = ctypes.c_void_p(4096)
    f = ctypes.c_float(1e-6)
    b = ctypes.c_double(1e6)
    assert L.tg_linear(p, 10, 12, p, 64, None, p, None) == 2                               # K % 8
    assert L.tg_linear(p, 10, 16, p, 48, None, p, None) == 2                               # N % 32
    assert L.tg_linear(p, -1, 16, p, 64, None, p, None) == 1
    assert L.tg_linear(p, 0, 16, p, 64, None, p, None) == 0                                # M = 0: no-op
    assert L.tg_linear(None, 10, 16, p, 64, None, p, None) == 1
    assert L.tg_linear(p, 10, 16, p, 64, ctypes.c_void_p(4098), p, None) == 3              # residual misaligned
    assert L.tg_qkv_rope(p, 10, 64, p, p, b, None, None, f, 4, 2, 96, p, p, p, None) == 2  # D
    assert L.tg_qkv_rope(p, 10, 60, p, p, b, None, None, f, 4, 2, 64, p, p, p, None) == 2  # d % 8
    assert L.tg_qkv_rope(p, 10, 64, p, p, ctypes.c_double(1.0), None, None, f, 4, 2, 64, p, p, p, None) == 1
    assert L.tg_qkv_rope(p, 10, 64, p, p, b, None, None, ctypes.c_float(-1.0), 4, 2, 64, p, p, p, None) == 1
    assert L.tg_qkv_rope(p, 10, 64, p, None, b, None, None, f, 4, 2, 64, p, p, p, None) == 1
    assert L.tg_qkv_rope(p, 0, 64, p, p, b, None, None, f, 4, 2, 64, p, p, p, None) == 0   # S = 0
    assert L.tg_qkv_rope(p, 10, 64, p, p, b, None, None, f, 4, 2, 64, ctypes.c_void_p(4097), p, p, None) == 3


def test_backward_workspace_size_and_argument_checks(L):
    L.tg_gated_attention_backward_workspace.restype = ctypes.c_size_t
    assert L.tg_gated_attention_backward_workspace(1000, 16) == 4 * 16 * (3 * 1024 + 8)   # padded to 1024 rows
    assert L.tg_gated_attention_backward_workspace(1, 1) == 1792                            # 385 floats, 256-byte multiple
    assert L.tg_gated_attention_backward_workspace(-1, 16) == 0
    p = ctypes.c_void_p(4096)
    f = ctypes.c_float(1.0)
    big = ctypes.c_size_t(1 << 30)
    args = lambda S, Hq, Hkv, D, ws=p, n=big, tau=f: (p, p, p, p, p, tau, p, None, p, p, S, Hq, Hkv, D, p, p, p, ws, n,  # noqa: E731
                                                      None)
    assert L.tg_gated_attention_backward(*args(100, 6, 4, 128)) == 1                       # Hq % Hkv
    assert L.tg_gated_attention_backward(*args(100, 4, 2, 96)) == 2                        # D
    assert L.tg_gated_attention_backward(*args(-1, 4, 2, 64)) == 1
    assert L.tg_gated_attention_backward(*args(100, 4, 2, 64, tau=ctypes.c_float(float("nan")))) == 1
    assert L.tg_gated_attention_backward(*args(100, 4, 2, 64, n=ctypes.c_size_t(1000))) == 1   # workspace too small
    assert "workspace" in _detail(L)
    assert L.tg_gated_attention_backward(*args(100, 4, 2, 64, ws=None)) == 1
    assert L.tg_gated_attention_backward(*args(100, 4, 2, 64, ws=ctypes.c_void_p(4100))) == 3
    assert L.tg_gated_attention_train(p, p, p, p, p, f, 10, 4, 2, 64, p, None, None, None) == 1   # lse NULL
    assert L.tg_gated_attention_train(p, p, p, p, p, f, 10, 4, 2, 64, p, p, ctypes.c_void_p(4104), None) == 3


def test_backward_varlen_workspace_and_argument_checks(L):
    L.tg_gated_attention_backward_varlen_workspace.restype = ctypes.c_size_t
    # 1000 packed rows in 3 requests: 1024 + 3 * 128 = 1408 rows per head (each request padded)
    assert L.tg_gated_attention_backward_varlen_workspace(1000, 3, 16) == (4 * 16 * (3 * 1408 + 11) + 255) // 256 * 256
    assert L.tg_gated_attention_backward_varlen_workspace(1000, 0, 16) == 0
    assert L.tg_gated_attention_backward_varlen_workspace(-1, 2, 16) == 0
    p = ctypes.c_void_p(4096)
    f = ctypes.c_float(1.0)
    big = ctypes.c_size_t(1 << 30)
    args = lambda cu, B, total, mx, n=big: (p, p, p, p, p, f, p, None, p, p, cu, B, total, mx, 4, 2, 64, p, p, p,  # noqa: E731
                                            p, n, None)
    assert L.tg_gated_attention_backward_varlen(*args(p, 0, 100, 50)) == 1        # B < 1
    assert L.tg_gated_attention_backward_varlen(*args(None, 2, 100, 50)) == 1     # cu_seqlens NULL
    assert L.tg_gated_attention_backward_varlen(*args(p, 2, 100, 101)) == 1       # max_seqlen > total
    assert L.tg_gated_attention_backward_varlen(*args(p, 2, 100, 50, n=ctypes.c_size_t(4 * 4 * 3 * 256))) == 1
    assert "workspace" in _detail(L)
    assert L.tg_gated_attention_train_varlen(p, p, p, p, p, f, None, 2, 10, 5, 4, 2, 64, p, p, None, None) == 1
    assert L.tg_gated_attention_train_varlen(p, p, p, p, p, f, p, 2, 10, 11, 4, 2, 64, p, p, None, None) == 1
    assert L.tg_gated_attention_train_varlen(p, p, p, p, p, f, p, 2, 10, 5, 4, 2, 64, p, None, None, None) == 1


def test_backward_noalloc_rejects_sizes_beyond_its_static_scratch(L):
    p = ctypes.c_void_p(4096)
    f = ctypes.c_float(1.0)
    # S = 30000 with 16 heads needs 4 * 16 * (3 * 30080 + 235) bytes > 4 MiB: rejected before any CUDA call
    assert L.tg_gated_attention_backward_noalloc(p, p, p, p, p, f, p, None, p, p, 30000, 16, 8, 128,
                                                 p, p, p, None) == 2
    assert "static scratch" in _detail(L) and "4194304" in _detail(L)
    assert L.tg_gated_attention_backward_noalloc(p, p, p, p, p, f, p, None, p, p, -1, 16, 8, 128, p, p, p, None) == 1


def test_select_fused_rejects_bad_arguments(L):
    p = ctypes.c_void_p(4096)
    ws = ctypes.c_size_t(1 << 20)
    args = lambda n=1000, d=64, h=64, k=10, cap=100, rows=50, hk=p, sk=p: (  # noqa: E731
        p, n, d, p, p, p, p, h, p, k, p, p, cap, p, hk, sk, rows, p, ws, None)
    assert L.tg_select_fused(*args(n=-1)) == 1
    assert L.tg_select_fused(*args(rows=101)) == 1          # n_rows > cap
    assert L.tg_select_fused(*args(d=12)) == 2              # d % 8
    assert L.tg_select_fused(*args(d=32768)) == 2           # d above the gather's limit
    assert L.tg_select_fused(*args(hk=None)) == 1           # rows requested without hidden_k


def test_probe_rejects_bad_limit(L):
    assert L.tg_probe_wait_timeout(0, None) == 1
    assert L.tg_probe_wait_timeout(3_000_000_000, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        _lib.lib()
