"""ctypes binding of libtokengate.so (include/tokengate.h).

Argument marshalling only: every function forwards torch CUDA tensors' device
pointers, sizes and the current CUDA stream to the C call of the same name and
raises ``TokenGateError`` on a non-TG_OK status.  No computation happens here
and there is no CPU fallback: if the library is missing the call fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_build", "libtokengate.so")

TG_OK = 0
TG_DEVERR_TIMEOUT = 1
TG_DEVERR_INDEX_OOB = 2
TG_DEVERR_K_GT_NDOC = 4
TG_DEVERR_CAPACITY = 8
TG_DEVERR_BAD_SEQLENS = 16

_lib = None


class TokenGateError(RuntimeError):
    def __init__(self, call: str, status: int, name: str, detail: str):
        super().__init__(f"{call} failed: {name}" + (f" ({detail})" if detail else ""))
        self.call = call
        self.status = status
        self.status_name = name
        self.detail = detail


_vp, _i64, _i32, _f32, _u32p = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.POINTER(ctypes.c_uint32)

_SIGNATURES = {
    "tg_abi_version": ([], ctypes.c_int),
    "tg_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "tg_last_error_detail": ([], ctypes.c_char_p),
    "tg_get_device_error": ([_vp, _u32p], ctypes.c_int),
    "tg_probe_wait_timeout": ([_i64, _vp], ctypes.c_int),
    "tg_gate_score": ([_vp, _i64, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _vp], ctypes.c_int),
    "tg_select_topk": ([_vp, _vp, _i64, _i64, _vp, _i64, _vp, _vp], ctypes.c_int),
    "tg_select_topk_varlen": ([_vp, _vp, _vp, _i32, _i64, _vp, _i64, _vp, _i64, _vp, _vp], ctypes.c_int),
    "tg_select_topk_sweep": ([_vp, _vp, _i64, _vp, _i32, _vp, _i64, _vp, _vp], ctypes.c_int),
    "tg_select_random_k": ([_vp, _i64, _i64, ctypes.c_uint64, _vp, _i64, _vp, _vp], ctypes.c_int),
    "tg_select_fused_workspace": ([_i64], ctypes.c_size_t),
    "tg_select_fused": ([_vp, _i64, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _i64, _vp, _vp, _i64, _vp, _vp, _vp, _i64, _vp,
                         ctypes.c_size_t, _vp], ctypes.c_int),
    "tg_gather": ([_vp, _i64, _i32, _vp, _i64, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "tg_gated_attention": ([_vp, _vp, _vp, _vp, _vp, _f32, _i64, _i32, _i32, _i32, _vp, _vp], ctypes.c_int),
    "tg_gated_attention_varlen": ([_vp, _vp, _vp, _vp, _vp, _f32, _vp, _i32, _i64, _i64, _i32, _i32, _i32, _vp, _vp],
                                  ctypes.c_int),
    "tg_gated_attention_train": ([_vp, _vp, _vp, _vp, _vp, _f32, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _vp],
                                 ctypes.c_int),
    "tg_gated_attention_backward_workspace": ([_i64, _i32], ctypes.c_size_t),
    "tg_gated_attention_backward": ([_vp, _vp, _vp, _vp, _vp, _f32, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _vp,
                                     _vp, _vp, _vp, ctypes.c_size_t, _vp], ctypes.c_int),
    "tg_gated_attention_train_varlen": ([_vp, _vp, _vp, _vp, _vp, _f32, _vp, _i32, _i64, _i64, _i32, _i32, _i32, _vp,
                                         _vp, _vp, _vp], ctypes.c_int),
    "tg_gated_attention_backward_varlen_workspace": ([_i64, _i32, _i32], ctypes.c_size_t),
    "tg_gated_attention_backward_varlen": ([_vp, _vp, _vp, _vp, _vp, _f32, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i64,
                                            _i32, _i32, _i32, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp], ctypes.c_int),
    "tg_gated_attention_backward_noalloc": ([_vp, _vp, _vp, _vp, _vp, _f32, _vp, _vp, _vp, _vp, _i64, _i32, _i32,
                                             _i32, _vp, _vp, _vp, _vp], ctypes.c_int),
    "tg_qkv_rope": ([_vp, _i64, _i32, _vp, _vp, ctypes.c_double, _vp, _vp, _f32, _i32, _i32, _i32, _vp, _vp, _vp, _vp],
                    ctypes.c_int),
    "tg_linear": ([_vp, _i64, _i32, _vp, _i32, _vp, _vp, _vp], ctypes.c_int),
}


def lib() -> ctypes.CDLL:
    """Load libtokengate.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m learned_token_pruning_mlp_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            if hasattr(L, name):
                fn = getattr(L, name)
                fn.argtypes = args
                fn.restype = res
        _lib = L
    return _lib


def _check(call: str, status: int) -> None:
    if status != TG_OK:
        L = lib()
        raise TokenGateError(call, status, L.tg_status_string(status).decode(), L.tg_last_error_detail().decode())


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: Optional[torch.Tensor], dtype, name: str):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def tg_abi_version() -> int:
    return int(lib().tg_abi_version())


def tg_get_device_error(stream=None) -> int:
    bits = ctypes.c_uint32(0)
    _check("tg_get_device_error", lib().tg_get_device_error(_stream(stream), ctypes.byref(bits)))
    return int(bits.value)


def tg_probe_wait_timeout(limit_ns: int, stream=None) -> None:
    _check("tg_probe_wait_timeout", lib().tg_probe_wait_timeout(int(limit_ns), _stream(stream)))


def tg_gate_score(hidden, W1, b1, W2, b2, scores=None, stream=None) -> torch.Tensor:
    n, d = hidden.shape
    h = W1.shape[0]
    if scores is None:
        scores = torch.empty(n, dtype=torch.float32, device=hidden.device)
    bf = torch.bfloat16
    _check("tg_gate_score", lib().tg_gate_score(
        _dev(hidden, bf, "hidden"), n, d, _dev(W1, bf, "W1"), _dev(b1, bf, "b1"), _dev(W2, bf, "W2"),
        _dev(b2, bf, "b2"), h, _dev(scores, torch.float32, "scores"), _stream(stream)))
    return scores


def tg_select_topk(scores, doc_mask, k: int, kept_idx=None, n_kept=None, cap: Optional[int] = None,
                   stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    n = scores.shape[0]
    if kept_idx is None:
        kept_idx = torch.empty(max(n, 1), dtype=torch.int32, device=scores.device)
    if n_kept is None:
        n_kept = torch.empty(1, dtype=torch.int32, device=scores.device)
    cap = kept_idx.numel() if cap is None else cap
    _check("tg_select_topk", lib().tg_select_topk(
        _dev(scores, torch.float32, "scores"), _dev(doc_mask, torch.uint8, "doc_mask"), n, int(k),
        _dev(kept_idx, torch.int32, "kept_idx"), int(cap), _dev(n_kept, torch.int32, "n_kept"), _stream(stream)))
    return kept_idx, n_kept


def tg_select_topk_varlen(scores, doc_mask, cu_seqlens, k_per_seq, max_seqlen: int, kept_idx=None, cu_kept=None,
                          cap: Optional[int] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    total = scores.shape[0]
    B = cu_seqlens.numel() - 1
    if kept_idx is None:
        kept_idx = torch.empty(max(total, 1), dtype=torch.int32, device=scores.device)
    if cu_kept is None:
        cu_kept = torch.empty(B + 1, dtype=torch.int32, device=scores.device)
    cap = kept_idx.numel() if cap is None else cap
    _check("tg_select_topk_varlen", lib().tg_select_topk_varlen(
        _dev(scores, torch.float32, "scores"), _dev(doc_mask, torch.uint8, "doc_mask"),
        _dev(cu_seqlens, torch.int32, "cu_seqlens"), B, total, _dev(k_per_seq, torch.int32, "k_per_seq"),
        int(max_seqlen), _dev(kept_idx, torch.int32, "kept_idx"), int(cap), _dev(cu_kept, torch.int32, "cu_kept"),
        _stream(stream)))
    return kept_idx, cu_kept


def tg_select_topk_sweep(scores, doc_mask, ks, kept_idx=None, n_kept=None, stride: Optional[int] = None,
                         stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    n = scores.shape[0]
    m = ks.numel()
    stride = max(n, 1) if stride is None else stride
    if kept_idx is None:
        kept_idx = torch.empty(max(m * stride, 1), dtype=torch.int32, device=scores.device)
    if n_kept is None:
        n_kept = torch.empty(max(m, 1), dtype=torch.int32, device=scores.device)
    _check("tg_select_topk_sweep", lib().tg_select_topk_sweep(
        _dev(scores, torch.float32, "scores"), _dev(doc_mask, torch.uint8, "doc_mask"), n,
        _dev(ks, torch.int32, "ks"), m, _dev(kept_idx, torch.int32, "kept_idx"), int(stride),
        _dev(n_kept, torch.int32, "n_kept"), _stream(stream)))
    return kept_idx, n_kept


def tg_select_random_k(doc_mask, k: int, seed: int, kept_idx=None, n_kept=None, cap: Optional[int] = None,
                       stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    n = doc_mask.shape[0]
    if kept_idx is None:
        kept_idx = torch.empty(max(n, 1), dtype=torch.int32, device=doc_mask.device)
    if n_kept is None:
        n_kept = torch.empty(1, dtype=torch.int32, device=doc_mask.device)
    cap = kept_idx.numel() if cap is None else cap
    _check("tg_select_random_k", lib().tg_select_random_k(
        _dev(doc_mask, torch.uint8, "doc_mask"), n, int(k), int(seed) & 0xFFFFFFFFFFFFFFFF,
        _dev(kept_idx, torch.int32, "kept_idx"), int(cap), _dev(n_kept, torch.int32, "n_kept"), _stream(stream)))
    return kept_idx, n_kept


def tg_select_fused_workspace(n: int) -> int:
    return int(lib().tg_select_fused_workspace(int(n)))


def tg_select_fused(hidden, W1, b1, W2, b2, doc_mask, k: int, n_rows: Optional[int] = None, scores=None,
                    kept_idx=None, n_kept=None, hidden_k=None, s_k=None, cap: Optional[int] = None, workspace=None,
                    stream=None):
    """Gate -> top-K -> gather in one call; returns (scores, kept_idx, n_kept, hidden_k, s_k)."""
    n, d = hidden.shape
    h = W1.shape[0]
    dev = hidden.device
    if scores is None:
        scores = torch.empty(n, dtype=torch.float32, device=dev)
    if kept_idx is None:
        kept_idx = torch.empty(max(n, 1), dtype=torch.int32, device=dev)
    if n_kept is None:
        n_kept = torch.empty(1, dtype=torch.int32, device=dev)
    cap = kept_idx.numel() if cap is None else cap
    if n_rows is None:
        n_rows = min(cap, n)
    if hidden_k is None:
        hidden_k = torch.empty((max(n_rows, 1), d), dtype=hidden.dtype, device=dev)
    if s_k is None:
        s_k = torch.empty(max(n_rows, 1), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(tg_select_fused_workspace(n), 16), dtype=torch.uint8, device=dev)
    bf = torch.bfloat16
    _check("tg_select_fused", lib().tg_select_fused(
        _dev(hidden, bf, "hidden"), n, d, _dev(W1, bf, "W1"), _dev(b1, bf, "b1"), _dev(W2, bf, "W2"),
        _dev(b2, bf, "b2"), h, _dev(doc_mask, torch.uint8, "doc_mask"), int(k), _dev(scores, torch.float32, "scores"),
        _dev(kept_idx, torch.int32, "kept_idx"), int(cap), _dev(n_kept, torch.int32, "n_kept"),
        _dev(hidden_k, bf, "hidden_k"), _dev(s_k, torch.float32, "s_k"), int(n_rows),
        _dev(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)))
    return scores, kept_idx, n_kept, hidden_k, s_k


def tg_gather(hidden, kept_idx, n_rows: Optional[int] = None, n_kept=None, hidden_k=None, scores=None, s_k=None,
              stream=None):
    n, d = hidden.shape
    n_rows = kept_idx.numel() if n_rows is None else n_rows
    if hidden_k is None:
        hidden_k = torch.empty((n_rows, d), dtype=hidden.dtype, device=hidden.device)
    if scores is not None and s_k is None:
        s_k = torch.empty(n_rows, dtype=torch.float32, device=hidden.device)
    _check("tg_gather", lib().tg_gather(
        _dev(hidden, torch.bfloat16, "hidden"), n, d, _dev(kept_idx, torch.int32, "kept_idx"), int(n_rows),
        _dev(n_kept, torch.int32, "n_kept"), _dev(hidden_k, torch.bfloat16, "hidden_k"),
        _dev(scores, torch.float32, "scores"), _dev(s_k, torch.float32, "s_k"), _stream(stream)))
    return hidden_k, s_k


def tg_gated_attention(Q, Kc, V, s, gain, tau: float, O=None, stream=None) -> torch.Tensor:
    S, Hq, D = Q.shape
    Hkv = Kc.shape[1]
    if O is None:
        O = torch.empty_like(Q)
    bf = torch.bfloat16
    _check("tg_gated_attention", lib().tg_gated_attention(
        _dev(Q, bf, "Q"), _dev(Kc, bf, "Kc"), _dev(V, bf, "V"), _dev(s, torch.float32, "s"),
        _dev(gain, torch.float32, "gain"), float(tau), S, Hq, Hkv, D, _dev(O, bf, "O"), _stream(stream)))
    return O


def tg_gated_attention_train(Q, Kc, V, s, gain, tau: float, O=None, lse=None, O32=None, keep_fp32=True,
                             stream=None):
    """Forward for training: returns (O bf16, lse fp32 [S, Hq], O32 fp32 [S, Hq, D] or None)."""
    S, Hq, D = Q.shape
    Hkv = Kc.shape[1]
    if O is None:
        O = torch.empty_like(Q)
    if lse is None:
        lse = torch.empty((S, Hq), dtype=torch.float32, device=Q.device)
    if O32 is None and keep_fp32:
        O32 = torch.empty((S, Hq, D), dtype=torch.float32, device=Q.device)
    bf = torch.bfloat16
    _check("tg_gated_attention_train", lib().tg_gated_attention_train(
        _dev(Q, bf, "Q"), _dev(Kc, bf, "Kc"), _dev(V, bf, "V"), _dev(s, torch.float32, "s"),
        _dev(gain, torch.float32, "gain"), float(tau), S, Hq, Hkv, D, _dev(O, bf, "O"),
        _dev(lse, torch.float32, "lse"), _dev(O32, torch.float32, "O32"), _stream(stream)))
    return O, lse, O32


def tg_gated_attention_backward_workspace(S: int, Hq: int) -> int:
    return int(lib().tg_gated_attention_backward_workspace(int(S), int(Hq)))


def tg_gated_attention_backward(Q, Kc, V, s, gain, tau: float, O, dO, lse, O32=None, ds=None, dgain=None,
                                dtau=None, workspace=None, stream=None):
    S, Hq, D = Q.shape
    Hkv = Kc.shape[1]
    dev = gain.device
    if ds is None:
        ds = torch.empty(S, dtype=torch.float32, device=dev)
    if dgain is None:
        dgain = torch.empty(Hq, dtype=torch.float32, device=dev)
    if dtau is None:
        dtau = torch.empty(1, dtype=torch.float32, device=dev)
    need = tg_gated_attention_backward_workspace(S, Hq)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    bf = torch.bfloat16
    _check("tg_gated_attention_backward", lib().tg_gated_attention_backward(
        _dev(Q, bf, "Q"), _dev(Kc, bf, "Kc"), _dev(V, bf, "V"), _dev(s, torch.float32, "s"),
        _dev(gain, torch.float32, "gain"), float(tau), _dev(O, bf, "O"), _dev(O32, torch.float32, "O32"),
        _dev(dO, bf, "dO"), _dev(lse, torch.float32, "lse"), S, Hq, Hkv, D, _dev(ds, torch.float32, "ds"),
        _dev(dgain, torch.float32, "dgain"), _dev(dtau, torch.float32, "dtau"),
        _dev(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)))
    return ds, dgain, dtau


def tg_gated_attention_varlen(Q, Kc, V, s, gain, tau: float, cu_seqlens, max_seqlen: int, O=None,
                              stream=None) -> torch.Tensor:
    total, Hq, D = Q.shape
    Hkv = Kc.shape[1]
    B = cu_seqlens.numel() - 1
    if O is None:
        O = torch.empty_like(Q)
    bf = torch.bfloat16
    _check("tg_gated_attention_varlen", lib().tg_gated_attention_varlen(
        _dev(Q, bf, "Q"), _dev(Kc, bf, "Kc"), _dev(V, bf, "V"), _dev(s, torch.float32, "s"),
        _dev(gain, torch.float32, "gain"), float(tau), _dev(cu_seqlens, torch.int32, "cu_seqlens"), B, total,
        int(max_seqlen), Hq, Hkv, D, _dev(O, bf, "O"), _stream(stream)))
    return O


def tg_gated_attention_train_varlen(Q, Kc, V, s, gain, tau: float, cu_seqlens, max_seqlen: int, O=None, lse=None,
                                   O32=None, keep_fp32=True, stream=None):
    """Training forward of a packed ragged batch: returns (O bf16, lse fp32 [total, Hq], O32 or None)."""
    total, Hq, D = Q.shape
    Hkv = Kc.shape[1]
    B = cu_seqlens.numel() - 1
    if O is None:
        O = torch.empty_like(Q)
    if lse is None:
        lse = torch.empty((total, Hq), dtype=torch.float32, device=Q.device)
    if O32 is None and keep_fp32:
        O32 = torch.empty((total, Hq, D), dtype=torch.float32, device=Q.device)
    bf = torch.bfloat16
    _check("tg_gated_attention_train_varlen", lib().tg_gated_attention_train_varlen(
        _dev(Q, bf, "Q"), _dev(Kc, bf, "Kc"), _dev(V, bf, "V"), _dev(s, torch.float32, "s"),
        _dev(gain, torch.float32, "gain"), float(tau), _dev(cu_seqlens, torch.int32, "cu_seqlens"), B, total,
        int(max_seqlen), Hq, Hkv, D, _dev(O, bf, "O"), _dev(lse, torch.float32, "lse"),
        _dev(O32, torch.float32, "O32"), _stream(stream)))
    return O, lse, O32


def tg_gated_attention_backward_varlen_workspace(total: int, B: int, Hq: int) -> int:
    return int(lib().tg_gated_attention_backward_varlen_workspace(int(total), int(B), int(Hq)))


def tg_gated_attention_backward_varlen(Q, Kc, V, s, gain, tau: float, O, dO, lse, cu_seqlens, max_seqlen: int,
                                       O32=None, ds=None, dgain=None, dtau=None, workspace=None, stream=None):
    total, Hq, D = Q.shape
    Hkv = Kc.shape[1]
    B = cu_seqlens.numel() - 1
    dev = gain.device
    if ds is None:
        ds = torch.empty(total, dtype=torch.float32, device=dev)
    if dgain is None:
        dgain = torch.empty(Hq, dtype=torch.float32, device=dev)
    if dtau is None:
        dtau = torch.empty(1, dtype=torch.float32, device=dev)
    if workspace is None:
        need = tg_gated_attention_backward_varlen_workspace(total, B, Hq)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    bf = torch.bfloat16
    _check("tg_gated_attention_backward_varlen", lib().tg_gated_attention_backward_varlen(
        _dev(Q, bf, "Q"), _dev(Kc, bf, "Kc"), _dev(V, bf, "V"), _dev(s, torch.float32, "s"),
        _dev(gain, torch.float32, "gain"), float(tau), _dev(O, bf, "O"), _dev(O32, torch.float32, "O32"),
        _dev(dO, bf, "dO"), _dev(lse, torch.float32, "lse"), _dev(cu_seqlens, torch.int32, "cu_seqlens"), B, total,
        int(max_seqlen), Hq, Hkv, D, _dev(ds, torch.float32, "ds"), _dev(dgain, torch.float32, "dgain"),
        _dev(dtau, torch.float32, "dtau"), _dev(workspace, torch.uint8, "workspace"), workspace.numel(),
        _stream(stream)))
    return ds, dgain, dtau


def tg_gated_attention_backward_noalloc(Q, Kc, V, s, gain, tau: float, O, dO, lse, O32=None, ds=None, dgain=None,
                                        dtau=None, stream=None):
    S, Hq, D = Q.shape
    Hkv = Kc.shape[1]
    dev = gain.device
    if ds is None:
        ds = torch.empty(S, dtype=torch.float32, device=dev)
    if dgain is None:
        dgain = torch.empty(Hq, dtype=torch.float32, device=dev)
    if dtau is None:
        dtau = torch.empty(1, dtype=torch.float32, device=dev)
    bf = torch.bfloat16
    _check("tg_gated_attention_backward_noalloc", lib().tg_gated_attention_backward_noalloc(
        _dev(Q, bf, "Q"), _dev(Kc, bf, "Kc"), _dev(V, bf, "V"), _dev(s, torch.float32, "s"),
        _dev(gain, torch.float32, "gain"), float(tau), _dev(O, bf, "O"), _dev(O32, torch.float32, "O32"),
        _dev(dO, bf, "dO"), _dev(lse, torch.float32, "lse"), S, Hq, Hkv, D, _dev(ds, torch.float32, "ds"),
        _dev(dgain, torch.float32, "dgain"), _dev(dtau, torch.float32, "dtau"), _stream(stream)))
    return ds, dgain, dtau


def tg_qkv_rope(hidden, W_qkv, positions, rope_base: float, Hq: int, Hkv: int, D: int, q_norm=None, k_norm=None,
                eps: float = 1e-6, Q=None, Kc=None, V=None, stream=None):
    S, d = hidden.shape
    bf = torch.bfloat16
    if Q is None:
        Q = torch.empty((S, Hq, D), dtype=bf, device=hidden.device)
    if Kc is None:
        Kc = torch.empty((S, Hkv, D), dtype=bf, device=hidden.device)
    if V is None:
        V = torch.empty((S, Hkv, D), dtype=bf, device=hidden.device)
    if W_qkv.shape != ((Hq + 2 * Hkv) * D, d):
        raise ValueError(f"W_qkv must be [{(Hq + 2 * Hkv) * D}, {d}], got {tuple(W_qkv.shape)}")
    if positions.numel() < S:
        raise ValueError("positions needs one entry per row")
    _check("tg_qkv_rope", lib().tg_qkv_rope(
        _dev(hidden, bf, "hidden"), S, d, _dev(W_qkv, bf, "W_qkv"), _dev(positions, torch.int32, "positions"),
        float(rope_base), _dev(q_norm, bf, "q_norm"), _dev(k_norm, bf, "k_norm"), float(eps), Hq, Hkv, D,
        _dev(Q, bf, "Q"), _dev(Kc, bf, "Kc"), _dev(V, bf, "V"), _stream(stream)))
    return Q, Kc, V


def tg_linear(x, W, residual=None, y=None, stream=None) -> torch.Tensor:
    M, K = x.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("W must be [N, K]")
    bf = torch.bfloat16
    if y is None:
        y = torch.empty((M, N), dtype=bf, device=x.device)
    _check("tg_linear", lib().tg_linear(
        _dev(x, bf, "x"), M, K, _dev(W, bf, "W"), N, _dev(residual, bf, "residual"), _dev(y, bf, "y"),
        _stream(stream)))
    return y
