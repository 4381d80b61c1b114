"""fp64 CPU oracle for the TokenGate pruned-prefill hot path.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg may import this package; the library never does,
and it shares no code with the CUDA path.

Two independent implementations live here:
  * ``oracle.c`` -- plain C, fp64, OpenMP over output rows (``liboracle.so``,
    compiled on first use or by ``oracle.build.build()``);
  * ``twin``     -- the same definitions in numpy fp64, for small sizes only.

Source: the MarkTechPost TokenGate article, sections "How does TokenGate
learned token pruning work?" (gate, top-K, question never pruned, pruned
forward, kept tokens at their prompt positions) and "What is token-gated
attention?" (score as logit bias, per-head gain, temperature).  Each function below restates the definition it follows.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np
import torch

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        vp, i64, i32, f64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        L.orc_gate_score.argtypes = [vp, i64, i32, vp, vp, vp, vp, i32, vp]
        L.orc_gate_score.restype = None
        L.orc_select_topk.argtypes = [vp, vp, i64, i64, vp]
        L.orc_select_topk.restype = i64
        L.orc_gather.argtypes = [vp, i32, vp, i64, vp, vp, vp]
        L.orc_gather.restype = None
        L.orc_gated_attention_rows.argtypes = [vp, vp, vp, vp, vp, f64, i64, i32, i32, i32, vp, i64, vp, vp]
        L.orc_gated_attention_rows.restype = None
        L.orc_splitmix64.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        L.orc_splitmix64.restype = ctypes.c_uint64
        L.orc_select_random_k.argtypes = [vp, i64, i64, ctypes.c_uint64, vp]
        L.orc_select_random_k.restype = i64
        L.orc_gated_attention_lse_rows.argtypes = [vp, vp, vp, vp, f64, i32, i32, i32, vp, i64, vp]
        L.orc_gated_attention_lse_rows.restype = None
        L.orc_gated_attention_backward.argtypes = [vp, vp, vp, vp, vp, f64, vp, i64, i32, i32, i32, vp, vp, vp]
        L.orc_gated_attention_backward.restype = None
        L.orc_qkv_rope_rows.argtypes = [vp, i32, vp, vp, f64, i32, i32, i32, vp, vp, f64, vp, i64, vp, vp, vp]
        L.orc_qkv_rope_rows.restype = None
        L.orc_linear_rows.argtypes = [vp, i32, vp, i32, vp, vp, i64, vp]
        L.orc_linear_rows.restype = None
        L.orc_num_threads.argtypes = []
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_set_num_threads.argtypes = [i32]
        L.orc_set_num_threads.restype = None
        _lib = L
    return _lib


def num_threads() -> int:
    return int(lib().orc_num_threads())


def set_num_threads(n: int) -> None:
    """Thread count of the oracle's parallel loops from now on (timing only; results are
    the same for any count)."""
    lib().orc_set_num_threads(int(n))


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _np(a, dtype) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------- gate
def gate_score(hidden, W1, b1, W2, b2) -> np.ndarray:
    """s_i = b2 + sum_j W2_j * SiLU(b1_j + W1[j,:] . x_i) in fp64 over the bf16 inputs."""
    n, d = hidden.shape
    h = W1.shape[0]
    hb, w1, bb1, w2, bb2 = (_bf16_bits(t) for t in (hidden, W1, b1, W2, b2))
    out = np.empty(n, dtype=np.float64)
    lib().orc_gate_score(_ptr(hb), n, d, _ptr(w1), _ptr(bb1), _ptr(w2), _ptr(bb2), h, _ptr(out))
    return out


# --------------------------------------------------------------------------- top-K
def select_topk(scores, doc_mask, k: int) -> np.ndarray:
    """Kept indices (ascending int32): the k best document tokens by (score desc, index asc),
    NaN below everything, plus every question token."""
    s = _np(scores, np.float32)
    m = _np(doc_mask, np.uint8)
    out = np.empty(max(len(s), 1), dtype=np.int32)
    cnt = lib().orc_select_topk(_ptr(s), _ptr(m), len(s), int(k), _ptr(out))
    return out[:cnt].copy()


def select_topk_varlen(scores, doc_mask, cu_seqlens: Sequence[int], ks: Sequence[int]):
    """Per-request selection of packed requests; indices are positions in the packed sequence.
    Returns (kept_idx int32, cu_kept int32[B+1])."""
    s = _np(scores, np.float32)
    m = _np(doc_mask, np.uint8)
    cu = [int(x) for x in cu_seqlens]
    parts, cu_kept = [], [0]
    for b in range(len(cu) - 1):
        lo, hi = cu[b], cu[b + 1]
        kept = select_topk(s[lo:hi], m[lo:hi], int(ks[b])) + lo
        parts.append(kept.astype(np.int32))
        cu_kept.append(cu_kept[-1] + len(kept))
    kept_all = np.concatenate(parts) if parts else np.zeros(0, np.int32)
    return kept_all, np.asarray(cu_kept, dtype=np.int32)


def select_topk_sweep(scores, doc_mask, ks: Sequence[int]):
    """The selection at every budget of ``ks``: a list of kept-index arrays."""
    return [select_topk(scores, doc_mask, int(k)) for k in ks]


def splitmix64(seed: int, index: int) -> int:
    """The (index + 1)-th output of SplitMix64 seeded with ``seed``."""
    return int(lib().orc_splitmix64(seed & 0xFFFFFFFFFFFFFFFF, index))


def select_random_k(doc_mask, k: int, seed: int) -> np.ndarray:
    """k uniformly random document tokens (SplitMix64 keys, ties to the lower index) plus
    every question token, ascending int32."""
    m = _np(doc_mask, np.uint8)
    out = np.empty(max(len(m), 1), dtype=np.int32)
    cnt = lib().orc_select_random_k(_ptr(m), len(m), int(k), seed & 0xFFFFFFFFFFFFFFFF, _ptr(out))
    return out[:cnt].copy()


# --------------------------------------------------------------------------- gather
def gather(hidden, kept, scores=None):
    """hidden_k[r] = hidden[kept[r]] (bf16 bit patterns, uint16) and s_k[r] = scores[kept[r]]."""
    hb = _bf16_bits(hidden)
    n, d = hb.shape
    kp = _np(kept, np.int32)
    hk = np.empty((len(kp), d), dtype=np.uint16)
    sk = None
    sp = None
    if scores is not None:
        sp = _np(scores, np.float32)
        sk = np.empty(len(kp), dtype=np.float32)
    lib().orc_gather(_ptr(hb), d, _ptr(kp), len(kp), _ptr(hk),
                     _ptr(sp) if sp is not None else None, _ptr(sk) if sk is not None else None)
    return hk, sk


# --------------------------------------------------------------------------- attention
def gated_attention(Q, K, V, s, gain, tau: float, rows: Optional[Sequence[int]] = None,
                    return_spread: bool = False):
    """O[i,h] = sum_{j<=i} softmax_j(tau*Q_ih.K_jg/sqrt(D) + gain_h*s_j) V_jg, g = h // (Hq/Hkv).
    Returns fp64 [len(rows), Hq, D] (all rows when ``rows`` is None).  With
    ``return_spread`` also returns spread[i,h,c] = sum_j softmax_j |V_jg[c] - O_ih[c]|,
    the weighted mean absolute deviation of the value rows: a bound on how far
    relative weight errors move the output, used to size tolerances (not part of
    the method)."""
    S, Hq, D = Q.shape
    Hkv = K.shape[1]
    qb, kb, vb = _bf16_bits(Q), _bf16_bits(K), _bf16_bits(V)
    sv = _np(s, np.float32)
    gv = _np(gain, np.float32)
    r = np.arange(S, dtype=np.int64) if rows is None else _np(rows, np.int64)
    out = np.empty((len(r), Hq, D), dtype=np.float64)
    spread = np.empty((len(r), Hq, D), dtype=np.float64) if return_spread else None
    lib().orc_gated_attention_rows(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(sv), _ptr(gv), float(tau),
                                   S, Hq, Hkv, D, _ptr(r), len(r), _ptr(out),
                                   _ptr(spread) if return_spread else None)
    return (out, spread) if return_spread else out


def gated_attention_varlen(Q, K, V, s, gain, tau: float, cu_seqlens: Sequence[int],
                           rows: Optional[Sequence[int]] = None, return_spread: bool = False):
    """Packed requests: each segment [cu[b], cu[b+1]) attends causally within itself only.
    ``rows`` are packed row indices (all rows when None); returns fp64 [len(rows), Hq, D]
    (and the spread, as in ``gated_attention``)."""
    cu = [int(x) for x in cu_seqlens]
    S, Hq, D = Q.shape
    rows_all = np.arange(S, dtype=np.int64) if rows is None else _np(rows, np.int64)
    out = np.empty((len(rows_all), Hq, D), dtype=np.float64)
    spread = np.empty((len(rows_all), Hq, D), dtype=np.float64) if return_spread else None
    for b in range(len(cu) - 1):
        lo, hi = cu[b], cu[b + 1]
        sel = np.nonzero((rows_all >= lo) & (rows_all < hi))[0]
        if len(sel) == 0:
            continue
        res = gated_attention(Q[lo:hi], K[lo:hi], V[lo:hi], _np(s, np.float32)[lo:hi], gain, tau,
                              rows=rows_all[sel] - lo, return_spread=return_spread)
        if return_spread:
            out[sel], spread[sel] = res
        else:
            out[sel] = res
    return (out, spread) if return_spread else out


def gated_attention_lse(Q, K, s, gain, tau: float, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """lse[r, h] = log sum_{j <= i} exp(tau*Q_ih.K_jg/sqrt(D) + gain_h*s_j), i = rows[r]; fp64 [R, Hq]."""
    S, Hq, D = Q.shape
    Hkv = K.shape[1]
    qb, kb = _bf16_bits(Q), _bf16_bits(K)
    sv, gv = _np(s, np.float32), _np(gain, np.float32)
    r = np.arange(S, dtype=np.int64) if rows is None else _np(rows, np.int64)
    out = np.empty((len(r), Hq), dtype=np.float64)
    lib().orc_gated_attention_lse_rows(_ptr(qb), _ptr(kb), _ptr(sv), _ptr(gv), float(tau), Hq, Hkv, D,
                                       _ptr(r), len(r), _ptr(out))
    return out


def gated_attention_backward(Q, K, V, s, gain, tau: float, dO):
    """Gradients of the loss with dL/dO = dO through token-gated attention:
    (ds [S], dgain [Hq], dtau) in fp64, with dl_ij = P_ij (dO_i.V_j - dO_i.O_i),
    ds_j = sum_{h,i} gain_h dl_ij, dgain_h = sum_{i,j} s_j dl_ij, dtau = sum dl_ij q_i.k_j/sqrt(D)."""
    S, Hq, D = Q.shape
    Hkv = K.shape[1]
    qb, kb, vb, db = _bf16_bits(Q), _bf16_bits(K), _bf16_bits(V), _bf16_bits(dO)
    sv, gv = _np(s, np.float32), _np(gain, np.float32)
    ds = np.empty(S, dtype=np.float64)
    dg = np.empty(Hq, dtype=np.float64)
    dt = np.empty(1, dtype=np.float64)
    lib().orc_gated_attention_backward(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(sv), _ptr(gv), float(tau), _ptr(db),
                                       S, Hq, Hkv, D, _ptr(ds), _ptr(dg), _ptr(dt))
    return ds, dg, float(dt[0])


# --------------------------------------------------------------------------- projections
def qkv_rope(hidden, W_qkv, positions, base: float, Hq: int, Hkv: int, D: int, q_norm=None, k_norm=None,
             eps: float = 1e-6, rows: Optional[Sequence[int]] = None):
    """[Q K V] = W_qkv x_i; optional per-head RMS norm of Q / K heads; rotary embedding of Q / K heads
    at ``positions[i]`` with pairs (j, j + D/2) and angles p * base^(-2j/D).
    Returns fp64 (Q [R, Hq, D], K [R, Hkv, D], V [R, Hkv, D]) for the listed rows (all when None)."""
    S, d = hidden.shape
    hb, wb = _bf16_bits(hidden), _bf16_bits(W_qkv)
    assert wb.shape == ((Hq + 2 * Hkv) * D, d)
    pv = _np(positions, np.int32)
    qn = _bf16_bits(q_norm) if q_norm is not None else None
    kn = _bf16_bits(k_norm) if k_norm is not None else None
    r = np.arange(S, dtype=np.int64) if rows is None else _np(rows, np.int64)
    Q = np.empty((len(r), Hq, D))
    K = np.empty((len(r), Hkv, D))
    V = np.empty((len(r), Hkv, D))
    lib().orc_qkv_rope_rows(_ptr(hb), d, _ptr(wb), _ptr(pv), float(base), Hq, Hkv, D,
                            _ptr(qn) if qn is not None else None, _ptr(kn) if kn is not None else None,
                            float(eps), _ptr(r), len(r), _ptr(Q), _ptr(K), _ptr(V))
    return Q, K, V


def linear(x, W, residual=None, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """y_i = W x_i (+ residual_i) in fp64 over the bf16 inputs; fp64 [len(rows), N]."""
    M, K = x.shape
    N = W.shape[0]
    xb, wb = _bf16_bits(x), _bf16_bits(W)
    rb = _bf16_bits(residual) if residual is not None else None
    r = np.arange(M, dtype=np.int64) if rows is None else _np(rows, np.int64)
    y = np.empty((len(r), N))
    lib().orc_linear_rows(_ptr(xb), K, _ptr(wb), N, _ptr(rb) if rb is not None else None, _ptr(r), len(r), _ptr(y))
    return y


def sampled_rows(S: int, seed: int, head: int = 128, tail: int = 128, rand: int = 256) -> np.ndarray:
    """Row sample for large cases: the first ``head`` rows, the last ``tail`` rows and ``rand``
    seeded random rows in between (sorted, unique)."""
    rng = np.random.default_rng(seed)
    parts = [np.arange(min(head, S)), np.arange(max(0, S - tail), S)]
    if S > head + tail:
        parts.append(rng.choice(np.arange(head, S - tail), size=min(rand, S - head - tail), replace=False))
    return np.unique(np.concatenate(parts)).astype(np.int64)
