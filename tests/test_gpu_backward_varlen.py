"""Backward of token-gated attention over a packed ragged batch (cu_seqlens), and its
training forward, vs the fp64 CPU oracle run request by request, through the C ABI.

Each request attends within itself only, so the oracle's gradients of request b are
those of its own slice: ds is request b's ds at its rows, dgain and dtau sum over the
requests.  Tolerances are those of the single-sequence tests (test_gpu_backward.py):
kernel parity when the GPU backward is fed the oracle's forward quantities, the chained
bounds when it follows the GPU training forward.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import learned_token_pruning_mlp_b200 as tg
from test_gpu_backward import assert_grads_close, assert_kernel_close
from test_gpu_parity import check_attention

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from learned_token_pruning_mlp_b200 import build
    build.build()
    tg.tg_get_device_error()
    yield


def _packed(lens, Hq, Hkv, D, seed, q_scale=1.0):
    total = int(sum(lens))
    g = torch.Generator().manual_seed(seed)
    Q = (torch.randn(total, Hq, D, generator=g) * q_scale).to(torch.bfloat16)
    K = torch.randn(total, Hkv, D, generator=g).to(torch.bfloat16)
    V = torch.randn(total, Hkv, D, generator=g).to(torch.bfloat16)
    dO = torch.randn(total, Hq, D, generator=g).to(torch.bfloat16)
    s = torch.randn(total, generator=g)
    gain = 0.5 + torch.rand(Hq, generator=g)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return Q, K, V, dO, s, gain, cu


def _oracle_per_request(Q, K, V, dO, s, gain, tau, cu):
    """ds at every packed row, dgain and dtau summed over the requests (the definition
    applied to each request's slice)."""
    Hq = Q.shape[1]
    ds = np.zeros(Q.shape[0])
    dg = np.zeros(Hq)
    dt = 0.0
    for b in range(len(cu) - 1):
        lo, hi = int(cu[b]), int(cu[b + 1])
        if hi == lo:
            continue
        rds, rdg, rdt = oracle.gated_attention_backward(Q[lo:hi], K[lo:hi], V[lo:hi], s[lo:hi], gain, tau, dO[lo:hi])
        ds[lo:hi] = rds
        dg += rdg
        dt += rdt
    return ds, dg, dt


def _oracle_forward(Q, K, s, V, gain, tau, cu):
    """O (fp64) and lse at every packed row, request by request."""
    O = oracle.gated_attention_varlen(Q, K, V, s, gain, tau, cu)
    lse = np.zeros((Q.shape[0], Q.shape[1]))
    for b in range(len(cu) - 1):
        lo, hi = int(cu[b]), int(cu[b + 1])
        if hi > lo:
            lse[lo:hi] = oracle.gated_attention_lse(Q[lo:hi], K[lo:hi], s[lo:hi], gain, tau)
    return O, lse


def _gpu_backward_varlen(Q, K, V, dO, s, gain, tau, cu, O, O32, lse, ws_fill=None):
    d = [t.to(DEV) for t in (Q, K, V, dO, s, gain)]
    d_cu = torch.as_tensor(cu).to(DEV)
    ws = None
    if ws_fill is not None:
        n = tg.tg_gated_attention_backward_varlen_workspace(Q.shape[0], len(cu) - 1, Q.shape[1])
        ws = torch.full((n,), ws_fill, dtype=torch.uint8, device=DEV)
    ds, dg, dt = tg.tg_gated_attention_backward_varlen(d[0], d[1], d[2], d[4], d[5], tau, O, d[3], lse, d_cu,
                                                       int(np.max(np.diff(cu))), O32=O32, workspace=ws)
    torch.cuda.synchronize()
    return ds.cpu().numpy().astype(np.float64), dg.cpu().numpy().astype(np.float64), float(dt.item())


@pytest.mark.parametrize("lens,Hq,Hkv,D,tau", [([300, 1, 0, 517, 129], 4, 2, 128, 1.1),
                                               ([64, 200, 37], 2, 1, 64, -0.7),
                                               ([128, 256, 129], 8, 8, 128, 2.5)])
def test_backward_varlen_kernel_matches_oracle_per_request(lens, Hq, Hkv, D, tau):
    Q, K, V, dO, s, gain, cu = _packed(lens, Hq, Hkv, D, sum(lens) + Hq)
    O_ref, lse_ref = _oracle_forward(Q, K, s, V, gain, tau, cu)
    O32 = torch.as_tensor(O_ref, dtype=torch.float32)
    got = _gpu_backward_varlen(Q, K, V, dO, s, gain, tau, cu, O32.to(torch.bfloat16).to(DEV), O32.to(DEV),
                               torch.as_tensor(lse_ref, dtype=torch.float32).to(DEV), ws_fill=0xAB)
    assert_kernel_close(got, _oracle_per_request(Q, K, V, dO, s, gain, tau, cu))
    assert tg.tg_get_device_error() == 0


def test_train_forward_varlen_then_backward_chained():
    lens = [300, 1, 517, 129]
    Q, K, V, dO, s, gain, cu = _packed(lens, 8, 2, 128, 77)
    d = [t.to(DEV) for t in (Q, K, V, s, gain)]
    d_cu = torch.as_tensor(cu).to(DEV)
    O, lse, O32 = tg.tg_gated_attention_train_varlen(d[0], d[1], d[2], d[3], d[4], 1.1, d_cu, max(lens))
    # the forward's outputs, each within the forward's budget
    check_attention(O.float().cpu().numpy(), Q, K, V, s, gain, 1.1, cu=cu)
    check_attention(O32.cpu().numpy(), Q, K, V, s, gain, 1.1, cu=cu, fp32_out=True)
    _, lse_ref = _oracle_forward(Q, K, s, V, gain, 1.1, cu)
    assert np.max(np.abs(lse.cpu().numpy() - lse_ref)) <= 4e-3
    # the plain varlen forward gives the same O
    O2 = tg.tg_gated_attention_varlen(d[0], d[1], d[2], d[3], d[4], 1.1, d_cu, max(lens))
    assert torch.equal(O, O2)
    got = _gpu_backward_varlen(Q, K, V, dO, s, gain, 1.1, cu, O, O32, lse)
    assert_grads_close(got, _oracle_per_request(Q, K, V, dO, s, gain, 1.1, cu))
    assert tg.tg_get_device_error() == 0


def test_backward_varlen_one_request_equals_single_sequence_bitwise():
    Q, K, V, dO, s, gain, cu = _packed([700], 16, 8, 128, 5)
    d = [t.to(DEV) for t in (Q, K, V, dO, s, gain)]
    O, lse, O32 = tg.tg_gated_attention_train(d[0], d[1], d[2], d[4], d[5], 1.1)
    single = tg.tg_gated_attention_backward(d[0], d[1], d[2], d[4], d[5], 1.1, O, d[3], lse, O32)
    packed = tg.tg_gated_attention_backward_varlen(d[0], d[1], d[2], d[4], d[5], 1.1, O, d[3], lse,
                                                   torch.as_tensor(cu).to(DEV), 700, O32=O32)
    torch.cuda.synchronize()
    for a, b, name in zip(packed, single, ("ds", "dgain", "dtau")):
        assert torch.equal(a, b), name


def test_backward_varlen_ragged_workload_lengths():
    """The ragged 4-request workload's kept lengths (K = N/8 plus the question:
    1152, 3328, 6656 and 9216 rows), two heads so the fp64 oracle finishes in seconds."""
    lens = [1152, 3328, 6656, 9216]
    Q, K, V, dO, s, gain, cu = _packed(lens, 2, 1, 128, 4)
    O_ref, lse_ref = _oracle_forward(Q, K, s, V, gain, 1.1, cu)
    O32 = torch.as_tensor(O_ref, dtype=torch.float32)
    got = _gpu_backward_varlen(Q, K, V, dO, s, gain, 1.1, cu, O32.to(torch.bfloat16).to(DEV), O32.to(DEV),
                               torch.as_tensor(lse_ref, dtype=torch.float32).to(DEV))
    assert_kernel_close(got, _oracle_per_request(Q, K, V, dO, s, gain, 1.1, cu))
    # a constant added to a request's scores leaves its softmax rows unchanged: the
    # request's score gradients sum to zero
    ds = got[0]
    for b in range(len(lens)):
        seg = ds[cu[b]:cu[b + 1]]
        assert abs(seg.sum()) <= 1e-3 * np.abs(seg).sum()
    assert tg.tg_get_device_error() == 0


def test_backward_varlen_malformed_offsets_set_the_status_bit():
    Q, K, V, dO, s, gain, _ = _packed([100, 50], 4, 2, 64, 9)
    d = [t.to(DEV) for t in (Q, K, V, dO, s, gain)]
    O, lse, O32 = tg.tg_gated_attention_train(d[0], d[1], d[2], d[4], d[5], 1.1)
    bad = torch.tensor([0, 100, 50, 150], dtype=torch.int32, device=DEV)  # decreasing
    tg.tg_gated_attention_backward_varlen(d[0], d[1], d[2], d[4], d[5], 1.1, O, d[3], lse, bad, 100, O32=O32)
    assert tg.tg_get_device_error() & tg.TG_DEVERR_BAD_SEQLENS
    # the context is still usable and a well-formed call is clean afterwards
    good = torch.tensor([0, 100, 150], dtype=torch.int32, device=DEV)
    tg.tg_gated_attention_backward_varlen(d[0], d[1], d[2], d[4], d[5], 1.1, O, d[3], lse, good, 100, O32=O32)
    assert tg.tg_get_device_error() == 0
