"""Both attention kernels against the fp64 oracle, through the C ABI.

tg_gated_attention (and its varlen / training forms) runs one of two kernels: the
two-tile kernel (one CTA per 256 query rows, head and request) or, when that grid would
hold at most 1.5 CTAs per SM, the persistent kernel (one CTA per SM working through single
128-row query tiles).  Heads are independent problems, so replicating the heads r times
(Q, K, V and the gains tiled along the head axis) moves a call to the two-tile kernel
without changing what each head computes: every case here runs on both kernels, is held
to the oracle's tolerance on each, and the r replicas of every head must agree bitwise.
"""
import numpy as np
import pytest
import torch

import oracle
import learned_token_pruning_mlp_b200 as tg
from test_gpu_parity import _attn_inputs, check_attention

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
KERNELS = ["persistent", "two_tile"]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from learned_token_pruning_mlp_b200 import build
    build.build()
    tg.tg_get_device_error()
    yield


def uses_persistent(max_seqlen, Hq, B=1):
    """The library's rule: the persistent kernel when the two-tile grid has at most 1.5
    CTAs per SM."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return 2 * (-(-max_seqlen // 256)) * Hq * B <= 3 * sms


def replication_for(kernel, max_seqlen, Hq, B=1):
    """How many times to replicate the heads so that the call runs ``kernel``."""
    if kernel == "persistent":
        if not uses_persistent(max_seqlen, Hq, B):
            pytest.skip("this size runs the two-tile kernel at any head count")
        return 1
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    per_head = -(-max_seqlen // 256) * Hq * B
    r = 1 if not uses_persistent(max_seqlen, Hq, B) else 3 * sms // (2 * per_head) + 1
    assert not uses_persistent(max_seqlen, Hq * r, B)
    return r


def tile_heads(r, Q, K, V, gain):
    return (Q.repeat(1, r, 1), K.repeat(1, r, 1), V.repeat(1, r, 1), None if gain is None else gain.repeat(r))


def first_replica(t, Hq, r):
    """Heads 0..Hq-1 of a head-replicated output, after checking every replica equals them."""
    parts = t.reshape(t.shape[0], r, Hq, *t.shape[2:])
    for i in range(1, r):
        assert torch.equal(parts[:, i], parts[:, 0]), f"replica {i} differs"
    return parts[:, 0].contiguous()


def run(kernel, fn, Q, K, V, s, gain, tau, *rest, max_seqlen=None, B=1, **kw):
    """fn(Q, K, V, s, gain, tau, *rest) on the requested kernel; outputs for the original heads."""
    Hq = Q.shape[1]
    r = replication_for(kernel, max_seqlen if max_seqlen is not None else Q.shape[0], Hq, B)
    Qr, Kr, Vr, gr = tile_heads(r, Q, K, V, gain)
    out = fn(Qr.to(DEV), Kr.to(DEV), Vr.to(DEV), None if s is None else s.to(DEV),
             None if gr is None else gr.to(DEV), tau, *rest, **kw)
    torch.cuda.synchronize()
    assert tg.tg_get_device_error() == 0
    if isinstance(out, tuple):
        return tuple(None if o is None else first_replica(o, Hq, r).cpu() for o in out)
    return first_replica(out, Hq, r).cpu()


def test_the_two_layer_shapes_of_the_bench_take_different_kernels():
    assert not uses_persistent(8704, 16)   # 128k context, K = 8192: 34 x 16 = 544 CTAs
    assert uses_persistent(1536, 16)       # 16k context, K = 1024: 6 x 16 = 96 CTAs
    assert uses_persistent(2560, 16)       # 160 CTAs on 148 SMs
    assert not uses_persistent(4608, 16)   # 288 CTAs


CASES = [(192, 4, 2, 64, 1.1), (300, 4, 2, 64, 2.5), (1000, 16, 8, 128, 1.1), (640, 4, 4, 128, -0.7),
         (257, 8, 2, 128, 0.0), (129, 2, 1, 64, 1e-3), (1, 4, 2, 128, 1.1), (2048, 16, 8, 128, 1.1)]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("S,Hq,Hkv,D,tau", CASES)
def test_gated_attention_on_both_kernels(kernel, S, Hq, Hkv, D, tau):
    Q, K, V, s, gain = _attn_inputs(S, Hq, Hkv, D, 3 * S + Hq + D)
    O = run(kernel, tg.tg_gated_attention, Q, K, V, s, gain, tau)
    check_attention(O.float().numpy(), Q, K, V, s, gain, tau, max_abs_below=2.0)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("D", [64, 128])
def test_rescale_stress_on_both_kernels(kernel, D):
    # scores that climb by ~18 base-2 logit units every 64 keys with one jump of ~140:
    # the running max grows past the rescale threshold in both halves of most KV tiles
    S = 1000
    Q, K, V, s, gain = _attn_inputs(S, 4, 2, D, 91)
    s = 0.2 * torch.arange(S, dtype=torch.float32)
    s[700:] += 100.0
    gain = torch.ones(4)
    O = run(kernel, tg.tg_gated_attention, Q, K, V, s, gain, 1.1)
    assert torch.isfinite(O.float()).all()
    check_attention(O.float().numpy(), Q, K, V, s, gain, 1.1, max_abs_below=2.0)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("S,Hq,Hkv,D,tau", [(700, 16, 8, 128, 1.1), (129, 2, 1, 128, -0.7), (200, 4, 2, 64, 0.0)])
def test_plain_causal_attention_on_both_kernels(kernel, S, Hq, Hkv, D, tau):
    Q, K, V, _, _ = _attn_inputs(S, Hq, Hkv, D, S + D)
    O = run(kernel, tg.tg_gated_attention, Q, K, V, None, None, tau)
    check_attention(O.float().numpy(), Q, K, V, np.zeros(S, np.float32), np.zeros(Hq, np.float32), tau)


@pytest.mark.parametrize("kernel", KERNELS)
def test_varlen_on_both_kernels(kernel):
    lens = [300, 1, 0, 1000, 129]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Q, K, V, s, gain = _attn_inputs(int(cu[-1]), 4, 2, 128, 5)
    O = run(kernel, tg.tg_gated_attention_varlen, Q, K, V, s, gain, 1.1, torch.as_tensor(cu).to(DEV), max(lens),
            max_seqlen=max(lens), B=len(lens))
    check_attention(O.float().numpy(), Q, K, V, s, gain, 1.1, cu=cu)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("S,Hq,Hkv,D,tau", [(700, 16, 8, 128, 1.1), (1000, 4, 2, 64, -0.7), (257, 8, 2, 128, 2.5)])
def test_training_forward_on_both_kernels(kernel, S, Hq, Hkv, D, tau):
    Q, K, V, s, gain = _attn_inputs(S, Hq, Hkv, D, S + 7)
    O, lse, O32 = run(kernel, tg.tg_gated_attention_train, Q, K, V, s, gain, tau)
    assert torch.equal(O32.to(torch.bfloat16), O)     # O is the bf16 rounding of O32
    check_attention(O.float().numpy(), Q, K, V, s, gain, tau, max_abs_below=2.0)
    check_attention(O32.numpy(), Q, K, V, s, gain, tau, fp32_out=True, max_abs_below=2.0)
    ref = oracle.gated_attention_lse(Q, K, s, gain, tau)
    assert np.max(np.abs(lse.numpy() - ref)) <= 4e-3
    O2 = run(kernel, tg.tg_gated_attention, Q, K, V, s, gain, tau)
    assert torch.equal(O, O2)                         # the extra outputs do not change O


@pytest.mark.parametrize("kernel", KERNELS)
def test_training_forward_varlen_on_both_kernels(kernel):
    lens = [300, 1, 517, 129]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Q, K, V, s, gain = _attn_inputs(int(cu[-1]), 8, 2, 128, 77)
    O, lse, O32 = run(kernel, tg.tg_gated_attention_train_varlen, Q, K, V, s, gain, 1.1,
                      torch.as_tensor(cu).to(DEV), max(lens), max_seqlen=max(lens), B=len(lens))
    check_attention(O.float().numpy(), Q, K, V, s, gain, 1.1, cu=cu)
    check_attention(O32.numpy(), Q, K, V, s, gain, 1.1, cu=cu, fp32_out=True)


@pytest.mark.parametrize("kernel", KERNELS)
def test_varlen_request_past_max_seqlen_sets_the_status_bit(kernel):
    """A request longer than the rows max_seqlen covers is reported, not silently cut; a
    well-formed call afterwards is clean."""
    lens = [300, 1000]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Q, K, V, s, gain = _attn_inputs(int(cu[-1]), 4, 2, 128, 12)
    r = replication_for(kernel, 100, 4, B=2)  # the kernel the bad call (max_seqlen 100) runs; the good one runs it too
    Qr, Kr, Vr, gr = tile_heads(r, Q, K, V, gain)
    d_cu = torch.as_tensor(cu).to(DEV)
    tg.tg_get_device_error()
    tg.tg_gated_attention_varlen(Qr.to(DEV), Kr.to(DEV), Vr.to(DEV), s.to(DEV), gr.to(DEV), 1.1, d_cu, 100)
    torch.cuda.synchronize()
    assert tg.tg_get_device_error() & tg.TG_DEVERR_BAD_SEQLENS
    tg.tg_gated_attention_varlen(Qr.to(DEV), Kr.to(DEV), Vr.to(DEV), s.to(DEV), gr.to(DEV), 1.1, d_cu, 1000)
    torch.cuda.synchronize()
    assert tg.tg_get_device_error() == 0
