"""Host threads calling the library at once, each on its own CUDA stream.

The C ABI allows concurrent calls from several host threads on different streams: the
per-device set-up (kernel attributes, symbol addresses) runs once under a library lock,
and such calls share only the status word.  A fresh process (so that the set-up itself
is raced) starts four threads together; each runs one call of the hot path repeatedly on
its own stream.  Every result must equal, bit for bit, the same call made afterwards on
one thread.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import threading
import torch
import learned_token_pruning_mlp_b200 as tg
from learned_token_pruning_mlp_b200 import workloads as W

dev = torch.device("cuda:0")
torch.cuda.set_device(dev)
w = W.get("tiny_n512")
hidden, W1, b1, W2, b2 = [t.to(dev) for t in W.gate_inputs(w)]
mask = W.doc_mask(w).to(dev)
n = hidden.shape[0]
k = w.segments[0].k
g = torch.Generator().manual_seed(3)
sel = torch.randn(n, generator=g).to(dev)
kept_ref, nk_ref = tg.tg_select_topk(sel, mask, k)  # rows for the gather, made before the race
torch.cuda.synchronize()
S = 700
Q = torch.randn(S, 8, 128, generator=g).to(torch.bfloat16).to(dev)
K = torch.randn(S, 4, 128, generator=g).to(torch.bfloat16).to(dev)
V = torch.randn(S, 4, 128, generator=g).to(torch.bfloat16).to(dev)
s = torch.randn(S, generator=g).to(dev)
gain = (0.5 + torch.rand(8, generator=g)).to(dev)
rows = int(nk_ref.item())

calls = {
    "gate": lambda: tg.tg_gate_score(hidden, W1, b1, W2, b2),
    "topk": lambda: tg.tg_select_topk(sel, mask, k)[0][:rows],  # the kept rows (the rest is unwritten)
    "gather": lambda: tg.tg_gather(hidden, kept_ref[:rows].contiguous())[0],
    "attention": lambda: tg.tg_gated_attention(Q, K, V, s, gain, 1.1),
}
start = threading.Barrier(len(calls))
got = {}
errors = []

def worker(name):
    try:
        torch.cuda.set_device(dev)
        stream = torch.cuda.Stream(dev)
        with torch.cuda.stream(stream):
            start.wait()
            outs = [calls[name]() for _ in range(20)]
        stream.synchronize()
        got[name] = outs
    except Exception as e:  # reported by the main thread
        errors.append(f"{name}: {e!r}")

threads = [threading.Thread(target=worker, args=(name,)) for name in calls]
for t in threads:
    t.start()
for t in threads:
    t.join()
assert not errors, errors
torch.cuda.synchronize()
assert tg.tg_get_device_error() & ~tg.TG_DEVERR_K_GT_NDOC == 0
for name, fn in calls.items():
    ref = fn()
    torch.cuda.synchronize()
    for i, out in enumerate(got[name]):
        assert torch.equal(out.view(torch.uint8), ref.view(torch.uint8)), f"{name} call {i} differs"
print("threads OK")
'''


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from learned_token_pruning_mlp_b200 import build
    build.build()
    yield


def test_threads_on_their_own_streams_match_one_thread():
    r = subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, (r.stdout[-2000:], r.stderr[-4000:])
    assert "threads OK" in r.stdout
