"""B200-native (sm_100a) library for the TokenGate pruned-prefill hot path.

The four calls (gate MLP scoring, top-K selection with the question kept, gather
of the kept rows, token-gated causal GQA attention) run in hand-written CUDA
kernels behind the C ABI of include/tokengate.h; this package is the thin
ctypes binding over it (``_lib``) plus seeded synthetic workloads
(``workloads``).  The projections around the attention of a pruned layer
(QKV with per-head norm and rotary embedding at the kept tokens' positions, and
the output projection with the residual add) sit behind the same ABI.  There is
no CPU fallback.
"""
from ._lib import (  # noqa: F401
    TG_DEVERR_BAD_SEQLENS,
    TG_DEVERR_CAPACITY,
    TG_DEVERR_INDEX_OOB,
    TG_DEVERR_K_GT_NDOC,
    TG_DEVERR_TIMEOUT,
    TokenGateError,
    lib,
    tg_abi_version,
    tg_gate_score,
    tg_gated_attention,
    tg_gated_attention_backward,
    tg_gated_attention_backward_noalloc,
    tg_gated_attention_backward_varlen,
    tg_gated_attention_backward_varlen_workspace,
    tg_gated_attention_backward_workspace,
    tg_gated_attention_train,
    tg_gated_attention_train_varlen,
    tg_gated_attention_varlen,
    tg_gather,
    tg_get_device_error,
    tg_linear,
    tg_probe_wait_timeout,
    tg_qkv_rope,
    tg_select_fused,
    tg_select_fused_workspace,
    tg_select_random_k,
    tg_select_topk,
    tg_select_topk_sweep,
    tg_select_topk_varlen,
)
