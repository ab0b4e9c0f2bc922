"""The Full-layer indexer fused with its streaming top-k (many queries, no
pool) against the same call split into scoring and selection (bit for bit:
same scores, exact selection both ways) and against the oracle's selection on
sampled queries."""
import numpy as np
import pytest

import kv_cache_csa2_b200 as K
import oracle as O
from kv_cache_csa2_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _device_clean():
    yield
    K.csa2_device_error()


def _case(r, B, Q, H, d, N, var=None, wdist="uniform"):
    v = 1.0 / d if var is None else var
    q = I.f32_to_bf16_bits((r.standard_normal((B, Q, H, d)) * np.sqrt(v)).astype(np.float32))
    k = I.f32_to_bf16_bits((r.standard_normal((B, N, d)) * np.sqrt(v)).astype(np.float32))
    w = (r.random((B, Q, H)) if wdist == "uniform" else r.standard_normal((B, Q, H))).astype(np.float32)
    return q, w, k


@pytest.mark.parametrize("B,Q,H,d,N,k_top,causal,wdist", [
    (1, 600, 64, 128, 20000, 2048, True, "normal"),      # prefill-like: 150 groups of 4 queries
    (2, 300, 8, 64, 9000, 256, False, "uniform"),        # small heads (16-wide groups)
    (1, 601, 2, 64, 5000, 700, True, "uniform"),         # ReLU with 2 heads: many exact-zero ties; ragged group
    (1, 592, 64, 128, 3000, 2048, True, "normal"),       # fewer visible entries than k for early queries
])
def test_fused_topk_equals_split_and_oracle(B, Q, H, d, N, k_top, causal, wdist, monkeypatch):
    r = np.random.default_rng(70)
    q, w, k = _case(r, B, Q, H, d, N, var=1.0 if wdist == "normal" else None, wdist=wdist)
    nv = None
    if causal:               # query i sees entries below N - Q/4 + i/4 (a chunk at the end of the context)
        nv = np.broadcast_to(np.minimum(N, N - Q // 4 + np.arange(Q) // 4 + 1), (B, Q)).astype(np.int32).copy()
        if N < 4 * k_top:
            nv[:, :8] = np.arange(1, 9) * 37                # a few queries with fewer than k visible
    dq, dw, dk = U.dev_bf16(q), U.dev(w), U.dev_bf16(k)
    dnv = U.dev(nv) if nv is not None else None
    K.reset_launch_counts()
    fused, _ = K.csa2_index_topk(K.FULL, dq, dw, dk, k_top, n_visible=dnv)
    n = K.launch_counts()
    assert n["index_scores"] == 1 and n["topk"] == 0          # one kernel, no selection launch
    monkeypatch.setenv("CSA2_NO_FUSED_TOPK", "1")
    split, _ = K.csa2_index_topk(K.FULL, dq, dw, dk, k_top, n_visible=dnv)
    monkeypatch.delenv("CSA2_NO_FUSED_TOPK")
    fused, split = fused.cpu().numpy(), split.cpu().numpy()
    assert np.array_equal(fused, split)
    # the oracle's selection rule on sampled queries
    sample = np.unique(np.concatenate([[0, Q - 1], r.choice(Q, 12, replace=False)]))
    s = O.index_scores(O.bf16_bits_to_float(q[:, sample]), w[:, sample].astype(np.float64),
                       O.bf16_bits_to_float(k), n_visible=nv[:, sample] if nv is not None else None)
    for b in range(B):
        for j, t in enumerate(sample):
            U.check_selection(fused[b, t], np.arange(N), s[b, j], k_top, f"b{b} q{t}")
