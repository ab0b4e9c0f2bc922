"""The two schedules of the tensor-core attention (64 heads x 512): a query's
128-row tiles spread over several CTAs (few queries) or run in sequence on one
CTA (many queries).  Both compute each tile and the tile-order combine with
the same instructions, so a query's output and lse must be the same bits
whichever schedule runs it -- the batch invariance of the pages ("读完这篇，你就
搞懂 DeepSeek v4 了", 批无关性) across batch sizes -- and match the float64
oracle (注意力计算, eq. 9)."""
import numpy as np
import pytest
import torch

import kv_cache_csa2_b200 as K
import oracle as O
from kv_cache_csa2_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

HA, D = 64, 512


@pytest.fixture(autouse=True)
def _device_clean():
    yield
    K.csa2_device_error()


def _case(seed, B, Q, N, k):
    r = np.random.default_rng(seed)
    q = I.f32_to_bf16_bits(r.standard_normal((B, Q, HA, D)).astype(np.float32))
    kv = I.f32_to_bf16_bits(r.standard_normal((B, N, D)).astype(np.float32))
    topk = np.full((B, Q, k), -1, dtype=np.int32)
    for b in range(B):
        for t in range(Q):
            # every third query keeps a ragged prefix (some all-empty tiles)
            n = int(r.integers(0, k + 1)) if (b + t) % 3 == 2 else k
            topk[b, t, :n] = np.sort(r.choice(N, size=n, replace=False))
    return q, kv, topk


def _both(monkeypatch, call):
    monkeypatch.setenv("CSA2_ATTN_SEQ", "0")
    split = call()
    monkeypatch.setenv("CSA2_ATTN_SEQ", "1")
    seq = call()
    monkeypatch.delenv("CSA2_ATTN_SEQ")
    return split, seq


@pytest.mark.parametrize("B,Q,N,k", [(2, 3, 5000, 2048), (1, 5, 3000, 1000), (2, 2, 900, 129),
                                     (1, 3, 400, 64), (1, 2, 9000, 4096), (3, 1, 2000, 1)])
def test_seq_equals_split_bitwise(B, Q, N, k, monkeypatch):
    q, kv, topk = _case(31, B, Q, N, k)
    args = (U.dev_bf16(q), U.dev_bf16(kv), U.dev(topk), D ** -0.5)
    (o1, l1), (o2, l2) = _both(monkeypatch, lambda: K.csa2_sparse_attn(*args))
    assert torch.equal(o1, o2), "outputs differ between the schedules"
    assert torch.equal(l1, l2), "lse differs between the schedules"
    o, _, l = O.sparse_attn(O.bf16_bits_to_float(q), O.bf16_bits_to_float(kv), topk, D ** -0.5)
    U.check_attn(U.host_bf16(o2), l2.cpu().numpy().astype(np.float64), o, l, f"seq k{k}")


def test_seq_many_queries_per_cta(monkeypatch):
    """More queries than SMs: each CTA runs several queries in a row (the q
    buffer and the accumulator are reused); the default choice takes this
    schedule at this size, and a query's bits equal the split schedule's."""
    B, Q, N, k = 2, 200, 3000, 384
    q, kv, topk = _case(32, B, Q, N, k)
    args = (U.dev_bf16(q), U.dev_bf16(kv), U.dev(topk), D ** -0.5)
    default_out, default_lse = K.csa2_sparse_attn(*args)
    (o1, l1), (o2, l2) = _both(monkeypatch, lambda: K.csa2_sparse_attn(*args))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(default_out, o2) and torch.equal(default_lse, l2)
    # a sample of queries against the oracle
    for b, t in [(0, 0), (0, 199), (1, 77), (1, 150)]:
        o, _, l = O.sparse_attn(O.bf16_bits_to_float(q[b:b + 1, t:t + 1]), O.bf16_bits_to_float(kv[b:b + 1]),
                                topk[b:b + 1, t:t + 1], D ** -0.5)
        U.check_attn(U.host_bf16(o2[b:b + 1, t:t + 1]), l2[b:b + 1, t:t + 1].cpu().numpy().astype(np.float64),
                     o, l, f"seq b{b} t{t}")


def test_seq_single_query_equals_batched(monkeypatch):
    """One query alone (split schedule) against the same query inside a large
    batch (sequential schedule): the same bits."""
    B, Q, N, k = 1, 300, 4000, 2048
    q, kv, topk = _case(33, B, Q, N, k)
    qd, kvd, td = U.dev_bf16(q), U.dev_bf16(kv), U.dev(topk)
    monkeypatch.delenv("CSA2_ATTN_SEQ", raising=False)
    big_out, big_lse = K.csa2_sparse_attn(qd, kvd, td, D ** -0.5)
    for t in (0, 131, 299):
        one_out, one_lse = K.csa2_sparse_attn(qd[:, t:t + 1].contiguous(), kvd, td[:, t:t + 1].contiguous(), D ** -0.5)
        assert torch.equal(one_out, big_out[:, t:t + 1]) and torch.equal(one_lse, big_lse[:, t:t + 1])


def test_seq_window_and_dense_bitwise(monkeypatch):
    """The window tile (sliding-window branch) and the dense rows (HCA) take
    the same schedules."""
    r = np.random.default_rng(34)
    B, Q, N, k, R, W = 2, 3, 3000, 1000, 300, 128
    q, kv, topk = _case(35, B, Q, N, k)
    win = I.f32_to_bf16_bits(r.standard_normal((B, R, D)).astype(np.float32))
    we = r.integers(0, R + 1, size=(B, Q)).astype(np.int32)
    args = (U.dev_bf16(q), U.dev_bf16(kv), U.dev(topk), D ** -0.5, U.dev_bf16(win), U.dev(we), W)
    (o1, l1), (o2, l2) = _both(monkeypatch, lambda: K.csa2_sparse_attn_swa(*args))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    nv = r.integers(0, 1500, size=(B, Q)).astype(np.int32)
    dense = (U.dev_bf16(q), U.dev_bf16(kv[:, :1500].copy()), D ** -0.5)
    (o1, l1), (o2, l2) = _both(monkeypatch, lambda: K.csa2_dense_attn(*dense, n_visible=U.dev(nv)))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
