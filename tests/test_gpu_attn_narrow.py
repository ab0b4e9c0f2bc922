"""The tensor-core attention for entries of width 128 (16, 32 or 64 heads, bf16
or FP4 rows) against the float64 oracle ("读完这篇，你就搞懂 DeepSeek v4 了",
注意力计算, eq. 9; FP4 rows as "Recall之王", FP4 主KV缓存): one tile, several
tiles with the last-CTA combine, ragged and empty selections, the window tile,
dense rows, more queries than one launch's partials hold, and the same bits
for a query alone and inside a batch."""
import numpy as np
import pytest
import torch

import kv_cache_csa2_b200 as K
import oracle as O
from kv_cache_csa2_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(autouse=True)
def _device_clean():
    yield
    K.csa2_device_error()


def _case(seed, B, Q, Ha, N, k):
    r = np.random.default_rng(seed)
    q = I.f32_to_bf16_bits(r.standard_normal((B, Q, Ha, D)).astype(np.float32))
    kv = I.f32_to_bf16_bits(r.standard_normal((B, N, D)).astype(np.float32))
    topk = np.full((B, Q, k), -1, dtype=np.int32)
    for b in range(B):
        for t in range(Q):
            n = int(r.integers(0, k + 1)) if (b + t) % 3 == 2 else k
            topk[b, t, :n] = np.sort(r.choice(N, size=n, replace=False))
    return q, kv, topk


def _kv_values(kv, fp4):
    if not fp4:
        return O.bf16_bits_to_float(kv)
    B, N, _ = kv.shape
    return O.fp4_unpack(*O.fp4_pack(O.bf16_bits_to_float(kv.reshape(-1, D)))).reshape(B, N, D)


def _attn(q, kv, topk, fp4, **kw):
    kvd = U.dev_bf16(kv)
    if fp4:
        codes, scales = K.csa2_fp4_pack(kvd)
        return K.csa2_sparse_attn(U.dev_bf16(q), codes, U.dev(topk), D ** -0.5, kv_scales=scales, **kw)
    return K.csa2_sparse_attn(U.dev_bf16(q), kvd, U.dev(topk), D ** -0.5, **kw)


@pytest.mark.parametrize("Ha", [16, 32, 64])
@pytest.mark.parametrize("fp4", [False, True])
@pytest.mark.parametrize("k", [1, 128, 129, 1000])
def test_narrow_parity(Ha, fp4, k):
    B, Q, N = 2, 3, 3000
    q, kv, topk = _case(41 + k, B, Q, Ha, N, k)
    out, lse = _attn(q, kv, topk, fp4)
    o, _, l = O.sparse_attn(O.bf16_bits_to_float(q), _kv_values(kv, fp4), topk, D ** -0.5)
    U.check_attn(U.host_bf16(out), lse.cpu().numpy().astype(np.float64), o, l, f"Ha{Ha} fp4{fp4} k{k}")


def test_narrow_many_queries_several_launches():
    """More queries than one launch's partials hold (64 heads, 8 tiles per
    query): the queries run in several launches over the same counters."""
    B, Q, Ha, N, k = 2, 200, 64, 4000, 1000
    q, kv, topk = _case(42, B, Q, Ha, N, k)
    out, lse = _attn(q, kv, topk, False)
    for b, t in [(0, 0), (0, 199), (1, 57), (1, 123)]:
        o, _, l = O.sparse_attn(O.bf16_bits_to_float(q[b:b + 1, t:t + 1]), O.bf16_bits_to_float(kv[b:b + 1]),
                                topk[b:b + 1, t:t + 1], D ** -0.5)
        U.check_attn(U.host_bf16(out[b:b + 1, t:t + 1]), lse[b:b + 1, t:t + 1].cpu().numpy().astype(np.float64),
                     o, l, f"b{b} t{t}")


def test_narrow_query_alone_equals_batched():
    B, Q, Ha, N, k = 1, 64, 16, 5000, 256
    q, kv, topk = _case(43, B, Q, Ha, N, k)
    qd, td = U.dev_bf16(q), U.dev(topk)
    codes, scales = K.csa2_fp4_pack(U.dev_bf16(kv))
    big_out, big_lse = K.csa2_sparse_attn(qd, codes, td, D ** -0.5, kv_scales=scales)
    for t in (0, 31, 63):
        one_out, one_lse = K.csa2_sparse_attn(qd[:, t:t + 1].contiguous(), codes, td[:, t:t + 1].contiguous(),
                                              D ** -0.5, kv_scales=scales)
        assert torch.equal(one_out, big_out[:, t:t + 1]) and torch.equal(one_lse, big_lse[:, t:t + 1])


@pytest.mark.parametrize("fp4", [False, True])
def test_narrow_window_and_dense(fp4):
    r = np.random.default_rng(44)
    B, Q, Ha, N, k, R, W = 2, 3, 16, 2000, 300, 200, 128
    q, kv, topk = _case(45, B, Q, Ha, N, k)
    win = I.f32_to_bf16_bits(r.standard_normal((B, R, D)).astype(np.float32))
    we = r.integers(0, R + 1, size=(B, Q)).astype(np.int32)
    kvd = U.dev_bf16(kv)
    if fp4:
        codes, scales = K.csa2_fp4_pack(kvd)
        out, lse = K.csa2_sparse_attn_swa(U.dev_bf16(q), codes, U.dev(topk), D ** -0.5, U.dev_bf16(win), U.dev(we), W,
                                          kv_scales=scales)
    else:
        out, lse = K.csa2_sparse_attn_swa(U.dev_bf16(q), kvd, U.dev(topk), D ** -0.5, U.dev_bf16(win), U.dev(we), W)
    o, _, l = O.sparse_attn_swa(O.bf16_bits_to_float(q), _kv_values(kv, fp4), topk, O.bf16_bits_to_float(win), we,
                                W, D ** -0.5)
    U.check_attn(U.host_bf16(out), lse.cpu().numpy().astype(np.float64), o, l, "window")
    nv = r.integers(0, 700, size=(B, Q)).astype(np.int32)
    kvs = kv[:, :700].copy()
    if fp4:
        codes, scales = K.csa2_fp4_pack(U.dev_bf16(kvs))
        out, lse = K.csa2_dense_attn(U.dev_bf16(q), codes, D ** -0.5, n_visible=U.dev(nv), kv_scales=scales)
    else:
        out, lse = K.csa2_dense_attn(U.dev_bf16(q), U.dev_bf16(kvs), D ** -0.5, n_visible=U.dev(nv))
    o, _, l = O.dense_attn(O.bf16_bits_to_float(q), _kv_values(kvs, fp4), D ** -0.5, n_visible=nv)
    U.check_attn(U.host_bf16(out), lse.cpu().numpy().astype(np.float64), o, l, "dense")
