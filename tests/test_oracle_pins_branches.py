"""Pins of the oracle's sliding-window branch, its log-sum-exp merge with the
CSA2 branch, HCA compression and HCA (dense) attention: hand-worked goldens,
closed forms and special cases, and checks against torch's float64 scaled
dot-product attention (a library routine that shares nothing with the
oracle)."""
import numpy as np
import pytest
import torch

import oracle as O
from tests.conftest import load_golden

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _sdpa(q, rows, scale, mask=None):
    """torch float64 SDPA of one query's heads q [Ha, D] over rows [n, D] (K = V)."""
    qt = torch.from_numpy(q)[None, :, None, :]               # [1, Ha, 1, D]
    kt = torch.from_numpy(rows)[None, None].expand(1, q.shape[0], -1, -1)
    m = None if mask is None else torch.from_numpy(mask)[None, None, None, :]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, attn_mask=m, scale=scale)[0, :, 0].numpy()


def _lse(q, rows, scale):
    return np.logaddexp.reduce(scale * (q @ rows.T), axis=1)


# ------------------------------------------------------------------ HCA compression

@pytest.mark.parametrize("case", ["two_groups", "bias_only"])
def test_hca_compress_golden(case):
    d, num = load_golden("hca_hand.json")
    c = d["compress"][case]
    e, e16 = O.compress_hca(np.array(num(c["c"]), float), np.array(num(c["z"]), float),
                            np.array(num(c["bias"]), float), c["m"])
    assert np.allclose(e, np.array(c["expect"]), atol=1e-6)
    assert np.array_equal(e16, O.round_to_bf16(e))


@pytest.mark.parametrize("m", [1, 3, 16, 128])
def test_hca_compress_closed_forms(m):
    r = np.random.default_rng(40)
    B, N, D = 2, 3, 5
    T = N * m + (m - 1)                                   # a trailing partial group is dropped
    # constant tokens: every entry is that constant
    c = np.full((B, T, D), 1.75)
    z = r.standard_normal((B, T, D))
    bias = r.standard_normal((m, D))
    e, _ = O.compress_hca(c, z, bias, m)
    assert e.shape == (B, N, D) and np.allclose(e, 1.75, rtol=1e-14)
    # zero logits and bias: the plain mean of each group
    c = r.standard_normal((B, T, D))
    e, _ = O.compress_hca(c, np.zeros_like(c), np.zeros((m, D)), m)
    want = c[:, :N * m].reshape(B, N, m, D).mean(axis=2)
    assert np.allclose(e, want, rtol=1e-12, atol=1e-14)
    # one logit far above the others: that token's value
    z = np.zeros_like(c)
    z[:, 0::m] = 80.0                                   # first token of each group dominates
    e, _ = O.compress_hca(c, z, np.zeros((m, D)), m)
    assert np.allclose(e, c[:, 0:N * m:m], rtol=1e-12, atol=1e-12)


def test_hca_compress_is_csa_compress_without_the_earlier_block():
    """CSA's entry j joins blocks j-1 and j; with the earlier block's bias at
    -inf it weighs block j alone, which is HCA's entry j (bias = the later
    half)."""
    r = np.random.default_rng(41)
    m, B, N, D = 4, 2, 5, 6
    c = r.standard_normal((B, N * m, D))
    z = r.standard_normal((B, N * m, D))
    b2 = r.standard_normal((m, D))
    csa_bias = np.concatenate([np.full((m, D), -np.inf), b2])
    e_csa, _ = O.compress(c, z, csa_bias, m)
    e_hca, _ = O.compress_hca(c, z, b2, m)
    assert np.allclose(e_csa, e_hca, rtol=1e-13, atol=1e-14)


# ------------------------------------------------------------------ HCA attention

def test_dense_attn_golden():
    d, num = load_golden("hca_hand.json")
    a = d["attn"]
    q = np.array(num(a["q"]), float)
    kv = np.array(num(a["kv"]), float)
    o, o16, lse = O.dense_attn(q, kv, a["scale"])
    assert np.allclose(o[0, 0, 0], a["expect_all"]["o"], atol=1e-7)
    assert abs(np.exp(lse[0, 0, 0]) - a["expect_all"]["lse_exp"]) < 1e-6
    o, _, lse = O.dense_attn(q, kv, a["scale"], n_visible=np.array([[2]]))
    assert np.allclose(o[0, 0, 0], a["expect_nvis2"]["o"], atol=1e-7)
    assert abs(np.exp(lse[0, 0, 0]) - a["expect_nvis2"]["lse_exp"]) < 1e-6


def test_dense_attn_equals_causally_masked_sdpa():
    r = np.random.default_rng(42)
    B, Q, Ha, D, N = 2, 4, 3, 8, 11
    q = r.standard_normal((B, Q, Ha, D))
    kv = r.standard_normal((B, N, D))
    nv = np.array([[11, 7, 1, 4], [3, 11, 9, 2]])
    o, _, lse = O.dense_attn(q, kv, 0.4, n_visible=nv)
    for b in range(B):
        for t in range(Q):
            mask = np.arange(N) < nv[b, t]
            assert np.allclose(o[b, t], _sdpa(q[b, t], kv[b], 0.4, mask), rtol=1e-12, atol=1e-13)
            assert np.allclose(lse[b, t], _lse(q[b, t], kv[b, :nv[b, t]], 0.4), rtol=1e-12)
    o, _, lse = O.dense_attn(q, kv, 0.4, n_visible=np.zeros((B, Q), int))
    assert np.all(o == 0) and np.all(lse == -np.inf)


# ------------------------------------------------------------------ window branch and merge

def test_swa_and_merge_golden():
    d, num = load_golden("swa_hand.json")
    q = np.array(num(d["q"]), float)
    kv = np.array(d["kv"], float)
    win = np.array(d["win"], float)
    topk = np.array(d["topk"])
    we = np.array(d["win_end"])
    x = d["expect"]
    o_c, _, l_c = O.sparse_attn(q, kv, topk, 1.0)
    o_w, l_w = O.swa_attn(q, win, we, d["W"], 1.0)
    assert np.allclose(o_c[0, 0, 0], x["o_csa"], atol=1e-7) and abs(np.exp(l_c[0, 0, 0]) - x["lse_csa_exp"]) < 1e-6
    assert np.allclose(o_w[0, 0, 0], x["o_win"], atol=1e-7) and abs(np.exp(l_w[0, 0, 0]) - x["lse_win_exp"]) < 1e-5
    o, o16, lse = O.sparse_attn_swa(q, kv, topk, win, we, d["W"], 1.0)
    assert np.allclose(o[0, 0, 0], x["o"], atol=1e-7) and abs(np.exp(lse[0, 0, 0]) - x["lse_exp"]) < 1e-5
    assert np.array_equal(o16, O.round_to_bf16(o))


def test_merge_equals_one_softmax_over_the_union_of_rows():
    """The merged branches equal torch SDPA over the selected entries and the
    window rows together."""
    r = np.random.default_rng(43)
    B, Q, Ha, D, N, R, W, k = 2, 3, 4, 16, 40, 30, 8, 6
    q = r.standard_normal((B, Q, Ha, D))
    kv = r.standard_normal((B, N, D))
    win = r.standard_normal((B, R, D))
    topk = np.full((B, Q, k), -1)
    we = np.array([[30, 5, 0], [17, 30, 3]])              # full, short (e < W) and empty windows
    for b in range(B):
        for t in range(Q):
            n = [k, 3, 0][t]
            topk[b, t, :n] = np.sort(r.choice(N, n, replace=False))
    o, _, lse = O.sparse_attn_swa(q, kv, topk, win, we, W, 0.25)
    for b in range(B):
        for t in range(Q):
            ids = topk[b, t][topk[b, t] >= 0]
            rows = np.concatenate([kv[b, ids], win[b, max(0, we[b, t] - W):we[b, t]]])
            if rows.shape[0] == 0:
                assert np.all(o[b, t] == 0) and np.all(lse[b, t] == -np.inf)
                continue
            assert np.allclose(o[b, t], _sdpa(q[b, t], rows, 0.25), rtol=1e-12, atol=1e-13)
            assert np.allclose(lse[b, t], _lse(q[b, t], rows, 0.25), rtol=1e-12)


def test_merge_with_an_empty_branch_is_the_other_branch():
    r = np.random.default_rng(44)
    o1 = r.standard_normal((3, 5))
    l1 = r.standard_normal(3)
    o, lse = O.lse_merge(o1, l1, np.zeros((3, 5)), np.full(3, -np.inf))
    assert np.allclose(o, o1, rtol=1e-15) and np.allclose(lse, l1, rtol=1e-15)
    o, lse = O.lse_merge(np.zeros((3, 5)), np.full(3, -np.inf), o1, l1)
    assert np.allclose(o, o1, rtol=1e-15) and np.allclose(lse, l1, rtol=1e-15)
    o, lse = O.lse_merge(np.zeros((3, 5)), np.full(3, -np.inf), np.zeros((3, 5)), np.full(3, -np.inf))
    assert np.all(o == 0) and np.all(lse == -np.inf)


def test_group_layer_with_window_merges_its_branch():
    """run_group's attention on a layer given a window equals sparse_attn_swa
    over that layer's selection."""
    r = np.random.default_rng(45)
    B, Q, H, d, N, Ha, D, k, R, W = 2, 1, 2, 8, 50, 2, 8, 5, 12, 4
    kv = r.standard_normal((B, N, D))
    ik = r.standard_normal((B, N, d))
    win = r.standard_normal((B, R, D))
    we = np.full((B, Q), R)
    layers = [{"q_attn": r.standard_normal((B, Q, Ha, D)), "q_index": r.standard_normal((B, Q, H, d)),
               "w_index": r.random((B, Q, H)), "swa": (win, we, W)},
              {"q_attn": r.standard_normal((B, Q, Ha, D))}]
    res = O.run_group(["full", "reuse"], layers, kv, ik, k, 0.3)
    for i in range(2):
        o, _, lse = (O.sparse_attn_swa(layers[i]["q_attn"], kv, res[i]["topk"], win, we, W, 0.3) if i == 0
                     else O.sparse_attn(layers[i]["q_attn"], kv, res[i]["topk"], 0.3))
        assert np.array_equal(res[i]["o"], o) and np.array_equal(res[i]["lse"], lse)


# ------------------------------------------------------------------ FP4 indexer, bf16 scores

def _fp4_exact_rows(r, shape, scale_exp):
    """Rows whose every 16-channel block holds E2M1 values times one power-of-two
    scale, with a +-6 in each block (so quantising them again changes nothing)."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    v = grid[r.integers(0, 8, shape)] * np.where(r.random(shape) < 0.5, -1.0, 1.0)
    v.reshape(-1, 16)[:, 0] = 6.0
    return v * 2.0 ** scale_exp


def test_index_fp4_golden():
    """d = 16, one head: q = (6, 1.5, 0, ..), k = (1.5, 1, 0, ..), both FP4
    exact with scale 1 (absmax 6); q.k = 9 + 1.5 = 10.5; w = 0.1 gives
    1.05000001...; bfloat16 keeps 8 significant bits, so in [1, 2) its values
    are 1/128 apart and the neighbours are 1 + 6/128 = 1.046875 (0.0031 away)
    and 1 + 7/128 = 1.0546875 (0.0047 away): the score is 1.046875."""
    q = np.zeros((1, 1, 1, 16))
    q[..., 0], q[..., 1] = 6.0, 1.5
    k = np.zeros((1, 2, 16))
    k[0, 0, 0], k[0, 0, 1], k[0, 0, 2] = 1.5, 1.0, 6.0        # the 6 pairs with q's 0
    k[0, 1, 0] = -6.0                                         # q.k = -36: ReLU gives 0
    w = np.array([[[np.float32(0.1)]]], dtype=np.float64)
    s = O.index_scores_fp4(q, w, k)
    assert s[0, 0, 0] == 1.046875 and s[0, 0, 1] == 0.0


def test_index_fp4_on_fp4_exact_inputs_is_rounded_exact_score():
    r = np.random.default_rng(46)
    q = _fp4_exact_rows(r, (2, 3, 4, 64), -3)
    k = _fp4_exact_rows(r, (2, 50, 64), -2)
    w = r.random((2, 3, 4))
    nv = np.array([[50, 10, 0], [1, 49, 50]])
    s = O.index_scores_fp4(q, w, k, n_visible=nv)
    assert np.array_equal(s, O.round_to_bf16(O.index_scores(q, w, k, n_visible=nv)))
    assert np.array_equal(s, O.round_to_bf16(s))              # bf16 values
    assert np.all(np.isneginf(s[0, 2])) and np.all(np.isneginf(s[1, 0, 1:]))


def test_index_fp4_quantises_q_and_k_like_the_main_kv_format():
    r = np.random.default_rng(47)
    q = r.standard_normal((1, 2, 3, 32))
    k = r.standard_normal((1, 40, 32))
    w = r.random((1, 2, 3))
    qd = O.fp4_unpack(*O.fp4_pack(q.reshape(-1, 32))).reshape(q.shape)
    kd = O.fp4_unpack(*O.fp4_pack(k.reshape(-1, 32))).reshape(k.shape)
    s = O.index_scores_fp4(q, w, k)
    # scores over the dequantised values, computed directly (ReLU, weighted head sum)
    direct = np.einsum("bqh,bqhn->bqn", w, np.maximum(np.einsum("bqhd,bnd->bqhn", qd, kd), 0.0))
    assert np.allclose(s, direct, rtol=2.0 ** -8, atol=0)
    assert not np.allclose(s, O.index_scores(q, w, k), rtol=1e-3)   # quantisation matters
    pool = np.sort(r.choice(40, (1, 2, 7)), axis=-1)
    sp = O.index_scores_fp4(q, w, k, pool=pool)
    assert np.array_equal(sp, np.take_along_axis(s, pool, axis=-1))
