"""Pins for the float64 oracle: every check compares it with something other
than itself -- hand-worked examples (tests/golden), closed forms, invariants,
library routines that implement a special case (torch SDPA, torch/ml_dtypes
float8/float4 rounding, scipy logsumexp), and brute force on tiny inputs.
Runs on the CPU."""
import itertools

import ml_dtypes
import numpy as np
import pytest
import scipy.special
import torch

import oracle as O
from tests.conftest import load_golden

A = np.asarray


# ----------------------------------------------------------------------------- bf16

def test_bf16_round_hand_values():
    x = A([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -30, -0.0, 2.0 ** -134, 3 * 2.0 ** -134,
           3.4e38, -3.4e38])
    want = A([1.0, 1 + 2 ** -6, 1 + 2 ** -7, -0.0, 0.0, 2.0 ** -132, np.inf, -np.inf])
    got = O.round_to_bf16(x)
    assert np.array_equal(got, want)
    assert np.signbit(got[3])


def test_bf16_round_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(1)
    x32 = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                          (rng.standard_normal(2000) * 1e-39).astype(np.float32),
                          rng.uniform(-1e38, 1e38, 2000).astype(np.float32)])
    want = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_to_bf16(x32.astype(np.float64)), want)


# ----------------------------------------------------------------------------- compression

@pytest.mark.parametrize("case", ["two_channels", "halo", "dominant"])
def test_compress_golden(case):
    d, num = load_golden("compress_hand.json")
    cs = d["cases"][case]
    e, _ = O.compress(A(num(cs["c"])), A(num(cs["z"])), A(num(cs["bias"])), cs["m"], cs["halo"])
    np.testing.assert_allclose(e, A(cs["expect"]), rtol=0, atol=1e-6)


def _rand_compress_inputs(rng, B, T, D, m, halo):
    t_in = T + (m if halo else 0)
    c = O.round_to_bf16(rng.standard_normal((B, t_in, D)))
    z = rng.standard_normal((B, t_in, D)).astype(np.float32).astype(np.float64)
    b = (0.3 * rng.standard_normal((2 * m, D))).astype(np.float32).astype(np.float64)
    return c, z, b


@pytest.mark.parametrize("m", [1, 2, 4])
def test_compress_closed_forms(m):
    rng = np.random.default_rng(m)
    B, T, D = 2, 8 * m + (m - 1), 5      # ragged tail: the last partial block forms no entry
    c, z, b = _rand_compress_inputs(rng, B, T, D, m, False)
    N = T // m
    # constant c over the sequence -> every entry equals it
    cc = np.broadcast_to(c[:, :1, :], c.shape).copy()
    e, e16 = O.compress(cc, z, b, m)
    assert e.shape == (B, N, D)
    np.testing.assert_allclose(e, np.broadcast_to(cc[:, :1, :], e.shape), rtol=1e-14, atol=0)
    assert np.array_equal(e16, np.broadcast_to(cc[:, :1, :], e.shape))
    # z = bias = 0 -> plain window mean (entry 0: block 0 only)
    e, _ = O.compress(c, np.zeros_like(z), np.zeros_like(b), m)
    for j in range(N):
        lo = max(0, (j - 1) * m)
        np.testing.assert_allclose(e[:, j], c[:, lo:(j + 1) * m].mean(axis=1), rtol=1e-13, atol=1e-15)
    # a per-channel constant added to every logit changes nothing (softmax shift)
    e1, _ = O.compress(c, z, b, m)
    e2, _ = O.compress(c, z + rng.standard_normal((B, 1, D)) * 7, b, m)
    np.testing.assert_allclose(e1, e2, rtol=1e-12, atol=1e-13)


def test_compress_m1_is_logistic_mix():
    # m = 1: entry j mixes tokens j-1 and j with weight sigmoid of the logit difference
    rng = np.random.default_rng(7)
    c, z, b = _rand_compress_inputs(rng, 1, 9, 3, 1, False)
    e, _ = O.compress(c, z, b, 1)
    np.testing.assert_allclose(e[:, 0], c[:, 0], rtol=1e-15)
    for j in range(1, 9):
        a = scipy.special.expit((z[:, j] + b[1]) - (z[:, j - 1] + b[0]))
        np.testing.assert_allclose(e[:, j], a * c[:, j] + (1 - a) * c[:, j - 1], rtol=1e-12, atol=1e-14)


def test_compress_halo_equals_prefix_of_longer_sequence():
    # compressing a chunk with its halo equals the matching entries of the whole sequence
    rng = np.random.default_rng(9)
    m = 4
    c, z, b = _rand_compress_inputs(rng, 2, 12 * m, 6, m, False)
    full, _ = O.compress(c, z, b, m)
    s = 5 * m
    part, _ = O.compress(c[:, s - m:], z[:, s - m:], b, m, has_left_halo=True)
    np.testing.assert_allclose(part, full[:, 5:], rtol=1e-14, atol=1e-15)


def test_compress_dominant_logit_selects_token():
    rng = np.random.default_rng(3)
    m, D = 4, 4
    c, z, b = _rand_compress_inputs(rng, 1, 6 * m, D, m, False)
    z = z.copy()
    z[0, 9, :] = 500.0          # token 9 is in blocks 2 -> entries 2 and 3
    e, _ = O.compress(c, z, b, m)
    np.testing.assert_allclose(e[0, 2], c[0, 9], rtol=1e-12)
    np.testing.assert_allclose(e[0, 3], c[0, 9], rtol=1e-12)


# ----------------------------------------------------------------------------- index score

def test_index_scores_golden():
    d, num = load_golden("index_hand.json")
    q, w, k = A(d["q"], float), A(d["w"], float), A(d["k"], float)
    np.testing.assert_array_equal(O.index_scores(q, w, k), A(d["expect_relu"]))
    np.testing.assert_array_equal(O.index_scores(q, w, k, act="identity"), A(d["expect_identity"]))
    np.testing.assert_array_equal(O.index_scores(q, w, k, n_visible=A(d["n_visible"])),
                                  A(num(d["expect_relu_nv2"])))
    np.testing.assert_array_equal(O.index_scores(q, w, k, pool=A(d["pool"])),
                                  A(num(d["expect_relu_pool"])))


def test_index_identity_act_is_dot_with_weighted_query():
    # without the ReLU the score is linear: s_j = k_j . (sum_h w_h q_h)
    rng = np.random.default_rng(11)
    B, Q, H, d, N = 2, 3, 5, 7, 11
    q, w, k = rng.standard_normal((B, Q, H, d)), rng.random((B, Q, H)), rng.standard_normal((B, N, d))
    s = O.index_scores(q, w, k, act="identity")
    for b in range(B):
        for t in range(Q):
            qbar = sum(w[b, t, h] * q[b, t, h] for h in range(H))
            np.testing.assert_allclose(s[b, t], k[b] @ qbar, rtol=1e-12, atol=1e-12)


def test_index_pool_scores_are_gathered_full_scores():
    rng = np.random.default_rng(12)
    B, Q, H, d, N, P = 2, 2, 4, 8, 40, 9
    q, w, k = rng.standard_normal((B, Q, H, d)), rng.random((B, Q, H)), rng.standard_normal((B, N, d))
    full = O.index_scores(q, w, k)
    pool = np.sort(rng.choice(N, size=(B, Q, P)), axis=-1)
    pool[:, :, -2:] = -1
    ps = O.index_scores(q, w, k, pool=pool)
    for b in range(B):
        for t in range(Q):
            ok = pool[b, t] >= 0
            np.testing.assert_array_equal(ps[b, t, ok], full[b, t, pool[b, t, ok]])
            assert np.all(ps[b, t, ~ok] == -np.inf)


def test_index_relu_kills_negative_heads():
    # single head, w = 1: score = max(q . k, 0); unit query picks one coordinate of k
    k = A([[[0.5, -2.0, 3.0], [-1.0, 1.0, 0.25]]])
    for i in range(3):
        q = np.zeros((1, 1, 1, 3))
        q[0, 0, 0, i] = 1.0
        s = O.index_scores(q, np.ones((1, 1, 1)), k)
        np.testing.assert_array_equal(s[0, 0], np.maximum(k[0, :, i], 0))


# ----------------------------------------------------------------------------- top-k

def test_topk_golden():
    d, num = load_golden("topk_hand.json")
    s = A(num(d["scores"]))
    for kk, want in d["expect"].items():
        assert O.select_top(s[None], int(kk))[0].tolist() == want


def _brute_topk(s, k):
    """Brute force: the chosen set is the one whose members all beat every
    non-member under (score desc, index asc).  Enumerate every subset."""
    n = len(s)
    sel = [i for i in range(n) if s[i] > -np.inf]
    k = min(k, len(sel))
    beats = lambda a, b: (s[a] > s[b]) or (s[a] == s[b] and a < b)
    good = [set(S) for S in itertools.combinations(sel, k)
            if all(beats(a, b) for a in S for b in sel if b not in S)]
    assert len(good) == 1
    return sorted(good[0])


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(5)
    for trial in range(60):
        n = int(rng.integers(1, 9))
        s = rng.integers(0, 3, size=n).astype(float)     # many ties
        s[rng.random(n) < 0.2] = -np.inf
        for k in range(1, n + 2):
            got = O.select_top(s[None], k)[0]
            want = _brute_topk(s, k)
            assert got[:len(want)].tolist() == want
            assert np.all(got[len(want):] == -1)


def test_pool_contains_topk():
    rng = np.random.default_rng(6)
    s = rng.standard_normal((3, 500)).round(1)            # ties
    pool = O.select_top(s, 64)
    top = O.select_top(s, 16)
    for r in range(3):
        assert set(top[r]) <= set(pool[r])


def test_topk_of_pool_is_topk_of_row():
    """The reading a Full layer's two-step selection rests on: selecting the
    k best inside the P best (k <= P), through the pool's positions, gives
    exactly the row's k best (same order and ties, -inf never chosen, pools
    padded with -1 when fewer than P entries are selectable)."""
    rng = np.random.default_rng(7)
    for trial in range(200):
        L = int(rng.integers(1, 400))
        s = rng.integers(-4, 4, size=(2, L)).astype(float)     # heavy ties
        s[rng.random((2, L)) < 0.3] = -np.inf
        if trial % 3 == 0:
            s = rng.standard_normal((2, L)).round(1)
        P = int(rng.integers(1, L + 50))
        k = int(rng.integers(1, P + 1))
        pool = O.select_top(s, P)
        g = np.where(pool >= 0, np.take_along_axis(s, np.maximum(pool, 0), 1), -np.inf)
        pos = O.select_top(g, k)
        two_step = np.where(pos >= 0, np.take_along_axis(pool, np.maximum(pos, 0), 1), -1)
        assert np.array_equal(two_step, O.select_top(s, k)), (trial, L, P, k)


# ----------------------------------------------------------------------------- attention

def test_attn_golden():
    d, num = load_golden("attn_hand.json")
    o, _, lse = O.sparse_attn(A(num(d["q"])), A(d["kv"], float), A(d["topk"]), 1.0)
    np.testing.assert_allclose(o, A(d["expect_o"]), atol=1e-7)
    np.testing.assert_allclose(lse, A(d["expect_lse"]), atol=1e-7)


def test_attn_all_entries_equals_dense_sdpa():
    # k = N: top-k attention is dense softmax attention over every entry
    rng = np.random.default_rng(8)
    B, Q, Ha, D, N = 2, 3, 4, 16, 37
    q, kv = rng.standard_normal((B, Q, Ha, D)), rng.standard_normal((B, N, D))
    topk = np.broadcast_to(np.arange(N), (B, Q, N))
    o, _, lse = O.sparse_attn(q, kv, topk, 0.3)
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)                   # [B, Ha, Q, D]
    kt = torch.from_numpy(kv)[:, None].expand(B, Ha, N, D)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, scale=0.3)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-12, atol=1e-12)
    logits = 0.3 * np.einsum("bqhd,bnd->bqhn", q, kv)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(logits, axis=-1), rtol=1e-12)


def test_attn_special_cases():
    rng = np.random.default_rng(10)
    B, Q, Ha, D, N = 1, 2, 3, 8, 20
    q, kv = rng.standard_normal((B, Q, Ha, D)), rng.standard_normal((B, N, D))
    # one selected row -> output is that row, lse is its logit
    o, _, lse = O.sparse_attn(q, kv, A([[[7, -1], [3, -1]]]), 0.5)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(kv[0, 7], (Ha, D)), rtol=1e-14)
    np.testing.assert_allclose(lse[0, 1], 0.5 * q[0, 1] @ kv[0, 3], rtol=1e-13)
    # zero query -> uniform weights -> mean of the selected rows
    ids = A([[[1, 4, 9, 2], [0, 5, 6, 19]]])
    o, _, lse = O.sparse_attn(np.zeros_like(q), kv, ids, 0.5)
    np.testing.assert_allclose(o[0, 1, 2], kv[0, [0, 5, 6, 19]].mean(axis=0), rtol=1e-13)
    np.testing.assert_allclose(lse[0, 0], np.log(4.0) * np.ones(Ha), rtol=1e-14)
    # order of the selected ids does not matter; empty selection -> 0 / -inf
    o1, _, _ = O.sparse_attn(q, kv, ids, 0.5)
    o2, _, _ = O.sparse_attn(q, kv, ids[..., ::-1], 0.5)
    np.testing.assert_allclose(o1, o2, rtol=1e-13)
    o, _, lse = O.sparse_attn(q, kv, -np.ones((1, 2, 3), dtype=int), 0.5)
    assert np.all(o == 0) and np.all(lse == -np.inf)


# ----------------------------------------------------------------------------- FP4

def test_e2m1_table_is_the_format():
    # OCP MX E2M1: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 is the sign
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert O.e2m1_value(np.arange(8)).tolist() == mags
    assert O.e2m1_value(np.arange(8, 16)).tolist() == [-v for v in mags]
    via_lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(O.e2m1_value(np.arange(16)), via_lib)


def test_e4m3_table_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = O.e4m3_value(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2
    assert np.array_equal(mine[~nan], ref[~nan])
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9


def test_fp4_golden():
    d, num = load_golden("fp4_hand.json")
    x = A(num(d["x"]))
    codes, scales = O.fp4_pack(x)
    assert codes.tolist() == d["expect_codes"]
    assert scales.tolist() == d["expect_scales"]
    u = O.fp4_unpack(codes, scales)
    want = A(num(d["expect_unpack"]))
    assert np.array_equal(u, want) and np.array_equal(np.signbit(u), np.signbit(want))


def test_fp4_scale_is_nearest_e4m3_of_absmax_over_6():
    rng = np.random.default_rng(13)
    x = O.round_to_bf16(rng.standard_normal((4000, 16)) * np.exp(rng.uniform(-8, 8, (4000, 1))))
    _, scales = O.fp4_pack(x)
    amax = np.abs(x).max(axis=1)
    ref = torch.from_numpy((amax / 6.0).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    big = amax / 6.0 >= 464.0            # torch gives NaN past the top; the format saturates
    ref = np.where(big, 0x7E, ref)
    assert np.array_equal(scales[:, 0], ref)


def test_fp4_codes_match_library_e2m1_rounding():
    # with a power-of-two scale x/s is exact, so library E2M1 rounding of x/s is the reference
    rng = np.random.default_rng(14)
    x = O.round_to_bf16(rng.standard_normal((5000, 16)) * 1.7)
    x[:, 0] = 6.0 * 2.0 ** rng.integers(-3, 4, size=5000)       # absmax/6 is a power of two
    x[:, 1:] = np.clip(x[:, 1:], -np.abs(x[:, :1]), np.abs(x[:, :1]))
    codes, scales = O.fp4_pack(x)
    s = O.e4m3_value(scales[:, 0].astype(int))
    np.testing.assert_array_equal(s, np.abs(x[:, 0]) / 6.0)
    r = (x / s[:, None]).astype(np.float32).astype(ml_dtypes.float4_e2m1fn)
    lib_codes = r.view(np.uint8).astype(np.int64) & 0xF
    mine = np.empty((5000, 16), dtype=np.int64)
    mine[:, 0::2] = codes & 0xF
    mine[:, 1::2] = codes >> 4
    assert np.array_equal(mine, lib_codes)


def test_fp4_round_trips():
    rng = np.random.default_rng(15)
    # unpack(pack(x)) == x for x on the grid of a block whose largest code is 6
    sc = 2.0 ** rng.integers(-6, 6, size=(300, 1)) * rng.choice([1, 1.25, 1.5, 1.75], size=(300, 1))
    v = O.e2m1_value(rng.integers(0, 16, size=(300, 16)))
    v[:, 3] = 6.0
    x = v * sc
    c, s = O.fp4_pack(x)
    assert np.array_equal(O.fp4_unpack(c, s), x)
    # pack(unpack(bytes)) == bytes for every valid block holding a +-6 code
    codes = rng.integers(0, 256, size=(2000, 8)).astype(np.uint8)
    codes[:, 0] = (codes[:, 0] & 0xF0) | 0x7
    scales = rng.integers(1, 0x7F, size=(2000, 1)).astype(np.uint8)
    c2, s2 = O.fp4_pack(O.fp4_unpack(codes, scales))
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)


def test_fp4_saturation_for_huge_values():
    # far past the top of both formats: scale 448 (0x7E), every code at +-6
    x = np.zeros((3, 16))
    x[0, :] = 1e30
    x[1, :] = -3e38
    x[2, 0], x[2, 1], x[2, 2] = 2700.0, -2688.0 * 1e6, 1.0
    c, s = O.fp4_pack(x)
    assert s.tolist() == [[0x7E], [0x7E], [0x7E]]
    assert c[0].tolist() == [0x77] * 8 and c[1].tolist() == [0xFF] * 8
    assert c[2, 0] == 0xF7            # 2700/448 > 6 -> 7; -2.688e9 -> -6 (0xF)
    assert (c[2, 1] & 0xF) == 0       # 1/448 rounds to 0


def test_fp4_zero_block():
    x = np.zeros((2, 32))
    x[1, 16:] = -0.0
    x[1, 5] = -0.0
    c, s = O.fp4_pack(x)
    assert np.all(s == 0)
    assert c[0].tolist() == [0] * 16
    assert c[1, 2] == 0x80 and c[1, 8:].tolist() == [0x88] * 8


# ----------------------------------------------------------------------------- layer modes

def _group_inputs(rng, B=2, N=96, D=16, Ha=3, Hi=4, d=8, n_layers=4):
    kv = O.round_to_bf16(rng.standard_normal((B, N, D)))
    ik = O.round_to_bf16(rng.standard_normal((B, N, d)))
    layers = [dict(q_attn=rng.standard_normal((B, 1, Ha, D)),
                   q_index=rng.standard_normal((B, 1, Hi, d)),
                   w_index=rng.random((B, 1, Hi))) for _ in range(n_layers)]
    return kv, ik, layers


def test_modes_reuse_and_reindex_invariants():
    rng = np.random.default_rng(16)
    kv, ik, layers = _group_inputs(rng)
    res = O.run_group(["full", "reuse", "reindex", "reuse"], layers, kv, ik, k_top=8, scale=0.25)
    # reuse keeps the most recent selection and attends with its own queries
    assert np.array_equal(res[1]["topk"], res[0]["topk"])
    assert np.array_equal(res[3]["topk"], res[2]["topk"])
    o, _, _ = O.sparse_attn(layers[1]["q_attn"], kv, res[0]["topk"], 0.25)
    np.testing.assert_array_equal(res[1]["o"], o)
    # reindex with the Full layer's own queries reproduces Full's selection
    same = [layers[0], layers[0]]
    r2 = O.run_group(["full", "reindex"], same, kv, ik, k_top=8, scale=0.25)
    assert np.array_equal(r2[1]["topk"], r2[0]["topk"])


def test_hierarchical_pool_invariants():
    rng = np.random.default_rng(17)
    kv, ik, layers = _group_inputs(rng, N=300)
    same = [layers[0]] * 3
    # pool = every entry: Reindex equals the flat Reindex
    r_all = O.run_group(["full", "reindex"], same[:2], kv, ik, k_top=10, scale=0.25, pool_size=300)
    r_flat = O.run_group(["full", "reindex"], same[:2], kv, ik, k_top=10, scale=0.25)
    assert np.array_equal(r_all[1]["topk"], r_flat[1]["topk"])
    # a real pool: with the Full layer's own queries, Reindex inside the pool gives Full's top-k
    r = O.run_group(["full", "reindex"], same[:2], kv, ik, k_top=10, scale=0.25, pool_size=40)
    assert np.array_equal(r[1]["topk"], r[0]["topk"])
    assert all(set(r[0]["topk"][b, 0]) <= set(r[0]["pool"][b, 0]) for b in range(2))
    # fresh queries: Reindex picks only pool members
    r = O.run_group(["full", "reindex", "reindex"], layers[:3], kv, ik, k_top=10, scale=0.25, pool_size=40)
    for b in range(2):
        assert set(r[2]["topk"][b, 0]) <= set(r[0]["pool"][b, 0])


def test_modes_before_full_rejected():
    rng = np.random.default_rng(18)
    kv, ik, layers = _group_inputs(rng)
    for mode in ("reindex", "reuse"):
        with pytest.raises(ValueError):
            O.run_group([mode], layers[:1], kv, ik, k_top=4, scale=1.0)
