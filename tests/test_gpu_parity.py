"""GPU parity: every CUDA kernel, called through the C ABI, against the
float64 oracle on the same seeded inputs.  Small cases span several tiles and
a ragged tail; the five workloads run at full size with sampled checks."""
import numpy as np
import pytest
import torch

import kv_cache_csa2_b200 as K
import oracle as O
from kv_cache_csa2_b200 import configs as C
from kv_cache_csa2_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _device_clean():
    yield
    K.csa2_device_error()          # no kernel recorded a device-side error


def _rng(seed):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ FP4 (bit-exact)

def _fp4_cases():
    r = _rng(1)
    x = r.standard_normal((1000, 128)).astype(np.float32) * np.exp(r.uniform(-6, 6, (1000, 1))).astype(np.float32)
    x[0] = 0.0
    x[1, :16] = -0.0
    x[2, :16] = np.float32(6.375)         # scale tie
    x[3, :] = np.float32(1e30)            # saturating scale
    x[4, :16] = np.float32(1e-6)          # scale underflows to 0
    x[5, :16] = [6, 3, 1.5, 0.75, -0.25, 5, 2.5, -6, 0, -0.0, 1, 0.5, 4, -3, 2, 1.25]
    return I.f32_to_bf16_bits(x)


@pytest.mark.parametrize("rows", [1, 7, 1000])
def test_fp4_pack_unpack_bit_exact(rows):
    bits = _fp4_cases()[:rows]
    codes, scales = K.csa2_fp4_pack(U.dev_bf16(bits))
    oc, os_ = O.fp4_pack(O.bf16_bits_to_float(bits))
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(scales.cpu().numpy(), os_)
    back = K.csa2_fp4_unpack(codes, scales)
    ou = O.fp4_unpack(oc, os_)
    got = U.host_bf16(back)
    assert np.array_equal(got, ou) and np.array_equal(np.signbit(got), np.signbit(ou))


def test_fp4_unpack_every_code_and_scale():
    codes = np.tile(np.arange(256, dtype=np.uint8), 2 * 127).reshape(-1, 8)        # [8128, 8]
    scales = np.repeat(np.arange(127, dtype=np.uint8), 64).reshape(-1, 1)           # [8128, 1]
    got = U.host_bf16(K.csa2_fp4_unpack(U.dev(codes), U.dev(scales)))
    want = O.fp4_unpack(codes, scales)
    assert np.array_equal(got, want)


@pytest.mark.slow
def test_fp4_pack_c3_full_size_sampled():
    wl = C.C3
    inp = I.make_inputs(wl, layers=False)
    kv = U.dev_bf16(inp["kv"])
    codes, scales = K.csa2_fp4_pack(kv)
    r = _rng(2)
    b = r.integers(0, wl.B, 4096)
    j = r.integers(0, wl.N, 4096)
    oc, os_ = O.fp4_pack(O.bf16_bits_to_float(inp["kv"][b, j]))
    assert np.array_equal(codes[torch.from_numpy(b), torch.from_numpy(j)].cpu().numpy(), oc)
    assert np.array_equal(scales[torch.from_numpy(b), torch.from_numpy(j)].cpu().numpy(), os_)


# ------------------------------------------------------------------ compression

def _check_compress(c_bits, z, bias, m, halo, out_gpu):
    exact, _ = O.compress(O.bf16_bits_to_float(c_bits), z.astype(np.float64),
                          bias.astype(np.float64), m, halo)
    got = U.host_bf16(out_gpu)
    # f32 arithmetic then one rounding: within one bf16 step of the exact value,
    # plus an absolute floor for cancellation (1e-6 of the largest |c| in use)
    tol = U.bf16_ulp(exact) + 1e-6 * np.abs(O.bf16_bits_to_float(c_bits)).max()
    assert np.all(np.abs(got - exact) <= tol), np.abs(got - exact).max()
    return exact, got


@pytest.mark.parametrize("m,halo,T,D", [(1, False, 37, 16), (2, False, 130, 64), (4, False, 1027, 128),
                                         (4, True, 1024, 512), (8, True, 96, 24)])
def test_compress_parity(m, halo, T, D):
    r = _rng(3)
    t_in = T + (m if halo else 0)
    c = I.f32_to_bf16_bits(r.standard_normal((3, t_in, D)).astype(np.float32))
    z = r.standard_normal((3, t_in, D)).astype(np.float32) * 2
    bias = r.standard_normal((2 * m, D)).astype(np.float32) * 0.3
    out = K.csa2_compress(U.dev_bf16(c), U.dev(z), U.dev(bias), m, has_left_halo=halo)
    assert out.shape == (3, T // m, D)
    _check_compress(c, z, bias, m, halo, out)


def test_compress_appends_into_kv_buffer():
    r = _rng(4)
    m, T, D, B = 4, 64, 32, 2
    c = I.f32_to_bf16_bits(r.standard_normal((B, T + m, D)).astype(np.float32))
    z = r.standard_normal((B, T + m, D)).astype(np.float32)
    bias = r.standard_normal((2 * m, D)).astype(np.float32)
    buf = torch.full((B, 100, D), 7.0, dtype=torch.bfloat16, device="cuda")
    K.csa2_compress(U.dev_bf16(c), U.dev(z), U.dev(bias), m, True, out=buf[:, 50:], out_batch_stride=100 * D)
    _check_compress(c, z, bias, m, True, buf[:, 50:66])
    assert torch.all(buf[:, :50] == 7) and torch.all(buf[:, 66:] == 7)


@pytest.mark.slow
@pytest.mark.parametrize("wl", [C.C1, C.C5], ids=["c1", "c5"])
def test_compress_workloads(wl):
    inp = I.make_inputs(wl, layers=False)
    out = K.csa2_compress(U.dev_bf16(inp["c"]), U.dev(inp["z"]), U.dev(inp["bias"]), wl.m,
                          has_left_halo=wl.halo)
    _check_compress(inp["c"], inp["z"], inp["bias"], wl.m, wl.halo, out)


# ------------------------------------------------------------------ indexer scores

def _index_inputs(r, B, Q, H, d, N, wdist="uniform"):
    q = I.f32_to_bf16_bits((r.standard_normal((B, Q, H, d)) / np.sqrt(d)).astype(np.float32))
    k = I.f32_to_bf16_bits((r.standard_normal((B, N, d)) / np.sqrt(d)).astype(np.float32))
    w = (r.random((B, Q, H)) if wdist == "uniform" else r.standard_normal((B, Q, H))).astype(np.float32)
    return q, w, k


def _score_tol(q, w, k, pool=None):
    """Bound for f32 accumulation: 1e-5 * sum_h |w_h| sum_i |q_hi k_ji|."""
    qa, ka = np.abs(O.bf16_bits_to_float(q)), np.abs(O.bf16_bits_to_float(k))
    return 1e-5 * O.index_scores(qa, np.abs(w), ka, pool=pool, act="identity") + 1e-12


@pytest.mark.parametrize("B,Q,H,d,N", [(2, 3, 8, 64, 1000), (1, 2, 64, 128, 777), (2, 1, 16, 32, 300),
                                       (1, 1, 128, 64, 129), (3, 2, 4, 256, 65),
                                       (1, 37, 8, 64, 500), (2, 9, 64, 128, 300), (1, 6, 48, 64, 1300),
                                       (3, 1, 64, 128, 128), (1, 1, 1, 128, 4000)])
@pytest.mark.parametrize("act", [K.ACT_RELU, K.ACT_IDENTITY])
def test_index_scores_parity(B, Q, H, d, N, act):
    r = _rng(5)
    q, w, k = _index_inputs(r, B, Q, H, d, N, "normal")
    nv = r.integers(0, N + 1, (B, Q)).astype(np.int32)
    nv[0, 0] = N
    got = K.csa2_index_scores(U.dev_bf16(q), U.dev(w), U.dev_bf16(k), n_visible=U.dev(nv), act=act).cpu().numpy()
    want = O.index_scores(O.bf16_bits_to_float(q), w.astype(np.float64), O.bf16_bits_to_float(k),
                          n_visible=nv, act="relu" if act == K.ACT_RELU else "identity")
    fin = np.isfinite(want)
    assert np.array_equal(np.isfinite(got), fin)
    tol = _score_tol(q, w, k)
    assert np.all(np.abs(got[fin] - want[fin]) <= tol[fin])


@pytest.mark.parametrize("B,Q,H,d,N,P", [(2, 2, 64, 128, 5000, 700), (3, 1, 8, 64, 2000, 300),
                                         (1, 3, 16, 128, 999, 129)])
def test_index_scores_pool_parity(B, Q, H, d, N, P):
    r = _rng(6)
    q, w, k = _index_inputs(r, B, Q, H, d, N)
    pool = np.sort(r.choice(N, size=(B, Q, P)), axis=-1).astype(np.int32)
    pool[:, :, -13:] = -1
    got = K.csa2_index_scores(U.dev_bf16(q), U.dev(w), U.dev_bf16(k), pool=U.dev(pool)).cpu().numpy()
    want = O.index_scores(O.bf16_bits_to_float(q), w.astype(np.float64), O.bf16_bits_to_float(k), pool=pool)
    fin = np.isfinite(want)
    assert np.array_equal(np.isfinite(got), fin)
    assert np.all(np.abs(got[fin] - want[fin]) <= _score_tol(q, w, k, pool=pool)[fin])


# ------------------------------------------------------------------ top-k (bit-exact on given scores)

def _score_rows(r, rows, L, kind):
    if kind == "ties":
        s = r.integers(-20, 20, (rows, L)).astype(np.float32)
    elif kind == "dense_ties":      # the threshold bin keeps most of the row in every pass
        s = np.where(r.random((rows, L)) < 0.8, np.float32(1.0), np.float32(2.0)).astype(np.float32)
    else:
        s = r.standard_normal((rows, L)).astype(np.float32)
    s[r.random((rows, L)) < 0.05] = -np.inf
    s[r.random((rows, L)) < 0.01] = np.nan
    return s


@pytest.mark.parametrize("rows,L,count", [(5, 1000, 37), (3, 4096, 2048), (2, 300, 1000), (1, 1, 1),
                                          (8, 16384, 2048), (2, 32768, 16384), (3, 20001, 5000),
                                          (4, 70000, 2048), (2, 262144, 16384), (64, 2000, 256),
                                          (200, 3000, 100), (5, 32765, 7000)])
@pytest.mark.parametrize("kind", ["normal", "ties", "dense_ties"])
def test_select_topk_exact(rows, L, count, kind):
    r = _rng(7)
    s = _score_rows(r, rows, L, kind)
    got = K.csa2_select_topk(U.dev(s), count).cpu().numpy()
    s64 = np.where(np.isnan(s), -np.inf, s).astype(np.float64)
    want = O.select_top(s64, count)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("rows,L,count", [(3, 4096, 2048), (8, 16384, 2048), (2, 32768, 16384),
                                          (3, 20001, 5000)])
@pytest.mark.parametrize("path", ["one_cta", "chunked"])
@pytest.mark.parametrize("kind", ["ties", "dense_ties"])
def test_select_topk_short_row_paths(rows, L, count, path, kind, monkeypatch):
    """Short rows of a small batch normally take the 8-CTA cluster kernel;
    the one-CTA kernel and the cooperative kernel's one-chunk path give the
    same result."""
    monkeypatch.setenv("CSA2_TOPK_NO_CLUSTER", "1")
    if path == "chunked":
        monkeypatch.setenv("CSA2_TOPK_NO_CTA", "1")
    r = _rng(17)
    s = _score_rows(r, rows, L, kind)
    got = K.csa2_select_topk(U.dev(s), count).cpu().numpy()
    want = O.select_top(np.where(np.isnan(s), -np.inf, s).astype(np.float64), count)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("case", ["all_equal", "nothing_selectable", "few_selectable", "one_key",
                                  "narrow_band", "odd_rows"])
def test_select_topk_cluster_edges(case):
    """Edge rows of the cluster kernel (8 rows, at most 32768 scores)."""
    r = _rng(19)
    rows, L, count = 8, 16384, 2048
    if case == "all_equal":
        s = np.full((rows, L), 0.5, dtype=np.float32)
    elif case == "nothing_selectable":
        s = np.where(r.random((rows, L)) < 0.5, np.float32(-np.inf), np.float32(np.nan)).astype(np.float32)
    elif case == "few_selectable":       # fewer selectable scores than count: -1 padding
        s = np.full((rows, L), -np.inf, dtype=np.float32)
        s[r.random((rows, L)) < 0.05] = 3.0
        s[:, 5] = 4.0
    elif case == "one_key":
        rows, L, count = 3, 1, 1
        s = r.standard_normal((rows, L)).astype(np.float32)
    elif case == "narrow_band":          # long common key prefix, many near-ties
        s = (1.0 + 1e-6 * r.integers(0, 50, (rows, L))).astype(np.float32)
    else:                                # row starts off 16 bytes: unvectorised loads
        rows, L, count = 5, 4099, 1000
        s = r.standard_normal((rows, L)).astype(np.float32)
    got = K.csa2_select_topk(U.dev(s), count).cpu().numpy()
    want = O.select_top(np.where(np.isnan(s), -np.inf, s).astype(np.float64), count)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("L", [3000, 100000])
def test_select_topk_signed_zero_ties(L):
    """-0 and +0 are the same score: ties between them go to the lower position."""
    r = _rng(18)
    s = np.where(r.random((2, L)) < 0.5, np.float32(0.0), np.float32(-0.0)).astype(np.float32)
    s[:, ::7] = 1.0
    got = K.csa2_select_topk(U.dev(s), L // 2).cpu().numpy()
    assert np.array_equal(got, O.select_top(s.astype(np.float64), L // 2))


@pytest.mark.parametrize("B,Q,H,d,N,k_top,P", [(2, 3, 16, 64, 5000, 300, 1000),
                                              (2, 2, 2, 32, 5000, 300, 4500),
                                              (3, 1, 8, 32, 70000, 100, 3000),
                                              (8, 1, 64, 128, 262144, 2048, 16384)])
@pytest.mark.parametrize("path", ["cluster", "multi"])
def test_index_topk_full_pool_and_topk(B, Q, H, d, N, k_top, P, path, monkeypatch):
    """A Full layer's two selections (the pool and the top-k) against the
    oracle's selection over the same scores (the scoring kernel is
    deterministic).  The cluster path selects the pool, then the top-k inside
    it; the cooperative kernel selects both in the same passes.  H = 2 leaves
    many scores at exactly 0 (ReLU), so ties reach into the pool."""
    if path == "multi":
        monkeypatch.setenv("CSA2_TOPK_NO_CLUSTER", "1")
    r = _rng(21)
    q, w, k = _index_inputs(r, B, Q, H, d, N)
    dq, dw, dk = U.dev_bf16(q), U.dev(w), U.dev_bf16(k)
    topk, pool = K.csa2_index_topk(K.FULL, dq, dw, dk, k_top, pool_size=P)
    s = K.csa2_index_scores(dq, dw, dk).cpu().numpy().astype(np.float64)
    assert np.array_equal(pool.cpu().numpy(), O.select_top(s, P))
    assert np.array_equal(topk.cpu().numpy(), O.select_top(s, k_top))


def test_select_topk_maps_ids():
    r = _rng(8)
    s = _score_rows(r, 4, 3000, "ties")
    ids = np.sort(r.choice(10 ** 6, size=(4, 3000), replace=False), axis=-1).astype(np.int32)
    got = K.csa2_select_topk(U.dev(s), 100, ids=U.dev(ids)).cpu().numpy()
    pos = O.select_top(np.where(np.isnan(s), -np.inf, s).astype(np.float64), 100)
    assert np.array_equal(got, np.where(pos >= 0, np.take_along_axis(ids, np.maximum(pos, 0), 1), -1))


# ------------------------------------------------------------------ attention

def _attn_case(r, B, Q, Ha, D, N, k, fp4):
    q = I.f32_to_bf16_bits(r.standard_normal((B, Q, Ha, D)).astype(np.float32))
    kv = I.f32_to_bf16_bits(r.standard_normal((B, N, D)).astype(np.float32))
    topk = np.full((B, Q, k), -1, dtype=np.int32)
    for b in range(B):
        for t in range(Q):
            n = int(r.integers(0, k + 1)) if (b + t) % 3 == 2 else k
            topk[b, t, :n] = np.sort(r.choice(N, size=n, replace=False))
    return q, kv, topk


@pytest.mark.parametrize("Ha,D,N,k,fp4", [(16, 128, 3000, 256, False), (16, 128, 3000, 256, True),
                                          (64, 512, 5000, 2048, False), (64, 512, 900, 100, False),
                                          (64, 512, 5000, 2048, True), (16, 512, 500, 33, False),
                                          (32, 128, 400, 17, True), (64, 512, 9000, 4096, False),
                                          (64, 512, 9000, 6000, False), (64, 512, 2000, 300, False),
                                          (64, 512, 3000, 129, False)])
def test_sparse_attn_parity(Ha, D, N, k, fp4):
    r = _rng(9)
    B, Q = 2, 3
    q, kv, topk = _attn_case(r, B, Q, Ha, D, N, k, fp4)
    kvd = U.dev_bf16(kv)
    scale = D ** -0.5
    if fp4:
        codes, scales = K.csa2_fp4_pack(kvd)
        out, lse = K.csa2_sparse_attn(U.dev_bf16(q), codes, U.dev(topk), scale, kv_scales=scales)
        kvv = O.fp4_unpack(*O.fp4_pack(O.bf16_bits_to_float(kv.reshape(-1, D)))).reshape(B, N, D)
    else:
        out, lse = K.csa2_sparse_attn(U.dev_bf16(q), kvd, U.dev(topk), scale)
        kvv = O.bf16_bits_to_float(kv)
    o, _, l = O.sparse_attn(O.bf16_bits_to_float(q), kvv, topk, scale)
    U.check_attn(U.host_bf16(out), lse.cpu().numpy().astype(np.float64), o, l, f"Ha{Ha} D{D} k{k}")


@pytest.mark.parametrize("max_ctas,k", [("8", 384), ("8", 1000), ("16", 1000), ("40", 1000)])
def test_sparse_attn_grid_waves(max_ctas, k, monkeypatch):
    """The tensor-core kernel runs a grid of whole queries (one CTA per
    128-row tile) and loops over the batch in waves; a smaller grid means more
    waves, with the same reduction order and so the same bits."""
    r = _rng(19)
    B, Q, Ha, D, N = 2, 3, 64, 512, 4000
    q, kv, topk = _attn_case(r, B, Q, Ha, D, N, k, False)
    args = (U.dev_bf16(q), U.dev_bf16(kv), U.dev(topk), D ** -0.5)
    full_out, full_lse = K.csa2_sparse_attn(*args)
    monkeypatch.setenv("CSA2_ATTN_MAX_CTAS", max_ctas)
    for _ in range(2):                       # twice in a row
        out, lse = K.csa2_sparse_attn(*args)
        assert torch.equal(out, full_out) and torch.equal(lse, full_lse)
    o, _, l = O.sparse_attn(O.bf16_bits_to_float(q), O.bf16_bits_to_float(kv), topk, D ** -0.5)
    U.check_attn(U.host_bf16(out), lse.cpu().numpy().astype(np.float64), o, l, f"ctas<={max_ctas}")


def test_sparse_attn_bounds_recorded_not_faulting():
    r = _rng(10)
    q, kv, topk = _attn_case(r, 1, 2, 16, 128, 50, 8, False)
    topk[0, 0, 3] = 50            # one past the end: the kernel checks, skips and records it
    out, lse = K.csa2_sparse_attn(U.dev_bf16(q), U.dev_bf16(kv), U.dev(topk), 0.1)
    with pytest.raises(K.CSA2Error) as e:
        K.csa2_device_error()
    assert e.value.status == 7
    ids = topk.copy()
    ids[0, 0, 3] = -1
    o, _, l = O.sparse_attn(O.bf16_bits_to_float(q), O.bf16_bits_to_float(kv), ids, 0.1)
    U.check_attn(U.host_bf16(out), lse.cpu().numpy().astype(np.float64), o, l)


# ------------------------------------------------------------------ the five workloads

def _small(wl, **kw):
    return wl.replace(name=wl.name + "_small", **kw)


SMALL = [
    _small(C.C1, L=2048, compress_new_tokens=2048),
    _small(C.C2, B=3, L=4 * 3000, k=300),
    _small(C.C3, B=3, L=4 * 4000, k=100),
    _small(C.C4, B=2, L=4 * 20000, P=3000, k=500),
    _small(C.C5, L=4 * 5000, Q=64, compress_new_tokens=64 * 4, q_pos0=4 * 5000 - 64 * 4, k=300),
]


@pytest.mark.parametrize("wl", SMALL, ids=[w.name for w in SMALL])
def test_group_small(wl):
    inp = I.make_inputs(wl, seed=11)
    gres, kv = U.gpu_group(wl, inp)
    ores, _ = U.oracle_group(wl, inp)
    U.compare_groups(wl, inp, gres, ores, kv=kv)


@pytest.mark.slow
@pytest.mark.parametrize("wl", [C.C1, C.C2, C.C3, C.C4, C.C6], ids=["c1", "c2", "c3", "c4", "c6"])
def test_group_full_size(wl):
    inp = I.make_inputs(wl)
    gres, kv = U.gpu_group(wl, inp)
    ores, _ = U.oracle_group(wl, inp)
    U.compare_groups(wl, inp, gres, ores, kv=kv)


@pytest.mark.slow
def test_group_c5_prefill_sampled():
    wl = C.C5
    inp = I.make_inputs(wl)
    gres, kv = U.gpu_group(wl, inp)
    r = _rng(12)
    sample = np.unique(np.concatenate([[0, wl.Q - 1], r.choice(wl.Q, 30, replace=False)]))
    ores, _ = U.oracle_group(wl, inp, sample=sample)
    U.compare_groups(wl, inp, gres, ores, sample=sample, kv=kv)


# ------------------------------------------------------------------ modes, launches, invariance

def test_reuse_runs_no_indexer_and_mode_order():
    wl = SMALL[1]
    inp = I.make_inputs(wl, seed=13)
    K.reset_launch_counts()
    U.gpu_group(wl, inp)
    n = K.launch_counts()
    # one Full layer: one scoring launch and one selection; five Reuse layers add attention only
    assert n["index_scores"] == 1 and n["topk"] >= 1
    assert n["attn"] >= 6
    g = K.Group(wl.B, 1, wl.N, wl.D, wl.Ha, wl.Hi, wl.d, wl.k, [K.REUSE, K.FULL])
    out = torch.empty(wl.B, 1, wl.Ha, wl.D, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(K.CSA2Error) as e:
        g.layer(0, U.dev_bf16(inp["layers"][1]["q_attn"]), out)
    assert e.value.status == 2
    g.close()


@pytest.mark.parametrize("which", [3, 2], ids=["tensor_core_attn", "split_cuda_core_attn_fp4"])
def test_batch_invariance_bitwise(which):
    """A query's selection and output do not depend on the batch it runs in
    (the tensor-core attention of 64 x 512 heads, and the split CUDA-core
    attention of 16 x 128 heads over FP4 entries)."""
    wl = SMALL[which]
    inp = I.make_inputs(wl, seed=14)
    full, _ = U.gpu_group(wl, inp)
    for b in range(wl.B):
        one = {k: (v[b:b + 1] if isinstance(v, np.ndarray) and v.ndim >= 2 else v) for k, v in inp.items()}
        one["layers"] = [{k: v[b:b + 1] for k, v in L.items()} for L in inp["layers"]]
        alone, _ = U.gpu_group(wl.replace(B=1), one)
        for i in range(wl.n_layers):
            assert np.array_equal(alone[i]["topk"][0], full[i]["topk"][b])
            assert np.array_equal(alone[i]["out"][0], full[i]["out"][b])
            assert np.array_equal(alone[i]["lse"][0], full[i]["lse"][b])
