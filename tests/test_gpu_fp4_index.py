"""GPU parity of the FP4 indexer (FP4 q and K, bf16 scores) through the C ABI
against the float64 oracle.  The FP4 codes and scales fed to the GPU are the
oracle's own (csa2_fp4_pack gives the same bytes; that is tested elsewhere),
so both sides score the same dequantised values."""
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


def _fp4(x):
    """Oracle FP4 codes/scales of x [..., d] (rows along the last dim)."""
    lead, d = x.shape[:-1], x.shape[-1]
    c, s = O.fp4_pack(x.reshape(-1, d))
    return c.reshape(*lead, d // 2), s.reshape(*lead, d // 16)


def _case(r, B, Q, H, d, N, wdist="uniform"):
    q = O.bf16_bits_to_float(I.f32_to_bf16_bits((r.standard_normal((B, Q, H, d)) / np.sqrt(d)).astype(np.float32)))
    k = O.bf16_bits_to_float(I.f32_to_bf16_bits((r.standard_normal((B, N, d)) / np.sqrt(d)).astype(np.float32)))
    w = (r.random((B, Q, H)) if wdist == "uniform" else r.standard_normal((B, Q, H))).astype(np.float32)
    return q, k, w


def _dequant(x):
    c, s = _fp4(x)
    return O.fp4_unpack(c.reshape(-1, c.shape[-1]), s.reshape(-1, s.shape[-1])).reshape(x.shape)


def _score_bound(q, w, k, pool=None):
    """f32 accumulation bound over the dequantised values (as the bf16 kernel's)."""
    qa, ka = np.abs(_dequant(q)), np.abs(_dequant(k))
    return 1e-5 * O.index_scores(qa, np.abs(w).astype(np.float64), ka, pool=pool, act="identity") + 1e-12


def _check_scores(got, q, w, k, act, nv=None, pool=None):
    exact = O.index_scores(_dequant(q), w.astype(np.float64), _dequant(k), n_visible=nv, pool=pool, act=act)
    want = O.index_scores_fp4(q, w.astype(np.float64), k, n_visible=nv, pool=pool, act=act)
    fin = np.isfinite(want)
    assert np.array_equal(np.isfinite(got), fin)
    # one rounding to bf16 of a value within the f32 accumulation bound of the exact score
    bound = U.bf16_ulp(exact[fin]) / 2 + _score_bound(q, w, k, pool)[fin] * 1.01
    assert np.all(np.abs(got[fin] - exact[fin]) <= bound)
    assert np.array_equal(got[fin], O.round_to_bf16(got[fin]))     # bf16 values
    assert np.mean(got[fin] == want[fin]) > 0.99


@pytest.mark.parametrize("B,Q,H,d,N", [(2, 3, 8, 64, 1000), (1, 2, 64, 128, 777), (2, 1, 16, 128, 300),
                                       (1, 1, 64, 128, 129), (3, 2, 4, 64, 65), (1, 5, 64, 128, 5000)])
@pytest.mark.parametrize("act", [K.ACT_RELU, K.ACT_IDENTITY])
def test_index_scores_fp4_parity(B, Q, H, d, N, act):
    r = np.random.default_rng(60)
    q, k, w = _case(r, B, Q, H, d, N, "normal")
    nv = r.integers(0, N + 1, (B, Q)).astype(np.int32)
    nv[0, 0] = N
    qc, qs = _fp4(q)
    kc, ks = _fp4(k)
    got = K.csa2_index_scores_fp4(U.dev(qc), U.dev(qs), U.dev(w), U.dev(kc), U.dev(ks), n_visible=U.dev(nv),
                                  act=act)
    got = got.float().cpu().numpy().astype(np.float64)
    _check_scores(got, q, w, k, "relu" if act == K.ACT_RELU else "identity", nv=nv)


@pytest.mark.parametrize("B,Q,H,d,N,P", [(2, 2, 64, 128, 5000, 700), (3, 1, 8, 64, 2000, 300)])
def test_index_scores_fp4_pool_parity(B, Q, H, d, N, P):
    r = np.random.default_rng(61)
    q, k, w = _case(r, B, Q, H, d, N)
    pool = np.sort(r.choice(N, size=(B, Q, P)), axis=-1).astype(np.int32)
    pool[:, :, -13:] = -1
    qc, qs = _fp4(q)
    kc, ks = _fp4(k)
    got = K.csa2_index_scores_fp4(U.dev(qc), U.dev(qs), U.dev(w), U.dev(kc), U.dev(ks), pool=U.dev(pool))
    _check_scores(got.float().cpu().numpy().astype(np.float64), q, w, k, "relu", pool=pool)


def _bf16_step(s_k):
    return U.bf16_ulp(s_k)


@pytest.mark.parametrize("B,Q,H,d,N,k_top,P", [(2, 2, 16, 64, 5000, 300, 1000),
                                              (8, 1, 64, 128, 65536, 2048, 8192)])
def test_index_topk_fp4_full_then_reindex(B, Q, H, d, N, k_top, P):
    """A Full layer (pool and top-k) then a Reindex layer inside the pool, on
    bf16 scores: the selections against the oracle's, with one bf16 step of
    the k-th score as the tie band (bf16 scores tie often)."""
    r = np.random.default_rng(62)
    q, k, w = _case(r, B, Q, H, d, N)
    qc, qs = _fp4(q)
    kc, ks = _fp4(k)
    dk = (U.dev(kc), U.dev(ks))
    topk, pool = K.csa2_index_topk_fp4(K.FULL, U.dev(qc), U.dev(qs), U.dev(w), *dk, k_top, pool_size=P)
    topk, pool = topk.cpu().numpy(), pool.cpu().numpy()
    s = O.index_scores_fp4(q, w.astype(np.float64), k)
    exact_pool = 0
    for b in range(B):
        for t in range(Q):
            exact_pool += U.check_selection(pool[b, t], np.arange(N), s[b, t], P, f"pool b{b}", tie_tol=_bf16_step)
            U.check_selection(topk[b, t], np.arange(N), s[b, t], k_top, f"topk b{b}", tie_tol=_bf16_step)
            assert np.all(np.isin(topk[b, t][topk[b, t] >= 0], pool[b, t]))
    # Reindex with fresh queries inside the oracle's pool (given to both sides)
    pool_o = O.select_top(s, P).astype(np.int32)
    q2, _, w2 = _case(r, B, Q, H, d, 1)
    q2c, q2s = _fp4(q2)
    top2, _ = K.csa2_index_topk_fp4(K.REINDEX, U.dev(q2c), U.dev(q2s), U.dev(w2), *dk, k_top,
                                    pool_in=U.dev(pool_o))
    top2 = top2.cpu().numpy()
    s2 = O.index_scores_fp4(q2, w2.astype(np.float64), k, pool=pool_o)
    for b in range(B):
        for t in range(Q):
            ok = pool_o[b, t] >= 0
            U.check_selection(top2[b, t], pool_o[b, t][ok], s2[b, t][ok], k_top, f"reindex b{b}",
                              tie_tol=_bf16_step)
