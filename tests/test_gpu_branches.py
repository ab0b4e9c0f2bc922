"""GPU parity of the rows beside the CSA2 path proper, through the C ABI,
against the float64 oracle: HCA compression and HCA (dense) attention, and
the sliding-window branch that joins the CSA2 selection in one softmax
(standalone and inside a layer group)."""
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
    K.csa2_device_error()


def _rng(seed):
    return np.random.default_rng(seed)


def _bf(r, shape, std=1.0):
    return I.f32_to_bf16_bits((r.standard_normal(shape) * std).astype(np.float32))


# ------------------------------------------------------------------ HCA compression

@pytest.mark.parametrize("m,T,D", [(1, 37, 16), (4, 1027, 128), (64, 64 * 5 + 7, 512),
                                   (128, 128 * 9, 512), (1024, 2048, 64)])
def test_compress_hca_parity(m, T, D):
    r = _rng(50)
    c = _bf(r, (2, T, D))
    z = (r.standard_normal((2, T, D)) * 2).astype(np.float32)
    bias = (r.standard_normal((m, D)) * 0.5).astype(np.float32)
    out = K.csa2_compress_hca(U.dev_bf16(c), U.dev(z), U.dev(bias), m)
    assert out.shape == (2, T // m, D)
    exact, _ = O.compress_hca(O.bf16_bits_to_float(c), z.astype(np.float64), bias.astype(np.float64), m)
    got = U.host_bf16(out)
    tol = U.bf16_ulp(exact) + 1e-6 * np.abs(O.bf16_bits_to_float(c)).max()
    assert np.all(np.abs(got - exact) <= tol), np.abs(got - exact).max()


def test_compress_hca_appends_into_kv_buffer():
    r = _rng(51)
    m, T, D, B = 16, 64, 32, 2
    c, z = _bf(r, (B, T, D)), r.standard_normal((B, T, D)).astype(np.float32)
    bias = r.standard_normal((m, D)).astype(np.float32)
    buf = torch.full((B, 10, D), 7.0, dtype=torch.bfloat16, device="cuda")
    K.csa2_compress_hca(U.dev_bf16(c), U.dev(z), U.dev(bias), m, out=buf[:, 3:], out_batch_stride=10 * D)
    exact, _ = O.compress_hca(O.bf16_bits_to_float(c), z.astype(np.float64), bias.astype(np.float64), m)
    assert np.all(np.abs(U.host_bf16(buf[:, 3:7]) - exact) <= U.bf16_ulp(exact) + 1e-6)
    assert torch.all(buf[:, :3] == 7) and torch.all(buf[:, 7:] == 7)


# ------------------------------------------------------------------ HCA attention

@pytest.mark.parametrize("Ha,D,N,fp4,causal", [(64, 512, 3000, False, False), (64, 512, 8192, False, True),
                                               (64, 512, 700, True, False), (16, 128, 2000, False, True),
                                               (16, 128, 1500, True, False), (64, 512, 9000, False, False)])
def test_dense_attn_parity(Ha, D, N, fp4, causal):
    r = _rng(52)
    B, Q = 2, 3
    q = _bf(r, (B, Q, Ha, D))
    kv = _bf(r, (B, N, D))
    nv = r.integers(0, N + 1, (B, Q)).astype(np.int32) if causal else None
    if causal:
        nv[0, 0], nv[1, 2] = N, 0                         # everything visible; nothing visible
    kvd = U.dev_bf16(kv)
    scale = D ** -0.5
    if fp4:
        codes, scales = K.csa2_fp4_pack(kvd)
        out, lse = K.csa2_dense_attn(U.dev_bf16(q), codes, scale, kv_scales=scales,
                                     n_visible=U.dev(nv) if causal else None)
        kvv = O.fp4_unpack(*O.fp4_pack(O.bf16_bits_to_float(kv.reshape(-1, D)))).reshape(B, N, D)
    else:
        out, lse = K.csa2_dense_attn(U.dev_bf16(q), kvd, scale, n_visible=U.dev(nv) if causal else None)
        kvv = O.bf16_bits_to_float(kv)
    o, _, l = O.dense_attn(O.bf16_bits_to_float(q), kvv, scale, n_visible=nv)
    U.check_attn(U.host_bf16(out), lse.cpu().numpy().astype(np.float64), o, l, f"dense Ha{Ha} D{D} N{N}")


# ------------------------------------------------------------------ sliding-window branch

def _swa_case(r, B, Q, Ha, D, N, k, R, W, prefill):
    q = _bf(r, (B, Q, Ha, D))
    kv = _bf(r, (B, N, D))
    win = _bf(r, (B, R, D))
    topk = np.full((B, Q, k), -1, dtype=np.int32)
    for b in range(B):
        for t in range(Q):
            n = int(r.integers(0, k + 1)) if (b + t) % 3 == 2 else k
            topk[b, t, :n] = np.sort(r.choice(N, size=n, replace=False))
    if prefill:      # query t sits on window row R - Q + t (its own token); early ones see < W rows
        we = np.broadcast_to(np.arange(R - Q + 1, R + 1, dtype=np.int32), (B, Q)).copy()
        we[0, 0] = 0                                      # an empty window
        we[-1, 0] = min(R, 3)                             # fewer rows than W
    else:            # decode: the last W rows
        we = np.full((B, Q), R, dtype=np.int32)
    return q, kv, win, topk, we


@pytest.mark.parametrize("Ha,D,N,k,R,W,prefill,fp4", [
    (64, 512, 5000, 2048, 128, 128, False, False),     # decode, tensor-core kernel, 17 tiles
    (64, 512, 3000, 300, 200, 128, True, False),       # prefill-like window ends
    (64, 512, 900, 0, 64, 64, True, False),            # no selected entries: the window alone
    (64, 512, 5000, 4096, 128, 100, False, False),     # W < 128, 33 tiles (two waves)
    (16, 128, 3000, 256, 160, 128, True, True),        # CUDA-core kernel, FP4 main KV, bf16 window
    (16, 128, 500, 33, 100, 64, False, False),
])
def test_sparse_attn_swa_parity(Ha, D, N, k, R, W, prefill, fp4):
    r = _rng(53)
    B, Q = 2, 3
    q, kv, win, topk, we = _swa_case(r, B, Q, Ha, D, N, k, R, W, prefill)
    kvd = U.dev_bf16(kv)
    scale = D ** -0.5
    args = dict(win=U.dev_bf16(win), win_end=U.dev(we), W=W)
    if fp4:
        codes, scales = K.csa2_fp4_pack(kvd)
        out, lse = K.csa2_sparse_attn_swa(U.dev_bf16(q), codes, U.dev(topk), scale, kv_scales=scales, **args)
        kvv = O.fp4_unpack(*O.fp4_pack(O.bf16_bits_to_float(kv.reshape(-1, D)))).reshape(B, N, D)
    else:
        out, lse = K.csa2_sparse_attn_swa(U.dev_bf16(q), kvd, U.dev(topk), scale, **args)
        kvv = O.bf16_bits_to_float(kv)
    o, _, l = O.sparse_attn_swa(O.bf16_bits_to_float(q), kvv, topk, O.bf16_bits_to_float(win), we, W, scale)
    U.check_attn(U.host_bf16(out), lse.cpu().numpy().astype(np.float64), o, l, f"swa Ha{Ha} k{k} W{W}")


def test_sparse_attn_swa_window_end_out_of_range_is_recorded():
    r = _rng(54)
    q, kv, win, topk, we = _swa_case(r, 1, 2, 64, 512, 600, 200, 64, 64, False)
    we[0, 1] = 65                                         # one past the window buffer
    K.csa2_sparse_attn_swa(U.dev_bf16(q), U.dev_bf16(kv), U.dev(topk), 0.05, win=U.dev_bf16(win),
                           win_end=U.dev(we), W=64)
    with pytest.raises(K.CSA2Error) as e:
        K.csa2_device_error()
    assert e.value.status == 7


def test_group_with_window_branches():
    """A small hierarchical group (F, Ri, U) whose every layer has its own
    window rows: the selection rule per selecting layer and the attention of
    every layer against the oracle's group with the same windows."""
    wl = C.C4.replace(name="c4_swa_small", B=2, L=4 * 20000, P=3000, k=500,
                      modes=("full", "reindex", "reuse"))
    inp = I.make_inputs(wl, seed=15)
    r = _rng(55)
    R, W = 128, 128
    wins = [_bf(r, (wl.B, R, wl.D)) for _ in wl.modes]
    we = np.full((wl.B, wl.Q), R, dtype=np.int32)
    kv, ik = U.dev_bf16(inp["kv"]), U.dev_bf16(inp["index_k"])
    g = K.Group(wl.B, wl.Q, wl.N, wl.D, wl.Ha, wl.Hi, wl.d, wl.k, list(wl.modes), P=wl.P, scale=wl.attn_scale)
    gres = []
    for i, mode in enumerate(wl.modes):
        L = inp["layers"][i]
        out = torch.empty(wl.B, wl.Q, wl.Ha, wl.D, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(wl.B, wl.Q, wl.Ha, dtype=torch.float32, device="cuda")
        kw = dict(kv=kv, index_k=ik) if mode == "full" else {}
        if mode != "reuse":
            kw.update(q_index=U.dev_bf16(L["q_index"]), w_index=U.dev(L["w_index"]))
        g.layer(i, U.dev_bf16(L["q_attn"]), out, lse, swa=(U.dev_bf16(wins[i]), U.dev(we), W), **kw)
        topk, _ = g.copy_selection()
        gres.append((topk.cpu().numpy(), U.host_bf16(out), lse.cpu().numpy().astype(np.float64)))
    K.csa2_device_error()
    g.close()
    layers = []
    for i, L in enumerate(inp["layers"]):
        d = {"q_attn": O.bf16_bits_to_float(L["q_attn"]),
             "swa": (O.bf16_bits_to_float(wins[i]), we, W)}
        if "q_index" in L:
            d["q_index"] = O.bf16_bits_to_float(L["q_index"])
            d["w_index"] = L["w_index"].astype(np.float64)
        layers.append(d)
    ores = O.run_group(list(wl.modes), layers, O.bf16_bits_to_float(inp["kv"]),
                       I.bf16_bits_to_f32(inp["index_k"]), wl.k, wl.attn_scale, pool_size=wl.P)
    for i in range(wl.n_layers):
        topk, out, lse = gres[i]
        same = np.array([[np.array_equal(topk[b, t], ores[i]["topk"][b, t]) for t in range(wl.Q)]
                         for b in range(wl.B)])
        assert same.any(), f"layer {i}: no exact selection"
        U.check_attn(out[same], lse[same], ores[i]["o"][same], ores[i]["lse"][same], f"layer {i}")
        # every query, on the oracle's selection
        o2, l2 = K.csa2_sparse_attn_swa(U.dev_bf16(inp["layers"][i]["q_attn"]), kv,
                                        U.dev(ores[i]["topk"].astype(np.int32)), wl.attn_scale,
                                        win=U.dev_bf16(wins[i]), win_end=U.dev(we), W=W)
        U.check_attn(U.host_bf16(o2), l2.cpu().numpy().astype(np.float64), ores[i]["o"], ores[i]["lse"],
                     f"layer {i} on the oracle's selection")
