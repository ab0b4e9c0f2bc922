"""Helpers for the GPU parity tests: moving seeded inputs to the device,
running a layer group through the C ABI, running the same group on the oracle,
and the comparison rules (with the tolerances stated once, here)."""
import numpy as np
import torch

import kv_cache_csa2_b200 as K
import oracle as O
from kv_cache_csa2_b200 import inputs as I

# Tolerances.  Attention: the stated bar for bf16 inputs with f32 accumulation.
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
LSE_ABS = 2e-3          # f32 logits over D <= 512 terms: bound ~5e-4, doubled
TIE_REL, TIE_ABS = 1e-3, 1e-6


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host_bf16(t):
    return I.bf16_bits_to_f32(host_bits(t)).astype(np.float64)


def bf16_ulp(x):
    """Spacing of bfloat16 numbers at |x| (2**-133 at and below the subnormal range)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax >= 2.0 ** -126, np.ldexp(1.0, (e - 7).astype(int)), 2.0 ** -133)


def check_selection(gpu_row, cand_ids, cand_scores, k, what="", tie_tol=None):
    """GPU top-k row (entry ids) against the oracle's scores of the candidates.

    The GPU set must be a valid selection (ascending, unique, candidates only,
    -1 padded, min(k, selectable) long).  It must equal the oracle's set except
    for entries whose oracle score lies within TIE_REL*|s_k| (floor TIE_ABS) of
    the oracle's k-th score s_k -- or within tie_tol(s_k) when given (bf16
    scores: one bf16 step).  Returns True when the sets are identical.
    """
    cand_ids = np.asarray(cand_ids)
    ok = cand_scores > -np.inf
    n = int(min(k, ok.sum()))
    g = np.asarray(gpu_row[:n], dtype=np.int64)
    assert np.all(np.asarray(gpu_row[n:]) == -1), f"{what}: padding"
    assert n == 0 or np.all(np.diff(g) > 0), f"{what}: not ascending/unique"
    pos = np.searchsorted(cand_ids, g)
    assert np.all(pos < len(cand_ids)) and np.all(cand_ids[np.minimum(pos, len(cand_ids) - 1)] == g), \
        f"{what}: picked a non-candidate"
    assert np.all(cand_scores[pos] > -np.inf), f"{what}: picked an unscored slot"
    if n == 0:
        return True
    opos = O.select_top(cand_scores[None], k)[0][:n]
    s_k = cand_scores[opos].min()
    tol = max(TIE_REL * abs(s_k), TIE_ABS) if tie_tol is None else float(tie_tol(s_k))
    g_only = np.setdiff1d(pos, opos)
    o_only = np.setdiff1d(opos, pos)
    assert np.all(cand_scores[g_only] >= s_k - tol), f"{what}: GPU pick below the tie band"
    assert np.all(cand_scores[o_only] <= s_k + tol), f"{what}: oracle pick missed outside the tie band"
    return g_only.size == 0


def check_attn(o_gpu, lse_gpu, o_exact, lse_exact, what=""):
    err = np.abs(o_gpu - o_exact)
    assert err.max() <= ATTN_MAX_ABS, f"{what}: max abs {err.max():.3g}"
    assert err.mean() <= ATTN_MEAN_ABS, f"{what}: mean abs {err.mean():.3g}"
    fin = np.isfinite(lse_exact)
    assert np.array_equal(np.isfinite(lse_gpu), fin), f"{what}: lse finiteness"
    if fin.any():
        d = np.abs(lse_gpu[fin] - lse_exact[fin]).max()
        assert d <= LSE_ABS, f"{what}: lse {d:.3g}"


# ---------------------------------------------------------------------------- groups

def _mode_ids(wl):
    return [{"full": K.FULL, "reindex": K.REINDEX, "reuse": K.REUSE}[m] for m in wl.modes]


def gpu_group(wl, inp):
    """Run workload wl's layer group through the C ABI.  Returns per-layer
    dicts of numpy arrays: topk, pool (Full with P), out (float64 values), lse;
    plus 'kv' (device tensor of the main KV as built on the GPU)."""
    B, Q, N, D = wl.B, wl.Q, wl.N, wl.D
    kv = torch.empty(B, N, D, dtype=torch.bfloat16, device="cuda")
    n_cached = inp["kv"].shape[1]
    if n_cached:
        kv[:, :n_cached] = dev_bf16(inp["kv"])
    if wl.compress_new_tokens:
        K.csa2_compress(dev_bf16(inp["c"]), dev(inp["z"]), dev(inp["bias"]), wl.m,
                        has_left_halo=wl.halo, out=kv[:, n_cached:], out_batch_stride=N * D)
    kv_scales = None
    kv_arg = kv
    if wl.kv_fp4:
        kv_arg, kv_scales = K.csa2_fp4_pack(kv)
    ik = dev_bf16(inp["index_k"])
    nv = dev(inp["n_visible"]) if inp["n_visible"] is not None else None
    g = K.Group(B, Q, N, D, wl.Ha, wl.Hi, wl.d, wl.k, _mode_ids(wl), P=wl.P, scale=wl.attn_scale,
                kv_fmt=K.KV_FP4 if wl.kv_fp4 else K.KV_BF16)
    res = []
    for i, mode in enumerate(wl.modes):
        L = inp["layers"][i]
        out = torch.empty(B, Q, wl.Ha, D, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(B, Q, wl.Ha, dtype=torch.float32, device="cuda")
        kw = {}
        if mode == "full":
            kw = dict(kv=kv_arg, kv_scales=kv_scales, index_k=ik, n_visible=nv)
        elif mode == "reindex":
            kw = dict(n_visible=nv)
        if mode != "reuse":
            kw.update(q_index=dev_bf16(L["q_index"]), w_index=dev(L["w_index"]))
        if "win" in L:                         # the layer's sliding-window rows
            kw["swa"] = (dev_bf16(L["win"]), dev(L["win_end"]), wl.swa)
        g.layer(i, dev_bf16(L["q_attn"]), out, lse, **kw)
        topk, pool = g.copy_selection()
        r = {"mode": mode, "topk": topk.cpu().numpy(), "out": host_bf16(out),
             "lse": lse.cpu().numpy().astype(np.float64)}
        if mode == "full" and pool is not None:
            r["pool"] = pool.cpu().numpy()
        res.append(r)
    K.csa2_device_error()
    g.close()
    return res, kv


def oracle_group(wl, inp, sample=None):
    """The same group on the oracle (queries restricted to `sample` if given)."""
    n_cached = inp["kv"].shape[1]
    new = None
    if wl.compress_new_tokens:
        _, new = O.compress(O.bf16_bits_to_float(inp["c"]), inp["z"].astype(np.float64),
                            inp["bias"].astype(np.float64), wl.m, wl.halo)
    kv_bits = inp["kv"]

    def rows(b, ids):
        ids = np.asarray(ids)
        out = np.empty((len(ids), wl.D))
        old = ids < n_cached
        out[old] = O.bf16_bits_to_float(kv_bits[b, ids[old]])
        if (~old).any():
            out[~old] = new[b, ids[~old] - n_cached]
        if wl.kv_fp4:
            out = O.fp4_unpack(*O.fp4_pack(out))
        return out

    sl = slice(None) if sample is None else sample
    layers = []
    for L in inp["layers"]:
        d = {"q_attn": O.bf16_bits_to_float(L["q_attn"][:, sl])}
        if "q_index" in L:
            d["q_index"] = O.bf16_bits_to_float(L["q_index"][:, sl])
            d["w_index"] = L["w_index"][:, sl].astype(np.float64)
        if "win" in L:
            d["swa"] = (O.bf16_bits_to_float(L["win"]), L["win_end"][:, sl], wl.swa)
        layers.append(d)
    nv = inp["n_visible"][:, sl] if inp["n_visible"] is not None else None
    ik = I.bf16_bits_to_f32(inp["index_k"])
    return O.run_group(list(wl.modes), layers, rows, ik, wl.k, wl.attn_scale, pool_size=wl.P,
                       n_visible=nv), new


def attn_on_selection(wl, kv, q_attn_bits, topk, win=None):
    """The attention kernel, through the C ABI, on a given selection (the
    oracle's) for the layer's queries: kv is the group's bf16 KV on the
    device (packed to FP4 here when the workload stores FP4), q_attn_bits the
    queries [B, Qs, Ha, D] as bf16 bits, topk int [B, Qs, k]; win = (window
    rows as bf16 bits, win_end) for a layer with the sliding-window branch."""
    kv_arg, scales = kv, None
    if wl.kv_fp4:
        kv_arg, scales = K.csa2_fp4_pack(kv)
    sel = dev(np.ascontiguousarray(topk, dtype=np.int32))
    if win is not None:
        out, lse = K.csa2_sparse_attn_swa(dev_bf16(q_attn_bits), kv_arg, sel, wl.attn_scale,
                                          win=dev_bf16(win[0]), win_end=dev(np.ascontiguousarray(win[1])),
                                          W=wl.swa, kv_scales=scales)
    else:
        out, lse = K.csa2_sparse_attn(dev_bf16(q_attn_bits), kv_arg, sel, wl.attn_scale, kv_scales=scales)
    return host_bf16(out), lse.cpu().numpy().astype(np.float64)


def compare_groups(wl, inp, gres, ores, sample=None, min_exact=0.5, kv=None):
    """Selection rule on every selecting layer, and attention on every layer.

    Attention is checked twice.  (1) The group's own output, on the queries
    whose selection equals the oracle's (the others differ only inside the
    tie band); at least one query per layer, and a fraction min_exact of
    them, must have that exact selection.  (2) When kv (the group's device
    KV) is given, the attention kernel re-run through the C ABI on the
    oracle's selection, for every query of the layer, against the oracle's
    output over that selection.  Only oracle data flows into the GPU; no GPU
    result is fed to the oracle.

    A Reindex layer with a pool is compared with the oracle only for queries
    whose GPU pool equals the oracle's pool; for the others the GPU row is
    checked to be a valid subset of the GPU's own pool."""
    sl = np.arange(wl.Q) if sample is None else np.asarray(sample)
    ik = I.bf16_bits_to_f32(inp["index_k"])
    same = np.ones((wl.B, len(sl)), dtype=bool)
    pool_o = pool_g = pool_same = None
    for i, (g, o) in enumerate(zip(gres, ores)):
        mode = g["mode"]
        if mode in ("full", "reindex"):
            L = inp["layers"][i]
            q = O.bf16_bits_to_float(L["q_index"][:, sl])
            w = L["w_index"][:, sl].astype(np.float64)
            nv = inp["n_visible"][:, sl] if inp["n_visible"] is not None else None
            use_pool = mode == "reindex" and wl.P > 0
            s = O.index_scores(q, w, ik, n_visible=None if use_pool else nv,
                               pool=pool_o if use_pool else None)
            same = np.zeros_like(same)
            if mode == "full" and wl.P > 0:
                pool_o, pool_g = o["pool"], g["pool"][:, sl]
                pool_same = np.zeros_like(same)
            for b in range(wl.B):
                for t, qi in enumerate(sl):
                    row = g["topk"][b, qi]
                    if use_pool and not pool_same[b, t]:
                        gp = pool_g[b, t]
                        sel = row[row >= 0]
                        assert np.all(np.isin(sel, gp[gp >= 0])) and np.all(np.diff(sel) > 0)
                        continue
                    if use_pool:
                        cand = pool_o[b, t]
                        ok = cand >= 0
                        ids, sc = cand[ok], s[b, t][ok]
                    else:
                        ids, sc = np.arange(wl.N), s[b, t]
                    same[b, t] = check_selection(row, ids, sc, wl.k, f"layer {i} b{b} q{qi}")
                    if mode == "full" and wl.P > 0:
                        pool_same[b, t] = check_selection(pool_g[b, t], ids, sc, wl.P,
                                                          f"pool b{b} q{qi}")
        assert same.any(), f"layer {i}: no query has the oracle's exact selection"
        assert same.mean() >= min_exact, f"layer {i}: only {same.mean():.2f} exact selections"
        gi = g["out"][:, sl][same]
        oi = o["o"][same]
        check_attn(gi, g["lse"][:, sl][same], oi, o["lse"][same], f"layer {i} ({mode})")
        if kv is not None:
            L = inp["layers"][i]
            q_bits = L["q_attn"][:, sl]
            win = (L["win"], L["win_end"][:, sl]) if "win" in L else None
            out_r, lse_r = attn_on_selection(wl, kv, q_bits, o["topk"], win=win)
            check_attn(out_r, lse_r, o["o"], o["lse"], f"layer {i} ({mode}) on the oracle's selection")
    return same
