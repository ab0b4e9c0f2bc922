"""Python binding of libcsa2 (the CSA2 hot path on B200).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libcsa2.so``; PyTorch supplies device memory and streams.  The functions
carry the C ABI's names (include/csa2.h) and take torch CUDA tensors.  If the
library is not built, importing works but the first call raises.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "CSA2Error", "lib", "lib_path", "FULL", "REINDEX", "REUSE", "KV_BF16", "KV_FP4", "ACT_RELU",
    "ACT_IDENTITY", "csa2_compress", "csa2_index_scores", "csa2_select_topk", "csa2_select_topk_noalloc",
    "csa2_index_topk",
    "csa2_sparse_attn", "csa2_sparse_attn_swa", "csa2_dense_attn", "csa2_compress_hca",
    "csa2_index_scores_fp4", "csa2_index_topk_fp4",
    "csa2_fp4_pack", "csa2_fp4_unpack", "Group", "csa2_device_error",
    "launch_counts", "reset_launch_counts", "set_fault", "set_device_wait", "EXPORTED_SYMBOLS",
]

FULL, REINDEX, REUSE = 0, 1, 2
KV_BF16, KV_FP4 = 0, 1
ACT_RELU, ACT_IDENTITY = 0, 1
_MODE = {"full": FULL, "reindex": REINDEX, "reuse": REUSE, FULL: FULL, REINDEX: REINDEX,
         REUSE: REUSE}

_P, _I, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


class CSA2Kv(ctypes.Structure):
    _fields_ = [("fmt", _I), ("data", _P), ("scales", _P), ("n", _I64), ("dim", _I)]


class CSA2GroupDesc(ctypes.Structure):
    _fields_ = [("B", _I), ("Q", _I), ("N", _I64), ("D", _I), ("Ha", _I), ("Hi", _I), ("d", _I),
                ("k", _I), ("P", _I), ("scale", _F), ("kv_fmt", _I), ("act", _I),
                ("n_layers", _I), ("modes", ctypes.POINTER(_I))]


class CSA2LayerIO(ctypes.Structure):
    _fields_ = [("kv", CSA2Kv), ("index_k", _P), ("n_visible", _P), ("q_index", _P),
                ("w_index", _P), ("q_attn", _P), ("out", _P), ("lse", _P),
                ("swa_kv", _P), ("swa_rows", _I64), ("swa_end", _P), ("swa_window", _I)]


# name -> (restype, argtypes); every symbol include/csa2.h declares
_SIGS = {
    "csa2_compress": (_I, [_P, _P, _P, _I, _I64, _I, _I, _I, _P, _I64, _P]),
    "csa2_index_scores": (_I, [_P, _P, _P, _I, _I, _I, _I, _I64, _P, _P, _I, _I, _P, _P]),
    "csa2_select_topk_workspace": (_SZ, [_I64, _I64, _I]),
    "csa2_select_topk": (_I, [_P, _I64, _I64, _I, _P, _P, _P, _SZ, _P]),
    "csa2_select_topk_noalloc": (_I, [_P, _I64, _I64, _I, _P, _P, _P]),
    "csa2_index_topk_workspace": (_SZ, [_I, _I, _I64, _I, _I, _I]),
    "csa2_index_topk": (_I, [_I, _P, _P, _P, _I, _I, _I, _I, _I64, _P, _P, _I, _I, _P, _P, _I, _I,
                             _P, _SZ, _P]),
    "csa2_sparse_attn_workspace": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "csa2_sparse_attn": (_I, [_I, _P, ctypes.POINTER(CSA2Kv), _P, _I, _I, _I, _I, _F, _P, _P, _P,
                              _SZ, _P]),
    "csa2_index_scores_fp4": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I64, _P, _P, _I, _I, _P, _P]),
    "csa2_index_topk_fp4": (_I, [_I, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I64, _P, _P, _I, _I, _P, _P,
                                 _I, _I, _P, _SZ, _P]),
    "csa2_sparse_attn_swa_workspace": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "csa2_sparse_attn_swa": (_I, [_I, _P, ctypes.POINTER(CSA2Kv), _P, _I, _I, _I, _I, _F, _P, _I64,
                                  _P, _I, _P, _P, _P, _SZ, _P]),
    "csa2_dense_attn_workspace": (_SZ, [_I, _I, _I, _I, _I64, _I]),
    "csa2_dense_attn": (_I, [_P, ctypes.POINTER(CSA2Kv), _P, _I, _I, _I, _F, _P, _P, _P, _SZ, _P]),
    "csa2_compress_hca": (_I, [_P, _P, _P, _I, _I64, _I, _I, _P, _I64, _P]),
    "csa2_fp4_pack": (_I, [_P, _I64, _I, _P, _P, _P]),
    "csa2_fp4_unpack": (_I, [_P, _P, _I64, _I, _P, _P]),
    "csa2_group_create": (_I, [ctypes.POINTER(_P), ctypes.POINTER(CSA2GroupDesc)]),
    "csa2_group_layer": (_I, [_P, _I, ctypes.POINTER(CSA2LayerIO), _P]),
    "csa2_group_selection": (_I, [_P, ctypes.POINTER(_P), ctypes.POINTER(_P)]),
    "csa2_group_copy_selection": (_I, [_P, _P, _P, _P]),
    "csa2_group_destroy": (None, [_P]),
    "csa2_status_string": (ctypes.c_char_p, [_I]),
    "csa2_last_error": (ctypes.c_char_p, []),
    "csa2_device_error": (_I, [_P]),
    "csa2_launch_counts": (_I, [ctypes.POINTER(_I64), _I]),
    "csa2_reset_launch_counts": (None, []),
    "csa2_set_fault": (_I, [ctypes.c_char_p]),
    "csa2_set_device_wait": (_I, [ctypes.c_uint64, _I]),
    "csa2_timing_enable": (_I, [_I]),
    "csa2_kernel_times": (_I, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I64), _I]),
    "csa2_timing_reset": (None, []),
    "csa2_version": (_I, []),
}
EXPORTED_SYMBOLS = tuple(_SIGS)

_LIB = None


def lib_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcsa2.so")


def lib():
    """Load libcsa2.so (raises if it is missing: there is no fallback path)."""
    global _LIB
    if _LIB is None:
        path = lib_path()
        if not os.path.exists(path):
            raise ImportError(f"{path} is not built; run `python -m kv_cache_csa2_b200.build`")
        L = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


class CSA2Error(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{lib().csa2_status_string(status).decode()}: {msg}")
        self.status = status


def _check(status: int) -> None:
    if status != 0:
        raise CSA2Error(status, lib().csa2_last_error().decode(errors="replace"))


def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, ndim, name):
    torch = _torch()
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype != dtype or t.dim() != ndim or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} with {ndim} dims, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")
    return t


# ------------------------------------------------------------------ (a1)
def csa2_compress(c, z, bias, m: int, has_left_halo: bool = False, out=None,
                  out_batch_stride: int = 0, stream=None):
    """Compress raw tokens (c bf16 / z f32 [B, T+halo, D], bias f32 [2m, D]) into entries."""
    torch = _torch()
    _need(c, torch.bfloat16, 3, "c")
    _need(z, torch.float32, 3, "z")
    _need(bias, torch.float32, 2, "bias")
    B, t_in, D = c.shape
    T = t_in - (m if has_left_halo else 0)
    if out is None:
        out = torch.empty(B, T // m, D, dtype=torch.bfloat16, device=c.device)
    _check(lib().csa2_compress(_ptr(c), _ptr(z), _ptr(bias), B, T, D, m, int(has_left_halo),
                               _ptr(out), out_batch_stride, _stream(stream)))
    return out


# ------------------------------------------------------------------ (a2, a3)
def csa2_index_scores(q, w, k, n_visible=None, pool=None, act: int = ACT_RELU, out=None,
                      stream=None):
    torch = _torch()
    _need(q, torch.bfloat16, 4, "q")
    _need(w, torch.float32, 3, "w")
    _need(k, torch.bfloat16, 3, "k")
    B, Q, H, d = q.shape
    N = k.shape[1]
    P = pool.shape[2] if pool is not None else 0
    if pool is not None:
        _need(pool, torch.int32, 3, "pool")
    if n_visible is not None:
        _need(n_visible, torch.int32, 2, "n_visible")
    if out is None:
        out = torch.empty(B, Q, P if pool is not None else N, dtype=torch.float32, device=q.device)
    _check(lib().csa2_index_scores(_ptr(q), _ptr(w), _ptr(k), B, Q, H, d, N, _ptr(n_visible),
                                   _ptr(pool), P, act, _ptr(out), _stream(stream)))
    return out


def csa2_index_scores_fp4(q_codes, q_scales, w, k_codes, k_scales, n_visible=None, pool=None,
                          act: int = ACT_RELU, out=None, stream=None):
    """FP4 indexer: q codes/scales [B,Q,H,d/2]/[B,Q,H,d/16], K codes/scales
    [B,N,d/2]/[B,N,d/16] (csa2_fp4_pack's format); returns bf16 scores."""
    torch = _torch()
    _need(q_codes, torch.uint8, 4, "q_codes")
    _need(k_codes, torch.uint8, 3, "k_codes")
    _need(w, torch.float32, 3, "w")
    B, Q, H, d2 = q_codes.shape
    N = k_codes.shape[1]
    P = pool.shape[2] if pool is not None else 0
    if out is None:
        out = torch.empty(B, Q, P if pool is not None else N, dtype=torch.bfloat16, device=q_codes.device)
    _check(lib().csa2_index_scores_fp4(_ptr(q_codes), _ptr(q_scales), _ptr(w), _ptr(k_codes),
                                       _ptr(k_scales), B, Q, H, 2 * d2, N, _ptr(n_visible), _ptr(pool),
                                       P, act, _ptr(out), _stream(stream)))
    return out


def csa2_index_topk_fp4(mode, q_codes, q_scales, w, k_codes, k_scales, k_top: int, n_visible=None,
                        pool_in=None, pool_size: int = 0, act: int = ACT_RELU, stream=None):
    """Scores (FP4 indexer, bf16) + selection for one Full / Reindex layer."""
    torch = _torch()
    mode = _MODE[mode]
    B, Q, H, d2 = q_codes.shape
    N = k_codes.shape[1]
    P_in = pool_in.shape[2] if pool_in is not None else 0
    topk = torch.empty(B, Q, k_top, dtype=torch.int32, device=q_codes.device)
    pool = (torch.empty(B, Q, pool_size, dtype=torch.int32, device=q_codes.device)
            if pool_size > 0 else None)
    nb = lib().csa2_index_topk_workspace(B, Q, N, P_in, k_top, pool_size)
    ws = _workspace(nb, q_codes.device)
    _check(lib().csa2_index_topk_fp4(mode, _ptr(q_codes), _ptr(q_scales), _ptr(w), _ptr(k_codes),
                                     _ptr(k_scales), B, Q, H, 2 * d2, N, _ptr(n_visible),
                                     _ptr(pool_in), P_in, k_top, _ptr(topk), _ptr(pool), pool_size,
                                     act, _ptr(ws), nb, _stream(stream)))
    return topk, pool


def _workspace(nbytes, device):
    torch = _torch()
    if nbytes == 0:
        return None
    return torch.empty(int(nbytes), dtype=torch.uint8, device=device)


def csa2_select_topk(scores, count: int, ids=None, out=None, stream=None):
    """Top-`count` positions of each row of scores [..., L] (ascending, -1 padded)."""
    torch = _torch()
    L = scores.shape[-1]
    rows = scores.numel() // max(L, 1)
    if out is None:
        out = torch.empty(*scores.shape[:-1], count, dtype=torch.int32, device=scores.device)
    nb = lib().csa2_select_topk_workspace(rows, L, count)
    ws = _workspace(nb, scores.device)
    _check(lib().csa2_select_topk(_ptr(scores), rows, L, count, _ptr(ids), _ptr(out), _ptr(ws),
                                  nb, _stream(stream)))
    return out


def csa2_select_topk_noalloc(scores, count: int, ids=None, out=None, stream=None):
    """csa2_select_topk with the library's static scratch (no workspace is allocated)."""
    torch = _torch()
    L = scores.shape[-1]
    rows = scores.numel() // max(L, 1)
    if out is None:
        out = torch.empty(*scores.shape[:-1], count, dtype=torch.int32, device=scores.device)
    _check(lib().csa2_select_topk_noalloc(_ptr(scores), rows, L, count, _ptr(ids), _ptr(out),
                                          _stream(stream)))
    return out


def csa2_index_topk(mode, q, w, k, k_top: int, n_visible=None, pool_in=None, pool_size: int = 0,
                    act: int = ACT_RELU, stream=None):
    """Scores + selection for one Full / Reindex layer.  Returns (topk, pool or None)."""
    torch = _torch()
    mode = _MODE[mode]
    B, Q, H, d = q.shape
    N = k.shape[1]
    P_in = pool_in.shape[2] if pool_in is not None else 0
    topk = torch.empty(B, Q, k_top, dtype=torch.int32, device=q.device)
    pool = (torch.empty(B, Q, pool_size, dtype=torch.int32, device=q.device)
            if pool_size > 0 else None)
    nb = lib().csa2_index_topk_workspace(B, Q, N, P_in, k_top, pool_size)
    ws = _workspace(nb, q.device)
    _check(lib().csa2_index_topk(mode, _ptr(q), _ptr(w), _ptr(k), B, Q, H, d, N, _ptr(n_visible),
                                 _ptr(pool_in), P_in, k_top, _ptr(topk), _ptr(pool), pool_size,
                                 act, _ptr(ws), nb, _stream(stream)))
    return topk, pool


# ------------------------------------------------------------------ (a4)
def make_kv(kv, scales=None):
    """csa2_kv for a bf16 [B, n, D] tensor, or FP4 codes uint8 [B, n, D/2] + scales [B, n, D/16]."""
    if scales is None:
        return CSA2Kv(KV_BF16, kv.data_ptr(), None, kv.shape[1], kv.shape[2])
    return CSA2Kv(KV_FP4, kv.data_ptr(), scales.data_ptr(), kv.shape[1], kv.shape[2] * 2)


def csa2_sparse_attn(q, kv, topk, scale: float, kv_scales=None, mode=FULL, out=None, lse=None,
                     stream=None):
    torch = _torch()
    _need(q, torch.bfloat16, 4, "q")
    _need(topk, torch.int32, 3, "topk")
    B, Q, Ha, D = q.shape
    k = topk.shape[2]
    desc = make_kv(kv, kv_scales)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Q, Ha, dtype=torch.float32, device=q.device)
    nb = lib().csa2_sparse_attn_workspace(B, Q, Ha, D, k, desc.fmt)
    ws = _workspace(nb, q.device)
    _check(lib().csa2_sparse_attn(_MODE[mode], _ptr(q), ctypes.byref(desc), _ptr(topk), B, Q, Ha,
                                  k, scale, _ptr(out), _ptr(lse), _ptr(ws), nb, _stream(stream)))
    return out, lse


def csa2_sparse_attn_swa(q, kv, topk, scale: float, win, win_end, W: int = 128, kv_scales=None,
                         mode=FULL, out=None, lse=None, stream=None):
    """Sparse attention with the layer's sliding-window branch in the same
    softmax: win bf16 [B, R, D] window rows, win_end int32 [B, Q]."""
    torch = _torch()
    _need(q, torch.bfloat16, 4, "q")
    _need(topk, torch.int32, 3, "topk")
    _need(win, torch.bfloat16, 3, "win")
    _need(win_end, torch.int32, 2, "win_end")
    B, Q, Ha, D = q.shape
    k = topk.shape[2]
    desc = make_kv(kv, kv_scales)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Q, Ha, dtype=torch.float32, device=q.device)
    nb = lib().csa2_sparse_attn_swa_workspace(B, Q, Ha, D, k, desc.fmt)
    ws = _workspace(nb, q.device)
    _check(lib().csa2_sparse_attn_swa(_MODE[mode], _ptr(q), ctypes.byref(desc), _ptr(topk), B, Q,
                                      Ha, k, scale, _ptr(win), win.shape[1], _ptr(win_end), W,
                                      _ptr(out), _ptr(lse), _ptr(ws), nb, _stream(stream)))
    return out, lse


def csa2_dense_attn(q, kv, scale: float, n_visible=None, kv_scales=None, out=None, lse=None,
                    stream=None):
    """HCA attention: every query attends to entries [0, n_visible) of its sequence."""
    torch = _torch()
    _need(q, torch.bfloat16, 4, "q")
    if n_visible is not None:
        _need(n_visible, torch.int32, 2, "n_visible")
    B, Q, Ha, D = q.shape
    desc = make_kv(kv, kv_scales)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Q, Ha, dtype=torch.float32, device=q.device)
    nb = lib().csa2_dense_attn_workspace(B, Q, Ha, D, desc.n, desc.fmt)
    ws = _workspace(nb, q.device)
    _check(lib().csa2_dense_attn(_ptr(q), ctypes.byref(desc), _ptr(n_visible), B, Q, Ha, scale,
                                 _ptr(out), _ptr(lse), _ptr(ws), nb, _stream(stream)))
    return out, lse


def csa2_compress_hca(c, z, bias, m: int, out=None, out_batch_stride: int = 0, stream=None):
    """HCA compression of raw tokens (c bf16 / z f32 [B, T, D], bias f32 [m, D])."""
    torch = _torch()
    _need(c, torch.bfloat16, 3, "c")
    _need(z, torch.float32, 3, "z")
    _need(bias, torch.float32, 2, "bias")
    B, T, D = c.shape
    if out is None:
        out = torch.empty(B, T // m, D, dtype=torch.bfloat16, device=c.device)
    _check(lib().csa2_compress_hca(_ptr(c), _ptr(z), _ptr(bias), B, T, D, m, _ptr(out),
                                   out_batch_stride, _stream(stream)))
    return out


# ------------------------------------------------------------------ (a5)
def csa2_fp4_pack(x, stream=None):
    torch = _torch()
    rows, D = x.reshape(-1, x.shape[-1]).shape
    codes = torch.empty(*x.shape[:-1], D // 2, dtype=torch.uint8, device=x.device)
    scales = torch.empty(*x.shape[:-1], D // 16, dtype=torch.uint8, device=x.device)
    _check(lib().csa2_fp4_pack(_ptr(x), rows, D, _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def csa2_fp4_unpack(codes, scales, stream=None):
    torch = _torch()
    D = codes.shape[-1] * 2
    rows = codes.numel() // (D // 2)
    x = torch.empty(*codes.shape[:-1], D, dtype=torch.bfloat16, device=codes.device)
    _check(lib().csa2_fp4_unpack(_ptr(codes), _ptr(scales), rows, D, _ptr(x), _stream(stream)))
    return x


# ------------------------------------------------------------------ (a6)
class Group:
    """A CSA2 layer group (Full / Reindex / Reuse modes) driven through the C ABI."""

    def __init__(self, B, Q, N, D, Ha, Hi, d, k, modes, P=0, scale=None, kv_fmt=KV_BF16,
                 act=ACT_RELU):
        self.modes = [_MODE[m] for m in modes]
        arr = (_I * len(self.modes))(*self.modes)
        self._modes_arr = arr
        desc = CSA2GroupDesc(B, Q, N, D, Ha, Hi, d, k, P,
                             (D ** -0.5) if scale is None else scale, kv_fmt, act,
                             len(self.modes), arr)
        h = _P()
        _check(lib().csa2_group_create(ctypes.byref(h), ctypes.byref(desc)))
        self._h = h
        self.desc = desc

    def layer(self, i, q_attn, out, lse=None, kv=None, kv_scales=None, index_k=None,
              q_index=None, w_index=None, n_visible=None, swa=None, stream=None):
        """swa: optional (win bf16 [B, R, D], win_end int32 [B, Q], W), this
        layer's own sliding-window rows."""
        io = CSA2LayerIO()
        if kv is not None:
            io.kv = make_kv(kv, kv_scales)
        io.index_k = _ptr(index_k)
        io.n_visible = _ptr(n_visible)
        io.q_index = _ptr(q_index)
        io.w_index = _ptr(w_index)
        io.q_attn = _ptr(q_attn)
        io.out = _ptr(out)
        io.lse = _ptr(lse)
        if swa is not None:
            win, win_end, W = swa
            io.swa_kv = _ptr(win)
            io.swa_rows = win.shape[1]
            io.swa_end = _ptr(win_end)
            io.swa_window = W
        _check(lib().csa2_group_layer(self._h, i, ctypes.byref(io), _stream(stream)))

    def selection(self):
        t, p = _P(), _P()
        _check(lib().csa2_group_selection(self._h, ctypes.byref(t), ctypes.byref(p)))
        return t.value, p.value

    def copy_selection(self, stream=None):
        """(topk [B,Q,k], pool [B,Q,P] or None) copies of the current selection."""
        torch = _torch()
        d = self.desc
        topk = torch.empty(d.B, d.Q, d.k, dtype=torch.int32, device="cuda")
        pool = torch.empty(d.B, d.Q, d.P, dtype=torch.int32, device="cuda") if d.P > 0 else None
        _check(lib().csa2_group_copy_selection(self._h, _ptr(topk), _ptr(pool), _stream(stream)))
        return topk, pool

    def close(self):
        if getattr(self, "_h", None) and self._h.value:
            lib().csa2_group_destroy(self._h)
            self._h = _P()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ------------------------------------------------------------------ errors, counters
def csa2_device_error(stream=None):
    """Synchronise and raise if a kernel recorded a device-side error."""
    _check(lib().csa2_device_error(_stream(stream)))


LAUNCH_KINDS = ("compress", "index_scores", "topk", "attn", "attn_combine", "fp4_pack",
                "fp4_unpack", "other", "index_pool")


def launch_counts() -> dict:
    arr = (_I64 * len(LAUNCH_KINDS))()
    lib().csa2_launch_counts(arr, len(LAUNCH_KINDS))
    return dict(zip(LAUNCH_KINDS, arr))


def reset_launch_counts() -> None:
    lib().csa2_reset_launch_counts()


def timing_enable(on: bool) -> None:
    """Bracket every library launch with CUDA events (instrumentation)."""
    _check(lib().csa2_timing_enable(int(bool(on))))


def timing_reset() -> None:
    lib().csa2_timing_reset()


def kernel_times() -> dict:
    """{kind: (total_ms, timed_launches)} since the last timing_reset()."""
    n = len(LAUNCH_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (_I64 * n)()
    lib().csa2_kernel_times(ms, cnt, n)
    return {k: (ms[i], cnt[i]) for i, k in enumerate(LAUNCH_KINDS)}


def set_fault(kind: str) -> None:
    _check(lib().csa2_set_fault(kind.encode()))


def set_device_wait(limit_ns: int = 0, unreachable: bool = False) -> None:
    """Bound of the cross-CTA device waits (0 = default, 1 s); `unreachable`
    makes each such wait run out (a test of the error path)."""
    _check(lib().csa2_set_device_wait(int(limit_ns), int(bool(unreachable))))
