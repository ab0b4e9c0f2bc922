"""Seeded synthetic inputs for the CSA2 workloads (numpy, host memory).

This module only draws random numbers and stores them in the input formats
(bfloat16 bit patterns, float32, int32).  It holds none of the method's
arithmetic, so both the CUDA path (through the tests and the benchmark) and
the float64 oracle can be fed from it.

Every tensor has its own stream of generators: chunk i of a tensor (2**22
values) is drawn by PCG64 seeded from the sequence (seed, crc32(workload
name), tensor id, i), so a tensor's values depend neither on which other
tensors were drawn nor on how many threads draw the chunks.  bfloat16 inputs
are drawn in float32 and rounded to the nearest bfloat16 (ties to even).
"""
from __future__ import annotations

import os
import zlib
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from .configs import FULL, REINDEX, Workload, n_visible

_CHUNK = 1 << 22
_THREADS = max(1, min(16, os.cpu_count() or 1))


class _Stream:
    """Identifies one tensor's random stream: (seed, workload name, tensor id)."""

    def __init__(self, seed: int, name: str, tensor_id: int):
        self.key = [int(seed), zlib.crc32(name.encode()), int(tensor_id)]

    def chunk(self, i: int) -> np.random.Generator:
        return np.random.Generator(np.random.PCG64(np.random.SeedSequence(self.key + [int(i)])))


def _rng(seed: int, name: str, tensor_id: int) -> _Stream:
    return _Stream(seed, name, tensor_id)


def _fill_chunks(n: int, fn) -> None:
    """Call fn(i, start, stop) for every chunk, on a thread pool."""
    spans = [(i, s, min(n, s + _CHUNK)) for i, s in enumerate(range(0, n, _CHUNK))]
    if len(spans) <= 1:
        for sp in spans:
            fn(*sp)
        return
    with ThreadPoolExecutor(_THREADS) as ex:
        list(ex.map(lambda sp: fn(*sp), spans))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    u = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float32 values (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(rng: _Stream, shape, var: float) -> np.ndarray:
    """N(0, var) drawn in float32, stored as bfloat16 bits."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    std = np.float32(np.sqrt(var))

    def fill(i, s, e):
        v = rng.chunk(i).standard_normal(e - s, dtype=np.float32)
        v *= std
        out[s:e] = f32_to_bf16_bits(v)

    _fill_chunks(n, fill)
    return out.reshape(shape)


def normal_f32(rng: _Stream, shape, var: float) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    std = np.float32(np.sqrt(var))

    def fill(i, s, e):
        out[s:e] = rng.chunk(i).standard_normal(e - s, dtype=np.float32)
        out[s:e] *= std

    _fill_chunks(n, fill)
    return out.reshape(shape)


def draw_w(rng: _Stream, shape, dist) -> np.ndarray:
    kind, par = dist
    if kind == "uniform":
        n = int(np.prod(shape))
        out = np.empty(n, dtype=np.float32)

        def fill(i, s, e):
            out[s:e] = rng.chunk(i).uniform(0.0, par, size=e - s)

        _fill_chunks(n, fill)
        return out.reshape(shape)
    return normal_f32(rng, shape, par)


def make_inputs(wl: Workload, seed: int = 0, layers: bool = True) -> dict:
    """Draw every input of one layer group of workload ``wl``.

    Returns a dict:
      kv        uint16 [B, N_cached, D]  cached entries (all N unless raw tokens are given)
      c, z      uint16 / float32 [B, T_in, D] raw tokens to compress (if any; T_in includes the halo)
      bias      float32 [2m, D]
      index_k   uint16 [B, N, d]
      n_visible int32 [B, Q] or None
      layers    list of dicts: q_attn uint16 [B,Q,Ha,D]; Full/Reindex layers also
                q_index uint16 [B,Q,Hi,d] and w_index float32 [B,Q,Hi]
    """
    nm = wl.name
    out: dict = {}
    new_entries = wl.compress_new_tokens // wl.m
    n_cached = wl.N - new_entries
    out["kv"] = normal_bf16(_rng(seed, nm, 1), (wl.B, n_cached, wl.D), wl.var_kv)
    if wl.compress_new_tokens:
        t_in = wl.compress_new_tokens + (wl.m if wl.halo else 0)
        out["c"] = normal_bf16(_rng(seed, nm, 2), (wl.B, t_in, wl.D), 1.0)
        out["z"] = normal_f32(_rng(seed, nm, 3), (wl.B, t_in, wl.D), 1.0)
        out["bias"] = normal_f32(_rng(seed, nm, 4), (2 * wl.m, wl.D), wl.var_bias)
    out["index_k"] = normal_bf16(_rng(seed, nm, 5), (wl.B, wl.N, wl.d), wl.index_var)
    out["n_visible"] = n_visible(wl)
    if layers:
        out["layers"] = [make_layer_inputs(wl, i, seed) for i in range(wl.n_layers)]
    return out


def make_layer_inputs(wl: Workload, i: int, seed: int = 0) -> dict:
    nm = wl.name
    mode = wl.modes[i]
    L = {"q_attn": normal_bf16(_rng(seed, nm, 100 + 10 * i), (wl.B, wl.Q, wl.Ha, wl.D), wl.var_attn_q)}
    if wl.swa:       # this layer's own window rows: the last swa tokens, every query sees all of them
        L["win"] = normal_bf16(_rng(seed, nm, 103 + 10 * i), (wl.B, wl.swa, wl.D), wl.var_kv)
        L["win_end"] = np.full((wl.B, wl.Q), wl.swa, dtype=np.int32)
    if mode in (FULL, REINDEX):
        var = wl.index_var if mode == FULL else wl.reindex_var
        L["q_index"] = normal_bf16(_rng(seed, nm, 101 + 10 * i), (wl.B, wl.Q, wl.Hi, wl.d), var)
        L["w_index"] = draw_w(_rng(seed, nm, 102 + 10 * i), (wl.B, wl.Q, wl.Hi), wl.w_dist)
    return L
