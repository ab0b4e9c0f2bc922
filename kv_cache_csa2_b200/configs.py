"""The five CSA2 workloads (shapes, layer modes, input distributions).

Host-side description only: no arithmetic of the method lives here.  Names
follow the pages' notation: B sequences, Q query tokens per sequence, L
context tokens, m tokens per compressed block, N = L // m entries, D main-KV
width, Ha attention heads, Hi / d indexer heads and width, k selected entries,
P hierarchical-indexer pool size.

Distribution notation: ``N(0, v)`` gives the *variance* v (so q, k of the
indexer at width d are drawn with variance 1/d).
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field

FULL, REINDEX, REUSE = "full", "reindex", "reuse"


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Q: int
    L: int
    m: int
    D: int
    Ha: int
    Hi: int
    d: int
    k: int
    P: int = 0                       # 0: no hierarchical pool
    modes: tuple = (FULL,)
    kv_fp4: bool = False
    scale: float = 0.0               # 0: 1/sqrt(D)
    compress_new_tokens: int = 0     # >0: the newest tokens are given raw (c_t, z_t) and compressed
    halo: bool = False               # the raw chunk carries the m tokens before it
    q_pos0: int = -1                 # >=0: causal prefill, query i sits at absolute position q_pos0 + i
    # input distributions: (kind, parameter) with kind "normal" (variance) or "uniform" (upper bound)
    var_index_qk: float = 0.0        # 0: 1/d
    var_reindex_q: float = 0.0       # 0: same as the Full layer's
    w_dist: tuple = ("uniform", 1.0)
    var_bias: float = 0.1
    var_attn_q: float = 1.0
    var_kv: float = 1.0
    swa: int = 0                     # >0: every layer also attends its own window of this many uncompressed rows

    @property
    def N(self) -> int:
        return self.L // self.m

    @property
    def attn_scale(self) -> float:
        return self.scale if self.scale > 0 else 1.0 / math.sqrt(self.D)

    @property
    def index_var(self) -> float:
        return self.var_index_qk if self.var_index_qk > 0 else 1.0 / self.d

    @property
    def reindex_var(self) -> float:
        return self.var_reindex_q if self.var_reindex_q > 0 else self.index_var

    @property
    def n_layers(self) -> int:
        return len(self.modes)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# C1: single Full layer, decode, batch 1, KV compressed from raw tokens.
C1 = Workload(name="c1_full_decode_8k", B=1, Q=1, L=8192, m=4, D=128, Ha=16, Hi=8, d=64,
              k=256, modes=(FULL,), compress_new_tokens=8192, var_bias=0.1)

# C2: decode group F + 5U, batch 32, 64K context, 512-wide bf16 KV.
C2 = Workload(name="c2_decode_f5u_64k", B=32, Q=1, L=65536, m=4, D=512, Ha=64, Hi=64, d=128,
              k=2048, modes=(FULL,) + (REUSE,) * 5)

# C3: FP4 main KV, shapes of C1, batch 64, 128K context, F + Ri + 4U.
C3 = Workload(name="c3_fp4_decode_f_ri_4u_128k", B=64, Q=1, L=131072, m=4, D=128, Ha=16, Hi=8,
              d=64, k=256, modes=(FULL, REINDEX) + (REUSE,) * 4, kv_fp4=True)

# C4: hierarchical indexer at 1M context, batch 8: F (pool 16384) + 3 Ri + 4 U.
C4 = Workload(name="c4_hier_decode_f_3ri_4u_1m", B=8, Q=1, L=1048576, m=4, D=512, Ha=64, Hi=64,
              d=128, k=2048, P=16384, modes=(FULL,) + (REINDEX,) * 3 + (REUSE,) * 4,
              var_reindex_q=1.0)

# C5: causal prefill chunk of 4096 tokens at the end of a 1M context, F + 5U.
C5 = Workload(name="c5_prefill_4096_at_1m", B=1, Q=4096, L=1048576, m=4, D=512, Ha=64, Hi=64,
              d=128, k=2048, modes=(FULL,) + (REUSE,) * 5, compress_new_tokens=4096, halo=True,
              q_pos0=1048576 - 4096, var_index_qk=1.0, w_dist=("normal", 1.0), var_bias=1.0)

# C6: C4 with the sliding-window branch the V4.1 layer layout gives every
# layer: 128 uncompressed rows per layer and sequence, N(0,1) (not one of the
# five benchmark workloads: the measurement of that branch at C4's scale).
C6 = C4.replace(name="c6_hier_decode_swa128_1m", swa=128)

CONFIGS = {1: C1, 2: C2, 3: C3, 4: C4, 5: C5, 6: C6}


def n_visible(wl: Workload):
    """Entries each query may see (None = all N).  A query at absolute
    position p sees the entries whose blocks are complete: j < (p + 1) // m."""
    if wl.q_pos0 < 0:
        return None
    import numpy as np
    pos = wl.q_pos0 + np.arange(wl.Q, dtype=np.int64)
    nv = np.minimum((pos + 1) // wl.m, wl.N).astype(np.int32)
    return np.broadcast_to(nv, (wl.B, wl.Q)).copy()
