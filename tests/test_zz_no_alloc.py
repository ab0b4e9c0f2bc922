"""csa2_select_topk_noalloc keeps its scratch in a static device array inside
the library, for callers that cannot allocate device memory (for example code
that runs while an allocator is locked, or a host runtime that hands the
library no workspace).  Checked here against csa2_select_topk (caller
workspace) and against the oracle's selection, on two calls in a row with new
data each time, for every path the selection takes:

  - an 8-CTA cluster per row and one CTA per row: no scratch at all;
  - several cooperating CTAs per row (rows longer than 262144 keys, or the
    cluster kernel switched off): the static scratch, whose counters are
    cleared before every launch.

Named to be collected last, so that it also runs after every other test in
the same process; it needs nothing from them."""
import ctypes

import numpy as np
import pytest
import torch

import kv_cache_csa2_b200 as K
import oracle as O

CAP = 4 << 20     # CSA2_SELECT_TOPK_NOALLOC_SCRATCH_BYTES


def _scores(seed, rows, L, ties):
    r = np.random.default_rng(seed)
    if ties:      # few distinct values: long runs of equal scores
        s = r.integers(0, 40, size=(rows, L)).astype(np.float32) * np.float32(0.25)
    else:
        s = r.standard_normal((rows, L)).astype(np.float32)
    s[:, ::97] = -np.inf                     # never selectable
    return s


def _pool_ids(seed, rows, L, N):
    r = np.random.default_rng(seed)
    ids = np.stack([np.sort(r.choice(N, L, replace=False)) for _ in range(rows)]).astype(np.int32)
    return ids


def _oracle(s, count, ids):
    pos = O.select_top(s.astype(np.float64), count)
    if ids is None:
        return pos
    return np.where(pos >= 0, np.take_along_axis(ids, np.maximum(pos, 0), 1), -1)


CASES = [
    # rows, L, count, ids, environment, uses scratch
    (5, 1000, 64, False, {}, False),                                     # cluster of 8 CTAs
    (64, 262144, 2048, False, {}, False),                                # cluster: rows < SMs
    (200, 3000, 100, True, {}, False),                                   # one CTA per row
    (5, 300000, 2048, False, {}, True),                                  # cooperating CTAs (37 per row)
    (20, 400000, 5000, True, {}, True),                                  # 49 per row, 20 rows
    (8, 100000, 2048, False, {"CSA2_TOPK_NO_CLUSTER": "1"}, True),       # 13 per row
]


@pytest.mark.gpu
@pytest.mark.parametrize("rows,L,count,with_ids,env,scratch", CASES)
def test_noalloc_matches_workspace_entry_point_and_oracle(rows, L, count, with_ids, env, scratch,
                                                          monkeypatch):
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    lib = K.lib()
    ws = lib.csa2_select_topk_workspace(rows, L, count)
    if scratch:   # the cooperative kernel runs on the static array
        assert 0 < ws <= CAP
    for call, ties in enumerate((False, True)):           # two calls in a row, new data each
        s = _scores(100 + call, rows, L, ties)
        ids = _pool_ids(7 + call, rows, L, 4 * L) if with_ids else None
        ds = torch.from_numpy(s).cuda()
        di = torch.from_numpy(ids).cuda() if ids is not None else None
        want = K.csa2_select_topk(ds, count, ids=di)
        got = K.csa2_select_topk_noalloc(ds, count, ids=di)
        again = K.csa2_select_topk_noalloc(ds, count, ids=di)
        torch.cuda.synchronize()
        assert torch.equal(got, want)
        assert torch.equal(again, want)
        assert np.array_equal(got.cpu().numpy(), _oracle(s, count, ids))
    K.csa2_device_error()


def test_noalloc_rejects_oversize_on_host():
    """A cooperative selection whose scratch exceeds the static array:
    CSA2_ERR_OOM with nothing enqueued (26 rows of 400000 keys need about
    4.3 MiB; 25 rows is the most the array holds on that path)."""
    lib = K.lib()
    rows, L, count = 26, 400000, 2048
    need = lib.csa2_select_topk_workspace(rows, L, count)
    assert need > CAP
    p = ctypes.c_void_p(256)
    st = lib.csa2_select_topk_noalloc(p, rows, L, count, None, p, None)
    assert st == 6
    msg = lib.csa2_last_error().decode()
    assert str(need) in msg and str(CAP) in msg
    assert lib.csa2_select_topk_workspace(25, L, count) <= CAP
    # empty work needs no scratch
    assert lib.csa2_select_topk_noalloc(None, 0, L, count, None, None, None) == 0
