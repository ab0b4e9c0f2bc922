"""csa2_select_topk_noalloc (library-owned static scratch) against
csa2_select_topk (caller workspace): the same selection bit for bit, on two
calls in a row, for every path the selection takes (one CTA per row, one CTA
per row of up to 32768 keys, several cooperating CTAs per row).  Named to be
collected last, so it also runs after every other test in the same process."""
import ctypes

import numpy as np
import pytest
import torch

import kv_cache_csa2_b200 as K

CAP = 4 << 20     # CSA2_SELECT_TOPK_NOALLOC_SCRATCH_BYTES


def _scores(seed, rows, L, ties):
    r = np.random.default_rng(seed)
    if ties:      # few distinct values: long runs of equal scores
        s = r.integers(0, 40, size=(rows, L)).astype(np.float32) * np.float32(0.25)
    else:
        s = r.standard_normal((rows, L)).astype(np.float32)
    s[:, ::97] = -np.inf                     # never selectable
    return torch.from_numpy(s).cuda()


def _pool_ids(seed, rows, L, N):
    r = np.random.default_rng(seed)
    ids = np.stack([np.sort(r.choice(N, L, replace=False)) for _ in range(rows)]).astype(np.int32)
    return torch.from_numpy(ids).cuda()


CASES = [
    # rows, L, count, ids: one-CTA-per-row kernel (no scratch), one CTA per
    # row (scratch, nothing cleared), cooperating CTAs (scratch, cleared)
    (5, 1000, 64, False),
    (8, 16384, 2048, True),
    (8, 262144, 2048, False),
    (3, 100000, 700, True),
]


@pytest.mark.gpu
@pytest.mark.parametrize("rows,L,count,with_ids", CASES)
def test_noalloc_matches_workspace_entry_point(rows, L, count, with_ids):
    assert K.lib().csa2_select_topk_workspace(rows, L, count) <= CAP
    for call, ties in enumerate((False, True)):           # two calls in a row, new data each
        scores = _scores(100 + call, rows, L, ties)
        ids = _pool_ids(7 + call, rows, L, 4 * L) if with_ids else None
        want = K.csa2_select_topk(scores, count, ids=ids)
        got = K.csa2_select_topk_noalloc(scores, count, ids=ids)
        again = K.csa2_select_topk_noalloc(scores, count, ids=ids)
        torch.cuda.synchronize()
        assert torch.equal(got, want)
        assert torch.equal(again, want)
    K.csa2_device_error()


def test_noalloc_rejects_oversize_on_host():
    """More rows than the static scratch holds: CSA2_ERR_OOM, nothing enqueued."""
    lib = K.lib()
    rows, L, count = 64, 262144, 2048
    need = lib.csa2_select_topk_workspace(rows, L, count)
    assert need > CAP
    p = ctypes.c_void_p(256)
    st = lib.csa2_select_topk_noalloc(p, rows, L, count, None, p, None)
    assert st == 6
    msg = lib.csa2_last_error().decode()
    assert str(need) in msg and str(CAP) in msg
    # empty work needs no scratch
    assert lib.csa2_select_topk_noalloc(None, 0, L, count, None, None, None) == 0
