"""Bounded device waits end in an error status, not a hang or a fault.

The cross-CTA waits (the multi-CTA top-k's row barrier, the attention
kernel's wait for another tile's partial) are pointed, through
csa2_set_device_wait, at a count that no CTA ever writes, with a 1 ms bound.
Each wait must run out, the kernel must finish, csa2_device_error must report
CSA2_ERR_TIMEOUT, and the next normal call in the same process must give the
oracle's result with no error recorded."""
import numpy as np
import pytest

import kv_cache_csa2_b200 as K
import oracle as O
from kv_cache_csa2_b200 import inputs as I
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

TIMEOUT = 5
LIMIT_NS = 1_000_000


@pytest.fixture(autouse=True)
def _restore_wait():
    yield
    K.set_device_wait(0, False)


def _expect_timeout():
    with pytest.raises(K.CSA2Error) as e:
        K.csa2_device_error()
    assert e.value.status == TIMEOUT


def test_topk_row_barrier_runs_out_then_recovers():
    r = np.random.default_rng(31)
    rows, L, count = 4, 300000, 2048           # 37 cooperating CTAs per row
    s = r.standard_normal((rows, L)).astype(np.float32)
    ds = U.dev(s)
    want = O.select_top(s.astype(np.float64), count)
    K.csa2_device_error()
    K.set_device_wait(LIMIT_NS, True)
    K.csa2_select_topk(ds, count)
    _expect_timeout()
    K.set_device_wait(0, False)
    got = K.csa2_select_topk(ds, count).cpu().numpy()
    K.csa2_device_error()
    assert np.array_equal(got, want)


def test_attention_partial_wait_runs_out_then_recovers():
    r = np.random.default_rng(32)
    B, Q, Ha, D, N, k = 2, 3, 64, 512, 5000, 2048   # 16 tiles per query on the tensor-core kernel
    q = I.f32_to_bf16_bits(r.standard_normal((B, Q, Ha, D)).astype(np.float32))
    kv = I.f32_to_bf16_bits(r.standard_normal((B, N, D)).astype(np.float32))
    topk = np.stack([np.stack([np.sort(r.choice(N, k, replace=False)) for _ in range(Q)])
                     for _ in range(B)]).astype(np.int32)
    args = (U.dev_bf16(q), U.dev_bf16(kv), U.dev(topk), D ** -0.5)
    K.csa2_device_error()
    K.set_device_wait(LIMIT_NS, True)
    K.csa2_sparse_attn(*args)
    _expect_timeout()
    K.set_device_wait(0, False)
    out, lse = K.csa2_sparse_attn(*args)
    K.csa2_device_error()
    o, _, l = O.sparse_attn(O.bf16_bits_to_float(q), O.bf16_bits_to_float(kv), topk, D ** -0.5)
    U.check_attn(U.host_bf16(out), lse.cpu().numpy().astype(np.float64), o, l, "after a timeout")
