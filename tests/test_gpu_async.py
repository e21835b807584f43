"""Asynchronous calls (externd_options.async_status / externd_batch_options.async_status).

The call queues its work on the stream and returns at once.  The caller's device int
receives the status when the stream reaches the end of the work.  The factors must equal
those of the synchronous call bit for bit, and a device-side timeout must arrive as the
status rather than as a return code.  Host buffers are refused before anything is queued.
"""
import ctypes

import numpy as np
import pytest
import torch

import ternary_rank_weight_b200 as ext
from ternary_rank_weight_b200 import _lib
from ternary_rank_weight_b200.workloads import llm_matrix

pytestmark = pytest.mark.gpu


def _status():
    return torch.full((1,), 12345, dtype=torch.int32, device="cuda")


def test_async_factor_equals_the_synchronous_call():
    A = torch.from_numpy(llm_matrix(300, 517, seed=5)).cuda()
    ref = ext.factor(A, 1.5, 0.7, seed=3, want_d64=True)
    st = _status()
    f = ext.factor(A, 1.5, 0.7, seed=3, want_d64=True, async_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(f.B, ref.B) and torch.equal(f.C, ref.C) and torch.equal(f.D, ref.D)
    assert torch.equal(f.d64, ref.d64) and torch.equal(f.energy, ref.energy)


def test_async_calls_queue_back_to_back_on_one_stream():
    """Three factorizations queued without waiting, then one synchronisation."""
    mats = [torch.from_numpy(llm_matrix(128, 192, seed=s)).cuda() for s in range(3)]
    refs = [ext.factor(A, 1.0, 1.0, seed=s) for s, A in enumerate(mats)]
    sts = [_status() for _ in mats]
    outs = [ext.factor(A, 1.0, 1.0, seed=s, async_status=st) for s, (A, st) in enumerate(zip(mats, sts))]
    torch.cuda.synchronize()
    for f, r, st in zip(outs, refs, sts):
        assert st.item() == 0
        assert torch.equal(f.B, r.B) and torch.equal(f.C, r.C) and torch.equal(f.D, r.D)


def test_async_batched_equals_the_synchronous_batch():
    mats = [torch.from_numpy(llm_matrix(96, 160, seed=10 + s)).cuda() for s in range(4)]
    mus, taus = [1.0, 2.0, 1.5, 1.0], [0.7, 1.0, 2.0, 0.7]
    ref, rst = ext.factor_batched(mats, mus, taus, seeds=[1, 2, 3, 4])
    assert rst == [0] * 4
    st = _status()
    res, _ = ext.factor_batched(mats, mus, taus, seeds=[1, 2, 3, 4], async_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    for a, b in zip(res, ref):
        assert torch.equal(a.B, b.B) and torch.equal(a.C, b.C) and torch.equal(a.D, b.D)


def test_async_timeout_arrives_as_the_status():
    """A CTA that never signals (the host-set test flag): the bounded waits run out and the
    status, not the return code, carries EXTERND_ETIMEOUT; the next call succeeds."""
    A = torch.from_numpy(llm_matrix(256, 256, seed=3)).cuda()
    st = _status()
    ext.factor(A, 1.0, 0.7, grid=4, fault_skip_cta=2, wait_limit_s=0.2, async_status=st)
    torch.cuda.synchronize()
    assert st.item() == ext.STATUS["ETIMEOUT"]
    f = ext.factor(A, 1.0, 0.7, grid=4)
    assert f.energy[-1].item() > 0.5


def test_async_refuses_host_buffers():
    """Host input or output buffers would need a synchronous copy: EINVAL, nothing queued."""
    A = np.ascontiguousarray(llm_matrix(64, 64, seed=1), dtype=np.float32)
    k = ext.rank(64, 64, 1.0)
    B = np.zeros((k, ext.trit_bytes(64)), dtype=np.uint8)
    C = np.zeros((k, ext.trit_bytes(64)), dtype=np.uint8)
    D = np.zeros(k, dtype=np.float32)
    st = _status()
    opt = _lib.Options()
    opt.async_status = st.data_ptr()
    rc = _lib.load().externd_factor_ex(A.ctypes.data, 64, 64, 1.0, 0.7, 15, 0, B.ctypes.data, D.ctypes.data,
                                       C.ctypes.data, None, None, ctypes.byref(opt))
    assert rc == ext.STATUS["EINVAL"]
    assert st.item() == 12345
    with pytest.raises(ValueError):
        ext.factor(torch.from_numpy(A), 1.0, 0.7, async_status=st)
