"""The allocation-free entry point, externd_factor_noalloc.

Some callers cannot let the library allocate device memory during a call: a
conversion or inference service whose memory pool already reserved the GPU, or
a caller that cannot take the device synchronisation an allocation may cause.
For them the library keeps its scratch in one static device array and this
entry point allocates nothing.  Here it must give the same factors as the
allocating entry point (same kernels, same partition, fixed-order reductions:
identical bits, which is within every tolerance of the parity tests), on two
calls in a row -- the second call reuses the scratch left by the first.
This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import ternary_rank_weight_b200 as ext
from ternary_rank_weight_b200.workloads import llm_matrix

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m,n,block", [(384, 512, 256), (64, 14000, 512), (80, 22000, 1024)])
def test_noalloc_matches_the_allocating_entry_point_on_two_calls(m, n, block):
    """One shape per build of the ALS machinery (256, 512 and 1024 threads per CTA, chosen by the
    work of one CTA): the allocation-free call hands its static array to the build the plan picks."""
    A = torch.from_numpy(llm_matrix(m, n, seed=7)).cuda()
    ref = ext.factor(A, 1.5, 0.7, iters=15, seed=3)
    assert ref.stats["block"] == block
    for call in range(2):
        out = (torch.full_like(ref.B, 0xAA), torch.full_like(ref.D, float("nan")),
               torch.full_like(ref.C, 0x55), torch.full_like(ref.energy, float("nan")))
        f = ext.factor_noalloc(A, 1.5, 0.7, iters=15, seed=3, out=out)
        torch.cuda.synchronize()
        assert torch.equal(f.B, ref.B), call
        assert torch.equal(f.C, ref.C), call
        assert torch.equal(f.D, ref.D), call
        assert torch.equal(f.energy, ref.energy), call
        # and therefore within the end-to-end parity tolerances
        assert abs(f.energy[-1].item() - ref.energy[-1].item()) < 2e-3


def test_noalloc_rejects_what_it_cannot_do_without_memory():
    big = torch.zeros((2048, 4096), device="cuda")      # 16 m n = 128 MiB of residual copies > scratch
    big[0, 0] = 1.0
    with pytest.raises(ext.ExterndError) as e:
        ext.factor_noalloc(big, 1.0, 0.7)
    assert e.value.status == ext.STATUS["ELIMIT"]
    # host buffers would need staging memory
    import ctypes
    from ternary_rank_weight_b200 import _lib
    host = np.ones((8, 8), dtype=np.float32)
    k = ext.rank(8, 8, 1.0)
    B = torch.empty((k, ext.trit_bytes(8)), dtype=torch.uint8, device="cuda")
    C = torch.empty_like(B)
    D = torch.empty((k,), device="cuda")
    rc = _lib.load().externd_factor_noalloc(host.ctypes.data, 8, 8, 1.0, 0.7, 15, 0, B.data_ptr(), D.data_ptr(),
                                            C.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
    assert rc == ext.STATUS["EINVAL"]


def test_noalloc_refuses_a_copy_and_leaves_the_stats_alone():
    A = torch.from_numpy(llm_matrix(128, 96, seed=9)).cuda()
    ref = ext.factor(A, 1.0, 0.7, seed=1)
    before = ext.last_stats()
    f = ext.factor_noalloc(A, 1.0, 0.7, seed=1)
    assert torch.equal(f.B, ref.B) and torch.equal(f.D, ref.D)
    assert ext.last_stats() == before          # this entry point records no figures
    with pytest.raises(ValueError):
        ext.factor_noalloc(A.t(), 1.0, 0.7)    # non-contiguous: would need a copy
