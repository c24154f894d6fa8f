"""The backward entry point that allocates no device memory.

dash_attn_bwd_noalloc exists for callers that cannot call cudaMalloc:
runtimes that serve all device memory from their own pool and forbid other
allocations, and embedded or certified deployments whose device footprint is
fixed before they start.  It takes all scratch from one static device array,
so on a deterministic schedule its results must equal the allocating entry
point's bit for bit, also when called twice in a row on an array that still
holds the previous call's contents; the atomic variant must agree within the
parity bound.  A device-side timeout must be visible through
dash_attn_noalloc_sync_status.

This file is collected last so that a run stopping at its first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import attention as A
from persistent_sm_attn_b200 import binding
from persistent_sm_attn_b200.inputs import draw

TOL = 5e-3  # the relative Frobenius bound used by every parity test


def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,S,D,causal,schedule", [
    (1, 2, 256, 64, False, "shift"),
    (2, 3, 512, 128, True, "sym_shift"),
    (1, 4, 384, 64, True, "descending"),
    (1, 2, 512, 128, False, "atomic"),
])
def test_noalloc_matches_allocating_entry_point(B, H, S, D, causal, schedule):
    _need_cuda()
    q, k, v, do = draw(B, H, S, D, 1.0, seed=77 + S + D, device="cuda")
    o, lse = binding.dash_attn_fwd(q, k, v, causal)
    ref = binding.dash_attn_bwd(q, k, v, o, do, lse, causal, schedule)
    assert binding.dash_attn_sync_status() == 0
    for call in range(2):  # the second call reuses an array holding the first call's data
        outs = [torch.full_like(q, float("nan")) for _ in range(3)]
        binding.dash_attn_bwd_noalloc(q, k, v, o, do, lse, causal, schedule, *outs)
        assert binding.dash_attn_noalloc_sync_status() == 0, call
        for got, want in zip(outs, ref):
            if schedule == "atomic":
                # nondeterministic: the order of its additions differs from run to run
                g = got.float().cpu().numpy()
                assert np.isfinite(g).all(), call
                assert A.rel_fro(g, want.float().cpu().numpy()) <= TOL, call
            else:
                assert torch.equal(got, want), (schedule, call)


@pytest.mark.gpu
def test_noalloc_timeout_is_reported_then_recovers():
    """A schedule table whose first dQ contributors never arrive (planted on
    the host) makes the ticket waits run out after a 2 ms limit; the status
    call reports it once, and the next call is correct again."""
    _need_cuda()
    B, H, S, D, causal, sched = 1, 2, 512, 64, False, "shift"
    q, k, v, do = draw(B, H, S, D, 1.0, seed=91, device="cuda")
    o, lse = binding.dash_attn_fwd(q, k, v, causal)
    ref = binding.dash_attn_bwd(q, k, v, o, do, lse, causal, sched)
    assert binding.dash_attn_sync_status() == 0
    outs = [torch.empty_like(q) for _ in range(3)]
    binding.dash_set_spin_limit_us(2000)  # 2 ms
    try:
        binding.dash_inject_fault(1)
        binding.dash_attn_bwd_noalloc(q, k, v, o, do, lse, causal, sched, *outs)
        assert binding.dash_attn_noalloc_sync_status() == 4  # DASH_ERR_TIMEOUT
        assert binding.dash_attn_noalloc_sync_status() == 0  # read and cleared
    finally:
        binding.dash_inject_fault(0)
        binding.dash_set_spin_limit_us(0)
    binding.dash_attn_bwd_noalloc(q, k, v, o, do, lse, causal, sched, *outs)
    assert binding.dash_attn_noalloc_sync_status() == 0
    for got, want in zip(outs, ref):
        assert torch.equal(got, want)


def test_noalloc_rejects_sizes_beyond_its_array():
    """A call whose scratch would not fit is refused before the device is touched."""
    lib = binding.load()
    buf = ctypes.create_string_buffer(64)
    al = ctypes.c_void_p((ctypes.addressof(buf) + 15) // 16 * 16)
    # 2 fp32 accumulators x 64 heads x 16384 rows x 128 columns = 1 GiB > 64 MiB
    rc = lib.dash_attn_bwd_noalloc(*([al] * 9), 4, 16, 16384, 128, 0, 2, None)
    assert rc == 5  # DASH_ERR_OOM
