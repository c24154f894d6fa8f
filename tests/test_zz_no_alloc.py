"""The backward entry point that allocates no device memory.

dash_attn_bwd_noalloc exists for callers that cannot call cudaMalloc (code
running while a stream is captured into a CUDA graph, runtimes that serve all
device memory from their own pool, embedded users with a fixed device
footprint).  It takes all scratch from one static device array, so its
results must match the allocating entry point's, also when called twice in a
row on an array that still holds the previous call's contents.

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


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,S,D,causal,schedule", [
    (1, 2, 256, 64, False, "shift"),
    (2, 3, 512, 128, True, "sym_shift"),
    (1, 4, 384, 64, True, "descending"),
])
def test_noalloc_matches_allocating_entry_point(B, H, S, D, causal, schedule):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    q, k, v, do = draw(B, H, S, D, 1.0, seed=77 + S + D, device="cuda")
    o, lse = binding.dash_attn_fwd(q, k, v, causal)
    ref = binding.dash_attn_bwd(q, k, v, o, do, lse, causal, schedule)
    assert binding.dash_attn_sync_status() == 0
    ref = [t.float().cpu().numpy() for t in ref]
    for call in range(2):  # the second call reuses an array holding the first call's data
        outs = [torch.full_like(q, float("nan")) for _ in range(3)]
        binding.dash_attn_bwd_noalloc(q, k, v, o, do, lse, causal, schedule, *outs)
        torch.cuda.synchronize()
        for got, want in zip(outs, ref):
            g = got.float().cpu().numpy()
            assert np.isfinite(g).all(), call
            assert A.rel_fro(g, want) <= TOL, call


def test_noalloc_rejects_sizes_beyond_its_array():
    """A call whose scratch would not fit is refused before the device is touched."""
    lib = binding.load()
    buf = ctypes.create_string_buffer(64)
    al = ctypes.c_void_p((ctypes.addressof(buf) + 15) // 16 * 16)
    # 64 heads x 16384 rows x 128 columns of fp32 accumulator = 512 MiB > 64 MiB
    rc = lib.dash_attn_bwd_noalloc(*([al] * 9), 4, 16, 16384, 128, 0, 2, None)
    assert rc == 5  # DASH_ERR_OOM
