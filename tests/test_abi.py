"""The C-ABI library loads without a GPU, exports every symbol its header
declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

from persistent_sm_attn_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "dash_attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dash_\w+)\s*\(", src)))


def test_header_symbols_exported(lib):
    names = _declared()
    assert len(names) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (dash_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    assert set(binding.EXPORTS) == set(names)


def test_status_strings(lib):
    for code, name in binding.STATUS.items():
        assert binding.dash_status_string(code) == name
    assert binding.dash_status_string(99) == "DASH_ERR_UNKNOWN"


def _bwd(lib, ptrs, B=1, H=1, S=128, D=64, causal=0, sched=2):
    return lib.dash_attn_bwd(*ptrs, B, H, S, D, causal, sched, None)


def test_argument_errors_need_no_gpu(lib):
    buf = ctypes.create_string_buffer(64)
    al = (ctypes.addressof(buf) + 15) // 16 * 16
    good = [ctypes.c_void_p(al)] * 9
    null = [ctypes.c_void_p(0)] + good[1:]
    mis = [ctypes.c_void_p(al + 2)] + good[1:]
    assert _bwd(lib, null) == 1                       # null pointer
    assert _bwd(lib, mis) == 1                        # misaligned
    assert _bwd(lib, good, D=96) == 2                 # head dim not provided
    assert _bwd(lib, good, S=200) == 2                # S not a multiple of 128
    assert _bwd(lib, good, S=0) == 2
    assert _bwd(lib, good, B=-1) == 1
    assert _bwd(lib, good, sched=9) == 1              # unknown schedule
    assert _bwd(lib, good, causal=1, sched=2) == 2    # shift needs a full mask
    assert _bwd(lib, good, causal=0, sched=3) == 2    # symmetric shift needs causal
    assert _bwd(lib, good, S=384, causal=1, sched=3) == 2   # odd tile count
    assert _bwd(lib, good, causal=2) == 1
    assert lib.dash_attn_fwd(*good[:5], 1, 1, 128, 80, 0, None) == 2
    assert lib.dash_sched_simulate(1, 4, 0, 2, 4, -1.0, 0.0, 0, 1, None, None, None, None) == 1
    assert lib.dash_sched_simulate(1, 4, 0, 2, 4, 1.0, 0.0, 0, 0, None, None, None, None) == 1
    assert lib.dash_sched_check(1, 4, 2, 4, None, 0) == 1
    # host-buffer path: null host pointers and bad shapes fail before any copy
    assert lib.dash_attn_bwd_host(*null, 1, 1, 128, 64, 0, 2, None) == 1
    assert lib.dash_attn_bwd_host(*good, 1, 1, 128, 96, 0, 2, None) == 2
    assert lib.dash_attn_bwd_host(*good, 1, 1, 128, 64, 1, 2, None) == 2
    # grouped-query entries: Hkv must divide H, with a power-of-two group
    gqa_b = lambda H, Hkv, S=128, D=64: lib.dash_attn_bwd_gqa(*good, 1, H, Hkv, S, D, 0, 2, None)
    gqa_f = lambda H, Hkv: lib.dash_attn_fwd_gqa(*good[:5], 1, H, Hkv, 128, 64, 0, None)
    for fn in (gqa_b, gqa_f):
        assert fn(4, 3) == 1                          # 3 does not divide 4
        assert fn(4, 0) == 1
        assert fn(4, -2) == 1
        assert fn(6, 2) == 2                          # 3 query heads per K/V head
        assert fn(12, 1) == 2
    assert gqa_b(8, 2, D=96) == 2
    assert lib.dash_attn_bwd_gqa(*null, 1, 8, 2, 128, 64, 0, 2, None) == 1
    # a part outside the table's heads
    for h0, h1 in ((0, 0), (2, 1), (-1, 1), (0, 5)):
        assert lib.dash_sched_table_part(4, 4, 0, 2, 8, h0, h1, None, 0) == -1


def test_dag_cycle_rejected():
    with pytest.raises(binding.DashError):
        binding.dash_dag_longest_path(2, [(0, 1, 1.0), (1, 0, 1.0)])


def test_empty_batches_are_no_ops_without_a_device(lib):
    """B = 0 or H = 0: nothing to compute, so every entry point returns DASH_OK after
    its argument checks and before any CUDA call (none can succeed on this host)."""
    buf = ctypes.create_string_buffer(64)
    al = (ctypes.addressof(buf) + 15) // 16 * 16
    good = [ctypes.c_void_p(al)] * 9
    for B, H in ((0, 4), (2, 0)):
        assert _bwd(lib, good, B=B, H=H) == 0
        assert lib.dash_attn_fwd(*good[:5], B, H, 128, 64, 0, None) == 0
        assert lib.dash_attn_bwd_gqa(*good, B, H, 1, 128, 64, 0, 2, None) == 0
        assert lib.dash_attn_fwd_gqa(*good[:5], B, H, 1, 128, 64, 0, None) == 0
        assert lib.dash_attn_bwd_host(*good, B, H, 256, 64, 1, 3, None) == 0
        assert lib.dash_attn_bwd_noalloc(*good, B, H, 256, 128, 1, 1, None) == 0
    # argument errors still come first
    assert _bwd(lib, good, B=0, D=96) == 2
    assert _bwd(lib, good, B=0, sched=9) == 1
