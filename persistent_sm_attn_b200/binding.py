"""ctypes binding of libdash_attn.so (argument marshalling only).

Every step of the backward runs in the library's CUDA kernels; this module
turns torch tensors into pointers and a stream handle, and raises
``DashError`` on a non-zero status.  It never falls back to another
implementation: if the library is missing or fails to load, ``load()``
raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdash_attn.so")

SCHEDULES = {"naive_asc": 0, "descending": 1, "shift": 2, "sym_shift": 3, "atomic": 4,
             "shift_pairs": 5, "sym_shift_pairs": 6}
STATUS = {0: "DASH_OK", 1: "DASH_ERR_INVALID_ARG", 2: "DASH_ERR_UNSUPPORTED", 3: "DASH_ERR_CUDA",
          4: "DASH_ERR_TIMEOUT", 5: "DASH_ERR_OOM", 6: "DASH_ERR_SCHEDULE"}

EXPORTS = ("dash_attn_fwd", "dash_attn_bwd", "dash_attn_sync_status", "dash_status_string",
           "dash_set_spin_limit_us", "dash_bwd_num_ctas", "dash_release_workspace",
           "dash_sched_table", "dash_sched_simulate", "dash_sched_simulate_gqa",
           "dash_dag_longest_path",
           "dash_profile_begin", "dash_profile_end", "dash_attn_bwd_noalloc",
           "dash_trace_bwd", "dash_inject_fault", "dash_sched_check", "dash_attn_bwd_host",
           "dash_sched_table_part", "dash_attn_fwd_gqa", "dash_attn_bwd_gqa",
           "dash_sched_table_gqa", "dash_attn_noalloc_sync_status",
           "dash_attn_bwd_gqa_split", "dash_bwd_gqa_split_for", "dash_set_dq_chain_mode",
           "dash_dq_chain_uses_red", "dash_set_head_interleave",
           "dash_bwd_head_interleave", "dash_set_slot_placement",
           "dash_slot_placement_by_smid", "dash_sched_table_pairs")


class DashError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


_lib = None


def load(path: str | None = None):
    """Load (building first if absent or stale) the shared library."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    if path is None:
        from . import build as _build
        try:
            _build.build()
        except Exception as e:  # no compiler on this machine: use what is there
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"libdash_attn.so is missing and could not be built: {e}")
        path = LIB_PATH
    lib = ctypes.CDLL(path)
    vp, i, ll, d = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_double
    P = ctypes.POINTER
    lib.dash_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, vp]
    lib.dash_attn_bwd.argtypes = [vp] * 9 + [i, i, i, i, i, i, vp]
    lib.dash_attn_bwd_noalloc.argtypes = [vp] * 9 + [i, i, i, i, i, i, vp]
    lib.dash_attn_bwd_host.argtypes = [vp] * 9 + [i, i, i, i, i, i, vp]
    lib.dash_attn_fwd_gqa.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
    lib.dash_attn_bwd_gqa.argtypes = [vp] * 9 + [i, i, i, i, i, i, i, vp]
    lib.dash_attn_bwd_gqa_split.argtypes = [vp] * 9 + [i, i, i, i, i, i, i, i, vp]
    lib.dash_bwd_gqa_split_for.argtypes = [i, i, i, i, i, i, i, P(i)]
    lib.dash_set_dq_chain_mode.argtypes = [i]
    lib.dash_dq_chain_uses_red.argtypes = [i, i, i, i, P(i)]
    lib.dash_set_head_interleave.argtypes = [i]
    lib.dash_set_slot_placement.argtypes = [i]
    lib.dash_slot_placement_by_smid.argtypes = [i, P(i)]
    lib.dash_bwd_head_interleave.argtypes = [i, i, i, i, i, i, P(i)]
    lib.dash_attn_sync_status.argtypes = [vp]
    lib.dash_attn_noalloc_sync_status.argtypes = [vp]
    lib.dash_status_string.argtypes = [i]
    lib.dash_status_string.restype = ctypes.c_char_p
    lib.dash_set_spin_limit_us.argtypes = [ll]
    lib.dash_inject_fault.argtypes = [i]
    lib.dash_bwd_num_ctas.argtypes = [i, i, P(i)]
    lib.dash_release_workspace.argtypes = []
    lib.dash_sched_table.argtypes = [i, i, i, i, i, vp, ll]
    lib.dash_sched_table.restype = ll
    lib.dash_sched_table_part.argtypes = [i, i, i, i, i, i, i, vp, ll]
    lib.dash_sched_table_part.restype = ll
    lib.dash_sched_table_gqa.argtypes = [i, i, i, i, i, i, vp, ll]
    lib.dash_sched_table_gqa.restype = ll
    lib.dash_sched_table_pairs.argtypes = [i, i, i, i, vp, ll]
    lib.dash_sched_table_pairs.restype = ll
    lib.dash_sched_simulate.argtypes = [i, i, i, i, i, d, d, i, i, P(d), P(d), P(d), P(ll)]
    lib.dash_sched_simulate_gqa.argtypes = [i, i, i, i, i, i, d, d, i, i, P(d), P(d), P(d),
                                            P(ll)]
    lib.dash_sched_check.argtypes = [i, i, i, i, vp, ll]
    lib.dash_dag_longest_path.argtypes = [i, i, vp, vp, vp, vp, vp, P(d)]
    lib.dash_trace_bwd.argtypes = [vp] * 9 + [i, i, i, i, i, i, vp, vp, ll, P(i), P(i)]
    lib.dash_profile_begin.argtypes = []
    lib.dash_profile_end.argtypes = [P(d), P(d), P(ll)]
    for name in EXPORTS:
        if name not in ("dash_status_string", "dash_sched_table", "dash_sched_table_part",
                        "dash_sched_table_gqa", "dash_attn_noalloc_sync_status",
                        "dash_sched_table_pairs"):
            getattr(lib, name).restype = ctypes.c_int
    if path == LIB_PATH:
        _lib = lib
    return lib


def _check(rc: int, what: str):
    if rc != 0:
        raise DashError(rc, what)


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _sched_id(schedule) -> int:
    return SCHEDULES[schedule] if isinstance(schedule, str) else int(schedule)


def _check_tensors(q, k, v, o=None, do=None, lse=None, outs=(), *, cuda=True, gqa=False):
    """Reject tensors whose shape, dtype, layout or device differs from what the C
    entry points read and write: q [B,H,S,D] bf16; k, v [B,Hkv,S,D] bf16 (Hkv = H
    unless gqa); o, do like q; lse [B,H,S] fp32; outs (dq, dk, dv) or (o, lse).
    The C ABI takes bare pointers, so a mismatch here would otherwise become an
    out-of-bounds device access."""
    import torch
    if q.dim() != 4:
        raise ValueError("q must be [B,H,S,D]")
    B, H, S, D = q.shape
    Hkv = k.shape[1] if gqa and k.dim() == 4 else H
    bf, f32 = torch.bfloat16, torch.float32
    want = [("q", q, (B, H, S, D), bf), ("k", k, (B, Hkv, S, D), bf), ("v", v, (B, Hkv, S, D), bf)]
    if o is not None:
        want.append(("o", o, (B, H, S, D), bf))
    if do is not None:
        want.append(("do", do, (B, H, S, D), bf))
    if lse is not None:
        want.append(("lse", lse, (B, H, S), f32))
    names = ("dq", "dk", "dv") if len(outs) == 3 else ("out", "lse_out")
    shapes = ((B, H, S, D), (B, Hkv, S, D), (B, Hkv, S, D)) if len(outs) == 3 else \
        ((B, H, S, D), (B, H, S))
    dtypes = (bf, bf, bf) if len(outs) == 3 else (bf, f32)
    want += [(n, t, sh, dt) for n, t, sh, dt in zip(names, outs, shapes, dtypes) if t is not None]
    for name, t, shape, dtype in want:
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {shape}")
        if t.dtype != dtype:
            raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if cuda and (not t.is_cuda or t.device != q.device):
            raise ValueError(f"{name} must be a CUDA tensor on {q.device}")
        if not cuda and t.is_cuda:
            raise ValueError(f"{name} must be a host tensor")


def dash_status_string(status: int) -> str:
    return load().dash_status_string(int(status)).decode()


def dash_attn_fwd(q, k, v, causal: bool, out=None, lse=None, stream=None):
    """O, LSE = attention forward (bf16 [B,H,S,D] CUDA tensors)."""
    import torch
    _check_tensors(q, k, v, outs=(out, lse))
    B, H, S, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    rc = load().dash_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, S, D,
                              int(bool(causal)), _stream_handle(stream))
    _check(rc, "dash_attn_fwd")
    return out, lse


def dash_attn_bwd(q, k, v, o, do, lse, causal: bool, schedule="shift", dq=None, dk=None,
                  dv=None, stream=None):
    """dQ, dK, dV of attention (bf16 [B,H,S,D], lse fp32 [B,H,S]; CUDA tensors)."""
    import torch
    _check_tensors(q, k, v, o, do, lse, (dq, dk, dv))
    B, H, S, D = q.shape
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    rc = load().dash_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                              _ptr(dk), _ptr(dv), B, H, S, D, int(bool(causal)),
                              _sched_id(schedule), _stream_handle(stream))
    _check(rc, "dash_attn_bwd")
    return dq, dk, dv


def dash_attn_fwd_gqa(q, k, v, causal: bool, out=None, lse=None, stream=None):
    """O, LSE of grouped-query attention: q [B,H,S,D], k and v [B,Hkv,S,D] (bf16
    CUDA tensors), query head h reading K/V head h // (H // Hkv)."""
    import torch
    _check_tensors(q, k, v, outs=(out, lse), gqa=True)
    B, H, S, D = q.shape
    Hkv = k.shape[1]
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    rc = load().dash_attn_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Hkv, S,
                                  D, int(bool(causal)), _stream_handle(stream))
    _check(rc, "dash_attn_fwd_gqa")
    return out, lse


def dash_attn_bwd_gqa(q, k, v, o, do, lse, causal: bool, schedule="shift", dq=None, dk=None,
                      dv=None, stream=None, split=None):
    """dQ [B,H,S,D], dK and dV [B,Hkv,S,D] of grouped-query attention (dK, dV summed
    over each K/V head's query heads).  split: sub-groups per K/V head (a power of
    two dividing H / Hkv); None or 0 lets the library choose."""
    import torch
    _check_tensors(q, k, v, o, do, lse, (dq, dk, dv), gqa=True)
    B, H, S, D = q.shape
    Hkv = k.shape[1]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk),
            _ptr(dv), B, H, Hkv, S, D, int(bool(causal)), _sched_id(schedule))
    if split is None:
        rc = load().dash_attn_bwd_gqa(*args, _stream_handle(stream))
    else:
        rc = load().dash_attn_bwd_gqa_split(*args, int(split), _stream_handle(stream))
    _check(rc, "dash_attn_bwd_gqa")
    return dq, dk, dv


def dash_bwd_gqa_split_for(num_ctas: int, B: int, Hkv: int, group: int, S: int, causal: bool,
                           schedule="shift") -> int:
    """The sub-group count dash_attn_bwd_gqa chooses (host only)."""
    n = ctypes.c_int(0)
    _check(load().dash_bwd_gqa_split_for(num_ctas, B, Hkv, group, S, int(bool(causal)),
                                         _sched_id(schedule), ctypes.byref(n)),
           "dash_bwd_gqa_split_for")
    return n.value


def dash_attn_bwd_host(q, k, v, o, do, lse, causal: bool, schedule="shift", dq=None, dk=None,
                       dv=None, stream=None):
    """The backward from host (CPU) tensors, pipelined over parts of the heads;
    results are bitwise those of dash_attn_bwd.  Page-locked tensors let the
    copies overlap the compute.  The outputs are valid once `stream` (default:
    torch's current stream) has completed."""
    import torch
    _check_tensors(q, k, v, o, do, lse, (dq, dk, dv), cuda=False)
    B, H, S, D = q.shape
    pin = q.is_pinned()
    dq = torch.empty(q.shape, dtype=q.dtype, pin_memory=pin) if dq is None else dq
    dk = torch.empty(k.shape, dtype=k.dtype, pin_memory=pin) if dk is None else dk
    dv = torch.empty(v.shape, dtype=v.dtype, pin_memory=pin) if dv is None else dv
    rc = load().dash_attn_bwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                                   _ptr(dq), _ptr(dk), _ptr(dv), B, H, S, D, int(bool(causal)),
                                   _sched_id(schedule), _stream_handle(stream))
    _check(rc, "dash_attn_bwd_host")
    return dq, dk, dv


def dash_attn_bwd_noalloc(q, k, v, o, do, lse, causal: bool, schedule, dq, dk, dv,
                          stream=None):
    """The backward through the entry point that allocates no device memory.
    Outputs must be preallocated; all scratch comes from the library's static
    device array (see include/dash_attn.h)."""
    for t in (dq, dk, dv):
        if t is None:
            raise ValueError("dash_attn_bwd_noalloc needs preallocated dq, dk, dv")
    _check_tensors(q, k, v, o, do, lse, (dq, dk, dv))
    B, H, S, D = q.shape
    rc = load().dash_attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                                      _ptr(dq), _ptr(dk), _ptr(dv), B, H, S, D,
                                      int(bool(causal)), _sched_id(schedule),
                                      _stream_handle(stream))
    _check(rc, "dash_attn_bwd_noalloc")
    return dq, dk, dv


def dash_attn_sync_status(stream=None) -> int:
    return int(load().dash_attn_sync_status(_stream_handle(stream)))


def dash_attn_noalloc_sync_status(stream=None) -> int:
    """Waits for the stream and returns (and clears) the status that
    dash_attn_bwd_noalloc's calls recorded on the current device."""
    return int(load().dash_attn_noalloc_sync_status(_stream_handle(stream)))


def dash_set_spin_limit_us(us: int) -> None:
    _check(load().dash_set_spin_limit_us(int(us)), "dash_set_spin_limit_us")


def dash_inject_fault(mode: int) -> None:
    """Arm (1) or cancel (0) the host-side fault for the next backward."""
    _check(load().dash_inject_fault(int(mode)), "dash_inject_fault")


def dash_bwd_num_ctas(device: int = 0, D: int = 128) -> int:
    n = ctypes.c_int(0)
    _check(load().dash_bwd_num_ctas(device, D, ctypes.byref(n)), "dash_bwd_num_ctas")
    return n.value


def dash_set_dq_chain_mode(mode: int) -> None:
    """0: the library picks per launch; 1: middle positions of the ordered dQ chains
    add with red in L2; 2: load-add-store on the SM (bitwise the same results)."""
    _check(load().dash_set_dq_chain_mode(int(mode)), "dash_set_dq_chain_mode")


def dash_dq_chain_uses_red(schedule: str, S: int, D: int = 128, heads_per_unit: int = 1) -> bool:
    """Whether a deterministic backward of this schedule, length and head dim, with this
    many query heads per unit of its table, adds its chains' middle positions with red
    under the current mode (host only)."""
    r = ctypes.c_int(0)
    _check(load().dash_dq_chain_uses_red(_sched_id(schedule), S, int(D), int(heads_per_unit),
                                         ctypes.byref(r)),
           "dash_dq_chain_uses_red")
    return bool(r.value)


def dash_set_slot_placement(mode: int) -> None:
    """1: each CTA runs the table slot of its SM id's rank; 2: CTA b runs slot b; 0:
    the library's choice (by SM id from 128 tiles).  Bitwise the same results."""
    _check(load().dash_set_slot_placement(int(mode)), "dash_set_slot_placement")


def dash_slot_placement_by_smid(S: int) -> bool:
    """Whether a backward of length S places the table's slots by SM id under the
    current mode (host only)."""
    r = ctypes.c_int(0)
    _check(load().dash_slot_placement_by_smid(int(S), ctypes.byref(r)),
           "dash_slot_placement_by_smid")
    return bool(r.value)


def dash_set_head_interleave(mode: int) -> None:
    """Heads per unit of a multi-head backward's table: 0 the library's choice, 1 never
    interleave, 2 or 4 that many whenever it divides B * H."""
    _check(load().dash_set_head_interleave(int(mode)), "dash_set_head_interleave")


def dash_bwd_head_interleave(num_ctas: int, D: int, schedule: str, n_heads: int, S: int,
                             causal: bool) -> int:
    """Heads per unit a multi-head backward takes under the current mode (host only)."""
    r = ctypes.c_int(0)
    _check(load().dash_bwd_head_interleave(num_ctas, D, _sched_id(schedule), n_heads, S,
                                           int(bool(causal)), ctypes.byref(r)),
           "dash_bwd_head_interleave")
    return r.value


def dash_release_workspace() -> None:
    _check(load().dash_release_workspace(), "dash_release_workspace")


def dash_sched_table(n_heads: int, N: int, causal: bool, schedule, num_ctas: int):
    """Rows (cta, head, kv, q, position, chain_index) as a list of tuples."""
    lib = load()
    sid = _sched_id(schedule)
    n = lib.dash_sched_table(n_heads, N, int(bool(causal)), sid, num_ctas, None, 0)
    if n < 0:
        raise DashError(int(-n), "dash_sched_table")
    buf = (ctypes.c_int * (6 * n))()
    lib.dash_sched_table(n_heads, N, int(bool(causal)), sid, num_ctas, buf, n)
    flat = list(buf)
    return [tuple(flat[6 * r: 6 * r + 6]) for r in range(n)]


def dash_sched_table_part(n_heads: int, N: int, causal: bool, schedule, num_ctas: int,
                          h0: int, h1: int):
    """Rows of the part of the table covering heads [h0, h1), heads renumbered
    from 0, as the host-buffer path launches it."""
    lib = load()
    sid = _sched_id(schedule)
    n = lib.dash_sched_table_part(n_heads, N, int(bool(causal)), sid, num_ctas, h0, h1, None, 0)
    if n < 0:
        raise DashError(int(-n), "dash_sched_table_part")
    buf = (ctypes.c_int * (6 * max(n, 1)))()
    lib.dash_sched_table_part(n_heads, N, int(bool(causal)), sid, num_ctas, h0, h1, buf, n)
    flat = list(buf)
    return [tuple(flat[6 * r: 6 * r + 6]) for r in range(n)]


def dash_sched_table_gqa(n_heads: int, group: int, N: int, causal: bool, schedule,
                         num_ctas: int):
    """Rows (cta, query head, kv, q, position, chain_index) of a grouped-query table."""
    lib = load()
    sid = _sched_id(schedule)
    n = lib.dash_sched_table_gqa(n_heads, group, N, int(bool(causal)), sid, num_ctas, None, 0)
    if n < 0:
        raise DashError(int(-n), "dash_sched_table_gqa")
    buf = (ctypes.c_int * (6 * max(n, 1)))()
    lib.dash_sched_table_gqa(n_heads, group, N, int(bool(causal)), sid, num_ctas, buf, n)
    flat = list(buf)
    return [tuple(flat[6 * r: 6 * r + 6]) for r in range(n)]


def dash_sched_table_pairs(n_heads: int, N: int, causal: bool, num_ctas: int):
    """Rows (cta, head, kv, q, position, chain_index) of the grid's CTA-pair table
    (SHIFT_PAIRS, or SYM_SHIFT_PAIRS when causal) for num_ctas CTAs (even): CTAs 2i and
    2i + 1 run KV tiles 2m and 2m + 1 over the same Q tiles with the same positions."""
    lib = load()
    n = lib.dash_sched_table_pairs(n_heads, N, int(causal), num_ctas, None, 0)
    if n < 0:
        raise DashError(int(-n), "dash_sched_table_pairs")
    buf = (ctypes.c_int * (6 * max(n, 1)))()
    lib.dash_sched_table_pairs(n_heads, N, int(causal), num_ctas, buf, n)
    flat = list(buf)
    return [tuple(flat[6 * r: 6 * r + 6]) for r in range(n)]


def dash_sched_simulate(n_heads: int, N: int, causal: bool, schedule, num_ctas: int,
                        w_compute: float, w_reduce: float, dq_buffers: int = 0,
                        dq_chains: int = 1):
    """(critical_path, makespan, bubble_time, stalls) of a schedule's DAG;
    dq_chains = 2 models the kernel's two accumulators per dQ block."""
    cp, mk, bt = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    st = ctypes.c_longlong()
    rc = load().dash_sched_simulate(n_heads, N, int(bool(causal)), _sched_id(schedule), num_ctas,
                                    float(w_compute), float(w_reduce), int(dq_buffers),
                                    int(dq_chains), ctypes.byref(cp), ctypes.byref(mk),
                                    ctypes.byref(bt), ctypes.byref(st))
    _check(rc, "dash_sched_simulate")
    return cp.value, mk.value, bt.value, st.value


def dash_sched_simulate_gqa(n_heads: int, group: int, N: int, causal: bool, schedule,
                            num_ctas: int, w_compute: float, w_reduce: float,
                            dq_buffers: int = 0, dq_chains: int = 1):
    """dash_sched_simulate over the grouped-query table (`group` query heads per K/V head)."""
    cp, mk, bt = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    st = ctypes.c_longlong()
    rc = load().dash_sched_simulate_gqa(n_heads, group, N, int(bool(causal)), _sched_id(schedule),
                                        num_ctas, float(w_compute), float(w_reduce),
                                        int(dq_buffers), int(dq_chains), ctypes.byref(cp),
                                        ctypes.byref(mk), ctypes.byref(bt), ctypes.byref(st))
    _check(rc, "dash_sched_simulate_gqa")
    return cp.value, mk.value, bt.value, st.value


def dash_sched_check(n_heads: int, N: int, causal: bool, num_ctas: int, rows) -> int:
    """Status of the library's checks on a caller-supplied table given as rows
    (cta, head, kv, q, position, chain_index): 0 valid, 6 a failed check
    (coverage, positions or a deadlocking ticket order), 1 malformed rows."""
    flat = [int(x) for r in rows for x in r]
    buf = (ctypes.c_int * max(len(flat), 1))(*flat)
    return int(load().dash_sched_check(n_heads, N, int(bool(causal)), num_ctas, buf, len(rows)))


def dash_dag_longest_path(n_nodes: int, edges):
    """(cp, depth list, height list) of a weighted DAG given as (u, v, w) edges."""
    m = len(edges)
    src = (ctypes.c_int * max(m, 1))(*[e[0] for e in edges])
    dst = (ctypes.c_int * max(m, 1))(*[e[1] for e in edges])
    w = (ctypes.c_double * max(m, 1))(*[float(e[2]) for e in edges])
    depth = (ctypes.c_double * max(n_nodes, 1))()
    height = (ctypes.c_double * max(n_nodes, 1))()
    cp = ctypes.c_double()
    rc = load().dash_dag_longest_path(n_nodes, m, src, dst, w, depth, height, ctypes.byref(cp))
    _check(rc, "dash_dag_longest_path")
    return cp.value, list(depth)[:n_nodes], list(height)[:n_nodes]


def dash_profile_begin() -> None:
    _check(load().dash_profile_begin(), "dash_profile_begin")


def dash_profile_end():
    """(main kernel ms summed, auxiliary kernels ms summed, backward calls)."""
    m, a, n = ctypes.c_double(), ctypes.c_double(), ctypes.c_longlong()
    _check(load().dash_profile_end(ctypes.byref(m), ctypes.byref(a), ctypes.byref(n)),
           "dash_profile_end")
    return m.value, a.value, n.value


def dash_trace_bwd(q, k, v, o, do, lse, causal: bool, schedule="shift", stream=None):
    """One traced backward; returns (dq, dk, dv, trace [ctas, rows, 16] uint64 ns),
    the events per pair listed at dash_trace_bwd in include/dash_attn.h."""
    import numpy as np
    import torch
    _check_tensors(q, k, v, o, do, lse)
    B, H, S, D = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    N = S // 128
    EV = 16
    cap = EV * (B * H * N * N + 1024 * (N + 1))   # >= ctas * rows_per_cta * EV
    buf = np.zeros(cap, dtype=np.uint64)
    nc, rows = ctypes.c_int(), ctypes.c_int()
    rc = load().dash_trace_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                               _ptr(dk), _ptr(dv), B, H, S, D, int(bool(causal)),
                               _sched_id(schedule), _stream_handle(stream),
                               buf.ctypes.data_as(ctypes.c_void_p), cap, ctypes.byref(nc),
                               ctypes.byref(rows))
    _check(rc, "dash_trace_bwd")
    n = nc.value * rows.value * EV
    if n > cap:
        raise RuntimeError("trace buffer too small")
    return dq, dk, dv, buf[:n].reshape(nc.value, rows.value, EV)
