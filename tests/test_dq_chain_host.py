"""Host-side choice of how the ordered dQ chains add a middle position (no GPU):
red in L2 for descending and naive ascending from 64 tiles by default, forced
either way by dash_set_dq_chain_mode, never for the atomic variant."""
import pytest

from persistent_sm_attn_b200 import binding


def test_default_choice():
    f = binding.dash_dq_chain_uses_red
    binding.dash_set_dq_chain_mode(0)
    assert f("descending", 8192) and f("naive_asc", 16384) and f("descending", 64 * 128)
    assert not f("descending", 63 * 128) and not f("naive_asc", 4096)
    assert not f("shift", 16384) and not f("sym_shift", 16384)
    assert not f("atomic", 16384)
    # at D=64, tables with two or more query heads per unit take red on every
    # deterministic schedule; at D=128 they do not
    assert f("sym_shift", 16384, 64, 2) and f("shift", 1024, 64, 4) and f("descending", 512, 64, 2)
    assert not f("sym_shift", 16384, 128, 2) and not f("sym_shift", 16384, 64, 1)
    assert not f("atomic", 16384, 64, 2)
    # CTA pairs keep the load-add-store unless red is forced
    assert not f("shift_pairs", 16384, 64, 1)


def test_forced_modes():
    f = binding.dash_dq_chain_uses_red
    try:
        binding.dash_set_dq_chain_mode(1)
        assert all(f(s, 256) for s in ("naive_asc", "descending", "shift", "sym_shift",
                                      "shift_pairs"))
        assert not f("atomic", 256)
        binding.dash_set_dq_chain_mode(2)
        assert not any(f(s, 16384) for s in ("naive_asc", "descending", "shift", "sym_shift"))
    finally:
        binding.dash_set_dq_chain_mode(0)


def test_argument_errors():
    for bad in (lambda: binding.dash_set_dq_chain_mode(3),
                lambda: binding.dash_set_dq_chain_mode(-1),
                lambda: binding.dash_dq_chain_uses_red("descending", 100),
                lambda: binding.dash_dq_chain_uses_red("descending", 0),
                lambda: binding.dash_dq_chain_uses_red("descending", 1024, 64, 0),
                lambda: binding.dash_dq_chain_uses_red("descending", 1024, 96, 1)):
        with pytest.raises(binding.DashError):
            bad()
