"""The Python binding's tensor checks (no GPU): every wrapper rejects tensors
whose shape, dtype, layout or device the C entry points would misread, before
anything reaches the library."""
import pytest
import torch

from persistent_sm_attn_b200 import binding


def _host(B=1, H=4, Hkv=4, S=256, D=64):
    q = torch.zeros(B, H, S, D, dtype=torch.bfloat16)
    k = torch.zeros(B, Hkv, S, D, dtype=torch.bfloat16)
    v = torch.zeros_like(k)
    o, do = torch.zeros_like(q), torch.zeros_like(q)
    lse = torch.zeros(B, H, S, dtype=torch.float32)
    return [q, k, v, o, do, lse]


def test_valid_tensors_pass():
    binding._check_tensors(*_host(), cuda=False)
    binding._check_tensors(*_host(Hkv=2), cuda=False, gqa=True)
    t = _host()
    binding._check_tensors(*t, (torch.zeros_like(t[0]), torch.zeros_like(t[1]),
                                torch.zeros_like(t[2])), cuda=False)


@pytest.mark.parametrize("index,bad", [
    (1, torch.zeros(1, 4, 128, 64, dtype=torch.bfloat16)),     # k with another S
    (2, torch.zeros(1, 4, 256, 128, dtype=torch.bfloat16)),    # v with another D
    (3, torch.zeros(1, 4, 256, 64, dtype=torch.float16)),      # o in fp16
    (4, torch.zeros(1, 2, 256, 64, dtype=torch.bfloat16)),     # dO with fewer heads
    (5, torch.zeros(1, 4, 256, dtype=torch.float64)),          # lse in fp64
    (5, torch.zeros(4, 256, dtype=torch.float32)),             # lse flattened
    (0, torch.zeros(1, 4, 64, 256, dtype=torch.bfloat16).transpose(2, 3)),  # q not contiguous
])
def test_host_path_rejects_mismatched_inputs(index, bad):
    t = _host()
    t[index] = bad
    with pytest.raises(ValueError):
        binding.dash_attn_bwd_host(*t, False, "shift")


def test_outputs_are_checked_too():
    t = _host()
    with pytest.raises(ValueError, match="dk"):
        binding.dash_attn_bwd_host(*t, False, "shift", dk=torch.zeros(1, 4, 256, 32,
                                                                      dtype=torch.bfloat16))


def test_device_entry_points_reject_host_tensors():
    t = _host()
    with pytest.raises(ValueError, match="CUDA"):
        binding.dash_attn_bwd(*t, False, "shift")
    with pytest.raises(ValueError, match="CUDA"):
        binding.dash_attn_fwd(*t[:3], False)
    with pytest.raises(ValueError):
        binding.dash_attn_bwd_noalloc(*t, False, "shift", None, None, None)


def test_multi_head_entry_rejects_grouped_kv_and_grouped_entry_accepts_it():
    t = _host(Hkv=2)
    with pytest.raises(ValueError, match="k has shape"):
        binding._check_tensors(*t, cuda=False)
    binding._check_tensors(*t, cuda=False, gqa=True)
    with pytest.raises(ValueError, match="dk"):
        binding._check_tensors(*t, (None, torch.zeros_like(t[0]), None), cuda=False, gqa=True)
