"""bsa_forward_host (host buffers in and out, copies overlapped with the
compute) against bsa_forward on device copies of the same inputs.

The host path cuts the job into independent (batch entry, key/value head
group) chunks and runs the same kernels on compact copies of each, so its
output must equal the device path's bit for bit; the device path itself is
checked against the oracle in the other GPU tests. The cases cover slot reuse
(more chunks than the two slots), head groups split within a batch entry,
grouped queries, the causal flag, float32 and e4m3 inputs, and pageable
(non-pinned) host memory.
"""
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import block_sparse_attention_19_b200 as m

    return m


CASES = [  # (B, N, H, H_kv, D, block_size, ratio, dtype, causal, pinned)
    (5, 1024, 4, 4, 64, 64, 0.3, "bf16", False, True),       # 5 chunks (one per batch entry), 2 slots
    (1, 65536, 4, 4, 128, 128, 0.1, "bf16", False, True),    # one head per chunk (67 MB each)
    (2, 32768, 8, 2, 128, 128, 0.2, "bf16", True, True),     # grouped queries, causal, 2 kv heads per chunk
    (3, 512, 2, 2, 64, 64, 0.5, "f32", False, False),        # float32, pageable host memory
    (2, 2048, 4, 2, 128, 64, 0.25, "e4m3", False, True),     # e4m3 inputs, bf16 output
    (1, 65536, 2, 2, 64, 64, 0.05, "f32", False, True),      # float32, one head per chunk (sums that round)
]


@pytest.mark.parametrize("ci", range(len(CASES)))
def test_host_path_equals_device_path(bsa, ci):
    B, N, H, Hkv, D, bs, ratio, dt, causal, pinned = CASES[ci]
    cfg = W.Config(f"host{ci}", B, N, H, D, bs, ratio, dt, 1.0, 1400 + ci, None, H_kv=Hkv)
    q, k, v = W.make_inputs(cfg, device="cuda")
    flags = bsa.BSA_FLAG_CAUSAL if causal else 0
    ref = bsa.bsa_forward(q, k, v, bs, ratio, flags=flags)
    hq, hk, hv = (x.cpu() for x in (q, k, v))
    if pinned:
        hq, hk, hv = (x.pin_memory() for x in (hq, hk, hv))
    need = bsa.bsa_forward_host_workspace_bytes(B, N, H, D, bs, ratio, q.dtype, H_kv=Hkv)
    assert need > 0
    o = bsa.bsa_forward_host(hq, hk, hv, bs, ratio, flags=flags)
    assert bsa.bsa_device_error() == 0
    assert o.device.type == "cpu" and o.dtype == ref.dtype and o.shape == ref.shape
    assert torch.equal(o, ref.cpu())
    # a second call into the same output and workspace (slots reused across calls)
    ws = torch.empty(need, device="cuda", dtype=torch.uint8)
    o.zero_()
    bsa.bsa_forward_host(hq, hk, hv, bs, ratio, out=o, flags=flags, workspace=ws)
    bsa.bsa_forward_host(hq, hk, hv, bs, ratio, out=o, flags=flags, workspace=ws)
    assert torch.equal(o, ref.cpu())


def test_host_path_rejects_device_tensors_and_small_workspace(bsa):
    q = torch.zeros(1, 512, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        bsa.bsa_forward_host(q.cuda(), q, q, 64, 0.5)
    ws = torch.empty(256, device="cuda", dtype=torch.uint8)
    with pytest.raises(bsa.BsaError, match="WORKSPACE"):
        bsa.bsa_forward_host(q, q, q, 64, 0.5, workspace=ws)


@pytest.mark.parametrize("dtype,D", [(torch.float32, 128), (torch.bfloat16, 64), (torch.float8_e4m3fn, 128)])
def test_pooling_does_not_depend_on_the_head_count(bsa, dtype, D):
    """Each block mean is summed in one fixed order whatever the number of
    heads in the tensor (the host-buffer path pools one head group at a time
    and must reproduce the whole-tensor result bit for bit). float32 data has
    sums that round, so a different order would show."""
    g = torch.Generator(device="cuda").manual_seed(1700)
    x = (torch.randn(2, 4096, 8, D, generator=g, device="cuda") * 3 + 1).to(dtype)
    full = bsa.bsa_block_pool(x, 256)
    for h in (0, 3, 7):
        one = bsa.bsa_block_pool(x[:, :, h:h + 1].contiguous(), 256)
        assert torch.equal(one[:, 0], full[:, h]), h
