"""bsa_forward_noalloc, the allocation-free forward, against bsa_forward.

Some callers cannot allocate device memory themselves: a plugin that runs
inside a host application owning the whole device-memory budget, or a loop in
which cudaMalloc (and the device synchronisation it may imply) is not allowed.
bsa_forward_noalloc serves them from a fixed scratch array built into the
library instead of a caller workspace. These tests call it through the C ABI
twice in a row -- the second call reuses the scratch the first one left
behind -- and compare each output with bsa_forward (caller workspace). Both
run the same kernels on the same inputs, so the outputs must be equal bit for
bit: any stale or overlapping scratch content would show. They also check
that sizes beyond the scratch are refused before anything runs.

This file is collected last on purpose and passes both on its own in a fresh
process and after the rest of the suite.
"""
import ctypes

import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 64 << 20  # BSA_NOALLOC_SCRATCH_BYTES in include/bsa.h


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import block_sparse_attention_19_b200 as m

    return m


def _noalloc_c_call(bsa, q, k, v, o, block_size, ratio):
    P = ctypes.c_void_p
    B, N, H, D = q.shape
    dt = 1 if q.dtype == torch.bfloat16 else 0
    stream = P(torch.cuda.current_stream().cuda_stream)
    return bsa.lib.bsa_forward_noalloc(P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()), P(o.data_ptr()),
                                       B, N, H, D, block_size, float(ratio), dt, stream)


def _same(got: torch.Tensor, want: torch.Tensor):
    d = (got.to(torch.float64) - want.to(torch.float64)).abs().max().item()
    assert torch.equal(got, want), f"outputs differ (max|d| = {d})"


CASES = [  # (B, N, H, D, block_size, ratio, dtype): two different problems, one after the other
    W.Config("first", 1, 4096, 4, 128, 128, 0.25, "bf16", 1.0, 31, None),
    W.Config("second", 2, 2048, 3, 64, 64, 0.45, "bf16", 1.0, 32, None),
    W.Config("fp32", 1, 512, 2, 64, 64, 0.25, "f32", 1.0, 33, None),
]


def test_noalloc_matches_bsa_forward_on_calls_in_a_row(bsa):
    for cfg in CASES:
        assert bsa.bsa_forward_workspace_bytes(cfg.B, cfg.N, cfg.H, cfg.D, cfg.block_size,
                                               cfg.topk_ratio) <= SCRATCH_BYTES
    outs = []
    for cfg in CASES:  # calls in a row, each leaving its intermediates in the shared scratch
        q, k, v = W.make_inputs(cfg, device="cuda")
        o = torch.empty_like(q)
        assert _noalloc_c_call(bsa, q, k, v, o, cfg.block_size, cfg.topk_ratio) == 0, \
            bsa.lib.bsa_last_error_detail().decode()
        outs.append((cfg, q, k, v, o))
    # the first problem again: the scratch now holds the last call's contents
    cfg, q, k, v, _ = outs[0]
    o_again = torch.empty_like(q)
    assert _noalloc_c_call(bsa, q, k, v, o_again, cfg.block_size, cfg.topk_ratio) == 0
    torch.cuda.synchronize()
    assert bsa.bsa_device_error() == 0
    for cfg, q, k, v, o in outs:
        ref = bsa.bsa_forward(q, k, v, cfg.block_size, cfg.topk_ratio)
        torch.cuda.synchronize()
        _same(o, ref)
    _same(o_again, outs[0][4])


def test_noalloc_refuses_sizes_beyond_its_scratch(bsa):
    # million-token problem: pooled q and k, the index list and the block scores need about 650 MB
    need = bsa.bsa_forward_workspace_bytes(1, 1 << 20, 8, 128, 256, 0.15)
    assert need > SCRATCH_BYTES
    P = ctypes.c_void_p
    fake = P(0x10000)  # never dereferenced: the size check comes first
    st = bsa.lib.bsa_forward_noalloc(fake, fake, fake, P(0x20000), 1, 1 << 20, 8, 128, 256, 0.15, 1, P(0))
    assert st == 4  # BSA_ERR_WORKSPACE
    assert "built-in scratch" in bsa.lib.bsa_last_error_detail().decode()
