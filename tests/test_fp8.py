"""GPU parity of the FP8 (E4M3) inputs against the float64 oracle.

Reading (page "2026 新一代卷积与 Transformer 网络架构", section "基准测试": SparseFormer
run in FP8; closing advice: use FP8 tensor cores): q, k, v are e4m3 values
and the method computed on them is unchanged; the oracle runs on their exact
values. The GPU path computes both products as tcgen05 kind::f8f6f4 with
float32 accumulation and rounds the softmax weights P to e4m3 for the P.V
product (row sums from float32 P); the output is bfloat16.

Tolerance, from that arithmetic: rounding P to e4m3 changes each weight by
at most 2^-4 of itself in e4m3's normal range (P >= 2^-6 of the row's running
max) and by at most the weight itself below it, so per output element
|d| <= 2^-4 (sum_t p_t |v_t|) / l + (sum over the small weights) / l + the
bfloat16 rounding of o. The first term is computed here exactly with the
oracle run on |v| (same weights); the small-weight term and the rounding are
covered by an absolute 2^-8 * max|v| and a relative 2^-8 |o|. Over a whole
output o's error is a weighted combination of the weights' rounding errors.
A weight p = 2^x rounded to nearest in e4m3 (spacing 2^-3 of its binade) has
an error uniform within half a spacing, so its relative error has rms
2^-4 / (sqrt(3) m) for mantissa m in [1, 2). The weights are exponentials of
smoothly spread logits, so their mantissas are log-uniform, E[1/m^2] =
3 / (8 ln 2), and the relative rms is 2^-4 sqrt(1 / (8 ln 2)) = 0.0265 (the
distribution-free bound, m -> 1, is 2^-4 / sqrt(3) = 0.036). Relative L2 of
the output: <= 0.03, that expectation with a 13% margin (measured 0.022 to
0.026 on these cases). Index lists follow the near-tie rule (pooling reads
the exact e4m3 values).
"""
import numpy as np
import pytest
import torch

import workloads as W
from test_causal import accept_causal_rows
from test_parity import _host, accept_index_rows, gpu_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import block_sparse_attention_19_b200 as m

    return m


def check_fp8_output(o_gpu, o_ref, o_abs, vmax):
    d = np.abs(o_gpu - o_ref)
    bound = 2.0 ** -4 * o_abs + 2.0 ** -8 * vmax + 2.0 ** -8 * np.abs(o_ref)
    rel = np.linalg.norm(o_gpu - o_ref) / np.linalg.norm(o_ref)
    print(f"fp8: max|d| {d.max():.3g}, max|d|/bound {(d / bound).max():.3g}, rel L2 {rel:.3g}")
    assert np.all(d <= bound), f"max|d|/bound = {(d / bound).max()}"
    assert rel <= 0.03, f"rel L2 = {rel}"


CASES = [  # (B, N, H, H_kv, D, block_size, ratio, causal)
    (1, 2048, 2, 2, 128, 128, 0.25, False),
    (1, 2048, 4, 2, 128, 128, 0.3, False),   # grouped queries, heads paired in a CTA
    (1, 1920, 2, 2, 128, 128, 0.4, True),    # causal, odd nb
    (1, 4096, 2, 2, 128, 256, 0.3, False),   # block_size 256
    (1, 1024, 2, 2, 128, 128, 1.0, False),   # k = nb
    (1, 2048, 2, 2, 128, 64, 0.25, False),   # block_size 64: two query blocks stacked per tile
    (1, 1344, 4, 2, 128, 64, 0.3, True),     # block_size 64, causal, nb 21 (a CTA with one block)
    # D = 64: 64-byte rows in the 64-byte swizzled layout
    (2, 8192, 4, 4, 64, 64, 0.3, False),     # the page's benchmark shape (seq 8192, D 64, block_size 64)
    (1, 2048, 2, 2, 64, 128, 0.25, False),
    (1, 2048, 4, 2, 64, 128, 0.3, False),    # grouped queries, heads paired in a CTA
    (1, 4096, 2, 2, 64, 256, 0.3, True),     # block_size 256, causal
    (1, 1344, 4, 2, 64, 64, 0.3, True),      # block_size 64, causal, nb 21
    (1, 1024, 2, 2, 64, 128, 1.0, False),    # k = nb
]


@pytest.mark.parametrize("ci", range(len(CASES)))
def test_fp8_full_path(bsa, oracle_mod, ci):
    B, N, H, Hkv, D, bs, ratio, causal = CASES[ci]
    cfg = W.Config(f"fp8{ci}", B, N, H, D, bs, ratio, "e4m3", 1.0, 950 + ci, None, H_kv=Hkv)
    q, k, v = W.make_inputs(cfg, device="cuda")
    assert q.dtype == torch.float8_e4m3fn
    flags = bsa.BSA_FLAG_CAUSAL if causal else 0
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(B, N, H, D, bs, ratio, H_kv=Hkv), device="cuda",
                     dtype=torch.uint8)
    o = bsa.bsa_forward(q, k, v, bs, ratio, workspace=ws, flags=flags)
    torch.cuda.synchronize()
    assert bsa.bsa_device_error() == 0 and o.dtype == torch.bfloat16
    _, _, idx_g = bsa.workspace_views(ws, B, N, H, D, bs, ratio, H_kv=Hkv)
    qa, ka, va = _host(q), _host(k), _host(v)
    ref = oracle_mod.forward_gqa(qa, ka, va, bs, ratio, causal=causal)
    g = idx_g.cpu().numpy()
    if causal:
        accept_causal_rows(g, ref["scores"], cfg.k, ref["idx"], False)
    else:
        accept_index_rows(g, ref["scores"], cfg.k, ref["idx"])
    gq = np.repeat(g, H // Hkv, axis=1)
    o_ref = oracle_mod.sparse_attn_gqa(qa, ka, va, gq, bs, causal=causal)
    # sum_t p_t |v_t| / l: the oracle on the same (exact) q, k with |v| as values
    q64, k64 = (x.to(torch.float64).cpu().numpy() for x in (q, k))
    vabs = np.abs(v.to(torch.float64).cpu().numpy())
    o_abs = oracle_mod.sparse_attn_gqa(q64, k64, vabs, gq, bs, causal=causal)
    rows = np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (B, H, cfg.nb)).copy()
    check_fp8_output(gpu_rows(o, rows, bs), o_ref, o_abs, vabs.max())


def test_fp8_attention_alone_d64(bsa, oracle_mod):
    """bsa_sparse_attn_fwd on e4m3 D = 64 inputs with random index rows
    (non-contiguous blocks), block_size 64 and 128."""
    for bs in (64, 128):
        cfg = W.Config("fp8_d64", 1, 4096, 2, 64, bs, 0.25, "e4m3", 1.0, 990 + bs, None)
        q, k, v = W.make_inputs(cfg, device="cuda")
        rng = np.random.default_rng(bs)
        idx = np.sort(np.stack([[rng.choice(cfg.nb, cfg.k, replace=False) for _ in range(cfg.nb)]
                                for _ in range(cfg.H)])[None], -1).astype(np.int32)
        o = bsa.bsa_sparse_attn_fwd(q, k, v, torch.from_numpy(idx).cuda(), bs)
        torch.cuda.synchronize()
        assert bsa.bsa_device_error() == 0
        o_ref = oracle_mod.sparse_attn(_host(q), _host(k), _host(v), idx, bs)
        q64, k64 = (x.to(torch.float64).cpu().numpy() for x in (q, k))
        vabs = np.abs(v.to(torch.float64).cpu().numpy())
        o_abs = oracle_mod.sparse_attn(q64, k64, vabs, idx, bs)
        rows = np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (1, 2, cfg.nb)).copy()
        check_fp8_output(gpu_rows(o, rows, bs), o_ref, o_abs, vabs.max())
