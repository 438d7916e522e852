"""GPU parity of the backward pass (bsa_sparse_attn_fwd_train +
bsa_sparse_attn_bwd) against the float64 oracle.

Reading: the top-k indices carry no gradient (the page listing's selection is
torch.topk indices), so the gradients are those of the attention over the
kept blocks with the lists held fixed; the oracle computes them in float64
from the same bf16 inputs and lists.

Tolerance, from the arithmetic: the GPU path rounds three things to bf16
(unit roundoff u = 2^-8, 8 significant bits): the softmax weights P (operand
of dV), the score gradients dS (operand of dQ and dK) and the gradients it
writes; sums are float32. Each gradient element passes through two of these
roundings, each with a relative rms error of about u / sqrt(3) * 0.73 = 1.6e-3
for log-uniformly spread mantissas, so about 2.3e-3 together. Per gradient
tensor: relative L2 <= 5e-3 (the forward's bf16 bar; measured at most 3.4e-3
over these cases) and max|d| <= 2e-2 * max|reference| (measured at most
7e-3).
"""
import numpy as np
import pytest
import torch

import workloads as W
from test_parity import _host, check_output, gpu_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import block_sparse_attention_19_b200 as m

    return m


def check_grad(got: torch.Tensor, ref: np.ndarray, name: str):
    g = got.to(torch.float64).cpu().numpy()
    d = np.abs(g - ref)
    rel = np.linalg.norm(g - ref) / np.linalg.norm(ref)
    print(f"{name}: max|d| {d.max():.3g} (max|ref| {np.abs(ref).max():.3g}), rel L2 {rel:.3g}")
    assert rel <= 5e-3, f"{name}: rel L2 {rel}"
    assert d.max() <= 2e-2 * np.abs(ref).max(), f"{name}: max|d| {d.max()}"


CASES = [  # (B, N, H, D, block_size, ratio, causal)
    (1, 2048, 2, 128, 128, 0.25, False),
    (1, 2048, 2, 64, 128, 0.3, True),
    (2, 1024, 2, 128, 256, 0.5, False),
    (1, 2048, 2, 128, 256, 0.5, True),
    (1, 1536, 2, 128, 128, 1.0, True),  # dense causal
    # block_size 64: two blocks stacked per 128-row tile (query and key side)
    (1, 2048, 2, 64, 64, 0.25, False),
    (2, 1024, 2, 128, 64, 0.3, True),
    (1, 1344, 2, 64, 64, 0.3, True),    # nb 21: the last tile holds one block
    (1, 1024, 2, 64, 64, 1.0, False),   # k = nb
]


@pytest.mark.parametrize("ci", range(len(CASES)))
def test_backward_matches_oracle(bsa, oracle_mod, ci):
    B, N, H, D, bs, ratio, causal = CASES[ci]
    cfg = W.Config(f"bwd{ci}", B, N, H, D, bs, ratio, "bf16", 1.0, 1100 + ci, None)
    q, k, v = W.make_inputs(cfg, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(1200 + ci)
    do = torch.randn(q.shape, generator=g, device="cuda").to(torch.bfloat16)
    flags = bsa.BSA_FLAG_CAUSAL if causal else 0
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(B, N, H, D, bs, ratio), device="cuda", dtype=torch.uint8)
    bsa.bsa_forward(q, k, v, bs, ratio, workspace=ws, flags=flags)
    idx = bsa.workspace_views(ws, B, N, H, D, bs, ratio)[2].clone()
    o, lse = bsa.bsa_sparse_attn_fwd_train(q, k, v, idx, bs, flags=flags)
    dq, dk, dv = bsa.bsa_sparse_attn_bwd(q, k, v, o, do, idx, lse, bs, flags=flags)
    torch.cuda.synchronize()
    assert bsa.bsa_device_error() == 0
    qa, ka, va, doa = (_host(x) for x in (q, k, v, do))
    il = idx.cpu().numpy()
    # the forward of the training entry point matches the oracle, and so does lse
    o_ref = oracle_mod.sparse_attn(qa, ka, va, il, bs, causal=causal)
    rows = np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (B, H, cfg.nb)).copy()
    check_output(gpu_rows(o, rows, bs), o_ref, "bf16")
    rq, rk, rv = oracle_mod.sparse_attn_bwd(qa, ka, va, doa, il, bs, causal=causal)
    check_grad(dq, rq, "dq")
    check_grad(dk, rk, "dk")
    check_grad(dv, rv, "dv")


def test_lse_is_the_log_softmax_denominator(bsa, oracle_mod):
    """lse_n = ln sum_t exp(scale q_n . k_t) over the kept tokens, checked
    against the same sum in float64 from the exact bf16 inputs."""
    cfg = W.Config("lse", 1, 1024, 2, 128, 128, 0.25, "bf16", 1.0, 1300, None)
    q, k, v = W.make_inputs(cfg, device="cuda")
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(1, 1024, 2, 128, 128, 0.25), device="cuda", dtype=torch.uint8)
    bsa.bsa_forward(q, k, v, 128, 0.25, workspace=ws)
    idx = bsa.workspace_views(ws, 1, 1024, 2, 128, 128, 0.25)[2].clone()
    _, lse = bsa.bsa_sparse_attn_fwd_train(q, k, v, idx, 128)
    torch.cuda.synchronize()
    qd, kd = q.double().cpu(), k.double().cpu()
    il = idx.cpu().numpy()
    want = np.empty((1, 2, 1024))
    for h in range(2):
        for i in range(8):
            keys = np.concatenate([np.arange(j * 128, j * 128 + 128) for j in il[0, h, i]])
            logits = (qd[0, i * 128:(i + 1) * 128, h] @ kd[0, keys, h].T).numpy() / np.sqrt(128)
            m = logits.max(axis=1, keepdims=True)
            want[0, h, i * 128:(i + 1) * 128] = (m + np.log(np.exp(logits - m).sum(axis=1, keepdims=True)))[:, 0]
    got = lse.double().cpu().numpy()
    assert np.abs(got - want).max() <= 1e-4 * max(1.0, np.abs(want).max())


def test_backward_refuses_uncovered_shapes(bsa):
    q = torch.zeros(1, 512, 2, 64, device="cuda", dtype=torch.float32)
    idx = torch.zeros(1, 2, 8, 2, device="cuda", dtype=torch.int32)
    with pytest.raises(bsa.BsaError, match="UNSUPPORTED"):
        bsa.bsa_sparse_attn_fwd_train(q, q, q, idx, 64)  # float32 inputs


GQA_CASES = [  # (B, N, H, H_kv, D, block_size, ratio, causal)
    (1, 2048, 4, 2, 128, 128, 0.25, False),
    (1, 2048, 6, 2, 64, 128, 0.3, True),     # G = 3
    (2, 1024, 4, 1, 128, 256, 0.5, False),   # all query heads in one group, block_size 256
    (1, 2048, 4, 2, 64, 64, 0.3, True),      # block_size 64, causal
    (1, 1344, 6, 2, 128, 64, 0.25, False),   # block_size 64, G = 3, nb 21
]


@pytest.mark.parametrize("ci", range(len(GQA_CASES)))
def test_backward_gqa_matches_oracle(bsa, oracle_mod, ci):
    """Grouped queries: dq per query head, dk and dv per key/value head. The
    reference is the oracle's per-head backward with k and v repeated to the
    query heads and each query head given its group's index lists; the
    gradient of a shared k (or v) is the sum of those per-head gradients over
    its group, which is exact."""
    B, N, H, Hkv, D, bs, ratio, causal = GQA_CASES[ci]
    cfg = W.Config(f"bwdg{ci}", B, N, H, D, bs, ratio, "bf16", 1.0, 1500 + ci, None, H_kv=Hkv)
    q, k, v = W.make_inputs(cfg, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(1600 + ci)
    do = torch.randn(q.shape, generator=g, device="cuda").to(torch.bfloat16)
    flags = bsa.BSA_FLAG_CAUSAL if causal else 0
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(B, N, H, D, bs, ratio, H_kv=Hkv), device="cuda",
                     dtype=torch.uint8)
    bsa.bsa_forward(q, k, v, bs, ratio, workspace=ws, flags=flags)
    idx = bsa.workspace_views(ws, B, N, H, D, bs, ratio, H_kv=Hkv)[2].clone()  # [B, H_kv, nb, k]
    o, lse = bsa.bsa_sparse_attn_fwd_train(q, k, v, idx, bs, flags=flags)
    dq, dk, dv = bsa.bsa_sparse_attn_bwd(q, k, v, o, do, idx, lse, bs, flags=flags)
    torch.cuda.synchronize()
    assert bsa.bsa_device_error() == 0
    assert dk.shape == k.shape and dv.shape == v.shape
    G = H // Hkv
    qa, ka, va, doa = (_host(x) for x in (q, k, v, do))
    idx_q = np.repeat(idx.cpu().numpy(), G, axis=1)
    rows = np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (B, H, cfg.nb)).copy()
    check_output(gpu_rows(o, rows, bs), oracle_mod.sparse_attn_gqa(qa, ka, va, idx_q, bs, causal=causal), "bf16")
    ke, ve = np.repeat(ka, G, axis=2), np.repeat(va, G, axis=2)
    rq, rk, rv = oracle_mod.sparse_attn_bwd(qa, ke, ve, doa, idx_q, bs, causal=causal)
    rk = rk.reshape(B, N, Hkv, G, D).sum(axis=3)
    rv = rv.reshape(B, N, Hkv, G, D).sum(axis=3)
    check_grad(dq, rq, "dq")
    check_grad(dk, rk, "dk")
    check_grad(dv, rv, "dv")


def test_backward_dq_at_c3_size_on_sampled_query_blocks(bsa, oracle_mod):
    """The c3 workload (B=2 N=32768 H=16 D=128 block_size=128 k=51): dq of a
    sample of query blocks (two per (b, h)) against the oracle, which sums a
    query block's own contributions in full when it is in the sample."""
    cfg = W.CONFIGS["c3"]
    B, N, H, D, bs, ratio = cfg.B, cfg.N, cfg.H, cfg.D, cfg.block_size, cfg.topk_ratio
    q, k, v = W.make_inputs(cfg, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(1700)
    do = torch.randn(q.shape, generator=g, device="cuda").to(torch.bfloat16)
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(B, N, H, D, bs, ratio), device="cuda", dtype=torch.uint8)
    bsa.bsa_forward(q, k, v, bs, ratio, workspace=ws)
    idx = bsa.workspace_views(ws, B, N, H, D, bs, ratio)[2].clone()
    o, lse = bsa.bsa_sparse_attn_fwd_train(q, k, v, idx, bs)
    dq, _, _ = bsa.bsa_sparse_attn_bwd(q, k, v, o, do, idx, lse, bs)
    torch.cuda.synchronize()
    assert bsa.bsa_device_error() == 0
    rows = W.sample_query_blocks(cfg, count=2)
    rq, _, _ = oracle_mod.sparse_attn_bwd(_host(q), _host(k), _host(v), _host(do), idx.cpu().numpy(), bs, rows=rows)
    # the sampled rows of dq, [B, H, nrows * bs, D]
    tok = (rows[..., None] * bs + np.arange(bs)).reshape(B, H, -1)
    got = dq.to(torch.float64).cpu().numpy()
    g_rows = np.stack([np.stack([got[b, tok[b, h], h] for h in range(H)]) for b in range(B)])
    r_rows = np.stack([np.stack([rq[b, tok[b, h], h] for h in range(H)]) for b in range(B)])
    d = np.abs(g_rows - r_rows)
    rel = np.linalg.norm(g_rows - r_rows) / np.linalg.norm(r_rows)
    print(f"c3 dq (sampled): max|d| {d.max():.3g} (max|ref| {np.abs(r_rows).max():.3g}), rel L2 {rel:.3g}")
    assert rel <= 5e-3 and d.max() <= 2e-2 * np.abs(r_rows).max()
