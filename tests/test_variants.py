"""GPU parity of the add-on variants against the float64 oracle.

Max pooling (BSA_FLAG_MAX_POOL; page "从M2.7到M3：多模态模型稀疏注意力架构设计与实现全解析",
§2.2, comparison table: block-based methods score a block by its
block-internal extreme value). Reading: the pooled vector of a block is its
element-wise maximum over the block's rows, for q and k alike; scores,
selection and attention are unchanged. The maximum of stored values is exact,
so the pooled tensors must equal the oracle's bit for bit; index lists follow
the near-tie rule and outputs the bf16 / f32 tolerances of test_parity.py.

Global heads (BSA_GLOBAL_HEAD_PERIOD(p); same page, §5.3): query heads
h % p == 0 attend to every key block, the others over their selection; the
oracle runs on index rows widened accordingly (FP8 inputs keep the FP8
tolerance of test_fp8.py).
"""
import numpy as np
import pytest
import torch

import workloads as W
from test_causal import accept_causal_rows
from test_parity import _host, accept_index_rows, check_output, gpu_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import block_sparse_attention_19_b200 as m

    return m


@pytest.mark.parametrize("case", [(2, 512, 3, 64, 64, "f32"), (1, 2048, 5, 128, 256, "bf16"),
                                  (3, 768, 7, 64, 128, "bf16"), (1, 1024, 2, 128, 128, "e4m3")],
                         ids=lambda c: "B{}N{}H{}D{}bs{}{}".format(*c))
def test_max_pool_stage_is_exact(bsa, oracle_mod, case):
    B, N, H, D, bs, dt = case
    cfg = W.Config("maxpool", B, N, H, D, bs, 0.5, dt, 1.0, 41, None)
    q, _, _ = W.make_inputs(cfg, device="cuda")
    p = bsa.bsa_block_pool(q, bs, flags=bsa.BSA_FLAG_MAX_POOL)
    torch.cuda.synchronize()
    want = oracle_mod.block_pool(_host(q), bs, pool="max")
    assert np.array_equal(p.cpu().numpy().astype(np.float64), want)


CASES = [  # (B, N, H, H_kv, D, block_size, ratio, dtype, causal)
    (2, 1024, 3, 3, 64, 64, 0.45, "bf16", False),    # block_size 64 (stacked query blocks)
    (1, 4096, 2, 2, 128, 128, 0.25, "bf16", False),
    (1, 4096, 2, 2, 128, 256, 0.3, "bf16", False),
    (1, 2048, 4, 2, 128, 128, 0.3, "bf16", False),   # grouped queries: group mean of the max-pooled queries
    (1, 3840, 2, 2, 64, 128, 0.3, "bf16", True),     # causal, odd nb
    (2, 512, 2, 2, 64, 64, 0.5, "f32", False),
    (1, 16384, 2, 2, 128, 128, 0.15, "bf16", False),  # nb = 128
]


@pytest.mark.parametrize("ci", range(len(CASES)))
def test_max_pool_full_path(bsa, oracle_mod, ci):
    B, N, H, Hkv, D, bs, ratio, dt, causal = CASES[ci]
    cfg = W.Config(f"maxpool{ci}", B, N, H, D, bs, ratio, dt, 1.0, 300 + ci, None, H_kv=Hkv)
    q, k, v = W.make_inputs(cfg, device="cuda")
    flags = bsa.BSA_FLAG_MAX_POOL | (bsa.BSA_FLAG_CAUSAL if causal else 0)
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(B, N, H, D, bs, ratio, H_kv=Hkv), device="cuda",
                     dtype=torch.uint8)
    o = bsa.bsa_forward(q, k, v, bs, ratio, workspace=ws, flags=flags)
    torch.cuda.synchronize()
    assert bsa.bsa_device_error() == 0
    qp_g, kp_g, idx_g = bsa.workspace_views(ws, B, N, H, D, bs, ratio, H_kv=Hkv)
    qa, ka, va = _host(q), _host(k), _host(v)
    ref = oracle_mod.forward_gqa(qa, ka, va, bs, ratio, causal=causal, pool="max")
    # the pooled tensors are exact
    assert np.array_equal(qp_g.cpu().numpy().astype(np.float64), ref["qp"])
    assert np.array_equal(kp_g.cpu().numpy().astype(np.float64), ref["kp"])
    g = idx_g.cpu().numpy()
    if causal:
        accept_causal_rows(g, ref["scores"], cfg.k, ref["idx"], False)
    else:
        accept_index_rows(g, ref["scores"], cfg.k, ref["idx"])
    o_ref = oracle_mod.sparse_attn_gqa(qa, ka, va, np.repeat(g, H // Hkv, axis=1), bs, causal=causal)
    rows = np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (B, H, cfg.nb)).copy()
    check_output(gpu_rows(o, rows, bs), o_ref, dt)


def test_max_pool_changes_the_selection(bsa):
    """On the synthetic inputs max and mean pooling keep different blocks in
    some rows (the flag reaches the kernels)."""
    cfg = W.Config("maxpool_diff", 1, 4096, 2, 128, 128, 0.25, "bf16", 1.0, 77, None)
    q, k, v = W.make_inputs(cfg, device="cuda")
    ws1, ws2 = (torch.empty(bsa.bsa_forward_workspace_bytes(1, 4096, 2, 128, 128, 0.25), device="cuda",
                            dtype=torch.uint8) for _ in range(2))
    bsa.bsa_forward(q, k, v, 128, 0.25, workspace=ws1)
    bsa.bsa_forward(q, k, v, 128, 0.25, workspace=ws2, flags=bsa.BSA_FLAG_MAX_POOL)
    torch.cuda.synchronize()
    i1 = bsa.workspace_views(ws1, 1, 4096, 2, 128, 128, 0.25)[2]
    i2 = bsa.workspace_views(ws2, 1, 4096, 2, 128, 128, 0.25)[2]
    assert not torch.equal(i1, i2)


# ---------------------------------------------------------------- global heads
# Reading ("从M2.7到M3" §5.3: one global head in every four): query head h is
# global when h % period == 0 and attends to every key block (blocks 0..i
# when causal); the other heads attend over their selection. The oracle runs
# on rows widened to nb entries: every block for global heads, the GPU's
# selection (near-tie rule as above) for the others.

GCASES = [  # (B, N, H, H_kv, D, block_size, ratio, dtype, causal, period)
    (1, 4096, 4, 4, 128, 128, 0.25, "bf16", False, 4),
    (1, 4096, 4, 2, 128, 128, 0.25, "bf16", False, 2),   # grouped queries: heads no longer paired in a CTA
    (2, 2048, 3, 3, 64, 64, 0.3, "bf16", True, 2),       # block_size 64 (stacked), causal
    (1, 4096, 4, 4, 64, 256, 0.3, "bf16", True, 4),      # block_size 256, causal
    (1, 1344, 2, 2, 64, 64, 0.3, "bf16", False, 1),      # every head dense, nb 21
    (1, 2048, 4, 4, 128, 128, 0.25, "e4m3", False, 4),
    (2, 512, 4, 4, 64, 64, 0.25, "f32", True, 4),
]


@pytest.mark.parametrize("ci", range(len(GCASES)))
def test_global_heads_full_path(bsa, oracle_mod, ci):
    B, N, H, Hkv, D, bs, ratio, dt, causal, period = GCASES[ci]
    cfg = W.Config(f"global{ci}", B, N, H, D, bs, ratio, dt, 1.0, 500 + ci, None, H_kv=Hkv)
    q, k, v = W.make_inputs(cfg, device="cuda")
    flags = bsa.BSA_GLOBAL_HEAD_PERIOD(period) | (bsa.BSA_FLAG_CAUSAL if causal else 0)
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(B, N, H, D, bs, ratio, H_kv=Hkv), device="cuda",
                     dtype=torch.uint8)
    o = bsa.bsa_forward(q, k, v, bs, ratio, workspace=ws, flags=flags)
    torch.cuda.synchronize()
    assert bsa.bsa_device_error() == 0
    g = bsa.workspace_views(ws, B, N, H, D, bs, ratio, H_kv=Hkv)[2].cpu().numpy()
    qa, ka, va = _host(q), _host(k), _host(v)
    ref = oracle_mod.forward_gqa(qa, ka, va, bs, ratio, causal=causal)
    if causal:
        accept_causal_rows(g, ref["scores"], cfg.k, ref["idx"], False)
    else:
        accept_index_rows(g, ref["scores"], cfg.k, ref["idx"])
    rows_w = oracle_mod.global_head_rows(np.repeat(g, H // Hkv, axis=1), cfg.nb, period, causal)
    o_ref = oracle_mod.sparse_attn_gqa(qa, ka, va, rows_w, bs, causal=causal)
    rows = np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (B, H, cfg.nb)).copy()
    got = gpu_rows(o, rows, bs)
    if dt == "e4m3":
        from test_fp8 import check_fp8_output
        q64, k64 = (x.to(torch.float64).cpu().numpy() for x in (q, k))
        vabs = np.abs(v.to(torch.float64).cpu().numpy())
        o_abs = oracle_mod.sparse_attn_gqa(q64, k64, vabs, rows_w, bs, causal=causal)
        check_fp8_output(got, o_ref, o_abs, vabs.max())
    else:
        check_output(got, o_ref, dt)


def test_global_heads_attention_entry_point_matches_dense_sdpa(bsa):
    """bsa_sparse_attn_fwd with every head global (period 1) is dense
    attention, whatever the index rows hold."""
    cfg = W.Config("global_sdpa", 1, 2048, 2, 128, 128, 0.25, "bf16", 1.0, 610, None)
    q, k, v = W.make_inputs(cfg, device="cuda")
    junk = torch.zeros((1, 2, cfg.nb, cfg.k), device="cuda", dtype=torch.int32)
    o = bsa.bsa_sparse_attn_fwd(q, k, v, junk, 128, flags=bsa.BSA_GLOBAL_HEAD_PERIOD(1))
    torch.cuda.synchronize()
    t = lambda x: x.to(torch.float64).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v)).permute(0, 2, 1, 3)
    d = (o.to(torch.float64) - ref).abs()
    rel = (torch.linalg.vector_norm(o.to(torch.float64) - ref) / torch.linalg.vector_norm(ref)).item()
    assert d.max().item() <= 2e-2 and rel <= 5e-3


def test_training_entry_points_refuse_global_heads(bsa):
    cfg = W.Config("global_train", 1, 1024, 2, 64, 128, 0.25, "bf16", 1.0, 611, None)
    q, k, v = W.make_inputs(cfg, device="cuda")
    idx = torch.zeros((1, 2, cfg.nb, cfg.k), device="cuda", dtype=torch.int32)
    with pytest.raises(bsa.BsaError, match="UNSUPPORTED"):
        bsa.bsa_sparse_attn_fwd_train(q, k, v, idx, 128, flags=bsa.BSA_GLOBAL_HEAD_PERIOD(2))


# ---------------------------------------------------------------- overlapping key windows
# Reading ("从M2.7到M3" §5.3, overlap_ratio = 0.25): key windows of block_size
# tokens overlap by ov = int(overlap_ratio * block_size) tokens (window e
# starts at min(e (block_size - ov), N - block_size)); query blocks stay
# disjoint; each row attends to the union of its kept windows' tokens. The
# oracle attends over explicit token sets built from the GPU's window lists.

OCASES = [  # (B, N, H, H_kv, D, block_size, ratio, overlap_ratio, dtype, flags)
    (1, 4096, 2, 2, 128, 128, 0.25, 0.25, "bf16", 0),
    (2, 2048, 3, 3, 64, 64, 0.3, 0.25, "bf16", 0),     # block_size 64 (stacked), 43 windows of 64
    (1, 4096, 2, 2, 128, 256, 0.3, 0.25, "bf16", 0),
    (1, 4096, 2, 2, 64, 256, 0.5, 0.6, "bf16", 0),     # overlap 153 > 128: a window's whole first tile repeats
    (1, 2048, 4, 2, 128, 128, 0.3, 0.25, "bf16", 0),   # grouped queries, heads paired in a CTA
    (1, 2048, 4, 4, 64, 128, 0.3, 0.25, "bf16", 0x200),  # global heads every 2
    (2, 512, 2, 2, 64, 64, 0.4, 0.25, "f32", 0),
    (1, 2048, 2, 2, 64, 128, 0.3, 0.25, "e4m3", 0),
    (1, 8192, 2, 2, 64, 64, 0.3, 0.25, "bf16", 0),     # the page's block size: last window moved back
]


@pytest.mark.parametrize("ci", range(len(OCASES)))
def test_overlap_full_path(bsa, oracle_mod, ci):
    B, N, H, Hkv, D, bs, ratio, ovr, dt, flags = OCASES[ci]
    cfg = W.Config(f"ovl{ci}", B, N, H, D, bs, ratio, dt, 1.0, 700 + ci, None, H_kv=Hkv)
    q, k, v = W.make_inputs(cfg, device="cuda")
    ws = torch.empty(bsa.bsa_forward_overlap_workspace_bytes(B, N, H, D, bs, ratio, ovr, H_kv=Hkv), device="cuda",
                     dtype=torch.uint8)
    o = bsa.bsa_forward_overlap(q, k, v, bs, ratio, ovr, workspace=ws, flags=flags)
    torch.cuda.synchronize()
    assert bsa.bsa_device_error() == 0
    qa, ka, va = _host(q), _host(k), _host(v)
    ref = oracle_mod.forward_overlap(qa, ka, va, bs, ratio, ovr)
    nbk = bsa.bsa_overlap_window_count(N, bs, ovr)
    assert nbk == ref["nbk"]
    _, kp_g, idx_g, _ = bsa.overlap_workspace_views(ws, B, N, H, D, bs, ratio, ovr, H_kv=Hkv)
    # window means: float32 sums of block_size values
    absmean = oracle_mod.window_pool(np.abs(k.to(torch.float64).cpu().numpy()), bs, ref["ov"])
    err = np.abs(kp_g.cpu().numpy().astype(np.float64) - ref["kp"])
    assert np.all(err <= (bs - 1) * 2.0 ** -24 * absmean * 1.0001 + 1e-30)
    g = idx_g.cpu().numpy()
    assert g.shape[-1] == ref["k"]
    accept_index_rows(g, ref["scores"], ref["k"], ref["idx"])
    # the union of the GPU's kept windows (global heads: every token)
    sets = oracle_mod.window_token_sets(g, N, bs, ref["ov"])
    o_ref = oracle_mod.attend_token_sets(qa, ka, va, sets, bs)
    if flags:
        period = flags >> 8
        dense = oracle_mod.attend_token_sets(qa, ka, va, [[[np.arange(N)] * cfg.nb] * Hkv] * B, bs)
        for h in range(0, H, period):
            o_ref[:, h] = dense[:, h]
    rows = np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (B, H, cfg.nb)).copy()
    got = gpu_rows(o, rows, bs)
    if dt == "e4m3":
        from test_fp8 import check_fp8_output
        q64, k64 = (x.to(torch.float64).cpu().numpy() for x in (q, k))
        vabs = np.abs(v.to(torch.float64).cpu().numpy())
        check_fp8_output(got, o_ref, oracle_mod.attend_token_sets(q64, k64, vabs, sets, bs), vabs.max())
    else:
        check_output(got, o_ref, dt)


def test_overlap_zero_is_the_plain_path(bsa):
    cfg = W.Config("ovl0", 1, 4096, 2, 128, 128, 0.25, "bf16", 1.0, 730, None)
    q, k, v = W.make_inputs(cfg, device="cuda")
    a = bsa.bsa_forward(q, k, v, 128, 0.25)
    b = bsa.bsa_forward_overlap(q, k, v, 128, 0.25, 0.0)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("bs,D", [(64, 64), (128, 128), (256, 64)])
def test_overlap_attention_alone_with_adjacent_windows(bsa, oracle_mod, bs, D):
    """bsa_sparse_attn_fwd_overlap on window lists made of runs of adjacent
    windows, so most kept windows share tokens with the previous one."""
    N, H, ovr = 4096, 2, 0.25
    cfg = W.Config("ovl_attn", 1, N, H, D, bs, 0.25, "bf16", 1.0, 740 + bs, None)
    q, k, v = W.make_inputs(cfg, device="cuda")
    nbk = bsa.bsa_overlap_window_count(N, bs, ovr)
    rng = np.random.default_rng(bs)
    kk = 6
    idx = np.empty((1, H, cfg.nb, kk), np.int32)
    for h in range(H):
        for i in range(cfg.nb):
            s0, s1 = sorted(rng.choice(nbk - 3, 2, replace=False))
            idx[0, h, i] = np.unique(np.concatenate([np.arange(s0, s0 + 3), np.arange(s1, s1 + 3)]))[:kk] \
                if s1 >= s0 + 3 else np.arange(s0, s0 + kk) % nbk
            idx[0, h, i] = np.sort(idx[0, h, i])
    o = bsa.bsa_sparse_attn_fwd_overlap(q, k, v, torch.from_numpy(idx).cuda(), bs, ovr)
    torch.cuda.synchronize()
    assert bsa.bsa_device_error() == 0
    sets = oracle_mod.window_token_sets(idx, N, bs, int(ovr * bs))
    o_ref = oracle_mod.attend_token_sets(_host(q), _host(k), _host(v), sets, bs)
    rows = np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (1, H, cfg.nb)).copy()
    check_output(gpu_rows(o, rows, bs), o_ref, "bf16")
