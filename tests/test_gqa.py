"""GPU parity of the grouped-query variant (H query heads, H_kv key/value
heads) against the float64 oracle.

Readings ("从M2.7到M3：多模态模型稀疏注意力架构设计与实现全解析" §3.1, a GQA-based
attention block): query head h reads key/value head h // G (G = H / H_kv);
each key/value head has one selection per query block, scored with the
group's pooled query (the mean of its G heads' block means).

Pass rules as in test_parity.py. The score bound gains (G + 1) 2^-24 times
the heads' mean |qbar| . |kbar| for the float32 group mean (a sum of G pooled
rows, scaled by 1/G).
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


CASES = [  # (B, N, H, H_kv, D, block_size, ratio, dtype, causal)
    (1, 2048, 4, 2, 128, 128, 0.25, "bf16", False),  # G 2: two heads of a group per CTA
    (1, 2048, 8, 2, 128, 128, 0.25, "bf16", True),   # G 4, causal
    (2, 2048, 6, 2, 64, 128, 0.3, "bf16", False),    # G 3 (odd): two query blocks per CTA, D 64
    (1, 1920, 4, 1, 128, 128, 0.3, "bf16", False),   # G 4, odd nb
    (1, 1920, 4, 1, 128, 128, 0.3, "bf16", True),
    (1, 4096, 4, 2, 128, 256, 0.3, "bf16", False),   # block_size 256
    (2, 2048, 4, 2, 64, 64, 0.3, "bf16", True),      # block_size 64
    (1, 1024, 4, 2, 64, 64, 0.5, "f32", False),      # float32
    (1, 1024, 6, 3, 128, 64, 0.25, "f32", True),
]


def _cfg(case, seed):
    B, N, H, Hkv, D, bs, ratio, dt, _ = case
    return W.Config(f"gqa{seed}", B, N, H, D, bs, ratio, dt, 1.0, seed, None, H_kv=Hkv)


@pytest.mark.parametrize("ci", range(len(CASES)))
def test_gqa_full_path(bsa, oracle_mod, ci):
    causal = CASES[ci][-1]
    cfg = _cfg(CASES[ci], 800 + ci)
    B, N, H, Hkv, D, bs = cfg.B, cfg.N, cfg.H, cfg.Hkv, cfg.D, cfg.block_size
    q, k, v = W.make_inputs(cfg, device="cuda")
    assert k.shape == (B, N, Hkv, D)
    flags = bsa.BSA_FLAG_CAUSAL if causal else 0
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(B, N, H, D, bs, cfg.topk_ratio, H_kv=Hkv),
                     device="cuda", dtype=torch.uint8)
    o = bsa.bsa_forward(q, k, v, bs, cfg.topk_ratio, workspace=ws, flags=flags)
    torch.cuda.synchronize()
    assert bsa.bsa_device_error() == 0
    _, _, idx_g = bsa.workspace_views(ws, B, N, H, D, bs, cfg.topk_ratio, H_kv=Hkv)
    qa, ka, va = _host(q), _host(k), _host(v)
    ref = oracle_mod.forward_gqa(qa, ka, va, bs, cfg.topk_ratio, causal=causal)
    g = idx_g.cpu().numpy()
    if causal:
        accept_causal_rows(g, ref["scores"], cfg.k, ref["idx"], False)
    else:
        accept_index_rows(g, ref["scores"], cfg.k, ref["idx"])
    o_ref = oracle_mod.sparse_attn_gqa(qa, ka, va, np.repeat(g, H // Hkv, axis=1), bs, causal=causal)
    rows = np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (B, H, cfg.nb)).copy()
    check_output(gpu_rows(o, rows, bs), o_ref, cfg.dtype)


@pytest.mark.parametrize("H,Hkv,nb,D", [(4, 2, 100, 128), (8, 2, 300, 64), (6, 3, 1024, 128), (4, 1, 1501, 64)])
def test_gqa_scores_and_selection_stage(bsa, oracle_mod, H, Hkv, nb, D):
    """bsa_block_scores_topk on per-head pooled queries and per-group pooled
    keys: the group-mean scores within the float32 FFMA bound (plus the float32
    mean), the index lists by the near-tie rule."""
    B = 1
    rng = np.random.default_rng(nb + H)
    qp = (rng.standard_normal((B, H, nb, D)) * 0.3 + rng.standard_normal((B, H, nb, 1))).astype(np.float32)
    kp = (rng.standard_normal((B, Hkv, nb, D)) * 0.3 + rng.standard_normal((B, Hkv, nb, 1))).astype(np.float32)
    kk = max(1, nb // 7)
    idx, S = bsa.bsa_block_scores_topk(torch.from_numpy(qp).cuda(), torch.from_numpy(kp).cuda(), kk, scores=True)
    torch.cuda.synchronize()
    qg = oracle_mod.group_pool(qp.astype(np.float64), Hkv)
    S_ref = oracle_mod.block_scores(qg, kp.astype(np.float64))
    G = H // Hkv
    kabs = np.abs(kp.astype(np.float64)).transpose(0, 1, 3, 2)
    absdot = np.matmul(np.abs(qg), kabs)
    # the float32 group mean rounds relative to the mean of the heads' |qbar|
    absdot_heads = np.matmul(oracle_mod.group_pool(np.abs(qp.astype(np.float64)), Hkv), kabs)
    bound = D * 2.0 ** -24 * absdot + (G + 1) * 2.0 ** -24 * absdot_heads
    err = np.abs(S.cpu().numpy().astype(np.float64) - S_ref)
    print(f"G={G} nb={nb} D={D}: score error {(err / (absdot_heads + 1e-30)).max():.3g} x sum|q k|")
    assert np.all(err <= bound + 1e-30), f"score error {(err / (absdot + 1e-30)).max():.3g} x sum|q k|"
    accept_index_rows(idx.cpu().numpy(), S_ref, kk, oracle_mod.topk(S_ref, kk))


def test_gqa_one_head_per_group_matches_the_plain_entry_point(bsa):
    """H_kv = H through the grouped entry point is the plain method, bit for bit."""
    cfg = W.Config("gqa1", 1, 2048, 4, 128, 128, 0.25, "bf16", 1.0, 850, None)
    q, k, v = W.make_inputs(cfg, device="cuda")
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(1, 2048, 4, 128, 128, 0.25), device="cuda", dtype=torch.uint8)
    o1 = bsa.bsa_forward(q, k, v, 128, 0.25, workspace=ws)
    o2 = torch.empty_like(q)
    P = __import__("ctypes").c_void_p
    st = bsa.lib.bsa_forward_gqa(P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()), P(o2.data_ptr()), 1, 2048,
                                 4, 4, 128, 128, 0.25, 1, 0, P(ws.data_ptr()), ws.numel(),
                                 P(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
