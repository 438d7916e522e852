"""Sizes past 32-bit element offsets: q, k, v of more than 2^31 elements.

B = 3, N = 2^20, H = 8, D = 128 (3 * 2^30 elements per tensor, 6.4 GB in
bfloat16), block_size 256 (nb = 4096), topk_ratio 0.02 (k = 81): the last
batch entry's rows lie beyond element 2^31 of q, k, v and o (byte offsets
past 2^32). The whole path runs on the GPU. The (b, h)
problems of the method are independent (pooling, scores, selection and
attention never mix heads or batch entries), so the oracle checks the slices
with the largest offsets on their own: pooled means in full, and the index
rows and outputs of sampled query blocks, the last block included.
"""
import numpy as np
import pytest
import torch

import workloads as W
from test_parity import accept_index_rows, check_output, check_pool, gpu_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import block_sparse_attention_19_b200 as m

    return m


def test_offsets_past_2_31_elements(bsa, oracle_mod):
    cfg = W.Config("large", 3, 1 << 20, 8, 128, 256, 0.02, "bf16", 1.0, 23, None)
    B, N, H, D, bs = cfg.B, cfg.N, cfg.H, cfg.D, cfg.block_size
    assert B * N * H * D > 2 ** 31
    q, k, v = W.make_inputs(cfg, device="cuda")
    torch.cuda.empty_cache()
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(B, N, H, D, bs, cfg.topk_ratio), device="cuda",
                     dtype=torch.uint8)
    o = bsa.bsa_forward(q, k, v, bs, cfg.topk_ratio, workspace=ws)
    torch.cuda.synchronize()
    assert bsa.bsa_device_error() == 0
    qp_g, kp_g, idx_g = bsa.workspace_views(ws, B, N, H, D, bs, cfg.topk_ratio)
    kk = oracle_mod.topk_count(cfg.nb, cfg.topk_ratio)
    assert kk == idx_g.shape[-1] == 81
    rng = np.random.default_rng(cfg.seed + 1000)
    for b, h in [(B - 1, H - 1), (B - 1, 0), (0, H - 1)]:
        def one(x):  # the (b, h) problem as a [1, N, 1, D] tensor
            return x[b:b + 1, :, h:h + 1, :].contiguous()

        qa, ka, va = W.to_oracle_array(one(q)), W.to_oracle_array(one(k)), W.to_oracle_array(one(v))
        qp = oracle_mod.block_pool(qa, bs)
        kp = oracle_mod.block_pool(ka, bs)
        check_pool(qp_g[b:b + 1, h:h + 1], one(q), qp, bs)
        check_pool(kp_g[b:b + 1, h:h + 1], one(k), kp, bs)
        picks = rng.choice(cfg.nb - 1, size=5, replace=False)
        rows = np.sort(np.append(picks, cfg.nb - 1)).astype(np.int32)[None, None, :]
        S = oracle_mod.block_scores(qp, kp, rows)
        idx_o = oracle_mod.topk(S, kk)
        r_t = torch.as_tensor(rows[0, 0], device="cuda", dtype=torch.long)
        g_idx = idx_g[b, h].index_select(0, r_t).cpu().numpy()[None, None]
        accept_index_rows(g_idx, S, kk, idx_o)
        o_ref = oracle_mod.sparse_attn(qa, ka, va, g_idx, bs, rows=rows)
        check_output(gpu_rows(one(o), rows, bs), o_ref, "bf16")
