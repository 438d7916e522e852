"""GPU parity of the causal variant (BSA_FLAG_CAUSAL, BSA_FLAG_FORCE_DIAG)
against the float64 oracle.

Readings (the mask of Softmax(Mask(QK^T/sqrt(d_k)))V on "从M2.7到M3：多模态模型稀疏
注意力架构设计与实现全解析" §2.1, made causal): query block i ranks only key blocks
j <= i and keeps min(k, i+1) of them (with the diagonal forced in when asked),
rows padded with -1; query token n never sees key token t > n.

Pass rules as in test_parity.py: index lists bit-exact except near ties
(tau = 1e-4 |t| around the k-th ranked score), outputs within the float32 /
bfloat16 tolerances against the oracle run on the GPU's lists.
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


def _flags(bsa, force_diag):
    return bsa.BSA_FLAG_CAUSAL | (bsa.BSA_FLAG_FORCE_DIAG if force_diag else 0)


def accept_causal_rows(gpu_idx, scores, k, oracle_idx, force_diag):
    """Causal index rows: exact where the oracle's list is not in a near tie;
    otherwise a valid causal list that keeps every candidate clearly above the
    oracle's last ranked score and none clearly below it. Row r of the
    all-rows score matrix is query block r % nb."""
    nb = scores.shape[-1]
    G = gpu_idx.reshape(-1, k)
    S = scores.reshape(-1, nb)
    O = oracle_idx.reshape(-1, k)
    for r in range(G.shape[0]):
        i = r % nb
        n = min(k, i + 1)
        g = G[r]
        assert np.all(g[n:] == -1), f"row {r}: padding"
        if np.array_equal(g, O[r]):
            continue
        v = g[:n]
        assert np.all(v >= 0) and np.all(v <= i), f"row {r}: ids outside [0, {i}]"
        assert np.all(np.diff(v) > 0), f"row {r}: ids not strictly ascending"
        if force_diag:
            assert v[-1] == i, f"row {r}: diagonal block missing"
            v = v[:-1]
        ncand = i if force_diag else i + 1
        cand = S[r, :ncand]
        if len(v) == 0:
            continue
        t = np.sort(cand)[::-1][len(v) - 1]
        tau = 1e-4 * abs(t)
        sel = np.zeros(ncand, bool)
        sel[v] = True
        assert np.all(sel[cand > t + tau]), f"row {r}: a block clearly above the cut is missing"
        assert not np.any(sel[cand < t - tau]), f"row {r}: a block clearly below the cut was kept"


CASES = [  # (B, N, H, D, block_size, ratio, dtype)
    (1, 2048, 2, 128, 128, 0.25, "bf16"),   # nb 16, k 4: rows 0-2 padded
    (2, 4096, 3, 64, 128, 0.3, "bf16"),     # D 64
    (1, 1920, 2, 128, 128, 0.4, "bf16"),    # odd nb: a CTA with one query tile
    (1, 4096, 2, 128, 256, 0.3, "bf16"),    # block_size 256: halves of the diagonal
    (2, 2048, 2, 64, 64, 0.3, "bf16"),      # block_size 64, odd k
    (1, 448, 2, 128, 64, 0.5, "bf16"),      # block_size 64, nb 7: stacked blocks with unequal counts
    (1, 1024, 2, 128, 128, 1.0, "bf16"),    # k = nb: dense causal attention
    (1, 1024, 2, 64, 64, 0.5, "f32"),       # float32 path
    (1, 512, 2, 128, 64, 0.25, "f32"),
]


def _cfg(case, seed):
    B, N, H, D, bs, ratio, dt = case
    return W.Config(f"causal{seed}", B, N, H, D, bs, ratio, dt, 1.0, seed, None)


@pytest.mark.parametrize("force_diag", [False, True])
@pytest.mark.parametrize("ci", range(len(CASES)))
def test_causal_full_path(bsa, oracle_mod, ci, force_diag):
    cfg = _cfg(CASES[ci], 500 + ci)
    B, N, H, D, bs = cfg.B, cfg.N, cfg.H, cfg.D, cfg.block_size
    q, k, v = W.make_inputs(cfg, device="cuda")
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(B, N, H, D, bs, cfg.topk_ratio), device="cuda",
                     dtype=torch.uint8)
    o = bsa.bsa_forward(q, k, v, bs, cfg.topk_ratio, workspace=ws, flags=_flags(bsa, force_diag))
    torch.cuda.synchronize()
    assert bsa.bsa_device_error() == 0
    _, _, idx_g = bsa.workspace_views(ws, B, N, H, D, bs, cfg.topk_ratio)
    qa, ka, va = _host(q), _host(k), _host(v)
    S = oracle_mod.block_scores(oracle_mod.block_pool(qa, bs), oracle_mod.block_pool(ka, bs))
    kk = cfg.k
    idx_o = oracle_mod.topk(S, kk, causal=True, force_diag=force_diag)
    g = idx_g.cpu().numpy()
    accept_causal_rows(g, S, kk, idx_o, force_diag)
    o_ref = oracle_mod.sparse_attn(qa, ka, va, g, bs, causal=True)
    rows = np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (B, H, cfg.nb)).copy()
    check_output(gpu_rows(o, rows, bs), o_ref, cfg.dtype)


@pytest.mark.parametrize("ci", [0, 2, 3, 4, 6])
def test_causal_attention_with_oracle_indices(bsa, oracle_mod, ci):
    """The attention kernel alone on the oracle's causal lists (padding
    included): isolates the token mask and the per-tile -1 handling."""
    cfg = _cfg(CASES[ci], 600 + ci)
    B, N, H, D, bs = cfg.B, cfg.N, cfg.H, cfg.D, cfg.block_size
    q, k, v = W.make_inputs(cfg, device="cuda")
    qa, ka, va = _host(q), _host(k), _host(v)
    S = oracle_mod.block_scores(oracle_mod.block_pool(qa, bs), oracle_mod.block_pool(ka, bs))
    for force_diag in (False, True):
        idx = oracle_mod.topk(S, cfg.k, causal=True, force_diag=force_diag)
        o = bsa.bsa_sparse_attn_fwd(q, k, v, torch.from_numpy(idx).cuda(), bs, flags=bsa.BSA_FLAG_CAUSAL)
        torch.cuda.synchronize()
        assert bsa.bsa_device_error() == 0
        o_ref = oracle_mod.sparse_attn(qa, ka, va, idx, bs, causal=True)
        rows = np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (B, H, cfg.nb)).copy()
        check_output(gpu_rows(o, rows, bs), o_ref, cfg.dtype)


@pytest.mark.parametrize("nb", [40, 100, 1024, 1501, 4500])
def test_causal_selection_on_integer_scores(bsa, oracle_mod, nb):
    """Integer-valued pooled inputs give exact scores with many ties: the
    causal index lists must equal the oracle's bit for bit (register paths,
    ragged rows and rows staged in shared memory)."""
    B, H, D = 1, 2, 64
    rng = np.random.default_rng(900 + nb)
    qp = rng.integers(-1, 2, (B, H, nb, D)).astype(np.float32)
    kp = rng.integers(-2, 3, (B, H, nb, D)).astype(np.float32)
    S_ref = oracle_mod.block_scores(qp.astype(np.float64), kp.astype(np.float64))
    for kk in sorted({1, 3, max(1, nb // 7), nb}):
        for force_diag in (False, True):
            idx = bsa.bsa_block_scores_topk(torch.from_numpy(qp).cuda(), torch.from_numpy(kp).cuda(), kk,
                                            flags=_flags(bsa, force_diag))
            torch.cuda.synchronize()
            want = oracle_mod.topk(S_ref, kk, causal=True, force_diag=force_diag)
            assert np.array_equal(idx.cpu().numpy(), want), f"k={kk} force_diag={force_diag}"


def test_causal_ratio_one_is_dense_causal_attention(bsa):
    """k = nb: every block j <= i is kept, so the output is dense causal
    attention (torch SDPA with is_causal, float32 math on the bf16 inputs)."""
    cfg = _cfg((1, 2048, 2, 128, 128, 1.0, "bf16"), 700)
    q, k, v = W.make_inputs(cfg, device="cuda")
    o = bsa.bsa_forward(q, k, v, 128, 1.0, flags=bsa.BSA_FLAG_CAUSAL)
    t = lambda x: x.float().permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=True).permute(0, 2, 1, 3)
    check_output(o.double().cpu().numpy(), ref.double().cpu().numpy(), "bf16")
