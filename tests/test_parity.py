"""GPU parity: every stage of the CUDA path against the float64 oracle.

Rules (from the method's definition and its pass criteria):
* pooled means: float32 summation error bound (bs - 1) * 2^-24 * mean|x|;
* block scores: they are computed on the tensor cores from a split of each
  float32 operand into two TF32 parts (three products, float32 accumulation)
  and must stay within the worst-case error of a float32 FFMA dot product of
  length D, D * 2^-24 * sum_d |qbar_d kbar_d| (the float32 accuracy the
  scores are meant to have);
* index lists: bit-exact, except that a key block whose oracle score lies
  within tau = 1e-4 * |t| of the oracle's k-th largest score t may be swapped
  (such a row must still hold k distinct ascending ids, contain every block
  above t + tau and none below t - tau); the oracle's attention is then
  computed with the GPU's list;
* outputs: float32 max|d| <= 1e-4; bfloat16 max|d| <= 2e-2 and relative L2
  <= 5e-3, against the oracle on the same (rounded) inputs.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


@pytest.fixture(scope="module")
def bsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import block_sparse_attention_19_b200 as m

    return m


def _host(x):
    return W.to_oracle_array(x)


def _as_f64(x: torch.Tensor) -> np.ndarray:
    return x.detach().to("cpu", torch.float64).numpy()


def check_pool(gpu_pooled: torch.Tensor, x: torch.Tensor, ref: np.ndarray, bs: int):
    B, N, H, D = x.shape
    absmean = np.abs(_as_f64(x)).reshape(B, N // bs, bs, H, D).mean(2).transpose(0, 2, 1, 3)
    bound = (bs - 1) * U32 * absmean * 1.0001 + 1e-30
    err = np.abs(_as_f64(gpu_pooled) - ref)
    assert np.all(err <= bound), f"pool error {err.max()} above bound"


def accept_index_rows(gpu_idx: np.ndarray, scores: np.ndarray, k: int, oracle_idx: np.ndarray):
    """Near-tie acceptance of GPU index rows against oracle scores. Returns the
    number of rows that differ from the oracle's (all of them accepted)."""
    nb = scores.shape[-1]
    G = gpu_idx.reshape(-1, k)
    S = scores.reshape(-1, nb)
    O = oracle_idx.reshape(-1, k)
    differ = 0
    for r in range(G.shape[0]):
        g = G[r]
        if np.array_equal(g, O[r]):
            continue
        differ += 1
        assert np.all(g >= 0) and np.all(g < nb), f"row {r}: ids out of range"
        assert np.all(np.diff(g) > 0), f"row {r}: ids not strictly ascending"
        t = np.sort(S[r])[::-1][k - 1]
        tau = 1e-4 * abs(t)
        sel = np.zeros(nb, bool)
        sel[g] = True
        must = S[r] > t + tau
        never = S[r] < t - tau
        assert np.all(sel[must]), f"row {r}: a block clearly above the k-th score is missing"
        assert not np.any(sel[never]), f"row {r}: a block clearly below the k-th score was kept"
    return differ


def check_output(o_gpu: np.ndarray, o_ref: np.ndarray, dtype: str):
    d = np.abs(o_gpu - o_ref)
    if dtype == "f32":
        assert d.max() <= 1e-4, f"max|d| = {d.max()}"
    else:
        rel = np.linalg.norm(o_gpu - o_ref) / np.linalg.norm(o_ref)
        print(f"{dtype}: max|d| {d.max():.3g}, rel L2 {rel:.3g}")
        assert d.max() <= 2e-2, f"max|d| = {d.max()}"
        assert rel <= 5e-3, f"rel L2 = {rel}"


def gpu_rows(o: torch.Tensor, rows: np.ndarray, bs: int) -> np.ndarray:
    """GPU output [B,N,H,D] gathered to the oracle's [B,H,nrows,bs,D] for `rows`."""
    B, N, H, D = o.shape
    ob = o.view(B, N // bs, bs, H, D).permute(0, 3, 1, 2, 4)  # [B,H,nb,bs,D]
    r = torch.as_tensor(rows, device=o.device, dtype=torch.long)
    g = torch.gather(ob, 2, r[..., None, None].expand(B, H, rows.shape[-1], bs, D))
    return g.to(torch.float64).cpu().numpy()


# ------------------------------------------------------------------ full path on the configs

def run_config(bsa, oracle_mod, cfg: W.Config, rows=None):
    q, k, v = W.make_inputs(cfg, device="cuda")
    B, N, H, D, bs = cfg.B, cfg.N, cfg.H, cfg.D, cfg.block_size
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(B, N, H, D, bs, cfg.topk_ratio), device="cuda",
                     dtype=torch.uint8)
    o = bsa.bsa_forward(q, k, v, bs, cfg.topk_ratio, workspace=ws)
    torch.cuda.synchronize()
    assert bsa.bsa_device_error() == 0
    qp_g, kp_g, idx_g = bsa.workspace_views(ws, B, N, H, D, bs, cfg.topk_ratio)
    rows = W.sample_query_blocks(cfg) if rows is None else rows
    qa, ka, va = _host(q), _host(k), _host(v)
    qp = oracle_mod.block_pool(qa, bs)
    kp = oracle_mod.block_pool(ka, bs)
    check_pool(qp_g, q, qp, bs)
    check_pool(kp_g, k, kp, bs)
    S = oracle_mod.block_scores(qp, kp, rows)
    kk = oracle_mod.topk_count(cfg.nb, cfg.topk_ratio)
    assert kk == cfg.k == idx_g.shape[-1]
    idx_o = oracle_mod.topk(S, kk)
    r_t = torch.as_tensor(rows, device="cuda", dtype=torch.long)
    g_idx = torch.gather(idx_g, 2, r_t[..., None].expand(B, H, rows.shape[-1], kk)).cpu().numpy()
    accept_index_rows(g_idx, S, kk, idx_o)
    o_ref = oracle_mod.sparse_attn(qa, ka, va, g_idx, bs, rows=rows)
    check_output(gpu_rows(o, rows, bs), o_ref, cfg.dtype)
    return o


@pytest.mark.parametrize("name", ["c1", "c2", "c3", "c4", "c5"])
def test_config_parity(bsa, oracle_mod, name):
    cfg = W.CONFIGS[name]
    run_config(bsa, oracle_mod, cfg)


def test_c1_ratio_one_is_dense_attention(bsa, oracle_mod):
    cfg = W.CONFIGS["c1"].with_ratio(1.0)
    o = run_config(bsa, oracle_mod, cfg)
    q, k, v = W.make_inputs(cfg, device="cuda")
    t = lambda x: x.to(torch.float64).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v)).permute(0, 2, 1, 3)
    assert (o.to(torch.float64) - ref).abs().max().item() <= 1e-4


# ------------------------------------------------------------------ stage by stage, small shapes

SMALL = [  # (B, N, H, D, bs, ratio, dtype) spanning several key tiles and a ragged tail
    (2, 1024, 3, 64, 64, 0.45, "bf16"),   # k = 7: odd, last tile has 64 keys
    (1, 2048, 2, 128, 64, 0.5, "bf16"),   # k = 16
    (2, 1024, 2, 64, 128, 0.5, "bf16"),   # k = 4
    (1, 2048, 3, 128, 128, 0.3, "bf16"),  # k = 4
    (1, 2048, 2, 64, 256, 0.5, "bf16"),   # k = 4, two parts and two tiles per block
    (1, 4096, 2, 128, 256, 0.25, "bf16"),  # k = 4
    (1, 512, 2, 128, 128, 1.0, "bf16"),   # k = nb (dense)
    (1, 1024, 1, 128, 128, 0.125, "bf16"),  # k = 1
    (1, 256, 2, 64, 256, 1.0, "bf16"),    # nb = 1
    # block_size 64 stacks query blocks 4u..4u+3 in one CTA: counts that leave
    # blocks absent
    (1, 64, 2, 64, 64, 1.0, "bf16"),      # nb = 1
    (1, 192, 2, 64, 64, 0.67, "bf16"),    # nb = 3: second stream with one block
    (2, 320, 2, 128, 64, 0.4, "bf16"),    # nb = 5: a CTA with one block
    (1, 384, 3, 64, 64, 0.5, "bf16"),     # nb = 6: a CTA with one stream
    (2, 512, 3, 64, 64, 0.5, "f32"),
    (1, 1024, 2, 128, 128, 0.5, "f32"),
    (1, 1024, 2, 64, 256, 0.5, "f32"),
]


def _small_cfg(case, seed=7, sigma=1.0):
    B, N, H, D, bs, ratio, dt = case
    return W.Config("small", B, N, H, D, bs, ratio, dt, sigma, seed, None)


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "B{}N{}H{}D{}bs{}r{}{}".format(*c))
def test_small_full_path(bsa, oracle_mod, case):
    run_config(bsa, oracle_mod, _small_cfg(case))


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "B{}N{}H{}D{}bs{}r{}{}".format(*c))
def test_attention_with_oracle_indices(bsa, oracle_mod, case):
    """bsa_sparse_attn_fwd alone, fed random (non-contiguous) ascending index lists."""
    cfg = _small_cfg(case, seed=11)
    q, k, v = W.make_inputs(cfg, device="cuda")
    rng = np.random.default_rng(5)
    kk = cfg.k
    idx = np.sort(np.stack([[[rng.choice(cfg.nb, kk, replace=False) for _ in range(cfg.nb)]
                             for _ in range(cfg.H)] for _ in range(cfg.B)]), -1).astype(np.int32)
    o = bsa.bsa_sparse_attn_fwd(q, k, v, torch.from_numpy(idx).cuda(), cfg.block_size)
    torch.cuda.synchronize()
    assert bsa.bsa_device_error() == 0
    ref = oracle_mod.sparse_attn(_host(q), _host(k), _host(v), idx, cfg.block_size)
    check_output(gpu_rows(o, np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (cfg.B, cfg.H, cfg.nb)).copy(),
                          cfg.block_size), ref, cfg.dtype)


@pytest.mark.parametrize("nb,D", [(8, 64), (100, 128), (300, 64), (1024, 128), (1501, 64), (4096, 128),
                                  (4500, 64), (8192, 64)])
def test_scores_topk_stage(bsa, oracle_mod, nb, D):
    """bsa_block_scores_topk fed float32 pooled inputs: scores within the
    float32 FFMA bound, index lists by the near-tie rule (ragged tiles, rows
    of up to 4096 keys in registers, rows of up to 6400 keys staged in shared
    memory, longer rows searched from L2, odd nb)."""
    B, H = 1, 2
    rng = np.random.default_rng(nb)
    qp = (rng.standard_normal((B, H, nb, D)) * 0.3 + rng.standard_normal((B, H, nb, 1))).astype(np.float32)
    kp = (rng.standard_normal((B, H, nb, D)) * 0.3 + rng.standard_normal((B, H, nb, 1))).astype(np.float32)
    for kk in sorted({1, max(1, nb // 7), nb}):
        idx, S = bsa.bsa_block_scores_topk(torch.from_numpy(qp).cuda(), torch.from_numpy(kp).cuda(), kk, scores=True)
        torch.cuda.synchronize()
        S_ref = oracle_mod.block_scores(qp.astype(np.float64), kp.astype(np.float64))
        absdot = np.matmul(np.abs(qp.astype(np.float64)), np.abs(kp.astype(np.float64)).transpose(0, 1, 3, 2))
        err = np.abs(S.cpu().numpy().astype(np.float64) - S_ref)
        rel = (err / (absdot + 1e-30)).max()
        print(f"nb={nb} D={D} k={kk}: score error {rel:.3g} x sum|q k| (2^{np.log2(rel + 1e-300):.1f})")
        # the float32 FFMA bound; a dropped cross term (hi.lo) of the split
        # would show up at about 2^-11
        assert np.all(err <= D * U32 * absdot + 1e-30), f"score error {rel:.3g} x sum|q k|"
        idx_ref = oracle_mod.topk(S_ref, kk)
        accept_index_rows(idx.cpu().numpy(), S_ref, kk, idx_ref)


@pytest.mark.parametrize("nb", [40, 100, 1024, 1501, 4500, 8192])
def test_integer_scores_with_many_ties(bsa, oracle_mod, nb):
    """Small-integer pooled inputs make every score an exact integer (or a
    zero of either sign), so ties straddle the k-th score in most rows: the
    index lists must equal the oracle's bit-exactly, lower ids winning, and
    -0 must tie with +0."""
    B, H, D = 1, 2, 64
    rng = np.random.default_rng(77 + nb)
    qp = rng.integers(-1, 2, (B, H, nb, D)).astype(np.float32)
    kp = rng.integers(-2, 3, (B, H, nb, D)).astype(np.float32)
    kp[:, :, ::7] = -0.0  # rows of negative zeros: their scores are zeros of either sign
    kp[:, :, 3::7] = 0.0
    S_ref = oracle_mod.block_scores(qp.astype(np.float64), kp.astype(np.float64))
    for kk in sorted({1, max(1, nb // 7), nb // 2, nb}):
        idx, S = bsa.bsa_block_scores_topk(torch.from_numpy(qp).cuda(), torch.from_numpy(kp).cuda(), kk,
                                           scores=True)
        torch.cuda.synchronize()
        assert np.array_equal(S.cpu().numpy().astype(np.float64), S_ref)  # exact: integers below 2^24
        assert np.array_equal(idx.cpu().numpy(), oracle_mod.topk(S_ref, kk)), f"k={kk}"


def test_exact_score_ties_pick_lower_block(bsa, oracle_mod):
    """Duplicated key blocks give exactly equal pooled keys, hence exact score
    ties on both sides: the lower block id must win, bit-exactly."""
    cfg = _small_cfg((1, 2048, 2, 128, 128, 0.25, "bf16"), seed=3)
    q, k, v = W.make_inputs(cfg, device="cuda")
    bs = cfg.block_size
    kb = k.view(cfg.B, cfg.nb, bs, cfg.H, cfg.D)
    kb[:, 9] = kb[:, 2]
    kb[:, 14] = kb[:, 2]
    kb[:, 5] = kb[:, 11]
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(cfg.B, cfg.N, cfg.H, cfg.D, bs, cfg.topk_ratio),
                     device="cuda", dtype=torch.uint8)
    o = bsa.bsa_forward(q, k, v, bs, cfg.topk_ratio, workspace=ws)
    torch.cuda.synchronize()
    _, _, idx_g = bsa.workspace_views(ws, cfg.B, cfg.N, cfg.H, cfg.D, bs, cfg.topk_ratio)
    qa, ka, va = _host(q), _host(k), _host(v)
    S = oracle_mod.block_scores(oracle_mod.block_pool(qa, bs), oracle_mod.block_pool(ka, bs))
    idx_o = oracle_mod.topk(S, cfg.k)
    g = idx_g.cpu().numpy()
    assert np.array_equal(g, idx_o)
    # the duplicated blocks (2, 9, 14) and (5, 11) never appear as the higher
    # copy without the lower one
    for row in g.reshape(-1, cfg.k):
        s = set(row.tolist())
        assert not ({9, 14} & s) or 2 in s
        assert 11 not in s or 5 in s
    ref = oracle_mod.sparse_attn(qa, ka, va, g, bs)
    check_output(gpu_rows(o, np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (1, 2, cfg.nb)).copy(), bs),
                 ref, "bf16")


def test_constant_scores_select_lowest_blocks(bsa, oracle_mod):
    """All block scores equal (constant k): every row keeps blocks 0..k-1."""
    cfg = _small_cfg((1, 1024, 2, 64, 64, 0.25, "bf16"), seed=4)
    q, _, v = W.make_inputs(cfg, device="cuda")
    k = torch.full_like(q, 0.5)
    ws = torch.empty(bsa.bsa_forward_workspace_bytes(1, 1024, 2, 64, 64, 0.25), device="cuda", dtype=torch.uint8)
    bsa.bsa_forward(q, k, v, 64, 0.25, workspace=ws)
    torch.cuda.synchronize()
    _, _, idx_g = bsa.workspace_views(ws, 1, 1024, 2, 64, 64, 0.25)
    want = np.broadcast_to(np.arange(cfg.k, dtype=np.int32), idx_g.shape)
    assert np.array_equal(idx_g.cpu().numpy(), want)


def test_large_logits_exercise_rescaling(bsa, oracle_mod):
    """Logits spread over tens of units with the largest blocks last, so the
    running max moves several times along a row (output rescaling path)."""
    cfg = _small_cfg((1, 4096, 2, 128, 128, 0.5, "bf16"), seed=9)
    q, k, v = W.make_inputs(cfg, device="cuda")
    ramp = torch.linspace(0.2, 3.0, cfg.nb, device="cuda").repeat_interleave(cfg.block_size)
    q = (q.float() * 2.5).to(torch.bfloat16)
    k = (k.float() * ramp[None, :, None, None]).to(torch.bfloat16)
    rng = np.random.default_rng(2)
    idx = np.sort(np.stack([[[rng.choice(cfg.nb, cfg.k, replace=False) for _ in range(cfg.nb)]
                             for _ in range(cfg.H)]]), -1).astype(np.int32)
    o = bsa.bsa_sparse_attn_fwd(q, k, v, torch.from_numpy(idx).cuda(), cfg.block_size)
    torch.cuda.synchronize()
    ref = oracle_mod.sparse_attn(_host(q), _host(k), _host(v), idx, cfg.block_size)
    check_output(gpu_rows(o, np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (1, 2, cfg.nb)).copy(),
                          cfg.block_size), ref, "bf16")


def test_pool_stage_alone(bsa, oracle_mod):
    for case in [(2, 512, 3, 64, 64, 0.5, "f32"), (1, 2048, 5, 128, 256, 0.5, "bf16"),
                 (3, 768, 7, 64, 128, 0.5, "bf16")]:
        cfg = _small_cfg(case, seed=13)
        q, _, _ = W.make_inputs(cfg, device="cuda")
        p = bsa.bsa_block_pool(q, cfg.block_size)
        torch.cuda.synchronize()
        check_pool(p, q, oracle_mod.block_pool(_host(q), cfg.block_size), cfg.block_size)


@pytest.mark.parametrize("H,Hkv", [(3, 3), (4, 2)])
def test_pool_qk_matches_separate_pooling(bsa, H, Hkv):
    """bsa_block_pool_qk (one launch for q and k when H = H_kv) gives the same
    bits as pooling each tensor alone."""
    cfg = W.Config("poolqk", 2, 2048, H, 128, 128, 0.5, "bf16", 1.0, 15, None, H_kv=Hkv)
    q, k, _ = W.make_inputs(cfg, device="cuda")
    qp, kp = bsa.bsa_block_pool_qk(q, k, 128)
    torch.cuda.synchronize()
    assert torch.equal(qp, bsa.bsa_block_pool(q, 128)) and torch.equal(kp, bsa.bsa_block_pool(k, 128))


def test_repeat_calls_are_deterministic(bsa):
    cfg = _small_cfg((1, 2048, 2, 128, 128, 0.3, "bf16"), seed=21)
    q, k, v = W.make_inputs(cfg, device="cuda")
    a = bsa.bsa_forward(q, k, v, 128, 0.3)
    b = bsa.bsa_forward(q, k, v, 128, 0.3)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
