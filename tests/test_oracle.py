"""Pins for the float64 oracle (CPU only).

Every oracle function is checked against something other than itself: a
hand-worked case with closed-form answers, library routines (numpy matmul,
numpy lexsort, torch scaled_dot_product_attention in float64), brute force on
tiny inputs and invariants of the definition.  The definition is the one on
"2026 新一代卷积与 Transformer 网络架构" (qqiyuan.cn), section
"SparseFormer 注意力实现", with the mask formula of
"从M2.7到M3：多模态模型稀疏注意力架构设计与实现全解析" §2.1.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))


def _rand(shape, seed, offsets=True, bs=None):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape)
    if offsets and bs:
        B, N, H, D = shape
        off = rng.standard_normal((B, N // bs, 1, H, D))
        x = (x.reshape(B, N // bs, bs, H, D) + off).reshape(shape)
    return x


def _closed(expr):
    return eval(expr, {"exp": math.exp})


# ---------------------------------------------------------------- hand-worked

def test_hw1_hand_worked(oracle_mod):
    g = json.load(open(os.path.join(HERE, "golden", "hw1.json")))
    shp = (g["B"], g["N"], g["H"], g["D"])
    q = np.array(g["q"], np.float64).reshape(shp)
    k = np.array(g["k"], np.float64).reshape(shp)
    v = np.array(g["v"], np.float64).reshape(shp)
    bs = g["block_size"]
    r = oracle_mod.forward(q, k, v, bs, g["topk_ratio"])
    assert r["k"] == g["k_selected"]
    np.testing.assert_array_equal(r["qp"][0, 0, :, 0], g["q_pooled"])
    np.testing.assert_array_equal(r["kp"][0, 0, :, 0], g["k_pooled"])
    np.testing.assert_array_equal(r["scores"][0, 0], g["scores"])
    np.testing.assert_array_equal(r["idx"][0, 0], g["idx"])
    o = oracle_mod.o_to_bnhd(r["o"]).reshape(-1)
    want = [_closed(e) for e in g["o_closed_form"]]
    np.testing.assert_allclose(o, want, rtol=1e-15, atol=0)
    # ratio 1.0: row 0 attends to every token (dense)
    rd = oracle_mod.forward(q, k, v, bs, 1.0)
    np.testing.assert_allclose(oracle_mod.o_to_bnhd(rd["o"]).reshape(-1)[0],
                               _closed(g["o_dense_row0_closed_form"]), rtol=1e-15)
    # exact tie: both key blocks score the same, the lower id wins
    kt = np.array(g["tie_variant"]["k"], np.float64).reshape(shp)
    rt = oracle_mod.forward(q, kt, v, bs, g["topk_ratio"])
    np.testing.assert_array_equal(rt["kp"][0, 0, :, 0], g["tie_variant"]["k_pooled"])
    np.testing.assert_array_equal(rt["idx"][0, 0], g["tie_variant"]["idx"])


def test_hw2_max_pool_hand_worked(oracle_mod):
    g = json.load(open(os.path.join(HERE, "golden", "hw2_max_pool.json")))
    shp = (g["B"], g["N"], g["H"], g["D"])
    q, k, v = (np.array(g[n], np.float64).reshape(shp) for n in ("q", "k", "v"))
    bs = g["block_size"]
    r = oracle_mod.forward(q, k, v, bs, g["topk_ratio"], pool="max")
    np.testing.assert_array_equal(r["qp"][0, 0, :, 0], g["q_pooled_max"])
    np.testing.assert_array_equal(r["kp"][0, 0, :, 0], g["k_pooled_max"])
    np.testing.assert_array_equal(r["scores"][0, 0], g["scores_max"])
    np.testing.assert_array_equal(r["idx"][0, 0], g["idx_max"])
    o = oracle_mod.o_to_bnhd(r["o"]).reshape(-1)
    np.testing.assert_allclose(o, [_closed(e) for e in g["o_closed_form"]], rtol=1e-15, atol=0)
    # the mean-pooled path keeps the other block in both rows
    np.testing.assert_array_equal(oracle_mod.forward(q, k, v, bs, g["topk_ratio"])["idx"][0, 0], g["idx_mean"])


# ---------------------------------------------------------------- max pooling, adaptive block size

@pytest.mark.parametrize("dtype", ["f32", "bf16", "e4m3"])
def test_max_pool_matches_numpy_max(oracle_mod, dtype):
    B, N, H, D, bs = 2, 96, 3, 16, 8
    x = torch.from_numpy(_rand((B, N, H, D), 70)).to({"f32": torch.float32, "bf16": torch.bfloat16,
                                                       "e4m3": torch.float8_e4m3fn}[dtype])
    xa = W.to_oracle_array(x)
    got = oracle_mod.block_pool(xa, bs, pool="max")
    want = x.to(torch.float64).numpy().reshape(B, N // bs, bs, H, D).max(axis=2).transpose(0, 2, 1, 3)
    np.testing.assert_array_equal(got, want)


def test_max_pool_brute_force_and_invariants(oracle_mod):
    B, N, H, D, bs = 1, 24, 2, 5, 4
    x = _rand((B, N, H, D), 71)
    got = oracle_mod.block_pool(x, bs, pool="max")
    for h in range(H):
        for i in range(N // bs):
            for d in range(D):
                assert got[0, h, i, d] == max(x[0, i * bs + t, h, d] for t in range(bs))
    # block_size 1 is the identity; rows permuted inside a block change nothing;
    # a constant block pools to its row; the maximum is never below the mean
    np.testing.assert_array_equal(oracle_mod.block_pool(x, 1, pool="max")[0].transpose(1, 0, 2), x[0])
    perm = np.concatenate([i * bs + np.random.default_rng(i).permutation(bs) for i in range(N // bs)])
    np.testing.assert_array_equal(oracle_mod.block_pool(x[:, perm], bs, pool="max"), got)
    c = np.repeat(x[:, ::bs], bs, axis=1)
    np.testing.assert_array_equal(oracle_mod.block_pool(c, bs, pool="max"), oracle_mod.block_pool(c, bs))
    assert np.all(got >= oracle_mod.block_pool(x, bs) - 1e-15)


@pytest.mark.parametrize("n,want", [(1, 64), (8192, 64), (499_999, 64), (500_000, 128), (999_999, 128),
                                    (1_000_000, 256), (1 << 40, 256), (0, -1), (-5, -1)])
def test_adaptive_block_size_thresholds(oracle_mod, n, want):
    # page "从M2.7到M3" §4.2: 64 below 500,000 tokens, 128 below 1,000,000, else 256
    assert oracle_mod.adaptive_block_size(n) == want


# ---------------------------------------------------------------- global heads
# Reading ("从M2.7到M3" §5.3): query head h is global when h % period == 0 and
# attends to every key block; the other heads keep their selection.

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H,Hkv,period", [(4, 4, 4), (4, 2, 2), (3, 3, 1), (6, 3, 4)])
def test_global_heads_are_dense_attention(oracle_mod, causal, H, Hkv, period):
    B, N, D, bs, ratio = 2, 96, 8, 8, 0.25
    q = _rand((B, N, H, D), 80, bs=bs)
    k = _rand((B, N, Hkv, D), 81, bs=bs)
    v = _rand((B, N, Hkv, D), 82, offsets=False)
    r = oracle_mod.forward_global(q, k, v, bs, ratio, period, causal=causal)
    o = oracle_mod.o_to_bnhd(r["o"])
    plain = oracle_mod.o_to_bnhd(oracle_mod.forward_gqa(q, k, v, bs, ratio, causal=causal)["o"])
    G = H // Hkv
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)
    kr, vr = np.repeat(k, G, axis=2), np.repeat(v, G, axis=2)
    dense = torch.nn.functional.scaled_dot_product_attention(t(q), t(kr), t(vr), is_causal=causal,
                                                             scale=1.0 / math.sqrt(D)).permute(0, 2, 1, 3).numpy()
    for h in range(H):
        want = dense[:, :, h] if h % period == 0 else plain[:, :, h]
        np.testing.assert_allclose(o[:, :, h], want, rtol=1e-12, atol=1e-12)


def test_global_head_rows_layout(oracle_mod):
    idx = np.array([[[[1], [0], [2]], [[2], [2], [0]]]], np.int32)  # B=1, H=2, nb=3, k=1
    w = oracle_mod.global_head_rows(idx, 3, 2, causal=True)
    np.testing.assert_array_equal(w[0, 0], [[0, -1, -1], [0, 1, -1], [0, 1, 2]])
    np.testing.assert_array_equal(w[0, 1], [[2, -1, -1], [2, -1, -1], [0, -1, -1]])
    w = oracle_mod.global_head_rows(idx, 3, 2)
    np.testing.assert_array_equal(w[0, 0], [[0, 1, 2]] * 3)


# ---------------------------------------------------------------- overlapping key windows
# Reading ("从M2.7到M3" §5.3, overlap_ratio = 0.25): key windows of block_size
# tokens start every block_size - ov tokens (the last one moved back to end at
# N); query blocks stay disjoint; each row attends to the union of its kept
# windows' tokens.

def test_hw3_overlap_hand_worked(oracle_mod):
    g = json.load(open(os.path.join(HERE, "golden", "hw3_overlap.json")))
    shp = (g["B"], g["N"], g["H"], g["D"])
    q, k, v = (np.array(g[n], np.float64).reshape(shp) for n in ("q", "k", "v"))
    r = oracle_mod.forward_overlap(q, k, v, g["block_size"], g["topk_ratio"], g["overlap_ratio"])
    np.testing.assert_array_equal(oracle_mod.window_starts(g["N"], g["block_size"], r["ov"]), g["window_starts"])
    np.testing.assert_array_equal(r["qp"][0, 0, :, 0], g["q_pooled"])
    np.testing.assert_array_equal(r["kp"][0, 0, :, 0], g["k_window_means"])
    np.testing.assert_array_equal(r["scores"][0, 0], g["scores"])
    assert r["k"] == g["k_selected"]
    np.testing.assert_array_equal(r["idx"][0, 0], g["idx"])
    o = oracle_mod.o_to_bnhd(r["o"]).reshape(-1)
    np.testing.assert_allclose(o, [_closed(e) for e in g["o_closed_form"]], rtol=1e-15, atol=0)


@pytest.mark.parametrize("H,Hkv", [(3, 3), (4, 2)])
def test_overlap_zero_is_the_plain_path(oracle_mod, H, Hkv):
    B, N, D, bs, ratio = 2, 96, 8, 8, 0.3
    q, k, v = _rand((B, N, H, D), 90, bs=bs), _rand((B, N, Hkv, D), 91, bs=bs), _rand((B, N, Hkv, D), 92)
    r = oracle_mod.forward_overlap(q, k, v, bs, ratio, 0.0)
    p = oracle_mod.forward_gqa(q, k, v, bs, ratio)
    np.testing.assert_array_equal(r["idx"], p["idx"])
    np.testing.assert_allclose(r["o"], p["o"], rtol=1e-12, atol=1e-12)


def test_overlap_all_windows_is_dense_attention(oracle_mod):
    B, N, H, D, bs = 1, 128, 2, 8, 16  # ov 4: windows start every 12 tokens, the last moved back to 112
    q, k, v = (_rand((B, N, H, D), s, bs=8) for s in (93, 94, 95))
    r = oracle_mod.forward_overlap(q, k, v, bs, 1.0, 0.25)
    assert r["nbk"] == 11 and r["k"] == 11
    o = oracle_mod.o_to_bnhd(r["o"])
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), scale=1.0 / math.sqrt(D))
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-12, atol=1e-12)


def test_window_pool_is_a_sliding_mean(oracle_mod):
    B, N, H, D, bs, ov = 2, 200, 3, 4, 16, 5
    x = _rand((B, N, H, D), 96)
    got = oracle_mod.window_pool(x, bs, ov)
    starts = oracle_mod.window_starts(N, bs, ov)
    assert starts[0] == 0 and starts[-1] == N - bs and np.all(np.diff(starts)[:-1] == bs - ov)
    slide = np.lib.stride_tricks.sliding_window_view(x, bs, axis=1).mean(axis=-1)  # [B, N-bs+1, H, D]
    np.testing.assert_allclose(got, slide[:, starts].transpose(0, 2, 1, 3), rtol=1e-13, atol=1e-13)


def test_overlapping_kept_windows_count_shared_tokens_once(oracle_mod):
    idx = np.array([[[[0, 1], [2, 4]]]], np.int32)  # two query blocks, windows of 8 starting every 6
    sets = oracle_mod.window_token_sets(idx, 32, 8, 2)
    np.testing.assert_array_equal(sets[0][0][0], np.arange(0, 14))
    np.testing.assert_array_equal(sets[0][0][1], np.concatenate([np.arange(12, 20), np.arange(24, 32)]))


# ---------------------------------------------------------------- k = int(ratio * nb)

@pytest.mark.parametrize("nb,ratio,want", [
    (8, 0.25, 2), (8, 1.0, 8), (128, 0.3, 38), (256, 0.2, 51), (1024, 0.15, 153),
    (4096, 0.15, 614), (100, 0.29, 28), (3, 0.1, 0), (10, 0.7, 7),
])
def test_topk_count_matches_python_int(oracle_mod, nb, ratio, want):
    assert int(ratio * nb) == want  # what the page's int(topk_ratio * num_blocks) gives
    assert oracle_mod.topk_count(nb, ratio) == want


# ---------------------------------------------------------------- pooling

def test_pool_block_size_one_is_identity(oracle_mod):
    x = _rand((2, 6, 3, 5), 1, offsets=False)
    p = oracle_mod.block_pool(x, 1)
    np.testing.assert_array_equal(p, x.transpose(0, 2, 1, 3))


def test_pool_constant_block_gives_the_row(oracle_mod):
    B, nb, bs, H, D = 2, 3, 4, 2, 8
    rows = _rand((B, nb, 1, H, D), 2, offsets=False)
    x = np.broadcast_to(rows, (B, nb, bs, H, D)).reshape(B, nb * bs, H, D)
    p = oracle_mod.block_pool(x, bs)
    np.testing.assert_allclose(p, rows[:, :, 0].transpose(0, 2, 1, 3), rtol=1e-15)


def test_pool_matches_numpy_mean(oracle_mod):
    B, N, H, D, bs = 2, 64, 3, 16, 8
    x = _rand((B, N, H, D), 3, bs=bs)
    p = oracle_mod.block_pool(x, bs)
    ref = x.reshape(B, N // bs, bs, H, D).mean(axis=2).transpose(0, 2, 1, 3)
    np.testing.assert_allclose(p, ref, rtol=1e-13, atol=1e-15)


def test_bf16_and_f32_inputs_convert_exactly(oracle_mod):
    B, N, H, D, bs = 1, 16, 2, 8, 4
    xt = torch.from_numpy(_rand((B, N, H, D), 4, bs=bs))
    for dt in (torch.bfloat16, torch.float32):
        x = xt.to(dt)
        arr = x.view(torch.int16).numpy().view(np.uint16) if dt == torch.bfloat16 else x.numpy()
        p = oracle_mod.block_pool(arr, 1)
        np.testing.assert_array_equal(p, x.to(torch.float64).numpy().transpose(0, 2, 1, 3))


# ---------------------------------------------------------------- block scores

def test_scores_match_numpy_matmul(oracle_mod):
    rng = np.random.default_rng(5)
    qp = rng.standard_normal((2, 3, 7, 16))
    kp = rng.standard_normal((2, 3, 7, 16))
    S = oracle_mod.block_scores(qp, kp)
    np.testing.assert_allclose(S, np.matmul(qp, kp.transpose(0, 1, 3, 2)), rtol=1e-13, atol=1e-13)
    # a sample of rows picks the same rows out of the full matrix
    rows = np.array([[[6, 1], [0, 3], [2, 2]], [[5, 4], [1, 0], [3, 6]]], np.int32)
    Sr = oracle_mod.block_scores(qp, kp, rows)
    full = np.matmul(qp, kp.transpose(0, 1, 3, 2))
    np.testing.assert_allclose(Sr, np.take_along_axis(full, rows[..., None].astype(np.int64), 2),
                               rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- top-k selection

def _brute_topk(S, k):
    out = np.empty(S.shape[:-1] + (k,), np.int32)
    flat = S.reshape(-1, S.shape[-1])
    for r, row in enumerate(flat):
        j = np.arange(row.size)
        order = np.lexsort((j, -row))  # score descending, then index ascending
        out.reshape(-1, k)[r] = np.sort(order[:k])
    return out


@pytest.mark.parametrize("seed", range(4))
def test_topk_matches_lexsort_brute_force_with_ties(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(5, 40))
    S = rng.integers(-3, 4, size=(3, 2, nb, nb)).astype(np.float64)  # many exact ties
    for k in (1, nb // 3 + 1, nb - 1, nb):
        np.testing.assert_array_equal(oracle_mod.topk(S, k), _brute_topk(S, k))


def test_topk_invariants(oracle_mod):
    rng = np.random.default_rng(7)
    S = rng.standard_normal((2, 3, 50, 50))
    idx = oracle_mod.topk(S, 13)
    assert np.all(np.diff(idx, axis=-1) > 0)  # ascending, distinct
    for r in range(idx.reshape(-1, 13).shape[0]):
        row = S.reshape(-1, 50)[r]
        sel = idx.reshape(-1, 13)[r]
        mask = np.zeros(50, bool)
        mask[sel] = True
        assert row[mask].min() >= row[~mask].max()
    np.testing.assert_array_equal(oracle_mod.topk(S, 50)[0, 0, 0], np.arange(50))


def test_topk_ties_go_to_lower_index(oracle_mod):
    S = np.array([[0.5, 2.0, 1.0, 2.0, 1.0, 1.0, -1.0]])
    np.testing.assert_array_equal(oracle_mod.topk(S, 1), [[1]])
    np.testing.assert_array_equal(oracle_mod.topk(S, 2), [[1, 3]])
    np.testing.assert_array_equal(oracle_mod.topk(S, 3), [[1, 2, 3]])
    np.testing.assert_array_equal(oracle_mod.topk(S, 4), [[1, 2, 3, 4]])


# ---------------------------------------------------------------- attention

def _masked_dense(q, k, v, idx, bs, scale):
    """Softmax(Mask(Q K^T * scale)) V with Mask from the selected blocks
    ([MSA] §2.1), written with numpy over [B,N,H,D] float64."""
    B, N, H, D = q.shape
    nb = N // bs
    out = np.empty_like(q)
    for b in range(B):
        for h in range(H):
            logits = (q[b, :, h] @ k[b, :, h].T) * scale
            mask = np.zeros((N, N), bool)
            for i in range(nb):
                for j in idx[b, h, i]:
                    mask[i * bs:(i + 1) * bs, j * bs:(j + 1) * bs] = True
            logits = np.where(mask, logits, -np.inf)
            w = np.exp(logits - logits.max(axis=1, keepdims=True))
            out[b, :, h] = (w / w.sum(axis=1, keepdims=True)) @ v[b, :, h]
    return out


def test_ratio_one_equals_dense_sdpa(oracle_mod):
    B, N, H, D, bs = 2, 64, 2, 16, 8
    q, k, v = (_rand((B, N, H, D), s, bs=bs) for s in (10, 11, 12))
    r = oracle_mod.forward(q, k, v, bs, 1.0)
    o = oracle_mod.o_to_bnhd(r["o"])
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)  # [B,H,N,D]
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v)).permute(0, 2, 1, 3)
    np.testing.assert_allclose(o, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_any_index_list_equals_masked_dense(oracle_mod):
    B, N, H, D, bs = 1, 48, 2, 8, 6
    q, k, v = (_rand((B, N, H, D), s, bs=bs) for s in (20, 21, 22))
    rng = np.random.default_rng(23)
    nb, kk = N // bs, 3
    idx = np.sort(np.stack([[[rng.choice(nb, kk, replace=False) for _ in range(nb)]
                             for _ in range(H)] for _ in range(B)]), axis=-1).astype(np.int32)
    for scale in (1.0 / math.sqrt(D), 0.37):
        o = oracle_mod.o_to_bnhd(oracle_mod.sparse_attn(q, k, v, idx, bs, scale=scale))
        np.testing.assert_allclose(o, _masked_dense(q, k, v, idx, bs, scale), rtol=1e-12, atol=1e-12)


def test_block_size_one_full_k_is_token_attention(oracle_mod):
    B, N, H, D = 1, 12, 1, 4
    q, k, v = (_rand((B, N, H, D), s, offsets=False) for s in (30, 31, 32))
    r = oracle_mod.forward(q, k, v, 1, 1.0)
    logits = q[0, :, 0] @ k[0, :, 0].T / 2.0
    w = np.exp(logits - logits.max(1, keepdims=True))
    ref = (w / w.sum(1, keepdims=True)) @ v[0, :, 0]
    np.testing.assert_allclose(oracle_mod.o_to_bnhd(r["o"])[0, :, 0], ref, rtol=1e-12, atol=1e-13)


def test_sampled_rows_match_full_run(oracle_mod):
    B, N, H, D, bs = 1, 64, 2, 8, 8
    q, k, v = (_rand((B, N, H, D), s, bs=bs) for s in (40, 41, 42))
    full = oracle_mod.forward(q, k, v, bs, 0.5)
    rows = np.array([[[1, 6], [0, 7]]], np.int32)
    part = oracle_mod.forward(q, k, v, bs, 0.5, rows=rows)
    for h in range(H):
        for r, i in enumerate(rows[0, h]):
            np.testing.assert_array_equal(part["idx"][0, h, r], full["idx"][0, h, i])
            np.testing.assert_array_equal(part["o"][0, h, r], full["o"][0, h, i])


# ---------------------------------------------------------------- invariants

@pytest.fixture(scope="module")
def small_case():
    B, N, H, D, bs = 2, 64, 2, 8, 8
    q, k, v = (_rand((B, N, H, D), s, bs=bs) for s in (50, 51, 52))
    return q, k, v, bs, 0.375


def test_shift_and_linearity_in_v(oracle_mod, small_case):
    q, k, v, bs, ratio = small_case
    o = oracle_mod.o_to_bnhd(oracle_mod.forward(q, k, v, bs, ratio)["o"])
    c = np.linspace(-1, 1, v.shape[-1])
    o_shift = oracle_mod.o_to_bnhd(oracle_mod.forward(q, k, v + c, bs, ratio)["o"])
    np.testing.assert_allclose(o_shift, o + c, rtol=1e-12, atol=1e-12)
    v2 = _rand(v.shape, 53, offsets=False)
    o2 = oracle_mod.o_to_bnhd(oracle_mod.forward(q, k, v2, bs, ratio)["o"])
    o_lin = oracle_mod.o_to_bnhd(oracle_mod.forward(q, k, 2.0 * v - 3.0 * v2, bs, ratio)["o"])
    np.testing.assert_allclose(o_lin, 2.0 * o - 3.0 * o2, rtol=1e-11, atol=1e-11)


def test_permutations_inside_blocks(oracle_mod, small_case):
    q, k, v, bs, ratio = small_case
    B, N, H, D = q.shape
    base = oracle_mod.forward(q, k, v, bs, ratio)
    o = oracle_mod.o_to_bnhd(base["o"])
    perm = np.arange(N).reshape(-1, bs)[:, ::-1].reshape(-1)  # reverse rows inside every block
    # permuting key rows (k and v together) inside blocks leaves o unchanged
    rk = oracle_mod.forward(q, k[:, perm], v[:, perm], bs, ratio)
    np.testing.assert_array_equal(rk["idx"], base["idx"])
    np.testing.assert_allclose(oracle_mod.o_to_bnhd(rk["o"]), o, rtol=1e-12, atol=1e-12)
    # permuting query rows inside blocks permutes the output rows the same way
    rq = oracle_mod.forward(q[:, perm], k, v, bs, ratio)
    np.testing.assert_allclose(oracle_mod.o_to_bnhd(rq["o"]), o[:, perm], rtol=1e-12, atol=1e-12)


def test_batch_head_permutation_and_block_relabel(oracle_mod, small_case):
    q, k, v, bs, ratio = small_case
    B, N, H, D = q.shape
    base = oracle_mod.forward(q, k, v, bs, ratio)
    o = oracle_mod.o_to_bnhd(base["o"])
    pb, ph = [1, 0], [1, 0]
    r = oracle_mod.forward(q[pb][:, :, ph], k[pb][:, :, ph], v[pb][:, :, ph], bs, ratio)
    np.testing.assert_allclose(oracle_mod.o_to_bnhd(r["o"]), o[pb][:, :, ph], rtol=1e-12, atol=1e-12)
    # relabel key blocks: swap key blocks 1 and 5 (k and v together)
    nb = N // bs
    bperm = np.arange(nb)
    bperm[[1, 5]] = bperm[[5, 1]]
    tok = (bperm[:, None] * bs + np.arange(bs)).reshape(-1)
    r2 = oracle_mod.forward(q, k[:, tok], v[:, tok], bs, ratio)
    relabeled = np.sort(bperm[base["idx"]], axis=-1)
    np.testing.assert_array_equal(r2["idx"], relabeled)
    np.testing.assert_allclose(oracle_mod.o_to_bnhd(r2["o"]), o, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- the definition, written out again

def test_matches_definition_written_out_in_numpy(oracle_mod):
    """The three steps of page "2026 新一代卷积与 Transformer 网络架构" (section
    "SparseFormer 注意力实现") written out independently of the C oracle: block
    means as explicit per-block sums, the selection as a full sort of
    (score descending, block id ascending), and each query row's softmax over
    the tokens of its kept blocks. The random data has no exact score ties."""
    B, N, H, D, bs, ratio = 2, 96, 3, 16, 8, 0.3
    q, k, v = (_rand((B, N, H, D), s, bs=bs).astype(np.float64) for s in (60, 61, 62))
    nb = N // bs
    kk = int(ratio * nb)
    want_idx = np.empty((B, H, nb, kk), np.int32)
    want_o = np.empty((B, N, H, D))
    for b in range(B):
        for h in range(H):
            qbar = [sum(q[b, i * bs + t, h] for t in range(bs)) / bs for i in range(nb)]
            kbar = [sum(k[b, j * bs + t, h] for t in range(bs)) / bs for j in range(nb)]
            for i in range(nb):
                score = [float(np.dot(qbar[i], kbar[j])) for j in range(nb)]
                ranked = sorted(range(nb), key=lambda j: (-score[j], j))
                kept = sorted(ranked[:kk])
                want_idx[b, h, i] = kept
                toks = [j * bs + t for j in kept for t in range(bs)]
                for t_q in range(bs):
                    n = i * bs + t_q
                    logits = np.array([np.dot(q[b, n, h], k[b, t, h]) for t in toks]) / math.sqrt(D)
                    w = np.exp(logits - logits.max())
                    want_o[b, n, h] = sum(w[c] * v[b, t, h] for c, t in enumerate(toks)) / w.sum()
    r = oracle_mod.forward(q, k, v, bs, ratio)
    np.testing.assert_array_equal(r["idx"], want_idx)
    np.testing.assert_allclose(oracle_mod.o_to_bnhd(r["o"]), want_o, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- causal variant
# Readings: query block i ranks only key blocks j <= i and keeps min(k, i+1)
# of them (with the diagonal forced in when asked), rows padded with -1; query
# token n never sees key token t > n ([MSA] §2.1, Mask(QK^T) with the causal mask).

def _lexsort_topk_causal(S, k, force_diag):
    out = np.full(S.shape[:-1] + (k,), -1, np.int32)
    for pos in np.ndindex(S.shape[:-1]):
        i = pos[-1]
        n = min(k, i + 1)
        cand = np.arange(i if force_diag else i + 1)
        order = cand[np.lexsort((cand, -S[pos][cand]))]
        keep = list(order[: (n - 1 if force_diag else n)]) + ([i] if force_diag else [])
        out[pos][:n] = np.sort(keep)
    return out


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("force_diag", [False, True])
def test_causal_topk_matches_lexsort_brute_force(oracle_mod, seed, force_diag):
    rng = np.random.default_rng(100 + seed)
    S = rng.integers(-3, 4, (2, 3, 9, 9)).astype(np.float64)  # many exact ties
    for k in (1, 3, 9):
        got = oracle_mod.topk(S, k, causal=True, force_diag=force_diag)
        np.testing.assert_array_equal(got, _lexsort_topk_causal(S, k, force_diag))


def test_causal_topk_invariants(oracle_mod):
    rng = np.random.default_rng(7)
    S = rng.standard_normal((1, 2, 16, 16))
    k = 5
    for fd in (False, True):
        idx = oracle_mod.topk(S, k, causal=True, force_diag=fd)
        for h in range(2):
            for i in range(16):
                row, n = idx[0, h, i], min(k, i + 1)
                valid = row[:n]
                assert (row[n:] == -1).all() and (valid >= 0).all() and (valid <= i).all()
                assert (np.diff(valid) > 0).all()
                if fd:
                    assert i in valid
                ranked = [j for j in valid if not (fd and j == i)]
                dropped = [j for j in range(i if fd else i + 1) if j not in valid]
                if ranked and dropped:
                    assert S[0, h, i, ranked].min() >= S[0, h, i, dropped].max()
    # rows named explicitly give the same lists as the all-rows run
    rows = np.array([[[3, 11, 15], [0, 7, 8]]])
    sub = np.take_along_axis(S, rows[..., None], 2)
    got = oracle_mod.topk(sub, k, causal=True, qblocks=rows)
    np.testing.assert_array_equal(got, np.take_along_axis(oracle_mod.topk(S, k, causal=True), rows[..., None], 2))


def test_causal_ratio_one_equals_causal_sdpa(oracle_mod):
    """k = nb keeps every block j <= i, so the method is dense causal attention
    (block_size 1 makes it token-level causal attention)."""
    B, N, H, D = 2, 64, 2, 16
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)  # [B,H,N,D]
    for bs in (1, 4, 8):
        q, k, v = (_rand((B, N, H, D), s, bs=bs) for s in (70, 71, 72))
        ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=True)
        for fd in (False, True):
            r = oracle_mod.forward(q, k, v, bs, 1.0, causal=True, force_diag=fd)
            np.testing.assert_allclose(oracle_mod.o_to_bnhd(r["o"]), ref.permute(0, 2, 1, 3).numpy(),
                                       rtol=1e-12, atol=1e-12)


def test_causal_index_list_equals_masked_dense(oracle_mod):
    """Any causal index list (with -1 padding) equals dense attention under the
    block mask and the token causal mask, built here in torch."""
    B, N, H, D, bs, kk = 1, 48, 2, 8, 6, 3
    nb = N // bs
    q, k, v = (_rand((B, N, H, D), s, bs=bs) for s in (80, 81, 82))
    rng = np.random.default_rng(83)
    idx = np.full((B, H, nb, kk), -1, np.int32)
    for h in range(H):
        for i in range(nb):
            n = min(kk, i + 1)
            idx[0, h, i, :n] = np.sort(rng.choice(i + 1, n, replace=False))
    o = oracle_mod.o_to_bnhd(oracle_mod.sparse_attn(q, k, v, idx, bs, causal=True))
    blk = np.zeros((B, H, nb, nb), bool)
    for h in range(H):
        for i in range(nb):
            blk[0, h, i, idx[0, h, i][idx[0, h, i] >= 0]] = True
    mask = torch.from_numpy(blk).repeat_interleave(bs, 2).repeat_interleave(bs, 3)
    mask &= torch.ones(N, N, dtype=torch.bool).tril()
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=mask)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-12, atol=1e-12)


def test_causal_future_tokens_change_nothing_before_them(oracle_mod):
    """Changing q, k, v in blocks >= c leaves selection and output of every
    query block < c bit-identical (pooling, scoring, selection and attention
    all look only backwards)."""
    B, N, H, D, bs, ratio, c = 1, 64, 2, 8, 4, 0.3, 9
    q, k, v = (_rand((B, N, H, D), s, bs=bs) for s in (90, 91, 92))
    q2, k2, v2 = (x.copy() for x in (q, k, v))
    rng = np.random.default_rng(93)
    for x in (q2, k2, v2):
        x[:, c * bs:] += rng.standard_normal(x[:, c * bs:].shape) * 3
    for fd in (False, True):
        r1 = oracle_mod.forward(q, k, v, bs, ratio, causal=True, force_diag=fd)
        r2 = oracle_mod.forward(q2, k2, v2, bs, ratio, causal=True, force_diag=fd)
        np.testing.assert_array_equal(r1["idx"][:, :, :c], r2["idx"][:, :, :c])
        np.testing.assert_array_equal(r1["o"][:, :, :c], r2["o"][:, :, :c])
        assert not np.array_equal(r1["o"][:, :, c:], r2["o"][:, :, c:])


def test_minus_one_entries_select_nothing(oracle_mod, small_case):
    q, k, v, bs, ratio = small_case
    r = oracle_mod.forward(q, k, v, bs, ratio)
    pad = np.concatenate([r["idx"], np.full(r["idx"].shape[:-1] + (2,), -1, np.int32)], -1)
    np.testing.assert_array_equal(oracle_mod.sparse_attn(q, k, v, pad, bs), r["o"])


# ---------------------------------------------------------------- grouped-query variant
# Readings: q has H heads, k and v Hkv = H / G; query head h reads key/value
# head h // G; one selection per key/value head, scored with the group's pooled
# query (mean of its heads' block means).

def _repeat_kv(x, G):
    return np.repeat(x, G, axis=2)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_ratio_one_equals_sdpa_with_repeated_kv(oracle_mod, causal):
    B, N, H, Hkv, D, bs = 2, 64, 6, 2, 16, 8
    q = _rand((B, N, H, D), 110, bs=bs)
    k, v = (_rand((B, N, Hkv, D), s, bs=bs) for s in (111, 112))
    r = oracle_mod.forward_gqa(q, k, v, bs, 1.0, causal=causal)
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(_repeat_kv(k, H // Hkv)),
                                                           t(_repeat_kv(v, H // Hkv)), is_causal=causal)
    np.testing.assert_allclose(oracle_mod.o_to_bnhd(r["o"]), ref.permute(0, 2, 1, 3).numpy(),
                               rtol=1e-12, atol=1e-12)


def test_gqa_group_score_is_mean_of_head_scores(oracle_mod):
    """By linearity the group score q̄_g . k̄_j equals the mean over the group's
    heads of q̄_h . k̄_j, computed here with numpy per head."""
    B, N, H, Hkv, D, bs = 1, 96, 8, 2, 16, 8
    q = _rand((B, N, H, D), 120, bs=bs)
    k, v = (_rand((B, N, Hkv, D), s, bs=bs) for s in (121, 122))
    r = oracle_mod.forward_gqa(q, k, v, bs, 0.25)
    qp = q.reshape(B, N // bs, bs, H, D).mean(2).transpose(0, 2, 1, 3)  # [B,H,nb,D]
    kp = k.reshape(B, N // bs, bs, Hkv, D).mean(2).transpose(0, 2, 1, 3)
    G = H // Hkv
    per_head = np.stack([qp[:, h] @ kp[:, h // G].transpose(0, 2, 1) for h in range(H)], 1)
    want = per_head.reshape(B, Hkv, G, N // bs, N // bs).mean(2)
    np.testing.assert_allclose(r["scores"], want, rtol=1e-12, atol=1e-12)


def test_gqa_attention_equals_per_head_attention_on_repeated_kv(oracle_mod):
    B, N, H, Hkv, D, bs, kk = 1, 48, 4, 2, 8, 6, 3
    nb = N // bs
    q = _rand((B, N, H, D), 130, bs=bs)
    k, v = (_rand((B, N, Hkv, D), s, bs=bs) for s in (131, 132))
    rng = np.random.default_rng(133)
    idx = np.sort(np.stack([[[rng.choice(nb, kk, replace=False) for _ in range(nb)]
                             for _ in range(H)]]), axis=-1).astype(np.int32)
    for causal in (False, True):
        got = oracle_mod.sparse_attn_gqa(q, k, v, idx, bs, causal=causal)
        want = oracle_mod.sparse_attn(q, _repeat_kv(k, H // Hkv), _repeat_kv(v, H // Hkv), idx, bs,
                                      causal=causal)
        np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13)


def test_gqa_head_permutation_within_a_group(oracle_mod):
    B, N, H, Hkv, D, bs = 1, 64, 6, 2, 8, 8
    q = _rand((B, N, H, D), 140, bs=bs)
    k, v = (_rand((B, N, Hkv, D), s, bs=bs) for s in (141, 142))
    r = oracle_mod.forward_gqa(q, k, v, bs, 0.375)
    perm = np.array([2, 0, 1, 4, 5, 3])  # within groups {0,1,2} and {3,4,5}
    r2 = oracle_mod.forward_gqa(q[:, :, perm], k, v, bs, 0.375)
    np.testing.assert_array_equal(r2["idx"], r["idx"])
    np.testing.assert_allclose(r2["o"], r["o"][:, perm], rtol=1e-12, atol=1e-12)


def test_gqa_with_one_head_per_group_is_the_plain_path(oracle_mod, small_case):
    q, k, v, bs, ratio = small_case
    for causal in (False, True):
        a = oracle_mod.forward(q, k, v, bs, ratio, causal=causal)
        b = oracle_mod.forward_gqa(q, k, v, bs, ratio, causal=causal)
        np.testing.assert_array_equal(a["idx"], b["idx"])
        np.testing.assert_allclose(a["o"], b["o"], rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- FP8 E4M3 inputs

def test_e4m3_decoding_matches_torch_for_every_code(oracle_mod):
    codes = torch.arange(256, dtype=torch.uint8)
    want = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle_mod.e4m3_to_double(c) for c in range(256)])
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2  # S.1111.111
    np.testing.assert_array_equal(got[~nan], want[~nan])


def test_e4m3_inputs_are_their_exact_values(oracle_mod):
    """The whole path on e4m3 bytes equals the path on the same values given
    as float64 (the conversion is exact, nothing else changes)."""
    B, N, H, D, bs = 1, 64, 2, 16, 8
    x = [torch.from_numpy(_rand((B, N, H, D), s, bs=bs)).to(torch.float8_e4m3fn) for s in (150, 151, 152)]
    raw = [t.view(torch.uint8).numpy() for t in x]
    f64 = [t.to(torch.float64).numpy() for t in x]
    for causal in (False, True):
        a = oracle_mod.forward(*raw, bs, 0.375, causal=causal)
        b = oracle_mod.forward(*f64, bs, 0.375, causal=causal)
        np.testing.assert_array_equal(a["idx"], b["idx"])
        np.testing.assert_array_equal(a["o"], b["o"])


# ---------------------------------------------------------------- backward pass
# Reading: the top-k indices carry no gradient, so the backward is the
# gradient of the attention over the kept blocks with the lists held fixed.

def _dense_mask(idx, bs, N, causal):
    B, H, nb, _ = idx.shape
    blk = np.zeros((B, H, nb, nb), bool)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                row = idx[b, h, i]
                blk[b, h, i, row[row >= 0]] = True
    m = torch.from_numpy(blk).repeat_interleave(bs, 2).repeat_interleave(bs, 3)
    if causal:
        m &= torch.ones(N, N, dtype=torch.bool).tril()
    return m


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_torch_autograd_of_masked_dense_attention(oracle_mod, causal):
    """float64 torch autograd of SDPA under the block (and causal) mask."""
    B, N, H, D, bs = 2, 48, 2, 8, 6
    q, k, v, do = (_rand((B, N, H, D), s, bs=bs) for s in (160, 161, 162, 163))
    r = oracle_mod.forward(q, k, v, bs, 0.4, causal=causal)
    dq, dk, dv = oracle_mod.sparse_attn_bwd(q, k, v, do, r["idx"], bs, causal=causal)
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3).clone().requires_grad_(True)
    tq, tk, tv = t(q), t(k), t(v)
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv,
                                                           attn_mask=_dense_mask(r["idx"], bs, N, causal))
    out.backward(torch.from_numpy(do).permute(0, 2, 1, 3))
    for got, ref in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(got, ref.grad.permute(0, 2, 1, 3).numpy(), rtol=1e-11, atol=1e-12)


def test_backward_matches_finite_differences(oracle_mod):
    """Central differences of sum(o * dO) on a tiny case, for a few entries of
    q, k and v (the selection is held fixed)."""
    B, N, H, D, bs = 1, 16, 1, 4, 4
    q, k, v, do = (_rand((B, N, H, D), s, bs=bs) for s in (170, 171, 172, 173))
    idx = oracle_mod.forward(q, k, v, bs, 0.5)["idx"]
    dq, dk, dv = oracle_mod.sparse_attn_bwd(q, k, v, do, idx, bs)

    def loss(qq, kk, vv):
        o = oracle_mod.o_to_bnhd(oracle_mod.sparse_attn(qq, kk, vv, idx, bs))
        return float((o * do).sum())

    eps = 1e-6
    rng = np.random.default_rng(174)
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(4):
            pos = tuple(int(rng.integers(0, s)) for s in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[pos] += eps
            minus[pos] -= eps
            args = lambda x: [x if n == name else a for n, a in (("q", q), ("k", k), ("v", v))]
            fd = (loss(*args(plus)) - loss(*args(minus))) / (2 * eps)
            assert abs(fd - grad[pos]) <= 1e-7 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])


def test_row_lists_broadcast_over_batch_and_heads_and_are_checked(oracle_mod):
    """A [1, 1, nrows] list of query blocks means the same blocks in every
    (b, h); lists that do not broadcast, or name blocks outside [0, nb), are
    refused before the C routines read them."""
    import workloads as W

    oracle = oracle_mod
    cfg = W.Config("rows", 2, 512, 3, 64, 64, 0.5, "f32", 1.0, 77, None)
    q, k, v = (W.to_oracle_array(x) for x in W.make_inputs(cfg, device="cpu"))
    full = oracle.forward(q, k, v, 64, 0.5)
    rows = np.array([[[1, 6]]], np.int32)
    part = oracle.forward(q, k, v, 64, 0.5, rows=rows)
    np.testing.assert_array_equal(part["idx"], full["idx"][:, :, [1, 6]])
    np.testing.assert_allclose(part["o"], full["o"][:, :, [1, 6]], rtol=0, atol=0)
    with pytest.raises(ValueError):
        oracle.forward(q, k, v, 64, 0.5, rows=np.zeros((3, 3, 2), np.int32))  # B = 2
    with pytest.raises(ValueError):
        oracle.forward(q, k, v, 64, 0.5, rows=np.array([[[8]]], np.int32))  # nb = 8
    with pytest.raises(ValueError):
        oracle.sparse_attn(q, k, v, full["idx"][:, :, :2], 64, rows=np.array([0, 1], np.int32))


def test_bench_cpu_sample_with_several_batch_entries():
    """The benchmark's oracle sample on a B = 2 workload (one head, sampled
    query blocks): it runs and counts the tokens of every batch entry."""
    import bench
    import workloads as W

    cfg = W.Config("bench_rows", 2, 1024, 2, 64, 64, 0.25, "bf16", 1.0, 78, None)
    q, k, v = W.make_inputs(cfg, device="cpu")
    tok, sec, thr = bench.oracle_sample(q, k, v, cfg, [1], 3, seed=5)
    assert tok == 3 * 64 * 2 and sec > 0 and thr >= 1
