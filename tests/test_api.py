"""C-ABI boundary checks that need no GPU: the library loads, exports every
function include/bsa.h declares, and rejects bad arguments on the host before
touching the device (no compute call is made here)."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bsa():
    from conftest import build_library

    build_library()
    import block_sparse_attention_19_b200 as m

    return m


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "bsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(bsa):
    declared = _declared_functions()
    assert len(declared) >= 9
    assert set(declared) == set(bsa.EXPORTED)
    lib = ctypes.CDLL(bsa.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name


@pytest.mark.parametrize("nb,ratio", [(8, 0.25), (8, 1.0), (128, 0.3), (256, 0.2), (1024, 0.15),
                                      (4096, 0.15), (100, 0.29), (3, 0.1), (7, 0.999999)])
def test_topk_count_is_python_int(bsa, nb, ratio):
    assert bsa.bsa_topk_count(nb, ratio) == int(ratio * nb)


@pytest.mark.parametrize("n,want", [(1, 64), (499_999, 64), (500_000, 128), (999_999, 128),
                                    (1_000_000, 256), (1 << 40, 256), (0, -1)])
def test_adaptive_block_size(bsa, oracle_mod, n, want):
    # the page's rule ("从M2.7到M3" §4.2), and the oracle's restatement of it
    assert bsa.bsa_adaptive_block_size(n) == want == oracle_mod.adaptive_block_size(n)


def test_topk_count_rejects_bad_input(bsa):
    assert bsa.bsa_topk_count(0, 0.5) == -1
    assert bsa.bsa_topk_count(8, -0.1) == -1
    assert bsa.bsa_topk_count(8, float("nan")) == -1
    assert bsa.bsa_topk_count(8, float("inf")) == -1


def test_workspace_bytes(bsa):
    # c4: pooled q and k [1,16,1024,128] f32 = 8 MiB each, idx [1,16,1024,153] i32,
    # block scores [1,16,1024,1024] f32 = 64 MiB
    got = bsa.bsa_forward_workspace_bytes(1, 131072, 16, 128, 128, 0.15)
    idx = 16 * 1024 * 153 * 4
    assert got == 2 * 8 * 2**20 + (idx + 255) // 256 * 256 + 64 * 2**20
    assert bsa.bsa_forward_workspace_bytes(1, 100, 2, 64, 64, 0.5) == 0  # N % block_size
    assert bsa.bsa_forward_workspace_bytes(1, 512, 2, 96, 64, 0.5) == 0  # D unsupported
    assert bsa.bsa_forward_workspace_bytes(1, 512, 2, 64, 64, 0.1) == 0  # k = 0


def test_status_strings(bsa):
    for code in range(7):
        s = bsa.lib.bsa_status_string(code).decode()
        assert s and s != "unknown status"
    assert bsa.lib.bsa_status_string(99).decode() == "unknown status"


# Fake, never-dereferenced pointer values: every case below fails validation on
# the host, before any CUDA call.
A = 0x10000  # 16-byte aligned
M = 0x10004  # misaligned


def _fwd(bsa, q=A, k=A, v=A, o=A + 0x100, B=1, N=512, H=2, D=64, bs=64, ratio=0.25, dt=1, ws=A + 0x200,
         wsb=1 << 30):
    P = ctypes.c_void_p
    return bsa.lib.bsa_forward(P(q), P(k), P(v), P(o), B, N, H, D, bs, ratio, dt, P(ws), wsb, P(0))


@pytest.mark.parametrize("kw,status", [
    (dict(q=0), 1), (dict(o=0), 1), (dict(N=500), 1), (dict(B=0), 1), (dict(N=0), 1), (dict(H=0), 1),
    (dict(B=-1), 1), (dict(ratio=0.1), 1),
    (dict(ratio=1.5), 1), (dict(ratio=float("nan")), 1), (dict(D=96), 2), (dict(bs=32, N=512), 2),
    (dict(dt=7), 2), (dict(q=M), 3), (dict(v=M), 3), (dict(ws=0), 4), (dict(wsb=16), 4),
    (dict(ws=A + 0x210), 3), (dict(o=A), 1),
])
def test_forward_rejects_bad_arguments(bsa, kw, status):
    assert _fwd(bsa, **kw) == status
    assert bsa.lib.bsa_last_error_detail().decode() != ""


def test_stage_entry_points_reject_bad_arguments(bsa):
    P = ctypes.c_void_p
    L = bsa.lib
    assert L.bsa_block_pool(P(0), P(A), 1, 512, 2, 64, 64, 1, P(0)) == 1
    assert L.bsa_block_pool(P(A), P(M), 1, 512, 2, 64, 64, 1, P(0)) == 3
    assert L.bsa_block_pool(P(A), P(A), 1, 500, 2, 64, 64, 1, P(0)) == 1
    assert L.bsa_block_scores_topk(P(A), P(A), P(0), P(A), 1, 2, 8, 64, 0, P(0)) == 1
    assert L.bsa_block_scores_topk(P(A), P(A), P(0), P(A), 1, 2, 8, 64, 9, P(0)) == 1
    assert L.bsa_block_scores_topk(P(A), P(A), P(M), P(A), 1, 2, 8, 64, 2, P(0)) == 3
    assert L.bsa_block_scores_topk(P(A), P(A), P(0), P(A), 1, 2, 8, 32, 2, P(0)) == 2
    assert L.bsa_block_scores_topk(P(A), P(A), P(0), P(A), 1, 2, 8, 64, 2, P(0)) == 1  # scores required
    assert L.bsa_sparse_attn_fwd(P(A), P(A), P(A), P(A), P(A + 0x100), 1, 512, 2, 64, 64, 9, 0.125, 1, P(0)) == 1
    assert L.bsa_sparse_attn_fwd(P(A), P(A), P(A), P(A), P(A + 0x100), 1, 512, 2, 64, 64, 2, -1.0, 1, P(0)) == 1
    assert L.bsa_sparse_attn_fwd(P(A), P(A), P(A), P(0), P(A + 0x100), 1, 512, 2, 64, 64, 2, 0.125, 1, P(0)) == 1
    assert L.bsa_sparse_attn_fwd(P(A), P(A), P(A), P(A), P(M), 1, 512, 2, 64, 64, 2, 0.125, 1, P(0)) == 3


def test_binding_fails_loudly_without_library(tmp_path):
    """Importing the package with the library absent raises instead of falling back."""
    import subprocess
    import sys

    pkg = tmp_path / "block_sparse_attention_19_b200"
    pkg.mkdir()
    (pkg / "__init__.py").write_text(open(os.path.join(ROOT, "block_sparse_attention_19_b200", "__init__.py")).read())
    r = subprocess.run([sys.executable, "-c", "import block_sparse_attention_19_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "libbsa.so is not built" in r.stderr


def test_ex_entry_points_reject_bad_flags(bsa):
    """Flag validation happens on the host before any device work."""
    bsa_lib = bsa.lib
    P = ctypes.c_void_p
    fake = P(0x10000)
    # unknown bit
    st = bsa_lib.bsa_forward_ex(fake, fake, fake, P(0x20000), 1, 1024, 2, 64, 64, 0.25, 1, 8, fake,
                                1 << 30, P(0))
    assert st == 1 and b"flag" in bsa_lib.bsa_last_error_detail()
    st = bsa_lib.bsa_block_pool_ex(fake, P(0x20000), 1, 1024, 2, 64, 64, 1, 8, P(0))
    assert st == 1 and b"flag" in bsa_lib.bsa_last_error_detail()
    # forcing the diagonal block only makes sense with the causal flag
    st = bsa_lib.bsa_sparse_attn_fwd_ex(fake, fake, fake, fake, P(0x20000), 1, 1024, 2, 64, 64, 4,
                                        0.125, 1, 2, P(0))
    assert st == 1 and b"CAUSAL" in bsa_lib.bsa_last_error_detail()
    st = bsa_lib.bsa_block_scores_topk_ex(fake, fake, fake, fake, 1, 2, 16, 64, 4, 8, P(0))
    assert st == 1


def _host_plan_bytes(B, N, H, Hkv, D, bs, ratio, es, oes, gqa_ws):
    """bsa_forward_host's workspace, restated from its documented chunking:
    chunks of one batch entry and the fewest consecutive key/value heads
    whose inputs and output reach 64 MB (else all of them); two slots of
    q, k, v, o copies and a forward workspace, each 256-byte aligned, when
    there is more than one chunk."""
    a = lambda x: (x + 255) // 256 * 256
    G = H // Hkv
    per_g = N * D * (G * es + 2 * es + G * oes)
    gc = next((g for g in range(1, Hkv + 1) if Hkv % g == 0 and g * per_g >= 64 << 20), Hkv)
    chunks = B * (Hkv // gc)
    slot = a(N * G * gc * D * es) + 2 * a(N * gc * D * es) + a(N * G * gc * D * oes) + a(gqa_ws(1, N, G * gc, gc))
    return (2 if chunks > 1 else 1) * slot


@pytest.mark.parametrize("B,N,H,Hkv,D,bs,ratio,dt", [
    (1, 131072, 16, 16, 128, 128, 0.15, torch.bfloat16),   # one head per chunk, 16 chunks
    (32, 8192, 16, 16, 64, 64, 0.3, torch.bfloat16),        # one batch entry per chunk
    (1, 1024, 4, 2, 64, 64, 0.5, torch.float32),            # a single chunk: one slot
    (2, 65536, 8, 2, 128, 128, 0.2, torch.float8_e4m3fn),   # e4m3 in, bf16 out
])
def test_host_workspace_bytes(bsa, B, N, H, Hkv, D, bs, ratio, dt):
    es = {torch.float32: 4, torch.bfloat16: 2, torch.float8_e4m3fn: 1}[dt]
    oes = 4 if dt == torch.float32 else 2
    gqa_ws = lambda b, n, h, hk: bsa.lib.bsa_forward_gqa_workspace_bytes(b, n, h, hk, D, bs, float(ratio))
    want = _host_plan_bytes(B, N, H, Hkv, D, bs, ratio, es, oes, gqa_ws)
    assert bsa.bsa_forward_host_workspace_bytes(B, N, H, D, bs, ratio, dt, H_kv=Hkv) == want


def test_host_workspace_bytes_rejects_bad_sizes(bsa):
    f = bsa.lib.bsa_forward_host_workspace_bytes
    assert f(1, 1000, 2, 2, 64, 64, 0.5, 1) == 0   # N not a multiple of block_size
    assert f(1, 1024, 3, 2, 64, 64, 0.5, 1) == 0   # H not a multiple of H_kv
    assert f(1, 1024, 2, 2, 64, 64, 0.01, 1) == 0  # k = 0
    assert f(1, 1024, 2, 2, 64, 64, 0.5, 7) == 0   # no such dtype


def test_polynomial_exp2_of_the_softmax():
    """The kernels' polynomial 2^x (one key pair in four of the softmax), as
    the header defines it, evaluated step by step in float32: the range
    split, the degree-3 polynomial and the exponent added through
    bits(x + 1.5 * 2^23) << 23. Its relative error stays below 1e-4 on the
    range the softmax uses (far below the bf16 rounding of P, up to 2^-8), and the
    clamp gives 2^-125-sized values below it."""
    import numpy as np

    src = open(os.path.join(ROOT, "block_sparse_attention_19_b200", "csrc", "bsa_ptx.cuh")).read()
    c = {k: np.float32(v) for k, v in re.findall(r"(kExp2C\d) = ([0-9.e+-]+)f", src)}
    assert len(c) == 4
    x = np.concatenate([np.linspace(-30, 8, 2_000_001), [-124.9, -125.0, -200.0, -1e30]]).astype(np.float32)
    xc = np.maximum(x, np.float32(-125.0))
    rnd = np.float32(12582912.0)
    t = (xc + rnd).astype(np.float32)
    f = (xc - (t - rnd)).astype(np.float32)
    p = c["kExp2C3"]
    for k in ("kExp2C2", "kExp2C1", "kExp2C0"):
        p = (p * f + c[k]).astype(np.float32)
    bits = (t.view(np.int32).astype(np.int64) * 8388608 + p.view(np.int32).astype(np.int64)) & 0xFFFFFFFF
    y = bits.astype(np.uint32).view(np.float32).astype(np.float64)
    ref = np.exp2(np.maximum(x.astype(np.float64), -125.0))
    assert np.all(np.abs(y / ref - 1) < 1e-4), np.abs(y / ref - 1).max()


def _host_fwd(bsa, q=A, k=A, v=A, o=A + 0x100, B=1, N=512, H=2, Hkv=2, D=64, bs=64, ratio=0.25, dt=1, flags=0,
              ws=A + 0x200, wsb=1 << 30):
    P = ctypes.c_void_p
    return bsa.lib.bsa_forward_host(P(q), P(k), P(v), P(o), B, N, H, Hkv, D, bs, ratio, dt, flags, P(ws), wsb,
                                    P(0))


@pytest.mark.parametrize("kw,status", [
    (dict(q=0), 1), (dict(o=0), 1), (dict(N=500), 1), (dict(Hkv=3), 1), (dict(ratio=0.01), 1),
    (dict(flags=8), 1), (dict(flags=2), 1), (dict(D=96), 2), (dict(dt=7), 2), (dict(ws=0), 4),
    (dict(wsb=16), 4), (dict(ws=A + 0x210), 3),
])
def test_host_entry_point_rejects_bad_arguments(bsa, kw, status):
    """bsa_forward_host validates on the host before touching a device (the
    host pointers are not dereferenced here)."""
    assert _host_fwd(bsa, **kw) == status


def _bwd_gqa(bsa, H=4, Hkv=2, D=64, bs=128, kk=2, dt=1, flags=0, scale=0.125, ws=A + 0x400, wsb=1 << 30, dq=A + 0x100):
    P = ctypes.c_void_p
    return bsa.lib.bsa_sparse_attn_bwd_gqa(P(A), P(A), P(A), P(A), P(A), P(A), P(A), P(dq), P(A + 0x200),
                                           P(A + 0x300), 1, 1024, H, Hkv, D, bs, kk, scale, dt, flags, P(ws), wsb,
                                           P(0))


@pytest.mark.parametrize("kw,status", [
    (dict(Hkv=3), 1), (dict(flags=0x100), 2), (dict(dt=0), 2), (dict(kk=0), 1), (dict(kk=9), 1),
    (dict(scale=0.0), 1), (dict(flags=2), 1), (dict(dq=A), 1), (dict(ws=0), 4), (dict(wsb=8), 4),
])
def test_grouped_backward_rejects_bad_arguments(bsa, kw, status):
    assert _bwd_gqa(bsa, **kw) == status


def test_grouped_training_workspace_is_per_key_value_head(bsa):
    """The backward's bit matrix is per key/value head, D per query head."""
    f = bsa.lib.bsa_sparse_attn_bwd_gqa_workspace_bytes
    a = lambda x: (x + 255) // 256 * 256
    B, N, H, Hkv, bs = 2, 8192, 8, 2, 128
    nb = N // bs
    assert f(B, N, H, Hkv, 128, bs) == a(B * Hkv * nb * ((nb + 31) // 32) * 4) + a(B * H * N * 4)
    assert bsa.lib.bsa_sparse_attn_bwd_workspace_bytes(B, N, H, 128, bs) == f(B, N, H, H, 128, bs)
    assert f(B, N, H, 3, 128, bs) == 0


def test_binding_refuses_mismatched_shapes_before_the_device(bsa):
    """The C ABI takes plain pointers, so the binding checks the tensors'
    shapes first: a mismatch would otherwise read past a buffer on the GPU.
    CPU tensors reach these checks before the device check."""
    q = torch.zeros(1, 512, 4, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 512, 2, 64, dtype=torch.bfloat16)
    bad = [
        lambda: bsa.bsa_forward(q, k, torch.zeros(1, 512, 4, 64, dtype=torch.bfloat16), 64, 0.5),  # v != k
        lambda: bsa.bsa_forward(q, torch.zeros(1, 512, 3, 64, dtype=torch.bfloat16),
                                torch.zeros(1, 512, 3, 64, dtype=torch.bfloat16), 64, 0.5),  # 4 % 3
        lambda: bsa.bsa_forward(q, torch.zeros(1, 256, 2, 64, dtype=torch.bfloat16),
                                torch.zeros(1, 256, 2, 64, dtype=torch.bfloat16), 64, 0.5),  # N differs
        lambda: bsa.bsa_forward(q, k, k, 64, 0.5, out=torch.zeros(1, 512, 2, 64, dtype=torch.bfloat16)),
        lambda: bsa.bsa_sparse_attn_fwd(q, k, k, torch.zeros(1, 4, 8, 2, dtype=torch.int32), 64),  # idx per kv head
        lambda: bsa.bsa_sparse_attn_fwd_train(q, k, k, torch.zeros(1, 2, 8, 2, dtype=torch.int32), 64,
                                              lse=torch.zeros(1, 512, 4)),
        lambda: bsa.bsa_sparse_attn_bwd(q, k, k, q, q[:, :256], torch.zeros(1, 2, 8, 2, dtype=torch.int32),
                                        torch.zeros(1, 4, 512), 64),  # do
        lambda: bsa.bsa_forward_noalloc(q, k, k, 64, 0.5),  # no grouped queries there
        lambda: bsa.bsa_forward_host(q, k, k, 64, 0.5, out=torch.zeros(1, 512, 4, 64)),  # out dtype
        lambda: bsa.bsa_block_scores_topk(torch.zeros(1, 4, 8, 64), torch.zeros(1, 2, 9, 64), 2),
        lambda: bsa.bsa_block_pool(q, 64, out=torch.zeros(1, 4, 4, 64)),
    ]
    for i, f in enumerate(bad):
        with pytest.raises((ValueError, TypeError)) as e:
            f()
        assert "CUDA tensor" not in str(e.value), (i, str(e.value))
    # consistent shapes pass these checks and stop at the device check
    idx = torch.zeros(1, 2, 8, 2, dtype=torch.int32)
    for f in (lambda: bsa.bsa_forward(q, k, k, 64, 0.5),
              lambda: bsa.bsa_sparse_attn_fwd(q, k, k, idx, 64),
              lambda: bsa.bsa_sparse_attn_fwd_train(q, k, k, idx, 64, lse=torch.zeros(1, 4, 512)),
              lambda: bsa.bsa_sparse_attn_bwd(q, k, k, q, q, idx, torch.zeros(1, 4, 512), 64),
              lambda: bsa.bsa_block_scores_topk(torch.zeros(1, 4, 8, 64), torch.zeros(1, 2, 8, 64), 2)):
        with pytest.raises(ValueError, match="CUDA tensor"):
            f()


# ---------------------------------------------------------------- overlapping key windows

@pytest.mark.parametrize("N,bs,ratio", [(4096, 128, 0.25), (8192, 64, 0.25), (131072, 128, 0.25), (2048, 256, 0.5),
                                        (1024, 128, 0.0), (128, 128, 0.25)])
def test_overlap_window_count_matches_the_oracle(bsa, oracle_mod, N, bs, ratio):
    assert bsa.bsa_overlap_window_count(N, bs, ratio) == len(oracle_mod.window_starts(N, bs, int(ratio * bs)))


def test_overlap_window_count_rejects_bad_input(bsa):
    assert bsa.bsa_overlap_window_count(1000, 128, 0.25) == -1  # N % block_size
    assert bsa.bsa_overlap_window_count(1024, 128, 1.0) == -1
    assert bsa.bsa_overlap_window_count(1024, 128, -0.1) == -1


def _ovl_fwd(bsa, flags=0, ratio=0.25, ovr=0.25, ws=A + 0x400, wsb=1 << 30, H=2, Hkv=2):
    P = ctypes.c_void_p
    return bsa.lib.bsa_forward_overlap(P(A), P(A + 0x100), P(A + 0x200), P(A + 0x300), 1, 1024, H, Hkv, 64, 128,
                                       ratio, ovr, 1, flags, P(ws), wsb, P(0))


@pytest.mark.parametrize("kw,status", [
    (dict(flags=1), 2), (dict(flags=4), 2), (dict(flags=8), 1), (dict(ovr=1.0), 1), (dict(ovr=-0.5), 1),
    (dict(ratio=0.01), 1), (dict(ws=0), 4), (dict(wsb=64), 4), (dict(ws=A + 0x410), 3), (dict(Hkv=3), 1),
])
def test_overlap_entry_point_rejects_bad_arguments(bsa, kw, status):
    """bsa_forward_overlap validates on the host before touching a device."""
    assert _ovl_fwd(bsa, **kw) == status


def test_overlap_workspace_bytes(bsa):
    # N 1024, block_size 128, overlap 32: 11 windows, k = int(0.25 * 11) = 2
    got = bsa.bsa_forward_overlap_workspace_bytes(1, 1024, 2, 64, 128, 0.25, 0.25)
    a = lambda x: (x + 255) // 256 * 256
    assert got == a(2 * 8 * 64 * 4) + a(2 * 11 * 64 * 4) + a(2 * 8 * 2 * 4) + a(2 * 8 * 11 * 4)
