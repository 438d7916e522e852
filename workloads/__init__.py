"""Seeded synthetic workloads for block-sparse attention.

This module only draws random inputs; it holds none of the method's
arithmetic, and both the CUDA path's tests/benchmark and the oracle's checks
take their inputs from here.

Recipe (the same for every config): with ``torch.Generator(device)`` seeded by
the config's seed, draw q, k, v as float32 [B, N, H, D] iid N(0, 1) in that
order, then per-block offsets q_off and k_off as float32 [B, nb, H, D] iid
N(0, sigma^2); add each offset to every row of its block of q (resp. k); cast
q, k, v to the config dtype (round to nearest even).  v gets no offset.  The
offsets give the block scores a structure, as on the page
"2026 新一代卷积与 Transformer 网络架构" (qqiyuan.cn), where a few blocks carry
most of the attention mass.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    B: int
    N: int
    H: int
    D: int
    block_size: int
    topk_ratio: float
    dtype: str  # "f32", "bf16" or "e4m3"
    offset_sigma: float
    seed: int
    sample_blocks: int | None  # query blocks per (b, h) the oracle checks; None = all
    note: str = ""
    H_kv: int | None = None  # key/value heads for grouped queries (None: H)

    @property
    def Hkv(self) -> int:
        return self.H if self.H_kv is None else self.H_kv

    @property
    def nb(self) -> int:
        return self.N // self.block_size

    @property
    def k(self) -> int:
        return int(self.topk_ratio * self.nb)

    @property
    def torch_dtype(self):
        return {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn}[self.dtype]

    @property
    def elem_bytes(self) -> int:
        return {"f32": 4, "bf16": 2, "e4m3": 1}[self.dtype]

    def with_ratio(self, ratio: float) -> "Config":
        return dataclasses.replace(self, topk_ratio=ratio, name=f"{self.name}@{ratio}")

    def describe(self) -> str:
        kv = "" if self.Hkv == self.H else f" H_kv={self.Hkv}"
        return (f"B={self.B} N={self.N} H={self.H}{kv} D={self.D} block_size={self.block_size} "
                f"(nb={self.nb}) topk_ratio={self.topk_ratio} (k={self.k}) {self.dtype}")


CONFIGS = {
    "c1": Config("c1", 1, 512, 2, 64, 64, 0.25, "f32", 1.0, 0, None,
                 "tiny fp32 non-causal MHA; also run at topk_ratio=1.0 (dense)"),
    "c2": Config("c2", 32, 8192, 16, 64, 64, 0.3, "bf16", 1.0, 1, None,
                 "page-1 benchmark shape: seq 8192, hidden 1024 = 16 x 64, batch 32"),
    "c3": Config("c3", 2, 32768, 16, 128, 128, 0.2, "bf16", 0.5, 2, None,
                 "closer block scores (offset sigma 0.5)"),
    "c4": Config("c4", 1, 131072, 16, 128, 128, 0.15, "bf16", 1.0, 3, 32,
                 "long context"),
    "c5": Config("c5", 1, 1048576, 8, 128, 256, 0.15, "bf16", 1.0, 4, 8,
                 "million-token context"),
}


def make_inputs(cfg: Config, device="cpu", seed: int | None = None):
    """Draw (q, k, v) for ``cfg`` on ``device`` following the module recipe."""
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed if seed is None else seed)
    # k and v have cfg.Hkv heads (= H unless grouped queries); the draw order
    # is the same either way
    shape = (cfg.B, cfg.N, cfg.H, cfg.D)
    kshape = (cfg.B, cfg.N, cfg.Hkv, cfg.D)
    q = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    k = torch.randn(kshape, generator=g, device=device, dtype=torch.float32)
    v = torch.randn(kshape, generator=g, device=device, dtype=torch.float32)
    q_off = torch.randn((cfg.B, cfg.nb, 1, cfg.H, cfg.D), generator=g, device=device,
                        dtype=torch.float32) * cfg.offset_sigma
    k_off = torch.randn((cfg.B, cfg.nb, 1, cfg.Hkv, cfg.D), generator=g, device=device,
                        dtype=torch.float32) * cfg.offset_sigma
    q.view(cfg.B, cfg.nb, cfg.block_size, cfg.H, cfg.D).add_(q_off)
    k.view(cfg.B, cfg.nb, cfg.block_size, cfg.Hkv, cfg.D).add_(k_off)
    dt = cfg.torch_dtype
    return q.to(dt), k.to(dt), v.to(dt)


def to_oracle_array(x: torch.Tensor):
    """Host numpy view of a tensor in the oracle's input convention
    (float32 as is, bfloat16 as raw uint16 bit patterns)."""
    x = x.detach().cpu().contiguous()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy().view("uint16")
    if x.dtype == torch.float8_e4m3fn:
        return x.view(torch.uint8).numpy()
    if x.dtype in (torch.float32, torch.float64):
        return x.numpy()
    raise TypeError(f"unsupported dtype {x.dtype}")


def sample_query_blocks(cfg: Config, count: int | None = None, seed_offset: int = 1000):
    """Per-(b, h) random query-block ids (sorted), drawn without replacement with
    numpy.random.default_rng(seed + seed_offset). Returns int32 [B, H, count]."""
    import numpy as np

    count = cfg.sample_blocks if count is None else count
    if count is None or count >= cfg.nb:
        return np.broadcast_to(np.arange(cfg.nb, dtype=np.int32), (cfg.B, cfg.H, cfg.nb)).copy()
    rng = np.random.default_rng(cfg.seed + seed_offset)
    rows = np.empty((cfg.B, cfg.H, count), np.int32)
    for b in range(cfg.B):
        for h in range(cfg.H):
            rows[b, h] = np.sort(rng.choice(cfg.nb, size=count, replace=False))
    return rows
