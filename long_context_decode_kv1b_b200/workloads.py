"""Seeded synthetic inputs for the five benchmark / parity configurations.

This module holds only input recipes (shapes, distributions, seeds); none of the method's
arithmetic.  Tests, ``bench.py`` and the oracle all draw their inputs from here.  Data is drawn
with ``torch.Generator`` on the requested device, chunk by chunk, so a 1M-token cache never has
to exist uncompressed in one piece; any chunk can be regenerated on its own (e.g. to hand one
kv-head to the CPU oracle).

The pages evaluate on GSM8K / MMLU / HumanEval / perplexity sets ("H1B-KV", abstract and
experiment highlights); these seeded Gaussian caches stand in for them.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

HEAD_DIM = 128


@dataclass(frozen=True)
class Config:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    dtype: torch.dtype
    seed: int
    rotation_seed: int = 0
    steps: int = 0            # decode steps (append one token per sequence + attend)
    chunk: int = 4096         # prefill encode chunk
    outliers: bool = False    # 4 key channels per kv-head scaled x10
    token_scale: bool = False  # per (b, token) log-uniform scale in [1/2, 2] on K and V
    heavy: int = 0            # tokens per (b, kv-head) aligned with the query direction
    p: float = 0.0            # Top-p threshold (0 = full attention)
    scale: float = 1.0 / math.sqrt(HEAD_DIM)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def capacity(self) -> int:
        n = self.L + self.steps
        return (n + 127) // 128 * 128


CONFIGS = {
    "c1": Config("c1", B=1, Hq=1, Hkv=1, L=4096, dtype=torch.float32, seed=1),
    "c2": Config("c2", B=1, Hq=32, Hkv=32, L=8192, dtype=torch.bfloat16, seed=2, outliers=True),
    "c3": Config("c3", B=8, Hq=32, Hkv=8, L=32768, dtype=torch.bfloat16, seed=3, steps=16, token_scale=True),
    "c4": Config("c4", B=8, Hq=32, Hkv=8, L=32768, dtype=torch.bfloat16, seed=4, heavy=64, p=0.9),
    "c5": Config("c5", B=1, Hq=32, Hkv=8, L=1048576, dtype=torch.bfloat16, seed=5, steps=32, outliers=True),
    # not one of the five parity configurations: the long context with 64 query heads per 8 kv heads
    # (G = 8, a common grouping), for measurement only
    "c5g8": Config("c5g8", B=1, Hq=64, Hkv=8, L=1048576, dtype=torch.bfloat16, seed=5, steps=32, outliers=True),
}

DESCRIPTIONS = {
    "c1": "single head, batch 1, head_dim 128, context 4096; K,V,q fp32 N(0,1); full attention",
    "c2": "Llama-2-7B-shaped decode: 32 MHA heads, batch 1, context 8192, bf16, 4 outlier key channels x10",
    "c3": "Llama-3-8B-shaped GQA decode: 32q/8kv, batch 8, context 32768, 16 append+attend steps, token scales",
    "c4": "Top-p p=0.9 on 32q/8kv, batch 8, context 32768, 64 heavy tokens per head",
    "c5": "long context: 32q/8kv, batch 1, context 1,048,576, 32 append+attend steps, outlier key channels",
    "c5g8": "long context with G = 8: 64q/8kv, batch 1, context 1,048,576, 32 append+attend steps, outlier key channels",
}


def outlier_channels(h: int) -> list[int]:
    """Key channels scaled x10 for kv-head h: (17h + 31j + 5) mod 128, j = 0..3."""
    return [(17 * h + 31 * j + 5) % HEAD_DIM for j in range(4)]


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _stream_seed(cfg: Config, stream: int, index: int) -> int:
    return (cfg.seed * 1_000_003 + stream * 97_409 + index * 7_919) % (2**62)


def queries(cfg: Config, step: int, device) -> torch.Tensor:
    """Query of decode step `step` (0 for single-attend configs): [B, Hq, 128] in cfg.dtype."""
    g = _gen(device, _stream_seed(cfg, 1, step))
    q = torch.randn((cfg.B, cfg.Hq, HEAD_DIM), generator=g, device=device, dtype=torch.float32)
    return q.to(cfg.dtype)


def _shape_kv(cfg: Config, K: torch.Tensor, V: torch.Tensor, g: torch.Generator, device) -> None:
    if cfg.outliers:
        for h in range(cfg.Hkv):
            K[:, :, h, outlier_channels(h)] *= 10.0
    if cfg.token_scale:
        n = K.shape[1]
        u = torch.rand((cfg.B, n), generator=g, device=device, dtype=torch.float32)
        s = torch.exp(math.log(0.5) + u * (math.log(2.0) - math.log(0.5)))
        K.mul_(s[:, :, None, None])
        V.mul_(s[:, :, None, None])


def prefill_chunk(cfg: Config, start: int, n: int, device) -> tuple[torch.Tensor, torch.Tensor]:
    """Prefill tokens [start, start + n) (start a multiple of cfg.chunk, n <= cfg.chunk).
    Returns K, V as [B, n, Hkv, 128] in cfg.dtype."""
    assert start % cfg.chunk == 0 and n <= cfg.chunk
    g = _gen(device, _stream_seed(cfg, 2, start // cfg.chunk))
    K = torch.randn((cfg.B, n, cfg.Hkv, HEAD_DIM), generator=g, device=device, dtype=torch.float32)
    V = torch.randn((cfg.B, n, cfg.Hkv, HEAD_DIM), generator=g, device=device, dtype=torch.float32)
    _shape_kv(cfg, K, V, g, device)
    if cfg.heavy:
        _plant_heavy(cfg, K, start, n, g, device)
    return K.to(cfg.dtype), V.to(cfg.dtype)


def heavy_tokens(cfg: Config, device) -> torch.Tensor:
    """[B, Hkv, heavy] distinct token positions (sorted) that carry the query direction."""
    g = _gen(device, _stream_seed(cfg, 3, 0))
    idx = torch.stack([torch.stack([torch.randperm(cfg.L, generator=g, device=device)[: cfg.heavy]
                                    for _ in range(cfg.Hkv)]) for _ in range(cfg.B)])
    return idx.sort(dim=-1).values


def _plant_heavy(cfg: Config, K: torch.Tensor, start: int, n: int, g: torch.Generator, device) -> None:
    # k = 3 sqrt(128) * qhat + N(0, 1) for the heavy tokens; qhat = normalised mean of the group's queries.
    q = queries(cfg, 0, device).to(torch.float32).view(cfg.B, cfg.Hkv, cfg.G, HEAD_DIM).mean(dim=2)
    qhat = q / q.norm(dim=-1, keepdim=True)
    pos = heavy_tokens(cfg, device)
    gn = _gen(device, _stream_seed(cfg, 4, start // cfg.chunk))
    for b in range(cfg.B):
        for h in range(cfg.Hkv):
            p = pos[b, h]
            p = p[(p >= start) & (p < start + n)] - start
            if p.numel():
                noise = torch.randn((p.numel(), HEAD_DIM), generator=gn, device=device, dtype=torch.float32)
                K[b, p, h, :] = 3.0 * math.sqrt(HEAD_DIM) * qhat[b, h][None, :] + noise


def step_kv(cfg: Config, step: int, device) -> tuple[torch.Tensor, torch.Tensor]:
    """The token appended at decode step `step`: K, V as [B, 1, Hkv, 128] in cfg.dtype."""
    g = _gen(device, _stream_seed(cfg, 5, step))
    K = torch.randn((cfg.B, 1, cfg.Hkv, HEAD_DIM), generator=g, device=device, dtype=torch.float32)
    V = torch.randn((cfg.B, 1, cfg.Hkv, HEAD_DIM), generator=g, device=device, dtype=torch.float32)
    _shape_kv(cfg, K, V, g, device)
    return K.to(cfg.dtype), V.to(cfg.dtype)


def prefill_chunks(cfg: Config, L: int | None = None):
    """(start, n) of the prefill chunks covering [0, L)."""
    L = cfg.L if L is None else L
    return [(s, min(cfg.chunk, L - s)) for s in range(0, L, cfg.chunk)]
