"""Seeded synthetic decode workloads for the proposal -> refine -> sparse-decode path.

This module only shapes random inputs; it holds none of the method's
arithmetic (no quantization, scoring, selection or attention).  Both the CUDA
path and the CPU oracle consume the arrays it produces: a parity test
generates one set of arrays and hands the same values to both sides.

The pages measure on Qwen3 models under a serving stack (Prism Attention,
sec. 5.1 "Models and Benchmarks", sec. 5.3 "End-to-end latency"); no model or
dataset is used here.  The stand-in is a Llama-3-8B-shaped attention cache
(32 query heads / 8 KV heads, head_dim 128) whose structure models the
pages' observation that salient tokens shift only locally from layer to
layer (sec. 3 "Observations"):

* layer-0 keys and values are N(0,1); every later layer adds 0.3 * N(0,1)
  drift to the previous layer's raw keys / values;
* rotary position embedding (rotate-half pairing of feature j with j + d/2,
  frequency theta_j = base^(-2j/d), base 1e6 as for Qwen3 -- the geometric
  frequency ladder of "Prism: Spectral-Aware Block-Sparse Attention",
  sec. "Spectral Structure of RoPE") is applied to keys at their position and
  to the decode query at position L_b - 1;
* a fixed set of planted salient positions per (sequence, KV head) gets, in
  every layer, a key of unchanged norm at cosine 0.8 to one query head of the
  group (round-robin over the group);
* bf16 caches are rounded from fp32 with round-to-nearest-even (torch's cast).

Random numbers come from torch generators seeded from (seed, layer, stream);
CPU and CUDA generators give different streams, so a parity test always
copies one generated array to the other side instead of regenerating it.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterator, List, Optional

import torch

DRIFT = 0.3
SALIENT_COS = 0.8


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    seqlens: tuple  # per-sequence context length L_b
    num_layers: int
    group: int  # a layer l is a proposal layer when l % group == 0
    kappa_p: int
    kappa: int
    dtype: str  # "f32" or "bf16"
    rope: bool
    rope_base: float = 1e6
    n_salient: int = 64  # planted positions per (sequence, KV head)
    salient_spans: int = 0  # >0: positions come in this many contiguous spans
    seed: int = 0

    @property
    def G(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def cu_seqlens(self) -> List[int]:
        out = [0]
        for L in self.seqlens:
            out.append(out[-1] + int(L))
        return out

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def is_proposal(self, layer: int) -> bool:
        return layer % self.group == 0

    @property
    def proposal_layers(self) -> List[int]:
        return [l for l in range(self.num_layers) if self.is_proposal(l)]

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


def _ragged_lengths(batch: int, lo: int, hi: int, seed: int) -> tuple:
    g = torch.Generator(device="cpu")
    g.manual_seed(1_000_003 * (seed + 1) + 17)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (batch,), generator=g))


def config(name: str) -> Config:
    """The five workload configurations, by name.

    tiny      -- CPU-checkable: B=1, 1 KV head, 4 query heads, d=64, L=1024,
                 4 layers (layer 0 proposal), kappa_p=256, kappa=64, fp32,
                 no RoPE, 16 planted positions.
    c8k       -- B=1, 32q/8kv, d=128, L=8192, bf16, 8 layers, proposal every
                 4 layers, kappa_p=1024, kappa=256, 64 planted positions.
    c32k_b4   -- B=4, L=32768, 32 layers, proposal every 8, kappa_p=8192,
                 kappa=2048, planted positions in 8 contiguous spans of 8.
    c128k     -- headline: B=1, L=131072, 32 layers, proposal every 8,
                 kappa_p=8192, kappa=2048 (planted like c8k).
    ragged16  -- B=16, L_b uniform in [4096, 65536], 32 layers, proposal
                 every 4, kappa_p=4096, kappa=1024.
    """
    if name == "tiny":
        return Config("tiny", 1, 4, 1, 64, (1024,), 4, 4, 256, 64, "f32", False, n_salient=16)
    if name == "c8k":
        return Config("c8k", 1, 32, 8, 128, (8192,), 8, 4, 1024, 256, "bf16", True)
    if name == "c32k_b4":
        return Config("c32k_b4", 4, 32, 8, 128, (32768,) * 4, 32, 8, 8192, 2048, "bf16", True,
                      salient_spans=8)
    if name == "c128k":
        return Config("c128k", 1, 32, 8, 128, (131072,), 32, 8, 8192, 2048, "bf16", True)
    if name == "ragged16":
        return Config("ragged16", 16, 32, 8, 128, _ragged_lengths(16, 4096, 65536, 0), 32, 4,
                      4096, 1024, "bf16", True)
    raise KeyError(name)


CONFIG_NAMES = ("tiny", "c8k", "c32k_b4", "c128k", "ragged16")


@dataclasses.dataclass
class Layer:
    index: int
    q: torch.Tensor  # [B][Hq][d]
    k: torch.Tensor  # [Hkv][T][d] packed over sequences
    v: torch.Tensor  # [Hkv][T][d]


def _gen(seed: int, layer: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + layer * 7919 + stream * 104_729) & 0x7FFF_FFFF_FFFF)
    return g


def salient_positions(cfg: Config) -> List[List[torch.Tensor]]:
    """Planted positions per (sequence, KV head), fixed across layers (CPU int64)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(cfg.seed * 31 + 5)
    out = []
    for b, L in enumerate(cfg.seqlens):
        row = []
        for h in range(cfg.num_kv_heads):
            n = min(cfg.n_salient, L)
            if cfg.salient_spans > 0 and n > 0:
                spans = cfg.salient_spans
                width = max(1, n // spans)
                starts = torch.randperm(max(1, L // width), generator=g)[:spans] * width
                pos = (starts[:, None] + torch.arange(width)[None, :]).reshape(-1)
                pos = pos[pos < L]
            else:
                pos = torch.randperm(L, generator=g)[:n]
            row.append(torch.sort(pos).values)
        out.append(row)
    return out


def _rope_tables(max_len: int, d: int, base: float, device):
    j = torch.arange(d // 2, dtype=torch.float64, device=device)
    theta = base ** (-2.0 * j / d)
    ang = torch.arange(max_len, dtype=torch.float64, device=device)[:, None] * theta[None, :]
    return torch.cos(ang).float(), torch.sin(ang).float()


def _rope(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor) -> torch.Tensor:
    # x [..., n, d], cos/sin [n, d/2]: rotate-half pairing (j, j + d/2)
    h = x.shape[-1] // 2
    a, b = x[..., :h], x[..., h:]
    return torch.cat([a * cos - b * sin, a * sin + b * cos], dim=-1)


def generate(cfg: Config, device="cpu", layers: Optional[List[int]] = None) -> Iterator[Layer]:
    """Yield the layers of one decode step's cache, in layer order.

    Layers are produced by a drifting running sum, so every layer up to the
    last requested one is computed; only the requested ones are yielded.
    """
    device = torch.device(device)
    want = set(range(cfg.num_layers)) if layers is None else set(layers)
    last = max(want) if want else -1
    T, Hkv, Hq, d, G = cfg.total_tokens, cfg.num_kv_heads, cfg.num_q_heads, cfg.head_dim, cfg.G
    cu = cfg.cu_seqlens
    pos = torch.cat([torch.arange(L, device=device) for L in cfg.seqlens]) if T else \
        torch.zeros(0, dtype=torch.long, device=device)
    if cfg.rope and T:
        cos_t, sin_t = _rope_tables(max(cfg.seqlens), d, cfg.rope_base, device)
    sal = salient_positions(cfg)
    kraw = vraw = None
    for l in range(last + 1):
        gk, gv, gq, gu = (_gen(cfg.seed, l, s, device) for s in range(4))
        if l == 0:
            kraw = torch.randn((Hkv, T, d), generator=gk, device=device)
            vraw = torch.randn((Hkv, T, d), generator=gv, device=device)
        else:
            kraw.add_(torch.randn((Hkv, T, d), generator=gk, device=device), alpha=DRIFT)
            vraw.add_(torch.randn((Hkv, T, d), generator=gv, device=device), alpha=DRIFT)
        if l not in want:
            continue
        q = torch.randn((cfg.batch, Hq, d), generator=gq, device=device)
        if cfg.rope and T:
            k = torch.empty_like(kraw)
            step = 1 << 20
            for s0 in range(0, T, step):
                s1 = min(T, s0 + step)
                p = pos[s0:s1]
                k[:, s0:s1] = _rope(kraw[:, s0:s1], cos_t[p], sin_t[p])
            qpos = torch.tensor([max(L - 1, 0) for L in cfg.seqlens], device=device)
            q = _rope(q, cos_t[qpos][:, None, :], sin_t[qpos][:, None, :])
        else:
            k = kraw.clone()
        # planted salient keys: cosine 0.8 with one query head of the group
        for b in range(cfg.batch):
            for h in range(Hkv):
                p = sal[b][h].to(device)
                n = p.numel()
                if n == 0:
                    continue
                rows = cu[b] + p
                heads = h * G + (torch.arange(n, device=device) % G)
                qh = q[b, heads]
                qhat = qh / qh.norm(dim=-1, keepdim=True).clamp_min(1e-30)
                u = torch.randn((n, d), generator=gu, device=device)
                u = u - (u * qhat).sum(-1, keepdim=True) * qhat
                u = u / u.norm(dim=-1, keepdim=True).clamp_min(1e-30)
                norm = k[h, rows].norm(dim=-1, keepdim=True)
                k[h, rows] = norm * (SALIENT_COS * qhat + math.sqrt(1 - SALIENT_COS ** 2) * u)
        dt = cfg.torch_dtype
        # copies: the running sums are updated in place by the next layer
        yield Layer(l, q.to(dt, copy=True).contiguous(), k.to(dt).contiguous(),
                    vraw.to(dt, copy=True).contiguous())
