"""Seeded synthetic workloads for the Q4 KV-cache path.

This module only *draws inputs*: raw K/V/query tensors, outlier channel
choices, evicted slot sets and block-table permutations.  It contains none
of the method's arithmetic (no rotation, no quantisation, no attention), so
both the CUDA path and the CPU oracle can consume the same bytes.

Workload shapes follow the agent-serving set-ups the source pages describe:
Gemma 3 12B and Llama 3.1 8B agents with 256-token paged blocks ("Agent
Memory Below the Prompt", gist.science summary of arXiv 2603.04428, section
2.1), Qwen2.5-14B sessions with evicted slots (IntentKV article, section on
invalidating instead of compacting) and Llama-3.1-8B mixed-width handoff
(QKVShare, gist.science summary of arXiv 2605.03884, "Methodologie").
There is no dataset or model weight on this path; values are N(0, 1).

Random streams are keyed by (seed, layer, stream id) through splitmix64 and
drawn with torch's Philox generator on the requested device, so a device
tensor and its host copy are the same bytes.  CPU and CUDA generators give
different streams for the same key; every comparison copies one side's
bytes to the other.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Tuple

import torch

BLOCK_TOKENS = 256
GROUP = 64

STREAM_K = 0
STREAM_V = 1
STREAM_Q = 2
STREAM_OUTLIER = 3
STREAM_EVICT = 4
STREAM_PERM = 5
STREAM_WIDTH = 6

# Share of tokens at each width {2, 4, 8, 16} for a mixed-width card.  QKVShare
# assigns widths per token from {2, 4, 8, FP16} with a learned controller and
# reports no distribution; this fixed synthetic mix stands in for it.
CARD_WIDTH_MIX = ((2, 0.25), (4, 0.45), (8, 0.20), (16, 0.10))

_MASK64 = (1 << 64) - 1


def _splitmix64(x: int) -> int:
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def derive_seed(seed: int, layer: int, stream: int) -> int:
    """63-bit generator seed for one (workload seed, layer, stream) triple."""
    h = _splitmix64(seed & _MASK64)
    h = _splitmix64(h ^ (layer & _MASK64))
    h = _splitmix64(h ^ (stream & _MASK64))
    return h & ((1 << 63) - 1)


def generator(seed: int, layer: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(derive_seed(seed, layer, stream))
    return g


def torch_dtype(name: str) -> torch.dtype:
    return {"fp16": torch.float16, "bf16": torch.bfloat16,
            "fp32": torch.float32}[name]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic serving shape: `batch` sessions of `ctx` cached tokens."""

    name: str
    layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    batch: int
    ctx: int
    dtype: str = "fp16"
    seed: int = 0
    outliers: Optional[str] = None      # "per_head" | "fraction" | None
    outlier_count: int = 0              # per KV head ("per_head") or total ("fraction")
    outlier_scale: float = 1.0
    q8_fraction: float = 0.0            # share of blocks stored 8-bit
    evict_fraction: float = 0.0         # share of slots remapped to the sentinel
    permuted_pool: bool = False         # block tables permute a shared pool
    prefill_tokens: int = 0             # bulk-quantised prefill tiled over the pool

    @property
    def gqa(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def blocks_per_seq(self) -> int:
        return -(-self.ctx // BLOCK_TOKENS)

    @property
    def n_blocks(self) -> int:
        return self.batch * self.blocks_per_seq

    @property
    def n_tokens(self) -> int:
        return self.batch * self.ctx

    @property
    def n_q8_blocks(self) -> int:
        return int(math.floor(self.q8_fraction * self.n_blocks))

    @property
    def n_evicted_per_seq(self) -> int:
        return int(math.floor(self.evict_fraction * self.ctx))

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads.  Seeds follow "config i -> seed i-1".
TINY = Workload("tiny_1x1024_gqa4_d128", layers=1, n_q_heads=32, n_kv_heads=8,
                head_dim=128, batch=1, ctx=1024, dtype="fp16", seed=0,
                outliers="per_head", outlier_count=4, outlier_scale=10.0)
GEMMA3_12B = Workload("gemma3_12b_5x8192_d256", layers=48, n_q_heads=16,
                      n_kv_heads=8, head_dim=256, batch=5, ctx=8192,
                      dtype="bf16", seed=1, outliers="fraction",
                      outlier_count=41, outlier_scale=8.0)
LLAMA31_8B_MIXED = Workload("llama31_8b_10x32768_mixed48", layers=32,
                            n_q_heads=32, n_kv_heads=8, head_dim=128,
                            batch=10, ctx=32768, dtype="fp16", seed=2,
                            q8_fraction=0.25)
QWEN25_14B_EVICT = Workload("qwen25_14b_32x16384_evict60", layers=48,
                            n_q_heads=40, n_kv_heads=8, head_dim=128,
                            batch=32, ctx=16384, dtype="fp16", seed=3,
                            evict_fraction=0.6)
SWEEP_BASE = Workload("llama31_8b_sweep", layers=1, n_q_heads=32,
                      n_kv_heads=8, head_dim=128, batch=1, ctx=4096,
                      dtype="fp16", seed=4, permuted_pool=True,
                      prefill_tokens=131072)
SWEEP_BATCHES = (1, 16, 64, 256)
SWEEP_CONTEXTS = (4096, 32768, 131072)

WORKLOADS = {w.name: w for w in (TINY, GEMMA3_12B, LLAMA31_8B_MIXED,
                                 QWEN25_14B_EVICT)}


def sweep_point(batch: int, ctx: int) -> Workload:
    return SWEEP_BASE.with_(name=f"llama31_8b_sweep_b{batch}_c{ctx}",
                            batch=batch, ctx=ctx)


def sweep_points() -> List[Workload]:
    return [sweep_point(b, c) for b in SWEEP_BATCHES for c in SWEEP_CONTEXTS]


# ---------------------------------------------------------------------------
# draws
# ---------------------------------------------------------------------------

def normal(shape, seed: int, layer: int, stream: int, device="cpu") -> torch.Tensor:
    g = generator(seed, layer, stream, device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def outlier_channels(w: Workload, layer: int) -> List[Tuple[int, int]]:
    """(kv_head, channel) pairs whose K values are scaled up in `layer`."""
    if w.outliers is None:
        return []
    g = generator(w.seed, layer, STREAM_OUTLIER, "cpu")
    if w.outliers == "per_head":
        out = []
        for h in range(w.n_kv_heads):
            chans = torch.randperm(w.head_dim, generator=g)[: w.outlier_count]
            out.extend((h, int(c)) for c in chans)
        return out
    if w.outliers == "fraction":
        flat = torch.randperm(w.n_kv_heads * w.head_dim, generator=g)[: w.outlier_count]
        return [(int(f) // w.head_dim, int(f) % w.head_dim) for f in flat]
    raise ValueError(w.outliers)


def kv_tokens(w: Workload, layer: int, n_tokens: int, device="cpu",
              first_token: int = 0):
    """K and V rows [n_tokens][n_kv_heads][head_dim] in the workload dtype.

    Values are drawn in fp32, outlier K channels are scaled in fp32 and the
    result is rounded once (round-to-nearest-even) to fp16/bf16.  Rows
    `first_token .. first_token+n_tokens` of the layer's full draw are
    returned (the full draw is generated and sliced, so any slice is
    consistent with the whole).
    """
    total = first_token + n_tokens
    shape = (total, w.n_kv_heads, w.head_dim)
    k = normal(shape, w.seed, layer, STREAM_K, device)
    v = normal(shape, w.seed, layer, STREAM_V, device)
    for h, c in outlier_channels(w, layer):
        k[:, h, c] *= w.outlier_scale
    dt = torch_dtype(w.dtype)
    return (k[first_token:].to(dt).contiguous(), v[first_token:].to(dt).contiguous())


def kv_layer(w: Workload, layer: int, device="cpu"):
    """All sessions' K/V for one layer: [batch*ctx][n_kv_heads][head_dim]."""
    n = w.prefill_tokens if w.prefill_tokens else w.n_tokens
    return kv_tokens(w, layer, n, device)


def query(w: Workload, layer: int, device="cpu") -> torch.Tensor:
    q = normal((w.batch, w.n_q_heads, w.head_dim), w.seed, layer, STREAM_Q, device)
    return q.to(torch_dtype(w.dtype)).contiguous()


def evicted_positions(w: Workload) -> List[torch.Tensor]:
    """Per session, the sorted logical token positions remapped to the sentinel.

    Exactly floor(evict_fraction * ctx) positions per session, uniform
    without replacement; one permutation per session is drawn in session
    order from one stream, and the same sets apply to every layer.
    """
    n = w.n_evicted_per_seq
    if n == 0:
        return [torch.zeros(0, dtype=torch.int64) for _ in range(w.batch)]
    g = generator(w.seed, 0, STREAM_EVICT, "cpu")
    out = []
    for _ in range(w.batch):
        perm = torch.randperm(w.ctx, generator=g)
        out.append(torch.sort(perm[:n]).values)
    return out


def identity_tables(w: Workload) -> torch.Tensor:
    """Session b owns blocks b*blocks_per_seq ... in order (int32 [B][nb])."""
    nb = w.blocks_per_seq
    return torch.arange(w.batch * nb, dtype=torch.int32).view(w.batch, nb)


def permuted_tables(w: Workload) -> torch.Tensor:
    """Distinct blocks per sequence drawn as a seeded permutation of the pool."""
    nb = w.blocks_per_seq
    g = generator(w.seed, 0, STREAM_PERM, "cpu")
    perm = torch.randperm(w.batch * nb, generator=g).to(torch.int32)
    return perm.view(w.batch, nb).contiguous()


def seq_lens(w: Workload) -> torch.Tensor:
    return torch.full((w.batch,), w.ctx, dtype=torch.int32)


def evicted_slot_ids(w: Workload, tables: torch.Tensor) -> torch.Tensor:
    """Physical slot ids (block*256 + offset) of every evicted position."""
    out = []
    for b, pos in enumerate(evicted_positions(w)):
        if pos.numel() == 0:
            continue
        blk = tables[b].to(torch.int64)[pos // BLOCK_TOKENS]
        out.append(blk * BLOCK_TOKENS + pos % BLOCK_TOKENS)
    if not out:
        return torch.zeros(0, dtype=torch.int64)
    return torch.cat(out)


def random_small(n_tokens: int, n_kv_heads: int, head_dim: int, dtype: str,
                 seed: int, layer: int = 0, device="cpu", scale: float = 1.0):
    """Free-form K/V draw for edge-case tests (ragged sizes, odd shapes)."""
    shape = (n_tokens, n_kv_heads, head_dim)
    k = normal(shape, seed, layer, STREAM_K, device) * scale
    v = normal(shape, seed, layer, STREAM_V, device) * scale
    dt = torch_dtype(dtype)
    return k.to(dt).contiguous(), v.to(dt).contiguous()


def token_widths(n_tokens: int, seed: int, layer: int = 0, device="cpu",
                 mix=CARD_WIDTH_MIX) -> torch.Tensor:
    """uint8 [n_tokens] widths drawn independently from `mix` (seeded)."""
    g = generator(seed, layer, STREAM_WIDTH, "cpu")
    values = torch.tensor([w for w, _ in mix], dtype=torch.uint8)
    probs = torch.tensor([p for _, p in mix], dtype=torch.float64)
    idx = torch.multinomial(probs, n_tokens, replacement=True, generator=g) if n_tokens else \
        torch.zeros(0, dtype=torch.int64)
    return values[idx].to(device)
