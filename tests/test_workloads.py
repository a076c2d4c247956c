"""The seeded synthetic inputs (host logic, no GPU): each stream is
reproducible from its key, the shapes and counts are the documented ones,
and the card widths follow their fixed mix."""
import collections

import torch

from decode_attention_q4kv_b200 import workloads as W


def test_streams_are_reproducible_and_distinct():
    a = W.normal((64, 8), seed=3, layer=1, stream=W.STREAM_K)
    b = W.normal((64, 8), seed=3, layer=1, stream=W.STREAM_K)
    c = W.normal((64, 8), seed=3, layer=1, stream=W.STREAM_V)
    d = W.normal((64, 8), seed=3, layer=2, stream=W.STREAM_K)
    assert torch.equal(a, b)
    assert not torch.equal(a, c) and not torch.equal(a, d)


def test_workload_shapes():
    g = W.GEMMA3_12B
    assert (g.batch, g.ctx, g.n_q_heads, g.n_kv_heads, g.head_dim, g.dtype) == (5, 8192, 16, 8, 256, "bf16")
    assert g.n_tokens == 40960 and g.n_blocks == 160 and g.gqa == 2
    e = W.QWEN25_14B_EVICT
    assert (e.batch, e.ctx, e.n_q_heads, e.head_dim) == (32, 16384, 40, 128) and e.gqa == 5
    assert e.n_evicted_per_seq == 9830                         # floor(0.6 * 16384)
    m = W.LLAMA31_8B_MIXED
    assert (m.batch, m.ctx, m.head_dim) == (10, 32768, 128)
    k, v = W.kv_tokens(W.TINY, 0, 300)
    assert k.shape == (300, 8, 128) and k.dtype == torch.float16 and torch.isfinite(k).all()


def test_evicted_slots_per_session():
    w = W.QWEN25_14B_EVICT.with_(batch=3, ctx=2048)
    tables = W.identity_tables(w)
    slots = W.evicted_slot_ids(w, tables)
    assert slots.numel() == 3 * w.n_evicted_per_seq
    per_seq = collections.Counter((slots // 256 // w.blocks_per_seq).tolist())
    assert all(n == w.n_evicted_per_seq for n in per_seq.values())
    assert slots.unique().numel() == slots.numel()              # without replacement


def test_permuted_tables_are_permutations_of_the_pool():
    w = W.sweep_point(16, 32768)
    t = W.permuted_tables(w)
    assert t.shape == (16, 128)
    flat = t.reshape(-1)
    assert flat.unique().numel() == flat.numel() and int(flat.min()) >= 0


def test_card_widths_follow_the_mix():
    n = 200000
    w = W.token_widths(n, seed=9)
    assert torch.equal(w, W.token_widths(n, seed=9))
    counts = collections.Counter(w.tolist())
    assert set(counts) == {2, 4, 8, 16}
    for width, share in W.CARD_WIDTH_MIX:
        assert abs(counts[width] / n - share) < 0.01, (width, counts[width] / n)
