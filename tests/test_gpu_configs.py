"""Parity at the workloads' full sizes, in the launch configuration bench.py
times (its Job: same pools, plans, fp16 output).  Sampled encoder rows are
compared bit for bit with the oracle; sampled (sequence, KV head) attention
rows are recomputed by the oracle from the same input bytes.  Layers are
sampled too (first and last, plus one in the middle where there are many)."""
import numpy as np
import pytest
import torch

from bench import Job, workload_by_name
from decode_attention_q4kv_b200 import workloads as W
from helpers import ATOL, RTOL_L2, host
from oracle import q4kv_oracle as O

pytestmark = pytest.mark.gpu


def _chunk_of_block(job, blk):
    """Input chunk (256 tokens) whose codes block `blk` holds."""
    if job.w.permuted_pool:
        return blk % (job.w.prefill_tokens // 256)
    return blk


def _check_encoder_rows(job, li, n=48, seed=0):
    """Random (block, head, slot) rows of the pool vs the oracle's encoding."""
    L = job.layers[li]
    pool = L["pool"]
    w = job.w
    rng = np.random.default_rng(seed)
    ids = job.last_ids.cpu().numpy() if job.last_ids is not None else None
    n_chunks = (w.prefill_tokens or w.n_tokens) // 256
    for _ in range(n):
        c = int(rng.integers(0, n_chunks))
        blk = int(ids[c]) if ids is not None else c
        h = int(rng.integers(0, w.n_kv_heads))
        slot = int(rng.integers(0, 256))
        tok = c * 256 + slot
        kv, dt = host(L["k"][tok, h][None])
        vv, _ = host(L["v"][tok, h][None])
        bits = 4 if blk < pool.n_q4_blocks else 8
        kf = O.rotate_f32(O.to_f32(kv, dt))
        for name, x in (("k", kf), ("v", O.to_f32(vv, dt))):
            codes, s_h, z_h = O.quantize_groups(x, bits)
            if bits == 4:
                got_c = getattr(pool, f"{name}_codes4")[blk, h, slot].cpu().numpy()
                got_p = getattr(pool, f"{name}_params4")[blk, h, slot].cpu().numpy()
                want_c = O.pack_nibbles(codes[0])
            else:
                i8 = blk - pool.n_q4_blocks
                got_c = getattr(pool, f"{name}_codes8")[i8, h, slot].cpu().numpy()
                got_p = getattr(pool, f"{name}_params8")[i8, h, slot].cpu().numpy()
                want_c = codes[0]
            np.testing.assert_array_equal(got_c, want_c, err_msg=f"{name} codes blk {blk} h {h} slot {slot}")
            want_p = np.stack([s_h[0], z_h[0]], axis=-1)
            np.testing.assert_array_equal(got_p.view(np.uint16), want_p.view(np.uint16))


def _check_attention(job, li, pairs, q8_chunks=None):
    """Oracle attention for (sequence, KV head) pairs from the same input bytes."""
    L = job.layers[li]
    w = job.w
    g = w.gqa
    tables = job.tables.cpu().numpy()
    evicted = W.evicted_positions(w) if w.evict_fraction else None
    out = L["out"].float().cpu().numpy()
    for b, kvh in pairs:
        nb = w.blocks_per_seq
        chunks = [_chunk_of_block(job, int(tables[b, i])) for i in range(nb)]
        toks = np.concatenate([np.arange(c * 256, c * 256 + 256) for c in chunks])[: w.ctx]
        tok_t = torch.from_numpy(toks).to(L["k"].device)
        kh, dt = host(L["k"][tok_t, kvh][:, None])
        vh, _ = host(L["v"][tok_t, kvh][:, None])
        wide = [bool(q8_chunks[c]) for c in chunks] if q8_chunks is not None else [False] * nb
        n8 = sum(wide)
        ids, i4, i8 = [], 0, 0
        for wd in wide:
            ids.append(nb - n8 + i8 if wd else i4)
            i8 += wd
            i4 += not wd
        ref = O.OraclePool(1, w.head_dim, nb - n8, n8)
        ref.quantize_blocks(kh, vh, dt, ids)
        if evicted is not None:
            pos = evicted[b].numpy()
            ref.invalidate_slots([ids[p // 256] * 256 + p % 256 for p in pos])
        qh, qdt = host(L["q"][b:b + 1, kvh * g:(kvh + 1) * g])
        want = O.decode_attention(ref, qh, qdt, np.array([ids]), [w.ctx])[0]
        got = out[b, kvh * g:(kvh + 1) * g]
        err = np.abs(got - want)
        atol = ATOL + 2.0 ** -11 * np.abs(want)            # fp16 output rounding on top
        assert np.all(err <= atol), f"b {b} kv {kvh}: max err {err.max():.3e}"
        rel = np.linalg.norm(got - want) / np.linalg.norm(want)
        assert rel <= RTOL_L2, f"b {b} kv {kvh}: rel {rel:.3e}"


def _run(name, layer_ids):
    w = workload_by_name(name)
    job = Job(w, torch.device("cuda", 0), 0, layer_ids)
    job.step()
    torch.cuda.synchronize()
    for L in job.layers:
        assert L["pool"].read_device_error() == 0
    return job


@pytest.mark.parametrize("name,layers", [("tiny", [0]), ("gemma", [0, 23, 47]), ("evict", [0, 47])])
def test_workload(name, layers):
    job = _run(name, layers)
    w = job.w
    rng = np.random.default_rng(1)
    for li in range(len(layers)):
        _check_encoder_rows(job, li, seed=li)
        pairs = [(0, 0), (w.batch - 1, w.n_kv_heads - 1), (int(rng.integers(w.batch)), int(rng.integers(w.n_kv_heads)))]
        _check_attention(job, li, pairs)


def test_mixed_workload():
    job = _run("mixed", [0, 31])
    w = job.w
    for li in range(2):
        L = job.layers[li]
        kh, dt = host(L["k"])
        am = O.block_absmean(kh, dt)
        want_ids = O.mixed_block_ids(am, w.n_q8_blocks, 0, w.n_blocks - w.n_q8_blocks)
        got_ids = job.ids_per_layer[li].cpu().numpy()
        np.testing.assert_array_equal(got_ids, want_ids)
        job.last_ids = job.ids_per_layer[li]
        _check_encoder_rows(job, li, seed=li)
        q8 = want_ids >= w.n_blocks - w.n_q8_blocks
        _check_attention(job, li, [(0, 0), (9, 7), (4, 3)], q8_chunks=q8)


@pytest.mark.parametrize("ctx", W.SWEEP_CONTEXTS)
@pytest.mark.parametrize("batch", W.SWEEP_BATCHES)
def test_sweep_point(batch, ctx):
    """Every point of the batch {1, 16, 64, 256} x context {4K, 32K, 128K}
    sweep, up to 256 x 128K (a 37.7 GB pool): sampled encoder rows bit-exact,
    three (sequence, KV head) rows against the oracle."""
    job = _run(f"sweep:{batch}:{ctx}", [0])
    _check_encoder_rows(job, 0)
    _check_attention(job, 0, [(0, 0), (batch - 1, 7), (batch // 2, 3)])
