"""Appending tokens in place ([AMBP] 2.1 items 3-4): the GPU encoder writes each
new token at its sequence's position through the block table, bit-identical
to the oracle; a generation step (append, then decode) matches the oracle's
attention."""
import numpy as np
import pytest
import torch

import decode_attention_q4kv_b200 as q4
from decode_attention_q4kv_b200 import _lib
from decode_attention_q4kv_b200 import workloads as W
from helpers import assert_close, assert_pool_equal, cuda, host
from oracle import q4kv_oracle as O

pytestmark = pytest.mark.gpu


def _grow(d, hkv, dtype, rotated, n_q4, n_q8, lens, new, tables, max_new, strided=False, seed=0):
    """Prefill each sequence's first lens[b] tokens, then append; returns (gpu pool, oracle pool, k, v)."""
    dev = cuda()
    B = len(lens)
    name = "fp16" if dtype == torch.float16 else "bf16"
    pool = q4.Q4KVPool(hkv, d, n_q4, n_q8, k_rotated=rotated, device=dev)
    ref = O.OraclePool(hkv, d, n_q4, n_q8, k_rotated=rotated)
    for b in range(B):
        if lens[b] == 0:
            continue
        k, v = W.random_small(lens[b], hkv, d, name, seed=seed + 10 * b)
        nb = -(-lens[b] // 256)
        ids = tables[b][:nb].tolist()
        pool.quantize(k.to(dev), v.to(dev), torch.tensor(ids, dtype=torch.int32, device=dev))
        kh, dt = host(k)
        vh, _ = host(v)
        ref.quantize_blocks(kh, vh, dt, ids)
    kn, vn = W.random_small(B * max_new, hkv, d, name, seed=seed + 999)
    kn = kn.view(B, max_new, hkv, d)
    vn = vn.view(B, max_new, hkv, d)
    if strided:   # each sequence's rows inside a wider buffer, tokens 2 rows apart
        big_k = torch.zeros(B, 2 * max_new + 1, hkv, d, dtype=dtype)
        big_v = torch.zeros_like(big_k)
        big_k[:, 0:2 * max_new:2] = kn
        big_v[:, 0:2 * max_new:2] = vn
        kd, vd = big_k.to(dev)[:, 0:2 * max_new:2], big_v.to(dev)[:, 0:2 * max_new:2]
    else:
        kd, vd = kn.to(dev), vn.to(dev)
    nn = None if new is None else torch.tensor(new, dtype=torch.int32, device=dev)
    pool.append(kd, vd, torch.as_tensor(tables, dtype=torch.int32).to(dev),
                torch.tensor(lens, dtype=torch.int32, device=dev), nn)
    torch.cuda.synchronize()
    kh, dt = host(kn.reshape(B * max_new, hkv, d))
    vh, _ = host(vn.reshape(B * max_new, hkv, d))
    ref.append_tokens(kh.reshape(B, max_new, hkv, d), vh.reshape(B, max_new, hkv, d), dt,
                      np.asarray(tables), lens, new)
    return pool, ref


@pytest.mark.parametrize("d,hkv,dtype,rotated", [(128, 8, torch.float16, True), (256, 8, torch.bfloat16, True),
                                                 (128, 3, torch.bfloat16, False), (256, 1, torch.float16, True),
                                                 (256, 5, torch.bfloat16, False)])
@pytest.mark.parametrize("strided", [False, True])
def test_append_bit_exact(d, hkv, dtype, rotated, strided):
    # ragged lengths: empty, mid-block, one token before a block boundary, a
    # full block; ragged counts including 0; blocks of both widths
    lens = [0, 100, 255, 256, 510]
    new = [3, 1, 3, 0, 2]
    tables = np.array([[0, 7], [2, 9], [4, 1], [6, 3], [5, 8]], dtype=np.int32)
    pool, ref = _grow(d, hkv, dtype, rotated, 6, 4, lens, new, tables, 3, strided, seed=d + hkv)
    assert pool.read_device_error() == 0
    assert_pool_equal(pool, ref)


def test_append_all_tokens_when_counts_omitted():
    lens = [17, 300]
    tables = np.array([[1, 0], [2, 3]], dtype=np.int32)
    pool, ref = _grow(128, 8, torch.float16, True, 4, 0, lens, None, tables, 4)
    assert pool.read_device_error() == 0
    assert_pool_equal(pool, ref)


def test_append_past_the_table_and_bad_block_raise_and_skip():
    dev = cuda()
    hkv, d = 2, 128
    pool = q4.Q4KVPool(hkv, d, 4, device=dev)
    before = [pool.k_codes4.clone(), pool.mask.clone()]
    k, v = W.random_small(4, hkv, d, "fp16", seed=5)
    k = k.view(2, 2, hkv, d).to(dev)
    v = v.view(2, 2, hkv, d).to(dev)
    tables = torch.tensor([[0], [1]], dtype=torch.int32, device=dev)
    # sequence 0 is full (256 tokens, one block): both new tokens fall past the table
    pool.append(k[:1], v[:1], tables[:1], torch.tensor([256], dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    assert pool.read_device_error() & _lib.DEVERR_SEQ_LEN
    assert torch.equal(pool.k_codes4, before[0]) and torch.equal(pool.mask, before[1])
    bad = torch.tensor([[7]], dtype=torch.int32, device=dev)
    pool.append(k[1:], v[1:], bad, torch.tensor([0], dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    assert pool.read_device_error() & _lib.DEVERR_BLOCK_ID
    assert torch.equal(pool.k_codes4, before[0])


def test_generation_step_append_then_decode():
    # one decode step of a batch: append the new token of every sequence, then
    # attend over the grown cache with the new token included
    dev = cuda()
    hkv, hq, d = 8, 32, 128
    lens = [700, 256, 1, 1023]
    B = len(lens)
    tables = np.arange(B * 4, dtype=np.int32)[::-1].copy().reshape(B, 4)
    pool, ref = _grow(d, hkv, torch.float16, True, B * 4, 0, lens, [1] * B, tables, 1, seed=3)
    assert pool.read_device_error() == 0
    q = torch.randn(B, hq, d, generator=torch.Generator().manual_seed(4)).to(torch.float16)
    grown = [n + 1 for n in lens]
    out = q4.decode_attention(pool, q.to(dev), torch.as_tensor(tables).to(dev),
                              torch.tensor(grown, dtype=torch.int32, device=dev), out_dtype=torch.float32)
    qh, dt = host(q)
    want = O.decode_attention(ref, qh, dt, tables, grown)
    assert_close(out, want, what="append + decode")


def _prefilled(d, hkv, dtype, rotated, n_q4, n_q8, lens, tables, seed, n_q2=0, fp8=False):
    """Two GPU pools and an oracle pool holding each sequence's first lens[b] tokens."""
    dev = cuda()
    name = "fp16" if dtype == torch.float16 else "bf16"
    pools = [q4.Q4KVPool(hkv, d, n_q4, n_q8, k_rotated=rotated, device=dev, n_q2_blocks=n_q2, fp8=fp8)
             for _ in range(2)]
    ref = O.OraclePool(hkv, d, n_q4, n_q8, k_rotated=rotated, n_q2=n_q2, fp8=fp8)
    for b, n in enumerate(lens):
        if n == 0:
            continue
        k, v = W.random_small(n, hkv, d, name, seed=seed + 10 * b)
        ids = tables[b][: -(-n // 256)].tolist()
        for p in pools:
            p.quantize(k.to(dev), v.to(dev), torch.tensor(ids, dtype=torch.int32, device=dev))
        kh, dt = host(k)
        vh, _ = host(v)
        ref.quantize_blocks(kh, vh, dt, ids)
    return pools, ref


# (D, Hq, Hkv, input dtype, rotated K, 8-bit blocks): both column layouts, both
# head sizes, 4-bit-only and mixed pools
@pytest.mark.parametrize("d,hq,hkv,dtype,rotated,n_q8", [(128, 40, 8, torch.float16, True, 0),
                                                         (128, 32, 8, torch.bfloat16, False, 6),
                                                         (256, 16, 8, torch.bfloat16, True, 0),
                                                         (256, 8, 4, torch.float16, True, 6)])
@pytest.mark.parametrize("n_splits", [0, 1, 3])
def test_append_decode_matches_separate_calls_and_oracle(d, hq, hkv, dtype, rotated, n_q8, n_splits):
    """The generation step in one call (one decode launch whose extra warp
    encodes the new rows before the producer reads their blocks) gives
    exactly the pool and the output of an append followed by a decode over
    the grown lengths, and the oracle's."""
    dev = cuda()
    lens = [0, 100, 255, 256, 700, 1023]        # empty, mid-block, a block boundary crossed, full blocks
    new = [3, 1, 3, 0, 2, 1]
    B, max_new, mb = len(lens), 3, 5
    g = torch.Generator().manual_seed(d + hq + n_splits)
    tables = torch.randperm(B * mb, generator=g).to(torch.int32).view(B, mb).numpy()
    (fused, sep), ref = _prefilled(d, hkv, dtype, rotated, B * mb - n_q8, n_q8, lens, tables, seed=d + n_q8)
    name = "fp16" if dtype == torch.float16 else "bf16"
    kn, vn = W.random_small(B * max_new, hkv, d, name, seed=77)
    kn, vn = kn.view(B, max_new, hkv, d), vn.view(B, max_new, hkv, d)
    q = torch.randn(B, hq, d, generator=g).to(dtype)
    tab = torch.as_tensor(tables).to(dev)
    lens_d = torch.tensor(lens, dtype=torch.int32, device=dev)
    nn = torch.tensor(new, dtype=torch.int32, device=dev)
    grown = [n + a for n, a in zip(lens, new)]
    plan = q4.DecodePlan(B, hq, hkv, d, mb, n_splits=n_splits)
    out = q4.append_decode(fused, kn.to(dev), vn.to(dev), q.to(dev), tab, lens_d, nn, out_dtype=torch.float32,
                           plan=plan)
    sep.append(kn.to(dev), vn.to(dev), tab, lens_d, nn)
    want_gpu = q4.decode_attention(sep, q.to(dev), tab, torch.tensor(grown, dtype=torch.int32, device=dev),
                                   out_dtype=torch.float32, plan=plan)
    torch.cuda.synchronize()
    assert fused.read_device_error() == 0
    assert torch.equal(out, want_gpu)
    kh, dt = host(kn.reshape(B * max_new, hkv, d))
    vh, _ = host(vn.reshape(B * max_new, hkv, d))
    ref.append_tokens(kh.reshape(B, max_new, hkv, d), vh.reshape(B, max_new, hkv, d), dt, tables, lens, new)
    assert_pool_equal(fused, ref)
    qh, qdt = host(q)
    assert_close(out, O.decode_attention(ref, qh, qdt, tables, grown), what=f"append + decode {d}/{hq}/{hkv}")


@pytest.mark.parametrize("d,hq,hkv", [(128, 40, 8), (256, 16, 8), (256, 16, 4)])   # heads, pairs, heads
@pytest.mark.parametrize("n_q8", [0, 7])
def test_append_decode_rows_across_split_and_block_boundaries(d, hq, hkv, n_q8):
    """New rows of one sequence that fall in two splits (and two blocks,
    of different widths when the pool has 8-bit blocks): each split's item
    encodes its own part, and the result equals the two calls and the
    oracle."""
    dev = cuda()
    lens = [510, 0, 1020, 255]          # + new: 510..512 and 1020..1024 cross a split (512 tokens) and a block
    new = [3, 2, 5, 1]
    B, max_new, mb = len(lens), 5, 5
    tables = torch.randperm(B * mb, generator=torch.Generator().manual_seed(d + 3)).to(torch.int32).view(B, mb).numpy()
    (fused, sep), ref = _prefilled(d, hkv, torch.bfloat16, True, B * mb - n_q8, n_q8, lens, tables, seed=d + 5)
    kn, vn = W.random_small(B * max_new, hkv, d, "bf16", seed=41)
    kn, vn = kn.view(B, max_new, hkv, d), vn.view(B, max_new, hkv, d)
    q = torch.randn(B, hq, d, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    tab = torch.as_tensor(tables).to(dev)
    lens_d = torch.tensor(lens, dtype=torch.int32, device=dev)
    nn = torch.tensor(new, dtype=torch.int32, device=dev)
    grown = [n + a for n, a in zip(lens, new)]
    plan = q4.DecodePlan(B, hq, hkv, d, mb, n_splits=3)
    assert plan.c.tokens_per_split == 512
    out = q4.append_decode(fused, kn.to(dev), vn.to(dev), q.to(dev), tab, lens_d, nn, out_dtype=torch.float32,
                           plan=plan)
    sep.append(kn.to(dev), vn.to(dev), tab, lens_d, nn)
    want_gpu = q4.decode_attention(sep, q.to(dev), tab, torch.tensor(grown, dtype=torch.int32, device=dev),
                                   out_dtype=torch.float32, plan=plan)
    torch.cuda.synchronize()
    assert fused.read_device_error() == 0
    assert torch.equal(out, want_gpu)
    kh, dt = host(kn.reshape(B * max_new, hkv, d))
    vh, _ = host(vn.reshape(B * max_new, hkv, d))
    ref.append_tokens(kh.reshape(B, max_new, hkv, d), vh.reshape(B, max_new, hkv, d), dt, tables, lens, new)
    assert_pool_equal(fused, ref)
    qh, qdt = host(q)
    assert_close(out, O.decode_attention(ref, qh, qdt, tables, grown), what=f"rows across splits {d}")


def test_append_decode_all_new_tokens_and_no_new_tokens():
    """n_new omitted: every sequence appends max_new; max_new = 0: a plain decode."""
    dev = cuda()
    d, hq, hkv = 128, 32, 8
    lens = [300, 511]
    B, mb = len(lens), 3
    tables = np.array([[4, 0, 2], [1, 5, 3]], dtype=np.int32)
    (fused, sep), ref = _prefilled(d, hkv, torch.float16, True, 6, 0, lens, tables, seed=9)
    kn, vn = W.random_small(B * 2, hkv, d, "fp16", seed=8)
    kn, vn = kn.view(B, 2, hkv, d).to(dev), vn.view(B, 2, hkv, d).to(dev)
    q = torch.randn(B, hq, d, generator=torch.Generator().manual_seed(2)).to(torch.float16).to(dev)
    tab = torch.as_tensor(tables).to(dev)
    lens_d = torch.tensor(lens, dtype=torch.int32, device=dev)
    none = q4.append_decode(fused, kn[:, :0], vn[:, :0], q, tab, lens_d, out_dtype=torch.float32)
    plain = q4.decode_attention(sep, q, tab, lens_d, out_dtype=torch.float32)
    assert torch.equal(none, plain)
    out = q4.append_decode(fused, kn, vn, q, tab, lens_d, out_dtype=torch.float32)
    sep.append(kn, vn, tab, lens_d)
    want = q4.decode_attention(sep, q, tab, lens_d + 2, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fused.read_device_error() == 0
    assert torch.equal(out, want)


@pytest.mark.parametrize("kind", ["q2mix", "fp8"])
def test_append_decode_other_block_classes(kind):
    """The generation step over a pool mixing 2-, 4- and 8-bit blocks, and
    over the FP8 comparison cache: equal to the two calls, and to the oracle."""
    dev = cuda()
    d, hq, hkv = 128, 32, 8
    lens = [0, 255, 300, 1000]
    new = [2, 3, 1, 2]
    B, max_new, mb = len(lens), 3, 4
    tables = torch.randperm(B * mb, generator=torch.Generator().manual_seed(5)).to(torch.int32).view(B, mb).numpy()
    if kind == "q2mix":
        (fused, sep), ref = _prefilled(d, hkv, torch.float16, True, 6, 4, lens, tables, seed=31, n_q2=6)
    else:
        (fused, sep), ref = _prefilled(d, hkv, torch.float16, False, 0, B * mb, lens, tables, seed=31, fp8=True)
    kn, vn = W.random_small(B * max_new, hkv, d, "fp16", seed=32)
    kn, vn = kn.view(B, max_new, hkv, d), vn.view(B, max_new, hkv, d)
    q = torch.randn(B, hq, d, generator=torch.Generator().manual_seed(6)).to(torch.float16)
    tab = torch.as_tensor(tables).to(dev)
    lens_d = torch.tensor(lens, dtype=torch.int32, device=dev)
    nn = torch.tensor(new, dtype=torch.int32, device=dev)
    grown = [n + a for n, a in zip(lens, new)]
    out = q4.append_decode(fused, kn.to(dev), vn.to(dev), q.to(dev), tab, lens_d, nn, out_dtype=torch.float32)
    sep.append(kn.to(dev), vn.to(dev), tab, lens_d, nn)
    want_gpu = q4.decode_attention(sep, q.to(dev), tab, torch.tensor(grown, dtype=torch.int32, device=dev),
                                   out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fused.read_device_error() == 0
    assert torch.equal(out, want_gpu)
    kh, dt = host(kn.reshape(B * max_new, hkv, d))
    vh, _ = host(vn.reshape(B * max_new, hkv, d))
    ref.append_tokens(kh.reshape(B, max_new, hkv, d), vh.reshape(B, max_new, hkv, d), dt, tables, lens, new)
    assert_pool_equal(fused, ref)
    qh, qdt = host(q)
    assert_close(out, O.decode_attention(ref, qh, qdt, tables, grown), what=f"append + decode, {kind}")


def test_append_decode_past_the_table_raises_and_completes():
    """An append that lands past the block table: the append skips the token
    and raises Q4KV_DEVERR_SEQ_LEN, the decode over the grown length (beyond
    the table) writes a zero row and raises the same bit; the other
    sequence is unaffected, and the call completes (the decode then never
    reads a block the append writes, so only its final grid wait orders them)."""
    dev = cuda()
    d, hq, hkv = 128, 16, 4
    lens = [256, 100]
    tables = np.array([[0], [1]], dtype=np.int32)
    (fused, sep), ref = _prefilled(d, hkv, torch.float16, True, 2, 0, lens, tables, seed=41)
    kn, vn = W.random_small(2, hkv, d, "fp16", seed=42)
    kn, vn = kn.view(2, 1, hkv, d).to(dev), vn.view(2, 1, hkv, d).to(dev)
    q = torch.randn(2, hq, d, generator=torch.Generator().manual_seed(43)).to(torch.float16).to(dev)
    tab = torch.as_tensor(tables).to(dev)
    lens_d = torch.tensor(lens, dtype=torch.int32, device=dev)
    out = q4.append_decode(fused, kn, vn, q, tab, lens_d, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fused.read_device_error() & _lib.DEVERR_SEQ_LEN
    assert torch.count_nonzero(out[0]) == 0
    sep.append(kn[1:], vn[1:], tab[1:], lens_d[1:])
    want = q4.decode_attention(sep, q[1:], tab[1:].clone(), lens_d[1:] + 1, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(out[1:], want)
