"""Paging blocks between the device pool and pinned host memory (the block
pool of "Agent Memory Below the Prompt", section 2.1 items 1 and 3).

Exported images are byte-identical to the oracle's images of the same blocks;
imported images rebuild exactly the blocks the oracle rebuilds; an image whose
header does not fit its target is refused; a full Gemma-shaped layer survives
a round trip at permuted ids (same decode output, bit for bit), also while a
decode of other blocks runs on another stream.  Both paths are covered: block
ids on the device (the paging kernel) and on the host (the copy engines)."""
import numpy as np
import pytest
import torch

import decode_attention_q4kv_b200 as q4
from decode_attention_q4kv_b200 import _lib
from decode_attention_q4kv_b200 import workloads as W
from helpers import assert_pool_equal, cuda, host, oracle_pool
from oracle import q4kv_oracle as O

pytestmark = pytest.mark.gpu
WHERE = ["device", "host"]


def _ids(values, where):
    t = torch.tensor(values, dtype=torch.int32)
    return t.to(cuda()) if where == "device" else t


def _gpu_pool_like(k, v, ids, n_q4, n_q8, evict=()):
    pool = q4.Q4KVPool(k.shape[1], k.shape[2], n_q4, n_q8, device=cuda())
    pool.quantize(k.to(cuda()), v.to(cuda()), torch.tensor(ids, dtype=torch.int32, device=cuda()))
    ref = oracle_pool(k, v, ids, n_q4, n_q8)
    if evict:
        pool.invalidate(torch.tensor(evict, dtype=torch.int64, device=cuda()))
        ref.invalidate_slots(evict)
    return pool, ref


@pytest.mark.parametrize("where", WHERE)
@pytest.mark.parametrize("d,dtype,hkv", [(128, "fp16", 3), (256, "bf16", 2)])
def test_export_is_the_oracle_image(d, dtype, hkv, where):
    n = 4 * 256 - 77
    k, v = W.random_small(n, hkv, d, dtype, seed=31 + d)
    pool, ref = _gpu_pool_like(k, v, [4, 1, 0, 5], 3, 3, evict=[3, 256 + 9, 5 * 256 + 200])
    ids = [5, 0, 4, 1, 3]                       # 8-bit, 4-bit, ... and one never written
    images = pool.export_blocks(_ids(ids, where))
    torch.cuda.synchronize()
    assert pool.read_device_error() == 0
    stride = pool.image_stride()
    assert stride == ref.image_stride() and images.shape == (len(ids), stride)
    got = images.numpy()
    for i, blk in enumerate(ids):
        want = ref.block_image(blk)
        np.testing.assert_array_equal(got[i, :want.size], want, err_msg=f"image of block {blk}")


@pytest.mark.parametrize("where", WHERE)
@pytest.mark.parametrize("fp8", [False, True])
def test_import_rebuilds_the_oracle_blocks(fp8, where):
    d, hkv = 128, 2
    n = 3 * 256 - 5
    k, v = W.random_small(n, hkv, d, "fp16", seed=41)
    if fp8:
        src = O.OraclePool(hkv, d, 0, 4, k_rotated=False, fp8=True)
        dst_gpu = q4.Q4KVPool(hkv, d, 0, 4, k_rotated=False, fp8=True, device=cuda())
        dst = O.OraclePool(hkv, d, 0, 4, k_rotated=False, fp8=True)
        moves = {2: 0, 0: 3, 1: 2}
        kh, dt = host(k)
        vh, _ = host(v)
        src.quantize_blocks(kh, vh, dt, [2, 0, 1])
    else:
        src = oracle_pool(k, v, [1, 3, 0], 2, 2)
        dst_gpu = q4.Q4KVPool(hkv, d, 2, 2, device=cuda())
        dst = O.OraclePool(hkv, d, 2, 2)
        moves = {1: 0, 3: 2, 0: 1}               # same class on both sides
    src.invalidate_slots([7, 256 + 100])
    stride = dst_gpu.image_stride()
    images = torch.zeros((len(moves), stride), dtype=torch.uint8, pin_memory=True)
    for i, a in enumerate(moves):
        img = src.block_image(a)
        images[i, :img.size] = torch.from_numpy(img)
        assert dst.load_block_image(moves[a], img)
    dst_gpu.import_blocks(images, _ids(list(moves.values()), where))
    torch.cuda.synchronize()
    assert dst_gpu.read_device_error() == 0
    if fp8:
        for name in "kv":
            np.testing.assert_array_equal(getattr(dst_gpu, f"{name}_codes8").cpu().numpy(), dst.codes8[name])
        np.testing.assert_array_equal(dst_gpu.mask.cpu().numpy().view(np.uint32), dst.mask)
    else:
        assert_pool_equal(dst_gpu, dst)


@pytest.mark.parametrize("where", WHERE)
def test_import_refuses_images_that_do_not_fit(where):
    d, hkv = 128, 2
    k, v = W.random_small(512, hkv, d, "fp16", seed=43)
    pool, ref = _gpu_pool_like(k, v, [0, 2], 2, 2)
    before = [t.clone() for t in (pool.k_codes4, pool.k_codes8, pool.v_params8, pool.mask)]
    stride = pool.image_stride()
    images = torch.zeros((3, stride), dtype=torch.uint8, pin_memory=True)
    img4 = ref.block_image(0)
    images[0, :img4.size] = torch.from_numpy(img4)          # a 4-bit image aimed at an 8-bit block
    bad = img4.copy()
    bad[0] ^= 0xFF                                           # broken magic aimed at a 4-bit block
    images[1, :bad.size] = torch.from_numpy(bad)
    other = O.OraclePool(4, d, 2, 2)                          # another Hkv
    img_o = other.block_image(1)
    images[2, :min(img_o.size, stride)] = torch.from_numpy(img_o[:stride])
    if where == "device":
        pool.import_blocks(images, _ids([3, 1, 0], where))
        torch.cuda.synchronize()
        assert pool.read_device_error() == _lib.DEVERR_IMAGE
    else:   # the host checks every header first and enqueues nothing
        for i, blk in enumerate([3, 1, 0]):
            with pytest.raises(q4.Q4KVError):
                pool.import_blocks(images[i:i + 1], _ids([blk], where))
    for a, b in zip(before, (pool.k_codes4, pool.k_codes8, pool.v_params8, pool.mask)):
        assert torch.equal(a, b)


def test_out_of_range_ids_are_reported_and_skipped():
    k, v = W.random_small(256, 2, 128, "fp16", seed=47)
    pool, ref = _gpu_pool_like(k, v, [0], 2, 0)
    images = pool.export_blocks(torch.tensor([7, 0, -1], dtype=torch.int32, device=cuda()))
    torch.cuda.synchronize()
    assert pool.read_device_error() == _lib.DEVERR_BLOCK_ID
    want = ref.block_image(0)
    np.testing.assert_array_equal(images.numpy()[1, :want.size], want)
    # image 0 was never written (its id was out of range): aimed at block 1 it is refused by its header
    before = pool.k_codes4[1].clone()
    pool.import_blocks(images, torch.tensor([1, 9, 1 << 20], dtype=torch.int32, device=cuda()))
    torch.cuda.synchronize()
    assert pool.read_device_error() == _lib.DEVERR_BLOCK_ID | _lib.DEVERR_IMAGE
    assert torch.equal(pool.k_codes4[1], before)
    # host ids are checked before anything is enqueued
    for bad in ([7], [0, -1]):
        with pytest.raises(q4.Q4KVError):
            pool.export_blocks(_ids(bad, "host"))
        with pytest.raises(q4.Q4KVError):
            pool.import_blocks(images[:len(bad)], _ids(bad, "host"))


def _gemma_layer():
    w = W.GEMMA3_12B
    k, v = W.kv_tokens(w, 0, w.n_tokens, cuda())
    nb = w.n_tokens // 256
    pool = q4.Q4KVPool(w.n_kv_heads, w.head_dim, nb, 0, device=cuda())
    pool.quantize(k, v, torch.arange(nb, dtype=torch.int32, device=cuda()))
    q = W.query(w, 0, cuda())
    tables = W.identity_tables(w).to(cuda())
    lens = torch.full((w.batch,), w.ctx, dtype=torch.int32, device=cuda())
    return w, pool, q, tables, lens


@pytest.mark.parametrize("where", WHERE)
def test_full_layer_round_trip_keeps_decode_bit_identical(where):
    w, a, q, tables, lens = _gemma_layer()
    nb = a.n_blocks
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(5)).to(torch.int32)
    images = a.export_blocks(_ids(list(range(nb)), where))
    torch.cuda.synchronize()
    b = q4.Q4KVPool(w.n_kv_heads, w.head_dim, nb, 0, device=cuda())
    b.import_blocks(images, perm.to(cuda()) if where == "device" else perm)   # block i of a -> perm[i] of b
    torch.cuda.synchronize()
    assert a.read_device_error() == 0 and b.read_device_error() == 0
    inv = perm.long().to(cuda())
    for name in ("k_codes4", "v_codes4", "k_params4", "v_params4", "mask"):
        assert torch.equal(getattr(b, name)[inv], getattr(a, name)), name
    out_a = q4.decode_attention(a, q, tables, lens)
    out_b = q4.decode_attention(b, q, perm.to(cuda())[tables.long()], lens)
    torch.cuda.synchronize()
    assert torch.equal(out_a, out_b)


@pytest.mark.parametrize("where", WHERE)
def test_import_on_a_second_stream_beside_decode(where):
    """Blocks of one set of sequences come in on one stream while decode
    reads other blocks of the same pool on another."""
    w, a, q, tables, lens = _gemma_layer()
    nb = a.n_blocks
    half = nb // 2
    images = a.export_blocks(torch.arange(half, dtype=torch.int32, device=cuda()))
    ref_out = q4.decode_attention(a, q[3:], tables[3:], lens[3:])   # sessions 3, 4 own blocks >= half
    torch.cuda.synchronize()
    pool = q4.Q4KVPool(w.n_kv_heads, w.head_dim, nb, 0, device=cuda())
    # the upper half is resident (a plain copy of the arrays); the lower half pages in beside decode
    for name in ("k_codes4", "v_codes4", "k_params4", "v_params4", "mask"):
        getattr(pool, name)[half:].copy_(getattr(a, name)[half:])
    torch.cuda.synchronize()
    s_copy, s_dec = torch.cuda.Stream(), torch.cuda.Stream()
    ids = _ids(list(range(half)), where)
    with torch.cuda.stream(s_copy):
        pool.import_blocks(images, ids)
    with torch.cuda.stream(s_dec):
        out = q4.decode_attention(pool, q[3:], tables[3:], lens[3:])
    torch.cuda.synchronize()
    assert pool.read_device_error() == 0
    assert torch.equal(out, ref_out)
    for name in ("k_codes4", "v_codes4", "k_params4", "v_params4", "mask"):
        assert torch.equal(getattr(pool, name), getattr(a, name)), name
