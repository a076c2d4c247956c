"""2-bit blocks in the paged pool (QKVShare, "Méthodologie": widths from
{2, 4, 8, FP16} in one cache), a third block class beside the 4- and 8-bit
ones: the encoder's codes, scales, zeros and masks are bit-identical to the
oracle's; decode over pools that mix 2-, 4- and 8-bit blocks in one sequence
is within the oracle tolerance in both column layouts and both head sizes;
append, dequantise, paging and invalidation handle the class."""
import numpy as np
import pytest
import torch

import decode_attention_q4kv_b200 as q4
from decode_attention_q4kv_b200 import workloads as W
from helpers import assert_close, assert_pool_equal, cuda, host, seq_tables
from oracle import q4kv_oracle as O

pytestmark = pytest.mark.gpu


class Mix:
    """Sequences in random blocks of a pool with n_q4 4-bit, n_q8 8-bit and
    n_q2 2-bit blocks (ids in that order), on the GPU and in the oracle."""

    def __init__(self, lens, hq, hkv, d, n_q4, n_q8, n_q2, dtype="fp16", seed=0, rotated=True):
        dev = cuda()
        self.lens = list(lens)
        nbs = [-(-n // 256) for n in self.lens]
        self.mb = max(1, max(nbs))
        n_pool = n_q4 + n_q8 + n_q2
        assert n_pool >= len(self.lens) * self.mb
        self.pool = q4.Q4KVPool(hkv, d, n_q4, n_q8, k_rotated=rotated, device=dev, n_q2_blocks=n_q2)
        self.ref = O.OraclePool(hkv, d, n_q4, n_q8, k_rotated=rotated, n_q2=n_q2)
        self.tables = seq_tables(len(self.lens), self.mb, n_pool, seed)
        for b, n in enumerate(self.lens):
            if n == 0:
                continue
            k, v = W.random_small(n, hkv, d, dtype, seed=500 * seed + b)
            ids = self.tables[b, : nbs[b]]
            self.pool.quantize(k.to(dev), v.to(dev), ids.to(dev))
            kh, dt = host(k)
            vh, _ = host(v)
            self.ref.quantize_blocks(kh, vh, dt, ids.tolist())
        g = torch.Generator().manual_seed(seed + 3)
        self.q = torch.randn((len(self.lens), hq, d), generator=g).to(W.torch_dtype(dtype))

    def classes(self):
        return {self.ref.bits(int(b)) for b in self.tables.view(-1)}

    def decode(self, n_splits=0):
        dev = cuda()
        plan = q4.DecodePlan(len(self.lens), self.q.shape[1], self.pool.n_kv_heads, self.q.shape[2], self.mb,
                             n_splits=n_splits)
        out = q4.decode_attention(self.pool, self.q.to(dev), self.tables.to(dev),
                                  torch.tensor(self.lens, dtype=torch.int32, device=dev),
                                  out_dtype=torch.float32, plan=plan)
        torch.cuda.synchronize()
        return out

    def oracle(self):
        qh, dt = host(self.q)
        return O.decode_attention(self.ref, qh, dt, self.tables.numpy(), self.lens)


@pytest.mark.parametrize("d,dtype,rotated", [(128, "fp16", True), (256, "bf16", True), (128, "bf16", False)])
def test_encode_bit_exact(d, dtype, rotated):
    m = Mix([1300, 517], 8, 4, d, 3, 2, 7, dtype=dtype, seed=1, rotated=rotated)
    assert 2 in m.classes()
    assert m.pool.read_device_error() == 0
    assert_pool_equal(m.pool, m.ref)


# (Hq, Hkv, D): pairs layout (g * D/64 <= 8) and heads layout, both head sizes
@pytest.mark.parametrize("hq,hkv,d", [(32, 8, 128), (40, 8, 128), (16, 8, 256), (16, 4, 256), (8, 1, 128)])
@pytest.mark.parametrize("n_splits", [0, 3])
def test_decode_over_mixed_2_4_8_blocks(hq, hkv, d, n_splits):
    m = Mix([2000, 777, 255], hq, hkv, d, 10, 6, 10, seed=2)
    assert m.classes() == {2, 4, 8}
    out = m.decode(n_splits)
    assert m.pool.read_device_error() == 0
    assert_close(out, m.oracle(), what=f"{hq}/{hkv}/{d} mixed 2/4/8, splits {n_splits}")


def test_decode_all_2bit_with_eviction():
    m = Mix([3000, 1024], 32, 8, 128, 0, 0, 24, seed=3)
    g = torch.Generator().manual_seed(4)
    slots = []
    for b, n in enumerate(m.lens):
        pos = torch.randperm(n, generator=g)[: n // 2]
        slots.append(m.tables[b].to(torch.int64)[pos // 256] * 256 + pos % 256)
    s = torch.cat(slots)
    m.pool.invalidate(s.to(cuda()))
    m.ref.invalidate_slots(s.tolist())
    assert_pool_equal(m.pool, m.ref)      # masks included
    out = m.decode()
    assert_close(out, m.oracle(), what="2-bit, half evicted")


def test_dequantize_2bit_blocks():
    m = Mix([700], 8, 2, 128, 1, 1, 3, seed=5)
    ids = [int(x) for x in m.tables[0, :3]]
    kd, vd = m.pool.dequantize(torch.tensor(ids, dtype=torch.int32, device=cuda()), unrotate_k=True)
    for i, blk in enumerate(ids):
        kh, vh = m.ref.dequantize_block(blk, unrotate_k=True)
        np.testing.assert_array_equal(kd[i].cpu().numpy(), kh)
        np.testing.assert_array_equal(vd[i].cpu().numpy(), vh)


def test_append_into_2bit_blocks():
    dev = cuda()
    d, hkv = 128, 4
    pool = q4.Q4KVPool(hkv, d, 2, 0, device=dev, n_q2_blocks=4)
    ref = O.OraclePool(hkv, d, 2, 0, n_q2=4)
    tables = np.array([[2, 3], [0, 4]], np.int32)         # sequence 0 all 2-bit, sequence 1 4-bit then 2-bit
    lens = [250, 254]
    for b in range(2):
        k, v = W.random_small(lens[b], hkv, d, "fp16", seed=60 + b)
        pool.quantize(k.to(dev), v.to(dev), torch.tensor(tables[b][:1], dtype=torch.int32, device=dev))
        kh, dt = host(k)
        vh, _ = host(v)
        ref.quantize_blocks(kh, vh, dt, tables[b][:1].tolist())
    kn, vn = W.random_small(2 * 5, hkv, d, "fp16", seed=70)
    pool.append(kn.view(2, 5, hkv, d).to(dev), vn.view(2, 5, hkv, d).to(dev), torch.tensor(tables).to(dev),
                torch.tensor(lens, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    kh, dt = host(kn)
    vh, _ = host(vn)
    ref.append_tokens(kh.reshape(2, 5, hkv, d), vh.reshape(2, 5, hkv, d), dt, tables, lens)
    assert pool.read_device_error() == 0
    assert_pool_equal(pool, ref)


@pytest.mark.parametrize("where", ["device", "host"])
def test_paging_2bit_images(where):
    m = Mix([600], 8, 2, 128, 2, 1, 3, seed=8)
    m.pool.invalidate(torch.tensor([m.tables[0, 0].item() * 256 + 7], dtype=torch.int64, device=cuda()))
    m.ref.invalidate_slots([m.tables[0, 0].item() * 256 + 7])
    ids = list(range(m.ref.n_blocks))
    t = torch.tensor(ids, dtype=torch.int32)
    images = m.pool.export_blocks(t.to(cuda()) if where == "device" else t)
    torch.cuda.synchronize()
    assert m.pool.image_stride() == m.ref.image_stride()
    for i, blk in enumerate(ids):
        want = m.ref.block_image(blk)
        np.testing.assert_array_equal(images.numpy()[i, :want.size], want, err_msg=f"block {blk}")
    other = q4.Q4KVPool(2, 128, 2, 1, device=cuda(), n_q2_blocks=3)
    other.import_blocks(images, t.to(cuda()) if where == "device" else t)
    torch.cuda.synchronize()
    assert other.read_device_error() == 0
    assert_pool_equal(other, m.ref)
