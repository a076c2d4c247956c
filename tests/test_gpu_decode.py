"""Decode-attention parity on the GPU against the oracle's fp64 attention over
the same quantised cache (max-abs 2e-3, relative L2 1e-2), plus the
invariances the method promises."""
import numpy as np
import pytest
import torch

import decode_attention_q4kv_b200 as q4
from decode_attention_q4kv_b200 import workloads as W
from helpers import assert_close, cuda, host, oracle_pool, seq_tables
from oracle import q4kv_oracle as O

pytestmark = pytest.mark.gpu


class Case:
    """A pool holding `lens` sequences in random physical blocks, GPU and oracle."""

    def __init__(self, lens, hq, hkv, d, dtype="fp16", seed=0, n_pool=None, q8_blocks=(),
                 rotated=True, mb=None):
        self.lens = list(lens)
        nbs = [-(-n // 256) for n in self.lens]
        self.mb = mb or max(1, max(nbs))
        self.n_pool = n_pool or len(self.lens) * self.mb + 3
        q8 = sorted(set(q8_blocks))
        self.n_q8 = len(q8)
        self.n_q4 = self.n_pool - self.n_q8
        dev = cuda()
        self.pool = q4.Q4KVPool(hkv, d, self.n_q4, self.n_q8, k_rotated=rotated, device=dev)
        self.ref = O.OraclePool(hkv, d, self.n_q4, self.n_q8, k_rotated=rotated)
        tabs = seq_tables(len(self.lens), self.mb, self.n_pool, seed)
        self.tables = tabs
        self.k, self.v = [], []
        for b, n in enumerate(self.lens):
            if n == 0:
                self.k.append(None)
                self.v.append(None)
                continue
            k, v = W.random_small(n, hkv, d, dtype, seed=1000 * seed + b)
            ids = tabs[b, : nbs[b]]
            self.pool.quantize(k.to(dev), v.to(dev), ids.to(dev))
            kh, dt = host(k)
            vh, _ = host(v)
            self.ref.quantize_blocks(kh, vh, dt, ids.tolist())
            self.k.append(k)
            self.v.append(v)
        g = torch.Generator().manual_seed(seed + 77)
        q = torch.randn((len(self.lens), hq, d), generator=g)
        self.q = q.to(W.torch_dtype(dtype))
        self.lens_t = torch.tensor(self.lens, dtype=torch.int32)

    def invalidate(self, slots):
        slots = torch.as_tensor(slots, dtype=torch.int64)
        self.pool.invalidate(slots.to(cuda()))
        self.ref.invalidate_slots(slots.tolist())

    def run(self, n_splits=0, out_dtype=torch.float32, scale=0.0, kernel=1):
        dev = cuda()
        plan = q4.DecodePlan(len(self.lens), self.q.shape[1], self.pool.n_kv_heads, self.q.shape[2],
                             self.mb, n_splits=n_splits)
        plan.c.kernel = kernel      # 1: tensor-core pipeline (default), 0: CUDA-core kernel
        out = q4.decode_attention(self.pool, self.q.to(dev), self.tables.to(dev), self.lens_t.to(dev),
                                  softmax_scale=scale, out_dtype=out_dtype, plan=plan)
        torch.cuda.synchronize()
        return out, plan

    def oracle(self, scale=0.0):
        qh, dt = host(self.q)
        return O.decode_attention(self.ref, qh, dt, self.tables.numpy(), self.lens, softmax_scale=scale)


def test_tiny_workload():
    w = W.TINY
    dev = cuda()
    k, v = W.kv_layer(w, 0)
    q = W.query(w, 0)
    pool = q4.Q4KVPool(w.n_kv_heads, w.head_dim, w.n_blocks, device=dev)
    tables = W.identity_tables(w)
    pool.quantize(k.to(dev), v.to(dev), tables.view(-1).to(dev))
    out = q4.decode_attention(pool, q.to(dev), tables.to(dev), W.seq_lens(w).to(dev), out_dtype=torch.float32)
    ref = oracle_pool(k, v, tables.view(-1).tolist(), w.n_blocks)
    qh, dt = host(q)
    want = O.decode_attention(ref, qh, dt, tables.numpy(), W.seq_lens(w).tolist())
    assert_close(out, want, what="tiny")
    assert pool.read_device_error() == 0


@pytest.mark.parametrize("kernel", [1, 0])
@pytest.mark.parametrize("n_splits", [0, 1, 2, 7, 64])
def test_ragged_lengths_and_splits(n_splits, kernel):
    c = Case([1000, 1, 257, 0, 513, 256], hq=32, hkv=8, d=128, seed=1)
    out, plan = c.run(n_splits, kernel=kernel)
    assert_close(out, c.oracle(), what=f"splits={plan.n_splits}")
    assert torch.all(out[3] == 0)


@pytest.mark.parametrize("hq,hkv,d,dtype", [(16, 8, 256, "bf16"), (40, 8, 128, "fp16"),
                                            (8, 8, 128, "fp16"), (8, 1, 128, "bf16"),
                                            (4, 1, 256, "fp16"), (12, 4, 128, "bf16")])
@pytest.mark.parametrize("kernel", [1, 0])
def test_gqa_shapes(hq, hkv, d, dtype, kernel):
    c = Case([700, 300], hq=hq, hkv=hkv, d=d, dtype=dtype, seed=2)
    out, _ = c.run(kernel=kernel)
    assert_close(out, c.oracle(), what=f"{hq}/{hkv}/{d}")


@pytest.mark.parametrize("d,hq", [(128, 32), (256, 16)])
def test_mixed_q8_blocks(d, hq):
    c = Case([900, 600], hq=hq, hkv=8, d=d, seed=3, n_pool=8, q8_blocks=(4, 5, 6))
    # make sure some sequence blocks are 8-bit: the table uses ids drawn from the whole pool
    assert any(int(x) >= c.n_q4 for x in c.tables.view(-1))
    for s in (0, 3):
        out, _ = c.run(s)
        assert_close(out, c.oracle(), what="mixed")


def test_eviction_mask_and_scribble_invariance():
    c = Case([2048, 1500], hq=40, hkv=8, d=128, seed=4)
    g = torch.Generator().manual_seed(5)
    slots = []
    for b, n in enumerate(c.lens):
        pos = torch.randperm(n, generator=g)[: int(0.6 * n)]
        blk = c.tables[b].to(torch.int64)[pos // 256]
        slots.append(blk * 256 + pos % 256)
    c.invalidate(torch.cat(slots))
    out, _ = c.run()
    assert_close(out, c.oracle(), what="evicted")
    # scribble random bytes (NaN patterns included) over every remapped slot's data
    mask = c.pool.mask.cpu().numpy().view(np.uint32)
    bits = np.unpackbits(mask.view(np.uint8), bitorder="little").reshape(mask.shape[0], 256).astype(bool)
    rng = np.random.default_rng(6)
    for name in ("k_codes4", "v_codes4", "k_params4", "v_params4"):
        t = getattr(c.pool, name)
        raw = t.view(torch.uint8).view(t.shape[0], t.shape[1], 256, -1)
        for blk in np.nonzero(bits.any(axis=1))[0]:
            sl = torch.from_numpy(np.nonzero(bits[blk])[0]).to(cuda())
            junk = torch.from_numpy(rng.integers(0, 256, size=(t.shape[1], len(sl), raw.shape[-1]),
                                                 dtype=np.uint8)).to(cuda())
            raw[blk][:, sl] = junk
    out2, _ = c.run()
    assert torch.equal(out, out2)


def test_all_masked_and_empty_rows_are_zero():
    c = Case([300, 0, 10], hq=8, hkv=2, d=128, seed=7)
    slots = [int(c.tables[0, t // 256]) * 256 + t % 256 for t in range(300)]
    c.invalidate(slots)
    for s in (0, 1, 3):
        out, _ = c.run(s)
        assert torch.all(out[0] == 0) and torch.all(out[1] == 0)
        assert_close(out, c.oracle(), what="masked")


def test_single_live_slot_returns_its_value():
    c = Case([700], hq=8, hkv=2, d=128, seed=8)
    keep = 333
    slots = [int(c.tables[0, t // 256]) * 256 + t % 256 for t in range(700) if t != keep]
    c.invalidate(slots)
    out, _ = c.run(3)
    blk = int(c.tables[0, keep // 256])
    _, vd = c.pool.dequantize(torch.tensor([blk], dtype=torch.int32, device=cuda()))
    v_keep = vd[0, :, keep % 256].cpu()                # [Hkv][D]
    want = v_keep.repeat_interleave(4, dim=0)
    assert torch.allclose(out[0].cpu(), want, atol=1e-6, rtol=0)


def test_block_permutation_invariance():
    lens = [800]
    a = Case(lens, hq=32, hkv=8, d=128, seed=9)
    b = Case(lens, hq=32, hkv=8, d=128, seed=9, n_pool=40)   # same data, other physical blocks
    assert not torch.equal(a.tables, b.tables)
    oa, _ = a.run(2)
    ob, _ = b.run(2)
    assert torch.equal(oa, ob)


@pytest.mark.parametrize("out_dtype", [torch.float16, torch.bfloat16])
def test_low_precision_outputs(out_dtype):
    c = Case([640, 129], hq=32, hkv=8, d=128, seed=10)
    o32, _ = c.run(2, torch.float32)
    olo, _ = c.run(2, out_dtype)
    assert torch.equal(olo, o32.to(out_dtype))
    ulp = 2.0 ** -10 if out_dtype == torch.float16 else 2.0 ** -7
    want = c.oracle()
    assert_close(olo, want, atol=2e-3 + ulp * float(np.abs(want).max()), what=str(out_dtype))


def test_softmax_scale_and_raw_keys():
    c = Case([500], hq=16, hkv=4, d=128, seed=11, rotated=False)
    out, _ = c.run(0, scale=0.05)
    assert_close(out, c.oracle(scale=0.05), what="raw keys, scale 0.05")


def test_bad_table_entry_and_length():
    c = Case([600, 600, 600], hq=8, hkv=2, d=128, seed=12)
    good, _ = c.run(2)
    torch.cuda.synchronize()
    assert c.pool.read_device_error() == 0
    c.tables[1, 1] = 10_000                       # block id beyond the pool
    c.lens_t[2] = 10 * 256                         # longer than the table allows
    out, _ = c.run(2)
    bits = c.pool.read_device_error()
    assert bits & 1 and bits & 2
    assert torch.all(out[1] == 0) and torch.all(out[2] == 0)
    assert torch.equal(out[0], good[0])


@pytest.mark.parametrize("kernel", [1, 0])
def test_long_sequences_with_mixed_widths_and_eviction(kernel):
    # long contexts accumulate many tiles: checks the offset-form value
    # accumulation and the lazy rescale over 32K tokens
    c = Case([32768, 20000], hq=8, hkv=2, d=128, seed=13, n_pool=300, q8_blocks=range(60))
    g = torch.Generator().manual_seed(14)
    slots = []
    for b, n in enumerate(c.lens):
        pos = torch.randperm(n, generator=g)[: n // 3]
        blk = c.tables[b].to(torch.int64)[pos // 256]
        slots.append(blk * 256 + pos % 256)
    c.invalidate(torch.cat(slots))
    want = c.oracle()
    for s in (0, 1):
        out, _ = c.run(s, kernel=kernel)
        assert_close(out, want, what=f"long, splits {s}")


@pytest.mark.parametrize("rotated", [True, False])
@pytest.mark.parametrize("big", [300.0, 3000.0, 30000.0])
def test_wide_dynamic_range_query(rotated, big):
    """Queries with one outlier channel per head (300, 3000 or 30000) and the
    rest N(0, 1e-2), fp16, over rotated and raw keys.  The decode kernel turns
    the (rotated) query into fixed point with one power-of-two scale per head,
    so the small channels keep only the precision the digits leave them; the
    outlier makes the softmax sharp, so near-ties between the top keys show
    any error of those small channels.  Element by element against the
    oracle's fp64 attention (max-abs 2e-3, relative L2 1e-2)."""
    c = Case([1200, 333, 2048], hq=32, hkv=8, d=128, seed=15, rotated=rotated)
    g = torch.Generator().manual_seed(16 + int(big))
    q = torch.randn(c.q.shape, generator=g) * 1e-2
    ch = torch.randint(0, q.shape[2], q.shape[:2], generator=g)
    q.scatter_(2, ch[..., None], big)
    c.q = q.to(torch.float16)
    for s in (0, 3):
        out, _ = c.run(s)
        assert_close(out, c.oracle(), what=f"outlier {big}, {'rotated' if rotated else 'raw'} keys, splits {s}")
