"""Encoder/decoder parity on the GPU: codes, scales, zeros, packed bytes and
masks bit-identical to the oracle; dequantisation bit-identical too."""
import numpy as np
import pytest
import torch

import decode_attention_q4kv_b200 as q4
from decode_attention_q4kv_b200 import workloads as W
from helpers import assert_pool_equal, cuda, host, nblocks, oracle_pool
from oracle import q4kv_oracle as O

pytestmark = pytest.mark.gpu


def _quantize_both(k, v, ids, n_q4, n_q8=0, rotated=True):
    dev = cuda()
    pool = q4.Q4KVPool(k.shape[1], k.shape[2], n_q4, n_q8, k_rotated=rotated, device=dev)
    pool.quantize(k.to(dev), v.to(dev), torch.tensor(ids, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    assert pool.read_device_error() == 0
    ref = oracle_pool(k, v, ids, n_q4, n_q8, rotated)
    return pool, ref


def test_tiny_workload_bit_exact():
    w = W.TINY
    k, v = W.kv_layer(w, 0)
    ids = list(range(w.n_blocks))
    pool, ref = _quantize_both(k, v, ids, w.n_blocks)
    assert_pool_equal(pool, ref)


@pytest.mark.parametrize("d,dtype,hkv", [(128, torch.float16, 8), (128, torch.bfloat16, 3),
                                         (256, torch.bfloat16, 8), (256, torch.float16, 1)])
@pytest.mark.parametrize("rotated", [True, False])
def test_ragged_tokens_permuted_blocks(d, dtype, hkv, rotated):
    n = 1000                                     # 3 full blocks and a 232-token tail
    k, v = W.random_small(n, hkv, d, "fp16" if dtype == torch.float16 else "bf16", seed=11 + d + hkv)
    ids = [5, 0, 3, 6]
    pool, ref = _quantize_both(k, v, ids, 8, rotated=rotated)
    assert_pool_equal(pool, ref)


@pytest.mark.parametrize("d,hkv,n", [(128, 5, 1000), (256, 6, 777), (256, 16, 515), (128, 16, 3),
                                     (256, 3, 1), (128, 2, 261)])
@pytest.mark.parametrize("strided", [False, True])
def test_encoder_unit_shapes(d, hkv, n, strided):
    # head counts that leave a partial head chunk per unit, token tails shorter
    # than a unit, one-token calls, and rows that are not contiguous in memory
    k, v = W.random_small(n, hkv, d, "bf16", seed=70 + d + hkv + n)
    nb = nblocks(n)
    ids = list(range(nb - 1, -1, -1))
    dev = cuda()
    if strided:   # token stride Hkv*D + 8: each token's heads are copied on their own
        kk = torch.zeros(n, hkv * d + 8, dtype=k.dtype, device=dev)
        vv = torch.zeros(n, hkv * d + 8, dtype=v.dtype, device=dev)
        kk[:, :hkv * d] = k.reshape(n, -1).to(dev)
        vv[:, :hkv * d] = v.reshape(n, -1).to(dev)
        kk = kk[:, :hkv * d].view(n, hkv, d)
        vv = vv[:, :hkv * d].view(n, hkv, d)
    else:
        kk, vv = k.to(dev), v.to(dev)
    pool = q4.Q4KVPool(hkv, d, nb, 0, device=dev)
    pool.quantize(kk, vv, torch.tensor(ids, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    assert pool.read_device_error() == 0
    assert_pool_equal(pool, oracle_pool(k, v, ids, nb, 0))


def test_mixed_widths_and_strided_input():
    n, hkv, d = 700, 4, 128
    k, v = W.random_small(n, hkv, d, "fp16", seed=3)
    # K and V as slices of one fused [n][2][Hkv][D] tensor: token stride 2*Hkv*D
    fused = torch.stack([k, v], dim=1).to(cuda())
    kk, vv = fused[:, 0], fused[:, 1]
    ids = [3, 1, 4]                              # chunk 0 -> 8-bit (id 3 >= n_q4=3), chunks 1, 2 -> 4-bit
    dev = cuda()
    pool = q4.Q4KVPool(hkv, d, 3, 2, device=dev)
    pool.quantize(kk, vv, torch.tensor(ids, dtype=torch.int32, device=dev))
    ref = oracle_pool(k, v, ids, 3, 2)
    assert_pool_equal(pool, ref)


def test_edge_values():
    hkv, d = 2, 128
    rng = np.random.default_rng(0)
    base = rng.standard_normal((256, hkv, d)).astype(np.float32)
    base[0] = 0.0                                  # all-zero token: s = 0, codes 0
    base[1] = -0.0                                 # negative zeros
    base[2] = 0.1                                  # constant, not fp16-exact
    base[3, :, :64] = 3000.0                       # large, still fp16-safe after rotation
    base[3, :, 64:] = -3000.0
    base[4] = np.float32(2.0 ** -24)               # fp16 subnormals
    base[5, :, ::2] = 1e-7
    base[6] = rng.standard_normal((hkv, d)) * 1e4
    grid = np.arange(64, dtype=np.float32)
    base[7, :, :64] = -1.5 + (grid % 16) * 0.25    # exact ramp
    base[7, :, 64:] = -1.5 + ((grid % 15) + 0.5) * 0.25   # ties
    base[7, :, 64] = -1.5
    base[7, :, 65] = 2.25
    k = torch.from_numpy(base.astype(np.float16))
    v = torch.from_numpy((base[::-1].copy()).astype(np.float16))
    pool, ref = _quantize_both(k, v, [0], 1)
    assert_pool_equal(pool, ref)
    pool, ref = _quantize_both(k, v, [0], 1, rotated=False)
    assert_pool_equal(pool, ref)


def test_q8_only_pool_and_single_token():
    k, v = W.random_small(1, 5, 256, "bf16", seed=9)
    pool, ref = _quantize_both(k, v, [2], 0, 3)
    assert_pool_equal(pool, ref)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.float16])
@pytest.mark.parametrize("unrotate", [False, True])
def test_dequantize_bit_exact(out_dtype, unrotate):
    n, hkv, d = 600, 3, 128
    k, v = W.random_small(n, hkv, d, "fp16", seed=21)
    ids = [2, 0, 4]
    pool, ref = _quantize_both(k, v, ids, 3, 2)
    slots = torch.tensor([0, 17, 255, 2 * 256 + 100, 4 * 256 + 3], dtype=torch.int64, device=cuda())
    pool.invalidate(slots)
    ref.invalidate_slots(slots.cpu().tolist())
    want = [0, 1, 2, 3, 4]
    kd, vd = pool.dequantize(torch.tensor(want, dtype=torch.int32, device=cuda()), out_dtype, unrotate)
    torch.cuda.synchronize()
    for i, blk in enumerate(want):
        rk, rv = ref.dequantize_block(blk, unrotate_k=unrotate)
        if out_dtype == torch.float16:
            rk, rv = rk.astype(np.float16), rv.astype(np.float16)
        np.testing.assert_array_equal(kd[i].cpu().numpy(), rk)
        np.testing.assert_array_equal(vd[i].cpu().numpy(), rv)


def test_invalidate_and_requantize():
    n, hkv, d = 512, 2, 128
    k, v = W.random_small(n, hkv, d, "fp16", seed=31)
    pool, ref = _quantize_both(k, v, [1, 0], 2)
    g = torch.Generator().manual_seed(0)
    slots = torch.randperm(512, generator=g)[:200]
    pool.invalidate(slots.to(cuda()))
    ref.invalidate_slots(slots.tolist())
    torch.cuda.synchronize()
    assert_pool_equal(pool, ref)
    # rewriting block 1 (chunk 0) makes its slots live again
    pool.quantize(k[:256].to(cuda()), v[:256].to(cuda()), torch.tensor([1], dtype=torch.int32, device=cuda()))
    kh, dt = host(k[:256])
    vh, _ = host(v[:256])
    ref.quantize_blocks(kh, vh, dt, [1])
    torch.cuda.synchronize()
    assert_pool_equal(pool, ref)


def test_out_of_range_ids_raise_device_error_and_skip():
    n, hkv, d = 300, 1, 128
    k, v = W.random_small(n, hkv, d, "fp16", seed=41)
    dev = cuda()
    pool = q4.Q4KVPool(hkv, d, 2, device=dev)
    before = pool.k_codes4.clone()
    pool.quantize(k.to(dev), v.to(dev), torch.tensor([7, -1], dtype=torch.int32, device=dev))
    bits = pool.read_device_error()
    assert bits & 1
    assert torch.equal(before, pool.k_codes4)
    assert pool.read_device_error() == 0           # cleared by the previous read
    pool.invalidate(torch.tensor([2 * 256, -5, 3], dtype=torch.int64, device=dev))
    assert pool.read_device_error() == 4
    assert int(pool.mask[0, 0].item()) == 8         # slot 3 was still set


def test_block_absmean_and_mixed_ids():
    w = W.LLAMA31_8B_MIXED.with_(batch=2, ctx=4096)
    k, v = W.kv_layer(w, 0)
    kd = k.to(cuda())
    am = q4.block_absmean(kd)
    kh, dt = host(k)
    ref = O.block_absmean(kh, dt)
    # fp16 sums of |x| are exact in fp64 here, so the two agree bit for bit
    np.testing.assert_array_equal(am.cpu().numpy(), ref)
    n_q8 = w.n_q8_blocks
    ids = q4.mixed_block_ids(am, n_q8, 0, w.n_blocks - n_q8)
    want = O.mixed_block_ids(ref, n_q8, 0, w.n_blocks - n_q8)
    np.testing.assert_array_equal(ids.cpu().numpy(), want)
    # ties go to the lower chunk index; a ragged last chunk averages its own tokens
    a = torch.tensor([1.0, 3.0, 3.0, 2.0, 3.0], dtype=torch.float64, device=cuda())
    assert q4.mixed_block_ids(a, 2, 0, 10).cpu().tolist() == [0, 10, 11, 1, 2]
    k2 = torch.full((300, 1, 128), -2.0, dtype=torch.bfloat16, device=cuda())
    k2[256:] = 0.5
    assert q4.block_absmean(k2).cpu().tolist() == [2.0, 0.5]


def test_large_block_ids_and_many_tokens():
    # 64 blocks, ids reversed: exercises a grid of many CTAs and long id lists
    n, hkv, d = 64 * 256, 8, 128
    k, v = W.random_small(n, hkv, d, "fp16", seed=51)
    ids = list(range(63, -1, -1))
    pool, ref = _quantize_both(k, v, ids, 64)
    assert_pool_equal(pool, ref, blocks=[0, 1, 31, 62, 63])


def test_constant_group_beside_a_clamped_group():
    # One warp item (4 tokens of one head at D = 128) whose groups take both
    # encoder paths: token 1's values are beyond the fp16 range (zero = inf,
    # the exact path), token 0 is a constant group whose value is not
    # fp16-exact (s = 0 with x - z > 0; the oracle codes it 0, and so must
    # either path).
    rng = np.random.default_rng(12)
    hkv, d = 1, 128
    base = rng.standard_normal((256, hkv, d)).astype(np.float32)
    base[0] = 1.1e-6                            # bf16 value above its fp16 rounding
    base[1] = 70000.0 + rng.standard_normal((hkv, d)) * 1000.0
    x = torch.from_numpy(base).to(torch.bfloat16)
    assert float(x[0, 0, 0]) > float(x[0, 0, 0].to(torch.float16))
    for rotated in (False, True):
        pool, ref = _quantize_both(x, x, [0], 1, rotated=rotated)
        assert_pool_equal(pool, ref)


def test_near_tie_values_take_the_exact_path():
    # V is stored unrotated, so its quotients can be placed on and next to
    # half-integers exactly: z = -1, s = 1/16 (all fp16-exact), values
    # z + (k + 1/2) s and their fp16 neighbours.
    rng = np.random.default_rng(61)
    n, hkv, d = 512, 2, 128
    base = np.full((n, hkv, d), -1.0, np.float32)
    k = rng.integers(0, 15, size=(n, hkv, d))
    vals = (-1.0 + (k + 0.5) / 16.0).astype(np.float16)
    nudge = rng.integers(-1, 2, size=vals.shape)
    bits = vals.view(np.uint16).astype(np.int32) + nudge
    vals = bits.astype(np.uint16).view(np.float16)
    base[:] = vals.astype(np.float32)
    base[:, :, 0::64] = -1.0                    # every group spans exactly [-1, -1 + 15/16]
    base[:, :, 1::64] = -1.0 + 15 / 16
    v = torch.from_numpy(base.astype(np.float16))
    kk = torch.from_numpy(rng.standard_normal((n, hkv, d)).astype(np.float16))
    for n_q8 in (0, 2):
        pool, ref = _quantize_both(kk, v, [0, 1], 2 - n_q8, n_q8)
        assert_pool_equal(pool, ref)


@pytest.mark.parametrize("scale,offset", [(1e-3, 0.0), (1.0, 0.0), (300.0, 0.0), (1.0, 900.0),
                                          (0.01, -40.0), (50.0, 3000.0)])
def test_distribution_sweep(scale, offset):
    # large offsets relative to the spread force the exact path (|z / s| > 2^10)
    n, hkv, d = 2048, 4, 128
    rng = np.random.default_rng(int(scale * 1000 + offset) % 2**31)
    x = rng.standard_normal((n, hkv, d)) * scale + offset
    k = torch.from_numpy(x.astype(np.float16))
    v = torch.from_numpy((x[::-1] * 0.5).copy().astype(np.float16))
    ids = list(range(8))
    pool, ref = _quantize_both(k, v, ids, 6, 2)
    assert_pool_equal(pool, ref)
    pool, ref = _quantize_both(k.to(torch.bfloat16), v.to(torch.bfloat16), ids, 8, 0)
    assert_pool_equal(pool, ref)
