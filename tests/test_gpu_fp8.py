"""The FP8 (OCP E4M3) comparison cache ([UQ]: the 4-bit cache is measured
against an FP8 KV cache): encoding and appending are bit-exact with the
oracle's E4M3 rounding, dequantisation is exact, and decode attention over it
is within tolerance of the oracle's fp64 attention."""
import numpy as np
import pytest
import torch

import decode_attention_q4kv_b200 as q4
from decode_attention_q4kv_b200 import _lib
from decode_attention_q4kv_b200 import workloads as W
from helpers import assert_close, cuda, host, nblocks
from oracle import q4kv_oracle as O

pytestmark = pytest.mark.gpu


def _both(k, v, ids, n_blocks):
    dev = cuda()
    pool = q4.Q4KVPool(k.shape[1], k.shape[2], 0, n_blocks, k_rotated=False, fp8=True, device=dev)
    pool.quantize(k.to(dev), v.to(dev), torch.tensor(ids, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    assert pool.read_device_error() == 0
    ref = O.OraclePool(k.shape[1], k.shape[2], 0, n_blocks, k_rotated=False, fp8=True)
    kh, dt = host(k)
    vh, _ = host(v)
    ref.quantize_blocks(kh, vh, dt, ids)
    return pool, ref


def _assert_fp8_equal(pool, ref):
    for name in "kv":
        np.testing.assert_array_equal(getattr(pool, f"{name}_codes8").cpu().numpy(), ref.codes8[name],
                                      err_msg=f"{name} E4M3 bytes")
    np.testing.assert_array_equal(pool.mask.cpu().numpy().view(np.uint32), ref.mask)


@pytest.mark.parametrize("d,dtype,hkv", [(128, "fp16", 8), (256, "bf16", 2), (128, "bf16", 3)])
def test_fp8_encode_bit_exact(d, dtype, hkv):
    n = 700
    k, v = W.random_small(n, hkv, d, dtype, seed=d + hkv)
    k = k.float()
    k[0] = 1000.0                     # saturates to 448
    k[1] = -600.0
    k[2] = 2.0 ** -12                 # below the smallest subnormal step
    k[3] = -0.0
    k[4, :, ::2] = 1.0625             # ties to even
    v = v.float() * 40.0
    tdt = torch.float16 if dtype == "fp16" else torch.bfloat16
    pool, ref = _both(k.to(tdt), v.to(tdt), list(range(nblocks(n) - 1, -1, -1)), nblocks(n))
    _assert_fp8_equal(pool, ref)
    # dequantisation is exact: E4M3 -> fp32
    kd, vd = pool.dequantize(torch.arange(nblocks(n), dtype=torch.int32, device=cuda()))
    for blk in range(nblocks(n)):
        rk, rv = ref.dequantize_block(blk)
        np.testing.assert_array_equal(kd[blk].cpu().numpy(), rk)
        np.testing.assert_array_equal(vd[blk].cpu().numpy(), rv)


def test_fp8_append_bit_exact():
    dev = cuda()
    hkv, d = 4, 128
    k, v = W.random_small(300, hkv, d, "fp16", seed=3)
    pool, ref = _both(k, v, [2, 0], 3)
    kn, vn = W.random_small(6, hkv, d, "fp16", seed=4)
    kn, vn = kn.view(2, 3, hkv, d), vn.view(2, 3, hkv, d)
    tables = np.array([[2, 0], [1, 0]], dtype=np.int32)
    lens, new = [300, 10], [3, 2]
    pool.append(kn.to(dev), vn.to(dev), torch.as_tensor(tables).to(dev),
                torch.tensor(lens, dtype=torch.int32, device=dev), torch.tensor(new, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    khn, dt = host(kn.reshape(6, hkv, d))
    vhn, _ = host(vn.reshape(6, hkv, d))
    ref.append_tokens(khn.reshape(2, 3, hkv, d), vhn.reshape(2, 3, hkv, d), dt, tables, lens, new)
    _assert_fp8_equal(pool, ref)


@pytest.mark.parametrize("hq,hkv,d,dtype,n_splits", [(32, 8, 128, "fp16", 0), (16, 8, 256, "bf16", 0),
                                                      (32, 8, 128, "fp16", 3), (8, 1, 128, "bf16", 1),
                                                      (16, 4, 256, "fp16", 2)])
def test_fp8_decode_matches_oracle(hq, hkv, d, dtype, n_splits):
    dev = cuda()
    lens = [1, 255, 700, 1300]
    B = len(lens)
    nb = max(nblocks(n) for n in lens)
    g = torch.Generator().manual_seed(hq + d)
    perm = torch.randperm(B * nb, generator=g).to(torch.int32).view(B, nb)
    k, v = W.random_small(B * nb * 256, hkv, d, dtype, seed=7 + d)
    ids = list(range(B * nb))
    pool, ref = _both(k, v, ids, B * nb)
    # remap a few slots to the sentinel
    slots = torch.tensor([int(perm[3, 0]) * 256 + 5, int(perm[2, 1]) * 256 + 100], dtype=torch.int64)
    pool.invalidate(slots.to(dev))
    ref.invalidate_slots(slots.tolist())
    q = torch.randn(B, hq, d, generator=g).to(torch.float16 if dtype == "fp16" else torch.bfloat16)
    plan = q4.DecodePlan(B, hq, hkv, d, nb, n_splits=n_splits)
    out = q4.decode_attention(pool, q.to(dev), perm.to(dev), torch.tensor(lens, dtype=torch.int32, device=dev),
                              out_dtype=torch.float32, plan=plan)
    qh, dt = host(q)
    want = O.decode_attention(ref, qh, dt, perm.numpy(), lens)
    assert_close(out, want, what="fp8 decode")
    assert pool.read_device_error() == 0


def test_fp8_pool_rejects_the_cuda_core_kernel():
    dev = cuda()
    k, v = W.random_small(256, 2, 128, "fp16", seed=1)
    pool, _ = _both(k, v, [0], 1)
    plan = q4.DecodePlan(1, 8, 2, 128, 1)
    plan.c.kernel = 0
    with pytest.raises(_lib.Q4KVError):
        q4.decode_attention(pool, torch.zeros(1, 8, 128, dtype=torch.float16, device=dev),
                            torch.zeros(1, 1, dtype=torch.int32, device=dev),
                            torch.tensor([256], dtype=torch.int32, device=dev), plan=plan)
