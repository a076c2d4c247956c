"""The allocation-free decode entry point, called through the C ABI.

Some callers cannot allocate device memory themselves (their device memory
belongs to another allocator, or their budget is fixed before they run), so
q4kv_decode_attention_static_scratch keeps the split partials in a
file-scope device array instead of a caller-provided workspace.  These tests
compare it with q4kv_decode_attention on the same inputs, twice in a row
(the array is shared and keeps the previous call's contents), and check that
a plan needing more scratch than the array holds is refused.  The file is
named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import decode_attention_q4kv_b200 as q4
from decode_attention_q4kv_b200 import _lib
from decode_attention_q4kv_b200 import workloads as W
from helpers import ATOL, RTOL_L2, assert_close, cuda, host, seq_tables
from oracle import q4kv_oracle as O

pytestmark = pytest.mark.gpu


def _setup(lens, hq, hkv, d, dtype, seed):
    dev = cuda()
    mb = max(1, max(-(-n // 256) for n in lens))
    n_pool = len(lens) * mb + 2
    pool = q4.Q4KVPool(hkv, d, n_pool, device=dev)
    ref = O.OraclePool(hkv, d, n_pool)
    tables = seq_tables(len(lens), mb, n_pool, seed)
    for b, n in enumerate(lens):
        k, v = W.random_small(n, hkv, d, dtype, seed=100 * seed + b)
        ids = tables[b, : -(-n // 256)]
        pool.quantize(k.to(dev), v.to(dev), ids.to(dev))
        kh, dt = host(k)
        vh, _ = host(v)
        ref.quantize_blocks(kh, vh, dt, [int(i) for i in ids])
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((len(lens), hq, d), generator=g).to(W.torch_dtype(dtype))
    qh, dt = host(q)
    want = O.decode_attention(ref, qh, dt, tables.numpy(), lens)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=dev)
    return pool, q.to(dev), tables.to(dev), lens_t, mb, want


def _static_call(pool, plan, q, tables, lens, out):
    lib = _lib.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.q4kv_decode_attention_static_scratch(
        ctypes.byref(pool.desc), ctypes.byref(plan.c), ctypes.c_void_p(q.data_ptr()),
        q4._IN_DTYPES[q.dtype], ctypes.c_void_p(tables.data_ptr()), ctypes.c_void_p(lens.data_ptr()),
        ctypes.c_float(0.0), ctypes.c_void_p(out.data_ptr()), q4._OUT_DTYPES[out.dtype], stream)


def test_static_scratch_matches_workspace_entry_point_twice():
    # The first case's plan needs more scratch than the second's, so the
    # second call runs over partials the first one left in the shared array:
    # any stale partial that leaked into a result would change its bits.
    cases = [([1500, 700, 33], 32, 8, 128, "fp16", 1, 9),
             ([4096, 300], 16, 8, 256, "bf16", 2, 5)]
    used = []
    for lens, hq, hkv, d, dtype, seed, splits in cases:
        pool, q, tables, lens_t, mb, expect = _setup(lens, hq, hkv, d, dtype, seed)
        plan = q4.DecodePlan(len(lens), hq, hkv, d, mb, n_splits=splits)
        assert 0 < plan.workspace_bytes <= 16 << 20
        used.append(plan.workspace_bytes)
        want = q4.decode_attention(pool, q, tables, lens_t, out_dtype=torch.float32, plan=plan)
        for _ in range(2):                            # two calls in a row on the same inputs
            got = torch.full_like(want, float("nan"))
            st = _static_call(pool, plan, q, tables, lens_t, got)
            assert st == _lib.OK, _lib.lib().q4kv_status_string(st)
            torch.cuda.synchronize()
            # same kernels, same plan: the results agree bit for bit
            assert torch.equal(got, want), float((got - want).abs().max())
        assert pool.read_device_error() == 0
        # and both are within the oracle's tolerance
        assert_close(got, expect, atol=ATOL, rtol_l2=RTOL_L2, what="static scratch")
    assert used[0] > used[1]


def test_static_scratch_rejects_oversized_plan():
    # 256 sequences x 40 heads x 64 splits x 130 floats: far beyond the 16 MiB array
    plan = q4.DecodePlan(256, 40, 8, 128, 64, n_splits=64, num_sms=148)
    assert plan.workspace_bytes > 16 << 20
    pool = q4.Q4KVPool(8, 128, 1, device=cuda())
    x = torch.zeros(16, dtype=torch.float16, device=cuda())
    st = _static_call(pool, plan, x, x.int(), x.int(), x)
    assert st == _lib.ERR_WORKSPACE
