"""Every wait in the kernels is bounded: a barrier that nothing completes makes
the wait give up, report Q4KV_DEVERR_TIMEOUT and return, and the context stays
usable (a decode right after it still matches the oracle)."""
import time

import pytest
import torch

import decode_attention_q4kv_b200 as q4
from decode_attention_q4kv_b200 import _lib
from decode_attention_q4kv_b200 import workloads as W
from helpers import assert_close, cuda, host, oracle_pool
from oracle import q4kv_oracle as O

pytestmark = pytest.mark.gpu


def test_wait_that_nothing_completes_gives_up_and_reports():
    dev = cuda()
    word = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    t0 = time.monotonic()
    _lib.check(_lib.lib().q4kv_selftest_bounded_wait(word.data_ptr(), 2000, stream), "selftest")
    torch.cuda.synchronize()
    assert time.monotonic() - t0 < 30.0
    assert int(word.item()) & _lib.DEVERR_TIMEOUT
    # the context is still usable: a small decode matches the oracle
    k, v = W.random_small(300, 2, 128, "fp16", seed=1)
    pool = q4.Q4KVPool(2, 128, 2, device=dev)
    pool.quantize(k.to(dev), v.to(dev), torch.tensor([1, 0], dtype=torch.int32, device=dev))
    q = torch.randn(1, 4, 128, generator=torch.Generator().manual_seed(2)).to(torch.float16)
    tables = torch.tensor([[1, 0]], dtype=torch.int32)
    out = q4.decode_attention(pool, q.to(dev), tables.to(dev), torch.tensor([300], dtype=torch.int32, device=dev),
                              out_dtype=torch.float32)
    qh, dt = host(q)
    want = O.decode_attention(oracle_pool(k, v, [1, 0], 2), qh, dt, tables.numpy(), [300])
    assert_close(out, want, what="decode after a timed-out wait")
    assert pool.read_device_error() == 0
