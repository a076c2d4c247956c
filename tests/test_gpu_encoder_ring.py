"""The encoder's stage ring at full size.

One layer of the Qwen2.5-14B eviction workload (32 sessions x 16384 tokens,
8 KV heads, D = 128, fp16 -- 524288 tokens, 1 GiB per tensor) is encoded in a
single launch, several hundred units per CTA, so every stage is reused many
times.  The FP8 consumers are faster than the copies that feed them: they
wait on nearly every unit, and a unit read before its own copy has landed
(an out-of-order phase) shows up as wrong bytes.  The whole output is checked
with torch on the device against what the formats fix element by element,
and sampled blocks bit for bit against the oracle.
"""
import numpy as np
import pytest
import torch

import decode_attention_q4kv_b200 as q4
from decode_attention_q4kv_b200 import workloads as W
from helpers import cuda, host, oracle_pool
from oracle import q4kv_oracle as O

pytestmark = pytest.mark.gpu

EVICT = W.QWEN25_14B_EVICT


def _layer():
    w = EVICT
    k, v = W.kv_tokens(w, 0, w.n_tokens, cuda())
    ids = torch.arange(w.n_tokens // 256, dtype=torch.int32, device=cuda())
    return w, k, v, ids


def _by_block(x, nb):
    """[n][H][D] tokens -> [block][H][slot][D] (the pool's order for identity block ids)."""
    return x.reshape(nb, 256, x.shape[1], x.shape[2]).permute(0, 2, 1, 3)


def _sample_blocks(nb, seed=0):
    rng = np.random.default_rng(seed)
    return sorted({0, nb - 1, *rng.choice(nb, 6, replace=False).tolist()})


def test_fp8_encoder_full_layer():
    w, k, v, ids = _layer()
    nb = ids.numel()
    pool = q4.Q4KVPool(w.n_kv_heads, w.head_dim, 0, nb, k_rotated=False, fp8=True, device=cuda())
    pool.quantize(k, v, ids)
    torch.cuda.synchronize()
    assert pool.read_device_error() == 0
    for name, x in (("k", k), ("v", v)):
        codes = getattr(pool, f"{name}_codes8")
        xf = _by_block(x, nb).float()
        d = codes.view(torch.float8_e4m3fn).float()   # E4M3 -> fp32 is exact
        # round to nearest on the E4M3 grid: spacing 2^(e-3), e = max(floor(log2|x|), -6);
        # these inputs stay far below the saturation point 448
        assert xf.abs().max().item() < 448.0
        _, ex = torch.frexp(xf)
        quantum = torch.ldexp(torch.ones_like(xf), torch.clamp(ex - 1, min=-6) - 3)
        err = (xf - d).abs()
        bad = (err > 0.5 * quantum) | (torch.signbit(xf) != torch.signbit(d)) & (d != 0)
        assert int(bad.sum().item()) == 0, f"{name}: {int(bad.sum().item())} bytes off the nearest E4M3 value"
        del xf, d, ex, quantum, err, bad
    # sampled blocks: the oracle's encoding, bit for bit
    kh, _ = host(k)
    vh, _ = host(v)
    for blk in _sample_blocks(nb):
        rows = slice(blk * 256, (blk + 1) * 256)
        for name, xh in (("k", kh), ("v", vh)):
            want = O.e4m3_encode(xh[rows].transpose(1, 0, 2))
            got = getattr(pool, f"{name}_codes8")[blk].cpu().numpy()
            np.testing.assert_array_equal(got, want, err_msg=f"{name} block {blk}")
    # every slot was written live
    assert int(pool.mask.abs().sum().item()) == 0


def test_q4_encoder_full_layer_values():
    """Values are coded unrotated: given each group's stored fp16 scale and
    zero, every code is fixed (round half to even of (x - z) / s, clamped to
    [0, 15]) and the scale and zero are fixed by the group's min and max."""
    w, k, v, ids = _layer()
    nb = ids.numel()
    pool = q4.Q4KVPool(w.n_kv_heads, w.head_dim, nb, 0, k_rotated=True, device=cuda())
    pool.quantize(k, v, ids)
    torch.cuda.synchronize()
    assert pool.read_device_error() == 0
    xf = _by_block(v, nb).float()                                   # [nb][H][256][D]
    g = xf.reshape(*xf.shape[:3], w.head_dim // 64, 64)
    mn, mx = g.amin(-1), g.amax(-1)
    s_want = ((mx - mn) / 15.0).half()
    z_want = mn.half()
    par = pool.v_params4                                            # [nb][H][256][ng][2]
    assert torch.equal(par[..., 0], s_want), "value scales"
    assert torch.equal(par[..., 1], z_want), "value zeros"
    sf = par[..., 0].float().unsqueeze(-1)
    zf = par[..., 1].float().unsqueeze(-1)
    q = torch.where(sf == 0, torch.zeros_like(g), torch.clamp(torch.round((g - zf) / sf), 0, 15))
    b = pool.v_codes4                                               # [nb][H][256][D/2]
    codes = torch.stack((b & 15, b >> 4), dim=-1).reshape(xf.shape).float()
    bad = int((codes != q.reshape(xf.shape)).sum().item())
    assert bad == 0, f"{bad} value codes differ from the group rule"
    del xf, g, q, codes
    # sampled blocks of both tensors against the oracle
    for blk in _sample_blocks(nb, seed=1):
        rows = slice(blk * 256, (blk + 1) * 256)
        ref = oracle_pool(k[rows], v[rows], [0], 1)
        for name in "kv":
            np.testing.assert_array_equal(getattr(pool, f"{name}_codes4")[blk].cpu().numpy(),
                                          ref.codes4[name][0], err_msg=f"{name} codes, block {blk}")
            np.testing.assert_array_equal(getattr(pool, f"{name}_params4")[blk].cpu().numpy().view(np.uint16),
                                          ref.params4[name][0].view(np.uint16),
                                          err_msg=f"{name} scale/zero bits, block {blk}")
