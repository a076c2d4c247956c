"""Per-token widths {2, 4, 8, FP16} in one cache: the card (QKVShare,
"Méthodologie").  Cards the kernels write are byte-identical to the oracle's;
decoding gives the oracle's rebuilt keys and values bit for bit; invalid
widths and damaged cards are reported without reading out of bounds; the
Llama-3.1-8B-shaped layer (327680 tokens) round-trips at full size."""
import numpy as np
import pytest
import torch

import decode_attention_q4kv_b200 as q4
from decode_attention_q4kv_b200 import _lib
from decode_attention_q4kv_b200 import workloads as W
from helpers import cuda, host
from oracle import q4kv_oracle as O

pytestmark = pytest.mark.gpu


def _err():
    return torch.zeros(4, dtype=torch.int32, device=cuda())


def _dirty(n_bytes):
    """Leave non-zero bytes in the allocator's free blocks, so that a card
    byte the kernels forget to write shows up."""
    junk = torch.full((n_bytes,), 0xA5, dtype=torch.uint8, device=cuda())
    del junk


@pytest.mark.parametrize("k_rotated", [True, False])
@pytest.mark.parametrize("d,dtype,hkv,n", [(128, "fp16", 3, 301), (256, "bf16", 2, 97), (128, "bf16", 8, 8195),
                                          (128, "fp16", 1, 4096)])
def test_card_bytes_equal_the_oracle(d, dtype, hkv, n, k_rotated):
    k, v = W.random_small(n, hkv, d, dtype, seed=d + n, scale=2.0)
    widths = W.token_widths(n, seed=n)
    if n > 8:
        widths[5] = 16
        widths[6] = 2
    err = _err()
    _dirty(q4.card_max_bytes(d, hkv, n) + (1 << 20))
    card = q4.card_encode(k.to(cuda()), v.to(cuda()), widths.to(cuda()), k_rotated=k_rotated, error_word=err)
    torch.cuda.synchronize()
    assert int(err[0]) == 0
    kh, dt = host(k)
    vh, _ = host(v)
    ref = O.card_encode(kh, vh, dt, widths.numpy(), k_rotated=k_rotated)
    got = card.cpu().numpy()
    np.testing.assert_array_equal(got[:ref.size], ref)
    # a caller's buffer is reused and gets the same bytes
    again = torch.full_like(card, 0x5A)
    assert q4.card_encode(k.to(cuda()), v.to(cuda()), widths.to(cuda()), k_rotated=k_rotated, out=again) is again
    np.testing.assert_array_equal(again.cpu().numpy()[:ref.size], ref)
    # decode: the oracle's rebuilt rows exactly (fp32) and their fp16 rounding
    k_hat, v_hat = O.card_decode(ref)
    kd, vd = q4.card_decode(card, n, hkv, d, error_word=err)
    kd16, vd16 = q4.card_decode(card, n, hkv, d, out_dtype=torch.float16, error_word=err)
    torch.cuda.synchronize()
    assert int(err[0]) == 0
    np.testing.assert_array_equal(kd.cpu().numpy(), k_hat)
    np.testing.assert_array_equal(vd.cpu().numpy(), v_hat)
    np.testing.assert_array_equal(kd16.cpu().numpy(), k_hat.astype(np.float16))
    np.testing.assert_array_equal(vd16.cpu().numpy(), v_hat.astype(np.float16))


def test_invalid_widths_take_no_bytes_and_are_reported():
    n, hkv, d = 40, 2, 128
    k, v = W.random_small(n, hkv, d, "fp16", seed=3)
    widths = torch.tensor([(2, 4, 8, 16, 0, 3, 255)[t % 7] for t in range(n)], dtype=torch.uint8)
    err = _err()
    card = q4.card_encode(k.to(cuda()), v.to(cuda()), widths.to(cuda()), error_word=err)
    torch.cuda.synchronize()
    assert int(err[0]) == _lib.DEVERR_WIDTH
    kh, dt = host(k)
    vh, _ = host(v)
    ref = O.card_encode(kh, vh, dt, widths.numpy())
    np.testing.assert_array_equal(card.cpu().numpy()[:ref.size], ref)
    err.zero_()
    kd, vd = q4.card_decode(card, n, hkv, d, error_word=err)
    torch.cuda.synchronize()
    assert int(err[0]) == 0
    k_hat, v_hat = O.card_decode(ref)
    np.testing.assert_array_equal(kd.cpu().numpy(), k_hat)
    np.testing.assert_array_equal(vd.cpu().numpy(), v_hat)


def test_damaged_cards_read_zero_and_report():
    n, hkv, d = 64, 2, 128
    k, v = W.random_small(n, hkv, d, "fp16", seed=5)
    widths = W.token_widths(n, seed=5).to(cuda())
    card = q4.card_encode(k.to(cuda()), v.to(cuda()), widths)
    torch.cuda.synchronize()
    offs_at = 64 + 64                                     # header, 64 width bytes
    bad = card.clone()
    bad[offs_at + 8 * 10:offs_at + 8 * 11] = torch.tensor(list((1 << 40).to_bytes(8, "little")),
                                                           dtype=torch.uint8, device=cuda())
    err = _err()
    kd, vd = q4.card_decode(bad, n, hkv, d, error_word=err)
    torch.cuda.synchronize()
    assert int(err[0]) == _lib.DEVERR_IMAGE
    assert not kd[10].any() and not vd[10].any()
    k_ok, v_ok = q4.card_decode(card, n, hkv, d)
    assert torch.equal(kd[11:], k_ok[11:]) and torch.equal(vd[:10], v_ok[:10])
    err.zero_()
    kd, vd = q4.card_decode(card, n - 1, hkv, d, error_word=err)    # the header says n tokens
    torch.cuda.synchronize()
    assert int(err[0]) == _lib.DEVERR_IMAGE and not kd.any() and not vd.any()


def test_full_layer_card_round_trip():
    """The Llama-3.1-8B-shaped layer (10 x 32768 tokens, 8 KV heads, D 128):
    the offset table in full, sampled records against the oracle, every FP16
    token exact and every decoded row within its width's error bound."""
    w = W.LLAMA31_8B_MIXED
    n = w.n_tokens
    k, v = W.kv_tokens(w, 0, n, cuda())
    widths = W.token_widths(n, seed=w.seed)
    card = q4.card_encode(k, v, widths.to(cuda()))
    kd, vd = q4.card_decode(card, n, w.n_kv_heads, w.head_dim)
    torch.cuda.synchronize()
    offs, _, o_at, p_at, total = O.card_layout(w.head_dim, w.n_kv_heads, widths.numpy())
    got_offs = card[o_at:o_at + 8 * (n + 1)].cpu().numpy().view("<i8")
    np.testing.assert_array_equal(got_offs, offs)
    assert O.card_header(card[:64].cpu().numpy())["payload_bytes"] == offs[-1]
    fp16 = widths == 16
    assert torch.equal(kd[fp16.to(cuda())], k[fp16.to(cuda())].float())
    assert torch.equal(vd[fp16.to(cuda())], v[fp16.to(cuda())].float())
    # values: within half a step of their group (plus the fp16 rounding of s and z)
    for wd in (2, 4, 8):
        sel = (widths == wd).to(cuda())
        x = v[sel].float().reshape(-1, w.n_kv_heads, w.head_dim // 64, 64)
        xh = vd[sel].reshape(x.shape)
        L = (1 << wd) - 1
        s = (x.amax(-1) - x.amin(-1)) / L
        bound = 0.5 * s + L * s * 2.0 ** -10 + x.amin(-1).abs() * 2.0 ** -10 + 1e-6
        assert bool(((xh - x).abs().amax(-1) <= bound).all()), wd
    # sampled tokens: the oracle's record bytes
    _, dt = host(k[:1])
    rng = np.random.default_rng(7)
    for t in sorted({0, n - 1, *rng.choice(n, 14, replace=False).tolist()}):
        kt, _ = host(k[t:t + 1])
        vt, _ = host(v[t:t + 1])
        ref = O.card_encode(kt, vt, dt, widths[t:t + 1].numpy())
        r_offs, _, _, r_p, _ = O.card_layout(w.head_dim, w.n_kv_heads, widths[t:t + 1].numpy())
        a = p_at + int(offs[t])
        np.testing.assert_array_equal(card[a:a + int(r_offs[1])].cpu().numpy(), ref[r_p:r_p + int(r_offs[1])],
                                      err_msg=f"token {t}")
