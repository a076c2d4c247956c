"""Pins for the CPU oracle against facts outside the oracle itself.

Each test checks the oracle against something the pages print (fixtures in
tests/golden), a closed form, a textbook identity, a library routine that
computes the same mathematics by another route, or brute force on tiny
inputs.  A dropped term, a wrong sign or index, a transposed operand or a
wrong rounding rule in the oracle fails at least one of them.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import scipy.special

from conftest import read_golden
from oracle import q4kv_oracle as O


def _hexf(s):
    return np.float32(float.fromhex(s))


# ---------------------------------------------------------------------------
# Walsh-Hadamard rotation
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64, 128, 256])
def test_fwht_is_sylvester_matrix(n):
    # transform of each basis vector gives one column of H (exact integers)
    H = O.fwht(np.eye(n), np.float64).T
    i = np.arange(n)
    popc = np.vectorize(lambda a: bin(a).count("1"))(i[:, None] & i[None, :])
    assert np.array_equal(H, (-1.0) ** popc)
    Hi = H.astype(np.int64)
    assert np.array_equal(Hi @ Hi.T, n * np.eye(n, dtype=np.int64))
    # textbook Sylvester construction (library routine)
    assert np.array_equal(Hi, scipy.linalg.hadamard(n))


def test_fwht_h2():
    assert np.array_equal(O.fwht(np.array([3.0, 5.0]), np.float64), [8.0, -2.0])


@pytest.mark.parametrize("n", [128, 256])
def test_fwht_matches_matrix_product(n):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, n))
    Hs = scipy.linalg.hadamard(n).astype(np.float64)
    assert np.allclose(O.fwht(x, np.float64), x @ Hs.T, rtol=0, atol=1e-11)
    # integer inputs are exact in binary32 as well
    xi = rng.integers(-1000, 1000, size=(5, n)).astype(np.float32)
    exact = xi.astype(np.int64) @ scipy.linalg.hadamard(n).T
    assert np.array_equal(O.fwht(xi, np.float32).astype(np.int64), exact)


@pytest.mark.parametrize("n", [64, 128, 256, 512])
def test_rotation_constant_is_nearest_binary32(n):
    c = O.rotation_constant(n)
    lo = np.nextafter(c, np.float32(0))
    hi = np.nextafter(c, np.float32(1))
    C, L, Hh = Fraction(float(c)), Fraction(float(lo)), Fraction(float(hi))
    target_sq = Fraction(1, n)                       # (1/sqrt n)^2
    assert ((L + C) / 2) ** 2 < target_sq < ((C + Hh) / 2) ** 2
    if n == 256:
        assert c == np.float32(0.0625)
    if n == 128:
        assert float(c) == float.fromhex("0x1.6a09e6p-4")


@pytest.mark.parametrize("n", [128, 256])
def test_rotation_special_vectors(n):
    c = O.rotation_constant(n)
    e0 = np.zeros(n, np.float32)
    e0[0] = 1
    assert np.array_equal(O.rotate_f32(e0), np.full(n, c, np.float32))
    ones = np.ones(n, np.float32)
    want = np.zeros(n, np.float32)
    want[0] = np.float32(n) * c
    assert np.array_equal(O.rotate_f32(ones), want)


def test_rotation_preserves_norm():
    rng = np.random.default_rng(2)
    for n in (128, 256):
        x = rng.standard_normal((64, n)).astype(np.float32)
        y = O.rotate_f32(x)
        r = np.linalg.norm(y.astype(np.float64), axis=1) / np.linalg.norm(x.astype(np.float64), axis=1)
        assert np.all(np.abs(r - 1) < 8 * math.log2(n) * 2.0 ** -24)


def test_stage_order_worked_example():
    g = read_golden("fwht_stage_order.txt")
    x = np.array([_hexf(s) for s in g["input_hex"].split()], np.float32)
    out = O.fwht(x, np.float32)
    assert out[0] == _hexf(g["ascending_out0_hex"])
    assert out[0] != _hexf(g["descending_out0_hex"])


def test_rotation_is_self_inverse():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((16, 128))
    assert np.allclose(O.rotate_f64(O.rotate_f64(x)), x, atol=1e-12)


# ---------------------------------------------------------------------------
# group quantiser and packing
# ---------------------------------------------------------------------------

def test_ramp_gives_exact_codes():
    g = read_golden("quantizer_cases.txt")
    z, s = float(g["ramp_z"]), float(g["ramp_s"])
    j = np.arange(64)
    x = (z + (j % 16) * s).astype(np.float32)[None, :]
    codes, s_h, z_h = O.quantize_groups(x, 4)
    assert s_h[0, 0] == np.float16(s) and z_h[0, 0] == np.float16(z)
    assert np.array_equal(codes[0], j % 16)
    assert np.array_equal(O.dequantize_groups(codes, s_h, z_h), x)


def test_ties_round_to_even():
    g = read_golden("quantizer_cases.txt")
    want = [int(v) for v in g["ties_expected"].split(",")]
    z, s = -1.5, 0.25
    vals = [z, z + 15 * s] + [z + (k + 0.5) * s for k in range(15)]
    x = np.array(vals + [z] * (64 - len(vals)), np.float32)[None, :]
    codes, s_h, z_h = O.quantize_groups(x, 4)
    assert s_h[0, 0] == np.float16(0.25) and z_h[0, 0] == np.float16(-1.5)
    assert codes[0, 0] == 0 and codes[0, 1] == 15
    assert list(codes[0, 2:17]) == want


def test_constant_group():
    g = read_golden("quantizer_cases.txt")
    v = float(g["constant_value"])
    x = np.full((1, 128), v, np.float32)
    codes, s_h, z_h = O.quantize_groups(x, 4)
    assert np.all(codes == 0) and np.all(s_h == 0)
    assert np.all(z_h.view(np.uint16) == int(g["constant_zero_fp16_bits"], 16))
    assert np.all(O.dequantize_groups(codes, s_h, z_h) == np.float32(np.float16(v)))


def test_signed_zero_never_reaches_params():
    for x in (np.full((1, 64), -0.0, np.float32), np.zeros((1, 64), np.float32)):
        x[0, 1::2] = -0.0
        codes, s_h, z_h = O.quantize_groups(x, 4)
        assert s_h.view(np.uint16)[0, 0] == 0 and z_h.view(np.uint16)[0, 0] == 0
        assert np.all(codes == 0)


def test_fp16_rounding_of_scale_is_ties_to_even():
    assert np.float16(np.float32(1 + 2.0 ** -11)) == np.float16(1.0)
    assert np.float16(np.float32(1 + 3 * 2.0 ** -11)) == np.float16(1 + 2.0 ** -9)


def test_scale_and_zero_definition():
    # mx - mn = 1.0 -> s = fl(1/15) -> fp16; zero = fp16(mn)
    x = np.linspace(0.3, 1.3, 64).astype(np.float32)
    x[0], x[-1] = np.float32(0.3), np.float32(1.3)
    codes, s_h, z_h = O.quantize_groups(x[None, :], 4)
    s32 = (np.float32(1.3) - np.float32(0.3)) / np.float32(15)
    assert s_h[0, 0] == np.float16(s32)
    assert z_h[0, 0] == np.float16(np.float32(0.3))
    # 8-bit uses 255 levels
    c8, s8, z8 = O.quantize_groups(x[None, :], 8)
    assert s8[0, 0] == np.float16((np.float32(1.3) - np.float32(0.3)) / np.float32(255))
    assert c8.max() == 255 and c8.min() == 0


def _roundtrip_bound(x, codes, s_h, z_h, bits):
    L = O.levels(bits)
    d = x.shape[-1]
    xs = x.reshape(x.shape[:-1] + (d // 64, 64)).astype(np.float64)
    sf = s_h.astype(np.float64)[..., None]
    zf = z_h.astype(np.float64)[..., None]
    xh = O.dequantize_groups(codes, s_h, z_h).reshape(xs.shape).astype(np.float64)
    err = np.abs(xs - xh)
    inner = np.maximum(0.5 * sf, np.maximum(zf - xs, xs - zf - L * sf))
    slack = 2.0 ** -18 * sf + np.spacing(np.abs(xh).astype(np.float32)).astype(np.float64)
    return err, inner + slack


@pytest.mark.parametrize("bits", [4, 8])
def test_roundtrip_error_bound_random(bits):
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((300, 128)) * rng.choice([0.01, 1, 30], size=(300, 1))).astype(np.float32)
    codes, s_h, z_h = O.quantize_groups(x, bits)
    err, bound = _roundtrip_bound(x, codes, s_h, z_h, bits)
    assert np.all(err <= bound)


def test_roundtrip_half_scale_when_params_exact():
    # values on an fp16-friendly grid: mn and s exact in fp16 -> |x - x_hat| <= s/2
    rng = np.random.default_rng(5)
    z = np.float32(-2.0)
    s = np.float32(0.25)
    inner = rng.uniform(0, 15, size=(200, 62)).astype(np.float32) * s + z
    x = np.concatenate([np.full((200, 1), z), np.full((200, 1), z + 15 * s), inner], axis=1)
    codes, s_h, z_h = O.quantize_groups(x.astype(np.float32), 4)
    assert np.all(s_h == np.float16(s)) and np.all(z_h == np.float16(z))
    xh = O.dequantize_groups(codes, s_h, z_h)
    assert np.all(np.abs(x - xh) <= s / 2)


def test_pack_order():
    g = read_golden("quantizer_cases.txt")
    assert O.pack_nibbles(np.array([1, 2], np.uint8))[0] == 0x21
    word = O.pack_nibbles(np.arange(8, dtype=np.uint8)).view("<u4")[0]
    assert word == int(g["packed_word_0to7"], 16)
    rng = np.random.default_rng(6)
    c = rng.integers(0, 16, size=(7, 128)).astype(np.uint8)
    assert np.array_equal(O.unpack_nibbles(O.pack_nibbles(c)), c)


def test_memory_saving_matches_page_figure():
    g = read_golden("page_figures.txt")
    fp16 = 2 * 128 * 2
    q4 = O.bytes_per_token_head(128, 4)
    assert q4 == 144
    saving = 100.0 * (1 - q4 / fp16)
    assert saving == 71.875
    assert abs(saving - float(g["q4_memory_saving_percent_approx"])) < 0.5
    assert int(g["q4_scale_bits"]) == 16 and int(g["q4_bias_bits"]) == 16
    assert O.BLOCK_TOKENS == int(g["block_tokens"])
    assert O.SENTINEL_LOGIT == float(g["sentinel_key"])
    assert 4 in [int(b) for b in g["mixed_bit_widths"].split(",")]
    assert 8 in [int(b) for b in g["mixed_bit_widths"].split(",")]


# ---------------------------------------------------------------------------
# pool and attention
# ---------------------------------------------------------------------------

def _pool_with(k, v, dtype="fp16", n_q4=None, n_q8=0, ids=None, rotated=True):
    n, hkv, d = k.shape
    nb = -(-n // 256)
    if n_q4 is None:
        n_q4 = nb
    pool = O.OraclePool(hkv, d, n_q4, n_q8, k_rotated=rotated)
    pool.quantize_blocks(k, v, dtype, list(range(nb)) if ids is None else ids)
    return pool


def _rand_kv(n, hkv, d, seed):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((n, hkv, d)).astype(np.float16)
    v = rng.standard_normal((n, hkv, d)).astype(np.float16)
    return k, v


def test_attention_matches_explicit_brute_force():
    """Independent route: explicit Hadamard matrix, scipy softmax, fp64."""
    d, hkv, hq, n = 128, 2, 8, 300
    k, v = _rand_kv(n, hkv, d, 7)
    pool = _pool_with(k, v)
    rng = np.random.default_rng(8)
    q = rng.standard_normal((1, hq, d)).astype(np.float16)
    tables = np.array([[0, 1]], np.int32)
    out = O.decode_attention(pool, q, "fp16", tables, [n])
    H = scipy.linalg.hadamard(d).astype(np.float64) / math.sqrt(d)
    kh = np.concatenate([pool.dequantize_block(b)[0] for b in (0, 1)], axis=1)[:, :n].astype(np.float64)
    vh = np.concatenate([pool.dequantize_block(b)[1] for b in (0, 1)], axis=1)[:, :n].astype(np.float64)
    for h in range(hq):
        kv = h // (hq // hkv)
        logits = (kh[kv] @ (H @ q[0, h].astype(np.float64))) / math.sqrt(d)
        want = scipy.special.softmax(logits) @ vh[kv]
        assert np.allclose(out[0, h], want, rtol=0, atol=1e-12)


def test_attention_rotation_consistency():
    """<Hq, Hk> = <q, k>: attending in the unrotated domain gives the same result."""
    d, n = 128, 256
    k, v = _rand_kv(n, 1, d, 9)
    pool = _pool_with(k, v)
    q = np.random.default_rng(10).standard_normal((1, 2, d)).astype(np.float16)
    out = O.decode_attention(pool, q, "fp16", np.array([[0]]), [n])
    k_un = pool.dequantize_block(0, unrotate_k=True)[0][0].astype(np.float64)
    vh = pool.dequantize_block(0)[1][0].astype(np.float64)
    for h in range(2):
        s = (k_un @ q[0, h].astype(np.float64)) / math.sqrt(d)
        want = scipy.special.softmax(s) @ vh
        assert np.allclose(out[0, h], want, atol=2e-5)


def test_single_live_slot_returns_its_value():
    d, n = 128, 200
    k, v = _rand_kv(n, 1, d, 11)
    pool = _pool_with(k, v)
    pool.invalidate_slots([t for t in range(n) if t != 57])
    q = np.random.default_rng(12).standard_normal((1, 4, d)).astype(np.float16)
    out = O.decode_attention(pool, q, "fp16", np.array([[0]]), [n])
    codes, s_h, z_h = pool.codes_params(0, "v")
    want = O.dequantize_groups(codes[0, 57], s_h[0, 57], z_h[0, 57]).astype(np.float64)
    for h in range(4):
        assert np.array_equal(out[0, h], want)


def test_sentinel_weight_is_exactly_zero():
    # exp(-1e4 - m) underflows to +0 in fp64 once m > -1e4 + 745
    assert np.exp(np.float64(O.SENTINEL_LOGIT) - (-9000.0)) == 0.0
    assert np.exp(np.float32(O.SENTINEL_LOGIT) - np.float32(-9000.0)) == 0.0
    d, n = 128, 512
    k, v = _rand_kv(n, 1, d, 13)
    pool = _pool_with(k, v)
    masked = list(range(0, n, 3))
    pool.invalidate_slots(masked)
    q = np.random.default_rng(14).standard_normal((1, 4, d)).astype(np.float16)
    out = O.decode_attention(pool, q, "fp16", np.array([[0, 1]]), [n])
    # same tokens with the masked ones removed: a fresh pool holding only live rows
    live = [t for t in range(n) if t not in set(masked)]
    pool2 = _pool_with(k[live], v[live])
    # the live rows quantise identically (per-vector groups), so values agree
    out2 = O.decode_attention(pool2, q, "fp16", np.array([[0, 1]]), [len(live)])
    assert np.allclose(out, out2, rtol=0, atol=1e-13)


def test_dequantize_applies_sentinel():
    d, n = 128, 256
    k, v = _rand_kv(n, 2, d, 25)
    pool = _pool_with(k, v)
    pool.invalidate_slots([0, 77, 255])
    for unrot in (False, True):
        kh, vh = pool.dequantize_block(0, unrotate_k=unrot)
        for t in (0, 77, 255):
            assert np.all(kh[:, t] == np.float32(-1e4)) and np.all(vh[:, t] == 0)
        assert np.all(vh[:, 1] != 0) or np.any(vh[:, 1] != 0)
    # live rows: K dequantises to code*s + z in the rotated domain; unrotating
    # brings it back within the quantiser's error of the raw key
    kh, _ = pool.dequantize_block(0, unrotate_k=True)
    assert np.abs(kh[:, 5] - k[5].astype(np.float32)).max() < 0.6


def test_all_masked_and_empty_give_zero():
    d, n = 128, 100
    k, v = _rand_kv(n, 1, d, 15)
    pool = _pool_with(k, v)
    q = np.random.default_rng(16).standard_normal((2, 2, d)).astype(np.float16)
    pool.invalidate_slots(range(n))
    out = O.decode_attention(pool, q, "fp16", np.array([[0], [0]]), [n, 0])
    assert np.all(out == 0)


def test_zero_query_averages_live_values():
    d, n = 128, 300
    k, v = _rand_kv(n, 1, d, 17)
    pool = _pool_with(k, v)
    q = np.zeros((1, 1, d), np.float16)
    out = O.decode_attention(pool, q, "fp16", np.array([[0, 1]]), [n])
    vh = np.concatenate([pool.dequantize_block(b)[1][0] for b in (0, 1)])[:n].astype(np.float64)
    assert np.allclose(out[0, 0], vh.mean(axis=0), atol=1e-13)


def test_gqa_head_mapping():
    # KV head j holds the constant value j + 1 in V; query head h must read j = h // g
    d, hkv, g, n = 128, 4, 3, 64
    rng = np.random.default_rng(18)
    k = rng.standard_normal((n, hkv, d)).astype(np.float16)
    v = np.broadcast_to(np.arange(1, hkv + 1, dtype=np.float16)[None, :, None], (n, hkv, d)).copy()
    pool = _pool_with(k, v)
    q = rng.standard_normal((1, hkv * g, d)).astype(np.float16)
    out = O.decode_attention(pool, q, "fp16", np.array([[0]]), [n])
    for h in range(hkv * g):
        assert np.allclose(out[0, h], h // g + 1, atol=1e-12)


def test_block_table_indirection_and_permutation():
    d, n = 128, 700
    k, v = _rand_kv(n, 2, d, 19)
    perm = [5, 2, 7]
    pool = O.OraclePool(2, d, 8, 0)
    pool.quantize_blocks(k, v, "fp16", perm)
    ref = _pool_with(k, v)
    q = np.random.default_rng(20).standard_normal((1, 4, d)).astype(np.float16)
    a = O.decode_attention(pool, q, "fp16", np.array([perm]), [n])
    b = O.decode_attention(ref, q, "fp16", np.array([[0, 1, 2]]), [n])
    assert np.array_equal(a, b)
    # a token's value is read from its own slot: the only live token at
    # position 300 (block 1 of the table, slot 44) is returned verbatim
    pool.invalidate_slots([blk * 256 + s for blk in perm for s in range(256)])
    pool.mask[perm[1], 44 // 32] &= np.uint32(~(1 << (44 % 32)) & 0xFFFFFFFF)
    c = O.decode_attention(pool, q, "fp16", np.array([perm]), [n])
    codes, s_h, z_h = pool.codes_params(perm[1], "v")
    want = O.dequantize_groups(codes[0, 44], s_h[0, 44], z_h[0, 44])
    assert np.array_equal(c[0, 0], want.astype(np.float64))


def test_softmax_scale_argument():
    d, n = 128, 64
    k, v = _rand_kv(n, 1, d, 21)
    pool = _pool_with(k, v)
    q = np.random.default_rng(22).standard_normal((1, 1, d)).astype(np.float16)
    a = O.decode_attention(pool, q, "fp16", np.array([[0]]), [n], softmax_scale=0.25)
    # doubling q (exact in fp16) and halving the scale leaves every logit unchanged
    q2 = (q.astype(np.float32) * 2).astype(np.float16)
    b = O.decode_attention(pool, q2, "fp16", np.array([[0]]), [n], softmax_scale=0.125)
    assert np.array_equal(a, b)
    # a non-positive scale selects 1/sqrt(D)
    c = O.decode_attention(pool, q, "fp16", np.array([[0]]), [n], softmax_scale=0)
    e = O.decode_attention(pool, q, "fp16", np.array([[0]]), [n], softmax_scale=1 / math.sqrt(d))
    assert np.array_equal(c, e)


def test_requantize_makes_slot_live():
    d, n = 128, 256
    k, v = _rand_kv(n, 1, d, 23)
    pool = _pool_with(k, v)
    pool.invalidate_slots([3, 4, 200])
    assert pool.masked(0)[[3, 4, 200]].all()
    pool.quantize_blocks(k, v, "fp16", [0])
    assert not pool.masked(0).any()


def test_q8_blocks_and_mixed_ids():
    d, n = 128, 512
    k, v = _rand_kv(n, 1, d, 24)
    pool = O.OraclePool(1, d, 1, 1)
    pool.quantize_blocks(k, v, "fp16", [1, 0])     # chunk 0 -> 8-bit block, chunk 1 -> 4-bit
    kh8, _ = pool.dequantize_block(1, unrotate_k=True)
    kh4, _ = pool.dequantize_block(0, unrotate_k=True)
    e8 = np.abs(kh8[0] - k[:256, 0].astype(np.float32)).max()
    e4 = np.abs(kh4[0] - k[256:, 0].astype(np.float32)).max()
    assert e8 < e4 / 8
    am = np.array([0.5, 2.0, 1.0, 2.0, 0.1])
    ids = O.mixed_block_ids(am, 2, q4_first=0, q8_first=100)
    # ranking: chunk 1 (2.0), chunk 3 (2.0, tie -> lower index first), chunk 2 ...
    assert list(ids) == [0, 100, 1, 101, 2]
    # with one 8-bit slot the tie between chunks 1 and 3 goes to chunk 1
    assert list(O.mixed_block_ids(am, 1, 0, 100)) == [0, 100, 1, 2, 3]


def test_block_absmean_closed_form():
    k = np.full((300, 2, 128), -1.5, np.float16)
    k[256:] = 0.25
    am = O.block_absmean(k, "fp16")
    assert list(am) == [1.5, 0.25]


def test_bf16_conversion_is_exact():
    bits = np.array([0x3F80, 0xC000, 0x3E80, 0x0001], np.uint16)   # 1, -2, 0.25, tiny
    f = O.to_f32(bits, "bf16")
    assert list(f[:3]) == [1.0, -2.0, 0.25]
    assert f[3] == np.float32(2.0 ** -133)


# ---------------------------------------------------------------------------
# Appending tokens in place
# ---------------------------------------------------------------------------

def test_append_equals_bulk_encoding_of_whole_sequences():
    # Growing sequences in place (ragged lengths, one crossing a block
    # boundary, one not growing, appended slots previously remapped) must leave
    # the pool exactly as encoding each whole sequence in one bulk call
    # through its block table.
    rng = np.random.default_rng(17)
    hkv, d = 3, 128
    lens, new = [300, 254, 40], [5, 4, 0]
    tables = np.array([[3, 0], [1, 2], [4, 5]])
    ks = [rng.standard_normal((lens[b] + new[b], hkv, d)).astype(np.float16) for b in range(3)]
    vs = [rng.standard_normal((lens[b] + new[b], hkv, d)).astype(np.float16) for b in range(3)]
    ref = O.OraclePool(hkv, d, 6)
    grown = O.OraclePool(hkv, d, 6)
    for b in range(3):
        nb = -(-(lens[b] + new[b]) // O.BLOCK_TOKENS)
        ref.quantize_blocks(ks[b], vs[b], "fp16", tables[b][:nb])
        nb0 = -(-lens[b] // O.BLOCK_TOKENS)
        grown.quantize_blocks(ks[b][:lens[b]], vs[b][:lens[b]], "fp16", tables[b][:nb0])
        slots = [int(tables[b][p // 256]) * 256 + p % 256 for p in range(lens[b], lens[b] + new[b])]
        grown.invalidate_slots(slots)
    kn = np.zeros((3, 5, hkv, d), np.float16)
    vn = np.zeros((3, 5, hkv, d), np.float16)
    for b in range(3):
        kn[b, :new[b]] = ks[b][lens[b]:]
        vn[b, :new[b]] = vs[b][lens[b]:]
    grown.append_tokens(kn, vn, "fp16", tables, lens, new)
    for name in "kv":
        np.testing.assert_array_equal(grown.codes4[name], ref.codes4[name])
        np.testing.assert_array_equal(grown.params4[name].view(np.uint16), ref.params4[name].view(np.uint16))
    np.testing.assert_array_equal(grown.mask, ref.mask)


# ---------------------------------------------------------------------------
# FP8 (OCP E4M3) comparison cache
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("x,byte", [
    (1.0, 0x38), (-1.0, 0xB8), (448.0, 0x7E), (-448.0, 0xFE), (500.0, 0x7E), (464.0, 0x7E),
    (2.0 ** -6, 0x08), (2.0 ** -9, 0x01), (0.0, 0x00), (-0.0, 0x80),
    (1.0625, 0x38),           # halfway between 1 and 1.125: ties to the even mantissa (1)
    (1.1875, 0x3A),           # halfway between 1.125 and 1.25: ties to 1.25
    (1.5 * 2.0 ** -9, 0x02),  # subnormal tie goes to the even count (2)
    (2.0 ** -10, 0x00),       # half the smallest subnormal rounds to +0
    (240.0, 0x77), (0.1, 0x1D)])
def test_e4m3_encoding_closed_forms(x, byte):
    # OCP E4M3: value = (1 + m/8) 2^(e - 7) for e in 1..15 (m = 7 with e = 15
    # is NaN, so the largest finite is 1.75 * 2^8 = 448), m/8 * 2^-6 for e = 0
    assert int(O.e4m3_encode(np.array([x], np.float32))[0]) == byte


def test_e4m3_round_trip_and_library_agreement():
    every = np.array([b for b in range(256) if b not in (0x7F, 0xFF)], np.uint8)   # all but NaN
    np.testing.assert_array_equal(O.e4m3_encode(O.e4m3_decode(every)), every)
    # torch's float8_e4m3fn conversion rounds to nearest even inside the range
    import torch
    x = np.clip(np.random.default_rng(5).standard_normal(100000) * 60, -448, 448).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(O.e4m3_encode(x), ref)


def test_fp8_pool_attention_matches_brute_force():
    rng = np.random.default_rng(9)
    hkv, hq, d, n = 1, 4, 128, 300
    k = rng.standard_normal((n, hkv, d)).astype(np.float16)
    v = rng.standard_normal((n, hkv, d)).astype(np.float16)
    pool = O.OraclePool(hkv, d, 0, 2, k_rotated=False, fp8=True)
    pool.quantize_blocks(k, v, "fp16", [1, 0])
    q = rng.standard_normal((1, hq, d)).astype(np.float16)
    out = O.decode_attention(pool, q, "fp16", np.array([[1, 0]]), [n])
    kd = O.e4m3_decode(O.e4m3_encode(k.astype(np.float32)))[:, 0].astype(np.float64)
    vd = O.e4m3_decode(O.e4m3_encode(v.astype(np.float32)))[:, 0].astype(np.float64)
    for h in range(hq):
        s = kd @ q[0, h].astype(np.float64) / math.sqrt(d)
        p = scipy.special.softmax(s)
        np.testing.assert_allclose(out[0, h], p @ vd, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# block images (paging between device and host)
# ---------------------------------------------------------------------------

def _mixed_pool(seed=11, hkv=2, d=128, fp8=False):
    rng = np.random.default_rng(seed)
    n = 3 * 256 - 40
    k = rng.standard_normal((n, hkv, d)).astype(np.float16)
    v = rng.standard_normal((n, hkv, d)).astype(np.float16)
    if fp8:
        pool = O.OraclePool(hkv, d, 0, 4, k_rotated=False, fp8=True)
        pool.quantize_blocks(k, v, "fp16", [2, 0, 3])
    else:
        pool = O.OraclePool(hkv, d, 2, 2)
        pool.quantize_blocks(k, v, "fp16", [1, 3, 0])           # 4-bit, 8-bit, 4-bit
    pool.invalidate_slots([5, 300, 3 * 256 + 7])
    return pool, rng


@pytest.mark.parametrize("fp8", [False, True])
def test_block_image_sizes_follow_the_per_token_byte_counts(fp8):
    """Header 16 B + mask 32 B + the block's bytes: 144 B per (token, KV
    head) for a 4-bit block at D = 128 (the page's ~72 % figure), 272 B for
    an 8-bit block, 256 B for an FP8 block."""
    pool, _ = _mixed_pool(fp8=fp8)
    per = {4: 144, 8: 272, 0x108: 256}
    for blk in range(pool.n_blocks):
        img = pool.block_image(blk)
        assert img.size == 48 + per[pool.block_class(blk)] * 256 * pool.hkv
    assert pool.image_stride() == 48 + (256 if fp8 else 272) * 256 * pool.hkv


def test_block_image_layout_by_independent_indexing():
    """Sampled bytes of the image sit where the layout puts them: K codes of
    (head h, slot t, byte i) at 16 + (h*256 + t)*row + i, V codes one section
    later, then the fp16 (scale, zero) pairs and the mask words."""
    pool, rng = _mixed_pool()
    for blk in (0, 3):
        img = pool.block_image(blk)
        assert img[:4].tobytes() == b"Q4KB"
        assert int.from_bytes(img[4:6].tobytes(), "little") == pool.block_class(blk)
        assert int.from_bytes(img[6:8].tobytes(), "little") == 128
        assert int.from_bytes(img[8:12].tobytes(), "little") == 2
        assert int.from_bytes(img[12:16].tobytes(), "little") == blk
        is4 = blk < pool.n_q4
        row = 64 if is4 else 128
        cbytes = 2 * 256 * row
        pbytes = 2 * 256 * 2 * 4
        kc = pool.codes4["k"][blk] if is4 else pool.codes8["k"][blk - 2]
        vc = pool.codes4["v"][blk] if is4 else pool.codes8["v"][blk - 2]
        vp = pool.params4["v"][blk] if is4 else pool.params8["v"][blk - 2]
        for _ in range(50):
            h, t, i = int(rng.integers(2)), int(rng.integers(256)), int(rng.integers(row))
            assert img[16 + (h * 256 + t) * row + i] == kc[h, t, i]
            assert img[16 + cbytes + (h * 256 + t) * row + i] == vc[h, t, i]
            g, e = int(rng.integers(2)), int(rng.integers(2))
            off = 16 + 2 * cbytes + pbytes + ((h * 256 + t) * 2 + g) * 4 + 2 * e
            assert img[off:off + 2].view(np.float16)[0].view(np.uint16) == vp[h, t, g, e].view(np.uint16)
        mask_off = 16 + 2 * cbytes + 2 * pbytes
        for w in range(8):
            assert int.from_bytes(img[mask_off + 4 * w:mask_off + 4 * w + 4].tobytes(), "little") == int(pool.mask[blk, w])


@pytest.mark.parametrize("fp8", [False, True])
def test_block_images_restore_blocks_exactly(fp8):
    """Loading every block's image into a fresh pool at a permuted id of the
    same class gives back the same dequantised blocks and the same attention."""
    src, rng = _mixed_pool(fp8=fp8)
    dst = (O.OraclePool(2, 128, 0, 4, k_rotated=False, fp8=True) if fp8 else O.OraclePool(2, 128, 2, 2))
    perm = {2: 0, 0: 3, 3: 2, 1: 1} if fp8 else {0: 1, 1: 0, 2: 3, 3: 2}   # same class both sides
    for a, b in perm.items():
        assert dst.load_block_image(b, src.block_image(a))
    for a, b in perm.items():
        for x, y in zip(src.dequantize_block(a), dst.dequantize_block(b)):
            np.testing.assert_array_equal(x, y)
        np.testing.assert_array_equal(src.masked(a), dst.masked(b))
    q = rng.standard_normal((1, 4, 128)).astype(np.float16)
    tbl = [2, 0, 3] if fp8 else [1, 3, 0]
    out_src = O.decode_attention(src, q, "fp16", np.array([tbl]), [3 * 256 - 40])
    out_dst = O.decode_attention(dst, q, "fp16", np.array([[perm[t] for t in tbl]]), [3 * 256 - 40])
    np.testing.assert_array_equal(out_src, out_dst)


def test_block_image_of_another_class_or_shape_is_refused():
    src, _ = _mixed_pool()
    dst = O.OraclePool(2, 128, 2, 2)
    before = dst.block_image(2).copy()
    assert not dst.load_block_image(2, src.block_image(0))      # 4-bit image into an 8-bit block
    np.testing.assert_array_equal(dst.block_image(2), before)
    other = O.OraclePool(4, 128, 2, 2)                          # another Hkv
    assert not other.load_block_image(0, src.block_image(0))
    bad = src.block_image(0).copy()
    bad[0] ^= 1                                                 # broken magic
    assert not dst.load_block_image(0, bad)


# ---------------------------------------------------------------------------
# the mixed-width card (per-token widths {2, 4, 8, FP16})
# ---------------------------------------------------------------------------

def test_code_packing_generalises_the_nibble_order():
    rng = np.random.default_rng(21)
    c4 = rng.integers(0, 16, (3, 128)).astype(np.uint8)
    np.testing.assert_array_equal(O.pack_codes(c4, 4), O.pack_nibbles(c4))
    assert O.pack_codes(np.array([[0, 1, 2, 3]], np.uint8), 2)[0, 0] == 0b11100100
    for bits in (2, 4, 8):
        c = rng.integers(0, 1 << bits, (5, 256)).astype(np.uint8)
        np.testing.assert_array_equal(O.unpack_codes(O.pack_codes(c, bits), bits), c)


def test_card_record_sizes():
    # per (token, KV head): K and V codes plus an fp16 (s, z) pair per group, or two raw 16-bit rows
    assert [O.card_record_bytes(128, w) for w in (2, 4, 8, 16)] == [80, 144, 272, 512]
    assert [O.card_record_bytes(256, w) for w in (2, 4, 8, 16)] == [160, 288, 544, 1024]
    assert O.card_record_bytes(128, 3) == 0
    offs, w_at, o_at, p_at, total = O.card_layout(128, 8, [2, 16, 4, 8, 5])
    assert list(offs) == [0, 640, 640 + 4096, 640 + 4096 + 1152, 640 + 4096 + 1152 + 2176,
                          640 + 4096 + 1152 + 2176]
    assert (w_at, o_at, p_at) == (64, 80, 128) and total == 128 + offs[-1]


def test_card_2bit_ramp_closed_form():
    x = np.zeros((1, 1, 128), np.float32)
    x[0, 0, :64] = np.arange(64)                 # s = 63 / 3 = 21, z = 0
    x[0, 0, 64:] = np.arange(64) * 0.5 - 7.0     # s = 31.5 / 3 = 10.5, z = -7
    card = O.card_encode(x.astype(np.float16), x.astype(np.float16), "fp16", [2], k_rotated=False)
    p_at = O.card_layout(128, 1, [2])[3]
    assert p_at == 64 + 16 + 16                  # header, one width byte, two offsets (each padded to 16)
    rec = card[p_at:p_at + 80]
    codes_v = O.unpack_codes(rec[32:64], 2)
    np.testing.assert_array_equal(codes_v[:64], np.floor(np.arange(64) / 21.0 + 0.5))
    np.testing.assert_array_equal(codes_v[64:], np.floor(np.arange(64) * 0.5 / 10.5 + 0.5))
    par = rec[64 + 8:80].view(np.float16)        # V (s, z) of both groups
    np.testing.assert_array_equal(par, np.array([21.0, 0.0, 10.5, -7.0], np.float16))


def test_card_4_and_8_bit_records_are_the_pool_encoding():
    rng = np.random.default_rng(23)
    n, hkv, d = 256, 2, 128
    k = rng.standard_normal((n, hkv, d)).astype(np.float16)
    v = rng.standard_normal((n, hkv, d)).astype(np.float16)
    widths = rng.choice([4, 8], n)
    card = O.card_encode(k, v, "fp16", widths)
    offs, _, _, p_at, _ = O.card_layout(d, hkv, widths)
    pool = O.OraclePool(hkv, d, 1, 1)
    pool.quantize_blocks(k, v, "fp16", [0])
    pool.quantize_blocks(k, v, "fp16", [1])
    for t in range(n):
        w, at = int(widths[t]), p_at + int(offs[t])
        blk = 0 if w == 4 else 1
        for h in range(hkv):
            rec = card[at:at + O.card_record_bytes(d, w)]
            cb = d * w // 8
            kc = pool.codes4["k"][0, h, t] if w == 4 else pool.codes8["k"][0, h, t]
            vc = pool.codes4["v"][0, h, t] if w == 4 else pool.codes8["v"][0, h, t]
            kp = (pool.params4 if w == 4 else pool.params8)["k"][0, h, t]
            vp = (pool.params4 if w == 4 else pool.params8)["v"][0, h, t]
            np.testing.assert_array_equal(rec[:cb], kc)
            np.testing.assert_array_equal(rec[cb:2 * cb], vc)
            np.testing.assert_array_equal(rec[2 * cb:].view(np.uint16),
                                          np.concatenate([kp.reshape(-1), vp.reshape(-1)]).view(np.uint16))
            at += O.card_record_bytes(d, w)
        assert blk in (0, 1)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_card_round_trip_bounds(dtype):
    rng = np.random.default_rng(29)
    n, hkv, d = 64, 2, 256
    kf = (rng.standard_normal((n, hkv, d)) * 3).astype(np.float32)
    vf = (rng.standard_normal((n, hkv, d)) * 3).astype(np.float32)
    if dtype == "fp16":
        k, v = kf.astype(np.float16), vf.astype(np.float16)
    else:   # bf16 as raw bits (truncated fp32 is an exact bf16 value)
        k = (kf.view(np.uint32) >> 16).astype(np.uint16)
        v = (vf.view(np.uint32) >> 16).astype(np.uint16)
    x_k, x_v = O.to_f32(k, dtype), O.to_f32(v, dtype)
    widths = np.array([(2, 4, 8, 16, 7)[t % 5] for t in range(n)])
    card = O.card_encode(k, v, dtype, widths)
    hd = O.card_header(card)
    assert hd["magic"] == b"QKVC" and hd["n_tokens"] == n and hd["raw_dtype"] == (0 if dtype == "fp16" else 1)
    k_hat, v_hat = O.card_decode(card)
    for t in range(n):
        w = int(widths[t])
        if w == 16:
            np.testing.assert_array_equal(k_hat[t], x_k[t])
            np.testing.assert_array_equal(v_hat[t], x_v[t])
            continue
        if w == 7:
            assert not k_hat[t].any() and not v_hat[t].any()
            continue
        L = (1 << w) - 1
        g = x_v[t].reshape(hkv, d // 64, 64)
        s = (g.max(-1) - g.min(-1)) / L
        bound = 0.5 * s + L * s * 2.0 ** -10 + np.abs(g.min(-1)) * 2.0 ** -10 + 1e-6
        err = np.abs(v_hat[t] - x_v[t]).reshape(hkv, d // 64, 64).max(-1)
        assert (err <= bound).all(), (w, err.max(), bound.min())
        # keys: the rotation is orthonormal, so the l2 error stays within the rotated one's bound
        kr = O.rotate_f32(x_k[t:t + 1])[0].reshape(hkv, d // 64, 64)
        sk = (kr.max(-1) - kr.min(-1)) / L
        lim = np.sqrt(64 * ((0.5 * sk + L * sk * 2.0 ** -10 + np.abs(kr.min(-1)) * 2.0 ** -10) ** 2).sum(-1))
        assert (np.linalg.norm(k_hat[t] - x_k[t], axis=-1) <= lim * 1.001 + 1e-4).all()


# ---------------------------------------------------------------------------
# 2-bit blocks in the paged pool (QKVShare, "Methodologie": widths {2, 4, 8,
# FP16} in one cache; a third block class after the 4- and 8-bit ones)
# ---------------------------------------------------------------------------

def _pool3(seed, d=128, hkv=2, n=700, rotated=True):
    """4-, 8- and 2-bit blocks in one pool: ids 0-1 4-bit, 2 8-bit, 3-4 2-bit."""
    k, v = _rand_kv(n, hkv, d, seed)
    pool = O.OraclePool(hkv, d, 2, 1, k_rotated=rotated, n_q2=2)
    pool.quantize_blocks(k, v, "fp16", [3, 1, 4])                # 2-bit, 4-bit, 2-bit
    return pool, k, v


def test_2bit_ids_follow_the_8bit_ones():
    pool = O.OraclePool(2, 128, 3, 2, n_q2=4)
    assert pool.n_blocks == 9
    assert [pool.bits(b) for b in range(9)] == [4, 4, 4, 8, 8, 2, 2, 2, 2]
    with pytest.raises(IndexError):
        pool.bits(9)


def test_2bit_ramp_codes_and_byte_layout():
    """Values z + k s (k = 0..3, representable s and z) give codes k; the
    stored byte i holds elements 4i .. 4i+3 at bits 0, 2, 4, 6."""
    z, s = np.float32(-1.5), np.float32(0.5)
    d, hkv = 128, 1
    j = np.arange(d)
    pattern = (j * 7 + j // 5) % 4                    # not a plain repeat: catches swapped elements
    x = (z + pattern * s).astype(np.float16)
    k = np.tile(x, (256, hkv, 1)).reshape(256, hkv, d)
    pool = O.OraclePool(hkv, d, 0, 0, k_rotated=False, n_q2=1)
    pool.quantize_blocks(k, k, "fp16", [0])
    for name in "kv":
        byte = pool.codes2[name][0, 0, 0]                # slot 0 of head 0
        want = [int(pattern[4 * i]) | int(pattern[4 * i + 1]) << 2 | int(pattern[4 * i + 2]) << 4
                | int(pattern[4 * i + 3]) << 6 for i in range(d // 4)]
        assert list(byte) == want
        par = pool.params2[name][0, 0, 0]
        assert np.all(par[:, 0] == np.float16(s)) and np.all(par[:, 1] == np.float16(z))


def test_2bit_codes_are_the_nearest_level():
    """Brute force: each code is the level k in {0..3} nearest to x in exact
    arithmetic, z_h + k s_h (elements within 1e-6 s of a midpoint skipped)."""
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((400, 128)) * rng.choice([0.05, 1, 20], size=(400, 1))).astype(np.float32)
    codes, s_h, z_h = O.quantize_groups(x, 2)
    xs = x.reshape(400, 2, 64).astype(np.float64)
    s = s_h.astype(np.float64)[..., None]
    z = z_h.astype(np.float64)[..., None]
    lv = z[..., None] + s[..., None] * np.arange(4)          # [400][2][1][4]
    dist = np.abs(xs[..., None] - lv)
    near = np.argmin(dist, axis=-1)
    srt = np.sort(dist, axis=-1)
    clear = (srt[..., 1] - srt[..., 0]) > 1e-6 * s
    got = codes.reshape(400, 2, 64)
    assert np.all(got[clear & (s > 0)] == near[clear & (s > 0)])
    assert clear.mean() > 0.99


def test_2bit_blocks_dequantise_by_independent_unpacking():
    """K_hat / V_hat of a 2-bit block rebuilt from the raw bytes with shifts
    and masks written here, scale and zero read from the params."""
    pool, _, _ = _pool3(22)
    for blk in (3, 4):
        kh, vh = pool.dequantize_block(blk)
        i2 = blk - pool.n_q4 - pool.n_q8
        for name, got in (("k", kh), ("v", vh)):
            raw = pool.codes2[name][i2].astype(np.uint32)          # [Hkv][256][32]
            c = np.stack([(raw >> (2 * m)) & 3 for m in range(4)], axis=-1).reshape(raw.shape[:-1] + (128,))
            par = pool.params2[name][i2].astype(np.float32)         # [Hkv][256][2][2]
            s = np.repeat(par[..., 0], 64, axis=-1)
            z = np.repeat(par[..., 1], 64, axis=-1)
            want = (c.astype(np.float32) * s + z).astype(np.float32)
            live = ~pool.masked(blk)
            assert np.array_equal(got[:, live], want[:, live])


def test_mixed_2_4_8_pool_attention_matches_brute_force():
    d, hkv, hq, n = 128, 2, 8, 700
    pool, _, _ = _pool3(23, d, hkv, n)
    pool.invalidate_slots([3 * 256 + 9, 1 * 256 + 40])
    rng = np.random.default_rng(24)
    q = rng.standard_normal((1, hq, d)).astype(np.float16)
    tables = np.array([[3, 1, 4]], np.int32)
    out = O.decode_attention(pool, q, "fp16", tables, [n])
    H = scipy.linalg.hadamard(d).astype(np.float64) / math.sqrt(d)
    kh = np.concatenate([pool.dequantize_block(b)[0] for b in (3, 1, 4)], axis=1)[:, :n].astype(np.float64)
    vh = np.concatenate([pool.dequantize_block(b)[1] for b in (3, 1, 4)], axis=1)[:, :n].astype(np.float64)
    masked = np.concatenate([pool.masked(b) for b in (3, 1, 4)])[:n]
    for h in range(hq):
        kv = h // (hq // hkv)
        logits = (kh[kv] @ (H @ q[0, h].astype(np.float64))) / math.sqrt(d)
        logits[masked] = O.SENTINEL_LOGIT
        want = scipy.special.softmax(logits) @ vh[kv]
        assert np.allclose(out[0, h], want, rtol=0, atol=1e-12)


def test_2bit_round_trip_bound():
    rng = np.random.default_rng(25)
    x = (rng.standard_normal((300, 128)) * rng.choice([0.01, 1, 30], size=(300, 1))).astype(np.float32)
    codes, s_h, z_h = O.quantize_groups(x, 2)
    assert codes.max() <= 3
    err, bound = _roundtrip_bound(x, codes, s_h, z_h, 2)
    assert np.all(err <= bound)


def test_2bit_block_image_size_and_restore():
    """A 2-bit block's image: header 16 B + mask 32 B + 80 B per (token, KV
    head) at D = 128 (two 32-byte code rows, two 8-byte param rows); loading
    it into another pool's 2-bit block restores the block exactly."""
    pool, _, _ = _pool3(26)
    img = pool.block_image(3)
    assert pool.block_class(3) == 2
    assert img.size == 48 + 80 * 256 * pool.hkv
    other = O.OraclePool(pool.hkv, pool.d, 2, 1, n_q2=2)
    assert other.load_block_image(4, img)
    assert np.array_equal(other.block_image(4)[16:], img[16:])
    assert not other.load_block_image(0, img)            # a 4-bit block refuses a 2-bit image
