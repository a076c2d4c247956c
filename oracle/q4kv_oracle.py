"""CPU oracle for the 4-bit paged KV cache and its decode attention.

TEST INFRASTRUCTURE.  Only the test suite, the smoke check in
``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` may import or run this module.  The product path never does:
the CUDA library has no CPU fallback and shares no code, constant or table
with this file.

What it computes, step by step, and where each step comes from:

  [AMBP]  "Agent Memory Below the Prompt: Persistent Q4 KV Cache for
          Multi-Agent LLM Inference on Edge Devices" (gist.science summary of
          arXiv 2603.04428).  Section 2.1, item 1: the cache is cut into
          256-token blocks.  Section 2.1, item 2: 4-bit codes packed into
          uint32 words with one 16-bit scale and one 16-bit bias per group,
          read directly by attention ("direct restore"), about 72 % smaller
          than FP16.  Section 2.1, item 3: attention batched over several
          agents' quantised caches.  Section 2.1, item 4: a prompt that
          extends a cached prefix grows the cache instead of being
          prefilled again.  Section 2.2: GQA models.
  [UQ]    UltraQuant news item (poko-everyday.com, arXiv 2606.20474),
          section "technology / business": a Walsh-Hadamard rotation before
          4-bit quantisation, with keys and values treated asymmetrically;
          the 4-bit cache is measured against an FP8 KV cache.
  [IKV]   IntentKV article (Qiita), section "invalidate instead of
          compacting": an evicted slot is re-pointed to a sentinel slot
          whose key is -1e4, so its softmax weight collapses to zero while
          every surviving slot keeps its position.
  [QKVS]  QKVShare (gist.science summary of arXiv 2605.03884),
          "Methodologie": bit widths drawn from {2, 4, 8, FP16}; the
          receiver dequantises the shared cache before use.

Readings taken where the pages leave a step open (each is restated in the
design notes):
  * groups are 64 consecutive values along head_dim of one (token, head)
    vector; scale s and zero z are fp16 (binary16), z is an additive offset;
  * the rotation is the orthonormal Sylvester-ordered Walsh-Hadamard
    transform c*H_D, c = binary32 nearest to 1/sqrt(D), butterflies applied
    in ascending stride order h = 1, 2, ..., D/2; K is rotated, V is not;
    the query is rotated by the same transform inside attention;
  * codes are computed from the *stored* fp16 s and z with binary32
    subtraction and division, rounded half to even, then clamped;
    min and max have +0.0 added so a signed zero never reaches the
    stored parameters;
  * nibble order: value 2i in the low nibble of byte i, so element j of a
    little-endian uint32 word sits at bits 4*(j mod 8);
  * an evicted slot's *logit* is -1e4 and its value is 0; its stored bytes
    stay where they are; one 256-bit mask per physical block, shared by
    all KV heads; writing a token into a slot makes the slot live again;
  * 8-bit blocks use the same steps with 255 levels, one code per byte;
    2-bit blocks ([QKVS] widths from {2, 4, 8, FP16}, here a third block
    class) the same steps with 3 levels, four codes per byte, element
    4i + m at bits 2m of byte i (the nibble order, generalised);
  * the FP8 comparison cache stores each raw value as one OCP E4M3 byte
    (bias 7, 3 mantissa bits, no infinities, largest finite 448), rounded
    to nearest with ties to even and saturated to +-448; no scale, no
    rotation (the plainest FP8 KV cache);
  * paging a block out of and back into the device ([AMBP] section 2.1,
    items 1 and 3: blocks move between memory and storage, one agent's
    cache is brought in while another decodes) copies its bytes unchanged:
    a block image is a 16-byte header followed by the block's sections in
    the pool's own layout, and loading it restores the block exactly;
  * per-token widths from {2, 4, 8, FP16} in one cache ([QKVS]
    "Methodologie": the CacheCard carries quantised groups and per-token
    widths, and the receiver rebuilds FP16 keys and values before use): a
    card holds each token at its own width with the pool's group coding
    (L = 2^w - 1; 2-bit codes four to a byte in the nibble order, generalised)
    or as its raw 16-bit rows, and decoding it dequantises and un-rotates.

Precision: the encoding steps (rotation, min/max, scale/zero, codes,
dequantisation) are binary32/binary16 by definition, so they are written
with numpy float32/float16 scalars-arrays, one IEEE operation per step and
no fused multiply-add.  Attention is fp64 over the dequantised cache.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

BLOCK_TOKENS = 256          # [AMBP] 2.1 item 1
GROUP = 64                  # values sharing one (scale, zero) pair
SENTINEL_LOGIT = -1.0e4     # [IKV]
MASK_WORDS = BLOCK_TOKENS // 32
# Block images [AMBP 2.1 item 1: blocks are paged between memory and storage]:
# a fixed 16-byte header, then the block's bytes as the pool holds them.
IMAGE_MAGIC = b"Q4KB"
IMAGE_HEADER_BYTES = 16


def levels(bits: int) -> int:
    """Largest code of a `bits`-wide unsigned code (15 for Q4, 255 for Q8)."""
    return (1 << bits) - 1


# ---------------------------------------------------------------------------
# input conversion (exact)
# ---------------------------------------------------------------------------

def to_f32(a: np.ndarray, dtype: str) -> np.ndarray:
    """fp16 / bf16 input -> binary32, exactly.

    fp16 arrives as np.float16; bf16 arrives as its raw uint16 bit pattern
    (numpy has no bfloat16), which is the upper half of a binary32.
    """
    if dtype == "fp16":
        return np.asarray(a, dtype=np.float16).astype(np.float32)
    if dtype == "bf16":
        bits = np.asarray(a, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
        return bits.view(np.float32)
    if dtype == "fp32":
        return np.asarray(a, dtype=np.float32)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# Walsh-Hadamard rotation [UQ]
# ---------------------------------------------------------------------------

def rotation_constant(d: int) -> np.float32:
    """c = binary32 nearest to 1/sqrt(d) for d a power of two.

    1/sqrt(2^k) is 2^(-k/2) for even k and sqrt(2) * 2^(-(k+1)/2) for odd k;
    both are formed from the correctly rounded double sqrt(2), then rounded
    once to binary32.
    """
    k = int(round(math.log2(d)))
    assert 1 << k == d, "head_dim must be a power of two"
    if k % 2 == 0:
        return np.float32(2.0 ** (-k // 2))
    return np.float32(math.sqrt(2.0) * 2.0 ** (-(k + 1) // 2))


def fwht(x: np.ndarray, dtype=np.float32) -> np.ndarray:
    """Unnormalised Sylvester-ordered Walsh-Hadamard transform, last axis.

    Stages run with stride h = 1, 2, 4, ..., n/2.  In each stage every pair
    (i, i+h) with bit h of i clear becomes (x_i + x_{i+h}, x_i - x_{i+h}),
    each sum and difference one IEEE operation in `dtype`.  The result is
    H_n x with H_n[i, j] = (-1)^popcount(i & j).
    """
    y = np.array(x, dtype=dtype, copy=True)
    n = y.shape[-1]
    h = 1
    while h < n:
        v = y.reshape(y.shape[:-1] + (n // (2 * h), 2, h))
        a = v[..., 0, :].copy()
        b = v[..., 1, :].copy()
        v[..., 0, :] = a + b
        v[..., 1, :] = a - b
        h *= 2
    return y


def rotate_f32(x: np.ndarray) -> np.ndarray:
    """c * H x in binary32: the butterflies, then one multiply by c."""
    d = x.shape[-1]
    return fwht(x, np.float32) * rotation_constant(d)


def rotate_f64(x: np.ndarray) -> np.ndarray:
    """(1/sqrt(D)) * H x in fp64 (used for the query inside attention)."""
    d = x.shape[-1]
    return fwht(x, np.float64) * (1.0 / math.sqrt(d))


# ---------------------------------------------------------------------------
# group quantisation [AMBP 2.1 item 2], [UQ], [QKVS]
# ---------------------------------------------------------------------------

def quantize_groups(x: np.ndarray, bits: int):
    """Quantise binary32 vectors x[..., D] group by group.

    Returns (codes uint8 [..., D], scale fp16 [..., D/64], zero fp16 [..., D/64]).
    Per group of 64 values:
      mn = min + 0, mx = max + 0                  (exact)
      s  = fl(fl(mx - mn) / L)                    L = 2^bits - 1
      s_h = fp16(s), z_h = fp16(mn)               round to nearest even
      code = 0 if s_h == 0 else clamp(rne(fl(fl(x - z_h) / s_h)), 0, L)
    """
    x = np.asarray(x, dtype=np.float32)
    d = x.shape[-1]
    assert d % GROUP == 0
    L = np.float32(levels(bits))
    g = x.reshape(x.shape[:-1] + (d // GROUP, GROUP))
    zero = np.float32(0.0)
    mn = g.min(axis=-1) + zero
    mx = g.max(axis=-1) + zero
    s = (mx - mn) / L
    s_h = s.astype(np.float16)
    z_h = mn.astype(np.float16)
    sf = s_h.astype(np.float32)[..., None]
    zf = z_h.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (g - zf) / sf
    q = np.clip(np.rint(t), zero, L)
    q = np.where(sf == zero, zero, q)
    return q.astype(np.uint8).reshape(x.shape), s_h, z_h


def dequantize_groups(codes: np.ndarray, s_h: np.ndarray, z_h: np.ndarray) -> np.ndarray:
    """x_hat = fl(code * s_h + z_h) in binary32 (code * s_h is exact)."""
    codes = np.asarray(codes)
    d = codes.shape[-1]
    c = codes.astype(np.float32).reshape(codes.shape[:-1] + (d // GROUP, GROUP))
    sf = np.asarray(s_h, dtype=np.float16).astype(np.float32)[..., None]
    zf = np.asarray(z_h, dtype=np.float16).astype(np.float32)[..., None]
    return (c * sf + zf).reshape(codes.shape)


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte: element 2i low nibble, 2i+1 high nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[..., 0::2] | (codes[..., 1::2] << np.uint8(4))).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & np.uint8(0x0F)
    out[..., 1::2] = packed >> np.uint8(4)
    return out


# ---------------------------------------------------------------------------
# FP8 E4M3 values of the comparison cache [UQ]
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """OCP E4M3 bytes of finite values x: round to nearest, ties to even, on
    the E4M3 grid (spacing 2^(e-3) for |x| in [2^e, 2^(e+1)), e >= -6, and
    2^-9 below 2^-6), then saturate to +-448."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    sign = np.signbit(x).astype(np.uint8) << np.uint8(7)
    a = np.minimum(a, E4M3_MAX)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    quantum = np.exp2(e - 3.0)
    r = np.minimum(np.rint(a / quantum) * quantum, E4M3_MAX)   # a / quantum is exact in fp64
    with np.errstate(divide="ignore"):
        er = np.floor(np.log2(np.where(r > 0, r, 1.0)))
    normal = r >= 2.0 ** -6
    exp_field = np.where(normal, er + 7.0, 0.0)
    mant = np.where(normal, r / np.exp2(er) - 1.0, r / 2.0 ** -9 / 8.0) * 8.0
    bits = (exp_field.astype(np.uint8) << np.uint8(3)) | np.rint(mant).astype(np.uint8)
    return (bits | sign).astype(np.uint8)


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    """binary32 value of OCP E4M3 bytes (every one is exact in binary32)."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int32)
    sign = np.where(b & 0x80, -1.0, 1.0)
    ef = (b >> 3) & 0xF
    mf = b & 0x7
    val = np.where(ef == 0, mf * 2.0 ** -9, (1.0 + mf / 8.0) * np.exp2(ef - 7.0))
    return (sign * val).astype(np.float32)


# ---------------------------------------------------------------------------
# the paged pool [AMBP 2.1 items 1-2], eviction mask [IKV]
# ---------------------------------------------------------------------------

class OraclePool:
    """Host model of the paged cache.

    Unified block ids: [0, n_q4) are 4-bit blocks, [n_q4, n_q4 + n_q8) are
    8-bit blocks, [n_q4 + n_q8, n_q4 + n_q8 + n_q2) are 2-bit blocks
    ([QKVS] "Methodologie": widths from {2, 4, 8, FP16} in one cache; here
    per block).  Per block and KV head: codes [256][D/2] (4-bit), [256][D]
    (8-bit) or [256][D/4] (2-bit, element 4i + m at bits 2m of byte i) and
    params [256][D/64][2] fp16 as (scale, zero).  mask[block][8] uint32:
    bit (slot mod 32) of word (slot / 32) set means the slot has been
    remapped to the sentinel.
    """

    def __init__(self, n_kv_heads: int, head_dim: int, n_q4: int, n_q8: int = 0,
                 k_rotated: bool = True, fp8: bool = False, n_q2: int = 0):
        if fp8 and (n_q4 or n_q2 or k_rotated):
            raise ValueError("an FP8 pool has only 8-bit blocks and raw keys")
        self.fp8 = fp8
        self.hkv = n_kv_heads
        self.d = head_dim
        self.n_q4 = n_q4
        self.n_q8 = n_q8
        self.k_rotated = k_rotated
        ng = head_dim // GROUP
        T = BLOCK_TOKENS
        self.codes4 = {s: np.zeros((n_q4, n_kv_heads, T, head_dim // 2), np.uint8) for s in "kv"}
        self.params4 = {s: np.zeros((n_q4, n_kv_heads, T, ng, 2), np.float16) for s in "kv"}
        self.codes8 = {s: np.zeros((n_q8, n_kv_heads, T, head_dim), np.uint8) for s in "kv"}
        self.params8 = {s: np.zeros((n_q8, n_kv_heads, T, ng, 2), np.float16) for s in "kv"}
        self.n_q2 = n_q2
        self.codes2 = {s: np.zeros((n_q2, n_kv_heads, T, head_dim // 4), np.uint8) for s in "kv"}
        self.params2 = {s: np.zeros((n_q2, n_kv_heads, T, ng, 2), np.float16) for s in "kv"}
        self.mask = np.zeros((n_q4 + n_q8 + n_q2, MASK_WORDS), np.uint32)

    @property
    def n_blocks(self) -> int:
        return self.n_q4 + self.n_q8 + self.n_q2

    def bits(self, blk: int) -> int:
        if not 0 <= blk < self.n_blocks:
            raise IndexError(f"block id {blk} outside [0, {self.n_blocks})")
        if blk < self.n_q4:
            return 4
        return 8 if blk < self.n_q4 + self.n_q8 else 2

    def _store(self, name: str, blk: int, slots, codes: np.ndarray, par: np.ndarray) -> None:
        """Write codes [Hkv][n][D] (unpacked) and params [Hkv][n][ng][2] of
        `slots` of block `blk` in the block's width."""
        bits = self.bits(blk)
        if bits == 4:
            self.codes4[name][blk, :, slots] = pack_nibbles(codes)
            self.params4[name][blk, :, slots] = par
        elif bits == 8:
            i8 = blk - self.n_q4
            self.codes8[name][i8, :, slots] = codes
            self.params8[name][i8, :, slots] = par
        else:
            i2 = blk - self.n_q4 - self.n_q8
            self.codes2[name][i2, :, slots] = pack_codes(codes, 2)
            self.params2[name][i2, :, slots] = par

    # -- writes ------------------------------------------------------------
    def quantize_blocks(self, k: np.ndarray, v: np.ndarray, dtype: str,
                        block_ids: Sequence[int]) -> None:
        """Encode tokens k/v [n][Hkv][D] into the pool.

        Token i goes to block block_ids[i // 256], slot i % 256; the slot's
        mask bit is cleared (a freshly written slot is live).
        """
        kf = to_f32(k, dtype)
        vf = to_f32(v, dtype)
        n = kf.shape[0]
        assert kf.shape == (n, self.hkv, self.d) and vf.shape == kf.shape
        for c in range(-(-n // BLOCK_TOKENS)):
            t0, t1 = c * BLOCK_TOKENS, min(n, (c + 1) * BLOCK_TOKENS)
            blk = int(block_ids[c])
            bits = self.bits(blk)
            kk = kf[t0:t1]
            if self.k_rotated:
                kk = rotate_f32(kk)
            for name, x in (("k", kk), ("v", vf[t0:t1])):
                if self.fp8:
                    self.codes8[name][blk, :, : t1 - t0] = e4m3_encode(x).transpose(1, 0, 2)
                    continue
                codes, s_h, z_h = quantize_groups(x, bits)       # [cnt][Hkv][D]
                codes = codes.transpose(1, 0, 2)                  # [Hkv][cnt][D]
                par = np.stack([s_h, z_h], axis=-1).transpose(1, 0, 2, 3)
                self._store(name, blk, slice(0, t1 - t0), codes, par)
            for slot in range(t1 - t0):
                self.mask[blk, slot // 32] &= np.uint32(~(1 << (slot % 32)) & 0xFFFFFFFF)

    def append_tokens(self, k: np.ndarray, v: np.ndarray, dtype: str, tables: np.ndarray,
                      seq_lens: Sequence[int], n_new: Optional[Sequence[int]] = None) -> None:
        """Grow each sequence's cache in place [AMBP 2.1 items 3-4].

        k, v: [B][T][Hkv][D].  Token i < n_new[b] (all T if None) of sequence
        b is the token at position p = seq_lens[b] + i, stored in block
        tables[b][p // 256], slot p % 256, with exactly the per-vector encoding
        quantize_blocks gives it; the slot's mask bit is cleared.
        """
        kf = to_f32(k, dtype)
        vf = to_f32(v, dtype)
        nb, nt = kf.shape[0], kf.shape[1]
        for b in range(nb):
            for i in range(nt if n_new is None else int(n_new[b])):
                p = int(seq_lens[b]) + i
                blk = int(tables[b][p // BLOCK_TOKENS])
                slot = p % BLOCK_TOKENS
                bits = self.bits(blk)
                kk = kf[b, i][None]                           # [1][Hkv][D]
                if self.k_rotated:
                    kk = rotate_f32(kk)
                for name, x in (("k", kk), ("v", vf[b, i][None])):
                    if self.fp8:
                        self.codes8[name][blk, :, slot] = e4m3_encode(x[0])
                        continue
                    codes, s_h, z_h = quantize_groups(x, bits)
                    par = np.stack([s_h[0], z_h[0]], axis=-1)  # [Hkv][D/64][2]
                    self._store(name, blk, slice(slot, slot + 1), codes[0][:, None], par[:, None])
                self.mask[blk, slot // 32] &= np.uint32(~(1 << (slot % 32)) & 0xFFFFFFFF)

    def invalidate_slots(self, slot_ids: Sequence[int]) -> None:
        """Remap physical slots (block*256 + offset) to the sentinel [IKV]."""
        for sid in slot_ids:
            sid = int(sid)
            blk, slot = divmod(sid, BLOCK_TOKENS)
            self.bits(blk)
            self.mask[blk, slot // 32] |= np.uint32(1 << (slot % 32))

    # -- block images: paging between device and host [AMBP 2.1 items 1, 3; 5] --
    def block_class(self, blk: int) -> int:
        """Class tag of a block's image: 2, 4 or 8 (code width) or 0x108 (FP8)."""
        bits = self.bits(blk)
        return 0x108 if self.fp8 else bits

    def image_sections(self, cls: int):
        """(name, bytes) of the sections of an image of class `cls`, in order."""
        row = {2: self.d // 4, 4: self.d // 2}.get(cls, self.d)
        codes = self.hkv * BLOCK_TOKENS * row
        params = 0 if cls == 0x108 else self.hkv * BLOCK_TOKENS * (self.d // GROUP) * 4
        secs = [("header", IMAGE_HEADER_BYTES), ("k_codes", codes), ("v_codes", codes)]
        if params:
            secs += [("k_params", params), ("v_params", params)]
        return secs + [("mask", MASK_WORDS * 4)]

    def image_stride(self) -> int:
        """Bytes between consecutive images: the largest class of the pool."""
        classes = [0x108] if self.fp8 else (([4] if self.n_q4 else []) + ([8] if self.n_q8 else [])
                                             + ([2] if self.n_q2 else []))
        return max(sum(b for _, b in self.image_sections(c)) for c in classes or [4])

    def _block_arrays(self, blk: int):
        """The block's arrays (views) in image order, header excluded."""
        if self.bits(blk) == 4:
            arrs = [self.codes4["k"][blk], self.codes4["v"][blk],
                    self.params4["k"][blk], self.params4["v"][blk]]
        elif self.bits(blk) == 2:
            i2 = blk - self.n_q4 - self.n_q8
            arrs = [self.codes2["k"][i2], self.codes2["v"][i2],
                    self.params2["k"][i2], self.params2["v"][i2]]
        else:
            i8 = blk - self.n_q4
            arrs = [self.codes8["k"][i8], self.codes8["v"][i8]]
            if not self.fp8:
                arrs += [self.params8["k"][i8], self.params8["v"][i8]]
        return arrs + [self.mask[blk]]

    def block_image(self, blk: int) -> np.ndarray:
        """uint8 image of block `blk`: a 16-byte header (magic 'Q4KB', class,
        head_dim, Hkv, source block id; little-endian) and then the block's
        bytes exactly as the pool holds them -- K codes, V codes, K params,
        V params (not for FP8), remap mask -- each section contiguous."""
        hdr = np.zeros(IMAGE_HEADER_BYTES, np.uint8)
        hdr[0:4] = np.frombuffer(IMAGE_MAGIC, np.uint8)
        hdr[4:6] = np.array([self.block_class(blk)], "<u2").view(np.uint8)
        hdr[6:8] = np.array([self.d], "<u2").view(np.uint8)
        hdr[8:12] = np.array([self.hkv], "<u4").view(np.uint8)
        hdr[12:16] = np.array([blk], "<i4").view(np.uint8)
        parts = [hdr] + [np.ascontiguousarray(a).reshape(-1).view(np.uint8) for a in self._block_arrays(blk)]
        return np.concatenate(parts)

    def image_matches(self, blk: int, image: np.ndarray) -> bool:
        """True when the header fits block `blk` of this pool (magic, class,
        head_dim, Hkv; the source id is not checked)."""
        h = np.asarray(image[:IMAGE_HEADER_BYTES], np.uint8)
        return (h[0:4].tobytes() == IMAGE_MAGIC
                and int(h[4:6].view("<u2")[0]) == self.block_class(blk)
                and int(h[6:8].view("<u2")[0]) == self.d
                and int(h[8:12].view("<u4")[0]) == self.hkv)

    def load_block_image(self, blk: int, image: np.ndarray) -> bool:
        """Replace block `blk` (codes, params, mask) by an image; an image
        whose header does not fit the block changes nothing (returns False)."""
        image = np.asarray(image, np.uint8)
        if not self.image_matches(blk, image):
            return False
        off = IMAGE_HEADER_BYTES
        for a in self._block_arrays(blk):
            nb = a.size * a.itemsize
            a[...] = image[off:off + nb].view(a.dtype).reshape(a.shape)
            off += nb
        return True

    # -- reads -------------------------------------------------------------
    def masked(self, blk: int) -> np.ndarray:
        """bool [256]: slot remapped to the sentinel."""
        words = self.mask[blk]
        return np.array([(int(words[t // 32]) >> (t % 32)) & 1 for t in range(BLOCK_TOKENS)],
                        dtype=bool)

    def codes_params(self, blk: int, name: str):
        """(codes uint8 [Hkv][256][D], scale fp16 [Hkv][256][ng], zero fp16)."""
        if self.bits(blk) == 4:
            codes = unpack_nibbles(self.codes4[name][blk])
            par = self.params4[name][blk]
        elif self.bits(blk) == 2:
            i2 = blk - self.n_q4 - self.n_q8
            codes = unpack_codes(self.codes2[name][i2], 2)
            par = self.params2[name][i2]
        else:
            codes = self.codes8[name][blk - self.n_q4]
            par = self.params8[name][blk - self.n_q4]
        return codes, par[..., 0], par[..., 1]

    def dequantize_block(self, blk: int, unrotate_k: bool = False):
        """Binary32 K_hat, V_hat [Hkv][256][D] with the sentinel applied.

        K is in the stored (rotated) domain unless `unrotate_k`; the inverse
        of c*H is c*H itself (H symmetric, H H^T = D I), applied with the
        same butterfly order.  Remapped slots read K = -1e4, V = 0.
        """
        out = []
        for name in "kv":
            if self.fp8:
                self.bits(blk)
                out.append(e4m3_decode(self.codes8[name][blk]))
                continue
            codes, s_h, z_h = self.codes_params(blk, name)
            x = dequantize_groups(codes, s_h, z_h)
            if name == "k" and unrotate_k and self.k_rotated:
                x = rotate_f32(x)
            out.append(x)
        k_hat, v_hat = out
        m = self.masked(blk)
        k_hat[:, m, :] = np.float32(SENTINEL_LOGIT)
        v_hat[:, m, :] = np.float32(0.0)
        return k_hat, v_hat


# ---------------------------------------------------------------------------
# decode attention [AMBP 2.1 items 2-3, 2.2], [IKV]
# ---------------------------------------------------------------------------

def decode_attention(pool: OraclePool, q: np.ndarray, q_dtype: str,
                     block_tables: np.ndarray, seq_lens: Sequence[int],
                     softmax_scale: Optional[float] = None,
                     heads: Optional[Sequence[tuple]] = None) -> np.ndarray:
    """fp64 single-token GQA attention over the paged quantised cache.

    For sequence b and query head h (KV head h // g): token t of the
    sequence lives in block block_tables[b][t // 256], slot t % 256.  Its
    logit is scale * <q_rot, K_hat_t> (q_rot = (1/sqrt D) H q when K is
    stored rotated), or -1e4 if the slot is remapped, in which case its
    value is 0.  Output = softmax(logits) . V_hat, softmax max-subtracted.
    A sequence with no tokens yields 0.

    `heads` optionally restricts the work to a list of (b, h) pairs; the
    other rows of the result stay 0.
    """
    qf = to_f32(q, q_dtype).astype(np.float64)
    B, Hq, D = qf.shape
    g = Hq // pool.hkv
    assert g * pool.hkv == Hq and D == pool.d
    if softmax_scale is None or softmax_scale <= 0:
        softmax_scale = 1.0 / math.sqrt(D)
    want = None if heads is None else {}
    if heads is not None:
        for b, h in heads:
            want.setdefault(int(b), []).append(int(h))
    out = np.zeros((B, Hq, D), np.float64)
    for b in range(B):
        if want is not None and b not in want:
            continue
        n = int(seq_lens[b])
        if n == 0:
            continue
        ks, vs, ms = [], [], []
        for c in range(-(-n // BLOCK_TOKENS)):
            cnt = min(BLOCK_TOKENS, n - c * BLOCK_TOKENS)
            blk = int(block_tables[b][c])
            k_hat, v_hat = pool.dequantize_block(blk)
            ks.append(k_hat[:, :cnt])
            vs.append(v_hat[:, :cnt])
            ms.append(pool.masked(blk)[:cnt])
        K = np.concatenate(ks, axis=1).astype(np.float64)    # [Hkv][n][D]
        V = np.concatenate(vs, axis=1).astype(np.float64)
        M = np.concatenate(ms)
        for h in (range(Hq) if want is None else want[b]):
            kv = h // g
            qv = rotate_f64(qf[b, h]) if pool.k_rotated else qf[b, h]
            s = softmax_scale * (K[kv] @ qv)
            s[M] = SENTINEL_LOGIT          # V_hat of these rows is already 0
            p = np.exp(s - s.max())
            out[b, h] = (p @ V[kv]) / p.sum()
    return out


# ---------------------------------------------------------------------------
# mixed 4/8-bit block selection [QKVS]
# ---------------------------------------------------------------------------

def block_absmean(k: np.ndarray, dtype: str) -> np.ndarray:
    """fp64 mean |K| of each 256-token chunk of raw (unrotated) keys [n][Hkv][D]."""
    kf = to_f32(k, dtype).astype(np.float64)
    n = kf.shape[0]
    out = []
    for c in range(-(-n // BLOCK_TOKENS)):
        chunk = np.abs(kf[c * BLOCK_TOKENS: (c + 1) * BLOCK_TOKENS])
        out.append(chunk.sum() / chunk.size)
    return np.array(out, dtype=np.float64)


def mixed_block_ids(absmean: np.ndarray, n_q8: int, q4_first: int, q8_first: int) -> np.ndarray:
    """Block id per chunk: the n_q8 chunks of highest mean |K| go 8-bit.

    Ranking is descending mean |K| with ties to the lower chunk index.  The
    k-th 8-bit chunk in chunk order gets id q8_first + k, the k-th 4-bit
    chunk gets q4_first + k.
    """
    n = len(absmean)
    order = sorted(range(n), key=lambda i: (-float(absmean[i]), i))
    chosen = set(order[:n_q8])
    ids = np.empty(n, np.int32)
    n8 = n4 = 0
    for i in range(n):
        if i in chosen:
            ids[i] = q8_first + n8
            n8 += 1
        else:
            ids[i] = q4_first + n4
            n4 += 1
    return ids


def bytes_per_token_head(head_dim: int, bits: int) -> int:
    """Stored bytes for one (token, KV head): K and V codes plus fp16 (s, z)."""
    code_bytes = head_dim * bits // 8
    param_bytes = (head_dim // GROUP) * 2 * 2
    return 2 * (code_bytes + param_bytes)


# ---------------------------------------------------------------------------
# per-token widths {2, 4, 8, FP16} in one cache: the card [QKVS "Methodologie"]
# ---------------------------------------------------------------------------
# QKVS gives every token a width from {2, 4, 8, FP16} and ships the cache as
# a compact artifact holding the quantised groups, the per-token widths and
# metadata; the receiver rebuilds FP16 keys and values from it before use.
# Reading: the card is a 64-byte header, the widths (one byte per token), the
# byte offset of every token's record, then the records.  A token's record is,
# for every KV head in order, its K codes, V codes, K (s, z) pairs and V (s, z)
# pairs at its width (the pool's group coding with L = 2^w - 1, K rotated when
# the card says so), or for an FP16 token its raw 16-bit K and V rows.
CARD_MAGIC = b"QKVC"
CARD_VERSION = 1
CARD_HEADER_BYTES = 64
CARD_WIDTHS = (2, 4, 8, 16)


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """bits-wide codes [..., D] -> bytes: element e sits at bits
    bits*(e mod 8/bits) of byte e*bits/8 (the nibble order, generalised)."""
    per = 8 // bits
    c = np.asarray(codes, np.uint32).reshape(codes.shape[:-1] + (codes.shape[-1] // per, per))
    out = np.zeros(c.shape[:-1], np.uint32)
    for e in range(per):
        out |= c[..., e] << np.uint32(bits * e)
    return out.astype(np.uint8)


def unpack_codes(packed: np.ndarray, bits: int) -> np.ndarray:
    per = 8 // bits
    p = np.asarray(packed, np.uint32)[..., None]
    shifts = np.arange(per, dtype=np.uint32) * np.uint32(bits)
    out = (p >> shifts) & np.uint32((1 << bits) - 1)
    return out.reshape(packed.shape[:-1] + (packed.shape[-1] * per,)).astype(np.uint8)


def card_record_bytes(head_dim: int, bits: int) -> int:
    """Bytes of one (token, KV head) record at width `bits`; 0 for a width
    outside {2, 4, 8, 16} (such a token is skipped)."""
    if bits == 16:
        return 4 * head_dim
    if bits in (2, 4, 8):
        return bytes_per_token_head(head_dim, bits)
    return 0


def _round16(x: int) -> int:
    return (x + 15) // 16 * 16


def card_layout(head_dim: int, n_kv_heads: int, widths: Sequence[int]):
    """(offsets of each token's record from the payload start, int64 [n + 1];
    byte offsets of the widths, the offsets table and the payload; total
    card bytes)."""
    n = len(widths)
    rec = np.array([n_kv_heads * card_record_bytes(head_dim, int(w)) for w in widths], np.int64)
    offs = np.zeros(n + 1, np.int64)
    offs[1:] = np.cumsum(rec)
    widths_at = CARD_HEADER_BYTES
    offsets_at = widths_at + _round16(n)
    payload_at = offsets_at + _round16(8 * (n + 1))
    return offs, widths_at, offsets_at, payload_at, payload_at + int(offs[-1])


def card_encode(k: np.ndarray, v: np.ndarray, dtype: str, widths: Sequence[int],
                k_rotated: bool = True) -> np.ndarray:
    """The card (uint8) of tokens k, v [n][Hkv][D] at per-token widths."""
    n, hkv, d = np.asarray(k).shape
    kf, vf = to_f32(k, dtype), to_f32(v, dtype)
    raw_k = np.asarray(k).view(np.uint16) if dtype == "fp16" else np.asarray(k, np.uint16)
    raw_v = np.asarray(v).view(np.uint16) if dtype == "fp16" else np.asarray(v, np.uint16)
    offs, w_at, o_at, p_at, total = card_layout(d, hkv, widths)
    card = np.zeros(total, np.uint8)
    hdr = card[:CARD_HEADER_BYTES]
    hdr[0:4] = np.frombuffer(CARD_MAGIC, np.uint8)
    hdr[4:24] = np.array([CARD_VERSION, d, hkv, n & 0xFFFFFFFF, n >> 32], "<u4").view(np.uint8)
    hdr[24:32] = np.array([int(k_rotated), 0 if dtype == "fp16" else 1], "<u4").view(np.uint8)
    hdr[32:40] = np.array([offs[-1]], "<i8").view(np.uint8)
    card[w_at:w_at + n] = np.asarray(widths, np.uint8)
    card[o_at:o_at + 8 * (n + 1)] = offs.astype("<i8").view(np.uint8)
    for t in range(n):
        w = int(widths[t])
        at = p_at + int(offs[t])
        if w == 16:
            for h in range(hkv):
                rec = np.concatenate([raw_k[t, h].astype("<u2").view(np.uint8),
                                      raw_v[t, h].astype("<u2").view(np.uint8)])
                card[at:at + rec.size] = rec
                at += rec.size
            continue
        if w not in (2, 4, 8):
            continue
        kk = rotate_f32(kf[t:t + 1])[0] if k_rotated else kf[t]
        ck, sk, zk = quantize_groups(kk, w)          # [Hkv][D], [Hkv][D/64]
        cv, sv, zv = quantize_groups(vf[t], w)
        for h in range(hkv):
            pk = np.stack([sk[h], zk[h]], axis=-1).reshape(-1).view(np.uint8)
            pv = np.stack([sv[h], zv[h]], axis=-1).reshape(-1).view(np.uint8)
            rec = np.concatenate([pack_codes(ck[h], w), pack_codes(cv[h], w), pk, pv])
            card[at:at + rec.size] = rec
            at += rec.size
    return card


def card_header(card: np.ndarray) -> dict:
    h = np.asarray(card[:CARD_HEADER_BYTES], np.uint8)
    u = h[4:32].view("<u4")
    return dict(magic=h[0:4].tobytes(), version=int(u[0]), head_dim=int(u[1]), n_kv_heads=int(u[2]),
                n_tokens=int(u[3]) | (int(u[4]) << 32), k_rotated=int(u[5]), raw_dtype=int(u[6]),
                payload_bytes=int(h[32:40].view("<i8")[0]))


def card_decode(card: np.ndarray):
    """Binary32 K_hat, V_hat [n][Hkv][D] of a card: x_hat = fl(code s + z),
    K un-rotated by c*H when stored rotated; FP16 tokens exactly; a token of
    an invalid width reads 0."""
    hd = card_header(card)
    n, hkv, d = hd["n_tokens"], hd["n_kv_heads"], hd["head_dim"]
    widths = np.asarray(card[CARD_HEADER_BYTES:CARD_HEADER_BYTES + n], np.uint8)
    offs, _, o_at, p_at, _ = card_layout(d, hkv, widths)
    stored = np.asarray(card[o_at:o_at + 8 * (n + 1)]).view("<i8")
    assert np.array_equal(stored, offs), "offset table does not match the widths"
    k_hat = np.zeros((n, hkv, d), np.float32)
    v_hat = np.zeros((n, hkv, d), np.float32)
    raw = "fp16" if hd["raw_dtype"] == 0 else "bf16"
    ng = d // GROUP
    for t in range(n):
        w = int(widths[t])
        at = p_at + int(offs[t])
        for h in range(hkv):
            if w == 16:
                rk = np.asarray(card[at:at + 2 * d]).view("<u2")
                rv = np.asarray(card[at + 2 * d:at + 4 * d]).view("<u2")
                k_hat[t, h] = to_f32(rk.view(np.float16) if raw == "fp16" else rk, raw)
                v_hat[t, h] = to_f32(rv.view(np.float16) if raw == "fp16" else rv, raw)
                at += 4 * d
                continue
            if w not in (2, 4, 8):
                continue
            cb = d * w // 8
            ck = unpack_codes(card[at:at + cb], w)
            cv = unpack_codes(card[at + cb:at + 2 * cb], w)
            pk = np.asarray(card[at + 2 * cb:at + 2 * cb + 4 * ng]).view(np.float16).reshape(ng, 2)
            pv = np.asarray(card[at + 2 * cb + 4 * ng:at + 2 * cb + 8 * ng]).view(np.float16).reshape(ng, 2)
            k_hat[t, h] = dequantize_groups(ck, pk[:, 0], pk[:, 1])
            v_hat[t, h] = dequantize_groups(cv, pv[:, 0], pv[:, 1])
            at += card_record_bytes(d, w)
        if w in (2, 4, 8) and hd["k_rotated"]:
            k_hat[t] = rotate_f32(k_hat[t:t + 1])[0]
    return k_hat, v_hat
