"""B200 (sm_100a) 4-bit paged KV cache and decode attention.

Python face of libq4kv.so (include/q4kv.h).  Every function here only checks
and marshals arguments -- device pointers, sizes and the current CUDA stream
-- and calls the C ABI; all computation runs in the library's CUDA kernels.
torch supplies device memory and streams.  There is no CPU path: without a
CUDA device and the library, these calls raise.

Format and method, by source page:
  * 256-token blocks, 4-bit codes with a 16-bit scale and bias per group,
    attention straight from the packed cache: "Agent Memory Below the
    Prompt" (gist.science summary of arXiv 2603.04428), sec. 2.1 items 1-3.
  * Walsh-Hadamard rotation of K, V unrotated: UltraQuant news item
    (arXiv 2606.20474), "技術/ビジネス面".
  * Evicted slots remapped to a zero-weight sentinel: IntentKV article
    (Qiita), "詰め直さずに「無効化」する".
  * Wider codes for some blocks, dequantisation for hand-off: QKVShare
    (gist.science summary of arXiv 2605.03884), "Méthodologie".
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import torch

from . import _lib
from ._lib import Q4KVError, check, lib

BLOCK_TOKENS = 256
GROUP = 64

_IN_DTYPES = {torch.float16: _lib.F16, torch.bfloat16: _lib.BF16}
_OUT_DTYPES = {torch.float32: _lib.F32, torch.float16: _lib.F16, torch.bfloat16: _lib.BF16}


def _stream(device: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _require_cuda(*ts: torch.Tensor) -> torch.device:
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("q4kv works on CUDA tensors only")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("all tensors must be on one device")
    return dev


class Q4KVPool:
    """Device storage of the paged cache plus its C descriptor.

    Unified block ids [0, n_q4_blocks) are 4-bit, [n_q4_blocks,
    n_q4_blocks + n_q8_blocks) are 8-bit, the next n_q2_blocks ids 2-bit.
    Tensors (row-major):
      k_codes4/v_codes4   uint8 [n_q4][Hkv][256][D/2]
      k_params4/v_params4 fp16  [n_q4][Hkv][256][D/64][2]   (scale, zero)
      k_codes8/v_codes8   uint8 [n_q8][Hkv][256][D]
      k_params8/v_params8 fp16  [n_q8][Hkv][256][D/64][2]
      k_codes2/v_codes2   uint8 [n_q2][Hkv][256][D/4]
      k_params2/v_params2 fp16  [n_q2][Hkv][256][D/64][2]
      mask                int32 [n_q4+n_q8+n_q2][8] (bit set = slot remapped)
      error_word          int32 [4] (word 0 holds device error bits)
    """

    def __init__(self, n_kv_heads: int, head_dim: int, n_q4_blocks: int, n_q8_blocks: int = 0,
                 k_rotated: bool = True, device="cuda", fp8: bool = False, n_q2_blocks: int = 0):
        self.device = torch.device(device)
        if self.device.type != "cuda":
            raise ValueError("Q4KVPool lives on a CUDA device")
        if fp8 and (n_q4_blocks or n_q2_blocks or k_rotated):
            raise ValueError("an FP8 pool has only 8-bit blocks (n_q4_blocks = n_q2_blocks = 0) and raw keys "
                             "(k_rotated = False)")
        self.fp8 = bool(fp8)
        self.n_kv_heads, self.head_dim = n_kv_heads, head_dim
        self.n_q4_blocks, self.n_q8_blocks, self.n_q2_blocks = n_q4_blocks, n_q8_blocks, n_q2_blocks
        self.k_rotated = bool(k_rotated)
        ng = head_dim // GROUP
        T = BLOCK_TOKENS

        def codes(n, width):
            return torch.zeros((n, n_kv_heads, T, width), dtype=torch.uint8, device=self.device)

        def params(n):
            return torch.zeros((n, n_kv_heads, T, ng, 2), dtype=torch.float16, device=self.device)

        self.k_codes4, self.v_codes4 = codes(n_q4_blocks, head_dim // 2), codes(n_q4_blocks, head_dim // 2)
        self.k_params4, self.v_params4 = params(n_q4_blocks), params(n_q4_blocks)
        self.k_codes8, self.v_codes8 = codes(n_q8_blocks, head_dim), codes(n_q8_blocks, head_dim)
        n_par8 = 0 if self.fp8 else n_q8_blocks                 # FP8 blocks carry no params
        self.k_params8, self.v_params8 = params(n_par8), params(n_par8)
        self.k_codes2, self.v_codes2 = codes(n_q2_blocks, head_dim // 4), codes(n_q2_blocks, head_dim // 4)
        self.k_params2, self.v_params2 = params(n_q2_blocks), params(n_q2_blocks)
        self.mask = torch.zeros((n_q4_blocks + n_q8_blocks + n_q2_blocks, 8), dtype=torch.int32,
                                device=self.device)
        self.error_word = torch.zeros(4, dtype=torch.int32, device=self.device)
        self.desc = _lib.PoolDesc(
            head_dim, n_kv_heads, int(self.k_rotated), n_q4_blocks, n_q8_blocks, int(self.fp8),
            self.k_codes4.data_ptr(), self.v_codes4.data_ptr(),
            self.k_params4.data_ptr(), self.v_params4.data_ptr(),
            self.k_codes8.data_ptr() if n_q8_blocks else 0,
            self.v_codes8.data_ptr() if n_q8_blocks else 0,
            self.k_params8.data_ptr() if n_q8_blocks else 0,
            self.v_params8.data_ptr() if n_q8_blocks else 0,
            self.mask.data_ptr(), self.error_word.data_ptr(),
            n_q2_blocks, 0,
            self.k_codes2.data_ptr() if n_q2_blocks else 0,
            self.v_codes2.data_ptr() if n_q2_blocks else 0,
            self.k_params2.data_ptr() if n_q2_blocks else 0,
            self.v_params2.data_ptr() if n_q2_blocks else 0)

    @property
    def n_blocks(self) -> int:
        return self.n_q4_blocks + self.n_q8_blocks + self.n_q2_blocks

    def nbytes(self) -> int:
        ts = (self.k_codes4, self.v_codes4, self.k_params4, self.v_params4, self.k_codes8,
              self.v_codes8, self.k_params8, self.v_params8, self.k_codes2, self.v_codes2,
              self.k_params2, self.v_params2, self.mask)
        return sum(t.numel() * t.element_size() for t in ts)

    # -- writes -------------------------------------------------------------
    def quantize(self, k: torch.Tensor, v: torch.Tensor, block_ids: torch.Tensor) -> None:
        """Encode K/V [n_tokens][Hkv][D] (fp16/bf16; the token axis may be strided)."""
        dev = _require_cuda(k, v, block_ids)
        if k.dtype != v.dtype or k.dtype not in _IN_DTYPES:
            raise ValueError("k and v must share dtype float16 or bfloat16")
        if k.shape != v.shape or k.dim() != 3 or k.stride() != v.stride():
            raise ValueError("k and v must be [n_tokens][Hkv][D] with equal strides")
        if k.stride(2) != 1 or k.stride(1) != k.shape[2]:
            raise ValueError("each token's [Hkv][D] row must be contiguous")
        ids = block_ids.to(torch.int32).contiguous()
        check(lib().q4kv_quantize_blocks(ctypes.byref(self.desc), _ptr(k), _ptr(v), _IN_DTYPES[k.dtype],
                                         k.shape[0], k.stride(0), _ptr(ids), _stream(dev)),
              "q4kv_quantize_blocks")

    def append(self, k: torch.Tensor, v: torch.Tensor, tables: torch.Tensor, seq_lens: torch.Tensor,
               n_new: Optional[torch.Tensor] = None) -> None:
        """Write new tokens k/v [B][T][Hkv][D] at each sequence's position.

        Token i < n_new[b] (all T when n_new is None) of sequence b goes to
        position seq_lens[b] + i through the block table tables [B][max_blocks];
        seq_lens holds the lengths before the append and is not modified.
        """
        dev = _require_cuda(k, v, tables, seq_lens)
        if k.dtype != v.dtype or k.dtype not in _IN_DTYPES:
            raise ValueError("k and v must share dtype float16 or bfloat16")
        if k.shape != v.shape or k.dim() != 4 or k.stride() != v.stride():
            raise ValueError("k and v must be [B][T][Hkv][D] with equal strides")
        if k.stride(3) != 1 or k.stride(2) != k.shape[3]:
            raise ValueError("each token's [Hkv][D] row must be contiguous")
        if tables.dim() != 2 or tables.shape[0] != k.shape[0] or seq_lens.shape != (k.shape[0],):
            raise ValueError("tables must be [B][max_blocks] and seq_lens [B]")
        tab = tables.to(torch.int32).contiguous()
        lens = seq_lens.to(torch.int32).contiguous()
        nn = None
        if n_new is not None:
            if n_new.shape != (k.shape[0],):
                raise ValueError("n_new must be [B]")
            _require_cuda(n_new)
            nn = n_new.to(torch.int32).contiguous()
        check(lib().q4kv_append_tokens(ctypes.byref(self.desc), _ptr(k), _ptr(v), _IN_DTYPES[k.dtype],
                                       k.shape[0], k.shape[1], _ptr(nn) if nn is not None else None,
                                       k.stride(0), k.stride(1), _ptr(tab), tab.shape[1], _ptr(lens),
                                       _stream(dev)),
              "q4kv_append_tokens")

    def invalidate(self, slot_ids: torch.Tensor) -> None:
        """Remap physical slots (block * 256 + offset) to the sentinel."""
        dev = _require_cuda(slot_ids)
        ids = slot_ids.to(torch.int64).contiguous()
        check(lib().q4kv_invalidate_slots(ctypes.byref(self.desc), _ptr(ids), ids.numel(), _stream(dev)),
              "q4kv_invalidate_slots")

    # -- paging between device and host -------------------------------------
    def image_stride(self) -> int:
        """Bytes between consecutive block images (the largest block class)."""
        out = ctypes.c_size_t(0)
        check(lib().q4kv_block_image_stride(ctypes.byref(self.desc), ctypes.byref(out)),
              "q4kv_block_image_stride")
        return int(out.value)

    def export_blocks(self, block_ids: torch.Tensor, images: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Images of the blocks into pinned host memory, uint8 [n][stride].

        Device ids: one kernel writes the images.  Host (CPU) ids: the copy
        engines do, with no kernel.  Enqueued on the current stream; the bytes
        are complete once that stream has passed the call."""
        ids = block_ids.to(torch.int32).contiguous()
        stride = self.image_stride()
        if images is None:
            images = torch.empty((ids.numel(), stride), dtype=torch.uint8, pin_memory=True)
        _check_images(images, ids.numel(), stride)
        if ids.device.type == "cpu":
            check(lib().q4kv_export_blocks_host_ids(ctypes.byref(self.desc), _ptr(ids), ids.numel(),
                                                    ctypes.c_void_p(images.data_ptr()), _stream(self.device)),
                  "q4kv_export_blocks_host_ids")
            return images
        dev = _require_cuda(ids)
        check(lib().q4kv_export_blocks(ctypes.byref(self.desc), _ptr(ids), ids.numel(),
                                       ctypes.c_void_p(images.data_ptr()), _stream(dev)),
              "q4kv_export_blocks")
        return images

    def import_blocks(self, images: torch.Tensor, block_ids: torch.Tensor) -> None:
        """Load pinned host images (uint8 [n][stride]) into blocks block_ids[i].

        Device ids: one kernel, headers checked on the device.  Host (CPU)
        ids: the copy engines, headers checked here first.  Enqueued on the
        current stream; `images` must stay unchanged until that stream has
        passed the call."""
        ids = block_ids.to(torch.int32).contiguous()
        _check_images(images, ids.numel(), self.image_stride())
        if ids.device.type == "cpu":
            check(lib().q4kv_import_blocks_host_ids(ctypes.byref(self.desc), ctypes.c_void_p(images.data_ptr()),
                                                    _ptr(ids), ids.numel(), _stream(self.device)),
                  "q4kv_import_blocks_host_ids")
            return
        dev = _require_cuda(ids)
        check(lib().q4kv_import_blocks(ctypes.byref(self.desc), ctypes.c_void_p(images.data_ptr()),
                                       _ptr(ids), ids.numel(), _stream(dev)),
              "q4kv_import_blocks")

    # -- reads --------------------------------------------------------------
    def dequantize(self, block_ids: torch.Tensor, out_dtype=torch.float32,
                   unrotate_k: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
        """K_hat, V_hat [n][Hkv][256][D]; remapped slots read K = -1e4, V = 0."""
        dev = _require_cuda(block_ids)
        ids = block_ids.to(torch.int32).contiguous()
        shape = (ids.numel(), self.n_kv_heads, BLOCK_TOKENS, self.head_dim)
        k = torch.empty(shape, dtype=out_dtype, device=dev)
        v = torch.empty(shape, dtype=out_dtype, device=dev)
        check(lib().q4kv_dequantize(ctypes.byref(self.desc), _ptr(ids), ids.numel(), _ptr(k), _ptr(v),
                                    _OUT_DTYPES[out_dtype], int(unrotate_k), _stream(dev)),
              "q4kv_dequantize")
        return k, v

    def read_device_error(self, clear: bool = True) -> int:
        """Synchronise the current stream and return the device error bits."""
        bits = ctypes.c_uint32(0)
        st = lib().q4kv_read_device_error(ctypes.byref(self.desc), ctypes.byref(bits), int(clear),
                                          _stream(self.device))
        if st not in (_lib.OK, _lib.ERR_DEVICE):
            check(st, "q4kv_read_device_error")
        return int(bits.value)


def card_max_bytes(head_dim: int, n_kv_heads: int, n_tokens: int) -> int:
    out = ctypes.c_size_t(0)
    check(lib().q4kv_card_max_bytes(head_dim, n_kv_heads, n_tokens, ctypes.byref(out)), "q4kv_card_max_bytes")
    return int(out.value)


def card_encode(k: torch.Tensor, v: torch.Tensor, widths: torch.Tensor, k_rotated: bool = True,
                error_word: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Card (device uint8) of K/V [n][Hkv][D] at per-token widths {2, 4, 8, 16}.

    `out` (device uint8, at least card_max_bytes) is reused when given; the
    card's own size is in its header (payload bytes) and its offset table."""
    dev = _require_cuda(k, v, widths)
    if k.dtype != v.dtype or k.dtype not in _IN_DTYPES or k.shape != v.shape or k.dim() != 3:
        raise ValueError("k and v must be [n][Hkv][D] of one dtype, float16 or bfloat16")
    if k.stride() != v.stride() or k.stride(2) != 1 or k.stride(1) != k.shape[2]:
        raise ValueError("each token's [Hkv][D] row must be contiguous, with equal strides for k and v")
    n, hkv, d = k.shape
    w = widths.to(torch.uint8).contiguous()
    need = card_max_bytes(d, hkv, n)
    if out is None:
        card = torch.empty(need, dtype=torch.uint8, device=dev)
    elif out.dtype != torch.uint8 or not out.is_contiguous() or out.numel() < need or out.device != dev:
        raise ValueError(f"out must be contiguous uint8 on {dev} with at least {need} bytes")
    else:
        card = out
    check(lib().q4kv_card_encode(d, hkv, int(k_rotated), _ptr(k), _ptr(v), _IN_DTYPES[k.dtype], n, k.stride(0),
                                 _ptr(w), _ptr(card), card.numel(), _ptr(error_word), _stream(dev)),
          "q4kv_card_encode")
    return card


def card_decode(card: torch.Tensor, n_tokens: int, n_kv_heads: int, head_dim: int, out_dtype=torch.float32,
                error_word: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """K_hat, V_hat [n][Hkv][D] rebuilt from a card."""
    dev = _require_cuda(card)
    shape = (n_tokens, n_kv_heads, head_dim)
    k = torch.empty(shape, dtype=out_dtype, device=dev)
    v = torch.empty(shape, dtype=out_dtype, device=dev)
    check(lib().q4kv_card_decode(_ptr(card), card.numel(), head_dim, n_kv_heads, n_tokens, _ptr(k), _ptr(v),
                                 _OUT_DTYPES[out_dtype], _ptr(error_word), _stream(dev)),
          "q4kv_card_decode")
    return k, v


def _check_images(images: torch.Tensor, n: int, stride: int) -> None:
    if images.device.type != "cpu" or not images.is_pinned():
        raise ValueError("block images live in pinned host memory")
    if images.dtype != torch.uint8 or not images.is_contiguous() or images.numel() < n * stride:
        raise ValueError(f"block images must be contiguous uint8 of at least {n} x {stride} bytes")


def block_absmean(k: torch.Tensor) -> torch.Tensor:
    """fp64 mean |K| per 256-token chunk of raw keys [n_tokens][Hkv][D]."""
    dev = _require_cuda(k)
    if k.dtype not in _IN_DTYPES or k.dim() != 3 or k.stride(2) != 1 or k.stride(1) != k.shape[2]:
        raise ValueError("k must be fp16/bf16 [n_tokens][Hkv][D] with contiguous rows")
    n = k.shape[0]
    out = torch.empty((n + BLOCK_TOKENS - 1) // BLOCK_TOKENS, dtype=torch.float64, device=dev)
    check(lib().q4kv_block_absmean(_ptr(k), _IN_DTYPES[k.dtype], n, k.stride(0), k.shape[1], k.shape[2],
                                   _ptr(out), _stream(dev)), "q4kv_block_absmean")
    return out


def mixed_block_ids(absmean: torch.Tensor, n_q8: int, q4_first: int = 0,
                    q8_first: Optional[int] = None) -> torch.Tensor:
    """Block id per chunk; the n_q8 chunks with the largest absmean get 8-bit ids."""
    dev = _require_cuda(absmean)
    a = absmean.to(torch.float64).contiguous()
    n = a.numel()
    if q8_first is None:
        q8_first = n - n_q8
    ids = torch.empty(n, dtype=torch.int32, device=dev)
    check(lib().q4kv_mixed_block_ids(_ptr(a), n, n_q8, q4_first, q8_first, _ptr(ids), _stream(dev)),
          "q4kv_mixed_block_ids")
    return ids


class DecodePlan:
    """Launch plan for one decode shape (split count, workspace size)."""

    def __init__(self, batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                 max_blocks_per_seq: int, n_splits: int = 0, num_sms: int = 0):
        self.c = _lib.DecodePlan()
        check(lib().q4kv_decode_plan_make(batch, n_q_heads, n_kv_heads, head_dim, max_blocks_per_seq,
                                          n_splits, num_sms, ctypes.byref(self.c)),
              "q4kv_decode_plan_make")

    def __getattr__(self, name):
        return getattr(self.__dict__["c"], name)

    def workspace(self, device) -> Optional[torch.Tensor]:
        n = self.c.workspace_bytes
        return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def decode_attention(pool: Q4KVPool, q: torch.Tensor, block_tables: torch.Tensor,
                     seq_lens: torch.Tensor, softmax_scale: float = 0.0, out_dtype=torch.float16,
                     plan: Optional[DecodePlan] = None, workspace: Optional[torch.Tensor] = None,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Single-token GQA attention of q [B][Hq][D] over the paged cache."""
    dev = _require_cuda(q, block_tables, seq_lens)
    if q.dtype not in _IN_DTYPES or q.dim() != 3 or not q.is_contiguous():
        raise ValueError("q must be contiguous fp16/bf16 [B][Hq][D]")
    tables = block_tables.to(torch.int32).contiguous()
    lens = seq_lens.to(torch.int32).contiguous()
    B, hq, d = q.shape
    if plan is None:
        plan = DecodePlan(B, hq, pool.n_kv_heads, d, tables.shape[1])
    if workspace is None:
        workspace = plan.workspace(dev)
    if out is None:
        out = torch.empty((B, hq, d), dtype=out_dtype, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib().q4kv_decode_attention(ctypes.byref(pool.desc), ctypes.byref(plan.c), _ptr(q),
                                      _IN_DTYPES[q.dtype], _ptr(tables), _ptr(lens),
                                      float(softmax_scale), _ptr(out), _OUT_DTYPES[out.dtype],
                                      _ptr(workspace), ws_bytes, _stream(dev)),
          "q4kv_decode_attention")
    return out


def append_decode(pool: Q4KVPool, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor,
                  block_tables: torch.Tensor, seq_lens: torch.Tensor, n_new: Optional[torch.Tensor] = None,
                  softmax_scale: float = 0.0, out_dtype=torch.float16, plan: Optional[DecodePlan] = None,
                  workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One generation step: append k_new/v_new [B][T][Hkv][D] at each
    sequence's position seq_lens[b] (lengths before the append, not
    modified), then decode q [B][Hq][D] over seq_lens[b] + n_new[b] tokens
    (+ T when n_new is None).  Same result as pool.append then
    decode_attention with the grown lengths, in one decode launch that
    encodes the new rows itself (FP8 pools and plan kernel 0: the append
    kernel, then a decode that overlaps it)."""
    dev = _require_cuda(k_new, v_new, q, block_tables, seq_lens)
    if k_new.dtype != v_new.dtype or k_new.dtype not in _IN_DTYPES:
        raise ValueError("k_new and v_new must share dtype float16 or bfloat16")
    if k_new.shape != v_new.shape or k_new.dim() != 4 or k_new.stride() != v_new.stride():
        raise ValueError("k_new and v_new must be [B][T][Hkv][D] with equal strides")
    if k_new.stride(3) != 1 or k_new.stride(2) != k_new.shape[3]:
        raise ValueError("each token's [Hkv][D] row must be contiguous")
    if q.dtype not in _IN_DTYPES or q.dim() != 3 or not q.is_contiguous():
        raise ValueError("q must be contiguous fp16/bf16 [B][Hq][D]")
    B, hq, d = q.shape
    tables = block_tables.to(torch.int32).contiguous()
    lens = seq_lens.to(torch.int32).contiguous()
    if k_new.shape[0] != B or tables.dim() != 2 or tables.shape[0] != B or lens.shape != (B,):
        raise ValueError("k_new, q, block_tables and seq_lens must share the batch")
    nn = None
    if n_new is not None:
        if n_new.shape != (B,):
            raise ValueError("n_new must be [B]")
        _require_cuda(n_new)
        nn = n_new.to(torch.int32).contiguous()
    if plan is None:
        plan = DecodePlan(B, hq, pool.n_kv_heads, d, tables.shape[1])
    if workspace is None:
        workspace = plan.workspace(dev)
    if out is None:
        out = torch.empty((B, hq, d), dtype=out_dtype, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(lib().q4kv_append_decode(ctypes.byref(pool.desc), ctypes.byref(plan.c), _ptr(k_new), _ptr(v_new),
                                   _IN_DTYPES[k_new.dtype], k_new.shape[1],
                                   _ptr(nn) if nn is not None else None, k_new.stride(0), k_new.stride(1),
                                   _ptr(q), _IN_DTYPES[q.dtype], _ptr(tables), _ptr(lens), float(softmax_scale),
                                   _ptr(out), _OUT_DTYPES[out.dtype], _ptr(workspace), ws_bytes, _stream(dev)),
          "q4kv_append_decode")
    return out


__all__ = ["Q4KVPool", "Q4KVError", "DecodePlan", "decode_attention", "append_decode", "block_absmean",
           "mixed_block_ids", "card_max_bytes", "card_encode", "card_decode", "BLOCK_TOKENS", "GROUP"]
