"""Host-only checks of the C ABI: the library loads without a GPU, exports
every function include/q4kv.h declares, sizes the pool as the format says,
makes launch plans, and rejects bad arguments before touching a device."""
import ctypes

import pytest

from decode_attention_q4kv_b200 import _lib

L = _lib.lib()
FAKE = 0x7F0000000000     # 4 KiB-aligned address never dereferenced: every call below is rejected first


def _pool(**kw):
    d = dict(head_dim=128, n_kv_heads=8, k_rotated=1, n_q4_blocks=4, n_q8_blocks=0, value_format=0,
             k_codes4=FAKE, v_codes4=FAKE, k_params4=FAKE, v_params4=FAKE,
             k_codes8=0, v_codes8=0, k_params8=0, v_params8=0, remap_mask=FAKE, error_word=0)
    d.update(kw)
    p = _lib.PoolDesc()
    for k, v in d.items():
        setattr(p, k, v)
    return p


def test_exports_every_declared_function():
    names = _lib.header_functions()
    assert len(names) == 23
    for n in names:
        assert hasattr(L, n), n
    # the binding declares a signature for each of them
    assert set(names) == set(_lib._SIGNATURES)


def test_abi_version_and_status_strings():
    assert L.q4kv_abi_version() == 4
    assert L.q4kv_status_string(0) == b"ok"
    assert b"workspace" in L.q4kv_status_string(_lib.ERR_WORKSPACE)
    assert L.q4kv_status_string(99) == b"unknown status"


def test_struct_layouts():
    assert ctypes.sizeof(_lib.PoolDesc) == 24 + 10 * 8 + 8 + 4 * 8
    assert _lib.PoolDesc.k_codes4.offset == 24
    assert _lib.PoolDesc.n_q2_blocks.offset == 24 + 10 * 8
    assert _lib.PoolDesc.k_codes2.offset == 24 + 10 * 8 + 8
    assert ctypes.sizeof(_lib.DecodePlan) == 40


def test_pool_array_bytes_give_144_bytes_per_token_head():
    cb, pb = ctypes.c_size_t(), ctypes.c_size_t()
    assert L.q4kv_pool_array_bytes(128, 1, 1, 4, ctypes.byref(cb), ctypes.byref(pb)) == 0
    assert (cb.value, pb.value) == (256 * 64, 256 * 2 * 4)
    per_token_head = 2 * (cb.value + pb.value) / 256
    assert per_token_head == 144
    assert L.q4kv_pool_array_bytes(128, 1, 1, 8, ctypes.byref(cb), ctypes.byref(pb)) == 0
    assert 2 * (cb.value + pb.value) / 256 == 272
    assert L.q4kv_pool_array_bytes(256, 1, 1, 4, ctypes.byref(cb), ctypes.byref(pb)) == 0
    assert 2 * (cb.value + pb.value) / 256 == 288
    assert L.q4kv_pool_array_bytes(96, 1, 1, 4, ctypes.byref(cb), ctypes.byref(pb)) == _lib.ERR_UNSUPPORTED
    assert L.q4kv_pool_array_bytes(128, 1, 1, 3, ctypes.byref(cb), ctypes.byref(pb)) == _lib.ERR_INVALID_ARG


def _plan(*args):
    p = _lib.DecodePlan()
    st = L.q4kv_decode_plan_make(*args, ctypes.byref(p))
    return st, p


@pytest.mark.parametrize("B,hq,hkv,d,mb", [(1, 32, 8, 128, 16), (64, 32, 8, 128, 512),
                                           (5, 16, 8, 256, 32), (32, 40, 8, 128, 64),
                                           (256, 32, 8, 128, 512), (1, 8, 8, 128, 1)])
def test_plan_covers_context(B, hq, hkv, d, mb):
    st, p = _plan(B, hq, hkv, d, mb, 0, 148)
    assert st == 0
    ctx = mb * 256
    assert p.tokens_per_split % 256 == 0 and p.kernel == 1
    assert p.n_splits * p.tokens_per_split >= ctx > (p.n_splits - 1) * p.tokens_per_split
    if p.n_splits > 1:
        assert p.workspace_bytes >= B * hq * p.n_splits * (d + 2) * 4
    else:
        assert p.workspace_bytes == 0
    # forcing the plan's own split count reproduces it
    st2, p2 = _plan(B, hq, hkv, d, mb, p.n_splits, 7)
    assert st2 == 0 and (p2.n_splits, p2.tokens_per_split, p2.workspace_bytes) == \
        (p.n_splits, p.tokens_per_split, p.workspace_bytes)


def test_plan_rejects_bad_shapes():
    assert _plan(1, 30, 8, 128, 4, 0, 148)[0] == _lib.ERR_INVALID_ARG      # Hq % Hkv != 0
    assert _plan(1, 72, 8, 128, 4, 0, 148)[0] == _lib.ERR_UNSUPPORTED      # g = 9
    assert _plan(1, 48, 8, 256, 4, 0, 148)[0] == _lib.ERR_UNSUPPORTED      # g*D/64 = 24
    assert _plan(1, 32, 8, 64, 4, 0, 148)[0] == _lib.ERR_UNSUPPORTED       # D = 64
    assert _plan(1, 32, 8, 128, 0, 0, 148)[0] == _lib.ERR_INVALID_ARG      # empty table
    assert _plan(-1, 32, 8, 128, 4, 0, 148)[0] == _lib.ERR_INVALID_ARG
    st, p = _plan(1, 32, 8, 128, 4, 100000, 148)                            # clamped to the context
    assert st == 0 and p.n_splits == 4 and p.tokens_per_split == 256 and p.kernel == 1


def test_quantize_rejects_bad_arguments_without_launching():
    p = _pool()
    q = L.q4kv_quantize_blocks
    assert q(None, FAKE, FAKE, 0, 10, 1024, FAKE, None) == _lib.ERR_INVALID_ARG
    assert q(ctypes.byref(_pool(head_dim=64)), FAKE, FAKE, 0, 10, 512, FAKE, None) == _lib.ERR_UNSUPPORTED
    assert q(ctypes.byref(p), FAKE, FAKE, 2, 10, 1024, FAKE, None) == _lib.ERR_INVALID_ARG       # fp32 input
    assert q(ctypes.byref(p), FAKE + 2, FAKE, 0, 10, 1024, FAKE, None) == _lib.ERR_INVALID_ARG   # misaligned
    assert q(ctypes.byref(p), FAKE, FAKE, 0, 10, 1000, FAKE, None) == _lib.ERR_INVALID_ARG       # stride < Hkv*D
    assert q(ctypes.byref(p), FAKE, FAKE, 0, 10, 1028, FAKE, None) == _lib.ERR_INVALID_ARG       # stride not 16 B
    assert q(ctypes.byref(p), FAKE, FAKE, 0, -1, 1024, FAKE, None) == _lib.ERR_INVALID_ARG
    assert q(ctypes.byref(p), FAKE, FAKE, 0, 10, 1024, None, None) == _lib.ERR_INVALID_ARG       # no block ids
    assert q(ctypes.byref(_pool(value_format=2)), FAKE, FAKE, 0, 10, 1024, FAKE, None) == _lib.ERR_INVALID_ARG
    assert q(ctypes.byref(_pool(k_codes4=0)), FAKE, FAKE, 0, 10, 1024, FAKE, None) == _lib.ERR_INVALID_ARG
    assert q(ctypes.byref(_pool(n_q8_blocks=2)), FAKE, FAKE, 0, 10, 1024, FAKE, None) == _lib.ERR_INVALID_ARG
    assert q(ctypes.byref(_pool(remap_mask=FAKE + 4)), FAKE, FAKE, 0, 10, 1024, FAKE, None) == _lib.ERR_INVALID_ARG
    # zero tokens is a no-op that succeeds
    assert q(ctypes.byref(p), FAKE, FAKE, 0, 0, 1024, FAKE, None) == 0


def test_other_entry_points_reject_bad_arguments():
    p = _pool()
    assert L.q4kv_dequantize(ctypes.byref(p), FAKE, 2, FAKE, FAKE, 1, 2, None) == _lib.ERR_INVALID_ARG
    assert L.q4kv_dequantize(ctypes.byref(p), FAKE, 2, FAKE, FAKE, 1, 0, None) == _lib.ERR_INVALID_ARG  # bf16 out
    assert L.q4kv_dequantize(ctypes.byref(p), FAKE, 2, FAKE + 8, FAKE, 2, 0, None) == _lib.ERR_INVALID_ARG
    assert L.q4kv_dequantize(ctypes.byref(p), FAKE, 0, FAKE, FAKE, 2, 0, None) == 0
    assert L.q4kv_invalidate_slots(ctypes.byref(p), FAKE, -1, None) == _lib.ERR_INVALID_ARG
    assert L.q4kv_invalidate_slots(ctypes.byref(p), None, 3, None) == _lib.ERR_INVALID_ARG
    assert L.q4kv_invalidate_slots(ctypes.byref(p), FAKE, 0, None) == 0
    assert L.q4kv_block_absmean(FAKE, 0, 10, 1000, 1, 3, FAKE, None) == _lib.ERR_INVALID_ARG
    assert L.q4kv_block_absmean(FAKE, 0, 10, 1028, 8, 128, FAKE, None) == _lib.ERR_INVALID_ARG
    assert L.q4kv_block_absmean(FAKE, 0, 0, 1024, 8, 128, FAKE, None) == 0
    assert L.q4kv_mixed_block_ids(FAKE, 70000, 1, 0, 0, FAKE, None) == _lib.ERR_INVALID_ARG
    assert L.q4kv_mixed_block_ids(FAKE, 10, 11, 0, 0, FAKE, None) == _lib.ERR_INVALID_ARG
    assert L.q4kv_mixed_block_ids(FAKE, 0, 0, 0, 0, FAKE, None) == 0


def test_append_rejects_bad_arguments_without_launching():
    p = _pool()
    a = L.q4kv_append_tokens

    def call(pool=p, k=FAKE, v=FAKE, dt=0, b=2, t=3, nn=None, ss=3 * 1024, ts=1024, tab=FAKE, mb=4, lens=FAKE):
        return a(ctypes.byref(pool), k, v, dt, b, t, nn, ss, ts, tab, mb, lens, None)

    assert call(dt=2) == _lib.ERR_INVALID_ARG                 # fp32 input
    assert call(b=-1) == _lib.ERR_INVALID_ARG
    assert call(t=-1) == _lib.ERR_INVALID_ARG
    assert call(k=FAKE + 8) == _lib.ERR_INVALID_ARG           # misaligned rows
    assert call(ts=1020) == _lib.ERR_INVALID_ARG              # token stride below Hkv*D
    assert call(ts=1028) == _lib.ERR_INVALID_ARG              # token stride not a 16-byte multiple
    assert call(ss=3 * 1024 + 4) == _lib.ERR_INVALID_ARG      # sequence stride not a 16-byte multiple
    assert call(tab=None) == _lib.ERR_INVALID_ARG
    assert call(lens=None) == _lib.ERR_INVALID_ARG
    assert call(mb=0) == _lib.ERR_INVALID_ARG
    assert call(nn=FAKE + 2) == _lib.ERR_INVALID_ARG
    assert call(pool=_pool(head_dim=96)) != 0
    assert call(b=0) == 0 and call(t=0) == 0                  # nothing to append: no launch


def test_decode_rejects_bad_arguments_without_launching():
    p = _pool()
    st, plan = _plan(2, 32, 8, 128, 4, 4, 148)
    assert st == 0 and plan.workspace_bytes > 0
    d = L.q4kv_decode_attention
    args = lambda **kw: dict(dict(q=FAKE, qd=0, tab=FAKE, lens=FAKE, scale=0.0, out=FAKE, od=1,
                                  ws=FAKE, wsb=plan.workspace_bytes), **kw)

    def call(pool=p, pl=plan, **kw):
        a = args(**kw)
        return d(ctypes.byref(pool), ctypes.byref(pl), a["q"], a["qd"], a["tab"], a["lens"], a["scale"],
                 a["out"], a["od"], a["ws"], a["wsb"], None)

    assert call(ws=0) == _lib.ERR_WORKSPACE
    assert call(wsb=plan.workspace_bytes - 1) == _lib.ERR_WORKSPACE
    assert call(ws=FAKE + 16) == _lib.ERR_WORKSPACE
    assert call(qd=2) == _lib.ERR_INVALID_ARG
    assert call(od=7) == _lib.ERR_INVALID_ARG
    assert call(q=FAKE + 2) == _lib.ERR_INVALID_ARG
    assert call(scale=float("nan")) == _lib.ERR_INVALID_ARG
    assert call(pool=_pool(n_kv_heads=4)) == _lib.ERR_INVALID_ARG       # plan and pool disagree
    bad = _lib.DecodePlan.from_buffer_copy(plan)
    bad.tokens_per_split += 64
    assert call(pl=bad) == _lib.ERR_INVALID_ARG                          # not a plan the library made
    for k in (2, -1):                                                    # only variants 0 and 1 exist
        bad = _lib.DecodePlan.from_buffer_copy(plan)
        bad.kernel = k
        assert call(pl=bad) == _lib.ERR_INVALID_ARG
    st, empty = _plan(0, 32, 8, 128, 4, 0, 148)
    assert st == 0
    assert call(pl=empty, ws=0, wsb=0) == 0                              # batch 0: nothing to do


def test_append_decode_rejects_bad_arguments_without_launching():
    """The fused generation step validates both the append and the decode
    arguments before it launches anything (a fake pointer would fault)."""
    p = _pool()
    st, plan = _plan(2, 32, 8, 128, 4, 4, 148)
    assert st == 0
    f = L.q4kv_append_decode

    def call(pool=p, pl=plan, k=FAKE, dt=0, t=3, nn=None, ss=3 * 1024, ts=1024, q=FAKE, qd=0, tab=FAKE,
             lens=FAKE, scale=0.0, out=FAKE, od=1, ws=FAKE, wsb=None):
        wsb = (pl.workspace_bytes if pl is not None else 0) if wsb is None else wsb
        return f(ctypes.byref(pool), None if pl is None else ctypes.byref(pl), k, k, dt, t, nn, ss, ts, q, qd,
                 tab, lens, scale, out, od, ws, wsb, None)

    assert call(pl=None) == _lib.ERR_INVALID_ARG
    assert call(dt=2) == _lib.ERR_INVALID_ARG                  # append: fp32 input
    assert call(k=FAKE + 8) == _lib.ERR_INVALID_ARG            # append: misaligned rows
    assert call(ts=1020) == _lib.ERR_INVALID_ARG               # append: token stride below Hkv*D
    assert call(t=-1) == _lib.ERR_INVALID_ARG
    assert call(nn=FAKE + 2) == _lib.ERR_INVALID_ARG
    assert call(lens=None) == _lib.ERR_INVALID_ARG
    assert call(qd=2) == _lib.ERR_INVALID_ARG                  # decode: bad query dtype
    assert call(out=FAKE + 4) == _lib.ERR_INVALID_ARG          # decode: misaligned output
    assert call(ws=0) == _lib.ERR_WORKSPACE                    # decode: missing workspace
    assert call(pool=_pool(n_kv_heads=4)) == _lib.ERR_INVALID_ARG
    bad = _lib.DecodePlan.from_buffer_copy(plan)
    bad.kernel = 3
    assert call(pl=bad) == _lib.ERR_INVALID_ARG
    st, empty = _plan(0, 32, 8, 128, 4, 0, 148)
    assert st == 0 and call(pl=empty, ws=0, wsb=0) == 0        # batch 0: nothing to do


def test_selftest_rejects_bad_arguments():
    assert L.q4kv_selftest_bounded_wait(None, 10, None) == _lib.ERR_INVALID_ARG
    assert L.q4kv_selftest_bounded_wait(FAKE + 2, 10, None) == _lib.ERR_INVALID_ARG
    assert L.q4kv_selftest_bounded_wait(FAKE, 0, None) == _lib.ERR_INVALID_ARG
    assert L.q4kv_selftest_bounded_wait(FAKE, (1 << 21) + 1, None) == _lib.ERR_INVALID_ARG


def test_read_device_error_without_word():
    p = _pool()
    bits = ctypes.c_uint32(123)
    assert L.q4kv_read_device_error(ctypes.byref(p), ctypes.byref(bits), 1, None) == 0
    assert bits.value == 0
    assert L.q4kv_read_device_error(None, ctypes.byref(bits), 1, None) == _lib.ERR_INVALID_ARG


def _stride(pool):
    out = ctypes.c_size_t(0)
    st = L.q4kv_block_image_stride(ctypes.byref(pool), ctypes.byref(out))
    return st, out.value


@pytest.mark.parametrize("d,hkv,n_q8,fp8", [(128, 8, 0, 0), (128, 8, 3, 0), (256, 4, 0, 0), (128, 2, 4, 1),
                                            (256, 8, 2, 0)])
def test_block_image_stride_matches_the_oracle(d, hkv, n_q8, fp8):
    from oracle import q4kv_oracle as O
    n_q4 = 0 if fp8 else 4
    kw = dict(head_dim=d, n_kv_heads=hkv, n_q4_blocks=n_q4, n_q8_blocks=n_q8, value_format=fp8,
              k_rotated=0 if fp8 else 1)
    if n_q8:
        kw.update(k_codes8=FAKE, v_codes8=FAKE, k_params8=FAKE, v_params8=FAKE)
    if fp8:
        kw.update(k_codes4=0, v_codes4=0, k_params4=0, v_params4=0, k_params8=0, v_params8=0)
    st, stride = _stride(_pool(**kw))
    assert st == 0
    ref = O.OraclePool(hkv, d, n_q4, n_q8, k_rotated=not fp8, fp8=bool(fp8))
    assert stride == ref.image_stride() and stride % 16 == 0


def test_paging_rejects_bad_arguments_without_launching():
    p = _pool()
    e, i = L.q4kv_export_blocks, L.q4kv_import_blocks
    assert _stride(_pool(head_dim=64))[0] == _lib.ERR_UNSUPPORTED
    assert L.q4kv_block_image_stride(ctypes.byref(p), None) == _lib.ERR_INVALID_ARG
    host = ctypes.create_string_buffer(1 << 16)                # pageable host memory
    addr = (ctypes.addressof(host) + 15) // 16 * 16
    eh, ih = L.q4kv_export_blocks_host_ids, L.q4kv_import_blocks_host_ids
    for call in (lambda ids, n, h: e(ctypes.byref(p), ids, n, h, None),
                 lambda ids, n, h: i(ctypes.byref(p), h, ids, n, None),
                 lambda ids, n, h: eh(ctypes.byref(p), ids, n, h, None),
                 lambda ids, n, h: ih(ctypes.byref(p), h, ids, n, None)):
        assert call(FAKE, -1, addr) == _lib.ERR_INVALID_ARG
        assert call(None, 2, addr) == _lib.ERR_INVALID_ARG
        assert call(FAKE + 2, 2, addr) == _lib.ERR_INVALID_ARG
        assert call(FAKE, 2, None) == _lib.ERR_INVALID_ARG
        assert call(FAKE, 2, addr + 8) == _lib.ERR_INVALID_ARG          # misaligned images
        assert call(FAKE, 2, addr) == _lib.ERR_INVALID_ARG              # not page-locked
        assert call(FAKE, 0, None) == 0                                 # nothing to move


@pytest.mark.parametrize("d,hkv,n", [(128, 8, 0), (128, 3, 301), (256, 2, 8195)])
def test_card_max_bytes_is_the_all_fp16_card(d, hkv, n):
    from oracle import q4kv_oracle as O
    out = ctypes.c_size_t(0)
    assert L.q4kv_card_max_bytes(d, hkv, n, ctypes.byref(out)) == 0
    assert out.value == O.card_layout(d, hkv, [16] * n)[4]


def test_card_calls_reject_bad_arguments_without_launching():
    out = ctypes.c_size_t(0)
    assert L.q4kv_card_max_bytes(64, 8, 10, ctypes.byref(out)) == _lib.ERR_UNSUPPORTED
    assert L.q4kv_card_max_bytes(128, 0, 10, ctypes.byref(out)) == _lib.ERR_INVALID_ARG
    assert L.q4kv_card_max_bytes(128, 8, -1, ctypes.byref(out)) == _lib.ERR_INVALID_ARG
    L.q4kv_card_max_bytes(128, 8, 10, ctypes.byref(out))
    big = out.value
    enc = lambda **kw: L.q4kv_card_encode(*[dict(dict(d=128, h=8, rot=1, k=FAKE, v=FAKE, dt=0, n=10, ts=1024,
                                                      w=FAKE, card=FAKE, cb=big, err=None, s=None), **kw)[x]
                                            for x in ("d", "h", "rot", "k", "v", "dt", "n", "ts", "w", "card",
                                                      "cb", "err", "s")])
    assert enc(cb=big - 1) == _lib.ERR_INVALID_ARG            # card too small for the worst case
    assert enc(card=FAKE + 8) == _lib.ERR_INVALID_ARG
    assert enc(w=None) == _lib.ERR_INVALID_ARG
    assert enc(rot=2) == _lib.ERR_INVALID_ARG
    assert enc(dt=2) == _lib.ERR_INVALID_ARG
    assert enc(ts=1000) == _lib.ERR_INVALID_ARG
    assert enc(d=96) == _lib.ERR_UNSUPPORTED
    assert enc(err=FAKE + 2) == _lib.ERR_INVALID_ARG
    dec = L.q4kv_card_decode
    assert dec(FAKE, big, 128, 8, 10, FAKE, FAKE, 1, None, None) == _lib.ERR_INVALID_ARG   # bf16 output
    assert dec(FAKE, 100, 128, 8, 10, FAKE, FAKE, 2, None, None) == _lib.ERR_INVALID_ARG   # no room for tables
    assert dec(FAKE + 4, big, 128, 8, 10, FAKE, FAKE, 2, None, None) == _lib.ERR_INVALID_ARG
    assert dec(FAKE, big, 128, 8, 10, FAKE + 4, FAKE, 2, None, None) == _lib.ERR_INVALID_ARG
    assert dec(FAKE, big, 128, 8, -1, FAKE, FAKE, 2, None, None) == _lib.ERR_INVALID_ARG
    assert dec(None, 0, 128, 8, 0, None, None, 2, None, None) == 0                       # nothing to rebuild


@pytest.mark.parametrize("shape,splits", [((5, 16, 8, 256, 32), 11),      # Gemma-3-12B shape, 5 x 8192
                                          ((10, 32, 8, 128, 128), 11),    # Llama-3.1-8B, 10 x 32768
                                          ((32, 40, 8, 128, 64), 4),      # Qwen2.5-14B, 32 x 16384
                                          ((16, 32, 8, 128, 128), 8),     # sweep 16 x 32K
                                          ((64, 32, 8, 128, 16), 2),      # sweep 64 x 4K
                                          ((1, 32, 8, 128, 512), 37)])    # sweep 1 x 128K
def test_default_split_counts_follow_the_measured_item_cost(shape, splits):
    """The cost model (waves x (blocks per item + 0.9)) on the workload shapes
    for a 148-SM B200.  Its per-item constant was fitted to forced-split decode
    timings: evicted Qwen 1/4/8 splits 197/179/191 us, sweep 16 x 32K
    1/5/8/11 splits 168/173/156/169 us, Llama mixed 1/5/8/11 splits
    207/138/146/134 us, Gemma 3/11 splits 38.8-47.7/37.4 us."""
    st, p = _plan(*shape, 0, 148)
    assert st == 0 and p.n_splits == splits


@pytest.mark.parametrize("shape", [(256, 32, 8, 128, 512), (64, 32, 8, 128, 512), (16, 32, 8, 128, 512),
                                   (1, 16, 8, 256, 4096)])
def test_default_items_are_at_most_64_blocks(shape):
    """Long contexts with many sequences: the cost model alone picks one split
    for 256 x 128K (every SM already has work), but a work item is capped at 64
    blocks (16384 tokens), since the fp32 value sums of one long item lose
    accuracy (measured: 2.2e-2 relative L2 at 131072 tokens per item, 2.7e-3
    at 32768).  A forced split count stays as given."""
    st, p = _plan(*shape, 0, 148)
    assert st == 0 and p.tokens_per_split <= 64 * 256
    assert p.n_splits * p.tokens_per_split >= shape[4] * 256
    st, p1 = _plan(*shape, 1, 148)
    assert st == 0 and p1.n_splits == 1
