"""Shared test helpers: move seeded inputs to the oracle, compare pools."""
import math

import numpy as np
import torch

from oracle import q4kv_oracle as O

DT = {torch.float16: "fp16", torch.bfloat16: "bf16"}

# Decode-attention tolerance: the oracle is fp64 attention over the same
# dequantised cache; pass iff max|a - b| <= 2e-3 and ||a - b|| / ||b|| <= 1e-2.
ATOL = 2e-3
RTOL_L2 = 1e-2


def host(t: torch.Tensor):
    """(numpy array, dtype name) of an fp16/bf16 tensor, bit-exact."""
    t = t.detach().cpu()
    if t.dtype == torch.float16:
        return t.numpy(), "fp16"
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16), "bf16"
    raise TypeError(t.dtype)


def oracle_pool(k: torch.Tensor, v: torch.Tensor, ids, n_q4: int, n_q8: int = 0,
                rotated: bool = True, n_q2: int = 0) -> O.OraclePool:
    kh, dt = host(k)
    vh, _ = host(v)
    pool = O.OraclePool(k.shape[1], k.shape[2], n_q4, n_q8, k_rotated=rotated, n_q2=n_q2)
    pool.quantize_blocks(kh, vh, dt, [int(i) for i in ids])
    return pool


def assert_pool_equal(gpu, ref: O.OraclePool, blocks=None):
    """Codes, scale/zero bits and remap mask bit-identical for `blocks` (an
    FP8 pool has E4M3 codes and the mask only)."""
    blocks = range(ref.n_blocks) if blocks is None else blocks
    for blk in blocks:
        blk = int(blk)
        if ref.fp8:
            for name in "kv":
                np.testing.assert_array_equal(getattr(gpu, f"{name}_codes8")[blk].cpu().numpy(),
                                              ref.codes8[name][blk], err_msg=f"{name} E4M3 codes, block {blk}")
            continue
        for name in "kv":
            if blk < ref.n_q4:
                g_codes = getattr(gpu, f"{name}_codes4")[blk].cpu().numpy()
                g_par = getattr(gpu, f"{name}_params4")[blk].cpu().numpy()
                r_codes = ref.codes4[name][blk]
                r_par = ref.params4[name][blk]
            elif blk >= ref.n_q4 + ref.n_q8:
                i = blk - ref.n_q4 - ref.n_q8
                g_codes = getattr(gpu, f"{name}_codes2")[i].cpu().numpy()
                g_par = getattr(gpu, f"{name}_params2")[i].cpu().numpy()
                r_codes = ref.codes2[name][i]
                r_par = ref.params2[name][i]
            else:
                i = blk - ref.n_q4
                g_codes = getattr(gpu, f"{name}_codes8")[i].cpu().numpy()
                g_par = getattr(gpu, f"{name}_params8")[i].cpu().numpy()
                r_codes = ref.codes8[name][i]
                r_par = ref.params8[name][i]
            np.testing.assert_array_equal(g_codes, r_codes, err_msg=f"{name} codes, block {blk}")
            np.testing.assert_array_equal(g_par.view(np.uint16), r_par.view(np.uint16),
                                          err_msg=f"{name} scale/zero bits, block {blk}")
    gm = gpu.mask.cpu().numpy().view(np.uint32)
    for blk in blocks:
        np.testing.assert_array_equal(gm[int(blk)], ref.mask[int(blk)], err_msg=f"mask {blk}")


def assert_close(gpu_out: torch.Tensor, ref: np.ndarray, atol=ATOL, rtol_l2=RTOL_L2, what=""):
    a = gpu_out.detach().float().cpu().numpy().astype(np.float64)
    b = np.asarray(ref, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    assert np.all(np.isfinite(a)), f"{what}: non-finite output"
    err = np.abs(a - b)
    mx = float(err.max()) if err.size else 0.0
    nb = float(np.linalg.norm(b))
    rel = float(np.linalg.norm(a - b)) / nb if nb > 0 else float(np.linalg.norm(a - b))
    assert mx <= atol, f"{what}: max abs error {mx:.3e} > {atol}"
    assert rel <= rtol_l2 or nb == 0 and mx <= atol, f"{what}: relative L2 error {rel:.3e} > {rtol_l2}"
    return mx, rel


def seq_tables(batch, blocks_per_seq, n_pool, seed):
    """Distinct random physical blocks per sequence (int32 [B][nb])."""
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n_pool, generator=g)[: batch * blocks_per_seq]
    return perm.view(batch, blocks_per_seq).to(torch.int32)


def scatter_tokens_to_ids(tables, seq_lens):
    """Chunk -> block id list for tokens laid out sequence after sequence."""
    ids = []
    for b, n in enumerate(seq_lens):
        nb = -(-int(n) // 256)
        ids.extend(int(x) for x in tables[b, :nb])
    return ids


def cuda():
    return torch.device("cuda", 0)


def nblocks(n):
    return -(-n // 256)


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def sqrt(x):
    return math.sqrt(x)
