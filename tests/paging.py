"""Test helper: lay dense per-request K/V (float64) out as a paged cache.

Used only to build oracle inputs by hand; it performs no attention arithmetic."""
import numpy as np

PAGE = 16


def paged(dense_k, dense_v, num_kv_heads, rng=None, fill_k=30.0, fill_v=-30.0):
    """dense_k / dense_v: list over requests of float64 [L_r, Hkv, d].

    Returns (k_pool, v_pool, block_table, kv_lens) with request i in block-table row i.
    Blocks are assigned in a random order when rng is given, else in order."""
    pages = [(k.shape[0] + PAGE - 1) // PAGE for k in dense_k]
    n = sum(pages) + 1
    d = dense_k[0].shape[-1]
    order = np.arange(n) if rng is None else rng.permutation(n)
    kp = np.full((n, num_kv_heads, PAGE, d), fill_k)
    vp = np.full((n, num_kv_heads, PAGE, d), fill_v)
    bt = np.full((len(dense_k), max(1, max(pages))), order[-1], dtype=np.int32)
    off = 0
    for r, (k, v) in enumerate(zip(dense_k, dense_v)):
        for p in range(pages[r]):
            blk = order[off]
            off += 1
            bt[r, p] = blk
            seg = slice(p * PAGE, min((p + 1) * PAGE, k.shape[0]))
            m = seg.stop - seg.start
            kp[blk, :, :m] = np.transpose(k[seg], (1, 0, 2))
            vp[blk, :, :m] = np.transpose(v[seg], (1, 0, 2))
    lens = np.asarray([k.shape[0] for k in dense_k], dtype=np.int32)
    return kp, vp, bt, lens
