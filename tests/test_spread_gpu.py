"""GPU parity at large score spreads: the softmax's running-max paths.

The prefill tile keeps a stale row max and rescales O in TMEM only when a
row's max grows by more than 2^8; decode rescales its accumulators on every
page.  N(0,1) inputs at scale 1/sqrt(d) almost never move the max that far,
so these batches make it move (what attention computes: POD-Attention
explainer, "Why this problem is worth solving"):
  * scale 1.0 at d = 128: scores have a standard deviation of about 11, and
    the row max keeps growing across the key tiles;
  * a prefill chunk whose later keys (in the prior context and inside the
    chunk) have a planted large q.k, so rows that see them jump by far more
    than 2^8 in the exp2 domain;
  * a decode request whose scores rise steadily along the keys, so every page
    moves the max.
Each runs fused and sequential and is compared element by element with the
float64 oracle at the same tolerance as the other parity tests; with
POD_FLAG_TRACE the kernel counts the prefill warps that took the rescale
branch, and the test requires that count to be positive.
"""
import numpy as np
import pytest

import synth
from oracle import attention as A
from prefill_decode_b200.device_batch import DeviceBatch

MAX_ABS, MEAN_ABS = 2e-2, 2e-3
PAGE = 16


@pytest.fixture(scope="module")
def env():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from prefill_decode_b200 import build
    build.build()
    import prefill_decode_b200 as pod
    return torch, pod


def _bf16(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _set_key(b, row, j, kvh, vec_bits):
    blk = int(b.block_table[row, j // PAGE])
    b.k_pool[blk, kvh, j % PAGE, :] = vec_bits


def _planted_batch():
    """Prefill 128 rows over 1000 earlier tokens (4 q heads, 1 kv head, d=128) + 2 decodes.
    Keys 900..909 (prior context) and 1050..1059 (inside the chunk) are 16 e_0; every
    query has q[0] = 16: those keys score 256 * scale = 22.6 above ~4 for the rest."""
    w = synth.custom("planted", 4, 1, 128, 128, 1000, [700, 2000], 31)
    b = synth.make_batch(w)
    big = np.zeros(128, dtype=np.float32)
    big[0] = 16.0
    for j in list(range(900, 910)) + list(range(1050, 1060)):
        _set_key(b, 0, j, 0, _bf16(big))
    b.q_prefill[:, :, 0] = _bf16(16.0)
    return b


def _rising_decode_batch():
    """Decodes whose score rises along the keys: K[j][0] = 60 j / L, q[0] = 16 (scale 1/sqrt(128)),
    so the max grows on every page; a small prefill rides along."""
    w = synth.custom("rising", 8, 2, 128, 64, 700, [2000, 333, 4100], 32)
    b = synth.make_batch(w)
    for r, L in enumerate(b.decode_lens.tolist()):
        row = b.num_prefill + r
        for kvh in range(2):
            for j in range(L):
                blk = int(b.block_table[row, j // PAGE])
                b.k_pool[blk, kvh, j % PAGE, 0] = _bf16(60.0 * j / L).reshape(-1)[0]
    b.q_decode[:, :, 0] = _bf16(16.0)
    return b


CASES = {
    "scale1_d128": lambda: synth.make_batch(
        synth.custom("scale1", 8, 2, 128, 256, 2500, [100, 1500, 5000], 30, scale=1.0)),
    "planted_keys": _planted_batch,
    "rising_decode": _rising_decode_batch,
}


def _run_and_check(env, b, flags, expect_rescale, **plan_kw):
    torch, pod = env
    db = DeviceBatch(torch, b)
    pl = db.plan(pod, flags=flags | pod.POD_FLAG_TRACE, **plan_kw)
    ws = db.workspace(pl)
    pl.upload(ws)
    trace = torch.zeros((pl.info.num_prefill_items + pl.info.num_decode_items, 4), dtype=torch.int32,
                        device="cuda")
    db.run(pod, pl, ws, trace=trace)
    torch.cuda.synchronize()
    assert db.error_word(pl, ws) == 0
    off = pl.info.rescale_count_offset
    rescales = int(ws[off:off + 4].view(torch.int32).item())
    op, od = db.outputs()
    w = b.workload
    rp = A.attend_prefill_batched(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_qo_lens,
                                  b.prefill_kv_lens, b.scale, w.num_kv_heads)
    rd = A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, w.num_kv_heads,
                         first_row=b.num_prefill)
    for name, got, ref in (("prefill", op, rp), ("decode", od, rd)):
        err = np.abs(got - ref)
        assert np.isfinite(got).all(), f"{name}: non-finite output"
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, f"{name}: max {err.max():.3e} mean {err.mean():.3e}"
    if expect_rescale:
        assert rescales > 0, "the lazy O rescale never ran"
    return rescales


@pytest.mark.gpu
@pytest.mark.parametrize("splits", [0, 1], ids=["split_rule", "no_split"])
@pytest.mark.parametrize("flags", [0, 1], ids=["fused", "sequential"])
@pytest.mark.parametrize("case", sorted(CASES))
def test_large_score_spread(env, case, flags, splits):
    """splits = 0: the plan rule cuts the prefill items into KV pieces here (the rescale then also
    runs inside pieces and the pieces are merged); splits = 1: whole items."""
    b = CASES[case]()
    _run_and_check(env, b, flags, expect_rescale=case != "rising_decode", max_prefill_splits=splits)


def test_planted_keys_dominate():
    """Sanity of the planted batch itself (CPU oracle): rows that see the planted keys return,
    to within the far smaller weight of every other key, the mean of those keys' values."""
    b = _planted_batch()
    w = b.workload
    ref = A.attend_prefill(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_ctx, b.scale, 1)
    V = A.gather_tokens(b.v_pool, b.block_table[0], 1128, 0)
    planted = list(range(900, 910)) + list(range(1050, 1060))
    for i in (0, 49, 59, 127):      # row i sees keys 0 .. 1000 + i
        seen = [j for j in planted if j <= 1000 + i]
        np.testing.assert_allclose(ref[i, 0], V[seen].mean(axis=0), atol=1e-3)
