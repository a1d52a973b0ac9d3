"""GPU parity of the FP8 (e4m3) KV cache for the decode branch (pod_attn_run_fp8kv).

The decode requests read e4m3 pages with one fp32 scale per kv head; the
prefill requests keep the bf16 pools (blog post "Prefill vs. Decode GPU
Utilization Imbalance", "Quantization and compression as a lever on both the
bandwidth and capacity problem": 8-bit KV halves the bytes decode streams).
The oracle is the float64 attention on the exactly decoded, scaled codes
(oracle/fp8.py); tolerance as every other parity test: max-abs <= 2e-2 and
mean-abs <= 2e-3 per output tensor, element by element."""
import numpy as np
import pytest

import synth
from oracle import attention as A
from oracle import fp8
from prefill_decode_b200.device_batch import DeviceBatch

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(scope="module")
def env():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from prefill_decode_b200 import build
    build.build()
    import prefill_decode_b200 as pod
    return torch, pod


def _check(got, ref, what):
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, f"{what}: max {err.max():.3e} mean {err.mean():.3e}"


def _oracle(b, c, dec_reqs=None, pre_rows=None):
    w = b.workload
    op = od = None
    if w.prefill_rows:
        op = A.attend_prefill_batched(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_qo_lens,
                                      b.prefill_kv_lens, b.scale, w.num_kv_heads, rows=pre_rows)
    if w.num_decode:
        K = fp8.dequant_pool(c.k_pool, c.k_scale)
        V = fp8.dequant_pool(c.v_pool, c.v_scale)
        od = A.attend_decode(b.q_decode, K, V, b.block_table, b.kv_lens, b.scale, w.num_kv_heads,
                             requests=dec_reqs, first_row=b.num_prefill)
    return op, od


def _run(env, b, c, **plan_kw):
    torch, pod = env
    db = DeviceBatch(torch, b).attach_fp8(c)
    pl = db.plan(pod, **plan_kw)
    ws = db.workspace(pl)
    pl.upload(ws)
    db.run_fp8(pod, pl, ws)
    torch.cuda.synchronize()
    assert db.error_word(pl, ws) == 0
    return db, pl, ws


SMALL = [
    synth.tiny(),
    synth.custom("fp8_ragged_d128_g4", 8, 2, 128, 300, 200, [1, 15, 16, 17, 100, 1000, 3000], 55),
    synth.custom("fp8_ragged_d64_g2", 4, 2, 64, 130, 33, [3, 64, 65, 700], 56),
    synth.custom("fp8_mha_g1", 4, 4, 128, 129, 0, [1, 2, 300], 57),
    synth.custom("fp8_g8", 16, 2, 128, 64, 1000, [5000, 17, 250], 58),
    synth.custom("fp8_decode_only", 8, 2, 128, 0, 0, [1, 16, 31, 4097, 9000], 59),
    synth.custom("fp8_g3", 6, 2, 128, 150, 300, [700, 3000, 33], 60),
    synth.custom("fp8_g5_d64", 10, 2, 64, 70, 90, [2600, 17], 61),
    synth.custom("fp8_g7", 28, 4, 128, 96, 200, [3500, 1, 640], 62),
    synth.custom_batched("fp8_batched", 8, 2, 128, [(300, 200), (1, 0), (0, 0), (129, 1000)], [1, 15, 17, 3000], 63),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("kw", [dict(), dict(flags=1), dict(flags=16), dict(flags=64), dict(max_waves=8)],
                         ids=["fused", "sequential", "two_streams", "four_warps", "many_splits"])
def test_fp8_small_batches_full_parity(env, w, kw):
    b = synth.make_batch(w)
    c = synth.fp8_cache(b)
    db, pl, ws = _run(env, b, c, **kw)
    op, od = db.outputs()
    rp, rd = _oracle(b, c)
    if rp is not None:
        _check(op, rp, f"{w.name} prefill")
    if rd is not None:
        _check(od, rd, f"{w.name} decode")


def test_fp8_nan_codes_past_the_end_are_ignored(env):
    """Slots past a request's length may hold any code, NaN (0x7F / 0xFF) included."""
    w = synth.custom("fp8_nan_tail", 8, 2, 128, 64, 100, [1, 17, 33, 250], 64)
    b = synth.make_batch(w)
    c = synth.fp8_cache(b)
    for r, L in enumerate(b.decode_lens.tolist()):
        row = b.num_prefill + r
        n = -(-L // 16)
        if L % 16:
            blk = int(b.block_table[row, n - 1])
            c.k_pool[blk, :, L % 16:, :] = 0x7F
            c.v_pool[blk, :, L % 16:, :] = 0xFF
    db, pl, ws = _run(env, b, c)
    _, od = db.outputs()
    _, rd = _oracle(b, c)
    _check(od, rd, "decode")


def test_fp8_halves_nothing_but_the_bytes(env):
    """The same batch through pod_attn_run (bf16) and pod_attn_run_fp8kv: prefill outputs are
    bit-identical (the prefill path is unchanged), decode outputs differ only by the quantisation."""
    torch, pod = env
    w = synth.custom("fp8_vs_bf16", 8, 2, 128, 200, 700, [100, 1000, 4000], 65)
    b = synth.make_batch(w)
    c = synth.fp8_cache(b)
    db, pl, ws = _run(env, b, c)
    o8 = db.o_pre.clone(), db.o_dec.clone()
    db.run(pod, pl, ws)
    torch.cuda.synchronize()
    assert torch.equal(o8[0], db.o_pre)
    diff = (o8[1].float() - db.o_dec.float()).abs().max().item()
    assert 0 < diff < 0.25


def _sampled(env, w, pre_rows, dec_reqs, **kw):
    torch, pod = env
    b = synth.make_batch(w)
    c = synth.fp8_cache(b)
    db, pl, ws = _run(env, b, c, **kw)
    op, od = db.outputs()
    rp, rd = _oracle(b, c, dec_reqs=dec_reqs, pre_rows=pre_rows)
    _check(op[pre_rows], rp, f"{w.name} prefill rows")
    _check(od[dec_reqs], rd, f"{w.name} decode requests")


def test_fp8_llama3_8b_mix_sampled(env):
    _sampled(env, synth.llama3_8b_mix(), [0, 127, 128, 383, 511], [0, 1, 31, 62, 63])


@pytest.mark.slow
def test_fp8_decode_heavy_mix_sampled(env):
    w = synth.decode_heavy_mix()
    lens = synth._draw_lengths(np.random.default_rng(w.seed), w)
    _sampled(env, w, [0, 255], sorted({0, int(np.argmax(lens)), int(np.argmin(lens)), 255}))


def test_fp8_bad_block_id_is_reported(env):
    torch, pod = env
    w = synth.custom("fp8_bad_block", 8, 2, 128, 0, 0, [100, 700], 66)
    b = synth.make_batch(w)
    c = synth.fp8_cache(b)
    b.block_table[b.num_prefill + 1, 3] = b.num_blocks + 5
    db = DeviceBatch(torch, b).attach_fp8(c)
    pl = db.plan(pod)
    ws = db.workspace(pl)
    pl.upload(ws)
    db.run_fp8(pod, pl, ws)
    torch.cuda.synchronize()
    assert db.error_word(pl, ws) == pod.POD_ERR_BOUNDS
