"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Tolerance (bf16 inputs, fp32 accumulation, bf16 outputs): max-abs <= 2e-2 and
mean-abs <= 2e-3 per output tensor.  Small batches are compared element by
element; the full-size workloads are compared on sampled rows that the oracle
computes one by one, in the same launch configuration the bench times.
"""
import numpy as np
import pytest

import synth
from oracle import attention as A
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


def _oracle(b, pre_rows=None, dec_reqs=None):
    w = b.workload
    op = od = None
    if w.prefill_rows:
        op = A.attend_prefill_batched(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_qo_lens,
                                      b.prefill_kv_lens, b.scale, w.num_kv_heads, rows=pre_rows)
    if w.num_decode:
        od = A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale,
                             w.num_kv_heads, requests=dec_reqs, first_row=b.num_prefill)
    return op, od


def _run(env, b, **plan_kw):
    torch, pod = env
    db = DeviceBatch(torch, b)
    pl = db.plan(pod, **plan_kw)
    ws = db.workspace(pl)
    pl.upload(ws)
    db.run(pod, pl, ws)
    torch.cuda.synchronize()
    assert db.error_word(pl, ws) == 0
    return db, pl, ws


SMALL = [
    synth.tiny(),
    synth.custom("ragged_d128_g4", 8, 2, 128, 300, 200, [1, 15, 16, 17, 100, 1000, 3000], 5),
    synth.custom("ragged_d64_g2", 4, 2, 64, 130, 33, [3, 64, 65, 700], 6),
    synth.custom("mha_g1", 4, 4, 128, 129, 0, [1, 2, 300], 7),
    synth.custom("g8", 16, 2, 128, 64, 1000, [5000, 17, 250], 8),
    synth.custom("decode_only", 8, 2, 128, 0, 0, [1, 16, 31, 4097, 9000], 9),
    synth.custom("prefill_only", 8, 2, 128, 257, 1500, [], 10),
    synth.custom("prefill_no_prior", 4, 1, 64, 200, 0, [40], 11),
    # group sizes that do not divide a warp (the split merge is specialised per group size)
    synth.custom("g3", 6, 2, 128, 150, 300, [700, 3000, 33], 13),
    synth.custom("g5_d64", 10, 2, 64, 70, 90, [2600, 17], 14),
    synth.custom("g6", 12, 2, 128, 64, 500, [4100, 260], 15),
    synth.custom("g7", 28, 4, 128, 96, 200, [3500, 1, 640], 16),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("flags", [0, 1, 64, 65], ids=["fused", "sequential", "four_warps", "four_warps_sequential"])
def test_small_batches_full_parity(env, w, flags):
    b = synth.make_batch(w)
    db, pl, ws = _run(env, b, flags=flags)
    op, od = db.outputs()
    rp, rd = _oracle(b)
    if rp is not None:
        _check(op, rp, f"{w.name} prefill")
    if rd is not None:
        _check(od, rd, f"{w.name} decode")


@pytest.mark.parametrize("kw", [dict(ctas_per_sm=1), dict(ratio=(0, 1)), dict(ratio=(1, 0)), dict(max_waves=8),
                                dict(min_chunk_pages=1), dict(num_sms=7), dict(flags=4, max_waves=8),
                                dict(flags=5, max_waves=8), dict(flags=16), dict(flags=16 | 4, max_waves=8),
                                dict(flags=32), dict(flags=64, ratio=(0, 1)), dict(flags=64 | 16),
                                dict(flags=64 | 4, max_waves=8), dict(flags=64 | 32)],
                         ids=["one_cta", "decode_first", "prefill_first", "many_splits", "tiny_splits", "few_sms",
                              "merge_kernel", "merge_kernel_sequential", "two_streams", "two_streams_merge_kernel",
                              "sm_partition", "four_warps_decode_first", "four_warps_two_streams",
                              "four_warps_merge_kernel", "four_warps_sm_partition"])
def test_knobs_keep_results(env, kw):
    w = synth.custom("knobs", 8, 2, 128, 300, 700, [16, 33, 1000, 2500, 4096], 12)
    b = synth.make_batch(w)
    db, pl, ws = _run(env, b, **kw)
    op, od = db.outputs()
    rp, rd = _oracle(b)
    _check(op, rp, "prefill")
    _check(od, rd, "decode")


BATCHED = [
    # several prefill requests (rows 0..NP-1): ragged chunks, one row, an empty request, no prior context
    synth.custom_batched("batched_ragged_d128", 8, 2, 128, [(300, 200), (1, 0), (0, 0), (129, 1000), (64, 64)],
                         [1, 15, 17, 1000, 3000], 17),
    synth.custom_batched("batched_d64_g4", 8, 2, 64, [(130, 33), (257, 0)], [700, 64], 18),
    synth.custom_batched("batched_g7", 28, 4, 128, [(96, 500), (40, 17)], [2100, 5], 20),
    synth.custom_batched("batched_prefill_only", 32, 8, 128, [(512, 1024), (200, 300), (100, 0)], [], 19),
    # no prefill request at all: the decodes own block-table rows from 0
    synth.custom_batched("batched_no_prefill", 8, 2, 128, [], [1, 16, 17, 3000, 250], 21),
]


@pytest.mark.parametrize("w", BATCHED, ids=lambda w: w.name)
@pytest.mark.parametrize("flags", [0, 1, 16, 64], ids=["fused", "sequential", "two_streams", "four_warps"])
def test_batched_full_parity(env, w, flags):
    b = synth.make_batch(w)
    db, pl, ws = _run(env, b, flags=flags)
    assert pl.info.num_prefill_requests == w.num_prefill
    op, od = db.outputs()
    rp, rd = _oracle(b)
    if rp is not None:
        _check(op, rp, f"{w.name} prefill")
    if rd is not None:
        _check(od, rd, f"{w.name} decode")


def test_batched_llama3_8b_mix_sampled(env):
    w = synth.batched_llama3_8b_mix()
    # first and last rows of each request (rows 0..511, 512..1023, 1024..1279) and a few in between
    rows = [0, 127, 128, 511, 512, 600, 1023, 1024, 1151, 1279]
    reqs = [0, 1, 31, 63]
    b = synth.make_batch(w)
    db, pl, ws = _run(env, b)
    op, od = db.outputs()
    rp, rd = _oracle(b, pre_rows=rows, dec_reqs=reqs)
    _check(op[rows], rp, "batched prefill rows")
    _check(od[reqs], rd, "batched decode requests")


def _sampled(env, w, pre_rows, dec_reqs, **kw):
    b = synth.make_batch(w)
    db, pl, ws = _run(env, b, **kw)
    op, od = db.outputs()
    rp, rd = _oracle(b, pre_rows=pre_rows, dec_reqs=dec_reqs)
    _check(op[pre_rows], rp, f"{w.name} prefill rows")
    _check(od[dec_reqs], rd, f"{w.name} decode requests")
    return db, pl, ws, b


def test_llama3_8b_mix_sampled(env):
    w = synth.llama3_8b_mix()
    rows = [0, 1, 127, 128, 200, 255, 256, 383, 384, 450, 510, 511]
    reqs = [0, 1, 7, 31, 32, 62, 63]
    db, pl, ws, b = _sampled(env, w, rows, reqs)
    assert pl.info.num_partials > 0       # the workload exercises split-KV + merge


def test_llama3_8b_mix_sampled_four_warps(env):
    """The same full-size batch with only warps 0-3 decoding (3-page rings)."""
    w = synth.llama3_8b_mix()
    _sampled(env, w, [0, 127, 128, 383, 511], [0, 1, 31, 63], flags=64)


@pytest.mark.slow
def test_long_context_mix_sampled(env):
    w = synth.long_context_mix()
    _sampled(env, w, [0, 129, 511, 640, 1000, 1023], [0, 50, 127])


@pytest.mark.slow
def test_decode_heavy_mix_sampled(env):
    w = synth.decode_heavy_mix()
    b_lens = synth._draw_lengths(np.random.default_rng(w.seed), w)
    longest = int(np.argmax(b_lens))
    shortest = int(np.argmin(b_lens))
    _sampled(env, w, [0, 127, 128, 255], sorted({0, longest, shortest, 255}))


def test_fused_equals_sequential(env):
    torch, pod = env
    w = synth.custom("fs", 32, 8, 128, 384, 1024, list(range(100, 4000, 150)), 13)
    b = synth.make_batch(w)
    outs = []
    for flags in (0, 1):
        db, pl, ws = _run(env, b, flags=flags)
        outs.append(db.outputs())
    np.testing.assert_allclose(outs[0][0], outs[1][0], atol=1e-2)
    np.testing.assert_allclose(outs[0][1], outs[1][1], atol=1e-2)


def test_repeat_runs_are_stable(env):
    """Counters are reset every run: ten back-to-back runs give identical bits."""
    torch, pod = env
    w = synth.custom("rep", 8, 2, 128, 256, 512, [100, 2000, 3000, 50], 14)
    b = synth.make_batch(w)
    db, pl, ws = _run(env, b)
    first = [t.clone() for t in (db.o_pre, db.o_dec)]
    for _ in range(10):
        db.run(pod, pl, ws)
    torch.cuda.synchronize()
    assert torch.equal(first[0], db.o_pre) and torch.equal(first[1], db.o_dec)


# ----------------------------------------------------------- prefill KV pieces
# Batches whose prefill items the plan cuts into KV pieces (merged by the CTA that finishes the
# item's last piece): d = 64 / 128, g = 1..8, ragged chunk ends, no prior context, several requests.
SPLIT = [
    synth.custom("split_d128_g4", 8, 2, 128, 300, 2500, [17, 1000, 3000], 40),
    synth.custom("split_d64_g2_prefill_only", 4, 2, 64, 70, 1800, [], 41),
    synth.custom("split_mha_g1", 4, 4, 128, 129, 1600, [33], 42),
    synth.custom("split_g8", 16, 2, 128, 64, 3000, [5000, 17], 43),
    synth.custom("split_g3_d64", 6, 2, 64, 200, 1200, [700], 44),
    synth.custom("split_g5", 10, 2, 128, 100, 900, [2600, 17], 45),
    synth.custom("split_g7", 28, 4, 128, 96, 1500, [3500, 1], 46),
    synth.custom("split_no_prior", 8, 2, 128, 1200, 0, [100, 900], 47),
    synth.custom_batched("split_batched", 8, 2, 128, [(300, 2000), (1, 900), (0, 0), (129, 3000)], [1, 1000], 48),
]


@pytest.mark.parametrize("w", SPLIT, ids=lambda w: w.name)
@pytest.mark.parametrize("flags", [0, 1, 16, 64], ids=["fused", "sequential", "two_streams", "four_warps"])
def test_split_prefill_full_parity(env, w, flags):
    b = synth.make_batch(w)
    db, pl, ws = _run(env, b, flags=flags)
    assert pl.info.num_prefill_partials > 0, "the batch should split its prefill"
    op, od = db.outputs()
    rp, rd = _oracle(b)
    _check(op, rp, f"{w.name} prefill")
    if rd is not None:
        _check(od, rd, f"{w.name} decode")


@pytest.mark.parametrize("kw", [dict(max_prefill_splits=2), dict(max_prefill_splits=16), dict(max_prefill_splits=1),
                                dict(flags=128), dict(flags=128 | 1), dict(flags=128, ctas_per_sm=1),
                                dict(flags=128, ratio=(0, 1)), dict(flags=128 | 32)],
                         ids=["cap2", "cap16", "never", "unlimited", "unlimited_sequential", "unlimited_one_cta",
                              "unlimited_decode_first", "unlimited_sm_partition"])
def test_split_knobs_keep_results(env, kw):
    w = synth.custom("split_knobs", 8, 2, 128, 300, 1700, [16, 1000, 2500, 4096], 49)
    b = synth.make_batch(w)
    db, pl, ws = _run(env, b, **kw)
    if kw.get("max_prefill_splits") != 1:
        assert pl.info.num_prefill_partials > 0
    op, od = db.outputs()
    rp, rd = _oracle(b)
    _check(op, rp, "prefill")
    _check(od, rd, "decode")


def test_llama3_8b_mix_sampled_unlimited_split(env):
    """The full-size bench batch with the co-located limit off: 256 prefill pieces merged in-kernel."""
    torch, pod = env
    w = synth.llama3_8b_mix()
    db, pl, ws, b = _sampled(env, w, [0, 1, 127, 128, 255, 256, 383, 384, 510, 511], [0, 31, 63],
                             flags=pod.POD_FLAG_PREFILL_SPLIT_UNLIMITED)
    assert pl.info.num_prefill_partials == 256
