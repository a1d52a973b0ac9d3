"""GPU checks of the error paths and the scheduler, with host-made faults only.

Nothing here faults, traps or hangs the GPU: bad block ids are read through
TMA past the tensor's end (zeros) and reported in the workspace error word;
the expired-wait path is exercised by a diagnostic flag that makes one thread
wait (1 ms limit) on a barrier nothing arrives at; the schedule is checked from
the per-item trace the kernel writes."""
from collections import defaultdict

import numpy as np
import pytest

import synth
from oracle import attention as A
from prefill_decode_b200.device_batch import DeviceBatch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from prefill_decode_b200 import build
    build.build()
    import prefill_decode_b200 as pod
    return torch, pod


def _close(got, ref):
    e = np.abs(got - ref)
    return np.isfinite(got).all() and e.max() <= 2e-2 and e.mean() <= 2e-3


W = synth.custom("robust", 8, 2, 128, 200, 300, [40, 700, 1500, 3000, 16], 31)


def test_expired_wait_is_reported_and_attention_still_runs(env):
    torch, pod = env
    b = synth.make_batch(W)
    db = DeviceBatch(torch, b)
    pl = db.plan(pod, flags=pod.POD_FLAG_SELFTEST_TIMEOUT)
    ws = db.workspace(pl)
    pl.upload(ws)
    db.run(pod, pl, ws)
    torch.cuda.synchronize()
    assert db.error_word(pl, ws) == pod.POD_ERR_TIMEOUT
    op, od = db.outputs()
    assert _close(op, A.attend_prefill(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_ctx, b.scale, 2))
    assert _close(od, A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, 2))
    # the context stays usable and the next run starts with a clean error word
    pl2 = db.plan(pod)
    ws2 = db.workspace(pl2)
    pl2.upload(ws2)
    db.run(pod, pl2, ws2)
    torch.cuda.synchronize()
    assert db.error_word(pl2, ws2) == 0


@pytest.mark.parametrize("flags", [0, 64], ids=["six_decode_warps", "four_decode_warps"])
@pytest.mark.parametrize("bad", [10 ** 6, -7])
def test_out_of_range_block_id_is_reported_not_faulted(env, bad, flags):
    torch, pod = env
    b = synth.make_batch(W)
    db = DeviceBatch(torch, b)
    bt = b.block_table.copy()
    bt[3, 5] = bad                     # decode request 2 (1500 tokens), page 5
    db.bt = torch.from_numpy(bt).cuda()
    pl = db.plan(pod, flags=flags)
    ws = db.workspace(pl)
    pl.upload(ws)
    db.run(pod, pl, ws)
    torch.cuda.synchronize()
    assert db.error_word(pl, ws) == pod.POD_ERR_BOUNDS
    off = pl.info.error_offset
    assert int(ws[off + 4:off + 8].view(torch.int32).item()) == bad
    # every other request is untouched
    op, od = db.outputs()
    rd = A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, 2)
    keep = [0, 1, 3, 4]
    assert _close(od[keep], rd[keep])
    assert np.isfinite(od[2]).all()


def test_lengths_that_disagree_with_the_plan_are_reported(env):
    torch, pod = env
    b = synth.make_batch(W)
    db = DeviceBatch(torch, b)
    lens = b.kv_lens.copy()
    lens[2] -= 50                       # the device says request 1 is shorter than the plan
    db.lens = torch.from_numpy(lens).cuda()
    pl = db.plan(pod)
    ws = db.workspace(pl)
    pl.upload(ws)
    db.run(pod, pl, ws)
    torch.cuda.synchronize()
    assert db.error_word(pl, ws) == pod.POD_ERR_PLAN_MISMATCH


@pytest.mark.parametrize("ratio,extra", [((0, 0), 0), ((1, 0), 0), ((0, 1), 0), ((0, 0), 64)],
                         ids=["proportional", "prefill_first", "decode_first", "proportional_four_warps"])
def test_schedule_trace(env, ratio, extra):
    """Every item runs exactly once; with two CTAs per SM and a 1:1 ratio each SM
    has one prefill-home and one decode-home CTA; 1:0 and 0:1 make every CTA
    prefill-home or decode-home."""
    torch, pod = env
    w = synth.custom("trace", 32, 8, 128, 512, 2048, list(range(300, 6000, 97)), 32)
    b = synth.make_batch(w)
    db = DeviceBatch(torch, b)
    pl = db.plan(pod, flags=pod.POD_FLAG_TRACE | extra, ratio=ratio)
    ws = db.workspace(pl)
    pl.upload(ws)
    n = pl.info.num_prefill_items + pl.info.num_decode_items
    trace = torch.zeros(n * 4, dtype=torch.int32, device="cuda")
    db.run(pod, pl, ws, trace=trace)
    torch.cuda.synchronize()
    assert db.error_word(pl, ws) == 0
    t = trace.view(n, 4).cpu().numpy()
    assert (t[:, 3] == 1).all(), "an item ran zero or several times"
    assert (t[:, 1] >= 0).all() and (t[:, 1] < pl.info.grid).all()
    home = {}
    for smid, cta, role, _ in t.tolist():
        assert home.setdefault(cta, (smid, role)) == (smid, role)
    per_sm = defaultdict(set)
    for cta, (smid, role) in home.items():
        per_sm[smid].add((cta, role))
    roles = [r for (_, r) in home.values()]
    if ratio == (1, 0):
        assert set(roles) == {0}
    elif ratio == (0, 1):
        assert set(roles) == {1}
    else:
        assert (pl.info.ratio_prefill, pl.info.ratio_decode) == (1, 1)
        for smid, ctas in per_sm.items():
            if len(ctas) == 2:
                assert sorted(r for _, r in ctas) == [0, 1], f"SM {smid}: {ctas}"
    op, od = db.outputs()
    rows = [0, 255, 256, 511]
    assert _close(op[rows], A.attend_prefill(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_ctx,
                                             b.scale, 8, rows=rows))


def test_out_of_range_block_id_in_a_batched_prefill_request(env):
    """A bad block id in prefill request 1 of a batched batch (its own
    block-table row) is reported in the error word; request 0 and the decodes
    are untouched."""
    torch, pod = env
    w = synth.custom_batched("robust_batched", 8, 2, 128, [(100, 300), (130, 200)], [500, 40], 33)
    b = synth.make_batch(w)
    db = DeviceBatch(torch, b)
    bt = b.block_table.copy()
    bad = 10 ** 7
    bt[1, 3] = bad                      # prefill request 1, page 3 (keys 48..63)
    db.bt = torch.from_numpy(bt).cuda()
    pl = db.plan(pod)
    ws = db.workspace(pl)
    pl.upload(ws)
    db.run(pod, pl, ws)
    torch.cuda.synchronize()
    assert db.error_word(pl, ws) == pod.POD_ERR_BOUNDS
    off = pl.info.error_offset
    assert int(ws[off + 4:off + 8].view(torch.int32).item()) == bad
    op, od = db.outputs()
    rp = A.attend_prefill_batched(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_qo_lens,
                                  b.prefill_kv_lens, b.scale, 2, rows=range(100))
    assert _close(op[:100], rp)
    rd = A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, 2, first_row=2)
    assert _close(od, rd)
    assert np.isfinite(op[100:]).all()


def test_split_prefill_trace_and_bad_block(env):
    """With prefill items cut into KV pieces every piece runs exactly once (trace), and a bad
    block id inside one piece is reported in the error word; the decodes stay correct."""
    torch, pod = env
    w = synth.custom("robust_split", 8, 2, 128, 256, 2000, [300, 1200], 34)
    b = synth.make_batch(w)
    db = DeviceBatch(torch, b)
    pl = db.plan(pod, flags=pod.POD_FLAG_TRACE)
    assert pl.info.num_prefill_partials > 0
    ws = db.workspace(pl)
    pl.upload(ws)
    n = pl.info.num_prefill_items + pl.info.num_decode_items
    trace = torch.zeros(n * 4, dtype=torch.int32, device="cuda")
    db.run(pod, pl, ws, trace=trace)
    torch.cuda.synchronize()
    assert db.error_word(pl, ws) == 0
    assert (trace.view(n, 4)[:, 3] == 1).all().item()
    rp = A.attend_prefill(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_ctx, b.scale, 2)
    assert _close(db.outputs()[0], rp)
    # now a bad block id on page 40 (keys 640..655) of the prefill request
    bt = b.block_table.copy()
    bt[0, 40] = 10 ** 6
    db.bt = torch.from_numpy(bt).cuda()
    pl2 = db.plan(pod)
    ws2 = db.workspace(pl2)
    pl2.upload(ws2)
    db.run(pod, pl2, ws2)
    torch.cuda.synchronize()
    assert db.error_word(pl2, ws2) == pod.POD_ERR_BOUNDS
    op, od = db.outputs()
    assert np.isfinite(op).all()
    rd = A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, 2)
    assert _close(od, rd)


@pytest.mark.parametrize("name", ["decode_splits", "prefill_pieces"])
def test_back_to_back_runs_reuse_the_workspace(env, name):
    """A fused launch leaves its counters at zero (last CTA out; merge counts by the warp that
    completes the merge), so repeated runs on one uploaded workspace stay correct without any
    clearing in between."""
    torch, pod = env
    w = W if name == "decode_splits" else synth.custom("robust_split", 8, 2, 128, 256, 2000, [300, 1200], 34)
    b = synth.make_batch(w)
    db = DeviceBatch(torch, b)
    pl = db.plan(pod)
    assert pl.info.num_merge_items > 0
    if name == "prefill_pieces":
        assert pl.info.num_prefill_partials > 0
    ws = db.workspace(pl)
    pl.upload(ws)
    rp = A.attend_prefill(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_ctx, b.scale, 2)
    rd = A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, 2)
    for _ in range(4):
        db.o_pre.fill_(float("nan"))
        db.o_dec.fill_(float("nan"))
        db.run(pod, pl, ws)
        torch.cuda.synchronize()
        assert db.error_word(pl, ws) == 0
        assert int(torch.count_nonzero(ws[:4096]).item()) == 0, "counters left non-zero"
        op, od = db.outputs()
        assert _close(op, rp) and _close(od, rd)


def test_error_word_tells_about_the_last_run_only(env):
    """A run that records an error publishes it; the next run on the same workspace, with the
    block table repaired and no upload in between, reports 0 and is correct."""
    torch, pod = env
    b = synth.make_batch(W)
    db = DeviceBatch(torch, b)
    good = db.bt
    bt = b.block_table.copy()
    bt[3, 5] = 10 ** 6                  # decode request 2 (1500 tokens), page 5
    pl = db.plan(pod)
    ws = db.workspace(pl)
    pl.upload(ws)
    db.bt = torch.from_numpy(bt).cuda()
    db.run(pod, pl, ws)
    torch.cuda.synchronize()
    assert db.error_word(pl, ws) == pod.POD_ERR_BOUNDS
    off = pl.info.error_offset
    assert int(ws[off + 4:off + 8].view(torch.int32).item()) == 10 ** 6
    db.bt = good
    db.run(pod, pl, ws)
    torch.cuda.synchronize()
    assert db.error_word(pl, ws) == 0
    assert int(ws[off + 4:off + 8].view(torch.int32).item()) == 0
    op, od = db.outputs()
    assert _close(op, A.attend_prefill(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_ctx, b.scale, 2))
    assert _close(od, A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, 2))
