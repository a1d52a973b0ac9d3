"""pod_attn_run_static: the entry point for callers that cannot allocate device
memory (for example a plugin inside an inference engine that keeps nearly all
HBM in its own pools, or a latency-critical caller that cannot pay for
cudaMalloc's implicit synchronisation).  It takes no workspace and runs on a
fixed device array owned by the library.  This file is collected last so a
failure here cannot hide the other tests; it passes alone in a fresh process
and after them."""
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


def _close(a, b):
    e = np.abs(a - b)
    return np.isfinite(a).all() and e.max() <= MAX_ABS and e.mean() <= MEAN_ABS


@pytest.mark.parametrize("heads", [(32, 8), (8, 2)], ids=["decode_splits", "decode_and_prefill_splits"])
def test_static_scratch_matches_workspace_entry_point(env, heads):
    torch, pod = env
    # decode splits (partials + merge) and a ragged multi-tile prefill, so the scratch is really used;
    # with 8/2 heads the prefill items are cut into KV pieces too, whose partials also live there
    Hq, Hkv = heads
    w = synth.custom("no_alloc", Hq, Hkv, 128, 300, 900, [17, 1000, 3000, 5000, 257], 21)
    b = synth.make_batch(w)
    db = DeviceBatch(torch, b)
    plan = db.plan(pod, max_waves=8)
    assert plan.info.num_partials > 0
    assert (plan.info.num_prefill_partials > 0) == (Hq == 8)
    assert plan.workspace_bytes <= (8 << 20)
    ws = db.workspace(plan)
    plan.upload(ws)
    db.run(pod, plan, ws)
    torch.cuda.synchronize()
    ref_pre, ref_dec = db.outputs()

    w = b.workload
    ora_pre = A.attend_prefill(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_ctx, b.scale,
                               w.num_kv_heads)
    ora_dec = A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, w.num_kv_heads)
    assert _close(ref_pre, ora_pre) and _close(ref_dec, ora_dec)

    L = pod.lib()
    for call in range(2):
        db.o_pre.fill_(0)
        db.o_dec.fill_(0)
        rc = L.pod_attn_run_static(plan.handle, db.q_pre.data_ptr(), db.q_dec.data_ptr(), db.k.data_ptr(),
                                   db.v.data_ptr(), b.num_blocks, db.bt.data_ptr(), db.bt.shape[1],
                                   db.lens.data_ptr(), b.scale, db.o_pre.data_ptr(), db.o_dec.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
        assert rc == 0, pod.status_string(rc)
        torch.cuda.synchronize()
        got_pre, got_dec = db.outputs()
        assert _close(got_pre, ref_pre), f"call {call}: prefill differs"
        assert _close(got_dec, ref_dec), f"call {call}: decode differs"
        # and against the float64 oracle, at the tolerance of every other parity test
        assert _close(got_pre, ora_pre), f"call {call}: prefill differs from the oracle"
        assert _close(got_dec, ora_dec), f"call {call}: decode differs from the oracle"


def test_static_scratch_rejects_oversized_plan(env):
    torch, pod = env
    # 512 decode requests x 8 kv heads, each split: partials far beyond 8 MiB
    plan = pod.Plan(32, 8, 128, 0, 0, [32768] * 512, max_waves=64)
    assert plan.workspace_bytes > (8 << 20)
    rc = pod.lib().pod_attn_run_static(plan.handle, None, 16, 16, 16, 10, 16, 1, None, 0.1, None, 16, None)
    assert rc == pod.POD_ERR_WORKSPACE
