"""C-ABI library checks that need no GPU: it loads, exports every entry point
that include/pod_attn.h declares, and its C++ planner reproduces the plan rule
of oracle/plan_ref.py bit for bit (tables, split size, ratio), including the
inputs it must reject."""
import ctypes
import os
import re

import numpy as np
import pytest

import synth
from oracle.plan_ref import plan_ref, plan_ref_batched, PlanError

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pod():
    from prefill_decode_b200 import build
    build.build()
    import prefill_decode_b200 as m
    m.lib()
    return m


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "pod_attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pod_attn_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol(pod):
    names = _declared_functions()
    assert len(names) >= 10
    L = ctypes.CDLL(pod.LIB_PATH)
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/pod_attn.h but not exported"
    assert sorted(pod.EXPORTED) == names


def test_status_strings(pod):
    assert pod.status_string(0) == "ok"
    assert "workspace" in pod.status_string(pod.POD_ERR_WORKSPACE)


CONFIGS = [synth.tiny(), synth.llama3_8b_mix(), synth.long_context_mix(), synth.decode_heavy_mix()] + synth.sweep_points()


def _lens(w):
    return [int(x) for x in synth._draw_lengths(np.random.default_rng(w.seed), w)]


def _c_plan(pod, Hq, Hkv, d, sms, P, KV, lens, **kw):
    """The same batch and knobs through the C planner (keyword names as plan_ref's)."""
    ratio = (kw.get("ratio_p", 0), kw.get("ratio_d", 0))
    flags = pod.POD_FLAG_DECODE_FOUR_WARPS if kw.get("decode_warps", 6) == 4 else 0
    if kw.get("split_unlimited", False):
        flags |= pod.POD_FLAG_PREFILL_SPLIT_UNLIMITED
    return pod.Plan(Hq, Hkv, d, P, KV, lens, num_sms=sms, ctas_per_sm=kw.get("ctas_per_sm", 0), ratio=ratio,
                    max_waves=kw.get("max_waves", 0), min_chunk_pages=kw.get("min_chunk_pages", 0),
                    max_prefill_splits=kw.get("prefill_splits", 0), flags=flags)


def _same_tables(pl, ref):
    pre, dec, mer = pl.tables()
    np.testing.assert_array_equal(pre, ref.prefill_items)
    np.testing.assert_array_equal(dec, ref.decode_items)
    np.testing.assert_array_equal(mer, ref.merge_items)
    np.testing.assert_array_equal(pl.prefill_merges(), ref.prefill_merge_items)
    i = pl.info
    assert (i.ctas_per_sm, i.ratio_prefill, i.ratio_decode, i.chunk_pages, i.num_partials) == (
        ref.ctas_per_sm, ref.ratio_p, ref.ratio_d, ref.chunk_pages, ref.num_partials)
    assert (i.num_prefill_items, i.num_prefill_partials, i.num_prefill_merge_items) == (
        len(ref.prefill_items), ref.num_prefill_partials, len(ref.prefill_merge_items))


def _compare(pod, Hq, Hkv, d, sms, P, KV, lens, **kw):
    ref = plan_ref(Hq, Hkv, d, sms, P, KV, lens, **kw)
    pl = _c_plan(pod, Hq, Hkv, d, sms, P, KV, lens, **kw)
    _same_tables(pl, ref)
    i = pl.info
    assert i.grid == sms * ref.ctas_per_sm
    return pl


@pytest.mark.parametrize("w", CONFIGS, ids=lambda w: w.name)
def test_c_plan_matches_plan_ref(pod, w):
    P, C = w.prefill_len, w.prefill_ctx
    pl = _compare(pod, w.num_q_heads, w.num_kv_heads, w.head_dim, 148, P, C + P, _lens(w))
    # algorithmic counts used by the roofline
    L = sum(_lens(w))
    assert pl.info.decode_flops == 4 * w.head_dim * w.num_q_heads * L
    assert pl.info.kv_bytes == 4 * w.head_dim * w.num_kv_heads * ((C + P if P else 0) + L)
    assert pl.info.prefill_flops == 4 * w.head_dim * w.num_q_heads * sum(C + i + 1 for i in range(P))


def test_c_plan_matches_plan_ref_random(pod):
    rng = np.random.default_rng(2024)
    for _ in range(80):
        Hkv = int(rng.choice([1, 2, 4, 8]))
        g = int(rng.choice([1, 2, 4, 8]))
        P = int(rng.choice([0, 1, 100, 128, 129, 513]))
        C = int(rng.integers(0, 4000)) if P else 0
        B = int(rng.integers(0 if P else 1, 50))
        lens = [int(x) for x in rng.integers(1, 9000, size=B)]
        kw = dict(ctas_per_sm=int(rng.choice([0, 1, 2])), max_waves=int(rng.choice([0, 1, 3])),
                  min_chunk_pages=int(rng.choice([0, 1, 4, 16])),
                  ratio_p=int(rng.choice([0, 0, 1, 2])), ratio_d=int(rng.choice([0, 0, 1, 3])),
                  decode_warps=int(rng.choice([4, 6])), prefill_splits=int(rng.choice([0, 0, 1, 2, 5, 16])),
                  split_unlimited=bool(rng.integers(0, 2)))
        _compare(pod, Hkv * g, Hkv, int(rng.choice([64, 128])), int(rng.integers(1, 200)), P, C + P, lens, **kw)


@pytest.mark.parametrize("bad,code", [
    (dict(Hq=30, Hkv=8), -1), (dict(Hq=32, Hkv=2), -2), (dict(d=96), -2), (dict(page=32), -2),
    (dict(sms=600), -1), (dict(ctas=4), -1), (dict(P=10, KV=5), -1), (dict(lens=[0]), -1),
    (dict(lens=[-3]), -1), (dict(lens=[1 << 25]), -1), (dict(ratio=(-1, 1)), -1),
])
def test_c_plan_rejects(pod, bad, code):
    a = dict(Hq=32, Hkv=8, d=128, page=16, sms=148, ctas=0, P=64, KV=128, lens=[100, 200], ratio=(0, 0))
    a.update(bad)
    with pytest.raises(pod.PodError) as e:
        pod.Plan(a["Hq"], a["Hkv"], a["d"], a["P"], a["KV"], a["lens"], num_sms=a["sms"], ctas_per_sm=a["ctas"],
                 ratio=a["ratio"], page_size=a["page"])
    assert e.value.status == code
    with pytest.raises(PlanError):
        plan_ref(a["Hq"], a["Hkv"], a["d"], a["sms"], a["P"], a["KV"], a["lens"], page_size=a["page"],
                 ctas_per_sm=a["ctas"], ratio_p=a["ratio"][0], ratio_d=a["ratio"][1])


def _compare_batched(pod, Hq, Hkv, d, sms, qo, kv, lens, **kw):
    ref = plan_ref_batched(Hq, Hkv, d, sms, qo, kv, lens, **kw)
    pl = _c_plan(pod, Hq, Hkv, d, sms, qo, kv, lens, **kw)
    _same_tables(pl, ref)
    np.testing.assert_array_equal(pl.prefill_requests(), ref.prefill_requests)
    i = pl.info
    assert (i.num_prefill_requests, i.num_prefill_rows) == (len(qo), sum(qo))
    # algorithmic counts over every prefill request
    assert i.prefill_flops == 4 * d * Hq * sum(sum(K - P + j + 1 for j in range(P)) for P, K in zip(qo, kv))
    assert i.kv_bytes == 4 * d * Hkv * (sum(K for P, K in zip(qo, kv) if P > 0) + sum(lens))
    assert i.qo_bytes == 4 * d * Hq * (sum(qo) + len(lens))
    return pl


def test_c_batched_plan_matches_plan_ref_random(pod):
    rng = np.random.default_rng(77)
    for _ in range(60):
        Hkv = int(rng.choice([1, 2, 8]))
        g = int(rng.choice([1, 4, 8]))
        NP = int(rng.integers(0, 7))
        qo = [int(rng.choice([0, 1, 64, 128, 300, 1025])) for _ in range(NP)]
        kv = [P + (int(rng.integers(0, 3000)) if P else int(rng.integers(0, 5))) for P in qo]
        lens = [int(x) for x in rng.integers(1, 6000, size=int(rng.integers(0, 30)))]
        kw = dict(ctas_per_sm=int(rng.choice([0, 1, 2])), max_waves=int(rng.choice([0, 1, 3])),
                  min_chunk_pages=int(rng.choice([0, 1, 16])), decode_warps=int(rng.choice([4, 6])),
                  prefill_splits=int(rng.choice([0, 0, 1, 3])), split_unlimited=bool(rng.integers(0, 2)))
        _compare_batched(pod, Hkv * g, Hkv, int(rng.choice([64, 128])), int(rng.integers(1, 200)), qo, kv, lens, **kw)


def test_c_single_form_equals_one_request_batch(pod):
    a = pod.Plan(32, 8, 128, 512, 4608, [1000, 3000], num_sms=148)
    b = pod.Plan(32, 8, 128, [512], [4608], [1000, 3000], num_sms=148)
    for x, y in zip(a.tables(), b.tables()):
        np.testing.assert_array_equal(x, y)
    np.testing.assert_array_equal(a.prefill_requests(), b.prefill_requests())
    assert a.workspace_bytes == b.workspace_bytes


@pytest.mark.parametrize("qo,kv", [([-1], [5]), ([10], [5]), ([1 << 24, 1], [1 << 24, 1])])
def test_c_batched_plan_rejects(pod, qo, kv):
    with pytest.raises(pod.PodError) as e:
        pod.Plan(8, 2, 128, qo, kv, [100], num_sms=148)
    assert e.value.status == pod.POD_ERR_INVALID_ARG


def test_run_rejects_bad_host_arguments(pod):
    """Argument validation happens on the host before any launch (no GPU needed)."""
    pl = pod.Plan(4, 2, 64, 64, 192, [64, 100], num_sms=4)
    ws = pl.workspace_bytes
    L = pod.lib()
    # null workspace
    assert L.pod_attn_run(pl.handle, 16, 16, 16, 16, 10, 16, 4, None, 0.125, 16, 16, None, ws, None, None) == -1
    # misaligned workspace
    assert L.pod_attn_run(pl.handle, 16, 16, 16, 16, 10, 16, 4, None, 0.125, 16, 16, 0x1010, ws, None, None) == -1
    # workspace too small
    assert L.pod_attn_run(pl.handle, 16, 16, 16, 16, 10, 16, 4, None, 0.125, 16, 16, 0x1000, 256, None, None) == -3
    # misaligned q pointer
    assert L.pod_attn_run(pl.handle, 17, 16, 16, 16, 10, 16, 4, None, 0.125, 16, 16, 0x1000, ws, None, None) == -1
    # bad scale
    assert L.pod_attn_run(pl.handle, 16, 16, 16, 16, 10, 16, 4, None, -1.0, 16, 16, 0x1000, ws, None, None) == -1
    # upload: too small / misaligned
    assert L.pod_attn_upload(pl.handle, 0x1000, 256, None) == -3
    assert L.pod_attn_upload(pl.handle, 0x1010, ws, None) == -1


def test_batched_run_rejects_bad_host_arguments(pod):
    """A batched plan validates its arguments on the host before any launch."""
    pl = pod.Plan(4, 2, 64, [64, 0, 30], [192, 0, 40], [64, 100], num_sms=4)
    ws = pl.workspace_bytes
    L = pod.lib()
    assert (pl.info.num_prefill_requests, pl.info.num_prefill_rows) == (3, 94)
    # prefill rows exist: q_prefill / o_prefill are required and 16-byte aligned
    assert L.pod_attn_run(pl.handle, None, 16, 16, 16, 10, 16, 4, None, 0.125, 16, 16, 0x1000, ws, None, None) == -1
    assert L.pod_attn_run(pl.handle, 16, 16, 16, 16, 10, 16, 4, None, 0.125, 24, 16, 0x1000, ws, None, None) == -1
    # tracing without a trace buffer
    tr = pod.Plan(4, 2, 64, [64], [192], [64], num_sms=4, flags=pod.POD_FLAG_TRACE)
    assert L.pod_attn_run(tr.handle, 16, 16, 16, 16, 10, 16, 4, None, 0.125, 16, 16, 0x1000, tr.workspace_bytes,
                          None, None) == -1


def test_decode_only_batched_plan_needs_no_prefill_pointers(pod):
    pl = pod.Plan(8, 2, 128, [], [], [1, 16, 3000], num_sms=148)
    assert (pl.info.num_prefill_requests, pl.info.num_prefill_items) == (0, 0)
    assert pl.prefill_requests().shape == (0, 4)
    # the workspace holds no prefill table and the decode side is planned as usual
    one = pod.Plan(8, 2, 128, 0, 0, [1, 16, 3000], num_sms=148)
    np.testing.assert_array_equal(pl.tables()[1], one.tables()[1])


def test_c_plan_rejects_too_many_heads_and_overflowing_work(pod):
    with pytest.raises(pod.PodError) as e:
        pod.Plan(4104, 513, 128, 64, 128, [100], num_sms=148)
    assert e.value.status == pod.POD_ERR_INVALID_ARG
    big = 1 << 24
    with pytest.raises(pod.PodError) as e:
        pod.Plan(4096, 512, 128, [big], [big], [100], num_sms=148)
    assert e.value.status == pod.POD_ERR_INVALID_ARG
    # the largest head count still plans, and agrees with the planner of record
    _compare_batched(pod, 4096, 512, 128, 148, [128], [1 << 20], [100])


def test_c_planner_matches_plan_ref_property(pod):
    """Property check over generated batches (hypothesis): the C planner and the
    written rule agree on every table, or both reject the batch."""
    from hypothesis import given, settings, HealthCheck, strategies as st

    chunk = st.tuples(st.sampled_from([0, 1, 2, 63, 64, 65, 127, 128, 129, 255, 256, 257, 1000]),
                      st.integers(0, 5000))
    batch = st.fixed_dictionaries(dict(
        Hkv=st.sampled_from([1, 2, 3, 8]), g=st.integers(1, 8), d=st.sampled_from([64, 128]),
        sms=st.integers(1, 300), chunks=st.lists(chunk, max_size=5),
        lens=st.lists(st.integers(1, 40000), max_size=40),
        ctas=st.sampled_from([0, 1, 2]), waves=st.integers(0, 4), minc=st.integers(0, 40),
        rp=st.integers(0, 3), rd=st.integers(0, 3), dw=st.sampled_from([4, 6]),
        ps=st.sampled_from([0, 1, 2, 4, 16, 17]), unl=st.booleans()))

    @settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])
    @given(batch)
    def check(x):
        qo = [P for P, _ in x["chunks"]]
        kv = [P + C if P else C % 3 for P, C in x["chunks"]]
        kw = dict(ctas_per_sm=x["ctas"], max_waves=x["waves"], min_chunk_pages=x["minc"],
                  ratio_p=x["rp"], ratio_d=x["rd"], decode_warps=x["dw"], prefill_splits=x["ps"],
                  split_unlimited=x["unl"])
        try:
            ref = plan_ref_batched(x["Hkv"] * x["g"], x["Hkv"], x["d"], x["sms"], qo, kv, x["lens"], **kw)
        except PlanError:
            ref = None
        if ref is None:
            with pytest.raises(pod.PodError):
                _c_plan(pod, x["Hkv"] * x["g"], x["Hkv"], x["d"], x["sms"], qo, kv, x["lens"], **kw)
            return
        _compare_batched(pod, x["Hkv"] * x["g"], x["Hkv"], x["d"], x["sms"], qo, kv, x["lens"], **kw)

    check()
