"""Host-side pieces of bench.py that need no GPU: the CPU-baseline sampling
(which rows and requests, how sampled oracle time scales to the whole batch)
for one and for several prefill requests, the device-code hash that keys the
committed ncu traffic figure, the plan digest replicas compare, and which arms'
step is a single kernel launch."""
import numpy as np
import pytest

import bench
import synth


def _batch(w):
    return synth.make_batch(w)


def test_prefill_row_keys_one_request():
    b = _batch(synth.custom("k1", 4, 2, 64, 5, 7, [3], 1))
    np.testing.assert_array_equal(bench.prefill_row_keys(b), [8, 9, 10, 11, 12])   # C + i + 1


def test_prefill_row_keys_several_requests():
    b = _batch(synth.custom_batched("k2", 4, 2, 64, [(3, 2), (0, 0), (2, 0)], [4], 2))
    np.testing.assert_array_equal(bench.prefill_row_keys(b), [3, 4, 5, 1, 2])


def test_sample_sets_and_extrapolation_cover_the_batch():
    b = _batch(synth.custom_batched("k3", 4, 2, 64, [(20, 10), (9, 0)], [30, 50, 70], 3))
    reqs, rows = bench.sample_sets(b, 4)
    assert reqs == [0] and rows == [0, 4, 8, 12, 16, 20, 24, 28]
    # sampled time t scales by (all keys) / (sampled keys) on each side
    keys = bench.prefill_row_keys(b)
    got = bench.extrapolate(b, reqs, rows, t_dec=1.0, t_pre=1.0)
    want = (30 + 50 + 70) / 30 + keys.sum() / keys[rows].sum()
    assert got == pytest.approx(want)


def test_kernel_hash_ignores_the_host_side_part(tmp_path):
    import os
    import shutil
    root = tmp_path
    for f in bench.KERNEL_SOURCES:
        os.makedirs(os.path.dirname(root / f), exist_ok=True)
        shutil.copy(os.path.join(bench.ROOT, f), root / f)
    base = bench.kernel_source_sha(str(root))
    cu = root / bench.KERNEL_SOURCES[0]
    cu.write_bytes(cu.read_bytes() + b"\n// a host-side edit\n")
    assert bench.kernel_source_sha(str(root)) == base
    data = cu.read_bytes()
    i = data.find(bench.HOST_SIDE_MARKER)
    assert i > 0
    cu.write_bytes(data[:i] + b"// a comment-only device-side edit\n/* and a block comment */\n" + data[i:])
    assert bench.kernel_source_sha(str(root)) == base
    cu.write_bytes(data[:i] + b"__device__ int pod_hash_probe;\n" + data[i:])
    assert bench.kernel_source_sha(str(root)) != base


def test_plan_digest_tracks_the_tables():
    from prefill_decode_b200 import build
    build.build()
    import prefill_decode_b200 as pod
    a = pod.Plan(8, 2, 128, 300, 900, [100, 2000], num_sms=148)
    b = pod.Plan(8, 2, 128, 300, 900, [100, 2000], num_sms=148)
    c = pod.Plan(8, 2, 128, 300, 900, [100, 2001], num_sms=148)
    assert bench.plan_digest(a) == bench.plan_digest(b) != bench.plan_digest(c)


def test_single_thread_oracle_figure_is_positive_and_scaled():
    b = synth.make_batch(synth.tiny())
    reqs, rows = bench.sample_sets(b, 2)
    v = bench.cpu_oracle_single_thread_us(b, reqs, rows)
    assert v > 0
    assert bench.blas_threads() >= 1


def test_single_launch_names_the_arms_whose_step_is_one_kernel():
    """The step of a plain fused plan is one launch (its kernel time is the back-to-back step time); the
    two-kernel arms, the traced path and the separate merge kernel are not."""
    import prefill_decode_b200 as pod

    class Info:
        def __init__(self, n_pre, n_dec):
            self.num_prefill_items, self.num_decode_items = n_pre, n_dec

    both = Info(4, 9)
    assert bench.single_launch({}, both)
    assert bench.single_launch(dict(ratio=(1, 0)), both)
    assert bench.single_launch(dict(flags=pod.POD_FLAG_SM_PARTITION | pod.POD_FLAG_DECODE_FOUR_WARPS), both)
    assert bench.single_launch(dict(flags=pod.POD_FLAG_PREFILL_SPLIT_UNLIMITED, max_prefill_splits=1), both)
    assert not bench.single_launch(dict(flags=pod.POD_FLAG_SEQUENTIAL), both)
    assert not bench.single_launch(dict(flags=pod.POD_FLAG_TWO_STREAMS), both)
    assert not bench.single_launch(dict(flags=pod.POD_FLAG_TRACE), both)
    assert not bench.single_launch(dict(flags=pod.POD_FLAG_MERGE_KERNEL), both)
    # two streams with one side empty falls back to the fused launch
    assert bench.single_launch(dict(flags=pod.POD_FLAG_TWO_STREAMS), Info(0, 9))
    assert bench.single_launch(dict(flags=pod.POD_FLAG_TWO_STREAMS), Info(4, 0))
