"""Host-side pieces of the benchmark that run without a GPU: the oracle's CPU baseline (the
numbers `bench.py` reports beside the GPU ones) and the fold's algorithmic flop count."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
import iskv_synth as syn  # noqa: E402


def test_cpu_baseline_reports_all_threads_and_one_thread():
    c = bench.cpu_baseline(tokens=2)
    assert c["kind"] == "oracle" and c["unit"] == bench.UNIT
    assert c["value"] > 0 and c["value_1_thread"] > 0
    assert c["cores"] >= 1 and c["host_cores"] >= 1
    assert "extrapolated" in c["sample"]


@pytest.mark.parametrize("wl_id", [1, 2, 3])
def test_fold_flops_counts_every_fold_of_the_append(wl_id):
    """The count grows with the number of folds: one block more adds exactly that fold's terms,
    and the first fold (k = 0) has no projection or rotation terms."""
    wl = syn.WORKLOADS[wl_id]
    b, d, r = wl.block, 128, (wl.rank_k, wl.rank_v)
    units = wl.n_layers * wl.batch * wl.n_kv_heads
    t1 = wl.window + b                        # exactly one fold
    first = sum(units * (4 * d * b * b - 4 * b ** 3 / 3 + 2 * b * b * b + 11 * b ** 3
                         + 2 * d * b * rr + 2 * b * d * rr) for rr in r)
    assert bench.fold_flops(wl, t1) == pytest.approx(first)
    t2 = t1 + b                               # a second fold, k = min(r, b), n_c = b
    second = 0.0
    for rr in r:
        k = min(rr, b)
        p = min(b, d - k)
        m, n = k + b, k + p
        second += units * (4 * b * d * k + 4 * d * b * p - 4 * p ** 3 / 3 + 2 * m * n * n
                           + 11 * n ** 3 + 2 * d * (k + p) * rr + 2 * b * k * rr + 2 * b * d * rr)
    assert bench.fold_flops(wl, t2) == pytest.approx(first + second)


def test_headline_step_holds_one_fold_of_every_unit():
    """A step is one fold period: exactly one block per unit crosses the window per step."""
    wl = bench.WL
    assert bench.TOK_PER_STEP == wl.block
    for t0 in (30000, 31999, 32640 - 128):
        assert wl.n_c(t0 + bench.TOK_PER_STEP) - wl.n_c(t0) == wl.block


def test_decode_bytes_counts_the_stored_factors():
    wl = bench.WL
    t = wl.tokens
    n = wl.n_c(t)
    per_unit = 4 * n * (32 + 64) + 2 * 2 * (t - n) * 128 + 4 * 128 * (32 + 64) + 2 * 4 * 4 * 128
    assert bench.decode_bytes(t) == 64 * per_unit
