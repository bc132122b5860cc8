"""Host-side helpers of bench.py: the packed per-step input buffer that the
end-to-end leg copies host -> device in one transfer."""
import importlib.util
import os

import numpy as np
import pytest
import torch

import fixtures

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_host", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


@pytest.mark.parametrize("T,H,k", [(1, 2048, 10), (64, 2048, 10), (7, 768, 16), (1, 256, 4)])
def test_packed_inputs_round_trip(bench, T, H, k):
    x = fixtures.make_x(31, T, H)
    st = fixtures.Stream(31, 5)
    ids = st.randint(T * k, 512).astype(np.int32).reshape(T, k)
    wt = st.uniform(T * k).astype(np.float32).reshape(T, k)
    pk = bench.pack_inputs(x, ids, wt)
    assert pk.dtype == np.uint8 and pk.nbytes == x.nbytes + ids.nbytes + wt.nbytes
    vx, vi, vw = bench.input_views(torch.from_numpy(pk), T, H, k)
    assert vx.dtype == torch.float32 and vi.dtype == torch.int32 and vw.dtype == torch.float32
    assert vx.is_contiguous() and vi.is_contiguous() and vw.is_contiguous()
    assert np.array_equal(vx.numpy(), x) and np.array_equal(vi.numpy(), ids) and np.array_equal(vw.numpy(), wt)
    # x leads the buffer; ids and weights start on 4-byte boundaries
    assert vi.data_ptr() - vx.data_ptr() == x.nbytes and (vw.data_ptr() - vx.data_ptr()) % 4 == 0


def test_steps_are_fixed_graph_replays(bench):
    """A step is a fixed number of layer calls, so --steps K times exactly K steps."""
    for cfg in (2, 3, 4, 5):
        assert bench.calls_per_step(cfg) == bench.GRAPH_CALLS[cfg] * bench.REPLAYS_PER_STEP[cfg]
    assert bench.calls_per_step(2) % bench.N_SETS == 0  # whole passes over the 48 disjoint decode sets


def test_clock_summary_uses_the_timed_window(bench):
    import datetime

    def row(t, mhz, cap="Not Active"):
        ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return [ts, "0", str(mhz), "1965", "700.0", "0x0", "Not Active", "Not Active", "Not Active", cap]

    rows = [row(100.0, 600), row(100.5, 1965, "Active"), row(100.6, 1965, "Active"), row(101.5, 700)]
    s = bench.ClockSampler.summarise(rows, (100.4, 100.7))
    assert s["sm_mhz"] == 1965 and s["samples_in_window"] == 2 and s["reasons"] == ["sw_power_cap"]
    s = bench.ClockSampler.summarise(rows, (200.0, 201.0))  # window too short for a sample: all rows
    assert s["samples_in_window"] == 0 and s["samples"] == 4
