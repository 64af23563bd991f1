"""Host logic of bench.py's timed region, on CPU with fakes: the NVML device is found by the
CUDA device's UUID (NVML numbers every GPU of the machine, CUDA only the visible ones), the
clock-event reasons are decoded from their bit mask, a region that saw a thermal or hardware
slowdown (or a median clock well below the maximum with no reason) is rejected and taken once
more, and with two gloo ranks both take the same number of replays when only one rank's record
is rejected."""
import os
import socket
import sys
import types

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def fake_nvml(uuids, mhz=1965, reasons=0, max_mhz=1965):
    """A stand-in for pynvml: device i has UUID uuids[i]; the clock and reasons are read from
    the module's attributes, so a test can change them while a sampler runs."""
    nv = types.SimpleNamespace(NVML_CLOCK_SM=1, mhz=mhz, reasons=reasons, inits=0)

    class NVMLError(Exception):
        pass

    def by_uuid(u):
        if u not in uuids:
            raise NVMLError("not found")
        return ("dev", uuids.index(u))

    def by_index(i):
        if not 0 <= i < len(uuids):
            raise NVMLError("bad index")
        return ("dev", i)

    def init():
        nv.inits += 1

    nv.nvmlInit = init
    nv.nvmlDeviceGetHandleByUUID = by_uuid
    nv.nvmlDeviceGetHandleByIndex = by_index
    nv.nvmlDeviceGetMaxClockInfo = lambda h, kind: max_mhz
    nv.nvmlDeviceGetClockInfo = lambda h, kind: nv.mhz
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: nv.reasons
    return nv


def test_nvml_device_found_by_uuid(monkeypatch):
    nv = fake_nvml(["GPU-aaaa", "GPU-bbbb", "GPU-cccc"])
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    s = bench.ClockSampler(0, uuid="bbbb")  # CUDA device 0 is the machine's GPU 1
    assert s.ok and s.h == ("dev", 1) and s.match == "uuid"
    s = bench.ClockSampler(0, uuid="GPU-cccc")
    assert s.h == ("dev", 2) and s.match == "uuid"
    s = bench.ClockSampler(1, uuid="dddd")  # unknown UUID: the index
    assert s.h == ("dev", 1) and s.match == "index"
    s = bench.ClockSampler(2)
    assert s.h == ("dev", 2) and s.match == "index"


def test_no_nvml_is_reported_not_guessed(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", None)  # import fails
    s = bench.ClockSampler(0)
    with s:
        pass
    assert not s.ok
    assert s.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}


def test_sampler_decodes_reasons(monkeypatch):
    nv = fake_nvml(["GPU-aaaa"], mhz=1800, reasons=0x4 | 0x40)  # sw_power_cap + hw_thermal_slowdown
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    with bench.ClockSampler(0, period=0.001, uuid="aaaa") as s:
        import time
        time.sleep(0.02)
    sm = s.summary()
    assert sm["sm_mhz"] == 1800 and sm["sm_max_mhz"] == 1965 and sm["samples"] >= 2
    assert sm["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert sm["nvml_device"] == "uuid"
    assert bench.ClockSampler.rejected(sm)


@pytest.mark.parametrize("summary,bad", [
    ({"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}, False),
    ({"sm_mhz": 1300, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}, False),  # kept and noted
    ({"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": ["hw_slowdown"]}, True),
    ({"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": ["sw_thermal_slowdown"]}, True),
    ({"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": ["gpu_idle", "hw_thermal_slowdown"]}, True),
    ({"sm_mhz": 1200, "sm_max_mhz": 1965, "reasons": []}, True),  # stuck low, no reason: a lock
    ({"sm_mhz": 1800, "sm_max_mhz": 1965, "reasons": []}, False),
    ({"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}, False),
])
def test_rejection_rule(summary, bad):
    assert bench.ClockSampler.rejected(summary) is bad


class FakeTorch:
    """torch.cuda's events and synchronize over a fake device clock that graph replays advance."""

    def __init__(self):
        self.now = 0.0
        self.syncs = 0
        fake = self

        class Event:
            def __init__(self, enable_timing=False):
                assert enable_timing
                self.at = None

            def record(self):
                self.at = fake.now

            def elapsed_time(self, other):
                return other.at - self.at

        def synchronize():
            fake.syncs += 1

        self.cuda = types.SimpleNamespace(Event=Event, synchronize=synchronize)


class FakeGraph:
    def __init__(self, t, durations):
        self.t, self.durations, self.replays = t, list(durations), 0

    def replay(self):
        self.t.now += self.durations[self.replays]
        self.replays += 1


def sampler_sequence(summaries):
    it = iter(summaries)

    class S:
        def __enter__(self):
            self.s = next(it)
            return self

        def __exit__(self, *a):
            return False

        def summary(self):
            return dict(self.s)

    return S


GOOD = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}
HOT = {"sm_mhz": 1600, "sm_max_mhz": 1965, "reasons": ["hw_thermal_slowdown"]}


def test_timed_replay_keeps_a_clean_region():
    t = FakeTorch()
    g = FakeGraph(t, [12.5, 99.0])
    ms, clocks = bench.timed_replay(t, g, "cpu", None, sampler_sequence([GOOD, GOOD]))
    assert ms == 12.5 and g.replays == 1 and clocks == GOOD


def test_timed_replay_retakes_a_rejected_region_once():
    t = FakeTorch()
    g = FakeGraph(t, [20.0, 12.5, 99.0])
    ms, clocks = bench.timed_replay(t, g, "cpu", None, sampler_sequence([HOT, GOOD, GOOD]))
    assert ms == 12.5 and g.replays == 2
    assert clocks["reasons"] == []
    assert clocks["rejected_runs"] == [{"ms": 20.0, "clocks": HOT, "on": "this rank"}]
    # rejected twice: the second is reported as it is, with its reasons, for the reader to judge
    t = FakeTorch()
    g = FakeGraph(t, [20.0, 21.0, 99.0])
    ms, clocks = bench.timed_replay(t, g, "cpu", None, sampler_sequence([HOT, HOT, GOOD]))
    assert ms == 21.0 and g.replays == 2 and clocks["reasons"] == ["hw_thermal_slowdown"]
    assert len(clocks["rejected_runs"]) == 1


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench as b
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = FakeTorch()
        g = FakeGraph(t, [10.0 + rank, 11.0 + rank, 99.0])
        seq = [GOOD, GOOD] if rank == 0 else [HOT, GOOD]  # only rank 1 saw a slowdown
        ms, clocks = b.timed_replay(t, g, "cpu", dist, sampler_sequence(seq))
        q.put((rank, g.replays, ms, [r["on"] for r in clocks.get("rejected_runs", [])]))
    finally:
        dist.destroy_process_group()


def test_ranks_agree_on_a_retake_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    # both ranks replay twice (same collective steps on every rank) and keep the second replay;
    # rank 0's clean first replay is dropped because rank 1's was rejected
    assert got == [(0, 2, 11.0, ["another rank"]), (1, 2, 12.0, ["this rank"])]


def test_oracle_baseline_on_several_threads():
    """The CPU baseline runs the oracle on independent row slices in several host threads at
    once; each thread's slices are its own and the bytes add up over all of them."""
    import numpy as np
    pool = [np.zeros((32, 2560), dtype=np.uint16), np.zeros((32, 9728), dtype=np.uint16)]  # bf16 bits
    v1, i1 = bench.oracle_throughput(pool, budget_s=0.05)
    v2, i2 = bench.oracle_throughput(pool, budget_s=0.05, threads=2)
    assert i1["threads"] == 1 and i2["threads"] == 2
    assert v1 > 0 and v2 > 0 and i2["samples"] >= 2
    assert i1["elements"] == sum(pool[k % 2].size for k in range(i1["samples"]))
    assert 1 <= bench.cpu_threads() <= 32


def test_oracle_pool_holds_the_workload_bits():
    """The baseline's slices are rows of the decoder stack exactly as the generator draws them."""
    import numpy as np
    import synthetic
    pool = bench.oracle_pool(n_slices=2, rows=2)
    cols = {c for _, _, c in synthetic.DECODER_LAYER}
    for xs in pool:
        assert xs.dtype == np.uint16 and xs.shape[0] == 2 and xs.shape[1] in cols
    # the first slice against the full tensor it was cut from
    rng = np.random.default_rng(12345)
    layer = int(rng.integers(synthetic.N_LAYERS))
    k = int(rng.integers(len(synthetic.DECODER_LAYER)))
    _, nrows, cols = synthetic.DECODER_LAYER[k]
    r0 = int(rng.integers(nrows - 2 + 1))
    w = synthetic.decoder_weight(layer, k)
    assert np.array_equal(pool[0], w[r0:r0 + 2])


def test_stack_step_bytes_are_the_survey_figures():
    """Per layer 280 698 880 B to MXFP6 E2M3 and 283 852 800 B to AXS-6 (values in + codes +
    scales), 36 layers per step."""
    b, n = bench.stack_step_bytes()
    assert n == 36 * 100925440
    assert b == 36 * (280698880 + 283852800)


def test_timed_region_with_a_set_status_word_reports_nothing():
    """The status check runs after every timed region; when it raises (a bounded wait ran out,
    so some outputs are incomplete), the exception leaves timed_replay and no time is returned."""
    t = FakeTorch()
    g = FakeGraph(t, [12.5, 99.0])

    class Timeout(RuntimeError):
        pass

    def check():
        raise Timeout("MXQ_ERR_TIMEOUT")

    with pytest.raises(Timeout):
        bench.timed_replay(t, g, "cpu", None, sampler_sequence([GOOD, GOOD]), after=check)
    calls = []
    ms, _ = bench.timed_replay(t, FakeGraph(t, [3.0, 4.0, 99.0]), "cpu", None, sampler_sequence([GOOD]),
                               replays=2, after=lambda: calls.append(1))
    assert ms == 7.0 and calls == [1]  # K replays in one region, one check after it
