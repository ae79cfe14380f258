"""Host-side logic of bench.py that needs no GPU: the clock record and the roofline byte counts."""
import os
import sys
import time

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


class FakeNvml:
    """Stands in for pynvml: a clock that steps through a list and fixed reason bits."""
    NVML_CLOCK_SM = 1

    def __init__(self, clocks, bits=0):
        self.clocks, self.bits, self.i = list(clocks), bits, 0

    def nvmlDeviceGetClockInfo(self, h, which):
        assert h == "gpu0" and which == 1
        v = self.clocks[min(self.i, len(self.clocks) - 1)]
        self.i += 1
        return v

    def nvmlDeviceGetMaxClockInfo(self, h, which):
        return 1965

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.bits


def test_summary_keeps_only_the_window():
    samples = [(0.0, 500, 0x1), (1.0, 1965, 0), (1.5, 1900, 0x4), (2.0, 1965, 0), (3.0, 300, 0x40)]
    s = bench.nvml_clock_summary(samples, (1.0, 2.0), 1965)
    assert s == {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"], "samples": 3}
    assert bench.nvml_clock_summary(samples, (5.0, 6.0), 1965) is None
    assert bench.nvml_clock_summary(samples, (None, None), 1965) is None


def test_every_reason_bit_is_named():
    bits = 0x8 | 0x40 | 0x20 | 0x4
    s = bench.nvml_clock_summary([(1.0, 1000, bits)], (0.0, 2.0), 1965)
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap", "sw_thermal_slowdown"]
    # idle (0x1) and application-clock (0x2) bits are not throttle reasons
    assert bench.nvml_clock_summary([(1.0, 1000, 0x3)], (0.0, 2.0), 1965)["reasons"] == []


def test_sample_loop_writes_parseable_lines(tmp_path):
    nv = FakeNvml([1965, 1950, 1965], bits=0x4)
    path = tmp_path / "s.txt"
    n = [0]

    def stop():
        n[0] += 1
        return n[0] > 3

    with open(path, "w") as f:
        f.write("max 1965\n")
        bench.nvml_sample_loop(nv, "gpu0", 0.0, f, stop)
        f.write("123.5 19")  # a line the sampler had not finished when it was ended
    samples, mx = bench.read_nvml_samples(str(path))
    assert mx == 1965
    assert [s[1:] for s in samples] == [(1965, 4), (1950, 4), (1965, 4)]
    assert samples[0][0] <= samples[1][0] <= samples[2][0]
    s = bench.nvml_clock_summary(samples, (samples[0][0], samples[-1][0]), mx)
    assert s == {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"], "samples": 3}


def test_sampler_process_without_a_gpu_ends_and_falls_back(tmp_path):
    # no driver here: the sampler process fails to start NVML and exits; the bench goes on with the
    # nvidia-smi record and never waits for the sampler's full start-up limit
    class Smi:
        def summary(self):
            return {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": [], "samples": 2}

    t0 = time.monotonic()
    with bench.NvmlClocks(("GPU-00000000-0000-0000-0000-000000000000", "00000000:00:00.0"),
                          path=str(tmp_path / "n.txt"), start_timeout=60.0) as c:
        c.mark_start()
        c.mark_end()
    assert time.monotonic() - t0 < 30.0
    assert c.proc is not None and c.proc.returncode is not None
    r = bench.clocks_record(c, Smi())
    assert r["samples"] == 2 and r["source"].startswith("nvidia-smi")


FAKE_PYNVML = """
NVML_CLOCK_SM = 1
def nvmlInit(): pass
def nvmlDeviceGetHandleByUUID(u):
    if u != "GPU-fake":
        raise RuntimeError("no such uuid")
    return 7
def nvmlDeviceGetHandleByPciBusId(b): return 7
def nvmlDeviceGetMaxClockInfo(h, w): return 1965
def nvmlDeviceGetClockInfo(h, w): return 1950
def nvmlDeviceGetCurrentClocksEventReasons(h): return 4
"""


def test_sampler_process_records_the_window(tmp_path, monkeypatch):
    # the whole sampler path, process included, against a fake NVML module found first on its path
    (tmp_path / "pynvml.py").write_text(FAKE_PYNVML)
    monkeypatch.setenv("PYTHONPATH", str(tmp_path))
    with bench.NvmlClocks(("GPU-fake", "00000000:00:00.0"), path=str(tmp_path / "n.txt")) as c:
        assert c.proc is not None and c.proc.poll() is None
        c.mark_start()
        time.sleep(0.1)
        c.mark_end()
    s = c.summary()
    assert s["sm_mhz"] == 1950 and s["sm_max_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"]
    assert s["samples"] >= 5
    assert not (tmp_path / "n.txt").exists() or os.environ.get("CSA2_CLOCKS_DIR")


def test_without_device_properties_no_sampler_starts():
    with bench.NvmlClocks(None) as c:
        c.mark_start()
        c.mark_end()
    assert c.proc is None and c.summary() is None


def test_record_prefers_the_samples_inside_the_region():
    class Smi:
        def summary(self):
            return {"sm_mhz": 1200, "sm_max_mhz": 1965, "reasons": [], "samples": 1}

    class Nvml:
        def summary(self):
            return bench.nvml_clock_summary([(1.0, 1965, 0)], (0.5, 1.5), 1965)

    r = bench.clocks_record(Nvml(), Smi())
    assert r["sm_mhz"] == 1965 and r["samples"] == 1 and r["smi_samples"] == 1 and r["smi_sm_mhz"] == 1200


def test_reindex_algorithmic_bytes_per_query():
    import workloads as W

    wl = W.WORKLOADS["reindex_b128_n1m"]
    ab = bench.algorithmic_bytes(wl)
    # 2000 pool blocks x 8 positions x 144 B indexer rows + pool ids + count + indexer query + indices
    assert ab["index"] == 2000 * 8 * 144 + 2000 * 4 + 4 + 4 * 64 * 2 + 512 * 4 == 2314564
    # 512 FP4 rows x 144 B + 128 window rows x 256 B + q + indices + out
    assert ab["attend"] == 512 * 144 + 128 * 256 + 4096 + 2048 + 4096


@pytest.mark.parametrize("v,expect", [(1.0, 1), (-3.5, -3.5)])
def test_reduce_max_single_rank_is_identity(v, expect):
    assert bench.reduce_max(v, "cpu", 1) == expect


def test_draft_rows_share_one_pass_over_the_keys():
    import workloads as W

    wl = W.WORKLOADS["draft_b64_n131072_tq5"]
    ab = bench.algorithmic_bytes(wl)
    # per step and sequence: every visible indexer row once, plus each row's query and indices
    assert ab["index"] * wl.tq == 131072 * 144 + 5 * (4 * 64 * 2 + 512 * 4)
    assert bench.e2e_call("draft").startswith("csa2_quantize_append")
    assert bench.e2e_call("reindex") == "csa2_decode_reindex"


def test_latent_workloads_bytes_flops_and_calls():
    """The pages' own shapes: the latent attention reads k latent entries (256 + 32 B), the window
    rows (512 B), q and writes out (64 x 512 bf16 each) and reads the indices; its two contractions
    take 2 x 2 x 64 x 512 flops per key. The indexer reads every visible MXFP4 key (68 B), its query
    (32 x 128 bf16) and position, and writes k indices."""
    import workloads as W

    wl = W.WORKLOADS["latent_b128_n131072"]
    assert bench.algorithmic_bytes(wl) == {"append": 0, "index": 0, "attend": 346112}
    assert 512 * 288 + 128 * 512 + 2 * 65536 + 2048 == 346112
    assert bench.latent_flops(wl) == 4 * 64 * 512 * 640
    assert bench.kernels_per_step(wl) == 1 and bench.e2e_call("latent") == "csa2_latent_attend"
    wi = W.WORKLOADS["latent_index_b128_n131072"]
    assert bench.algorithmic_bytes(wi)["index"] == 131072 * 68 + 32 * 128 * 2 + 8 + 512 * 4
    assert bench.kernels_per_step(wi) == 3 and bench.e2e_call("latent_index") == "csa2_latent_index_topk"
