"""Host-side pieces of bench.py that need no GPU: the key that ties the
recorded ncu traffic to the kernel code, and the byte model's write
reduction on every workload (the C/2 bar of the measurement)."""
import os

import pytest

import bench
from recurrent_state_head_b200 import synth

CODE = """// a comment
__device__ float f(float x) {   /* block
   comment */ return x * 2.f; }
"""


def test_code_digest_ignores_comments_and_blank_space(tmp_path):
    a, b, c = tmp_path / "a.cuh", tmp_path / "b.cuh", tmp_path / "c.cuh"
    a.write_text(CODE)
    b.write_text(CODE.replace("// a comment", "// another comment\n\n").replace("   ", " "))
    c.write_text(CODE.replace("2.f", "3.f"))
    assert bench.kernel_source_digest(str(a)) == bench.kernel_source_digest(str(b))
    assert bench.kernel_source_digest(str(a)) != bench.kernel_source_digest(str(c))


def test_recorded_traffic_follows_the_committed_profile():
    """While the committed append summary was taken on the current kernel
    code, the bench reports its traffic, within a few percent of the
    algorithmic bytes of one launch at the cycle's mean log length; once the
    code has changed since, the bench reports none."""
    import re
    w = synth.WORKLOADS["gdn-b128-h16-d128-c8"]
    prof = os.path.join(bench.ROOT, "profiles", f"append_kernel_{w.name}.md")
    src = os.path.join(bench.ROOT, "recurrent_state_head_b200", "csrc", "kernels.cuh")
    m = re.search(r"kernel_code_sha256:\s*([0-9a-f]{64})", open(prof).read())
    t = bench.recorded_traffic(w.name)
    if m and m.group(1) == bench.kernel_source_digest(src):
        bm = bench.bytes_model(w)
        algo = w.heads * sum(bm["append"](3))
        assert t is not None and 0.95 < t / algo < 1.1
    else:
        assert t is None


def test_recorded_traffic_absent_for_unprofiled_workload():
    assert bench.recorded_traffic("no-such-workload") is None


@pytest.mark.parametrize("name", [n for n in synth.WORKLOADS if "stack24" not in n or "b128" in n])
def test_write_reduction_meets_half_capacity(name):
    w = synth.WORKLOADS[name]
    bm = bench.bytes_model(w)
    ratio = bm["eager"][1] / bm["token_write"]
    assert ratio >= w.C / 2, (name, ratio)
    # the merge-token never writes more than the separate merge
    assert bm["token_write"] <= bench.bytes_model(w, fold=False)["token_write"]


def test_config_object_and_l2_wording():
    """Both arms print the same config object; a working set below the
    126 MB L2 is labelled as such."""
    big = synth.WORKLOADS["gdn-b128-h16-d128-c8"]
    small = synth.WORKLOADS["gdn-b1-h2-d64-c4-fp32"]
    cb = bench.workload_config(big, 4, 1)
    assert cb["workload"] == big.name and cb["layers_rotated"] == 4
    assert cb["l2"].startswith("inputs larger than L2")
    assert "fits in L2" in bench.workload_config(small, 4, 1)["l2"]
    assert set(cb) == set(bench.workload_config(small, 4, 1))


@pytest.mark.parametrize("name", ["gdn-b128-h16-d128-c8", "kda-b128-h32-d128-c4",
                                  "rwkv6-b128-h32-d64-c8"])
def test_device_drawn_timing_inputs(name):
    """The sweep's device-drawn states and tokens have the workload's shapes,
    dtypes and distributions (checked on the CPU generator)."""
    import torch
    from recurrent_state_head_b200 import device as D
    w = synth.WORKLOADS[name].with_(B=4)
    g = torch.Generator(device="cpu")
    g.manual_seed(1)
    S = D.draw_state(w, 0, "cpu", g)
    assert S.shape == (w.heads, w.dk, w.dv) and S.dtype == torch.float32
    assert abs(float(S.std()) - w.init_std) < 0.1 * w.init_std
    x = D.draw_tokens(w, 3, "cpu", g)
    assert x["q"].shape == (3, w.heads, w.dk) and x["v"].shape == (3, w.heads, w.dv)
    assert x["g"].shape == (3, w.heads, w.m) and x["beta"].shape == (3, w.heads)
    assert x["q"].dtype == D.TORCH_DTYPE[w.in_dtype]
    assert bool((x["g"] < 0).all())
    if w.op == synth.RWKV6:
        assert bool((x["beta"] == 0).all())
    else:
        norms = x["k"].float().norm(dim=-1)
        assert bool(((norms - 1).abs() < 1e-2).all())
        assert bool(((x["beta"] > 0) & (x["beta"] < 1)).all())


class _FakeNVML:
    """Stands in for pynvml: a GPU whose (SM clock, clock-event reasons)
    samples follow a script, the last entry repeating."""
    NVML_CLOCK_SM = 1

    def __init__(self, script):
        self.script = list(script)
        self.calls = 0

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByUUID(self, uuid):
        return "h"

    def nvmlDeviceGetHandleByIndex(self, i):
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        return self.script[min(self.calls, len(self.script) - 1)][0]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        r = self.script[min(self.calls, len(self.script) - 1)][1]
        self.calls += 1
        return r


def test_clock_sampler_with_fake_nvml(monkeypatch):
    """The sampler has its first sample before the timed region starts,
    drops idle samples from the median and reports every reason seen."""
    import sys
    import time
    import torch
    fake = _FakeNVML([(345, 0x1)] + [(1800, 0x4)] * 4 + [(1965, 0x0)])
    monkeypatch.setitem(sys.modules, "pynvml", fake)

    class Props:
        uuid = "0000"
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda d: Props())

    class Dev:
        index = 0
    with bench.ClockSampler(Dev(), period_s=0.001) as clk:
        assert len(clk.samples) >= 1            # taken before the region
        t0 = time.time()
        while fake.calls < 16 and time.time() - t0 < 5:
            time.sleep(0.002)
    s = clk.summary()
    assert s["sm_max_mhz"] == 1965
    assert s["samples"] >= 10
    assert s["sm_mhz"] == 1965                  # idle sample left out
    assert s["reasons"] == ["sw_power_cap"]


def test_reference_arm_line(monkeypatch, capsys):
    """`--impl reference` (the oracle on the host cores) prints one JSON line
    with the native arm's config object and the contract's keys; under a
    launcher, ranks other than 0 print nothing and return."""
    import json
    w = "gdn-b1-h2-d64-c4-fp32"
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--workload", w, "--steps", "1", "--warmup", "3"])
    assert capsys.readouterr().out == ""
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    bench.main(["--impl", "reference", "--workload", w, "--steps", "1", "--warmup", "3"])
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    r = json.loads(lines[0])
    assert r["impl"] == "reference" and r["value"] > 0 and r["unit"] == "tok/s"
    assert r["config"] == bench.workload_config(synth.WORKLOADS[w], 4, 1)
    assert r["cpu_baseline"]["kind"] == "oracle" and r["cpu_baseline"]["cores"] >= 1
    assert r["e2e"] == {"value": r["value"], "unit": "tok/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    for k in ("metric", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data"):
        assert k in r


def test_cold_rotation_reaches_four_times_l2():
    """Every workload's cold figures rotate enough layers that the working
    set is at least 4x the L2; a layer that fits in L2 also gets a hot
    figure."""
    for name in (bench.DEFAULT_WORKLOAD,) + bench.EXTRA_WORKLOADS:
        w = synth.WORKLOADS[name]
        R = bench.cold_layers(w, 4)
        assert R >= 4
        assert bench.working_set(w, R) >= 4 * bench.L2_BYTES
        assert R == 4 or bench.working_set(w, R - 1) < 4 * bench.L2_BYTES
    assert bench.cold_layers(synth.WORKLOADS["rwkv6-b128-h32-d64-c8"], 4) == 7
    assert bench.working_set(synth.WORKLOADS["rwkv6-b128-h32-d64-c8"], 1) < bench.L2_BYTES
