"""Host-side rules of bench.py and of the committed profile summaries.

* A DRAM-traffic figure from an ncu capture is reported only while the
  kernel sources still hash to the capture's source hash; after any kernel
  change the bench reports traffic as null.
* Every profile summary gives the command that produced it: ncu with
  --clock-control none, running bench.py (a committed file) with options the
  bench accepts, and each workload it names exists.
"""
import glob
import json
import os
import re
import shlex

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_traffic_only_for_matching_sources(monkeypatch):
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    wl, kernels = next(iter(t.items()))
    kernel, entry = next(iter(kernels.items()))
    monkeypatch.setattr(bench, "kernel_source_sha", lambda k: entry["source_sha"])
    assert bench.profiled_traffic(kernel, wl) == entry["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "kernel_source_sha", lambda k: "0" * 16)
    assert bench.profiled_traffic(kernel, wl) is None
    # an unprofiled kernel or workload has no figure
    assert bench.profiled_traffic("gemm", "no_such_workload") is None


@pytest.mark.parametrize("kernel", sorted(bench.KERNEL_SOURCES))
def test_source_hash_covers_every_file_of_the_kernel(tmp_path, monkeypatch, kernel):
    """A kernel's hash changes when any file it is built from changes, and
    only then."""
    src = os.path.join(ROOT, "w8a8_int8_quantized_rmsnorm_b200", "csrc")
    fake = tmp_path / "w8a8_int8_quantized_rmsnorm_b200" / "csrc"
    fake.mkdir(parents=True)
    for name in sorted(os.listdir(src)):
        with open(os.path.join(src, name), "rb") as f:
            (fake / name).write_bytes(f.read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_sha(kernel)
    for name in sorted(os.listdir(fake)):
        before = (fake / name).read_bytes()
        (fake / name).write_bytes(before + b"\n")
        changed = bench.kernel_source_sha(kernel) != h0
        assert changed == (name in bench.KERNEL_SOURCES[kernel]), name
        (fake / name).write_bytes(before)
    assert bench.kernel_source_sha(kernel) == h0


def test_replay_count_bounds():
    # one rank: enough replays for MIN_TIMED_MS, within the bounds
    assert bench.agreed_replays(1000.0, 1, "cpu") == bench.MIN_REPLAYS
    assert bench.agreed_replays(bench.MIN_TIMED_MS / 20, 1, "cpu") == 20
    assert bench.agreed_replays(1e-6, 1, "cpu") == bench.MAX_REPLAYS


def _commands(text):
    """The shell commands of a summary: indented lines, backslash-joined."""
    lines, cur = [], ""
    for ln in text.splitlines():
        if not ln.startswith("    "):
            if cur:
                lines.append(cur)
                cur = ""
            continue
        part = ln.strip()
        cur = (cur + " " + part[:-1].strip()) if part.endswith("\\") else (cur + " " + part)
        if not part.endswith("\\"):
            lines.append(cur.strip())
            cur = ""
    return [c for c in lines if c]


@pytest.mark.parametrize("path", sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))),
                         ids=os.path.basename)
def test_profile_commands_run_committed_files(path, monkeypatch):
    with open(path) as f:
        cmds = _commands(f.read())
    ncu = [c for c in cmds if "ncu " in c]
    assert ncu, "a profile summary names the ncu command that produced it"
    for c in ncu:
        assert "--clock-control none" in c
        prog = re.split(r"\s[>&|]", c[c.index("python "):])[0]
        argv = shlex.split(prog)
        assert argv[1] == "bench.py" and os.path.exists(os.path.join(ROOT, argv[1]))
        # the bench accepts the options (argparse exits on an unknown one)
        monkeypatch.setattr("sys.argv", argv[1:])
        args = bench.parse()
        assert args.workload in bench.workloads.WORKLOADS


def test_cpu_baseline_reports_all_cores_and_one_thread():
    """The oracle's CPU baseline, on a tiny budget: the multi-threaded figure
    and the single-thread one, both in tokens/s of the workload."""
    w = bench.workloads.WORKLOADS["single_linear_m32"]
    r = bench.cpu_baseline(w, target_s=0.2, single_s=0.2)
    assert r["kind"] == "oracle" and r["unit"] == "tokens/s" and r["value"] > 0
    assert r["cores"] >= 1
    assert r["single_thread"]["cores"] == 1 and r["single_thread"]["value"] > 0


def test_clock_summary_counts_only_the_timed_region():
    """Samples before and after the timed region (idle clocks) are left out;
    the throttle reasons are those seen inside it."""
    def line(mhz, cap):
        return f"0, {mhz}, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, {cap}"
    lines = [(0.5, line(1965, "Not Active")), (1.0, line(1440, "Active")),
             (1.1, line(1425, "Active")), (1.2, line(1455, "Not Active")),
             (2.5, line(1965, "Not Active")), (3.0, "garbage")]
    r = bench.summarize_clocks(lines, 0.9, 2.0)
    assert r["samples"] == 3 and r["sm_mhz"] == 1440.0 and r["sm_min_mhz"] == 1425.0
    assert r["reasons"] == ["sw_power_cap"] and r["sm_max_mhz"] == 1965.0
    assert bench.summarize_clocks(lines)["samples"] == 5
