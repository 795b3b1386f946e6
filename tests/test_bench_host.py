"""Host logic of bench.py (CPU only): the launch count it claims, the radix
pass count, the clock-sample parsing and the traffic lookup that is only
trusted while the profiled kernel source is unchanged."""
import hashlib
import json
import os

import pytest

import bench
from atomic_expert_layer_b200 import configs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("G,passes", [(1, 0), (2, 1), (256, 1), (257, 2), (13285, 2),
                                      (65536, 2), (65537, 3)])
def test_radix_passes(G, passes):
    assert bench.radix_passes(G) == passes


def test_launches_per_step_matches_the_profiled_step():
    # the headline step in the committed launch list: GEMM, two axis kernels,
    # merge, scan, two radix scatters, histogram scan, group pass, token pass
    assert bench.launches_per_step(configs.HEADLINE) == 10
    # decode batches (L <= 16) run the whole step as one cooperative launch
    assert bench.launches_per_step(configs.sweep(16)) == 1
    assert bench.launches_per_step(configs.sweep(1)) == 1
    # the skewed layer adds the tensor-core expert path: 8 launches
    # (use, mark, scan, list, gather, split, two GEMMs); its 8192 groups need
    # two radix passes, like the headline
    assert bench.launches_per_step(configs.SKEW) == 10 + 8


def test_clock_summary_reads_reasons_and_load_median(tmp_path):
    s = bench.ClockSampler(0)
    s.path = str(tmp_path / "clocks.csv")
    with open(s.path, "w") as f:
        f.write("0, 1965, 1965, 120.0, 0x0, Not Active, Not Active, Not Active, Not Active\n")
        f.write("0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n")
        f.write("0, 1700, 1965, 1000.0, 0x4, Not Active, Not Active, Not Active, Active\n")
        f.write("garbage line\n")
    out = s.summary()
    assert out["samples"] == 3 and out["samples_under_load"] == 2
    assert out["sm_mhz"] == pytest.approx(1750.0)           # median of the loaded samples
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]
    assert not os.path.exists(s.path)                         # the sample file is removed


def test_traffic_only_for_the_profiled_source(tmp_path):
    # the committed capture is trusted only for the source whose hash it
    # records; any other source (e.g. a later edit) gives no traffic figure
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))["grouped_expert_stage"]
    src = os.path.join(ROOT, "atomic_expert_layer_b200", "csrc", "expert.cu")
    cur = open(src, "rb").read()
    got = bench.traffic_from_profile(src)
    if hashlib.sha256(cur).hexdigest() == rec["source_sha256"]:
        assert got == rec["dram_bytes_per_launch_full_size"] and got > 1e9
    else:
        assert got is None
    other = tmp_path / "expert.cu"
    other.write_bytes(cur + b"\n// changed\n")
    assert bench.traffic_from_profile(str(other)) is None
