"""The commands written in profiles/ still name things that exist: every
kernel_cases case they run is one the harness knows and dispatches, every
bench.py flag is one bench.py parses, and every --workload is a workload of
synth.WORKLOADS; so each summary's command can be run again as written."""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _profiles_text():
    return "\n".join(open(p, encoding="utf-8").read() for p in glob.glob(os.path.join(ROOT, "profiles", "*.md")))


def test_kernel_cases_named_in_profiles_exist():
    from flow_matching_video_b200 import kernel_cases
    src = open(os.path.join(ROOT, "flow_matching_video_b200", "kernel_cases.py"), encoding="utf-8").read()
    body = src[src.index("def make_case"):]
    for case in kernel_cases.CASES:   # each listed case is dispatched by make_case
        assert f'"{case}"' in body, case
    used = set(re.findall(r"kernel_cases ([a-z][a-z0-9_]*)", _profiles_text()))
    assert used and used <= set(kernel_cases.CASES), used - set(kernel_cases.CASES)


def test_bench_flags_and_workloads_named_in_profiles_exist():
    from flow_matching_video_b200 import synth
    text = _profiles_text()
    bench_src = open(os.path.join(ROOT, "bench.py"), encoding="utf-8").read()
    flags = set()
    for line in re.findall(r"bench\.py[^\n|`]*", text):
        flags |= set(re.findall(r"(--[a-z0-9-]+)", line))
    assert flags
    for f in flags:
        assert f'"{f}"' in bench_src, f
    for wl in set(re.findall(r"--workload ([A-Za-z0-9_-]+)", text)):
        assert wl in synth.WORKLOADS, wl
