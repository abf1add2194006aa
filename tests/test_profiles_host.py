"""The bench's per-kernel DRAM traffic figures are the ones the committed
one-kernel ncu summaries report (the first figure of each summary is the
default kernel's), and every summary names the command that made it."""
import os
import re

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")
FILES = {
    "tc_prep": "ncu_tc_prep_h16_t8k.md",
    "tc_scan_fwd": "ncu_tc_scan_fwd_h16_t8k.md",
    "tc_out_og": "ncu_tc_out_og_h16_t8k.md",
    "tc_scan_bwd": "ncu_tc_scan_bwd_h16_t8k.md",
    "tc_grad": "ncu_tc_grad_h16_t8k.md",
}


def test_bench_traffic_matches_the_profiles():
    assert set(bench.MEASURED_TRAFFIC) == set(FILES)
    for kernel, name in FILES.items():
        text = open(os.path.join(PROFILES, name)).read()
        m = re.search(r"\((\d+) B per chunk-head\)", text)
        assert m, name
        assert float(m.group(1)) == bench.MEASURED_TRAFFIC[kernel], (kernel, m.group(1))


def test_every_summary_gives_its_command():
    for name in sorted(os.listdir(PROFILES)):
        text = open(os.path.join(PROFILES, name)).read()
        assert "--clock-control none" in text, name
        assert "python bench.py" in text, name
