"""The committed ncu summaries: each names the command that made it and only
committed files; the bench's roofline reads DRAM traffic from one of them."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")


def test_every_summary_states_its_command_and_runs_committed_files_only():
    names = sorted(os.listdir(PROFILES))
    assert names
    for name in names:
        assert name.endswith((".txt", ".md")), name
        text = open(os.path.join(PROFILES, name)).read()
        assert "command" in text, f"{name} gives no command"
        assert "_work/" not in text and "/root/" not in text, f"{name} names a scratch or machine path"
        assert len(text) < 16_000, f"{name} is not a short summary"


def test_bench_profile_carries_sha_and_traffic():
    text = open(os.path.join(PROFILES, "k_fused_cluster_n128_p128.txt")).read()
    assert re.search(r"^kernel_source_sha: [0-9a-f]{16}$", text, re.M)
    assert re.search(r"^dram_bytes_per_launch: \d+$", text, re.M)
