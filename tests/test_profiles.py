"""The committed ncu summaries: readable, current, and reproducible from
committed files.

`bench.py` reports a kernel's DRAM traffic only from a summary captured from
the current CUDA sources; these checks fail when a kernel source changes and
the traffic figures are not captured again."""
import os
import re

import bench

PROFILES = os.path.join(bench.ROOT, "profiles")


def _summaries():
    return sorted(f for f in os.listdir(PROFILES) if f.endswith((".md", ".txt")))


def test_decode_traffic_matches_the_current_sources():
    for kind in ("lod_decode", "lod_decode_int4"):
        t = bench.profiled_traffic(kind, "decode_gqa_128k_bf16")
        assert t is not None, "%s traffic was captured from other CUDA sources" % kind
        assert 10_000_000 < t < 1_000_000_000


def test_summaries_run_committed_files_only():
    for f in _summaries():
        text = open(os.path.join(PROFILES, f)).read()
        assert "_work" not in text, f
        # every capture names its command, and every command gives --clock-control none
        joined = re.sub(r"\\\n\s*", " ", text)  # shell line continuations
        cmds = [ln.strip() for ln in joined.splitlines() if re.match(r"\s*ncu\s", ln)]
        assert cmds, "%s names no ncu command" % f
        for ln in cmds:
            assert "--clock-control none" in ln, (f, ln)
        # the programs the commands run are committed files of this repository
        for script in re.findall(r"\bpython3? ([\w./-]+\.py)\b", joined):
            assert os.path.exists(os.path.join(bench.ROOT, script)), (f, script)


def test_summaries_are_short_text():
    for f in os.listdir(PROFILES):
        assert f.endswith((".md", ".txt")), f
        assert os.path.getsize(os.path.join(PROFILES, f)) < 16 * 1024, f
