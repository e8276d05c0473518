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


def test_decode_traffic_is_reported_only_for_the_current_sources():
    """bench.py takes a kernel's DRAM traffic from its committed summary only
    while the CUDA sources hash to the value recorded there; otherwise the
    line's traffic is null (the counters no longer describe the kernel)."""
    for kind in ("lod_decode", "lod_decode_int4"):
        path = os.path.join(PROFILES, "%s_decode_gqa_128k_bf16.md" % kind)
        text = open(path).read()
        rec = re.search(r"csrc_sha256:\s*(\w+)", text)
        val = re.search(r"traffic_bytes_per_launch:\s*(\d+)", text)
        files = re.search(r"csrc_files:\s*(.+)", text)
        assert rec and val and files, path
        assert 10_000_000 < int(val.group(1)) < 1_000_000_000
        t = bench.profiled_traffic(kind, "decode_gqa_128k_bf16")
        if rec.group(1) == bench.csrc_hash(files.group(1).split()):
            assert t == int(val.group(1))
        else:
            assert t is None


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
