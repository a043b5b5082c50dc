"""The committed ncu summaries that bench.py reads, and its mirror of a library
default (CPU only).

bench.py takes `roofline.traffic` from a summary's machine-readable block only
while the kernel's sources hash to the value recorded there; these checks keep
the blocks well formed and the rule itself honest.
"""
import re
from pathlib import Path

import bench

ROOT = Path(__file__).resolve().parents[1]
PROFILES = sorted((ROOT / "profiles").glob("*.md"))


def blocks():
    for f in PROFILES:
        text = f.read_text()
        if "machine-readable" not in text:
            continue
        kv = dict(re.findall(r"^(kernel|dram_bytes_per_launch|source_sha256): (.+)$", text, re.M))
        yield f, kv


def test_profiles_are_short_text_with_their_command():
    assert PROFILES
    for f in PROFILES:
        assert f.stat().st_size < 16 * 1024, f.name
        text = f.read_text()
        assert "ncu " in text and "--clock-control none" in text, f.name


def test_machine_readable_blocks_are_well_formed():
    seen = 0
    for f, kv in blocks():
        seen += 1
        assert set(kv) == {"kernel", "dram_bytes_per_launch", "source_sha256"}, f.name
        name = kv["kernel"].split("<")[0]
        assert name in bench.KERNEL_SOURCES, f.name
        assert int(kv["dram_bytes_per_launch"]) > 0, f.name
        assert re.fullmatch(r"[0-9a-f]{64}", kv["source_sha256"]), f.name
    assert seen >= 1


def test_traffic_is_used_only_while_the_sources_match():
    for f, kv in blocks():
        name = kv["kernel"].split("<")[0]
        current = bench.kernel_source_sha256(name) == kv["source_sha256"]
        got = bench.profiled_traffic(kv["kernel"])
        if current:
            assert got == int(kv["dram_bytes_per_launch"]), f.name
        else:
            assert got is None, f.name
    assert bench.profiled_traffic("no_such_kernel<1>") is None


def test_bench_mirrors_the_combine_threshold():
    """bench.py counts a tcgen05 plan's combine launch with the library's default
    threshold; the two must not drift apart."""
    src = (ROOT / "kv_cache_decode_03_b200" / "csrc" / "kvc_api.cu").read_text()
    m = re.search(r"#define KVC_TC_COMBINE_MIN_BYTES \((\d+) << (\d+)\)", src)
    assert m, "KVC_TC_COMBINE_MIN_BYTES default not found"
    assert bench.TC_COMBINE_MIN_BYTES == int(m.group(1)) << int(m.group(2))
