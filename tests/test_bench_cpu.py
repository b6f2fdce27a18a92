"""Host logic of bench.py that decides whether committed ncu figures still describe the kernels."""
import json
import os

import bench


def test_code_lines_drop_comments_keep_strings():
    src = 'asm("mov.u32 %0, 1; // not a comment");  // a comment\n\n  // whole-line comment\nint x = 1;   \n'
    assert bench.code_lines(src) == ['asm("mov.u32 %0, 1; // not a comment");', "int x = 1;"]


def test_source_sha_ignores_comments_but_not_code():
    files = {rel: open(os.path.join(bench.ROOT, rel)).read() for rel in bench.KERNEL_SOURCES}
    base = bench.source_sha(lambda rel: files[rel])
    assert base == bench.source_sha()
    first = bench.KERNEL_SOURCES[0]
    commented = dict(files)
    commented[first] = "// an added comment line\n" + files[first].replace("\n", "  // trailing note\n", 1)
    assert bench.source_sha(lambda rel: commented[rel]) == base
    changed = dict(files)
    changed[first] = files[first] + "\nconstexpr int kProbeOnly = 1;\n"
    assert bench.source_sha(lambda rel: changed[rel]) != base


def test_committed_traffic_matches_current_code():
    """Every traffic entry is keyed to a code hash; the ones keyed to the current code are what
    the bench reports, and each names the profile summary it comes from."""
    p = os.path.join(bench.ROOT, "profiles", "ncu_traffic.txt")
    with open(p) as fh:
        entries = json.load(fh)
    assert entries, "no traffic figures committed"
    for name, e in entries.items():
        assert e["dram_bytes_per_launch"] > 0
        assert os.path.exists(os.path.join(bench.ROOT, "profiles", e["from"].split()[0])), e["from"]
        if e["source_sha"] == bench.source_sha():
            assert bench.ncu_traffic(name) == e["dram_bytes_per_launch"]
        else:
            assert bench.ncu_traffic(name) is None

