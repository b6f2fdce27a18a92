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
        if name == "group_sparse_step":
            assert e["dram_bytes_per_step"] > 0
            for f in e["from"].split(", "):
                assert os.path.exists(os.path.join(bench.ROOT, "profiles", f.split()[0])), f
            got = bench.ncu_sparse_traffic()
            if e["source_sha"] == bench.source_sha(files=bench.SPARSE_SOURCES):
                assert got["dram_bytes_per_step"] == e["dram_bytes_per_step"]
            else:
                assert got is None
            continue
        assert e["dram_bytes_per_step"] > 0
        assert os.path.exists(os.path.join(bench.ROOT, "profiles", e["from"].split()[0])), e["from"]
        if e["source_sha"] == bench.source_sha():
            assert bench.ncu_traffic(name) == e["dram_bytes_per_step"]
        else:
            assert bench.ncu_traffic(name) is None


def test_peak_choice_follows_the_timed_region():
    p, kind = bench.choose_peak(0.1, 1658.4, 1375.3, "measured")
    assert p == 1658.4 and "burst" in kind
    p, kind = bench.choose_peak(5.0, 1658.4, 1375.3, "measured")
    assert p == 1375.3 and "sustained" in kind


def test_pct_of_peak_denominators():
    clk = {"sm_mhz": 1965.0}
    out = bench.pct_of_peak(1350.0, 1658.4, 1375.3, "measured", clk)
    assert out["nominal"] == 60.0
    assert abs(out["burst"] - 100 * 1350 / 1658.4) < 0.01
    # 148 SMs x 8192 FLOP per clock at 1965 MHz
    assert abs(out["at_sampled_clock_tflops"] - 148 * 8192 * 1965e6 / 1e12) < 0.1
    assert "at_sampled_clock" not in bench.pct_of_peak(1350.0, 1658.4, 1375.3, "measured", None)


def test_clock_window_keeps_only_samples_inside_the_timed_region():
    t = bench.parse_smi_time("2026/12/02 16:15:00.250")
    assert t is not None and abs(bench.parse_smi_time("2026/12/02 16:15:01.250") - t - 1.0) < 1e-6
    rows = [dict(ts=t + i * 0.02, sm=(800.0 if i < 5 else 1965.0), smax=1965.0, power=300.0 + i,
                 hw="Not Active", hwt="Not Active", swt="Not Active",
                 swp=("Active" if i == 7 else "Not Active")) for i in range(10)]
    inside = bench.summarize_clocks(rows, t + 0.1, t + 0.18)  # samples 5..9
    assert inside["samples"] == 5 and inside["sm_mhz"] == 1965.0
    assert inside["reasons"] == ["sw_power_cap"] and inside["power_w_max"] == 309.0
    assert bench.summarize_clocks(rows, t + 5, t + 6) is None
    assert bench.summarize_clocks(rows)["samples"] == 10


def test_sparse_algorithmic_bytes_at_workload3():
    """The least traffic of select + fwd + bwd at 16384 x 1024 -> 4096, G 64, K 8, spg 8: about
    0.38 GB, far below the row-buffer design's traffic."""
    alg = bench.sparse_step_algorithmic_bytes(16384, 1024, 4096, 64, 8, 8)
    assert 0.37e9 < alg < 0.39e9
    R = 16384 * 8 + 64 * 64  # padded pair rows of a balanced selection
    design = bench.sparse_step_design_bytes(16384, 1024, 4096, 64, 8, 8, R)
    assert 3 * alg < design < 1.7e9  # mostly the per-pair y and dx rows: 4 x 277 MB
    # the algorithmic bytes do not depend on the padding and grow with the number of groups kept
    assert bench.sparse_step_algorithmic_bytes(16384, 1024, 4096, 64, 4, 8) < alg


def test_selection_check_counts_rows_against_the_oracle():
    """The bench's CPU-leg check: the oracle's own choice differs nowhere; a row with one group
    swapped for an unchosen one is counted."""
    import numpy as np
    import torch

    import oracle as O
    from swiglu_feed_forward_b200 import synth
    w = synth.WORKLOADS[3]
    inp = synth.workload_inputs(3, with_dy=False)
    x, wg = (inp[k].to(torch.float64).numpy() for k in ("x", "w_gate"))
    sub = O.make_subsample_index(w["d_ff"], w["group_size"], w["samples_per_group"], w["seed"])
    bias = synth.balance_bias(w["d_ff"] // w["group_size"], w["seed"]).to(torch.float64).numpy()
    ref = O.topk_groups(O.group_energy(x, wg, w["group_size"], sub, bias), w["num_active_groups"])
    out = bench.selection_check(torch.from_numpy(ref.astype(np.int32)))
    assert out["rows_differing"] == 0 and out["rows_differing_outside_near_ties"] == 0
    assert out["tokens"] == w["M"] and out["near_tie_rows"] >= 0
    bad = ref.copy()
    spare = [c for c in range(w["d_ff"] // w["group_size"]) if c not in bad[0]][0]
    bad[0, 0] = spare
    out = bench.selection_check(torch.from_numpy(bad.astype(np.int32)))
    assert out["rows_differing"] == 1

