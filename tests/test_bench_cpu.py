"""Host logic of the benchmark: the early-exit round schedule it assumes
matches the header's constants, its byte accounting is the per-row sum it
claims to be, and the kernel-source hash that ties a committed ncu capture
to the code it measured ignores comments only."""
import os
import re
import shutil
import subprocess

import numpy as np

import bench
import psi_inputs
import rejection_sampling_verify_b200 as psi

CFG = psi_inputs.CONFIGS


def _header_define(name):
    text = open(bench.os.path.join(bench.ROOT, "include", "psi_verify.h")).read()
    return int(re.search(rf"#define\s+{name}\s+(\d+)", text).group(1))


def test_schedule_constants_come_from_the_header():
    for name in ("PSI_SAMPLED_ROUND_POSITIONS", "PSI_GREEDY_ROUND_POSITIONS",
                 "PSI_SAMPLED_SHORT_ROUNDS", "PSI_GREEDY_SHORT_ROUNDS",
                 "PSI_EARLY_EXIT_MIN_N"):
        assert getattr(psi, name) == _header_define(name)


def test_rounds_partition_the_positions():
    for name in ("large_batch_nucleus", "max_batch_greedy", "single_stream", "tiny"):
        cfg = CFG[name]
        r = bench.sampled_rounds(cfg)
        assert r[0][0] == 0 and r[-1][1] == cfg.B + 1
        assert all(a[1] == b[0] and a[0] < a[1] for a, b in zip(r, r[1:]))
        if cfg.N < psi.PSI_EARLY_EXIT_MIN_N:
            assert r == [(0, cfg.B + 1)]
        else:
            short, rs = ((psi.PSI_GREEDY_SHORT_ROUNDS, psi.PSI_GREEDY_ROUND_POSITIONS)
                         if cfg.temperature == 0 else
                         (psi.PSI_SAMPLED_SHORT_ROUNDS, psi.PSI_SAMPLED_ROUND_POSITIONS))
            assert all(b - a == rs for a, b in r[:short])


def test_rows_read_counts_rounds_up_to_the_emitting_position():
    cfg = CFG["large_batch_nucleus"]  # rounds (0, 2), (2, 4), (4, 9), B = 8
    assert bench.sampled_rounds(cfg) == [(0, 2), (2, 4), (4, 9)]
    # emitting position 0..1: round 0 only = 2 AR + 2 draft rows; 2..3: rounds
    # 0 and 1 = 8 rows; later: all 17
    assert bench.rows_read(cfg, np.array([1, 2])) == 2 * 4
    assert bench.rows_read(cfg, np.array([3, 4])) == 2 * 8
    assert bench.rows_read(cfg, np.array([5, 9])) == 2 * 17
    g = CFG["max_batch_greedy"]  # AR rows only
    assert bench.rows_read(g, np.array([1])) == 3
    assert bench.rows_read(g, np.array([17])) == 17


def test_main_launch_bytes_is_the_first_round():
    cfg = CFG["large_batch_nucleus"]
    assert bench.main_launch_bytes(cfg) == cfg.N * 4 * cfg.V * 2
    g = CFG["max_batch_greedy"]
    assert bench.main_launch_bytes(g) == g.N * 3 * g.V * 2
    t = CFG["tree_greedy"]
    assert bench.main_launch_bytes(t) == bench.algorithmic_bytes(t)
    assert bench.algorithmic_bytes(cfg) == 1322450944


# ---- the kernel-source hash behind `traffic` ----------------------------------------

def test_tree_rows_read_follows_the_matches():
    """The greedy tree walk reads the root's row and each matched node's:
    node 0 (token 1) and node 1 (token 1, a duplicate sibling) match the
    root's argmax 1; node 2 matches node 0's row; node 3's parent row (node 1)
    has argmax 0, not its token; node 4 hangs off the unmatched node 3; node 5
    has an invalid parent."""
    am = np.array([[1, 2, 0, 5, 4, 3, 0]])   # argmax of rows 0..M (row k+1 = node k)
    tok = np.array([[1, 1, 2, 3, 4, 0]])
    par = np.array([[-1, -1, 0, 1, 3, 7]])
    assert bench.tree_rows_read(am, tok, par) == 1 + 3
    # nothing matched: the root's row only; two trees add up
    assert bench.tree_rows_read(np.array([[9, 0, 0]]), np.array([[1, 2]]), np.array([[-1, 0]])) == 1
    assert bench.tree_rows_read(np.concatenate([am, am]), np.concatenate([tok, tok]),
                                np.concatenate([par, par])) == 8


def test_comment_stripping_matches_the_compiler():
    """gcc's own comment removal (-fpreprocessed) leaves the same code, up to
    whitespace (gcc also drops `#pragma once` from a main file)."""
    for f in bench.kernel_source_files():
        text = open(f, encoding="utf-8").read()
        mine = "".join(bench.strip_c_comments(text).split()).replace("#pragmaonce", "")
        g = subprocess.run(["gcc", "-fpreprocessed", "-dD", "-E", "-P", "-x", "c++", f],
                           capture_output=True, text=True, check=True)
        assert mine == "".join(g.stdout.split()), os.path.basename(f)


def test_strip_keeps_literals_and_code():
    src = 'a = "// not a comment"; /* gone */ b = \'/\'; // gone\nc = "x\\"y"; /*\n*/ d;'
    out = bench.strip_c_comments(src)
    assert '"// not a comment"' in out and "'/'" in out and '"x\\"y"' in out
    # a block comment is one space, even across lines
    assert "gone" not in out and out.splitlines()[-1] == 'c = "x\\"y";   d;'


def test_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    root = tmp_path / "repo"
    shutil.copytree(os.path.join(bench.ROOT, "rejection_sampling_verify_b200", "csrc"),
                    root / "rejection_sampling_verify_b200" / "csrc")
    (root / "include").mkdir()
    shutil.copy(os.path.join(bench.ROOT, "include", "psi_verify.h"), root / "include")
    monkeypatch.setattr(bench, "ROOT", str(root))
    h0 = bench.kernel_source_hash()
    assert h0 == bench.kernel_source_hash()
    f = root / "rejection_sampling_verify_b200" / "csrc" / "psi_scan.cu"
    text = f.read_text()
    f.write_text("// a new comment line\n\n" + text.replace("\n", "  \n", 3) + "\n/* and a block */\n")
    assert bench.kernel_source_hash() == h0
    f.write_text(text.replace("kStages = 6", "kStages = 5", 1))
    assert bench.kernel_source_hash() != h0


# ---- the reference arm (the oracle, on the host) -------------------------------------

def test_reference_arm_prints_the_contract_line():
    """`--impl reference` runs the oracle as it stands on the host (no GPU)
    and prints one JSON line with the same metric, unit and config keys."""
    import json
    import sys
    import time
    t0 = time.perf_counter()
    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl",
                        "reference", "--config", "tiny", "--steps", "3", "--warmup", "1"],
                       capture_output=True, text=True, timeout=600, cwd=bench.ROOT, check=True)
    wall = time.perf_counter() - t0
    line = json.loads(r.stdout.strip().splitlines()[-1])
    # the step time is the one measured: the timed steps fit in the run
    assert line["ms_per_step"] * line["steps"] / 1000.0 <= wall
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "blocks/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 3 and line["warmup"] == 1
    assert line["config"]["workload"] == "tiny"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == bench.host_cores()
    assert cb["value"] == line["value"] and line["sequences_per_step"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "blocks/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
