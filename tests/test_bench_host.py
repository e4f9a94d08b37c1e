"""Host-side bookkeeping of bench.py (no GPU): the rows a walking greedy call
reads, the byte counts built on them, and the translation units that key
the ncu traffic records."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from speculative_decoding_verification_87_b200 import workloads as wl  # noqa: E402


def test_chain_rows_read_match_oracle_accept_lengths(orc):
    # a linear walk reads rows 0..n of each request: sum(n + 1)
    for seed in range(3):
        w = wl.greedy_linear(seed=seed, batch=24, k=5, vocab=300)
        o = orc.verify_greedy(w.target, w.tokens, w.vocab)
        assert bench.walk_rows_read("greedy-walk", w) == int((o["acc"] + 1).sum())


def test_tree_rows_read_on_a_hand_built_tree():
    # root 0 with children 1, 2 (same token), 1 -> 3, 2 -> 4; argmax of every
    # row is token 5, except node 1's row (token 6)
    V = 8
    t = np.zeros((1, 5, V), np.float32)
    t[0, :, 5] = 1.0
    t[0, 1, 5], t[0, 1, 6] = 0.0, 1.0
    parents = np.array([[-1, 0, 0, 1, 2]], np.int32)
    tokens = np.array([[-1, 5, 5, 5, 5]], np.int32)
    w = wl.TreeWorkload("hand", t, t, tokens, parents, 2, V, 1.0, "f32")
    # kept: root, 1 and 2 (both match the root's argmax), 4 (matches node 2's
    # argmax); node 3 does not match node 1's argmax
    assert bench.walk_rows_read("tree-walk", w) == 4


def test_tree_rows_read_bounds_and_chain_equivalence(orc):
    w = wl.draft_tree(seed=1, batch=4, vocab=500, level_widths=(1, 3, 3, 2))
    o = orc.verify_tree(w.target, None, w.node_tokens, w.parents, w.max_depth, w.vocab, False,
                        1.0, 0, 0)
    read = bench.walk_rows_read("tree-walk", w)
    # every node on each chosen path is kept, and no more than all nodes
    assert int((o["acc"] + 1).sum()) <= read <= w.batch * w.num_nodes
    lin = wl.greedy_linear(seed=4, batch=10, k=3, vocab=200)
    c = wl.chain_tree_from_linear(lin)
    assert bench.walk_rows_read("tree-walk", c) == bench.walk_rows_read("greedy-walk", lin)


def test_walk_bytes_are_the_rows_read():
    w = wl.greedy_linear(seed=2, batch=16, k=4, vocab=1000)
    rows, full, _ = bench.workload_facts("greedy", w)
    rows_w, walk, cfg = bench.workload_facts("greedy-walk", w)
    read = bench.walk_rows_read("greedy-walk", w)
    assert rows_w == rows == 16 * 5
    assert cfg["rows_read_per_step"] == read
    assert full - walk == (rows - read) * 1000 * 2 == cfg["bytes_avoided_per_step"]
    assert "(walk)" in cfg["workload"]


def test_translation_units():
    main = bench.tu_files("specverify.cu")
    assert {"specverify.cu", "sv_common.cuh", "sv_fused.cuh", "sv_verify.cuh"} <= set(main)
    assert "sv_walk.cuh" not in main and "walk.cu" not in main
    assert bench.tu_files("walk.cu") == ["sv_common.cuh", "sv_exp64.cuh", "sv_walk.cuh", "walk.cu"]
    assert bench.tu_digest("walk.cu") != bench.tu_digest("specverify.cu")


def test_empirical_alpha():
    a = bench.empirical_alpha([0, 1, 2, 2, 3, -1], 5)
    assert a[0] == 4 / 5 and a[1] == 3 / 4 and a[2] == 1 / 3 and a[3] == 0.0 and a[4] is None
    assert bench.empirical_alpha([], 2) == [None, None]
    # all drafts kept: every position accepts
    assert bench.empirical_alpha([5, 5, 5], 5) == [1.0] * 5


def test_whole_job_rates():
    # 64 requests a step, 10 steps, 2 ranks, 5 ms: requests and rows per second
    assert bench.whole_job_rate(64, 10, 2, 5.0) == 64 * 10 * 2 / 0.005


def test_greedy_forms_share_the_workload_bytes():
    # the streamed and the workspace-free greedy forms time the same call on
    # the same rows: identical row and byte counts, distinct workload names
    w = wl.greedy_linear(seed=3, batch=8, k=4, vocab=1000)
    rows, full, cfg = bench.workload_facts("greedy", w)
    rows_c, full_c, cfg_c = bench.workload_facts("greedy-cluster", w)
    assert (rows, full) == (rows_c, full_c)
    assert cfg["workload"] != cfg_c["workload"] and "workspace-free" in cfg_c["workload"]
    assert "greedy-cluster" in bench.KERNEL_OF


def test_traffic_records_are_keyed_and_current():
    # every committed record names a workload the bench produces, a summary
    # that exists, and carries DRAM bytes; a record whose sources changed
    # since its capture reads as unmeasured
    import json
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    assert rec
    for key, e in rec.items():
        assert os.path.exists(os.path.join(ROOT, e["summary"])), key
        assert e["dram_read_bytes"] > 0 and e["dram_write_bytes"] >= 0
        assert e["tu"] in ("specverify.cu", "walk.cu")
        traffic, src = bench.measured_traffic(key)
        if e["tu_sha256"] == bench.tu_digest(e["tu"]):
            assert traffic == e["dram_read_bytes"] + e["dram_write_bytes"] and src == e["summary"]
        else:
            assert traffic is None
    assert bench.measured_traffic("no such workload") == (None, None)
