"""Host-side logic of bench.py on the CPU: how the option flags name and
configure a workload, and which arm each flag dispatches to.  No GPU work."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_tree_flags_configure_and_name_the_workload():
    args = bench.parse_args(["--config", "5", "--tree-fanout", "16"])
    w = bench.workload_of(args)
    assert (w.tree_fanout, w.tree_beam) == (16, w.top_k)      # the beam defaults to top_k
    assert w.name.endswith("+tree16x16")
    args = bench.parse_args(["--config", "2", "--tree-fanout", "16", "--tree-beam", "4",
                             "--consensus"])
    w = bench.workload_of(args)
    assert (w.tree_fanout, w.tree_beam, w.consensus) == (16, 4, True)
    assert bench.tree_of(w) == (16, 4)
    assert "two-level routing fanout=16 beam=4" in bench.workload_config(w, args)["workload"]
    flat = bench.workload_of(bench.parse_args([]))
    assert bench.tree_of(flat) == (0, 0) and "two-level" not in \
        bench.workload_config(flat, bench.parse_args([]))["workload"]


def test_mode_flags_dispatch_to_their_arms(monkeypatch):
    seen = []
    for name in ("run_ssa", "run_reference", "run_decode", "run_reference_decode",
                 "run_backward", "run_reference_backward"):
        monkeypatch.setattr(bench, name, lambda args, n=name: seen.append(n))
    cases = [([], "run_ssa"), (["--impl", "reference"], "run_reference"),
             (["--decode"], "run_decode"), (["--decode", "--impl", "reference"],
                                            "run_reference_decode"),
             (["--backward"], "run_backward"),
             (["--backward", "--impl", "reference"], "run_reference_backward")]
    for argv, want in cases:
        seen.clear()
        bench.main(argv)
        assert seen == [want], argv


def test_default_run_is_the_headline_workload():
    args = bench.parse_args([])
    # the largest workload that fits one GPU: the million-token prefill
    assert (args.gpus, args.config, args.steps >= 1, args.warmup >= 3) == (1, 5, True, True)
    w = bench.workload_of(args)
    assert (w.name, w.tree_fanout, w.consensus, w.beta) == ("gqa-clustered-1m", 0, False, 0.0)
    assert w.N == 1 << 20
