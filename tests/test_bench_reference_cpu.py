"""The reference arm of bench.py (the oracle timed on the host cores) on CPU:
exactly K timed steps after W warm-up steps, a sample sized to the budget, and
the JSON line the contract asks for.  Run on the tiny byte-level model so it
takes seconds; the arm itself is model-agnostic."""
import argparse
import contextlib
import io
import json


def test_sample_length_fits_budget():
    import bench
    seqs = (64, 32, 16)
    # forward + backward 0.8 s at 64 tokens, optimiser 0.1 s
    assert bench.ref_sample_seq(0.8, 0.1, 1.0, seqs) == 64
    assert bench.ref_sample_seq(0.8, 0.1, 0.6, seqs) == 32     # 0.1 + 0.4
    assert bench.ref_sample_seq(0.8, 0.1, 0.35, seqs) == 16    # 0.1 + 0.2
    assert bench.ref_sample_seq(0.8, 0.1, 0.05, seqs) == 16    # nothing fits: the smallest


def test_reference_arm_json_line(monkeypatch):
    import bench
    from scratch_decoder_only_b200 import configs as CF
    monkeypatch.setattr(bench, "WL", CF.TINY_BYTE)
    monkeypatch.setattr(bench, "REF_SEQS", (64, 32, 16))
    args = argparse.Namespace(steps=3, warmup=2, gpus=1, impl="reference")
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(args, rank=0, world=1)
    lines = [l for l in out.getvalue().splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["steps"] == 3 and d["warmup"] == 2 and d["n_gpus"] == 1
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["config"]["workload"] == CF.TINY_BYTE.name
    assert d["ms_per_step"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_do_nothing():
    import bench
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(argparse.Namespace(steps=1, warmup=1), rank=1, world=2)
    assert out.getvalue() == ""


def test_oracle_trainer_carries_state():
    import numpy as np
    import bench
    from scratch_decoder_only_b200 import configs as CF
    tr = bench.OracleTrainer(CF.TINY_BYTE)
    p0 = tr.p.copy()
    tr.step(16)
    p1 = tr.p.copy()
    tr.step(16)
    assert tr.t == 2
    assert not np.array_equal(p0, p1) and not np.array_equal(p1, tr.p)
    assert np.all(tr.v >= 0) and np.any(tr.m != 0)
