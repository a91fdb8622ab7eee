"""Host-side arithmetic of the benchmark (CPU): the algorithmic bytes and flops that
every reported rate divides by, and the reading of a committed ncu summary."""
import hashlib
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle as O  # noqa: E402
from oracle import prefill_oracle as PF  # noqa: E402
from head_partitioned_sparse_b200 import synth  # noqa: E402


@pytest.mark.parametrize("T,start,n_sink,window", [(1, 0, 4, 16), (70, 0, 4, 16), (50, 33, 0, 8), (40, 100, 7, 1),
                                                   (64, 5, 100, 3)])
def test_prefill_flops_counts_every_attended_pair(T, start, n_sink, window):
    head_mask = [1, 0, 0, 1]
    G = 2
    pairs = 0
    for g, m in enumerate(head_mask):
        for t in range(start, start + T):
            pairs += G * len(PF.prefill_keys(t, bool(m), n_sink, window))
    assert bench.prefill_flops(T, start, head_mask, G, n_sink, window) == 4.0 * 128 * pairs


def test_algorithmic_bytes_of_a_ragged_batch():
    inp = synth.make_inputs("tiny", 0, overrides={"B": 3, "L": 700, "window": 32, "dtype": "bf16"},
                            seq_lens=[700, 450, 3])
    rng = np.random.default_rng(0)
    counts = rng.integers(0, 100, size=(inp.B, inp.Hkv))
    got = bench.algorithmic_bytes(inp, counts, 2)
    idx = contig = 0
    for b in range(inp.B):
        L = int(inp.seq_lens[b])
        sw = len(O.sink_window(L, inp.n_sink, inp.window))
        for g in range(inp.Hkv):
            contig += sw
            idx += 32 * L if inp.head_mask[g] else 0
    row = 2 * 128 * 2
    assert got["idx"] == idx and got["contig_rows"] == contig and got["selected_rows"] == counts.sum()
    assert got["total"] == idx + (contig + counts.sum()) * row + inp.B * inp.Hq * 128 * (2 + 4)


def test_recorded_traffic_needs_the_profiled_source(tmp_path, monkeypatch):
    csrc = tmp_path / "head_partitioned_sparse_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "k.cu").write_text("// kernel\n")
    sha = hashlib.sha256(b"// kernel\n").hexdigest()
    (tmp_path / "profiles" / "k.md").write_text(
        f"kernel_source_sha256: {sha}\n\ndram_bytes_per_launch_full_workload: 12345\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("k.cu", "k.md") == 12345.0
    (csrc / "k.cu").write_text("// kernel, changed\n")
    assert bench.recorded_traffic("k.cu", "k.md") is None      # stale counters are not reported
    assert bench.recorded_traffic("k.cu", "missing.md") is None
