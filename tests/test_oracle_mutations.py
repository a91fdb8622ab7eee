"""Planted mistakes in the oracles are caught by the pins (CPU).

Each case copies the oracle package, the pin tests (with their fixtures) and the
synthetic-input module into a scratch directory, applies one textual mutation to one
oracle file there (a dropped term, a wrong sign, an off-by-one, a transposed operand, a
wrong reduction), and runs the pin file of that oracle in a subprocess: it must fail.
The unmutated copy must pass, which shows the harness itself is sound.  Nothing here
touches the repository's own files.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PINS = {
    "spa_oracle.py": "test_oracle_pins.py",
    "aoh_oracle.py": "test_oracle_aoh.py",
    "prefill_oracle.py": "test_oracle_prefill.py",
}

# (oracle file, text, replacement, what the mistake is)
MUTATIONS = [
    ("spa_oracle.py", "x2 * c + x1 * s", "x2 * c - x1 * s", "RoPE rotation sign"),
    ("spa_oracle.py", "-2.0 * i / head_dim", "-1.0 * i / head_dim", "RoPE frequencies"),
    ("spa_oracle.py", "kept = np.sort(order[before_sorted < p])", "kept = np.sort(order[before_sorted <= p])",
     "top-p keeps one token too many"),
    ("spa_oracle.py", "return a.mean(axis=0), a", "return a.sum(axis=0), a", "group sum instead of mean"),
    ("spa_oracle.py", "softmax(np.float64(idx_scale) * scores", "softmax(scores", "index temperature dropped"),
    ("spa_oracle.py", "order = np.lexsort((pos, -pi))            #", "order = np.lexsort((-pos, -pi))            #",
     "ties broken by the highest position"),
    ("spa_oracle.py", "s = set(range(min(max(n_sink, 0), L)))", "s = set(range(min(max(n_sink, 0), L) + 1))",
     "one sink too many"),
    ("spa_oracle.py", ") / np.sqrt(np.float64(d))", ")", "attention scale dropped"),
    ("spa_oracle.py", "@ np.asarray(P_k_g, np.float64).T)", "@ np.asarray(P_k_g, np.float64).T[::-1])",
     "index projector rows permuted"),
    ("spa_oracle.py", "t = L - 1", "t = L", "decode query position"),
    ("spa_oracle.py", "kept_blocks = bidx if p >= 1.0 else np.sort(order[before_sorted < p])",
     "kept_blocks = bidx if p >= 1.0 else np.sort(order[before_sorted <= p])", "block top-p keeps one block too many"),
    ("spa_oracle.py", "bmass = np.array([pi[b * block:(b + 1) * block].sum()",
     "bmass = np.array([pi[b * block:(b + 1) * block].max()", "block scored by its maximum"),
    ("spa_oracle.py", "s.update(range(max(0, L - max(window, 0)), L))",
     "s.update(range(max(0, L - max(window, 0) + 1), L))", "window one position short"),
    ("spa_oracle.py", "return softmax(s, axis=-1) @ np.asarray(V, np.float64)",
     "return softmax(s, axis=0) @ np.asarray(V, np.float64)", "attention softmax over the wrong axis"),
    ("aoh_oracle.py", "np.exp(-np.sum(p * np.log(p)))", "np.exp(-np.sum(p * np.log2(p)))", "entropy in bits"),
    ("aoh_oracle.py", "return (Wq @ Wq.T) @ (Wk @ Wk.T)", "return (Wq @ Wk.T) @ (Wk @ Wq.T)", "proxy matrix operands"),
    ("aoh_oracle.py", "_, R = np.linalg.qr(Wk.T)", "_, R = np.linalg.qr(Wq.T)", "kernel operator operands"),
    ("aoh_oracle.py", ".reshape(Hkv, -1).mean(axis=1)", ".reshape(Hkv, -1).max(axis=1)", "group maximum"),
    ("aoh_oracle.py", "order = np.lexsort((np.arange(er_kv.size), er_kv))",
     "order = np.lexsort((np.arange(er_kv.size), -er_kv))", "highest rank labelled retrieval"),
    ("prefill_oracle.py", "return np.arange(t + 1, dtype=np.int64)", "return np.arange(t, dtype=np.int64)",
     "causal mask drops the diagonal"),
    ("prefill_oracle.py", "return sink_window(t + 1, n_sink, window)", "return sink_window(t, n_sink, window)",
     "window ends one position early"),
    ("prefill_oracle.py", "q = rope(to_f64(q_chunk[b, h, i]), t, rope_theta)",
     "q = rope(to_f64(q_chunk[b, h, i]), i, rope_theta)", "query rotated to its chunk row"),
    ("prefill_oracle.py", "g = h // G", "g = h % Hkv", "GQA head mapping"),
    ("prefill_oracle.py", "keys = prefill_keys(t, bool(head_mask[g]), n_sink, window)",
     "keys = prefill_keys(t, not head_mask[g], n_sink, window)", "retrieval and streaming heads swapped"),
    ("aoh_oracle.py", "p = s / s.sum()", "p = s / s.max()", "singular values normalised by the largest"),
]


def _scratch(tmp, oracle_file=None, old=None, new=None):
    """A scratch copy of what the pins import, with one mutation applied."""
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(tmp, "oracle"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    pkg = os.path.join(tmp, "head_partitioned_sparse_b200")
    os.makedirs(pkg)
    for f in ("__init__.py", "synth.py"):
        shutil.copy(os.path.join(ROOT, "head_partitioned_sparse_b200", f), pkg)
    tests = os.path.join(tmp, "tests")
    os.makedirs(tests)
    for f in ["conftest.py", "index_band.py"] + sorted(set(PINS.values())):
        shutil.copy(os.path.join(ROOT, "tests", f), tests)
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(tests, "golden"))
    if oracle_file:
        path = os.path.join(tmp, "oracle", oracle_file)
        src = open(path).read()
        assert src.count(old) >= 1, f"mutation anchor not found in {oracle_file}: {old!r}"
        open(path, "w").write(src.replace(old, new, 1))


def _run_pins(tmp, pin_file):
    env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join("tests", pin_file), "-x", "-q",
                        "-p", "no:cacheprovider"], cwd=tmp, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-600:]


@pytest.mark.parametrize("oracle_file", sorted(PINS))
def test_unmutated_copy_passes_its_pins(tmp_path, oracle_file):
    _scratch(str(tmp_path))
    rc, out = _run_pins(str(tmp_path), PINS[oracle_file])
    assert rc == 0, out


@pytest.mark.parametrize("case", MUTATIONS, ids=[m[3] for m in MUTATIONS])
def test_planted_mistake_is_caught(tmp_path, case):
    oracle_file, old, new, _ = case
    _scratch(str(tmp_path), oracle_file, old, new)
    rc, out = _run_pins(str(tmp_path), PINS[oracle_file])
    assert rc != 0, f"the pins did not notice: {case[3]}\n{out}"
