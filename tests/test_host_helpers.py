"""Host helpers beside the kernels, on the CPU: the suffix bound the cascade
takes, and the bench's rule that a committed DRAM-traffic figure is reported
only while the kernel sources it was measured on are unchanged."""
import importlib.util
import json
import os

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_suffix_blocks_bound():
    from paged_kv_cache_459_b200 import pkv
    lens = np.array([17, 32, 100, 1])
    pb = np.array([0, 1, 5, 0])
    # ceil(len / 16) - prefix blocks: 2, 1, 2, 1
    assert pkv.suffix_blocks_bound(lens, pb) == 2
    assert pkv.suffix_blocks_bound(np.array([16]), np.array([1])) == 1   # never below one block
    assert pkv.suffix_blocks_bound(np.array([], np.int64), np.array([], np.int64)) == 0


def _bench(tmp_path):
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    csrc = tmp_path / "paged_kv_cache_459_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    bench.ROOT = str(tmp_path)
    return bench, csrc


def test_committed_traffic_follows_the_sources(tmp_path):
    bench, csrc = _bench(tmp_path)
    (csrc / "a.cu").write_text("kernel a\n")
    (csrc / "b.cuh").write_text("helpers\n")
    sha = bench.source_sha(str(csrc / "a.cu"), str(csrc / "b.cuh"))
    rec = {"w": {"k": {"dram_bytes_per_launch": 123, "source": ["a.cu", "b.cuh"], "source_sha": sha}},
           "v": {"k": {"dram_bytes_per_launch": 7, "source": "a.cu",
                       "source_sha": bench.source_sha(str(csrc / "a.cu"))}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.committed_traffic("k", "w") == 123
    assert bench.committed_traffic("k", "v") == 7
    assert bench.committed_traffic("k", "missing") is None
    (csrc / "b.cuh").write_text("helpers, changed\n")     # a source changed since the capture
    assert bench.committed_traffic("k", "w") is None
    assert bench.committed_traffic("k", "v") == 7          # its own source is unchanged


def test_source_sha_depends_on_every_file_and_order(tmp_path):
    bench, csrc = _bench(tmp_path)
    (csrc / "x").write_text("1")
    (csrc / "y").write_text("2")
    a = bench.source_sha(str(csrc / "x"), str(csrc / "y"))
    assert a != bench.source_sha(str(csrc / "x"))
    assert a == bench.source_sha(str(csrc / "x"), str(csrc / "y"))
    assert len(a) == 12
