"""bench.py's roofline accounting (no GPU): the algorithmic byte counts it divides by, and the
rule that ncu traffic is reported only for the indexer source that was captured."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from synth.configs import CSA_1M  # noqa: E402


def test_bytes_per_query_at_1m():
    cfg = CSA_1M
    keys = cfg.Nc * (32 + 2)                       # MXFP4: 32 packed bytes + 2 E8M0 scales
    rows = (cfg.k + cfg.W) * (64 + 4 + 128)        # E4M3 half + fp32 scale + bf16 RoPE half
    qo = 2 * cfg.H * cfg.d * 2 + cfg.HI * cfg.dI * 2 + cfg.HI * 4 + 4
    assert (cfg.Nc, cfg.k, cfg.W, cfg.H, cfg.d, cfg.HI, cfg.dI) == (262144, 1024, 128, 128, 128, 16, 64)
    assert bench.bytes_per_query(cfg) == keys + rows + qo == 9206340


def test_indexer_bytes_per_launch():
    # keys read + bf16 scores written, 8 sequences
    assert bench.indexer_bytes_per_launch(CSA_1M, 8) == 8 * 262144 * 36 == 75497472


def test_traffic_only_for_the_captured_source(monkeypatch):
    import hashlib
    src = os.path.join(ROOT, "heavily_compressed_long_b200", "csrc", "indexer.cu")
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    per = bench.INDEXER_TRAFFIC["bytes_per_seq"]
    monkeypatch.setitem(bench.INDEXER_TRAFFIC, "source_sha256_16", h)
    assert bench.indexer_traffic(8) == pytest.approx(8 * per)
    monkeypatch.setitem(bench.INDEXER_TRAFFIC, "source_sha256_16", "0" * 16)
    assert bench.indexer_traffic(8) is None


def test_rank_sequences_partition():
    got = [bench.rank_sequences(8, r) for r in range(4)]
    flat = [s for part in got for s in part]
    assert flat == list(range(32)) and all(len(p) == 8 for p in got)
