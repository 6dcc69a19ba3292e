"""The N>1 path on CPU: two gloo ranks (no GPU).

The hot path shards over independent sequences (weak scaling): every rank decodes its own
sequences and nothing crosses ranks on the data path; only the timing is reduced (max over
ranks).  These tests run the bench's sharding and reduction helpers in two processes and check
that the union of the ranks' decodes (computed with the CPU oracle) is exactly what one process
computes for all sequences."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _decode(seqs):
    """Tiny CSA decode for the given global sequence ids through the oracle:
    compress -> index scores -> top-k -> attention.  Returns o [n, 1, H, d] fp64."""
    import oracle
    from synth import gen
    from synth.configs import CSA_TINY, scaled
    cfg = scaled(CSA_TINY, L=512, k=16, W=16)
    kv, g = gen.raw_kv(cfg, seqs, 0, cfg.L), gen.gate(cfg, seqs, 0, cfg.L)
    bias = gen.bias(cfg, 2 * cfg.m)
    q, qI = gen.queries(cfg, seqs), gen.index_queries(cfg, seqs)
    w, kI = gen.head_weights(cfg, seqs), gen.index_keys(cfg, seqs)
    pos = gen.query_positions(cfg, len(seqs))
    ent = oracle.compress(kv, g, bias, cfg.m, True)
    ent16 = torch.from_numpy(oracle.round_bf16(ent).astype(np.float32)).to(torch.bfloat16)
    s = oracle.index_scores(oracle.FMT_BF16, qI, w, kI, pos, cfg.m)
    idx = oracle.topk(s, pos, cfg.m, cfg.k)
    o, _ = oracle.csa_attn(q, oracle.KV(0, ent16, cfg.Nc), idx, oracle.KV(0, kv, cfg.L), cfg.W, pos)
    return o


def _worker(rank, world, port, n_per_rank, out_path):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        seqs = bench.rank_sequences(n_per_rank, rank)
        o = torch.from_numpy(_decode(seqs))
        parts = [torch.empty_like(o) for _ in range(world)]
        dist.all_gather(parts, o)                   # test-only: collect for comparison
        slowest = bench.max_over_ranks(10.0 + rank, world, torch.device("cpu"))
        if rank == 0:
            torch.save({"parts": parts, "slowest": slowest, "seqs": [bench.rank_sequences(n_per_rank, r)
                                                                    for r in range(world)]}, out_path)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_sharded_decode_equals_single_process(world, tmp_path):
    n_per_rank = 2
    out = str(tmp_path / "res.pt")
    mp.start_processes(_worker, args=(world, _free_port(), n_per_rank, out), nprocs=world,
                       join=True, start_method="spawn")
    res = torch.load(out)
    assert res["slowest"] == 10.0 + world - 1            # max over ranks
    flat = [s for part in res["seqs"] for s in part]
    assert flat == list(range(world * n_per_rank))      # disjoint, covering, in rank order
    full = torch.from_numpy(_decode(flat))
    assert torch.equal(torch.cat(res["parts"]), full)


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.rank_sequences(8, 0) == list(range(8))
    assert bench.rank_sequences(8, 3) == list(range(24, 32))
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
