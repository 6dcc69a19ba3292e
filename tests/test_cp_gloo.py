"""Context-parallel CSA decode on CPU: two (and three) gloo ranks share one sequence's entries.

heavily_compressed_long_b200.cp.CsaDecodeCP runs its real exchange and merge logic -- the
slicing, the move of the query positions to each slice, the two all-gathers over a gloo
process group, the global selection from the gathered candidates and the log-sum-exp merge --
with the data steps done by the CPU oracle (OracleOps below stands in for the CUDA library,
which these CPU-only tests cannot load).  The result must equal one process computing the same
decode over the whole sequence: the selected indices exactly, the output within the bf16
rounding of the ranks' partial outputs."""
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


class _KV:
    """A bf16 store for the oracle: rows [B, cap, d]."""

    def __init__(self, data):
        self.data, self.cap = data, data.shape[1]


class OracleOps:
    """The CP data steps on the CPU with the oracle (test stand-in for the CUDA library)."""

    @staticmethod
    def index_scores(op_fmt, qI, w, kI, q_pos, m, scores, Nc=None, qI_sf=None, kI_sf=None):
        import oracle
        s = oracle.index_scores(oracle.FMT_BF16, qI, w, kI[:, :Nc].contiguous(), q_pos, m)
        scores.copy_(torch.from_numpy(s).to(scores.dtype))

    @staticmethod
    def topk(scores, q_pos, m, k, idx):
        import oracle
        idx.copy_(torch.from_numpy(oracle.topk(scores.double(), q_pos, m, k)))

    @staticmethod
    def cp_candidates(scores, idx, e0, cand_s, cand_i):
        B = scores.shape[0]
        for b in range(B):
            for j, li in enumerate(idx[b, 0].tolist()):
                cand_s[b, j] = float(scores[b, 0, li]) if li >= 0 else float("-inf")
                cand_i[b, j] = e0 + li if li >= 0 else -1

    @staticmethod
    def cp_own(pos, gathered_idx, e0, e1, sel, own):
        B, _, k = pos.shape
        for b in range(B):
            g = [int(gathered_idx[b, p]) for p in pos[b, 0].tolist() if p >= 0]
            g = [x for x in g if x >= 0]
            mine = [x - e0 for x in g if e0 <= x < e1]
            sel[b, 0] = torch.tensor(g + [-1] * (k - len(g)), dtype=torch.int32)
            own[b, 0] = torch.tensor(mine + [-1] * (k - len(mine)), dtype=torch.int32)

    @staticmethod
    def sparse_attn(q, kvc, Nc, idx, raw, L, W, q_pos, out, lse=None, q_gamma=None):
        import oracle
        o, l = oracle.csa_attn(q, oracle.KV(oracle.FMT_BF16, kvc.data, kvc.cap), idx,
                               oracle.KV(oracle.FMT_BF16, raw.data, raw.cap), W, q_pos)
        out.copy_(torch.from_numpy(o).to(out.dtype))
        lse.copy_(torch.from_numpy(l).to(lse.dtype))

    @staticmethod
    def lse_merge(o_parts, lse_parts, out, lse_out=None, sink=None):
        o = o_parts.double()
        l = lse_parts.double()
        M = l.max(0).values
        w = torch.where(l > float("-inf"), torch.exp(l - M), torch.zeros_like(l))
        den = w.sum(0)
        res = (w.unsqueeze(-1) * o).sum(0) / den.clamp_min(1e-300).unsqueeze(-1)
        out.copy_(res.to(out.dtype))
        if lse_out is not None:
            lse_out.copy_((M + torch.log(den)).to(lse_out.dtype))


def _problem():
    from synth import gen
    from synth.configs import CSA_TINY, scaled
    cfg = scaled(CSA_TINY, B=2, L=4 * 700 + 2, k=48, W=32, seed=31)
    bs = [0, 1]
    kvc = gen.comp_kv(cfg, bs, cfg.Nc)
    raw = gen.raw_kv(cfg, bs, 0, cfg.L)
    q, qI = gen.queries(cfg, bs), gen.index_queries(cfg, bs)
    w, kI = gen.head_weights(cfg, bs), gen.index_keys(cfg, bs)
    pos = torch.tensor([[cfg.L - 1], [cfg.L - 7]], dtype=torch.int32)
    return cfg, kvc, raw, q, qI, w, kI, pos


def _reference():
    """One process over the whole sequence, with the scores rounded to fp32 as the candidates
    carry them."""
    import oracle
    cfg, kvc, raw, q, qI, w, kI, pos = _problem()
    s = oracle.index_scores(oracle.FMT_BF16, qI, w, kI, pos, cfg.m).astype(np.float32).astype(np.float64)
    idx = oracle.topk(s, pos, cfg.m, cfg.k)
    o, l = oracle.csa_attn(q, oracle.KV(0, kvc, cfg.Nc), idx, oracle.KV(0, raw, cfg.L), cfg.W, pos)
    return idx, o, l


def _worker(rank, world, port, out_path):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from heavily_compressed_long_b200.api import HCL_FP32
        from heavily_compressed_long_b200.cp import CsaDecodeCP, TorchComm
        cfg, kvc, raw, q, qI, w, kI, pos = _problem()
        cp = CsaDecodeCP(rank, world, cfg.Nc, cfg.L, cfg.W, cfg.m, cfg.k, cfg.H, score_fmt=HCL_FP32,
                         comm=TorchComm(), ops=OracleOps, device="cpu")
        e0, e1 = cp.e0, cp.e1
        out, lse, sel = cp.step(q, qI, w, kI[:, e0:e1].contiguous(), _KV(kvc[:, e0:e1].contiguous()),
                                _KV(raw), pos)
        if rank == 0:
            torch.save({"out": out, "lse": lse, "sel": sel}, out_path)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_cp_decode_matches_one_process(tmp_path, world):
    out_path = str(tmp_path / "cp.pt")
    mp.start_processes(_worker, args=(world, _free_port(), out_path), nprocs=world,
                       start_method="spawn", join=True)
    got = torch.load(out_path)
    idx, o, l = _reference()
    assert np.array_equal(got["sel"].numpy(), idx)
    assert np.abs(got["out"].double().numpy() - o).max() <= 1e-2
    assert np.abs(got["lse"].double().numpy() - l).max() <= 1e-5
