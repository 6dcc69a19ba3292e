"""Context-parallel CSA decode: one sequence's compressed entries sharded over ranks.

[Austery's talk notes, infrastructure section: context parallelism] Rank r of G holds the
contiguous entry slice [e0, e1) of every sequence -- its index keys and compressed KV rows --
and the rank holding the last entries also holds the raw sliding window.  One decode step:

  select_local  the rank scores its slice (the lightning indexer, with the query positions
                moved to the slice's origin) and keeps its local top-k, turned into (score,
                global index) candidates;
  exchange 1    all ranks gather the candidates, rank by rank (= ascending global index);
  attend        every rank selects the k best of the gathered list -- the global top-k, since an
                entry among the k best overall is among the k best of its own slice (ties to the
                lower index in both) -- and attends over the selected entries it owns (plus the
                window on the last rank), keeping the partial (o, lse);
  exchange 2    all ranks gather the partials;
  merge         log-sum-exp merge of the partials (an attention sink enters once, here).

Every data step is a libhcl call; this module only marshals buffers and issues the two
all-gathers (torch.distributed: NCCL on GPUs).  The compute calls go through `ops` (default:
the CUDA library), so the exchange and merge logic can also run with another implementation of
the same calls."""
import math

import torch

from . import api
from .api import HCL_BF16, HCL_FP32, KV


class CudaOps:
    """The data steps on the GPU (libhcl)."""
    index_scores = staticmethod(api.hcl_csa_index_scores)
    topk = staticmethod(api.hcl_csa_topk)
    cp_candidates = staticmethod(api.hcl_cp_candidates)
    cp_own = staticmethod(api.hcl_cp_own)
    sparse_attn = staticmethod(api.hcl_csa_sparse_attn)
    lse_merge = staticmethod(api.hcl_lse_merge)


class TorchComm:
    """all_gather over a torch.distributed process group, along a new leading rank axis."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def all_gather(self, t):
        t = t.contiguous()
        flat = torch.empty((self.world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype,
                           device=t.device)
        self.dist.all_gather_into_tensor(flat, t, group=self.group)
        return flat.view((self.world,) + tuple(t.shape))


def slice_bounds(Nc, world, rank):
    """Contiguous entry slice [e0, e1) of `rank`: equal shares, the last rank taking the rest."""
    per = -(-Nc // world)
    e0 = min(Nc, rank * per)
    return e0, min(Nc, e0 + per)


class CsaDecodeCP:
    """One rank's part of a context-parallel CSA decode step for B sequences (Tq = 1).

    qI bf16 [B,1,HI,dI]; w fp32 [B,1,HI]; kI: this rank's index keys [B, e1-e0, dI] (bf16, or
    MXFP4 packed with kI_sf); kvc: this rank's entry rows (api.KV, cap >= e1-e0, local index);
    raw: the window store (api.KV; used on the last rank only); q bf16 [B,1,H,d]; q_pos int32
    [B,1] absolute positions."""

    def __init__(self, rank, world, Nc, L, W, m, k, H, d=128, op_fmt=HCL_BF16, score_fmt=HCL_FP32,
                 comm=None, ops=CudaOps, device="cuda"):
        self.rank, self.world, self.Nc, self.L, self.W, self.m, self.k = rank, world, Nc, L, W, m, k
        self.H, self.d, self.op_fmt, self.score_fmt = H, d, op_fmt, score_fmt
        self.e0, self.e1 = slice_bounds(Nc, world, rank)
        self.comm, self.ops, self.device = comm, ops, device
        self.last = rank == world - 1

    # ---- phase 1: local scores, local top-k, candidates --------------------------------------
    def select_local(self, qI, w, kI, q_pos, kI_sf=None, qI_sf=None):
        B = w.shape[0]
        n_loc = self.e1 - self.e0
        # positions relative to the slice's first entry (entry e0 becomes local entry 0)
        pos_loc = (q_pos - self.m * self.e0).to(torch.int32)
        sdt = torch.bfloat16 if self.score_fmt == HCL_BF16 else torch.float32
        self.scores = torch.empty(B, 1, max(n_loc, 1), dtype=sdt, device=self.device)
        self.idx_loc = torch.full((B, 1, self.k), -1, dtype=torch.int32, device=self.device)
        if n_loc > 0:
            self.ops.index_scores(self.op_fmt, qI, w, kI, pos_loc, self.m, self.scores[:, :, :n_loc],
                                  Nc=n_loc, qI_sf=qI_sf, kI_sf=kI_sf)
            self.ops.topk(self.scores[:, :, :n_loc].contiguous(), pos_loc, self.m, self.k, self.idx_loc)
        cand_s = torch.empty(B, self.k, dtype=torch.float32, device=self.device)
        cand_i = torch.empty(B, self.k, dtype=torch.int32, device=self.device)
        self.ops.cp_candidates(self.scores[:, :, :max(n_loc, 1)].contiguous(), self.idx_loc, self.e0,
                               cand_s, cand_i)
        return cand_s, cand_i

    # ---- phase 2: global selection from the gathered candidates, attention over own rows ----
    def attend(self, gath_s, gath_i, q, kvc: KV, raw: KV, q_pos, q_gamma=None):
        """gath_s / gath_i: [world, B, k] gathered candidates.  Returns (o, lse, sel)."""
        G, B, k = gath_s.shape
        n = G * k
        # per sequence, the gathered candidates in rank order: [B, 1, n]
        s_rows = gath_s.permute(1, 0, 2).reshape(B, 1, n).contiguous()
        i_rows = gath_i.permute(1, 0, 2).reshape(B, n).contiguous()
        allvis = torch.full((B, 1), n - 1, dtype=torch.int32, device=self.device)
        pos = torch.empty(B, 1, k, dtype=torch.int32, device=self.device)
        self.ops.topk(s_rows, allvis, 1, k, pos)
        sel = torch.empty(B, 1, k, dtype=torch.int32, device=self.device)
        own = torch.empty(B, 1, k, dtype=torch.int32, device=self.device)
        self.ops.cp_own(pos, i_rows, self.e0, self.e1, sel, own)
        o = torch.empty(B, 1, self.H, self.d, dtype=torch.bfloat16, device=self.device)
        lse = torch.empty(B, 1, self.H, dtype=torch.float32, device=self.device)
        W = self.W if self.last else 0
        n_loc = max(self.e1 - self.e0, 1)
        self.ops.sparse_attn(q, kvc, n_loc, own, raw, self.L, W, q_pos, o, lse=lse,
                             q_gamma=q_gamma)
        return o, lse, sel

    # ---- phase 3: merge of the gathered partials -------------------------------------------
    def merge(self, gath_o, gath_lse, sink=None):
        G = gath_o.shape[0]
        out = torch.empty(gath_o.shape[1:], dtype=torch.bfloat16, device=self.device)
        lse = torch.empty(gath_lse.shape[1:], dtype=torch.float32, device=self.device)
        self.ops.lse_merge(gath_o.contiguous(), gath_lse.contiguous(), out, lse_out=lse, sink=sink)
        return out, lse

    def step(self, q, qI, w, kI, kvc: KV, raw: KV, q_pos, kI_sf=None, sink=None, q_gamma=None):
        """The whole step with the two all-gathers; returns (out, lse, selected indices)."""
        cand_s, cand_i = self.select_local(qI, w, kI, q_pos, kI_sf=kI_sf)
        gs, gi = self.comm.all_gather(cand_s), self.comm.all_gather(cand_i)
        o, lse, sel = self.attend(gs, gi, q, kvc, raw, q_pos, q_gamma=q_gamma)
        go, gl = self.comm.all_gather(o), self.comm.all_gather(lse)
        out, lse_out = self.merge(go, gl, sink=sink)
        return out, lse_out, sel
