"""Composition of the hot-path calls for the three workload shapes, on caller-provided CUDA
tensors: a CSA decode step, an HCA layer (prefill chunk or decode), and a CSA/HCA layer pair
over a chunked prefill.  Owns the intermediate buffers (scores, indices, workspaces) so a step
allocates nothing; every step is a sequence of libhcl calls on one stream."""
import math

import torch

from . import api
from .api import HCL_BF16, HCL_FP32, HCL_MXFP4, KV


class CsaDecode:
    """One query per sequence: [quantise q_I] -> index scores -> top-k -> sparse attention.

    q [B,1,H,d] bf16; qI [B,1,HI,dI] bf16; w [B,1,HI] fp32; keys: bf16 [B,cap,dI], or MXFP4
    packed [B,cap,dI/2] + kI_sf [B,cap,dI/32]; kvc / raw: api.KV stores; q_pos [B,1] int32."""

    def __init__(self, q, qI, w, kI, kvc: KV, Nc, raw: KV, L, W, q_pos, m=4, k=1024,
                 op_fmt=HCL_BF16, score_fmt=HCL_FP32, kI_sf=None, sink=None, q_gamma=None,
                 q_eps=1e-6):
        self.q, self.qI, self.w, self.kI, self.kI_sf = q, qI, w, kI, kI_sf
        self.q_gamma, self.q_eps = q_gamma, q_eps
        self.kvc, self.raw, self.Nc, self.L, self.W, self.q_pos = kvc, raw, Nc, L, W, q_pos
        self.m, self.k, self.op_fmt, self.score_fmt, self.sink = m, k, op_fmt, score_fmt, sink
        B, _, H, d = q.shape
        HI, dI = qI.shape[-2], qI.shape[-1]
        dev = q.device
        self.B, self.H, self.HI = B, H, HI
        if op_fmt == HCL_MXFP4:
            self.qI_packed = torch.empty(B, 1, HI, dI // 2, dtype=torch.uint8, device=dev)
            self.qI_sf = torch.empty(B, 1, HI, dI // 32, dtype=torch.uint8, device=dev)
        sdt = torch.bfloat16 if score_fmt == HCL_BF16 else torch.float32
        self.scores = torch.empty(B, 1, Nc, dtype=sdt, device=dev)
        self.idx = torch.empty(B, 1, k, dtype=torch.int32, device=dev)
        self.out = torch.empty(B, 1, H, d, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(B, 1, H, dtype=torch.float32, device=dev)
        n = api.csa_sparse_attn_workspace_bytes(B, 1, H, k, W)
        self.attn_ws = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
        n = api.decode_step_workspace_bytes(B, H, HI, Nc, k, W, op_fmt, score_fmt)
        self.step_ws = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def launches_per_step(self, fused=True):
        """Kernels one step launches: the fused C-ABI step as the library reports it, or with
        step_parts() indexer, top-k, attention (+ split merge) and, for MXFP4 keys, a separate
        q_I quantisation."""
        if fused:
            return api.lib().hcl_csa_decode_step_kernels(self.B, self.H, self.HI, self.Nc, self.k,
                                                         self.W, self.op_fmt, self.score_fmt,
                                                         self.kvc.fmt)
        n = 3 + (1 if self.op_fmt == HCL_MXFP4 else 0)
        need = api.csa_sparse_attn_workspace_bytes(self.B, 1, self.H, self.k, self.W)
        return n + (1 if need else 0)

    def step_parts(self, stream=None):
        """The four calls one by one, keeping the intermediates (scores, idx)."""
        qI, qI_sf = self.qI, None
        if self.op_fmt == HCL_MXFP4:
            api.hcl_quant_mxfp4(self.qI, self.qI_packed, self.qI_sf, stream=stream)
            qI, qI_sf = self.qI_packed, self.qI_sf
        api.hcl_csa_index_scores(self.op_fmt, qI, self.w, self.kI, self.q_pos, self.m, self.scores,
                                 Nc=self.Nc, qI_sf=qI_sf, kI_sf=self.kI_sf, status=self.status,
                                 stream=stream)
        api.hcl_csa_topk(self.scores, self.q_pos, self.m, self.k, self.idx, status=self.status,
                         stream=stream)
        api.hcl_csa_sparse_attn(self.q, self.kvc, self.Nc, self.idx, self.raw, self.L, self.W,
                                self.q_pos, self.out, lse=self.lse, sink=self.sink,
                                ws=self.attn_ws, status=self.status, q_gamma=self.q_gamma,
                                q_eps=self.q_eps, stream=stream)
        return self.out

    def step(self, stream=None):
        """The fused C-ABI decode step (same kernels, one call)."""
        api.hcl_csa_decode_step(self.q, self.qI, self.w, self.op_fmt, self.kI, self.kvc, self.Nc,
                                self.m, self.k, self.raw, self.L, self.W, self.q_pos, self.out,
                                score_fmt=self.score_fmt, kI_sf=self.kI_sf, lse=self.lse,
                                idx_out=self.idx, sink=self.sink, ws=self.step_ws,
                                status=self.status, q_gamma=self.q_gamma, q_eps=self.q_eps,
                                stream=stream)
        return self.out


class HcaLayer:
    """HCA attention over the compressed entries plus the raw window for Tq queries per
    sequence (a prefill chunk, or Tq = 1 for decode); optionally compresses entries first."""

    def __init__(self, q, kvh: KV, Nh, mh, raw: KV, L, W, q_pos, sink=None, q_gamma=None,
                 q_eps=1e-6):
        self.q, self.kvh, self.Nh, self.mh, self.raw, self.L, self.W = q, kvh, Nh, mh, raw, L, W
        self.q_pos, self.sink, self.q_gamma, self.q_eps = q_pos, sink, q_gamma, q_eps
        B, Tq, H, d = q.shape
        self.out = torch.empty(B, Tq, H, d, dtype=torch.bfloat16, device=q.device)
        self.lse = torch.empty(B, Tq, H, dtype=torch.float32, device=q.device)
        n = api.hca_dense_attn_workspace_bytes(B, Tq, H, Nh, W)
        self.ws = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=q.device)

    def step(self, stream=None):
        api.hcl_hca_dense_attn(self.q, self.kvh, self.Nh, self.mh, self.raw, self.L, self.W,
                               self.q_pos, self.out, lse=self.lse, sink=self.sink, ws=self.ws,
                               status=self.status, q_gamma=self.q_gamma, q_eps=self.q_eps,
                               stream=stream)
        return self.out


class PairPrefill:
    """Alternating CSA/HCA layer pair over a chunk of new tokens appended to a context:
    compress the new CSA and HCA entries, score all CSA entries for every new query, top-k,
    CSA sparse attention, HCA dense attention.

    raw_kv / gate [1, L, d] bf16 (context + chunk); entries before the chunk are expected in
    comp_csa / comp_hca already (bf16 [1, cap, d]); qI [1,Tq,HI,dI] bf16, w [1,Tq,HI];
    q_csa / q_hca [1,Tq,H,d]; kI [1,Nc,dI] bf16."""

    def __init__(self, raw_kv, gate, bias_csa, bias_hca, comp_csa, comp_hca, q_csa, q_hca, qI, w,
                 kI, q_pos, chunk_begin, m=4, mh=128, k=1024, W=128, score_fmt=HCL_BF16):
        self.raw_kv, self.gate, self.bias_csa, self.bias_hca = raw_kv, gate, bias_csa, bias_hca
        self.comp_csa, self.comp_hca, self.q_csa, self.q_hca = comp_csa, comp_hca, q_csa, q_hca
        self.qI, self.w, self.kI, self.q_pos = qI, w, kI, q_pos
        self.m, self.mh, self.k, self.W, self.score_fmt = m, mh, k, W, score_fmt
        B, L, d = raw_kv.shape
        Tq, H = q_csa.shape[1], q_csa.shape[2]
        self.L = L
        self.Nc = -(-L // m)
        self.Nh = -(-L // mh)
        self.csa_begin = chunk_begin // m
        self.hca_begin = chunk_begin // mh
        dev = raw_kv.device
        sdt = torch.bfloat16 if score_fmt == HCL_BF16 else torch.float32
        self.scores = torch.empty(B, Tq, self.Nc, dtype=sdt, device=dev)
        self.idx = torch.empty(B, Tq, k, dtype=torch.int32, device=dev)
        self.raw = KV(raw_kv)
        self.kvc = KV(comp_csa)
        self.kvh = KV(comp_hca)
        self.out_csa = torch.empty(B, Tq, H, d, dtype=torch.bfloat16, device=dev)
        self.lse_csa = torch.empty(B, Tq, H, dtype=torch.float32, device=dev)
        n = api.csa_sparse_attn_workspace_bytes(B, Tq, H, k, W)
        self.ws_csa = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
        self.hca = HcaLayer(q_hca, self.kvh, self.Nh, mh, self.raw, L, W, q_pos)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def compress_prior(self, stream=None):
        """Entries of the context before the chunk (set-up, not part of a step)."""
        if self.csa_begin:
            api.hcl_csa_compress(self.raw_kv, self.gate, self.bias_csa, self.m, self.comp_csa,
                                 0, self.csa_begin, stream=stream)
        if self.hca_begin:
            api.hcl_hca_compress(self.raw_kv, self.gate, self.bias_hca, self.mh, self.comp_hca,
                                 0, self.hca_begin, stream=stream)

    def step(self, stream=None):
        api.hcl_csa_compress(self.raw_kv, self.gate, self.bias_csa, self.m, self.comp_csa,
                             self.csa_begin, self.Nc, stream=stream)
        api.hcl_hca_compress(self.raw_kv, self.gate, self.bias_hca, self.mh, self.comp_hca,
                             self.hca_begin, self.Nh, stream=stream)
        api.hcl_csa_index_scores(HCL_BF16, self.qI, self.w, self.kI, self.q_pos, self.m,
                                 self.scores, Nc=self.Nc, status=self.status, stream=stream)
        api.hcl_csa_topk(self.scores, self.q_pos, self.m, self.k, self.idx, status=self.status,
                         stream=stream)
        api.hcl_csa_sparse_attn(self.q_csa, self.kvc, self.Nc, self.idx, self.raw, self.L, self.W,
                                self.q_pos, self.out_csa, lse=self.lse_csa, ws=self.ws_csa,
                                status=self.status, stream=stream)
        self.hca.step(stream=stream)
        return self.out_csa, self.hca.out

    def launches_per_step(self):
        n = 6
        if api.csa_sparse_attn_workspace_bytes(*self.idx.shape[:2], self.q_csa.shape[2], self.k, self.W):
            n += 1
        if api.hca_dense_attn_workspace_bytes(*self.q_hca.shape[:3], self.Nh, self.W):
            n += 1
        return n
