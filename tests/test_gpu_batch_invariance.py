"""Batch-invariant kernels [Tripbot §8, infrastructure table: batch-invariant, deterministic
kernels; Austery's talk notes, infrastructure section]: a sequence's decode result must be
bitwise the same whatever batch it is decoded in.

The 128K-context CSA decode workload (32 sequences, 32768 entries each, 64 heads, top-512 plus
a 128-token window, planted high-scoring entries) runs as one batch of 32, as a batch of the
first 7 and as the first sequence alone, through the fused C-ABI decode step and through the
separate calls.  Selected indices, outputs and log-sum-exps of every shared sequence must be
equal bit for bit.  (The selection is exact, so it cannot depend on how the top-k is spread
over blocks; the attention splits each sequence's row list by its length only, and merges the
splits in a fixed order.)"""
import pytest
import torch

from heavily_compressed_long_b200.api import HCL_BF16, HCL_FP32, KV
from heavily_compressed_long_b200.pipeline import CsaDecode
from synth import gen
from synth.configs import CSA_128K
from tests.helpers import cuda

pytestmark = pytest.mark.gpu


def _run(cfg, seqs, fused):
    B, L, W, Nc = len(seqs), cfg.L, cfg.W, cfg.Nc
    q, qI, w = gen.queries(cfg, seqs), gen.index_queries(cfg, seqs), gen.head_weights(cfg, seqs)
    kI = gen.index_keys(cfg, seqs)
    kvc = gen.comp_kv(cfg, seqs, Nc)
    rows = gen.raw_kv(cfg, seqs, L - W, L)
    ring = torch.empty_like(rows)
    for j, t in enumerate(range(L - W, L)):
        ring[:, t % W] = rows[:, j]
    pos = gen.query_positions(cfg, B)
    pipe = CsaDecode(cuda(q), cuda(qI), cuda(w), cuda(kI), KV(cuda(kvc)), Nc, KV(cuda(ring)), L, W,
                     cuda(pos), m=cfg.m, k=cfg.k, op_fmt=HCL_BF16, score_fmt=HCL_FP32)
    if fused:
        pipe.step()
    else:
        pipe.step_parts()
    torch.cuda.synchronize()
    assert pipe.status.item() == 0
    return pipe.idx.cpu(), pipe.out.cpu(), pipe.lse.cpu()


@pytest.mark.parametrize("fused", [True, False])
def test_csa_decode_128k_batch_invariant(hcl, fused):
    """bf16 index operands, fp32 scores: the separate top-k and attention kernels."""
    cfg = CSA_128K
    full = _run(cfg, list(range(32)), fused)
    seven = _run(cfg, list(range(7)), fused)
    one = _run(cfg, [0], fused)
    for a, b in zip(full, seven):
        assert torch.equal(a[:7], b)
    for a, b in zip(full, one):
        assert torch.equal(a[:1], b)


def _run_mxfp4(cfg, seqs):
    """The 1M-decode path's formats (MXFP4 keys, bf16 scores, FP8 split KV rows) through the fused
    step, whose selection and attention run as one cluster kernel per sequence."""
    from heavily_compressed_long_b200 import api
    from heavily_compressed_long_b200.api import HCL_BF16, HCL_MXFP4
    B, L, W, Nc = len(seqs), cfg.L, cfg.W, cfg.Nc
    dev = "cuda"
    kp = torch.empty(B, Nc, 32, dtype=torch.uint8, device=dev)
    ks = torch.empty(B, Nc, 2, dtype=torch.uint8, device=dev)
    cn = torch.empty(B, Nc, 64, dtype=torch.uint8, device=dev)
    cs = torch.empty(B, Nc, dtype=torch.float32, device=dev)
    cr = torch.empty(B, Nc, 64, dtype=torch.bfloat16, device=dev)
    api.hcl_quant_mxfp4(cuda(gen.index_keys(cfg, seqs)), kp, ks)
    api.hcl_quant_kv_fp8(cuda(gen.comp_kv(cfg, seqs, Nc)), cn, cs, cr)
    rn = torch.empty(B, W, 64, dtype=torch.uint8, device=dev)
    rs = torch.empty(B, W, dtype=torch.float32, device=dev)
    rr = torch.empty(B, W, 64, dtype=torch.bfloat16, device=dev)
    api.hcl_quant_kv_fp8(cuda(gen.raw_kv(cfg, seqs, L - W, L)), rn, rs, rr)
    q, qI, w = gen.queries(cfg, seqs), gen.index_queries(cfg, seqs), gen.head_weights(cfg, seqs)
    pos = gen.query_positions(cfg, B)
    pipe = CsaDecode(cuda(q), cuda(qI), cuda(w), kp, KV(cn, cs, cr), Nc, KV(rn, rs, rr), L, W,
                     cuda(pos), m=cfg.m, k=cfg.k, op_fmt=HCL_MXFP4, score_fmt=HCL_BF16, kI_sf=ks)
    pipe.step()
    torch.cuda.synchronize()
    assert pipe.status.item() == 0
    return pipe.idx.cpu(), pipe.out.cpu(), pipe.lse.cpu()


def test_csa_decode_mxfp4_batch_invariant(hcl):
    from synth.configs import CSA_1M, scaled
    cfg = scaled(CSA_1M, L=4 * 70000)
    full = _run_mxfp4(cfg, [0, 1, 2])
    one = _run_mxfp4(cfg, [1])
    for a, b in zip(full, one):
        assert torch.equal(a[1:2], b)
