"""End-to-end GPU parity at the five workloads' full sizes.

The GPU runs every sequence and query of a workload through the same calls the benchmark
times; the oracle recomputes sampled sequences / query rows from the same seeded inputs.
Stored entries and scores compare within 1 bf16 ulp (bf16) or 1e-3 norm-wise (fp32);
quantised caches compare bit-exact.  A selection is not unique where scores tie within the
ambiguity band (|s - s_k| <= max(1e-3 |s_k|, 1 bf16 ulp)), so it is checked in two parts: the
part outside the band must equal the oracle's top-k, and the GPU's selection must be a valid
one (unique, visible, ascending, of the right size).  The oracle then attends over that very
validated selection and every sampled row's attention must agree with it within 2e-2 (bf16
KV) / 5e-2 (FP8 KV) -- on every sampled row, whether or not the selection equals the
oracle's own."""
import numpy as np
import pytest
import torch

import oracle
from heavily_compressed_long_b200.api import HCL_BF16, HCL_FP32, HCL_MXFP4, KV
from heavily_compressed_long_b200.pipeline import CsaDecode, HcaLayer, PairPrefill
from synth import gen
from synth.configs import CSA_128K, CSA_1M, CSA_TINY, HCA_64K, PAIR_PREFILL, scaled
from tests.helpers import as_f64, bf16_out_ratio, check_topk_band, cuda, rel_rowwise

pytestmark = pytest.mark.gpu


def bf16_of(x64):
    """oracle fp64 values rounded by the oracle to bf16, as a bf16 tensor (exact conversion)."""
    return torch.from_numpy(oracle.round_bf16(x64).astype(np.float32)).to(torch.bfloat16)


def ring_of(rows, L, W):
    """raw rows for tokens [L-W, L) -> ring slots t % W."""
    ring = torch.empty_like(rows)
    for j, t in enumerate(range(L - W, L)):
        ring[:, t % W] = rows[:, j]
    return ring


def _attn_rows_match(gpu_idx, ref_idx):
    return [i for i in range(len(ref_idx)) if np.array_equal(gpu_idx[i], ref_idx[i])]


# =========================================================================================

def test_cfg1_csa_tiny_end_to_end(hcl):
    cfg = CSA_TINY
    bs = [0]
    kv, g = gen.raw_kv(cfg, bs, 0, cfg.L), gen.gate(cfg, bs, 0, cfg.L)
    bias = gen.bias(cfg, 2 * cfg.m)
    q, qI, w, kI = gen.queries(cfg, bs), gen.index_queries(cfg, bs), gen.head_weights(cfg, bs), gen.index_keys(cfg, bs)
    pos = gen.query_positions(cfg, 1)
    Nc = cfg.Nc
    # oracle chain
    ent = oracle.compress(kv, g, bias, cfg.m, True)
    ent16 = bf16_of(ent)
    s_ref = oracle.index_scores(oracle.FMT_BF16, qI, w, kI, pos, cfg.m)
    # GPU chain
    comp = torch.empty(1, Nc, cfg.d, dtype=torch.bfloat16, device="cuda")
    hcl.hcl_csa_compress(cuda(kv), cuda(g), cuda(bias), cfg.m, comp)
    pipe = CsaDecode(cuda(q), cuda(qI), cuda(w), cuda(kI), KV(comp), Nc, KV(cuda(kv)), cfg.L, cfg.W,
                     cuda(pos), m=cfg.m, k=cfg.k, op_fmt=HCL_BF16, score_fmt=HCL_FP32)
    pipe.step_parts()
    torch.cuda.synchronize()
    assert bf16_out_ratio(as_f64(comp), ent) <= 1.0
    assert rel_rowwise(as_f64(pipe.scores), s_ref) <= 1e-3
    gidx = pipe.idx.cpu().numpy()
    check_topk_band(gidx[0, 0], s_ref[0, 0], Nc, cfg.k, False)
    o_ref, l_ref = oracle.csa_attn(q, oracle.KV(0, ent16, Nc), gidx, oracle.KV(0, kv, cfg.L), cfg.W, pos)
    assert np.abs(as_f64(pipe.out) - o_ref).max() <= 2e-2
    assert np.abs(as_f64(pipe.lse) - l_ref).max() <= 2e-2
    # the fused C-ABI decode step launches the same kernels: identical bits
    out1, idx1 = pipe.out.clone(), pipe.idx.clone()
    pipe.step()
    torch.cuda.synchronize()
    assert torch.equal(out1, pipe.out) and torch.equal(idx1, pipe.idx)
    assert pipe.status.item() == 0


# =========================================================================================

def test_cfg2_hca_prefill_and_decode(hcl):
    cfg = HCA_64K
    B, L, d, mh, W = cfg.B, cfg.L, cfg.d, cfg.mh, cfg.W
    Nh = cfg.Nh
    bs = list(range(B))
    kv, g = gen.raw_kv(cfg, bs, 0, L), gen.gate(cfg, bs, 0, L)
    bias = gen.bias(cfg, mh)
    comp = torch.empty(B, Nh, d, dtype=torch.bfloat16, device="cuda")
    kvg = cuda(kv)
    hcl.hcl_hca_compress(kvg, cuda(g), cuda(bias), mh, comp)
    q = gen.queries(cfg, bs)                                  # [B, 2048, 16, 128]
    pos = gen.query_positions(cfg, B)
    pre = HcaLayer(cuda(q), KV(comp), Nh, mh, KV(kvg), L, W, cuda(pos))
    pre.step()
    qd = q[:, -1:].contiguous()
    dec = HcaLayer(cuda(qd), KV(comp), Nh, mh, KV(kvg), L, W, cuda(pos[:, -1:].contiguous()))
    dec.step()
    torch.cuda.synchronize()
    sample_b = [0, B - 1]
    rows = np.r_[0:cfg.Tq:97, cfg.Tq - 1]
    for b in sample_b:
        ent = oracle.compress(kv[b:b + 1], g[b:b + 1], bias, mh, False)
        assert bf16_out_ratio(as_f64(comp[b:b + 1]), ent) <= 1.0
        ent16 = bf16_of(ent)
        qs = q[b:b + 1, rows].contiguous()
        ps = pos[b:b + 1, rows].contiguous()
        o_ref, l_ref = oracle.hca_attn(qs, oracle.KV(0, ent16, Nh), Nh, mh, oracle.KV(0, kv[b:b + 1], L), W, ps)
        assert np.abs(as_f64(pre.out[b:b + 1, rows]) - o_ref).max() <= 2e-2
        assert np.abs(as_f64(pre.lse[b:b + 1, rows]) - l_ref).max() <= 2e-2
        assert np.abs(as_f64(dec.out[b:b + 1]) - o_ref[:, -1:]).max() <= 2e-2


# =========================================================================================

def test_cfg3_csa_128k_planted(hcl):
    cfg = CSA_128K
    B, L, d, W, Nc = cfg.B, cfg.L, cfg.d, cfg.W, cfg.Nc
    bs = list(range(B))
    q, qI, w = gen.queries(cfg, bs), gen.index_queries(cfg, bs), gen.head_weights(cfg, bs)
    kI = gen.index_keys(cfg, bs)
    kvc = gen.comp_kv(cfg, bs, Nc)
    raw_rows = gen.raw_kv(cfg, bs, L - W, L)
    ring = ring_of(raw_rows, L, W)
    pos = gen.query_positions(cfg, B)
    pipe = CsaDecode(cuda(q), cuda(qI), cuda(w), cuda(kI), KV(cuda(kvc)), Nc, KV(cuda(ring)), L, W,
                     cuda(pos), m=cfg.m, k=cfg.k, op_fmt=HCL_BF16, score_fmt=HCL_FP32)
    pipe.step_parts()
    torch.cuda.synchronize()
    gidx = pipe.idx.cpu().numpy()
    for b in range(B):                        # generator invariant: every pick is planted
        assert set(gidx[b, 0].tolist()) <= set(gen.planted_set(cfg, b).tolist())
    for b in [0, 13, B - 1]:
        sl = slice(b, b + 1)
        s_ref = oracle.index_scores(oracle.FMT_BF16, qI[sl], w[sl], kI[sl], pos[sl], cfg.m)
        assert rel_rowwise(as_f64(pipe.scores[sl]), s_ref) <= 1e-3
        check_topk_band(gidx[b, 0], s_ref[0, 0], Nc, cfg.k, False)
        o_ref, l_ref = oracle.csa_attn(q[sl], oracle.KV(0, kvc[sl], Nc), gidx[sl],
                                       oracle.KV(0, ring[sl], W), W, pos[sl])
        assert np.abs(as_f64(pipe.out[sl]) - o_ref).max() <= 2e-2
        assert np.abs(as_f64(pipe.lse[sl]) - l_ref).max() <= 2e-2
    assert pipe.status.item() == 0


# =========================================================================================

def test_cfg4_csa_1m_mxfp4_fp8(hcl):
    cfg = CSA_1M
    B, L, d, W, Nc, HI = cfg.B, cfg.L, cfg.d, cfg.W, cfg.Nc, cfg.HI
    dev = "cuda"
    kI_p = torch.empty(B, Nc, 32, dtype=torch.uint8, device=dev)
    kI_s = torch.empty(B, Nc, 2, dtype=torch.uint8, device=dev)
    c_n = torch.empty(B, Nc, 64, dtype=torch.uint8, device=dev)
    c_s = torch.empty(B, Nc, dtype=torch.float32, device=dev)
    c_r = torch.empty(B, Nc, 64, dtype=torch.bfloat16, device=dev)
    for b in range(B):                         # quantise the caches on the GPU, one sequence at a time
        hcl.hcl_quant_mxfp4(cuda(gen.index_keys(cfg, [b])), kI_p[b:b + 1], kI_s[b:b + 1])
        hcl.hcl_quant_kv_fp8(cuda(gen.comp_kv(cfg, [b], Nc)), c_n[b:b + 1], c_s[b:b + 1], c_r[b:b + 1])
    bs = list(range(B))
    raw_rows = gen.raw_kv(cfg, bs, L - W, L)
    ring = ring_of(raw_rows, L, W)
    r_n = torch.empty(B, W, 64, dtype=torch.uint8, device=dev)
    r_s = torch.empty(B, W, dtype=torch.float32, device=dev)
    r_r = torch.empty(B, W, 64, dtype=torch.bfloat16, device=dev)
    hcl.hcl_quant_kv_fp8(cuda(ring), r_n, r_s, r_r)
    q, qI, w = gen.queries(cfg, bs), gen.index_queries(cfg, bs), gen.head_weights(cfg, bs)
    pos = gen.query_positions(cfg, B)
    pipe = CsaDecode(cuda(q), cuda(qI), cuda(w), kI_p, KV(c_n, c_s, c_r), Nc, KV(r_n, r_s, r_r), L, W,
                     cuda(pos), m=cfg.m, k=cfg.k, op_fmt=HCL_MXFP4, score_fmt=HCL_BF16, kI_sf=kI_s)
    pipe.step_parts()
    torch.cuda.synchronize()
    gidx = pipe.idx.cpu().numpy()
    for b in [0, B - 1]:
        sl = slice(b, b + 1)
        # caches: the GPU quantiser's bits equal the oracle's
        kp, ks = oracle.quant_mxfp4(gen.index_keys(cfg, [b]))
        assert np.array_equal(kI_p[sl].cpu().numpy(), kp) and np.array_equal(kI_s[sl].cpu().numpy(), ks)
        cn, cs, cr = oracle.quant_kv_fp8(gen.comp_kv(cfg, [b], Nc))
        assert np.array_equal(c_n[sl].cpu().numpy(), cn)
        assert np.array_equal(c_s[sl].cpu().numpy().view(np.uint32), cs.view(np.uint32))
        rn, rs, rr = oracle.quant_kv_fp8(ring[sl])
        qp, qs = oracle.quant_mxfp4(qI[sl])
        assert np.array_equal(pipe.qI_packed[sl].cpu().numpy(), qp)
        s_ref = oracle.index_scores(oracle.FMT_MXFP4, qp, w[sl], kp, pos[sl], cfg.m, qI_sf=qs,
                                    kI_sf=ks, bf16_scores=True)
        assert bf16_out_ratio(as_f64(pipe.scores[sl]), s_ref) <= 1.0
        check_topk_band(gidx[b, 0], s_ref[0, 0], Nc, cfg.k, True)
        okc = oracle.KV(oracle.FMT_FP8SPLIT, cn, Nc, scale=cs, rope=cr)
        okr = oracle.KV(oracle.FMT_FP8SPLIT, rn, W, scale=rs, rope=rr)
        o_ref, l_ref = oracle.csa_attn(q[sl], okc, gidx[sl], okr, W, pos[sl])
        assert np.abs(as_f64(pipe.out[sl]) - o_ref).max() <= 5e-2
        assert np.abs(as_f64(pipe.lse[sl]) - l_ref).max() <= 5e-2
    assert pipe.status.item() == 0
    # the fused C-ABI decode step (q_I quantised inside the indexer, the top-k from its group
    # summaries): the same selection bit for bit, and its attention against the oracle on
    # every sequence.  Repeated steps on the same workspace must give the same bits.
    idx1 = pipe.idx.clone()
    pipe.idx.fill_(-7)
    pipe.step()
    torch.cuda.synchronize()
    assert torch.equal(idx1, pipe.idx)
    assert pipe.status.item() == 0
    out1, lse1 = pipe.out.clone(), pipe.lse.clone()
    for _ in range(3):
        pipe.idx.fill_(-7)
        pipe.out.zero_()
        pipe.step()
        torch.cuda.synchronize()
        assert torch.equal(idx1, pipe.idx)
        assert torch.equal(out1, pipe.out) and torch.equal(lse1, pipe.lse)
    assert pipe.status.item() == 0
    # a wait that ran to its bounded limit (about a second) would show here even if its result
    # were not reported: 20 steps take about 1 ms, the bound is generous
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(20):
        pipe.step()
    e1.record()
    torch.cuda.synchronize()
    assert e0.elapsed_time(e1) / 20 < 5.0
    assert pipe.status.item() == 0
    for b in range(B):
        sl = slice(b, b + 1)
        cn, cs, cr = oracle.quant_kv_fp8(gen.comp_kv(cfg, [b], Nc))
        rn, rs, rr = oracle.quant_kv_fp8(ring[sl])
        okc = oracle.KV(oracle.FMT_FP8SPLIT, cn, Nc, scale=cs, rope=cr)
        okr = oracle.KV(oracle.FMT_FP8SPLIT, rn, W, scale=rs, rope=rr)
        o_ref, l_ref = oracle.csa_attn(q[sl], okc, gidx[sl], okr, W, pos[sl])
        assert np.abs(as_f64(pipe.out[sl]) - o_ref).max() <= 5e-2
        assert np.abs(as_f64(pipe.lse[sl]) - l_ref).max() <= 5e-2


# =========================================================================================

def test_cfg5_pair_prefill(hcl):
    cfg = PAIR_PREFILL
    L, d, W, m, mh, HI = cfg.L, cfg.d, cfg.W, cfg.m, cfg.mh, cfg.HI
    Nc, Nh, Tq = cfg.Nc, cfg.Nh, cfg.Tq
    bs = [0]
    kv, g = gen.raw_kv(cfg, bs, 0, L), gen.gate(cfg, bs, 0, L)
    b_csa, b_hca = gen.bias(cfg, 2 * m, 0), gen.bias(cfg, mh, 1)
    q_csa = gen.queries(cfg, bs)
    q_hca = gen.queries(scaled(cfg, seed=cfg.seed + 1), bs)
    qI, w, kI = gen.index_queries(cfg, bs), gen.head_weights(cfg, bs), gen.index_keys(cfg, bs)
    pos = gen.query_positions(cfg, 1)
    comp_csa = torch.zeros(1, Nc, d, dtype=torch.bfloat16, device="cuda")
    comp_hca = torch.zeros(1, Nh, d, dtype=torch.bfloat16, device="cuda")
    pp = PairPrefill(cuda(kv), cuda(g), cuda(b_csa), cuda(b_hca), comp_csa, comp_hca, cuda(q_csa),
                     cuda(q_hca), cuda(qI), cuda(w), cuda(kI), cuda(pos), cfg.first_pos, m=m, mh=mh,
                     k=cfg.k, W=W, score_fmt=HCL_BF16)
    pp.compress_prior()
    pp.step()
    torch.cuda.synchronize()
    ent_c = oracle.compress(kv, g, b_csa, m, True)
    ent_h = oracle.compress(kv, g, b_hca, mh, False)
    assert bf16_out_ratio(as_f64(comp_csa), ent_c) <= 1.0
    assert bf16_out_ratio(as_f64(comp_hca), ent_h) <= 1.0
    rows = np.unique(np.r_[0:Tq:67, Tq - 1])
    ps = pos[:, rows].contiguous()
    s_ref = oracle.index_scores(oracle.FMT_BF16, qI[:, rows].contiguous(), w[:, rows].contiguous(),
                                kI, ps, m, bf16_scores=True)
    assert bf16_out_ratio(as_f64(pp.scores[:, rows]), s_ref) <= 1.0
    gidx = np.ascontiguousarray(pp.idx[:, rows].cpu().numpy())
    for r in range(len(rows)):                 # every sampled row's selection is checked
        nvis = oracle.num_visible(int(ps[0, r]), m, Nc)
        check_topk_band(gidx[0, r], s_ref[0, r], nvis, cfg.k, True)
    o_ref, l_ref = oracle.csa_attn(q_csa[:, rows].contiguous(), oracle.KV(0, bf16_of(ent_c), Nc), gidx,
                                   oracle.KV(0, kv, L), W, ps)
    assert np.abs(as_f64(pp.out_csa[:, rows]) - o_ref).max() <= 2e-2
    assert np.abs(as_f64(pp.lse_csa[:, rows]) - l_ref).max() <= 2e-2
    oh_ref, lh_ref = oracle.hca_attn(q_hca[:, rows].contiguous(), oracle.KV(0, bf16_of(ent_h), Nh), Nh, mh,
                                     oracle.KV(0, kv, L), W, ps)
    assert np.abs(as_f64(pp.hca.out[:, rows]) - oh_ref).max() <= 2e-2
    assert pp.status.item() == 0
