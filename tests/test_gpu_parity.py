"""GPU parity of every libhcl kernel against the CPU oracle, on seeded inputs that span several
tiles and a ragged tail.  Inputs come from synth/ or the oracle; every expected value is the
oracle's, computed from those inputs.  Two results are not unique, and there a GPU output is
checked for validity instead: a top-k selection inside the ambiguity band (the oracle then
attends over the GPU's validated selection), and the fused step's exact top-k of the very bf16
scores the GPU produced (those scores are first checked against the oracle's).  Tolerances: entries and scores rel <= 1e-3 (norm-wise
per row, fp32 output) or 1 bf16 ulp (bf16 output); top-k exact for identical scores;
attention max abs <= 2e-2 (bf16 KV) / 5e-2 (FP8 non-RoPE dims); quantisers bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from synth import gen
from tests.helpers import as_f64, bf16_out_ratio, check_topk_band, cuda, rel_rowwise

pytestmark = pytest.mark.gpu
RNG = np.random.default_rng(20261202)


def rbf16(*shape, std=1.0):
    return gen.to_bf16((RNG.standard_normal(shape) * std).astype(np.float32))


def u8(t):
    return t.cpu().numpy().astype(np.uint8)


# =========================================================================================
# a3: quantisers (bit-exact)

def test_quant_kv_fp8_bitexact(hcl):
    x = rbf16(1000, 128, std=2.0)
    x[3] = 0
    x[7, :64] = 0
    x[11, :64] = gen.to_bf16(np.full(64, 3e-38, np.float32))  # tiny values
    x[13, 5] = 1e30
    nope, scale, rope = oracle.quant_kv_fp8(x)
    xg = cuda(x)
    gn = torch.empty(1000, 64, dtype=torch.uint8, device="cuda")
    gs = torch.empty(1000, dtype=torch.float32, device="cuda")
    gr = torch.empty(1000, 64, dtype=torch.bfloat16, device="cuda")
    hcl.hcl_quant_kv_fp8(xg, gn, gs, gr)
    torch.cuda.synchronize()
    assert np.array_equal(u8(gn), nope)
    assert np.array_equal(gs.cpu().numpy().view(np.uint32), scale.view(np.uint32))
    assert np.array_equal(gen.bf16_bits(gr.cpu()), rope)


def test_quant_mxfp4_bitexact(hcl):
    x = rbf16(777, 64, std=1.5)
    x[0] = 0                                                     # zero blocks
    x[1, :32] = gen.to_bf16(RNG.standard_normal(32).astype(np.float32) * 1e-38)  # subnormal range
    x[2, 32:] = gen.to_bf16(RNG.standard_normal(32).astype(np.float32) * 1e30)
    x[3] = gen.to_bf16(np.tile(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0], np.float32), 8))
    packed, sf = oracle.quant_mxfp4(x)
    gp = torch.empty(777, 32, dtype=torch.uint8, device="cuda")
    gs = torch.empty(777, 2, dtype=torch.uint8, device="cuda")
    hcl.hcl_quant_mxfp4(cuda(x), gp, gs)
    torch.cuda.synchronize()
    assert np.array_equal(u8(gs), sf)
    assert np.array_equal(u8(gp), packed)


# =========================================================================================
# a1/a2: compressor

@pytest.mark.parametrize("B,L,m,overlap", [(1, 4096, 4, True), (2, 1027, 4, True),
                                           (2, 128 * 37 + 5, 128, False), (1, 300, 1, False)])
def test_compress(hcl, B, L, m, overlap):
    d = 128
    x, g = rbf16(B, L, d), rbf16(B, L, d)
    span = 2 * m if overlap else m
    bias = torch.from_numpy((RNG.standard_normal(span) * 0.1).astype(np.float32))
    ref = oracle.compress(x, g, bias, m, overlap)
    n = ref.shape[1]
    fn = hcl.hcl_csa_compress if overlap else hcl.hcl_hca_compress
    out32 = torch.full((B, n + 3, d), float("nan"), device="cuda")
    fn(cuda(x), cuda(g), cuda(bias), m, out32)
    out16 = torch.empty(B, n, d, dtype=torch.bfloat16, device="cuda")
    fn(cuda(x), cuda(g), cuda(bias), m, out16)
    torch.cuda.synchronize()
    assert rel_rowwise(as_f64(out32[:, :n]), ref) <= 1e-3
    assert torch.isnan(out32[:, n:]).all()              # nothing written past the entries
    assert bf16_out_ratio(as_f64(out16), ref) <= 1.0


@pytest.mark.parametrize("B,L,m,overlap", [(1, 4096, 4, True), (2, 1027, 4, True),
                                           (2, 128 * 37 + 5, 128, False)])
def test_compress_rmsnorm(hcl, B, L, m, overlap):
    """The compressor's RMSNorm epilogue against or_rmsnorm applied to or_compress (entries
    normalised after pooling, before the output rounding)."""
    d, eps = 128, 1e-6
    x, g = rbf16(B, L, d), rbf16(B, L, d)
    span = 2 * m if overlap else m
    bias = torch.from_numpy((RNG.standard_normal(span) * 0.1).astype(np.float32))
    gamma = torch.from_numpy((1.0 + 0.25 * RNG.standard_normal(d)).astype(np.float32))
    ref = oracle.rmsnorm(oracle.compress(x, g, bias, m, overlap), gamma, eps)
    n = ref.shape[1]
    fn = hcl.hcl_csa_compress if overlap else hcl.hcl_hca_compress
    out32 = torch.empty(B, n, d, device="cuda")
    fn(cuda(x), cuda(g), cuda(bias), m, out32, gamma=cuda(gamma), eps=eps)
    out16 = torch.empty(B, n, d, dtype=torch.bfloat16, device="cuda")
    fn(cuda(x), cuda(g), cuda(bias), m, out16, gamma=cuda(gamma), eps=eps)
    torch.cuda.synchronize()
    assert rel_rowwise(as_f64(out32), ref) <= 1e-3
    assert bf16_out_ratio(as_f64(out16), ref) <= 1.0


def test_compress_entry_range(hcl):
    B, L, d = 1, 2000, 128
    x, g = rbf16(B, L, d), rbf16(B, L, d)
    bias = torch.from_numpy((RNG.standard_normal(8) * 0.1).astype(np.float32))
    ref = oracle.compress(x, g, bias, 4, True, 100, 137)
    out = torch.zeros(B, 500, d, device="cuda")
    hcl.hcl_csa_compress(cuda(x), cuda(g), cuda(bias), 4, out, 100, 137)
    torch.cuda.synchronize()
    o = as_f64(out)
    assert rel_rowwise(o[:, 100:137], ref) <= 1e-3
    assert np.all(o[:, :100] == 0) and np.all(o[:, 137:] == 0)


# =========================================================================================
# a4: lightning indexer

def _positions(B, Tq, hi):
    return torch.from_numpy(RNG.integers(0, hi, (B, Tq)).astype(np.int32))


@pytest.mark.parametrize("B,Tq,HI,Nc,cap", [(1, 1, 4, 1024, 1024), (3, 1, 8, 1000, 1003),
                                            (2, 1, 16, 3001, 3001), (2, 37, 16, 700, 704),
                                            (1, 20, 5, 257, 260)])
def test_index_scores_bf16(hcl, B, Tq, HI, Nc, cap):
    qI, kI = rbf16(B, Tq, HI, 64), rbf16(B, cap, 64)
    w = torch.from_numpy(RNG.random((B, Tq, HI)).astype(np.float32))
    pos = _positions(B, Tq, 4 * Nc + 8)
    pos[0, 0] = 4 * Nc + 100                               # all visible
    if Tq > 1:
        pos[0, 1] = 2                                       # nothing visible
    ref = oracle.index_scores(oracle.FMT_BF16, qI, w, kI[:, :Nc], pos, 4)
    out = torch.empty(B, Tq, Nc, device="cuda")
    hcl.hcl_csa_index_scores(hcl.HCL_BF16, cuda(qI), cuda(w), cuda(kI), cuda(pos), 4, out, Nc=Nc)
    torch.cuda.synchronize()
    assert rel_rowwise(as_f64(out), ref) <= 1e-3


@pytest.mark.parametrize("B,Tq,Nc,cap", [(2, 1, 2999, 3000), (1, 1, 262144 // 16, 262144 // 16),
                                         (1, 9, 500, 512)])
def test_index_scores_mxfp4_bf16_scores(hcl, B, Tq, Nc, cap):
    HI = 16
    qb, kb = rbf16(B, Tq, HI, 64), rbf16(B, cap, 64)
    qp, qs = oracle.quant_mxfp4(qb)
    kp, ks = oracle.quant_mxfp4(kb)
    w = torch.from_numpy(RNG.random((B, Tq, HI)).astype(np.float32))
    pos = torch.full((B, Tq), 4 * cap + 3, dtype=torch.int32)
    if Tq > 1:
        pos[0] = torch.arange(Tq) * 97
    ref = oracle.index_scores(oracle.FMT_MXFP4, qp, w, kp[:, :Nc], pos, 4, qI_sf=qs,
                              kI_sf=ks[:, :Nc], bf16_scores=True)
    out = torch.empty(B, Tq, Nc, dtype=torch.bfloat16, device="cuda")
    t = lambda a: cuda(torch.from_numpy(np.ascontiguousarray(a)))
    hcl.hcl_csa_index_scores(hcl.HCL_MXFP4, t(qp), cuda(w), t(kp), cuda(pos), 4, out, Nc=Nc,
                             qI_sf=t(qs), kI_sf=t(ks))
    torch.cuda.synchronize()
    assert bf16_out_ratio(as_f64(out), ref) <= 1.0


@pytest.mark.parametrize("B,Nc,cap,nvis,fp32", [
    (3, 5000, 5008, (5000, 1237, 0), True),     # vector fp32 stores, visibility inside a row
    (3, 5000, 5008, (4999, 1, 2050), False),    # vector bf16 stores, ragged visibility
    (1, 70001, 70008, (70001,), False),         # many blocks per row, scalar tail stores
    (2, 512, 512, (512, 511), True),            # exactly one 512-key tile
    (1, 3, 8, (3,), True),                      # fewer keys than one packed row group
])
def test_index_scores_mxfp4_decode(hcl, B, Nc, cap, nvis, fp32):
    """Decode (one query) with MXFP4 operands: keys packed four to a 128-byte row.  Covers
    partial tiles, rows whose visible prefix ends inside a four-key group and both score
    formats (the in-kernel quantisation of bf16 index queries is covered by the fused decode
    step's bitwise comparison with the separate calls)."""
    HI = 16
    qb, kb = rbf16(B, 1, HI, 64), rbf16(B, cap, 64)
    qp, qs = oracle.quant_mxfp4(qb)
    kp, ks = oracle.quant_mxfp4(kb)
    w = torch.from_numpy(RNG.random((B, 1, HI)).astype(np.float32))
    pos = torch.tensor([[4 * v - 1 if v > 0 else 2] for v in nvis], dtype=torch.int32)
    ref = oracle.index_scores(oracle.FMT_MXFP4, qp, w, kp[:, :Nc], pos, 4, qI_sf=qs,
                              kI_sf=ks[:, :Nc], bf16_scores=not fp32)
    t = lambda a: cuda(torch.from_numpy(np.ascontiguousarray(a)))
    dt = torch.float32 if fp32 else torch.bfloat16
    out = torch.empty(B, 1, Nc, dtype=dt, device="cuda")
    hcl.hcl_csa_index_scores(hcl.HCL_MXFP4, t(qp), cuda(w), t(kp), cuda(pos), 4, out, Nc=Nc,
                             qI_sf=t(qs), kI_sf=t(ks))
    torch.cuda.synchronize()
    if fp32:
        assert rel_rowwise(as_f64(out), ref) <= 1e-3
    else:
        assert bf16_out_ratio(as_f64(out), ref) <= 1.0


def test_index_scores_deterministic(hcl):
    qI, kI = cuda(rbf16(2, 1, 16, 64)), cuda(rbf16(2, 5000, 64))
    w = cuda(torch.rand(2, 1, 16))
    pos = cuda(torch.full((2, 1), 20000, dtype=torch.int32))
    a = torch.empty(2, 1, 5000, device="cuda")
    b = torch.empty_like(a)
    hcl.hcl_csa_index_scores(hcl.HCL_BF16, qI, w, kI, pos, 4, a)
    hcl.hcl_csa_index_scores(hcl.HCL_BF16, qI, w, kI, pos, 4, b)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# =========================================================================================
# a5: top-k (identical scores on both sides -> exact)

@pytest.mark.parametrize("fmt,B,Tq,Nc,k", [("fp32", 1, 1, 1024, 64), ("fp32", 4, 1, 32768, 512),
                                           ("bf16", 2, 1, 262144, 1024), ("bf16", 3, 5, 66560, 1024),
                                           ("fp32", 2, 3, 5000, 4096), ("bf16", 1, 2, 70000, 1)])
def test_topk_exact(hcl, fmt, B, Tq, Nc, k):
    s = np.round(RNG.standard_normal((B, Tq, Nc)) * 4, 2).astype(np.float32)   # many ties
    s[0, 0, 100:400] = 7.25
    pos = torch.full((B, Tq), 4 * Nc + 10, dtype=torch.int32)
    if Tq > 1:
        pos[-1, 1] = 4 * (Nc // 3) + 1
    if fmt == "bf16":
        st = gen.to_bf16(s)
        sref = st.double().numpy()
    else:
        st = torch.from_numpy(s)
        sref = s.astype(np.float64)
    want = oracle.topk(sref, pos, 4, k)
    out = torch.empty(B, Tq, k, dtype=torch.int32, device="cuda")
    hcl.hcl_csa_topk(cuda(st), cuda(pos), 4, k, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), want)


@pytest.mark.parametrize("off,B,Nc,k,kind", [
    (3, 3, 100003, 1024, "ties"),      # rows start at every alignment, heavy ties
    (5, 2, 262147, 1024, "normal"),
    (1, 1, 9999, 2000, "ties"),
    (7, 2, 40000, 1, "ties"),
    (2, 1, 50000, 1000, "equal"),      # one value everywhere: the tie run spans every block
    (0, 2, 131072, 1024, "runs"),      # long equal runs across block boundaries
])
def test_topk_bf16_layouts(hcl, off, B, Nc, k, kind):
    """bf16 rows whose first key sits at any position of a 16-byte vector (the score tensor is
    an element-offset view), lengths that are no multiple of 8, and threshold ties spread over
    the cluster's blocks."""
    if kind == "equal":
        s = np.full((B, 1, Nc), 3.0, np.float32)
    elif kind == "runs":
        s = np.repeat(np.round(RNG.standard_normal((B, 1, Nc // 4096)), 1), 4096, axis=2)
        s = s.astype(np.float32)
    elif kind == "ties":
        s = np.round(RNG.standard_normal((B, 1, Nc)) * 2, 1).astype(np.float32)
    else:
        s = RNG.standard_normal((B, 1, Nc)).astype(np.float32)
    st = gen.to_bf16(s)
    pos = torch.full((B, 1), 4 * Nc + 3, dtype=torch.int32)
    want = oracle.topk(st.double().numpy(), pos, 4, k)
    store = torch.zeros(B * Nc + 16, dtype=torch.bfloat16, device="cuda")
    view = store[off:off + B * Nc].view(B, 1, Nc)
    view.copy_(cuda(st))
    out = torch.empty(B, 1, k, dtype=torch.int32, device="cuda")
    hcl.hcl_csa_topk(view, cuda(pos), 4, k, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), want)


def test_topk_fewer_visible_and_negative(hcl):
    s = torch.randn(3, 2, 5000)
    s[1] = -torch.rand(2, 5000) * 1e3
    s[2, :, ::7] = float("-inf")
    pos = torch.tensor([[11, -1], [4 * 5000, 4 * 300], [4 * 5000 + 3, 999]], dtype=torch.int32)
    want = oracle.topk(s.double().numpy(), pos, 4, 512)
    out = torch.empty(3, 2, 512, dtype=torch.int32, device="cuda")
    hcl.hcl_csa_topk(cuda(s), cuda(pos), 4, 512, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), want)


# =========================================================================================
# a6/a7: attention (same idx on both sides)

def _kv_pair(ent, raw, fp8):
    """oracle KV + GPU KV of the same stored values (FP8 split rows quantised by the oracle)."""
    if not fp8:
        return (oracle.KV(oracle.FMT_BF16, ent, ent.shape[1]), hcl_kv(ent),
                oracle.KV(oracle.FMT_BF16, raw, raw.shape[1]), hcl_kv(raw))
    out = []
    for t in (ent, raw):
        n, s, r = oracle.quant_kv_fp8(t)
        out.append(oracle.KV(oracle.FMT_FP8SPLIT, n, t.shape[1], scale=s, rope=r))
        out.append(hcl_kv(torch.from_numpy(n), torch.from_numpy(s), torch.from_numpy(r.view(np.int16)).view(torch.bfloat16)))
    return tuple(out)


def _split3(nsr, cap):
    """(codes, scale, rope) of oracle.quant_kv_fp8 -> the arguments of an FP8-split oracle.KV."""
    n, sc, r = nsr
    return n, cap, sc, r


def hcl_kv(data, scale=None, rope=None):
    from heavily_compressed_long_b200.api import KV
    return KV(cuda(data), None if scale is None else cuda(scale), None if rope is None else cuda(rope))


@pytest.mark.parametrize("B,Tq,H,Nc,k,W,fp8,sink", [
    (1, 1, 8, 1024, 64, 64, False, False),      # cfg-1 shape
    (2, 1, 64, 5000, 512, 128, False, True),    # split-KV + sink
    (2, 1, 128, 9000, 1024, 128, True, False),  # cfg-4 shape, FP8 split rows
    (2, 1, 100, 5000, 512, 128, True, True),    # heads over two blocks: slices of 64 and 36
    (3, 1, 72, 4000, 300, 64, False, False),    # slices of 64 and 8
    (1, 3, 16, 700, 100, 37, False, False),     # ragged list, several queries
    (2, 2, 128, 3000, 64, 0, True, True),       # no window
    (1, 1, 128, 9000, 4096, 128, True, True),   # long list: splits merged via the workspace
    # prefill chunks (>= 32 groups of 128 / H queries): the tcgen05 flash kernel, each query's
    # own selection concatenated per block
    (1, 80, 64, 3000, 256, 64, False, False),
    (2, 130, 32, 2000, 100, 37, True, True),
])
def test_csa_attn(hcl, B, Tq, H, Nc, k, W, fp8, sink):
    d, L = 128, 4 * Nc + 11
    ent, raw = rbf16(B, Nc, d), rbf16(B, L, d)
    q = rbf16(B, Tq, H, d)
    pos = torch.from_numpy(RNG.integers(L - 300, L, (B, Tq)).astype(np.int32))
    idx = np.stack([[np.sort(RNG.choice(Nc, k, replace=False)) for _ in range(Tq)] for _ in range(B)]).astype(np.int32)
    idx[0, 0, -5:] = -1
    sk = torch.from_numpy(RNG.standard_normal(H).astype(np.float32)) if sink else None
    okc, gkc, okr, gkr = _kv_pair(ent, raw, fp8)
    o_ref, l_ref = oracle.csa_attn(q, okc, idx, okr, W, pos, sink=sk)
    out = torch.empty(B, Tq, H, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Tq, H, device="cuda")
    hcl.hcl_csa_sparse_attn(cuda(q), gkc, Nc, cuda(torch.from_numpy(idx)), gkr, L, W, cuda(pos), out,
                            lse=lse, sink=None if sk is None else cuda(sk))
    torch.cuda.synchronize()
    tol = 5e-2 if fp8 else 2e-2
    assert np.abs(as_f64(out) - o_ref).max() <= tol
    assert np.abs(as_f64(lse) - l_ref).max() <= tol


def _normed_q(q, gamma, eps):
    """The oracle's RMSNorm of every query head row, rounded to bf16 (the attention's operand
    precision), as a bf16 tensor."""
    qn = oracle.round_bf16(oracle.rmsnorm(q, gamma, eps))
    return torch.from_numpy(qn.astype(np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("B,Tq,H,Nc,k,W,fp8", [
    (1, 1, 8, 1024, 64, 64, False),             # cfg-1 shape
    (2, 1, 128, 9000, 1024, 128, True),         # cfg-4 shape (tcgen05 decode kernel)
    (1, 3, 16, 700, 100, 37, False),            # several queries (mma.sync kernel)
])
def test_csa_attn_query_rmsnorm(hcl, B, Tq, H, Nc, k, W, fp8):
    """Attention on RMS-normalised queries: the oracle normalises q (fp64, then bf16) and
    attends; the kernels normalise in their query load."""
    d, L, eps = 128, 4 * Nc + 11, 1e-6
    ent, raw = rbf16(B, Nc, d), rbf16(B, L, d)
    q = rbf16(B, Tq, H, d, std=3.0)
    gamma = torch.from_numpy((1.0 + 0.25 * RNG.standard_normal(d)).astype(np.float32))
    pos = torch.from_numpy(RNG.integers(L - 300, L, (B, Tq)).astype(np.int32))
    idx = np.stack([[np.sort(RNG.choice(Nc, k, replace=False)) for _ in range(Tq)] for _ in range(B)]).astype(np.int32)
    okc, gkc, okr, gkr = _kv_pair(ent, raw, fp8)
    o_ref, l_ref = oracle.csa_attn(_normed_q(q, gamma, eps), okc, idx, okr, W, pos)
    out = torch.empty(B, Tq, H, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Tq, H, device="cuda")
    hcl.hcl_csa_sparse_attn(cuda(q), gkc, Nc, cuda(torch.from_numpy(idx)), gkr, L, W, cuda(pos), out,
                            lse=lse, q_gamma=cuda(gamma), q_eps=eps)
    torch.cuda.synchronize()
    tol = 5e-2 if fp8 else 2e-2
    assert np.abs(as_f64(out) - o_ref).max() <= tol
    assert np.abs(as_f64(lse) - l_ref).max() <= tol


@pytest.mark.parametrize("Tq", [40, 300])     # mma.sync kernel, tcgen05 flash kernel
def test_hca_attn_query_rmsnorm(hcl, Tq):
    B, H, L, W, d, mh, eps = 2, 16, 128 * 30 + 9, 128, 128, 128, 1e-6
    Nh = -(-L // mh)
    ent, raw = rbf16(B, Nh, d), rbf16(B, L, d)
    q = rbf16(B, Tq, H, d, std=0.5)
    gamma = torch.from_numpy((1.0 + 0.25 * RNG.standard_normal(d)).astype(np.float32))
    pos = torch.arange(L - Tq, L, dtype=torch.int32).repeat(B, 1).contiguous()
    okc, gkc, okr, gkr = _kv_pair(ent, raw, False)
    o_ref, l_ref = oracle.hca_attn(_normed_q(q, gamma, eps), okc, Nh, mh, okr, W, pos)
    out = torch.empty(B, Tq, H, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Tq, H, device="cuda")
    hcl.hcl_hca_dense_attn(cuda(q), gkc, Nh, mh, gkr, L, W, cuda(pos), out, lse=lse,
                           q_gamma=cuda(gamma), q_eps=eps)
    torch.cuda.synchronize()
    assert np.abs(as_f64(out) - o_ref).max() <= 2e-2
    assert np.abs(as_f64(lse) - l_ref).max() <= 2e-2


@pytest.mark.parametrize("B,Tq,H,L,W,fp8,sink", [
    (2, 64, 16, 128 * 40, 128, False, False),
    (2, 1, 16, 128 * 40 + 77, 128, False, False),
    (1, 37, 64, 128 * 20 + 3, 128, False, False),
    (1, 5, 128, 128 * 9, 16, True, False),
    # >= 32 query groups: the tcgen05 flash kernel (prefill), with ragged last groups
    (2, 300, 16, 128 * 20 + 3, 128, False, False),
    (1, 261, 32, 128 * 33 + 100, 128, True, True),
    (1, 70, 64, 128 * 12, 200, False, True),
    (1, 40, 128, 128 * 4 + 9, 128, False, False),
    # bf16 rows: two query groups per block (warp-specialised); an odd group count leaves the
    # last block's second tile empty; a chunk at the start of the context (no visible entries
    # for the first queries, windows reaching before token 0)
    (3, 520, 16, 128 * 40 + 1, 128, False, False),
    (1, 300, 16, 300, 128, False, True),
    (1, 33 * 4, 32, 128 * 7 + 5, 64, False, False),
])
def test_hca_attn(hcl, B, Tq, H, L, W, fp8, sink):
    d, mh = 128, 128
    Nh = -(-L // mh)
    ent, raw = rbf16(B, Nh, d), rbf16(B, L, d)
    q = rbf16(B, Tq, H, d)
    pos = torch.arange(L - Tq, L, dtype=torch.int32).repeat(B, 1).contiguous()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sk = torch.from_numpy(RNG.standard_normal(H).astype(np.float32)) if sink else None
    okc, gkc, okr, gkr = _kv_pair(ent, raw, fp8)
    o_ref, l_ref = oracle.hca_attn(q, okc, Nh, mh, okr, W, pos, sink=sk)
    out = torch.empty(B, Tq, H, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Tq, H, device="cuda")
    hcl.hcl_hca_dense_attn(cuda(q), gkc, Nh, mh, gkr, L, W, cuda(pos), out, lse=lse,
                           sink=None if sk is None else cuda(sk), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    tol = 5e-2 if fp8 else 2e-2
    assert np.abs(as_f64(out) - o_ref).max() <= tol
    assert np.abs(as_f64(lse) - l_ref).max() <= tol


def test_attn_ring_window(hcl):
    B, H, d, W, Nc = 2, 16, 128, 128, 500
    L = 4 * Nc
    raw = rbf16(B, L, d)
    ring = torch.zeros(B, W, d, dtype=torch.bfloat16)
    for t in range(L - W, L):
        ring[:, t % W] = raw[:, t]
    ent, q = rbf16(B, Nc, d), rbf16(B, 1, H, d)
    pos = torch.full((B, 1), L - 1, dtype=torch.int32)
    idx = torch.from_numpy(np.sort(RNG.choice(Nc, (B, 1, 64)), -1).astype(np.int32))
    o_ref, _ = oracle.csa_attn(q, oracle.KV(0, ent, Nc), idx, oracle.KV(0, raw, L), W, pos)
    out = torch.empty(B, 1, H, d, dtype=torch.bfloat16, device="cuda")
    hcl.hcl_csa_sparse_attn(cuda(q), hcl_kv(ent), Nc, cuda(idx), hcl_kv(ring), L, W, cuda(pos), out)
    torch.cuda.synchronize()
    assert np.abs(as_f64(out) - o_ref).max() <= 2e-2


# =========================================================================================
# failure detection (no GPU fault: bounded waits and skipped out-of-range indices)

def test_bounded_wait_reports_timeout(hcl):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    hcl.hcl_selftest_bounded_wait(status, limit_us=2000)
    torch.cuda.synchronize()
    assert status.item() & 8
    x = torch.ones(1000, device="cuda")                  # the context is still usable
    assert float((x * 2).sum()) == 2000.0


def test_out_of_range_index_is_skipped_and_reported(hcl):
    B, H, d, Nc, W = 1, 16, 128, 300, 16
    L = 4 * Nc
    ent, raw, q = rbf16(B, Nc, d), rbf16(B, L, d), rbf16(B, 1, H, d)
    pos = torch.full((B, 1), L - 1, dtype=torch.int32)
    idx = torch.tensor([[[3, 17, 250, Nc + 5, 10 ** 6, -7]]], dtype=torch.int32)
    clean = torch.tensor([[[3, 17, 250, -1, -1, -1]]], dtype=torch.int32)
    o_ref, _ = oracle.csa_attn(q, oracle.KV(0, ent, Nc), clean, oracle.KV(0, raw, L), W, pos)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(B, 1, H, d, dtype=torch.bfloat16, device="cuda")
    hcl.hcl_csa_sparse_attn(cuda(q), hcl_kv(ent), Nc, cuda(idx), hcl_kv(raw), L, W, cuda(pos), out,
                            status=status)
    torch.cuda.synchronize()
    assert status.item() & 16
    assert np.abs(as_f64(out) - o_ref).max() <= 2e-2


def test_invalid_arguments_rejected(hcl):
    from heavily_compressed_long_b200._lib import HclError
    x = torch.zeros(10, 48, dtype=torch.bfloat16, device="cuda")
    p = torch.empty(10, 24, dtype=torch.uint8, device="cuda")
    s = torch.empty(10, 1, dtype=torch.uint8, device="cuda")
    with pytest.raises(HclError):
        hcl.hcl_quant_mxfp4(x, p, s)                       # cols not a multiple of 32
    q = torch.zeros(1, 1, 4, 32, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(HclError):                          # dI != 64 is unsupported
        hcl.hcl_csa_index_scores(hcl.HCL_BF16, q, torch.ones(1, 1, 4, device="cuda"),
                                 torch.zeros(1, 8, 32, dtype=torch.bfloat16, device="cuda"),
                                 torch.zeros(1, 1, dtype=torch.int32, device="cuda"), 4,
                                 torch.empty(1, 1, 8, device="cuda"))


# =========================================================================================
# fused decode step: MXFP4 keys + bf16 scores select from the indexer's per-16-entry summaries

@pytest.mark.parametrize("B,Nc,k,nvis,ties,plant,qnorm", [
    (3, 70000, 1024, (70000, 5000, 700), False, None, False),  # the last row: fewer than k visible
    (2, 40000, 512, (40000, 39999), True, None, False),   # many equal scores, visibility mid-group
    (1, 4096, 1024, (1030,), True, None, False),          # just above k visible
    (2, 262144, 1024, (262144, 131075), False, None, False),   # full decode length
    (2, 262144, 1024, (262144, 262143), False, None, True),    # with RMS-normalised queries
    # keys doubled in the groups the top-k samples (every 16th group) of the first P*16
    # groups: the sampled lower bound overshoots, so the exact k-th largest maximum is taken;
    # P = 200 keeps the multi-candidate groups within the shared-memory pool, P = 1024 does not
    (1, 262144, 1024, (262144,), False, (200, 2.0), False),
    (1, 262144, 1024, (262144,), False, (1024, 2.0), False),
])
def test_decode_step_group_maxima(hcl, B, Nc, k, nvis, ties, plant, qnorm):
    """The fused step's top-k (group summaries lower bound): the GPU's bf16 scores against the
    oracle's scores of the same MXFP4 operands (quantised by the oracle); the selection against
    the oracle's top-k with the ambiguity band and, exactly, against the oracle's top-k of the
    very scores the GPU produced (the kernel must select exactly, ties to the lower index);
    attention against the oracle over that selection; the fused step (selection + attention in
    one kernel) with the same selection bit for bit and its attention against the oracle."""
    from heavily_compressed_long_b200.api import HCL_BF16, HCL_MXFP4, KV
    from heavily_compressed_long_b200.pipeline import CsaDecode
    H, HI, W, d = 16, 16, 128, 128
    L = 4 * Nc
    kb = rbf16(B, Nc, 64)
    if ties:                                   # few distinct key rows -> heavily tied scores
        kb = kb[:, RNG.integers(0, 37, Nc)]
    if plant is not None:
        P, gain = plant
        e = np.arange(Nc)
        sampled = torch.from_numpy((((e // 16) % 16) == 0) & (e < 256 * P))
        kf = kb.float()
        kf[:, sampled] *= gain                 # a power of two: exact in bf16 and MXFP4
        kb = kf.to(torch.bfloat16)
    kp = torch.empty(B, Nc, 32, dtype=torch.uint8, device="cuda")
    ks = torch.empty(B, Nc, 2, dtype=torch.uint8, device="cuda")
    hcl.hcl_quant_mxfp4(cuda(kb), kp, ks)
    ent = rbf16(B, Nc, d)
    cn = torch.empty(B, Nc, 64, dtype=torch.uint8, device="cuda")
    cs = torch.empty(B, Nc, dtype=torch.float32, device="cuda")
    cr = torch.empty(B, Nc, 64, dtype=torch.bfloat16, device="cuda")
    hcl.hcl_quant_kv_fp8(cuda(ent), cn, cs, cr)
    raw = rbf16(B, W, d)
    rn = torch.empty(B, W, 64, dtype=torch.uint8, device="cuda")
    rs = torch.empty(B, W, dtype=torch.float32, device="cuda")
    rr = torch.empty(B, W, 64, dtype=torch.bfloat16, device="cuda")
    hcl.hcl_quant_kv_fp8(cuda(raw), rn, rs, rr)
    q, qI = rbf16(B, 1, H, d), rbf16(B, 1, HI, 64)
    w = torch.from_numpy(RNG.random((B, 1, HI)).astype(np.float32))
    pos = torch.tensor([[4 * v - 1] for v in nvis], dtype=torch.int32)
    gamma = (torch.from_numpy((1.0 + 0.25 * RNG.standard_normal(d)).astype(np.float32))
             if qnorm else None)
    pipe = CsaDecode(cuda(q), cuda(qI), cuda(w), kp, KV(cn, cs, cr), Nc, KV(rn, rs, rr), L, W,
                     cuda(pos), m=4, k=k, op_fmt=HCL_MXFP4, score_fmt=HCL_BF16, kI_sf=ks,
                     q_gamma=None if gamma is None else cuda(gamma))
    pipe.step_parts()
    torch.cuda.synchronize()
    kpo, kso = oracle.quant_mxfp4(kb)
    assert np.array_equal(kp.cpu().numpy(), kpo) and np.array_equal(ks.cpu().numpy(), kso)
    qpo, qso = oracle.quant_mxfp4(qI)
    s_ref = oracle.index_scores(oracle.FMT_MXFP4, qpo, w, kpo, pos, 4, qI_sf=qso, kI_sf=kso,
                                bf16_scores=True)
    assert bf16_out_ratio(as_f64(pipe.scores), s_ref) <= 1.0
    gidx = pipe.idx.cpu().numpy()
    for b in range(B):
        check_topk_band(gidx[b, 0], s_ref[b, 0], min(nvis[b], Nc), k, True)
    want = oracle.topk(as_f64(pipe.scores), pos, 4, k)
    assert np.array_equal(gidx, want)
    okc = oracle.KV(oracle.FMT_FP8SPLIT, *_split3(oracle.quant_kv_fp8(ent), Nc))
    okr = oracle.KV(oracle.FMT_FP8SPLIT, *_split3(oracle.quant_kv_fp8(raw), W))
    o_ref, l_ref = oracle.csa_attn(q if gamma is None else _normed_q(q, gamma, 1e-6), okc, gidx,
                                   okr, W, pos)
    assert np.abs(as_f64(pipe.out) - o_ref).max() <= 5e-2
    assert np.abs(as_f64(pipe.lse) - l_ref).max() <= 5e-2
    # the fused C-ABI step (selection and attention in one cluster kernel per sequence): the
    # same selection bit for bit, and its attention against the oracle over it
    idx1 = pipe.idx.clone()
    pipe.idx.fill_(-7)
    pipe.out.zero_()
    pipe.step()
    torch.cuda.synchronize()
    assert torch.equal(pipe.idx, idx1)
    assert np.abs(as_f64(pipe.out) - o_ref).max() <= 5e-2
    assert np.abs(as_f64(pipe.lse) - l_ref).max() <= 5e-2
    assert pipe.status.item() == 0
