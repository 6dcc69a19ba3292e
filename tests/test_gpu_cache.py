"""Decode-time cache maintenance (hcl_cache_append) [Yanbaoke §5 KV cache management;
Austery's talk notes, infrastructure section: a heterogeneous KV cache].

Two sequences decode 640 consecutive tokens each (starting at positions 1001 and 1004, so their
entries complete at different steps) into a CSA layer's cache (raw window and entries as FP8
split rows, MXFP4 index keys) and an HCA layer's cache (bf16 raw window and entries), with and
without the RMSNorm of the entries.  After the last step every cache is compared with a
recomputation from scratch over the whole token history:
  - the raw windows and the index keys bit for bit with the oracle's quantisers applied to the
    generated tokens / keys (those values are exact inputs, so the results are unique);
  - the pooled entries within the compressor tolerance of the oracle's pooling (and RMSNorm),
    after the FP8 quantisation bound for split rows;
  - the pooled entries bit for bit with the library's own batch compressor and quantiser run
    over the full history (the append uses the same arithmetic), which also shows that rows
    past the last completed entry were not written."""
import numpy as np
import pytest
import torch

import oracle
from heavily_compressed_long_b200.api import KV
from synth import gen
from synth.configs import CSA_TINY, scaled
from tests.helpers import as_f64, bf16_out_ratio, cuda

pytestmark = pytest.mark.gpu
T_STEPS = 640


def _split(B, cap, dev="cuda"):
    return (torch.zeros(B, cap, 64, dtype=torch.uint8, device=dev),
            torch.ones(B, cap, dtype=torch.float32, device=dev),
            torch.zeros(B, cap, 64, dtype=torch.bfloat16, device=dev))


def _deq_split(n, s, r):
    """fp64 values of split rows [.., 64 codes], [..], [.., 64 bf16] (decoded by the oracle)."""
    codes = n.cpu().numpy()
    lut = np.array([oracle.e4m3_to_f64(c) for c in range(256)])
    lo = lut[codes] * s.cpu().numpy().astype(np.float64)[..., None]
    return np.concatenate([lo, as_f64(r)], -1)


@pytest.mark.parametrize("norm", [False, True])
def test_cache_append_640_steps(hcl, norm):
    from heavily_compressed_long_b200 import api
    B, d, m, mh, W, dI, S = 2, 128, 4, 128, 128, 64, 128
    t0 = [1001, 1004]
    L = max(t0) + T_STEPS
    cfg = scaled(CSA_TINY, B=B, L=L, seed=777)
    bs = list(range(B))
    x = gen.raw_kv(cfg, bs, 0, L)                       # [B, L, d] bf16
    g = gen.gate(cfg, bs, 0, L)
    nce = -(-L // m)
    kI_full = gen.comp_kv(cfg, bs, nce, tid=91)[..., :dI].contiguous()   # one index key per entry
    b_csa = gen.bias(cfg, 2 * m, 0)
    b_hca = gen.bias(cfg, mh, 1)
    gamma = torch.from_numpy((1.0 + 0.25 * np.random.default_rng(5).standard_normal(d))
                             .astype(np.float32)) if norm else None
    eps = 1e-6
    dev = "cuda"
    xg, gg = cuda(x), cuda(g)
    gam = None if gamma is None else cuda(gamma)

    # ---- caches at the start: entries complete before t0[b] from the batch compressors
    cap_c, cap_h = nce + 8, -(-L // mh) + 2
    kvc_n, kvc_s, kvc_r = _split(B, cap_c)
    kI_p = torch.zeros(B, cap_c, dI // 2, dtype=torch.uint8, device=dev)
    kI_s = torch.zeros(B, cap_c, dI // 32, dtype=torch.uint8, device=dev)
    kvh = torch.zeros(B, cap_h, d, dtype=torch.bfloat16, device=dev)
    rawc = _split(B, W)
    rawh = torch.zeros(B, W, d, dtype=torch.bfloat16, device=dev)
    stc = [torch.zeros(B, S, d, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    sth = [torch.zeros(B, S, d, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    for b in range(B):
        sl = slice(b, b + 1)
        nc0, nh0 = t0[b] // m, t0[b] // mh
        tmp = torch.empty(1, cap_c, d, dtype=torch.bfloat16, device=dev)
        api.hcl_csa_compress(xg[sl, :t0[b]], gg[sl, :t0[b]], cuda(b_csa), m, tmp, 0, nc0, gamma=gam, eps=eps)
        api.hcl_quant_kv_fp8(tmp[:, :nc0].contiguous(), kvc_n[sl, :nc0], kvc_s[sl, :nc0], kvc_r[sl, :nc0])
        api.hcl_quant_mxfp4(cuda(kI_full[sl, :nc0]), kI_p[sl, :nc0], kI_s[sl, :nc0])
        api.hcl_hca_compress(xg[sl, :t0[b]], gg[sl, :t0[b]], cuda(b_hca), mh, kvh[sl], 0, nh0, gamma=gam, eps=eps)
        for u in range(t0[b] - S, t0[b]):
            for st in (stc, sth):
                st[0][b, u % S] = xg[b, u]
                st[1][b, u % S] = gg[b, u]
            rawh[b, u % W] = xg[b, u]
        ring = torch.stack([xg[b, u] for u in range(t0[b] - W, t0[b])])   # tokens in order
        slot_order = [u % W for u in range(t0[b] - W, t0[b])]
        qn, qs, qr = (t.clone() for t in _split(1, W))
        api.hcl_quant_kv_fp8(ring.unsqueeze(0).contiguous(), qn, qs, qr)
        for j, sl_ in enumerate(slot_order):
            rawc[0][b, sl_], rawc[1][b, sl_], rawc[2][b, sl_] = qn[0, j], qs[0, j], qr[0, j]
    KVC, RAWC = KV(kvc_n, kvc_s, kvc_r), KV(*rawc)
    KVH, RAWH = KV(kvh), KV(rawh)

    # ---- 640 decode steps, one append per layer per step
    kIg = cuda(kI_full)
    for s in range(T_STEPS):
        t = torch.tensor([t0[0] + s, t0[1] + s], dtype=torch.int32, device=dev)
        kv_new = torch.stack([xg[b, t0[b] + s] for b in range(B)]).contiguous()
        g_new = torch.stack([gg[b, t0[b] + s] for b in range(B)]).contiguous()
        kI_new = torch.stack([kIg[b, (t0[b] + s) // m] for b in range(B)]).contiguous()
        api.hcl_cache_append(kv_new, g_new, t, stc[0], stc[1], RAWC, kvc=KVC, bias_csa=cuda(b_csa),
                             m=m, kI_new=kI_new, kI=kI_p, kI_sf=kI_s, gamma=gam, eps=eps)
        api.hcl_cache_append(kv_new, g_new, t, sth[0], sth[1], RAWH, kvh=KVH, bias_hca=cuda(b_hca),
                             mh=mh, gamma=gam, eps=eps)
    torch.cuda.synchronize()

    for b in range(B):
        sl = slice(b, b + 1)
        tend = t0[b] + T_STEPS                         # tokens [0, tend) seen
        nc, nh = tend // m, tend // mh                 # entries complete
        xs, gs = x[sl, :tend], g[sl, :tend]
        # raw windows: the last W tokens, by slot, bit for bit
        toks = list(range(tend - W, tend))
        on, os_, orp = oracle.quant_kv_fp8(x[b, toks])
        slots = [u % W for u in toks]
        assert np.array_equal(rawc[0][b, slots].cpu().numpy(), on)
        assert np.array_equal(rawc[1][b, slots].cpu().numpy().view(np.uint32), os_.view(np.uint32))
        assert np.array_equal(gen.bf16_bits(rawc[2][b, slots].cpu()), orp)
        assert torch.equal(rawh[b, slots].cpu(), x[b, toks])
        # index keys: the oracle's MXFP4 of the generated keys, bit for bit
        kp_o, ks_o = oracle.quant_mxfp4(kI_full[b, :nc])
        assert np.array_equal(kI_p[b, :nc].cpu().numpy(), kp_o)
        assert np.array_equal(kI_s[b, :nc].cpu().numpy(), ks_o)
        # CSA entries: oracle pooling (+ RMSNorm) within the FP8 bound
        ref = oracle.compress(xs, gs, b_csa, m, True, 0, nc)[0]
        if norm:
            ref = oracle.rmsnorm(ref, gamma, eps)
        deq = _deq_split(kvc_n[b, :nc], kvc_s[b, :nc], kvc_r[b, :nc])
        amax = np.abs(ref[:, :64]).max(1, keepdims=True)
        err = np.abs(deq[:, :64] - ref[:, :64])
        assert np.all(err <= 0.07 * np.abs(ref[:, :64]) + 2e-3 * amax + 1e-30)
        assert bf16_out_ratio(deq[:, 64:], ref[:, 64:]) <= 1.0
        # ... and bit for bit the batch compressor + quantiser over the whole history
        full = torch.empty(1, cap_c, d, dtype=torch.bfloat16, device=dev)
        api.hcl_csa_compress(xg[sl, :tend], gg[sl, :tend], cuda(b_csa), m, full, 0, nc, gamma=gam, eps=eps)
        fn, fs, fr = (t.clone() for t in _split(1, cap_c))
        api.hcl_quant_kv_fp8(full[:, :nc].contiguous(), fn[:, :nc], fs[:, :nc], fr[:, :nc])
        torch.cuda.synchronize()
        assert torch.equal(kvc_n[b, :nc], fn[0, :nc]) and torch.equal(kvc_s[b, :nc], fs[0, :nc])
        assert torch.equal(kvc_r[b, :nc], fr[0, :nc])
        assert int(kvc_n[b, nc:].count_nonzero()) == 0          # nothing past the last entry
        # HCA entries (bf16): oracle within 1 bf16 ulp + 1e-3, and the batch compressor bitwise
        ref_h = oracle.compress(xs, gs, b_hca, mh, False, 0, nh)[0]
        if norm:
            ref_h = oracle.rmsnorm(ref_h, gamma, eps)
        assert bf16_out_ratio(as_f64(kvh[b, :nh]), ref_h) <= 1.0
        fullh = torch.zeros(1, cap_h, d, dtype=torch.bfloat16, device=dev)
        api.hcl_hca_compress(xg[sl, :tend], gg[sl, :tend], cuda(b_hca), mh, fullh, 0, nh, gamma=gam, eps=eps)
        torch.cuda.synchronize()
        assert torch.equal(kvh[b], fullh[0])
