"""Context-parallel CSA decode through the CUDA library on one GPU.

The ranks' phases of heavily_compressed_long_b200.cp.CsaDecodeCP run one after another in one
process and the all-gathers are done by stacking the ranks' tensors (no kernel ever waits on
another rank).  Checked against the oracle: the selection outside the ambiguity band equals the
oracle's top-k over the whole sequence and is identical on every rank, and bit for bit the
selection of the single-device path (same per-entry scores); the merged attention within 2e-2
of the oracle over that selection, with and without a sink."""
import numpy as np
import pytest
import torch

import oracle
from heavily_compressed_long_b200.api import HCL_BF16, HCL_FP32, KV
from heavily_compressed_long_b200.cp import CsaDecodeCP
from heavily_compressed_long_b200.pipeline import CsaDecode
from synth import gen
from synth.configs import CSA_TINY, scaled
from tests.helpers import as_f64, check_topk_band, cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,sink", [(2, False), (3, True)])
def test_cp_decode_ranks_on_one_gpu(hcl, world, sink):
    cfg = scaled(CSA_TINY, B=2, L=4 * 5000 + 2, H=16, k=256, W=64, seed=77)
    bs = [0, 1]
    Nc, L, W, m, k, H = cfg.Nc, cfg.L, cfg.W, cfg.m, cfg.k, cfg.H
    kvc = gen.comp_kv(cfg, bs, Nc)
    raw = gen.raw_kv(cfg, bs, 0, L)
    q, qI = gen.queries(cfg, bs), gen.index_queries(cfg, bs)
    w, kI = gen.head_weights(cfg, bs), gen.index_keys(cfg, bs)
    pos = torch.tensor([[L - 1], [L - 37]], dtype=torch.int32)
    sk = torch.from_numpy(np.random.default_rng(3).standard_normal(H).astype(np.float32)) if sink else None
    qg, qIg, wg, posg, rawkv = cuda(q), cuda(qI), cuda(w), cuda(pos), KV(cuda(raw))
    ranks = [CsaDecodeCP(r, world, Nc, L, W, m, k, H, score_fmt=HCL_FP32) for r in range(world)]
    cands = [cp.select_local(qIg, wg, cuda(kI[:, cp.e0:cp.e1]), posg) for cp in ranks]
    gs = torch.stack([c[0] for c in cands])
    gi = torch.stack([c[1] for c in cands])
    parts = [cp.attend(gs, gi, qg, KV(cuda(kvc[:, cp.e0:cp.e1])), rawkv, posg) for cp in ranks]
    sels = [p_[2] for p_ in parts]
    for s_ in sels[1:]:
        assert torch.equal(s_, sels[0])
    go = torch.stack([p_[0] for p_ in parts])
    gl = torch.stack([p_[1] for p_ in parts])
    out, lse = ranks[0].merge(go, gl, sink=None if sk is None else cuda(sk))
    torch.cuda.synchronize()
    sel = sels[0].cpu().numpy()
    # the selection: the oracle's top-k outside the band, and the single-device selection
    s_ref = oracle.index_scores(oracle.FMT_BF16, qI, w, kI, pos, m)
    for b in range(2):
        check_topk_band(sel[b, 0], s_ref[b, 0], oracle.num_visible(int(pos[b, 0]), m, Nc), k, False)
    one = CsaDecode(qg, qIg, wg, cuda(kI), KV(cuda(kvc)), Nc, rawkv, L, W, posg, m=m, k=k,
                    op_fmt=HCL_BF16, score_fmt=HCL_FP32)
    one.step_parts()
    torch.cuda.synchronize()
    assert np.array_equal(one.idx.cpu().numpy(), sel)
    o_ref, l_ref = oracle.csa_attn(q, oracle.KV(0, kvc, Nc), sel, oracle.KV(0, raw, L), W, pos, sink=sk)
    assert np.abs(as_f64(out) - o_ref).max() <= 2e-2
    assert np.abs(as_f64(lse) - l_ref).max() <= 2e-2
