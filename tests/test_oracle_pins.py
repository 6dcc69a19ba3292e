"""Pins of the CPU oracle against what the pages and mathematics fix (no GPU).

Every test here checks the oracle against something other than itself: a library routine
(torch / numpy / scipy), a closed form, an invariant of the method, a value the pages
print, or brute force on tiny inputs.  Together they are chosen so that a dropped term, a
wrong sign, a wrong slot or index, or a transposed operand in the oracle fails at least one
of them (tests/test_oracle_mutants.py plants such mistakes and checks that).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from synth import gen
from synth.configs import CSA_TINY, scaled

GOLD = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def bf16(a):
    return gen.to_bf16(np.asarray(a, np.float32))


def f64(t):
    return t.to(torch.float64).numpy()


def rand_bf16(*shape, std=1.0):
    return bf16(RNG.standard_normal(shape).astype(np.float32) * std)


# =========================================================================================
# scalar formats

def test_bf16_rounding_matches_torch(orc):
    x = np.concatenate([RNG.standard_normal(4000) * 10.0 ** RNG.integers(-30, 30, 4000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.0078125, 3.0e38, 1e-40, -1e-39]])
    x32 = x.astype(np.float32)           # fp32-representable inputs: torch rounds fp32->bf16
    want = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.f64_to_bf16(float(v)) for v in x32], np.uint16)
    assert np.array_equal(got, want)
    # decoding is exact
    assert all(orc.bf16_to_f64(int(h)) == float(torch.tensor([int(np.int16(h))], dtype=torch.int16)
                                               .view(torch.bfloat16).float()) for h in want[:200])


def test_bf16_ties_to_even(orc):
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to the even mantissa (1.0)
    assert orc.f64_to_bf16(1.0 + 2.0 ** -8) == 0x3F80
    assert orc.f64_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert orc.f64_to_bf16(float("inf")) == 0x7F80
    assert orc.f64_to_bf16(-float("inf")) == 0xFF80


def _fixture(name):
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                a, c, v = line.split()
                rows.append((float(a), int(c, 16), float(v)))
    return rows


def test_e4m3_golden_codes(orc):
    for x, code, val in _fixture("e4m3_codes.txt"):
        assert orc.f32_to_e4m3(x) == code, x
        assert orc.e4m3_to_f64(code) == val
        if abs(x) <= 464:   # torch's cast saturates differently above the RNE range
            t = torch.tensor([x], dtype=torch.float32).to(torch.float8_e4m3fn)
            assert t.view(torch.uint8).item() == code, x


def test_e4m3_matches_torch_cast(orc):
    # all finite codes, their midpoints and random values within the finite range
    vals = [orc.e4m3_to_f64(c) for c in range(256) if not (c & 0x7F) == 0x7F]
    mids = [(a + b) / 2 for a, b in zip(sorted(vals)[:-1], sorted(vals)[1:])]
    rnd = list(RNG.uniform(-448, 448, 3000)) + list(RNG.standard_normal(2000) * 1e-2)
    xs = np.array(vals + mids + rnd, np.float32)
    xs = xs[np.abs(xs) <= 448]
    want = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.f32_to_e4m3(float(v)) for v in xs], np.uint8)
    # torch keeps -0 for negative underflow as well; compare codes exactly
    assert np.array_equal(got, want)


def test_e2m1_golden(orc):
    for x, code, val in _fixture("e2m1_rne.txt"):
        assert orc.f32_to_e2m1(x) == code, x
        assert orc.e2m1_to_f64(code) == val
        assert math.copysign(1, orc.e2m1_to_f64(code)) == math.copysign(1, val)


def test_e2m1_is_nearest(orc):
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6.0])
    for x in RNG.uniform(-6, 6, 2000):
        v = orc.e2m1_to_f64(orc.f32_to_e2m1(float(np.float32(x))))
        assert abs(abs(v) - abs(x)) <= np.min(np.abs(grid - abs(x))) + 1e-12


def test_e8m0(orc):
    assert orc.e8m0_to_f64(127) == 1.0
    assert orc.e8m0_to_f64(130) == 8.0
    assert orc.e8m0_to_f64(0) == 2.0 ** -127
    assert math.isnan(orc.e8m0_to_f64(255))


# =========================================================================================
# a3: quantisers

def test_quant_kv_fp8_against_torch(orc):
    kv = rand_bf16(257, 128, std=3.0)
    kv[5, :64] = 0                          # amax = 0 row -> scale 1, zero codes
    nope, scale, rope = orc.quant_kv_fp8(kv)
    x = kv.float().numpy()
    amax = np.abs(x[:, :64]).max(1)
    want_scale = np.where(amax > 0, (amax / np.float32(448.0)).astype(np.float32), np.float32(1))
    assert np.array_equal(scale, want_scale.astype(np.float32))
    q = (x[:, :64] / want_scale[:, None]).astype(np.float32)
    want = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(nope, want)
    assert np.array_equal(rope, gen.bf16_bits(kv[:, 64:]))
    assert np.all(nope[5] == 0) and scale[5] == 1.0
    # the largest element of each row decodes back to +-amax (448 * scale)
    dec = np.array([[orc.e4m3_to_f64(int(c)) for c in r] for r in nope[:20]]) * scale[:20, None]
    assert np.allclose(np.abs(dec).max(1), amax[:20], rtol=1e-6)


def test_quant_mxfp4_scale_rule_and_roundtrip(orc):
    # Each block: exactly representable values {0,.5,...,6} * 2^e with the max element 6*2^e
    # or 4*2^e round-trip exactly; the stored exponent is floor(log2 amax) - 2.
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6.0])
    rows = []
    exps = []
    for r in range(64):
        e = int(RNG.integers(-20, 20))
        vals = RNG.choice(grid, 64) * RNG.choice([-1, 1], 64)
        top = 6.0 if r % 2 else 4.0
        vals[0], vals[32] = top, -top
        rows.append(vals * 2.0 ** e)
        exps.append(e)
    x = bf16(np.array(rows))
    packed, sf = orc.quant_mxfp4(x)
    for r in range(64):
        assert list(sf[r]) == [exps[r] + 127] * 2      # floor(log2(4 or 6 * 2^e)) - 2 = e
    dec = np.zeros((64, 64))
    for r in range(64):
        for c in range(64):
            nib = (packed[r, c // 2] >> (4 * (c % 2))) & 15
            dec[r, c] = orc.e2m1_to_f64(int(nib)) * orc.e8m0_to_f64(int(sf[r, c // 32]))
    assert np.array_equal(dec, x.double().numpy())


def test_quant_mxfp4_packing_and_zero_block(orc):
    x = np.zeros((1, 64), np.float32)
    x[0, 0], x[0, 1] = 0.5 * 2 ** -2 * 4, 1.0     # amax 1 -> e = -2, X = 1/4 -> codes 2 (0.5/.25=2), 4
    x[0, 1] = 1.0
    packed, sf = orc.quant_mxfp4(bf16(x))
    assert sf[0, 0] == 125 and sf[0, 1] == 127        # zero block stores 2^0
    assert packed[0, 0] == (4 | (6 << 4))              # 0.5/0.25 = 2 -> code 4; 1/.25 = 4 -> code 6
    assert np.all(packed[0, 16:] == 0)


def test_quant_mxfp4_is_nearest_per_block(orc):
    x = rand_bf16(40, 64, std=2.0)
    packed, sf = orc.quant_mxfp4(x)
    xv = x.double().numpy()
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6.0])
    for r in range(40):
        for blk in range(2):
            amax = np.abs(xv[r, blk * 32:(blk + 1) * 32]).max()
            X = 2.0 ** (math.floor(math.log2(amax)) - 2)
            assert orc.e8m0_to_f64(int(sf[r, blk])) == X
            for c in range(blk * 32, blk * 32 + 32):
                nib = (packed[r, c // 2] >> (4 * (c % 2))) & 15
                v = orc.e2m1_to_f64(int(nib))
                err = abs(abs(v) - min(abs(xv[r, c]) / X, 6.0))
                assert err <= np.min(np.abs(grid - min(abs(xv[r, c]) / X, 6.0))) + 1e-12
                assert v == 0 or np.sign(v) == np.sign(xv[r, c])


# =========================================================================================
# a1/a2: compressor

def test_entry_counts_match_pages(orc):
    pc = json.load(open(os.path.join(GOLD, "page_constants.json")))
    m, mh = pc["csa_ratio_m"]["value"], pc["hca_ratio_m_prime"]["value"]
    c = pc["csa_entries_1M"]
    assert orc.num_entries(c["tokens"], m) == c["entries"]
    h = pc["hca_entries_1M"]
    assert abs(orc.num_entries(h["tokens"], mh) - h["entries"]) <= h["rel_tol"] * h["entries"]
    # and with the workload's 2^20 tokens
    assert orc.num_entries(1 << 20, 4) == 262144 and orc.num_entries(1 << 20, 128) == 8192


@pytest.mark.parametrize("m,overlap,L", [(4, True, 37), (4, True, 64), (128, False, 300), (1, False, 9)])
def test_compress_constant_tokens_pool_to_themselves(orc, m, overlap, L):
    d = 16
    const = RNG.standard_normal(d).astype(np.float32)
    x = bf16(np.broadcast_to(const, (2, L, d)))
    g = rand_bf16(2, L, d, std=3.0)
    bias = torch.from_numpy(RNG.standard_normal(2 * m if overlap else m).astype(np.float32))
    out = orc.compress(x, g, bias, m, overlap)
    assert out.shape == (2, -(-L // m), d)
    assert np.allclose(out, f64(x[0, 0])[None, None, :], rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("m,overlap,L", [(4, True, 23), (128, False, 300), (2, False, 7)])
def test_compress_zero_gate_is_mean_of_present_slots(orc, m, overlap, L):
    d = 8
    x = rand_bf16(1, L, d)
    g = bf16(np.zeros((1, L, d)))
    bias = torch.zeros(2 * m if overlap else m)
    out = orc.compress(x, g, bias, m, overlap)
    xv = f64(x[0])
    for i in range(-(-L // m)):
        # CSA entry i: previous window's last m tokens (C^b) and the current m tokens (C^a)
        lo = m * (i - 1) if overlap else m * i
        toks = [t for t in range(lo, m * i + m) if 0 <= t < L]
        assert np.allclose(out[0, i], xv[toks].mean(0), rtol=1e-12, atol=1e-12)


def test_compress_bias_selects_slot(orc):
    # A dominant bias on slot j makes entry i equal to token t_j = m(i-1) + j: pins the
    # slot order (C^b first, then C^a) and the direction of the softmax.
    m, L, d = 4, 40, 8
    x = rand_bf16(1, L, d)
    g = bf16(np.zeros((1, L, d)))
    xv = f64(x[0])
    for j in range(2 * m):
        b = np.full(2 * m, -60.0, np.float32)
        b[j] = 60.0
        out = orc.compress(x, g, torch.from_numpy(b), m, True)
        for i in range(1, L // m):
            assert np.allclose(out[0, i], xv[m * (i - 1) + j], rtol=0, atol=1e-12)


def test_compress_gate_is_per_channel(orc):
    # A dominant gate logit on (token t, channel c) makes channel c of every entry pooling t
    # equal to x[t, c] while the other channels stay pooled.
    m, L, d = 4, 16, 4
    x = rand_bf16(1, L, d)
    gz = np.zeros((1, L, d), np.float32)
    gz[0, 9, 2] = 80.0
    out = orc.compress(x, bf16(gz), torch.zeros(8), m, True)
    xv = f64(x[0])
    for i in (2, 3):       # token 9 is in C^a of entry 2 and C^b of entry 3
        assert abs(out[0, i, 2] - xv[9, 2]) < 1e-12
        assert abs(out[0, i, 1] - xv[m * (i - 1):m * i + m, 1].mean()) < 1e-12


def test_compress_matches_grouping_example(orc):
    # The pages' 8-token example: C1 from t1..t4, C2 from t5..t8.  Biasing the pool onto the
    # current group (C^a) reproduces exactly those groups.
    pc = json.load(open(os.path.join(GOLD, "page_constants.json")))["grouping_example"]
    m = pc["m"]
    x = rand_bf16(1, 8, 4)
    b = np.array([-80.0] * m + [0.0] * m, np.float32)
    out = orc.compress(x, bf16(np.zeros((1, 8, 4))), torch.from_numpy(b), m, True)
    xv = f64(x[0])
    for i, grp in enumerate(pc["current_groups_1based"]):
        assert np.allclose(out[0, i], xv[[t - 1 for t in grp]].mean(0), atol=1e-12)


def test_compress_softmax_weights_against_scipy(orc):
    from scipy.special import softmax
    m, L, d = 4, 12, 3
    x = rand_bf16(1, L, d)
    g = rand_bf16(1, L, d, std=2.0)
    bias = torch.from_numpy(RNG.standard_normal(8).astype(np.float32))
    out = orc.compress(x, g, bias, m, True)
    xv, gv, bv = f64(x[0]), f64(g[0]), bias.double().numpy()
    i, ch = 2, 1
    toks = list(range(4, 12))
    wts = softmax(np.array([gv[t, ch] for t in toks]) + bv)
    assert abs(out[0, i, ch] - float(wts @ xv[toks, ch])) < 1e-12


def test_compress_span_one_is_identity(orc):
    x = rand_bf16(2, 11, 16)
    out = orc.compress(x, rand_bf16(2, 11, 16), torch.zeros(1), 1, False)
    assert np.array_equal(out, f64(x))


def test_compress_entry_range(orc):
    x, g = rand_bf16(1, 50, 8), rand_bf16(1, 50, 8)
    bias = torch.from_numpy(RNG.standard_normal(8).astype(np.float32))
    full = orc.compress(x, g, bias, 4, True)
    part = orc.compress(x, g, bias, 4, True, 5, 9)
    assert np.array_equal(part[0], full[0, 5:9])


# =========================================================================================
# visibility, a4: indexer

def test_visibility_is_entry_completion(orc):
    # entry i (last token m*i + m - 1) is visible at position p iff that token is <= p
    for m in (1, 4, 128):
        for p in range(0, 700, 7):
            want = sum(1 for i in range(1000) if m * i + m - 1 <= p)
            assert orc.num_visible(p, m, 1000) == want
    assert orc.num_visible(-1, 4, 10) == 0 and orc.num_visible(10 ** 6, 4, 10) == 10


def test_index_single_head_is_relu_matmul(orc):
    Nc, dI = 97, 64
    q = rand_bf16(1, 1, 1, dI)
    k = rand_bf16(1, Nc, dI)
    w = torch.ones(1, 1, 1)
    pos = torch.tensor([[10 ** 6]], dtype=torch.int32)
    s = orc.index_scores(oracle.FMT_BF16, q, w, k, pos, 4)
    ref = torch.relu(k[0].double() @ q[0, 0, 0].double()).numpy()
    assert np.allclose(s[0, 0], ref, rtol=1e-14, atol=1e-14)


def test_index_head_weights_and_linearity(orc):
    B, Tq, HI, dI, Nc = 2, 3, 4, 64, 50
    q = rand_bf16(B, Tq, HI, dI)
    k = rand_bf16(B, Nc, dI)
    pos = torch.full((B, Tq), 10 ** 6, dtype=torch.int32)
    w1 = torch.from_numpy(RNG.random((B, Tq, HI)).astype(np.float32))
    w2 = torch.from_numpy(RNG.random((B, Tq, HI)).astype(np.float32))
    s1 = orc.index_scores(0, q, w1, k, pos, 4)
    s2 = orc.index_scores(0, q, w2, k, pos, 4)
    s12 = orc.index_scores(0, q, w1.double().add(w2.double()).float(), k, pos, 4)
    w12 = (w1.double() + w2.double()).float().double()
    assert np.allclose(s12, s1 + s2, rtol=1e-5)     # w1+w2 rounded to fp32 -> small slack
    # one-hot weights select one head: s = relu(q_h . k)
    for h in range(HI):
        w = torch.zeros(B, Tq, HI)
        w[..., h] = 1
        s = orc.index_scores(0, q, w, k, pos, 4)
        ref = torch.relu(torch.einsum("btc,bnc->btn", q[:, :, h].double(), k.double())).numpy()
        assert np.allclose(s, ref, rtol=1e-14, atol=1e-13)
    del w12


def test_index_masks_invisible_entries(orc):
    Nc = 40
    q, k = rand_bf16(1, 3, 2, 64), rand_bf16(1, Nc, 64)
    w = torch.ones(1, 3, 2)
    pos = torch.tensor([[0, 18, 19]], dtype=torch.int32)
    s = orc.index_scores(0, q, w, k, pos, 4)
    assert np.all(np.isneginf(s[0, 0]))                  # p=0: no complete entry
    assert np.all(np.isfinite(s[0, 1, :4])) and np.all(np.isneginf(s[0, 1, 4:]))   # 4*4+3 > 18
    assert np.all(np.isfinite(s[0, 2, :5])) and np.all(np.isneginf(s[0, 2, 5:]))   # 4*4+3 = 19


def test_index_mxfp4_is_exact(orc):
    # MXFP4 operands: products of E2M1 * 2^e values are exact, so the fp64 oracle must equal
    # an exact matmul of the independently decoded operands.
    B, Tq, HI, dI, Nc = 1, 2, 3, 64, 33
    qb, kb = rand_bf16(B, Tq, HI, dI), rand_bf16(B, Nc, dI)
    qp, qs = orc.quant_mxfp4(qb)
    kp, ks = orc.quant_mxfp4(kb)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6.0])

    def decode(p, s):
        lo, hi = p & 15, p >> 4
        nib = np.stack([lo, hi], -1).reshape(p.shape[:-1] + (p.shape[-1] * 2,))
        val = grid[nib & 7] * np.where(nib & 8, -1.0, 1.0)
        return val * np.repeat(2.0 ** (s.astype(np.float64) - 127), 32, axis=-1)

    qd, kd = decode(qp, qs), decode(kp, ks)
    w = torch.from_numpy(RNG.random((B, Tq, HI)).astype(np.float32))
    pos = torch.full((B, Tq), 10 ** 6, dtype=torch.int32)
    s = orc.index_scores(oracle.FMT_MXFP4, qp, w, kp, pos, 4, qI_sf=qs, kI_sf=ks)
    dots = np.einsum("bthc,bnc->bthn", qd, kd)
    ref = np.einsum("bth,bthn->btn", w.double().numpy(), np.maximum(dots, 0))
    assert np.allclose(s, ref, rtol=1e-15, atol=0)


# =========================================================================================
# a5: top-k

def _brute_topk(s, nvis, k):
    order = np.lexsort((np.arange(nvis), -s[:nvis]))   # score desc, then index asc
    sel = np.sort(order[:k])
    return np.concatenate([sel, -np.ones(k - len(sel), int)])


def test_topk_against_sort(orc):
    B, Tq, Nc, k = 3, 4, 300, 37
    s = RNG.standard_normal((B, Tq, Nc))
    s[0, 0, :50] = 0.5                                   # ties
    s = np.round(s, 1)                                   # many more ties
    pos = torch.tensor(RNG.integers(0, 4 * Nc + 10, (B, Tq)), dtype=torch.int32)
    idx = orc.topk(s, pos, 4, k)
    for b in range(B):
        for t in range(Tq):
            nvis = min(Nc, (int(pos[b, t]) + 1) // 4)
            assert np.array_equal(idx[b, t], _brute_topk(s[b, t], nvis, k))


def test_topk_selection_property(orc):
    s = np.round(RNG.standard_normal((1, 1, 500)), 2)
    idx = orc.topk(s, torch.tensor([[10 ** 6]], dtype=torch.int32), 4, 64)[0, 0]
    sel = set(idx.tolist())
    worst_in = min(s[0, 0, list(sel)])
    for i in range(500):
        if i not in sel:
            assert s[0, 0, i] < worst_in or (s[0, 0, i] == worst_in and i > max(
                j for j in sel if s[0, 0, j] == worst_in))
    assert list(idx) == sorted(idx)


def test_topk_fewer_visible_than_k(orc):
    s = RNG.standard_normal((1, 2, 100))
    idx = orc.topk(s, torch.tensor([[39, 2]], dtype=torch.int32), 4, 16)
    assert list(idx[0, 0]) == list(range(10)) + [-1] * 6
    assert list(idx[0, 1]) == [-1] * 16


def test_topk_all_equal_takes_lowest(orc):
    s = np.zeros((1, 1, 64))
    idx = orc.topk(s, torch.tensor([[1000]], dtype=torch.int32), 4, 10)
    assert list(idx[0, 0]) == list(range(10))


def test_topk_planted_generator(orc):
    cfg = scaled(CSA_TINY, planted=0.05, HI=8, k=32, seed=77)
    qI, kI, w = gen.index_queries(cfg, [0]), gen.index_keys(cfg, [0]), gen.head_weights(cfg, [0])
    pos = gen.query_positions(cfg, 1)
    s = orc.index_scores(0, qI, w, kI, pos, cfg.m)
    idx = orc.topk(s, pos, cfg.m, cfg.k)
    assert set(idx[0, 0].tolist()) <= set(gen.planted_set(cfg, 0).tolist())


# =========================================================================================
# a6/a7: attention

def _kv(t, cap=None):
    return oracle.KV(oracle.FMT_BF16, t, t.shape[1] if cap is None else cap)


def test_attn_m1_full_selection_is_causal_sdpa(orc):
    # m = 1 with one-token pools, k >= L and no window: standard causal attention
    B, L, H, d = 2, 24, 3, 32
    x = rand_bf16(B, L, d)
    ent = orc.compress(x, rand_bf16(B, L, d), torch.zeros(1), 1, False)
    assert np.array_equal(ent, f64(x))
    q = rand_bf16(B, L, H, d)
    pos = torch.arange(L, dtype=torch.int32).repeat(B, 1)
    s = orc.index_scores(0, rand_bf16(B, L, 1, 64), torch.ones(B, L, 1), rand_bf16(B, L, 64), pos, 1)
    idx = orc.topk(s, pos, 1, L)
    o, lse = orc.csa_attn(q, _kv(x), idx, _kv(x), 0, pos)
    qd = q.double().permute(0, 2, 1, 3)                         # [B,H,L,d]
    kv = x.double().unsqueeze(1).expand(B, H, L, d)
    ref = torch.nn.functional.scaled_dot_product_attention(qd, kv, kv, is_causal=True)
    assert np.allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-12, atol=1e-12)
    logits = (qd @ kv.transpose(-1, -2)) / math.sqrt(d)
    logits = logits.masked_fill(torch.ones(L, L, dtype=torch.bool).triu(1), -float("inf"))
    assert np.allclose(lse, torch.logsumexp(logits, -1).permute(0, 2, 1).numpy(), atol=1e-12)


def test_attn_window_only_is_banded_sdpa(orc):
    B, L, H, d, W = 1, 30, 2, 16, 5
    x = rand_bf16(B, L, d)
    q = rand_bf16(B, L, H, d)
    pos = torch.arange(L, dtype=torch.int32).unsqueeze(0)
    idx = -torch.ones(B, L, 4, dtype=torch.int32)
    o, _ = orc.csa_attn(q, _kv(rand_bf16(B, 8, d)), idx, _kv(x), W, pos)
    i = torch.arange(L)
    mask = (i[None, :] <= i[:, None]) & (i[None, :] > i[:, None] - W)
    qd = q.double().permute(0, 2, 1, 3)
    kv = x.double().unsqueeze(1).expand(B, H, L, d)
    ref = torch.nn.functional.scaled_dot_product_attention(qd, kv, kv, attn_mask=mask)
    assert np.allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-12, atol=1e-12)


def test_attn_full_selection_equals_dense_hca_math(orc):
    # k >= number of entries: CSA equals dense attention over the compressed KV (ratio 4)
    B, L, H, d, W = 2, 64, 4, 32, 7
    ent = rand_bf16(B, 16, d)
    raw = rand_bf16(B, L, d)
    q = rand_bf16(B, 3, H, d)
    pos = torch.tensor([[63, 40, 9], [17, 3, 60]], dtype=torch.int32)
    s = RNG.standard_normal((B, 3, 16))
    idx = orc.topk(s, pos, 4, 16)
    oc, lc = orc.csa_attn(q, _kv(ent), idx, _kv(raw), W, pos)
    oh, lh = orc.hca_attn(q, _kv(ent), 16, 4, _kv(raw), W, pos)
    assert np.allclose(oc, oh, rtol=1e-13, atol=1e-13) and np.allclose(lc, lh, atol=1e-13)


def test_attn_single_item(orc):
    d = 64
    x = rand_bf16(1, 9, d)
    q = rand_bf16(1, 1, 2, d)
    idx = torch.tensor([[[3, -1, -1]]], dtype=torch.int32)
    o, lse = orc.csa_attn(q, _kv(x), idx, _kv(x), 0, torch.tensor([[100]], dtype=torch.int32))
    assert np.array_equal(o[0, 0, 0], f64(x[0, 3])) and np.array_equal(o[0, 0, 1], f64(x[0, 3]))
    assert np.allclose(lse[0, 0], (q[0, 0].double() @ x[0, 3].double()).numpy() / 8.0, atol=1e-13)


def test_attn_two_pass_matches_scipy_softmax(orc):
    from scipy.special import softmax
    d = 16
    ent, raw = rand_bf16(1, 12, d, std=4.0), rand_bf16(1, 20, d, std=4.0)
    q = rand_bf16(1, 1, 1, d, std=4.0)
    idx = torch.tensor([[[0, 5, 7, 11]]], dtype=torch.int32)
    o, lse = orc.csa_attn(q, _kv(ent), idx, _kv(raw), 3, torch.tensor([[19]], dtype=torch.int32))
    rows = np.concatenate([f64(ent[0, [0, 5, 7, 11]]), f64(raw[0, 17:20])])
    z = rows @ f64(q[0, 0, 0]) / 4.0
    assert np.allclose(o[0, 0, 0], softmax(z) @ rows, rtol=1e-12, atol=1e-12)
    from scipy.special import logsumexp
    assert abs(lse[0, 0, 0] - logsumexp(z)) < 1e-12


def test_attn_window_and_entries_are_not_deduplicated(orc):
    # A window row identical to a selected entry counts twice in the softmax.
    d = 8
    raw = rand_bf16(1, 10, d)
    ent = raw[:, 9:10].clone()                                 # entry 0 == raw token 9
    q = rand_bf16(1, 1, 1, d)
    o, _ = orc.csa_attn(q, _kv(ent), torch.tensor([[[0]]], dtype=torch.int32), _kv(raw), 2,
                        torch.tensor([[9]], dtype=torch.int32))
    rows = np.stack([f64(raw[0, 9]), f64(raw[0, 8]), f64(raw[0, 9])])
    z = rows @ f64(q[0, 0, 0]) / math.sqrt(d)
    p = np.exp(z - z.max()) / np.exp(z - z.max()).sum()
    assert np.allclose(o[0, 0, 0], p @ rows, atol=1e-13)


def test_attn_sink_takes_mass(orc):
    B, L, H, d, W = 1, 40, 4, 16, 6
    ent, raw = rand_bf16(B, 10, d), rand_bf16(B, L, d)
    q = rand_bf16(B, 2, H, d)
    pos = torch.tensor([[39, 20]], dtype=torch.int32)
    idx = torch.tensor([[[1, 4, 6, -1], [0, 2, 3, 4]]], dtype=torch.int32)
    sink = torch.from_numpy(RNG.standard_normal(H).astype(np.float32))
    o0, l0 = orc.csa_attn(q, _kv(ent), idx, _kv(raw), W, pos)
    o1, l1 = orc.csa_attn(q, _kv(ent), idx, _kv(raw), W, pos, sink=sink)
    sd = sink.double().numpy()
    assert np.allclose(l1, np.logaddexp(l0, sd[None, None, :]), atol=1e-13)
    assert np.allclose(o1, o0 * np.exp(l0 - l1)[..., None], atol=1e-13)
    o2, l2 = orc.csa_attn(q, _kv(ent), idx, _kv(raw), W, pos, sink=torch.full((H,), -1e30))
    assert np.allclose(o2, o0, atol=1e-14)


def test_attn_ring_buffer_equals_linear(orc):
    B, L, H, d, W = 2, 50, 2, 16, 8
    raw = rand_bf16(B, L, d)
    ring = torch.zeros(B, W, d, dtype=torch.bfloat16)
    for t in range(L - W, L):
        ring[:, t % W] = raw[:, t]
    ent = rand_bf16(B, 12, d)
    q = rand_bf16(B, 1, H, d)
    pos = torch.full((B, 1), L - 1, dtype=torch.int32)
    idx = torch.tensor([[[1, 5, 9]], [[0, 2, 11]]], dtype=torch.int32)
    a = orc.csa_attn(q, _kv(ent), idx, _kv(raw), W, pos)
    b = orc.csa_attn(q, _kv(ent), idx, _kv(ring, W), W, pos)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_attn_fp8split_rows_decode(orc):
    # split rows decode as E4M3 * scale for the first half and bf16 for the RoPE half
    B, N, d = 1, 6, 128
    ent = rand_bf16(B, N, d)
    nope, scale, rope = orc.quant_kv_fp8(ent)
    kv = oracle.KV(oracle.FMT_FP8SPLIT, nope, N, scale=scale, rope=rope)
    q = rand_bf16(B, 1, 1, d)
    for j in range(N):
        o, _ = orc.csa_attn(q, kv, torch.tensor([[[j]]], dtype=torch.int32), _kv(ent), 0,
                            torch.tensor([[10 ** 6]], dtype=torch.int32))
        t = torch.from_numpy(nope[0, j].copy()).view(torch.float8_e4m3fn).double().numpy()
        want = np.concatenate([t * float(scale[0, j]), f64(ent[0, j, 64:])])
        assert np.array_equal(o[0, 0, 0], want)
    # and the quantised row stays within E4M3's half-ulp (2^-4 relative) of the bf16 row
    assert np.allclose(want[:64], f64(ent[0, N - 1, :64]), rtol=2 ** -4, atol=float(scale[0, -1]) * 2 ** -9)


def test_hca_visibility_and_empty(orc):
    d = 8
    ent, raw = rand_bf16(1, 4, d), rand_bf16(1, 600, d)
    q = rand_bf16(1, 3, 1, d)
    pos = torch.tensor([[126, 127, 300]], dtype=torch.int32)
    o, lse = orc.hca_attn(q, _kv(ent), 4, 128, _kv(raw), 0, pos)
    assert np.all(o[0, 0] == 0) and np.isneginf(lse[0, 0, 0])       # nothing visible, W = 0
    assert np.array_equal(o[0, 1, 0], f64(ent[0, 0]))                 # entry 0 complete at 127
    z = f64(ent[0, :2]) @ f64(q[0, 2, 0]) / math.sqrt(d)
    p = np.exp(z - z.max()) / np.exp(z - z.max()).sum()
    assert np.allclose(o[0, 2, 0], p @ f64(ent[0, :2]), atol=1e-13)  # entries 0, 1 at p=300


# -----------------------------------------------------------------------------------------
# RMSNorm of queries and entries [Tripbot §5]: hand values, identities, and torch's own
# RMSNorm as an independent implementation.

def test_rmsnorm_hand_values(orc):
    # x = (3, 4): mean of squares 12.5
    out = orc.rmsnorm(np.array([[3.0, 4.0]]), eps=0.0)
    assert np.allclose(out, np.array([[3.0, 4.0]]) / math.sqrt(12.5), rtol=0, atol=1e-15)
    # a constant row of 1e-3 with eps = 1e-6: mean square equals eps -> 1e-3 / sqrt(2e-6)
    out = orc.rmsnorm(np.full((1, 128), 1e-3), eps=1e-6)
    assert np.allclose(out, 1.0 / math.sqrt(2.0), rtol=1e-14, atol=0)
    # a zero row stays zero (eps keeps the denominator finite)
    assert np.array_equal(orc.rmsnorm(np.zeros((2, 64))), np.zeros((2, 64)))


def test_rmsnorm_identities(orc):
    rng = np.random.default_rng(11)
    x = rng.standard_normal((5, 128))
    y = orc.rmsnorm(x, eps=0.0)
    # unit root-mean-square per row, direction kept, invariant to a positive scale
    assert np.allclose(np.sqrt((y * y).mean(-1)), 1.0, rtol=1e-14)
    assert np.allclose(y / np.linalg.norm(y, axis=-1, keepdims=True),
                       x / np.linalg.norm(x, axis=-1, keepdims=True), rtol=1e-13)
    assert np.allclose(orc.rmsnorm(7.5 * x, eps=0.0), y, rtol=1e-13)
    # gamma multiplies per channel
    gamma = rng.random(128).astype(np.float32) + 0.5
    assert np.allclose(orc.rmsnorm(x, gamma, eps=0.0), y * gamma.astype(np.float64), rtol=1e-14)
    # rows are independent
    assert np.allclose(orc.rmsnorm(x[2:3], eps=0.0), y[2:3], rtol=0, atol=0)


def test_rmsnorm_against_torch(orc):
    rng = np.random.default_rng(12)
    x = rng.standard_normal((3, 4, 128)) * 3.0
    gamma = (rng.random(128) + 0.25).astype(np.float32)
    want = torch.nn.functional.rms_norm(torch.from_numpy(x), (128,),
                                        torch.from_numpy(gamma.astype(np.float64)), eps=1e-6)
    got = orc.rmsnorm(x, gamma, eps=1e-6)
    assert np.allclose(got, want.numpy(), rtol=1e-13, atol=1e-15)
    # bf16 input (as the queries and entries are stored) is read exactly
    xb = gen.to_bf16(x.astype(np.float32))
    assert np.allclose(orc.rmsnorm(xb, gamma), orc.rmsnorm(xb.double().numpy(), gamma), rtol=0, atol=0)
