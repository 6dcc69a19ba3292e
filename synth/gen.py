"""Seeded synthetic inputs for the hybrid-attention workloads.

Every tensor is drawn from numpy's Philox generator keyed by (workload seed, tensor id,
sequence, row block), so any sequence or row range can be regenerated on its own
(full-size parity tests only rebuild the rows they check).  Values are drawn in fp32 and
stored in the formats the path consumes (bf16 bits, fp32, int32).  This module holds none
of the method's arithmetic: no pooling, scoring, selection, attention or quantisation.
Both the CPU oracle and the CUDA library receive exactly these tensors.
"""
import numpy as np
import torch

from .configs import Workload

# tensor ids (part of the Philox key)
T_KV_RAW, T_GATE, T_BIAS, T_Q, T_QI, T_W, T_KI, T_KVC, T_KVH, T_PLANT, T_SINK = range(1, 12)

ROW_BLOCK = 4096  # rows per independently keyed block


def _rng(seed: int, tid: int, b: int, block: int) -> np.random.Generator:
    ss = np.random.SeedSequence([seed & 0xFFFFFFFF, tid, b, block])
    key = ss.generate_state(2, np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def rows_normal(seed, tid, b, r0, r1, width, std=1.0):
    """fp32 N(0, std^2) rows [r0, r1) of a (sequence b, tensor tid) stream, shape [r1-r0, width]."""
    out = np.empty((max(r1 - r0, 0), width), np.float32)
    blk0, blk1 = r0 // ROW_BLOCK, (r1 - 1) // ROW_BLOCK if r1 > r0 else -1
    for blk in range(blk0, blk1 + 1):
        base = blk * ROW_BLOCK
        vals = _rng(seed, tid, b, blk).standard_normal((ROW_BLOCK, width), dtype=np.float32)
        lo, hi = max(r0, base), min(r1, base + ROW_BLOCK)
        out[lo - r0:hi - r0] = vals[lo - base:hi - base]
    if std != 1.0:
        out *= np.float32(std)
    return out


def rows_uniform(seed, tid, b, n, width):
    return _rng(seed, tid, b, 0).random((n, width), dtype=np.float32)


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """fp32 numpy -> bf16 torch (round to nearest even; storage conversion only)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 torch tensor -> its raw uint16 bits as numpy (no copy of values' meaning)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------------------------------
# per-tensor generators

def raw_kv(cfg: Workload, bs, r0: int, r1: int) -> torch.Tensor:
    """Raw (already rotated) KV rows [len(bs), r1-r0, d] bf16 ~ N(0,1)."""
    return to_bf16(np.stack([rows_normal(cfg.seed, T_KV_RAW, b, r0, r1, cfg.d) for b in bs]))


def gate(cfg: Workload, bs, r0: int, r1: int) -> torch.Tensor:
    """Per-token, per-channel gate logits [len(bs), r1-r0, d] bf16 ~ N(0,1)."""
    return to_bf16(np.stack([rows_normal(cfg.seed, T_GATE, b, r0, r1, cfg.d) for b in bs]))


def bias(cfg: Workload, span: int, which: int = 0) -> torch.Tensor:
    """Learned position bias, one fp32 scalar per pooled slot, ~ N(0, bias_std^2)."""
    return torch.from_numpy(rows_normal(cfg.seed, T_BIAS, which, 0, 1, span, cfg.bias_std)[0].copy())


def queries(cfg: Workload, bs) -> torch.Tensor:
    """Attention queries [len(bs), Tq, H, d] bf16 ~ N(0,1)."""
    return to_bf16(np.stack([rows_normal(cfg.seed, T_Q, b, 0, cfg.Tq * cfg.H, cfg.d)
                             .reshape(cfg.Tq, cfg.H, cfg.d) for b in bs]))


def comp_kv(cfg: Workload, bs, n: int, tid: int = T_KVC) -> torch.Tensor:
    """A directly generated compressed-KV cache [len(bs), n, d] bf16 ~ N(0,1) (decode configs)."""
    return to_bf16(np.stack([rows_normal(cfg.seed, tid, b, 0, n, cfg.d) for b in bs]))


def head_weights(cfg: Workload, bs) -> torch.Tensor:
    """Indexer head weights w [len(bs), Tq, HI] fp32 ~ U(0,1)."""
    return torch.from_numpy(np.stack([rows_uniform(cfg.seed, T_W, b, cfg.Tq, cfg.HI) for b in bs]))


def _plant(cfg: Workload, b: int):
    """Planted direction u (unit, dI) and the planted entry set of sequence b."""
    rng = _rng(cfg.seed, T_PLANT, b, 0)
    u = rng.standard_normal(cfg.dI).astype(np.float64)
    u /= np.linalg.norm(u)
    n_plant = int(cfg.planted * cfg.Nc)
    S = np.sort(rng.choice(cfg.Nc, size=n_plant, replace=False))
    return u, S


PLANT_KEY_GAIN = 6.0    # planted keys:   k_i + 6 u
PLANT_Q_GAIN = 2.0      # index queries:  2 u + 0.1 eps_h
PLANT_Q_NOISE = 0.1


def index_keys(cfg: Workload, bs) -> torch.Tensor:
    """Lightning-indexer keys K_I [len(bs), Nc, dI] bf16 ~ N(0,1), planted if cfg.planted."""
    out = []
    for b in bs:
        k = rows_normal(cfg.seed, T_KI, b, 0, cfg.Nc, cfg.dI)
        if cfg.planted > 0:
            u, S = _plant(cfg, b)
            k[S] += (PLANT_KEY_GAIN * u).astype(np.float32)
        out.append(k)
    return to_bf16(np.stack(out))


def index_queries(cfg: Workload, bs) -> torch.Tensor:
    """Lightning-indexer queries q_I [len(bs), Tq, HI, dI] bf16."""
    out = []
    for b in bs:
        q = rows_normal(cfg.seed, T_QI, b, 0, cfg.Tq * cfg.HI, cfg.dI).reshape(cfg.Tq, cfg.HI, cfg.dI)
        if cfg.planted > 0:
            u, _ = _plant(cfg, b)
            q = (PLANT_Q_GAIN * u + PLANT_Q_NOISE * q).astype(np.float32)
        out.append(q)
    return to_bf16(np.stack(out))


def planted_set(cfg: Workload, b: int) -> np.ndarray:
    return _plant(cfg, b)[1]


def query_positions(cfg: Workload, nb: int) -> torch.Tensor:
    """Absolute query positions [nb, Tq] int32: a contiguous chunk ending at L-1."""
    p = torch.arange(cfg.first_pos, cfg.first_pos + cfg.Tq, dtype=torch.int32)
    return p.unsqueeze(0).repeat(nb, 1).contiguous()


def sink_logits(cfg: Workload) -> torch.Tensor:
    """Optional per-head attention-sink logits [H] fp32 ~ N(0,1)."""
    return torch.from_numpy(rows_normal(cfg.seed, T_SINK, 0, 0, 1, cfg.H)[0].copy())
