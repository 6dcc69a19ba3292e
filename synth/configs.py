"""The five synthetic workloads of the CSA/HCA hybrid-attention hot path.

Shapes, ratios and selection sizes follow the DeepSeek-V4 write-ups:
  * CSA ratio m=4 with an overlapped 2m pooling window, top-k 1024 (Pro) / 512 (Flash)
    ("论文解读｜DeepSeek-V4：百万 token 上下文的效率革命", blog.tripbot.top, §3.1;
    gitcode.csdn.net "CSA / HCA 混合注意力" article, §1.1 and its "工程细节" paragraph);
  * HCA ratio m'=128, dense attention over all compressed entries (same pages, §3.2 / §1.2);
  * a 128-token raw sliding-window branch on both (blog.tripbot.top §3.3);
  * MXFP4 indexer operands, BF16 index scores, FP8 non-RoPE / BF16 RoPE KV storage
    (gitcode.csdn.net §1.4).
This module only describes workloads; it holds none of the method's arithmetic.
"""
from dataclasses import dataclass, field, replace


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "csa_decode" | "hca" | "pair_prefill"
    B: int               # sequences
    L: int               # raw tokens in the context (query positions are < L)
    H: int               # query heads sharing the one KV head
    d: int = 128         # head dim; dims 64..127 are the (pre-rotated) RoPE dims
    m: int = 4           # CSA compression ratio (overlapped window of 2m tokens)
    mh: int = 128        # HCA compression ratio (non-overlapped)
    HI: int = 0          # lightning-indexer heads
    dI: int = 64         # lightning-indexer head dim
    k: int = 0           # top-k
    W: int = 128         # raw sliding window
    Tq: int = 1          # queries per sequence
    q_pos0: int = -1     # position of the first query (-1: L - Tq)
    idx_fmt: str = "bf16"    # indexer operand format: "bf16" | "mxfp4"
    score_fmt: str = "fp32"  # index score format: "fp32" | "bf16"
    kv_fmt: str = "bf16"     # compressed/raw KV storage: "bf16" | "fp8split"
    planted: float = 0.0     # fraction of entries planted to score high (cfg 3)
    bias_std: float = 0.1    # position-bias std
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def first_pos(self) -> int:
        return self.L - self.Tq if self.q_pos0 < 0 else self.q_pos0

    @property
    def Nc(self) -> int:       # CSA entries: ceil(L / m)
        return -(-self.L // self.m)

    @property
    def Nh(self) -> int:       # HCA entries: ceil(L / m')
        return -(-self.L // self.mh)


# Config 1: CSA decode, tiny (the parity case; seed 0).
CSA_TINY = Workload(name="csa_decode_tiny_L4096", kind="csa_decode", B=1, L=4096, H=8,
                    HI=4, k=64, W=64, Tq=1, idx_fmt="bf16", score_fmt="fp32",
                    kv_fmt="bf16", seed=0)

# Config 2: HCA layer, prefill (2048-query causal chunk at the end) and decode.
HCA_64K = Workload(name="hca_L65536_B4", kind="hca", B=4, L=65536, H=16, W=128,
                   Tq=2048, seed=2000)

# Config 3: CSA decode at 128K, Flash-like, planted 5% high-scoring entries.
CSA_128K = Workload(name="csa_decode_L131072_B32", kind="csa_decode", B=32, L=131072,
                    H=64, HI=8, k=512, W=128, Tq=1, idx_fmt="bf16", score_fmt="fp32",
                    kv_fmt="bf16", planted=0.05, seed=3000)

# Config 4: CSA decode at 1M, Pro-like: MXFP4 indexer, BF16 scores, FP8/BF16 split KV.
CSA_1M = Workload(name="csa_decode_L1048576_B8", kind="csa_decode", B=8, L=1048576,
                  H=128, HI=16, k=1024, W=128, Tq=1, idx_fmt="mxfp4", score_fmt="bf16",
                  kv_fmt="fp8split", seed=4000)

# Config 5: alternating CSA/HCA layer pair, 4096-token chunked prefill on a 262144 context.
PAIR_PREFILL = Workload(name="csa_hca_pair_prefill_ctx262144_new4096", kind="pair_prefill",
                        B=1, L=262144 + 4096, H=64, HI=16, k=1024, W=128, Tq=4096,
                        q_pos0=262144, idx_fmt="bf16", score_fmt="bf16", kv_fmt="bf16",
                        seed=5000)

CONFIGS = [CSA_TINY, HCA_64K, CSA_128K, CSA_1M, PAIR_PREFILL]
BY_NAME = {c.name: c for c in CONFIGS}


def scaled(cfg: Workload, **kw) -> Workload:
    """A smaller copy of a workload (same structure, fewer sequences/tokens)."""
    return replace(cfg, **kw)
