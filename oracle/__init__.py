"""CPU oracle of the CSA/HCA hybrid-attention hot path (fp64, plain C, see hcl_oracle.c).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's CPU-baseline
leg are the only callers.  The CUDA library never imports, links or calls this package,
and this package never imports the CUDA library.

Arguments are numpy arrays (bf16 is passed as its uint16 bits) or CPU torch tensors.
"""
import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# HCL_ORACLE_LIB points the oracle at another build of hcl_oracle.c (the mutation tests
# load deliberately broken copies this way to show that the pins catch them).
_LIB_PATH = os.environ.get("HCL_ORACLE_LIB") or os.path.join(_HERE, "liboracle.so")
_lib = None

FMT_BF16, FMT_FP32, FMT_FP8SPLIT, FMT_MXFP4 = 0, 1, 2, 3


def build(force: bool = False) -> str:
    from .build import build_oracle
    return build_oracle(force=force)


def lib():
    global _lib
    if _lib is None:
        if os.environ.get("HCL_ORACLE_LIB"):
            pass
        elif not os.path.exists(_LIB_PATH) or (
                os.path.getmtime(_LIB_PATH) < os.path.getmtime(os.path.join(_HERE, "hcl_oracle.c"))):
            build()
        _lib = ctypes.CDLL(_LIB_PATH)
        _declare(_lib)
    return _lib


P = ctypes.c_void_p
I = ctypes.c_int
LG = ctypes.c_long
D = ctypes.c_double


def _declare(L):
    L.or_bf16_to_f64.argtypes = [ctypes.c_uint16]; L.or_bf16_to_f64.restype = D
    L.or_f64_to_bf16.argtypes = [D]; L.or_f64_to_bf16.restype = ctypes.c_uint16
    L.or_e4m3_to_f64.argtypes = [ctypes.c_uint8]; L.or_e4m3_to_f64.restype = D
    L.or_f32_to_e4m3.argtypes = [ctypes.c_float]; L.or_f32_to_e4m3.restype = ctypes.c_uint8
    L.or_e2m1_to_f64.argtypes = [ctypes.c_uint8]; L.or_e2m1_to_f64.restype = D
    L.or_f32_to_e2m1.argtypes = [ctypes.c_float]; L.or_f32_to_e2m1.restype = ctypes.c_uint8
    L.or_e8m0_to_f64.argtypes = [ctypes.c_uint8]; L.or_e8m0_to_f64.restype = D
    L.or_num_visible.argtypes = [LG, I, LG]; L.or_num_visible.restype = LG
    L.or_compress.argtypes = [P, P, P, I, LG, I, I, I, LG, LG, P]; L.or_compress.restype = None
    L.or_index_scores.argtypes = [I, P, P, P, P, P, I, I, I, I, LG, P, I, P]
    L.or_index_scores.restype = None
    L.or_round_bf16.argtypes = [P, LG]; L.or_round_bf16.restype = None
    L.or_topk.argtypes = [P, I, I, LG, P, I, I, P]; L.or_topk.restype = None
    kv = [I, P, P, P, LG]
    L.or_csa_attn.argtypes = [P, I, I, I, I] + kv + [P, I] + kv + [I, P, D, P, P, P]
    L.or_csa_attn.restype = None
    L.or_hca_attn.argtypes = [P, I, I, I, I] + kv + [LG, I] + kv + [I, P, D, P, P, P]
    L.or_hca_attn.restype = None
    L.or_quant_kv_fp8.argtypes = [P, LG, I, P, P, P]; L.or_quant_kv_fp8.restype = None
    L.or_quant_mxfp4.argtypes = [P, LG, I, P, P]; L.or_quant_mxfp4.restype = None
    L.or_rmsnorm.argtypes = [P, LG, I, P, D, P]; L.or_rmsnorm.restype = None


# ------------------------------------------------------------------------------------------
# array plumbing

def _np(a, dtype=None):
    """torch/numpy -> C-contiguous numpy; bf16 torch tensors become their uint16 bits."""
    if a is None:
        return None
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype == torch.bfloat16:
                a = a.view(torch.int16).numpy().view(np.uint16)
            elif a.dtype == torch.float8_e4m3fn:
                a = a.view(torch.uint8).numpy()
            else:
                a = a.numpy()
    except ImportError:
        pass
    a = np.ascontiguousarray(a)
    if dtype is not None and a.dtype != dtype:
        a = a.astype(dtype)
    return a


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class KV:
    """A KV store in one of the path's formats.

    fmt FMT_BF16: data = bf16 bits [B, cap, d];
    fmt FMT_FP8SPLIT: data = E4M3 codes [B, cap, d/2], scale = fp32 [B, cap],
                      rope = bf16 bits [B, cap, d/2].
    Row t of sequence b is slot t % cap (cap == L: linear storage; cap < L: a ring)."""

    def __init__(self, fmt, data, cap, scale=None, rope=None):
        self.fmt = fmt
        self.data = _np(data, np.uint16 if fmt == FMT_BF16 else np.uint8)
        self.scale = _np(scale, np.float32)
        self.rope = _np(rope, np.uint16)
        self.cap = int(cap)

    def args(self):
        return [self.fmt, _p(self.data), _p(self.scale), _p(self.rope), self.cap]


# ------------------------------------------------------------------------------------------
# scalar helpers

def bf16_to_f64(h: int) -> float: return lib().or_bf16_to_f64(h)
def f64_to_bf16(x: float) -> int: return lib().or_f64_to_bf16(x)
def e4m3_to_f64(c: int) -> float: return lib().or_e4m3_to_f64(c)
def f32_to_e4m3(x: float) -> int: return lib().or_f32_to_e4m3(x)
def e2m1_to_f64(c: int) -> float: return lib().or_e2m1_to_f64(c)
def f32_to_e2m1(x: float) -> int: return lib().or_f32_to_e2m1(x)
def e8m0_to_f64(c: int) -> float: return lib().or_e8m0_to_f64(c)
def num_visible(p: int, m: int, n: int) -> int: return lib().or_num_visible(p, m, n)


def num_entries(L: int, m: int) -> int:
    """Entries produced from L raw tokens at ratio m: ceil(L / m)."""
    return -(-L // m)


# ------------------------------------------------------------------------------------------
# hot-path steps

def compress(x, g, bias, m, overlap, e0=0, e1=None):
    """Softmax-gated pooling (CSA: overlap=True, span 2m; HCA: overlap=False, span m).
    x, g: bf16 [B, L, d]; bias: fp32 [span]. Returns fp64 [B, e1-e0, d]."""
    x, g = _np(x, np.uint16), _np(g, np.uint16)
    bias = _np(bias, np.float32)
    B, L, d = x.shape
    if e1 is None:
        e1 = num_entries(L, m)
    assert bias.shape[0] == (2 * m if overlap else m)
    out = np.empty((B, e1 - e0, d), np.float64)
    lib().or_compress(_p(x), _p(g), _p(bias), B, L, d, m, int(bool(overlap)), e0, e1, _p(out))
    return out


def index_scores(fmt, qI, w, kI, q_pos, m, qI_sf=None, kI_sf=None, bf16_scores=False):
    """Lightning-indexer scores fp64 [B, Tq, Nc] (-inf for entries not yet visible).
    fmt FMT_BF16: qI bf16 [B,Tq,HI,dI], kI bf16 [B,Nc,dI];
    fmt FMT_MXFP4: qI packed [B,Tq,HI,dI/2] + qI_sf [B,Tq,HI,dI/32], kI packed [B,Nc,dI/2]
    + kI_sf [B,Nc,dI/32].  bf16_scores rounds the result to bf16 (ties to even)."""
    w = _np(w, np.float32)
    q_pos = _np(q_pos, np.int32)
    B, Tq, HI = w.shape
    if fmt == FMT_BF16:
        qI, kI = _np(qI, np.uint16), _np(kI, np.uint16)
        dI = qI.shape[-1]
        Nc = kI.shape[1]
    else:
        qI, kI = _np(qI, np.uint8), _np(kI, np.uint8)
        qI_sf, kI_sf = _np(qI_sf, np.uint8), _np(kI_sf, np.uint8)
        dI = qI.shape[-1] * 2
        Nc = kI.shape[1]
    s = np.empty((B, Tq, Nc), np.float64)
    lib().or_index_scores(fmt, _p(qI), _p(qI_sf), _p(w), _p(kI), _p(kI_sf), B, Tq, HI, dI, Nc,
                          _p(q_pos), m, _p(s))
    if bf16_scores:
        lib().or_round_bf16(_p(s), s.size)
    return s


def round_bf16(s):
    s = np.array(s, dtype=np.float64, copy=True, order="C")
    lib().or_round_bf16(_p(s), s.size)
    return s


def topk(s, q_pos, m, k):
    """Top-k visible entries per row, ascending index order, -1 padded. int32 [B,Tq,k]."""
    s = _np(s, np.float64)
    q_pos = _np(q_pos, np.int32)
    B, Tq, Nc = s.shape
    idx = np.empty((B, Tq, k), np.int32)
    lib().or_topk(_p(s), B, Tq, Nc, _p(q_pos), m, k, _p(idx))
    return idx


def csa_attn(q, kvc: KV, idx, raw: KV, W, q_pos, scale=None, sink=None):
    """CSA attention over selected entries + raw window. q bf16 [B,Tq,H,d].
    Returns (o fp64 [B,Tq,H,d], lse fp64 [B,Tq,H])."""
    q = _np(q, np.uint16)
    idx = _np(idx, np.int32)
    q_pos = _np(q_pos, np.int32)
    sink = _np(sink, np.float32)
    B, Tq, H, d = q.shape
    k = idx.shape[-1]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    o = np.empty((B, Tq, H, d), np.float64)
    lse = np.empty((B, Tq, H), np.float64)
    lib().or_csa_attn(_p(q), B, Tq, H, d, *kvc.args(), _p(idx), k, *raw.args(), W, _p(q_pos),
                      scale, _p(sink), _p(o), _p(lse))
    return o, lse


def hca_attn(q, kvh: KV, Nh, mh, raw: KV, W, q_pos, scale=None, sink=None):
    """HCA dense attention over visible entries + raw window. Returns (o, lse) fp64."""
    q = _np(q, np.uint16)
    q_pos = _np(q_pos, np.int32)
    sink = _np(sink, np.float32)
    B, Tq, H, d = q.shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    o = np.empty((B, Tq, H, d), np.float64)
    lse = np.empty((B, Tq, H), np.float64)
    lib().or_hca_attn(_p(q), B, Tq, H, d, *kvh.args(), Nh, mh, *raw.args(), W, _p(q_pos),
                      scale, _p(sink), _p(o), _p(lse))
    return o, lse


def rmsnorm(x, gamma=None, eps=1e-6):
    """RMSNorm over the last axis in fp64: x / sqrt(mean(x^2) + eps) * gamma.  x: fp64, or
    bf16 (uint16 bits / torch bfloat16), any leading shape; gamma fp32 [d] or None."""
    a = _np(x)
    xd = dequant_bf16(a) if a.dtype == np.uint16 else np.ascontiguousarray(a, dtype=np.float64)
    d = xd.shape[-1]
    rows = xd.size // d if d else 0
    out = np.empty_like(xd)
    g = _np(gamma, np.float32)
    lib().or_rmsnorm(_p(xd), rows, d, _p(g), float(eps), _p(out))
    return out


def quant_kv_fp8(kv):
    """bf16 [..., d] -> (E4M3 codes [..., d/2] uint8, fp32 scale [...], bf16 bits [..., d/2])."""
    kv = _np(kv, np.uint16)
    d = kv.shape[-1]
    lead = kv.shape[:-1]
    rows = int(np.prod(lead)) if lead else 1
    nope = np.empty(lead + (d // 2,), np.uint8)
    scale = np.empty(lead, np.float32)
    rope = np.empty(lead + (d // 2,), np.uint16)
    lib().or_quant_kv_fp8(_p(kv), rows, d, _p(nope), _p(scale), _p(rope))
    return nope, scale, rope


def quant_mxfp4(x):
    """bf16 [..., cols] -> (packed uint8 [..., cols/2], E8M0 uint8 [..., cols/32])."""
    x = _np(x, np.uint16)
    cols = x.shape[-1]
    lead = x.shape[:-1]
    rows = int(np.prod(lead)) if lead else 1
    packed = np.empty(lead + (cols // 2,), np.uint8)
    sf = np.empty(lead + (cols // 32,), np.uint8)
    lib().or_quant_mxfp4(_p(x), rows, cols, _p(packed), _p(sf))
    return packed, sf


def dequant_bf16(bits):
    """bf16 bits -> fp64 values (exact)."""
    b = _np(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)
