"""Python binding of libhcl with the C ABI's names; torch tensors in, argument marshalling only.

Every function takes CUDA tensors (device memory owned by the caller) and enqueues the
corresponding libhcl call on the current torch stream (or `stream`).  No arithmetic of the
method happens here.  Formats: HCL_BF16 / HCL_FP32 / HCL_FP8SPLIT / HCL_MXFP4.
"""
import ctypes
import math

import torch

from . import _lib
from ._lib import (HCL_BF16, HCL_FP32, HCL_FP8SPLIT, HCL_MXFP4, check, hcl_kv_t, lib)

__all__ = ["KV", "hcl_csa_compress", "hcl_hca_compress", "hcl_quant_kv_fp8", "hcl_quant_mxfp4",
           "hcl_csa_index_scores", "hcl_csa_topk", "hcl_csa_sparse_attn", "hcl_hca_dense_attn",
           "hcl_csa_decode_step", "hcl_cache_append", "hcl_selftest_bounded_wait", "HCL_BF16", "HCL_FP32",
           "HCL_FP8SPLIT", "HCL_MXFP4"]


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libhcl takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libhcl takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class KV:
    """A KV store (see hcl_kv_t): bf16 rows [B, cap, d], or split rows: e4m3 codes
    [B, cap, d/2] (uint8), fp32 scale [B, cap], bf16 RoPE half [B, cap, d/2]."""

    def __init__(self, data, scale=None, rope=None):
        self.data, self.scale, self.rope = data, scale, rope
        self.fmt = HCL_FP8SPLIT if scale is not None else HCL_BF16
        self.cap = data.shape[1]
        self._c = hcl_kv_t(self.fmt, self.cap, _ptr(data).value, None if scale is None else _ptr(scale).value,
                           None if rope is None else _ptr(rope).value)

    def ref(self):
        return ctypes.byref(self._c)


def _fmt_of(t):
    return HCL_FP32 if t.dtype == torch.float32 else HCL_BF16


def hcl_csa_compress(kv, gate, bias, m, out, entry_begin=0, entry_end=None, gamma=None,
                     eps=1e-6, stream=None):
    """gamma (fp32 [d] CUDA tensor): RMSNorm each pooled entry (x / rms(x) * gamma)."""
    B, L, d = kv.shape
    if entry_end is None:
        entry_end = -(-L // m)
    check(lib().hcl_csa_compress(_ptr(kv), _ptr(gate), _ptr(bias), B, L, d, m, entry_begin,
                                 entry_end, _ptr(out), _fmt_of(out), out.shape[1], _ptr(gamma),
                                 eps, _stream(stream)))
    return out


def hcl_hca_compress(kv, gate, bias, m, out, entry_begin=0, entry_end=None, gamma=None,
                     eps=1e-6, stream=None):
    B, L, d = kv.shape
    if entry_end is None:
        entry_end = -(-L // m)
    check(lib().hcl_hca_compress(_ptr(kv), _ptr(gate), _ptr(bias), B, L, d, m, entry_begin,
                                 entry_end, _ptr(out), _fmt_of(out), out.shape[1], _ptr(gamma),
                                 eps, _stream(stream)))
    return out


def hcl_quant_kv_fp8(kv, nope, scale, rope, stream=None):
    d = kv.shape[-1]
    rows = kv.numel() // d
    check(lib().hcl_quant_kv_fp8(_ptr(kv), rows, d, _ptr(nope), _ptr(scale), _ptr(rope),
                                 _stream(stream)))


def hcl_quant_mxfp4(x, packed, sf, stream=None):
    cols = x.shape[-1]
    rows = x.numel() // cols
    check(lib().hcl_quant_mxfp4(_ptr(x), rows, cols, _ptr(packed), _ptr(sf), _stream(stream)))


def hcl_csa_index_scores(op_fmt, qI, w, kI, q_pos, m, scores, Nc=None, qI_sf=None, kI_sf=None,
                         status=None, stream=None):
    B, Tq, HI = w.shape
    dI = qI.shape[-1] * (2 if op_fmt == HCL_MXFP4 else 1)
    cap = kI.shape[1]
    Nc = cap if Nc is None else Nc
    check(lib().hcl_csa_index_scores(op_fmt, _ptr(qI), _ptr(qI_sf), _ptr(w), _ptr(kI), _ptr(kI_sf),
                                     B, Tq, HI, dI, Nc, cap, _ptr(q_pos), m, _ptr(scores),
                                     _fmt_of(scores), _ptr(status), _stream(stream)))
    return scores


def hcl_csa_topk(scores, q_pos, m, k, idx, status=None, stream=None):
    B, Tq, Nc = scores.shape
    fmt = _fmt_of(scores)
    wsb = lib().hcl_csa_topk_workspace_bytes(B, Tq, Nc, k, fmt)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=scores.device) if wsb else None
    check(lib().hcl_csa_topk(_ptr(scores), fmt, B, Tq, Nc, _ptr(q_pos), m, k, _ptr(idx), _ptr(ws),
                             wsb, _ptr(status), _stream(stream)))
    return idx


def csa_sparse_attn_workspace_bytes(B, Tq, H, k, W):
    return lib().hcl_csa_sparse_attn_workspace_bytes(B, Tq, H, k, W)


def hcl_csa_sparse_attn(q, kvc: KV, Nc, idx, raw: KV, L, W, q_pos, out, lse=None, scale=None,
                        sink=None, ws=None, status=None, q_gamma=None, q_eps=1e-6, stream=None):
    B, Tq, H, d = q.shape
    k = idx.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    need = csa_sparse_attn_workspace_bytes(B, Tq, H, k, W)
    if ws is None and need:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    check(lib().hcl_csa_sparse_attn(_ptr(q), B, Tq, H, d, kvc.ref(), Nc, _ptr(idx), k, raw.ref(),
                                    L, W, _ptr(q_pos), scale, _ptr(sink), _ptr(q_gamma), q_eps,
                                    _ptr(out), _ptr(lse),
                                    _ptr(ws), 0 if ws is None else ws.numel(), _ptr(status),
                                    _stream(stream)))
    return out


def hca_dense_attn_workspace_bytes(B, Tq, H, Nh, W):
    return lib().hcl_hca_dense_attn_workspace_bytes(B, Tq, H, Nh, W)


def hcl_hca_dense_attn(q, kvh: KV, Nh, mh, raw: KV, L, W, q_pos, out, lse=None, scale=None,
                       sink=None, ws=None, status=None, q_gamma=None, q_eps=1e-6, stream=None):
    B, Tq, H, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    need = hca_dense_attn_workspace_bytes(B, Tq, H, Nh, W)
    if ws is None and need:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    check(lib().hcl_hca_dense_attn(_ptr(q), B, Tq, H, d, kvh.ref(), Nh, mh, raw.ref(), L, W,
                                   _ptr(q_pos), scale, _ptr(sink), _ptr(q_gamma), q_eps, _ptr(out),
                                   _ptr(lse), _ptr(ws),
                                   0 if ws is None else ws.numel(), _ptr(status), _stream(stream)))
    return out


def decode_step_workspace_bytes(B, H, HI, Nc, k, W, op_fmt, score_fmt):
    return lib().hcl_csa_decode_step_workspace_bytes(B, H, HI, Nc, k, W, op_fmt, score_fmt)


def hcl_csa_decode_step(q, qI, w, op_fmt, kI, kvc: KV, Nc, m, k, raw: KV, L, W, q_pos, out,
                        score_fmt=HCL_FP32, kI_sf=None, lse=None, idx_out=None, scale=None,
                        sink=None, ws=None, status=None, q_gamma=None, q_eps=1e-6, stream=None):
    """One CSA decode step (Tq = 1): MXFP4-quantise qI (MXFP4 keys only), score, top-k, attend."""
    B, _, H, d = q.shape
    HI, dI = qI.shape[-2], qI.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    need = decode_step_workspace_bytes(B, H, HI, Nc, k, W, op_fmt, score_fmt)
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    check(lib().hcl_csa_decode_step(_ptr(q), _ptr(qI), _ptr(w), op_fmt, _ptr(kI), _ptr(kI_sf),
                                    kI.shape[1], score_fmt, B, H, HI, dI, d, kvc.ref(), Nc, m, k,
                                    raw.ref(), L, W, _ptr(q_pos), scale, _ptr(sink), _ptr(q_gamma),
                                    q_eps, _ptr(out), _ptr(lse), _ptr(idx_out), _ptr(ws), ws.numel(),
                                    _ptr(status),
                                    _stream(stream)))
    return out


def hcl_cache_append(kv_new, gate_new, t_new, stage_kv, stage_gate, raw: KV, kvc: KV = None,
                     bias_csa=None, m=4, kI_new=None, kI=None, kI_sf=None, kvh: KV = None,
                     bias_hca=None, mh=128, gamma=None, eps=1e-6, stream=None):
    """Append one token per sequence (kv_new / gate_new bf16 [B, d], t_new int32 [B]) to one
    layer's cache: staging rings, raw window store, and the CSA (kvc, index keys kI: bf16
    [B, cap, dI], or MXFP4 packed uint8 [B, cap, dI/2] with kI_sf) or HCA (kvh) entry it
    completes."""
    B, d = kv_new.shape
    kI_fmt = HCL_MXFP4 if kI_sf is not None else HCL_BF16
    dI = 0 if kI is None else (kI.shape[-1] * (2 if kI_fmt == HCL_MXFP4 else 1))
    check(lib().hcl_cache_append(_ptr(kv_new), _ptr(gate_new), _ptr(kI_new), _ptr(t_new), B, d, dI,
                                 _ptr(stage_kv), _ptr(stage_gate), stage_kv.shape[1], raw.ref(),
                                 None if kvc is None else kvc.ref(), _ptr(bias_csa), m, kI_fmt,
                                 _ptr(kI), _ptr(kI_sf), 0 if kI is None else kI.shape[1],
                                 None if kvh is None else kvh.ref(), _ptr(bias_hca), mh,
                                 _ptr(gamma), eps, None, _stream(stream)))


def hcl_cp_candidates(scores, idx, e0, cand_scores, cand_idx, status=None, stream=None):
    """Local top-k (idx [B, 1, k]) over a rank's scores [B, 1, Nc_local] -> (fp32 score, global
    index) candidates [B, k]."""
    B, _, Nc_local = scores.shape
    k = idx.shape[-1]
    check(lib().hcl_cp_candidates(_ptr(scores), _fmt_of(scores), _ptr(idx), B, Nc_local, k, e0,
                                  _ptr(cand_scores), _ptr(cand_idx), _ptr(status), _stream(stream)))


def hcl_cp_own(pos, gathered_idx, e0, e1, sel_out, own_out, stream=None):
    """pos [B, 1, k] selected positions in the gathered list gathered_idx [B, n] -> global
    selection sel_out [B, 1, k] and this rank's local share own_out [B, 1, k]."""
    B, n = gathered_idx.shape
    k = pos.shape[-1]
    check(lib().hcl_cp_own(_ptr(pos), _ptr(gathered_idx), B, n, k, e0, e1, _ptr(sel_out),
                           _ptr(own_out), _stream(stream)))


def hcl_lse_merge(o_parts, lse_parts, out, lse_out=None, sink=None, stream=None):
    """o_parts bf16 [G, B, Tq, H, d], lse_parts fp32 [G, B, Tq, H] -> out [B, Tq, H, d]."""
    G = o_parts.shape[0]
    H, d = o_parts.shape[-2], o_parts.shape[-1]
    rows = lse_parts[0].numel()
    check(lib().hcl_lse_merge(_ptr(o_parts), _ptr(lse_parts), G, rows, d, H, _ptr(sink), _ptr(out),
                              _ptr(lse_out), _stream(stream)))


def hcl_selftest_bounded_wait(status, limit_us=1000, stream=None):
    check(lib().hcl_selftest_bounded_wait(_ptr(status), limit_us, _stream(stream)))
