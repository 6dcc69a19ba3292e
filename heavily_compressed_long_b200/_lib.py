"""ctypes declarations of libhcl's C ABI (include/hcl.h).  Argument marshalling only.

Loading fails loudly when the in-tree libhcl.so is missing: there is no fallback path.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhcl.so")

HCL_OK, HCL_ERR_INVALID_ARG, HCL_ERR_UNSUPPORTED, HCL_ERR_CUDA = 0, 1, 2, 4
HCL_ERR_TIMEOUT, HCL_ERR_DEVICE_FAULT = 8, 16
HCL_BF16, HCL_FP32, HCL_FP8SPLIT, HCL_MXFP4 = 0, 1, 2, 3

P = ctypes.c_void_p
I = ctypes.c_int
I64 = ctypes.c_int64
F = ctypes.c_float
SZ = ctypes.c_size_t


class hcl_kv_t(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("cap", ctypes.c_int32), ("data", P), ("scale", P),
                ("rope", P)]


KVP = ctypes.POINTER(hcl_kv_t)

# name -> (restype, argtypes)
SIGNATURES = {
    "hcl_version": (ctypes.c_char_p, []),
    "hcl_last_error": (ctypes.c_char_p, []),
    "hcl_csa_compress": (I, [P, P, P, I, I, I, I, I, I, P, I, I, P, F, P]),
    "hcl_hca_compress": (I, [P, P, P, I, I, I, I, I, I, P, I, I, P, F, P]),
    "hcl_quant_kv_fp8": (I, [P, I64, I, P, P, P, P]),
    "hcl_quant_mxfp4": (I, [P, I64, I, P, P, P]),
    "hcl_csa_index_scores": (I, [I, P, P, P, P, P, I, I, I, I, I, I, P, I, P, I, P, P]),
    "hcl_csa_topk_workspace_bytes": (SZ, [I, I, I, I, I]),
    "hcl_csa_topk": (I, [P, I, I, I, I, P, I, I, P, P, SZ, P, P]),
    "hcl_csa_sparse_attn_workspace_bytes": (SZ, [I, I, I, I, I]),
    "hcl_csa_sparse_attn": (I, [P, I, I, I, I, KVP, I, P, I, KVP, I, I, P, F, P, P, F, P, P, P, SZ,
                                P, P]),
    "hcl_csa_sparse_attn_noalloc": (I, [P, I, I, I, I, KVP, I, P, I, KVP, I, I, P, F, P, P, P, P, P]),
    "hcl_hca_dense_attn_workspace_bytes": (SZ, [I, I, I, I, I]),
    "hcl_hca_dense_attn": (I, [P, I, I, I, I, KVP, I, I, KVP, I, I, P, F, P, P, F, P, P, P, SZ, P,
                               P]),
    "hcl_csa_decode_step_workspace_bytes": (SZ, [I, I, I, I, I, I, I, I]),
    "hcl_csa_decode_step_kernels": (I, [I, I, I, I, I, I, I, I, I]),
    "hcl_csa_decode_step": (I, [P, P, P, I, P, P, I, I, I, I, I, I, I, KVP, I, I, I, KVP, I, I,
                                P, F, P, P, F, P, P, P, P, SZ, P, P]),
    "hcl_cache_append": (I, [P, P, P, P, I, I, I, P, P, I, KVP, KVP, P, I, I, P, P, I, KVP, P, I,
                             P, F, P, P]),
    "hcl_cp_candidates": (I, [P, I, P, I, I, I, I, P, P, P, P]),
    "hcl_cp_own": (I, [P, P, I, I, I, I, I, P, P, P]),
    "hcl_lse_merge": (I, [P, P, I, I64, I, I, P, P, P, P]),
    "hcl_selftest_bounded_wait": (I, [P, I, P]),
}

_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build the CUDA library first "
                "(python -m heavily_compressed_long_b200.build or __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


class HclError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"libhcl error {code}: {msg}")
        self.code = code


def check(code):
    if code != HCL_OK:
        raise HclError(code, lib().hcl_last_error().decode(errors="replace"))
    return code
