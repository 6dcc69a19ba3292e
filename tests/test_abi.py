"""The C ABI (no GPU): libhcl.so loads, exports every function include/hcl.h declares, the
ctypes binding declares each with the header's arity, and host-side argument validation
rejects bad calls before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hcl.h")


def header_functions():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    out = {}
    for m in re.finditer(r"HCL_API\s+[\w\s\*]+?\b(hcl_\w+)\s*\(([^)]*)\)\s*;", txt, flags=re.S):
        args = [a.strip() for a in m.group(2).split(",") if a.strip() and a.strip() != "void"]
        out[m.group(1)] = len(args)
    return out


@pytest.fixture(scope="module")
def libhcl():
    from heavily_compressed_long_b200 import build as b
    b.build()
    from heavily_compressed_long_b200 import _lib
    return _lib


def test_header_parses():
    fns = header_functions()
    for name in ["hcl_csa_compress", "hcl_hca_compress", "hcl_csa_index_scores", "hcl_csa_topk",
                 "hcl_csa_sparse_attn", "hcl_hca_dense_attn", "hcl_quant_kv_fp8", "hcl_quant_mxfp4",
                 "hcl_csa_decode_step", "hcl_last_error"]:
        assert name in fns


def test_every_declared_symbol_is_exported(libhcl):
    so = ctypes.CDLL(libhcl.LIB_PATH)
    for name in header_functions():
        assert hasattr(so, name), f"{name} not exported"


def test_binding_arity_matches_header(libhcl):
    fns = header_functions()
    assert set(fns) == set(libhcl.SIGNATURES), set(fns) ^ set(libhcl.SIGNATURES)
    for name, n in fns.items():
        assert len(libhcl.SIGNATURES[name][1]) == n, name


def test_version_and_error_strings(libhcl):
    L = libhcl.lib()
    assert b"sm_100a" in L.hcl_version()


def test_host_validation_without_device(libhcl):
    L = libhcl.lib()
    fake = ctypes.c_void_p(1 << 20)
    # MXFP4 needs cols % 32 == 0
    assert L.hcl_quant_mxfp4(fake, 10, 48, fake, fake, None) == libhcl.HCL_ERR_INVALID_ARG
    assert b"multiple of 32" in L.hcl_last_error()
    # indexer: only dI == 64
    rc = L.hcl_csa_index_scores(libhcl.HCL_BF16, fake, None, fake, fake, None, 1, 1, 4, 32, 8, 8,
                                fake, 4, fake, libhcl.HCL_FP32, None, None)
    assert rc == libhcl.HCL_ERR_UNSUPPORTED
    # top-k: k out of range
    rc = L.hcl_csa_topk(fake, libhcl.HCL_FP32, 1, 1, 100, fake, 4, 5000, fake, None, 0, None, None)
    assert rc == libhcl.HCL_ERR_INVALID_ARG
    # compressor: entry range beyond ceil(L/m)
    rc = L.hcl_csa_compress(fake, fake, fake, 1, 40, 128, 4, 0, 11, fake, libhcl.HCL_FP32, 64, None,
                            0.0, None)
    assert rc == libhcl.HCL_ERR_INVALID_ARG
    # misaligned pointer
    rc = L.hcl_quant_kv_fp8(ctypes.c_void_p((1 << 20) + 4), 4, 128, fake, fake, fake, None)
    assert rc == libhcl.HCL_ERR_INVALID_ARG
    # attention: d != 128 unsupported; kv descriptor format check
    kv = libhcl.hcl_kv_t(libhcl.HCL_BF16, 16, fake.value, None, None)
    rc = L.hcl_csa_sparse_attn(fake, 1, 1, 8, 64, ctypes.byref(kv), 16, fake, 4, ctypes.byref(kv),
                               64, 8, fake, 0.1, None, None, 0.0, fake, None, None, 0, None, None)
    assert rc == libhcl.HCL_ERR_UNSUPPORTED
    bad = libhcl.hcl_kv_t(7, 16, fake.value, None, None)
    rc = L.hcl_csa_sparse_attn(fake, 1, 1, 8, 128, ctypes.byref(bad), 16, fake, 4, ctypes.byref(kv),
                               64, 8, fake, 0.1, None, None, 0.0, fake, None, None, 0, None, None)
    assert rc == libhcl.HCL_ERR_INVALID_ARG
    # empty problems are a no-op success
    assert L.hcl_quant_mxfp4(None, 0, 64, None, None, None) == libhcl.HCL_OK


def test_workspace_queries(libhcl):
    L = libhcl.lib()
    # decode at B = 8, H = 128, k + W = 1152: the splits merge inside a cluster, no workspace
    assert L.hcl_csa_sparse_attn_workspace_bytes(8, 1, 128, 1024, 128) == 0
    # one sequence with k = 4096 splits into more pieces than a cluster holds -> workspace
    assert L.hcl_csa_sparse_attn_workspace_bytes(1, 1, 128, 4096, 128) > 0
    # a prefill chunk with many queries does not split
    assert L.hcl_csa_sparse_attn_workspace_bytes(1, 4096, 64, 1024, 128) == 0
    assert L.hcl_csa_decode_step_workspace_bytes(8, 128, 16, 262144, 1024, 128,
                                                 libhcl.HCL_MXFP4, libhcl.HCL_BF16) > 8 * 262144 * 2
    # MXFP4 keys + bf16 scores: the workspace also holds 5 bytes per 16-entry group of every row
    # (largest, second largest, position of the largest) for the top-k; fp32 scores do not
    for Nc in (262144, 70000, 4096):
        ngp = ((Nc + 15) // 16 + 15) // 16 * 16
        with_sum = L.hcl_csa_decode_step_workspace_bytes(8, 128, 16, Nc, 1024, 128,
                                                         libhcl.HCL_MXFP4, libhcl.HCL_BF16)
        scores_only = 8 * Nc * 2 + 8 * 1024 * 4
        assert with_sum >= scores_only + 8 * ngp * 5
    fp32 = L.hcl_csa_decode_step_workspace_bytes(8, 128, 16, 262144, 1024, 128,
                                                 libhcl.HCL_MXFP4, libhcl.HCL_FP32)
    assert fp32 >= 8 * 262144 * 4 and fp32 < 8 * 262144 * 4 + 8 * 16384 * 5
