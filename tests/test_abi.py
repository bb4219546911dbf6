"""CPU tests of the C ABI: the library loads, exports every function include/tq.h declares,
its host-side builders (codebook, signs, QJL matrix, record sizes) agree with the oracle,
and invalid arguments are rejected with a status code before any device work."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import oracle as O
from tests.conftest import ROOT

tq = pytest.importorskip("quantized_decode_attention_kv_b200.tq")


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "tq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_\w+)\s*\(", text)))


def test_header_functions_are_exported_and_bound():
    names = _declared_functions()
    assert len(names) >= 13
    lib = ctypes.CDLL(tq.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
        assert n in tq.EXPORTS, n


def test_library_links_only_cuda_runtime_and_system_libs():
    # the product is self-contained: no torch symbols in the boundary
    out = os.popen(f"nm -D --undefined-only {tq.LIB_PATH}").read()
    assert "torch" not in out and "c10" not in out


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("d", [16, 64, 128, 256])
def test_codebook_matches_oracle(bits, d):
    c, b = tq.tq_make_codebook(bits, d)
    oc, ob = O.codebook(bits, d)
    # the library rounds its double codebook to float32: within one float32 ulp of the oracle
    for got, want in ((c, oc), (b, ob)):
        ulp = np.spacing(np.abs(want).astype(np.float32)).astype(np.float64) + 1e-30
        assert np.all(np.abs(got.astype(np.float64) - want) <= ulp)
    assert np.all(c[: len(c) // 2] == -c[::-1][: len(c) // 2])


@pytest.mark.parametrize("d", [16, 64, 128, 256])
def test_sign_vector_matches_oracle(d):
    for seed in (0, 1, 77, 2**40 + 3):
        bits = np.unpackbits(tq.tq_make_signs(seed, d), bitorder="little")
        assert np.array_equal(bits == 1, O.rotation_signs(seed, d) == -1.0)
    assert tq.tq_make_signs(0, 128).nbytes == 16


@pytest.mark.parametrize("m,d", [(64, 64), (8, 16), (128, 128), (256, 32)])
def test_qjl_matrix_matches_oracle(m, d):
    S = tq.tq_make_qjl_matrix(1, m, d)
    ref = O.qjl_matrix(1, m, d)
    # both sides round a double Box-Muller value to float32; libm and Python's math may differ
    # by an ulp in double, which can move the float32 result by at most one ulp
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(S.astype(np.float64) - ref) <= ulp)
    assert np.mean(S.astype(np.float64) == ref) > 0.999


@pytest.mark.parametrize("d", [16, 64, 128, 256])
@pytest.mark.parametrize("bits,mode,m", [(1, 0, 0), (2, 0, 0), (3, 0, 0), (4, 0, 0),
                                         (1, 1, 0), (2, 1, 0), (2, 1, 64), (3, 1, 8)])
def test_record_sizes_match_oracle(d, bits, mode, m):
    mm = m or d
    assert tq.tq_code_bytes(d, bits, mode, m) == O.code_bytes(d, bits, mode)
    assert tq.tq_sign_bytes(d, bits, mode, m) == O.sign_bytes(d, bits, mode, mm)
    assert tq.tq_record_bytes(d, bits, mode, m) == O.record_bytes(d, bits, mode, mm)


def test_record_bytes_reproduce_published_ratios():
    assert tq.tq_record_bytes(128, 3) == 50 and 256 / 50 == 5.12
    assert tq.tq_record_bytes(64, 2, tq.TQ_PROD, 64) == 20


def test_host_helpers_reject_bad_arguments():
    lib = tq.lib
    buf = np.zeros(64, dtype=np.float32)
    assert lib.tq_make_codebook(0, 128, buf.ctypes.data, buf.ctypes.data) == tq.TQ_ERR_UNSUPPORTED
    assert lib.tq_make_codebook(5, 128, buf.ctypes.data, buf.ctypes.data) == tq.TQ_ERR_UNSUPPORTED
    assert lib.tq_make_codebook(3, 96, buf.ctypes.data, buf.ctypes.data) == tq.TQ_ERR_UNSUPPORTED
    assert lib.tq_make_codebook(3, 512, buf.ctypes.data, buf.ctypes.data) == tq.TQ_ERR_UNSUPPORTED
    assert lib.tq_make_codebook(3, 128, None, buf.ctypes.data) == tq.TQ_ERR_INVALID_ARG
    assert "bits" in tq.last_error() or "pointer" in tq.last_error()
    assert lib.tq_make_qjl_matrix(1, 12, 64, buf.ctypes.data) == tq.TQ_ERR_UNSUPPORTED
    assert lib.tq_make_qjl_matrix(1, 512, 64, buf.ctypes.data) == tq.TQ_ERR_UNSUPPORTED
    assert lib.tq_make_signs(0, 100, buf.ctypes.data) == tq.TQ_ERR_UNSUPPORTED
    assert lib.tq_code_bytes(100, tq.tq_qcfg(3, 0, 0)) == 0
    assert lib.tq_record_bytes(128, tq.tq_qcfg(2, 1, 12)) == 0
    assert lib.tq_record_bytes(128, tq.tq_qcfg(2, 7, 0)) == 0


def _cache(**kw):
    base = dict(B=2, Hkv=2, T_cap=64, d=128, seed=0, kc=tq.tq_qcfg(4, 0, 0), vc=tq.tq_qcfg(2, 0, 0),
                k_codes=16, v_codes=16, k_norm=16, v_norm=16, k_signs=None, v_signs=None,
                k_rnorm=None, v_rnorm=None, k_qjl=None, v_qjl=None)
    base.update(kw)
    c = tq.tq_cache()
    for k, v in base.items():
        setattr(c, k, v)
    return c


def test_device_entry_points_validate_before_launch():
    # every case fails in argument checking, so no CUDA call is made (this box has no GPU)
    lib = tq.lib
    P = 4096  # a fake, 16-byte aligned "device" address: never dereferenced on these paths
    c = _cache()
    ref = ctypes.byref
    assert lib.tq_quantize_kv(P, P, 1, 4, 0, None, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_quantize_kv(None, None, 1, 4, 0, ref(c), None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_quantize_kv(P, P, 9, 4, 0, ref(c), None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_quantize_kv(P, P, 1, 4, 62, ref(c), None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_quantize_kv(P, P, 1, -1, 0, ref(c), None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_quantize_kv(P + 2, P, 1, 4, 0, ref(c), None) == tq.TQ_ERR_INVALID_ARG
    # T = 0 is a no-op success
    assert lib.tq_quantize_kv(P, P, 1, 0, 64, ref(c), None) == tq.TQ_OK
    bad_d = _cache(d=96)
    assert lib.tq_quantize_kv(P, P, 1, 4, 0, ref(bad_d), None) == tq.TQ_ERR_UNSUPPORTED
    bad_bits = _cache(kc=tq.tq_qcfg(5, 0, 0))
    assert lib.tq_quantize_kv(P, P, 1, 4, 0, ref(bad_bits), None) == tq.TQ_ERR_UNSUPPORTED
    e2m1_3bit = _cache(kc=tq.tq_qcfg(3, tq.TQ_E2M1, 0))  # E2M1 codes are 4 bits
    assert lib.tq_quantize_kv(P, P, 1, 4, 0, ref(e2m1_3bit), None) == tq.TQ_ERR_UNSUPPORTED
    assert "TQ_E2M1" in tq.last_error()
    assert tq.tq_record_bytes(128, 4, tq.TQ_E2M1) == tq.tq_record_bytes(128, 4, tq.TQ_MSE) == 66
    prod_missing = _cache(kc=tq.tq_qcfg(2, 1, 0))
    assert lib.tq_quantize_kv(P, P, 1, 4, 0, ref(prod_missing), None) == tq.TQ_ERR_INVALID_ARG
    assert "TQ_PROD" in tq.last_error()
    misaligned = _cache(k_codes=P + 4)
    assert lib.tq_quantize_kv(P, P, 1, 4, 0, ref(misaligned), None) == tq.TQ_ERR_INVALID_ARG
    # decode: Hq not a multiple of Hkv, T_len out of range, null workspace
    assert lib.tq_decode_attention(P, 1, 3, 8, 0.1, ref(c), P, P, 1 << 20, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_decode_attention(P, 1, 4, 0, 0.1, ref(c), P, P, 1 << 20, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_decode_attention(P, 1, 4, 65, 0.1, ref(c), P, P, 1 << 20, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_decode_attention(P, 1, 4, 8, float("nan"), ref(c), P, P, 1 << 20, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_decode_attention(None, 1, 4, 8, 0.1, ref(c), P, P, 1 << 20, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_decode_workspace_bytes(2, 3, 8, ref(c)) == 0
    assert lib.tq_dequantize(ref(c), 2, 8, P, 0, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_dequantize(ref(c), 0, 65, P, 0, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_dequantize(ref(c), 0, 0, P, 0, None) == tq.TQ_OK
    assert lib.tq_decode_attention_bf16(P, 3, P, P, 2, 2, 64, 8, 128, 0.1, P, P, 1, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_decode_attention_bf16(P, 4, P, P, 2, 2, 64, 8, 96, 0.1, P, P, 1, None) == tq.TQ_ERR_UNSUPPORTED
    assert lib.tq_decode_bf16_workspace_bytes(2, 3, 2, 8, 128) == 0


def test_binding_refuses_host_tensors():
    import torch
    cache = type("C", (), {})()
    with pytest.raises(tq.TQError):
        tq.tq_quantize_kv(torch.zeros(1, 1, 4, 128), None, cache)


def _fake_cache(B, Hkv, T_cap, d, kb, km, vb, vm, m=0):
    """A tq_cache whose pointers are aligned placeholders: tq_launch_counts inspects shapes and
    bit-widths only and never touches device memory."""
    c = tq.tq_cache()
    c.B, c.Hkv, c.T_cap, c.d, c.seed = B, Hkv, T_cap, d, 0
    c.kc = tq.tq_qcfg(kb, km, m)
    c.vc = tq.tq_qcfg(vb, vm, m)
    for i, f in enumerate(("k_codes", "v_codes", "k_norm", "v_norm", "k_signs", "v_signs",
                           "k_rnorm", "v_rnorm", "k_qjl", "v_qjl")):
        setattr(c, f, 0x10000 * (i + 1))
    return c


@pytest.mark.parametrize("cfg,dtype,Hq,want", [
    # 16-bit MSE write: one launch for K and V; MSE d=128 decode: decode (which prepares its
    # queries itself) and combine
    ((16, 8, 32768, 128, 4, O.MSE, 2, O.MSE), 1, 32, (1, 2)),
    ((4, 8, 1024, 128, 3, O.MSE, 3, O.MSE), 2, 32, (1, 2)),
    # fp32 input takes the per-vector kernel, one launch per tensor
    ((1, 1, 1024, 128, 4, O.MSE, 4, O.MSE), 0, 1, (2, 2)),
    # d = 64 TurboQuant_prod with 64 sketch rows: tensor-core write and decode (G <= 2)
    ((64, 12, 8192, 64, 2, O.PROD, 2, O.PROD, 64), 1, 12, (1, 3)),
    ((64, 12, 8192, 64, 2, O.PROD, 2, O.PROD, 64), 1, 48, (1, 2)),
    # shapes without a tensor-core kernel: per-vector write, split-K decode + combine
    ((2, 2, 100, 256, 4, O.MSE, 2, O.MSE), 1, 4, (2, 2)),
    ((2, 2, 100, 128, 4, O.MSE, 2, O.MSE), 1, 2 * 32, (1, 2)),
])
def test_launch_counts_follow_the_kernel_selection(cfg, dtype, Hq, want):
    c = _fake_cache(*cfg)
    nq, nd = ctypes.c_int(-1), ctypes.c_int(-1)
    st = tq.lib.tq_launch_counts(ctypes.byref(c), dtype, 1, Hq, min(c.T_cap, 100), ctypes.byref(nq),
                                 ctypes.byref(nd))
    assert st == tq.TQ_OK, tq.last_error()
    assert (nq.value, nd.value) == want


def test_launch_counts_reject_bad_arguments():
    c = _fake_cache(1, 2, 10, 128, 4, O.MSE, 2, O.MSE)
    n = ctypes.c_int(0)
    assert tq.lib.tq_launch_counts(ctypes.byref(c), 7, 1, 2, 5, ctypes.byref(n), None) == tq.TQ_ERR_INVALID_ARG
    assert tq.lib.tq_launch_counts(ctypes.byref(c), 1, 1, 3, 5, ctypes.byref(n), None) == tq.TQ_ERR_INVALID_ARG
    assert tq.lib.tq_launch_counts(ctypes.byref(c), 1, 1, 2, 11, ctypes.byref(n), None) == tq.TQ_ERR_INVALID_ARG


def test_varlen_decode_validates_before_any_device_work():
    c = _fake_cache(3, 2, 64, 128, 4, O.MSE, 2, O.MSE)
    lens = (ctypes.c_int * 3)(10, 0, 5)
    out = ctypes.c_void_p(0x100000)
    st = tq.lib.tq_decode_attention_varlen(out, 1, 8, ctypes.cast(lens, ctypes.c_void_p), 0.1,
                                           ctypes.byref(c), out, out, 1 << 20, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "T_lens[1]" in tq.last_error()
    lens[1] = 65  # above T_cap
    assert tq.lib.tq_decode_attention_varlen(out, 1, 8, ctypes.cast(lens, ctypes.c_void_p), 0.1,
                                             ctypes.byref(c), out, out, 1 << 20, None) == tq.TQ_ERR_INVALID_ARG
    assert tq.lib.tq_decode_attention_varlen(out, 1, 8, None, 0.1, ctypes.byref(c), out, out, 1 << 20,
                                             None) == tq.TQ_ERR_INVALID_ARG
    assert tq.lib.tq_decode_varlen_workspace_bytes(8, ctypes.byref(c), None) == 0
    # TurboQuant_prod records with 32 sketch rows have no ragged (tensor-core) kernel
    p = _fake_cache(3, 2, 64, 64, 2, O.PROD, 2, O.PROD, 32)
    lens[1] = 7
    assert tq.lib.tq_decode_attention_varlen(out, 1, 4, ctypes.cast(lens, ctypes.c_void_p), 0.1,
                                             ctypes.byref(p), out, out, 1 << 20, None) == tq.TQ_ERR_UNSUPPORTED
    # more sequences than one launch's parameters carry
    big = _fake_cache(513, 1, 16, 128, 4, O.MSE, 2, O.MSE)
    many = (ctypes.c_int * 513)(*([4] * 513))
    assert tq.lib.tq_decode_attention_varlen(out, 1, 4, ctypes.cast(many, ctypes.c_void_p), 0.1,
                                             ctypes.byref(big), out, out, 1 << 20, None) == tq.TQ_ERR_UNSUPPORTED
