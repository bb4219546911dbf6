"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded
inputs, at sizes the oracle finishes in seconds that still span several tiles and a ragged
tail, plus edge cases. Full-size workloads are in test_gpu_workloads.py."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - the GPU tier always has a device
    pytest.skip("needs a CUDA device", allow_module_level=True)

from quantized_decode_attention_kv_b200 import tq  # noqa: E402
from quantized_decode_attention_kv_b200.workloads import random_kv  # noqa: E402

DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def _inputs(B, Hkv, T, d, dtype, seed, outliers=False, zero_at=None, scale=1.0):
    K, V = random_kv(B, Hkv, T, d, dtype=torch.float32, seed=seed, scale=scale)
    if outliers:
        K[..., :3] *= 20.0
    if zero_at is not None:
        K[0, 0, zero_at] = 0.0
        V[0, 0, zero_at] = 0.0
    return K.to(dtype), V.to(dtype)


# ------------------------------------------------------------------ quantize
QUANT_CASES = [
    # d, k(bits, mode), v(bits, mode), m
    (128, (4, O.MSE), (2, O.MSE), 0),
    (128, (3, O.MSE), (3, O.MSE), 0),
    (128, (1, O.MSE), (4, O.MSE), 0),
    (64, (2, O.PROD), (2, O.PROD), 64),
    (64, (1, O.PROD), (3, O.PROD), 32),
    (64, (1, O.PROD), (2, O.PROD), 64),
    (16, (3, O.MSE), (1, O.MSE), 0),
    (16, (2, O.PROD), (4, O.PROD), 8),
    (32, (4, O.MSE), (2, O.PROD), 0),
    (256, (4, O.MSE), (3, O.MSE), 0),
    (256, (2, O.PROD), (2, O.MSE), 256),
]


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("case", QUANT_CASES, ids=lambda c: f"d{c[0]}-k{c[1]}-v{c[2]}-m{c[3]}")
def test_quantize_matches_oracle(case, dtype):
    d, (kb, km), (vb, vm), m = case
    B, Hkv, T, T_cap, t_off = 2, 3, 37, 50, 6
    K, V = _inputs(B, Hkv, T, d, DT[dtype], seed=d + kb, outliers=True, zero_at=5)
    cache = tq.TQCache(B, Hkv, T_cap, d, kb, vb, km, vm, m, m, seed=11, qjl_seed=5)
    tq.tq_quantize_kv(K.cuda(), V.cuda(), cache, t_offset=t_off)
    torch.cuda.synchronize()
    for side, X, bits, mode in (("k", K, kb, km), ("v", V, vb, vm)):
        recs = P.oracle_records(P.to_np(X), bits, mode, 11, 5, m or None)
        st = P.compare_records(cache, side, recs, t_offset=t_off)
        assert st["flipped_near_boundary"] <= st["near_boundary"]
    # positions outside [t_off, t_off + T) stay untouched (zero)
    assert int(cache["k_norm"][:, :, :t_off].abs().sum()) == 0
    assert int(cache["v_norm"][:, :, t_off + T:].abs().sum()) == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", [(128, (4, O.MSE), (2, O.MSE), 0), (64, (2, O.PROD), (2, O.PROD), 64)],
                         ids=["d128-mse", "d64-prod"])
def test_quantize_norms_beyond_fp16_range(case, dtype):
    # per-token scales from 1e2 to 3e6: norms from ~1e3 to ~3e7, so about half of them exceed
    # the largest fp16 value and round to +inf in the stored norm (round to nearest, as the
    # oracle's float32 -> float16 conversion does); the codes are those of the unit vector
    d, (kb, km), (vb, vm), m = case
    B, Hkv, T = 2, 2, 40
    K, V = random_kv(B, Hkv, T, d, dtype=torch.float32, seed=77)
    sc = torch.logspace(2, 6.5, T, dtype=torch.float32).view(1, 1, T, 1)
    K, V = (K * sc).to(DT[dtype]), (V * sc.flip(2)).to(DT[dtype])
    cache = tq.TQCache(B, Hkv, T, d, kb, vb, km, vm, m, m, seed=3, qjl_seed=9)
    tq.tq_quantize_kv(K.cuda(), V.cuda(), cache)
    torch.cuda.synchronize()
    saturated = 0
    for side, X, bits, mode in (("k", K, kb, km), ("v", V, vb, vm)):
        recs = P.oracle_records(P.to_np(X), bits, mode, 3, 9, m or None)
        P.compare_records(cache, side, recs)
        saturated += sum(int(np.sum(np.isinf(r.norm16.astype(np.float64)))) for r in recs)
    assert 0.3 * 2 * B * Hkv * T <= saturated <= 0.7 * 2 * B * Hkv * T


def test_quantize_only_keys_or_values():
    d = 64
    K, V = _inputs(1, 2, 20, d, torch.bfloat16, seed=3)
    cache = tq.TQCache(1, 2, 20, d, 4, 2)
    tq.tq_quantize_kv(None, V.cuda(), cache)
    torch.cuda.synchronize()
    assert int(cache["k_norm"].abs().sum()) == 0
    P.compare_records(cache, "v", P.oracle_records(P.to_np(V), 2, O.MSE, 0, 1, None))
    tq.tq_quantize_kv(K.cuda(), None, cache)
    torch.cuda.synchronize()
    P.compare_records(cache, "k", P.oracle_records(P.to_np(K), 4, O.MSE, 0, 1, None))


def test_quantize_is_deterministic_and_per_head_independent():
    d, B, H, T = 128, 2, 4, 300
    K, V = _inputs(B, H, T, d, torch.bfloat16, seed=9, outliers=True)
    c1 = tq.TQCache(B, H, T, d, 4, 2)
    c2 = tq.TQCache(B, H, T, d, 4, 2)
    tq.tq_quantize_kv(K.cuda(), V.cuda(), c1)
    tq.tq_quantize_kv(K.cuda(), V.cuda(), c2)
    one = tq.TQCache(1, 1, T, d, 4, 2)
    tq.tq_quantize_kv(K[1:2, 2:3].contiguous().cuda(), V[1:2, 2:3].contiguous().cuda(), one)
    torch.cuda.synchronize()
    for key in ("k_codes", "v_codes", "k_norm", "v_norm"):
        assert torch.equal(c1[key], c2[key])
        assert torch.equal(c1[key][1, 2], one[key][0, 0])


# ------------------------------------------------------------------ dequantize
@pytest.mark.parametrize("case", QUANT_CASES, ids=lambda c: f"d{c[0]}-k{c[1]}-v{c[2]}-m{c[3]}")
def test_dequantize_matches_oracle(case):
    d, (kb, km), (vb, vm), m = case
    B, Hkv, T = 2, 2, 45
    K, V = _inputs(B, Hkv, T, d, torch.float32, seed=d * 3 + vb, scale=7.0)
    cache = tq.TQCache(B, Hkv, T + 3, d, kb, vb, km, vm, m, m, seed=4, qjl_seed=9)
    for side, X, bits, mode in (("k", K, kb, km), ("v", V, vb, vm)):
        recs = P.oracle_records(P.to_np(X), bits, mode, 4, 9, m or None)
        P.upload(cache, side, recs)
        out = torch.empty(B, Hkv, T, d, device="cuda", dtype=torch.float32)
        tq.tq_dequantize(cache, 0 if side == "k" else 1, T, out)
        torch.cuda.synchronize()
        want = np.stack([O.dequantize(r) for r in recs]).reshape(B, Hkv, T, d)
        n16 = np.stack([r.norm16.astype(np.float64) for r in recs]).reshape(B, Hkv, T, 1)
        err = np.abs(P.to_np(out) - want) / np.maximum(n16, 1e-30)
        assert err.max() <= P.DEQUANT_ATOL, err.max()
        for dt in (torch.bfloat16, torch.float16):
            o2 = torch.empty(B, Hkv, T, d, device="cuda", dtype=dt)
            tq.tq_dequantize(cache, 0 if side == "k" else 1, T, o2)
            assert torch.allclose(o2.float(), out.to(dt).float(), rtol=0, atol=0)


# ------------------------------------------------------------------ decode
DECODE_CASES = [
    # d, G, Hkv, k(bits, mode), v(bits, mode), m, T_len, T_cap
    (128, 4, 2, (4, O.MSE), (2, O.MSE), 0, 1000, 1030),
    (128, 1, 1, (4, O.MSE), (4, O.MSE), 0, 1024, 1024),
    (128, 8, 1, (3, O.MSE), (3, O.MSE), 0, 777, 800),
    (128, 5, 2, (4, O.MSE), (2, O.MSE), 0, 300, 300),
    (64, 1, 3, (2, O.PROD), (2, O.PROD), 64, 520, 520),
    (64, 2, 2, (1, O.PROD), (3, O.PROD), 32, 129, 140),
    (16, 4, 2, (3, O.MSE), (1, O.MSE), 0, 257, 260),
    (32, 16, 1, (4, O.MSE), (2, O.PROD), 0, 200, 200),
    (256, 2, 2, (4, O.MSE), (2, O.MSE), 0, 390, 400),
    (256, 3, 1, (2, O.PROD), (4, O.MSE), 128, 128, 128),
    (128, 32, 1, (4, O.MSE), (2, O.MSE), 0, 64, 64),
    (128, 4, 2, (4, O.MSE), (2, O.MSE), 0, 1, 10),
    # the other key/value bit-widths of the tensor-core kernel, ragged tails
    (128, 2, 3, (3, O.MSE), (2, O.MSE), 0, 613, 640),
    (128, 6, 1, (4, O.MSE), (3, O.MSE), 0, 450, 450),
    (128, 3, 2, (3, O.MSE), (4, O.MSE), 0, 95, 100),
    # the tensor-core TurboQuant_prod kernel with two query heads per KV head
    (64, 2, 2, (2, O.PROD), (2, O.PROD), 64, 333, 340),
]


def _decode_case(case, q_dtype, k_scale=1.0, seed=0):
    d, G, Hkv, (kb, km), (vb, vm), m, T_len, T_cap = case
    B = 2
    Hq = G * Hkv
    K, V = _inputs(B, Hkv, T_cap, d, torch.float32, seed=seed + d + G, outliers=True, scale=k_scale)
    g = torch.Generator().manual_seed(seed + 17)
    q = torch.randn(B, Hq, d, generator=g).to(q_dtype)
    return B, Hq, K, V, q


@pytest.mark.parametrize("case", DECODE_CASES, ids=lambda c: f"d{c[0]}-G{c[1]}-H{c[2]}-k{c[3]}-v{c[4]}-T{c[6]}")
def test_decode_over_oracle_records_matches_oracle(case):
    d, G, Hkv, (kb, km), (vb, vm), m, T_len, T_cap = case
    B, Hq, K, V, q = _decode_case(case, torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    cache = tq.TQCache(B, Hkv, T_cap, d, kb, vb, km, vm, m, m, seed=21, qjl_seed=2)
    k_recs = P.oracle_records(P.to_np(K), kb, km, 21, 2, m or None)
    v_recs = P.oracle_records(P.to_np(V), vb, vm, 21, 2, m or None)
    P.upload(cache, "k", k_recs)
    P.upload(cache, "v", v_recs)
    out = torch.empty(B, Hq, d, device="cuda")
    ws = tq.workspace(tq.tq_decode_workspace_bytes(cache, Hq, T_len))
    tq.tq_decode_attention(q.cuda(), cache, T_len, scale, out, ws)
    torch.cuda.synchronize()
    want = P.oracle_decode(P.to_np(q), k_recs, v_recs, B, Hkv, scale, T_len)
    P.assert_attention_close(P.to_np(out), want)


@pytest.mark.parametrize("q_dtype", [torch.float32, torch.float16])
def test_decode_query_dtypes(q_dtype):
    case = DECODE_CASES[0]
    d, G, Hkv, (kb, km), (vb, vm), m, T_len, T_cap = case
    B, Hq, K, V, q = _decode_case(case, q_dtype, seed=5)
    cache = tq.TQCache(B, Hkv, T_cap, d, kb, vb, km, vm)
    k_recs = P.oracle_records(P.to_np(K), kb, km, 0, 1, None)
    v_recs = P.oracle_records(P.to_np(V), vb, vm, 0, 1, None)
    P.upload(cache, "k", k_recs)
    P.upload(cache, "v", v_recs)
    out = torch.empty(B, Hq, d, device="cuda")
    ws = tq.workspace(tq.tq_decode_workspace_bytes(cache, Hq, T_len))
    tq.tq_decode_attention(q.cuda(), cache, T_len, 0.3, out, ws)
    torch.cuda.synchronize()
    P.assert_attention_close(P.to_np(out), P.oracle_decode(P.to_np(q), k_recs, v_recs, B, Hkv, 0.3, T_len))


@pytest.mark.parametrize("G,kb,vb,T", [(8, 4, 2, 700), (4, 4, 2, 2000), (3, 3, 3, 1500), (2, 4, 4, 900)])
def test_decode_with_large_key_norms(G, kb, vb, T):
    # keys 50x the values' norm ("What the Paper Doesn't Tell You", Finding 1): near-one-hot
    # softmax, where score precision decides the output; every query-group width and key
    # bit-width of the tensor-core kernel (the last score n-tile full or half used)
    case = (128, G, 1, (kb, O.MSE), (vb, O.MSE), 0, T, T)
    B, Hq, K, V, q = _decode_case(case, torch.bfloat16, k_scale=50.0, seed=3 + G)
    cache = tq.TQCache(B, 1, T, 128, kb, vb)
    k_recs = P.oracle_records(P.to_np(K), kb, O.MSE, 0, 1, None)
    v_recs = P.oracle_records(P.to_np(V), vb, O.MSE, 0, 1, None)
    P.upload(cache, "k", k_recs)
    P.upload(cache, "v", v_recs)
    out = torch.empty(B, Hq, 128, device="cuda")
    ws = tq.workspace(tq.tq_decode_workspace_bytes(cache, Hq, T))
    tq.tq_decode_attention(q.cuda(), cache, T, 128 ** -0.5, out, ws)
    torch.cuda.synchronize()
    P.assert_attention_close(P.to_np(out), P.oracle_decode(P.to_np(q), k_recs, v_recs, B, 1, 128 ** -0.5))


@pytest.mark.parametrize("case", DECODE_CASES[:6], ids=lambda c: f"d{c[0]}-G{c[1]}-k{c[3]}-v{c[4]}")
def test_quantize_then_decode_end_to_end(case):
    d, G, Hkv, (kb, km), (vb, vm), m, T_len, T_cap = case
    B, Hq, K, V, q = _decode_case(case, torch.bfloat16, seed=8)
    Kb, Vb = K.to(torch.bfloat16), V.to(torch.bfloat16)
    cache = tq.TQCache(B, Hkv, T_cap, d, kb, vb, km, vm, m, m, seed=6, qjl_seed=3)
    # prefill T_len - 1 tokens, then append the last one (decode-time write)
    tq.tq_quantize_kv(Kb[:, :, : T_len - 1].contiguous().cuda(), Vb[:, :, : T_len - 1].contiguous().cuda(),
                      cache, 0) if T_len > 1 else None
    tq.tq_quantize_kv(Kb[:, :, T_len - 1:T_len].contiguous().cuda(), Vb[:, :, T_len - 1:T_len].contiguous().cuda(),
                      cache, T_len - 1)
    out = torch.empty(B, Hq, d, device="cuda")
    ws = tq.workspace(tq.tq_decode_workspace_bytes(cache, Hq, T_len))
    tq.tq_decode_attention(q.cuda(), cache, T_len, d ** -0.5, out, ws)
    torch.cuda.synchronize()
    k_recs = P.oracle_records(P.to_np(Kb[:, :, :T_len]), kb, km, 6, 3, m or None)
    v_recs = P.oracle_records(P.to_np(Vb[:, :, :T_len]), vb, vm, 6, 3, m or None)
    want = P.oracle_decode(P.to_np(q), k_recs, v_recs, B, Hkv, d ** -0.5)
    P.assert_attention_close(P.to_np(out), want)


@pytest.mark.parametrize("q_dtype", [torch.bfloat16, torch.float32])
def test_decode_zero_query_head_attends_uniformly(q_dtype):
    # an all-zero query has no fixed-point scale: its scores are all zero (uniform weights)
    # while the other heads of the same KV head decode normally; so has a query of subnormal
    # size (exact scores below 1e-30)
    case = (128, 4, 2, (4, O.MSE), (2, O.MSE), 0, 333, 333)
    B, Hq, K, V, q = _decode_case(case, q_dtype, seed=12)
    q[0, 1] = 0.0
    q[1, 6] = 0.0
    q[1, 5] = (q[1, 5].float() * 1e-39).to(q_dtype)
    cache = tq.TQCache(B, 2, 333, 128, 4, 2)
    k_recs = P.oracle_records(P.to_np(K), 4, O.MSE, 0, 1, None)
    v_recs = P.oracle_records(P.to_np(V), 2, O.MSE, 0, 1, None)
    P.upload(cache, "k", k_recs)
    P.upload(cache, "v", v_recs)
    out = torch.empty(B, Hq, 128, device="cuda")
    ws = tq.workspace(tq.tq_decode_workspace_bytes(cache, Hq, 333))
    tq.tq_decode_attention(q.cuda(), cache, 333, 128 ** -0.5, out, ws)
    torch.cuda.synchronize()
    want = P.oracle_decode(P.to_np(q), k_recs, v_recs, B, 2, 128 ** -0.5)
    P.assert_attention_close(P.to_np(out), want)
    vh = O.dequantize(v_recs[0])
    np.testing.assert_allclose(want[0, 1], vh.mean(axis=0), rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("case", [
    (128, 4, 2, (4, O.MSE), (2, O.MSE), 0, 333, 333),    # tensor-core MSE kernel
    (128, 8, 1, (3, O.MSE), (3, O.MSE), 0, 200, 200),    # tensor-core MSE kernel, two n-tiles
    (256, 2, 2, (4, O.MSE), (2, O.MSE), 0, 150, 150),    # generic split-K kernel
    (64, 1, 3, (2, O.PROD), (2, O.PROD), 64, 140, 140),  # TurboQuant_prod, one head per KV head
    (64, 2, 2, (2, O.PROD), (2, O.PROD), 64, 140, 140),  # TurboQuant_prod, two heads per KV head
], ids=lambda c: f"d{c[0]}-G{c[1]}-k{c[3]}-v{c[4]}")
def test_decode_non_finite_query_heads_give_nan(case):
    # a query head holding a NaN or an infinity has NaN scores in exact arithmetic, so its
    # attention output is NaN; the other heads of the same KV head decode as usual
    d, G, Hkv, (kb, km), (vb, vm), m, T, _ = case
    B, Hq, K, V, q = _decode_case(case, torch.bfloat16, seed=14)
    bad = [(0, 0), (1, Hq - 1)]
    q[0, 0, 3] = float("nan")
    q[1, Hq - 1, 7] = float("inf")
    cache = tq.TQCache(B, Hkv, T, d, kb, vb, km, vm, m, m, seed=4, qjl_seed=2)
    k_recs = P.oracle_records(P.to_np(K), kb, km, 4, 2, m or None)
    v_recs = P.oracle_records(P.to_np(V), vb, vm, 4, 2, m or None)
    P.upload(cache, "k", k_recs)
    P.upload(cache, "v", v_recs)
    out = torch.empty(B, Hq, d, device="cuda")
    ws = tq.workspace(tq.tq_decode_workspace_bytes(cache, Hq, T))
    tq.tq_decode_attention(q.cuda(), cache, T, d ** -0.5, out, ws)
    torch.cuda.synchronize()
    got = P.to_np(out)
    qf = P.to_np(q)
    for b, h in bad:
        assert np.isnan(got[b, h]).all(), f"head ({b},{h}) should be NaN"
        qf[b, h] = 0.0  # the oracle's answer for the finite heads does not depend on these
    want = P.oracle_decode(qf, k_recs, v_recs, B, Hkv, d ** -0.5)
    for b in range(B):
        for h in range(Hq):
            if (b, h) not in bad:
                assert np.isfinite(got[b, h]).all()
                assert P.rel_l2(got[b, h], want[b, h]) <= P.ATTN_RTOL, (b, h)


def test_bf16_decode_non_finite_query_heads_give_nan():
    for d, G, Hkv in ((128, 4, 2), (64, 1, 3)):
        B, T = 2, 260
        Hq = G * Hkv
        K, V = random_kv(B, Hkv, T, d, dtype=torch.bfloat16, seed=d)
        q = torch.randn(B, Hq, d, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
        q[0, 1, 0] = float("nan")
        q[1, 0, 5] = float("-inf")
        out = torch.empty(B, Hq, d, device="cuda")
        ws = tq.workspace(tq.tq_decode_bf16_workspace_bytes(B, Hq, Hkv, T, d))
        tq.tq_decode_attention_bf16(q.cuda(), K.cuda(), V.cuda(), T, d ** -0.5, out, ws)
        torch.cuda.synchronize()
        got = P.to_np(out)
        qf = P.to_np(q)
        for b, h in ((0, 1), (1, 0)):
            assert np.isnan(got[b, h]).all()
            qf[b, h] = 0.0
        want = O.gqa_decode(qf, P.to_np(K), P.to_np(V), d ** -0.5)
        for b in range(B):
            for h in range(Hq):
                if (b, h) not in ((0, 1), (1, 0)):
                    assert P.rel_l2(got[b, h], want[b, h]) <= P.ATTN_RTOL


def test_decode_rejects_small_workspace_and_empty_context():
    cache = tq.TQCache(1, 1, 64, 128, 4, 2)
    q = torch.zeros(1, 4, 128, device="cuda", dtype=torch.bfloat16)
    out = torch.empty(1, 4, 128, device="cuda")
    need = tq.tq_decode_workspace_bytes(cache, 4, 64)
    small = tq.workspace(need - 64)
    with pytest.raises(tq.TQError) as e:
        tq.tq_decode_attention(q, cache, 64, 0.1, out, small[: (need - 64) // 4 - 8])
    assert e.value.status == tq.TQ_ERR_WORKSPACE
    with pytest.raises(tq.TQError) as e:
        tq.tq_decode_attention(q, cache, 0, 0.1, out, tq.workspace(need))
    assert e.value.status == tq.TQ_ERR_INVALID_ARG


# ------------------------------------------------------------------ bf16 comparator
@pytest.mark.parametrize("d,G,Hkv,T_len,T_cap", [(128, 4, 2, 1000, 1024), (64, 1, 3, 129, 140),
                                                  (256, 8, 1, 300, 300), (16, 2, 2, 1, 4),
                                                  (128, 8, 1, 777, 800), (128, 1, 3, 33, 40),
                                                  (128, 3, 2, 1, 5), (128, 16, 1, 100, 100)])
def test_bf16_decode_matches_oracle(d, G, Hkv, T_len, T_cap):
    B, Hq = 2, G * Hkv
    K, V = _inputs(B, Hkv, T_cap, d, torch.bfloat16, seed=d + G, outliers=True)
    q = torch.randn(B, Hq, d, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    out = torch.empty(B, Hq, d, device="cuda")
    ws = tq.workspace(tq.tq_decode_bf16_workspace_bytes(B, Hq, Hkv, T_len, d))
    tq.tq_decode_attention_bf16(q.cuda(), K.cuda(), V.cuda(), T_len, d ** -0.5, out, ws)
    torch.cuda.synchronize()
    want = O.gqa_decode(P.to_np(q), P.to_np(K)[:, :, :T_len], P.to_np(V)[:, :, :T_len], d ** -0.5)
    P.assert_attention_close(P.to_np(out), want)


@pytest.mark.parametrize("d,kcfg,vcfg,m,dtype", [
    (128, (4, O.MSE), (2, O.MSE), 0, torch.bfloat16),   # tensor-core Hadamard, 16-vector groups
    (128, (3, O.MSE), (2, O.MSE), 0, torch.float16),
    (64, (3, O.MSE), (1, O.MSE), 0, torch.bfloat16),    # streaming quantiser, 128-vector batches
    (64, (2, O.PROD), (2, O.PROD), 64, torch.bfloat16),  # tcgen05 sketch quantiser, 128-vector tiles
    (64, (1, O.PROD), (2, O.PROD), 64, torch.bfloat16),
    (64, (2, O.PROD), (1, O.PROD), 64, torch.float16),
])
def test_bulk_quantize_with_ragged_batches_and_offset(d, kcfg, vcfg, m, dtype):
    # 3 x 7 x 1000 = 21000 vectors per tensor: above the few-token path, and neither a whole
    # number of 128-vector batches or tiles nor of 16-vector groups; written at offset 5 of
    # T_cap 1010
    B, Hkv, T, T_cap, t_off = 3, 7, 1000, 1010, 5
    (kb, km), (vb, vm) = kcfg, vcfg
    K, V = _inputs(B, Hkv, T, d, dtype, seed=d + kb + vb, outliers=True, zero_at=17)
    cache = tq.TQCache(B, Hkv, T_cap, d, kb, vb, km, vm, m, m, seed=13, qjl_seed=7)
    tq.tq_quantize_kv(K.cuda(), V.cuda(), cache, t_offset=t_off)
    torch.cuda.synchronize()
    heads = [(0, 0), (1, 3), (2, 6)]  # includes the last (b, KV head): the ragged end
    for side, X, bits, mode in (("k", K, kb, km), ("v", V, vb, vm)):
        Xn = P.to_np(X)
        recs = [P.oracle_records(Xn[b:b + 1, h:h + 1], bits, mode, 13, 7, m or None)[0] for b, h in heads]
        P.compare_records(cache, side, recs, t_offset=t_off, heads=heads)
    assert int(cache["k_norm"][:, :, :t_off].abs().sum()) == 0
    assert int(cache["v_norm"][:, :, t_off + T:].abs().sum()) == 0
    assert tq.tq_device_faults() == 0


@pytest.mark.parametrize("d,kcfg,vcfg,m", [
    (128, (4, O.MSE), (2, O.MSE), 0),        # tensor-core writer, 16-vector groups
    (64, (2, O.PROD), (1, O.PROD), 64),      # tcgen05 writer, 128-vector tiles
])
def test_bulk_quantize_short_context_wraps_records(d, kcfg, vcfg, m):
    # T = 5 < 16: one 16-vector group spans several (batch, KV head) slices, so the record
    # index wraps inside a group; 600 x 8 x 5 = 24000 vectors per tensor keeps the bulk kernels
    B, Hkv, T, T_cap, t_off = 600, 8, 5, 9, 3
    (kb, km), (vb, vm) = kcfg, vcfg
    K, V = _inputs(B, Hkv, T, d, torch.bfloat16, seed=77 + d, outliers=True)
    cache = tq.TQCache(B, Hkv, T_cap, d, kb, vb, km, vm, m, m, seed=17, qjl_seed=9)
    tq.tq_quantize_kv(K.cuda(), V.cuda(), cache, t_offset=t_off)
    torch.cuda.synchronize()
    heads = [(0, 0), (0, 7), (1, 2), (299, 4), (599, 7)]
    for side, X, bits, mode in (("k", K, kb, km), ("v", V, vb, vm)):
        Xn = P.to_np(X)
        recs = [P.oracle_records(Xn[b:b + 1, h:h + 1], bits, mode, 17, 9, m or None)[0] for b, h in heads]
        P.compare_records(cache, side, recs, t_offset=t_off, heads=heads)
    assert int(cache["k_norm"][:, :, :t_off].abs().sum()) == 0
    assert int(cache["v_norm"][:, :, t_off + T:].abs().sum()) == 0
    assert tq.tq_device_faults() == 0
