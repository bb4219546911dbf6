"""GPU parity of TurboQuant_mse records on the E2M1 (Blackwell FP4) grid: the library's writers
put the same codes as the oracle (bit-exact away from boundaries), and decode and prefill over
E2M1 keys match the oracle's attention over the dequantised cache ("Where This Fits in the
Inference Stack", Blackwell FP4)."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from quantized_decode_attention_kv_b200 import tq  # noqa: E402
from quantized_decode_attention_kv_b200.workloads import random_kv  # noqa: E402


@pytest.mark.parametrize("d,B,Hkv,T,dtype", [
    (128, 2, 4, 300, torch.bfloat16),  # bulk write
    (128, 3, 2, 1, torch.float16),     # one new token
    (64, 2, 3, 77, torch.float32),
])
def test_e2m1_write_matches_oracle(d, B, Hkv, T, dtype):
    K, V = random_kv(B, Hkv, T, d, dtype=torch.float32, seed=T + d)
    K[..., :3] *= 20.0
    Kd, Vd = K.to(dtype), V.to(dtype)
    cache = tq.TQCache(B, Hkv, T + 5, d, 4, 2, tq.TQ_E2M1, tq.TQ_MSE, seed=11)
    tq.tq_quantize_kv(Kd.cuda(), Vd.cuda(), cache, 2)
    torch.cuda.synchronize()
    k_recs = P.oracle_records(P.to_np(Kd), 4, O.E2M1, 11, 1, None)
    v_recs = P.oracle_records(P.to_np(Vd), 2, O.MSE, 11, 1, None)
    P.compare_records(cache, "k", k_recs, t_offset=2)
    P.compare_records(cache, "v", v_recs, t_offset=2)


@pytest.mark.parametrize("d,G,Hkv,vb,T", [
    (128, 4, 2, 2, 700),   # tensor-core decode
    (128, 8, 1, 3, 333),
    (128, 16, 1, 2, 200),  # more query heads per KV head than the tensor-core kernel takes
    (64, 2, 2, 4, 129),
])
def test_e2m1_decode_matches_oracle(d, G, Hkv, vb, T):
    B, Hq = 2, G * Hkv
    K, V = random_kv(B, Hkv, T, d, dtype=torch.float32, seed=T)
    K[..., :3] *= 50.0  # keys at 50x the values' norm
    q = torch.randn(B, Hq, d, generator=torch.Generator().manual_seed(T)).to(torch.bfloat16)
    cache = tq.TQCache(B, Hkv, T, d, 4, vb, tq.TQ_E2M1, tq.TQ_MSE, seed=7)
    k_recs = P.oracle_records(P.to_np(K), 4, O.E2M1, 7, 1, None)
    v_recs = P.oracle_records(P.to_np(V), vb, O.MSE, 7, 1, None)
    P.upload(cache, "k", k_recs)
    P.upload(cache, "v", v_recs)
    out = torch.empty(B, Hq, d, device="cuda")
    ws = tq.workspace(tq.tq_decode_workspace_bytes(cache, Hq, T))
    tq.tq_decode_attention(q.cuda(), cache, T, d ** -0.5, out, ws)
    torch.cuda.synchronize()
    want = P.oracle_decode(P.to_np(q), k_recs, v_recs, B, Hkv, d ** -0.5)
    P.assert_attention_close(P.to_np(out), want)


@pytest.mark.parametrize("G,vb,Lq,t0,k_scale", [
    (4, 2, 200, 150, 20.0),
    (4, 2, 64, 0, 1.0),      # one tile, causal inside the chunk
    (4, 3, 1, 500, 1.0),     # a single query: a decode step
    (8, 4, 300, 130, 1.0),   # eight query heads per KV head
    (2, 2, 128, 1000, 50.0), # keys at 50x the values' norm: near one-hot rows
    (1, 3, 300, 64, 1.0),
])
def test_e2m1_prefill_matches_oracle(G, vb, Lq, t0, k_scale):
    # E2M1 keys enter the score MMAs as E2M1 operands (kind::f8f6f4) against the query in four
    # E4M3 parts
    B, Hkv = 2, 2
    Hq, T = G * Hkv, t0 + Lq
    K, V = random_kv(B, Hkv, T, 128, dtype=torch.float32, seed=9 + G + t0, scale=k_scale)
    K[..., :3] *= 20.0 if k_scale == 1.0 else 1.0
    q = torch.randn(B, Lq, Hq, 128, generator=torch.Generator().manual_seed(10 + Lq)).to(torch.bfloat16)
    cache = tq.TQCache(B, Hkv, T, 128, 4, vb, tq.TQ_E2M1, tq.TQ_MSE, seed=5)
    k_recs = P.oracle_records(P.to_np(K), 4, O.E2M1, 5, 1, None)
    v_recs = P.oracle_records(P.to_np(V), vb, O.MSE, 5, 1, None)
    P.upload(cache, "k", k_recs)
    P.upload(cache, "v", v_recs)
    out = torch.empty(B, Lq, Hq, 128, device="cuda")
    tq.tq_prefill_attention(q.cuda(), cache, t0, 128 ** -0.5, out)
    torch.cuda.synchronize()
    assert tq.tq_device_faults() == 0
    want = O.prefill_compressed(P.to_np(q), k_recs, v_recs, B, Hkv, t0, 128 ** -0.5)
    P.assert_attention_close(P.to_np(out).reshape(B * Lq, Hq, 128), want.reshape(B * Lq, Hq, 128))


def test_e2m1_prefill_last_query_equals_decode_over_device_written_records():
    B, Hkv, G, t0, Lq = 2, 2, 4, 333, 200
    Hq, T = G * Hkv, t0 + Lq
    K, V = random_kv(B, Hkv, T, 128, dtype=torch.bfloat16, seed=14)
    cache = tq.TQCache(B, Hkv, T, 128, 4, 2, tq.TQ_E2M1, tq.TQ_MSE, seed=3)
    tq.tq_quantize_kv(K.contiguous().cuda(), V.contiguous().cuda(), cache, 0)
    q = torch.randn(B, Lq, Hq, 128, generator=torch.Generator().manual_seed(15)).to(torch.bfloat16).cuda()
    out = torch.empty(B, Lq, Hq, 128, device="cuda")
    tq.tq_prefill_attention(q, cache, t0, 128 ** -0.5, out)
    dec = torch.empty(B, Hq, 128, device="cuda")
    ws = tq.workspace(tq.tq_decode_workspace_bytes(cache, Hq, T))
    tq.tq_decode_attention(q[:, -1].contiguous(), cache, T, 128 ** -0.5, dec, ws)
    torch.cuda.synchronize()
    assert tq.tq_device_faults() == 0
    P.assert_attention_close(P.to_np(out[:, -1]), P.to_np(dec))


def test_e2m1_keys_cost_more_attention_error_than_lloyd_max_keys():
    # the measured price of the FP4 grid: attention over E2M1 keys vs exact attention, against
    # the same with 4-bit Lloyd-Max keys (values fp32 exact in both), on the GPU decode
    B, Hkv, G, T, d = 4, 2, 4, 2048, 128
    K, V = random_kv(B, Hkv, T, d, dtype=torch.float32, seed=3)
    q = torch.randn(B, G * Hkv, d, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    exact = O.gqa_decode(P.to_np(q), P.to_np(K), P.to_np(V), d ** -0.5)
    errs = {}
    for mode in (tq.TQ_MSE, tq.TQ_E2M1):
        cache = tq.TQCache(B, Hkv, T, d, 4, 4, mode, tq.TQ_MSE, seed=2)
        tq.tq_quantize_kv(K.cuda(), V.cuda(), cache)
        out = torch.empty(B, G * Hkv, d, device="cuda")
        ws = tq.workspace(tq.tq_decode_workspace_bytes(cache, G * Hkv, T))
        tq.tq_decode_attention(q.cuda(), cache, T, d ** -0.5, out, ws)
        torch.cuda.synchronize()
        errs[mode] = P.rel_l2(P.to_np(out), exact)
    assert errs[tq.TQ_E2M1] > errs[tq.TQ_MSE]
