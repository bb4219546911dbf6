"""GPU parity of the prefill (chunked) attention over the compressed cache: the tcgen05 kernel,
called through the C ABI, against the oracle's causal chunk attention over the dequantised
cache ("Where This Fits in the Inference Stack", Decode Throughput vs. Time to First Token)."""
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


def _case(B, Hkv, G, T_cap, k_scale, seed, q_dtype=torch.bfloat16):
    K, V = random_kv(B, Hkv, T_cap, 128, dtype=torch.float32, seed=seed, scale=k_scale)
    K[..., :3] *= 20.0 if k_scale == 1.0 else 1.0
    return K, V


def _check(got, want):
    B, Lq, Hq, d = want.shape
    P.assert_attention_close(got.reshape(B * Lq, Hq, d), want.reshape(B * Lq, Hq, d))


@pytest.mark.parametrize("G,kb,vb,Lq,t0,k_scale", [
    (4, 4, 2, 64, 0, 1.0),       # one full tile of the chunk itself
    (4, 4, 2, 300, 0, 1.0),      # several query blocks and KV tiles, causal inside the chunk
    (4, 4, 2, 1, 777, 1.0),      # a single query: a decode step
    (4, 3, 3, 128, 200, 1.0),    # 3-bit keys and values, prefix + chunk
    (8, 4, 2, 300, 130, 1.0),    # eight query heads per KV head (16 positions per block)
    (8, 3, 3, 64, 1000, 50.0),   # keys at 50x the values' norm: near one-hot rows
    (4, 4, 3, 128, 1, 50.0),
    (2, 4, 4, 300, 64, 1.0),     # two heads per KV head, 4-bit values
    (1, 3, 2, 128, 500, 1.0),    # one head per KV head
])
def test_prefill_over_oracle_records_matches_oracle(G, kb, vb, Lq, t0, k_scale):
    B, Hkv = 2, 2
    Hq = G * Hkv
    T = t0 + Lq
    T_cap = T + 9
    K, V = _case(B, Hkv, G, T_cap, k_scale, seed=Lq + t0 + G)
    q = torch.randn(B, Lq, Hq, 128, generator=torch.Generator().manual_seed(t0 + 1)).to(torch.bfloat16)
    cache = tq.TQCache(B, Hkv, T_cap, 128, kb, vb, seed=9)
    k_recs = P.oracle_records(P.to_np(K[:, :, :T]), kb, O.MSE, 9, 1, None)
    v_recs = P.oracle_records(P.to_np(V[:, :, :T]), vb, O.MSE, 9, 1, None)
    P.upload(cache, "k", k_recs)
    P.upload(cache, "v", v_recs)
    out = torch.full((B, Lq, Hq, 128), float("nan"), device="cuda")
    tq.tq_prefill_attention(q.cuda(), cache, t0, 128 ** -0.5, out)
    torch.cuda.synchronize()
    assert tq.tq_device_faults() == 0
    want = O.prefill_compressed(P.to_np(q), k_recs, v_recs, B, Hkv, t0, 128 ** -0.5)
    _check(P.to_np(out), want)


def test_prefill_after_device_write_and_last_query_equals_decode():
    # the chunk is written by the library's quantiser (prefix first, then the chunk), the
    # prefill of the chunk matches the oracle over the device's own records, and its last query
    # equals a decode call over the same cache
    B, Hkv, G, t0, Lq = 2, 2, 4, 333, 200
    Hq, T = G * Hkv, t0 + Lq
    K, V = random_kv(B, Hkv, T, 128, dtype=torch.bfloat16, seed=4)
    cache = tq.TQCache(B, Hkv, T, 128, 4, 2, seed=3)
    tq.tq_quantize_kv(K[:, :, :t0].contiguous().cuda(), V[:, :, :t0].contiguous().cuda(), cache, 0)
    tq.tq_quantize_kv(K[:, :, t0:].contiguous().cuda(), V[:, :, t0:].contiguous().cuda(), cache, t0)
    q = torch.randn(B, Lq, Hq, 128, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).cuda()
    out = torch.empty(B, Lq, Hq, 128, device="cuda")
    tq.tq_prefill_attention(q, cache, t0, 128 ** -0.5, out)
    dec = torch.empty(B, Hq, 128, device="cuda")
    ws = tq.workspace(tq.tq_decode_workspace_bytes(cache, Hq, T))
    tq.tq_decode_attention(q[:, -1].contiguous(), cache, T, 128 ** -0.5, dec, ws)
    torch.cuda.synchronize()
    P.assert_attention_close(P.to_np(out[:, -1]), P.to_np(dec))
    recs = {}
    for side, bits in (("k", 4), ("v", 2)):
        codes = cache[f"{side}_codes"].cpu().numpy()
        norms = cache[f"{side}_norm"].cpu().numpy().view(np.float16)
        recs[side] = [O.records_from_packed(bits, O.MSE, 128, codes[b, h], norms[b, h], seed=3)
                      for b in range(B) for h in range(Hkv)]
    want = O.prefill_compressed(P.to_np(q), recs["k"], recs["v"], B, Hkv, t0, 128 ** -0.5)
    _check(P.to_np(out), want)


def test_prefill_rejects_unsupported_configurations():
    q = torch.zeros(1, 4, 4, 128, device="cuda", dtype=torch.bfloat16)
    out = torch.zeros(1, 4, 4, 128, device="cuda")
    for kb, vb, km in ((2, 2, tq.TQ_MSE), (4, 2, tq.TQ_PROD), (4, 1, tq.TQ_MSE)):
        cache = tq.TQCache(1, 1, 16, 128, kb, vb, km)
        with pytest.raises(tq.TQError) as e:
            tq.tq_prefill_attention(q, cache, 0, 0.1, out)
        assert e.value.status == tq.TQ_ERR_UNSUPPORTED
    cache = tq.TQCache(1, 1, 16, 128, 4, 2)
    with pytest.raises(tq.TQError) as e:
        tq.tq_prefill_attention(q, cache, 13, 0.1, out)  # t0 + Lq > T_cap
    assert e.value.status == tq.TQ_ERR_INVALID_ARG
    q3 = torch.zeros(1, 4, 3, 128, device="cuda", dtype=torch.bfloat16)  # 3 heads per KV head
    out3 = torch.zeros(1, 4, 3, 128, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_prefill_attention(q3, cache, 0, 0.1, out3)
    assert e.value.status == tq.TQ_ERR_UNSUPPORTED
    assert int(out.abs().sum()) == 0
