"""GPU parity of the ragged decode call: sequence b attends to its first T_lens[b] cached
positions. Checked against the oracle sequence by sequence, through the C ABI."""
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

CASES = [
    # d, G, Hkv, k(bits, mode), v(bits, mode), T_lens, T_cap
    (128, 4, 2, (4, O.MSE), (2, O.MSE), [1, 700, 16, 33, 1024, 257], 1024),  # 12-warp CTAs
    (128, 8, 1, (4, O.MSE), (2, O.MSE), [500, 3, 64, 1000], 1000),           # 8 query heads
    (128, 2, 3, (3, O.MSE), (3, O.MSE), [129, 2, 600], 640),                  # 4-warp CTAs
    # TurboQuant_prod, d = 64, 64 sketch rows: one query head per KV head (byte-table scores)
    # and two (tensor-core scores)
    (64, 1, 3, (2, O.PROD), (2, O.PROD), [1, 520, 17, 64, 300], 520),
    (64, 2, 2, (2, O.PROD), (2, O.PROD), [333, 5, 129, 2, 400, 48], 400),
]


def _setup(d, G, Hkv, kcfg, vcfg, T_lens, T_cap, seed):
    (kb, km), (vb, vm) = kcfg, vcfg
    B, Hq = len(T_lens), G * Hkv
    K, V = random_kv(B, Hkv, T_cap, d, dtype=torch.float32, seed=seed)
    K[..., :3] *= 20.0
    g = torch.Generator().manual_seed(seed + 1)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    cache = tq.TQCache(B, Hkv, T_cap, d, kb, vb, km, vm, 0, 0, seed=31, qjl_seed=3)
    k_recs = P.oracle_records(P.to_np(K), kb, km, 31, 3, None)
    v_recs = P.oracle_records(P.to_np(V), vb, vm, 31, 3, None)
    P.upload(cache, "k", k_recs)
    P.upload(cache, "v", v_recs)
    return B, Hq, q, cache, k_recs, v_recs


def _check_sequences(out, q, k_recs, v_recs, T_lens, Hkv, scale, seqs):
    qn, on = P.to_np(q), P.to_np(out)
    for b in seqs:
        want = P.oracle_decode(qn[b:b + 1], k_recs[b * Hkv:(b + 1) * Hkv], v_recs[b * Hkv:(b + 1) * Hkv],
                               1, Hkv, scale, T_lens[b])
        P.assert_attention_close(on[b:b + 1], want)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"G{c[1]}-H{c[2]}-k{c[3][0]}-v{c[4][0]}-B{len(c[5])}")
def test_varlen_decode_matches_oracle(case):
    d, G, Hkv, kcfg, vcfg, T_lens, T_cap = case
    B, Hq, q, cache, k_recs, v_recs = _setup(d, G, Hkv, kcfg, vcfg, T_lens, T_cap, seed=5 + G)
    scale = 1.0 / math.sqrt(d)
    out = torch.empty(B, Hq, d, device="cuda")
    ws = tq.workspace(tq.tq_decode_varlen_workspace_bytes(cache, Hq, T_lens))
    tq.tq_decode_attention_varlen(q.cuda(), cache, T_lens, scale, out, ws)
    torch.cuda.synchronize()
    _check_sequences(out, q, k_recs, v_recs, T_lens, Hkv, scale, range(B))


def test_varlen_many_short_sequences():
    # 300 sequences of 1..200 tokens: many (sequence, KV head) segments per CTA
    rng = np.random.default_rng(3)
    T_lens = [int(t) for t in rng.integers(1, 201, size=300)]
    B, Hq, q, cache, k_recs, v_recs = _setup(128, 4, 1, (4, O.MSE), (2, O.MSE), T_lens, 200, seed=9)
    out = torch.empty(B, Hq, 128, device="cuda")
    ws = tq.workspace(tq.tq_decode_varlen_workspace_bytes(cache, Hq, T_lens))
    tq.tq_decode_attention_varlen(q.cuda(), cache, T_lens, 128 ** -0.5, out, ws)
    torch.cuda.synchronize()
    _check_sequences(out, q, k_recs, v_recs, T_lens, 1, 128 ** -0.5, [0, 1, 2, 57, 150, 298, 299])


def test_varlen_with_equal_lengths_equals_the_uniform_call():
    T_lens = [333] * 4
    B, Hq, q, cache, _, _ = _setup(128, 4, 2, (4, O.MSE), (2, O.MSE), T_lens, 400, seed=2)
    out_v = torch.empty(B, Hq, 128, device="cuda")
    out_u = torch.empty(B, Hq, 128, device="cuda")
    ws_v = tq.workspace(tq.tq_decode_varlen_workspace_bytes(cache, Hq, T_lens))
    ws_u = tq.workspace(tq.tq_decode_workspace_bytes(cache, Hq, 333))
    tq.tq_decode_attention_varlen(q.cuda(), cache, T_lens, 0.1, out_v, ws_v)
    tq.tq_decode_attention(q.cuda(), cache, 333, 0.1, out_u, ws_u)
    torch.cuda.synchronize()
    torch.testing.assert_close(out_v, out_u, rtol=1e-5, atol=1e-6)


def test_varlen_rejects_unsupported_configurations():
    cache = tq.TQCache(2, 2, 64, 64, 2, 2, O.PROD, O.PROD, 32, 32)  # 32 sketch rows
    with pytest.raises(tq.TQError) as e:
        tq.tq_decode_varlen_workspace_bytes(cache, 2, [10, 20])
    assert "tensor-core configuration" in str(e.value)


def test_varlen_prod_with_equal_lengths_equals_the_uniform_call():
    T_lens = [300] * 3
    B, Hq, q, cache, _, _ = _setup(64, 2, 2, (2, O.PROD), (2, O.PROD), T_lens, 320, seed=7)
    out_v = torch.empty(B, Hq, 64, device="cuda")
    out_u = torch.empty(B, Hq, 64, device="cuda")
    ws_v = tq.workspace(tq.tq_decode_varlen_workspace_bytes(cache, Hq, T_lens))
    ws_u = tq.workspace(tq.tq_decode_workspace_bytes(cache, Hq, 300))
    tq.tq_decode_attention_varlen(q.cuda(), cache, T_lens, 0.125, out_v, ws_v)
    tq.tq_decode_attention(q.cuda(), cache, 300, 0.125, out_u, ws_u)
    torch.cuda.synchronize()
    torch.testing.assert_close(out_v, out_u, rtol=1e-5, atol=1e-6)
