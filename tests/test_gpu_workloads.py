"""Full-size workloads on the GPU, in the launch configuration bench.py times: every
workload is quantised and decoded at its real size through the C ABI, and sampled
(batch, KV head) slices are checked against the oracle (codes, norms, and the attention of
that KV head's query heads over the full context)."""
import numpy as np
import pytest
import torch

import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from quantized_decode_attention_kv_b200 import tq  # noqa: E402
from quantized_decode_attention_kv_b200.workloads import WORKLOADS, make_inputs  # noqa: E402


def _cache_for(w):
    return tq.TQCache(w.B, w.Hkv, w.T, w.d, w.k_bits, w.v_bits, w.k_mode, w.v_mode, w.qjl_m,
                      w.qjl_m, seed=w.seed, qjl_seed=w.qjl_seed)


def _check_full(w, layer=0, samples=((0, 0), (-1, -1))):
    K, V, q = make_inputs(w, device="cuda", layer=layer)
    cache = _cache_for(w)
    tq.tq_quantize_kv(K, V, cache)
    out = torch.empty(w.B, w.Hq, w.d, device="cuda")
    ws = tq.workspace(tq.tq_decode_workspace_bytes(cache, w.Hq, w.T))
    tq.tq_decode_attention(q, cache, w.T, w.scale, out, ws)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    G = w.G
    stats = []
    for b, h in samples:
        b %= w.B
        h %= w.Hkv
        recs = {}
        for side, X, bits, mode in (("k", K, w.k_bits, w.k_mode), ("v", V, w.v_bits, w.v_mode)):
            r = O.quantize(P.to_np(X[b, h]), bits, mode, seed=w.seed, qjl_seed=w.qjl_seed,
                           m=w.qjl_m or None)
            stats.append(P.compare_records(cache, side, [r], heads=[(b, h)]))
            recs[side] = r
        qs = P.to_np(q[b:b + 1, h * G:(h + 1) * G])
        want = O.decode_compressed(qs, [recs["k"]], [recs["v"]], 1, 1, w.scale)
        P.assert_attention_close(P.to_np(out[b:b + 1, h * G:(h + 1) * G]), want)
    del K, V, cache
    torch.cuda.empty_cache()
    return stats


@pytest.mark.parametrize("name", ["tiny_single_head_fp32", "llama3_8b_decode_32k", "gpt2_prod_2bit",
                                  "llama3_8b_128k_3bit", "llama70b_asym_16k", "llama3_8b_32k_3p5bit"])
def test_full_size_workload_sampled_parity(name):
    w = WORKLOADS[name]
    stats = _check_full(w)
    near = sum(s["near_boundary"] for s in stats)
    coords = sum(s["coords"] for s in stats)
    # the exemption band is 2e-5 wide around each boundary: for near-Gaussian z that is about
    # 2e-5 * sum_j pdf(beta_j) < 1e-4 of the coordinates
    assert near <= 3e-4 * coords


def test_full_size_bf16_boundary_layer():
    # layers kept unquantised in the 70B-shaped workload run the bf16 kernel at full size
    w = WORKLOADS["llama70b_asym_16k"]
    K, V, q = make_inputs(w, device="cuda", layer=0)
    out = torch.empty(w.B, w.Hq, w.d, device="cuda")
    ws = tq.workspace(tq.tq_decode_bf16_workspace_bytes(w.B, w.Hq, w.Hkv, w.T, w.d))
    tq.tq_decode_attention_bf16(q, K, V, w.T, w.scale, out, ws)
    torch.cuda.synchronize()
    G = w.G
    for b, h in ((0, 0), (w.B - 1, w.Hkv - 1)):
        want = O.gqa_decode(P.to_np(q[b:b + 1, h * G:(h + 1) * G]), P.to_np(K[b:b + 1, h:h + 1]),
                            P.to_np(V[b:b + 1, h:h + 1]), w.scale)
        P.assert_attention_close(P.to_np(out[b:b + 1, h * G:(h + 1) * G]), want)


@pytest.mark.parametrize("name,T,kmode", [
    ("llama3_8b_decode_32k", 65536, tq.TQ_MSE),    # the bench's 64K prefill chunk (K4/V2)
    ("llama3_8b_128k_3bit", 131072, tq.TQ_MSE),    # the bench's 128K prefill chunk (K3/V3)
    ("llama3_8b_decode_32k", 65536, tq.TQ_E2M1),   # 64K with keys on the E2M1 grid
])
def test_full_size_prefill_sampled_parity(name, T, kmode):
    # the chunk bench.py times: batch 4, 1024 queries at the end of the cache; sampled
    # (batch, KV head) slices: records against the oracle, and the first and last query rows of
    # the slice's query heads against the oracle's causal attention over its dequantised records
    import dataclasses
    w = dataclasses.replace(WORKLOADS[name], B=4, T=T)
    Lq, t0 = 1024, T - 1024
    K, V, _ = make_inputs(w, device="cuda")
    cache = tq.TQCache(w.B, w.Hkv, w.T, w.d, w.k_bits, w.v_bits, kmode, tq.TQ_MSE, seed=w.seed)
    tq.tq_quantize_kv(K, V, cache)
    q = torch.randn(w.B, Lq, w.Hq, w.d, generator=torch.Generator(device="cuda").manual_seed(77),
                    device="cuda").to(torch.bfloat16)
    out = torch.empty(w.B, Lq, w.Hq, w.d, device="cuda")
    tq.tq_prefill_attention(q, cache, t0, w.scale, out)
    torch.cuda.synchronize()
    assert tq.tq_device_faults() == 0
    G = w.G
    for b, h in ((0, 0), (w.B - 1, w.Hkv - 1)):
        recs = {}
        for side, X, bits, mode in (("k", K, w.k_bits, O.E2M1 if kmode == tq.TQ_E2M1 else O.MSE),
                                    ("v", V, w.v_bits, O.MSE)):
            r = O.quantize(P.to_np(X[b, h]), bits, mode, seed=w.seed)
            P.compare_records(cache, side, [r], heads=[(b, h)])
            recs[side] = r
        # the first and the last 8 query rows of the chunk (each block the oracle's own causal
        # chunk starting at its position)
        for i0 in (0, Lq - 8):
            qs = P.to_np(q[b:b + 1, i0:i0 + 8, h * G:(h + 1) * G])
            want = O.prefill_compressed(qs, [recs["k"]], [recs["v"]], 1, 1, t0 + i0, w.scale)
            got = P.to_np(out[b:b + 1, i0:i0 + 8, h * G:(h + 1) * G])
            P.assert_attention_close(got.reshape(8, G, w.d), want.reshape(8, G, w.d))
    del K, V, cache
    torch.cuda.empty_cache()


@pytest.mark.parametrize("page,ragged", [(64, False), (16, True), (32, True), (256, True)],
                         ids=["page64-full", "page16-ragged", "page32-ragged", "page256-ragged"])
def test_full_size_paged_decode_sampled_parity(page, ragged):
    # the bench's paged case (Llama-3.1-8B-shaped layer, batch 16, 32K context, pages scattered
    # over the pool by a seeded permutation) and ragged lengths in [T/4, T] at other page sizes:
    # every CTA walks many page chunks. The paged call must agree with the dense
    # per-sequence-length call on the same inputs (the two writers store the same records), and sampled
    # (batch, KV head) slices must match the oracle over their own lengths.
    w = WORKLOADS["llama3_8b_decode_32k"]
    K, V, q = make_inputs(w, device="cuda")
    if ragged:
        g = torch.Generator().manual_seed(99 + page)
        lens = torch.randint(w.T // 4, w.T + 1, (w.B,), generator=g).tolist()
    else:
        lens = [w.T] * w.B
    maxp = (w.T + page - 1) // page
    npages = w.B * maxp
    bt = torch.randperm(npages, generator=torch.Generator().manual_seed(4321)).to(torch.int32)
    pc = tq.TQPagedCache(w.B, w.Hkv, w.d, page, npages, maxp, w.k_bits, w.v_bits,
                         bt.reshape(w.B, maxp).cuda(), seed=w.seed)
    tq.tq_quantize_kv_paged(K, V, pc, 0)
    out = torch.empty(w.B, w.Hq, w.d, device="cuda")
    ws = tq.workspace(tq.tq_decode_paged_workspace_bytes(pc, w.Hq, lens))
    tq.tq_decode_attention_paged(q, pc, lens, w.scale, out, ws)
    dense = _cache_for(w)
    tq.tq_quantize_kv(K, V, dense)
    out_d = torch.empty_like(out)
    ws_d = tq.workspace(tq.tq_decode_varlen_workspace_bytes(dense, w.Hq, lens))
    tq.tq_decode_attention_varlen(q, dense, lens, w.scale, out_d, ws_d)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    # same records, another assignment of tiles to warps: only rounding differs (each warp's
    # softmax reference sets the fp16 rounding of its weights)
    P.assert_attention_close(P.to_np(out), P.to_np(out_d))
    G = w.G
    for b, h in ((0, 0), (w.B - 1, w.Hkv - 1)):
        T = lens[b]
        recs = {side: O.quantize(P.to_np(X[b, h, :T]), bits, O.MSE, seed=w.seed)
                for side, X, bits in (("k", K, w.k_bits), ("v", V, w.v_bits))}
        qs = P.to_np(q[b:b + 1, h * G:(h + 1) * G])
        want = O.decode_compressed(qs, [recs["k"]], [recs["v"]], 1, 1, w.scale)
        P.assert_attention_close(P.to_np(out[b:b + 1, h * G:(h + 1) * G]), want)
    del K, V, pc, dense, ws, ws_d
    torch.cuda.empty_cache()
