"""The decode step (quantise the new token, decode over the cache) captured in a CUDA graph
through the public API and replayed: a serving loop launches it without host work per kernel.
The replay must write the same records and outputs as eager calls."""
import math

import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from quantized_decode_attention_kv_b200 import tq  # noqa: E402
from quantized_decode_attention_kv_b200.workloads import random_kv  # noqa: E402


@pytest.mark.parametrize("d,G,Hkv,kcfg,vcfg,m,T", [
    (128, 4, 2, (4, tq.TQ_MSE), (2, tq.TQ_MSE), 0, 700),
    (64, 1, 3, (2, tq.TQ_PROD), (2, tq.TQ_PROD), 64, 300),
])
def test_decode_step_replays_from_a_cuda_graph(d, G, Hkv, kcfg, vcfg, m, T):
    B, Hq = 2, G * Hkv
    K, V = random_kv(B, Hkv, T, d, dtype=torch.bfloat16, seed=T)
    K, V = K.cuda(), V.cuda()
    q = torch.randn(B, Hq, d, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).cuda()
    scale = 1.0 / math.sqrt(d)
    eager = tq.TQCache(B, Hkv, T, d, kcfg[0], vcfg[0], kcfg[1], vcfg[1], m, m)
    graphed = tq.TQCache(B, Hkv, T, d, kcfg[0], vcfg[0], kcfg[1], vcfg[1], m, m)
    for c in (eager, graphed):
        tq.tq_quantize_kv(K[:, :, : T - 1].contiguous(), V[:, :, : T - 1].contiguous(), c)
    k_new = K[:, :, T - 1:].contiguous()
    v_new = V[:, :, T - 1:].contiguous()
    out_e = torch.empty(B, Hq, d, device="cuda")
    out_g = torch.full((B, Hq, d), float("nan"), device="cuda")
    ws_e = tq.workspace(tq.tq_decode_workspace_bytes(eager, Hq, T))
    ws_g = tq.workspace(tq.tq_decode_workspace_bytes(graphed, Hq, T))

    tq.tq_quantize_kv(k_new, v_new, eager, t_offset=T - 1)
    tq.tq_decode_attention(q, eager, T, scale, out_e, ws_e)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm up on the capture stream's side, as torch requires
        tq.tq_quantize_kv(k_new, v_new, graphed, t_offset=T - 1)
        tq.tq_decode_attention(q, graphed, T, scale, out_g, ws_g)
    torch.cuda.current_stream().wait_stream(side)
    out_g.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        tq.tq_quantize_kv(k_new, v_new, graphed, t_offset=T - 1)
        tq.tq_decode_attention(q, graphed, T, scale, out_g, ws_g)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.isfinite(out_g).all()
    # equal to fp32 rounding (the TurboQuant_prod merge adds warps' partials with shared-memory
    # atomics, whose order is not fixed)
    torch.testing.assert_close(out_g, out_e, rtol=1e-5, atol=1e-6)
    for key in ("k_codes", "v_codes", "k_norm", "v_norm"):
        assert torch.equal(graphed[key], eager[key]), key


def test_ragged_and_paged_decode_replay_from_a_cuda_graph():
    # per-sequence lengths travel as launch parameters: the graph keeps the captured lengths
    B, Hkv, G, d, T, page = 3, 2, 4, 128, 640, 64
    Hq, lens = G * Hkv, [640, 17, 300]
    K, V = random_kv(B, Hkv, T, d, dtype=torch.bfloat16, seed=11)
    K, V = K.cuda(), V.cuda()
    q = torch.randn(B, Hq, d, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).cuda()
    dense = tq.TQCache(B, Hkv, T, d, 4, 2)
    tq.tq_quantize_kv(K, V, dense)
    maxp = T // page
    bt = torch.randperm(B * maxp, generator=torch.Generator().manual_seed(2)).to(torch.int32)
    paged = tq.TQPagedCache(B, Hkv, d, page, B * maxp, maxp, 4, 2, bt.reshape(B, maxp).cuda())
    tq.tq_quantize_kv_paged(K, V, paged)
    ws_r = tq.workspace(tq.tq_decode_varlen_workspace_bytes(dense, Hq, lens))
    ws_p = tq.workspace(tq.tq_decode_paged_workspace_bytes(paged, Hq, lens))
    eager_r, eager_p = torch.empty(B, Hq, d, device="cuda"), torch.empty(B, Hq, d, device="cuda")
    tq.tq_decode_attention_varlen(q, dense, lens, 0.1, eager_r, ws_r)
    tq.tq_decode_attention_paged(q, paged, lens, 0.1, eager_p, ws_p)
    out_r = torch.full((B, Hq, d), float("nan"), device="cuda")
    out_p = torch.full((B, Hq, d), float("nan"), device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        tq.tq_decode_attention_varlen(q, dense, lens, 0.1, out_r, ws_r)
        tq.tq_decode_attention_paged(q, paged, lens, 0.1, out_p, ws_p)
    torch.cuda.current_stream().wait_stream(side)
    out_r.fill_(float("nan"))
    out_p.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        tq.tq_decode_attention_varlen(q, dense, lens, 0.1, out_r, ws_r)
        tq.tq_decode_attention_paged(q, paged, lens, 0.1, out_p, ws_p)
    lens[1] = 600  # the host array may change after capture: the graph keeps its values
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    torch.testing.assert_close(out_r, eager_r, rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(out_p, eager_p, rtol=1e-5, atol=1e-6)
