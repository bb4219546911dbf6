"""GPU parity of the paged cache: records at page block_table[b][t / page_size], head h, slot
t % page_size. Writes are checked byte for byte against dense writes of the same input and
against the oracle; decode against the oracle per sequence, through the C ABI."""
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


def _block_table(B, max_pages, num_pages, seed):
    """Each sequence gets max_pages distinct pages, scattered over the pool."""
    perm = np.random.default_rng(seed).permutation(num_pages)[: B * max_pages]
    return torch.from_numpy(perm.reshape(B, max_pages).astype(np.int32)).cuda()


class _DenseView:
    """The paged pools gathered into the dense [B][Hkv][T][...] layout (what compare_records reads)."""

    def __init__(self, cache: tq.TQPagedCache, T: int):
        bt = cache.block_table.cpu().numpy()
        t = np.arange(T)
        pages = bt[:, t // cache.page_size].astype(np.int64)  # [B][T]
        slots = np.broadcast_to(t % cache.page_size, pages.shape).astype(np.int64)
        self.Hkv = cache.Hkv
        self.tensors = {}
        for key in ("k_codes", "v_codes", "k_norm", "v_norm", "k_signs", "v_signs", "k_rnorm", "v_rnorm"):
            if cache[key] is None:
                self.tensors[key] = None
                continue
            pool = cache[key].cpu()
            g = pool[torch.from_numpy(pages)[:, None, :], torch.arange(cache.Hkv)[None, :, None],
                     torch.from_numpy(slots)[:, None, :]]
            self.tensors[key] = g

    def __getitem__(self, key):
        return self.tensors[key]


def _scatter(cache: tq.TQPagedCache, side: str, recs):
    """Write oracle records of every (b, h) into the pools through the block table."""
    bt = cache.block_table.cpu().numpy()
    prod = cache[f"{side}_signs"] is not None
    codes, norm = cache[f"{side}_codes"].cpu(), cache[f"{side}_norm"].cpu()
    if prod:
        signs, rnorm = cache[f"{side}_signs"].cpu(), cache[f"{side}_rnorm"].cpu()
    for idx, r in enumerate(recs):
        b, h = divmod(idx, cache.Hkv)
        t = np.arange(r.norm16.shape[0])
        pg, sl = torch.from_numpy(bt[b, t // cache.page_size].astype(np.int64)), torch.from_numpy(t % cache.page_size)
        codes[pg, h, sl] = torch.from_numpy(r.packed.copy())
        norm[pg, h, sl] = torch.from_numpy(r.norm16.view(np.int16).copy())
        if prod:
            signs[pg, h, sl] = torch.from_numpy(r.qjl_packed.copy())
            rnorm[pg, h, sl] = torch.from_numpy(r.rnorm16.view(np.int16).copy())
    cache[f"{side}_codes"].copy_(codes)
    cache[f"{side}_norm"].copy_(norm)
    if prod:
        cache[f"{side}_signs"].copy_(signs)
        cache[f"{side}_rnorm"].copy_(rnorm)
    torch.cuda.synchronize()


@pytest.mark.parametrize("page_size,kb,vb,B,Hkv,T", [
    (32, 4, 2, 4, 8, 400),   # 12800 vectors per tensor: the bulk tensor-core writer
    (16, 3, 3, 2, 2, 50),    # few vectors: the one-warp-per-vector writer
])
def test_paged_write_matches_dense_write_and_oracle(page_size, kb, vb, B, Hkv, T):
    max_pages = (T + 1 + page_size - 1) // page_size
    num_pages = B * max_pages + 5
    K, V = random_kv(B, Hkv, T + 1, 128, dtype=torch.float32, seed=41)
    K[..., :3] *= 20.0
    Kb, Vb = K.to(torch.bfloat16), V.to(torch.bfloat16)
    paged = tq.TQPagedCache(B, Hkv, 128, page_size, num_pages, max_pages, kb, vb,
                            _block_table(B, max_pages, num_pages, 7), seed=13)
    dense = tq.TQCache(B, Hkv, max_pages * page_size, 128, kb, vb, seed=13)
    # prefill T positions, then append one (a decode-time write)
    for c in (paged, dense):
        write = tq.tq_quantize_kv_paged if c is paged else tq.tq_quantize_kv
        write(Kb[:, :, :T].contiguous().cuda(), Vb[:, :, :T].contiguous().cuda(), c, 0)
        write(Kb[:, :, T:].contiguous().cuda(), Vb[:, :, T:].contiguous().cuda(), c, T)
    torch.cuda.synchronize()
    view = _DenseView(paged, T + 1)
    for key in ("k_codes", "v_codes", "k_norm", "v_norm"):
        assert torch.equal(view[key], dense[key][:, :, : T + 1].cpu()), key
    heads = [(0, 0), (B - 1, Hkv - 1)]
    for side, X, bits in (("k", Kb, kb), ("v", Vb, vb)):
        Xn = P.to_np(X)
        recs = [P.oracle_records(Xn[b:b + 1, h:h + 1], bits, O.MSE, 13, 1, None)[0] for b, h in heads]
        P.compare_records(view, side, recs, heads=heads)


@pytest.mark.parametrize("page_size,G,Hkv,kb,vb", [(16, 4, 2, 4, 2), (64, 8, 1, 4, 2), (32, 2, 3, 3, 3)])
def test_paged_decode_matches_oracle(page_size, G, Hkv, kb, vb):
    T_lens = [1, 500, 17, 640, 333]
    B, Hq, T_cap = len(T_lens), G * Hkv, 640
    max_pages = T_cap // page_size
    num_pages = B * max_pages + 3
    K, V = random_kv(B, Hkv, T_cap, 128, dtype=torch.float32, seed=19)
    K[..., :3] *= 20.0
    g = torch.Generator().manual_seed(20)
    q = torch.randn(B, Hq, 128, generator=g).to(torch.bfloat16)
    cache = tq.TQPagedCache(B, Hkv, 128, page_size, num_pages, max_pages, kb, vb,
                            _block_table(B, max_pages, num_pages, 3), seed=31)
    k_recs = P.oracle_records(P.to_np(K), kb, O.MSE, 31, 3, None)
    v_recs = P.oracle_records(P.to_np(V), vb, O.MSE, 31, 3, None)
    _scatter(cache, "k", k_recs)
    _scatter(cache, "v", v_recs)
    scale = 1.0 / math.sqrt(128)
    out = torch.empty(B, Hq, 128, device="cuda")
    ws = tq.workspace(tq.tq_decode_paged_workspace_bytes(cache, Hq, T_lens))
    tq.tq_decode_attention_paged(q.cuda(), cache, T_lens, scale, out, ws)
    torch.cuda.synchronize()
    qn, on = P.to_np(q), P.to_np(out)
    for b, T in enumerate(T_lens):
        want = P.oracle_decode(qn[b:b + 1], k_recs[b * Hkv:(b + 1) * Hkv], v_recs[b * Hkv:(b + 1) * Hkv],
                               1, Hkv, scale, T)
        P.assert_attention_close(on[b:b + 1], want)
    # the same records in the dense layout give the same outputs up to rounding: the paged walk
    # deals page chunks to the warps, so each warp's softmax reference (and with it the fp16
    # rounding of its weights) can differ from the dense walk's
    dense = tq.TQCache(B, Hkv, T_cap, 128, kb, vb, seed=31)
    P.upload(dense, "k", k_recs)
    P.upload(dense, "v", v_recs)
    out_d = torch.empty_like(out)
    ws_d = tq.workspace(tq.tq_decode_varlen_workspace_bytes(dense, Hq, T_lens))
    tq.tq_decode_attention_varlen(q.cuda(), dense, T_lens, scale, out_d, ws_d)
    torch.cuda.synchronize()
    P.assert_attention_close(P.to_np(out), P.to_np(out_d))


@pytest.mark.parametrize("page_size,B,Hkv,T", [
    (32, 4, 6, 300),  # 7200 vectors per tensor: the bulk tcgen05 writer
    (16, 2, 2, 40),   # few vectors: the warp-level writer
])
def test_paged_prod_write_matches_dense_write_and_oracle(page_size, B, Hkv, T):
    # TurboQuant_prod, head_dim 64, 64 sketch rows: codes, QJL signs, norms and residual norms
    max_pages = (T + 1 + page_size - 1) // page_size
    num_pages = B * max_pages + 5
    K, V = random_kv(B, Hkv, T + 1, 64, dtype=torch.float32, seed=43)
    Kb, Vb = K.to(torch.bfloat16), V.to(torch.bfloat16)
    paged = tq.TQPagedCache(B, Hkv, 64, page_size, num_pages, max_pages, 2, 2,
                            _block_table(B, max_pages, num_pages, 9), seed=13,
                            k_mode=tq.TQ_PROD, v_mode=tq.TQ_PROD, qjl_seed=5)
    dense = tq.TQCache(B, Hkv, max_pages * page_size, 64, 2, 2, tq.TQ_PROD, tq.TQ_PROD, 0, 0, seed=13, qjl_seed=5)
    for c in (paged, dense):
        write = tq.tq_quantize_kv_paged if c is paged else tq.tq_quantize_kv
        write(Kb[:, :, :T].contiguous().cuda(), Vb[:, :, :T].contiguous().cuda(), c, 0)
        write(Kb[:, :, T:].contiguous().cuda(), Vb[:, :, T:].contiguous().cuda(), c, T)
    torch.cuda.synchronize()
    view = _DenseView(paged, T + 1)
    for side in ("k", "v"):
        for key in ("codes", "signs", "norm", "rnorm"):
            k = f"{side}_{key}"
            assert torch.equal(view[k], dense[k][:, :, : T + 1].cpu()), k
    heads = [(0, 0), (B - 1, Hkv - 1)]
    for side, X in (("k", Kb), ("v", Vb)):
        Xn = P.to_np(X)
        recs = [P.oracle_records(Xn[b:b + 1, h:h + 1], 2, O.PROD, 13, 5, None)[0] for b, h in heads]
        P.compare_records(view, side, recs, heads=heads)


@pytest.mark.parametrize("page_size,G,Hkv", [(16, 1, 3), (32, 2, 2), (64, 1, 2)])
def test_paged_prod_decode_matches_oracle(page_size, G, Hkv):
    # one query head per KV head: byte-table scores; two: tensor-core scores
    T_lens = [1, 500, 17, 640, 333, 64]
    B, Hq, T_cap, d = len(T_lens), G * Hkv, 640, 64
    max_pages = T_cap // page_size
    num_pages = B * max_pages + 3
    K, V = random_kv(B, Hkv, T_cap, d, dtype=torch.float32, seed=23)
    K[..., :3] *= 20.0
    g = torch.Generator().manual_seed(24)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    cache = tq.TQPagedCache(B, Hkv, d, page_size, num_pages, max_pages, 2, 2,
                            _block_table(B, max_pages, num_pages, 4), seed=31,
                            k_mode=tq.TQ_PROD, v_mode=tq.TQ_PROD, qjl_seed=3)
    k_recs = P.oracle_records(P.to_np(K), 2, O.PROD, 31, 3, None)
    v_recs = P.oracle_records(P.to_np(V), 2, O.PROD, 31, 3, None)
    _scatter(cache, "k", k_recs)
    _scatter(cache, "v", v_recs)
    scale = 1.0 / math.sqrt(d)
    out = torch.empty(B, Hq, d, device="cuda")
    ws = tq.workspace(tq.tq_decode_paged_workspace_bytes(cache, Hq, T_lens))
    tq.tq_decode_attention_paged(q.cuda(), cache, T_lens, scale, out, ws)
    torch.cuda.synchronize()
    qn, on = P.to_np(q), P.to_np(out)
    for b, T in enumerate(T_lens):
        want = P.oracle_decode(qn[b:b + 1], k_recs[b * Hkv:(b + 1) * Hkv], v_recs[b * Hkv:(b + 1) * Hkv],
                               1, Hkv, scale, T)
        P.assert_attention_close(on[b:b + 1], want)
    # the same records in the dense layout give the same outputs
    dense = tq.TQCache(B, Hkv, T_cap, d, 2, 2, tq.TQ_PROD, tq.TQ_PROD, 0, 0, seed=31, qjl_seed=3)
    P.upload(dense, "k", k_recs)
    P.upload(dense, "v", v_recs)
    out_d = torch.empty_like(out)
    ws_d = tq.workspace(tq.tq_decode_varlen_workspace_bytes(dense, Hq, T_lens))
    tq.tq_decode_attention_varlen(q.cuda(), dense, T_lens, scale, out_d, ws_d)
    torch.cuda.synchronize()
    torch.testing.assert_close(out, out_d, rtol=1e-5, atol=1e-6)


def test_paged_cache_rejects_unsupported_layouts():
    bt = torch.zeros(2, 4, dtype=torch.int32, device="cuda")
    with pytest.raises(tq.TQError):
        cache = tq.TQPagedCache(2, 1, 128, 24, 8, 4, 4, 2, bt)  # page size not a power of two
        tq.tq_decode_paged_workspace_bytes(cache, 4, [10, 20])
    cache = tq.TQPagedCache(2, 1, 128, 16, 8, 4, 4, 2, bt)
    with pytest.raises(tq.TQError):
        tq.tq_decode_paged_workspace_bytes(cache, 4, [10, 65])  # longer than 4 pages of 16
    x = torch.zeros(2, 1, 3, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_quantize_kv_paged(x, x, cache, 0)  # fp32 input has no paged writer
    assert e.value.status == tq.TQ_ERR_UNSUPPORTED
    # TurboQuant_prod pages hold head_dim 64 only; mixed modes are not paged
    for d, km, vm in ((128, tq.TQ_PROD, tq.TQ_PROD), (64, tq.TQ_PROD, tq.TQ_MSE)):
        c = tq.TQPagedCache(2, 1, d, 16, 8, 4, 2, 2, bt, k_mode=km, v_mode=vm)
        with pytest.raises(tq.TQError) as e:
            tq.tq_decode_paged_workspace_bytes(c, 2, [10, 20])  # a size query: 0 bytes and the message
        assert "paged caches hold" in str(e.value)
