"""The allocation-free decode entry point (tq_decode_attention_noalloc), called through the C
ABI, against the workspace entry point (tq_decode_attention) on the same cache.

Some callers cannot allocate device memory where they call decode attention: runtimes that
own every byte of device memory through their own pool, decode loops that must not call
cudaMalloc/cudaFree (those can stall the device), plugin interfaces with no workspace
argument. For them libtq keeps the split-K partials in a fixed 8 MiB device array of its own.
This file is collected last on purpose; it must pass alone in a fresh process and after the
rest of the suite (the shared array then holds whatever earlier calls left in it)."""
import math

import pytest
import torch

from tests import parity as P

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from quantized_decode_attention_kv_b200 import tq  # noqa: E402
from quantized_decode_attention_kv_b200.workloads import random_kv  # noqa: E402


@pytest.mark.parametrize("d,G,Hkv,kcfg,vcfg,T", [
    (128, 4, 2, (4, tq.TQ_MSE), (2, tq.TQ_MSE), 3000),
    (64, 1, 3, (2, tq.TQ_PROD), (2, tq.TQ_PROD), 777),
    (128, 4, 2, (4, tq.TQ_MSE), (3, tq.TQ_MSE), 1500),   # 3-bit values (the 3.5-bit reading)
    (256, 2, 2, (4, tq.TQ_MSE), (2, tq.TQ_MSE), 390),    # generic split-K kernel + its combine
    (32, 16, 1, (3, tq.TQ_MSE), (2, tq.TQ_MSE), 200),    # generic kernel, many heads per KV head
])
def test_noalloc_decode_matches_workspace_decode_on_two_calls(d, G, Hkv, kcfg, vcfg, T):
    B, Hq = 3, G * Hkv
    K, V = random_kv(B, Hkv, T, d, dtype=torch.bfloat16, seed=d + T)
    q = torch.randn(B, Hq, d, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16).cuda()
    cache = tq.TQCache(B, Hkv, T, d, kcfg[0], vcfg[0], kcfg[1], vcfg[1])
    tq.tq_quantize_kv(K.cuda(), V.cuda(), cache)
    scale = 1.0 / math.sqrt(d)
    ref = torch.empty(B, Hq, d, device="cuda")
    ws = tq.workspace(tq.tq_decode_workspace_bytes(cache, Hq, T))
    tq.tq_decode_attention(q, cache, T, scale, ref, ws)
    for call in range(2):  # the second call finds the first call's partials in the scratch
        out = torch.full((B, Hq, d), float("nan"), device="cuda")
        tq.tq_decode_attention_noalloc(q, cache, T, scale, out)
        torch.cuda.synchronize()
        P.assert_attention_close(P.to_np(out), P.to_np(ref))


def test_noalloc_decode_rejects_shapes_beyond_the_fixed_scratch():
    # 512 x 32 query heads of d=128 need 512*32*132*4 bytes of partials (> 8 MiB)
    B, H, d = 512, 32, 128
    cache = tq.TQCache(B, H, 1, d, 4, 2)
    q = torch.zeros(B, H, d, device="cuda", dtype=torch.bfloat16)
    out = torch.zeros(B, H, d, device="cuda")
    assert tq.tq_decode_workspace_bytes(cache, H, 1) > 8 << 20
    with pytest.raises(tq.TQError) as e:
        tq.tq_decode_attention_noalloc(q, cache, 1, 0.1, out)
    assert e.value.status == tq.TQ_ERR_WORKSPACE
    assert "fixed scratch" in str(e.value)
    assert int(out.abs().sum()) == 0  # nothing ran
