"""Helpers for GPU-vs-oracle parity tests: run the oracle on the same seeded inputs, upload
oracle records into a device cache, and compare device records with the oracle's.

Comparison rules (the two sides decide in different precisions: float64 here, float32 on the
device):
  * codes: bit-exact, except coordinates whose oracle z lies within 1e-5 of a decision
    boundary (N(0,1) scale); those are counted and returned.
  * QJL sign bits: bit-exact for vectors whose codes all match, except rows with
    |(S r)_j| < 1e-5 * ||r||.
  * fp16 norms (and residual norms): bit-exact unless the exact value is within a relative
    1e-5 of a float16 rounding tie, where either neighbour is accepted.
  * dequantised vectors: |x_hat_gpu - x_hat| / ||x|| <= 1e-5 per coordinate.
  * attention: relative L2 <= 2e-3 (whole output and each query head).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from quantized_decode_attention_kv_b200 import tq

BOUNDARY_EPS = 1e-5
ATTN_RTOL = 2e-3
DEQUANT_ATOL = 1e-5


def to_np(x: torch.Tensor) -> np.ndarray:
    return x.detach().float().cpu().numpy().astype(np.float64)


def oracle_records(X: np.ndarray, bits: int, mode: int, seed: int, qjl_seed: int, m: int | None):
    """Oracle records per (b, h) of X [B, Hkv, T, d], row-major list."""
    B, H = X.shape[:2]
    return [O.quantize(X[b, h], bits, mode, seed=seed, qjl_seed=qjl_seed, m=m)
            for b in range(B) for h in range(H)]


def upload(cache: tq.TQCache, side: str, recs, t_offset: int = 0) -> None:
    """Write oracle records into the device cache at positions [t_offset, t_offset + T)."""
    H = cache.Hkv
    for idx, r in enumerate(recs):
        b, h = divmod(idx, H)
        T = r.norm16.shape[0]
        sl = slice(t_offset, t_offset + T)
        if cache[f"{side}_codes"] is not None:
            cache[f"{side}_codes"][b, h, sl] = torch.from_numpy(r.packed.copy())
        cache[f"{side}_norm"][b, h, sl] = torch.from_numpy(r.norm16.view(np.int16).copy())
        if r.mode == O.PROD:
            cache[f"{side}_signs"][b, h, sl] = torch.from_numpy(r.qjl_packed.copy())
            cache[f"{side}_rnorm"][b, h, sl] = torch.from_numpy(r.rnorm16.view(np.int16).copy())
    torch.cuda.synchronize()


def _fp16_ambiguous(exact: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):  # norms past the fp16 range round to inf on both sides
        lo = (exact * (1 - 1e-5)).astype(np.float32).astype(np.float16)
        hi = (exact * (1 + 1e-5)).astype(np.float32).astype(np.float16)
    return lo != hi


def _fp16_close(got16: np.ndarray, want16: np.ndarray, exact: np.ndarray) -> np.ndarray:
    same = got16.view(np.int16) == want16.view(np.int16)
    amb = _fp16_ambiguous(exact)
    with np.errstate(over="ignore", invalid="ignore"):
        nbr = np.abs(got16.astype(np.float64) - exact) <= np.abs(
            np.spacing(np.abs(exact).astype(np.float16)).astype(np.float64))
    return same | (amb & nbr)


def compare_records(cache: tq.TQCache, side: str, recs, t_offset: int = 0, heads=None) -> dict:
    """Assert device records equal the oracle's under the rules above; return counts.
    ``heads`` lists the (b, h) of each record; by default records cover every (b, h) in
    row-major order."""
    H = cache.Hkv
    wbits = recs[0].bits - 1 if recs[0].mode == O.PROD else recs[0].bits
    d = recs[0].d
    codes_dev = _Lazy(cache[f"{side}_codes"]) if cache[f"{side}_codes"] is not None else None
    norm_dev = _Lazy(cache[f"{side}_norm"], np.float16)
    if recs[0].mode == O.PROD:
        signs_dev = _Lazy(cache[f"{side}_signs"])
        rn_dev = _Lazy(cache[f"{side}_rnorm"], np.float16)
    stats = {"coords": 0, "near_boundary": 0, "flipped_near_boundary": 0, "sign_rows": 0,
             "flipped_signs_near_zero": 0}
    for idx, r in enumerate(recs):
        b, h = divmod(idx, H) if heads is None else heads[idx]
        T = r.norm16.shape[0]
        sl = slice(t_offset, t_offset + T)
        near = O.boundary_distance(r) < BOUNDARY_EPS
        if wbits > 0:
            got = O.unpack_bits(codes_dev[b, h, sl], wbits, d)
            bad = got != r.codes
            assert not np.any(bad & ~near), (
                f"{side}[{b},{h}]: {int(np.sum(bad & ~near))} code mismatches away from boundaries")
            stats["flipped_near_boundary"] += int(np.sum(bad))
            row_ok = ~np.any(bad, axis=1)
        else:
            row_ok = np.ones(T, dtype=bool)
        stats["coords"] += near.size
        stats["near_boundary"] += int(np.sum(near))
        ok = _fp16_close(norm_dev[b, h, sl], r.norm16, r.norm)
        assert np.all(ok), f"{side}[{b},{h}] norm mismatch at {np.nonzero(~ok)[0][:5]}"
        if r.mode == O.PROD:
            got_bits = O.unpack_bits(signs_dev[b, h, sl], 1, r.m)
            near_s = np.abs(r.proj) < BOUNDARY_EPS * r.rnorm[:, None]
            bad_s = (got_bits != r.qjl_bits) & row_ok[:, None]
            assert not np.any(bad_s & ~near_s), f"{side}[{b},{h}] QJL sign mismatches"
            stats["sign_rows"] += int(np.sum(row_ok))
            stats["flipped_signs_near_zero"] += int(np.sum(bad_s))
            okr = _fp16_close(rn_dev[b, h, sl], r.rnorm16, r.rnorm) | ~row_ok
            assert np.all(okr), f"{side}[{b},{h}] residual-norm mismatch"
    return stats


class _Lazy:
    """Index a device tensor as [b, h, slice] and copy only that slice to the host."""

    def __init__(self, t: torch.Tensor, view=None):
        self.t, self.view = t, view

    def __getitem__(self, key):
        a = self.t[key].cpu().numpy()
        return a.view(self.view) if self.view is not None else a


def rel_l2(got: np.ndarray, want: np.ndarray) -> float:
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def assert_attention_close(got: np.ndarray, want: np.ndarray, tol: float = ATTN_RTOL) -> float:
    """Whole-output and per-head relative L2 within ``tol``; returns the worst per-head value."""
    assert rel_l2(got, want) <= tol, rel_l2(got, want)
    worst = 0.0
    for b in range(want.shape[0]):
        for h in range(want.shape[1]):
            e = rel_l2(got[b, h], want[b, h])
            worst = max(worst, e)
    assert worst <= tol, worst
    return worst


def oracle_decode(q: np.ndarray, k_recs, v_recs, B: int, Hkv: int, scale: float, T_len: int | None = None):
    """Oracle attention over the dequantised cache (optionally the first T_len tokens)."""
    if T_len is not None:
        k_recs = [_head(r, T_len) for r in k_recs]
        v_recs = [_head(r, T_len) for r in v_recs]
    return O.decode_compressed(q, k_recs, v_recs, B, Hkv, scale)


def _head(r, n):
    return O.records_from_packed(r.bits, r.mode, r.d, r.packed[:n], r.norm16[:n],
                                 r.qjl_packed[:n] if r.mode == O.PROD else None,
                                 r.rnorm16[:n] if r.mode == O.PROD else None,
                                 seed=r.seed, qjl_seed=r.qjl_seed, m=r.m)
