"""Helpers shared by the GPU tests: run the CUDA path through the C ABI and compare it with
the fp64 oracle.

Acceptance bar of this path (bf16 in, fp32 accumulate, bf16 out):
max |gpu - oracle| <= 1e-2 and ||gpu - oracle||_2 / ||oracle||_2 <= 2e-3 against the fp64
oracle. A second, tighter check compares with the oracle rounded to bf16 (RNE): every element must
be within one bf16 ulp of the correctly rounded value, plus an absolute slack of 4e-6 times
the largest output magnitude. The slack covers outputs that are small because their terms
cancel: there the fp32 accumulation error (relative to the terms, ~1e-6) exceeds the ulp of
the tiny result. The check holds only if the fp32 work before the final rounding is
accurate to well under half an ulp of typical outputs.
"""
from __future__ import annotations

import numpy as np
import torch

import block_masked_window_b200 as bmw
import oracle

MAX_ABS = 1e-2
REL_L2 = 2e-3


def to_dev(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().to("cuda")


def run_step(li, seq_lens, max_seq, W, algo=bmw.LA_ALGO_AUTO, mask_mode=bmw.LA_MASK_PBD,
             Hq=16, Hkv=2, scale=None, ws=None, return_cache=False):
    """Append + attention for one layer through the C ABI. Returns the bf16 output (CPU)."""
    B = li.q.shape[0]
    cfg = bmw.Config.make(B, Hq, Hkv, max_seq, scale=scale, mask_mode=mask_mode, algo=algo)
    q = to_dev(li.q)
    kc, vc = to_dev(li.k_cache), to_dev(li.v_cache)
    kn, vn = to_dev(li.k_new), to_dev(li.v_new)
    sl = to_dev(seq_lens)
    out = torch.full_like(q, float("nan"))
    ws = ws or bmw.Workspace(cfg, W)
    bmw.la_pbd_step(cfg, q, kn, vn, kc, vc, sl, W, out, ws)
    torch.cuda.synchronize()
    if return_cache:
        return out.cpu(), kc.cpu(), vc.cpu(), ws
    return out.cpu()


def oracle_step(li, seq_lens, scale, mask="pbd"):
    return oracle.pbd_step(li.q, li.k_cache, li.v_cache, li.k_new, li.v_new, seq_lens, scale,
                           mask=mask)


def errors(gpu: torch.Tensor, ref: np.ndarray):
    g = gpu.to(torch.float64).numpy()
    diff = g - ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    return max_abs, rel


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    a = np.abs(x)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_parity(gpu: torch.Tensor, ref: np.ndarray, what: str = ""):
    assert torch.isfinite(gpu).all(), f"{what}: non-finite output"
    max_abs, rel = errors(gpu, ref)
    assert max_abs <= MAX_ABS, f"{what}: max |err| {max_abs:.3e} > {MAX_ABS}"
    assert rel <= REL_L2, f"{what}: rel L2 {rel:.3e} > {REL_L2}"
    # within one bf16 ulp of the correctly rounded oracle value
    rounded = torch.from_numpy(ref).to(torch.bfloat16).to(torch.float64).numpy()
    g = gpu.to(torch.float64).numpy()
    slack = 4e-6 * float(np.abs(ref).max()) if ref.size else 0.0
    dev = np.abs(g - rounded)
    off = dev > bf16_ulp(ref) * 1.0001 + slack
    assert not off.any(), (f"{what}: {int(off.sum())} elements beyond 1 ulp of bf16(oracle); "
                           f"worst {float(dev[off].max()):.3e} at |ref| {float(np.abs(ref[off]).min()):.3e}")
    print(f"[parity] {what}: max_abs={max_abs:.3e} rel_l2={rel:.3e} "
          f"ulp_exact={float((dev <= bf16_ulp(ref) * 1.0001).mean()):.6f}")
    return max_abs, rel
