"""GPU parity of the block-causal prefill kernel (la_block_prefill) against the fp64 oracle.

Tolerance: the bar of the whole path, max |gpu - oracle| <= 1e-2 and relative L2 <= 2e-3
(bf16 in, fp32 accumulate, bf16 out). The PV product takes the probabilities in fp16 with V
converted to fp16 (exact over the data's range), or, for query tiles that read a V tile
outside that range, as two bf16 parts (P = P_hi + P_lo, residual ~2^-17 P) times bf16 V.
Either way the product adds little to the bf16 output rounding (~1.7e-3 relative L2 on
N(0,1) data); both paths are exercised below. The decode path's extra one-ulp check is not
applied: the prefill's 128-key tiles change the fp32 summation order over thousands of keys.
"""
import dataclasses

import numpy as np
import pytest
import torch

import block_masked_window_b200 as bmw
import oracle
import workloads
from gpu_util import errors, to_dev

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_L2 = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_lib):
    return cuda_lib


def run_prefill(pi, bs, Hq=16, Hkv=2):
    B, T = pi.q.shape[0], pi.q.shape[1]
    cfg = bmw.Config.make(B, Hq, Hkv, pi.k_cache.shape[2])
    out = torch.full((B, T, Hq, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    ws = bmw.PrefillWorkspace(cfg, T)
    bmw.la_block_prefill(cfg, to_dev(pi.q), to_dev(pi.k_cache), to_dev(pi.v_cache),
                         to_dev(pi.seq_lens), bs, out, ws)
    torch.cuda.synchronize()
    return out.cpu(), ws


def oracle_prefill(pi, b, bs):
    n = int(pi.seq_lens[b])
    ids = np.arange(n) // bs
    k = pi.k_cache[b, :, :n].permute(1, 0, 2)
    v = pi.v_cache[b, :, :n].permute(1, 0, 2)
    return oracle.block_prefill_attention(pi.q[b, :n], k, v, ids, pi.scale)


def check(gpu, ref, what):
    assert torch.isfinite(gpu).all(), f"{what}: non-finite output"
    max_abs, rel = errors(gpu, ref)
    print(f"[parity] {what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}")
    assert max_abs <= MAX_ABS, f"{what}: max |err| {max_abs:.3e}"
    assert rel <= REL_L2, f"{what}: rel L2 {rel:.3e}"


@pytest.mark.parametrize("lens,bs,t_max", [
    ((300,), 6, None),              # ragged last tile, PBD window size
    ((128, 1, 515), 4, 520),        # exact tile, single token, rows past T_b are padding
    ((257,), 1, None),              # block size 1: plain causal attention
    ((200,), 256, None),            # one block covers everything: bidirectional
    ((1000, 37), 6, 1024),
])
def test_prefill_parity(lens, bs, t_max):
    pi = workloads.prefill_case(lens, seed=61, t_max=t_max, stale_fill=float("nan"))
    out, ws = run_prefill(pi, bs)
    assert bmw.la_pbd_check(ws) == 0
    for b, n in enumerate(lens):
        check(out[b, :n], oracle_prefill(pi, b, bs), f"prefill T={n} bs={bs}")
        assert torch.equal(out[b, n:], torch.zeros_like(out[b, n:])), "rows past T_b"


@pytest.mark.parametrize("Hq,Hkv", [(16, 2), (8, 8), (4, 1)])
def test_prefill_gqa(Hq, Hkv):
    pi = workloads.prefill_case((390,), num_q_heads=Hq, num_kv_heads=Hkv, seed=63)
    out, _ = run_prefill(pi, 6, Hq=Hq, Hkv=Hkv)
    check(out[0], oracle_prefill(pi, 0, 6), f"prefill GQA {Hq}/{Hkv}")


def test_prefill_long_sampled_rows():
    """A 16K-token prefill (the pages' long contexts): rows sampled across the sequence, in
    every query tile position class (first, middle, last, block edges), against the
    single-row oracle."""
    n, bs = 16384, 6
    pi = workloads.prefill_case((n,), seed=67)
    out, ws = run_prefill(pi, bs)
    assert bmw.la_pbd_check(ws) == 0
    k = pi.k_cache[0, :, :n].permute(1, 0, 2)
    v = pi.v_cache[0, :, :n].permute(1, 0, 2)
    ids = np.arange(n) // bs
    rows = [0, 1, 5, 6, 127, 128, 129, 4095, 8190, 8191, 12000, 16379, 16380, 16383]
    got = torch.stack([out[0, i] for i in rows])
    ref = np.stack([oracle.block_prefill_row(pi.q[0, i], k, v, i, ids, pi.scale) for i in rows])
    check(got, ref, "prefill 16K sampled rows")


def test_prefill_invalid_length_flagged():
    pi = workloads.prefill_case((100, 50), seed=69, t_max=128)
    pi.seq_lens[1] = 200     # longer than t_max
    out, ws = run_prefill(pi, 6)
    assert bmw.la_pbd_check(ws) == 5
    assert torch.equal(out[1], torch.zeros_like(out[1]))
    check(out[0, :100], oracle_prefill(pi, 0, 6), "valid sequence beside an invalid one")


@pytest.mark.parametrize("scale_log2", [17, -12])
def test_prefill_v_outside_fp16_range(scale_log2):
    """V scaled by 2^17 (beyond fp16) or 2^-12 (below the fp16 path's lower bound): every
    query tile takes the bf16 P_hi + P_lo path. Scaling V by a power of two scales the
    output exactly (no overflow or underflow in bf16), so out * 2^-s must meet the bars
    against the oracle on the unscaled V."""
    lens, bs = (300,), 6
    pi = workloads.prefill_case(lens, seed=73)
    ref = oracle_prefill(pi, 0, bs)
    pi.v_cache = pi.v_cache * (2.0 ** scale_log2)
    out, ws = run_prefill(pi, bs)
    assert bmw.la_pbd_check(ws) == 0
    check(out[0, :300].float() * (2.0 ** -scale_log2), ref, f"prefill V x 2^{scale_log2}")


def test_prefill_mixed_paths():
    """One 128-row V tile beyond fp16 (rows [256, 384) x 2^17): the query tiles that read it
    take the bf16 path, the others the fp16 path, in the same launch. The outputs span five
    orders of magnitude and some are small sums of large terms, whose fp32 accumulation
    error scales with the terms, not with the sum. So the bar is relative L2 plus max |err|
    relative to max(1, sum_j p_ij |v_j|) (the oracle on |V|)."""
    n, bs = 640, 6
    pi = workloads.prefill_case((n,), seed=75)
    pi.v_cache[0, :, 256:384] = pi.v_cache[0, :, 256:384] * 2.0 ** 17
    out, ws = run_prefill(pi, bs)
    assert bmw.la_pbd_check(ws) == 0
    ref = oracle_prefill(pi, 0, bs)
    mag = oracle_prefill(dataclasses.replace(pi, v_cache=pi.v_cache.abs()), 0, bs)
    got = out[0, :n].double().numpy()
    assert np.isfinite(got).all()
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    worst = (np.abs(got - ref) / np.maximum(1.0, mag)).max()
    print(f"[parity] prefill mixed paths: rel_l2={rel:.3e} max_err_over_magnitude={worst:.3e}")
    assert rel <= REL_L2 and worst <= MAX_ABS
    # Query rows < 252 (block 6) see only keys [0, 252), none of the scaled rows, so they meet
    # the absolute bar too: rows [0, 128) from the fp16 path, rows [128, 252) from the bf16
    # path (their query tile also holds rows that see the scaled tile).
    check(out[0, :252], ref[:252], "prefill rows before the scaled tile")
