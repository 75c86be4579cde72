"""GPU test of the device-side failure detection: a bounded wait that runs out.

Every wait of the tensor-core kernels is bounded. la_pbd_selftest_timeout runs one attention
call in which the MMA thread withholds the completion signal of its first S^T product, with
every wait limited to 1 ms: nothing else ever completes that barrier, so the softmax warps'
wait for it runs out. No trap, fault or endless loop is involved. The kernel must raise the
sticky LA_ERR_TIMEOUT flag, drain what it has in flight, free its tensor memory and return.
The test checks the status, that it arrives quickly, and that the context, the tensor memory of
the SMs that ran it and the same workspace then serve normal calls that match the oracle.
"""
import time

import pytest
import torch

import block_masked_window_b200 as bmw
import workloads
from gpu_util import assert_parity, errors, oracle_step, to_dev

pytestmark = pytest.mark.gpu

LA_ERR_TIMEOUT = 6


def test_bounded_wait_runs_out_and_context_recovers(cuda_lib):
    wl = workloads.WORKLOADS["tiny"]
    wi = workloads.generate(wl)
    li = wi.layers[0]
    cfg = bmw.Config.make(wl.batch, wl.num_q_heads, wl.num_kv_heads, wi.max_seq,
                          algo=bmw.LA_ALGO_TCGEN05)
    q, kc, vc, sl = to_dev(li.q), to_dev(li.k_cache), to_dev(li.v_cache), to_dev(wi.seq_lens)
    bmw.la_kv_append(cfg, to_dev(li.k_new), to_dev(li.v_new), kc, vc, sl, wl.window)
    ws = bmw.Workspace(cfg, wl.window)
    out = torch.full_like(q, float("nan"))
    t0 = time.perf_counter()
    bmw.la_pbd_selftest_timeout(cfg, q, kc, vc, sl, wl.window, out, ws, 1_000_000)
    st = bmw.la_pbd_check(ws)
    elapsed = time.perf_counter() - t0
    assert st == LA_ERR_TIMEOUT, bmw.la_status_string(st)
    assert elapsed < 5.0, elapsed
    assert bmw.la_pbd_check(ws) == 0          # read and cleared

    # The same workspace serves a normal call, whose result matches the oracle.
    ref = oracle_step(li, wi.seq_lens, wl.scale)
    out = torch.full_like(q, float("nan"))
    bmw.la_pbd_attn(cfg, q, kc, vc, sl, wl.window, out, ws)
    torch.cuda.synchronize()
    assert bmw.la_pbd_check(ws) == 0
    assert_parity(out.cpu(), ref, "after the timeout self-test")


def test_every_sm_allocates_after_timeouts(cuda_lib):
    """Timed-out CTAs on many SMs free their tensor memory: a full-grid call afterwards (one
    CTA per SM, each allocating all 512 columns) completes and matches the oracle."""
    wl = workloads.WORKLOADS["tiny"]
    wi = workloads.random_case(40, [100 + 37 * i for i in range(40)], 6, seed=91)
    li = wi.layers[0]
    cfg = bmw.Config.make(40, 16, 2, wi.max_seq, algo=bmw.LA_ALGO_TCGEN05)
    q, kc, vc, sl = to_dev(li.q), to_dev(li.k_cache), to_dev(li.v_cache), to_dev(wi.seq_lens)
    bmw.la_kv_append(cfg, to_dev(li.k_new), to_dev(li.v_new), kc, vc, sl, 6)
    ws = bmw.Workspace(cfg, 6)
    out = torch.empty_like(q)
    for _ in range(2):
        bmw.la_pbd_selftest_timeout(cfg, q, kc, vc, sl, 6, out, ws, 1_000_000)
        assert bmw.la_pbd_check(ws) == LA_ERR_TIMEOUT
    bmw.la_pbd_attn(cfg, q, kc, vc, sl, 6, out, ws)
    torch.cuda.synchronize()
    assert bmw.la_pbd_check(ws) == 0
    assert_parity(out.cpu(), oracle_step(li, wi.seq_lens, wi.workload.scale), "after timeouts")


@pytest.mark.parametrize("name,fused", [("tiny", False), ("single_image", True),
                                        ("ragged", True), ("ragged", False)])
def test_rejected_early_plan_gives_the_same_result(cuda_lib, name, fused):
    """The attention kernel issues its first copies from a plan made before its dependency
    wait and checks that plan afterwards. With the check forced to fail, the kernel drains
    those copies, initialises its barriers again and follows the plan made after the wait:
    the output and the caches must be bit-identical to a normal call."""
    wl = workloads.WORKLOADS[name]
    wi = workloads.generate(wl, layers=1)
    li = wi.layers[0]
    cfg = bmw.Config.make(wl.batch, wl.num_q_heads, wl.num_kv_heads, wi.max_seq,
                          algo=bmw.LA_ALGO_TCGEN05)
    results = []
    for replan in (False, True):
        q, kc, vc, sl = to_dev(li.q), to_dev(li.k_cache), to_dev(li.v_cache), to_dev(wi.seq_lens)
        kn, vn = to_dev(li.k_new), to_dev(li.v_new)
        ws = bmw.Workspace(cfg, wl.window)
        out = torch.full_like(q, float("nan"))
        if not fused:
            bmw.la_kv_append(cfg, kn, vn, kc, vc, sl, wl.window)
        if replan:
            bmw.la_pbd_selftest_replan(cfg, q, kn if fused else None, vn if fused else None,
                                       kc, vc, sl, wl.window, out, ws)
        elif fused:
            bmw.la_pbd_step(cfg, q, kn, vn, kc, vc, sl, wl.window, out, ws)
        else:
            bmw.la_pbd_attn(cfg, q, kc, vc, sl, wl.window, out, ws)
        torch.cuda.synchronize()
        assert bmw.la_pbd_check(ws) == 0
        results.append((out.cpu(), kc.cpu(), vc.cpu()))
    assert torch.equal(results[0][0], results[1][0])
    assert torch.equal(results[0][1], results[1][1]) and torch.equal(results[0][2], results[1][2])
    assert_parity(results[1][0], oracle_step(li, wi.seq_lens, wl.scale), f"re-plan {name}")


def test_prefill_bounded_wait_runs_out_and_context_recovers(cuda_lib):
    """The block-causal prefill kernel under the same self-test: the QK^T-issuing thread
    withholds the completion signal of the first S product of key half 0, so that half's
    softmax wait runs out after 1 ms. The other roles (the second key half, both issuing
    threads, both producers) must stop at their next bounded wait, drain, free the tensor
    memory and return with LA_ERR_TIMEOUT raised; the same workspace then serves a normal
    prefill that matches the oracle."""
    import numpy as np
    import oracle
    lens, bs = (300, 1000), 6
    pi = workloads.prefill_case(lens, seed=63, t_max=1024)
    B, T = pi.q.shape[0], pi.q.shape[1]
    cfg = bmw.Config.make(B, 16, 2, pi.k_cache.shape[2])
    q, kc, vc, sl = to_dev(pi.q), to_dev(pi.k_cache), to_dev(pi.v_cache), to_dev(pi.seq_lens)
    ws = bmw.PrefillWorkspace(cfg, T)
    out = torch.full((B, T, 16, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    t0 = time.perf_counter()
    bmw.la_block_prefill_selftest_timeout(cfg, q, kc, vc, sl, bs, out, ws, 1_000_000)
    st = bmw.la_pbd_check(ws)
    elapsed = time.perf_counter() - t0
    assert st == LA_ERR_TIMEOUT, bmw.la_status_string(st)
    assert elapsed < 5.0, elapsed
    assert bmw.la_pbd_check(ws) == 0          # read and cleared

    out = torch.full((B, T, 16, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    bmw.la_block_prefill(cfg, q, kc, vc, sl, bs, out, ws)
    torch.cuda.synchronize()
    assert bmw.la_pbd_check(ws) == 0
    out = out.cpu()
    for b, n in enumerate(lens):
        ids = np.arange(n) // bs
        k = pi.k_cache[b, :, :n].permute(1, 0, 2)
        v = pi.v_cache[b, :, :n].permute(1, 0, 2)
        ref = oracle.block_prefill_attention(pi.q[b, :n], k, v, ids, pi.scale)
        # (the prefill's bars: max |err| and relative L2; its tiles sum thousands of keys, so
        # the decode path's one-ulp check does not apply)
        assert torch.isfinite(out[b, :n]).all()
        max_abs, rel = errors(out[b, :n], ref)
        assert max_abs <= 1e-2 and rel <= 2e-3, (max_abs, rel)
