"""GPU test of la_pbd_attn_static, the entry point for callers that cannot allocate.

Callers such as an engine plugin that is handed no scratch memory, or a decode loop where
cudaMalloc is forbidden (it can synchronise the device), use la_pbd_attn_static instead of
la_pbd_attn: the library supplies the scratch from one 32 MiB device array per GPU. This test
calls it through the C ABI twice in a row and checks each output against la_pbd_attn with a
caller workspace and against the fp64 oracle, within the parity tolerance used by the other
GPU tests. The single-image layer (one sequence, split over several CTAs) puts split partial
results in the shared array; the ragged batch covers many sequences and the prefix sums the
merge reads for batches above 32. It lives in its own file, collected last, and passes alone
in a fresh process as well as after the other tests.
"""
import ctypes

import pytest
import torch

import block_masked_window_b200 as bmw
import oracle
import workloads
from gpu_util import errors

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_L2 = 2e-3


def _close(a, b):
    a, b = a.double(), b.double()
    return float((a - b).abs().max()) <= MAX_ABS and float((a - b).norm() / b.norm()) <= REL_L2


@pytest.mark.parametrize("workload", ["single_image", "ragged"])
@pytest.mark.parametrize("algo", [bmw.LA_ALGO_TCGEN05, bmw.LA_ALGO_SIMT], ids=["tcgen05", "simt"])
def test_static_entry_matches_workspace_entry(cuda_lib, algo, workload):
    wl = workloads.WORKLOADS[workload]
    wi = workloads.generate(wl, layers=1)
    li = wi.layers[0]
    cfg = bmw.Config.make(wl.batch, wl.num_q_heads, wl.num_kv_heads, wi.max_seq, algo=algo)
    dev = lambda t: t.contiguous().cuda()  # noqa: E731
    q, kc, vc, sl = dev(li.q), dev(li.k_cache), dev(li.v_cache), dev(wi.seq_lens)
    bmw.la_kv_append(cfg, dev(li.k_new), dev(li.v_new), kc, vc, sl, wl.window)
    ref = torch.empty_like(q)
    bmw.la_pbd_attn(cfg, q, kc, vc, sl, wl.window, ref, bmw.Workspace(cfg, wl.window))
    exact = oracle.pbd_step(li.q, li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens,
                            wl.scale)
    lib = bmw.load()
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        st = lib.la_pbd_attn_static(ctypes.byref(cfg), q.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                    sl.data_ptr(), wl.window, out.data_ptr(), stream)
        assert st == 0, bmw.la_status_string(st)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert _close(out.cpu(), ref.cpu())
        max_abs, rel = errors(out.cpu(), exact)
        assert max_abs <= MAX_ABS and rel <= REL_L2, (max_abs, rel)


def test_static_entry_rejects_oversized_problem(cuda_lib):
    # W * G = 128 rows per slot and 4096 sequences need far more than 32 MiB of scratch.
    cfg = bmw.Config.make(4096, 16, 2, 64)
    lib = bmw.load()
    st = lib.la_pbd_attn_static(ctypes.byref(cfg), 256, 256, 256, 256, 16, 256, None)
    assert st == 3  # LA_ERR_WORKSPACE, nothing enqueued
