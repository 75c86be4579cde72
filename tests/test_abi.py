"""CPU checks of the C ABI: the library loads, exports every declared symbol, and its host-side
validation rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

import block_masked_window_b200 as bmw

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "la_pbd.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(la_[a-z_]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from block_masked_window_b200 import build
    build.build()
    return bmw.load()


def test_header_declares_binding_symbols():
    assert declared_functions() == sorted(bmw.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_version_and_status_strings(lib):
    assert bmw.la_version() == 100
    for code in range(7):
        s = bmw.la_status_string(code)
        assert isinstance(s, str) and s
    assert bmw.la_status_string(99) == "unknown status"


def _cfg(**kw):
    base = dict(batch=1, num_q_heads=16, num_kv_heads=2, max_seq=128)
    base.update(kw)
    return bmw.Config.make(**base)


@pytest.mark.parametrize("kw,W,expect", [
    (dict(), 0, 1),                        # window 0
    (dict(), 17, 1),                       # window > 16
    (dict(batch=0), 6, 1),
    (dict(batch=5000), 6, 1),
    (dict(head_dim=64), 6, 2),
    (dict(num_q_heads=15), 6, 2),          # Hq % Hkv != 0
    (dict(num_kv_heads=1), 16, 2),         # W * G = 256 > 128
    (dict(mask_mode=7), 6, 1),
    (dict(algo=9), 6, 1),
    (dict(algo=1, num_kv_heads=1), 6, 2),  # tensor-core kernel needs W * G <= 80
    (dict(max_seq=0), 6, 1),
    (dict(batch=4096, num_kv_heads=16, num_q_heads=16, max_seq=1 << 20), 6, 2),
])
def test_host_validation(lib, kw, W, expect):
    cfg = _cfg(**kw)
    st = lib.la_pbd_attn(ctypes.byref(cfg), 16, 16, 16, 16, W, 16, 256, 1 << 30, None)
    assert st == expect
    assert bmw.la_pbd_workspace_bytes(cfg, W) == 0


def test_null_and_misaligned_pointers(lib):
    cfg = _cfg()
    # null q
    assert lib.la_pbd_attn(ctypes.byref(cfg), 0, 16, 16, 16, 6, 16, 256, 1 << 30, None) == 1
    # misaligned k_cache (not 16-byte aligned)
    assert lib.la_pbd_attn(ctypes.byref(cfg), 16, 24, 16, 16, 6, 16, 256, 1 << 30, None) == 1
    # misaligned seq_lens
    assert lib.la_pbd_attn(ctypes.byref(cfg), 16, 16, 16, 18, 6, 16, 256, 1 << 30, None) == 1
    assert lib.la_kv_append(ctypes.byref(cfg), 0, 16, 16, 16, 16, 6, None) == 1
    assert lib.la_kv_append(ctypes.byref(cfg), 16, 16, 16, 16, 16, 0, None) == 1
    assert lib.la_pbd_step(ctypes.byref(cfg), 16, 16, 16, 16, 16, 16, 6, 0, 256, 1 << 30, None) == 1
    # null config
    assert lib.la_pbd_attn(None, 16, 16, 16, 16, 6, 16, 256, 1 << 30, None) == 1
    # workspace checks that need no device
    assert lib.la_pbd_workspace_init(0, 1 << 20, None) == 3
    assert lib.la_pbd_workspace_init(256, 16, None) == 3
    assert lib.la_pbd_check(0, None) == 3
    assert lib.la_pbd_check(100, None) == 3


def test_binding_rejects_cpu_tensors(lib):
    import torch
    cfg = _cfg(max_seq=8)
    q = torch.zeros(1, 6, 16, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        bmw.la_kv_append(cfg, q[:, :, :2], q[:, :, :2], torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16),
                         torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16),
                         torch.zeros(1, dtype=torch.int32), 6)


def test_noop_chain_validates_before_launching(lib):
    # every one of these is rejected on the host, before any CUDA call
    assert lib.la_noop_chain(-1, 1, 32, None) == 1
    assert lib.la_noop_chain(4, 0, 32, None) == 1
    assert lib.la_noop_chain(4, 1, 0, None) == 1
    assert lib.la_noop_chain(4, 1, 1025, None) == 1
    assert lib.la_noop_chain(0, 1, 32, None) == 0     # nothing to launch


def test_selftest_timeout_validates_before_launching(lib):
    cfg = _cfg()
    # wait limits outside [1 us, 2 s] are rejected before any CUDA call
    for limit in (0, 999, 3_000_000_000):
        assert lib.la_pbd_selftest_timeout(ctypes.byref(cfg), 16, 16, 16, 16, 6, 16, 256, 1 << 30,
                                           limit, None) == 1


def test_prefill_selftest_timeout_validates_before_launching(lib):
    cfg = _cfg(max_seq=1024)
    # wait limits outside [1 us, 2 s] are rejected before any CUDA call
    for limit in (0, 999, 3_000_000_000):
        assert lib.la_block_prefill_selftest_timeout(ctypes.byref(cfg), 16, 16, 16, 16, 256, 6,
                                                     16, 256, 1 << 30, limit, None) == 1
    # and so are the prefill's own argument errors (a null q), with a valid limit
    assert lib.la_block_prefill_selftest_timeout(ctypes.byref(cfg), None, 16, 16, 16, 256, 6,
                                                 16, 256, 1 << 30, 1_000_000, None) == 1


def test_algo_choice_without_gpu(lib):
    # kernel choice is host logic: tcgen05 up to 80 rows per KV head, CUDA cores above
    assert bmw.la_pbd_algo(_cfg(), 6) == bmw.LA_ALGO_TCGEN05
    assert bmw.la_pbd_algo(_cfg(), 10) == bmw.LA_ALGO_TCGEN05
    assert bmw.la_pbd_algo(_cfg(), 11) == bmw.LA_ALGO_SIMT
    assert bmw.la_pbd_algo(_cfg(algo=bmw.LA_ALGO_SIMT), 6) == bmw.LA_ALGO_SIMT
    assert lib.la_pbd_algo(ctypes.byref(_cfg()), 17) == -1
    assert lib.la_pbd_algo(ctypes.byref(_cfg(algo=1)), 11) == -2


def test_prefill_workspace_layout_without_gpu(lib):
    # header (256 B), one int32 flag per 128-row V tile, then the fp16 copy of V at a 1024-byte
    # boundary: B * Hkv * ceil(t_max / 128) * 128 rows of 256 bytes
    cfg = _cfg(max_seq=16384)
    tiles = 1 * 2 * 128
    assert bmw.la_block_prefill_workspace_bytes(cfg, 16384) == 2048 + tiles * 128 * 256
    assert bmw.la_block_prefill_workspace_bytes(cfg, 1) == 1024 + 2 * 128 * 256
    assert bmw.la_block_prefill_workspace_bytes(cfg, 0) == 0
    assert bmw.la_block_prefill_workspace_bytes(_cfg(head_dim=64), 128) == 0
    # a workspace below that size is rejected on the host, before any CUDA call
    need = bmw.la_block_prefill_workspace_bytes(cfg, 300)
    args = (16, 16, 16, 16, 300, 6, 16, 256)
    assert lib.la_block_prefill(ctypes.byref(cfg), *args, need - 1, None) == 3
    assert lib.la_block_prefill(ctypes.byref(cfg), *args[:-1], 0, need, None) == 3
