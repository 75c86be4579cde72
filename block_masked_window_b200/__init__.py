"""Python binding of ``libla_pbd.so``, the B200 PBD window-attention library.

Argument marshalling only: every step of the computation runs in the library's CUDA kernels
(see ``include/la_pbd.h`` for the C ABI). The functions take torch CUDA tensors for device
memory and use torch's current CUDA stream; they never fall back to another implementation:
if the shared library is missing or fails to load, they raise.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

__all__ = [
    "LA_MASK_PBD", "LA_MASK_CAUSAL_WINDOW", "LA_ALGO_AUTO", "LA_ALGO_TCGEN05", "LA_ALGO_SIMT",
    "LaError", "Config", "load", "library_path", "la_version", "la_status_string",
    "la_pbd_workspace_bytes", "la_pbd_workspace_init", "la_kv_append", "la_pbd_attn",
    "la_pbd_step", "la_pbd_check", "la_pbd_attn_static", "la_pbd_plan", "la_pbd_plan_params",
    "la_noop_chain", "la_pbd_attn_varwin", "la_pbd_algo", "chosen_algo",
    "la_pbd_selftest_timeout", "la_pbd_selftest_replan", "la_block_prefill_selftest_timeout",
    "la_pbd_step_varwin", "la_block_prefill", "la_block_prefill_workspace_bytes",
    "la_pbd_attn_paged", "la_pbd_step_paged", "Workspace", "PrefillWorkspace",
    "EXPORTED_SYMBOLS",
]

LA_MASK_PBD = 0
LA_MASK_CAUSAL_WINDOW = 1
LA_ALGO_AUTO = 0
LA_ALGO_TCGEN05 = 1
LA_ALGO_SIMT = 2

LA_OK = 0
LA_ERR_INVALID_ARG_CODE = 1
STATUS_NAMES = {0: "LA_OK", 1: "LA_ERR_INVALID_ARG", 2: "LA_ERR_UNSUPPORTED",
                3: "LA_ERR_WORKSPACE", 4: "LA_ERR_CUDA", 5: "LA_ERR_SEQ_OVERFLOW",
                6: "LA_ERR_TIMEOUT"}

EXPORTED_SYMBOLS = ["la_version", "la_status_string", "la_pbd_workspace_bytes",
                    "la_pbd_workspace_init", "la_kv_append", "la_pbd_attn", "la_pbd_step",
                    "la_pbd_check", "la_pbd_attn_static", "la_pbd_plan", "la_pbd_plan_params",
                    "la_noop_chain", "la_pbd_algo", "la_pbd_selftest_timeout",
                    "la_pbd_selftest_replan", "la_block_prefill_selftest_timeout",
                    "la_pbd_attn_varwin", "la_pbd_step_varwin", "la_block_prefill",
                    "la_block_prefill_workspace_bytes", "la_pbd_attn_paged", "la_pbd_step_paged"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB: Optional[ctypes.CDLL] = None


class LaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} "
                         f"({la_status_string(status) if _LIB else ''})")


class Config(ctypes.Structure):
    """Mirror of ``la_pbd_cfg``."""
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("max_seq", ctypes.c_int32), ("scale", ctypes.c_float),
                ("mask_mode", ctypes.c_int32), ("algo", ctypes.c_int32)]

    @classmethod
    def make(cls, batch, num_q_heads, num_kv_heads, max_seq, head_dim=128, scale=None,
             mask_mode=LA_MASK_PBD, algo=LA_ALGO_AUTO) -> "Config":
        if scale is None:
            scale = 1.0 / math.sqrt(head_dim)
        return cls(batch, num_q_heads, num_kv_heads, head_dim, max_seq, scale, mask_mode, algo)


def library_path() -> str:
    return os.path.join(_HERE, "libla_pbd.so")


def load() -> ctypes.CDLL:
    """Load the shared library (raises if it has not been built)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m block_masked_window_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    cfgp = ctypes.POINTER(Config)
    lib.la_version.restype = i32
    lib.la_version.argtypes = []
    lib.la_status_string.restype = ctypes.c_char_p
    lib.la_status_string.argtypes = [i32]
    lib.la_pbd_workspace_bytes.restype = sz
    lib.la_pbd_workspace_bytes.argtypes = [cfgp, i32]
    lib.la_pbd_workspace_init.restype = i32
    lib.la_pbd_workspace_init.argtypes = [vp, sz, vp]
    lib.la_kv_append.restype = i32
    lib.la_kv_append.argtypes = [cfgp, vp, vp, vp, vp, vp, i32, vp]
    lib.la_pbd_attn.restype = i32
    lib.la_pbd_attn.argtypes = [cfgp, vp, vp, vp, vp, i32, vp, vp, sz, vp]
    lib.la_pbd_step.restype = i32
    lib.la_pbd_step.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, i32, vp, vp, sz, vp]
    lib.la_pbd_check.restype = i32
    lib.la_pbd_check.argtypes = [vp, vp]
    lib.la_pbd_attn_static.restype = i32
    lib.la_pbd_attn_static.argtypes = [cfgp, vp, vp, vp, vp, i32, vp, vp]
    lib.la_pbd_attn_varwin.restype = i32
    lib.la_pbd_attn_varwin.argtypes = [cfgp, vp, vp, vp, vp, vp, i32, vp, vp, sz, vp]
    lib.la_pbd_step_varwin.restype = i32
    lib.la_pbd_step_varwin.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, sz, vp]
    lib.la_block_prefill.restype = i32
    lib.la_block_prefill.argtypes = [cfgp, vp, vp, vp, vp, i32, i32, vp, vp, sz, vp]
    lib.la_block_prefill_selftest_timeout.restype = i32
    lib.la_block_prefill_selftest_timeout.argtypes = [cfgp, vp, vp, vp, vp, i32, i32, vp, vp, sz,
                                                      ctypes.c_int64, vp]
    lib.la_block_prefill_workspace_bytes.restype = sz
    lib.la_block_prefill_workspace_bytes.argtypes = [cfgp, i32]
    lib.la_pbd_attn_paged.restype = i32
    lib.la_pbd_attn_paged.argtypes = [cfgp, vp, vp, vp, vp, i32, i32, i32, vp, i32, vp, vp, sz, vp]
    lib.la_pbd_step_paged.restype = i32
    lib.la_pbd_step_paged.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, i32, vp, vp,
                                      sz, vp]
    lib.la_pbd_plan.restype = i32
    lib.la_pbd_plan.argtypes = [cfgp, i32, vp, i32, i32, i32, vp, i32]
    lib.la_pbd_plan_params.restype = i32
    lib.la_pbd_plan_params.argtypes = [i32, vp, vp]
    lib.la_noop_chain.restype = i32
    lib.la_noop_chain.argtypes = [i32, i32, i32, vp]
    lib.la_pbd_algo.restype = i32
    lib.la_pbd_algo.argtypes = [cfgp, i32]
    lib.la_pbd_selftest_replan.restype = i32
    lib.la_pbd_selftest_replan.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, i32, vp, vp, sz, vp]
    lib.la_pbd_selftest_timeout.restype = i32
    lib.la_pbd_selftest_timeout.argtypes = [cfgp, vp, vp, vp, vp, i32, vp, vp, sz, ctypes.c_int64,
                                            vp]
    _LIB = lib
    return lib


def la_version() -> int:
    return load().la_version()


def la_status_string(status: int) -> str:
    return load().la_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != LA_OK:
        raise LaError(status, where)


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _stream(stream) -> int:
    if stream is not None:
        return int(stream) if isinstance(stream, int) else int(stream.cuda_stream)
    import torch
    return int(torch.cuda.current_stream().cuda_stream)


_DTYPES = {}


def _check_tensor(t, name, dtype_name, shape=None):
    if not _DTYPES:
        import torch
        _DTYPES.update({"bf16": torch.bfloat16, "i32": torch.int32})
    if t.dtype is not _DTYPES[dtype_name]:
        raise TypeError(f"{name}: expected {dtype_name}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and t.shape != shape:
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def la_pbd_workspace_bytes(cfg: Config, window_len: int) -> int:
    return int(load().la_pbd_workspace_bytes(ctypes.byref(cfg), int(window_len)))


def la_pbd_workspace_init(workspace, stream=None) -> None:
    _check(load().la_pbd_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                        _stream(stream)), "la_pbd_workspace_init")


def la_block_prefill_workspace_bytes(cfg: Config, t_max: int) -> int:
    return int(load().la_block_prefill_workspace_bytes(ctypes.byref(cfg), int(t_max)))


class Workspace:
    """A device workspace sized by ``la_pbd_workspace_bytes`` (allocated through torch)."""

    def __init__(self, cfg: Config, window_len: int, device=None, nbytes: Optional[int] = None):
        import torch
        n = la_pbd_workspace_bytes(cfg, window_len) if nbytes is None else int(nbytes)
        if n == 0:
            raise LaError(2, "la_pbd_workspace_bytes")
        self.nbytes = n
        self.buf = torch.empty(n + 256, dtype=torch.uint8, device=device or "cuda")
        off = (-self.buf.data_ptr()) % 256
        self.tensor = self.buf[off:off + n]
        la_pbd_workspace_init(self.tensor)

    def data_ptr(self) -> int:
        return int(self.tensor.data_ptr())


class PrefillWorkspace(Workspace):
    """A device workspace sized by ``la_block_prefill_workspace_bytes``."""

    def __init__(self, cfg: Config, t_max: int, device=None):
        n = la_block_prefill_workspace_bytes(cfg, t_max)
        if n == 0:
            raise LaError(2, "la_block_prefill_workspace_bytes")
        super().__init__(cfg, 1, device=device, nbytes=n)


def _shapes(cfg: Config, W: int):
    B, Hq, Hkv, D, S = cfg.batch, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, cfg.max_seq
    return (B, W, Hq, D), (B, Hkv, S, D), (B, W, Hkv, D)


def la_kv_append(cfg: Config, k_new, v_new, k_cache, v_cache, seq_lens, window_len: int,
                 stream=None) -> None:
    W = int(window_len)
    _, cache_shape, new_shape = _shapes(cfg, W)
    _check_tensor(k_new, "k_new", "bf16", new_shape)
    _check_tensor(v_new, "v_new", "bf16", new_shape)
    _check_tensor(k_cache, "k_cache", "bf16", cache_shape)
    _check_tensor(v_cache, "v_cache", "bf16", cache_shape)
    _check_tensor(seq_lens, "seq_lens", "i32", (cfg.batch,))
    _check(load().la_kv_append(ctypes.byref(cfg), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                               _ptr(v_cache), _ptr(seq_lens), W, _stream(stream)),
           "la_kv_append")


def la_pbd_attn(cfg: Config, q, k_cache, v_cache, seq_lens, window_len: int, out,
                workspace: Workspace, stream=None) -> None:
    W = int(window_len)
    q_shape, cache_shape, _ = _shapes(cfg, W)
    _check_tensor(q, "q", "bf16", q_shape)
    _check_tensor(k_cache, "k_cache", "bf16", cache_shape)
    _check_tensor(v_cache, "v_cache", "bf16", cache_shape)
    _check_tensor(seq_lens, "seq_lens", "i32", (cfg.batch,))
    _check_tensor(out, "out", "bf16", q_shape)
    _check(load().la_pbd_attn(ctypes.byref(cfg), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                              _ptr(seq_lens), W, _ptr(out), workspace.data_ptr(),
                              workspace.nbytes, _stream(stream)), "la_pbd_attn")


def la_pbd_step(cfg: Config, q, k_new, v_new, k_cache, v_cache, seq_lens, window_len: int, out,
                workspace: Workspace, stream=None) -> None:
    W = int(window_len)
    q_shape, cache_shape, new_shape = _shapes(cfg, W)
    _check_tensor(q, "q", "bf16", q_shape)
    _check_tensor(k_new, "k_new", "bf16", new_shape)
    _check_tensor(v_new, "v_new", "bf16", new_shape)
    _check_tensor(k_cache, "k_cache", "bf16", cache_shape)
    _check_tensor(v_cache, "v_cache", "bf16", cache_shape)
    _check_tensor(seq_lens, "seq_lens", "i32", (cfg.batch,))
    _check_tensor(out, "out", "bf16", q_shape)
    _check(load().la_pbd_step(ctypes.byref(cfg), _ptr(q), _ptr(k_new), _ptr(v_new),
                              _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), W, _ptr(out),
                              workspace.data_ptr(), workspace.nbytes, _stream(stream)),
           "la_pbd_step")


def la_pbd_check(workspace: Workspace, stream=None) -> int:
    """Synchronise and return the sticky device status (0 = LA_OK); clears it."""
    return int(load().la_pbd_check(workspace.data_ptr(), _stream(stream)))


def la_pbd_attn_static(cfg: Config, q, k_cache, v_cache, seq_lens, window_len: int, out,
                       stream=None) -> None:
    """Window attention without a caller-provided workspace.

    For callers that cannot allocate device memory (an engine plugin given no scratch, a
    loop where cudaMalloc is not allowed): the library keeps one 32 MiB scratch array per
    GPU. Calls that overlap on the GPU share that array and race; serialise them.
    """
    W = int(window_len)
    q_shape, cache_shape, _ = _shapes(cfg, W)
    _check_tensor(q, "q", "bf16", q_shape)
    _check_tensor(k_cache, "k_cache", "bf16", cache_shape)
    _check_tensor(v_cache, "v_cache", "bf16", cache_shape)
    _check_tensor(seq_lens, "seq_lens", "i32", (cfg.batch,))
    _check_tensor(out, "out", "bf16", q_shape)
    _check(load().la_pbd_attn_static(ctypes.byref(cfg), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                     _ptr(seq_lens), W, _ptr(out), _stream(stream)),
           "la_pbd_attn_static")


def la_pbd_plan(cfg: Config, window_len: int, seq_lens, num_ctas: int, unit_keys: int,
                seg_units: int = 0):
    """Host-side split-KV work plan (no GPU work): a list of (cta, b, h, j0, j1, slot)
    tuples in CTA order; slot is -1 for a segment that is a whole sequence."""
    lens = (ctypes.c_int32 * cfg.batch)(*[int(x) for x in seq_lens])
    lib = load()
    n = lib.la_pbd_plan(ctypes.byref(cfg), int(window_len), ctypes.cast(lens, ctypes.c_void_p),
                        int(num_ctas), int(unit_keys), int(seg_units), None, 0)
    if n < 0:
        raise LaError(-n, "la_pbd_plan")
    buf = (ctypes.c_int32 * (6 * max(n, 1)))()
    m = lib.la_pbd_plan(ctypes.byref(cfg), int(window_len), ctypes.cast(lens, ctypes.c_void_p),
                        int(num_ctas), int(unit_keys), int(seg_units),
                        ctypes.cast(buf, ctypes.c_void_p), n)
    if m != n:
        raise LaError(LA_ERR_INVALID_ARG_CODE, "la_pbd_plan")
    return [tuple(buf[6 * i: 6 * i + 6]) for i in range(n)]


def la_noop_chain(launches: int, ctas: int, threads: int, stream=None) -> None:
    """Enqueue `launches` empty kernels (launch-floor measurements)."""
    _check(load().la_noop_chain(int(launches), int(ctas), int(threads), _stream(stream)),
           "la_noop_chain")


def la_pbd_selftest_timeout(cfg: Config, q, k_cache, v_cache, seq_lens, window_len: int, out,
                            workspace: Workspace, wait_limit_ns: int, stream=None) -> None:
    """Enqueue the failure-detection self-test (one attention call whose first S^T completion
    is withheld, every wait limited to `wait_limit_ns`); la_pbd_check then gives 6
    (LA_ERR_TIMEOUT)."""
    W = int(window_len)
    q_shape, cache_shape, _ = _shapes(cfg, W)
    _check_tensor(q, "q", "bf16", q_shape)
    _check_tensor(k_cache, "k_cache", "bf16", cache_shape)
    _check_tensor(v_cache, "v_cache", "bf16", cache_shape)
    _check_tensor(seq_lens, "seq_lens", "i32", (cfg.batch,))
    _check_tensor(out, "out", "bf16", q_shape)
    _check(load().la_pbd_selftest_timeout(ctypes.byref(cfg), _ptr(q), _ptr(k_cache),
                                          _ptr(v_cache), _ptr(seq_lens), W, _ptr(out),
                                          workspace.data_ptr(), workspace.nbytes,
                                          int(wait_limit_ns), _stream(stream)),
           "la_pbd_selftest_timeout")


def la_pbd_selftest_replan(cfg: Config, q, k_new, v_new, k_cache, v_cache, seq_lens,
                           window_len: int, out, workspace: Workspace, stream=None) -> None:
    """Enqueue la_pbd_attn (k_new, v_new None) or la_pbd_step with the plan made before the
    dependency wait forced to be rejected (self-test of the kernel's re-plan path)."""
    W = int(window_len)
    q_shape, cache_shape, new_shape = _shapes(cfg, W)
    _check_tensor(q, "q", "bf16", q_shape)
    if k_new is not None:
        _check_tensor(k_new, "k_new", "bf16", new_shape)
        _check_tensor(v_new, "v_new", "bf16", new_shape)
    _check_tensor(k_cache, "k_cache", "bf16", cache_shape)
    _check_tensor(v_cache, "v_cache", "bf16", cache_shape)
    _check_tensor(seq_lens, "seq_lens", "i32", (cfg.batch,))
    _check_tensor(out, "out", "bf16", q_shape)
    _check(load().la_pbd_selftest_replan(ctypes.byref(cfg), _ptr(q), _ptr(k_new), _ptr(v_new),
                                         _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), W,
                                         _ptr(out), workspace.data_ptr(), workspace.nbytes,
                                         _stream(stream)),
           "la_pbd_selftest_replan")


def la_pbd_algo(cfg: Config, window_len: int) -> int:
    """The attention kernel (LA_ALGO_TCGEN05 or LA_ALGO_SIMT) the library runs for `cfg`."""
    r = int(load().la_pbd_algo(ctypes.byref(cfg), int(window_len)))
    if r < 0:
        raise LaError(-r, "la_pbd_algo")
    return r


chosen_algo = la_pbd_algo


def la_pbd_plan_params(algo: int):
    """(unit_keys, seg_units) of the plan that attention kernel `algo` follows."""
    unit, seg = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(load().la_pbd_plan_params(int(algo), ctypes.byref(unit), ctypes.byref(seg)),
           "la_pbd_plan_params")
    return unit.value, seg.value


def la_pbd_attn_varwin(cfg: Config, q, k_cache, v_cache, seq_lens, window_lens, window_max: int,
                       out, workspace: Workspace, stream=None) -> None:
    """Window attention with per-sequence window lengths (q, out padded to window_max rows)."""
    W = int(window_max)
    q_shape, cache_shape, _ = _shapes(cfg, W)
    _check_tensor(q, "q", "bf16", q_shape)
    _check_tensor(k_cache, "k_cache", "bf16", cache_shape)
    _check_tensor(v_cache, "v_cache", "bf16", cache_shape)
    _check_tensor(seq_lens, "seq_lens", "i32", (cfg.batch,))
    _check_tensor(window_lens, "window_lens", "i32", (cfg.batch,))
    _check_tensor(out, "out", "bf16", q_shape)
    _check(load().la_pbd_attn_varwin(ctypes.byref(cfg), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                     _ptr(seq_lens), _ptr(window_lens), W, _ptr(out),
                                     workspace.data_ptr(), workspace.nbytes, _stream(stream)),
           "la_pbd_attn_varwin")


def la_pbd_step_varwin(cfg: Config, q, k_new, v_new, k_cache, v_cache, seq_lens, window_lens,
                       window_max: int, out, workspace: Workspace, stream=None) -> None:
    """Append rows w < W_b of k_new/v_new, then window attention with per-sequence windows."""
    W = int(window_max)
    q_shape, cache_shape, new_shape = _shapes(cfg, W)
    _check_tensor(q, "q", "bf16", q_shape)
    _check_tensor(k_new, "k_new", "bf16", new_shape)
    _check_tensor(v_new, "v_new", "bf16", new_shape)
    _check_tensor(k_cache, "k_cache", "bf16", cache_shape)
    _check_tensor(v_cache, "v_cache", "bf16", cache_shape)
    _check_tensor(seq_lens, "seq_lens", "i32", (cfg.batch,))
    _check_tensor(window_lens, "window_lens", "i32", (cfg.batch,))
    _check_tensor(out, "out", "bf16", q_shape)
    _check(load().la_pbd_step_varwin(ctypes.byref(cfg), _ptr(q), _ptr(k_new), _ptr(v_new),
                                     _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens),
                                     _ptr(window_lens), W, _ptr(out), workspace.data_ptr(),
                                     workspace.nbytes, _stream(stream)),
           "la_pbd_step_varwin")


def la_block_prefill(cfg: Config, q, k_cache, v_cache, seq_lens, block_size: int, out,
                     workspace: Workspace, stream=None) -> None:
    """Block-causal prefill attention: q, out [B, T, Hq, D]; caches [B, Hkv, S, D] holding
    each sequence's keys in rows [0, T_b); seq_lens = T_b; workspace from
    ``PrefillWorkspace(cfg, T)``."""
    B, T = int(q.shape[0]), int(q.shape[1])
    Hq, Hkv, D, S = cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, cfg.max_seq
    _check_tensor(q, "q", "bf16", (B, T, Hq, D))
    _check_tensor(k_cache, "k_cache", "bf16", (B, Hkv, S, D))
    _check_tensor(v_cache, "v_cache", "bf16", (B, Hkv, S, D))
    _check_tensor(seq_lens, "seq_lens", "i32", (B,))
    _check_tensor(out, "out", "bf16", (B, T, Hq, D))
    _check(load().la_block_prefill(ctypes.byref(cfg), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                   _ptr(seq_lens), T, int(block_size), _ptr(out),
                                   workspace.data_ptr(), workspace.nbytes, _stream(stream)),
           "la_block_prefill")


def la_block_prefill_selftest_timeout(cfg: Config, q, k_cache, v_cache, seq_lens, block_size: int,
                                      out, workspace: Workspace, wait_limit_ns: int,
                                      stream=None) -> None:
    """Enqueue the prefill failure-detection self-test (one la_block_prefill whose first S
    completion of key half 0 is withheld, every wait limited to `wait_limit_ns`);
    la_pbd_check then gives 6 (LA_ERR_TIMEOUT)."""
    B, T = int(q.shape[0]), int(q.shape[1])
    Hq, Hkv, D, S = cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, cfg.max_seq
    _check_tensor(q, "q", "bf16", (B, T, Hq, D))
    _check_tensor(k_cache, "k_cache", "bf16", (B, Hkv, S, D))
    _check_tensor(v_cache, "v_cache", "bf16", (B, Hkv, S, D))
    _check_tensor(seq_lens, "seq_lens", "i32", (B,))
    _check_tensor(out, "out", "bf16", (B, T, Hq, D))
    _check(load().la_block_prefill_selftest_timeout(
        ctypes.byref(cfg), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), T,
        int(block_size), _ptr(out), workspace.data_ptr(), workspace.nbytes, int(wait_limit_ns),
        _stream(stream)), "la_block_prefill_selftest_timeout")


def _check_paged(cfg, q, k_pool, v_pool, block_table, seq_lens, W, out):
    B, Hq, Hkv, D = cfg.batch, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim
    _check_tensor(q, "q", "bf16", (B, W, Hq, D))
    _check_tensor(out, "out", "bf16", (B, W, Hq, D))
    _check_tensor(k_pool, "k_pool", "bf16")
    _check_tensor(v_pool, "v_pool", "bf16", tuple(k_pool.shape))
    if k_pool.dim() != 4 or k_pool.shape[1] != Hkv or k_pool.shape[3] != D:
        raise ValueError(f"k_pool: expected [num_pages, {Hkv}, page_size, {D}], got {tuple(k_pool.shape)}")
    _check_tensor(block_table, "block_table", "i32")
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError(f"block_table: expected [{B}, pages_per_seq], got {tuple(block_table.shape)}")
    _check_tensor(seq_lens, "seq_lens", "i32", (B,))
    return int(k_pool.shape[0]), int(k_pool.shape[2]), int(block_table.shape[1])


def la_pbd_attn_paged(cfg: Config, q, k_pool, v_pool, block_table, seq_lens, window_len: int,
                      out, workspace: Workspace, stream=None) -> None:
    """Window attention over paged caches: pools [num_pages, Hkv, page_size, D], block_table
    [B, pages_per_seq] (page of each page_size run of keys)."""
    W = int(window_len)
    num_pages, page_size, pps = _check_paged(cfg, q, k_pool, v_pool, block_table, seq_lens, W, out)
    _check(load().la_pbd_attn_paged(ctypes.byref(cfg), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                    _ptr(block_table), pps, page_size, num_pages, _ptr(seq_lens),
                                    W, _ptr(out), workspace.data_ptr(), workspace.nbytes,
                                    _stream(stream)), "la_pbd_attn_paged")


def la_pbd_step_paged(cfg: Config, q, k_new, v_new, k_pool, v_pool, block_table, seq_lens,
                      window_len: int, out, workspace: Workspace, stream=None) -> None:
    """Append the window into its pages, then window attention over the paged caches (one
    launch)."""
    W = int(window_len)
    num_pages, page_size, pps = _check_paged(cfg, q, k_pool, v_pool, block_table, seq_lens, W, out)
    _check_tensor(k_new, "k_new", "bf16", (cfg.batch, W, cfg.num_kv_heads, cfg.head_dim))
    _check_tensor(v_new, "v_new", "bf16", (cfg.batch, W, cfg.num_kv_heads, cfg.head_dim))
    _check(load().la_pbd_step_paged(ctypes.byref(cfg), _ptr(q), _ptr(k_new), _ptr(v_new),
                                    _ptr(k_pool), _ptr(v_pool), _ptr(block_table), pps, page_size,
                                    num_pages, _ptr(seq_lens), W, _ptr(out), workspace.data_ptr(),
                                    workspace.nbytes, _stream(stream)), "la_pbd_step_paged")
