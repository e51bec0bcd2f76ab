"""ctypes binding of libonebit (include/onebit.h), one Python function per C
entry point, with the same names.  Marshalling only: every step of the
method runs in the library's CUDA kernels.  A non-OK status raises
OnebitError; there is no fallback of any kind when the library is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(HERE, "libonebit.so")

OB_ABI_VERSION = 1
OB_MAX_WORKERS = 64
OB_TENSOR_ALIGN = 128

OB_OK = 0
OB_ERR_INVALID_ARG = 1
OB_ERR_PHASE = 2
OB_ERR_ALIGN = 3
OB_ERR_WORKSPACE = 4
OB_ERR_OOM = 5
OB_ERR_CUDA = 6
OB_ERR_DEVICE_TIMEOUT = 7

OB_STATE_P = 0
OB_STATE_M = 1
OB_STATE_V = 2
OB_STATE_D = 3
OB_STATE_E_WORKER = 4
OB_STATE_E_SERVER = 5
OB_STATE_S_WORKER = 6
OB_STATE_S_SERVER = 7
OB_STATE_BITS_WORKER = 8
OB_STATE_BITS_SERVER = 9
OB_STATE_STEP = 10
OB_STATE_RATIO = 11

OB_STATIC_MAX_ELEMENTS = 1 << 26

OB_K_WARMUP = 0
OB_K_FREEZE = 1
OB_K_PACK = 2
OB_K_PACK_SCALE = 3
OB_K_SERVER = 4
OB_K_SERVER_SCALE = 5
OB_K_APPLY = 6
OB_NUM_KERNELS = 7

# Every symbol include/onebit.h declares.
EXPORTS = (
    "ob_status_string", "ob_abi_version", "ob_layout", "ob_chunk_range", "ob_workspace_bytes",
    "ob_create", "ob_destroy", "ob_warmup_adam_step", "ob_freeze_variance", "ob_compressed_step",
    "ob_host_staging_bytes", "ob_compressed_step_host", "ob_read_state", "ob_write_state",
    "ob_profile_enable", "ob_profile_read", "ob_kernel_name", "ob_test_fail_host_alloc",
    "ob_onebit_compress_static", "ob_set_lr", "ob_graph_enable",
    "ob_server_shard_range", "ob_set_server_shard", "ob_worker_stage", "ob_worker_exchange_buffers",
    "ob_server_stage", "ob_server_exchange_buffers", "ob_apply_update", "ob_set_layerwise",
    "ob_set_peer_words",
)


__all__ = [name for name in EXPORTS] + [
    "OnebitError", "lib", "status_name", "LIBRARY", "pointer_array",
    "OB_ABI_VERSION", "OB_MAX_WORKERS", "OB_TENSOR_ALIGN", "OB_STATIC_MAX_ELEMENTS",
    "OB_OK", "OB_ERR_INVALID_ARG", "OB_ERR_PHASE", "OB_ERR_ALIGN", "OB_ERR_WORKSPACE",
    "OB_ERR_OOM", "OB_ERR_CUDA", "OB_ERR_DEVICE_TIMEOUT",
    "OB_STATE_P", "OB_STATE_M", "OB_STATE_V", "OB_STATE_D", "OB_STATE_E_WORKER",
    "OB_STATE_E_SERVER", "OB_STATE_S_WORKER", "OB_STATE_S_SERVER", "OB_STATE_BITS_WORKER",
    "OB_STATE_BITS_SERVER", "OB_STATE_STEP", "OB_STATE_RATIO",
    "OB_LAYERWISE_OFF", "OB_LAYERWISE_STEP", "OB_LAYERWISE_FROZEN", "layerwise_mode",
    "OB_K_WARMUP", "OB_K_FREEZE", "OB_K_PACK", "OB_K_PACK_SCALE", "OB_K_SERVER",
    "OB_K_SERVER_SCALE", "OB_K_APPLY", "OB_NUM_KERNELS",
]


class OnebitError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = int(status)
        self.call = call
        super().__init__(f"{call}: {status_name(status)}")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libonebit.so (built in-tree).  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIBRARY):
        raise RuntimeError(
            f"{LIBRARY} is not built; run `python -m error_compensated_bit_adam_b200.build` "
            "(or __graft_entry__.build()).  There is no fallback implementation.")
    L = ctypes.CDLL(LIBRARY)
    i32, i64, f32, vp, sz = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
    P64 = ctypes.POINTER(i64)
    sig = {
        "ob_status_string": (ctypes.c_char_p, [i32]),
        "ob_abi_version": (i32, []),
        "ob_layout": (i32, [i32, P64, P64, P64]),
        "ob_chunk_range": (i32, [i64, i32, i32, P64, P64]),
        "ob_workspace_bytes": (i32, [i32, P64, i32, ctypes.POINTER(sz)]),
        "ob_create": (i32, [i32, P64, i32, f32, f32, f32, f32, vp, vp, sz, vp, ctypes.POINTER(vp)]),
        "ob_destroy": (None, [vp]),
        "ob_warmup_adam_step": (i32, [vp, vp]),
        "ob_freeze_variance": (i32, [vp]),
        "ob_compressed_step": (i32, [vp, vp]),
        "ob_host_staging_bytes": (i32, [vp, ctypes.POINTER(sz)]),
        "ob_compressed_step_host": (i32, [vp, vp, vp, sz, vp]),
        "ob_read_state": (i32, [vp, i32, i32, vp, sz]),
        "ob_write_state": (i32, [vp, i32, i32, vp, sz]),
        "ob_profile_enable": (i32, [vp, i32]),
        "ob_profile_read": (i32, [vp, ctypes.POINTER(ctypes.c_double), P64, i32]),
        "ob_kernel_name": (ctypes.c_char_p, [i32]),
        "ob_test_fail_host_alloc": (None, [i32]),
        "ob_onebit_compress_static": (i32, [vp, i64, vp, vp, vp, vp]),
        "ob_set_lr": (i32, [vp, f32]),
        "ob_graph_enable": (i32, [vp, i32]),
        "ob_server_shard_range": (i32, [i32, P64, i32, i32, i32, ctypes.POINTER(i32),
                                        ctypes.POINTER(i32), P64, P64]),
        "ob_set_server_shard": (i32, [vp, i32, i32]),
        "ob_worker_stage": (i32, [vp, vp, i32, i32]),
        "ob_worker_exchange_buffers": (i32, [vp, ctypes.POINTER(vp), ctypes.POINTER(sz),
                                             ctypes.POINTER(vp), ctypes.POINTER(sz)]),
        "ob_server_stage": (i32, [vp]),
        "ob_server_exchange_buffers": (i32, [vp, ctypes.POINTER(vp), ctypes.POINTER(sz),
                                             ctypes.POINTER(vp), ctypes.POINTER(sz)]),
        "ob_apply_update": (i32, [vp]),
        "ob_set_layerwise": (i32, [vp, i32]),
        "ob_set_peer_words": (i32, [vp, i32, vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    if L.ob_abi_version() != OB_ABI_VERSION:
        raise RuntimeError("libonebit ABI version mismatch")
    _lib = L
    return L


def status_name(status: int) -> str:
    try:
        return lib().ob_status_string(int(status)).decode()
    except Exception:  # the library may be what failed to load
        return f"status {status}"


def _check(status: int, call: str) -> None:
    if status != OB_OK:
        raise OnebitError(status, call)


def _i64_array(values: Sequence[int]):
    arr = (ctypes.c_int64 * max(1, len(values)))(*[int(v) for v in values])
    return arr


def _ptrs(ptrs: Sequence[int]):
    """A C array of pointers (a ctypes pointer array is passed through)."""
    if isinstance(ptrs, ctypes.Array):
        return ptrs
    arr = (ctypes.c_void_p * max(1, len(ptrs)))()
    for i, p in enumerate(ptrs):
        arr[i] = int(p)
    return arr


def pointer_array(ptrs: Sequence[int]):
    """A reusable C array of device pointers for the step calls."""
    return _ptrs(list(ptrs))


# --------------------------------------------------------------- host only

def ob_status_string(status: int) -> str:
    return lib().ob_status_string(int(status)).decode()


def ob_abi_version() -> int:
    return int(lib().ob_abi_version())


def ob_layout(numel: Sequence[int]) -> Tuple[List[int], int]:
    """Tensor offsets and n_padded of the padded layout."""
    n = len(numel)
    offs = (ctypes.c_int64 * max(1, n))()
    total = ctypes.c_int64()
    _check(lib().ob_layout(n, _i64_array(numel), offs, ctypes.byref(total)), "ob_layout")
    return [int(offs[i]) for i in range(n)], int(total.value)


def ob_chunk_range(numel: int, W: int, j: int) -> Tuple[int, int]:
    b, e = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().ob_chunk_range(int(numel), int(W), int(j), ctypes.byref(b), ctypes.byref(e)),
           "ob_chunk_range")
    return int(b.value), int(e.value)


def ob_workspace_bytes(numel: Sequence[int], W: int) -> int:
    out = ctypes.c_size_t()
    _check(lib().ob_workspace_bytes(len(numel), _i64_array(numel), int(W), ctypes.byref(out)),
           "ob_workspace_bytes")
    return int(out.value)


def ob_kernel_name(kernel_id: int) -> Optional[str]:
    r = lib().ob_kernel_name(int(kernel_id))
    return None if r is None else r.decode()


def ob_test_fail_host_alloc(countdown: int) -> None:
    lib().ob_test_fail_host_alloc(int(countdown))


# ----------------------------------------------------------------- context

def ob_create(numel: Sequence[int], W: int, beta1: float, beta2: float, eps: float, lr: float,
              d_params: int, d_workspace: int, workspace_bytes: int, cuda_stream: int) -> int:
    """Returns the context handle (an opaque integer)."""
    out = ctypes.c_void_p()
    _check(lib().ob_create(len(numel), _i64_array(numel), int(W), float(beta1), float(beta2),
                           float(eps), float(lr), int(d_params), int(d_workspace),
                           int(workspace_bytes), int(cuda_stream), ctypes.byref(out)), "ob_create")
    return int(out.value)


def ob_destroy(ctx: int) -> None:
    lib().ob_destroy(int(ctx) if ctx else None)


def ob_warmup_adam_step(ctx: int, d_grads: Sequence[int]) -> None:
    _check(lib().ob_warmup_adam_step(ctx, _ptrs(d_grads)), "ob_warmup_adam_step")


def ob_freeze_variance(ctx: int) -> None:
    _check(lib().ob_freeze_variance(ctx), "ob_freeze_variance")


def ob_compressed_step(ctx: int, d_grads: Sequence[int]) -> None:
    _check(lib().ob_compressed_step(ctx, _ptrs(d_grads)), "ob_compressed_step")


def ob_host_staging_bytes(ctx: int) -> int:
    out = ctypes.c_size_t()
    _check(lib().ob_host_staging_bytes(ctx, ctypes.byref(out)), "ob_host_staging_bytes")
    return int(out.value)


def ob_compressed_step_host(ctx: int, h_grads: Sequence[int], d_staging: int, staging_bytes: int,
                            h_server_scales: Optional[int]) -> None:
    _check(lib().ob_compressed_step_host(ctx, _ptrs(h_grads), int(d_staging), int(staging_bytes),
                                         int(h_server_scales) if h_server_scales else None),
           "ob_compressed_step_host")


def ob_read_state(ctx: int, kind: int, index: int, host_dst: int, nbytes: int) -> None:
    _check(lib().ob_read_state(ctx, int(kind), int(index), int(host_dst), int(nbytes)),
           "ob_read_state")


def ob_write_state(ctx: int, kind: int, index: int, host_src: int, nbytes: int) -> None:
    _check(lib().ob_write_state(ctx, int(kind), int(index), int(host_src), int(nbytes)),
           "ob_write_state")


def ob_set_lr(ctx: int, lr: float) -> None:
    _check(lib().ob_set_lr(ctx, float(lr)), "ob_set_lr")


# ob_set_layerwise modes (include/onebit.h)
OB_LAYERWISE_OFF, OB_LAYERWISE_STEP, OB_LAYERWISE_FROZEN = 0, 1, 2


def layerwise_mode(mode) -> int:
    """An OB_LAYERWISE_* mode from an int, a bool (True: per-step ratios) or
    a name ("off", "step", "frozen")."""
    if isinstance(mode, bool) or mode is None:
        return OB_LAYERWISE_STEP if mode else OB_LAYERWISE_OFF
    if isinstance(mode, str):
        names = {"off": OB_LAYERWISE_OFF, "step": OB_LAYERWISE_STEP, "frozen": OB_LAYERWISE_FROZEN}
        if mode not in names:
            raise ValueError(f"layerwise mode {mode!r}: one of {sorted(names)}")
        return names[mode]
    return int(mode)


def ob_set_layerwise(ctx: int, mode) -> None:
    _check(lib().ob_set_layerwise(ctx, layerwise_mode(mode)), "ob_set_layerwise")


def ob_graph_enable(ctx: int, on: bool) -> None:
    _check(lib().ob_graph_enable(ctx, 1 if on else 0), "ob_graph_enable")


def ob_profile_enable(ctx: int, on: bool) -> None:
    _check(lib().ob_profile_enable(ctx, 1 if on else 0), "ob_profile_enable")


def ob_profile_read(ctx: int, reset: bool = False) -> Tuple[List[float], List[int]]:
    ms = (ctypes.c_double * OB_NUM_KERNELS)()
    n = (ctypes.c_int64 * OB_NUM_KERNELS)()
    _check(lib().ob_profile_read(ctx, ms, n, 1 if reset else 0), "ob_profile_read")
    return [float(v) for v in ms], [int(v) for v in n]


# ------------------------------------------------------------ split step

def ob_server_shard_range(numel: Sequence[int], W: int, n_shards: int,
                          shard: int) -> Tuple[int, int, int, int]:
    """(chunk_begin, chunk_end, word_begin, word_end) of one shard."""
    cb, ce = ctypes.c_int(), ctypes.c_int()
    wb, we = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().ob_server_shard_range(len(numel), _i64_array(numel), int(W), int(n_shards), int(shard),
                                       ctypes.byref(cb), ctypes.byref(ce), ctypes.byref(wb),
                                       ctypes.byref(we)), "ob_server_shard_range")
    return cb.value, ce.value, wb.value, we.value


def ob_set_server_shard(ctx: int, n_shards: int, shard: int) -> None:
    _check(lib().ob_set_server_shard(ctx, int(n_shards), int(shard)), "ob_set_server_shard")


def ob_worker_stage(ctx: int, d_grads: Sequence[int], w_begin: int, w_count: int) -> None:
    _check(lib().ob_worker_stage(ctx, _ptrs(d_grads), int(w_begin), int(w_count)), "ob_worker_stage")


def _buffers(fn, ctx: int, call: str) -> Tuple[int, int, int, int]:
    a, b = ctypes.c_void_p(), ctypes.c_void_p()
    na, nb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(fn(ctx, ctypes.byref(a), ctypes.byref(na), ctypes.byref(b), ctypes.byref(nb)), call)
    return int(a.value or 0), int(na.value), int(b.value or 0), int(nb.value)


def ob_worker_exchange_buffers(ctx: int) -> Tuple[int, int, int, int]:
    """(d_bits, bits_row_bytes, d_scales, scales_row_bytes)."""
    return _buffers(lib().ob_worker_exchange_buffers, ctx, "ob_worker_exchange_buffers")


def ob_server_stage(ctx: int) -> None:
    _check(lib().ob_server_stage(ctx), "ob_server_stage")


def ob_server_exchange_buffers(ctx: int) -> Tuple[int, int, int, int]:
    """(d_sbits, sbits_bytes, d_scales, scales_bytes)."""
    return _buffers(lib().ob_server_exchange_buffers, ctx, "ob_server_exchange_buffers")


def ob_apply_update(ctx: int) -> None:
    _check(lib().ob_apply_update(ctx), "ob_apply_update")


def ob_set_peer_words(ctx: int, d_worker_bits: Sequence[int], d_server_bits: Sequence[int]) -> None:
    """Fused word exchanges of the split step (empty lists turn them off)."""
    n = len(d_worker_bits)
    assert len(d_server_bits) == n
    _check(lib().ob_set_peer_words(ctx, n, _ptrs(d_worker_bits) if n else None,
                                   _ptrs(d_server_bits) if n else None), "ob_set_peer_words")


# ------------------------------------------------------ allocation-free call

def ob_onebit_compress_static(d_x: int, n: int, d_bits: int, d_error: int, d_scale: int,
                              cuda_stream: int) -> None:
    """1-bit compression of one device vector with the library's static
    scratch: for callers that cannot allocate device memory."""
    _check(lib().ob_onebit_compress_static(int(d_x) or None, int(n), int(d_bits) or None,
                                           int(d_error) or None, int(d_scale) or None,
                                           int(cuda_stream) or None),
           "ob_onebit_compress_static")
