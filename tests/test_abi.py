"""The C-ABI library on the CPU: it loads, exports every declared symbol, and
its host-only calls (layout, chunks, workspace size, validation that
happens before any CUDA call) behave as include/onebit.h states.  No
compute call runs here."""
import ctypes
import os
import re

import pytest

import error_compensated_bit_adam_b200 as ob
from error_compensated_bit_adam_b200 import _binding as B
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "onebit.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^OB_API\s+[\w\s\*]*?\b(ob_\w+)\s*\(", text, re.M)))


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    L = B.lib()
    for name in names:
        assert hasattr(L, name), name
    assert sorted(B.EXPORTS) == names


def test_abi_version_and_status_strings():
    assert B.ob_abi_version() == B.OB_ABI_VERSION
    for code, name in [(0, "OB_OK"), (1, "OB_ERR_INVALID_ARG"), (2, "OB_ERR_PHASE"),
                       (3, "OB_ERR_ALIGN"), (4, "OB_ERR_WORKSPACE"), (5, "OB_ERR_OOM"),
                       (6, "OB_ERR_CUDA"), (7, "OB_ERR_DEVICE_TIMEOUT")]:
        assert B.ob_status_string(code) == name
    assert B.ob_status_string(99) == "OB_UNKNOWN_STATUS"
    assert [B.ob_kernel_name(k) for k in range(B.OB_NUM_KERNELS)] == [
        "ob_warmup_kernel", "ob_freeze_kernel", "ob_pack_kernel", "ob_scale_kernel:worker",
        "ob_server_kernel", "ob_scale_kernel:server", "ob_apply_kernel"]
    assert B.ob_kernel_name(B.OB_NUM_KERNELS) is None


def test_layout_pads_each_tensor_to_128():
    numel = [1, 0, 127, 128, 129, 4096, 5]
    offs, total = B.ob_layout(numel)
    assert offs == [0, 128, 128, 256, 384, 640, 4736]
    assert total == 4864
    for o in offs:
        assert o % B.OB_TENSOR_ALIGN == 0


def test_chunk_range_agrees_with_oracle():
    o = oracle.default()
    for W in (1, 2, 3, 4, 5, 8, 16, 31, 32, 63, 64):
        for n in (0, 1, 31, 32, 33, 100, 127, 128, 129, 1000, 4095, 4096, 4097, 65537, 1 << 20,
                  1_000_003, 335_544_320):
            for j in range(W):
                assert B.ob_chunk_range(n, W, j) == o.chunk_range(n, W, j), (n, W, j)


def test_workspace_bytes_accounts_for_every_state_buffer():
    n = 1 << 20
    for W in (1, 4, 64):
        ws = B.ob_workspace_bytes([n], W)
        # m, v, W error buffers, y: 4 bytes each per element; signs W/8 + 1/8
        assert ws >= (3 + W) * 4 * n + (W + 1) * n // 8
        assert ws < (3 + W) * 4 * n + (W + 1) * n // 8 + (W + 1) * 8 * (n // 4096 + W) + (16 << 20)


@pytest.mark.parametrize("numel,W", [([], 4), ([-1], 4), ([10], 0), ([10], 65)])
def test_invalid_lists_are_rejected(numel, W):
    with pytest.raises(B.OnebitError) as ei:
        B.ob_workspace_bytes(numel, W)
    assert ei.value.status == B.OB_ERR_INVALID_ARG


def test_chunk_range_rejects_bad_arguments():
    for args in [(-1, 4, 0), (10, 0, 0), (10, 65, 0), (10, 4, 4), (10, 4, -1)]:
        with pytest.raises(B.OnebitError) as ei:
            B.ob_chunk_range(*args)
        assert ei.value.status == B.OB_ERR_INVALID_ARG


def _create(numel, W, params=256, ws=256, ws_bytes=None, out=True):
    L = B.lib()
    arr = (ctypes.c_int64 * len(numel))(*numel)
    handle = ctypes.c_void_p()
    if ws_bytes is None:
        ws_bytes = 1 << 62
    return L.ob_create(len(numel), arr, W, 0.9, 0.999, 1e-8, 1e-4, params, ws, ws_bytes, None,
                       ctypes.byref(handle) if out else None)


def test_create_validates_before_touching_the_gpu():
    assert _create([100], 4, out=False) == B.OB_ERR_INVALID_ARG
    assert _create([100], 4, params=None) == B.OB_ERR_INVALID_ARG
    assert _create([100], 4, ws=None) == B.OB_ERR_INVALID_ARG
    assert _create([100], 4, params=256 + 4) == B.OB_ERR_ALIGN
    assert _create([100], 4, ws=256 + 16) == B.OB_ERR_ALIGN
    assert _create([100], 0) == B.OB_ERR_INVALID_ARG
    assert _create([100], 65) == B.OB_ERR_INVALID_ARG
    assert _create([-5], 4) == B.OB_ERR_INVALID_ARG
    need = B.ob_workspace_bytes([100], 4)
    assert _create([100], 4, ws_bytes=need - 1) == B.OB_ERR_WORKSPACE
    L = B.lib()
    handle = ctypes.c_void_p()
    arr = (ctypes.c_int64 * 1)(100)
    for beta1, beta2, eps in [(1.0, 0.999, 1e-8), (0.9, -0.1, 1e-8), (0.9, 0.999, 0.0)]:
        assert L.ob_create(1, arr, 4, beta1, beta2, eps, 1e-4, 256, 256, 1 << 62, None,
                           ctypes.byref(handle)) == B.OB_ERR_INVALID_ARG


def test_injected_host_allocation_failure():
    B.ob_test_fail_host_alloc(1)
    with pytest.raises(B.OnebitError) as ei:
        B.ob_workspace_bytes([1000, 2000], 4)
    assert ei.value.status == B.OB_ERR_OOM
    B.ob_test_fail_host_alloc(2)
    assert _create([1000], 4) == B.OB_ERR_OOM
    B.ob_test_fail_host_alloc(0)
    assert B.ob_workspace_bytes([1000, 2000], 4) > 0


def test_unknown_or_destroyed_context_is_rejected():
    L = B.lib()
    bogus = ctypes.c_void_p(0x1000)
    assert L.ob_freeze_variance(bogus) == B.OB_ERR_INVALID_ARG
    assert L.ob_compressed_step(bogus, None) == B.OB_ERR_INVALID_ARG
    assert L.ob_freeze_variance(None) == B.OB_ERR_INVALID_ARG
    assert L.ob_worker_stage(bogus, None, 0, 1) == B.OB_ERR_INVALID_ARG
    assert L.ob_server_stage(bogus) == B.OB_ERR_INVALID_ARG
    assert L.ob_apply_update(bogus) == B.OB_ERR_INVALID_ARG
    assert L.ob_set_server_shard(bogus, 1, 0) == B.OB_ERR_INVALID_ARG
    out_p, out_n = ctypes.c_void_p(), ctypes.c_size_t()
    assert L.ob_worker_exchange_buffers(bogus, ctypes.byref(out_p), ctypes.byref(out_n),
                                        ctypes.byref(out_p), ctypes.byref(out_n)) == B.OB_ERR_INVALID_ARG
    L.ob_destroy(bogus)  # ignored
    L.ob_destroy(None)


def test_product_package_does_not_touch_the_oracle():
    pkg = os.path.join(ROOT, "error_compensated_bit_adam_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".c")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"\boracle\b", text.replace("the oracle", "")), f


def test_binding_constants_match_the_header_defines():
    """Every integer #define of include/onebit.h has the binding's value."""
    text = open(HEADER).read()
    defines = re.findall(r"^#define\s+(OB_\w+)\s+\(?\(?(?:int64_t\))?\s*([0-9x]+)\s*(?:<<\s*(\d+))?\)?", text, re.M)
    assert defines
    for name, value, shift in defines:
        v = int(value, 0) << (int(shift) if shift else 0)
        assert getattr(B, name) == v, name
    assert {"OB_LAYERWISE_OFF", "OB_LAYERWISE_STEP", "OB_LAYERWISE_FROZEN"} <= {d[0] for d in defines}
    assert [B.layerwise_mode(m) for m in (False, True, "off", "step", "frozen", 2)] == [0, 1, 0, 1, 2, 2]
    with pytest.raises(ValueError):
        B.layerwise_mode("sometimes")
