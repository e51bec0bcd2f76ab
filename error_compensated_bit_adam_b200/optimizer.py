"""User-facing wrapper of a libonebit context.

PyTorch supplies the device memory (parameters, workspace, staging) and the
CUDA stream; every step runs in libonebit's kernels through the C ABI.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Union

import numpy as np
import torch

from . import _binding as B

_STATE_DTYPE = {
    B.OB_STATE_P: np.float32, B.OB_STATE_M: np.float32, B.OB_STATE_V: np.float32,
    B.OB_STATE_D: np.float32, B.OB_STATE_E_WORKER: np.float32, B.OB_STATE_E_SERVER: np.float32,
    B.OB_STATE_S_WORKER: np.float32, B.OB_STATE_S_SERVER: np.float32,
    B.OB_STATE_BITS_WORKER: np.uint32, B.OB_STATE_BITS_SERVER: np.uint32,
    B.OB_STATE_STEP: np.int64, B.OB_STATE_RATIO: np.float32,
}

Grads = Union[torch.Tensor, Sequence[torch.Tensor]]


class OneBitAdam:
    """1-bit Adam over W data-parallel workers simulated on one GPU.

    numel: element counts of the tensors.  params: a float32 CUDA tensor of
    n_padded elements in the padded layout (see ``layout``), updated in
    place; a zero tensor is made if omitted.  Gradients are passed as a
    [W, n_padded] float32 CUDA tensor or a list of W such vectors.
    layerwise=True (or "step") runs 1-bit LAMB instead (ob_set_layerwise):
    every tensor's step scaled by its trust ratio ||p|| / ||u||, recomputed
    every step; layerwise="frozen" keeps the last warmup step's ratios from
    the freeze on.
    """

    def __init__(self, numel: Sequence[int], W: int, *, beta1: float = 0.9, beta2: float = 0.999,
                 eps: float = 1e-8, lr: float = 1e-4, params: Optional[torch.Tensor] = None,
                 device: Union[str, torch.device, None] = None,
                 stream: Optional[torch.cuda.Stream] = None, layerwise: Union[bool, str] = False):
        self.numel = [int(n) for n in numel]
        self.W = int(W)
        self.offsets, self.n_padded = B.ob_layout(self.numel)
        self.device = torch.device(device if device is not None else
                                   (params.device if params is not None else "cuda"))
        if params is None:
            params = torch.zeros(self.n_padded, dtype=torch.float32, device=self.device)
        if (params.dtype != torch.float32 or not params.is_cuda or not params.is_contiguous()
                or params.numel() != self.n_padded):
            raise ValueError(f"params must be a contiguous float32 CUDA tensor of {self.n_padded} "
                             "elements")
        self.params = params
        self.workspace_bytes = B.ob_workspace_bytes(self.numel, self.W)
        self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=self.device)
        self.stream = stream if stream is not None else torch.cuda.current_stream(self.device)
        self._staging: Optional[torch.Tensor] = None
        self._ptr_cache = {}
        self.ctx = 0
        with torch.cuda.device(self.device):
            self.ctx = B.ob_create(self.numel, self.W, beta1, beta2, eps, lr, params.data_ptr(),
                                   self.workspace.data_ptr(), self.workspace_bytes,
                                   self.stream.cuda_stream)
            if B.layerwise_mode(layerwise) != B.OB_LAYERWISE_OFF:
                B.ob_set_layerwise(self.ctx, layerwise)

    # ------------------------------------------------------------ helpers
    def layout(self):
        return self.offsets, self.n_padded

    def _ptrs(self, grads: Grads):
        """The W gradient pointers as a C array.  A [W, n_padded] tensor is
        checked once and its rows' addresses computed from its base; the
        array is kept per base address, so stepping on the same gradient
        buffers again costs no marshalling."""
        if isinstance(grads, torch.Tensor):
            if (grads.dtype != torch.float32 or not grads.is_cuda or not grads.is_contiguous()
                    or tuple(grads.shape) != (self.W, self.n_padded)):
                raise ValueError(f"gradients must be a contiguous float32 CUDA tensor of shape "
                                 f"({self.W}, {self.n_padded}) or a list of {self.W} vectors")
            base = grads.data_ptr()
            arr = self._ptr_cache.get(base)
            if arr is None:
                if len(self._ptr_cache) >= 8:
                    self._ptr_cache.clear()
                row = self.n_padded * 4
                arr = self._ptr_cache[base] = B.pointer_array([base + w * row for w in range(self.W)])
            return arr
        rows = list(grads)
        if len(rows) != self.W:
            raise ValueError(f"expected {self.W} gradients")
        for g in rows:
            if (g.dtype != torch.float32 or not g.is_cuda or not g.is_contiguous()
                    or g.numel() != self.n_padded):
                raise ValueError("each gradient must be a contiguous float32 CUDA vector of "
                                 f"{self.n_padded} elements")
        return [g.data_ptr() for g in rows]

    # -------------------------------------------------------------- steps
    def warmup_step(self, grads: Grads) -> None:
        B.ob_warmup_adam_step(self.ctx, self._ptrs(grads))

    def freeze(self) -> None:
        B.ob_freeze_variance(self.ctx)

    def step(self, grads: Grads) -> None:
        B.ob_compressed_step(self.ctx, self._ptrs(grads))

    def step_host(self, host_grads: torch.Tensor, server_scales: Optional[np.ndarray] = None) -> None:
        """Compressed step with gradients in (preferably pinned) host memory,
        a [W, n_padded] float32 CPU tensor.  Blocks until the step is done."""
        if (host_grads.is_cuda or host_grads.dtype != torch.float32
                or not host_grads.is_contiguous() or tuple(host_grads.shape) != (self.W, self.n_padded)):
            raise ValueError("host_grads must be a contiguous float32 CPU tensor [W, n_padded]")
        if self._staging is None:
            nbytes = B.ob_host_staging_bytes(self.ctx)
            self._staging = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        out = None
        if server_scales is not None:
            assert server_scales.dtype == np.float32 and server_scales.size == len(self.numel) * self.W
            out = server_scales.ctypes.data
        B.ob_compressed_step_host(self.ctx, [host_grads[w].data_ptr() for w in range(self.W)],
                                  self._staging.data_ptr(), self._staging.numel(), out)

    # -------------------------------------------------------------- state
    def _shape(self, kind: int):
        T, W, n = len(self.numel), self.W, self.n_padded
        if kind in (B.OB_STATE_S_WORKER,):
            return (W, T)
        if kind in (B.OB_STATE_S_SERVER,):
            return (T, W)
        if kind in (B.OB_STATE_BITS_WORKER, B.OB_STATE_BITS_SERVER):
            return (n // 32,)
        if kind == B.OB_STATE_STEP:
            return (3,)
        if kind == B.OB_STATE_RATIO:
            return (T,)
        return (n,)

    def read(self, kind: int, index: int = 0) -> np.ndarray:
        out = np.empty(self._shape(kind), _STATE_DTYPE[kind])
        B.ob_read_state(self.ctx, kind, index, out.ctypes.data, out.nbytes)
        return out

    def write(self, kind: int, index: int, value: np.ndarray) -> None:
        arr = np.ascontiguousarray(value, _STATE_DTYPE[kind]).reshape(self._shape(kind))
        B.ob_write_state(self.ctx, kind, index, arr.ctypes.data, arr.nbytes)

    def set_lr(self, lr: float) -> None:
        B.ob_set_lr(self.ctx, lr)

    def graph(self, on: bool = True) -> None:
        """Replay the compressed step as one CUDA graph (small tensor lists)."""
        B.ob_graph_enable(self.ctx, on)

    def profile(self, on: bool = True) -> None:
        B.ob_profile_enable(self.ctx, on)

    def profile_read(self, reset: bool = False):
        ms, n = B.ob_profile_read(self.ctx, reset)
        return {B.ob_kernel_name(k): (ms[k], n[k]) for k in range(B.OB_NUM_KERNELS)}

    def close(self) -> None:
        if self.ctx:
            B.ob_destroy(self.ctx)
            self.ctx = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
