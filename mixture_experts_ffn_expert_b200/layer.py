"""Torch-facing wrapper of the C ABI: checks tensors, owns the workspace, and
passes data pointers and the current CUDA stream to ``moe_forward``.

PyTorch only provides device memory and streams here; all arithmetic runs in
libmoe_ffn.so. A missing library raises instead of falling back to anything.
"""
from __future__ import annotations

from typing import Dict, Optional

import torch

from .binding import (MOE_OPTION_BIAS_SELECTION_ONLY, MOE_OPTION_CAPACITY_FACTOR_PERMILLE,
                      MOE_OPTION_CTAS_PER_SM, MOE_OPTION_DOWN_TILE_COLS, MOE_OPTION_GATHER_ROWS,
                      MOE_OPTION_EXPERT_CAPACITY, MOE_OPTION_FUSED_ROUTER,
                      MOE_OPTION_MERGE_SHARED, MOE_OPTION_PAIR_MIN_ROWS,
                      MOE_OPTION_INTERLEAVE, MOE_OPTION_SHARED_CONCURRENT,
                      MOE_OPTION_SWIGLU_TILE_COLS, MOE_OPTION_TILE_ROWS, MOE_OPTION_WIDE_TILES,
                      MoEError, Plan)

__all__ = ["MoELayer", "MoEError"]


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


class MoELayer:
    """One MoE feed-forward layer shape bound to a CUDA device.

    ``weights`` holds W_g (N_r, d), W1, W3 (N_r, f, d), W2 (N_r, d, f) and, when
    n_shared > 0, W1s, W3s (N_s*f, d), W2s (d, N_s*f), all bf16 contiguous on
    the device; ``bias`` is an optional fp32 (N_r,) logit bias. ``capacity``
    (seats per expert per forward) or ``capacity_factor`` (the library gives each
    expert ceil(factor * T * top_k / N_r) seats per forward over T tokens) turns
    on token dropping; ``bias_selection_only`` makes the bias choose experts
    without entering the gates; the other options (``fused_router``,
    ``swiglu_tile_cols``, ``tile_rows``, ``interleave``, ``shared_concurrent``,
    ``ctas_per_sm``, ``down_tile_cols``, ``gather_rows`` among them) only select
    kernels, tile orders or streams.
    """

    def __init__(self, d: int, f: int, n_routed: int, top_k: int, n_shared: int,
                 renorm: bool, weights: Dict[str, Optional[torch.Tensor]],
                 bias: Optional[torch.Tensor] = None, device=None,
                 pair_min_rows: Optional[int] = None, wide_tiles: Optional[int] = None,
                 merge_shared: Optional[int] = None, capacity: Optional[int] = None,
                 bias_selection_only: bool = False, capacity_factor: Optional[float] = None,
                 fused_router: Optional[int] = None,
                 swiglu_tile_cols: Optional[int] = None,
                 shared_concurrent: Optional[int] = None,
                 tile_rows: Optional[int] = None, interleave: Optional[int] = None,
                 ctas_per_sm: Optional[int] = None, down_tile_cols: Optional[int] = None,
                 gather_rows: Optional[int] = None):
        dev = torch.device(device) if device is not None else torch.device("cuda")
        if dev.type == "cuda" and dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        if self.device.type != "cuda":
            raise MoEError(2, "MoELayer runs on a CUDA device only")
        with torch.cuda.device(self.device):
            self.plan = Plan(d, f, n_routed, top_k, n_shared, renorm)
        if pair_min_rows is not None:
            self.plan.set_option(MOE_OPTION_PAIR_MIN_ROWS, pair_min_rows)
        if wide_tiles is not None:
            self.plan.set_option(MOE_OPTION_WIDE_TILES, wide_tiles)
        if merge_shared is not None:
            self.plan.set_option(MOE_OPTION_MERGE_SHARED, merge_shared)
        if fused_router is not None:
            self.plan.set_option(MOE_OPTION_FUSED_ROUTER, fused_router)
        if swiglu_tile_cols is not None:
            self.plan.set_option(MOE_OPTION_SWIGLU_TILE_COLS, swiglu_tile_cols)
        if shared_concurrent is not None:
            self.plan.set_option(MOE_OPTION_SHARED_CONCURRENT, shared_concurrent)
        if tile_rows is not None:
            self.plan.set_option(MOE_OPTION_TILE_ROWS, tile_rows)
        if interleave is not None:
            self.plan.set_option(MOE_OPTION_INTERLEAVE, interleave)
        if ctas_per_sm is not None:
            self.plan.set_option(MOE_OPTION_CTAS_PER_SM, ctas_per_sm)
        if down_tile_cols is not None:
            self.plan.set_option(MOE_OPTION_DOWN_TILE_COLS, down_tile_cols)
        if gather_rows is not None:
            self.plan.set_option(MOE_OPTION_GATHER_ROWS, gather_rows)
        # seats per expert per forward (token dropping); None or 0: dropless
        if capacity and capacity_factor:
            raise MoEError(2, "give either capacity or capacity_factor, not both")
        if capacity:
            self.plan.set_option(MOE_OPTION_EXPERT_CAPACITY, capacity)
        if capacity_factor:
            if capacity_factor <= 0:
                raise MoEError(2, "capacity factor must be positive")
            self.plan.set_option(MOE_OPTION_CAPACITY_FACTOR_PERMILLE,
                                 int(round(capacity_factor * 1000)))
        self.bias_selection_only = bool(bias_selection_only)
        if bias_selection_only:
            self.plan.set_option(MOE_OPTION_BIAS_SELECTION_ONLY, 1)
        self.d, self.f, self.n_routed, self.top_k, self.n_shared = d, f, n_routed, top_k, n_shared
        self.renorm = bool(renorm)
        shapes = {"W_g": (n_routed, d), "W1": (n_routed, f, d), "W3": (n_routed, f, d),
                  "W2": (n_routed, d, f)}
        if n_shared > 0:
            shapes.update({"W1s": (n_shared * f, d), "W3s": (n_shared * f, d),
                           "W2s": (d, n_shared * f)})
        self.w: Dict[str, Optional[torch.Tensor]] = {"W1s": None, "W3s": None, "W2s": None}
        for name, shp in shapes.items():
            t = weights.get(name)
            if t is None or tuple(t.shape) != shp or t.dtype != torch.bfloat16 \
                    or not t.is_contiguous() or t.device != self.device:
                raise MoEError(2, f"{name} must be a contiguous bf16 {shp} tensor on {self.device}")
            self.w[name] = t
        self.bias = None
        if bias is not None:
            if tuple(bias.shape) != (n_routed,) or bias.dtype != torch.float32 \
                    or bias.device != self.device or not bias.is_contiguous():
                raise MoEError(2, "bias must be a contiguous fp32 (N_r,) tensor on the device")
            self.bias = bias
        self.plan.set_logit_bias(_ptr(self.bias))
        self.workspace: Optional[torch.Tensor] = None
        self._ws_T = -1

    def ensure_workspace(self, T: int) -> None:
        need = self.plan.workspace_bytes(T)
        if self.workspace is None or self.workspace.numel() < need:
            self.workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=self.device)
            self.plan.set_workspace(self.workspace.data_ptr(), self.workspace.numel())

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """out (T, d) bf16 = shared(x) + sum of gated routed experts, no residual."""
        if x.dim() != 2 or x.shape[1] != self.d or x.dtype != torch.bfloat16 \
                or not x.is_contiguous() or x.device != self.device:
            raise MoEError(2, f"x must be a contiguous bf16 (T, {self.d}) tensor on {self.device}")
        T = x.shape[0]
        if out is None:
            out = torch.empty_like(x)
        self.ensure_workspace(T)
        w = self.w
        stream = torch.cuda.current_stream(self.device).cuda_stream
        self.plan.forward(T, x.data_ptr(), w["W_g"].data_ptr(), w["W1"].data_ptr(),
                          w["W3"].data_ptr(), w["W2"].data_ptr(), _ptr(w["W1s"]),
                          _ptr(w["W3s"]), _ptr(w["W2s"]), out.data_ptr(), stream)
        self._ws_T = T
        return out

    __call__ = forward

    def routing(self) -> Dict[str, torch.Tensor]:
        """idx, w, counts, offsets, perm_src, inv_pos of the last forward (device tensors)."""
        T, k, n = self._ws_T, self.top_k, self.n_routed
        dev = self.device
        r = {"idx": torch.empty((T, k), dtype=torch.int32, device=dev),
             "w": torch.empty((T, k), dtype=torch.float32, device=dev),
             "counts": torch.empty((n,), dtype=torch.int32, device=dev),
             "offsets": torch.empty((n + 1,), dtype=torch.int32, device=dev),
             "perm_src": torch.empty((T * k,), dtype=torch.int32, device=dev),
             "inv_pos": torch.empty((T, k), dtype=torch.int32, device=dev)}
        stream = torch.cuda.current_stream(dev).cuda_stream
        self.plan.get_routing(T, r["idx"].data_ptr(), r["w"].data_ptr(), r["counts"].data_ptr(),
                              r["offsets"].data_ptr(), stream)
        self.plan.get_permutation(T, r["perm_src"].data_ptr(), r["inv_pos"].data_ptr(), stream)
        return r

    def capacity_seats(self, T: int) -> int:
        """Seats per expert a forward over T tokens uses (0: dropless)."""
        return self.plan.capacity_seats(T)

    def device_status(self) -> int:
        return self.plan.device_status()
