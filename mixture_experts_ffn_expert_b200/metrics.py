"""Work accounting used to turn measured times into throughput figures.

FLOPs count one multiply-add as 2 FLOPs ("MoE：细粒度专家与共享专家（shared
expert）", budget section: an expert costs 3*d*f multiply-adds per token) over
the selected experts only (no padding, none of the dense all-expert work
routing avoids). Bytes count the HBM traffic a perfect implementation cannot
avoid: x in and out (bf16), the router matrix, the shared weights and every
routed expert that received at least one token. Intermediates (grouped rows,
hidden activations) are implementation choices and are not counted at the
layer level; per kernel, the bytes are the kernel's own inputs and outputs.
"""
from __future__ import annotations

from typing import Optional, Tuple

from .inputs import LayerShape

__all__ = ["layer_flops", "layer_bytes", "kernel_work"]


def layer_flops(shape: LayerShape, T: Optional[int] = None) -> int:
    """Router 2*T*d*N_r + routed 6*T*k*d*f + shared 6*T*d*N_s*f."""
    T = shape.T if T is None else T
    return (2 * T * shape.d * shape.n_routed
            + 6 * T * shape.top_k * shape.d * shape.f
            + 6 * T * shape.d * shape.n_shared * shape.f)


def layer_bytes(shape: LayerShape, touched_experts: int,
                T: Optional[int] = None) -> int:
    """2 bytes x (T*d in + T*d out + N_r*d router + 3*d*N_s*f shared
    + touched*3*d*f routed)."""
    T = shape.T if T is None else T
    d, f = shape.d, shape.f
    return 2 * (2 * T * d + shape.n_routed * d + 3 * d * shape.n_shared * f
                + touched_experts * 3 * d * f)


def kernel_work(name: str, shape: LayerShape, T: int, touched: int) -> Tuple[int, int]:
    """(flops, bytes) one launch of the named kernel cannot avoid: its inputs,
    outputs and weights. `touched` = routed experts that received a row. A GEMM
    variant tag ("[pair]", "[pair512]") does not change the work, except
    "[+shared]": the shared expert's GEMM merged into the routed launch."""
    d, f, n, k = shape.d, shape.f, shape.n_routed, shape.top_k
    A, nsf = T * k, shape.n_shared * shape.f
    base, _, tag = name.partition("[")
    table = {
        "router_gemm": (2 * T * d * n, 2 * n * d + 2 * T * d + 4 * T * n),
        "route_topk": (0, 4 * T * n + 8 * A),
        # fused router: scores, softmax, top-k, gates and the chunk histogram
        "route_fused": (2 * T * d * n, 2 * n * d + 2 * T * d + 8 * A),
        "route_scan": (0, 0),
        "route_scatter": (0, 2 * T * d + 2 * A * d + 12 * A),
        "grouped_gate_up": (4 * A * d * f, touched * 4 * d * f + 2 * A * d + 2 * A * f),
        "grouped_down": (2 * A * d * f, touched * 2 * d * f + 2 * A * f + 2 * A * d),
        "shared_gate_up": (4 * T * d * nsf, 4 * nsf * d + 2 * T * d + 2 * T * nsf),
        "shared_down": (2 * T * d * nsf, 2 * nsf * d + 2 * T * nsf + 4 * T * d),
        "combine": (0, 2 * A * d + (4 * T * d if nsf else 0) + 2 * T * d + 8 * A),
    }
    fl, by = table.get(base, (0, 0))
    if "+shared" in tag:
        sf, sb = table["shared_" + base.split("_", 1)[1]]
        fl, by = fl + sf, by + sb
    return fl, by
