"""Work accounting used to turn measured times into throughput figures.

FLOPs count one multiply-add as 2 FLOPs over the selected experts only (no
padding, none of the dense all-expert work routing avoids). Bytes count the
HBM traffic a perfect implementation cannot avoid: x in and out back (bf16),
the router matrix, the shared weights and every routed expert that received at
least one token. Intermediates (grouped rows, hidden activations) are
implementation choices and are not counted.
"""
from __future__ import annotations

from typing import Optional

from .inputs import LayerShape

__all__ = ["layer_flops", "layer_bytes", "gate_up_flops", "down_flops"]


def layer_flops(shape: LayerShape, T: Optional[int] = None) -> int:
    """Router 2*T*d*N_r + routed 6*T*k*d*f + shared 6*T*d*N_s*f."""
    T = shape.T if T is None else T
    return (2 * T * shape.d * shape.n_routed
            + 6 * T * shape.top_k * shape.d * shape.f
            + 6 * T * shape.d * shape.n_shared * shape.f)


def gate_up_flops(shape: LayerShape, T: Optional[int] = None) -> int:
    """Routed gate + up projections: 4*T*k*d*f."""
    T = shape.T if T is None else T
    return 4 * T * shape.top_k * shape.d * shape.f


def down_flops(shape: LayerShape, T: Optional[int] = None) -> int:
    """Routed down projection: 2*T*k*d*f."""
    T = shape.T if T is None else T
    return 2 * T * shape.top_k * shape.d * shape.f


def layer_bytes(shape: LayerShape, touched_experts: int,
                T: Optional[int] = None) -> int:
    """2 bytes x (T*d in + T*d out + N_r*d router + 3*d*N_s*f shared
    + touched*3*d*f routed)."""
    T = shape.T if T is None else T
    d, f = shape.d, shape.f
    return 2 * (2 * T * d + shape.n_routed * d + 3 * d * shape.n_shared * f
                + touched_experts * 3 * d * f)
