"""Algorithmic work of one block step: the bytes it must move at least once and the
matrix FLOPs it applies.  Used for the roofline figures of the benchmark."""
from __future__ import annotations

from typing import Dict, List

from .inputs import Q4K_BLOCK_BYTES, Q4K_BLOCK_ELEMS, Dims


def step_bytes(dims: Dims, ctx_after: List[int], n_new: List[int]) -> Dict[str, float]:
    """Weights once, the KV window each block row can see, the appended rows, taps and gathered rows.

    ctx_after: cached tokens per request after this step's append (L_b)."""
    H, F, T, R, V = dims.hidden, dims.ffn, dims.n_taps, dims.rank, dims.vocab
    hq, hkv, hd = dims.n_q * dims.head_dim, dims.n_kv * dims.head_dim, dims.head_dim
    # bytes per weight the step streams: Q4_K and MLX 4-bit both as 144-byte records per 256 weights;
    # bf16 and Q8_0 (decoded to bf16 when the weights are prepared) as 2 bytes
    per_w = Q4K_BLOCK_BYTES / Q4K_BLOCK_ELEMS if dims.wfmt in (0, 2) else 2.0
    layer_mats = (hq * H + 2 * hkv * H + H * hq + 2 * F * H + H * F) * per_w
    dyn = (2 * (H // 4) * H + 2 * H) * 2.0
    norms = (2 * H + 2 * hd) * 2.0
    B, Bk = len(ctx_after), dims.block
    kv_read = 0.0
    for L in ctx_after:
        visible = min(L, dims.window - 1)  # cache keys block position 0 can see
        kv_read += visible * hkv * 2 * 2 * dims.layers
    kv_write = float(sum(n_new) * hkv * 2 * 2 * dims.layers)
    out = {
        "layers": dims.layers * (layer_mats + dyn + norms),
        "fc": H * T * H * per_w + 2 * H * 2.0,
        "lm_head": V * H * 2.0,
        "sel_proj": R * H * 2.0,
        "kv_read": kv_read,
        "kv_write": kv_write,
        "taps": float(sum(n_new) * T * H * 2),
        "gathered_rows": B * Bk * H * 2.0 + B * (1 + 2 * dims.topk * (Bk - 1)) * R * 2.0,
    }
    out["total"] = sum(out.values())
    return out


def lmhead_bytes(dims: Dims, rows: int) -> float:
    """One LM-head + top-16 launch: the output head and the selector projection once, plus its rows."""
    return (dims.vocab + dims.rank) * dims.hidden * 2.0 + rows * dims.hidden * 2.0


def lmhead_flops(dims: Dims, rows: int) -> float:
    """2 x multiply-adds of one output-head launch (head and selector projection) over `rows`."""
    return 2.0 * rows * (dims.vocab + dims.rank) * dims.hidden


def step_flops(dims: Dims, batch: int) -> float:
    """2 x multiply-adds of the matrices applied (block rows, context rows, drafted rows)."""
    H, F, T, R, V = dims.hidden, dims.ffn, dims.n_taps, dims.rank, dims.vocab
    hq, hkv = dims.n_q * dims.head_dim, dims.n_kv * dims.head_dim
    mb = batch * dims.block
    per_layer = mb * (2 * (H // 4) * H + hq * H + H * hq + 3 * F * H) + 2 * mb * 2 * hkv * H
    return 2.0 * (dims.layers * per_layer + mb * T * H * H + batch * (dims.block - 1) * (V + R) * H)


def launches_per_step(dims: Dims, batch: int, step_kernels: int) -> int:
    """Kernels launched per drafted step: the draft step's (as the library reports them) plus the
    acceptance kernel."""
    return step_kernels + 1
