"""Seeded synthetic inputs for the DFlash 2 drafter block step.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It only describes shapes and draws random tensors; it holds
none of the block step's arithmetic.  The one encoder here, ``quantize_q4k``,
turns random fp32 matrices into Q4_K super-block bytes: the drafter card
(FastFlowLM model card, "Weights" row) ships its fc/q/k/v/o/MLP matrices
already in Q4_K, so quantisation is how the synthetic weight *file* is made,
not a step of the draft.  Both sides then decode the same bytes with code of
their own.

Shapes come from the FastFlowLM model card ("Draft" and "Taps" rows: 5
Qwen3-style layers, hidden 5120, FFN 17408, 32/8 heads of 128, window 2048,
block 8, top 16, rank 256, taps of target layers 5/19/33/47/61) and the
aiqre.com model page (vocabulary 248,320; context 262,144).

Q4_K byte layout (one 144-byte super-block of 256 consecutive weights of a row):
  bytes 0..1    d     fp16, little endian
  bytes 2..3    dmin  fp16
  bytes 4..9    eight 6-bit sub-block scales sc_j, j = 0..7, bit 6j of the
                48-bit little-endian integer formed by these bytes
  bytes 10..15  eight 6-bit sub-block mins m_j, same packing
  bytes 16..143 256 4-bit codes q_e: byte 16 + e/2, low nibble for even e
  weight e = d*sc_{e/32}*q_e - dmin*m_{e/32}
"""
from __future__ import annotations

import dataclasses
import math
import zlib
from typing import Dict, List, Optional

import torch

Q4K_BLOCK_ELEMS = 256
Q4K_BLOCK_BYTES = 144


@dataclasses.dataclass(frozen=True)
class Dims:
    layers: int
    hidden: int
    ffn: int
    n_q: int
    n_kv: int
    head_dim: int
    window: int
    vocab: int
    n_taps: int
    block: int
    topk: int
    rank: int
    page_size: int = 16
    rope_theta: float = 1.0e6
    rms_eps: float = 1.0e-6
    wfmt: int = 0  # layer + fc matrices: 0 = Q4_K, 1 = bf16, 2 = MLX 4-bit group-64, 3 = Q8_0

    @property
    def drafted(self) -> int:
        return self.block - 1


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dims: Dims
    batch: int
    ctx_lo: int              # cached tokens before the step, uniform in [lo, hi]
    ctx_hi: int
    shuffled_pages: bool     # physical page order is a seeded permutation
    window_pages_only: bool  # only pages that the window can reach are backed
    tap_outliers: bool       # 1% of tap channels scaled x20
    target_mode: str         # "uniform" or "first_mismatch"
    seed: int
    description: str = ""
    weight_seed: int = 0     # seed of the weight set (0: use ``seed``)

    @property
    def wseed(self) -> int:
        return self.weight_seed or self.seed


TINY = Dims(layers=1, hidden=512, ffn=1536, n_q=4, n_kv=1, head_dim=128, window=64,
            vocab=8192, n_taps=2, block=8, topk=16, rank=64)
FULL = Dims(layers=5, hidden=5120, ffn=17408, n_q=32, n_kv=8, head_dim=128, window=2048,
            vocab=248320, n_taps=5, block=8, topk=16, rank=256)
FULL_BF16_B5 = dataclasses.replace(FULL, block=5, wfmt=1)

WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", TINY, 1, 128, 128, False, False, False, "uniform", 1001,
                     "tiny drafter, 1 request, 128 cached tokens"),
    "full_b1": Workload("full_b1", FULL, 1, 4096, 4096, False, False, False, "first_mismatch", 1002,
                        "full DFlash2 shape, 1 request, 4096 cached tokens"),
    "full_b8_paged": Workload("full_b8_paged", FULL, 8, 2048, 32768, True, False, False,
                              "first_mismatch", 1003,
                              "full shape, 8 requests, 2048..32768 cached, shuffled 16-token pages", 1002),
    "full_b64": Workload("full_b64", FULL, 64, 512, 8192, False, False, False, "first_mismatch", 1004,
                         "full shape, 64 requests (512 block rows), 512..8192 cached", 1002),
    "full_bf16_b16": Workload("full_bf16_b16", FULL_BF16_B5, 16, 1, 262144, False, True, True,
                              "first_mismatch", 1005,
                              "bf16 layers, block 5, 16 requests, up to 262144 cached, 1% tap outliers"),
    # profiling case: full layer shapes, one layer, a 65536-token vocabulary (about 1.7 GB on the device)
    "prof_small": Workload("prof_small", dataclasses.replace(FULL, layers=1, vocab=65536), 1, 4096, 4096, False, False,
                           False, "first_mismatch", 1006, "profiling case: 1 full-shape layer, vocab 65536"),
    # the same for 64 requests (the tensor-core products and head), about 2.5 GB on the device
    "prof_b64": Workload("prof_b64", dataclasses.replace(FULL, layers=1, vocab=65536), 64, 512, 4096, False, False,
                         False, "first_mismatch", 1007, "profiling case: 1 full-shape layer, vocab 65536, 64 requests"),
}


def _gen(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1000003 + zlib.crc32(name.encode())) & 0x7FFFFFFFFFFFFFFF)
    return g


def _normal(shape, std, mean, seed, name, device, dtype=torch.bfloat16, chunk_rows=4096):
    """N(mean, std^2) drawn in fp32 and stored as ``dtype`` (row chunks bound the fp32 temp)."""
    g = _gen(seed, name, device)
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(shape[0], -1) if len(shape) > 1 else out.view(1, -1)
    for r0 in range(0, flat.shape[0], chunk_rows):
        r1 = min(flat.shape[0], r0 + chunk_rows)
        t = torch.randn((r1 - r0, flat.shape[1]), generator=g, device=device, dtype=torch.float32)
        flat[r0:r1] = (t * std + mean).to(dtype)
    return out


def quantize_q4k(w: torch.Tensor) -> torch.Tensor:
    """fp32 [N, K] -> uint8 [N, K/256*144] Q4_K super-blocks (layout in the module docstring).

    Per 32-weight sub-block: offset = -min(0, min w), scale = (max w - min)/15.
    Per super-block: d = max scale/63 and dmin = max offset/63, rounded to fp16;
    6-bit sc_j, m_j and 4-bit codes by round-half-even, clamped to their ranges.
    """
    assert w.dim() == 2 and w.shape[1] % Q4K_BLOCK_ELEMS == 0
    n, k = w.shape
    nb = k // Q4K_BLOCK_ELEMS
    x = w.float().reshape(n, nb, 8, 32)
    mn = x.amin(-1).clamp(max=0.0)
    mx = x.amax(-1)
    scale = (mx - mn) / 15.0
    mofs = -mn
    d16 = (scale.amax(-1) / 63.0).to(torch.float16)
    dm16 = (mofs.amax(-1) / 63.0).to(torch.float16)
    d = d16.float().unsqueeze(-1)
    dm = dm16.float().unsqueeze(-1)
    one = torch.ones_like(d)
    sc = torch.where(d > 0, torch.round(scale / torch.where(d > 0, d, one)), 0.0).clamp(0, 63)
    mm = torch.where(dm > 0, torch.round(mofs / torch.where(dm > 0, dm, one)), 0.0).clamp(0, 63)
    es = (d * sc).unsqueeze(-1)
    em = (dm * mm).unsqueeze(-1)
    q = torch.where(es > 0, torch.round((x + em) / torch.where(es > 0, es, torch.ones_like(es))),
                    torch.zeros_like(x)).clamp(0, 15).to(torch.int32)

    out = torch.empty((n, nb, Q4K_BLOCK_BYTES), dtype=torch.uint8, device=w.device)
    dbits = d16.view(torch.int16).to(torch.int32) & 0xFFFF
    dmbits = dm16.view(torch.int16).to(torch.int32) & 0xFFFF
    out[..., 0] = (dbits & 0xFF).to(torch.uint8)
    out[..., 1] = (dbits >> 8).to(torch.uint8)
    out[..., 2] = (dmbits & 0xFF).to(torch.uint8)
    out[..., 3] = (dmbits >> 8).to(torch.uint8)
    sh = torch.arange(8, device=w.device, dtype=torch.int64) * 6
    scp = (sc.to(torch.int64) << sh).sum(-1)
    mmp = (mm.to(torch.int64) << sh).sum(-1)
    for i in range(6):
        out[..., 4 + i] = ((scp >> (8 * i)) & 0xFF).to(torch.uint8)
        out[..., 10 + i] = ((mmp >> (8 * i)) & 0xFF).to(torch.uint8)
    qf = q.reshape(n, nb, 256)
    out[..., 16:] = (qf[..., 0::2] | (qf[..., 1::2] << 4)).to(torch.uint8)
    return out.reshape(n, nb * Q4K_BLOCK_BYTES)


def quantize_mlx4(w: torch.Tensor) -> torch.Tensor:
    """fp32 [N, K] -> uint8 [N, K/64*36]: MLX-style 4-bit groups of 64 (the MLX sidecar card ships
    4-bit group-64 weights).  Per group: 32 bytes of codes (element e at byte e/2, low nibble
    first), then the bf16 scale and bias; weight = scale * q + bias.  Scale (max - min)/15 and bias
    = min, both rounded to bf16 first; codes by round-half-even of (w - bias)/scale, clamped."""
    assert w.dim() == 2 and w.shape[1] % 64 == 0
    n, k = w.shape
    x = w.float().reshape(n, k // 64, 64)
    mn, mx = x.amin(-1), x.amax(-1)
    sc = ((mx - mn) / 15.0).to(torch.bfloat16)
    bi = mn.to(torch.bfloat16)
    scf, bif = sc.float().unsqueeze(-1), bi.float().unsqueeze(-1)
    q = torch.where(scf > 0, torch.round((x - bif) / torch.where(scf > 0, scf, torch.ones_like(scf))),
                    torch.zeros_like(x)).clamp(0, 15).to(torch.int32)
    out = torch.empty((n, k // 64, 36), dtype=torch.uint8, device=w.device)
    out[..., :32] = (q[..., 0::2] | (q[..., 1::2] << 4)).to(torch.uint8)
    sb = sc.view(torch.int16).to(torch.int32) & 0xFFFF
    bb = bi.view(torch.int16).to(torch.int32) & 0xFFFF
    out[..., 32] = (sb & 0xFF).to(torch.uint8)
    out[..., 33] = (sb >> 8).to(torch.uint8)
    out[..., 34] = (bb & 0xFF).to(torch.uint8)
    out[..., 35] = (bb >> 8).to(torch.uint8)
    return out.reshape(n, k // 64 * 36)


def quantize_q8_0(w: torch.Tensor) -> torch.Tensor:
    """fp32 [N, K] -> uint8 [N, K/32*34]: Q8_0 blocks of 32 (the GGUF listing ships Q8_0 files):
    fp16 d = max|w|/127, then 32 signed codes round-half-even(w/d) clamped to [-127, 127]."""
    assert w.dim() == 2 and w.shape[1] % 32 == 0
    n, k = w.shape
    x = w.float().reshape(n, k // 32, 32)
    d16 = (x.abs().amax(-1) / 127.0).to(torch.float16)
    d = d16.float().unsqueeze(-1)
    q = torch.where(d > 0, torch.round(x / torch.where(d > 0, d, torch.ones_like(d))),
                    torch.zeros_like(x)).clamp(-127, 127).to(torch.int32)
    out = torch.empty((n, k // 32, 34), dtype=torch.uint8, device=w.device)
    db = d16.view(torch.int16).to(torch.int32) & 0xFFFF
    out[..., 0] = (db & 0xFF).to(torch.uint8)
    out[..., 1] = (db >> 8).to(torch.uint8)
    out[..., 2:] = (q & 0xFF).to(torch.uint8)
    return out.reshape(n, k // 32 * 34)


# bytes per row per 256 weights of each storage format of fc and the layer matrices
FORMAT_BYTES_PER_256 = {0: Q4K_BLOCK_BYTES, 1: 512, 2: 4 * 36, 3: 8 * 34}


def _linear(out_f, in_f, dims: Dims, seed, name, device, quantized: bool):
    """A linear layer [out_f, in_f] with N(0, 0.02) weights, stored in the format dims.wfmt
    (0 = Q4_K, 1 = bf16, 2 = MLX 4-bit group-64, 3 = Q8_0)."""
    if not quantized or dims.wfmt == 1:
        return _normal((out_f, in_f), 0.02, 0.0, seed, name, device)
    enc = {0: quantize_q4k, 2: quantize_mlx4, 3: quantize_q8_0}[dims.wfmt]
    g = _gen(seed, name, device)
    out = torch.empty((out_f, in_f // 256 * FORMAT_BYTES_PER_256[dims.wfmt]), dtype=torch.uint8, device=device)
    step = 2048
    for r0 in range(0, out_f, step):
        r1 = min(out_f, r0 + step)
        w = torch.randn((r1 - r0, in_f), generator=g, device=device, dtype=torch.float32) * 0.02
        out[r0:r1] = enc(w)
    return out


def make_weights(dims: Dims, seed: int, device="cpu") -> dict:
    """All drafter weights for ``dims``; every tensor has its own seeded stream."""
    H, F, T, R, V = dims.hidden, dims.ffn, dims.n_taps, dims.rank, dims.vocab
    hq, hkv, hd = dims.n_q * dims.head_dim, dims.n_kv * dims.head_dim, dims.head_dim
    qz = dims.wfmt != 1
    norm = lambda n, name: _normal((n,), 0.01, 1.0, seed, name, device)
    w = {
        "fc": _linear(H, T * H, dims, seed, "fc", device, qz),
        "fc_norm": norm(H, "fc_norm"),
        "layers": [],
        "final_norm": norm(H, "final_norm"),
        "embed": _normal((V, H), 0.02, 0.0, seed, "embed", device),
        "lm_head": _normal((V, H), 0.02, 0.0, seed, "lm_head", device),
        "sel_proj": _normal((R, H), 0.02, 0.0, seed, "sel_proj", device),
        "cb_a": _normal((V, R), 0.05, 0.0, seed, "cb_a", device),
        "cb_b": _normal((V, R), 0.05, 0.0, seed, "cb_b", device),
    }
    for l in range(dims.layers):
        p = f"l{l}."
        w["layers"].append({
            "wq": _linear(hq, H, dims, seed, p + "wq", device, qz),
            "wk": _linear(hkv, H, dims, seed, p + "wk", device, qz),
            "wv": _linear(hkv, H, dims, seed, p + "wv", device, qz),
            "wo": _linear(H, hq, dims, seed, p + "wo", device, qz),
            "wg": _linear(F, H, dims, seed, p + "wg", device, qz),
            "wu": _linear(F, H, dims, seed, p + "wu", device, qz),
            "wd": _linear(H, F, dims, seed, p + "wd", device, qz),
            "ln1": norm(H, p + "ln1"),
            "ln2": norm(H, p + "ln2"),
            "qn": norm(hd, p + "qn"),
            "kn": norm(hd, p + "kn"),
            "dc_w": _normal((2 * (H // 4), H), 0.02, 0.0, seed, p + "dc_w", device),
            "dc_s0": _normal((H,), 0.01, 1.0, seed, p + "dc_s0", device),
            "dc_s1": _normal((H,), 0.01, 0.0, seed, p + "dc_s1", device),
        })
    return w


def context_lengths(wl: Workload) -> List[int]:
    g = torch.Generator().manual_seed(wl.seed * 7 + 3)
    if wl.ctx_lo == wl.ctx_hi:
        return [wl.ctx_lo] * wl.batch
    return [int(v) for v in torch.randint(wl.ctx_lo, wl.ctx_hi + 1, (wl.batch,), generator=g)]


def make_state(wl: Workload, device="cpu", extra_tokens: int = 0, seq_len: Optional[List[int]] = None,
               n_new: Optional[List[int]] = None) -> dict:
    """Per-step inputs and the paged KV cache of ``wl``.

    Cache layout per layer and for K and V alike: bf16 [num_pages, n_kv, page_size, head_dim];
    ``page_table`` int32 [B, max_pages] maps logical page i of request b (tokens 16i..16i+15)
    to a physical page, -1 where nothing is backed.  ``extra_tokens`` reserves room for that
    many appended tokens past this step (benchmarks that run many steps).
    """
    dims = wl.dims
    B, Bk, P = wl.batch, dims.block, dims.page_size
    lens = list(seq_len) if seq_len is not None else context_lengths(wl)
    nn = list(n_new) if n_new is not None else [Bk] * B
    cap = [L + Bk + extra_tokens for L in lens]
    max_pages = max((c + P - 1) // P for c in cap)
    # which logical pages are backed
    backed = []
    for b in range(B):
        npg = (cap[b] + P - 1) // P
        if wl.window_pages_only:
            # first cache key that block position 0 can see after this step's append
            first_tok = max(0, lens[b] + nn[b] - dims.window + 1)
            backed.append(list(range(first_tok // P, npg)))
        else:
            backed.append(list(range(npg)))
    total = sum(len(x) for x in backed)
    phys = torch.arange(total, dtype=torch.int32)
    if wl.shuffled_pages:
        phys = phys[torch.randperm(total, generator=torch.Generator().manual_seed(wl.seed * 13 + 5))]
    pt = torch.full((B, max_pages), -1, dtype=torch.int32)
    k = 0
    for b in range(B):
        for lp in backed[b]:
            pt[b, lp] = phys[k]
            k += 1
    shape = (total, dims.n_kv, P, dims.head_dim)
    kc = [_normal(shape, 1.0, 0.0, wl.seed, f"k{l}", device) for l in range(dims.layers)]
    vc = [_normal(shape, 1.0, 0.0, wl.seed, f"v{l}", device) for l in range(dims.layers)]

    taps = _normal((B, Bk, dims.n_taps * dims.hidden), 1.0, 0.0, wl.seed, "taps", device)
    if wl.tap_outliers:
        g = _gen(wl.seed, "outliers", "cpu")
        nch = dims.n_taps * dims.hidden
        idx = torch.randperm(nch, generator=g)[: max(1, nch // 100)].to(device)
        taps[..., idx] = (taps[..., idx].float() * 20.0).to(torch.bfloat16)
    for b in range(B):
        taps[b, nn[b]:] = 0
    g = _gen(wl.seed, "block_tokens", "cpu")
    bt = torch.full((B, Bk), dims.vocab - 1, dtype=torch.int32)  # mask id V-1 at positions 1..D
    bt[:, 0] = torch.randint(0, dims.vocab - 1, (B,), generator=g, dtype=torch.int32)
    return {
        "seq_len": torch.tensor(lens, dtype=torch.int32, device=device),
        "n_new": torch.tensor(nn, dtype=torch.int32, device=device),
        "block_tokens": bt.to(device),
        "taps": taps,
        "page_table": pt.to(device),
        "max_pages": max_pages,
        "k_cache": kc,
        "v_cache": vc,
    }


def make_targets(wl: Workload, path: Optional[torch.Tensor] = None, step: int = 0) -> torch.Tensor:
    """Target tokens int32 [B, block] (the target's argmax for block positions 1..block).

    "uniform": uniform ids.  "first_mismatch": the drafted ``path`` copied up to a seeded
    first mismatch position m in 0..block-1 (m = block-1 means all drafted tokens match),
    a different id at m, uniform ids after it.
    """
    dims = wl.dims
    B, Bk, V = wl.batch, dims.block, dims.vocab
    g = torch.Generator().manual_seed(wl.seed * 31 + 17 + step)
    t = torch.randint(0, V, (B, Bk), generator=g, dtype=torch.int32)
    if wl.target_mode == "uniform":
        return t
    assert path is not None
    p = path.detach().to("cpu", torch.int32)
    m = torch.randint(0, Bk, (B,), generator=g)
    for b in range(B):
        mb = int(m[b])
        t[b, :mb] = p[b, :mb]
        if mb < Bk - 1:
            t[b, mb] = (int(p[b, mb]) + 1 + int(t[b, mb]) % (V - 1)) % V
    return t
