"""ctypes front end of the CPU oracle (``dflash2_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  It shares no
code with the CUDA path: it takes host tensors (numpy or CPU torch) and calls
the plain C oracle, which computes in double precision.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dflash2_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_dflash2.so")
MAX_LAYERS = 8


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (portable flags: the library travels between hosts)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Dims(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("layers", "hidden", "ffn", "n_q", "n_kv", "head_dim", "window",
                                         "vocab", "n_taps", "block", "topk", "rank", "page_size", "wfmt")] + \
               [("rope_theta", C.c_double), ("rms_eps", C.c_double)]


class Layer(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("wq", "wk", "wv", "wo", "wg", "wu", "wd", "ln1", "ln2", "qn", "kn",
                                          "dc_w", "dc_s0", "dc_s1")]


class Weights(C.Structure):
    _fields_ = [("fc", C.c_void_p), ("fc_norm", C.c_void_p), ("layer", Layer * MAX_LAYERS)] + \
               [(n, C.c_void_p) for n in ("final_norm", "embed", "lm_head", "sel_proj", "cb_a", "cb_b")]


class Trace(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("hidden", "ctx", "final_h", "cand", "cand_logit", "z", "q0", "k0")]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _lib.orc_bf16.restype = C.c_double
        _lib.orc_fp16.restype = C.c_double
        _lib.orc_to_bf16.restype = C.c_uint16
        _lib.orc_to_bf16.argtypes = [C.c_double]
        _lib.orc_draft_request.restype = C.c_int
        _lib.orc_attention.restype = C.c_int
        _lib.orc_num_threads.restype = C.c_int
    return _lib


# ---------------------------------------------------------------- helpers

def _np(t, dtype=None):
    """Contiguous numpy view of a CPU torch tensor or numpy array (bf16 -> uint16 bits)."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            t = t.detach().cpu().contiguous()
            if t.dtype == torch.bfloat16 or t.dtype == torch.float16:
                t = t.view(torch.int16)
                a = t.numpy().view(np.uint16)
            else:
                a = t.numpy()
            return np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))
    except ImportError:
        pass
    a = np.asarray(t)
    return np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def dims_struct(d) -> Dims:
    return Dims(d.layers, d.hidden, d.ffn, d.n_q, d.n_kv, d.head_dim, d.window, d.vocab, d.n_taps, d.block,
                d.topk, d.rank, d.page_size, d.wfmt, float(d.rope_theta), float(d.rms_eps))


class HostWeights:
    """Keeps numpy copies alive and exposes the C weight struct."""

    def __init__(self, w: dict):
        self.keep = []

        def k(t):
            a = _np(t)
            self.keep.append(a)
            return _p(a)

        s = Weights()
        s.fc, s.fc_norm = k(w["fc"]), k(w["fc_norm"])
        for i, L in enumerate(w["layers"]):
            for n in Layer._fields_:
                setattr(s.layer[i], n[0], k(L[n[0]]))
        for n in ("final_norm", "embed", "lm_head", "sel_proj", "cb_a", "cb_b"):
            setattr(s, n, k(w[n]))
        self.struct = s


# ---------------------------------------------------------------- primitives

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_bf16(x: float) -> int:
    return int(lib().orc_to_bf16(float(x)))


def q4k_dequant(blocks) -> np.ndarray:
    b = _np(blocks, np.uint8).reshape(-1)
    assert b.size % 144 == 0
    out = np.empty(b.size // 144 * 256, np.float64)
    lib().orc_q4k_dequant(_p(b), C.c_int64(b.size // 144), _p(out))
    return out


def mlx4_dequant(groups) -> np.ndarray:
    b = _np(groups, np.uint8).reshape(-1)
    assert b.size % 36 == 0
    out = np.empty(b.size // 36 * 64, np.float64)
    lib().orc_mlx4_dequant(_p(b), C.c_int64(b.size // 36), _p(out))
    return out


def q8_0_dequant(blocks) -> np.ndarray:
    b = _np(blocks, np.uint8).reshape(-1)
    assert b.size % 34 == 0
    out = np.empty(b.size // 34 * 32, np.float64)
    lib().orc_q8_0_dequant(_p(b), C.c_int64(b.size // 34), _p(out))
    return out


def matmul(fmt: int, W, N: int, K: int, X: np.ndarray) -> np.ndarray:
    w = _np(W)
    x = np.ascontiguousarray(X, np.float64).reshape(-1, K)
    y = np.empty((x.shape[0], N), np.float64)
    lib().orc_matmul(fmt, _p(w), N, K, _p(x), x.shape[0], _p(y))
    return y


def rmsnorm(x: np.ndarray, w_bf16, eps: float) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float64)
    w = _np(w_bf16, np.uint16)
    y = np.empty_like(x)
    lib().orc_rmsnorm(_p(x), x.size, _p(w), C.c_double(eps), _p(y))
    return y


def rope(v: np.ndarray, pos: int, theta: float) -> np.ndarray:
    v = np.array(v, np.float64, copy=True)
    lib().orc_rope(_p(v), v.size, C.c_int64(pos), C.c_double(theta))
    return v


def dynconv(x: np.ndarray, dc_w, s0, s1) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float64)
    Bk, H = x.shape
    y = np.empty_like(x)
    lib().orc_dynconv(Bk, H, _p(x), _p(_np(dc_w, np.uint16)), _p(_np(s0, np.uint16)), _p(_np(s1, np.uint16)), _p(y))
    return y


def attention(dims, q, kb, vb, kcache, vcache, page_table, Lb: int):
    q = np.ascontiguousarray(q, np.float64)
    kb = np.ascontiguousarray(kb, np.float64)
    vb = np.ascontiguousarray(vb, np.float64)
    kc, vc = _np(kcache, np.uint16), _np(vcache, np.uint16)
    pt = _np(page_table, np.int32)
    o = np.empty_like(q)
    ds = dims_struct(dims)
    err = lib().orc_attention(C.byref(ds), q.shape[0], _p(q), _p(kb), _p(vb), _p(kc), _p(vc), _p(pt),
                              pt.size, C.c_int64(Lb), _p(o))
    return err, o


def topk(logits: np.ndarray, k: int):
    lg = np.ascontiguousarray(logits, np.float64)
    ids = np.empty(k, np.int32)
    vals = np.empty(k, np.float64)
    lib().orc_topk(_p(lg), lg.size, k, _p(ids), _p(vals))
    return ids, vals


def viterbi(unary: np.ndarray, trans: np.ndarray):
    u = np.ascontiguousarray(unary, np.float64)
    D, K = u.shape
    tr = np.ascontiguousarray(trans, np.float64).reshape(D, K, K)
    idx = np.empty(D, np.int32)
    sc = np.empty(D, np.float64)
    lib().orc_viterbi(D, K, _p(u), _p(tr), _p(idx), _p(sc))
    return idx, sc


def selector(cand, cand_logit, z, x0: int, cb_a, cb_b):
    cand = _np(cand, np.int32)
    D, K = cand.shape
    cl = np.ascontiguousarray(cand_logit, np.float64)
    zz = np.ascontiguousarray(z, np.float64)
    R = zz.shape[1]
    path = np.empty(D, np.int32)
    sc = np.empty(D, np.float64)
    lib().orc_selector(D, K, R, _p(cand), _p(cl), _p(zz), int(x0), _p(_np(cb_a, np.uint16)),
                       _p(_np(cb_b, np.uint16)), _p(path), _p(sc))
    return path, sc


def selector_trans(cand, z, x0: int, cb_a, cb_b) -> np.ndarray:
    """Transition scores tau [D][K][K] of the selector (row = source index, column = destination)."""
    cand = _np(cand, np.int32)
    D, K = cand.shape
    zz = np.ascontiguousarray(z, np.float64)
    tr = np.empty((D, K, K), np.float64)
    lib().orc_selector_trans(D, K, zz.shape[1], _p(cand), _p(zz), int(x0), _p(_np(cb_a, np.uint16)),
                             _p(_np(cb_b, np.uint16)), _p(tr))
    return tr


def accept(draft, target):
    d = _np(draft, np.int32)
    t = _np(target, np.int32)
    B, Bk = t.shape
    acc = np.empty(B, np.int32)
    em = np.empty((B, Bk), np.int32)
    lib().orc_accept(B, Bk, _p(d), _p(t), _p(acc), _p(em))
    return acc, em


def accept_chain(draft, target, mask_id: int):
    """Acceptance plus the next round's n_new and block tokens (see orc_accept_chain)."""
    d = _np(draft, np.int32)
    t = _np(target, np.int32)
    B, Bk = t.shape
    acc = np.empty(B, np.int32)
    em = np.empty((B, Bk), np.int32)
    nn = np.empty(B, np.int32)
    bt = np.empty((B, Bk), np.int32)
    lib().orc_accept_chain(B, Bk, int(mask_id), _p(d), _p(t), _p(acc), _p(em), _p(nn), _p(bt))
    return acc, em, nn, bt


def accept_sampled(draft, p, u_acc, u_s, q=None):
    """Exact rejection-sampling acceptance (see orc_accept_sampled).  draft int32 [B][D], p fp32
    [B][Bk][V], u_acc fp32 [B][D], u_s uint32 [B], q fp32 [B][D][V] or None (point mass)."""
    d = _np(draft, np.int32)
    pp = np.ascontiguousarray(_np(p), np.float32)
    B, Bk, V = pp.shape
    qq = None if q is None else np.ascontiguousarray(_np(q), np.float32)
    ua = np.ascontiguousarray(_np(u_acc), np.float32)
    us = np.ascontiguousarray(_np(u_s).astype(np.uint32))
    acc = np.empty(B, np.int32)
    em = np.empty((B, Bk), np.int32)
    lib().orc_accept_sampled(B, Bk, V, _p(d), _p(pp), _p(qq), _p(ua), _p(us), _p(acc), _p(em))
    return acc, em


def lmhead_topk(hn_bf16, lm_head, k: int):
    hn = _np(hn_bf16, np.uint16)
    rows, H = hn.shape
    lm = _np(lm_head, np.uint16)
    V = lm.size // H
    ids = np.empty((rows, k), np.int32)
    vals = np.empty((rows, k), np.float64)
    lib().orc_lmhead_topk(rows, H, V, k, _p(hn), _p(lm), _p(ids), _p(vals))
    return ids, vals


def logits_at(hn_bf16, lm_head, ids):
    hn = _np(hn_bf16, np.uint16)
    rows, H = hn.shape
    ids = _np(ids, np.int32)
    out = np.empty(ids.shape, np.float64)
    lib().orc_logits_at(rows, H, ids.shape[1], _p(hn), _p(_np(lm_head, np.uint16)), _p(ids), _p(out))
    return out


def num_threads() -> int:
    return int(lib().orc_num_threads())


# ---------------------------------------------------------------- the block step

def draft_request(dims, hw: HostWeights, taps_b, n_new: int, btok_b, k_cache, v_cache, page_table_b,
                  seq_len: int, trace: bool = False):
    """One request's block step.  ``k_cache``/``v_cache``: lists of per-layer uint16 numpy arrays,
    updated in place.  Returns (err, path, scores, new_seq_len, traces)."""
    D, H, K, R, Bk = dims.block - 1, dims.hidden, dims.topk, dims.rank, dims.block
    taps = _np(taps_b, np.uint16)
    bt = _np(btok_b, np.int32)
    pt = _np(page_table_b, np.int32)
    kp = (C.c_void_p * MAX_LAYERS)(*[_p(a) for a in k_cache])
    vp = (C.c_void_p * MAX_LAYERS)(*[_p(a) for a in v_cache])
    sl = C.c_int32(seq_len)
    path = np.empty(D, np.int32)
    scores = np.empty(D, np.float32)
    tr = None
    trs = None
    if trace:
        tr = {
            "hidden": np.zeros((dims.layers + 1, Bk, H)),
            "ctx": np.zeros((Bk, H)),
            "final_h": np.zeros((D, H)),
            "cand": np.zeros((D, K), np.int32),
            "cand_logit": np.zeros((D, K)),
            "z": np.zeros((D, R)),
            "q0": np.zeros((Bk, dims.n_q * dims.head_dim)),
            "k0": np.zeros((Bk, dims.n_kv * dims.head_dim)),
        }
        trs = Trace(*[_p(tr[n]) for n, _ in Trace._fields_])
    ds = dims_struct(dims)
    err = lib().orc_draft_request(C.byref(ds), C.byref(hw.struct), _p(taps), int(n_new), _p(bt), kp, vp, _p(pt),
                                  pt.size, C.byref(sl), _p(path), _p(scores),
                                  C.byref(trs) if trs is not None else None)
    return err, path, scores, sl.value, tr
