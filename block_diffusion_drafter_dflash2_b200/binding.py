"""Thin ctypes binding of ``libdflash2.so`` (include/dflash2.h): argument marshalling only.

Every step of the block step runs in the library's CUDA kernels.  PyTorch is
used for device memory and streams.  There is no fallback: loading fails
loudly when the library is missing, and the calls need a CUDA device.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

import torch

MAX_LAYERS = 8
_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdflash2.so")

ERR_NAMES = {0: "OK", -1: "ARG", -2: "SHAPE", -3: "ALIGN", -4: "WORKSPACE", -5: "CUDA", -6: "LAYOUT",
             -7: "STATIC_LIMIT"}
STATIC_SCRATCH_BYTES = 16 << 20
DEV_TOKEN, DEV_PAGE, DEV_NONFINITE, DEV_TIMEOUT = 1, 2, 4, 8


class Config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("layers", "hidden", "ffn", "n_q", "n_kv", "head_dim", "window", "vocab",
                                         "n_taps", "block", "topk", "rank", "page_size")] + \
               [("rope_theta", C.c_float), ("rms_eps", C.c_float), ("wfmt", C.c_int32)]


LAYER_FIELDS = ("wq", "wk", "wv", "wo", "wg", "wu", "wd", "ln1", "ln2", "qn", "kn", "dc_w", "dc_s0", "dc_s1")


class LayerWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in LAYER_FIELDS]


class Weights(C.Structure):
    _fields_ = [("fc", C.c_void_p), ("fc_norm", C.c_void_p), ("layer", LayerWeights * MAX_LAYERS)] + \
               [(n, C.c_void_p) for n in ("final_norm", "embed", "lm_head", "sel_proj", "cb_a", "cb_b")] + \
               [("prepared", C.c_int32)]


class KV(C.Structure):
    _fields_ = [("k", C.c_void_p * MAX_LAYERS), ("v", C.c_void_p * MAX_LAYERS), ("page_table", C.c_void_p),
                ("max_pages", C.c_int32), ("num_pages", C.c_int32), ("seq_len", C.c_void_p)]


class Inputs(C.Structure):
    _fields_ = [("taps", C.c_void_p), ("n_new", C.c_void_p), ("block_tokens", C.c_void_p)]


class Debug(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("hidden", "ctx", "final_h", "cand", "cand_logit", "z", "ev_lm_begin",
                                          "ev_lm_end")]


class InputsMut(C.Structure):
    _fields_ = [("taps", C.c_void_p), ("n_new", C.c_void_p), ("block_tokens", C.c_void_p)]


EXPORTS = ("dflash2_workspace_size", "dflash2_prepared_size", "dflash2_prepare_weights", "dflash2_draft_step",
           "dflash2_draft_step_static", "dflash2_accept", "dflash2_accept_sampled", "dflash2_accept_chain", "dflash2_spec_round",
           "dflash2_spec_step_host", "dflash2_device_error", "dflash2_step_kernels", "dflash2_strerror",
           "dflash2_head_shard_size", "dflash2_prepare_head_shard", "dflash2_draft_step_head_shard",
           "dflash2_select")

_lib = None


def load(path: str = LIB_PATH):
    """Load the CUDA library; raises when it is not built (there is no CPU fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libdflash2.so not built at {path}; run block_diffusion_drafter_dflash2_b200/build.py")
    lib = C.CDLL(path)
    lib.dflash2_workspace_size.restype = C.c_size_t
    lib.dflash2_workspace_size.argtypes = [C.POINTER(Config), C.c_int32]
    lib.dflash2_prepared_size.restype = C.c_size_t
    lib.dflash2_prepared_size.argtypes = [C.POINTER(Config)]
    lib.dflash2_prepare_weights.argtypes = [C.POINTER(Config), C.POINTER(Weights), C.c_void_p, C.c_size_t,
                                            C.POINTER(Weights), C.c_void_p]
    lib.dflash2_draft_step.argtypes = [C.POINTER(Config), C.POINTER(Weights), C.POINTER(Inputs), C.POINTER(KV),
                                       C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.POINTER(Debug),
                                       C.c_void_p]
    lib.dflash2_draft_step_static.argtypes = [C.POINTER(Config), C.POINTER(Weights), C.POINTER(Inputs),
                                              C.POINTER(KV), C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p,
                                              C.POINTER(Debug), C.c_void_p]
    lib.dflash2_accept.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p]
    lib.dflash2_head_shard_size.restype = C.c_size_t
    lib.dflash2_head_shard_size.argtypes = [C.POINTER(Config), C.c_int32]
    lib.dflash2_prepare_head_shard.argtypes = [C.POINTER(Config), C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p,
                                               C.c_size_t, C.c_void_p]
    lib.dflash2_draft_step_head_shard.argtypes = [C.POINTER(Config), C.POINTER(Weights), C.c_void_p, C.c_int32,
                                                  C.c_int32, C.POINTER(Inputs), C.POINTER(KV), C.c_int32, C.c_void_p,
                                                  C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]
    lib.dflash2_select.argtypes = [C.POINTER(Config), C.POINTER(Weights), C.c_int32, C.c_int32] + \
        [C.c_void_p] * 7 + [C.c_size_t, C.c_void_p]
    lib.dflash2_accept_sampled.argtypes = [C.c_void_p] * 5 + [C.c_int32] * 3 + [C.c_void_p] * 3
    lib.dflash2_accept_chain.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_int32, C.c_int32] + [C.c_void_p] * 5
    lib.dflash2_spec_round.argtypes = [C.POINTER(Config), C.POINTER(Weights), C.POINTER(InputsMut), C.POINTER(KV),
                                       C.c_int32, C.c_void_p, C.c_void_p, C.c_int32] + [C.c_void_p] * 5 + \
        [C.c_size_t, C.c_void_p]
    lib.dflash2_spec_step_host.argtypes = [C.POINTER(Config), C.POINTER(Weights), C.POINTER(KV), C.c_int32] + \
        [C.c_void_p] * 9 + [C.c_void_p, C.c_size_t, C.c_void_p]
    lib.dflash2_device_error.argtypes = [C.c_void_p, C.POINTER(C.c_int32), C.c_void_p]
    lib.dflash2_step_kernels.restype = C.c_int32
    lib.dflash2_step_kernels.argtypes = [C.POINTER(Config), C.c_int32]
    lib.dflash2_strerror.restype = C.c_char_p
    lib.dflash2_strerror.argtypes = [C.c_int]
    _lib = lib
    return lib


class DFlash2Error(RuntimeError):
    pass


def check(rc: int, what: str = "call"):
    if rc != 0:
        raise DFlash2Error(f"{what}: {ERR_NAMES.get(rc, rc)} ({load().dflash2_strerror(rc).decode()})")


def config(d) -> Config:
    return Config(d.layers, d.hidden, d.ffn, d.n_q, d.n_kv, d.head_dim, d.window, d.vocab, d.n_taps, d.block,
                  d.topk, d.rank, d.page_size, float(d.rope_theta), float(d.rms_eps), d.wfmt)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None) -> C.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def weights_struct(w: dict, prepared: int = 0) -> Weights:
    s = Weights()
    s.fc, s.fc_norm = w["fc"].data_ptr(), w["fc_norm"].data_ptr()
    for i, L in enumerate(w["layers"]):
        for n in LAYER_FIELDS:
            setattr(s.layer[i], n, L[n].data_ptr())
    for n in ("final_norm", "embed", "lm_head", "sel_proj", "cb_a", "cb_b"):
        setattr(s, n, w[n].data_ptr())
    s.prepared = prepared
    return s


def kv_struct(state: dict) -> KV:
    kv = KV()
    for i, (k, v) in enumerate(zip(state["k_cache"], state["v_cache"])):
        kv.k[i] = k.data_ptr()
        kv.v[i] = v.data_ptr()
    kv.page_table = state["page_table"].data_ptr()
    kv.max_pages = int(state["page_table"].shape[1])
    kv.num_pages = int(state["k_cache"][0].shape[0])
    kv.seq_len = state["seq_len"].data_ptr()
    return kv


class Drafter:
    """Prepared weights + workspace for ``batch`` requests on the current CUDA device."""

    def __init__(self, dims, weights: dict, batch: int, stream=None):
        self.lib = load()
        self.dims = dims
        self.batch = batch
        self.cfg = config(dims)
        self.weights = weights  # keeps the device tensors alive
        dev = weights["lm_head"].device
        canon = weights_struct(weights, 0)
        nprep = self.lib.dflash2_prepared_size(C.byref(self.cfg))
        self.prepared_buf = torch.empty(max(nprep, 16), dtype=torch.uint8, device=dev)
        self.w = Weights()
        check(self.lib.dflash2_prepare_weights(C.byref(self.cfg), C.byref(canon), _ptr(self.prepared_buf), nprep,
                                               C.byref(self.w), _stream(stream)), "prepare_weights")
        self.ws_bytes = self.lib.dflash2_workspace_size(C.byref(self.cfg), batch)
        if self.ws_bytes == 0:
            raise DFlash2Error("configuration not supported (workspace size 0)")
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev)

    def draft_step(self, inputs: dict, state: dict, out_path: torch.Tensor, out_scores: torch.Tensor,
                   debug: Optional[dict] = None, stream=None, kv: Optional[KV] = None):
        ins = Inputs(inputs["taps"].data_ptr(), inputs["n_new"].data_ptr(), inputs["block_tokens"].data_ptr())
        kvs = kv if kv is not None else kv_struct(state)
        dbg = None
        if debug:
            dbg = Debug()
            for n, _ in Debug._fields_:
                v = debug.get(n)
                if v is None:
                    continue
                setattr(dbg, n, v.cuda_event if isinstance(v, torch.cuda.Event) else v.data_ptr())
        rc = self.lib.dflash2_draft_step(C.byref(self.cfg), C.byref(self.w), C.byref(ins), C.byref(kvs), self.batch,
                                         _ptr(out_path), _ptr(out_scores), _ptr(self.workspace), self.ws_bytes,
                                         C.byref(dbg) if dbg is not None else None, _stream(stream))
        check(rc, "draft_step")

    def draft_step_static(self, inputs: dict, state: dict, out_path: torch.Tensor, out_scores: torch.Tensor,
                          dev_err: Optional[torch.Tensor] = None, stream=None, kv: Optional[KV] = None):
        """The allocation-free entry point: same step, scratch compiled into the library (no workspace)."""
        ins = Inputs(inputs["taps"].data_ptr(), inputs["n_new"].data_ptr(), inputs["block_tokens"].data_ptr())
        kvs = kv if kv is not None else kv_struct(state)
        rc = self.lib.dflash2_draft_step_static(C.byref(self.cfg), C.byref(self.w), C.byref(ins), C.byref(kvs),
                                                self.batch, _ptr(out_path), _ptr(out_scores), _ptr(dev_err), None,
                                                _stream(stream))
        check(rc, "draft_step_static")

    def accept(self, draft: torch.Tensor, target: torch.Tensor, accepted: torch.Tensor, emitted: torch.Tensor,
               stream=None):
        check(self.lib.dflash2_accept(_ptr(draft), _ptr(target), self.batch, self.dims.block, _ptr(accepted),
                                      _ptr(emitted), _stream(stream)), "accept")

    def accept_sampled(self, draft, p_target, u_accept, u_sample, accepted, emitted, q_draft=None, stream=None):
        """Exact rejection-sampling acceptance (sampled decoding)."""
        check(self.lib.dflash2_accept_sampled(_ptr(draft), _ptr(p_target), _ptr(q_draft), _ptr(u_accept),
                                              _ptr(u_sample), self.batch, self.dims.block, int(p_target.shape[-1]),
                                              _ptr(accepted), _ptr(emitted), _stream(stream)), "accept_sampled")

    def accept_chain(self, draft, target, mask_id: int, accepted, emitted, n_new_next, block_tokens_next,
                     stream=None):
        """Acceptance plus the next round's n_new and block tokens, on the device."""
        check(self.lib.dflash2_accept_chain(_ptr(draft), _ptr(target), self.batch, self.dims.block, int(mask_id),
                                            _ptr(accepted), _ptr(emitted), _ptr(n_new_next),
                                            _ptr(block_tokens_next), _stream(stream)), "accept_chain")

    def spec_round(self, inputs: dict, state: dict, prev_path, target, mask_id: int, accepted, emitted, out_path,
                   out_scores, stream=None, kv: Optional[KV] = None):
        """Chained acceptance of the previous draft, then the next draft step; inputs["n_new"] and
        inputs["block_tokens"] are overwritten with the next round's values on the device."""
        ins = InputsMut(inputs["taps"].data_ptr(), inputs["n_new"].data_ptr(), inputs["block_tokens"].data_ptr())
        kvs = kv if kv is not None else kv_struct(state)
        check(self.lib.dflash2_spec_round(C.byref(self.cfg), C.byref(self.w), C.byref(ins), C.byref(kvs),
                                          self.batch, _ptr(prev_path), _ptr(target), int(mask_id), _ptr(accepted),
                                          _ptr(emitted), _ptr(out_path), _ptr(out_scores), _ptr(self.workspace),
                                          self.ws_bytes, _stream(stream)), "spec_round")

    def spec_step_host(self, state: dict, taps_h, n_new_h, block_tokens_h, target_h, path_h, scores_h, accepted_h,
                       emitted_h, stream=None, kv: Optional[KV] = None) -> int:
        """Host-buffer round trip (inputs in, outputs back, stream synchronised); returns the device
        error bits.  With page-locked buffers the library's kernels read and write them in place."""
        kvs = kv if kv is not None else kv_struct(state)
        if getattr(self, "_err_h", None) is None:
            self._err_h = torch.zeros(1, dtype=torch.int32).pin_memory()
        self._err_h.zero_()
        rc = self.lib.dflash2_spec_step_host(
            C.byref(self.cfg), C.byref(self.w), C.byref(kvs), self.batch, _ptr(taps_h), _ptr(n_new_h),
            _ptr(block_tokens_h), _ptr(target_h), _ptr(path_h), _ptr(scores_h), _ptr(accepted_h), _ptr(emitted_h),
            _ptr(self._err_h), _ptr(self.workspace), self.ws_bytes, _stream(stream))
        check(rc, "spec_step_host")
        return int(self._err_h[0])

    def step_kernels(self) -> int:
        """Kernels one draft_step launches."""
        return int(self.lib.dflash2_step_kernels(C.byref(self.cfg), self.batch))

    def device_error(self, stream=None) -> int:
        out = C.c_int32(0)
        check(self.lib.dflash2_device_error(_ptr(self.workspace), C.byref(out), _stream(stream)), "device_error")
        return out.value
