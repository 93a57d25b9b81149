"""The C ABI library loads on a host without a GPU and exports every declared entry point;
host-side validation answers before any device work."""
import ctypes as C
import os
import re

import pytest

from block_diffusion_drafter_dflash2_b200 import build, inputs
from block_diffusion_drafter_dflash2_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def declared():
    txt = open(os.path.join(ROOT, "include", "dflash2.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(dflash2_\w+)\s*\(", txt)))


def test_every_declared_symbol_is_exported(lib):
    names = declared()
    assert set(names) == set(binding.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_strerror_and_sizes(lib):
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert lib.dflash2_strerror(code)
    cfg = binding.config(inputs.TINY)
    assert lib.dflash2_workspace_size(C.byref(cfg), 1) > 0
    d = inputs.TINY
    H, F, HQ, HKV = d.hidden, d.ffn, d.n_q * 128, d.n_kv * 128
    mats = H * d.n_taps * H + d.layers * (HQ * H + 2 * HKV * H + H * HQ + 3 * F * H)
    dyn = d.layers * 2 * (H // 4) * H * 2
    head = -(-(d.vocab + d.rank) // 256) * 256 * H * 2  # output head + selector projection, whole 16-tile records
    # prepared copy: the Q4_K matrices keep their size, bf16 matrices theirs, and the output head is
    # held twice (the streaming kernel's records and the tensor-core operand layout)
    assert lib.dflash2_prepared_size(C.byref(cfg)) == mats // 256 * 144 + dyn + 2 * head
    full = binding.config(inputs.FULL)
    # full drafter: 973.2 MB of Q4_K matrices + 131.1 MB dynamic-convolution generators + 2 x 2545.5 MB head
    assert abs(lib.dflash2_prepared_size(C.byref(full)) / 1e6 - (973.2 + 131.1 + 2 * 2545.5)) < 1.0
    bf = binding.config(inputs.FULL_BF16_B5)
    assert lib.dflash2_prepared_size(C.byref(bf)) > lib.dflash2_prepared_size(C.byref(full))


@pytest.mark.parametrize("field,value", [("head_dim", 64), ("page_size", 32), ("topk", 8), ("block", 1),
                                         ("block", 17), ("hidden", 500), ("n_kv", 3), ("rank", 512),
                                         ("vocab", 8200), ("layers", 9), ("wfmt", 4)])
def test_unsupported_config_is_rejected(lib, field, value):
    cfg = binding.config(inputs.TINY)
    setattr(cfg, field, value)
    assert lib.dflash2_workspace_size(C.byref(cfg), 1) == 0
    rc = lib.dflash2_draft_step(C.byref(cfg), None, None, None, 1, None, None, None, 0, None, None)
    assert rc == -2


def test_null_arguments_are_rejected(lib):
    cfg = binding.config(inputs.TINY)
    assert lib.dflash2_draft_step(C.byref(cfg), None, None, None, 1, None, None, None, 0, None, None) == -1
    w = binding.Weights()
    assert lib.dflash2_draft_step(C.byref(cfg), C.byref(w), None, None, 0, None, None, None, 0, None, None) == -1
    assert lib.dflash2_accept(None, None, 1, 8, None, None, None) == -1
    out = C.c_int32()
    assert lib.dflash2_device_error(None, C.byref(out), None) == -1
    # the host-buffer round validates its host pointers, batch and workspace before any CUDA call
    h = [C.c_int32() for _ in range(8)]
    ptrs = [C.addressof(v) for v in h]
    assert lib.dflash2_spec_step_host(C.byref(cfg), C.byref(w), None, 1, None, *ptrs[1:8], None, None, 0,
                                      None) == -1
    assert lib.dflash2_spec_step_host(C.byref(cfg), C.byref(w), None, 0, *ptrs, None, ptrs[0], 0, None) == -1
    assert lib.dflash2_spec_step_host(C.byref(cfg), C.byref(w), None, 1, *ptrs, None, None, 0, None) == -1
    # the host-buffer round rejects a missing KV cache before it copies anything (weights valid-looking)
    ws = C.create_string_buffer(512)
    ws_al = (C.addressof(ws) + 255) // 256 * 256
    assert lib.dflash2_spec_step_host(C.byref(cfg), C.byref(w), None, 1, *ptrs, None, ws_al, 1 << 40, None) in (-1, -6)
    # sampled acceptance: every pointer but q (optional), a positive batch, block >= 2 and vocab >= 1
    assert lib.dflash2_accept_sampled(None, *ptrs[1:5], 1, 8, 10, ptrs[5], ptrs[6], None) == -1
    assert lib.dflash2_accept_sampled(*ptrs[:5], 0, 8, 10, ptrs[5], ptrs[6], None) == -1
    assert lib.dflash2_accept_sampled(*ptrs[:5], 1, 1, 10, ptrs[5], ptrs[6], None) == -1
    assert lib.dflash2_accept_sampled(*ptrs[:5], 1, 8, 0, ptrs[5], ptrs[6], None) == -1
    assert lib.dflash2_accept_sampled(*ptrs[:5], 1, 8, 10, None, ptrs[6], None) == -1
    # chained acceptance: every pointer, a positive batch, block >= 2 and mask_id >= 0 are required
    assert lib.dflash2_accept_chain(None, ptrs[1], 1, 8, 5, *ptrs[2:6], None) == -1
    assert lib.dflash2_accept_chain(*ptrs[:2], 0, 8, 5, *ptrs[2:6], None) == -1
    assert lib.dflash2_accept_chain(*ptrs[:2], 1, 1, 5, *ptrs[2:6], None) == -1
    assert lib.dflash2_accept_chain(*ptrs[:2], 1, 8, -1, *ptrs[2:6], None) == -1
    assert lib.dflash2_accept_chain(*ptrs[:2], 1, 8, 5, ptrs[2], ptrs[3], None, ptrs[5], None) == -1
    ins = binding.InputsMut()
    assert lib.dflash2_spec_round(C.byref(cfg), C.byref(w), C.byref(ins), None, 1, *ptrs[:2], 5, *ptrs[2:6], ws_al,
                                  1 << 30, None) == -1
    ins = binding.InputsMut(ptrs[0], ptrs[1], ptrs[2])
    assert lib.dflash2_spec_round(C.byref(cfg), C.byref(w), C.byref(ins), None, 1, *ptrs[:2], inputs.TINY.vocab,
                                  *ptrs[2:6], ws_al, 1 << 30, None) == -1
    assert lib.dflash2_spec_round(C.byref(cfg), C.byref(w), C.byref(ins), None, 1, *ptrs[:2], 5, *ptrs[2:6], ws_al,
                                  1 << 30, None) == -6  # (unprepared weights: rejected before anything is queued)


def test_unprepared_q4k_weights_are_rejected(lib):
    cfg = binding.config(inputs.TINY)
    w = binding.Weights()
    w.prepared = 0
    ins, kv = binding.Inputs(), binding.KV()
    buf = C.create_string_buffer(64)
    rc = lib.dflash2_draft_step(C.byref(cfg), C.byref(w), C.byref(ins), C.byref(kv), 1, buf, buf, buf, 0, None,
                                None)
    assert rc == -6


@pytest.mark.parametrize("dims_name,batch,umma_products", [
    ("tiny", 3, 1),   # 24 block rows stream; only q/k/v (48 rows: block + context) on the tensor cores
    ("tiny", 4, 6),   # 32 rows: every layer product and fc on the tensor cores
    ("full", 1, 0),   # 8 rows (16 for q/k/v): all streamed
    ("full", 2, 5),   # q/k/v of 5 layers at 32 rows
    ("full", 4, 26),  # 5 layers x 5 products + fc
    ("full", 64, 26),
])
def test_tensor_core_products_from_32_rows(lib, dims_name, batch, umma_products):
    """A product runs on the tensor cores (two launches: product and fix-up) from 32 activation rows
    on; the plan is visible on the host through the per-step launch count."""
    dims = inputs.TINY if dims_name == "tiny" else inputs.FULL
    cfg = binding.config(dims)
    base = 3 + 6 * dims.layers + 1 + 1 + 1
    assert lib.dflash2_step_kernels(C.byref(cfg), batch) == base + umma_products


def test_step_kernel_count_without_a_device(lib):
    cfg = binding.config(inputs.TINY)
    # embed, fc, fc norm | 7 per layer | final norm, LM head, selector tau + Viterbi
    assert lib.dflash2_step_kernels(C.byref(cfg), 1) == 3 + 6 * inputs.TINY.layers + 1 + 1 + 1
    assert lib.dflash2_step_kernels(C.byref(cfg), 0) == 0
    cfg.head_dim = 64
    assert lib.dflash2_step_kernels(C.byref(cfg), 1) == 0
