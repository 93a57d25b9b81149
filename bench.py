"""Benchmark of the DFlash 2 drafter block step on B200.

One step = dflash2_draft_step + dflash2_accept for the whole batch (full drafter
shape, 1 request, 4096 cached tokens, block of 8).  Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dflash2|reference]

Multi-GPU: one process per GPU (torchrun); requests are sharded across ranks, each
rank runs its own replica on its own requests, no collective on the data path
(weak scaling).  Timing: CUDA events on the launching stream, barrier +
synchronize on both sides, max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_diffusion_drafter_dflash2_b200 import accounting, inputs  # noqa: E402

NOMINAL_HBM_GBS = 8000.0


def head_traffic_ratio():
    """DRAM bytes per algorithmic byte of the streaming LM-head kernel, from the machine-readable
    summary of its small-case ncu capture; None when the summary is missing or the kernel's source
    has changed since the capture (the counters then describe another kernel)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "ncu_k_slmhead_prof_small.json")) as f:
            cap = json.load(f)
        with open(os.path.join(ROOT, "block_diffusion_drafter_dflash2_b200", "csrc", "stream.cuh")) as f:
            src = f.read()
    except (OSError, ValueError):
        return None
    i = src.find("__global__ void __launch_bounds__(kGemvThreads, 1) k_slmhead")
    if i < 0 or hashlib.sha256(src[i:].encode()).hexdigest() != cap.get("kernel_source_sha256"):
        return None
    return float(cap["dram_bytes_per_algorithmic_byte"])


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def bf16_sustained_tflops():
    """Measured sustained dense bf16 rate (the step is long), else the recipe's fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.idx)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = [r.split(",") for r in (self.out or "").strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i] and "Not" not in r[5 + i]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def all_max(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def oracle_step_time(wl, weights_host, hw, st_host, reps_budget_s: float, max_reps: int):
    """Time the oracle's block step for request 0 (as it stands) on the host cores."""
    import oracle
    from tests.parity import snapshot_request
    times = []
    t_all = time.perf_counter()
    while len(times) < max_reps:
        sn = snapshot_request(wl, st_host, 0)
        t0 = time.perf_counter()
        err, *_ = oracle.draft_request(wl.dims, hw, sn["taps"], sn["n"], sn["btok"], sn["kc"], sn["vc"], sn["pt"],
                                       sn["L0"])
        times.append(time.perf_counter() - t0)
        assert err == 0
        if time.perf_counter() - t_all > reps_budget_s:
            break
    return times, oracle.num_threads()


def host_state_for_request0(st: dict) -> dict:
    return {k: ([t.cpu() for t in v] if isinstance(v, list) else (v.cpu() if isinstance(v, torch.Tensor) else v))
            for k, v in st.items()}


def host_copy_weights(w: dict):
    import oracle
    hw_t = {k: v.cpu() for k, v in w.items() if k != "layers"}
    hw_t["layers"] = [{k: v.cpu() for k, v in L.items()} for L in w["layers"]]
    return hw_t, oracle.HostWeights(hw_t)


def bench_config(wl, ws: int) -> dict:
    """The workload description both arms print."""
    d = wl.dims
    return {"workload": wl.name, "requests_per_gpu": wl.batch, "context": wl.ctx_lo, "block": d.block,
            "layers": d.layers, "hidden": d.hidden, "vocab": d.vocab,
            "parallelism": f"replicas x{ws} (requests sharded, no collective)",
            "l2": "inputs larger than L2 (3.7 GB of weights streamed per step)"}


def run_reference(args, ws, rank):
    """The reference arm: the CPU oracle as it stands, timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    wl = inputs.WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = inputs.make_weights(wl.dims, wl.wseed, dev)
    st = inputs.make_state(wl, dev)
    hw_t, hw = host_copy_weights(w)
    del w
    st_h = host_state_for_request0(st)
    # one untimed oracle step (each takes seconds on the host cores; the timed steps are bounded by
    # --ref-budget-s): the line reports the warm-up it ran
    warm = min(args.warmup, 1)
    for _ in range(warm):
        oracle_step_time(wl, hw_t, hw, st_h, 0.0, 1)
    times, cores = oracle_step_time(wl, hw_t, hw, st_h, args.ref_budget_s, args.steps)
    per = sum(times) / len(times)
    value = 1.0 / per
    line = {
        "impl": "reference", "metric": "DFlash2 draft steps/s (8-token block)", "value": value,
        "unit": "steps/s", "n_gpus": ws, "steps": len(times), "warmup": warm, "ms_per_step": per * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(wl, ws),
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": cores, "kind": "oracle",
                         "sample": f"{len(times)} full block steps of request 0 (fp64 C oracle, OpenMP)"},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="dflash2", choices=["dflash2", "reference"])
    ap.add_argument("--workload", default="full_b1", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0)
    ap.add_argument("--ref-budget-s", type=float, default=90.0)
    ap.add_argument("--e2e-steps", type=int, default=0, help="0: same as --steps")
    args = ap.parse_args()
    ws, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, ws, rank)
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    assert torch.cuda.is_available(), "the CUDA path needs a GPU"
    from block_diffusion_drafter_dflash2_b200.binding import Drafter, kv_struct

    wl = inputs.WORKLOADS[args.workload]
    dims = wl.dims
    B, Bk, D = wl.batch, dims.block, dims.block - 1
    dev = torch.device("cuda", local)
    K, W = args.steps, max(3, args.warmup)
    E = args.e2e_steps or K
    total_steps = W + K + E + 2
    w = inputs.make_weights(dims, wl.wseed, dev)
    st = inputs.make_state(wl, dev, extra_tokens=Bk * total_steps + Bk)
    dr = Drafter(dims, w, B)
    kv = kv_struct(st)
    ins = {"taps": st["taps"], "n_new": st["n_new"], "block_tokens": st["block_tokens"]}
    path = torch.zeros((B, D), dtype=torch.int32, device=dev)
    scores = torch.zeros((B, D), dtype=torch.float32, device=dev)
    acc = torch.zeros((B,), dtype=torch.int32, device=dev)
    em = torch.zeros((B, Bk), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    # first step: its path seeds the target tokens (first mismatch at a seeded position)
    dr.draft_step(ins, st, path, scores, kv=kv)
    target = inputs.make_targets(wl, path).to(dev)
    dr.accept(path, target, acc, em)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in ev:  # create the events (the library records them again inside the step)
        a.record(stream)
        b.record(stream)

    def step(i=None):
        dbg = {"ev_lm_begin": ev[i][0], "ev_lm_end": ev[i][1]} if i is not None else None
        dr.draft_step(ins, st, path, scores, debug=dbg, kv=kv)
        dr.accept(path, target, acc, em)

    for _ in range(W):
        step()
    torch.cuda.synchronize()
    assert dr.device_error() == 0, "device error during warm-up"

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        barrier(ws)
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(K):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(ws)
    ms = t0.elapsed_time(t1) / K
    ms_max = all_max(ms, ws)
    # accepted drafted tokens per request in the last timed step (synthetic targets: the first
    # mismatch sits at a seeded position, so this is the workload's own distribution)
    acc_hist = [int(v) for v in torch.bincount(acc.long().cpu(), minlength=Bk)[:Bk]]
    lm_ms = sum(a.elapsed_time(b) for a, b in ev) / K
    assert dr.device_error() == 0, "device error during the timed steps"

    # end to end through the host-buffer C call (inputs in, path/accepted out, every step)
    taps_h = st["taps"].cpu().pin_memory()
    nn_h = st["n_new"].cpu().pin_memory()
    bt_h = st["block_tokens"].cpu().pin_memory()
    tg_h = target.cpu().pin_memory()
    path_h = torch.empty((B, D), dtype=torch.int32).pin_memory()
    sc_h = torch.empty((B, D), dtype=torch.float32).pin_memory()
    acc_h = torch.empty((B,), dtype=torch.int32).pin_memory()
    em_h = torch.empty((B, Bk), dtype=torch.int32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (taps_h, nn_h, bt_h, tg_h))
    d2h = sum(t.numel() * t.element_size() for t in (path_h, sc_h, acc_h, em_h)) + 4
    dr.spec_step_host(st, taps_h, nn_h, bt_h, tg_h, path_h, sc_h, acc_h, em_h, kv=kv)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(E):
        derr = dr.spec_step_host(st, taps_h, nn_h, bt_h, tg_h, path_h, sc_h, acc_h, em_h, kv=kv)
        assert derr == 0
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    e2e_ms = all_max(e0.elapsed_time(e1) / E, ws)

    L_after = [int(v) + Bk for v in inputs.context_lengths(wl)]
    byt = accounting.step_bytes(dims, L_after, [Bk] * B)
    hbm, peak_kind = peaks()
    tpk, tpk_kind = bf16_sustained_tflops()
    flops = accounting.step_flops(dims, B)
    nk = dr.step_kernels()
    traffic = None
    rk_bytes = accounting.lmhead_bytes(dims, B * D)
    rk_gbs = rk_bytes / (lm_ms * 1e-3) / 1e9
    if B * D <= 8:
        rk_name = "k_slmhead (LM head + streaming top-16 + selector projection)"
        ratio = head_traffic_ratio()  # captured for the streaming kernel
        if ratio is not None:
            traffic = ratio * rk_bytes  # small-case capture scaled by the launch's bytes
        roof = {"bound": "hbm", "achieved": rk_gbs, "peak": hbm, "unit": "GB/s", "frac": rk_gbs / hbm}
    else:
        rk_name = "k_umma_head (tcgen05 LM head + top-16 + selector projection)"
        hflops = accounting.lmhead_flops(dims, B * D)
        tf = hflops / (lm_ms * 1e-3) / 1e12
        if B * D >= 128:  # a dense contraction: the tensor pipe bounds it
            roof = {"bound": "tensor", "achieved": tf, "peak": tpk, "unit": "TFLOP/s", "frac": tf / tpk}
        else:
            roof = {"bound": "hbm", "achieved": rk_gbs, "peak": hbm, "unit": "GB/s", "frac": rk_gbs / hbm}
    value = ws / (ms_max * 1e-3)  # draft steps/s over all ranks (one step = a rank's whole batch)
    line = {
        "metric": "DFlash2 draft steps/s (8-token block)",
        "value": value,
        "unit": "steps/s",
        "n_gpus": ws,
        "steps": K,
        "warmup": W,
        "ms_per_step": ms_max,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "q4k/bf16 weights, bf16 activations, fp32 accumulate",
        "data": "synthetic (seeded N(0,0.02) weights quantised to Q4_K, bf16 LM head/codebooks, N(0,1) taps and KV)",
        "config": bench_config(wl, ws),
        "request_steps_per_s": value * B,
        "accepted_hist": {"counts_by_accepted_0_to_7": acc_hist, "kind": "synthetic targets (seeded first mismatch)"},
        "step_hbm": {"algorithmic_bytes": byt["total"], "achieved_gbs": byt["total"] / (ms_max * 1e-3) / 1e9,
                     "frac_of_8tbs": byt["total"] / (ms_max * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
                     "frac_of_measured": byt["total"] / (ms_max * 1e-3) / 1e9 / hbm, "peak_kind": peak_kind},
        # the matrix products as a contraction (the bound of the 64-request workload), against the
        # measured sustained bf16 dense rate
        "step_tensor": {"flops": flops, "achieved_tflops": flops / (ms_max * 1e-3) / 1e12, "peak_tflops": tpk,
                        "frac": flops / (ms_max * 1e-3) / 1e12 / tpk, "peak_kind": tpk_kind,
                        "path": ("tcgen05 (TMEM) products above 64 block rows" if B * Bk > 64 else
                                 "mma.sync m16n8k16 streaming engine")},
        "roofline": {"kernel": rk_name, **roof, "traffic": traffic, "algorithmic_bytes": rk_bytes,
                     "avg_launch_ms": lm_ms,
                     "peak_kind": peak_kind if roof["bound"] == "hbm" else f"{tpk_kind} sustained bf16"},
        "e2e": {"value": ws / (e2e_ms * 1e-3), "unit": "steps/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": accounting.launches_per_step(dims, B, nk) * K,
        "clocks": clk.summary(),
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        hw_t, hw = host_copy_weights(w)
        st0 = inputs.make_state(wl, dev)
        st_h = host_state_for_request0(st0)
        del st0
        times, cores = oracle_step_time(wl, hw_t, hw, st_h, args.cpu_budget_s, 50)
        line["cpu_baseline"] = {"value": len(times) / sum(times), "unit": "steps/s", "cores": cores, "kind": "oracle",
                                "sample": f"{len(times)} full block steps of request 0 (fp64 C oracle, OpenMP)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
