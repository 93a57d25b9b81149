"""Shared parity machinery: run the CUDA path through the C ABI, run the oracle on
the same seeded inputs, compare.

Tolerances (the drafter's bf16-activation path against the fp64 oracle):
  * continuous tensors (hidden states, context rows, final rows, appended cache
    rows, candidate logits end to end): max |gpu - oracle| / max |oracle| <= 2e-2
    per row (per head vector for the cache rows), so an error confined to one row
    or head cannot hide under another row's larger values;
  * the selector's end-to-end path: the oracle's own path equals the GPU's, or the
    oracle scores the GPU's path within the bound the 2e-2 logit tolerance allows
    (twice the per-position tolerance, summed over the positions);
  * top-16 ids of every row are distinct;
  * stage-wise (the oracle fed the GPU's own bf16 operands, so only fp32
    accumulation order differs): logits and selector projection within 1e-3
    relative; top-16 ids identical except where the oracle's logits of the
    swapped ids lie within 1e-3 of each other; the selector path identical except
    where the oracle's scores of the two paths lie within 1e-3 * max(1, |score|);
  * integers (accepted length, emitted tokens, untouched cache rows): bit-exact.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from block_diffusion_drafter_dflash2_b200 import inputs

TOL = 2e-2
STAGE_TOL = 1e-3


def maxrel(g, o) -> float:
    """Worst row of max |g - o| / max |o| (each row normalised by its own largest oracle value;
    the last axis is the row)."""
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    if not o.size:
        return 0.0
    g = g.reshape(-1, o.shape[-1])
    o = o.reshape(-1, o.shape[-1])
    den = np.maximum(np.max(np.abs(o), axis=1), 1e-30)
    return float(np.max(np.max(np.abs(g - o), axis=1) / den))


def bits(t: torch.Tensor) -> np.ndarray:
    return oracle._np(t, np.uint16)


def f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return oracle.bf16_to_f64(bits(t))
    return t.detach().cpu().double().numpy()


def snapshot_request(wl: inputs.Workload, st: dict, b: int) -> dict:
    """Everything the oracle needs for request b, taken before the GPU step mutates the cache:
    the pages the window and this step's appends touch, gathered into a compact local cache."""
    d = wl.dims
    L0 = int(st["seq_len"][b])
    n = int(st["n_new"][b])
    Lb = L0 + n
    first = max(0, Lb - d.window + 1) // d.page_size
    last = (Lb - 1) // d.page_size
    phys = st["page_table"][b, first:last + 1].long()
    assert bool((phys >= 0).all()), "window pages must be backed"
    kc = [oracle._np(k.index_select(0, phys), np.uint16).copy() for k in st["k_cache"]]
    vc = [oracle._np(v.index_select(0, phys), np.uint16).copy() for v in st["v_cache"]]
    pt = np.full(last + 1, -1, np.int32)
    pt[first:] = np.arange(last + 1 - first, dtype=np.int32)
    return dict(b=b, L0=L0, n=n, first=first, last=last, phys=phys, kc=kc, vc=vc, kc0=[a.copy() for a in kc],
                vc0=[a.copy() for a in vc], pt=pt, taps=oracle._np(st["taps"][b]).copy(),
                btok=oracle._np(st["block_tokens"][b], np.int32).copy())


def run_gpu(wl: inputs.Workload, weights: dict, sample, state: dict | None = None):
    """Run the CUDA step once (with every debug output) and snapshot the sampled requests."""
    from block_diffusion_drafter_dflash2_b200.binding import Drafter
    d = wl.dims
    B, Bk, D, H = wl.batch, d.block, d.block - 1, d.hidden
    st = state if state is not None else inputs.make_state(wl, "cuda")
    snaps = {b: snapshot_request(wl, st, b) for b in sample}
    seq_before = st["seq_len"].clone()
    dr = Drafter(d, weights, B)
    dev = "cuda"
    path = torch.full((B, D), -7, dtype=torch.int32, device=dev)
    scores = torch.full((B, D), float("nan"), dtype=torch.float32, device=dev)
    dbg = {
        "hidden": torch.zeros((d.layers + 1, B * Bk, H), dtype=torch.float32, device=dev),
        "ctx": torch.zeros((B * Bk, H), dtype=torch.bfloat16, device=dev),
        "final_h": torch.zeros((B * D, H), dtype=torch.bfloat16, device=dev),
        "cand": torch.zeros((B * D, 16), dtype=torch.int32, device=dev),
        "cand_logit": torch.zeros((B * D, 16), dtype=torch.float32, device=dev),
        "z": torch.zeros((B * D, d.rank), dtype=torch.float32, device=dev),
    }
    dr.draft_step({"taps": st["taps"], "n_new": st["n_new"], "block_tokens": st["block_tokens"]}, st, path, scores,
                  debug=dbg)
    torch.cuda.synchronize()
    err = dr.device_error()
    return dict(wl=wl, drafter=dr, state=st, snaps=snaps, seq_before=seq_before, path=path, scores=scores, dbg=dbg,
                err=err)


def host_weights(weights: dict) -> tuple:
    """Host copies of the weights (the oracle's inputs) and the oracle's weight struct."""
    hw_t = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in weights.items() if k != "layers"}
    hw_t["layers"] = [{k: v.cpu() for k, v in L.items()} for L in weights["layers"]]
    return hw_t, oracle.HostWeights(hw_t)


def check_topk_row(g_ids, g_vals, o_ids, o_vals, o_at_g) -> None:
    """Top-16 of one row: GPU ids/logits against the oracle's, fed the same bf16 operand."""
    assert len(set(np.asarray(g_ids).tolist())) == len(g_ids), ("duplicate candidate ids", g_ids)
    # the GPU's own order: logit descending, smaller id first among equal logits
    for i in range(len(g_ids) - 1):
        assert g_vals[i] > g_vals[i + 1] or (g_vals[i] == g_vals[i + 1] and g_ids[i] < g_ids[i + 1]), \
            ("GPU list out of order", g_ids, g_vals)
    assert np.max(np.abs(g_vals - o_at_g) / np.maximum(1.0, np.abs(o_at_g))) <= STAGE_TOL, (g_vals, o_at_g)
    if np.array_equal(g_ids, o_ids):
        return
    thr = o_vals[-1]
    for i, gid in enumerate(g_ids):
        if gid not in set(o_ids.tolist()):
            assert o_at_g[i] >= thr - STAGE_TOL, ("GPU kept a candidate well below the 16th", gid, o_at_g[i], thr)
    # order may differ only among near-equal logits
    assert np.all(np.diff(o_at_g) <= STAGE_TOL), ("GPU order disagrees beyond near-ties", o_at_g)


def check_request(run: dict, hw_t: dict, hw: oracle.HostWeights, b: int, check_selector_e2e: bool = True) -> dict:
    wl = run["wl"]
    d = wl.dims
    Bk, D, H, K = d.block, d.block - 1, d.hidden, d.topk
    sn = run["snaps"][b]
    err, o_path, o_scores, o_sl, tr = oracle.draft_request(d, hw, sn["taps"], sn["n"], sn["btok"], sn["kc"], sn["vc"],
                                                           sn["pt"], sn["L0"], trace=True)
    assert err == 0, f"oracle error {err}"
    assert run["err"] == 0, f"device error bits {run['err']}"
    dbg = run["dbg"]
    rows = slice(b * Bk, (b + 1) * Bk)
    drows = slice(b * D, (b + 1) * D)
    report = {}
    # continuous values end to end
    hid = f64(dbg["hidden"][:, rows])
    for l in range(d.layers + 1):
        report[f"hidden{l}"] = maxrel(hid[l], tr["hidden"][l])
        assert report[f"hidden{l}"] <= TOL, (l, report)
    n = sn["n"]
    if n:
        report["ctx"] = maxrel(f64(dbg["ctx"][rows][:n]), tr["ctx"][:n])
        assert report["ctx"] <= TOL, report
    g_fh = dbg["final_h"][drows]
    report["final_h"] = maxrel(f64(g_fh), tr["final_h"])
    assert report["final_h"] <= TOL, report
    # cache: appended rows close, all other rows of the touched pages untouched
    L0 = sn["L0"]
    for l in range(d.layers):
        gk = oracle._np(run["state"]["k_cache"][l].index_select(0, sn["phys"]), np.uint16)
        gv = oracle._np(run["state"]["v_cache"][l].index_select(0, sn["phys"]), np.uint16)
        new = np.zeros(gk.shape[0] * d.page_size, bool)
        new[L0 - sn["first"] * d.page_size: L0 - sn["first"] * d.page_size + n] = True
        new = new.reshape(gk.shape[0], d.page_size)
        for g_, o_, before in ((gk, sn["kc"][l], sn["kc0"][l]), (gv, sn["vc"][l], sn["vc0"][l])):
            gt = np.transpose(g_, (0, 2, 1, 3))  # [page][slot][head][dim]
            ot = np.transpose(o_, (0, 2, 1, 3))
            bt = np.transpose(before, (0, 2, 1, 3))
            assert np.array_equal(gt[~new], bt[~new]), "GPU wrote outside the appended rows"
            if n:  # [rows][head][dim]: one tolerance per head vector
                r = maxrel(oracle.bf16_to_f64(gt[new]), oracle.bf16_to_f64(ot[new]))
                report[f"cache{l}"] = max(report.get(f"cache{l}", 0.0), r)
                assert r <= TOL, report
    # stage-wise top-16: oracle LM head on the GPU's own bf16 rows
    lm = hw_t["lm_head"]
    o_ids, o_vals = oracle.lmhead_topk(g_fh, lm, K)
    g_ids = dbg["cand"][drows].cpu().numpy()
    g_vals = dbg["cand_logit"][drows].cpu().double().numpy()
    o_at_g = oracle.logits_at(g_fh, lm, g_ids)
    for t in range(D):
        check_topk_row(g_ids[t], g_vals[t], o_ids[t], o_vals[t], o_at_g[t])
    # stage-wise selector projection
    z_o = oracle.matmul(1, hw_t["sel_proj"], d.rank, H, f64(g_fh))
    g_z = dbg["z"][drows].cpu().double().numpy()
    report["z"] = maxrel(g_z, z_o)
    assert report["z"] <= STAGE_TOL, report
    # stage-wise selector: the oracle's Viterbi on the GPU's candidates, logits and z
    g_path = run["path"][b].cpu().numpy()
    g_scores = run["scores"][b].cpu().double().numpy()
    x0 = int(sn["btok"][0])
    s_path, s_scores = oracle.selector(g_ids, g_vals, g_z, x0, hw_t["cb_a"], hw_t["cb_b"])
    if not np.array_equal(s_path, g_path):
        tau = oracle.selector_trans(g_ids, g_z, x0, hw_t["cb_a"], hw_t["cb_b"])
        idx = [int(np.where(g_ids[t] == g_path[t])[0][0]) for t in range(D)]
        sc = g_vals[0, idx[0]] + tau[0, 0, idx[0]]
        for t in range(1, D):
            sc += g_vals[t, idx[t]] + tau[t, idx[t - 1], idx[t]]
        assert abs(sc - s_scores[-1]) <= STAGE_TOL * max(1.0, abs(s_scores[-1])), ("path differs beyond a near-tie",
                                                                                    g_path, s_path)
        report["path_near_tie"] = True
    else:
        assert np.all(np.abs(g_scores - s_scores) <= STAGE_TOL * np.maximum(1.0, np.abs(s_scores))), (g_scores, s_scores)
    # candidate logits end to end (oracle rows, GPU ids)
    lm_rows = oracle.bf16_to_f64(oracle._np(lm[torch.as_tensor(g_ids.reshape(-1), dtype=torch.long)])).reshape(D, K, H)
    e2e = np.einsum("tkh,th->tk", lm_rows, tr["final_h"])
    report["cand_logit_e2e"] = maxrel(g_vals, e2e)
    assert report["cand_logit_e2e"] <= TOL, report
    # seq_len advanced by n_new
    assert int(run["state"]["seq_len"][b]) == int(run["seq_before"][b]) + n
    # the oracle's own end-to-end path against the GPU's: equal, or the oracle scores both paths
    # within the bound the end-to-end logit tolerance allows
    report["oracle_path_equal_gpu_path"] = bool(np.array_equal(o_path, g_path))
    if not report["oracle_path_equal_gpu_path"]:
        margin, bound = e2e_path_margin(hw_t, tr, x0, o_path, g_path)
        report["e2e_path_margin"], report["e2e_path_bound"] = margin, bound
        assert margin <= bound, ("end-to-end path differs beyond the logit tolerance", o_path, g_path, margin, bound)
    return report


def e2e_path_margin(hw_t: dict, tr: dict, x0: int, o_path, g_path):
    """The oracle's score of its own path minus its score of the GPU's path (both in the oracle's
    fp64 logits and transitions), and the largest gap the 2e-2 end-to-end tolerance permits:
    a path's score moves by at most TOL * (max |logit| + max |transition|) per position, and
    the GPU maximised its own scores, so the oracle's two scores differ by at most twice that
    summed over the positions."""
    lm, A, Bc = hw_t["lm_head"], hw_t["cb_a"], hw_t["cb_b"]
    fh, z = tr["final_h"], tr["z"]
    D = fh.shape[0]

    def rows(t, ids):
        return oracle.bf16_to_f64(oracle._np(t[torch.as_tensor(np.asarray(ids, np.int64))]))

    def score(path):
        prev = np.concatenate([[x0], path[:-1]])
        lg = np.einsum("th,th->t", rows(lm, path), fh)
        tau = np.einsum("tr,tr,tr->t", rows(A, prev), z, rows(Bc, path))
        return float(lg.sum() + tau.sum())

    cand = tr["cand"]
    bound = 0.0
    for t in range(D):
        lmax = float(np.max(np.abs(tr["cand_logit"][t])))
        srcs = [x0] if t == 0 else cand[t - 1]
        tmax = float(np.max(np.abs(rows(A, srcs) * z[t]) @ np.abs(rows(Bc, cand[t])).T))
        bound += 2.0 * TOL * (lmax + tmax)
    return score(np.asarray(o_path)) - score(np.asarray(g_path)), bound


def check_accept(run: dict) -> None:
    wl = run["wl"]
    dr = run["drafter"]
    B, Bk = wl.batch, wl.dims.block
    target = inputs.make_targets(wl, run["path"]).to("cuda")
    acc = torch.full((B,), -5, dtype=torch.int32, device="cuda")
    em = torch.full((B, Bk), -5, dtype=torch.int32, device="cuda")
    dr.accept(run["path"], target, acc, em)
    torch.cuda.synchronize()
    o_acc, o_em = oracle.accept(run["path"].cpu(), target.cpu())
    assert np.array_equal(acc.cpu().numpy(), o_acc) and np.array_equal(em.cpu().numpy(), o_em)
