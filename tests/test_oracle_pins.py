"""Pins for the CPU oracle: closed forms, invariants, brute force and library routines.

Each test fixes the oracle to something other than itself, chosen so that a
plausible slip (a dropped term, a wrong sign or index, a transposed operand)
fails at least one of them.
"""
import dataclasses
import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle
from block_diffusion_drafter_dflash2_b200 import inputs

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))
rng = np.random.default_rng(1234)


def bf16_bits(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(b):
    return oracle.bf16_to_f64(b)


# ------------------------------------------------------------------ number formats

def test_fp16_decode_matches_numpy():
    bits = np.concatenate([np.arange(0, 0x7C00, 7, dtype=np.uint16), np.array([1, 2, 0x3C00, 0x8001, 0xBC00], np.uint16)])
    lib = oracle.lib()
    ours = np.array([lib.orc_fp16(int(b)) for b in bits])
    ref = bits.view(np.float16).astype(np.float64)
    assert np.array_equal(ours, ref)


def test_bf16_round_half_even_matches_torch():
    x = np.concatenate([rng.standard_normal(4000).astype(np.float32) * 10.0 ** rng.integers(-6, 6, 4000),
                        np.float32([1 + 2 ** -8, 1 + 3 * 2 ** -8, -1 - 2 ** -8, 3.0e38])])
    ours = np.array([oracle.to_bf16(float(v)) for v in x], np.uint16)
    assert np.array_equal(ours, bf16_bits(x))


# ------------------------------------------------------------------ Q4_K

def _pack_block(d16, dm16, sc, mn, q):
    """Hand packing of one super-block from the byte layout (independent of the generator)."""
    b = bytearray(144)
    b[0:2] = np.float16(d16).tobytes()
    b[2:4] = np.float16(dm16).tobytes()
    s = sum(int(v) << (6 * j) for j, v in enumerate(sc))
    m = sum(int(v) << (6 * j) for j, v in enumerate(mn))
    b[4:10] = s.to_bytes(6, "little")
    b[10:16] = m.to_bytes(6, "little")
    for e in range(0, 256, 2):
        b[16 + e // 2] = int(q[e]) | (int(q[e + 1]) << 4)
    return np.frombuffer(bytes(b), np.uint8)


def test_q4k_hand_block():
    # d = 1, dmin = 0.5, sc_j = j + 1, m_j = 2j, q_e = e mod 16:
    # weight e = (j+1)*(e mod 16) - 0.5*2j = (j+1)*(e mod 16) - j, j = e // 32
    sc = [j + 1 for j in range(8)]
    mn = [2 * j for j in range(8)]
    q = [e % 16 for e in range(256)]
    got = oracle.q4k_dequant(_pack_block(1.0, 0.5, sc, mn, q))
    want = np.array([(e // 32 + 1) * (e % 16) - e // 32 for e in range(256)], np.float64)
    assert np.array_equal(got, want)


def test_q4k_each_nibble_moves_one_weight():
    sc = [63, 1, 7, 33, 2, 60, 5, 19]
    mn = [0, 63, 1, 2, 40, 3, 9, 17]
    q = list(rng.integers(0, 15, 256))
    base = oracle.q4k_dequant(_pack_block(0.25, 0.125, sc, mn, q))
    for e in [0, 1, 31, 32, 63, 100, 129, 200, 255]:
        q2 = list(q)
        q2[e] += 1
        diff = oracle.q4k_dequant(_pack_block(0.25, 0.125, sc, mn, q2)) - base
        assert np.count_nonzero(diff) == 1 and diff[e] == 0.25 * sc[e // 32]


def test_q4k_all_zero_block_is_exact():
    z = torch.zeros((4, 512))
    assert np.array_equal(oracle.q4k_dequant(inputs.quantize_q4k(z)), np.zeros(4 * 512))


def test_mlx4_hand_group_and_round_trip():
    """MLX 4-bit group-64: a hand-packed group decodes to scale * q + bias exactly (scale 0.5,
    bias -3, q = e mod 16), nibble order low first; the synthetic quantiser's round trip on
    N(0, 0.02) rows has the relative L2 error of 4-bit codes over a group's range (about 0.1)."""
    q = [e % 16 for e in range(64)]
    b = bytearray(36)
    for e in range(0, 64, 2):
        b[e // 2] = q[e] | (q[e + 1] << 4)
    b[32:34] = bf16_bits([0.5]).tobytes()
    b[34:36] = bf16_bits([-3.0]).tobytes()
    got = oracle.mlx4_dequant(np.frombuffer(bytes(b), np.uint8))
    assert np.array_equal(got, 0.5 * np.array(q) - 3.0)
    w = torch.randn(64, 512, generator=torch.Generator().manual_seed(5)) * 0.02
    enc = inputs.quantize_mlx4(w)
    dec = oracle.mlx4_dequant(enc.numpy()).reshape(64, 512)
    rel = np.linalg.norm(dec - w.double().numpy()) / np.linalg.norm(w.double().numpy())
    assert 0.05 < rel < 0.15, rel


def test_q8_0_hand_block_and_round_trip():
    """Q8_0: a hand-packed block decodes to d * q exactly (d = 0.25, q = -127, -3, 0, 5, 127, ...);
    the round trip on N(0, 0.02) rows has the error of 8-bit codes (well under 1 %)."""
    qv = np.array([-127, -3, 0, 5, 127] + list(range(-13, 14)), np.int8)
    b = np.frombuffer(np.float16(0.25).tobytes() + qv.tobytes(), np.uint8)
    got = oracle.q8_0_dequant(b)
    assert np.array_equal(got, 0.25 * qv.astype(np.float64))
    w = torch.randn(64, 512, generator=torch.Generator().manual_seed(6)) * 0.02
    dec = oracle.q8_0_dequant(inputs.quantize_q8_0(w).numpy()).reshape(64, 512)
    rel = np.linalg.norm(dec - w.double().numpy()) / np.linalg.norm(w.double().numpy())
    assert 0.001 < rel < 0.01, rel


@pytest.mark.parametrize("fmt", [2, 3])
def test_matmul_of_alternate_codecs_matches_decoded_numpy(fmt):
    N, K = 48, 512
    w = torch.randn(N, K, generator=torch.Generator().manual_seed(7 + fmt)) * 0.02
    enc = (inputs.quantize_mlx4 if fmt == 2 else inputs.quantize_q8_0)(w)
    dec = (oracle.mlx4_dequant if fmt == 2 else oracle.q8_0_dequant)(enc.numpy()).reshape(N, K)
    x = rng.standard_normal((5, K))
    assert np.allclose(oracle.matmul(fmt, enc, N, K, x), x @ dec.T, rtol=1e-12, atol=1e-12)


def test_q4k_round_trip_matches_card_error():
    """FastFlowLM card: about 0.07 relative L2 per Q4_K matrix (N(0, 0.02) weights here)."""
    w = torch.randn((256, 4096), generator=torch.Generator().manual_seed(7)) * 0.02
    deq = oracle.q4k_dequant(inputs.quantize_q4k(w)).reshape(w.shape)
    wd = w.double().numpy()
    rel = np.linalg.norm(deq - wd) / np.linalg.norm(wd)
    card = GOLD["q4k_relative_l2_per_matrix"]["value"]
    assert 0.04 <= rel <= 0.10, rel
    assert abs(rel - card) < 0.03
    # every weight within one quantisation step of its sub-block (codes never saturate badly)
    blk = (wd - deq).reshape(256, -1, 32)
    rng_ = wd.reshape(256, -1, 32)
    step = (rng_.max(-1) - np.minimum(rng_.min(-1), 0)) / 15.0
    assert np.all(np.abs(blk).max(-1) <= step * 1.2 + 1e-9)


# ------------------------------------------------------------------ matmul

@pytest.mark.parametrize("fmt", [0, 1])
def test_matmul_matches_numpy(fmt):
    N, K, M = 48, 512, 5
    if fmt == 0:
        W = inputs.quantize_q4k(torch.randn((N, K)) * 0.02)
        dense = oracle.q4k_dequant(W).reshape(N, K)
    else:
        Wf = rng.standard_normal((N, K)).astype(np.float32)
        W = bf16_bits(Wf)
        dense = bits_to_f64(W)
    X = rng.standard_normal((M, K))
    got = oracle.matmul(fmt, W, N, K, X)
    assert np.allclose(got, X @ dense.T, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ RMSNorm, RoPE

def test_rmsnorm_closed_forms():
    x = rng.standard_normal(512) * 3.0
    one = bf16_bits(np.ones(512))
    y = oracle.rmsnorm(x, one, 0.0)
    assert np.isclose(np.sqrt(np.mean(y ** 2)), 1.0, atol=1e-12)
    assert np.allclose(oracle.rmsnorm(7.5 * x, one, 0.0), y, atol=1e-12)
    w = bf16_bits(rng.uniform(0.5, 2.0, 512))
    assert np.allclose(oracle.rmsnorm(x, w, 0.0), y * bits_to_f64(w), atol=1e-12)
    # eps enters under the square root: mean(x^2) = 1 exactly for a +-1 vector
    s = np.where(rng.random(512) < 0.5, -1.0, 1.0)
    assert np.allclose(oracle.rmsnorm(s, one, 0.25), s / np.sqrt(1.25), atol=1e-14)


def test_rope_invariants():
    hd, theta = 128, 1.0e6
    q = rng.standard_normal(hd)
    k = rng.standard_normal(hd)
    assert np.allclose(oracle.rope(q, 0, theta), q, atol=0)
    r = oracle.rope(q, 12345, theta)
    half = hd // 2
    assert np.allclose(q[:half] ** 2 + q[half:] ** 2, r[:half] ** 2 + r[half:] ** 2, atol=1e-10)
    a = np.dot(oracle.rope(q, 100, theta), oracle.rope(k, 37, theta))
    b = np.dot(oracle.rope(q, 5100, theta), oracle.rope(k, 5037, theta))
    assert np.isclose(a, b, atol=1e-9)
    # pair i rotates by pos * theta^(-2i/hd): measure the angle of unit vectors e_i
    for i in [0, 1, 10, 63]:
        e = np.zeros(hd)
        e[i] = 1.0
        pos = 3
        v = oracle.rope(e, pos, theta)
        ang = np.arctan2(v[i + half], v[i])
        want = np.angle(np.exp(1j * pos * theta ** (-2.0 * i / hd)))
        assert np.isclose(ang, want, atol=1e-12)
        assert np.count_nonzero(np.abs(v) > 1e-15) <= 2


# ------------------------------------------------------------------ dynamic convolution

def _dc_tensors(H, w_val=None, s0=1.0, s1=0.0):
    G = H // 4
    W = bf16_bits(np.zeros((2 * G, H)) if w_val is None else w_val)
    return W, bf16_bits(np.full(H, s0)), bf16_bits(np.full(H, s1))


def test_dynconv_special_cases():
    Bk, H = 8, 64
    x = rng.standard_normal((Bk, H))
    W, s0, s1 = _dc_tensors(H)
    assert np.allclose(oracle.dynconv(x, W, s0, s1), x, atol=0)
    W, s0, s1 = _dc_tensors(H, s0=1.0, s1=1.0)
    prev = np.vstack([np.zeros((1, H)), x[:-1]])
    assert np.allclose(oracle.dynconv(x, W, s0, s1), x + prev, atol=1e-15)


def test_dynconv_causal_and_grouped():
    Bk, H = 8, 64
    G = H // 4
    x = rng.standard_normal((Bk, H))
    Wv = rng.standard_normal((2 * G, H)) * 0.3
    W, s0, s1 = _dc_tensors(H, Wv, 1.0, 0.5)
    y = oracle.dynconv(x, W, s0, s1)
    x2 = x.copy()
    x2[5] += rng.standard_normal(H)
    y2 = oracle.dynconv(x2, W, s0, s1)
    assert np.array_equal(y[:5], y2[:5]) and not np.allclose(y[5], y2[5])
    # one saturated gate row r (< H/4) moves exactly channels 4r..4r+3 of the current tap
    Wv = np.zeros((2 * G, H))
    Wv[3, :] = 1000.0
    W, s0, s1 = _dc_tensors(H, Wv, 1.0, 0.0)
    x = np.abs(rng.standard_normal((Bk, H))) + 0.1
    y = oracle.dynconv(x, W, s0, s1)
    ch = np.zeros(H, bool)
    ch[12:16] = True
    assert np.allclose(y[:, ch], 2.0 * x[:, ch], atol=1e-12)
    assert np.allclose(y[:, ~ch], x[:, ~ch], atol=0)
    # a saturated gate in the second half drives the previous tap of the same 4 channels
    Wv = np.zeros((2 * G, H))
    Wv[G + 2, :] = 1000.0
    W, s0, s1 = _dc_tensors(H, Wv, 1.0, 0.0)
    y = oracle.dynconv(x, W, s0, s1)
    prev = np.vstack([np.zeros((1, H)), x[:-1]])
    ch = np.zeros(H, bool)
    ch[8:12] = True
    assert np.allclose(y[:, ch], x[:, ch] + prev[:, ch], atol=1e-12)
    assert np.allclose(y[:, ~ch], x[:, ~ch], atol=0)


# ------------------------------------------------------------------ attention

def _attn_setup(nq=4, nkv=2, window=40, L0=70, n_new=5, Bk=6, pages=8):
    d = inputs.Dims(layers=1, hidden=256, ffn=256, n_q=nq, n_kv=nkv, head_dim=128, window=window, vocab=64,
                    n_taps=1, block=Bk, topk=4, rank=4)
    hd = 128
    kc = bf16_bits(rng.standard_normal((pages, nkv, 16, hd)))
    vc = bf16_bits(rng.standard_normal((pages, nkv, 16, hd)))
    pt = np.array(rng.permutation(pages), np.int32)
    q = rng.standard_normal((Bk, nq * hd))
    kb = rng.standard_normal((Bk, nkv * hd))
    vb = rng.standard_normal((Bk, nkv * hd))
    return d, q, kb, vb, kc, vc, pt, L0 + n_new


def _cache_rows(cache, pt, head, j0, j1):
    return np.stack([bits_to_f64(cache[pt[j // 16], head, j % 16]) for j in range(j0, j1)]) if j1 > j0 \
        else np.zeros((0, 128))


def test_attention_zero_query_is_window_mean():
    """q = 0 makes the softmax uniform: the output is the mean of exactly the visible values."""
    d, q, kb, vb, kc, vc, pt, Lb = _attn_setup()
    q[:] = 0
    err, o = oracle.attention(d, q, kb, vb, kc, vc, pt, Lb)
    assert err == 0
    grp = d.n_q // d.n_kv
    for t in range(d.block):
        j0 = max(0, Lb + t - d.window + 1)
        for h in range(d.n_q):
            kvh = h // grp
            vis = np.vstack([_cache_rows(vc, pt, kvh, j0, Lb), vb[:, kvh * 128:(kvh + 1) * 128]])
            assert np.allclose(o[t, h * 128:(h + 1) * 128], vis.mean(0), atol=1e-12)


def test_attention_one_dominant_key_and_gqa_mapping():
    d, q, kb, vb, kc, vc, pt, Lb = _attn_setup()
    # make block key 2 of kv head 1 dominate for every query of heads 2, 3
    kb[:, 128:] = 0
    kb[2, 128:] = 1.0
    q[:, 2 * 128:4 * 128] = 400.0
    kc_z = kc.copy()
    kc_z[:, 1] = 0  # cache keys of kv head 1 score 0
    err, o = oracle.attention(d, q, kb, vb, kc_z, vc, pt, Lb)
    assert err == 0
    for h in (2, 3):
        assert np.allclose(o[:, h * 128:(h + 1) * 128], np.broadcast_to(vb[2, 128:], (d.block, 128)), atol=1e-9)
    # constant values for kv head 0 -> heads 0, 1 return the constant whatever the scores
    vc_c = vc.copy()
    vc_c[:, 0] = bf16_bits(np.full(128, 0.75))
    vb_c = vb.copy()
    vb_c[:, :128] = 0.75
    err, o = oracle.attention(d, q, kb, vb_c, kc, vc_c, pt, Lb)
    assert np.allclose(o[:, :2 * 128], 0.75, atol=1e-12)


def test_attention_window_bounds():
    d, q, kb, vb, kc, vc, pt, Lb = _attn_setup()
    err, o = oracle.attention(d, q, kb, vb, kc, vc, pt, Lb)
    # keys older than the window of block row 0 do not matter
    first = Lb - d.window + 1
    kc2, vc2 = kc.copy(), vc.copy()
    for j in range(0, first):
        kc2[pt[j // 16], :, j % 16] = bf16_bits(rng.standard_normal((d.n_kv, 128)))
        vc2[pt[j // 16], :, j % 16] = bf16_bits(rng.standard_normal((d.n_kv, 128)))
    _, o2 = oracle.attention(d, q, kb, vb, kc2, vc2, pt, Lb)
    assert np.array_equal(o, o2)
    # the key at first is seen by row 0 only; the key at first + 1 by rows 0 and 1
    kc3 = kc.copy()
    kc3[pt[first // 16], :, first % 16] = bf16_bits(rng.standard_normal((d.n_kv, 128)))
    _, o3 = oracle.attention(d, q, kb, vb, kc3, vc, pt, Lb)
    assert not np.allclose(o3[0], o[0]) and np.array_equal(o3[1:], o[1:])
    # pages wholly before the window may be unmapped; an unmapped page inside it is an error
    pt2 = pt.copy()
    pt2[: first // 16] = -1
    err2, o4 = oracle.attention(d, q, kb, vb, kc, vc, pt2, Lb)
    assert err2 == 0 and np.array_equal(o4, o)
    pt3 = pt.copy()
    pt3[(Lb - 1) // 16] = -1
    err3, _ = oracle.attention(d, q, kb, vb, kc, vc, pt3, Lb)
    assert err3 != 0


def test_attention_short_context_sees_all():
    """Lb < window: every cached key and every block key is visible to every row."""
    d, q, kb, vb, kc, vc, pt, Lb = _attn_setup(window=4096, L0=20, n_new=3)
    q[:] = 0
    err, o = oracle.attention(d, q, kb, vb, kc, vc, pt, Lb)
    vis = np.vstack([_cache_rows(vc, pt, 0, 0, Lb), vb[:, :128]])
    assert err == 0 and np.allclose(o[:, :128], vis.mean(0), atol=1e-12)


def _brute_attention(d, q, kb, vb, kc, vc, pt, Lb):
    """Attention from its textbook definition, one (block row, query head) at a time: collect
    the keys the row may see (cache positions inside the window, looked up page by page, then
    every block key), scores q.k / sqrt(head_dim), softmax, weighted sum of the values."""
    hd, grp = d.head_dim, d.n_q // d.n_kv
    o = np.zeros_like(q)
    for t in range(d.block):
        p = Lb + t
        j0 = max(0, p - d.window + 1)
        for h in range(d.n_q):
            kvh = h // grp
            keys = [bits_to_f64(kc[pt[j // 16], kvh, j % 16]) for j in range(j0, Lb)]
            vals = [bits_to_f64(vc[pt[j // 16], kvh, j % 16]) for j in range(j0, Lb)]
            keys += [kb[u, kvh * hd:(kvh + 1) * hd] for u in range(d.block)]
            vals += [vb[u, kvh * hd:(kvh + 1) * hd] for u in range(d.block)]
            s = np.array([float(np.dot(q[t, h * hd:(h + 1) * hd], k)) for k in keys]) / np.sqrt(hd)
            w = np.exp(s - s.max())
            w /= w.sum()
            o[t, h * hd:(h + 1) * hd] = sum(wi * v for wi, v in zip(w, vals))
    return o


@pytest.mark.parametrize("window,L0,n_new", [(40, 70, 5), (4096, 20, 3), (17, 33, 6)])
def test_attention_matches_brute_force_softmax(window, L0, n_new):
    """Random, non-degenerate queries (scores of order one, so neither uniform nor saturated),
    GQA groups of 2, a shuffled page table and the window cutting through pages: every output
    element equals the brute-force softmax attention."""
    d, q, kb, vb, kc, vc, pt, Lb = _attn_setup(window=window, L0=L0, n_new=n_new)
    err, o = oracle.attention(d, q, kb, vb, kc, vc, pt, Lb)
    assert err == 0
    want = _brute_attention(d, q, kb, vb, kc, vc, pt, Lb)
    assert np.allclose(o, want, rtol=0, atol=1e-12)
    s = q[0, :128] @ kb[:, :128].T / np.sqrt(128)
    assert 0.3 < s.std() < 3.0  # the case exercises the softmax away from its limits


def test_attention_softmax_scale_closed_form():
    """Two visible keys (a one-token window leaves only the block's two keys) along one axis:
    the weights are exp(a c_u / sqrt(128)) normalised, so with c_0 - c_1 = sqrt(128) ln 3 the
    head with a = 1 returns 3/4 of value 0 and 1/4 of value 1, the head with a = 2 returns
    9/10 and 1/10.  Any other score scale (1/128, none) moves these numbers."""
    d = inputs.Dims(layers=1, hidden=256, ffn=256, n_q=2, n_kv=1, head_dim=128, window=1, vocab=64,
                    n_taps=1, block=2, topk=4, rank=4)
    hd = 128
    kc = bf16_bits(rng.standard_normal((1, 1, 16, hd)))
    vc = bf16_bits(rng.standard_normal((1, 1, 16, hd)))
    pt = np.zeros(1, np.int32)
    q = np.zeros((2, 2 * hd))
    q[:, 0] = 1.0
    q[:, hd] = 2.0
    kb = np.zeros((2, hd))
    kb[0, 0] = 0.5 + np.sqrt(128.0) * np.log(3.0)
    kb[1, 0] = 0.5
    vb = np.zeros((2, hd))
    vb[0, 1] = 1.0
    vb[1, 2] = 1.0
    err, o = oracle.attention(d, q, kb, vb, kc, vc, pt, 3)
    assert err == 0
    for t in range(2):
        assert np.allclose(o[t, [1, 2]], [0.75, 0.25], atol=1e-12)
        assert np.allclose(o[t, [hd + 1, hd + 2]], [0.9, 0.1], atol=1e-12)


# ------------------------------------------------------------------ top-k

def test_topk_matches_full_sort_with_ties():
    for n, k in [(1000, 16), (40, 16), (16, 16), (5000, 3)]:
        x = np.round(rng.standard_normal(n) * 4) / 4  # many exact ties
        ids, vals = oracle.topk(x, k)
        order = np.lexsort((np.arange(n), -x))[:k]  # value descending, id ascending
        assert np.array_equal(ids, order) and np.array_equal(vals, x[order])


# ------------------------------------------------------------------ Viterbi

def _brute_force_path(unary, trans):
    D, K = unary.shape
    best, arg = None, None
    for p in itertools.product(range(K), repeat=D):
        s = unary[0, p[0]] + trans[0, 0, p[0]]
        for t in range(1, D):
            s += unary[t, p[t]] + trans[t, p[t - 1], p[t]]
        if best is None or s > best:  # first (lexicographically smallest) maximiser kept
            best, arg = s, p
    return np.array(arg), best


@pytest.mark.parametrize("D,K", [(1, 5), (2, 4), (4, 6), (5, 7)])
def test_viterbi_matches_exhaustive(D, K):
    for _ in range(5):
        u = rng.standard_normal((D, K)) * 3
        tr = rng.standard_normal((D, K, K)) * 3
        idx, sc = oracle.viterbi(u, tr)
        p, best = _brute_force_path(u, tr)
        assert np.array_equal(idx, p)
        assert np.isclose(sc[-1], best, atol=1e-12)
        # prefix scores are the partial sums of the chosen path
        s = u[0, p[0]] + tr[0, 0, p[0]]
        assert np.isclose(sc[0], s)
        for t in range(1, D):
            s += u[t, p[t]] + tr[t, p[t - 1], p[t]]
            assert np.isclose(sc[t], s)


def test_viterbi_exhaustive_full_block_16_candidates():
    """All 16^7 paths of a block of 8 (7 drafted tokens, top 16) scored one by one."""
    D, K = 7, 16
    u = rng.standard_normal((D, K)) * 4
    tr = rng.standard_normal((D, K, K)) * 4
    idx, sc = oracle.viterbi(u, tr)
    # prefix part over positions 0..2 (4096 prefixes), suffix part over 3..6 given position 2
    j = np.indices((K,) * 3).reshape(3, -1)
    pre = u[0, j[0]] + tr[0, 0, j[0]] + u[1, j[1]] + tr[1, j[0], j[1]] + u[2, j[2]] + tr[2, j[1], j[2]]
    s = np.indices((K,) * 4).reshape(4, -1)
    suf_wo = u[3, s[0]] + u[4, s[1]] + tr[4, s[0], s[1]] + u[5, s[2]] + tr[5, s[1], s[2]] + u[6, s[3]] + tr[6, s[2], s[3]]
    best, arg = -np.inf, None
    for c0 in range(0, pre.size, 256):
        tot = pre[c0:c0 + 256, None] + tr[3][j[2, c0:c0 + 256]][:, s[0]] + suf_wo[None, :]
        m = tot.max()
        if m > best:
            f = np.argmax(tot)
            best, arg = m, (c0 + f // tot.shape[1], f % tot.shape[1])
    path = np.concatenate([j[:, arg[0]], s[:, arg[1]]])
    assert np.array_equal(idx, path) and np.isclose(sc[-1], best, atol=1e-9)


def test_viterbi_zero_transitions_is_greedy_and_ties_pick_smaller():
    u = rng.standard_normal((6, 16))
    idx, _ = oracle.viterbi(u, np.zeros((6, 16, 16)))
    assert np.array_equal(idx, u.argmax(1))
    u = np.zeros((3, 4))
    idx, sc = oracle.viterbi(u, np.zeros((3, 4, 4)))
    assert np.array_equal(idx, [0, 0, 0]) and np.all(sc == 0)


# ------------------------------------------------------------------ selector

def test_selector_zero_codebooks_is_top1_path():
    D, K, R, V = 7, 16, 8, 64
    cand = np.stack([rng.permutation(V)[:K] for _ in range(D)]).astype(np.int32)
    cl = -np.sort(-rng.standard_normal((D, K)), axis=1)
    z = rng.standard_normal((D, R))
    zero = bf16_bits(np.zeros((V, R)))
    path, sc = oracle.selector(cand, cl, z, 5, zero, zero)
    assert np.array_equal(path, cand[:, 0]) and np.allclose(sc, np.cumsum(cl[:, 0]))


def test_selector_chain_codebooks_force_consecutive_ids():
    """A = identity, B = identity shifted by one: tau(a -> b) = z_t[a] iff b = a + 1.
    With a large z the chosen path follows x0+1, x0+2, ... even from low candidate ranks,
    which pins the source (previous position / first block token) and destination roles."""
    D, K, V = 7, 16, 64
    R = V
    A = np.eye(V)
    Bc = np.zeros((V, V))
    for b in range(1, V):
        Bc[b, b - 1] = 1.0
    x0 = 20
    g = np.random.default_rng(77)  # own stream: independent of the order the other tests run in
    cand = np.zeros((D, K), np.int32)
    for t in range(D):
        # the alternative first token x0 + 30 below must have no chain successor among the candidates
        others = [i for i in g.permutation(V) if i != x0 + 1 + t and i != x0 + 31][:K - 1]
        cand[t] = others[:K - 1 - (t % 5)] + [x0 + 1 + t] + others[K - 1 - (t % 5):K - 1]
    cl = -np.sort(-g.standard_normal((D, K)), axis=1)
    z = np.full((D, R), 50.0)
    path, sc = oracle.selector(cand, cl, z, x0, bf16_bits(A), bf16_bits(Bc))
    assert np.array_equal(path, x0 + 1 + np.arange(D))
    # another first token loses exactly the first transition (z = 50) and nothing else
    path2, sc2 = oracle.selector(cand, cl, z, x0 + 30, bf16_bits(A), bf16_bits(Bc))
    assert np.array_equal(path2, path) and np.allclose(sc - sc2, 50.0, atol=1e-9)


# ------------------------------------------------------------------ acceptance

def test_accept_invariants():
    B, Bk = 200, 8
    D = Bk - 1
    draft = rng.integers(0, 5, (B, D)).astype(np.int32)
    target = rng.integers(0, 5, (B, Bk)).astype(np.int32)
    m = rng.integers(0, Bk, B)
    for b in range(B):
        target[b, :m[b]] = draft[b, :m[b]]
        if m[b] < D:
            target[b, m[b]] = draft[b, m[b]] + 1
    acc, em = oracle.accept(draft, target)
    assert np.array_equal(acc, m)
    for b in range(B):
        n = acc[b]
        assert 0 <= n <= D
        assert np.array_equal(em[b, :n], draft[b, :n]) and em[b, n] == target[b, n]
        assert np.all(em[b, n + 1:] == -1)
    assert np.all((acc == D) == np.all(draft == target[:, :D], axis=1))


def test_accept_chain_next_round_inputs():
    """The next round starts from the token the target kept (emitted[n], its own argmax at the
    first disagreement, or its bonus token after a full match) and fuses n + 1 new context rows:
    the n accepted drafted tokens and that token."""
    B, Bk, mask = 300, 8, 8191
    D = Bk - 1
    draft = rng.integers(0, 6, (B, D)).astype(np.int32)
    target = rng.integers(0, 6, (B, Bk)).astype(np.int32)
    m = rng.integers(0, Bk, B)
    for b in range(B):
        target[b, :m[b]] = draft[b, :m[b]]
        if m[b] < D:
            target[b, m[b]] = draft[b, m[b]] + 1
    acc, em, nn, bt = oracle.accept_chain(draft, target, mask)
    acc0, em0 = oracle.accept(draft, target)
    assert np.array_equal(acc, acc0) and np.array_equal(em, em0) and np.array_equal(acc, m)
    assert np.array_equal(nn, m + 1) and np.all((nn >= 1) & (nn <= Bk))
    for b in range(B):
        assert bt[b, 0] == em[b, m[b]] == target[b, m[b]]
        assert np.all(bt[b, 1:] == mask)
        # after a full match the next block starts from the bonus token (the target's 8th)
        if m[b] == D:
            assert bt[b, 0] == target[b, D]


def _grid_uniforms(N, M):
    """u_acc on the midpoints of N cells of [0,1), u_s on the midpoints of M cells of 2^32."""
    ua = ((np.arange(N) + 0.5) / N).astype(np.float32)
    us = (((np.arange(M) + 0.5) / M) * 2.0 ** 32).astype(np.uint64).astype(np.uint32)
    return np.repeat(ua, M), np.tile(us, N)


@pytest.mark.parametrize("with_q", [False, True])
def test_sampled_accept_is_lossless_on_a_uniform_grid(with_q):
    """The defining property of exact rejection sampling: over uniform u_acc and u_s (an exact
    midpoint grid here), the first emitted token is distributed as the target's p_0, whatever the
    draft distribution q (drafted token d drawn from q) or, by default, a fixed drafted token."""
    V, N, M = 5, 400, 512
    p0 = np.array([0.05, 0.4, 0.25, 0.1, 0.2], np.float32)
    pD = np.array([0.3, 0.1, 0.1, 0.2, 0.3], np.float32)
    q0 = np.array([0.3, 0.1, 0.4, 0.15, 0.05], np.float32)
    ua, us = _grid_uniforms(N, M)
    B = ua.size
    freq = np.zeros(V)
    for d in range(V):
        weight = q0[d] if with_q else (1.0 if d == 2 else 0.0)
        if weight == 0:
            continue
        p = np.broadcast_to(np.stack([p0, pD]), (B, 2, V)).copy()
        q = np.broadcast_to(q0, (B, 1, V)).copy() if with_q else None
        acc, em = oracle.accept_sampled(np.full((B, 1), d, np.int32), p, ua.reshape(B, 1), us, q=q)
        freq += weight * np.bincount(em[:, 0], minlength=V) / B
    assert np.allclose(freq, p0, atol=1.0 / N + 1.0 / M + 1e-6), (freq, p0)


def test_sampled_accept_special_cases():
    V, Bk = 50, 8
    D = Bk - 1
    B = 64
    draft = rng.integers(0, V, (B, D)).astype(np.int32)
    ua = rng.random((B, D)).astype(np.float32)
    us = rng.integers(0, 2 ** 32, B, dtype=np.uint64).astype(np.uint32)
    # the target is certain of every drafted token: all accepted, the bonus from p_D (one-hot 7)
    p = np.zeros((B, Bk, V), np.float32)
    for b in range(B):
        p[b, np.arange(D), draft[b]] = 1.0
    p[:, D, 7] = 1.0
    acc, em = oracle.accept_sampled(draft, p, ua, us)
    assert np.all(acc == D) and np.array_equal(em[:, :D], draft) and np.all(em[:, D] == 7)
    # the target gives the first drafted token probability 0: rejected at 0 whatever u, and the
    # resampled token is never the drafted one; u_acc = 0 accepts exactly the tokens with p > 0
    p = rng.random((B, Bk, V)).astype(np.float32)
    p /= p.sum(-1, keepdims=True)
    p[np.arange(B), 0, draft[:, 0]] = 0.0
    acc, em = oracle.accept_sampled(draft, p, ua, us)
    assert np.all(acc == 0) and np.all(em[:, 0] != draft[:, 0]) and np.all(em[:, 1:] == -1)
    acc0, _ = oracle.accept_sampled(draft, p, np.zeros_like(ua), us)
    assert np.all(acc0 == 0)
    p[np.arange(B), 0, draft[:, 0]] = 1e-30
    acc1, _ = oracle.accept_sampled(draft, p, np.zeros_like(ua), us)
    assert np.all(acc1 >= 1)


def test_sampled_residual_search_matches_searchsorted():
    """The resampled token is the inverse CDF of the fixed-point residual: numpy's searchsorted on
    the running sums of floor(max(0, p - q) * 2^32) gives the same token, u_s = 0 and 2^32 - 1
    included (first and last token of nonzero residual)."""
    V, B = 1000, 200
    p = rng.random((B, 2, V)).astype(np.float32) ** 3
    p /= p.sum(-1, keepdims=True)
    q = rng.random((B, 1, V)).astype(np.float32) ** 3
    q /= q.sum(-1, keepdims=True)
    p[:2, 0, :3] = 0.0  # leading tokens without residual mass: u_s = 0 must skip them
    draft = rng.integers(0, V, (B, 1)).astype(np.int32)
    ua = np.full((B, 1), 0.999999, np.float32)  # rejections (unless p(d) >= q(d))
    us = rng.integers(0, 2 ** 32, B, dtype=np.uint64).astype(np.uint32)
    us[:2] = [0, 2 ** 32 - 1]
    acc, em = oracle.accept_sampled(draft, p, ua, us, q=q)
    for b in range(B):
        if acc[b] == 1:
            continue
        r = np.maximum(np.float32(0), p[b, 0] - q[b, 0])
        fx = np.floor(r.astype(np.float64) * 2.0 ** 32).astype(np.uint64)
        cum = np.cumsum(fx, dtype=np.uint64)
        t = (int(us[b]) * int(cum[-1])) >> 32
        want = int(np.searchsorted(cum, np.uint64(t), side="right"))
        assert em[b, 0] == want, (b, em[b, 0], want)
        if b == 0:
            assert want == int(np.nonzero(fx)[0][0])
        if b == 1:
            assert want == int(np.nonzero(fx)[0][-1])
    # a threshold exactly on a running sum: p = (1/4, 1/4, 1/2), q = (0, 0, 1) leaves the residual
    # (1/4, 1/4, 0), in fixed point (2^30, 2^30, 0), T = 2^31; u_s = 2^31 gives t = 2^30 = the first
    # running sum, and the token is the first whose running sum exceeds t: token 1
    p3 = np.array([[[0.25, 0.25, 0.5], [1 / 3, 1 / 3, 1 / 3]]], np.float32)
    acc, em = oracle.accept_sampled(np.array([[2]], np.int32), p3, np.array([[0.99]], np.float32),
                                    np.array([2 ** 31], np.uint32), q=np.array([[[0.0, 0.0, 1.0]]], np.float32))
    assert acc[0] == 0 and em[0, 0] == 1


# ------------------------------------------------------------------ whole step

def _tiny_step(wl=None, mutate=None, trace=True, state=None):
    wl = wl or inputs.WORKLOADS["tiny"]
    w = inputs.make_weights(wl.dims, wl.seed)
    if mutate:
        mutate(w)
    st = state or inputs.make_state(wl)
    hw = oracle.HostWeights(w)
    kc = [oracle._np(t).copy() for t in st["k_cache"]]
    vc = [oracle._np(t).copy() for t in st["v_cache"]]
    res = oracle.draft_request(wl.dims, hw, st["taps"][0], int(st["n_new"][0]), st["block_tokens"][0], kc, vc,
                               st["page_table"][0], int(st["seq_len"][0]), trace=trace)
    return w, st, kc, vc, res


def test_step_structure_tiny():
    w, st, kc, vc, (err, path, scores, sl, tr) = _tiny_step()
    d = inputs.WORKLOADS["tiny"].dims
    assert err == 0 and sl == int(st["seq_len"][0]) + int(st["n_new"][0])
    for t in range(d.block - 1):
        assert path[t] in tr["cand"][t]
        assert np.all(np.diff(tr["cand_logit"][t]) <= 0)
    assert np.all(np.isfinite(scores))
    # only positions L0..Lb-1 of the cache changed
    L0, Lb = int(st["seq_len"][0]), sl
    k0 = oracle._np(st["k_cache"][0])
    pt = oracle._np(st["page_table"][0])
    for cache, before in ((kc[0], k0), (vc[0], oracle._np(st["v_cache"][0]))):
        changed = np.argwhere(np.any(cache != before, axis=(1, 3)))  # (physical page, slot)
        touched = {int(np.where(pt == p)[0][0]) * 16 + int(s) for p, s in changed}
        assert touched == set(range(L0, Lb))
    # the candidate logits are the LM head applied to the final-normed rows
    hn = tr["final_h"]
    lm = oracle.bf16_to_f64(oracle._np(w["lm_head"])).reshape(d.vocab, d.hidden)
    full = hn @ lm.T
    for t in range(d.block - 1):
        ids, vals = oracle.topk(full[t], d.topk)
        assert np.array_equal(ids, tr["cand"][t]) and np.allclose(vals, tr["cand_logit"][t], atol=1e-9)


def test_step_with_zero_output_projections_keeps_embeddings():
    """W_o = W_d = 0 turns every layer into the identity on the residual stream, so the
    final rows are RMSNorm(embedding) exactly."""
    def mut(w):
        for L in w["layers"]:
            L["wo"] = torch.zeros_like(L["wo"])
            L["wd"] = torch.zeros_like(L["wd"])
    w, st, kc, vc, (err, path, scores, sl, tr) = _tiny_step(mutate=mut)
    d = inputs.WORKLOADS["tiny"].dims
    E = oracle.bf16_to_f64(oracle._np(w["embed"])).reshape(d.vocab, d.hidden)
    bt = oracle._np(st["block_tokens"][0])
    for t in range(1, d.block):
        want = oracle.rmsnorm(E[bt[t]], w["final_norm"], d.rms_eps)
        assert np.allclose(tr["final_h"][t - 1], want, atol=1e-12)


def _bf16_layers_tiny():
    d = dataclasses.replace(inputs.TINY, wfmt=1)
    return dataclasses.replace(inputs.WORKLOADS["tiny"], dims=d)


# (gate a, up b) per MLP channel j: the channel's gate row is a/H, its up row b/H, so on a row of
# ones the gate is a*c and the up value b*c (c = 1/sqrt(1 + eps), the RMSNorm of a constant row)
_MLP_CASES = [(40.0, 0.5), (-40.0, 3.0), (0.0, 5.0), (1.0, 1.0), (1.5, 1.0), (-1.5, 1.0), (2.5, -2.0)]


def test_mlp_branch_gate_goes_through_silu():
    """One layer with W_o = 0 (attention adds nothing), embeddings of ones and ln2 = 1, so the MLP
    sees a constant row; W_d copies channel j of the SwiGLU product back onto hidden unit j.
    Saturated gates fix the roles (SiLU on W_g's output, multiplying W_u's): gate +40 passes the
    up value through (x sigma(x) -> x), gate -40 blocks it, gate 0 gives exactly 0; the pair
    +-1.5 pins silu(x) - silu(-x) = x; gate 1 gives sigma(1) = 1 / (1 + e^-1)."""
    wl = _bf16_layers_tiny()
    d = wl.dims
    H, F = d.hidden, d.ffn

    def mut(w):
        w["embed"].fill_(1.0)
        L = w["layers"][0]
        L["wo"].zero_()
        L["ln2"].fill_(1.0)
        wg = torch.zeros(F, H)
        wu = torch.zeros(F, H)
        wd = torch.zeros(H, F)
        for j, (a, b) in enumerate(_MLP_CASES):
            wg[j] = a / H
            wu[j] = b / H
            wd[j, j] = 1.0
        L["wg"] = wg.to(torch.bfloat16)
        L["wu"] = wu.to(torch.bfloat16)
        L["wd"] = wd.to(torch.bfloat16)
        assert torch.equal(L["wg"].float(), wg) and torch.equal(L["wu"].float(), wu)  # exact in bf16

    w, st, kc, vc, (err, path, scores, sl, tr) = _tiny_step(wl=wl, mutate=mut)
    assert err == 0
    c = 1.0 / np.sqrt(1.0 + d.rms_eps)
    h0, h1 = tr["hidden"][0], tr["hidden"][1]
    assert np.all(h0 == 1.0)
    for t in range(d.block):
        y = h1[t] - 1.0
        assert abs(y[0] - 40 * c * 0.5 * c) <= 1e-9              # open gate: u passes
        assert abs(y[1]) <= 1e-12                                  # closed gate: nothing
        assert y[2] == 0.0                                         # silu(0) = 0
        assert abs(y[3] - 0.7310585786300049) <= 1e-5              # sigma(1), the logistic function
        assert abs((y[4] - y[5]) - 1.5 * c * c) <= 1e-12           # silu(x) - silu(-x) = x
        assert y[6] < 0 and abs(y[6] / (-2.0 * c) - 2.5 * c / (1 + np.exp(-2.5 * c))) <= 1e-12
        assert np.all(y[len(_MLP_CASES):] == 0.0)


def _angle_mod_pi(x0, x1):
    return np.mod(np.arctan2(x1, x0), np.pi)


def _pos_mod_pi(p):
    return np.mod(float(p), np.pi)


def test_qk_norm_precedes_rope_at_absolute_positions():
    """Query head 0 and key head 0 of layer 0 carry one nonzero input dimension (dim 0, the sum
    of the row); q/k-norm weights differ between dim 0 and its RoPE partner dim 64.  Norm first,
    then rotation: the pair (0, 64) has amplitude qn[0] * sqrt(128) and angle = position (mod pi,
    the sign of the sum being unknown) with frequency theta^0 = 1.  Rotation first would give
    amplitudes mixed from qn[0] and qn[64] and a different angle.  Block rows sit at Lb + t
    (queries and block keys); context rows are appended to the cache at L0 + i."""
    wl = _bf16_layers_tiny()
    d = wl.dims

    def mut(w):
        L = w["layers"][0]
        for n in ("wq", "wk"):
            L[n].zero_()
            L[n][0] = 1.0
        L["qn"].fill_(1.0)
        L["qn"][0], L["qn"][64] = 1.5, 0.5
        L["kn"].fill_(1.0)
        L["kn"][0], L["kn"][64] = 0.75, 1.25

    w, st, kc, vc, (err, path, scores, sl, tr) = _tiny_step(wl=wl, mutate=mut)
    assert err == 0
    L0, n = int(st["seq_len"][0]), int(st["n_new"][0])
    Lb = L0 + n
    hd = d.head_dim
    for name, trace, wt in (("q", tr["q0"], 1.5), ("k", tr["k0"], 0.75)):
        for t in range(d.block):
            v = trace[t]
            others = np.ones(v.size, bool)
            others[[0, 64]] = False
            assert np.all(v[others] == 0.0), name
            assert abs(np.hypot(v[0], v[64]) - wt * np.sqrt(hd)) <= 1e-3, (name, t)
            diff = abs(_angle_mod_pi(v[0], v[64]) - _pos_mod_pi(Lb + t))
            assert min(diff, np.pi - diff) <= 1e-9, (name, t)
    # context keys in the cache (bf16): position L0 + i, amplitude kn[0] * sqrt(128)
    pt = oracle._np(st["page_table"][0])
    for i in range(n):
        pos = L0 + i
        row = bits_to_f64(kc[0][pt[pos // 16], 0, pos % 16])
        others = np.ones(hd, bool)
        others[[0, 64]] = False
        assert np.all(row[others] == 0.0)
        assert abs(np.hypot(row[0], row[64]) - 0.75 * np.sqrt(hd)) <= 0.75 * np.sqrt(hd) * 2 ** -7
        diff = abs(_angle_mod_pi(row[0], row[64]) - _pos_mod_pi(pos))
        assert min(diff, np.pi - diff) <= 2 ** -6, i


def test_step_ignores_cache_outside_window():
    wl = inputs.WORKLOADS["tiny"]
    st = inputs.make_state(wl)
    *_, (e1, p1, s1, _, t1) = _tiny_step(state=st)
    st2 = inputs.make_state(wl)
    Lb = int(st2["seq_len"][0]) + int(st2["n_new"][0])
    first = Lb - wl.dims.window + 1
    pt = st2["page_table"][0]
    for j in range(first):
        st2["k_cache"][0][pt[j // 16], :, j % 16] = 3.0
        st2["v_cache"][0][pt[j // 16], :, j % 16] = -2.0
    *_, (e2, p2, s2, _, t2) = _tiny_step(state=st2)
    assert e1 == e2 == 0 and np.array_equal(p1, p2) and np.array_equal(s1, s2)
    # a change inside the window does move the result
    st3 = inputs.make_state(wl)
    st3["v_cache"][0][pt[(Lb - 10) // 16], :, (Lb - 10) % 16] = 50.0
    *_, (e3, p3, s3, _, t3) = _tiny_step(state=st3)
    assert not np.allclose(t3["hidden"][-1], t1["hidden"][-1])


def test_kv_bytes_per_token_matches_page():
    d = inputs.FULL
    per_token = d.layers * d.n_kv * d.head_dim * 2 * 2  # K and V, 16-bit
    assert per_token == GOLD["kv_bytes_per_token_16bit"]["value"]


def test_parameter_count_consistency():
    """Named tensors of the full drafter (with the dynamic-convolution reading) land within
    0.01% of the published 1,924,404,480 parameters (aiqre.com, Specification)."""
    d = inputs.FULL
    H, F, T = d.hidden, d.ffn, d.n_taps
    hq, hkv = d.n_q * d.head_dim, d.n_kv * d.head_dim
    layer = hq * H + 2 * hkv * H + H * hq + 3 * F * H + 2 * H + 2 * d.head_dim + 2 * (H // 4) * H + 2 * H
    total = d.layers * layer + T * H * H + H + H + d.rank * H + 2 * d.vocab * d.rank
    pub = GOLD["parameters"]["value"]
    assert abs(total - pub) / pub < 1e-4
