// Candidate merge, selector transition scores and the Viterbi path, one CTA per
// request (FastFlowLM card: "picks one coherent path through its top 16
// candidates per position"; "Weights" row: selector projection and two
// 248320 x 256 codebooks).
//
// Transition score (the reading fixed for the pages' unnamed formula):
//   tau_t(a -> b) = sum_r A[a][r] * z_t[r] * Bc[b][r],  z_t = W_s h~_t,
// sources at position 0 = the block's first token, at t > 0 the candidates of
// t-1; unary = candidate logit;
//   delta_0(j) = u_0(j) + tau_0(x0 -> c_0j)
//   delta_t(j) = u_t(j) + max_i (delta_{t-1}(i) + tau_t(c_{t-1,i} -> c_tj)),
// smaller candidate index on ties.  fp32 throughout.
#pragma once
#include "common.cuh"

namespace dfl {

constexpr int kMaxD = 15;
constexpr int kMaxR = 256;

struct SelParams {
  const float* cand_val;  // [nparts][rows_total][16], each list sorted
  const int32_t* cand_id;
  int nparts, rows_total;
  const float* z;  // [rows_total][R]
  int R, V, Bk;
  const uint16_t *cb_a, *cb_b;
  const int32_t* block_tokens;
  int32_t* out_path;
  float* out_scores;
  int32_t* seq_len;
  const int32_t* n_new;
  int32_t* dbg_cand;
  float* dbg_logit;
  int* err;
};

// Transition scores and the Viterbi path of request b from its merged candidates (cand, cl in
// shared memory), run by the first NTHR threads (named barrier 1).  As, Wj: shared scratch of
// 16 x 256 floats each.  Writes out_path / out_scores and advances seq_len[b].
template <int NTHR>
DEVI void selector_core(const SelParams& p, int b, int (*cand)[kTopK], float (*cl)[kTopK], float (*As)[kMaxR],
                        float (*Wj)[kTopK]) {
  __shared__ float tau[kTopK][kTopK];
  __shared__ float delta[kMaxD][kTopK];
  __shared__ int bp[kMaxD][kTopK];
  __shared__ int src_ids[kTopK];
  const int D = p.Bk - 1, R = p.R;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 2. per position: transition scores tau_t, then one Viterbi step in warp 0
  //    (lane j of warp 0 holds delta_t(j))
  float d = 0.f;
  for (int t = 0; t < D; ++t) {
    const int nsrc = t == 0 ? 1 : kTopK;
    if (threadIdx.x < kTopK) {
      int a = t == 0 ? p.block_tokens[b * p.Bk] : cand[t - 1][threadIdx.x];
      if (a < 0 || a >= p.V) a = 0;
      src_ids[threadIdx.x] = a;
    }
    consumers_sync<NTHR>();
    const float* zt = p.z + (size_t)(b * D + t) * R;
    const int R8 = R / 8;
    for (int i = threadIdx.x; i < kTopK * R8; i += NTHR) {
      const int j = i / R8, r = (i % R8) * 8;
      const uint4 bv = *reinterpret_cast<const uint4*>(p.cb_b + (size_t)cand[t][j] * R + r);
      const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        Wj[r + 2 * e][j] = __ldcg(zt + r + 2 * e) * bf2f(bw[e] & 0xffff);
        Wj[r + 2 * e + 1][j] = __ldcg(zt + r + 2 * e + 1) * bf2f(bw[e] >> 16);
      }
      if (j < nsrc) {
        const uint4 av = *reinterpret_cast<const uint4*>(p.cb_a + (size_t)src_ids[j] * R + r);
        const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          As[j][r + 2 * e] = bf2f(aw[e] & 0xffff);
          As[j][r + 2 * e + 1] = bf2f(aw[e] >> 16);
        }
      }
    }
    consumers_sync<NTHR>();
    {
      const int i = threadIdx.x / kTopK, j = threadIdx.x % kTopK;
      if (i < nsrc) {
        float s = 0.f;
        for (int r = 0; r < R; ++r) s = fmaf(As[i][r], Wj[r][j], s);
        tau[i][j] = s;
      }
    }
    consumers_sync<NTHR>();
    if (warp == 0) {
      const int j = lane & 15;
      int bi = 0;
      if (t == 0) {
        d = cl[0][j] + tau[0][j];
      } else {
        float best = 0.f;
        bi = -1;
        for (int i = 0; i < kTopK; ++i) {
          const float s = __shfl_sync(0xffffffffu, d, i) + tau[i][j];
          if (bi < 0 || s > best) { best = s; bi = i; }
        }
        d = cl[t][j] + best;
      }
      if (lane < kTopK) { delta[t][j] = d; bp[t][j] = bi; }
    }
  }
  consumers_sync<NTHR>();
  if (threadIdx.x == 0) {
    int jj = 0;
    for (int i = 1; i < kTopK; ++i)
      if (delta[D - 1][i] > delta[D - 1][jj]) jj = i;
    for (int t = D - 1; t >= 0; --t) {
      p.out_path[b * D + t] = cand[t][jj];
      p.out_scores[b * D + t] = delta[t][jj];
      jj = bp[t][jj];
    }
    p.seq_len[b] += p.n_new[b];
  }
}

// Final top-16 of one drafted row from `nparts` sorted partial lists ([part][rows_total][16]),
// by one warp.  T0 = max(best 16th entry of a list, 16th best list head) bounds the final 16th
// from below (either way at least 16 entries reach it), so only list prefixes >= T0 are
// gathered (sv/si, `cap` >= 512 entries; usually a few dozen) and an exact selection runs on
// them.  If more than `cap` survive (pathological ties) an exact per-lane insertion merge of
// every list runs instead, in the same buffers.  Lane 0 writes out_v/out_id[0..15].
DEVI void merge_lists_row(const float* cv, const int32_t* ci, int nparts, int rows_total, int row, float* sv, int* si,
                          int cap, int* surv, float* out_v, int* out_id) {
  const int lane = threadIdx.x & 31;
  float T0 = -INFINITY;
  float heads[8];
  int nh = 0;
  for (int part = lane; part < nparts; part += 32) {
    const size_t o = ((size_t)part * rows_total + row) * kTopK;
    T0 = fmaxf(T0, __ldcg(cv + o + kTopK - 1));
    if (nh < 8) heads[nh++] = __ldcg(cv + o);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) T0 = fmaxf(T0, __shfl_xor_sync(0xffffffffu, T0, o));
  if (nparts <= 8 * 32) {
    // 16th largest head: 16 rounds of a warp max, removing one occurrence each time
    float hb = -INFINITY;
    for (int k = 0; k < kTopK; ++k) {
      float lb = -INFINITY;
      int li_ = -1;
      for (int i = 0; i < nh; ++i)
        if (heads[i] > lb) { lb = heads[i]; li_ = i; }
      float m = lb;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const unsigned who = __ballot_sync(0xffffffffu, li_ >= 0 && lb == m);
      if (who && lane == __ffs(who) - 1) heads[li_] = -INFINITY;
      hb = m;
    }
    T0 = fmaxf(T0, hb);
  }
  if (lane == 0) *surv = 0;
  __syncwarp();
  for (int part = lane; part < nparts; part += 32) {
    const size_t o = ((size_t)part * rows_total + row) * kTopK;
    for (int k = 0; k < kTopK; ++k) {
      const float v = __ldcg(cv + o + k);
      if (!(v >= T0)) break;  // lists are sorted
      const int slot = atomicAdd(surv, 1);
      if (slot < cap) {
        sv[slot] = v;
        si[slot] = __ldcg(ci + o + k);
      }
    }
  }
  __syncwarp();
  const int n = *surv;
  if (n <= cap) {
    for (int k = 0; k < kTopK; ++k) {
      float bv = -INFINITY;
      int bid = 0x7fffffff, bslot = -1;
      for (int i = lane; i < n; i += 32)
        if (better(sv[i], si[i], bv, bid)) { bv = sv[i]; bid = si[i]; bslot = i; }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oid = __shfl_xor_sync(0xffffffffu, bid, o);
        const int os = __shfl_xor_sync(0xffffffffu, bslot, o);
        if (better(ov, oid, bv, bid) || (ov == bv && oid == bid && os > bslot)) { bv = ov; bid = oid; bslot = os; }
      }
      if (lane == 0) {
        out_id[k] = bid;
        out_v[k] = bv;
        if (bslot >= 0) { sv[bslot] = -INFINITY; si[bslot] = 0x7fffffff; }
      }
      __syncwarp();
    }
    return;
  }
  // pathological ties: exact per-lane insertion merge of every list, then 16 rounds over lane heads
  float* lv = sv + lane * kTopK;
  int* li = si + lane * kTopK;
  __syncwarp();
  for (int k = 0; k < kTopK; ++k) { lv[k] = -INFINITY; li[k] = 0x7fffffff; }
  for (int part = lane; part < nparts; part += 32) {
    const size_t o = ((size_t)part * rows_total + row) * kTopK;
    for (int k = 0; k < kTopK; ++k) {
      const float v = __ldcg(cv + o + k);
      const int id = __ldcg(ci + o + k);
      if (!better(v, id, lv[kTopK - 1], li[kTopK - 1])) break;
      int pos = kTopK - 1;
      while (pos > 0 && better(v, id, lv[pos - 1], li[pos - 1])) {
        lv[pos] = lv[pos - 1];
        li[pos] = li[pos - 1];
        --pos;
      }
      lv[pos] = v;
      li[pos] = id;
    }
  }
  __syncwarp();
  int head = 0;
  for (int k = 0; k < kTopK; ++k) {
    float bv = head < kTopK ? lv[head] : -INFINITY;
    int bid = head < kTopK ? li[head] : 0x7fffffff;
    int bl = lane;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oid = __shfl_xor_sync(0xffffffffu, bid, o);
      const int ol = __shfl_xor_sync(0xffffffffu, bl, o);
      if (better(ov, oid, bv, bid) || (ov == bv && oid == bid && ol < bl)) { bv = ov; bid = oid; bl = ol; }
    }
    if (lane == 0) {
      out_id[k] = bid;
      out_v[k] = bv;
    }
    if (lane == bl) ++head;
  }
  __syncwarp();
}

__global__ void __launch_bounds__(256) k_selector(SelParams p) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x, D = p.Bk - 1;
  const int warp = threadIdx.x >> 5;
  __shared__ int cand[kMaxD][kTopK];
  __shared__ float cl[kMaxD][kTopK];
  // phase 1: per-lane merge lists [warps][32][16] (values, then ids); phase 2: codebook rows
  __shared__ __align__(16) float big[2 * kTopK * kMaxR];
  float(*As)[kMaxR] = reinterpret_cast<float(*)[kMaxR]>(big);
  float(*Wj)[kTopK] = reinterpret_cast<float(*)[kTopK]>(big + kTopK * kMaxR);  // [r][j]: conflict-free reads

  // 1. merge the CTA lists of each drafted position into the final top-16
  constexpr int kCap = 512;
  __shared__ int surv_n[kWarps];
  for (int t = warp; t < D; t += kWarps) {
    float* sv = big + warp * kCap;
    int* si = reinterpret_cast<int*>(big + kWarps * kCap) + warp * kCap;
    merge_lists_row(p.cand_val, p.cand_id, p.nparts, p.rows_total, b * D + t, sv, si, kCap, &surv_n[warp], cl[t],
                    cand[t]);
  }
  __syncthreads();
  if (threadIdx.x < D * kTopK) {
    const int t = threadIdx.x / kTopK, k = threadIdx.x % kTopK;
    const float v = cl[t][k];
    int id = cand[t][k];
    if (!isfinite(v)) set_err(p.err, DFLASH2_DEV_NONFINITE);
    if (id < 0 || id >= p.V) {
      set_err(p.err, DFLASH2_DEV_NONFINITE);
      cand[t][k] = 0;
    }
  }
  __syncthreads();

  selector_core<256>(p, b, cand, cl, As, Wj);
  if (p.dbg_cand && threadIdx.x < D * kTopK) {
    const int t = threadIdx.x / kTopK, k = threadIdx.x % kTopK;
    p.dbg_cand[(b * D + t) * kTopK + k] = cand[t][k];
    p.dbg_logit[(b * D + t) * kTopK + k] = cl[t][k];
  }
}

}  // namespace dfl
