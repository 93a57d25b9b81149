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
#include <climits>

#include "common.cuh"

namespace dfl {

// Integer keys that order like the floats (no NaN): a warp max/min of floats in one redux.
DEVI int order_key(float f) {
  const int k = __float_as_int(f);
  return k >= 0 ? k : k ^ 0x7fffffff;
}
DEVI float key_float(int k) { return __int_as_float(k >= 0 ? k : k ^ 0x7fffffff); }

constexpr int kMaxD = 15;
constexpr int kSelSpreadSmem = 160 * 1024;  // dynamic shared memory reserved per selector CTA (one per SM)
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

// Final top-16 of one drafted row from `nparts` sorted partial lists ([part][rows_total][16]),
// by one warp.  T0 = max(best 16th entry of a list, 16th best list head) bounds the final 16th
// from below (either way at least 16 entries reach it), so only list prefixes >= T0 are
// gathered (sv/si, `cap` >= 512 entries; usually a few dozen) and an exact selection runs on
// them.  If more than `cap` survive (pathological ties) an exact per-lane insertion merge of
// every list runs instead, in the same buffers.  Lane 0 writes out_v/out_id[0..15].
DEVI void merge_lists_row(const float* cv, const int32_t* ci, int nparts, int rows_total, int row, float* sv, int* si,
                          int cap, int* surv, float* out_v, int* out_id) {
  const int lane = threadIdx.x & 31;
  // the lane's first 8 lists (parts lane, lane + 32, ...): their heads stay in registers (fully
  // unrolled, no local memory) and all 16 loads go out together
  float T0 = -INFINITY;
  float heads[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int part = lane + 32 * q;
    heads[q] = -INFINITY;
    if (part < nparts) {
      const size_t o = ((size_t)part * rows_total + row) * kTopK;
      T0 = fmaxf(T0, __ldcg(cv + o + kTopK - 1));
      heads[q] = __ldcg(cv + o);
    }
  }
  for (int part = lane + 256; part < nparts; part += 32)
    T0 = fmaxf(T0, __ldcg(cv + ((size_t)part * rows_total + row) * kTopK + kTopK - 1));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) T0 = fmaxf(T0, __shfl_xor_sync(0xffffffffu, T0, o));
  if (nparts <= 8 * 32) {
    // 16th largest head: 16 rounds of a warp max (one redux on order-preserving integer keys),
    // removing one occurrence each time
    int hk[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) hk[q] = order_key(heads[q]);
    int hb = INT_MIN;
    for (int k = 0; k < kTopK; ++k) {
      int lb = INT_MIN, li_ = -1;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (hk[q] > lb) {
          lb = hk[q];
          li_ = q;
        }
      const int m = __reduce_max_sync(0xffffffffu, lb);
      const unsigned who = __ballot_sync(0xffffffffu, li_ >= 0 && lb == m);
      if (who && lane == __ffs(who) - 1) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q == li_) hk[q] = INT_MIN;
      }
      hb = m;
    }
    if (hb != INT_MIN) T0 = fmaxf(T0, key_float(hb));
  }
  if (lane == 0) *surv = 0;
  __syncwarp();
  // survivors: each sorted list contributes a prefix >= T0.  The lane's lists (at most 8) are read
  // 4 entries at a time, all of them together, so a round costs one L2 round trip; the ids of the
  // survivors are fetched afterwards in one batch (si holds the entry's offset until then).
  {
    unsigned live = 0;  // bit q: the lane's list q may continue
    int nq = 0;
    for (int part = lane; part < nparts && nq < 8; part += 32) live |= 1u << nq++;
    for (int k0 = 0; k0 < kTopK && __any_sync(0xffffffffu, live != 0); k0 += 4) {
      float4 v4[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (live >> q & 1u)
          v4[q] = __ldcg(reinterpret_cast<const float4*>(cv + ((size_t)(lane + 32 * q) * rows_total + row) * kTopK + k0));
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (!(live >> q & 1u)) continue;
        const float e4[4] = {v4[q].x, v4[q].y, v4[q].z, v4[q].w};
        const size_t o = ((size_t)(lane + 32 * q) * rows_total + row) * kTopK + k0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (!(e4[e] >= T0)) {  // lists are sorted: this one is done
            live &= ~(1u << q);
            break;
          }
          const int slot = atomicAdd(surv, 1);
          if (slot < cap) {
            sv[slot] = e4[e];
            si[slot] = (int)(o + e);
          }
        }
      }
    }
    // more than 8 lists per lane (over 256 parts): the rest one entry at a time
    for (int part = lane + 256; part < nparts; part += 32) {
      const size_t o = ((size_t)part * rows_total + row) * kTopK;
      for (int k = 0; k < kTopK; ++k) {
        const float v = __ldcg(cv + o + k);
        if (!(v >= T0)) break;
        const int slot = atomicAdd(surv, 1);
        if (slot < cap) {
          sv[slot] = v;
          si[slot] = (int)(o + k);
        }
      }
    }
    __syncwarp();
    const int ns = min(*surv, cap);
#pragma unroll 4
    for (int i = lane; i < ns; i += 32) si[i] = __ldcg(ci + si[i]);
  }
  __syncwarp();
  const int n = *surv;
  if (n <= 64) {
    // few survivors (the usual case): each one's rank is the number of survivors better than it
    // (ids are distinct, so ranks are), and the 16 best go straight to their places
    if (lane < kTopK) {
      out_v[lane] = -INFINITY;
      out_id[lane] = 0x7fffffff;
    }
    __syncwarp();
    for (int e = lane; e < n; e += 32) {
      const float v = sv[e];
      const int id = si[e];
      int rank = 0;
      for (int i = 0; i < n; ++i) rank += better(sv[i], si[i], v, id) ? 1 : 0;
      if (rank < kTopK) {
        out_v[rank] = v;
        out_id[rank] = id;
      }
    }
    __syncwarp();
    return;
  }
  if (n <= cap) {
    for (int k = 0; k < kTopK; ++k) {
      float bv = -INFINITY;
      int bid = 0x7fffffff, bslot = -1;
      for (int i = lane; i < n; i += 32)
        if (better(sv[i], si[i], bv, bid)) { bv = sv[i]; bid = si[i]; bslot = i; }
      // best value (redux on order-preserving keys), then the smallest id among its holders
      const int mk = __reduce_max_sync(0xffffffffu, order_key(bv));
      const int mid = __reduce_min_sync(0xffffffffu, order_key(bv) == mk ? bid : 0x7fffffff);
      const unsigned who = __ballot_sync(0xffffffffu, order_key(bv) == mk && bid == mid && bslot >= 0);
      if (lane == 0) {
        out_id[k] = mid;
        out_v[k] = key_float(mk);
      }
      if (who && lane == __ffs(who) - 1) {
        sv[bslot] = -INFINITY;
        si[bslot] = 0x7fffffff;
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

// Transition scores of position t of request b, tau[i][j] = sum_r A[src_i][r] z_t[r] B[cand_j][r]
// for sources i < nsrc (t = 0: the block's first token; t > 0: the candidates of t-1), by the
// first NTHR (>= 256) threads (named barrier 1).  As, Wj: shared scratch of 16 x 256 floats each.
template <int NTHR>
DEVI void selector_tau(const SelParams& p, int b, int t, const int* src_ids, int nsrc, const int* cand_t,
                       float (*As)[kMaxR], float (*Wj)[kTopK], float* tau) {
  const int D = p.Bk - 1, R = p.R, R8 = R / 8;
  const float* zt = p.z + (size_t)(b * D + t) * R;
  // every thread issues the loads of all its items (codebook rows are random HBM rows) before
  // converting any of them
  constexpr int kIt = (kTopK * (kMaxR / 8) + NTHR - 1) / NTHR;
  uint4 bv[kIt], av[kIt];
  float4 z0[kIt], z1[kIt];
#pragma unroll
  for (int k = 0; k < kIt; ++k) {
    const int i = threadIdx.x + k * NTHR, j = i / R8, r = (i % R8) * 8;
    if (i < kTopK * R8) {
      bv[k] = *reinterpret_cast<const uint4*>(p.cb_b + (size_t)cand_t[j] * R + r);
      z0[k] = __ldcg(reinterpret_cast<const float4*>(zt + r));
      z1[k] = __ldcg(reinterpret_cast<const float4*>(zt + r + 4));
      if (j < nsrc) av[k] = *reinterpret_cast<const uint4*>(p.cb_a + (size_t)src_ids[j] * R + r);
    }
  }
#pragma unroll
  for (int k = 0; k < kIt; ++k) {
    const int i = threadIdx.x + k * NTHR, j = i / R8, r = (i % R8) * 8;
    if (i >= kTopK * R8) continue;
    const uint32_t bw[4] = {bv[k].x, bv[k].y, bv[k].z, bv[k].w};
    const float zz[8] = {z0[k].x, z0[k].y, z0[k].z, z0[k].w, z1[k].x, z1[k].y, z1[k].z, z1[k].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      Wj[r + 2 * e][j] = zz[2 * e] * bf2f(bw[e] & 0xffff);
      Wj[r + 2 * e + 1][j] = zz[2 * e + 1] * bf2f(bw[e] >> 16);
    }
    if (j < nsrc) {
      const uint32_t aw[4] = {av[k].x, av[k].y, av[k].z, av[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        As[j][r + 2 * e] = bf2f(aw[e] & 0xffff);
        As[j][r + 2 * e + 1] = bf2f(aw[e] >> 16);
      }
    }
  }
  consumers_sync<NTHR>();
  const int i = threadIdx.x / kTopK, j = threadIdx.x % kTopK;
  if (i < nsrc) {
    float s4[4] = {0.f, 0.f, 0.f, 0.f};  // four independent chains, added in a fixed order
    for (int r = 0; r < R; r += 4) {
#pragma unroll
      for (int e = 0; e < 4; ++e) s4[e] = fmaf(As[i][r + e], Wj[r + e][j], s4[e]);
    }
    tau[i * kTopK + j] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
  }
}

// Viterbi over the D positions of request b by one warp (lane j < 16 holds delta_t(j)):
//   delta_0(j) = cl_0(j) + tau_0(0, j),  delta_t(j) = cl_t(j) + max_i (delta_{t-1}(i) + tau_t(i, j)),
// first maximum on ties (smallest i; at the end smallest j).  Writes the path and its running
// scores and advances seq_len[b] by n_new[b].  cl/cand: [D][16], tau: [D][16][16] (global).
// SH: cl/cand/tau are in shared memory (plain loads); otherwise global, written by other CTAs (L2).
template <bool SH = false>
DEVI void selector_viterbi(const SelParams& p, int b, const float* cl, const int32_t* cand, const float* tau) {
  auto ldf = [](const float* a) { return SH ? *a : __ldcg(a); };
  auto ldi = [](const int32_t* a) { return SH ? *a : __ldcg(a); };
  const int lane = threadIdx.x & 31, j = lane & 15, D = p.Bk - 1;
  float d = 0.f;
  float dl[kMaxD];
  int bp[kMaxD];
#pragma unroll
  for (int t = 0; t < kMaxD; ++t) {
    dl[t] = 0.f;
    bp[t] = 0;
    if (t >= D) continue;
    const float* tt = tau + (size_t)t * kTopK * kTopK;
    const float c = ldf(cl + t * kTopK + j);
    if (t == 0) {
      d = c + ldf(tt + j);
    } else {
      // all 16 shuffles and loads go out together; the first maximum wins
      float sc[kTopK];
#pragma unroll
      for (int i = 0; i < kTopK; ++i) sc[i] = __shfl_sync(0xffffffffu, d, i) + ldf(tt + i * kTopK + j);
      float best = sc[0];
      int bi = 0;
#pragma unroll
      for (int i = 1; i < kTopK; ++i)
        if (sc[i] > best) { best = sc[i]; bi = i; }
      d = c + best;
      bp[t] = bi;
    }
    dl[t] = d;
  }
  int jj = 0;
  float bestd = __shfl_sync(0xffffffffu, d, 0);
  for (int i = 1; i < kTopK; ++i) {
    const float v = __shfl_sync(0xffffffffu, d, i);
    if (v > bestd) { bestd = v; jj = i; }
  }
#pragma unroll
  for (int t = kMaxD - 1; t >= 0; --t) {
    if (t >= D) continue;
    const float sc = __shfl_sync(0xffffffffu, dl[t], jj);
    const int prev = __shfl_sync(0xffffffffu, bp[t], jj);
    if (lane == 0) {
      p.out_path[b * D + t] = ldi(cand + t * kTopK + jj);
      p.out_scores[b * D + t] = sc;
    }
    jj = prev;
  }
  if (lane == 0 && p.seq_len) p.seq_len[b] += p.n_new[b];
}

// Final candidates of row (b, t) from the CTA lists into cl/cand (shared), ids outside [0, V)
// (and non-finite logits) flagged and replaced by 0.  One warp; sv/si: >= 512 entries each.
DEVI void selector_row(const SelParams& p, int row, float* sv, int* si, int* surv, float* cl, int* cand) {
  merge_lists_row(p.cand_val, p.cand_id, p.nparts, p.rows_total, row, sv, si, 512, surv, cl, cand);
  __syncwarp();
  const int lane = threadIdx.x & 31;
  if (lane < kTopK) {
    if (!isfinite(cl[lane])) set_err(p.err, DFLASH2_DEV_NONFINITE);
    if (cand[lane] < 0 || cand[lane] >= p.V) {
      set_err(p.err, DFLASH2_DEV_NONFINITE);
      cand[lane] = 0;
    }
  }
  __syncwarp();
}

// One CTA per (position t, request b): final candidates of rows t (and t-1, the sources), then
// tau_t -> tau_g[b][t]; row t's candidates -> cl_g/cand_g (and the debug outputs).  The last of a
// request's D CTAs to finish (arrival ticket per request, acq_rel; rearmed by it) runs the
// request's Viterbi path.
__global__ void __launch_bounds__(256) k_sel_tau(SelParams p, float* tau_g, float* cl_g, int32_t* cand_g,
                                                 int* tickets) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x, b = blockIdx.y, D = p.Bk - 1, warp = threadIdx.x >> 5;
  __shared__ int cand[2][kTopK];
  __shared__ float cl[2][kTopK];
  __shared__ int src[kTopK];
  __shared__ int surv[2];
  __shared__ __align__(16) float big[2 * kTopK * kMaxR];
  float(*As)[kMaxR] = reinterpret_cast<float(*)[kMaxR]>(big);
  float(*Wj)[kTopK] = reinterpret_cast<float(*)[kTopK]>(big + kTopK * kMaxR);  // [r][j]: conflict-free reads
  // warp 0: row t; warp 1: row t - 1 (the sources), each in its own part of `big`
  if (warp == 0 || (warp == 1 && t > 0)) {
    float* sv = big + warp * 1024;
    int* si = reinterpret_cast<int*>(big + warp * 1024 + 512);
    selector_row(p, b * D + t - warp, sv, si, &surv[warp], cl[1 - warp], cand[1 - warp]);
  }
  __syncthreads();
  if (threadIdx.x < kTopK) {
    const size_t o = (size_t)(b * D + t) * kTopK + threadIdx.x;
    cl_g[o] = cl[1][threadIdx.x];
    cand_g[o] = cand[1][threadIdx.x];
    if (p.dbg_cand) {
      p.dbg_cand[o] = cand[1][threadIdx.x];
      p.dbg_logit[o] = cl[1][threadIdx.x];
    }
    if (t == 0) {
      if (threadIdx.x == 0) {
        int a = p.block_tokens[b * p.Bk];
        src[0] = (a < 0 || a >= p.V) ? 0 : a;
      }
    } else {
      src[threadIdx.x] = cand[0][threadIdx.x];
    }
  }
  __syncthreads();
  selector_tau<256>(p, b, t, src, t == 0 ? 1 : kTopK, cand[1], As, Wj, tau_g + (size_t)(b * D + t) * kTopK * kTopK);
  __shared__ int s_last;
  __syncthreads();  // this CTA's tau, cl and cand stores precede its arrival
  if (threadIdx.x == 0) {
    int prev;
    asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], 1;" : "=r"(prev) : "l"(tickets + b) : "memory");
    s_last = prev == D - 1;
    if (s_last) tickets[b] = 0;
  }
  __syncthreads();
  if (!s_last) return;
  // the request's scores and candidates into shared memory in one round trip, then the path
  float* tau_s = big;                                        // [D][16][16]
  float* cl_s = big + kMaxD * kTopK * kTopK;                 // [D][16]
  int* cd_s = reinterpret_cast<int*>(cl_s + kMaxD * kTopK);  // [D][16]
  const float* tb = tau_g + (size_t)b * D * kTopK * kTopK;
  for (int i = threadIdx.x; i < D * kTopK * kTopK / 4; i += blockDim.x)
    reinterpret_cast<float4*>(tau_s)[i] = __ldcg(reinterpret_cast<const float4*>(tb) + i);
  for (int i = threadIdx.x; i < D * kTopK; i += blockDim.x) {
    cl_s[i] = __ldcg(cl_g + (size_t)b * D * kTopK + i);
    cd_s[i] = __ldcg(cand_g + (size_t)b * D * kTopK + i);
  }
  __syncthreads();
  if (warp == 0) selector_viterbi<true>(p, b, cl_s, cd_s, tau_s);
}

// A vocabulary shard's local candidates: the final top-16 of each row from the head CTAs' lists
// (`nparts` sorted lists [part][rows][16]) into out_v/out_id [rows][16], one warp per row; the
// selector that would advance seq_len runs on another rank, so this kernel advances it
// (seq_len[b] += n_new[b]).
__global__ void __launch_bounds__(128) k_merge_rows(const float* __restrict__ cv, const int32_t* __restrict__ ci,
                                                    int nparts, int rows, float* __restrict__ out_v,
                                                    int32_t* __restrict__ out_id, int32_t* __restrict__ seq_len,
                                                    const int32_t* __restrict__ n_new, int B) {
  pdl_trigger();
  pdl_wait();
  __shared__ __align__(16) float sv[4][512];
  __shared__ __align__(16) int si[4][512];
  __shared__ int surv[4];
  const int warp = threadIdx.x >> 5, row = blockIdx.x * 4 + warp;
  if (row < rows)
    merge_lists_row(cv, ci, nparts, rows, row, sv[warp], si[warp], 512, &surv[warp], out_v + (size_t)row * kTopK,
                    out_id + (size_t)row * kTopK);
  if (blockIdx.x == 0 && seq_len)
    for (int b = threadIdx.x; b < B; b += blockDim.x) seq_len[b] += n_new[b];
}

}  // namespace dfl
