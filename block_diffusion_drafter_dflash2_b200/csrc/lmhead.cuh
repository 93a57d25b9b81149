// Shared output head + streaming top-16 (FastFlowLM card: the output projection
// over the 248320-token vocabulary, 16 candidates kept per drafted position),
// with the selector projection z = W_s h~ riding along as extra tiles.
//
// This kernel serves more than 8 drafted rows (16 per pass); up to 8 rows use
// the TMA-ring engine k_slmhead.  Persistent CTAs of 8 warps.  The final-normed
// rows (bf16) sit in shared memory; each warp streams prepared 16-row vocabulary
// tiles (16-byte streaming loads, two 128-wide K steps in flight) through
// mma.sync m16n8k16 with the vocabulary as the M side.  Logits never leave the
// SM: after each tile every lane offers its values to a per-warp, per-row
// sorted top-16 list in shared memory (threshold test first; insertions
// serialised over the warp by ballot).  At the end the CTA merges its 8 warp
// lists into one sorted list per row; the selector kernel merges the CTAs'.
// Order: larger logit first, smaller token id on ties.
#pragma once
#include "common.cuh"

namespace dfl {

struct LmParams {
  const uint8_t* W;        // prepared bf16 tiles of [lm_head; sel_proj]
  int V, R, H;
  const uint16_t* X;       // final-normed rows of this pass [rows][H]
  int rows;                // rows in this pass (<= 8*NT)
  int row_base;            // absolute index of the pass's first row
  int rows_total;
  float* z;                // [rows_total][R]
  float* cand_val;         // [gridDim.x][rows_total][16]
  int32_t* cand_id;
};

DEVI void topk_insert(float* lv, int* li, float v, int id) {
  if (!better(v, id, lv[kTopK - 1], li[kTopK - 1])) return;
  int pos = kTopK - 1;
  while (pos > 0 && better(v, id, lv[pos - 1], li[pos - 1])) {
    lv[pos] = lv[pos - 1];
    li[pos] = li[pos - 1];
    --pos;
  }
  lv[pos] = v;
  li[pos] = id;
}

template <int NT>
__global__ void __launch_bounds__(kWarps * 32) k_lmhead_topk(LmParams p) {
  constexpr int R8 = NT * 8;
  extern __shared__ __align__(128) uint8_t smem[];
  const int H = p.H, stride = H * 2 + 64;
  uint8_t* Xs = smem;
  float* lv_all = reinterpret_cast<float*>(smem + R8 * stride);       // [warps][R8][16]
  int* li_all = reinterpret_cast<int*>(lv_all + kWarps * R8 * kTopK);  // [warps][R8][16]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;

  for (int i = threadIdx.x; i < R8 * (H / 8); i += blockDim.x) {
    const int r = i / (H / 8), v = i % (H / 8);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < p.rows) val = *reinterpret_cast<const uint4*>(p.X + (size_t)r * H + v * 8);
    *reinterpret_cast<uint4*>(Xs + r * stride + v * 16) = val;
  }
  for (int i = threadIdx.x; i < kWarps * R8 * kTopK; i += blockDim.x) {
    lv_all[i] = -INFINITY;
    li_all[i] = 0x7fffffff;
  }
  __syncthreads();
  float* lv = lv_all + warp * R8 * kTopK;
  int* li = li_all + warp * R8 * kTopK;

  const int vt = p.V / 16, total = vt + p.R / 16;
  const int wg = blockIdx.x * kWarps + warp, nw = gridDim.x * kWarps;
  const int ntiles = wg < total ? (total - wg + nw - 1) / nw : 0;
  const int spt = H / 64;  // 64-wide K steps per tile
  const int nit = ntiles * spt;
  const int ntact = (p.rows + 7) >> 3;

  // prepared bf16 [lm_head; sel_proj]: 2048 bytes per (tile, 64-wide step), 16 tiles per record
  auto load = [&](uint4 (&w)[4], int it) {
    const int tile = wg + (it / spt) * nw;
    const uint8_t* b =
        p.W + (((size_t)(tile / kHeadTiles) * spt + it % spt) * kHeadTiles + tile % kHeadTiles) * 2048 + lane * 16;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      w[2 * j] = ldg_stream(b + j * 1024);
      w[2 * j + 1] = ldg_stream(b + j * 1024 + 512);
    }
  };
  float acc[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

  auto finish_tile = [&](int it) {
    const int tile = wg + (it / spt) * nw;
    if (tile >= vt) {
      const int c0 = (tile - vt) * 16;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = nt * 8 + 2 * t + (e & 1);
          if (nt < ntact && r < p.rows) p.z[(size_t)(p.row_base + r) * p.R + c0 + g + 8 * (e >> 1)] = acc[nt][e];
        }
    } else {
      const int id0 = tile * 16;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (nt >= ntact) continue;
        bool want = false;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = nt * 8 + 2 * t + (e & 1);
          if (r < p.rows && better(acc[nt][e], id0 + g + 8 * (e >> 1), lv[r * kTopK + kTopK - 1], li[r * kTopK + kTopK - 1]))
            want = true;
        }
        unsigned m = __ballot_sync(0xffffffffu, want);
        while (m) {
          const int l = __ffs(m) - 1;
          if (lane == l) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int r = nt * 8 + 2 * t + (e & 1);
              if (r < p.rows) topk_insert(lv + r * kTopK, li + r * kTopK, acc[nt][e], id0 + g + 8 * (e >> 1));
            }
          }
          __syncwarp();
          m &= m - 1;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  };

  if (nit > 0) {
    uint4 wa[4], wb[4];
    load(wa, 0);
    if (1 < nit) load(wb, 1);
    for (int it = 0; it < nit; it += 2) {
      {
        const int kbyte = (it % spt) * 128;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint4 u = wa[2 * j], v = wa[2 * j + 1];
          const uint32_t a0[4] = {u.x, v.x, u.y, v.y}, a1[4] = {u.z, v.z, u.w, v.w};
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            if (nt < ntact) {
              const uint4 bx = *reinterpret_cast<const uint4*>(Xs + (nt * 8 + g) * stride + kbyte + j * 64 + t * 16);
              mma16816(acc[nt], a0, bx.x, bx.y);
              mma16816(acc[nt], a1, bx.z, bx.w);
            }
          }
        }
        if (it + 2 < nit) load(wa, it + 2);
        if ((it % spt) == spt - 1) finish_tile(it);
      }
      if (it + 1 < nit) {
        const int kbyte = ((it + 1) % spt) * 128;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint4 u = wb[2 * j], v = wb[2 * j + 1];
          const uint32_t a0[4] = {u.x, v.x, u.y, v.y}, a1[4] = {u.z, v.z, u.w, v.w};
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            if (nt < ntact) {
              const uint4 bx = *reinterpret_cast<const uint4*>(Xs + (nt * 8 + g) * stride + kbyte + j * 64 + t * 16);
              mma16816(acc[nt], a0, bx.x, bx.y);
              mma16816(acc[nt], a1, bx.z, bx.w);
            }
          }
        }
        if (it + 3 < nit) load(wb, it + 3);
        if (((it + 1) % spt) == spt - 1) finish_tile(it + 1);
      }
    }
  }
  __syncthreads();
  // merge the 8 warp lists of each row: lane holds 4 entries (warp lane/4, entries 4*(lane%4)..+3)
  for (int r = warp; r < p.rows; r += kWarps) {
    float v[4];
    int id[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int src = ((lane >> 2) * R8 + r) * kTopK + (lane & 3) * 4 + i;
      v[i] = lv_all[src];
      id[i] = li_all[src];
    }
    for (int k = 0; k < kTopK; ++k) {
      int bi = 0;
#pragma unroll
      for (int i = 1; i < 4; ++i)
        if (better(v[i], id[i], v[bi], id[bi])) bi = i;
      float bv = v[0];
      int bid = id[0];
#pragma unroll
      for (int i = 1; i < 4; ++i)
        if (i == bi) { bv = v[i]; bid = id[i]; }
      int bl = lane;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oid = __shfl_xor_sync(0xffffffffu, bid, o);
        const int ol = __shfl_xor_sync(0xffffffffu, bl, o);
        if (better(ov, oid, bv, bid) || (ov == bv && oid == bid && ol < bl)) {
          bv = ov;
          bid = oid;
          bl = ol;
        }
      }
      if (lane == 0) {
        const size_t o = ((size_t)blockIdx.x * p.rows_total + p.row_base + r) * kTopK + k;
        p.cand_val[o] = bv;
        p.cand_id[o] = bid;
      }
      if (lane == bl) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (i == bi) { v[i] = -INFINITY; id[i] = 0x7fffffff; }
      }
    }
  }
}

}  // namespace dfl
