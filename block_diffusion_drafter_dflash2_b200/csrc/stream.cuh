// Weight-streaming engine of the block step (all of its matrices are read once
// per step, so the step is bound by HBM bandwidth).
//
// One CTA per SM, warp-specialised: a producer warp streams tile-contiguous
// weight chunks (prepared layouts, below) into a per-warp ring of shared-memory
// slots with 1-D bulk copies on the TMA engine, completion counted on mbarriers;
// 8 consumer warps each own one 16-feature tile at a time and run warp
// mma.sync m16n8k16 with the weights as the M side and the step's few
// activation rows (staged once in shared memory) as the N side.  The producer
// starts before the activations exist (the weights do not depend on the
// previous kernel), so with programmatic dependent launch the weight stream
// overlaps the previous kernel's tail and this kernel's own prologue.
//
// Prepared layouts (made by dflash2_prepare_weights, values unchanged):
//  * Q4_K: per 16-row tile and 256-wide super-block a 2304-byte record: 2048
//    bytes of 4-bit codes in mma A-fragment order, then the 16 canonical 16-byte
//    scale records of the tile's rows (see q4_unit).
//  * bf16: per 16-row tile and 128-wide K step a 4096-byte record: for each
//    32-wide sub-block j, 512 bytes holding lane L = (g, t)'s 8 values
//    W[row g][32j + 8t ..] then 512 bytes for row g + 8.
//
// Work split of the GEMV (stream-K): the (column group, K unit) plane is cut
// into gridDim.x equal contiguous ranges, so every SM streams the same number
// of bytes.  A column group (8 tiles = 128 outputs; 4 gate + 4 up tiles when
// paired) that straddles ranges gets one fp32 partial per range; the last CTA
// to finish a group (arrival ticket, nobody waits) sums the partials in range
// order — deterministic — and runs the epilogue.
#pragma once
#include "gemv.cuh"

namespace dfl {

constexpr int kConsumers = 8;
constexpr int kStreamThreads = (kConsumers + 1) * 32;

template <bool Q4>
struct Ring;
template <>
struct Ring<true> {
  static constexpr int kSlot = kQ4Bytes, kNS = 6, kUnitK = 256;
};
template <>
struct Ring<false> {
  static constexpr int kSlot = 4096, kNS = 4, kUnitK = 128;
};

DEVI void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory"); }
DEVI void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

struct SGemvParams {
  GemvSeg seg[3];
  int nseg;
  int paired;
  const uint16_t* X;  // bf16 activations [rows][ldx]
  int ldx;
  int rows;           // activation rows (max over segments)
  int U;              // K units per tile (Q4: K/256, bf16: K/128)
  int groups, mgroups;
  long long W;        // groups * mgroups * U
  int kc_units;       // units per shared-memory X chunk
  float* part;        // partials [piece][rows][ldo]
  int ldo;
  long long piece_stride;
  int* counters;      // [mgroups * groups]
  int epi;
  float* y;
  int ldy;
  uint16_t* act;
  int F;
  QkvEpi qkv;
  int* err;
};

// Owner CTA of global position x when [0, W) is cut into P ranges [c*W/P, (c+1)*W/P).
DEVI long long sk_owner(long long x, long long W, long long P) { return ((x + 1) * P + W - 1) / W - 1; }

// Tile of consumer warp w in column group grp; -1 when idle.
DEVI int sk_tile(const SGemvParams& p, int grp, int w, int& si) {
  if (p.paired) {
    si = w >> 2;
    const int tile = grp * 4 + (w & 3);
    return tile < p.seg[si].tiles ? tile : -1;
  }
  int gt = grp * kConsumers + w, acc = 0;
  for (int s = 0; s < p.nseg; ++s) {
    if (gt < acc + p.seg[s].tiles) {
      si = s;
      return gt - acc;
    }
    acc += p.seg[s].tiles;
  }
  si = -1;
  return -1;
}

DEVI int sk_rows(const SGemvParams& p, int si, int mz, int R) {
  if (si < 0) return 0;
  int r = p.seg[si].rows - mz;
  return r > R ? R : (r < 0 ? 0 : r);
}

DEVI float sum_pieces(const SGemvParams& p, int npieces, int row, int col) {
  const float* b = p.part + (size_t)row * p.ldo + col;
  float v = 0.f;
  for (int s = 0; s < npieces; ++s) v += __ldcg(b + (size_t)s * p.piece_stride);
  return v;
}

// Epilogue of one column group over rows [mz, mz + R) (consumer threads only).
DEVI void sk_fixup(const SGemvParams& p, int grp, int mz, int R, int npieces) {
  const int tid = threadIdx.x, nthr = kConsumers * 32, warp = tid >> 5, lane = tid & 31;
  if (p.paired) {
    const int f0 = grp * 64;
    const int rows = sk_rows(p, 0, mz, R);
    for (int i = tid; i < rows * 64; i += nthr) {
      const int r = i >> 6, f = f0 + (i & 63);
      if (f >= p.F) continue;
      const float gv = sum_pieces(p, npieces, mz + r, p.seg[0].out_col + f);
      const float uv = sum_pieces(p, npieces, mz + r, p.seg[1].out_col + f);
      p.act[(size_t)(mz + r) * p.F + f] = f2bf(gv / (1.f + __expf(-gv)) * uv);
    }
    return;
  }
  int si = -1;
  const int tile0 = sk_tile(p, grp, 0, si);
  if (tile0 < 0) return;
  int ncol = (p.seg[si].tiles - tile0) * 16;
  ncol = ncol > 128 ? 128 : ncol;
  const int col0 = p.seg[si].out_col + tile0 * 16;
  const int rows = sk_rows(p, si, mz, R);
  if (p.epi == EPI_QKV) {
    const int head = tile0 / 8;
    for (int r = warp; r < rows; r += kConsumers) {
      float x[4];
      const int dims[4] = {2 * lane, 2 * lane + 1, 64 + 2 * lane, 65 + 2 * lane};
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] = sum_pieces(p, npieces, mz + r, col0 + dims[i]);
      qkv_head_row(p.qkv, si, head, mz + r, x, lane);
    }
    return;
  }
  for (int i = tid; i < rows * ncol; i += nthr) {
    const int r = i / ncol, c = col0 + i % ncol;
    const float v = sum_pieces(p, npieces, mz + r, c);
    float* y = p.y + (size_t)(mz + r) * p.ldy + c;
    if (p.epi == EPI_RESID) *y += v;
    else *y = v;
  }
}

template <int NT, bool Q4>
__global__ void __launch_bounds__(kStreamThreads, 1) k_sgemv(SGemvParams p) {
  using RC = Ring<Q4>;
  constexpr int R = NT * 8;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[kConsumers][RC::kNS];
  __shared__ __align__(8) uint64_t empty[kConsumers][RC::kNS];
  __shared__ int s_last;
  uint8_t* ring = smem;
  uint8_t* Xs = smem + kConsumers * RC::kNS * RC::kSlot;
  const int stride = p.kc_units * RC::kUnitK * 2 + 64;
  float* Xsum = reinterpret_cast<float*>(Xs + R * stride);
  float2* coef_all = reinterpret_cast<float2*>(Xsum + (Q4 ? p.kc_units * 8 * R : 0));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;

  if (threadIdx.x == 0) {
    for (int w = 0; w < kConsumers; ++w)
      for (int s = 0; s < RC::kNS; ++s) {
        mbar_init(&full[w][s], 1);
        mbar_init(&empty[w][s], 1);
      }
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger();
  const long long P = gridDim.x, c = blockIdx.x;
  const long long x0 = c * p.W / P, x1 = (c + 1) * p.W / P;

  if (warp == kConsumers) {
    // ---- producer: weights only, so it may run ahead of the previous kernel ----
    if (lane != 0) return;
    int cnt[kConsumers];
    for (int w = 0; w < kConsumers; ++w) cnt[w] = 0;
    for (long long x = x0; x < x1;) {
      const int gidx = (int)(x / p.U), ua = (int)(x % p.U);
      const int ub = (int)((x1 - x) < (long long)(p.U - ua) ? ua + (x1 - x) : p.U);
      const int grp = gidx % p.groups, mz = (gidx / p.groups) * 64;
      const uint8_t* src[kConsumers];
      for (int w = 0; w < kConsumers; ++w) {
        int si;
        const int tile = sk_tile(p, grp, w, si);
        src[w] = (tile >= 0 && sk_rows(p, si, mz, R) > 0)
                     ? p.seg[si].W + ((size_t)tile * p.U) * RC::kSlot
                     : nullptr;
      }
      for (int u = ua; u < ub; ++u)
        for (int w = 0; w < kConsumers; ++w) {
          if (!src[w]) continue;
          const int slot = cnt[w] % RC::kNS, round = cnt[w] / RC::kNS;
          if (round > 0 && !mbar_wait_bounded(&empty[w][slot], (round - 1) & 1)) {
            set_err(p.err, DFLASH2_DEV_TIMEOUT);
            return;
          }
          mbar_expect_tx(&full[w][slot], RC::kSlot);
          bulk_g2s(ring + (w * RC::kNS + slot) * RC::kSlot, src[w] + (size_t)u * RC::kSlot, RC::kSlot, &full[w][slot]);
          ++cnt[w];
        }
      x += ub - ua;
    }
    return;
  }

  // ---- consumers ----
  pdl_wait();  // activations and the partial/ticket buffers come from earlier kernels
  float2* coef = coef_all + warp * 128;
  int cnt = 0;
  bool dead = false;
  for (long long x = x0; x < x1;) {
    const int gidx = (int)(x / p.U), ua = (int)(x % p.U);
    const int ub = (int)((x1 - x) < (long long)(p.U - ua) ? ua + (x1 - x) : p.U);
    const int grp = gidx % p.groups, mz = (gidx / p.groups) * 64;
    int si;
    const int tile = sk_tile(p, grp, warp, si);
    const int my_rows = tile >= 0 ? sk_rows(p, si, mz, R) : 0;
    const int ntact = (my_rows + 7) >> 3;
    int stage_rows = p.rows - mz;
    stage_rows = stage_rows > R ? R : stage_rows;
    float acc[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    for (int c0 = ua; c0 < ub; c0 += p.kc_units) {
      const int cu = (ub - c0) < p.kc_units ? (ub - c0) : p.kc_units;
      // stage X[mz.., c0*unitK ..] and, for Q4_K, the 32-wide sums
      consumers_sync();
      const int vec_per_row = cu * RC::kUnitK / 8;
      const uint16_t* X = p.X + (size_t)mz * p.ldx + (size_t)c0 * RC::kUnitK;
      for (int i = threadIdx.x; i < R * vec_per_row; i += kConsumers * 32) {
        const int r = i / vec_per_row, v = i % vec_per_row;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (r < stage_rows) val = *reinterpret_cast<const uint4*>(X + (size_t)r * p.ldx + v * 8);
        *reinterpret_cast<uint4*>(Xs + r * stride + v * 16) = val;
      }
      consumers_sync();
      if (Q4) {
        for (int i = threadIdx.x; i < R * cu * 8; i += kConsumers * 32) {
          const int r = i % R, j = i / R;
          const uint16_t* row = reinterpret_cast<const uint16_t*>(Xs + r * stride) + j * 32;
          float s = 0.f;
#pragma unroll 8
          for (int k = 0; k < 32; ++k) s += bf2f(row[k]);
          Xsum[j * R + r] = s;
        }
        consumers_sync();
      }
      if (ntact == 0) continue;
      for (int u = c0; u < c0 + cu; ++u) {
        const int slot = cnt % RC::kNS;
        // a consumer never leaves early (the named barriers count on it): after an expired
        // wait it flags the error and skips its remaining work
        if (!dead && !mbar_wait_bounded(&full[warp][slot], (cnt / RC::kNS) & 1)) {
          set_err(p.err, DFLASH2_DEV_TIMEOUT);
          dead = true;
        }
        ++cnt;
        if (dead) continue;
        const uint8_t* sb = ring + (warp * RC::kNS + slot) * RC::kSlot;
        if (Q4) {
          uint4 q[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) q[i] = *reinterpret_cast<const uint4*>(sb + (i * 32 + lane) * 16);
          const uint4 sc = *reinterpret_cast<const uint4*>(sb + 2048 + (lane >> 1) * 16);
          q4_unit<NT>(q, sc, coef, Xs, stride, Xsum + (u - c0) * 8 * R, (u - c0) * 512, ntact, acc, lane);
        } else {
          uint4 wv[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            wv[2 * j] = *reinterpret_cast<const uint4*>(sb + j * 1024 + lane * 16);
            wv[2 * j + 1] = *reinterpret_cast<const uint4*>(sb + j * 1024 + 512 + lane * 16);
          }
          bf16_step<NT>(wv, Xs, stride, (u - c0) * 256, ntact, acc, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[warp][slot]);
      }
    }
    // partial of this piece
    const long long gstart = (long long)gidx * p.U;
    const long long first = sk_owner(gstart, p.W, P);
    const int piece = (int)(c - first);
    const int npieces = (int)(sk_owner(gstart + p.U - 1, p.W, P) - first + 1);
    if (ntact > 0) {
      float* out = p.part + (size_t)piece * p.piece_stride + (size_t)mz * p.ldo;
      const int out_col = p.seg[si].out_col + tile * 16;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (nt < ntact) {
          const int r0 = nt * 8 + 2 * t;
          if (r0 < my_rows) {
            out[(size_t)r0 * p.ldo + out_col + g] = acc[nt][0];
            out[(size_t)r0 * p.ldo + out_col + g + 8] = acc[nt][2];
          }
          if (r0 + 1 < my_rows) {
            out[(size_t)(r0 + 1) * p.ldo + out_col + g] = acc[nt][1];
            out[(size_t)(r0 + 1) * p.ldo + out_col + g + 8] = acc[nt][3];
          }
        }
      }
    }
    __threadfence();
    consumers_sync();
    if (threadIdx.x == 0) {
      const int prev = atomicAdd(p.counters + gidx, 1);
      s_last = prev == npieces - 1;
      if (s_last) p.counters[gidx] = 0;
    }
    consumers_sync();
    if (s_last) {
      __threadfence();
      sk_fixup(p, grp, mz, R, npieces);
    }
    x += ub - ua;
  }
}

// ---------------------------------------------------------------------------
// Shared output head + streaming top-16 (<= 8 drafted rows), same engine: the
// prepared [V + R rows] bf16 matrix (output head, then the selector projection)
// is cut into 8-tile sets handed round-robin to the persistent CTAs.
struct SLmParams {
  const uint8_t* W;  // prepared bf16 tiles of [lm_head; sel_proj]
  int V, R, H;
  const uint16_t* X;  // final-normed rows [rows][H]
  int rows;
  float* z;           // [rows][R]
  float* cand_val;    // [gridDim.x][rows][16]
  int32_t* cand_id;
  int* err;
};

__global__ void __launch_bounds__(kStreamThreads, 1) k_slmhead(SLmParams p) {
  using RC = Ring<false>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[kConsumers][RC::kNS];
  __shared__ __align__(8) uint64_t empty[kConsumers][RC::kNS];
  const int H = p.H, stride = H * 2 + 64;
  uint8_t* ring = smem;
  uint8_t* Xs = smem + kConsumers * RC::kNS * RC::kSlot;
  float* lv_all = reinterpret_cast<float*>(Xs + 8 * stride);          // [warps][8][16]
  int* li_all = reinterpret_cast<int*>(lv_all + kConsumers * 8 * kTopK);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int vt = p.V / 16, total = vt + p.R / 16, S = H / 128;
  const int nsets = (total + kConsumers - 1) / kConsumers;

  if (threadIdx.x == 0) {
    for (int w = 0; w < kConsumers; ++w)
      for (int s = 0; s < RC::kNS; ++s) {
        mbar_init(&full[w][s], 1);
        mbar_init(&empty[w][s], 1);
      }
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger();

  if (warp == kConsumers) {
    if (lane != 0) return;
    int cnt[kConsumers];
    for (int w = 0; w < kConsumers; ++w) cnt[w] = 0;
    for (int set = blockIdx.x; set < nsets; set += gridDim.x)
      for (int s = 0; s < S; ++s)
        for (int w = 0; w < kConsumers; ++w) {
          const int tile = set * kConsumers + w;
          if (tile >= total) continue;
          const int slot = cnt[w] % RC::kNS, round = cnt[w] / RC::kNS;
          if (round > 0 && !mbar_wait_bounded(&empty[w][slot], (round - 1) & 1)) {
            set_err(p.err, DFLASH2_DEV_TIMEOUT);
            return;
          }
          mbar_expect_tx(&full[w][slot], RC::kSlot);
          bulk_g2s(ring + (w * RC::kNS + slot) * RC::kSlot, p.W + ((size_t)tile * S + s) * RC::kSlot, RC::kSlot,
                   &full[w][slot]);
          ++cnt[w];
        }
    return;
  }

  for (int i = threadIdx.x; i < kConsumers * 8 * kTopK; i += kConsumers * 32) {
    lv_all[i] = -INFINITY;
    li_all[i] = 0x7fffffff;
  }
  pdl_wait();
  for (int i = threadIdx.x; i < 8 * (H / 8); i += kConsumers * 32) {
    const int r = i / (H / 8), v = i % (H / 8);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < p.rows) val = *reinterpret_cast<const uint4*>(p.X + (size_t)r * H + v * 8);
    *reinterpret_cast<uint4*>(Xs + r * stride + v * 16) = val;
  }
  consumers_sync();
  float* lv = lv_all + warp * 8 * kTopK;
  int* li = li_all + warp * 8 * kTopK;
  int cnt = 0;
  bool ok = true;
  for (int set = blockIdx.x; set < nsets && ok; set += gridDim.x) {
    const int tile = set * kConsumers + warp;
    if (tile >= total) continue;
    float acc[1][4] = {{0.f, 0.f, 0.f, 0.f}};
    for (int s = 0; s < S; ++s) {
      const int slot = cnt % RC::kNS;
      if (!mbar_wait_bounded(&full[warp][slot], (cnt / RC::kNS) & 1)) {
        set_err(p.err, DFLASH2_DEV_TIMEOUT);
        ok = false;
        break;
      }
      const uint8_t* sb = ring + (warp * RC::kNS + slot) * RC::kSlot;
      uint4 wv[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        wv[2 * j] = *reinterpret_cast<const uint4*>(sb + j * 1024 + lane * 16);
        wv[2 * j + 1] = *reinterpret_cast<const uint4*>(sb + j * 1024 + 512 + lane * 16);
      }
      bf16_step<1>(wv, Xs, stride, s * 256, 1, acc, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[warp][slot]);
      ++cnt;
    }
    if (!ok) break;
    if (tile >= vt) {
      const int c0 = (tile - vt) * 16;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = 2 * t + (e & 1);
        if (r < p.rows) p.z[(size_t)r * p.R + c0 + g + 8 * (e >> 1)] = acc[0][e];
      }
    } else {
      const int id0 = tile * 16;
      bool want = false;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = 2 * t + (e & 1);
        if (r < p.rows && better(acc[0][e], id0 + g + 8 * (e >> 1), lv[r * kTopK + kTopK - 1], li[r * kTopK + kTopK - 1]))
          want = true;
      }
      unsigned m = __ballot_sync(0xffffffffu, want);
      while (m) {
        const int l = __ffs(m) - 1;
        if (lane == l) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int r = 2 * t + (e & 1);
            if (r < p.rows) topk_insert(lv + r * kTopK, li + r * kTopK, acc[0][e], id0 + g + 8 * (e >> 1));
          }
        }
        __syncwarp();
        m &= m - 1;
      }
    }
  }
  consumers_sync();
  // merge the 8 warp lists of each row
  for (int r = warp; r < p.rows; r += kConsumers) {
    float v[4];
    int id[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int src = ((lane >> 2) * 8 + r) * kTopK + (lane & 3) * 4 + i;
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
        if (better(ov, oid, bv, bid) || (ov == bv && oid == bid && ol < bl)) { bv = ov; bid = oid; bl = ol; }
      }
      if (lane == 0) {
        const size_t o = ((size_t)blockIdx.x * p.rows + r) * kTopK + k;
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

// Canonical bf16 [N][K] -> prepared tiles [N/16][K/128][4096 B].
__global__ void k_bf16_prepare(const uint16_t* __restrict__ src, uint8_t* __restrict__ dst, int N, int K) {
  const int S = K / 128, s = blockIdx.x, T = blockIdx.y, lane = threadIdx.x, g = lane >> 2, t = lane & 3;
  uint8_t* out = dst + ((size_t)T * S + s) * 4096;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const size_t k = (size_t)s * 128 + j * 32 + t * 8;
    *reinterpret_cast<uint4*>(out + j * 1024 + lane * 16) =
        *reinterpret_cast<const uint4*>(src + (size_t)(T * 16 + g) * K + k);
    *reinterpret_cast<uint4*>(out + j * 1024 + 512 + lane * 16) =
        *reinterpret_cast<const uint4*>(src + (size_t)(T * 16 + g + 8) * K + k);
  }
}

}  // namespace dfl
