// Weight-streaming engine of the block step (all of its matrices are read once
// per step, so the step is bound by HBM bandwidth).
//
// One CTA per SM, warp-specialised: one producer thread streams weight
// records into a ring of shared-memory slots with 1-D bulk copies on the TMA
// engine (completion counted on mbarriers); 8 consumer warps each own one
// 16-feature tile of the current 8-tile column group and run warp mma.sync
// m16n8k16 with the weights as the M side and the step's few activation rows
// (brought into shared memory by bulk copies as well) as the N side.  The
// producer starts before the activations exist (the weights do not depend on
// the previous kernel), so with programmatic dependent launch the weight
// stream overlaps the previous kernel's tail and this kernel's prologue.
//
// Prepared layouts (made by dflash2_prepare_weights, values unchanged): the
// 8 tiles of a column group are interleaved per K unit, so one bulk copy moves
// a whole group's unit (18 KB of Q4_K, 16 KB of bf16):
//  * Q4_K: per tile and 256-wide super-block a 2304-byte record: 2048 bytes of
//    4-bit codes in mma A-fragment order, then the 16 canonical 16-byte scale
//    records of the tile's rows (see q4_unit).
//  * bf16: per tile and 64-wide K step a 2048-byte record: for each 32-wide
//    sub-block j, 512 bytes holding lane L = (g, t)'s 8 values W[row g][32j + 8t ..]
//    then 512 bytes for row g + 8.
//  * gate/up of the MLP are interleaved 4 + 4 tiles per group, so one CTA holds
//    both halves of the SwiGLU for 64 features.
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

constexpr int kConsumers = 8;                          // consumer warps of the LM-head kernel = tiles per group
constexpr int kGemvSets = 2;                           // GEMV: two warp sets alternate ring slots
constexpr int kGemvConsumers = kGemvSets * kConsumers;
constexpr int kGemvThreads = (kGemvConsumers + 1) * 32;
constexpr int kSGemvThreads = (kGemvConsumers + 2) * 32;  // streamed GEMV: + a watcher warp

template <bool Q4>
struct Ring;
template <>
struct Ring<true> {
  static constexpr int kUnitBytes = kQ4Bytes, kSlot = 8 * kQ4Bytes, kNS = 6, kUnitK = 256;
};
template <>
struct Ring<false> {
  static constexpr int kUnitBytes = 2048, kSlot = 8 * 2048, kNS = 8, kUnitK = 64;
};

DEVI void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Hand a ring slot back to the producer: dep folds one word of every load this lane made from
// the slot, and the warp vote on it cannot complete until all lanes' loads have landed in
// registers; the arrive consumes the vote, so it is issued only then.  The consumers call it
// after the math on the slot's bytes: releasing between the loads and the math measured no
// faster and, at 64 activation rows, let results go wrong.
DEVI void slot_release(uint64_t* bar, uint32_t dep, int lane) {
  const unsigned v = __ballot_sync(0xffffffffu, dep == 0x9e3779b9u);
  if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)), "r"(v) : "memory");
}

struct SGemvParams {
  GemvSeg seg[3];     // output column ranges; weights of a paired launch live in seg[0].W
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
  float* ssp;         // EPI_RESID: per-row sums of squares of the new rows, or null
  int ssp_rows;       // row stride of ssp: [column group][quarter][ssp_rows]
  // RMSNorm folded into the products.  EPI_RESID with hw: also hw = bf16(h_new * hw_w) (the next
  // norm's weight applied, its row scale not); the consumer of hw (EPI_STORE / EPI_SWIGLU with
  // rs_in) multiplies its outputs by the row scale rs = 1/sqrt(mean(h^2) + eps) from rs_in, the
  // quarter-column sums of squares the residual epilogue left.
  uint16_t* hw;
  const uint16_t* hw_w;
  int hw_ld;
  const float* rs_in;
  int rs_H;
  float eps;
  // EPI_DYNCONV (paired gate generators a0 | a1 of the two-tap convolution): y_t = (s0 + tanh a0)
  // x_t + (s1 + tanh a1) x_{t-1} with x = RMSNorm(h; dyn_w) formed from the residual rows dyn_h
  const float* dyn_h;
  const uint16_t *dyn_w, *dyn_s0, *dyn_s1;
  uint16_t* dyn_y;  // bf16 [rows][rs_H]
  int Bk;
  int* err;
  // tensor-core path: the row scales of rs_in, computed once per product by its kernel, [rows]
  float* rs_glob;
  int mlx;  // 4-bit records carry MLX group-64 (scale, bias) pairs instead of Q4_K scale records
  int un;   // tensor-core path: activation rows per tile (the MMA's N and the TMA box height)
  int upair;  // and 1 when a tile is two 256-row halves sharing each weight stage
};

// Row scales of rows [mz, mz + rows) from quarter-column sums of squares (ssp layout
// [H/128][4][ldr]) into s_rs[0 .. rows); warp r handles row r.  Consumer threads (barrier 1).
DEVI void rows_scale(const float* ssp, int ldr, int H, float eps, int mz, int rows, float* s_rs) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nq = (H >> 7) * 4;
  for (int r = warp; r < rows; r += kGemvConsumers) {
    float q = 0.f;
    for (int i = lane; i < nq; i += 32) q += __ldcg(ssp + (size_t)i * ldr + mz + r);
    q = warp_sum(q);
    if (lane == 0) s_rs[r] = rsqrtf(q / H + eps);
  }
  consumers_sync<kGemvConsumers * 32>();
}

// Arrival ticket of a split-K group, taken by thread 0 right after a CTA barrier: the acq_rel
// atomic releases the CTA's partial stores (ordered before it by the barrier) and acquires the
// earlier arrivals', so the last arrival can read every partial after its next barrier.
DEVI int ticket_acq_rel(int* ctr) {
  int prev;
  asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], 1;" : "=r"(prev) : "l"(ctr) : "memory");
  return prev;
}

// Arrival of a non-designated split-K piece: a release reduction, after a CTA barrier that orders
// the CTA's partial stores before it; nobody waits for it to complete.
DEVI void arrive_release(int* ctr) {
  asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(ctr) : "memory");
}
// Wait (bounded) until the other `others` pieces of a split-K group have arrived, with acquire
// loads; false when the limit expired.
DEVI bool await_pieces(const int* ctr, int others) {
  for (long long i = 0; i < (kWaitLimit >> 4); ++i) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= others) return true;
    __nanosleep(128);
  }
  return false;
}

// Owner CTA of global position x when [0, W) is cut into P ranges [c*W/P, (c+1)*W/P).
DEVI long long sk_owner(long long x, long long W, long long P) { return ((x + 1) * P + W - 1) / W - 1; }

// Tile (output columns) of consumer warp w in column group grp.
DEVI int sk_tile(const SGemvParams& p, int grp, int w, int& si) {
  if (p.paired) {
    si = w >> 2;
    return grp * 4 + (w & 3);
  }
  int gt = grp * kConsumers + w, acc = 0;
  for (int s = 0; s < p.nseg; ++s) {
    if (gt < acc + p.seg[s].tiles) {
      si = s;
      return gt - acc;
    }
    acc += p.seg[s].tiles;
  }
  si = 0;
  return -1;
}

// Weight records of column group grp (one group record per K unit).
template <bool Q4>
DEVI const uint8_t* sk_group_src(const SGemvParams& p, int grp) {
  if (p.paired) return p.seg[0].W + (size_t)grp * p.U * Ring<Q4>::kSlot;
  int acc = 0;
  for (int s = 0; s < p.nseg; ++s) {
    const int ng = p.seg[s].tiles / 8;
    if (grp < acc + ng) return p.seg[s].W + (size_t)(grp - acc) * p.U * Ring<Q4>::kSlot;
    acc += ng;
  }
  return nullptr;
}

DEVI int sk_rows(const SGemvParams& p, int si, int mz, int R) {
  int r = p.seg[si].rows - mz;
  return r > R ? R : (r < 0 ? 0 : r);
}

// Sum of the split-K partials of one output in piece order (deterministic); the loads go out in
// batches of 8 before they are added, so a fix-up costs one or two L2 round trips, not npieces.
DEVI float sum_pieces(const SGemvParams& p, int npieces, int row, int col) {
  const float* b = p.part + (size_t)row * p.ldo + col;
  float v = 0.f;
  for (int s0 = 0; s0 < npieces; s0 += 8) {
    float x[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) x[k] = s0 + k < npieces ? __ldcg(b + (size_t)(s0 + k) * p.piece_stride) : 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) v += x[k];
  }
  return v;
}

// Split-K sums of up to 4 outputs (row[k], col[k]; ok[k] false: 0), each in piece order (the same
// additions as sum_pieces); the loads of a round of 4 pieces for all 4 outputs go out together, so
// a fix-up thread pays one L2 round trip per 4 pieces rather than one per output.
DEVI void sum_pieces4(const SGemvParams& p, int npieces, const int (&row)[4], const int (&col)[4],
                      const bool (&ok)[4], float (&v)[4]) {
  const float* b[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    b[k] = p.part + (size_t)row[k] * p.ldo + col[k];
    v[k] = 0.f;
  }
  for (int s0 = 0; s0 < npieces; s0 += 4) {
    float x[4][4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        x[k][j] = ok[k] && s0 + j < npieces ? __ldcg(b[k] + (size_t)(s0 + j) * p.piece_stride) : 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int j = 0; j < 4; ++j) v[k] += x[k][j];
  }
}

// Split-K sums of N outputs (row[k], col[k]; ok[k] false: 0), each in piece order (the same
// additions as sum_pieces); all loads of a round of 4 pieces for all N outputs go out together.
template <int N>
DEVI void sum_pieces_n(const SGemvParams& p, int npieces, const int (&row)[N], const int (&col)[N],
                       const bool (&ok)[N], float (&v)[N]) {
  const float* b[N];
#pragma unroll
  for (int k = 0; k < N; ++k) {
    b[k] = p.part + (size_t)row[k] * p.ldo + col[k];
    v[k] = 0.f;
  }
  for (int s0 = 0; s0 < npieces; s0 += 4) {
    float x[N][4];
#pragma unroll
    for (int k = 0; k < N; ++k)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        x[k][j] = ok[k] && s0 + j < npieces ? __ldcg(b[k] + (size_t)(s0 + j) * p.piece_stride) : 0.f;
#pragma unroll
    for (int k = 0; k < N; ++k)
#pragma unroll
      for (int j = 0; j < 4; ++j) v[k] += x[k][j];
  }
}

// Split-K sums of N groups of 4 consecutive outputs (row[k], col[k] .. col[k] + 3, col[k] a
// multiple of 4; ok[k] false: 0), each output in piece order (the same additions as sum_pieces),
// with 16-byte loads: all loads of a round of 2 pieces for all N groups go out together.
template <int N>
DEVI void sum_pieces_q(const SGemvParams& p, int npieces, const int (&row)[N], const int (&col)[N],
                       const bool (&ok)[N], float4 (&v)[N]) {
  const float* b[N];
#pragma unroll
  for (int k = 0; k < N; ++k) {
    b[k] = p.part + (size_t)row[k] * p.ldo + col[k];
    v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int s0 = 0; s0 < npieces; s0 += 2) {
    float4 x[N][2];
#pragma unroll
    for (int k = 0; k < N; ++k)
#pragma unroll
      for (int j = 0; j < 2; ++j)
        x[k][j] = ok[k] && s0 + j < npieces
                      ? __ldcg(reinterpret_cast<const float4*>(b[k] + (size_t)(s0 + j) * p.piece_stride))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < N; ++k)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        v[k].x += x[k][j].x;
        v[k].y += x[k][j].y;
        v[k].z += x[k][j].z;
        v[k].w += x[k][j].w;
      }
  }
}

DEVI uint2 pack_bf4(float a, float b, float c, float d) { return make_uint2(pack_bf2(a, b), pack_bf2(c, d)); }

// Epilogue of one column group over rows [mz, mz + R) (consumer threads only).
// rs_pre: row scales of rows [0, rows) computed at the kernel's start (single row group), or null.
template <int E = -1>
DEVI void sk_fixup(const SGemvParams& p, int grp, int mz, int R, int npieces, const float* rs_pre = nullptr) {
  const int epi = E >= 0 ? E : p.epi;  // a compile-time epilogue lets a kernel drop the other branches
  const int tid = threadIdx.x, nthr = kGemvConsumers * 32, warp = tid >> 5, lane = tid & 31;
  __shared__ float s_rs[72];
  const float* rsv = s_rs;
  if (p.paired) {
    const int f0 = grp * 64;
    const int rows = sk_rows(p, 0, mz, R);
    // the convolution's x_{t-1} of the group's first row may be the previous row group's last
    const int pre = epi == EPI_DYNCONV && mz > 0 ? 1 : 0;
    if (p.rs_in) {
      if (p.rs_glob) rsv = p.rs_glob + (mz - pre);
      else if (rs_pre && mz == 0) rsv = rs_pre;
      else rows_scale(p.rs_in, p.ssp_rows, p.rs_H, p.eps, mz - pre, rows + pre, s_rs);
    }
    if (epi != EPI_DYNCONV) {
      // two groups of 4 features (gate and up partials each) per thread per round, 16-byte loads
      constexpr int NQ = 2;
      for (int i0 = tid; i0 < rows * 16; i0 += NQ * nthr) {
        float4 sv[2 * NQ];
        {
          int rw[2 * NQ], cl[2 * NQ];
          bool okk[2 * NQ];
#pragma unroll
          for (int k = 0; k < NQ; ++k) {
            const int i = i0 + k * nthr, r = i >> 4, f = f0 + (i & 15) * 4;
            okk[2 * k] = okk[2 * k + 1] = i < rows * 16;
            rw[2 * k] = rw[2 * k + 1] = mz + r;
            cl[2 * k] = p.seg[0].out_col + f;
            cl[2 * k + 1] = p.seg[1].out_col + f;
          }
          sum_pieces_q<2 * NQ>(p, npieces, rw, cl, okk, sv);
        }
#pragma unroll
        for (int k = 0; k < NQ; ++k) {
          const int i = i0 + k * nthr, r = i >> 4, f = f0 + (i & 15) * 4;
          if (i >= rows * 16) continue;
          const float sc = p.rs_in ? rsv[r] : 1.f;
          const float4 g = make_float4(sv[2 * k].x * sc, sv[2 * k].y * sc, sv[2 * k].z * sc, sv[2 * k].w * sc);
          const float4 u =
              make_float4(sv[2 * k + 1].x * sc, sv[2 * k + 1].y * sc, sv[2 * k + 1].z * sc, sv[2 * k + 1].w * sc);
          if (epi == EPI_SWIGLU) {
            *reinterpret_cast<uint2*>(p.act + (size_t)(mz + r) * p.F + f) =
                pack_bf4(g.x / (1.f + __expf(-g.x)) * u.x, g.y / (1.f + __expf(-g.y)) * u.y,
                         g.z / (1.f + __expf(-g.z)) * u.z, g.w / (1.f + __expf(-g.w)) * u.w);
          } else {  // EPI_STORE
            *reinterpret_cast<float4*>(p.y + (size_t)(mz + r) * p.ldy + p.seg[0].out_col + f) = g;
            *reinterpret_cast<float4*>(p.y + (size_t)(mz + r) * p.ldy + p.seg[1].out_col + f) = u;
          }
        }
      }
      return;
    }
    // the convolution: four outputs per thread per round, all their partial loads in flight together
    constexpr int NO = 4;
    for (int i0 = tid; i0 < rows * 64; i0 += NO * nthr) {
      float gv[NO], uv[NO];
      float4 hc[NO], hp[NO];
      uint2 wv[NO], e0[NO], e1[NO];
      {
        int rw[2 * NO], cl[2 * NO];
        bool okk[2 * NO];
        float sv[2 * NO];
#pragma unroll
        for (int k = 0; k < NO; ++k) {
          const int i = i0 + k * nthr, r = i >> 6, f = f0 + (i & 63);
          okk[2 * k] = okk[2 * k + 1] = i < rows * 64;
          rw[2 * k] = rw[2 * k + 1] = mz + r;
          cl[2 * k] = p.seg[0].out_col + f;
          cl[2 * k + 1] = p.seg[1].out_col + f;
          // the convolution's operands go out with the partial loads
          hc[k] = hp[k] = make_float4(0.f, 0.f, 0.f, 0.f);
          wv[k] = e0[k] = e1[k] = make_uint2(0, 0);
          if (okk[2 * k] && epi == EPI_DYNCONV) {
            const int row = mz + r, H = p.rs_H;
            hc[k] = __ldcg(reinterpret_cast<const float4*>(p.dyn_h + (size_t)row * H + 4 * f));
            if (row % p.Bk > 0) hp[k] = __ldcg(reinterpret_cast<const float4*>(p.dyn_h + (size_t)(row - 1) * H + 4 * f));
            wv[k] = *reinterpret_cast<const uint2*>(p.dyn_w + 4 * f);
            e0[k] = *reinterpret_cast<const uint2*>(p.dyn_s0 + 4 * f);
            e1[k] = *reinterpret_cast<const uint2*>(p.dyn_s1 + 4 * f);
          }
        }
        sum_pieces_n<2 * NO>(p, npieces, rw, cl, okk, sv);
#pragma unroll
        for (int k = 0; k < NO; ++k) {
          gv[k] = sv[2 * k];
          uv[k] = sv[2 * k + 1];
        }
      }
#pragma unroll
      for (int k = 0; k < NO; ++k) {
        const int i = i0 + k * nthr, r = i >> 6, f = f0 + (i & 63);
        if (i >= rows * 64) continue;
        const float sc = p.rs_in ? rsv[pre + r] : 1.f;
        const float g = gv[k] * sc, u = uv[k] * sc;
        if (epi == EPI_SWIGLU) {
          p.act[(size_t)(mz + r) * p.F + f] = f2bf(g / (1.f + __expf(-g)) * u);
        } else if (epi == EPI_STORE) {
          p.y[(size_t)(mz + r) * p.ldy + p.seg[0].out_col + f] = g;
          p.y[(size_t)(mz + r) * p.ldy + p.seg[1].out_col + f] = u;
        } else {  // EPI_DYNCONV: channels 4f .. 4f + 3 of block row mz + r, gates (g, u) of that row
          const int row = mz + r, t = row % p.Bk, H = p.rs_H;
          const float a0 = tanhf(g), a1 = tanhf(u), rc = rsv[pre + r];
          const float rp = t > 0 ? rsv[pre + r - 1] : 0.f;
          const float4 c4 = hc[k], p4 = hp[k];
          const uint2 w2 = wv[k], s0 = e0[k], s1 = e1[k];
          const float n0 = bf2f(w2.x & 0xffff), n1 = bf2f(w2.x >> 16), n2 = bf2f(w2.y & 0xffff), n3 = bf2f(w2.y >> 16);
          const float y0 = (bf2f(s0.x & 0xffff) + a0) * (c4.x * rc * n0) + (bf2f(s1.x & 0xffff) + a1) * (p4.x * rp * n0);
          const float y1 = (bf2f(s0.x >> 16) + a0) * (c4.y * rc * n1) + (bf2f(s1.x >> 16) + a1) * (p4.y * rp * n1);
          const float y2 = (bf2f(s0.y & 0xffff) + a0) * (c4.z * rc * n2) + (bf2f(s1.y & 0xffff) + a1) * (p4.z * rp * n2);
          const float y3 = (bf2f(s0.y >> 16) + a0) * (c4.w * rc * n3) + (bf2f(s1.y >> 16) + a1) * (p4.w * rp * n3);
          *reinterpret_cast<uint2*>(p.dyn_y + (size_t)row * H + 4 * f) = make_uint2(pack_bf2(y0, y1), pack_bf2(y2, y3));
        }
      }
    }
    return;
  }
  int si = 0;
  const int tile0 = sk_tile(p, grp, 0, si);
  if (tile0 < 0) return;
  const int col0 = p.seg[si].out_col + tile0 * 16;
  const int rows = sk_rows(p, si, mz, R);
  if (p.rs_in && epi == EPI_STORE) {
    if (p.rs_glob) rsv = p.rs_glob + mz;
    else if (rs_pre && mz == 0) rsv = rs_pre;
    else rows_scale(p.rs_in, p.ssp_rows, p.rs_H, p.eps, mz, rows, s_rs);
  }
  if (epi == EPI_QKV) {
    const int head = tile0 / 8;
    for (int r = warp; r < rows; r += kGemvConsumers) {
      float x[4];
      const int rw[4] = {mz + r, mz + r, mz + r, mz + r};
      const int cl[4] = {col0 + 2 * lane, col0 + 2 * lane + 1, col0 + 64 + 2 * lane, col0 + 65 + 2 * lane};
      const bool okk[4] = {true, true, true, true};
      const QkvPre pre = qkv_prefetch(p.qkv, si, mz + r, lane);  // in flight with the partial loads
      sum_pieces4(p, npieces, rw, cl, okk, x);
      qkv_head_row(p.qkv, si, head, mz + r, x, lane, pre);
    }
    return;
  }
  // four groups of 4 consecutive columns per thread per round: all their partial loads (and the
  // residual reads) are in flight together before any store; a warp covers one row's 128 columns
  constexpr int NR = 4;
  for (int i0 = tid; i0 < rows * 32; i0 += NR * nthr) {
    float4 v[NR], old[NR];
    uint2 hwv[NR];
    {
      int rw[NR], cl[NR];
      bool okk[NR];
#pragma unroll
      for (int k = 0; k < NR; ++k) {
        const int i = i0 + k * nthr;
        rw[k] = mz + (i >> 5);
        cl[k] = col0 + (i & 31) * 4;
        okk[k] = i < rows * 32;
        // L2 read: another CTA may have written the residual row
        old[k] = okk[k] && epi == EPI_RESID
                     ? __ldcg(reinterpret_cast<const float4*>(p.y + (size_t)rw[k] * p.ldy + cl[k]))
                     : make_float4(0.f, 0.f, 0.f, 0.f);
        hwv[k] = okk[k] && epi == EPI_RESID && p.hw ? *reinterpret_cast<const uint2*>(p.hw_w + cl[k])
                                                     : make_uint2(0u, 0u);
      }
      sum_pieces_q<NR>(p, npieces, rw, cl, okk, v);
    }
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      const int i = i0 + k * nthr, r = i >> 5, c = col0 + (i & 31) * 4;
      if (i >= rows * 32) break;  // warp-uniform: rows * 32 is a multiple of 32
      float* y = p.y + (size_t)(mz + r) * p.ldy + c;
      if (epi == EPI_RESID) {
        const float4 nv = make_float4(old[k].x + v[k].x, old[k].y + v[k].y, old[k].z + v[k].z, old[k].w + v[k].w);
        *reinterpret_cast<float4*>(y) = nv;
        if (p.hw)
          *reinterpret_cast<uint2*>(p.hw + (size_t)(mz + r) * p.hw_ld + c) =
              pack_bf4(nv.x * bf2f(hwv[k].x & 0xffff), nv.y * bf2f(hwv[k].x >> 16), nv.z * bf2f(hwv[k].y & 0xffff),
                       nv.w * bf2f(hwv[k].y >> 16));
        if (p.ssp) {  // sum of squares of each 32-column quarter of the new row (8 lanes), for the next RMSNorm
          float q = nv.x * nv.x + nv.y * nv.y + nv.z * nv.z + nv.w * nv.w;
          q += __shfl_xor_sync(0xffffffffu, q, 1);
          q += __shfl_xor_sync(0xffffffffu, q, 2);
          q += __shfl_xor_sync(0xffffffffu, q, 4);
          if ((lane & 7) == 0) p.ssp[((size_t)(col0 >> 7) * 4 + (lane >> 3)) * p.ssp_rows + mz + r] = q;
        }
      } else {
        const float sc = p.rs_in ? rsv[r] : 1.f;
        *reinterpret_cast<float4*>(y) = make_float4(v[k].x * sc, v[k].y * sc, v[k].z * sc, v[k].w * sc);
      }
    }
  }
}

// Bring rows [0, nrows) of an X chunk (row stride ldx elements, `bytes` per row) into Xs (row
// stride `stride` bytes) with bulk copies on xbar; rows [nrows, R) are zeroed.  Consumer threads.
// Work done while a staging copy is in flight: a folded RMSNorm's row scales (once).
struct StageRs {
  const SGemvParams* p;
  float* s_rs;
  bool pending;
};

template <int NTHR>
DEVI void stage_x_chunk(const uint16_t* X, int ldx, int nrows, int R, int bytes, uint8_t* Xs, int stride,
                        uint64_t* xbar, uint32_t& xph, int* err, StageRs* rs = nullptr) {
  consumers_sync<NTHR>();  // every consumer is done with the previous chunk
  if (threadIdx.x == 0) {
    mbar_expect_tx(xbar, (uint32_t)(nrows * bytes));
    for (int r = 0; r < nrows; ++r) bulk_g2s(Xs + r * stride, X + (size_t)r * ldx, bytes, xbar);
  }
  for (int i = threadIdx.x; i < (R - nrows) * (bytes / 16); i += NTHR) {
    const int r = nrows + i / (bytes / 16), v = i % (bytes / 16);
    *reinterpret_cast<uint4*>(Xs + r * stride + v * 16) = make_uint4(0, 0, 0, 0);
  }
  if (rs && rs->pending) {  // (rows_scale ends with the consumer barrier)
    rows_scale(rs->p->rs_in, rs->p->ssp_rows, rs->p->rs_H, rs->p->eps, 0, rs->p->rows, rs->s_rs);
    rs->pending = false;
  } else {
    consumers_sync<NTHR>();
  }
  if (!mbar_wait_sleep_bounded(xbar, xph) && threadIdx.x == 0) set_err(err, DFLASH2_DEV_TIMEOUT);
  xph ^= 1u;
}

template <int NT, bool Q4>
__global__ void __launch_bounds__(kSGemvThreads, 1) k_sgemv(SGemvParams p) {
  using RC = Ring<Q4>;
  constexpr int R = NT * 8;
  constexpr int NC = kGemvConsumers * 32;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[RC::kNS];
  __shared__ __align__(8) uint64_t empty[RC::kNS];
  __shared__ __align__(8) uint64_t xbar;
  __shared__ __align__(8) uint64_t seen;  // the watcher saw the other pieces of the last group
  __shared__ int s_last;
  uint8_t* ring = smem;
  uint8_t* Xs = smem + RC::kNS * RC::kSlot;
  const int stride = p.kc_units * RC::kUnitK * 2 + 64;
  float2* coef_all = reinterpret_cast<float2*>(Xs + R * stride);                // [16 warps][128]
  float* red = reinterpret_cast<float*>(coef_all + kGemvConsumers * 128);       // [8][32][NT*4]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int set = warp / kConsumers, wt = warp % kConsumers;

  if (threadIdx.x == 0) {
    for (int s = 0; s < RC::kNS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);  // the 8 warps of the set that owns the slot
    }
    mbar_init(&xbar, 1);
    mbar_init(&seen, 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger();
  const long long P = gridDim.x, c = blockIdx.x;
  const long long x0 = c * p.W / P, x1 = (c + 1) * p.W / P;

  if (warp == kGemvConsumers + 1) {
    // ---- watcher: when this CTA fixes up the group its range ends in, wait for that group's
    // other pieces now, so the consumers find them arrived when they get there ----
    if (lane != 0 || x1 <= x0) return;
    const long long gstart = (x1 - 1) / p.U * p.U;
    const int gidx = (int)(gstart / p.U);
    const long long first = sk_owner(gstart, p.W, P);
    const int npieces = (int)(sk_owner(gstart + p.U - 1, p.W, P) - first + 1);
    if (c != first || npieces < 2) return;
    s_last = await_pieces(p.counters + gidx, npieces - 1) ? 1 : 0;
    mbar_arrive(&seen);  // (release: orders the flag and the acquired arrivals before the consumers)
    return;
  }

  if (warp == kGemvConsumers) {
    // ---- producer: weights only, so it may run ahead of the previous kernel ----
    if (lane != 0) return;
    int cnt = 0;
    for (long long x = x0; x < x1;) {
      const int gidx = (int)(x / p.U), ua = (int)(x % p.U);
      const int ub = (int)((x1 - x) < (long long)(p.U - ua) ? ua + (x1 - x) : p.U);
      const int grp = gidx % p.groups, mz = (gidx / p.groups) * 64;
      int si;
      sk_tile(p, grp, 0, si);
      if (sk_rows(p, si, mz, R) > 0) {
        const uint8_t* src = sk_group_src<Q4>(p, grp);
        for (int u = ua; u < ub; ++u) {
          const int slot = cnt % RC::kNS, round = cnt / RC::kNS;
          if (round > 0 && !mbar_wait_bounded(&empty[slot], (round - 1) & 1)) {
            set_err(p.err, DFLASH2_DEV_TIMEOUT);
            return;
          }
          mbar_expect_tx(&full[slot], RC::kSlot);
          bulk_g2s(ring + slot * RC::kSlot, src + (size_t)u * RC::kSlot, RC::kSlot, &full[slot]);
          ++cnt;
        }
      }
      x += ub - ua;
    }
    return;
  }

  // ---- consumers: ring slot k is consumed by warp set (k & 1) ----
  pdl_wait();  // activations and the partial/ticket buffers come from earlier kernels
  // a folded RMSNorm's row scales, computed now (off the fix-up's critical path) when all rows
  // form one row group
  __shared__ float s_rs0[64];
  const bool rs_early = p.rs_in && p.rows <= 64;
  StageRs srs{&p, s_rs0, rs_early};  // computed while the first activation copy is in flight
  float2* coef = coef_all + warp * 128;
  int cnt = 0, staged_mz = -1;
  uint32_t xph = 0;
  bool dead = false;
  for (long long x = x0; x < x1;) {
    const int gidx = (int)(x / p.U), ua = (int)(x % p.U);
    const int ub = (int)((x1 - x) < (long long)(p.U - ua) ? ua + (x1 - x) : p.U);
    const int grp = gidx % p.groups, mz = (gidx / p.groups) * 64;
    int si;
    const int tile = sk_tile(p, grp, wt, si);
    const int my_rows = sk_rows(p, si, mz, R);
    const int ntact = (my_rows + 7) >> 3;
    int stage_rows = p.rows - mz;
    stage_rows = stage_rows > R ? R : stage_rows;
    float acc[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    if (ntact > 0) {
      const bool whole = p.kc_units >= p.U;  // all of K fits: stage X once per row group and keep it
      for (int c0 = ua; c0 < ub; c0 += p.kc_units) {
        const int cu = (ub - c0) < p.kc_units ? (ub - c0) : p.kc_units;
        int base = c0;
        if (whole) {
          base = 0;
          if (staged_mz != mz) {
            stage_x_chunk<NC>(p.X + (size_t)mz * p.ldx, p.ldx, stage_rows, R, p.U * RC::kUnitK * 2, Xs, stride, &xbar,
                              xph, p.err, &srs);
            staged_mz = mz;
          }
        } else {
          stage_x_chunk<NC>(p.X + (size_t)mz * p.ldx + (size_t)c0 * RC::kUnitK, p.ldx, stage_rows, R,
                            cu * RC::kUnitK * 2, Xs, stride, &xbar, xph, p.err, &srs);
        }
        for (int u = c0; u < c0 + cu; ++u) {
          const int slot = cnt % RC::kNS;
          const bool mine = (cnt & 1) == set;
          const uint32_t par = (cnt / RC::kNS) & 1;
          ++cnt;
          if (!mine) continue;
          // a consumer never leaves early (the named barriers count on it): after an expired
          // wait it flags the error and skips its remaining work
          if (!dead && !mbar_wait_sleep_bounded(&full[slot], par)) {
            set_err(p.err, DFLASH2_DEV_TIMEOUT);
            dead = true;
          }
          if (dead) continue;
          const uint8_t* sb = ring + slot * RC::kSlot + wt * RC::kUnitBytes;
          if (Q4) {
            uint4 q[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) q[i] = lds_slot(sb + (i * 32 + lane) * 16);
            const uint4 sc = lds_slot(sb + 2048 + (lane >> 1) * 16);
            q4_unit<NT>(q, sc, coef, Xs, stride, (u - base) * 512, ntact, acc, lane, p.mlx != 0);
            slot_release(&empty[slot], q[0].x ^ q[1].x ^ q[2].x ^ q[3].x ^ sc.x, lane);
          } else {
            uint4 wv[4];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              wv[2 * j] = lds_slot(sb + j * 1024 + lane * 16);
              wv[2 * j + 1] = lds_slot(sb + j * 1024 + 512 + lane * 16);
            }
            bf16_step<NT, 2>(wv, Xs, stride, (u - base) * 128, ntact, acc, lane);
            slot_release(&empty[slot], wv[0].x ^ wv[1].x ^ wv[2].x ^ wv[3].x, lane);
          }
        }
      }
    }
    // the two sets' accumulators meet in shared memory; set 0 writes the piece's partial
    if (ntact > 0 && set == 1) {
      float* rd = red + (wt * 32 + lane) * (NT * 4);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) rd[nt * 4 + e] = acc[nt][e];
    }
    consumers_sync<NC>();
    const long long gstart = (long long)gidx * p.U;
    const long long first = sk_owner(gstart, p.W, P);
    const int piece = (int)(c - first);
    const int npieces = (int)(sk_owner(gstart + p.U - 1, p.W, P) - first + 1);
    if (ntact > 0 && set == 0) {
      const float* rd = red + (wt * 32 + lane) * (NT * 4);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] += rd[nt * 4 + e];
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
    // split-K: the owner of the group's first unit (it reaches the group last, at the end of its
    // range, unless the whole group lies inside it) sums the partials in range order
    // (deterministic) and runs the epilogue; the other owners post their arrival and go on
    consumers_sync<NC>();
    if (c != first) {
      if (threadIdx.x == 0) arrive_release(p.counters + gidx);
    } else {
      bool go = true;  // a group inside this range has no other pieces
      if (npieces > 1) {  // the group this range ends in: the watcher waited for its pieces
        go = mbar_wait_bounded(&seen, 0) && s_last != 0;
        if (!go && threadIdx.x == 0) set_err(p.err, DFLASH2_DEV_TIMEOUT);
        if (threadIdx.x == 0) p.counters[gidx] = 0;  // every piece has arrived: rearm
      }
      if (go && ntact > 0) sk_fixup(p, grp, mz, R, npieces, rs_early ? s_rs0 : nullptr);
    }
    x += ub - ua;
  }
}

// ---------------------------------------------------------------------------
// Shared output head + streaming top-16 (<= 8 drafted rows), same engine: the prepared
// [V + R rows] bf16 matrix (output head, then the selector projection) is stored in records of
// 16 tiles per 64-wide K step (32 KB, one bulk copy), handed out record by record to the
// persistent CTAs.  All 16 consumer warps take every slot: warp (half, wt) owns tile
// 8 * half + wt of the record and accumulates it over all K steps.  Logits never leave the SM:
// after its tile each warp offers the values to its own per-row sorted top-16 lists in shared
// memory; at the end the CTA merges its 16 warp lists, and the selector merges the CTAs'.

// Offer one tile's logits (this lane: rows 2t, 2t+1 at vocabulary ids id0 + g and id0 + g + 8,
// i.e. acc[e] at row 2t + (e & 1), id id0 + g + 8 * (e >> 1)) to the warp's sorted per-row lists
// lists[r * 16 + k] = (value bits, id), best first.  Entries beating a row's current 16th are
// inserted one at a time, the 16 list positions shifting in parallel across lanes 0-15.
DEVI void offer_tile(uint2* lists, const float (&acc)[4], int id0, int rows, int lane) {
  const int g = lane >> 2, t = lane & 3;
  unsigned m[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int r = 2 * t + (e & 1);
    bool want = false;
    if (r < rows) {
      const uint2 last = lists[r * kTopK + kTopK - 1];
      want = better(acc[e], id0 + g + 8 * (e >> 1), __uint_as_float(last.x), (int)last.y);
    }
    m[e] = __ballot_sync(0xffffffffu, want);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    while (m[e]) {
      const int src = __ffs(m[e]) - 1;
      m[e] &= m[e] - 1;
      const float v = __shfl_sync(0xffffffffu, acc[e], src);
      const int id = id0 + (src >> 2) + 8 * (e >> 1);
      uint2* L = lists + (2 * (src & 3) + (e & 1)) * kTopK;
      const uint2 cur = lane < kTopK ? L[lane] : make_uint2(0u, 0u);
      const bool ahead = lane < kTopK && better(__uint_as_float(cur.x), (int)cur.y, v, id);
      const int pos = __popc(__ballot_sync(0xffffffffu, ahead));  // entries that stay ahead (a prefix)
      __syncwarp();
      if (pos < kTopK) {
        if (lane >= pos && lane < kTopK - 1) L[lane + 1] = cur;
        if (lane == pos) L[pos] = make_uint2(__float_as_uint(v), (unsigned)id);
      }
      __syncwarp();
    }
  }
}

// Merge the 16 warp lists of each row into the CTA's list -> cand_val/cand_id[part][row][16].
// Lane l owns a sorted run of 8 entries (warp list l/2, entries 8*(l&1) .. +7) and a read position;
// each round the warp picks the best run head (ties: lower lane) and that lane advances.
// rows_total / row0: the output lists are [part][rows_total][16], this CTA's rows start at row0.
DEVI void merge_warp_lists(const uint2* lists, int rows, float* cand_val, int32_t* cand_id, int part, int warp,
                           int nwarps, int lane, int rows_total = -1, int row0 = 0) {
  if (rows_total < 0) rows_total = rows;
  for (int r = warp; r < rows; r += nwarps) {
    const uint2* run = lists + ((lane >> 1) * 8 + r) * kTopK + (lane & 1) * 8;
    int pos = 0;
    for (int kk = 0; kk < kTopK; ++kk) {
      const uint2 e = pos < 8 ? run[pos] : make_uint2(__float_as_uint(-INFINITY), 0x7fffffffu);
      float bv = __uint_as_float(e.x);
      int bid = (int)e.y, bl = lane;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oid = __shfl_xor_sync(0xffffffffu, bid, o);
        const int ol = __shfl_xor_sync(0xffffffffu, bl, o);
        if (better(ov, oid, bv, bid) || (ov == bv && oid == bid && ol < bl)) { bv = ov; bid = oid; bl = ol; }
      }
      if (lane == 0) {
        const size_t o = ((size_t)part * rows_total + row0 + r) * kTopK + kk;
        cand_val[o] = bv;
        cand_id[o] = bid;
      }
      if (lane == bl) ++pos;
    }
  }
}

struct SLmParams {
  const uint8_t* W;  // prepared bf16 records of [lm_head; sel_proj]
  int V, R, H;
  const uint16_t* X;  // final-normed rows [rows][H]
  int rows;           // all rows; groups of 8 (row group g: rows 8g .. 8g + 7)
  int groups;         // row groups: CTA b works on vocabulary part b / groups for row group b % groups
  float* z;           // [rows][R]
  float* cand_val;    // [parts][rows][16]
  int32_t* cand_id;
  float* part;        // split records' partial accumulators [groups][parts][2][16 warps][32 lanes][4]
  int* counters;      // [groups][records] arrival tickets, zero before the launch (the last arrival re-zeroes)
  int* err;
  int id0;            // vocabulary id of the head's first row (a shard of the vocabulary; 0 for the whole head)
};

constexpr int kHeadSlot = kHeadTiles * 2048;  // one record step: 32 KB
constexpr int kHeadNS = 4;

// Work split: stream-K over (record, K step) units, CTA c taking [c*W/P, (c+1)*W/P) of the
// W = records * (H/64) steps, so every SM streams the same number of bytes.  A record cut between
// CTAs leaves each owner's accumulators in `part`; the last owner to arrive (arrival ticket, no
// waiting) adds them in owner order (deterministic) and offers the tile's logits.
__global__ void __launch_bounds__(kGemvThreads, 1) k_slmhead(SLmParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[kHeadNS];
  __shared__ __align__(8) uint64_t empty[kHeadNS];
  __shared__ __align__(8) uint64_t xbar;
  __shared__ int s_last;
  constexpr int NC = kGemvConsumers * 32;
  const int H = p.H, stride = H * 2 + 64;
  uint8_t* ring = smem;
  uint8_t* Xs = smem + kHeadNS * kHeadSlot;
  uint2* lists = reinterpret_cast<uint2*>(Xs + 8 * stride);  // [16 warps][8 rows][16]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int half = warp >> 3, wt = warp & 7;
  const int vt = p.V / 16, total = vt + p.R / 16, S = H / 64;
  const int nrec = (total + kHeadTiles - 1) / kHeadTiles;
  // row group g of vocabulary part c: the groups of one part are neighbours in launch order, so
  // they stream the same records at about the same time (HBM once, L2 for the others)
  const int G = p.groups, grp = blockIdx.x % G, row0 = grp * 8;
  const int rows = p.rows - row0 < 8 ? p.rows - row0 : 8;
  const long long W = (long long)nrec * S, P = gridDim.x / G, c = blockIdx.x / G;
  float* part_g = p.part + (size_t)grp * P * 2 * kGemvConsumers * 32 * 4;
  int* ctr_g = p.counters + (size_t)grp * nrec;
  const long long x0 = c * W / P, x1 = (c + 1) * W / P;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kHeadNS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGemvConsumers);
    }
    mbar_init(&xbar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger();

  if (warp == kGemvConsumers) {
    // ---- producer: this CTA's range of record steps is one contiguous stretch of the head ----
    if (lane != 0) return;
    int cnt = 0;
    for (long long x = x0; x < x1; ++x) {
      const int slot = cnt % kHeadNS, round = cnt / kHeadNS;
      if (round > 0 && !mbar_wait_bounded(&empty[slot], (round - 1) & 1)) {
        set_err(p.err, DFLASH2_DEV_TIMEOUT);
        return;
      }
      mbar_expect_tx(&full[slot], kHeadSlot);
      bulk_g2s(ring + slot * kHeadSlot, p.W + (size_t)x * kHeadSlot, kHeadSlot, &full[slot]);
      ++cnt;
    }
    return;
  }

  for (int i = threadIdx.x; i < kGemvConsumers * 8 * kTopK; i += NC)
    lists[i] = make_uint2(__float_as_uint(-INFINITY), 0x7fffffffu);
  pdl_wait();
  uint32_t xph = 0;
  stage_x_chunk<NC>(p.X + (size_t)row0 * H, H, rows, 8, H * 2, Xs, stride, &xbar, xph, p.err);
  uint2* my = lists + warp * 8 * kTopK;
  int cnt = 0;
  bool dead = false;
  const int rec_first = (int)(x0 / S);
  for (long long x = x0; x < x1;) {
    const int rec = (int)(x / S), s0 = (int)(x % S);
    const int s1 = (x1 - x) < (long long)(S - s0) ? s0 + (int)(x1 - x) : S;
    const int tile = rec * kHeadTiles + half * 8 + wt;
    float acc[1][4] = {{0.f, 0.f, 0.f, 0.f}};
    for (int s = s0; s < s1; ++s) {
      const int slot = cnt % kHeadNS;
      if (!dead && !mbar_wait_sleep_bounded(&full[slot], (cnt / kHeadNS) & 1)) {
        set_err(p.err, DFLASH2_DEV_TIMEOUT);
        dead = true;
      }
      ++cnt;
      if (dead) continue;
      const uint8_t* sb = ring + slot * kHeadSlot + (half * 8 + wt) * 2048;
      uint4 wv[4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        wv[2 * j] = lds_slot(sb + j * 1024 + lane * 16);
        wv[2 * j + 1] = lds_slot(sb + j * 1024 + 512 + lane * 16);
      }
      bf16_step<1, 2>(wv, Xs, stride, s * 128, 1, acc, lane);
      slot_release(&empty[slot], wv[0].x ^ wv[1].x ^ wv[2].x ^ wv[3].x, lane);
    }
    x += s1 - s0;
    bool have = true;
    if (s0 > 0 || s1 < S) {
      // a record cut between CTAs: owners first..last of its steps
      const long long ux = (long long)rec * S;
      const long long first = sk_owner(ux, W, P), last = sk_owner(ux + S - 1, W, P);
      const int k = rec == rec_first ? 0 : 1;
      float4* mine = reinterpret_cast<float4*>(part_g) + ((c * 2 + k) * kGemvConsumers + warp) * 32 + lane;
      *mine = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
      consumers_sync<NC>();
      if (threadIdx.x == 0) {
        const int prev = ticket_acq_rel(ctr_g + rec);
        s_last = prev == (int)(last - first);
        if (s_last) ctr_g[rec] = 0;
      }
      consumers_sync<NC>();
      have = s_last != 0;
      if (have) {
        float a[4] = {0.f, 0.f, 0.f, 0.f};
        for (long long o = first; o <= last; ++o) {
          float4 v;
          if (o == c) {
            v = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
          } else {
            const int ko = rec == (int)((o * W / P) / S) ? 0 : 1;
            v = __ldcg(reinterpret_cast<const float4*>(part_g) + ((o * 2 + ko) * kGemvConsumers + warp) * 32 + lane);
          }
          a[0] += v.x;
          a[1] += v.y;
          a[2] += v.z;
          a[3] += v.w;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[0][e] = a[e];
      }
    }
    if (!have || dead || tile >= total) continue;
    if (tile >= vt) {
      const int c0 = (tile - vt) * 16;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = 2 * t + (e & 1);
        if (r < rows) p.z[(size_t)(row0 + r) * p.R + c0 + g + 8 * (e >> 1)] = acc[0][e];
      }
    } else {
      offer_tile(my, acc[0], p.id0 + tile * 16, rows, lane);
    }
  }
  consumers_sync<NC>();
  merge_warp_lists(lists, rows, p.cand_val, p.cand_id, (int)c, warp, kGemvConsumers, lane, p.rows, row0);
}

}  // namespace dfl
