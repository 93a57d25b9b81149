// Persistent block step for one request (block <= 8): the whole step in one launch.
//
// At batch 1 every matrix of the step is streamed once and the work between them is tiny, so
// a step of ~50 separate kernels spends much of its time in launch, ramp-up and drain.  Here one
// CTA per SM (cooperative launch, so all are resident) runs every op of the step in order,
// separated by grid barriers where an op reads what another CTA wrote.  The producer warp never
// takes part in the barriers: it walks the step's whole sequence of streamed matrices (fc, the
// five layers' W_dc, q|k|v, W_o, gate|up, W_d, then the output head) and keeps the CTA's ring of
// three 36 KB shared-memory slots full with 1-D bulk copies, so HBM streams continuously across
// op boundaries, attention and barriers.  A slot holds two consecutive K units of one column
// group (large copies: the copy engine sustains near-peak HBM bandwidth at 32 KB per copy, not at
// 16 KB); all 16 consumer warps take every slot, warps 0-7 the first unit's 8 tiles and warps
// 8-15 the second's, and release it as soon as its bytes are in registers.
//
// RMSNorms and the dynamic convolution are computed inside the activation staging of the GEMV
// that consumes them.  The per-row RMS comes from sums of squares that the residual epilogues
// leave per 32-column quarter (no extra pass over the rows), and each CTA stages only the K range
// of its own units.  Data written by other CTAs is read through L2 (ld.cg) or by bulk copies.
#pragma once
#include "attention.cuh"
#include "selector.cuh"
#include "stream.cuh"

namespace dfl {

constexpr int kPUnits = 2;                      // K units per ring slot
constexpr int kPSlot = kQ4Bytes * 8 * kPUnits;  // two Q4_K group units (36864 B), two bf16 64-wide steps or one head record step (32768 B)
constexpr int kPNS = 3;
constexpr int kPThreads = kGemvThreads;     // 16 consumer warps + 1 producer warp
constexpr int kPNC = kGemvConsumers * 32;   // consumer threads
constexpr int kPXBytes = 82944;             // activation staging (8 rows x 5120 bf16 + padding); attention buffers
constexpr int kPWshBytes = 4096;            // attention-combine weights [16 warps][64] floats
constexpr long long kBarrierSpin = 1ll << 24;
constexpr unsigned long long kBarrierNs = 2000000000ull;  // 2 s

enum : int { STG_COPY = 0, STG_NORM = 1, STG_DYNCONV = 2 };

struct PGemv {
  SGemvParams g;            // segments, stream-K plan, epilogue; g.X for STG_COPY
  int P;                    // CTAs the K units are split over (min(#SMs, W)); CTAs >= P have no share
  int q4;                   // 1: Q4_K units of 256; 0: bf16 steps of 64
  int stage;
  const uint16_t* nw;       // STG_NORM / STG_DYNCONV: RMSNorm weight [H] applied to h
  const float* gdc;         // STG_DYNCONV: gates [Mb][H/2]
  const uint16_t *s0, *s1;  // STG_DYNCONV: static taps [H]
  const uint16_t* ctx;      // STG_DYNCONV: context rows [Mb][H] (operand rows Mb..2Mb-1)
};

struct PLayer {
  PGemv dc, qkv, o, gu, dn;
  uint16_t *kc, *vc;
};

struct StepParams {
  int layers, Bk, Mb, H, D, V, R;
  float eps;
  const int32_t* block_tokens;
  const uint16_t* embed;
  PGemv fc;
  const uint16_t* fc_norm;
  const float* fcout;       // fc output [Mb][H]
  uint16_t* ctx;            // [Mb][H]
  const int32_t* n_new;
  PLayer L[DFLASH2_MAX_LAYERS];
  AttnParams ap;            // kc / vc set per layer
  uint16_t* ob;
  const uint8_t* head;      // prepared [lm_head; sel_proj]
  const uint16_t* final_norm;
  float* z;
  float* cand_val;          // [gridDim.x][D][16]
  int32_t* cand_id;
  float* cand_fval;         // merged [D][16]
  int32_t* cand_fid;
  float* tau;               // selector transition scores [D][16][16]
  SelParams sel;
  float* h;
  float* ssp;               // sums of squares of h: [H/128 column groups][4 quarters][Mb]
  unsigned* gbar;
  int* err;
  float* dbg_hidden;
  uint16_t* dbg_ctx;
  uint16_t* dbg_final_h;
};
static_assert(sizeof(StepParams) <= 32000, "step parameters must fit the kernel parameter space");

// ---------------------------------------------------------------------------- grid barrier
// Arrival counter in global memory, zeroed before the launch; epoch counts the barriers passed.
// Bounded wait: after kBarrierNs of wall time, or as soon as any CTA has flagged a timeout, the
// error bit is set and the CTA carries on (results are then garbage, but every CTA finishes
// quickly instead of timing out once per remaining barrier).
DEVI unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

DEVI void grid_sync(unsigned* gbar, unsigned& epoch, int* err) {
  consumers_sync<kPNC>();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned target = (epoch + 1) * gridDim.x;
    atomicAdd(gbar, 1u);
    bool ok = false;
    const unsigned long long t0 = global_ns();
    for (long long i = 0; i < kBarrierSpin; ++i) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(gbar) : "memory");
      if (v >= target) {
        ok = true;
        break;
      }
      if ((i & 255) == 255 &&
          ((*(volatile int*)err & DFLASH2_DEV_TIMEOUT) || global_ns() - t0 > kBarrierNs))
        break;
      __nanosleep(32);
    }
    if (!ok) set_err(err, DFLASH2_DEV_TIMEOUT);
    __threadfence();
  }
  ++epoch;
  consumers_sync<kPNC>();
}

// ---------------------------------------------------------------------------- work split
// This CTA's share [x0, x1) of a product's W = groups * U units (contiguous, stream-K order).
DEVI void pg_range(const PGemv& pg, long long& x0, long long& x1) {
  const long long P = pg.P, c = blockIdx.x, W = pg.g.W;
  x0 = c < P ? c * W / P : 0;
  x1 = c < P ? (c + 1) * W / P : 0;
}

// Stage the whole K once when this CTA's share covers at least one full group and K fits the
// staging area; otherwise stage per chunk of kc_units (only the K range of its own units).
DEVI bool pg_whole(const PGemv& pg, long long x0, long long x1) {
  return pg.g.kc_units >= pg.g.U && x1 - x0 >= pg.g.U;
}

// ---------------------------------------------------------------------------- producer
struct PRing {
  uint8_t* ring;
  uint64_t *full, *empty;
};

DEVI bool produce_slot(const PRing& r, int& cnt, const uint8_t* src, int bytes, int* err) {
  const int slot = cnt % kPNS, round = cnt / kPNS;
  if (round > 0 && !mbar_wait_bounded(&r.empty[slot], (round - 1) & 1)) {
    set_err(err, DFLASH2_DEV_TIMEOUT);
    return false;
  }
  mbar_expect_tx(&r.full[slot], bytes);
  bulk_g2s(r.ring + slot * kPSlot, src, bytes, &r.full[slot]);
  ++cnt;
  return true;
}

// Same slot sequence as consume_gemv: per group segment, per staging chunk, up to 2 units a slot.
DEVI bool produce_gemv(const PGemv& pg, const PRing& r, int& cnt, int* err) {
  const SGemvParams& p = pg.g;
  const int rec = pg.q4 ? kQ4Bytes * 8 : 2048 * 8;
  long long x0, x1;
  pg_range(pg, x0, x1);
  const int kc = pg_whole(pg, x0, x1) ? p.U : p.kc_units;
  for (long long x = x0; x < x1;) {
    const int gidx = (int)(x / p.U), ua = (int)(x % p.U);
    const int ub = (int)((x1 - x) < (long long)(p.U - ua) ? ua + (x1 - x) : p.U);
    const int grp = gidx % p.groups;
    const uint8_t* src = pg.q4 ? sk_group_src<true>(p, grp) : sk_group_src<false>(p, grp);
    for (int c0 = ua; c0 < ub; c0 += kc) {
      const int cu = (ub - c0) < kc ? (ub - c0) : kc;
      for (int k = 0; k < cu; k += kPUnits) {
        const int n = (cu - k) < kPUnits ? (cu - k) : kPUnits;
        if (!produce_slot(r, cnt, src + (size_t)(c0 + k) * rec, n * rec, err)) return false;
      }
    }
    x += ub - ua;
  }
  return true;
}

// Output head records (16 tiles x one 64-wide step = 32 KB) of this CTA: rec = c, c + P, ...
DEVI bool produce_head(const StepParams& S, const PRing& r, int& cnt) {
  const int total = S.V / 16 + S.R / 16, nrec = (total + kHeadTiles - 1) / kHeadTiles, St = S.H / 64;
  const int P = gridDim.x, c = blockIdx.x;
  for (int rec = c; rec < nrec; rec += P)
    for (int s = 0; s < St; ++s)
      if (!produce_slot(r, cnt, S.head + ((size_t)rec * St + s) * kHeadSlot, kHeadSlot, S.err)) return false;
  return true;
}

// ---------------------------------------------------------------------------- consumers
struct PState {
  uint8_t* ring;
  uint64_t *full, *empty, *xbar, *abar;
  uint8_t* Xs;      // kPXBytes
  float2* coef;     // [16 warps][128]
  float* red;       // [8][32][8]
  float* rs;        // [16] row scales
  float* wsh;       // [16 warps][64] attention-combine weights
  int* row_ok;      // [64]
  int cnt;
  uint32_t xph, aph;
  bool dead;
};

// Wait for ring position st.cnt (every consumer warp takes every slot); false after a timeout.
DEVI bool slot_wait(PState& st, int& slot, int* err) {
  slot = st.cnt % kPNS;
  const uint32_t par = (st.cnt / kPNS) & 1;
  ++st.cnt;
  if (!st.dead && !mbar_wait_sleep_bounded(&st.full[slot], par)) {
    set_err(err, DFLASH2_DEV_TIMEOUT);
    st.dead = true;
  }
  return !st.dead;
}

// rs[r] = 1/sqrt(mean(h[r]^2) + eps) for rows r < nrows, from the quarter-column sums of squares
// the residual epilogues (and the embedding) left in S.ssp.  Warp r handles row r.
DEVI void rs_from_ssp(const StepParams& S, int nrows, PState& st) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nq = (S.H >> 7) * 4;
  if (warp < nrows) {
    float s = 0.f;
    for (int i = lane; i < nq; i += 32) s += __ldcg(S.ssp + (size_t)i * S.Mb + warp);
    s = warp_sum(s);
    if (lane == 0) st.rs[warp] = rsqrtf(s / S.H + S.eps);
  }
  consumers_sync<kPNC>();
}

// Activation columns [k0, k0 + ncols) of rows [0, R) into Xs, computed from h (stage != COPY):
// x = h * rs * w (RMSNorm), and for STG_DYNCONV y_t = (s0 + tanh g0) x_t + (s1 + tanh g1) x_{t-1}
// for the block rows followed by the context rows.  Loads are issued in batches of kB items per
// thread before any use, so the L2 round trips overlap.
template <int R>
__device__ __noinline__ void stage_computed(const PGemv& pg, const StepParams& S, int k0, int ncols, int stride, PState& st) {
  constexpr int kB = 2;
  consumers_sync<kPNC>();  // previous chunk consumed
  const int H = S.H, G = H / 4, n4 = ncols / 4, total = R * n4;
  const bool dyn = pg.stage == STG_DYNCONV;
  const int nrows = dyn ? 2 * S.Mb : S.Mb;
  for (int i0 = threadIdx.x; i0 < total; i0 += kB * kPNC) {
    float4 hv[kB], hp[kB];
    uint2 wv[kB], cx[kB];
    float g0[kB], g1[kB];
#pragma unroll
    for (int b = 0; b < kB; ++b) {
      const int i = i0 + b * kPNC, r = i / n4, c = k0 + (i % n4) * 4;
      hv[b] = hp[b] = make_float4(0.f, 0.f, 0.f, 0.f);
      wv[b] = cx[b] = make_uint2(0, 0);
      g0[b] = g1[b] = 0.f;
      if (i < total && r < nrows) {
        if (dyn && r >= S.Mb) {
          cx[b] = __ldcg(reinterpret_cast<const uint2*>(pg.ctx + (size_t)(r - S.Mb) * H + c));
        } else {
          wv[b] = __ldg(reinterpret_cast<const uint2*>(pg.nw + c));
          hv[b] = __ldcg(reinterpret_cast<const float4*>(S.h + (size_t)r * H + c));
          if (dyn) {
            g0[b] = __ldcg(pg.gdc + (size_t)r * (H / 2) + c / 4);
            g1[b] = __ldcg(pg.gdc + (size_t)r * (H / 2) + G + c / 4);
            if (r % S.Bk > 0) hp[b] = __ldcg(reinterpret_cast<const float4*>(S.h + (size_t)(r - 1) * H + c));
          }
        }
      }
    }
#pragma unroll
    for (int b = 0; b < kB; ++b) {
      const int i = i0 + b * kPNC, r = i / n4, c = k0 + (i % n4) * 4;
      if (i >= total) break;
      uint2 out = cx[b];
      if (r < nrows && !(dyn && r >= S.Mb)) {
        const float w0 = bf2f(wv[b].x & 0xffff), w1 = bf2f(wv[b].x >> 16), w2 = bf2f(wv[b].y & 0xffff),
                    w3 = bf2f(wv[b].y >> 16);
        const float rs = st.rs[r];
        float x0 = hv[b].x * rs * w0, x1 = hv[b].y * rs * w1, x2 = hv[b].z * rs * w2, x3 = hv[b].w * rs * w3;
        if (dyn) {
          const float a0 = tanhf(g0[b]), a1 = tanhf(g1[b]);
          const float rp = r % S.Bk > 0 ? st.rs[r - 1] : 0.f;
          const float p0 = hp[b].x * rp * w0, p1 = hp[b].y * rp * w1, p2 = hp[b].z * rp * w2, p3 = hp[b].w * rp * w3;
          const uint2 a = __ldg(reinterpret_cast<const uint2*>(pg.s0 + c));
          const uint2 e = __ldg(reinterpret_cast<const uint2*>(pg.s1 + c));
          x0 = (bf2f(a.x & 0xffff) + a0) * x0 + (bf2f(e.x & 0xffff) + a1) * p0;
          x1 = (bf2f(a.x >> 16) + a0) * x1 + (bf2f(e.x >> 16) + a1) * p1;
          x2 = (bf2f(a.y & 0xffff) + a0) * x2 + (bf2f(e.y & 0xffff) + a1) * p2;
          x3 = (bf2f(a.y >> 16) + a0) * x3 + (bf2f(e.y >> 16) + a1) * p3;
        }
        out = make_uint2(pack_bf2(x0, x1), pack_bf2(x2, x3));
      }
      *reinterpret_cast<uint2*>(st.Xs + r * stride + (c - k0) * 2) = out;
    }
  }
  consumers_sync<kPNC>();
}

// Split-K epilogue of one column group (outlined: it runs once per group, off the hot loop).
__device__ __noinline__ void fixup_group(const SGemvParams& p, int grp, int R, int npieces) {
  sk_fixup(p, grp, 0, R, npieces);
}

// One streamed product (the phase functions are outlined so that each gets the whole register
// budget of the kernel; Q4 is a template parameter so each instance carries one decode path).
template <int NT, bool Q4>
__device__ __noinline__ void consume_gemv_t(const PGemv& pg, const StepParams& S, PState& st) {
  const SGemvParams& p = pg.g;
  constexpr int R = NT * 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int half = warp >> 3, wt = warp & 7;  // unit of the slot, tile of the group
  constexpr int unitK = Q4 ? 256 : 64, unitB = Q4 ? kQ4Bytes : 2048, rec = unitB * 8;
  const int stride = p.kc_units * unitK * 2 + 64;
  long long x0, x1;
  pg_range(pg, x0, x1);
  const bool whole = pg_whole(pg, x0, x1);
  const int kc = whole ? p.U : p.kc_units;
  const long long P = pg.P, c = blockIdx.x;
  __shared__ int s_last;
  if (pg.stage != STG_COPY && x1 > x0) rs_from_ssp(S, S.Mb, st);
  float2* coef = st.coef + warp * 128;
  bool staged = false;
  for (long long x = x0; x < x1;) {
    const int gidx = (int)(x / p.U), ua = (int)(x % p.U);
    const int ub = (int)((x1 - x) < (long long)(p.U - ua) ? ua + (x1 - x) : p.U);
    const int grp = gidx % p.groups;
    int si;
    const int tile = sk_tile(p, grp, wt, si);
    const int my_rows = sk_rows(p, si, 0, R);
    const int ntact = (my_rows + 7) >> 3;
    const int stage_rows = p.rows > R ? R : p.rows;
    float acc[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    for (int c0 = ua; c0 < ub; c0 += kc) {
      const int cu = (ub - c0) < kc ? (ub - c0) : kc;
      const int base = whole ? 0 : c0;
      if (!whole || !staged) {
        const int k0 = base * unitK, nk = (whole ? p.U : cu) * unitK;
        if (pg.stage == STG_COPY) {
          if (threadIdx.x == 0) fence_proxy_async();
          stage_x_chunk<kPNC>(p.X + k0, p.ldx, stage_rows, R, nk * 2, st.Xs, stride, st.xbar, st.xph, p.err);
        } else {
          stage_computed<R>(pg, S, k0, nk, stride, st);
        }
        staged = true;
      }
      for (int k = 0; k < cu; k += kPUnits) {
        int slot;
        if (!slot_wait(st, slot, p.err)) continue;
        const int u = c0 + k + half;
        const bool have = k + half < cu;
        const uint8_t* sb = st.ring + slot * kPSlot + half * rec + wt * unitB;
        if (Q4) {
          const uint4 z4 = make_uint4(0, 0, 0, 0);
          uint4 q[4] = {z4, z4, z4, z4}, sc = z4;
          if (have) {
#pragma unroll
            for (int i = 0; i < 4; ++i) q[i] = lds_slot(sb + (i * 32 + lane) * 16);
            sc = lds_slot(sb + 2048 + (lane >> 1) * 16);
          }
          if (have && ntact > 0) q4_unit<NT>(q, sc, coef, st.Xs, stride, (u - base) * 512, ntact, acc, lane);
          slot_release(&st.empty[slot], q[0].x ^ q[1].x ^ q[2].x ^ q[3].x ^ sc.x, lane);
        } else {
          uint4 wv[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
          if (have) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              wv[2 * j] = lds_slot(sb + j * 1024 + lane * 16);
              wv[2 * j + 1] = lds_slot(sb + j * 1024 + 512 + lane * 16);
            }
          }
          if (have && ntact > 0) bf16_step<NT, 2>(wv, st.Xs, stride, (u - base) * 128, ntact, acc, lane);
          slot_release(&st.empty[slot], wv[0].x ^ wv[1].x ^ wv[2].x ^ wv[3].x, lane);
        }
      }
    }
    // the two halves' accumulators meet in shared memory; half 0 writes the piece's partial
    if (ntact > 0 && half == 1) {
      float* rd = st.red + (wt * 32 + lane) * 8;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) rd[nt * 4 + e] = acc[nt][e];
    }
    consumers_sync<kPNC>();
    const long long gstart = (long long)gidx * p.U;
    const long long first = sk_owner(gstart, p.W, P);
    const int piece = (int)(c - first);
    const int npieces = (int)(sk_owner(gstart + p.U - 1, p.W, P) - first + 1);
    if (ntact > 0 && half == 0) {
      const float* rd = st.red + (wt * 32 + lane) * 8;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] += rd[nt * 4 + e];
      float* out = p.part + (size_t)piece * p.piece_stride;
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
    consumers_sync<kPNC>();
    if (threadIdx.x == 0) {
      const int prev = ticket_acq_rel(p.counters + gidx);
      s_last = prev == npieces - 1;
      if (s_last) p.counters[gidx] = 0;
    }
    consumers_sync<kPNC>();
    if (s_last && ntact > 0) fixup_group(p, grp, R, npieces);
    x += ub - ua;
  }
}

template <int NT>
DEVI void consume_gemv(const PGemv& pg, const StepParams& S, PState& st) {
  if (pg.q4) consume_gemv_t<NT, true>(pg, S, st);
  else consume_gemv_t<NT, false>(pg, S, st);
}

// Final-normed rows 1..D of the block -> Xs rows 0..D-1 (rows D..7 zero), batched loads.
DEVI void stage_final_rows(const StepParams& S, int stride, PState& st) {
  constexpr int kB = 4;
  const int H = S.H, n4 = H / 4, total = 8 * n4, D = S.D, c = blockIdx.x;
  for (int i0 = threadIdx.x; i0 < total; i0 += kB * kPNC) {
    float4 hv[kB];
    uint2 wv[kB];
#pragma unroll
    for (int b = 0; b < kB; ++b) {
      const int i = i0 + b * kPNC, r = i / n4, cc = (i % n4) * 4;
      hv[b] = make_float4(0.f, 0.f, 0.f, 0.f);
      wv[b] = make_uint2(0, 0);
      if (i < total && r < D) {
        hv[b] = __ldcg(reinterpret_cast<const float4*>(S.h + (size_t)(r + 1) * H + cc));
        wv[b] = __ldg(reinterpret_cast<const uint2*>(S.final_norm + cc));
      }
    }
#pragma unroll
    for (int b = 0; b < kB; ++b) {
      const int i = i0 + b * kPNC, r = i / n4, cc = (i % n4) * 4;
      if (i >= total) break;
      uint2 out = make_uint2(0, 0);
      if (r < D) {
        const float rs = st.rs[r + 1];
        out = make_uint2(pack_bf2(hv[b].x * rs * bf2f(wv[b].x & 0xffff), hv[b].y * rs * bf2f(wv[b].x >> 16)),
                         pack_bf2(hv[b].z * rs * bf2f(wv[b].y & 0xffff), hv[b].w * rs * bf2f(wv[b].y >> 16)));
        if (S.dbg_final_h && c == 0) *reinterpret_cast<uint2*>(S.dbg_final_h + (size_t)r * H + cc) = out;
      }
      *reinterpret_cast<uint2*>(st.Xs + r * stride + cc * 2) = out;
    }
  }
}

// Output head + top-16 of the drafted rows; this CTA's lists -> cand_val/cand_id[blockIdx.x].
// Every consumer warp takes every slot (one 32 KB record step): warp (half, wt) owns tile
// 8 * half + wt of the record, then offers its logits to its own per-row lists.
__device__ __noinline__ void consume_head(const StepParams& S, PState& st) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int half = warp >> 3, wt = warp & 7;
  const int H = S.H, stride = H * 2 + 64, vt = S.V / 16, total = vt + S.R / 16;
  const int nrec = (total + kHeadTiles - 1) / kHeadTiles, St = H / 64, P = gridDim.x, c = blockIdx.x, D = S.D;
  uint2* lists = reinterpret_cast<uint2*>(st.coef);  // [16 warps][8 rows][16], in the scale-table region
  rs_from_ssp(S, S.Bk, st);
  stage_final_rows(S, stride, st);
  for (int i = threadIdx.x; i < kGemvConsumers * 8 * kTopK; i += kPNC)
    lists[i] = make_uint2(__float_as_uint(-INFINITY), 0x7fffffffu);
  consumers_sync<kPNC>();
  uint2* my = lists + warp * 8 * kTopK;
  for (int rec = c; rec < nrec; rec += P) {
    const int tile = rec * kHeadTiles + half * 8 + wt;
    float acc[1][4] = {{0.f, 0.f, 0.f, 0.f}};
    for (int s = 0; s < St; ++s) {
      int slot;
      if (!slot_wait(st, slot, S.err)) continue;
      const uint8_t* sb = st.ring + slot * kPSlot + (half * 8 + wt) * 2048;
      uint4 wv[4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        wv[2 * j] = lds_slot(sb + j * 1024 + lane * 16);
        wv[2 * j + 1] = lds_slot(sb + j * 1024 + 512 + lane * 16);
      }
      bf16_step<1, 2>(wv, st.Xs, stride, s * 128, 1, acc, lane);
      slot_release(&st.empty[slot], wv[0].x ^ wv[1].x ^ wv[2].x ^ wv[3].x, lane);
    }
    if (st.dead || tile >= total) continue;
    if (tile >= vt) {
      const int c0 = (tile - vt) * 16;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = 2 * t + (e & 1);
        if (r < D) S.z[(size_t)r * S.R + c0 + g + 8 * (e >> 1)] = acc[0][e];
      }
    } else {
      offer_tile(my, acc[0], tile * 16, D, lane);
    }
  }
  consumers_sync<kPNC>();
  merge_warp_lists(lists, D, S.cand_val, S.cand_id, c, warp, kGemvConsumers, lane);
}

// Context row c = RMSNorm(fc output row c; fc_norm), or zero past the request's new rows; one
// CTA, the row's loads issued together (kB float4 per consumer thread cover H <= 8192).
__device__ __noinline__ void ctx_row(const StepParams& S, int c, PState& st) {
  constexpr int kB = 4;
  const int H = S.H, n4 = H / 4, t = c % S.Bk, b = c / S.Bk;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint16_t* dst = S.ctx + (size_t)c * H;
  const bool live = t < S.n_new[b];
  const float4* src = reinterpret_cast<const float4*>(S.fcout + (size_t)c * H);
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 v[kB];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < kB; ++k) {
    const int i = threadIdx.x + k * kPNC;
    v[k] = (live && i < n4) ? __ldcg(src + i) : zero;
    ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
  }
  for (int i = threadIdx.x + kB * kPNC; i < n4; i += kPNC) {
    const float4 u = live ? __ldcg(src + i) : zero;
    ss += u.x * u.x + u.y * u.y + u.z * u.z + u.w * u.w;
  }
  ss = warp_sum(ss);
  if (lane == 0) st.red[warp] = ss;
  consumers_sync<kPNC>();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kGemvConsumers; ++w) tot += st.red[w];
  const float r = live ? rsqrtf(tot / H + S.eps) : 0.f;
  auto put = [&](int i, const float4& u) {
    const uint2 wv = __ldg(reinterpret_cast<const uint2*>(S.fc_norm + 4 * i));
    const uint2 o = make_uint2(pack_bf2(u.x * r * bf2f(wv.x & 0xffff), u.y * r * bf2f(wv.x >> 16)),
                               pack_bf2(u.z * r * bf2f(wv.y & 0xffff), u.w * r * bf2f(wv.y >> 16)));
    *reinterpret_cast<uint2*>(dst + 4 * i) = o;
    if (S.dbg_ctx) *reinterpret_cast<uint2*>(S.dbg_ctx + (size_t)c * H + 4 * i) = o;
  };
#pragma unroll
  for (int k = 0; k < kB; ++k) {
    const int i = threadIdx.x + k * kPNC;
    if (i < n4) put(i, v[k]);
  }
  for (int i = threadIdx.x + kB * kPNC; i < n4; i += kPNC) put(i, live ? __ldcg(src + i) : zero);
}

__global__ void __launch_bounds__(kPThreads, 1) k_step_persistent(const __grid_constant__ StepParams S) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[kPNS];
  __shared__ __align__(8) uint64_t empty[kPNS];
  __shared__ __align__(8) uint64_t xbar, abar;
  __shared__ float rs[16];
  __shared__ int row_ok[kAttnKeys];
  __shared__ int cand_s[2][kTopK];  // selector: candidates of rows t - 1 and t
  __shared__ float cl_s[2][kTopK];
  __shared__ int src_s[kTopK];
  __shared__ int sel_n[2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPNS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGemvConsumers);  // every consumer warp releases every slot
    }
    mbar_init(&xbar, 1);
    mbar_init(&abar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  PRing ring{smem, full, empty};

  if (warp == kGemvConsumers) {
    // ---- producer: the step's streamed matrices in order; never waits on a grid barrier ----
    if (lane != 0) return;
    int cnt = 0;
    if (!produce_gemv(S.fc, ring, cnt, S.err)) return;
    for (int l = 0; l < S.layers; ++l) {
      if (!produce_gemv(S.L[l].dc, ring, cnt, S.err)) return;
      if (!produce_gemv(S.L[l].qkv, ring, cnt, S.err)) return;
      if (!produce_gemv(S.L[l].o, ring, cnt, S.err)) return;
      if (!produce_gemv(S.L[l].gu, ring, cnt, S.err)) return;
      if (!produce_gemv(S.L[l].dn, ring, cnt, S.err)) return;
    }
    produce_head(S, ring, cnt);
    return;
  }

  PState st;
  st.ring = smem;
  st.full = full;
  st.empty = empty;
  st.xbar = &xbar;
  st.abar = &abar;
  st.Xs = smem + kPNS * kPSlot;
  st.coef = reinterpret_cast<float2*>(st.Xs + kPXBytes);
  st.red = reinterpret_cast<float*>(st.coef + kGemvConsumers * 128);
  st.wsh = st.red + kConsumers * 32 * 8;
  st.rs = rs;
  st.row_ok = row_ok;
  st.cnt = 0;
  st.xph = st.aph = 0;
  st.dead = false;
  unsigned epoch = 0;
  const int c = blockIdx.x, P = gridDim.x, H = S.H;

  // A1: block rows from the shared embedding table (CTA r: row r), with the row's quarter-column
  // sums of squares for the first RMSNorm
  if (c < S.Mb) {
    int id = S.block_tokens[c];
    if (id < 0 || id >= S.V) {
      if (threadIdx.x == 0) set_err(S.err, DFLASH2_DEV_TOKEN);
      id = 0;
    }
    const uint16_t* erow = S.embed + (size_t)id * H;
    const uint4* e = reinterpret_cast<const uint4*>(erow);
    for (int i = threadIdx.x; i < H / 8; i += kPNC) {
      const uint4 v = e[i];
      float4* o = reinterpret_cast<float4*>(S.h + (size_t)c * H + i * 8);
      o[0] = make_float4(bf2f(v.x & 0xffff), bf2f(v.x >> 16), bf2f(v.y & 0xffff), bf2f(v.y >> 16));
      o[1] = make_float4(bf2f(v.z & 0xffff), bf2f(v.z >> 16), bf2f(v.w & 0xffff), bf2f(v.w >> 16));
      if (S.dbg_hidden) {
        reinterpret_cast<float4*>(S.dbg_hidden + (size_t)c * H + i * 8)[0] = o[0];
        reinterpret_cast<float4*>(S.dbg_hidden + (size_t)c * H + i * 8)[1] = o[1];
      }
    }
    for (int q = warp; q < (H >> 7) * 4; q += kGemvConsumers) {
      const float v = bf2f(erow[q * 32 + lane]);
      const float s = warp_sum(v * v);
      if (lane == 0) S.ssp[(size_t)q * S.Mb + c] = s;
    }
  }
  // A2: fc over the taps, then its RMSNorm into the context rows (CTA r: row r)
  consume_gemv<1>(S.fc, S, st);
  grid_sync(S.gbar, epoch, S.err);
  if (c < S.Mb) ctx_row(S, c, st);
  grid_sync(S.gbar, epoch, S.err);

  for (int l = 0; l < S.layers; ++l) {
    const PLayer& L = S.L[l];
    consume_gemv<1>(L.dc, S, st);  // x = RMSNorm(h; ln1) staged in place; g = W_dc x
    grid_sync(S.gbar, epoch, S.err);
    consume_gemv<2>(L.qkv, S, st);  // y = dynconv(x, g) and context rows; q/k norm, RoPE, append
    grid_sync(S.gbar, epoch, S.err);
    {
      AttnParams ap = S.ap;
      ap.kc = L.kc;
      ap.vc = L.vc;
      const int nitems = ap.nkv * (ap.NC + 1);
      for (int it = c; it < nitems; it += P) attn_item<2, kPNC>(ap, it % (ap.NC + 1), it / (ap.NC + 1), 0, st.Xs, st.row_ok);
      grid_sync(S.gbar, epoch, S.err);
      const int G = ap.nq / ap.nkv, nw = ap.nkv * G * ap.Bk;
      for (int it = c * kGemvConsumers + warp; it < nw; it += P * kGemvConsumers)
        attn_combine_warp(ap, S.ob, it % (G * ap.Bk), it / (G * ap.Bk), 0, st.wsh + warp * 64);
    }
    grid_sync(S.gbar, epoch, S.err);
    consume_gemv<1>(L.o, S, st);  // h += W_o o
    grid_sync(S.gbar, epoch, S.err);
    consume_gemv<1>(L.gu, S, st);  // x2 = RMSNorm(h; ln2) staged in place; SwiGLU in the epilogue
    grid_sync(S.gbar, epoch, S.err);
    consume_gemv<1>(L.dn, S, st);  // h += W_d act
    grid_sync(S.gbar, epoch, S.err);
    if (S.dbg_hidden && c < S.Mb)
      for (int i = threadIdx.x; i < H / 4; i += kPNC)
        reinterpret_cast<float4*>(S.dbg_hidden + ((size_t)(l + 1) * S.Mb + c) * H)[i] =
            __ldcg(reinterpret_cast<const float4*>(S.h + (size_t)c * H) + i);
  }
  consume_head(S, st);
  grid_sync(S.gbar, epoch, S.err);
  // A6: CTA t < D: final candidates of rows t and t - 1, then the transition scores tau_t
  if (c < S.D) {
    const int t = c;
    float* sv = reinterpret_cast<float*>(st.Xs) + warp * 1024;
    int* si = reinterpret_cast<int*>(st.Xs) + warp * 1024 + 512;
    if (warp == 0 || (warp == 1 && t > 0)) selector_row(S.sel, t - warp, sv, si, &sel_n[warp], cl_s[1 - warp], cand_s[1 - warp]);
    consumers_sync<kPNC>();
    if (threadIdx.x < kTopK) {
      S.cand_fval[t * kTopK + threadIdx.x] = cl_s[1][threadIdx.x];
      S.cand_fid[t * kTopK + threadIdx.x] = cand_s[1][threadIdx.x];
      if (S.sel.dbg_cand) {
        S.sel.dbg_cand[t * kTopK + threadIdx.x] = cand_s[1][threadIdx.x];
        S.sel.dbg_logit[t * kTopK + threadIdx.x] = cl_s[1][threadIdx.x];
      }
      if (t == 0) {
        if (threadIdx.x == 0) {
          const int a = S.block_tokens[0];
          src_s[0] = (a < 0 || a >= S.V) ? 0 : a;
        }
      } else {
        src_s[threadIdx.x] = cand_s[0][threadIdx.x];
      }
    }
    consumers_sync<kPNC>();
    float(*As)[kMaxR] = reinterpret_cast<float(*)[kMaxR]>(st.Xs + 8192);
    float(*Wj)[kTopK] = reinterpret_cast<float(*)[kTopK]>(st.Xs + 8192 + kTopK * kMaxR * 4);
    selector_tau<kPNC>(S.sel, 0, t, src_s, t == 0 ? 1 : kTopK, cand_s[1], As, Wj, S.tau + (size_t)t * kTopK * kTopK);
  }
  grid_sync(S.gbar, epoch, S.err);
  if (c == 0 && warp == 0) selector_viterbi(S.sel, 0, S.cand_fval, S.cand_fid, S.tau);
}

}  // namespace dfl
