// Batched layer products on the 5th-generation tensor cores (tcgen05 / TMEM).
//
// When the step carries many block rows (many requests), a layer product is a dense
// contraction: Y[row][feature] = sum_k X[row][k] W[feature][k] with a few hundred rows.  The
// streaming mma.sync engine (stream.cuh) re-reads its activation fragments from shared memory
// for every weight fragment, so there it is bound by shared-memory operand traffic; this kernel
// feeds the tensor cores from shared-memory descriptors instead and accumulates in TMEM.
//
// One CTA per SM (stream-K over the same (column group, row chunk, K unit) plane as the
// streaming engine, so the split-K pieces, their order and the fix-up epilogues are shared):
//  * warp 0, one thread: TMA (cp.async.bulk.tensor, no multicast) of the activation tile
//    [256 rows][64 k] bf16 into a 128-byte-swizzled K-major stage;
//  * warps 4-7: weight producers.  They read the prepared records of the column group (128
//    features = 8 tiles of 16, the layout of dflash2_prepare_weights) straight from global
//    memory and write the [128 features][64 k] bf16 operand into the same swizzled K-major
//    layout.  Q4_K codes become bf16 128+q with one LOP3 (0x4300 | q), widen exactly to fp32,
//    and w = (128+q) * (d sc_j) - (dmin m_j + 128 d sc_j) is formed by a packed fp32 fused
//    multiply-add and rounded once to bf16 (the only rounding of a weight; rounding the
//    sub-block scale or min to bf16 first would bias all 32 weights of a sub-block alike);
//    bf16 weights are moved as they are.  After the K range of a
//    piece they read the accumulator back (tcgen05.ld) and store the fp32 partial;
//  * warp 1: allocates 256 TMEM columns; one thread issues tcgen05.mma (kind::f16, bf16 x bf16
//    -> fp32, M = 128 features, N = 256 rows, K = 16) and commits each stage back to the
//    producers and each finished piece to the epilogue.
// Every mbarrier wait is bounded; an expired wait sets DFLASH2_DEV_TIMEOUT and the waiting role
// skips its remaining work, so the CTA still exits and frees its TMEM.
#pragma once
#include <cuda.h>

#include "stream.cuh"

namespace dfl {

constexpr int kUmmaRows = 256;                     // activation rows per tile (MMA N)
constexpr int kUmmaStages = 3;                     // operand stages (64-wide K)
constexpr int kUmmaRaw = 3;                        // raw weight-record slots (one prepared K unit each)
constexpr int kUmmaABytes = 128 * 128;             // [128 features][64 k] bf16
constexpr int kUmmaBBytes = kUmmaRows * 128;       // [256 rows][64 k] bf16
constexpr int kUmmaRawBytes = 8 * kQ4Bytes;        // one group unit (Q4_K 18 KB; bf16 units are 16 KB)
constexpr int kUmmaDq = 16;                        // weight-operand warps (a tile's 32-wide half each)
constexpr int kUmmaThreads = (4 + kUmmaDq + 4) * 32; // roles below
constexpr int kUHeadThreads = 16 * 32;               // the output head's roles
constexpr int kUmmaSmem = kUmmaStages * (kUmmaABytes + kUmmaBBytes) + kUmmaRaw * kUmmaRawBytes + 1024;
constexpr int kUmmaPairSmem = 2 * (kUmmaABytes + 2 * kUmmaBBytes) + kUmmaRaw * kUmmaRawBytes + 1024;
constexpr int kUmmaTmemCols = 512;                 // two 256-column accumulators

// ---- tcgen05 / TMA wrappers (one instruction each) ----
DEVI void tmem_alloc(uint32_t* dst_smem, int cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(cols)
               : "memory");
}
DEVI void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
DEVI void tmem_dealloc(uint32_t taddr, int cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
DEVI void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
DEVI void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
DEVI void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 inputs, fp32 accumulate)
DEVI void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane (warp w reads lanes 32*(w%4) ..)
DEVI void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
DEVI void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Generic-proxy shared-memory writes made visible to the async proxy (the tensor cores).
DEVI void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// 2-D tiled TMA load (no multicast): box at (x elements along K, y rows) of the tensor map.
DEVI void tma_load_2d(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor of a K-major operand stored as 8-row x 128-byte swizzled atoms
// (rows 128 bytes apart, 8-row groups 1024 bytes apart): start address, leading offset 16 B,
// stride offset 1024 B, descriptor version 1, layout SWIZZLE_128B.
DEVI uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
         ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
// Instruction descriptor: fp32 accumulator, bf16 A and B, both K-major, M = 128, N = n (a multiple
// of 16 up to 256).
DEVI constexpr uint32_t umma_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
constexpr uint32_t kUmmaIdesc = umma_idesc(kUmmaRows);

// Byte offset of the 16-byte chunk c (k = 8c .. 8c+7) of row m in a 128-byte-swizzled stage.
DEVI uint32_t sw128_off(int m, int c) { return (uint32_t)(m * 128 + ((c ^ (m & 7)) << 4)); }

DEVI bool wait_or_die(uint64_t* bar, uint32_t parity, bool& dead, int* err) {
  if (dead) return false;
  if (!mbar_wait_bounded(bar, parity)) {
    set_err(err, DFLASH2_DEV_TIMEOUT);
    dead = true;
    return false;
  }
  return true;
}

// (D, C) of sub-block j from a canonical 16-byte Q4_K scale record: D = d*sc_j and
// C = -(dmin*m_j + 128*D), so that w = (128 + q)*D + C.  d*sc_j and dmin*m_j are exact in fp32
// (an fp16 times a 6-bit integer); C carries one fp32 rounding, 2^-17 of a quantisation step.
DEVI float2 q4_scale_dc(const uint4 sc, int j) {
  const float d = __half2float(__ushort_as_half((unsigned short)(sc.x & 0xffffu)));
  const float dm = __half2float(__ushort_as_half((unsigned short)(sc.x >> 16)));
  const unsigned long long scp = (unsigned long long)sc.y | ((unsigned long long)(sc.z & 0xffffu) << 32);
  const unsigned long long mp = (unsigned long long)(sc.z >> 16) | ((unsigned long long)sc.w << 16);
  const float D = d * (float)((scp >> (6 * j)) & 63u), M = dm * (float)((mp >> (6 * j)) & 63u);
  return make_float2(D, -fmaf(128.f, D, M));
}

// bf16 pair (128 + q0, 128 + q1) -> the two weights in fp32 (exact widening, one fused
// multiply-add each on the packed pair), rounded once to a bf16 pair.
DEVI uint32_t q4_pair(uint32_t v, float2 dc) {
  const float2 x = make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
  const float2 w = ffma2(x, make_float2(dc.x, dc.x), make_float2(dc.y, dc.y));
  return pack_bf2(w.x, w.y);
}

// One row's 8 consecutive weights from two code words (nibble slots of the prepared record: word
// bits 4s hold slot s; row g takes slots 0,4 | 2,6 with shifts 0 | 8, row g+8 the same with an
// extra shift of 4), dequantised to 4 bf16 pairs.
DEVI uint4 q4_chunk(uint32_t w0, uint32_t w1, int rs, float2 dc) {
  const uint32_t k128 = 0x43004300u;  // bf16 pair (128, 128)
  const uint32_t a = ((w0 >> rs) & 0x000F000Fu) | k128, b = ((w0 >> (rs + 8)) & 0x000F000Fu) | k128;
  const uint32_t c = ((w1 >> rs) & 0x000F000Fu) | k128, d = ((w1 >> (rs + 8)) & 0x000F000Fu) | k128;
  return make_uint4(q4_pair(a, dc), q4_pair(b, dc), q4_pair(c, dc), q4_pair(d, dc));
}

// Row scales 1/sqrt(mean(h^2) + eps) of rows [r0, r1) from quarter-column sums of squares
// (layout [H/128][4][ldr]) into rs[row]; one warp.
DEVI void rows_scale_global(const float* ssp, int ldr, int H, float eps, int r0, int r1, float* rs) {
  const int lane = threadIdx.x & 31, nq = (H >> 7) * 4;
  for (int r = r0; r < r1; ++r) {
    float q = 0.f;
    for (int i = lane; i < nq; i += 32) q += __ldcg(ssp + (size_t)i * ldr + r);
    q = warp_sum(q);
    if (lane == 0) rs[r] = rsqrtf(q / H + eps);
  }
}

// Roles (24 warps): warp 0 one thread: activation TMA; warp 1: TMEM allocation, one thread issues
// the MMAs; warp 2 one thread: raw weight records into the raw ring (bulk copies, started before
// the dependency wait: the weights do not depend on earlier kernels); warp 3: the row scales of
// a folded RMSNorm for the fix-up (p.rs_glob); warps 4-19: the weight operand from the raw ring,
// one 32-wide half of one 16-feature tile each (four warps per SM sub-partition, so their
// latencies hide behind one another's work: the dequantisation's dependent chains bounded the
// kernel with one or two per sub-partition); warps 20-23: epilogue (TMEM lane = operand row), on
// two accumulators alternating by piece, or (PAIR) on the two halves of each piece in turn.
template <bool Q4, bool PAIR>
__global__ void __launch_bounds__(kUmmaThreads, 1) k_umma(const __grid_constant__ CUtensorMap tmx, SGemvParams p) {
  // PAIR: a tile is two 256-row halves sharing each weight stage (the operand is dequantised once
  // for both), accumulated in all 512 TMEM columns; two stages of 80 KB instead of three of 48 KB
  constexpr int NS = PAIR ? 2 : kUmmaStages;
  constexpr int BST = PAIR ? 2 * kUmmaBBytes : kUmmaBBytes;
  constexpr int MROWS = PAIR ? 2 * kUmmaRows : kUmmaRows;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t xfull[NS], afull[NS], sempty[NS];
  __shared__ __align__(8) uint64_t rfull[kUmmaRaw], rempty[kUmmaRaw];
  __shared__ __align__(8) uint64_t accfull[2], accempty[2];
  __shared__ uint32_t tmem_base_sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* As = smem;                    // [NS][128 x 128 B]
  uint8_t* Bs = As + NS * kUmmaABytes;   // [NS][1 or 2 halves][256 x 128 B]
  uint8_t* Rs = Bs + NS * BST;           // [raw slots][group unit]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kSub = Q4 ? 4 : 1;  // 64-wide stages per prepared K unit
  constexpr int kUnitK = Q4 ? 256 : 64;
  constexpr int kRawUnit = Ring<Q4>::kSlot;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&afull[s], kUmmaDq);
      mbar_init(&sempty[s], 1);
    }
    for (int r = 0; r < kUmmaRaw; ++r) {
      mbar_init(&rfull[r], 1);
      mbar_init(&rempty[r], kUmmaDq);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kUmmaTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  pdl_trigger();
  const long long P = gridDim.x, c = blockIdx.x;
  const long long x0 = c * p.W / P, x1 = (c + 1) * p.W / P;

  if (warp == 0) {
    // ---- activation producer (TMA) ----
    if (lane == 0) {
      pdl_wait();  // the activations come from the previous kernel
      bool dead = false;
      int cnt = 0;
      for (long long x = x0; x < x1 && !dead;) {
        const int gidx = (int)(x / p.U), ua = (int)(x % p.U);
        const int ub = (int)((x1 - x) < (long long)(p.U - ua) ? ua + (x1 - x) : p.U);
        const int grp = gidx % p.groups, mz = (gidx / p.groups) * MROWS;
        int si;
        sk_tile(p, grp, 0, si);
        if (sk_rows(p, si, mz, MROWS) > 0) {
          const bool h2 = PAIR && sk_rows(p, si, mz + kUmmaRows, kUmmaRows) > 0;  // second half rows
          for (int u = ua; u < ub && !dead; ++u)
            for (int sub = 0; sub < kSub && !dead; ++sub, ++cnt) {
              const int s = cnt % NS, round = cnt / NS;
              if (round > 0 && !wait_or_die(&sempty[s], (round - 1) & 1, dead, p.err)) break;
              mbar_expect_tx(&xfull[s], (uint32_t)p.un * 128u * (h2 ? 2u : 1u));  // boxes: un rows of 64 k
              tma_load_2d(Bs + s * BST, &tmx, u * kUnitK + sub * 64, mz, &xfull[s]);
              if (h2) tma_load_2d(Bs + s * BST + kUmmaBBytes, &tmx, u * kUnitK + sub * 64, mz + kUmmaRows, &xfull[s]);
            }
        }
        x += ub - ua;
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      bool dead = false;
      int cnt = 0, piece = 0;
      for (long long x = x0; x < x1 && !dead;) {
        const int gidx = (int)(x / p.U), ua = (int)(x % p.U);
        const int ub = (int)((x1 - x) < (long long)(p.U - ua) ? ua + (x1 - x) : p.U);
        const int grp = gidx % p.groups, mz = (gidx / p.groups) * MROWS;
        int si;
        sk_tile(p, grp, 0, si);
        if (sk_rows(p, si, mz, MROWS) > 0) {
          const bool h2 = PAIR && sk_rows(p, si, mz + kUmmaRows, kUmmaRows) > 0;
          // a pair tile fills all 512 columns, so its pieces take turns with the epilogue
          const int buf = PAIR ? 0 : piece & 1, use = PAIR ? piece : piece >> 1;
          if (use > 0 && !wait_or_die(&accempty[buf], (use - 1) & 1, dead, p.err)) break;
          tc_fence_after();
          const uint32_t acc = tmem + (uint32_t)(buf * kUmmaRows);
          const uint32_t idesc = umma_idesc(p.un);  // N = the tile's rows
          bool first = true;
          for (int u = ua; u < ub && !dead; ++u)
            for (int sub = 0; sub < kSub && !dead; ++sub, ++cnt) {
              const int s = cnt % NS;
              const uint32_t par = (cnt / NS) & 1;
              if (!wait_or_die(&xfull[s], par, dead, p.err) || !wait_or_die(&afull[s], par, dead, p.err)) break;
              tc_fence_after();
              const uint64_t ad = sw128_desc(smem_u32(As + s * kUmmaABytes));
              const uint64_t bd = sw128_desc(smem_u32(Bs + s * BST));
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {  // 16-wide K slices: +32 bytes inside the swizzled rows
                tc_mma(acc, ad + 2 * kk, bd + 2 * kk, idesc, (first && kk == 0) ? 0u : 1u);
                if (h2)  // the second half: the same weights, rows 256 on, accumulator columns 256 on
                  tc_mma(acc + (uint32_t)kUmmaRows, ad + 2 * kk, bd + (uint64_t)(kUmmaBBytes >> 4) + 2 * kk, idesc,
                         (first && kk == 0) ? 0u : 1u);
              }
              first = false;
              tc_commit(&sempty[s]);  // the stage is free once these MMAs have read it
            }
          if (!dead) tc_commit(&accfull[buf]);  // the piece's accumulator is complete
          ++piece;
        }
        x += ub - ua;
      }
    }
  } else if (warp == 2) {
    // ---- raw weight records (bulk copies; before the dependency wait) ----
    if (lane == 0) {
      bool dead = false;
      int cnt = 0;
      for (long long x = x0; x < x1 && !dead;) {
        const int gidx = (int)(x / p.U), ua = (int)(x % p.U);
        const int ub = (int)((x1 - x) < (long long)(p.U - ua) ? ua + (x1 - x) : p.U);
        const int grp = gidx % p.groups, mz = (gidx / p.groups) * MROWS;
        int si;
        sk_tile(p, grp, 0, si);
        if (sk_rows(p, si, mz, MROWS) > 0) {
          const uint8_t* src = sk_group_src<Q4>(p, grp);
          for (int u = ua; u < ub && !dead; ++u, ++cnt) {
            const int r = cnt % kUmmaRaw, round = cnt / kUmmaRaw;
            if (round > 0 && !wait_or_die(&rempty[r], (round - 1) & 1, dead, p.err)) break;
            mbar_expect_tx(&rfull[r], kRawUnit);
            bulk_g2s(Rs + r * kUmmaRawBytes, src + (size_t)u * kRawUnit, kRawUnit, &rfull[r]);
          }
        }
        x += ub - ua;
      }
    }
  } else if (warp == 3) {
    // ---- row scales of a folded RMSNorm for the fix-up (rows split over the CTAs) ----
    if (p.rs_glob) {
      pdl_wait();  // the sums of squares come from the previous product's epilogue
      const int r0 = (int)(c * p.rows / P), r1 = (int)((c + 1) * p.rows / P);
      rows_scale_global(p.rs_in, p.ssp_rows, p.rs_H, p.eps, r0, r1, p.rs_glob);
    }
  } else if (warp < 4 + kUmmaDq) {
    // ---- weight operand: raw ring -> swizzled K-major stage (warp = one tile of the group) ----
    // warp = one 32-wide half jh of every 64-wide stage of tile tl
    const int tl = (warp - 4) % 8, jh = (warp - 4) / 8, g = lane >> 2, t = lane & 3;
    bool dead = false;
    int cnt = 0, ucnt = 0;
    for (long long x = x0; x < x1;) {
      const int gidx = (int)(x / p.U), ua = (int)(x % p.U);
      const int ub = (int)((x1 - x) < (long long)(p.U - ua) ? ua + (x1 - x) : p.U);
      const int grp = gidx % p.groups, mz = (gidx / p.groups) * MROWS;
      int si0;
      sk_tile(p, grp, 0, si0);
      if (sk_rows(p, si0, mz, MROWS) > 0) {
        for (int u = ua; u < ub; ++u, ++ucnt) {
          const int r = ucnt % kUmmaRaw;
          wait_or_die(&rfull[r], (ucnt / kUmmaRaw) & 1, dead, p.err);
          const uint8_t* raw = Rs + r * kUmmaRawBytes;
          // 4-bit records: this lane's scale records (rows g, g+8 of its tile), decoded once per
          // unit (Q4_K: d, dmin and the packed 6-bit fields; MLX: the record's four bf16 pairs)
          float dd[2], dm[2];
          unsigned long long scp[2], mp[2];
          uint4 mrec[2];
          if (Q4 && !dead) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const uint4 sc = *reinterpret_cast<const uint4*>(raw + tl * kQ4Bytes + 2048 + (g + 8 * e) * 16);
              mrec[e] = sc;
              dd[e] = __half2float(__ushort_as_half((unsigned short)(sc.x & 0xffffu)));
              dm[e] = __half2float(__ushort_as_half((unsigned short)(sc.x >> 16)));
              scp[e] = (unsigned long long)sc.y | ((unsigned long long)(sc.z & 0xffffu) << 32);
              mp[e] = (unsigned long long)(sc.z >> 16) | ((unsigned long long)sc.w << 16);
            }
          }
#pragma unroll
          for (int sub = 0; sub < kSub; ++sub, ++cnt) {
            const int s = cnt % NS, round = cnt / NS;
            uint8_t* a = As + s * kUmmaABytes;
            // features g and g + 8 of tile tl go to operand rows 16 tl + a8(g) and + 8: a8 puts the
            // two features of each 8-lane store phase 4 rows apart, so that the phase's 16-byte
            // chunks land in distinct swizzled bank groups (the epilogue maps TMEM lanes back)
            const int m0 = tl * 16 + ((g >> 1) | ((g & 1) << 2));
            // the operand values are formed from the raw unit first, so that only the stores wait
            // for the tensor cores to free the stage
            uint4 rg = make_uint4(0u, 0u, 0u, 0u), rh = rg;
            if (!dead) {
              const uint8_t* rec = raw + tl * (Q4 ? kQ4Bytes : 2048);
              {
                const int jj = jh;  // this warp's 32-wide sub-block of the stage
                if (Q4) {
                  const uint4 q = *reinterpret_cast<const uint4*>(rec + (sub * 32 + lane) * 16);
                  const uint32_t w0 = jj ? q.z : q.x, w1 = jj ? q.w : q.y;
                  const int j = 2 * sub + jj;
                  float2 dc[2];
#pragma unroll
                  for (int e = 0; e < 2; ++e) {
                    if (p.mlx) {  // group j/2: w = scale*q + bias = (128+q)*scale + (bias - 128*scale)
                      const uint4 r = mrec[e];
                      const uint32_t wg = (j >> 1) == 0 ? r.x : (j >> 1) == 1 ? r.y : (j >> 1) == 2 ? r.z : r.w;
                      const float D = bf2f((uint16_t)(wg & 0xffffu)), B = bf2f((uint16_t)(wg >> 16));
                      dc[e] = make_float2(D, fmaf(-128.f, D, B));
                    } else {
                      const float D = dd[e] * (float)((scp[e] >> (6 * j)) & 63u);
                      const float M = dm[e] * (float)((mp[e] >> (6 * j)) & 63u);
                      dc[e] = make_float2(D, -fmaf(128.f, D, M));
                    }
                  }
                  rg = q4_chunk(w0, w1, 0, dc[0]);
                  rh = q4_chunk(w0, w1, 4, dc[1]);
                } else {  // bf16 record: W[row g][32jj + 8t ..] at jj*1024 + lane*16, row g+8 at +512
                  rg = *reinterpret_cast<const uint4*>(rec + jj * 1024 + lane * 16);
                  rh = *reinterpret_cast<const uint4*>(rec + jj * 1024 + 512 + lane * 16);
                }
              }
            }
            if (round > 0) wait_or_die(&sempty[s], (round - 1) & 1, dead, p.err);
            if (!dead) {
              *reinterpret_cast<uint4*>(a + sw128_off(m0, 4 * jh + t)) = rg;
              *reinterpret_cast<uint4*>(a + sw128_off(m0 + 8, 4 * jh + t)) = rh;
            }
            fence_proxy_async_smem();  // these generic writes feed the tensor cores (async proxy)
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[s]);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&rempty[r]);  // the raw unit has been read
        }
      }
      x += ub - ua;
    }
  } else {
    // ---- epilogue: TMEM -> fp32 partial [piece][row][ldo], accumulators alternate by piece ----
    const int ew = warp - (4 + kUmmaDq);  // = warp % 4: TMEM lanes 32*ew ..
    bool dead = false, waited = false;
    int piece = 0;
    for (long long x = x0; x < x1;) {
      const int gidx = (int)(x / p.U), ua = (int)(x % p.U);
      const int ub = (int)((x1 - x) < (long long)(p.U - ua) ? ua + (x1 - x) : p.U);
      const int grp = gidx % p.groups, mz = (gidx / p.groups) * MROWS;
      int si0;
      sk_tile(p, grp, 0, si0);
      if (sk_rows(p, si0, mz, MROWS) > 0) {
        if (!waited) {
          pdl_wait();  // the partial buffer may still be read by the previous product's fix-up
          waited = true;
        }
        const int buf = PAIR ? 0 : piece & 1, use = PAIR ? piece : piece >> 1;
        const int pc = (int)(c - sk_owner((long long)gidx * p.U, p.W, P));
        if (wait_or_die(&accfull[buf], use & 1, dead, p.err)) {
          tc_fence_after();
          const int m = ew * 32 + lane;  // TMEM lane = operand row: feature 16 (m / 16) + fo
          const int fo = (m & 8) | ((m & 3) << 1) | ((m >> 2) & 1);
          int si;
          const int tile = sk_tile(p, grp, m >> 4, si);
#pragma unroll 1
          for (int h = 0; h < (PAIR ? 2 : 1); ++h) {  // the tile's halves: rows mz + 256 h ..
            const int mh = mz + h * kUmmaRows;
            const int rows = tile >= 0 ? sk_rows(p, si, mh, kUmmaRows) : 0;
            float* out = p.part + (size_t)pc * p.piece_stride + (size_t)mh * p.ldo +
                         (tile >= 0 ? p.seg[si].out_col + tile * 16 + fo : 0);
            const uint32_t tbase = tmem + ((uint32_t)(ew * 32) << 16) + (uint32_t)((buf + h) * kUmmaRows);
            for (int n0 = 0; n0 < rows && n0 < p.un; n0 += 32) {
              uint32_t v[32];
              tmem_ld32(tbase + (uint32_t)n0, v);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (n0 + i < rows) out[(size_t)(n0 + i) * p.ldo] = __uint_as_float(v[i]);
            }
          }
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&accempty[buf]);
        ++piece;
      }
      x += ub - ua;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kUmmaTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Output head + top-16 for many drafted rows on the tensor cores.  The head ([V + R] rows: the
// output head, then the selector projection) has a second prepared copy in the tcgen05 operand
// layout: record rec, K step st (256 features x 64 k bf16, 32 KB) at ((rec * S + st) * 32 KB),
// feature f's 16-byte chunk c (k = 8c ..) at f * 128 + ((c ^ (f % 8)) * 16) (128-byte swizzle,
// K-major), so one bulk copy lands it as the MMA's B operand.  The rows are the M side (two
// 128-row accumulators in TMEM, 512 columns), the 256 features of a record the N side, so after a
// record each thread holds one row's 256 logits and offers them to that row's top-16, kept sorted
// in its registers.
//  * warp 0, one thread: TMA of the rows' [256][64] bf16 slice per K step (no multicast);
//  * warp 2, one thread: bulk copy of the record step (weights: before the dependency wait);
//  * warp 1: TMEM allocation and the MMA issue (2 x 4 per K step), commits;
//  * warps 4-7: the per-record top-16 epilogue.
// CTA c works on row tile c % nrt and on records c / nrt, c / nrt + P / nrt, ...; its lists are
// part c / nrt of the candidate lists ([P / nrt][rows][16]) that the selector merges.
struct UHeadParams {
  const uint8_t* Wsw;  // swizzled head records
  int V, R, H, rows, nrec, nrt;
  int id0;             // vocabulary id of the head's first row (a shard of the vocabulary; 0 for the whole head)
  float* z;           // [rows][R]
  float* cand_val;    // [parts][rows][16]
  int32_t* cand_id;
  int* err;
};

constexpr int kUHeadStages = 3;
constexpr int kUHeadStage = 2 * 32768;  // A: 256 rows x 128 B, B: 256 features x 128 B
constexpr int kUHeadSmem = kUHeadStages * kUHeadStage + 1024;

// Canonical bf16 head rows -> the swizzled operand copy (one CTA of 256 threads per record step).
__global__ void k_head_sw_prepare(const uint16_t* __restrict__ lm_head, const uint16_t* __restrict__ sel_proj,
                                  uint8_t* __restrict__ dst, int V, int R, int H) {
  const int S = H / 64, st = blockIdx.x, rec = blockIdx.y, f = threadIdx.x;
  const int row = rec * 256 + f;
  const uint16_t* src = row < V ? lm_head + (size_t)row * H : (row < V + R ? sel_proj + (size_t)(row - V) * H : nullptr);
  uint8_t* out = dst + ((size_t)rec * S + st) * 32768 + (size_t)f * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 v = src ? *reinterpret_cast<const uint4*>(src + (size_t)st * 64 + 8 * c) : make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(out + ((c ^ (f & 7)) << 4)) = v;
  }
}

// Insert (v, id) into a sorted 16-entry list held in registers (best first; the caller has checked
// that it beats the last entry): it replaces the last entry and bubbles up.
DEVI void reg_list_insert(float (&lv)[16], int (&li)[16], float v, int id) {
  lv[15] = v;
  li[15] = id;
#pragma unroll
  for (int k = 15; k > 0; --k) {
    const bool up = better(lv[k], li[k], lv[k - 1], li[k - 1]);
    const float a = lv[k], b = lv[k - 1];
    const int ia = li[k], ib = li[k - 1];
    lv[k] = up ? b : a;
    li[k] = up ? ib : ia;
    lv[k - 1] = up ? a : b;
    li[k - 1] = up ? ia : ib;
  }
}

__global__ void __launch_bounds__(kUHeadThreads, 1) k_umma_head(const __grid_constant__ CUtensorMap tmx, UHeadParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t xfull[kUHeadStages], bfull[kUHeadStages], sempty[kUHeadStages];
  __shared__ __align__(8) uint64_t accfull[2], accempty[2];
  __shared__ uint32_t tmem_base_sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.H / 64;
  const int P = gridDim.x, c = blockIdx.x, nparts = P / p.nrt, rt = c % p.nrt, part = c / p.nrt;
  const int row0 = rt * 256;
  const int trows = p.rows - row0 < 256 ? p.rows - row0 : 256;
  const int nmc = trows > 128 ? 2 : 1;  // 128-row accumulators this row tile needs
  // with one accumulator (at most 128 rows) the records alternate between TMEM columns 0 and 256,
  // so that the next record's MMAs run while the epilogue drains this one
  auto acc_buf = [&](int it) { return nmc == 1 ? (it & 1) : 0; };
  auto acc_use = [&](int it) { return nmc == 1 ? (it >> 1) : it; };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kUHeadStages; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&bfull[s], 1);
      mbar_init(&sempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  pdl_trigger();

  if (warp == 0 || warp == 2) {
    if (lane == 0) {  // ---- warp 0: activation rows (TMA); warp 2: weight record steps (bulk) ----
      const bool act = warp == 0;
      if (act) pdl_wait();
      bool dead = false;
      int cnt = 0;
      for (int rec = part; rec < p.nrec && !dead; rec += nparts)
        for (int st = 0; st < S && !dead; ++st, ++cnt) {
          const int s = cnt % kUHeadStages, round = cnt / kUHeadStages;
          if (round > 0 && !wait_or_die(&sempty[s], (round - 1) & 1, dead, p.err)) break;
          uint8_t* stage = smem + s * kUHeadStage;
          if (act) {
            mbar_expect_tx(&xfull[s], 32768);
            tma_load_2d(stage, &tmx, st * 64, row0, &xfull[s]);
          } else {
            mbar_expect_tx(&bfull[s], 32768);
            bulk_g2s(stage + 32768, p.Wsw + ((size_t)rec * S + st) * 32768, 32768, &bfull[s]);
          }
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer ----
      bool dead = false;
      int cnt = 0, it = 0;
      for (int rec = part; rec < p.nrec && !dead; rec += nparts, ++it) {
        const int buf = acc_buf(it), use = acc_use(it);
        if (use > 0 && !wait_or_die(&accempty[buf], (use - 1) & 1, dead, p.err)) break;
        tc_fence_after();
        for (int st = 0; st < S && !dead; ++st, ++cnt) {
          const int s = cnt % kUHeadStages;
          const uint32_t par = (cnt / kUHeadStages) & 1;
          if (!wait_or_die(&xfull[s], par, dead, p.err) || !wait_or_die(&bfull[s], par, dead, p.err)) break;
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * kUHeadStage), b0 = a0 + 32768;
          const uint64_t bd = sw128_desc(b0);
          for (int mc = 0; mc < nmc; ++mc) {
            const uint64_t ad = sw128_desc(a0 + mc * 16384);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_mma(tmem + (buf + mc) * 256, ad + 2 * kk, bd + 2 * kk, kUmmaIdesc, (st == 0 && kk == 0) ? 0u : 1u);
          }
          tc_commit(&sempty[s]);
        }
        if (!dead) tc_commit(&accfull[buf]);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ---- per-record top-16 epilogue: thread = row (TMEM lane 32*dw + lane of each accumulator) ----
    const int dw = warp - 4;
    float lv[2][16];
    int li[2][16];
#pragma unroll
    for (int mc = 0; mc < 2; ++mc)
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        lv[mc][k] = -INFINITY;
        li[mc][k] = 0x7fffffff;
      }
    bool dead = false;
    int it = 0;
    pdl_wait();  // (outputs; the dependency also orders the lists after the previous step's readers)
    for (int rec = part; rec < p.nrec; rec += nparts, ++it) {
      const int buf = acc_buf(it), use = acc_use(it);
      if (wait_or_die(&accfull[buf], use & 1, dead, p.err)) {
        tc_fence_after();
#pragma unroll
        for (int mc = 0; mc < 2; ++mc) {
          if (mc >= nmc) break;
          const int rl = mc * 128 + dw * 32 + lane, row = row0 + rl;
          for (int n0 = 0; n0 < 256; n0 += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + ((uint32_t)(dw * 32) << 16) + (uint32_t)((buf + mc) * 256 + n0), r);
            tmem_ld_wait();
            if (rl < trows) {
              const int f0 = rec * 256 + n0, g0 = f0 + p.id0;  // g0: vocabulary id of feature f0
              const int nv = min(32, max(0, p.V - f0));          // head features of this chunk
              // the features that beat the row's 16th entry (compact: one compare each), then one
              // insertion site for the few that do (the list's 16th only rises as entries go in)
              const float th = lv[mc][15];
              const int thi = li[mc][15];
              unsigned m = 0;
#pragma unroll
              for (int i = 0; i < 32; ++i) m |= (i < nv && better(__uint_as_float(r[i]), g0 + i, th, thi)) ? 1u << i : 0u;
              while (m) {
                const int i = __ffs(m) - 1;
                m &= m - 1;
                float x = __uint_as_float(r[0]);
#pragma unroll
                for (int k = 1; k < 32; ++k) x = k == i ? __uint_as_float(r[k]) : x;
                if (better(x, g0 + i, lv[mc][15], li[mc][15])) reg_list_insert(lv[mc], li[mc], x, g0 + i);
              }
              if (f0 + 32 > p.V) {  // selector projection features of this chunk
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                  const int f = f0 + i;
                  if (f >= p.V && f < p.V + p.R) p.z[(size_t)row * p.R + (f - p.V)] = __uint_as_float(r[i]);
                }
              }
            }
          }
        }
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[buf]);
    }
    // this CTA's lists -> part `part` of the candidate lists
#pragma unroll
    for (int mc = 0; mc < 2; ++mc) {
      const int rl = mc * 128 + dw * 32 + lane;
      if (rl < trows) {
        const size_t o = ((size_t)part * p.rows + row0 + rl) * kTopK;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          p.cand_val[o + k] = lv[mc][k];
          p.cand_id[o + k] = li[mc][k];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Split-K fix-up of the tensor-core products: the CTA of (fr-row group, column group) sums the
// pieces of its tile in piece order (deterministic) and runs the product's fused epilogue.
// P: the tensor-core launch's grid size (p.W its stream-K plane).  E: the epilogue, fixed at compile
// time so that the light ones (residual, SwiGLU, store) fit two CTAs per SM.
template <int E, int MINB>
// fr: rows per CTA (16, 32 or 64; fewer rows give few-row products more CTAs in flight).
__global__ void __launch_bounds__(kGemvConsumers * 32, MINB) k_umma_fixup(SGemvParams p, int P, int fr) {
  pdl_trigger();
  pdl_wait();
  const int grp = blockIdx.x % p.groups, mz = (blockIdx.x / p.groups) * fr;
  const long long gidx = (long long)(mz / (p.upair ? 2 * kUmmaRows : kUmmaRows)) * p.groups + grp;
  const long long gstart = gidx * p.U;
  const long long first = sk_owner(gstart, p.W, P);
  const int npieces = (int)(sk_owner(gstart + p.U - 1, p.W, P) - first + 1);
  int si;
  sk_tile(p, grp, 0, si);
  if (sk_rows(p, si, mz, fr) <= 0) return;
  sk_fixup<E>(p, grp, mz, fr, npieces, nullptr);
}

}  // namespace dfl
