// Sliding-window GQA attention for many requests (FastFlowLM card, "Draft" row: 32 query / 8
// key-value heads of 128, sliding window 2048): one CTA per (request, kv head) streams the
// window's cache pages through a ring of TMA stages.
//
// With many requests the cluster kernel (attention.cuh) runs thousands of short CTAs, one per SM at
// a time, each paying the whole load-compute-merge latency.  Here a cluster of S CTAs (S = 1 when
// the (request, kv head) pairs alone fill the SMs two deep) owns a pair for the whole window, CTA
// r of it taking chunks r, r + S, ...; two CTAs share an SM, and the loads run ahead of the math:
//  * warp 4, one thread: for each 64-key chunk (4 pages of 16 tokens), the 4 KiB K and V rows of
//    this kv head in each page by 2-D TMA (cp.async.bulk.tensor, no multicast) as two 64-dim boxes
//    with 128-byte swizzle into one of two 32 KB stages; unmapped pages are skipped and flagged;
//  * warps 0-3: warp (qt, kh) takes query tile qt (16 of the kv head's G x Bk query vectors) and
//    key half kh (32 keys) of every chunk: S = Q K^T and P V on mma.sync m16n8k16 with an online
//    softmax (running max, sum and output in registers); then the block's own keys (all visible);
//    the two key halves of a query tile merge in shared memory, then the S CTAs' (max, sum,
//    output) merge over distributed shared memory, CTA r finishing 32/S of the query vectors.
// Visibility as everywhere: block row t at position p = Lb + t sees cache keys
// max(0, p - W + 1) <= j < Lb and every block key.  Softmax in fp32, scale 1/sqrt(128).
#pragma once
#include <cuda.h>

#include "attention.cuh"
#include "umma.cuh"

namespace dfl {

constexpr int kAttnStreamMinBatch = 8;  // requests from which the streaming kernel is used
constexpr int kAsStages = 2;
constexpr int kAsKeys = 64;                  // cache keys per stage (4 pages)
constexpr int kAsHalf = kAsKeys * 128;       // one 64-dim half of a stage's K or V: 8 KB (128-byte rows)
constexpr int kAsStage = 4 * kAsHalf;        // K lo | K hi | V lo | V hi
constexpr int kAsBlk = 4 * 16 * 128;         // the block keys (<= 16) in the same layout: 8 KB
constexpr int kAsQ = 32 * 256;               // 32 query vectors x 128 bf16
constexpr int kAsThreads = 5 * 32;
constexpr int kAsSmem = kAsStages * kAsStage + kAsBlk + kAsQ + 1024;
constexpr int kAsMaxPages = 256;  // page-table entries a CTA reads ahead (64 chunks: windows to 4032)

// byte offset of dims [8c, 8c + 8) of key row r in a 128-byte-swizzled half block
DEVI uint32_t as_off(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// S for NT * 8 keys (NT n-tiles of 8) of one 16-query tile; kbase: the K half-blocks (dims 0..63 at
// +0, 64..127 at +half), keys key0 .. key0 + 8 NT - 1 of them.
template <int NT>
DEVI void as_scores(const uint32_t (&qa)[8][4], const uint8_t* kbase, int half, int key0, float (&s)[4][4], int lane) {
#pragma unroll
  for (int n = 0; n < 4; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int hf = ks >> 2, c = (ks & 3) * 2 + ((lane >> 3) & 1);
#pragma unroll
    for (int n = 0; n < NT; n += 2) {  // two n-tiles per ldmatrix: lanes 16-31 address tile n + 1
      const int r = key0 + (n + (lane >> 4)) * 8 + (lane & 7);
      uint32_t b[4];
      ldmatrix_x4(b, kbase + hf * half + as_off(r, c));
      mma16816(s[n], qa[ks], b[0], b[1]);
      mma16816(s[n + 1], qa[ks], b[2], b[3]);
    }
  }
}

// P V for the same keys (KK steps of 16): o[16 dim tiles][4] += P (s, already exponentiated) x V.
template <int KK>
DEVI void as_pv(const float (&s)[4][4], const uint8_t* vbase, int half, int key0, float (&o)[16][4], int lane) {
#pragma unroll
  for (int kk = 0; kk < KK; ++kk) {
    uint32_t a[4];
    a[0] = pack_bf2(s[2 * kk][0], s[2 * kk][1]);
    a[1] = pack_bf2(s[2 * kk][2], s[2 * kk][3]);
    a[2] = pack_bf2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
    a[3] = pack_bf2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
    const int r = key0 + kk * 16 + (lane & 15);
#pragma unroll
    for (int n = 0; n < 16; n += 2) {  // two dim tiles per ldmatrix: lanes 16-31 address tile n + 1
      const int nn = n + (lane >> 4);
      uint32_t b[4];
      ldmatrix_x4_trans(b, vbase + (nn >> 3) * half + as_off(r, nn & 7));
      mma16816(o[n], a, b[0], b[1]);
      mma16816(o[n + 1], a, b[2], b[3]);
    }
  }
}

// Online softmax update of one warp's two rows (h = 0, 1: query vectors g, g + 8 of its tile) with
// this chunk's masked scores (already scaled to log2 units, -inf where not visible); only the first
// NT n-tiles hold keys.
template <int NT>
DEVI void as_softmax(float (&s)[4][4], float (&m)[2], float (&l)[2], float (&o)[16][4]) {
  float mx[2] = {m[0], m[1]};
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) mx[e >> 1] = fmaxf(mx[e >> 1], s[n][e]);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
  }
  float corr[2], add[2] = {0.f, 0.f};
#pragma unroll
  for (int h = 0; h < 2; ++h) corr[h] = mx[h] == -INFINITY ? 1.f : exp2f(m[h] - mx[h]);
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float mm = mx[e >> 1];
      const float pv = mm == -INFINITY ? 0.f : exp2f(s[n][e] - mm);
      s[n][e] = pv;
      add[e >> 1] += pv;
    }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    add[h] += __shfl_xor_sync(0xffffffffu, add[h], 1);
    add[h] += __shfl_xor_sync(0xffffffffu, add[h], 2);
    l[h] = l[h] * corr[h] + add[h];
    m[h] = mx[h];
  }
  if (__any_sync(0xffffffffu, corr[0] != 1.f || corr[1] != 1.f)) {  // (most chunks keep the max)
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      o[n][0] *= corr[0];
      o[n][1] *= corr[0];
      o[n][2] *= corr[1];
      o[n][3] *= corr[1];
    }
  }
}

// tmk / tmv: the layer's K and V caches as [pages * nkv * 16 rows][128] bf16 tensors (boxes of 16
// rows x 64 dims, 128-byte swizzle).  Grid (S, nkv, B), clusters of (S, 1, 1), S in 1..8.
// Requires G * Bk <= 32 (two query tiles).
__global__ void __launch_bounds__(kAsThreads, 2) k_attn_stream(const __grid_constant__ CUtensorMap tmk,
                                                              const __grid_constant__ CUtensorMap tmv, AttnParams p,
                                                              uint16_t* __restrict__ ob) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kAsStages], empty[kAsStages];
  __shared__ int pvalid[kAsStages];  // bit i: page i of the stage's chunk is mapped
  __shared__ int s_pg[kAsMaxPages];  // physical page of (local chunk i, page pi) at 4 i + pi
  __shared__ float mrg_m[2][16], mrg_l[2][16];
  __shared__ float fin_m[32], fin_l[32];  // this CTA's running max and sum per query vector
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* stages = smem;
  uint8_t* blk = smem + kAsStages * kAsStage;  // block keys: K lo | K hi | V lo | V hi, 16 rows each
  uint16_t* Qs = reinterpret_cast<uint16_t*>(blk + kAsBlk);  // [32][128] bf16
  const int S = gridDim.x, rank = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.nq / p.nkv, nqv = G * p.Bk;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kAsStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    fence_mbar_init();
  }
  // Keys of pages that are never loaded (past the window's end, or unmapped) get P = 0, and their V
  // rows must be finite for 0 x V to vanish: the stages start zeroed, and later hold only loaded rows.
  for (int i = threadIdx.x; i < kAsStages * kAsStage / 16; i += kAsThreads)
    reinterpret_cast<uint4*>(stages)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  __syncthreads();
  pdl_trigger();
  pdl_wait();  // the queries, the block's keys and this step's context rows come from the QKV kernel
  const long long S0 = p.seq_len[b], Lb = S0 + p.n_new[b];
  long long s0 = Lb - p.W + 1;
  if (s0 < 0) s0 = 0;
  const long long cs = (s0 / kPage) * kPage;
  const int nc = (int)((Lb - cs + kAsKeys - 1) / kAsKeys);
  const int nloc = nc > rank ? (nc - rank + S - 1) / S : 0;  // this CTA's chunks: rank + i S

  if (warp == 4) {
    // ---- producer: this CTA's share of the window's pages, chunk by chunk ----
    // page (local chunk i, page pi): -2 past the cached tokens (nothing to load), -1 unmapped
    auto page_of = [&](int i, int pi) -> int {
      const long long j0 = cs + (long long)(rank + i * S) * kAsKeys + pi * kPage;  // first token
      if (j0 >= Lb) return -2;
      const long long lp = j0 / kPage;
      int g = lp < p.max_pages ? p.page_table[(size_t)b * p.max_pages + lp] : -1;
      if (g >= p.num_pages || g < 0) {
        g = -1;
        set_err(p.err, DFLASH2_DEV_PAGE);
      }
      return g;
    };
    // the whole warp reads the page-table entries ahead, all loads in flight together (one by
    // one they put a global-memory round trip per page on the chunk's critical path)
    const int npre = nloc * 4 < kAsMaxPages ? nloc * 4 : kAsMaxPages;
    for (int k = lane; k < npre; k += 32) s_pg[k] = page_of(k >> 2, k & 3);
    __syncwarp();
    if (lane == 0) {
      bool dead = false;
      int issued = 0;
      for (int i = 0; i < nloc && !dead; ++i) {
        const int s = i % kAsStages, round = i / kAsStages;
        if (round > 0 && !wait_or_die(&empty[s], (round - 1) & 1, dead, p.err)) break;
        int pg[4], pv = 0;
        uint32_t bytes = 0;
        for (int pi = 0; pi < 4; ++pi) {
          const int g = 4 * i + pi < npre ? s_pg[4 * i + pi] : page_of(i, pi);
          if (g >= 0) bytes += 4 * 2048;
          pg[pi] = g;
          pv |= (g >= 0 ? 1 : 0) << pi;
        }
        pvalid[s] = pv;
        uint8_t* st = stages + s * kAsStage;
        if (bytes) {
          mbar_expect_tx(&full[s], bytes);
          for (int pi = 0; pi < 4; ++pi)
            if (pg[pi] >= 0) {
              const int row = (pg[pi] * p.nkv + kvh) * kPage;
              tma_load_2d(st + 0 * kAsHalf + pi * 2048, &tmk, 0, row, &full[s]);
              tma_load_2d(st + 1 * kAsHalf + pi * 2048, &tmk, 64, row, &full[s]);
              tma_load_2d(st + 2 * kAsHalf + pi * 2048, &tmv, 0, row, &full[s]);
              tma_load_2d(st + 3 * kAsHalf + pi * 2048, &tmv, 64, row, &full[s]);
            }
        } else {
          mbar_arrive(&full[s]);  // (releases the page flags)
        }
        issued = i + 1;
      }
      // the CTA must not retire with copies into its shared memory still in flight (the math warps
      // may have stopped early on a timeout): wait, bounded, for the last stages issued
      for (int i = issued > kAsStages ? issued - kAsStages : 0; i < issued; ++i) {
        bool d2 = false;
        wait_or_die(&full[i % kAsStages], (i / kAsStages) & 1, d2, p.err);
      }
    }
    __syncwarp();
  } else {

  // ---- math warps: stage Q and the block keys (cp.async), then stream the chunks ----
  for (int i = threadIdx.x; i < 32 * 16; i += 128) {  // Q: 32 vectors x 16 chunks of 16 B
    const int qv = i >> 4, ch = i & 15;
    const bool ok = qv < nqv;
    const uint16_t* src = p.qb;
    if (ok) src += ((size_t)(b * p.Bk + qv / G) * p.nq + kvh * G + qv % G) * kHeadDim + ch * 8;
    cp_async16(reinterpret_cast<uint8_t*>(Qs) + qv * 256 + ch * 16, src, ok);
  }
  for (int i = threadIdx.x; i < 2 * 16 * 16; i += 128) {  // block keys: {K, V} x 16 rows x 16 chunks
    const int kv = i >> 8, r = (i >> 4) & 15, ch = i & 15;
    const bool ok = r < p.Bk;
    const uint16_t* src = kv ? p.vb : p.kb;
    if (ok) src += ((size_t)(b * p.Bk + r) * p.nkv + kvh) * kHeadDim + ch * 8;
    cp_async16(blk + (2 * kv + (ch >> 3)) * (16 * 128) + as_off(r, ch & 7), src, ok);
  }
  cp_async_wait_all();
  asm volatile("bar.sync 1, 128;" ::: "memory");
  const int qt = warp & 1, kh = warp >> 1, g = lane >> 2, t4 = lane & 3;
  uint32_t qa[8][4];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
    ldmatrix_x4(qa[ks], reinterpret_cast<const uint8_t*>(Qs) + (qt * 16 + (lane & 15)) * 256 + (ks * 16 + (lane >> 4) * 8) * 2);
  // window start of each of the thread's two rows relative to the first cached key of the walk:
  // block row t sees cache keys j >= Lb + t - W + 1 (padding vectors see no key)
  int trow[2];
  long long lo0[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int qv = qt * 16 + g + 8 * h;
    trow[h] = qv < nqv ? qv / G : -1;
    lo0[h] = trow[h] >= 0 ? Lb + trow[h] - p.W + 1 - cs : (long long)INT_MAX;
  }
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f}, o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  bool dead = false;
  for (int i = 0; i < nloc; ++i) {
    const int c = rank + i * S, s = i % kAsStages;
    if (!wait_or_die(&full[s], (i / kAsStages) & 1, dead, p.err)) break;
    const uint8_t* st = stages + s * kAsStage;
    float sc[4][4];
    as_scores<4>(qa, st, kAsHalf, kh * 32, sc, lane);
    // mask: key kk of the chunk (cache key j = cs + 64c + kk) is visible to the row iff its page is
    // mapped, j < Lb and j >= Lb + t - W + 1; chunk-relative bounds in int, clamped to [0, 65]
    const long long c64 = (long long)c * kAsKeys;
    const int hi = (int)min(max(Lb - cs - c64, 0ll), 65ll);
    int lo[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) lo[h] = (int)min(max(lo0[h] - c64, 0ll), 65ll);
    const int pv = pvalid[s];
    if (__all_sync(0xffffffffu, lo[0] == 0 && lo[1] == 0 && hi >= kAsKeys && pv == 0xF)) {
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[n][e] *= p.scale_log2;
    } else {
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kk = kh * 32 + n * 8 + 2 * t4 + (e & 1);
          const bool vis = kk >= lo[e >> 1] && kk < hi && ((pv >> (kk >> 4)) & 1);
          sc[n][e] = vis ? sc[n][e] * p.scale_log2 : -INFINITY;
        }
    }
    as_softmax<4>(sc, m, l, o);
    as_pv<2>(sc, st + 2 * kAsHalf, kAsHalf, kh * 32, o, lane);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);  // this warp's reads of the stage are done
  }
  // the block's own keys (rows 0 .. Bk-1 of the block area, zero-filled to 16), all visible, in CTA
  // 0 of the cluster: both key halves score the 16 rows, half kh keeps rows 8kh .. 8kh + 7
  if (!dead && rank == 0) {
    float sc[4][4];
    as_scores<2>(qa, blk, 16 * 128, 0, sc, lane);
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kk = n * 8 + 2 * t4 + (e & 1);
        const bool vis = trow[e >> 1] >= 0 && kk < p.Bk && n == kh;
        sc[n][e] = vis ? sc[n][e] * p.scale_log2 : -INFINITY;
      }
    as_softmax<2>(sc, m, l, o);
    as_pv<1>(sc, blk + 2 * (16 * 128), 16 * 128, 0, o, lane);
  }
  // ---- merge the two key halves of each query tile into this CTA's (max, sum, output) ----
  asm volatile("bar.sync 1, 128;" ::: "memory");  // every warp is done with the stages and blk
  float* red = reinterpret_cast<float*>(stages);                  // [qt][16 rows][128], key half 1
  float* fin = reinterpret_cast<float*>(stages) + 2 * 16 * 128;  // [32 vectors][128], unnormalised
  if (kh == 1) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = g + 8 * h;
#pragma unroll
      for (int n = 0; n < 16; ++n)
        *reinterpret_cast<float2*>(red + ((size_t)qt * 16 + row) * 128 + n * 8 + 2 * t4) =
            make_float2(o[n][2 * h], o[n][2 * h + 1]);
      if (t4 == 0) {
        mrg_m[qt][row] = m[h];
        mrg_l[qt][row] = l[h];
      }
    }
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
  if (kh == 0) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = g + 8 * h, qv = qt * 16 + row;
      const float m1 = mrg_m[qt][row], l1 = mrg_l[qt][row];
      const float M = fmaxf(m[h], m1);
      const float w0 = M == -INFINITY ? 0.f : exp2f(m[h] - M), w1 = M == -INFINITY ? 0.f : exp2f(m1 - M);
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        const float2 v1 = *reinterpret_cast<const float2*>(red + ((size_t)qt * 16 + row) * 128 + n * 8 + 2 * t4);
        *reinterpret_cast<float2*>(fin + (size_t)qv * 128 + n * 8 + 2 * t4) =
            make_float2(w0 * o[n][2 * h] + w1 * v1.x, w0 * o[n][2 * h + 1] + w1 * v1.y);
      }
      if (t4 == 0) {
        fin_m[qv] = M;
        fin_l[qv] = w0 * l[h] + w1 * l1;
      }
    }
  }
  }  // math warps
  // ---- the cluster's CTAs merge: CTA `rank` finishes query vectors [rank * 32 / S, ...) ----
  cluster_sync_all();  // every CTA's (max, sum, output) is in its shared memory
  {
    float* fin = reinterpret_cast<float*>(stages) + 2 * 16 * 128;
    const int v0 = rank * 32 / S, v1 = (rank + 1) * 32 / S;
    for (int i = threadIdx.x; i < (v1 - v0) * 64; i += kAsThreads) {
      const int qv = v0 + i / 64, d = (i % 64) * 2;
      if (qv >= nqv) continue;
      float M = -INFINITY;
      for (int r = 0; r < S; ++r) M = fmaxf(M, ld_cluster_f32(cluster_map(&fin_m[qv], r)));
      float L = 0.f, x = 0.f, y = 0.f;
      for (int r = 0; r < S; ++r) {
        const float mr = ld_cluster_f32(cluster_map(&fin_m[qv], r));
        const float wr = mr == -INFINITY ? 0.f : exp2f(mr - M);
        const float2 orr = ld_cluster_f32x2(cluster_map(fin + (size_t)qv * 128 + d, r));
        L += wr * ld_cluster_f32(cluster_map(&fin_l[qv], r));
        x += wr * orr.x;
        y += wr * orr.y;
      }
      const float inv = L > 0.f ? 1.f / L : 0.f;
      uint16_t* dst = ob + ((size_t)(b * p.Bk + qv / G) * p.nq + kvh * G + qv % G) * kHeadDim;
      *reinterpret_cast<uint32_t*>(dst + d) = pack_bf2(x * inv, y * inv);
    }
  }
  cluster_sync_all();  // no CTA leaves while another still reads its shared memory
}

}  // namespace dfl
