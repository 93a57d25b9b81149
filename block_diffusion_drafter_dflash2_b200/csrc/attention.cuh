// Sliding-window GQA attention of the block rows over the paged KV cache.
//
// Work split (flash-decoding): one CTA per (request, kv head, chunk of 64 cache
// keys = 4 pages) plus one CTA for the block's own keys.  The query vectors of
// a kv head's group (G query heads x Bk block rows, padded to 16-row mma
// tiles) attend to the chunk; each math warp owns 16 query vectors.  K and V
// rows of the chunk are loaded into shared memory (272-byte padded stride) by
// every thread of the CTA with 16-byte L2 loads, all issued before any store
// (64 rows of 256 bytes as one bulk copy per row cost more in copy-engine
// overhead than they move).  Scores and P.V use mma.sync m16n8k16; softmax
// statistics are fp32.  A combine kernel merges the chunk partials.
//
// Visibility (FastFlowLM card, "Draft" row: sliding window 2048): block row t
// sits at position p = Lb + t (Lb = cached tokens after this step's append);
// cache key j is visible iff max(0, p - W + 1) <= j < Lb; all block keys are
// visible to all block rows.
#pragma once
#include <climits>

#include "common.cuh"

namespace dfl {

struct AttnParams {
  const uint16_t *qb, *kb, *vb;  // [Mb][nq|nkv][128]
  const uint16_t *kc, *vc;       // this layer's cache [pages][nkv][16][128]
  const int32_t* page_table;
  int max_pages, num_pages;
  const int32_t *seq_len, *n_new;  // seq_len before the step (advanced later by the selector kernel)
  int Bk, nq, nkv, W;
  int NC;    // cache chunks per (request, kv head); chunk index NC = the block keys
  int QVP;   // query vectors per (request, kv head), padded to 16
  float *part_o, *part_ml;  // [B][nkv][NC+1][QVP][128], [B][nkv][NC+1][QVP][2]
  float scale_log2;         // log2(e) / sqrt(128)
  int* err;
};

DEVI void attn_geometry(const AttnParams& p, int b, long long& Lb, long long& cs, int& nact) {
  Lb = (long long)p.seq_len[b] + p.n_new[b];
  long long s0 = Lb - p.W + 1;
  if (s0 < 0) s0 = 0;
  cs = (s0 / kPage) * kPage;
  nact = (int)((Lb - cs + kAttnKeys - 1) / kAttnKeys);
}

// One chunk item (request b, kv head kvh, chunk c) processed by the first NTHR threads of the CTA
// (named barrier 1); warps 0..MT-1 do the math.  buf: (MT*16 + 2*64) * 272 bytes of shared memory;
// row_ok: 64 ints.
// Returns without touching anything when the chunk lies outside the request's window.
template <int MT, int NTHR>
DEVI void attn_item(const AttnParams& p, int c, int kvh, int b, uint8_t* buf, int* row_ok) {
  uint16_t* Qs = reinterpret_cast<uint16_t*>(buf);
  uint16_t* Ks = Qs + MT * 16 * kAttnStride;
  uint16_t* Vs = Ks + kAttnKeys * kAttnStride;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.nq / p.nkv, nqv = G * p.Bk;
  long long Lb, cs;
  int nact;
  attn_geometry(p, b, Lb, cs, nact);
  const bool blk = c == p.NC;
  if (!blk && c >= nact) return;
  const long long key0 = cs + (long long)c * kAttnKeys;
  consumers_sync<NTHR>();  // the buffer is free (previous item done)
  // queries of this (request, kv head): vector qv = t*G + gi -> head kvh*G + gi of block row t.
  // Every thread issues its 8 loads before any store (no load->store chains).
  {
    constexpr int kQv = MT * 16 * 16;  // 16-byte vectors of the query tile
    constexpr int kPer = (kQv + NTHR - 1) / NTHR;
    uint4 qv8[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int i = threadIdx.x + k * NTHR, qv = i >> 4, v = i & 15;
      qv8[k] = make_uint4(0, 0, 0, 0);
      if (i < kQv && qv < nqv) {
        const int t = qv / G, gi = qv % G;
        qv8[k] = __ldcg(reinterpret_cast<const uint4*>(p.qb + ((size_t)(b * p.Bk + t) * p.nq + kvh * G + gi) * kHeadDim + v * 8));
      }
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int i = threadIdx.x + k * NTHR, qv = i >> 4, v = i & 15;
      if (i < kQv) *reinterpret_cast<uint4*>(Qs + qv * kAttnStride + v * 8) = qv8[k];
    }
  }
  if (blk) {
    // the block's own keys: Bk rows loaded (4 vectors per thread at most), the rest zero
    for (int i = threadIdx.x; i < kAttnKeys * 16; i += NTHR) {
      const int u = i >> 4, v = i & 15;
      if (u >= p.Bk) {
        *reinterpret_cast<uint4*>(Ks + u * kAttnStride + v * 8) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(Vs + u * kAttnStride + v * 8) = make_uint4(0, 0, 0, 0);
      }
    }
    {
      constexpr int kPerK = (16 * 16 + NTHR - 1) / NTHR;  // Bk <= 16 rows x 16 vectors
      uint4 kv4[kPerK], vv4[kPerK];
#pragma unroll
      for (int k = 0; k < kPerK; ++k) {
        const int i = threadIdx.x + k * NTHR, u = i >> 4, v = i & 15;
        if (u < p.Bk) {
          const size_t off = ((size_t)(b * p.Bk + u) * p.nkv + kvh) * kHeadDim + v * 8;
          kv4[k] = __ldcg(reinterpret_cast<const uint4*>(p.kb + off));
          vv4[k] = __ldcg(reinterpret_cast<const uint4*>(p.vb + off));
        }
      }
#pragma unroll
      for (int k = 0; k < kPerK; ++k) {
        const int i = threadIdx.x + k * NTHR, u = i >> 4, v = i & 15;
        if (u < p.Bk) {
          *reinterpret_cast<uint4*>(Ks + u * kAttnStride + v * 8) = kv4[k];
          *reinterpret_cast<uint4*>(Vs + u * kAttnStride + v * 8) = vv4[k];
        }
      }
    }
    if (threadIdx.x < kAttnKeys) row_ok[threadIdx.x] = threadIdx.x < p.Bk;
    consumers_sync<NTHR>();
  } else {
    // the chunk's 64 cache keys (4 pages) with 16-byte L2 loads by every thread, all issued before
    // any store; keys past the request's length or on unmapped pages read as zero and are masked
    constexpr int kVec = kAttnKeys * 16;  // 16-byte vectors per K (or V) chunk
    constexpr int kPerKV = (kVec + NTHR - 1) / NTHR;
    uint4 kr[kPerKV], vr[kPerKV];
#pragma unroll
    for (int k = 0; k < kPerKV; ++k) {
      const int i = threadIdx.x + k * NTHR, kk = i >> 4, v = i & 15;
      kr[k] = vr[k] = make_uint4(0, 0, 0, 0);
      if (i < kVec) {
        const long long j = key0 + kk;
        bool ok = false;
        if (j < Lb) {
          const int lp = (int)(j / kPage);
          const int32_t pg = lp < p.max_pages ? p.page_table[(size_t)b * p.max_pages + lp] : -1;
          ok = pg >= 0 && pg < p.num_pages;
          if (ok) {
            const size_t off = (((size_t)pg * p.nkv + kvh) * kPage + j % kPage) * kHeadDim + v * 8;
            kr[k] = __ldcg(reinterpret_cast<const uint4*>(p.kc + off));
            vr[k] = __ldcg(reinterpret_cast<const uint4*>(p.vc + off));
          } else if (v == 0) {
            set_err(p.err, DFLASH2_DEV_PAGE);
          }
        }
        if (v == 0) row_ok[kk] = ok;
      }
    }
#pragma unroll
    for (int k = 0; k < kPerKV; ++k) {
      const int i = threadIdx.x + k * NTHR, kk = i >> 4, v = i & 15;
      if (i < kVec) {
        *reinterpret_cast<uint4*>(Ks + kk * kAttnStride + v * 8) = kr[k];
        *reinterpret_cast<uint4*>(Vs + kk * kAttnStride + v * 8) = vr[k];
      }
    }
    consumers_sync<NTHR>();
  }
  if (warp >= MT) return;

  // ---- S = Q K^T for this warp's 16 query vectors x 64 keys ----
  const int g = lane >> 2, t4 = lane & 3;
  float s[8][4];
#pragma unroll
  for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
  const uint16_t* Qw = Qs + warp * 16 * kAttnStride;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    uint32_t a[4];
    ldmatrix_x4(a, Qw + (lane & 15) * kAttnStride + ks * 16 + (lane >> 4) * 8);
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      uint32_t b0, b1;
      ldmatrix_x2(b0, b1, Ks + (n * 8 + (lane & 7)) * kAttnStride + ks * 16 + ((lane >> 3) & 1) * 8);
      mma16816(s[n], a, b0, b1);
    }
  }
  // ---- mask, chunk-local softmax (log2 domain) ----
  float mrow[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int n = 0; n < 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int qv = warp * 16 + g + 8 * (e >> 1);
      const int kk = n * 8 + 2 * t4 + (e & 1);
      bool vis = qv < nqv && row_ok[kk];
      if (vis && !blk) {
        const long long j = key0 + kk;
        const long long pos = Lb + qv / G;
        vis = j >= pos - p.W + 1;
      }
      const float v = vis ? s[n][e] * p.scale_log2 : -INFINITY;
      s[n][e] = v;
      mrow[e >> 1] = fmaxf(mrow[e >> 1], v);
    }
  float lrow[2] = {0.f, 0.f};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    mrow[h] = fmaxf(mrow[h], __shfl_xor_sync(0xffffffffu, mrow[h], 1));
    mrow[h] = fmaxf(mrow[h], __shfl_xor_sync(0xffffffffu, mrow[h], 2));
  }
#pragma unroll
  for (int n = 0; n < 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float m = mrow[e >> 1];
      const float pv = m == -INFINITY ? 0.f : exp2f(s[n][e] - m);
      s[n][e] = pv;
      lrow[e >> 1] += pv;
    }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 1);
    lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 2);
  }
  // ---- O = P V ----
  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint32_t a[4];
    a[0] = pack_bf2(s[2 * kk][0], s[2 * kk][1]);
    a[1] = pack_bf2(s[2 * kk][2], s[2 * kk][3]);
    a[2] = pack_bf2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
    a[3] = pack_bf2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      uint32_t b0, b1;
      ldmatrix_x2_trans(b0, b1, Vs + (kk * 16 + (lane & 15)) * kAttnStride + n * 8);
      mma16816(o[n], a, b0, b1);
    }
  }
  // ---- write the chunk partial ----
  const size_t base = (((size_t)b * p.nkv + kvh) * (p.NC + 1) + c) * p.QVP + warp * 16;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = g + 8 * h;
    float* orow = p.part_o + (base + row) * kHeadDim;
#pragma unroll
    for (int n = 0; n < 16; ++n)
      *reinterpret_cast<float2*>(orow + n * 8 + 2 * t4) = make_float2(o[n][2 * h], o[n][2 * h + 1]);
    if (t4 == 0) *reinterpret_cast<float2*>(p.part_ml + (base + row) * 2) = make_float2(mrow[h], lrow[h]);
  }
}


constexpr int kAttnThreads = 256;  // loaders; the first MT warps also do the math

template <int MT>  // 16-row query tiles per CTA (= math warps)
__global__ void __launch_bounds__(kAttnThreads) k_attn_chunk(AttnParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int row_ok[kAttnKeys];
  pdl_trigger();
  pdl_wait();
  attn_item<MT, kAttnThreads>(p, blockIdx.x, blockIdx.y, blockIdx.z, smem, row_ok);
}

// One warp per (request, kv head, query vector): merge the chunk partials -> o bf16 [Mb][nq][128].
// Lanes read the chunks' (m, l) in parallel; the weighted sum streams 16-byte rows.
DEVI void attn_combine_warp(const AttnParams& p, uint16_t* __restrict__ ob, int qv, int kvh, int b, float* wsh) {
  const int lane = threadIdx.x & 31;
  const int G = p.nq / p.nkv;
  if (qv >= G * p.Bk) return;
  long long Lb, cs;
  int nact;
  attn_geometry(p, b, Lb, cs, nact);
  if (nact > p.NC) nact = p.NC;
  const int nc = nact + 1;  // cache chunks + the block-key chunk (index NC)
  const size_t base = ((size_t)b * p.nkv + kvh) * (p.NC + 1);
  float m[2], l[2];
  float M = -INFINITY;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = lane + 32 * h;
    m[h] = -INFINITY;
    l[h] = 0.f;
    if (i < nc) {
      const int c = i < nact ? i : p.NC;
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.part_ml + ((base + c) * p.QVP + qv) * 2));
      m[h] = ml.x;
      l[h] = ml.y;
    }
    M = fmaxf(M, m[h]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float L = 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = lane + 32 * h;
    const float w = (m[h] == -INFINITY) ? 0.f : exp2f(m[h] - M);
    if (i < 64) wsh[i] = w;
    L += w * l[h];
  }
  L = warp_sum(L);
  __syncwarp();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
  for (int i = 0; i < nc; ++i) {
    const int c = i < nact ? i : p.NC;
    const float w = wsh[i];
    const float4 v = __ldcg(reinterpret_cast<const float4*>(p.part_o + ((base + c) * p.QVP + qv) * kHeadDim + lane * 4));
    acc.x += w * v.x;
    acc.y += w * v.y;
    acc.z += w * v.z;
    acc.w += w * v.w;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const int t = qv / G, gi = qv % G;
  uint16_t* dst = ob + ((size_t)(b * p.Bk + t) * p.nq + kvh * G + gi) * kHeadDim + lane * 4;
  *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf2(acc.x * inv, acc.y * inv), pack_bf2(acc.z * inv, acc.w * inv));
}

__global__ void k_attn_combine(AttnParams p, uint16_t* __restrict__ ob) {
  __shared__ float wsh[4][64];
  pdl_trigger();
  pdl_wait();
  const int wi = threadIdx.x >> 5;
  attn_combine_warp(p, ob, blockIdx.x * (blockDim.x >> 5) + wi, blockIdx.y, blockIdx.z, wsh[wi]);
}

}  // namespace dfl

namespace dfl {

// ---------------------------------------------------------------------------
// Sliding-window attention of one (request, kv head) on a cluster of 8 CTAs, merge included.
// The keys seen by the block's queries are the cache window [cs, Lb) followed by the block's own
// Bk keys; CTA r of the cluster takes keys [r*KC, (r+1)*KC) of that sequence.  Its warps split
// them into 4 quarters (warp = quarter * MT + query tile): S = Q K^T and P.V on mma.sync with a
// quarter-local softmax, the quarters merged in shared memory into the CTA's (m, l, o), then the 8
// CTAs' partials merged over distributed shared memory, each CTA finishing 1/8 of the query
// vectors.  The merge order is fixed, so the result does not depend on timing.
//
// Cache rows below seq_len were written by earlier steps and are not touched during this one,
// so they are fetched (cp.async) before waiting on the previous kernel; the rows that kernel
// writes (this step's context rows, the block's keys and the queries) are fetched after.
constexpr int kClusterCtas = 8;

DEVI void cp_async16(void* dst, const void* src, bool pred) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(pred ? 16 : 0)
               : "memory");
}
DEVI void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
DEVI uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
DEVI void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// shared-memory address of `p` in CTA `rank` of the cluster
DEVI uint32_t cluster_map(const void* p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  return a;
}
DEVI float ld_cluster_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}
DEVI float2 ld_cluster_f32x2(uint32_t a) {
  float2 v;
  asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a) : "memory");
  return v;
}

constexpr int kClRedStride = kHeadDim + 8;  // floats per row of the quarter partials (bank spread)

// Dynamic shared memory of k_attn_cluster: queries + KC key rows + KC value rows, bf16, padded rows.
constexpr size_t attn_cluster_smem(int MT, int KC) { return (size_t)(MT * 16 + 2 * KC) * kAttnStride * 2; }

// MT 16-row query tiles; KG key groups (warp = group * MT + tile); NTK 8-key tiles per group
// (KC = KG * 8 * NTK keys per CTA).
template <int MT, int NTK, int KG = 4>
__global__ void __launch_bounds__(MT * KG * 32, 1) k_attn_cluster(AttnParams p, uint16_t* __restrict__ ob) {
  constexpr int NT = MT * KG * 32, kQv = MT * 16, KQ = 8 * NTK, KC = KG * KQ, kQpc = kQv / kClusterCtas;
  static_assert(MT <= 2 && NTK % 2 == 0 && KC % kPage == 0, "shape");
  static_assert(MT * KG * 16 * kClRedStride * 4 <= 2 * KC * kAttnStride * 2, "group partials fit over K/V");
  static_assert(kQpc >= 1 && kQpc * 64 <= NT, "one output pair per thread in the cluster merge");
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int row_ok[KC];  // 0 masked, 1 cache key (window applies), 2 block key
  __shared__ int pgs[KC / kPage];
  __shared__ float red_m[MT * KG][16], red_l[MT * KG][16];
  __shared__ float cm[kQv], cl[kQv], qw[kQv][KG];
  uint16_t* Qs = reinterpret_cast<uint16_t*>(smem);
  uint16_t* Ks = Qs + kQv * kAttnStride;
  uint16_t* Vs = Ks + KC * kAttnStride;
  float* red_o = reinterpret_cast<float*>(Ks);  // [MT*KG warps][16][kClRedStride] after the math
  pdl_trigger();
  const uint32_t r = cluster_rank();
  const int kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.nq / p.nkv, nqv = G * p.Bk;
  // step inputs: no kernel of this step writes them, and the step's opening memsets order every
  // earlier writer (host staging, the previous round's acceptance) before this launch
  const long long S0 = p.seq_len[b];
  const long long Lb = S0 + p.n_new[b];
  long long s0 = Lb - p.W + 1;
  if (s0 < 0) s0 = 0;
  const long long cs = (s0 / kPage) * kPage;
  const long long ncache = Lb - cs;
  const long long k0 = (long long)r * KC;  // cs + k0 is page aligned (KC is a multiple of kPage)
  // this CTA's rows: [0, o_end) cache rows of earlier steps, [o_end, c_end) this step's context
  // rows, [c_end, b_end) the block's keys, [b_end, KC) nothing (masked, zero)
  auto clampkc = [](long long x) { return (int)(x < 0 ? 0 : (x > KC ? KC : x)); };
  const int o_end = clampkc(S0 - cs - k0), c_end = clampkc(ncache - k0), b_end = clampkc(ncache + p.Bk - k0);
  const int u0 = (int)(k0 - ncache);  // block key of row kk: kk + u0
  constexpr int RP = NT / 16;          // rows per pass (16 lanes per row)
  const int v = threadIdx.x & 15, slot = threadIdx.x >> 4;
  const size_t page_stride = (size_t)p.nkv * kPage * kHeadDim;
  const uint16_t* kc0 = p.kc + (size_t)kvh * kPage * kHeadDim + v * 8;
  const uint16_t* vc0 = p.vc + (size_t)kvh * kPage * kHeadDim + v * 8;

  for (int i = threadIdx.x; i < KC / kPage; i += NT) {
    int pg = -1;
    if (i * kPage < c_end) {
      const long long lp = (cs + k0) / kPage + i;
      pg = lp < p.max_pages ? p.page_table[(size_t)b * p.max_pages + lp] : -1;
      if (pg >= p.num_pages) pg = -1;
    }
    pgs[i] = pg;
  }
  __syncthreads();
  // one cache row: 16 lanes, 16 bytes each; an unmapped page reads as zero and flags the error
  auto cache_row = [&](int kk) {
    const int pg = pgs[kk / kPage];
    const bool ok = pg >= 0;
    const size_t off = ok ? (size_t)pg * page_stride + (size_t)(kk % kPage) * kHeadDim : 0;
    cp_async16(Ks + kk * kAttnStride + v * 8, kc0 + off, ok);
    cp_async16(Vs + kk * kAttnStride + v * 8, vc0 + off, ok);
    if (v == 0) {
      row_ok[kk] = ok ? 1 : 0;
      if (!ok) set_err(p.err, DFLASH2_DEV_PAGE);
    }
  };
  // ---- before the wait: cache rows of earlier steps; rows past everything read as zero ----
  for (int kk = slot; kk < o_end; kk += RP) cache_row(kk);
  for (int kk = b_end + slot; kk < KC; kk += RP) {
    cp_async16(Ks + kk * kAttnStride + v * 8, p.kc, false);
    cp_async16(Vs + kk * kAttnStride + v * 8, p.vc, false);
    if (v == 0) row_ok[kk] = 0;
  }
  pdl_wait();  // queries, the block's keys and this step's context rows come from the QKV kernel
  for (int kk = o_end + slot; kk < c_end; kk += RP) cache_row(kk);
  for (int kk = c_end + slot; kk < b_end; kk += RP) {
    const size_t off = ((size_t)(b * p.Bk + kk + u0) * p.nkv + kvh) * kHeadDim + v * 8;
    cp_async16(Ks + kk * kAttnStride + v * 8, p.kb + off, true);
    cp_async16(Vs + kk * kAttnStride + v * 8, p.vb + off, true);
    if (v == 0) row_ok[kk] = 2;
  }
  for (int qv = slot; qv < kQv; qv += RP) {
    const bool ok = qv < nqv;
    const uint16_t* src = p.qb;
    if (ok) src += ((size_t)(b * p.Bk + qv / G) * p.nq + kvh * G + qv % G) * kHeadDim + v * 8;
    cp_async16(Qs + qv * kAttnStride + v * 8, src, ok);
  }
  cp_async_wait_all();
  __syncthreads();

  // ---- warp (qt, kq): 16 query vectors x KQ keys ----
  const int qt = warp % MT, kq = warp / MT, g = lane >> 2, t4 = lane & 3;
  float s[NTK][4];
#pragma unroll
  for (int n = 0; n < NTK; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
  const uint16_t* Qw = Qs + qt * 16 * kAttnStride;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    uint32_t a[4];
    ldmatrix_x4(a, Qw + (lane & 15) * kAttnStride + ks * 16 + (lane >> 4) * 8);
#pragma unroll
    for (int n = 0; n < NTK; ++n) {
      uint32_t b0, b1;
      ldmatrix_x2(b0, b1, Ks + (kq * KQ + n * 8 + (lane & 7)) * kAttnStride + ks * 16 + ((lane >> 3) & 1) * 8);
      mma16816(s[n], a, b0, b1);
    }
  }
  // key kk (cache) is inside the window of block row t iff t <= tmax0 + kk
  const int tmax0 = (int)(cs + k0 - Lb + p.W - 1);
  int trow[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int qv = qt * 16 + g + 8 * h;
    trow[h] = qv < nqv ? qv / G : INT_MAX;  // INT_MAX: padding vector, sees nothing
  }
  float mrow[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int n = 0; n < NTK; ++n) {
    const int kb0 = kq * KQ + n * 8 + 2 * t4;
    const int ty[2] = {row_ok[kb0], row_ok[kb0 + 1]};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int h = e >> 1, type = ty[e & 1];
      const bool vis = trow[h] != INT_MAX && (type == 2 || (type == 1 && trow[h] <= tmax0 + kb0 + (e & 1)));
      const float x = vis ? s[n][e] * p.scale_log2 : -INFINITY;
      s[n][e] = x;
      mrow[h] = fmaxf(mrow[h], x);
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    mrow[h] = fmaxf(mrow[h], __shfl_xor_sync(0xffffffffu, mrow[h], 1));
    mrow[h] = fmaxf(mrow[h], __shfl_xor_sync(0xffffffffu, mrow[h], 2));
  }
  float lrow[2] = {0.f, 0.f};
#pragma unroll
  for (int n = 0; n < NTK; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float m = mrow[e >> 1];
      const float pv = m == -INFINITY ? 0.f : exp2f(s[n][e] - m);
      s[n][e] = pv;
      lrow[e >> 1] += pv;
    }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 1);
    lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 2);
  }
  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < NTK / 2; ++kk) {
    uint32_t a[4];
    a[0] = pack_bf2(s[2 * kk][0], s[2 * kk][1]);
    a[1] = pack_bf2(s[2 * kk][2], s[2 * kk][3]);
    a[2] = pack_bf2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
    a[3] = pack_bf2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      uint32_t b0, b1;
      ldmatrix_x2_trans(b0, b1, Vs + (kq * KQ + kk * 16 + (lane & 15)) * kAttnStride + n * 8);
      mma16816(o[n], a, b0, b1);
    }
  }
  __syncthreads();  // K/V are no longer read: their space takes the quarter partials
  {
    float* ro = red_o + (size_t)warp * 16 * kClRedStride;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = g + 8 * h;
#pragma unroll
      for (int n = 0; n < 16; ++n)
        *reinterpret_cast<float2*>(ro + row * kClRedStride + n * 8 + 2 * t4) = make_float2(o[n][2 * h], o[n][2 * h + 1]);
      if (t4 == 0) {
        red_m[warp][row] = mrow[h];
        red_l[warp][row] = lrow[h];
      }
    }
  }
  __syncthreads();
  // ---- merge the quarters; the CTA's o lands in quarter 0's rows (row qv of red_o) ----
  if (threadIdx.x < kQv) {
    const int qv = threadIdx.x, qtt = qv / 16, row = qv % 16;
    float M = -INFINITY;
#pragma unroll
    for (int q = 0; q < KG; ++q) M = fmaxf(M, red_m[q * MT + qtt][row]);
    float L = 0.f;
#pragma unroll
    for (int q = 0; q < KG; ++q) {
      const int wq = q * MT + qtt;
      const float wgt = M == -INFINITY ? 0.f : exp2f(red_m[wq][row] - M);
      qw[qv][q] = wgt;
      L += wgt * red_l[wq][row];
    }
    cm[qv] = M;
    cl[qv] = L;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kQv * kHeadDim; i += NT) {
    const int qv = i / kHeadDim, d = i % kHeadDim, qtt = qv / 16, row = qv % 16;
    float O = 0.f;
#pragma unroll
    for (int q = 0; q < KG; ++q) O += qw[qv][q] * red_o[((size_t)(q * MT + qtt) * 16 + row) * kClRedStride + d];
    red_o[(size_t)qv * kClRedStride + d] = O;  // only this thread reads or writes this element
  }
  cluster_sync_all();
  // ---- merge the cluster's 8 partials: this CTA finishes query vectors r*kQpc .. +kQpc-1 ----
  if (threadIdx.x < kQpc * 64) {
    const int qv = (int)r * kQpc + threadIdx.x / 64, d = (threadIdx.x % 64) * 2;
    float mc[kClusterCtas], M = -INFINITY;
#pragma unroll
    for (int c = 0; c < kClusterCtas; ++c) {
      mc[c] = ld_cluster_f32(cluster_map(cm + qv, c));
      M = fmaxf(M, mc[c]);
    }
    float L = 0.f;
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int c = 0; c < kClusterCtas; ++c) {
      const float wgt = mc[c] == -INFINITY ? 0.f : exp2f(mc[c] - M);
      L += wgt * ld_cluster_f32(cluster_map(cl + qv, c));
      const float2 v = ld_cluster_f32x2(cluster_map(red_o + (size_t)qv * kClRedStride + d, c));
      acc.x += wgt * v.x;
      acc.y += wgt * v.y;
    }
    if (qv < nqv) {
      const float inv = L > 0.f ? 1.f / L : 0.f;
      uint16_t* dst = ob + ((size_t)(b * p.Bk + qv / G) * p.nq + kvh * G + qv % G) * kHeadDim + d;
      *reinterpret_cast<uint32_t*>(dst) = pack_bf2(acc.x * inv, acc.y * inv);
    }
  }
  cluster_sync_all();  // no CTA leaves while another still reads its shared memory
}

}  // namespace dfl
