// Row-wise kernels of the block step: embedding gather, residual + RMSNorm,
// two-tap dynamic convolution, SwiGLU combine, q/k norm + RoPE + cache append,
// greedy acceptance.
#pragma once
#include "common.cuh"

namespace dfl {

// h[r] = E[block_tokens[r]] (fp32); ids outside [0, V) flag DFLASH2_DEV_TOKEN and read row 0.
__global__ void k_embed(const int32_t* __restrict__ tok, const uint16_t* __restrict__ E, float* __restrict__ h,
                        int H, int V, int* err) {
  const int r = blockIdx.x;
  int id = tok[r];
  if (id < 0 || id >= V) {
    if (threadIdx.x == 0) set_err(err, DFLASH2_DEV_TOKEN);
    id = 0;
  }
  const uint16_t* e = E + (size_t)id * H;
  for (int c = threadIdx.x; c < H; c += blockDim.x) h[(size_t)r * H + c] = bf2f(e[c]);
}

struct NormParams {
  float* h;            // residual stream [rows][H]; read (+ partials) and written back, or null
  const float* part;   // partial sums [nsplit][rows][ldp] added to the row (from column pcol), or null
  int nsplit;
  long long split_stride;
  int ldp, pcol;
  const uint16_t* w;   // RMSNorm weight [H]
  float eps;
  int H;
  uint16_t* out_bf;    // normalised row as bf16 (mode-dependent row index), or null
  int ldob;
  float* out_f;        // normalised row as fp32 [rows][H], or null
  int mode;            // 0 plain; 1 context rows (zero rows t >= n_new); 2 final (rows t >= 1 -> b*(Bk-1)+t-1)
  const int32_t* n_new;
  int Bk;
};

// One CTA per row: v = h + sum_s part_s; h = v; y = v / sqrt(mean v^2 + eps) * w.
__global__ void __launch_bounds__(256) k_norm(NormParams p) {
  extern __shared__ float vrow[];
  __shared__ float red[8];
  const int r = blockIdx.x, H = p.H;
  const int b = r / p.Bk, t = r % p.Bk;
  if (p.mode == 1 && t >= p.n_new[b]) {
    for (int c = threadIdx.x; c < H; c += blockDim.x) p.out_bf[(size_t)r * p.ldob + c] = 0;
    return;
  }
  float ss = 0.f;
  for (int c = threadIdx.x; c < H; c += blockDim.x) {
    float v = p.h ? p.h[(size_t)r * H + c] : 0.f;
    if (p.part)
      for (int s = 0; s < p.nsplit; ++s) v += p.part[s * p.split_stride + (size_t)r * p.ldp + p.pcol + c];
    if (p.h) p.h[(size_t)r * H + c] = v;
    vrow[c] = v;
    ss += v * v;
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float rs = rsqrtf(red[0] / H + p.eps);
  int orow = r;
  if (p.mode == 2) {
    if (t == 0) return;
    orow = b * (p.Bk - 1) + t - 1;
  }
  for (int c = threadIdx.x; c < H; c += blockDim.x) {
    const float y = vrow[c] * rs * bf2f(p.w[c]);
    if (p.out_bf) p.out_bf[(size_t)orow * p.ldob + c] = f2bf(y);
    if (p.out_f) p.out_f[(size_t)r * H + c] = y;
  }
}

// y_t[c] = (s0[c] + tanh g_t[c/4]) x_t[c] + (s1[c] + tanh g_t[H/4 + c/4]) x_{t-1}[c], x_{-1} = 0.
__global__ void k_dynconv(const float* __restrict__ xf, const float* __restrict__ gpart, int nsplit,
                          long long split_stride, int ldg, const uint16_t* __restrict__ s0,
                          const uint16_t* __restrict__ s1, int H, int Bk, uint16_t* __restrict__ y) {
  const int r = blockIdx.x, t = r % Bk, G = H / 4;
  for (int c = threadIdx.x; c < H; c += blockDim.x) {
    float g0 = 0.f, g1 = 0.f;
    for (int s = 0; s < nsplit; ++s) {
      g0 += gpart[s * split_stride + (size_t)r * ldg + c / 4];
      g1 += gpart[s * split_stride + (size_t)r * ldg + G + c / 4];
    }
    const float xc = xf[(size_t)r * H + c];
    const float xp = t > 0 ? xf[(size_t)(r - 1) * H + c] : 0.f;
    y[(size_t)r * H + c] = f2bf((bf2f(s0[c]) + tanhf(g0)) * xc + (bf2f(s1[c]) + tanhf(g1)) * xp);
  }
}

// act[r][f] = silu(sum_s gate) * sum_s up; gate in columns [0, F), up in [F, 2F) of the partials.
__global__ void k_silu_mul(const float* __restrict__ part, int nsplit, long long split_stride, int ldp, int rows,
                           int F, uint16_t* __restrict__ act) {
  const size_t n = (size_t)rows * F;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t r = i / F, f = i % F;
    float g = 0.f, u = 0.f;
    for (int s = 0; s < nsplit; ++s) {
      g += part[s * split_stride + r * ldp + f];
      u += part[s * split_stride + r * ldp + F + f];
    }
    act[i] = f2bf(g / (1.f + __expf(-g)) * u);
  }
}

struct RopeParams {
  const float* part;  // q|k|v partial sums [nsplit][2*Mb][ldp]: rows [0,Mb) block, [Mb,2Mb) context
  int nsplit;
  long long split_stride;
  int ldp;
  const uint16_t *qn, *kn;
  float eps;
  double log2_theta;
  int Bk, nq, nkv, Mb;
  const int32_t *seq_len, *n_new;
  uint16_t *qb, *kb, *vb;   // [Mb][heads][128] bf16
  uint16_t *kc, *vc;        // this layer's cache [pages][nkv][16][128]
  const int32_t* page_table;
  int max_pages, num_pages;
  int* err;
};

// One warp per (row, head slot); slots: n_q query heads, n_kv key heads, n_kv value heads.
// Lane L holds dims {2L, 2L+1, 64+2L, 65+2L}: the RoPE pairs (i, i+64) stay inside the lane.
__global__ void k_qk_rope_append(RopeParams p) {
  const int lane = threadIdx.x & 31;
  const int slot = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int r = blockIdx.y;
  const int nslot = p.nq + 2 * p.nkv;
  if (slot >= nslot) return;
  const bool ctx = r >= p.Mb;
  const int rr = ctx ? r - p.Mb : r;
  const int b = rr / p.Bk, t = rr % p.Bk;
  const int L0 = p.seq_len[b], nn = p.n_new[b];
  if (ctx && (slot < p.nq || t >= nn)) return;
  int kind, head, col;
  if (slot < p.nq) { kind = 0; head = slot; col = slot * kHeadDim; }
  else if (slot < p.nq + p.nkv) { kind = 1; head = slot - p.nq; col = p.nq * kHeadDim + head * kHeadDim; }
  else { kind = 2; head = slot - p.nq - p.nkv; col = (p.nq + p.nkv) * kHeadDim + head * kHeadDim; }
  const int dims[4] = {2 * lane, 2 * lane + 1, 64 + 2 * lane, 65 + 2 * lane};
  float x[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float v = 0.f;
    for (int s = 0; s < p.nsplit; ++s) v += p.part[s * p.split_stride + (size_t)r * p.ldp + col + dims[i]];
    x[i] = v;
  }
  if (kind < 2) {
    const uint16_t* w = kind == 0 ? p.qn : p.kn;
    float ss = warp_sum(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]);
    const float rs = rsqrtf(ss / kHeadDim + p.eps);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = x[i] * rs * bf2f(w[dims[i]]);
    // RoPE (rotate-half) at the absolute position; angle reduced in double, rotated in fp32
    const long long pos = ctx ? (long long)L0 + t : (long long)L0 + nn + t;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int fi = dims[i];  // 0..63
      const double inv = exp2(-(2.0 * fi / kHeadDim) * p.log2_theta);
      double a = (double)pos * inv;
      a -= 6.283185307179586 * rint(a / 6.283185307179586);
      float sn, cs;
      sincosf((float)a, &sn, &cs);
      const float x0 = x[i], x1 = x[i + 2];
      x[i] = x0 * cs - x1 * sn;
      x[i + 2] = x1 * cs + x0 * sn;
    }
  }
  uint16_t* dst;
  if (!ctx) {
    uint16_t* base = kind == 0 ? p.qb : (kind == 1 ? p.kb : p.vb);
    const int nh = kind == 0 ? p.nq : p.nkv;
    dst = base + ((size_t)r * nh + head) * kHeadDim;
  } else {
    const long long pos = (long long)L0 + t;
    const int lp = (int)(pos / kPage);
    const int pg = lp < p.max_pages ? p.page_table[(size_t)b * p.max_pages + lp] : -1;
    if (pg < 0 || pg >= p.num_pages) {
      if (lane == 0) set_err(p.err, DFLASH2_DEV_PAGE);
      return;
    }
    uint16_t* base = kind == 1 ? p.kc : p.vc;
    dst = base + (((size_t)pg * p.nkv + head) * kPage + pos % kPage) * kHeadDim;
  }
  *reinterpret_cast<uint32_t*>(dst + 2 * lane) = pack_bf2(x[0], x[1]);
  *reinterpret_cast<uint32_t*>(dst + 64 + 2 * lane) = pack_bf2(x[2], x[3]);
}

__global__ void k_accept(const int32_t* __restrict__ draft, const int32_t* __restrict__ target, int B, int Bk,
                         int32_t* __restrict__ accepted, int32_t* __restrict__ emitted) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int D = Bk - 1;
  int n = 0;
  while (n < D && draft[b * D + n] == target[b * Bk + n]) ++n;
  accepted[b] = n;
  for (int i = 0; i < Bk; ++i) emitted[b * Bk + i] = i < n ? draft[b * D + i] : (i == n ? target[b * Bk + n] : -1);
}

}  // namespace dfl
