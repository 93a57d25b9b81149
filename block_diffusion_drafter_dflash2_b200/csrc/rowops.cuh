// Row-wise kernels of the block step: embedding gather, RMSNorm, greedy acceptance.
#pragma once
#include "common.cuh"
#include "gemv.cuh"

namespace dfl {

// h[r] = E[block_tokens[r]] (fp32); ids outside [0, V) flag DFLASH2_DEV_TOKEN and read row 0.
// Also the first RMSNorm's inputs: hw[r] = bf16(h[r] * w) and the row's sums of squares per
// 32-column quarter, ssp[q][ldr] (the consumer applies the row scale).
// Per-step RoPE tables (QkvEpi::rope / rpage), filled by the embedding kernel: CTA r does block
// row r and context row r.
struct RopeInit {
  const int32_t *seq_len, *n_new, *page_table;
  int max_pages, num_pages, Bk, Mb;
  double log2_theta;
  float2* rope;
  int2* rpage;
};

__global__ void k_embed(const int32_t* __restrict__ tok, const uint16_t* __restrict__ E, float* __restrict__ h,
                        int H, int V, int* err, uint16_t* __restrict__ hw, const uint16_t* __restrict__ w,
                        float* __restrict__ ssp, int ldr, RopeInit ri) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (ri.rope && threadIdx.x < 128) {
    const int b = r / ri.Bk, t = r % ri.Bk, j = threadIdx.x & 63;
    const long long L0 = ri.seq_len[b], nn = ri.n_new[b];
    const bool ctxrow = threadIdx.x >= 64;
    const long long pos = ctxrow ? L0 + t : L0 + nn + t;
    ri.rope[((size_t)(ctxrow ? ri.Mb + r : r)) * 64 + j] = rope_cs(pos, j, ri.log2_theta);
    if (ctxrow && j == 0) {
      int2 d = make_int2(-2, 0);
      if (t < nn) {
        const int lp = (int)(pos / kPage);
        const int pg = lp < ri.max_pages ? ri.page_table[(size_t)b * ri.max_pages + lp] : -1;
        d = make_int2(pg >= 0 && pg < ri.num_pages ? pg : -1, (int)(pos % kPage));
      }
      ri.rpage[r] = d;
    }
  }
  int id = tok[r];
  if (id < 0 || id >= V) {
    if (threadIdx.x == 0) set_err(err, DFLASH2_DEV_TOKEN);
    id = 0;
  }
  const uint16_t* erow = E + (size_t)id * H;
  const uint4* e = reinterpret_cast<const uint4*>(erow);
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    const uint4 v = e[c], wv = reinterpret_cast<const uint4*>(w)[c];
    float4* o = reinterpret_cast<float4*>(h + (size_t)r * H + c * 8);
    o[0] = make_float4(bf2f(v.x & 0xffff), bf2f(v.x >> 16), bf2f(v.y & 0xffff), bf2f(v.y >> 16));
    o[1] = make_float4(bf2f(v.z & 0xffff), bf2f(v.z >> 16), bf2f(v.w & 0xffff), bf2f(v.w >> 16));
    const uint32_t vv[4] = {v.x, v.y, v.z, v.w}, ww[4] = {wv.x, wv.y, wv.z, wv.w};
    uint32_t out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      out[k] = pack_bf2(bf2f(vv[k] & 0xffff) * bf2f(ww[k] & 0xffff), bf2f(vv[k] >> 16) * bf2f(ww[k] >> 16));
    reinterpret_cast<uint4*>(hw + (size_t)r * H)[c] = make_uint4(out[0], out[1], out[2], out[3]);
  }
  for (int q = warp; q < H / 32; q += blockDim.x >> 5) {
    const float v = bf2f(erow[q * 32 + lane]);
    const float s = warp_sum(v * v);
    if (lane == 0) ssp[(size_t)q * ldr + r] = s;
  }
}

struct NormParams {
  const float* in;     // fp32 rows [rows][H]: the residual stream or the fc output
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

// One CTA per row: y = x / sqrt(mean x^2 + eps) * w, 16-byte loads.
__global__ void __launch_bounds__(256) k_norm(NormParams p) {
  extern __shared__ float4 vrow4[];
  __shared__ float red[8];
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x, H4 = p.H / 4;
  const int b = r / p.Bk, t = r % p.Bk;
  if (p.mode == 1 && t >= p.n_new[b]) {
    for (int c = threadIdx.x; c < H4; c += blockDim.x)
      *reinterpret_cast<uint2*>(p.out_bf + (size_t)r * p.ldob + 4 * c) = make_uint2(0, 0);
    return;
  }
  if (p.mode == 2 && t == 0) return;
  const float4* __restrict__ in = reinterpret_cast<const float4*>(p.in + (size_t)r * p.H);
  float ss = 0.f;
  {
    float4 v4[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int c = threadIdx.x + k * blockDim.x;
      if (c < H4) v4[k] = in[c];
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int c = threadIdx.x + k * blockDim.x;
      if (c >= H4) break;
      vrow4[c] = v4[k];
      ss += v4[k].x * v4[k].x + v4[k].y * v4[k].y + v4[k].z * v4[k].z + v4[k].w * v4[k].w;
    }
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
  const float rs = rsqrtf(red[0] / p.H + p.eps);
  const int orow = p.mode == 2 ? b * (p.Bk - 1) + t - 1 : r;
  // the weight loads go first: with the stores in the same loop the compiler cannot prove the
  // global pointers apart and would serialise a load->store round trip per iteration
  const uint2* __restrict__ w2 = reinterpret_cast<const uint2*>(p.w);
  uint16_t* __restrict__ ob = p.out_bf ? p.out_bf + (size_t)orow * p.ldob : nullptr;
  float4* __restrict__ of = p.out_f ? reinterpret_cast<float4*>(p.out_f + (size_t)r * p.H) : nullptr;
  constexpr int kMaxIt = 16;  // H <= 16384 over 256 threads
  uint2 wv[kMaxIt];
#pragma unroll
  for (int k = 0; k < kMaxIt; ++k) {
    const int c = threadIdx.x + k * blockDim.x;
    if (c < H4) wv[k] = w2[c];
  }
#pragma unroll
  for (int k = 0; k < kMaxIt; ++k) {
    const int c = threadIdx.x + k * blockDim.x;
    if (c >= H4) break;
    const float4 v = vrow4[c];
    const float y0 = v.x * rs * bf2f(wv[k].x & 0xffff), y1 = v.y * rs * bf2f(wv[k].x >> 16);
    const float y2 = v.z * rs * bf2f(wv[k].y & 0xffff), y3 = v.w * rs * bf2f(wv[k].y >> 16);
    if (ob) *reinterpret_cast<uint2*>(ob + 4 * c) = make_uint2(pack_bf2(y0, y1), pack_bf2(y2, y3));
    if (of) of[c] = make_float4(y0, y1, y2, y3);
  }
}

// Greedy acceptance of request b: the longest prefix on which draft and target agree, then the
// emitted tokens (accepted drafts, the target's token after them, -1 padding).
DEVI void accept_request(const int32_t* __restrict__ draft, const int32_t* __restrict__ target, int b, int Bk,
                         int32_t* __restrict__ accepted, int32_t* __restrict__ emitted) {
  const int D = Bk - 1;
  int n = 0;
  while (n < D && draft[b * D + n] == target[b * Bk + n]) ++n;
  accepted[b] = n;
  for (int i = 0; i < Bk; ++i) emitted[b * Bk + i] = i < n ? draft[b * D + i] : (i == n ? target[b * Bk + n] : -1);
}

__global__ void k_accept(const int32_t* __restrict__ draft, const int32_t* __restrict__ target, int B, int Bk,
                         int32_t* __restrict__ accepted, int32_t* __restrict__ emitted) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) accept_request(draft, target, b, Bk, accepted, emitted);
}

// Acceptance that also writes the next round's draft inputs: n_new_next[b] = accepted + 1 (the
// accepted drafted tokens and the target's own token become the next context rows) and the next
// block = [target[b][accepted], mask_id, ...].  One thread per request; the next-round buffers may
// be the step's own n_new / block_tokens (the step that read them has finished on this stream).
__global__ void k_accept_chain(const int32_t* __restrict__ draft, const int32_t* __restrict__ target, int B, int Bk,
                               int32_t mask_id, int32_t* __restrict__ accepted, int32_t* __restrict__ emitted,
                               int32_t* __restrict__ n_new_next, int32_t* __restrict__ btok_next) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  accept_request(draft, target, b, Bk, accepted, emitted);
  const int n = accepted[b];
  n_new_next[b] = n + 1;
  btok_next[(size_t)b * Bk] = target[(size_t)b * Bk + n];
  for (int i = 1; i < Bk; ++i) btok_next[(size_t)b * Bk + i] = mask_id;
}

// Host-buffer round, page-locked buffers (device-addressable): the small inputs (n_new [B], block
// tokens and targets [Mb]) gathered into the workspace by one kernel instead of three copies.
__global__ void k_stage_host_inputs(const int32_t* __restrict__ n_new_h, const int32_t* __restrict__ btok_h,
                                    const int32_t* __restrict__ tgt_h, int B, int Mb, int32_t* __restrict__ n_new,
                                    int32_t* __restrict__ btok, int32_t* __restrict__ tgt) {
  for (int i = threadIdx.x; i < B; i += blockDim.x) n_new[i] = n_new_h[i];
  for (int i = threadIdx.x; i < Mb; i += blockDim.x) {
    btok[i] = btok_h[i];
    tgt[i] = tgt_h[i];
  }
}

// ... and the round's results written straight to them: the draft path and scores [B][Bk-1], the
// acceptance (accepted [B], emitted [B][Bk]) and, when err_h is set, the device error word.
__global__ void k_accept_to_host(const int32_t* __restrict__ draft, const float* __restrict__ scores,
                                 const int32_t* __restrict__ target, int B, int Bk, const int* __restrict__ err,
                                 int32_t* __restrict__ path_h, float* __restrict__ scores_h,
                                 int32_t* __restrict__ accepted_h, int32_t* __restrict__ emitted_h,
                                 int32_t* __restrict__ err_h) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < B * (Bk - 1)) {
    path_h[i] = draft[i];
    scores_h[i] = scores[i];
  }
  if (i < B) accept_request(draft, target, i, Bk, accepted_h, emitted_h);
  if (i == 0 && err_h) *err_h = *err;
}

}  // namespace dfl
