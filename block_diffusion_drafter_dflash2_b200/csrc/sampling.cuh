// Exact rejection-sampling acceptance of a drafted path for sampled decoding (MLX sidecar card,
// "Contents": lossless acceptance when sampling; Mindket listing, "For newcomers and experts").
// The selector picks its path deterministically, so the draft's distribution at a position is the
// point mass on its token unless the caller supplies one.  Rule: accept d_i with probability
// min(1, p_i(d_i) / q_i(d_i)), in order; at the first rejection emit a token drawn from
// max(0, p_i - q_i); after a full match emit one drawn from p_D.  Every decision is exact
// (integers, or an fp32 x fp32 product formed exactly in double), so it does not depend on the
// order of any sum: accept iff u * q(d) < p(d); the residual in 32-bit fixed point
// floor(max(0, r) * 2^32), its total T as a 64-bit integer, the threshold floor(u_s * T / 2^32),
// and the emitted token is the first whose running sum exceeds it.  fp32 values below the normal
// range count as zero (flushed by bit pattern, independent of the compiler's denormal mode).
#pragma once
#include "common.cuh"

namespace dfl {

constexpr int kSampThreads = 1024;

DEVI float flush32(float v) { return (__float_as_uint(v) & 0x7F800000u) == 0 ? 0.f : v; }
DEVI unsigned long long fixed32(float r) {
  return r > 0.f ? (unsigned long long)floor((double)r * 4294967296.0) : 0ull;
}
// residual of token x: p - q, p without the drafted token (point mass), or p (dtok < 0)
DEVI float residual(const float* __restrict__ p, const float* __restrict__ q, int dtok, int x) {
  if (dtok < 0) return flush32(__ldg(p + x));
  if (q) return flush32(__fsub_rn(flush32(__ldg(p + x)), flush32(__ldg(q + x))));
  return x == dtok ? flush32(__fsub_rn(flush32(__ldg(p + x)), 1.f)) : flush32(__ldg(p + x));
}

DEVI unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// p: [B][Bk][V], q: [B][D][V] or null, u_acc: [B][D], u_s: [B].  One CTA per request.
__global__ void __launch_bounds__(kSampThreads) k_accept_sampled(const int32_t* __restrict__ draft,
                                                                 const float* __restrict__ p,
                                                                 const float* __restrict__ q,
                                                                 const float* __restrict__ u_acc,
                                                                 const uint32_t* __restrict__ u_s, int Bk, int V,
                                                                 int32_t* __restrict__ accepted,
                                                                 int32_t* __restrict__ emitted) {
  constexpr int NW = kSampThreads / 32;
  __shared__ int s_n, s_tok, s_warp, s_dtok;
  __shared__ unsigned long long s_wsum[NW], s_pre[NW + 1];
  const int b = blockIdx.x, D = Bk - 1, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    int n = 0;
    while (n < D) {
      const int d = draft[(size_t)b * D + n];
      if (d < 0 || d >= V) break;  // outside the vocabulary: probability 0, rejected (never used as an index)
      const float* pr = p + ((size_t)b * Bk + n) * V;
      const double qd = q ? (double)flush32(q[((size_t)b * D + n) * V + d]) : 1.0;
      if ((double)flush32(u_acc[(size_t)b * D + n]) * qd < (double)flush32(pr[d])) ++n;
      else break;
    }
    s_n = n;
    s_dtok = n < D ? draft[(size_t)b * D + n] : -1;
    s_tok = -1;
    s_warp = -1;
  }
  __syncthreads();
  const int n = s_n;
  const float* pr = p + ((size_t)b * Bk + n) * V;
  const float* qr = (q && n < D) ? q + ((size_t)b * D + n) * V : nullptr;
  const int seg = (V + NW - 1) / NW, x0 = warp * seg, x1 = min(V, x0 + seg);
  int dtok = s_dtok;
  unsigned long long T = 0;
  for (int pass = 0; pass < 2; ++pass) {  // pass 1 only when the residual is empty: sample p
    unsigned long long acc = 0;
    for (int x = x0 + lane; x < x1; x += 32) acc += fixed32(residual(pr, qr, dtok, x));
    acc = warp_sum_u64(acc);
    if (lane == 0) s_wsum[warp] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned long long run = 0;
      for (int w = 0; w < NW; ++w) {
        s_pre[w] = run;
        run += s_wsum[w];
      }
      s_pre[NW] = run;
    }
    __syncthreads();
    T = s_pre[NW];
    if (T > 0 || dtok < 0) break;
    dtok = -1;
    __syncthreads();
  }
  if (T > 0) {
    const unsigned long long t = __umul64hi((unsigned long long)u_s[b] << 32, T);  // floor(u_s * T / 2^32)
    if (lane == 0 && s_pre[warp] <= t && t < s_pre[warp + 1]) s_warp = warp;
    __syncthreads();
    if (warp == s_warp) {
      unsigned long long run = s_pre[warp];
      for (int base = x0; base < x1; base += 32) {
        const int x = base + lane;
        unsigned long long v = x < x1 ? fixed32(residual(pr, qr, dtok, x)) : 0ull;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {  // inclusive scan over the 32 lanes
          const unsigned long long u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
        const unsigned m = __ballot_sync(0xffffffffu, run + v > t);
        if (m) {
          if (lane == 0) s_tok = base + __ffs(m) - 1;
          break;
        }
        run += __shfl_sync(0xffffffffu, v, 31);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int tok = T > 0 ? (s_tok >= 0 ? s_tok : V - 1) : 0;
    accepted[b] = n;
    for (int i = 0; i < Bk; ++i)
      emitted[(size_t)b * Bk + i] = i < n ? draft[(size_t)b * D + i] : (i == n ? tok : -1);
  }
}

}  // namespace dfl
