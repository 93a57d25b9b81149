// Skinny GEMM Y[m][n] = sum_k W[n][k] X[m][k] for the block step's few rows
// (8 block rows per request, 16 with the context rows), weights streamed once
// from HBM.  Weights are the M side of a warp mma.sync m16n8k16 ("swap AB"): a
// warp owns 16 output features and streams them along K; the activations,
// staged once per CTA in shared memory, are the n = 8 side.
//
// Q4_K (prepared layout, one 2304-byte record per 16-feature tile and
// 256-wide super-block): 2048 bytes of codes arranged so that lane (g, t)
// reads one 16-byte vector per pair of 32-wide sub-blocks holding exactly its
// mma A-fragment nibbles (rows g and g+8, k = 8t..8t+7 of each sub-block),
// followed by the 16 canonical 16-byte scale records of the tile's features.
// A nibble q becomes the bf16 value 128+q with one LOP3 (0x4300 | q); the
// offset and the sub-block scale/min are applied per 32-wide sub-block on the
// fp32 accumulators:
//   y += (d*sc_j) * S_j - (dmin*m_j + 128*d*sc_j) * X_j,
//   S_j = sum_k (128+q_k) x_k,  X_j = sum_k x_k  (bf16 x as fed to the mma).
// The logical k order inside an mma is permuted identically on A and B, which
// leaves the dot product unchanged.
#pragma once
#include "common.cuh"

namespace dfl {

struct GemvSeg {
  const uint8_t* W;  // prepared Q4_K tiles or bf16 [N][K]
  int tiles;         // N / 16
  int rows;          // activation rows this matrix is applied to (<= staged rows)
  int out_col;       // first output column
};

struct GemvParams {
  GemvSeg seg[3];
  int nseg;
  const uint16_t* X;  // bf16 activations [rows][ldx]
  int ldx;
  int rows_stage;     // rows staged in shared memory (max over segments)
  int K;              // reduction length (multiple of 256)
  int units_per_split;
  int kc_units;       // units staged per shared-memory chunk
  float* out;         // fp32 partial sums [split][rows][ldo]
  int ldo;
  long long split_stride;
  int m_group_rows;   // rows per grid.z group (64)
};

template <int NT>
struct GemvSmem {
  static constexpr int kRows = NT * 8;
};

DEVI int gemv_stride_bytes(int kc_units) { return kc_units * kUnit * 2 + 64; }

// Stage X[:, k0 : k0+cu*256] into shared memory (rows >= rows_valid zero-filled)
// and, for Q4_K, the 32-wide sums X_j.
template <int NT, bool Q4>
DEVI void gemv_stage(const GemvParams& p, const uint16_t* X, int rows_valid, int u0, int cu, uint8_t* Xs,
                     float* Xsum, int stride) {
  constexpr int R = NT * 8;
  const int vec_per_row = cu * kUnit / 8;  // 16-byte vectors
  for (int i = threadIdx.x; i < R * vec_per_row; i += blockDim.x) {
    int r = i / vec_per_row, v = i % vec_per_row;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < rows_valid) val = *reinterpret_cast<const uint4*>(X + (size_t)r * p.ldx + (size_t)u0 * kUnit + v * 8);
    *reinterpret_cast<uint4*>(Xs + r * stride + v * 16) = val;
  }
  if (Q4) {
    __syncthreads();
    const int nsub = cu * 8;
    for (int i = threadIdx.x; i < R * nsub; i += blockDim.x) {
      int r = i % R, j = i / R;
      const uint16_t* row = reinterpret_cast<const uint16_t*>(Xs + r * stride) + j * 32;
      float s = 0.f;
#pragma unroll 8
      for (int k = 0; k < 32; ++k) s += bf2f(row[k]);
      Xsum[j * R + r] = s;
    }
  }
}

template <int NT>
DEVI void q4_unit(const uint4 (&q)[4], const uint4 sc, float2* coef, const uint8_t* Xs, int stride,
                  const float* Xsum_u, int kbyte, int ntact, float (&acc)[NT][4], int lane) {
  constexpr int R = NT * 8;
  const int g = lane >> 2, t = lane & 3;
  {
    // lane decodes (d*sc_j, dmin*m_j + 128*d*sc_j) of feature lane/2, sub-blocks 4*(lane&1) .. +3
    const int f = lane >> 1, jb = (lane & 1) * 4;
    const float d = __half2float(__ushort_as_half((unsigned short)(sc.x & 0xffffu)));
    const float dm = __half2float(__ushort_as_half((unsigned short)(sc.x >> 16)));
    const uint32_t sb = (lane & 1) ? ((sc.y >> 24) | ((sc.z & 0xffffu) << 8)) : (sc.y & 0xffffffu);
    const uint32_t mb = (lane & 1) ? (sc.w >> 8) : ((sc.z >> 16) | ((sc.w & 0xffu) << 16));
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float D = d * (float)((sb >> (6 * i)) & 63u);
      const float M = fmaf(128.f, D, dm * (float)((mb >> (6 * i)) & 63u));
      coef[(jb + i) * 16 + f] = make_float2(D, M);
    }
    __syncwarp();
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t w0 = (j & 1) ? q[j >> 1].z : q[j >> 1].x;
    const uint32_t w1 = (j & 1) ? q[j >> 1].w : q[j >> 1].y;
    uint32_t a0[4], a1[4];
    a0[0] = (w0 & 0x000F000Fu) | 0x43004300u;
    a0[1] = ((w0 >> 4) & 0x000F000Fu) | 0x43004300u;
    a0[2] = ((w0 >> 8) & 0x000F000Fu) | 0x43004300u;
    a0[3] = ((w0 >> 12) & 0x000F000Fu) | 0x43004300u;
    a1[0] = (w1 & 0x000F000Fu) | 0x43004300u;
    a1[1] = ((w1 >> 4) & 0x000F000Fu) | 0x43004300u;
    a1[2] = ((w1 >> 8) & 0x000F000Fu) | 0x43004300u;
    a1[3] = ((w1 >> 12) & 0x000F000Fu) | 0x43004300u;
    const float2 cg = coef[j * 16 + g], ch = coef[j * 16 + g + 8];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      if (nt < ntact) {
        const uint4 bx = *reinterpret_cast<const uint4*>(Xs + (nt * 8 + g) * stride + kbyte + j * 64 + t * 16);
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        mma16816(s, a0, bx.x, bx.y);
        mma16816(s, a1, bx.z, bx.w);
        const float2 xs = *reinterpret_cast<const float2*>(Xsum_u + j * R + nt * 8 + 2 * t);
        acc[nt][0] = fmaf(cg.x, s[0], fmaf(-cg.y, xs.x, acc[nt][0]));
        acc[nt][1] = fmaf(cg.x, s[1], fmaf(-cg.y, xs.y, acc[nt][1]));
        acc[nt][2] = fmaf(ch.x, s[2], fmaf(-ch.y, xs.x, acc[nt][2]));
        acc[nt][3] = fmaf(ch.x, s[3], fmaf(-ch.y, xs.y, acc[nt][3]));
      }
    }
  }
}

// bf16 weights: one 128-wide K step = 8 16-byte vectors per lane (rows g, g+8; 4 sub-blocks of 32).
template <int NT>
DEVI void bf16_step(const uint4 (&w)[8], const uint8_t* Xs, int stride, int kbyte, int ntact, float (&acc)[NT][4],
                    int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 u = w[2 * j], v = w[2 * j + 1];
    const uint32_t a0[4] = {u.x, v.x, u.y, v.y};
    const uint32_t a1[4] = {u.z, v.z, u.w, v.w};
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      if (nt < ntact) {
        const uint4 bx = *reinterpret_cast<const uint4*>(Xs + (nt * 8 + g) * stride + kbyte + j * 64 + t * 16);
        mma16816(acc[nt], a0, bx.x, bx.y);
        mma16816(acc[nt], a1, bx.z, bx.w);
      }
    }
  }
}

template <int NT, bool Q4>
__global__ void __launch_bounds__(kWarps * 32) k_gemv(GemvParams p) {
  constexpr int R = NT * 8;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int stride = gemv_stride_bytes(p.kc_units);
  uint8_t* Xs = smem;
  float* Xsum = reinterpret_cast<float*>(smem + R * stride);
  float2* coef = reinterpret_cast<float2*>(Xsum + (Q4 ? p.kc_units * 8 * R : 0)) + warp * 128;

  // the warp's tile
  int gt = blockIdx.x * kWarps + warp, si = -1, tile = 0;
  {
    int acc_t = 0;
    for (int s = 0; s < p.nseg; ++s) {
      if (gt < acc_t + p.seg[s].tiles) {
        si = s;
        tile = gt - acc_t;
        break;
      }
      acc_t += p.seg[s].tiles;
    }
  }
  const int mz = blockIdx.z * p.m_group_rows;
  const uint16_t* X = p.X + (size_t)mz * p.ldx;
  int stage_rows = p.rows_stage - mz;
  stage_rows = stage_rows > R ? R : stage_rows;
  int my_rows = 0;
  const uint8_t* W = nullptr;
  int out_col = 0;
  if (si >= 0) {
    my_rows = p.seg[si].rows - mz;
    my_rows = my_rows > R ? R : (my_rows < 0 ? 0 : my_rows);
    W = p.seg[si].W;
    out_col = p.seg[si].out_col + tile * 16;
  }
  const int ntact = (my_rows + 7) >> 3;
  const bool active = si >= 0 && ntact > 0;

  const int nunits = p.K / kUnit;
  const int u_lo = blockIdx.y * p.units_per_split;
  int u_hi = u_lo + p.units_per_split;
  u_hi = u_hi > nunits ? nunits : u_hi;

  float acc[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

  for (int c0 = u_lo; c0 < u_hi; c0 += p.kc_units) {
    const int cu = (u_hi - c0) < p.kc_units ? (u_hi - c0) : p.kc_units;
    __syncthreads();
    gemv_stage<NT, Q4>(p, X, stage_rows, c0, cu, Xs, Xsum, stride);
    __syncthreads();
    if (!active) continue;
    if (Q4) {
      // stream this warp's tile: 2304 bytes per super-block, two super-blocks in flight
      const uint8_t* base = W + ((size_t)tile * nunits) * kQ4Bytes;
      uint4 qa[4], qb[4], sa, sb;
      auto load = [&](uint4 (&q)[4], uint4& s, int u) {
        const uint8_t* b = base + (size_t)u * kQ4Bytes;
#pragma unroll
        for (int i = 0; i < 4; ++i) q[i] = ldg_stream(b + (i * 32 + lane) * 16);
        s = ldg_stream(b + 2048 + (lane >> 1) * 16);
      };
      load(qa, sa, c0);
      if (c0 + 1 < c0 + cu) load(qb, sb, c0 + 1);
      for (int u = c0; u < c0 + cu; u += 2) {
        q4_unit<NT>(qa, sa, coef, Xs, stride, Xsum + (u - c0) * 8 * R, (u - c0) * 512, ntact, acc, lane);
        if (u + 2 < c0 + cu) load(qa, sa, u + 2);
        if (u + 1 < c0 + cu) {
          q4_unit<NT>(qb, sb, coef, Xs, stride, Xsum + (u + 1 - c0) * 8 * R, (u + 1 - c0) * 512, ntact, acc, lane);
          if (u + 3 < c0 + cu) load(qb, sb, u + 3);
        }
      }
    } else {
      const uint16_t* Wr = reinterpret_cast<const uint16_t*>(W) + (size_t)(tile * 16 + g) * p.K;
      const size_t row8 = (size_t)8 * p.K;
      const int s_lo = c0 * 2, s_hi = (c0 + cu) * 2;  // 128-wide steps
      uint4 wa[8], wb[8];
      auto load = [&](uint4 (&w)[8], int s) {
        const uint16_t* b = Wr + (size_t)s * 128 + t * 8;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          w[2 * j] = ldg_stream(b + j * 32);
          w[2 * j + 1] = ldg_stream(b + row8 + j * 32);
        }
      };
      load(wa, s_lo);
      if (s_lo + 1 < s_hi) load(wb, s_lo + 1);
      for (int s = s_lo; s < s_hi; s += 2) {
        bf16_step<NT>(wa, Xs, stride, (s - s_lo) * 256, ntact, acc, lane);
        if (s + 2 < s_hi) load(wa, s + 2);
        if (s + 1 < s_hi) {
          bf16_step<NT>(wb, Xs, stride, (s + 1 - s_lo) * 256, ntact, acc, lane);
          if (s + 3 < s_hi) load(wb, s + 3);
        }
      }
    }
  }
  if (!active) return;
  float* out = p.out + (size_t)blockIdx.y * p.split_stride + (size_t)mz * p.ldo;
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

// Canonical Q4_K [N][K/256][144 B] -> prepared tiles [N/16][K/256][2304 B].
__global__ void k_q4k_prepare(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int N, int K) {
  const int nsb = K / kUnit, s = blockIdx.x, T = blockIdx.y, lane = threadIdx.x;
  const int g = lane >> 2, t = lane & 3;
  const uint8_t* bg = src + ((size_t)(T * 16 + g) * nsb + s) * 144;
  const uint8_t* bh = src + ((size_t)(T * 16 + g + 8) * nsb + s) * 144;
  auto q = [](const uint8_t* b, int e) -> uint32_t {
    const uint32_t v = b[16 + (e >> 1)];
    return (e & 1) ? (v >> 4) : (v & 15u);
  };
  uint32_t w[8][2];
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int e = 32 * j + 8 * t + 4 * h;
      // nibble slots: 0:(g,e) 4:(g,e+1) 1:(g+8,e) 5:(g+8,e+1) 2:(g,e+2) 6:(g,e+3) 3:(g+8,e+2) 7:(g+8,e+3)
      w[j][h] = q(bg, e) | (q(bh, e) << 4) | (q(bg, e + 2) << 8) | (q(bh, e + 2) << 12) | (q(bg, e + 1) << 16) |
                (q(bh, e + 1) << 20) | (q(bg, e + 3) << 24) | (q(bh, e + 3) << 28);
    }
  uint8_t* out = dst + ((size_t)T * nsb + s) * kQ4Bytes;
#pragma unroll
  for (int p = 0; p < 4; ++p)
    reinterpret_cast<uint4*>(out)[p * 32 + lane] = make_uint4(w[2 * p][0], w[2 * p][1], w[2 * p + 1][0], w[2 * p + 1][1]);
  if (lane < 16) {
    const uint8_t* b = src + ((size_t)(T * 16 + lane) * nsb + s) * 144;
    for (int i = 0; i < 16; ++i) out[2048 + lane * 16 + i] = b[i];
  }
}

}  // namespace dfl
