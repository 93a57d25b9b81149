// Per-warp compute pieces of the skinny GEMM Y[m][n] = sum_k W[n][k] X[m][k]
// (the block step's few rows: 8 block rows per request, 16 with the context
// rows).  Weights are the M side of a warp mma.sync m16n8k16 ("swap AB"): a
// warp owns 16 output features; the activations, staged in shared memory, are
// the n = 8 side.
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
//   S_j = sum_k (128+q_k) x_k,  X_j = sum_k x_k  (bf16 x as fed to the mma; X_j comes
//   from a second mma with an all-ones A operand).
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

enum : int { EPI_STORE = 0, EPI_RESID = 1, EPI_SWIGLU = 2, EPI_QKV = 3, EPI_DYNCONV = 4 };

// Fused epilogue of the q|k|v projection: per-head q/k RMSNorm, RoPE at the absolute
// position, block rows -> qb/kb/vb, context rows (t < n_new) -> the layer's paged cache.
struct QkvEpi {
  const uint16_t *qn, *kn;
  float eps;
  double log2_theta;
  int Bk, nq, nkv, Mb;
  const int32_t *seq_len, *n_new;
  uint16_t *qb, *kb, *vb;  // [Mb][heads][128]
  uint16_t *kc, *vc;       // [pages][nkv][16][128]
  const int32_t* page_table;
  int max_pages, num_pages;
  // Optional per-step tables (null: computed here): rope[row][j] = (cos, sin) of row's position
  // times theta^(-2j/128), rows [0, Mb) block rows then [Mb, 2Mb) context rows; rpage[ctx row] =
  // (page, slot) of its cache position, page -2 for rows past n_new, -1 for an unmapped page.
  const float2* rope;
  const int2* rpage;
  int* err;
};

// RoPE angle of position pos for frequency j: pos * theta^(-2j/128) reduced modulo 2 pi in double,
// then sin/cos in fp32.
DEVI float2 rope_cs(long long pos, int j, double log2_theta) {
  const double inv = exp2(-(2.0 * j / kHeadDim) * log2_theta);
  double a = (double)pos * inv;
  a -= 6.283185307179586 * rint(a / 6.283185307179586);
  float sn, cs;
  sincosf((float)a, &sn, &cs);
  return make_float2(cs, sn);
}

// One Q4_K group unit (16 rows x 256 k of one tile) against NT 8-row activation tiles.
// q: the lane's 64 bytes of 4-bit codes (mma fragment order), sc: its feature's scale record.
// Per 32-wide sub-block j: S = sum (128 + q) x by mma on the codes with the 0x4300 exponent
// (bf16 128 + q exactly), X = sum x by an mma with all-ones weights, then
// y += D*S - M*X with D = d*sc_j, M = dmin*m_j + 128*D.
// The 16-byte scale record of a feature row per 256-wide K unit: Q4_K's canonical record (d, dmin,
// 6-bit scales and mins), or for MLX 4-bit group-64 weights (mlx) four (scale, bias) bf16 pairs,
// one per 64-wide group: word g = scale | bias << 16, weight = scale * q + bias.
template <int NT>
DEVI void q4_unit(const uint4 (&q)[4], const uint4 sc, float2* coef, const uint8_t* Xs, int stride, int kbyte,
                  int ntact, float (&acc)[NT][4], int lane, bool mlx) {
  const int g = lane >> 2, t = lane & 3;
  // A = 1.0 in every slot: the mma then yields X_j = sum_k x_k (bf16 x, fp32 accumulate) per row
  const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};
  {
    // lane decodes (D_j, M_j) with weight = D_j * (128 + q) - M_j of feature lane/2, sub-blocks
    // 4*(lane&1) .. +3: Q4_K D = d*sc_j, M = dmin*m_j + 128*D; MLX D = scale, M = 128*scale - bias
    const int f = lane >> 1, jb = (lane & 1) * 4;
    __syncwarp();
    if (mlx) {
      const uint32_t w0 = (lane & 1) ? sc.z : sc.x, w1 = (lane & 1) ? sc.w : sc.y;  // groups jb/2, jb/2 + 1
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t wg = i < 2 ? w0 : w1;
        const float D = bf2f((uint16_t)(wg & 0xffffu)), B = bf2f((uint16_t)(wg >> 16));
        coef[(jb + i) * 16 + f] = make_float2(D, fmaf(128.f, D, -B));
      }
    } else {
      const float d = __half2float(__ushort_as_half((unsigned short)(sc.x & 0xffffu)));
      const float dm = __half2float(__ushort_as_half((unsigned short)(sc.x >> 16)));
      const uint32_t sb = (lane & 1) ? ((sc.y >> 24) | ((sc.z & 0xffffu) << 8)) : (sc.y & 0xffffffu);
      const uint32_t mb = (lane & 1) ? (sc.w >> 8) : ((sc.z >> 16) | ((sc.w & 0xffu) << 16));
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float D = d * (float)((sb >> (6 * i)) & 63u);
        const float M = fmaf(128.f, D, dm * (float)((mb >> (6 * i)) & 63u));
        coef[(jb + i) * 16 + f] = make_float2(D, M);
      }
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
        float s[4] = {0.f, 0.f, 0.f, 0.f}, xs[4] = {0.f, 0.f, 0.f, 0.f};
        mma16816(s, a0, bx.x, bx.y);
        mma16816(s, a1, bx.z, bx.w);
        mma16816(xs, ones, bx.x, bx.y);
        mma16816(xs, ones, bx.z, bx.w);
        // acc += D * S - M * X, two accumulators per packed FMA
        float2 a01 = make_float2(acc[nt][0], acc[nt][1]), a23 = make_float2(acc[nt][2], acc[nt][3]);
        a01 = ffma2(make_float2(-cg.y, -cg.y), make_float2(xs[0], xs[1]), a01);
        a01 = ffma2(make_float2(cg.x, cg.x), make_float2(s[0], s[1]), a01);
        a23 = ffma2(make_float2(-ch.y, -ch.y), make_float2(xs[2], xs[3]), a23);
        a23 = ffma2(make_float2(ch.x, ch.x), make_float2(s[2], s[3]), a23);
        acc[nt][0] = a01.x;
        acc[nt][1] = a01.y;
        acc[nt][2] = a23.x;
        acc[nt][3] = a23.y;
      }
    }
  }
}

// bf16 weights: one K step of NJ 32-wide sub-blocks = 2*NJ 16-byte vectors per lane (rows g, g+8).
template <int NT, int NJ>
DEVI void bf16_step(const uint4 (&w)[2 * NJ], const uint8_t* Xs, int stride, int kbyte, int ntact, float (&acc)[NT][4],
                    int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
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

// q/k RMSNorm + RoPE of one head of one row (lane holds dims 2L, 2L+1, 64+2L, 65+2L), then store.
// Operands of one (kind, row) epilogue that do not depend on the product, when the per-step
// tables are in use: the context row's cache slot, the q/k norm weights and the RoPE factors of
// this lane's dimensions.  Loaded before the split-K partials so that all come back together.
struct QkvPre {
  int2 dstpg;
  float w[4];
  float2 cs[2];
};

DEVI QkvPre qkv_prefetch(const QkvEpi& e, int kind, int row, int lane) {
  QkvPre q;
  q.dstpg = make_int2(0, 0);
  q.w[0] = q.w[1] = q.w[2] = q.w[3] = 1.f;
  q.cs[0] = q.cs[1] = make_float2(1.f, 0.f);
  if (!e.rope) return q;
  if (row >= e.Mb) q.dstpg = e.rpage[row - e.Mb];
  if (kind < 2) {
    const uint16_t* w = kind == 0 ? e.qn : e.kn;
    q.w[0] = bf2f(w[2 * lane]);
    q.w[1] = bf2f(w[2 * lane + 1]);
    q.w[2] = bf2f(w[64 + 2 * lane]);
    q.w[3] = bf2f(w[65 + 2 * lane]);
    q.cs[0] = e.rope[(size_t)row * 64 + 2 * lane];
    q.cs[1] = e.rope[(size_t)row * 64 + 2 * lane + 1];
  }
  return q;
}

// pre: qkv_prefetch of the same (kind, row).
DEVI void qkv_head_row(const QkvEpi& e, int kind, int head, int row, const float (&xin)[4], int lane,
                       const QkvPre& pre) {
  const bool ctx = row >= e.Mb;
  const int rr = ctx ? row - e.Mb : row;
  const int b = rr / e.Bk, t = rr % e.Bk;
  int L0 = 0, nn = 0;
  int2 dstpg = make_int2(0, 0);
  if (e.rope) {
    if (ctx) {
      dstpg = pre.dstpg;
      if (dstpg.x == -2) return;  // past the request's new rows
    }
  } else {
    L0 = e.seq_len[b];
    nn = e.n_new[b];
    if (ctx && t >= nn) return;
  }
  float x[4] = {xin[0], xin[1], xin[2], xin[3]};
  const int dims[4] = {2 * lane, 2 * lane + 1, 64 + 2 * lane, 65 + 2 * lane};
  if (kind < 2) {
    const uint16_t* w = kind == 0 ? e.qn : e.kn;
    const float ss = warp_sum(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]);
    const float rs = rsqrtf(ss / kHeadDim + e.eps);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = x[i] * rs * (e.rope ? pre.w[i] : bf2f(w[dims[i]]));
    const long long pos = ctx ? (long long)L0 + t : (long long)L0 + nn + t;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float2 c = e.rope ? pre.cs[i] : rope_cs(pos, dims[i], e.log2_theta);
      const float x0 = x[i], x1 = x[i + 2];
      x[i] = x0 * c.x - x1 * c.y;
      x[i + 2] = x1 * c.x + x0 * c.y;
    }
  }
  uint16_t* dst;
  if (!ctx) {
    uint16_t* base = kind == 0 ? e.qb : (kind == 1 ? e.kb : e.vb);
    const int nh = kind == 0 ? e.nq : e.nkv;
    dst = base + ((size_t)row * nh + head) * kHeadDim;
  } else {
    if (!e.rope) {
      const long long pos = (long long)L0 + t;
      const int lp = (int)(pos / kPage);
      const int pg = lp < e.max_pages ? e.page_table[(size_t)b * e.max_pages + lp] : -1;
      dstpg = make_int2(pg >= 0 && pg < e.num_pages ? pg : -1, (int)(pos % kPage));
    }
    if (dstpg.x < 0) {
      if (lane == 0) set_err(e.err, DFLASH2_DEV_PAGE);
      return;
    }
    dst = (kind == 1 ? e.kc : e.vc) + (((size_t)dstpg.x * e.nkv + head) * kPage + dstpg.y) * kHeadDim;
  }
  *reinterpret_cast<uint32_t*>(dst + 2 * lane) = pack_bf2(x[0], x[1]);
  *reinterpret_cast<uint32_t*>(dst + 64 + 2 * lane) = pack_bf2(x[2], x[3]);
}

// Placement of 16-row tile T of a matrix in a group-interleaved prepared buffer: tile T' = T + tile0
// sits in group T' / per_grp at slot slot0 + T' % per_grp; a group record of one K unit holds its 8
// slots back to back, so one bulk copy brings a whole group's unit.
// Tile T of a matrix goes to record grp = (T + tile0) / per_grp, position slot0 + (T + tile0) % per_grp
// of the `rec` tiles a record holds (per K unit s).
struct PrepPlace {
  int tile0, per_grp, slot0, rec;
};
DEVI size_t prep_offset(const PrepPlace& pl, int T, int s, int U, int unit_bytes) {
  const int tt = T + pl.tile0, grp = tt / pl.per_grp, slot = pl.slot0 + tt % pl.per_grp;
  return (((size_t)grp * U + s) * pl.rec + slot) * unit_bytes;
}

// Canonical Q4_K [N][K/256][144 B] -> prepared tiles (group records of 8 x 2304 B per super-block).
__global__ void k_q4k_prepare(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int N, int K, PrepPlace pl) {
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
  uint8_t* out = dst + prep_offset(pl, T, s, nsb, kQ4Bytes);
#pragma unroll
  for (int p = 0; p < 4; ++p)
    reinterpret_cast<uint4*>(out)[p * 32 + lane] = make_uint4(w[2 * p][0], w[2 * p][1], w[2 * p + 1][0], w[2 * p + 1][1]);
  if (lane < 16) {
    const uint8_t* b = src + ((size_t)(T * 16 + lane) * nsb + s) * 144;
    for (int i = 0; i < 16; ++i) out[2048 + lane * 16 + i] = b[i];
  }
}

// MLX 4-bit group-64 rows (per group of 64: 32 bytes of codes, low nibble first, then the bf16
// scale and bias) -> the same prepared records as Q4_K: the codes in mma fragment order and, per
// feature row, a 16-byte record of the unit's four (scale, bias) pairs.
__global__ void k_mlx4_prepare(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int N, int K, PrepPlace pl) {
  const int nsb = K / kUnit, ng = K / 64, s = blockIdx.x, T = blockIdx.y, lane = threadIdx.x;
  const int g = lane >> 2, t = lane & 3;
  const uint8_t* rg = src + (size_t)(T * 16 + g) * ng * 36;
  const uint8_t* rh = src + (size_t)(T * 16 + g + 8) * ng * 36;
  auto q = [&](const uint8_t* row, int e) -> uint32_t {
    const int k = s * kUnit + e;
    const uint32_t v = row[(k >> 6) * 36 + ((k & 63) >> 1)];
    return (k & 1) ? (v >> 4) : (v & 15u);
  };
  uint32_t w[8][2];
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int e = 32 * j + 8 * t + 4 * h;
      w[j][h] = q(rg, e) | (q(rh, e) << 4) | (q(rg, e + 2) << 8) | (q(rh, e + 2) << 12) | (q(rg, e + 1) << 16) |
                (q(rh, e + 1) << 20) | (q(rg, e + 3) << 24) | (q(rh, e + 3) << 28);
    }
  uint8_t* out = dst + prep_offset(pl, T, s, nsb, kQ4Bytes);
#pragma unroll
  for (int p = 0; p < 4; ++p)
    reinterpret_cast<uint4*>(out)[p * 32 + lane] = make_uint4(w[2 * p][0], w[2 * p][1], w[2 * p + 1][0], w[2 * p + 1][1]);
  if (lane < 16) {
    const uint8_t* row = src + (size_t)(T * 16 + lane) * ng * 36;
    uint32_t r[4];
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
      const uint8_t* gp = row + (size_t)(s * 4 + gi) * 36 + 32;
      r[gi] = (uint32_t)gp[0] | ((uint32_t)gp[1] << 8) | ((uint32_t)gp[2] << 16) | ((uint32_t)gp[3] << 24);
    }
    *reinterpret_cast<uint4*>(out + 2048 + lane * 16) = make_uint4(r[0], r[1], r[2], r[3]);
  }
}

// Q8_0 rows (blocks of 32: fp16 d, 32 signed codes) -> the prepared bf16 records: each weight d*q
// (exact in fp32) rounded once to bf16; the step then streams them as bf16 weights.
__global__ void k_q80_prepare(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int N, int K, PrepPlace pl) {
  const int S = K / 64, nb = K / 32, s = blockIdx.x, T = blockIdx.y, lane = threadIdx.x, g = lane >> 2, t = lane & 3;
  uint8_t* out = dst + prep_offset(pl, T, s, S, 2048);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint8_t* blk = src + ((size_t)(T * 16 + g + 8 * h) * nb + (size_t)s * 2 + j) * 34;
      const float d = __half2float(__ushort_as_half((unsigned short)(blk[0] | (blk[1] << 8))));
      uint32_t r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int k = t * 8 + 2 * i;
        r[i] = pack_bf2(d * (float)(int8_t)blk[2 + k], d * (float)(int8_t)blk[3 + k]);
      }
      *reinterpret_cast<uint4*>(out + j * 1024 + h * 512 + lane * 16) = make_uint4(r[0], r[1], r[2], r[3]);
    }
  }
}

// Canonical bf16 [N][K] -> prepared tiles (group records of 8 x 2048 B per 64-wide K step): for each
// 32-wide sub-block j, 512 bytes of lane (g, t)'s W[row g][32j + 8t ..], then 512 bytes for row g + 8.
__global__ void k_bf16_prepare(const uint16_t* __restrict__ src, uint8_t* __restrict__ dst, int N, int K,
                               PrepPlace pl) {
  const int S = K / 64, s = blockIdx.x, T = blockIdx.y, lane = threadIdx.x, g = lane >> 2, t = lane & 3;
  uint8_t* out = dst + prep_offset(pl, T, s, S, 2048);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const size_t k = (size_t)s * 64 + j * 32 + t * 8;
    *reinterpret_cast<uint4*>(out + j * 1024 + lane * 16) =
        *reinterpret_cast<const uint4*>(src + (size_t)(T * 16 + g) * K + k);
    *reinterpret_cast<uint4*>(out + j * 1024 + 512 + lane * 16) =
        *reinterpret_cast<const uint4*>(src + (size_t)(T * 16 + g + 8) * K + k);
  }
}

}  // namespace dfl
