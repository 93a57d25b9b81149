// C ABI of the DFlash 2 drafter block step (include/dflash2.h): argument
// validation, workspace layout and the launch sequence of the sm_100a kernels.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>

#include "attention.cuh"
#include "attn_stream.cuh"
#include "common.cuh"
#include "gemv.cuh"
#include "rowops.cuh"
#include "sampling.cuh"
#include "selector.cuh"
#include "stream.cuh"
#include "umma.cuh"

using namespace dfl;

namespace {

struct GemvPlan {
  int NT = 1, R = 8, groups = 1, mgroups = 1, U = 1, P = 1, kc_units = 1, max_pieces = 1;
  long long W = 1;
  size_t smem = 0;
  bool umma = false;  // tensor-core (tcgen05) product + fix-up instead of the streaming engine
  int un = 0;         // its activation rows per tile (MMA N): all rows up to 256, rounded up to 16
  bool upair = false; // its tiles are two 256-row halves (more than 256 rows)
  bool mlx = false;   // 4-bit records hold MLX group-64 (scale, bias) pairs
  int rows = 0, K = 0;
};

// From this many activation rows on a product runs on the tcgen05 tensor cores (k_umma, the
// tile's N = the rows rounded up to 16): the streaming engine's warps re-read every activation
// fragment from shared memory for each weight fragment, which at 32 rows and more costs more than
// the tensor-core path's dequantisation (measured: full shape at 4, 5 and 8 requests 2.29 -> 2.04,
// 2.97 -> 2.11 and 3.67 -> 2.14 ms per step; at 24 rows the streaming engine is still ahead).
constexpr int kUmmaMinRows = 32;

struct Plan {
  int B, Bk, D, Mb, H, F, HQ, HKV, T, V, R, nsm, G, QV, QVP, MT, NC;
  int attn_ntk;  // > 0: attention as one cluster kernel, attn_kg key groups of 8*attn_ntk keys per CTA; 0: chunks + merge
  int attn_kg;
  bool attn_stream;  // streaming CTAs per (request, kv head) with TMA-staged pages (many requests)
  int attn_split;    // its cluster size: CTAs sharing one (request, kv head)'s window
  bool q4, mlx;
  GemvPlan fc, dc, qkv, o, gu, dn;
  size_t off_cfv, off_cfi, off_ssp, off_tau, off_hpart, off_rope, off_rpage;
  int lm_nparts, lm_rows, lm_groups;
  size_t lm_smem;
  bool lm_umma;                  // output head on the tensor cores (k_umma_head)
  int lm_uP, lm_unrt, lm_unrec;  // its grid, row tiles of 256 and head records
  int sel_parts;                 // candidate lists per row the selector merges
  size_t off_err, off_h, off_xf, off_xb, off_yb, off_part, off_qb, off_kb, off_vb, off_ao, off_aml, off_ob,
      off_act, off_hn, off_cv, off_ci, off_z, off_g, off_ctr, off_rsg;
  size_t ctr_layer[5], ctr_per_layer, ctr_fc, ctr_head, ctr_sel, ctr_total;
  size_t off_s_taps, off_s_nnew, off_s_btok, off_s_tgt, off_s_path, off_s_scores, off_s_acc, off_s_emit;
  size_t step_bytes, total;
};

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

constexpr int kSmemLimit = 227 * 1024;
constexpr int kStaticSmem = 2048;  // mbarriers and flags of the streaming kernels

// tiles: 16-row tiles over all segments; paired: gate/up (groups = tiles / 8 still, 4 + 4 tiles each)
GemvPlan plan_gemv(int tiles, int rows, int K, bool q4, int nsm) {
  GemvPlan g;
  g.rows = rows;
  g.K = K;
  if (rows >= kUmmaMinRows) {
    g.umma = true;
    g.R = kUmmaRows;
    g.un = rows >= kUmmaRows ? kUmmaRows : (rows + 15) / 16 * 16;
    g.NT = 8;
    g.groups = (tiles + kConsumers - 1) / kConsumers;
    g.U = K / (q4 ? Ring<true>::kUnitK : Ring<false>::kUnitK);
    // 4-bit weights and more than 256 rows: tiles of two 256-row halves, each weight stage
    // dequantised once for both, as long as every CTA still gets 8 or more K units (measured: bf16
    // weights, and products as small as W_o, run faster with double-buffered 256-row tiles)
    const int mg1 = (rows + kUmmaRows - 1) / kUmmaRows, mg2 = (rows + 2 * kUmmaRows - 1) / (2 * kUmmaRows);
    g.upair = q4 && rows > kUmmaRows && (long long)g.groups * mg2 * g.U >= 8LL * nsm;
    g.mgroups = g.upair ? mg2 : mg1;
    g.W = (long long)g.groups * g.mgroups * g.U;
    g.P = (int)std::min<long long>(nsm, g.W);
    g.max_pieces = (int)((long long)(g.U - 1) * g.P / g.W) + 2;
    g.kc_units = g.U;
    g.smem = g.upair ? kUmmaPairSmem : kUmmaSmem;
    return g;
  }
  g.R = rows <= 8 ? 8 : rows <= 16 ? 16 : rows <= 32 ? 32 : 64;
  g.NT = g.R / 8;
  g.mgroups = g.R == 64 ? (rows + 63) / 64 : 1;
  g.groups = (tiles + kConsumers - 1) / kConsumers;
  const int unitK = q4 ? Ring<true>::kUnitK : Ring<false>::kUnitK, slot = q4 ? Ring<true>::kSlot : Ring<false>::kSlot;
  const int ns = q4 ? Ring<true>::kNS : Ring<false>::kNS;
  g.U = K / unitK;
  g.W = (long long)g.groups * g.mgroups * g.U;
  g.P = (int)std::min<long long>(nsm, g.W);
  g.max_pieces = (int)((long long)(g.U - 1) * g.P / g.W) + 2;
  const int ring = ns * slot;
  const int per_unit = g.R * unitK * 2;
  const int extra = kGemvConsumers * 1024 + kConsumers * 32 * g.NT * 4 * 4;  // per-warp scale tables, set reduction
  const int budget = kSmemLimit - kStaticSmem - ring - extra - 64 * g.R;
  g.kc_units = std::max(1, std::min(g.U, budget / per_unit));
  g.smem = (size_t)ring + (size_t)g.R * (g.kc_units * unitK * 2 + 64) + extra;
  return g;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Device address of a page-locked host buffer (under unified addressing every page-locked
// allocation is mapped into the device's address space), or null for pageable or misaligned memory.
void* host_mapped(const void* h) {
  if (!h || ((uintptr_t)h & 3u)) return nullptr;
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, h) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

bool cfg_ok(const dflash2_config* c) {
  if (!c) return false;
  const long long HQ = (long long)c->n_q * c->head_dim;
  return c->layers >= 1 && c->layers <= DFLASH2_MAX_LAYERS && c->head_dim == kHeadDim && c->page_size == kPage &&
         c->topk == kTopK && c->block >= 2 && c->block <= kMaxD + 1 && c->n_kv >= 1 && c->n_q % c->n_kv == 0 &&
         (c->n_q / c->n_kv) * c->block <= 64 && c->hidden % kUnit == 0 && c->ffn % kUnit == 0 &&
         HQ % kUnit == 0 && ((long long)c->n_taps * c->hidden) % kUnit == 0 && c->n_taps >= 1 &&
         c->vocab % 16 == 0 && c->vocab > 0 && c->rank % 16 == 0 && c->rank >= 16 && c->rank <= kMaxR &&
         c->window >= 1 && c->window <= 4032 && c->hidden <= 16384 && (c->wfmt >= 0 && c->wfmt <= 3) && c->rope_theta > 0.f &&
         c->rms_eps >= 0.f;
}

// The output head's launch shape for Vh head rows (the whole vocabulary, or a shard of it) plus the
// selector projection.
void plan_head(Plan& p, int Vh) {
  const int lm_tiles = Vh / 16 + p.R / 16;
  // the streaming head takes any number of rows in groups of 8 (one launch, a CTA per group and
  // vocabulary part)
  p.lm_groups = (p.lm_rows + 7) / 8;
  p.lm_smem = (size_t)kHeadNS * kHeadSlot + (size_t)8 * (p.H * 2 + 64) + (size_t)kGemvConsumers * 8 * kTopK * 8;
  p.lm_nparts = (int)std::min<long long>(p.nsm, (long long)((lm_tiles + kHeadTiles - 1) / kHeadTiles) * (p.H / 64));
  // more than one group of 8 drafted rows: the head is a dense contraction on the tensor cores
  p.lm_umma = p.lm_rows > 8;
  p.lm_unrt = (p.lm_rows + 255) / 256;
  p.lm_unrec = (lm_tiles + kHeadTiles - 1) / kHeadTiles;
  p.lm_uP = std::max(1, p.nsm / p.lm_unrt) * p.lm_unrt;
  p.sel_parts = p.lm_umma ? p.lm_uP / p.lm_unrt : p.lm_nparts;
}

Plan make_plan(const dflash2_config* c, int B) {
  Plan p;
  p.B = B;
  p.Bk = c->block;
  p.D = c->block - 1;
  p.Mb = B * c->block;
  p.H = c->hidden;
  p.F = c->ffn;
  p.HQ = c->n_q * kHeadDim;
  p.HKV = c->n_kv * kHeadDim;
  p.T = c->n_taps;
  p.V = c->vocab;
  p.R = c->rank;
  p.nsm = device_sms();
  p.q4 = c->wfmt == 0 || c->wfmt == 2;  // 4-bit records (Q4_K or MLX group-64); bf16 and Q8_0 stream bf16
  p.mlx = c->wfmt == 2;
  p.G = c->n_q / c->n_kv;
  p.QV = p.G * p.Bk;
  p.QVP = (p.QV + 15) / 16 * 16;
  p.MT = p.QVP / 16;
  p.NC = (c->window + kPage - 2 + kAttnKeys - 1) / kAttnKeys;
  {
    // the cluster's 8 CTAs cover the window's keys (page aligned) and the block's keys
    const int need = (c->window + kPage - 2 + p.Bk + kClusterCtas - 1) / kClusterCtas;
    p.attn_ntk = 0;
    p.attn_kg = 4;
    if (p.MT <= 2) {
      for (int ntk : {4, 8})
        if (32 * ntk >= need) {
          p.attn_ntk = ntk;
          break;
        }
      if (!p.attn_ntk && 6 * 48 >= need) {  // 6 key groups of 48 keys: 12 warps per CTA
        p.attn_ntk = 6;
        p.attn_kg = 6;
      }
      if (!p.attn_ntk)
        for (int ntk : {10, 12})
          if (32 * ntk >= need) {
            p.attn_ntk = ntk;
            break;
          }
    }
  }
  // With 8 or more requests the (request, kv head) pairs fill the SMs two deep, and a CTA that keeps
  // its window's pages streaming beats clusters that each pay the whole load-compute-merge latency.
  p.attn_stream = B >= kAttnStreamMinBatch && p.QV <= 32;
  // CTAs per (request, kv head) for the streaming kernel: the fewest (a power of two, at most 8)
  // that give about two CTAs per SM
  p.attn_split = 1;
  while (p.attn_split < 8 && (long long)B * c->n_kv * p.attn_split * 5 < 4LL * 2 * p.nsm) p.attn_split *= 2;
  p.fc = plan_gemv(p.H / 16, p.Mb, p.T * p.H, p.q4, p.nsm);
  p.dc = plan_gemv((p.H / 2) / 16, p.Mb, p.H, false, p.nsm);
  p.qkv = plan_gemv((p.HQ + 2 * p.HKV) / 16, 2 * p.Mb, p.H, p.q4, p.nsm);
  p.o = plan_gemv(p.H / 16, p.Mb, p.HQ, p.q4, p.nsm);
  p.gu = plan_gemv(2 * p.F / 16, p.Mb, p.H, p.q4, p.nsm);
  p.dn = plan_gemv(p.H / 16, p.Mb, p.F, p.q4, p.nsm);
  for (GemvPlan* g : {&p.fc, &p.dc, &p.qkv, &p.o, &p.gu, &p.dn}) g->mlx = p.mlx;
  p.lm_rows = B * p.D;
  plan_head(p, p.V);
  const int lm_tiles = p.V / 16 + p.R / 16;

  auto part_bytes = [&](const GemvPlan& g, int rows, int ldo) { return (size_t)g.max_pieces * rows * ldo * 4; };
  size_t part = 0;
  part = std::max(part, part_bytes(p.fc, p.Mb, p.H));
  part = std::max(part, part_bytes(p.dc, p.Mb, p.H / 2));
  part = std::max(part, part_bytes(p.qkv, 2 * p.Mb, p.HQ + 2 * p.HKV));
  part = std::max(part, part_bytes(p.o, p.Mb, p.H));
  part = std::max(part, part_bytes(p.gu, p.Mb, 2 * p.F));
  part = std::max(part, part_bytes(p.dn, p.Mb, p.H));
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t r = o;
    o = align256(o + bytes);
    return r;
  };
  p.off_err = take(256);
  p.off_h = take((size_t)p.Mb * p.H * 4);
  p.off_xf = take((size_t)p.Mb * p.H * 4);
  p.off_xb = take((size_t)p.Mb * p.H * 2);
  p.off_yb = take((size_t)2 * p.Mb * p.H * 2);
  p.off_part = take(part);
  p.off_qb = take((size_t)p.Mb * p.HQ * 2);
  p.off_kb = take((size_t)p.Mb * p.HKV * 2);
  p.off_vb = take((size_t)p.Mb * p.HKV * 2);
  const size_t nchunk = (size_t)B * c->n_kv * (p.NC + 1) * p.QVP;
  p.off_ao = take(nchunk * kHeadDim * 4);
  p.off_aml = take(nchunk * 2 * 4);
  p.off_ob = take((size_t)p.Mb * p.HQ * 2);
  p.off_act = take((size_t)p.Mb * p.F * 2);
  p.off_hn = take((size_t)std::max(p.lm_rows, 1) * p.H * 2);
  const size_t nlists = (size_t)std::max(p.lm_nparts, p.sel_parts);
  p.off_cv = take(nlists * p.lm_rows * kTopK * 4);
  p.off_ci = take(nlists * p.lm_rows * kTopK * 4);
  p.off_cfv = take((size_t)p.lm_rows * kTopK * 4);
  p.off_cfi = take((size_t)p.lm_rows * kTopK * 4);
  p.off_ssp = take((size_t)(p.H / 128) * 4 * p.Mb * 4);
  p.off_tau = take((size_t)p.lm_rows * kTopK * kTopK * 4);
  p.off_rope = take((size_t)2 * p.Mb * 64 * 8);
  p.off_rpage = take((size_t)p.Mb * 8);
  p.off_hpart = take((size_t)p.lm_groups * p.lm_nparts * 2 * kGemvConsumers * 32 * 4 * 4);
  p.off_z = take((size_t)p.lm_rows * p.R * 4);
  p.off_g = take((size_t)p.Mb * (p.H / 2) * 4);
  p.off_rsg = take((size_t)2 * p.Mb * 4);  // row scales of a folded RMSNorm (tensor-core products)
  // arrival tickets of the split-K GEMVs: one per (column group, row group) and launch
  auto nctr = [](const GemvPlan& g) { return (size_t)g.groups * g.mgroups; };
  const GemvPlan* lp[5] = {&p.dc, &p.qkv, &p.o, &p.gu, &p.dn};
  p.ctr_fc = nctr(p.fc);
  size_t acc = 0;
  for (int i = 0; i < 5; ++i) {
    p.ctr_layer[i] = acc;
    acc += nctr(*lp[i]);
  }
  p.ctr_per_layer = acc;
  p.ctr_head = p.ctr_fc + (size_t)c->layers * p.ctr_per_layer;  // the streaming head's record tickets
  p.ctr_sel = p.ctr_head + (size_t)p.lm_groups * ((lm_tiles + kHeadTiles - 1) / kHeadTiles);  // selector tickets
  p.ctr_total = p.ctr_sel + (size_t)B;
  p.off_ctr = take(p.ctr_total * 4);
  p.step_bytes = o;
  p.off_s_taps = take((size_t)p.Mb * p.T * p.H * 2);
  p.off_s_nnew = take((size_t)B * 4);
  p.off_s_btok = take((size_t)p.Mb * 4);
  p.off_s_tgt = take((size_t)p.Mb * 4);
  p.off_s_path = take((size_t)B * p.D * 4);
  p.off_s_scores = take((size_t)B * p.D * 4);
  p.off_s_acc = take((size_t)B * 4);
  p.off_s_emit = take((size_t)p.Mb * 4);
  p.total = o;
  return p;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(ws) + off);
}

bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15u) == 0; }

constexpr int kMaxDevices = 64;

// Opt kernel k into `bytes` of dynamic shared memory on the current device.  CUDA keeps this
// attribute per device, so it is recorded per device in `done` (one array per kernel); host
// threads that race here set the same value, which is harmless.
template <typename... KArgs>
cudaError_t smem_optin(void (*k)(KArgs...), int bytes, std::atomic<int>* done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (done[dev].load(std::memory_order_acquire) == bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  done[dev].store(bytes, std::memory_order_release);
  return cudaSuccess;
}

// Launch with programmatic dependent launch: the kernel may start while the previous kernel on
// the stream drains; every kernel launched this way calls griddepcontrol.wait before it touches
// data written by earlier kernels.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, args...);
}

template <int NT, bool Q4>
cudaError_t launch_sgemv_t(const GemvPlan& g, const SGemvParams& prm, cudaStream_t s) {
  static std::atomic<int> attr[kMaxDevices];
  const cudaError_t e = smem_optin(k_sgemv<NT, Q4>, kSmemLimit - kStaticSmem, attr);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_sgemv<NT, Q4>, dim3(g.P), dim3(kSGemvThreads), g.smem, s, prm);
}

struct Epi {
  int mode = EPI_STORE;
  float* y = nullptr;
  int ldy = 0;
  uint16_t* act = nullptr;
  int F = 0;
  QkvEpi qkv{};
  // RMSNorm folding (see SGemvParams): residual epilogues write hw and ssp; consumers scale by rs
  float* ssp = nullptr;
  int ssp_rows = 0;
  uint16_t* hw = nullptr;
  const uint16_t* hw_w = nullptr;
  int hw_ld = 0;
  const float* rs_in = nullptr;
  int rs_H = 0;
  float eps = 0.f;
  const float* dyn_h = nullptr;
  const uint16_t *dyn_w = nullptr, *dyn_s0 = nullptr, *dyn_s1 = nullptr;
  uint16_t* dyn_y = nullptr;
  int Bk = 1;
  float* rs_glob = nullptr;  // tensor-core products with rs_in: [rows] row-scale buffer
};

SGemvParams sgemv_params(const GemvPlan& g, const GemvSeg* segs, int nseg, bool paired, const uint16_t* X, int ldx,
                         int rows, float* part, int ldo, int out_rows, int* counters, const Epi& e, int* err) {
  SGemvParams prm;
  memset(&prm, 0, sizeof(prm));
  for (int i = 0; i < nseg; ++i) prm.seg[i] = segs[i];
  prm.nseg = nseg;
  prm.paired = paired ? 1 : 0;
  prm.X = X;
  prm.ldx = ldx;
  prm.rows = rows;
  prm.U = g.U;
  prm.groups = g.groups;
  prm.mgroups = g.mgroups;
  prm.W = g.W;
  prm.kc_units = g.kc_units;
  prm.part = part;
  prm.ldo = ldo;
  prm.piece_stride = (long long)out_rows * ldo;
  prm.counters = counters;
  prm.epi = e.mode;
  prm.y = e.y;
  prm.ldy = e.ldy;
  prm.act = e.act;
  prm.F = e.F;
  prm.qkv = e.qkv;
  prm.ssp = e.ssp;
  prm.ssp_rows = e.ssp_rows;
  prm.hw = e.hw;
  prm.hw_w = e.hw_w;
  prm.hw_ld = e.hw_ld;
  prm.rs_in = e.rs_in;
  prm.rs_H = e.rs_H;
  prm.eps = e.eps;
  prm.dyn_h = e.dyn_h;
  prm.dyn_w = e.dyn_w;
  prm.dyn_s0 = e.dyn_s0;
  prm.dyn_s1 = e.dyn_s1;
  prm.dyn_y = e.dyn_y;
  prm.Bk = e.Bk;
  prm.err = err;
  prm.rs_glob = (g.umma && e.rs_in) ? e.rs_glob : nullptr;
  prm.mlx = g.mlx ? 1 : 0;
  prm.un = g.un;
  prm.upair = g.upair ? 1 : 0;
  return prm;
}

// cuTensorMapEncodeTiled, reached through the runtime's driver entry point (no link against the
// driver library).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static std::atomic<EncodeTiledFn> fn{nullptr};
  EncodeTiledFn f = fn.load(std::memory_order_acquire);
  if (f) return f;
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !ptr) {
    (void)cudaGetLastError();
    return nullptr;
  }
  f = reinterpret_cast<EncodeTiledFn>(ptr);
  fn.store(f, std::memory_order_release);
  return f;
}

// Tensor map of a bf16 activation matrix [rows][ldx] (K valid columns): boxes of 64 columns x
// box_rows rows, 128-byte swizzle (the tcgen05 K-major operand layout); rows past the end read as
// zero.
cudaError_t make_act_tmap(CUtensorMap* tm, const uint16_t* X, int K, int ldx, int rows, int box_rows = kUmmaRows) {
  const EncodeTiledFn f = encode_tiled();
  if (!f) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ldx * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = f(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Tensor-core product (stream-K pieces into the partial buffer) and its fix-up kernel (piece sums
// in order + the product's epilogue), both with programmatic dependent launch.
template <bool Q4, bool PAIR>
cudaError_t launch_umma_k(const GemvPlan& g, const SGemvParams& prm, const CUtensorMap& tm, cudaStream_t s) {
  static std::atomic<int> attr[kMaxDevices];
  const int smem = PAIR ? kUmmaPairSmem : kUmmaSmem;
  const cudaError_t e = smem_optin(k_umma<Q4, PAIR>, smem, attr);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_umma<Q4, PAIR>, dim3(g.P), dim3(kUmmaThreads), (size_t)smem, s, tm, prm);
}

template <bool Q4>
cudaError_t launch_umma_t(const GemvPlan& g, const SGemvParams& prm, cudaStream_t s) {
  CUtensorMap tm;
  cudaError_t e = make_act_tmap(&tm, prm.X, g.K, prm.ldx, prm.rows, g.un);
  if (e != cudaSuccess) return e;
  e = g.upair ? launch_umma_k<Q4, true>(g, prm, tm, s) : launch_umma_k<Q4, false>(g, prm, tm, s);
  if (e != cudaSuccess) return e;
  // rows per fix-up CTA: 64, halved (down to 16) while the grid would leave SMs idle (the fix-ups
  // of products with few column groups are latency-bound)
  int fr = 64;
  while (fr > 16 && (long long)prm.groups * ((prm.rows + fr - 1) / fr) < g.P) fr /= 2;
  const int fix_blocks = prm.groups * ((prm.rows + fr - 1) / fr);
  const dim3 fg(fix_blocks), fb(kGemvConsumers * 32);
  switch (prm.epi) {
    case EPI_RESID: return launch_pdl(k_umma_fixup<EPI_RESID, 2>, fg, fb, 0, s, prm, g.P, fr);
    case EPI_SWIGLU: return launch_pdl(k_umma_fixup<EPI_SWIGLU, 2>, fg, fb, 0, s, prm, g.P, fr);
    case EPI_STORE: return launch_pdl(k_umma_fixup<EPI_STORE, 2>, fg, fb, 0, s, prm, g.P, fr);
    case EPI_QKV: return launch_pdl(k_umma_fixup<EPI_QKV, 1>, fg, fb, 0, s, prm, g.P, fr);
    default: return launch_pdl(k_umma_fixup<EPI_DYNCONV, 1>, fg, fb, 0, s, prm, g.P, fr);
  }
}

cudaError_t launch_gemv(const GemvPlan& g, bool q4, const GemvSeg* segs, int nseg, bool paired, const uint16_t* X,
                        int ldx, int rows, float* part, int ldo, int out_rows, int* counters, const Epi& e, int* err,
                        cudaStream_t s) {
  const SGemvParams prm = sgemv_params(g, segs, nseg, paired, X, ldx, rows, part, ldo, out_rows, counters, e, err);
  if (g.umma) return q4 ? launch_umma_t<true>(g, prm, s) : launch_umma_t<false>(g, prm, s);
  switch (g.NT * 2 + (q4 ? 1 : 0)) {
    case 2: return launch_sgemv_t<1, false>(g, prm, s);
    case 3: return launch_sgemv_t<1, true>(g, prm, s);
    case 4: return launch_sgemv_t<2, false>(g, prm, s);
    case 5: return launch_sgemv_t<2, true>(g, prm, s);
    case 8: return launch_sgemv_t<4, false>(g, prm, s);
    case 9: return launch_sgemv_t<4, true>(g, prm, s);
    case 16: return launch_sgemv_t<8, false>(g, prm, s);
    case 17: return launch_sgemv_t<8, true>(g, prm, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_norm(const NormParams& np, int rows, cudaStream_t s) {
  return launch_pdl(k_norm, dim3(rows), dim3(256), np.H * sizeof(float), s, np);
}

template <int MT>
cudaError_t launch_attn_t(const Plan& P, const AttnParams& ap, cudaStream_t s) {
  static std::atomic<int> attr[kMaxDevices];
  const size_t smem = (size_t)(MT * 16 + 2 * kAttnKeys) * kAttnStride * 2;
  const cudaError_t e = smem_optin(k_attn_chunk<MT>, (int)smem, attr);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_attn_chunk<MT>, dim3(P.NC + 1, ap.nkv, P.B), dim3(kAttnThreads), smem, s, ap);
}

// Tensor map of one layer's K or V cache viewed as [pages * nkv * 16 rows][128] bf16: boxes of
// 16 rows (one page of one kv head) x 64 dims, 128-byte swizzle.
cudaError_t make_kv_tmap(CUtensorMap* tm, const uint16_t* cache, int num_pages, int nkv) {
  const EncodeTiledFn f = encode_tiled();
  if (!f) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)num_pages * nkv * kPage};
  const cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kPage};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = f(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(cache), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_attn_stream(const Plan& P, const AttnParams& ap, uint16_t* ob, cudaStream_t s) {
  static std::atomic<int> attr[kMaxDevices];
  cudaError_t e = smem_optin(k_attn_stream, kAsSmem, attr);
  if (e != cudaSuccess) return e;
  CUtensorMap tk, tv;
  if ((e = make_kv_tmap(&tk, ap.kc, ap.num_pages, ap.nkv)) != cudaSuccess) return e;
  if ((e = make_kv_tmap(&tv, ap.vc, ap.num_pages, ap.nkv)) != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P.attn_split, ap.nkv, P.B);
  cfg.blockDim = dim3(kAsThreads);
  cfg.dynamicSmemBytes = kAsSmem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = P.attn_split;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k_attn_stream, tk, tv, ap, ob);
}

template <int MT, int NTK, int KG>
cudaError_t launch_attn_cluster_t(const Plan& P, const AttnParams& ap, uint16_t* ob, cudaStream_t s) {
  static std::atomic<int> attr[kMaxDevices];
  const size_t smem = attn_cluster_smem(MT, KG * 8 * NTK);
  const cudaError_t e = smem_optin(k_attn_cluster<MT, NTK, KG>, (int)smem, attr);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kClusterCtas, ap.nkv, P.B);
  cfg.blockDim = dim3(MT * KG * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = kClusterCtas;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k_attn_cluster<MT, NTK, KG>, ap, ob);
}

template <int MT>
cudaError_t launch_attn_cluster_mt(const Plan& P, const AttnParams& ap, uint16_t* ob, cudaStream_t s) {
  if (P.attn_kg == 6) return launch_attn_cluster_t<MT, 6, 6>(P, ap, ob, s);
  switch (P.attn_ntk) {
    case 4: return launch_attn_cluster_t<MT, 4, 4>(P, ap, ob, s);
    case 8: return launch_attn_cluster_t<MT, 8, 4>(P, ap, ob, s);
    case 10: return launch_attn_cluster_t<MT, 10, 4>(P, ap, ob, s);
    default: return launch_attn_cluster_t<MT, 12, 4>(P, ap, ob, s);
  }
}

int fail(cudaError_t e) { return e == cudaSuccess ? DFLASH2_OK : DFLASH2_ERR_CUDA; }

#define CK(expr)                          \
  do {                                    \
    cudaError_t e_ = (expr);              \
    if (e_ != cudaSuccess) return fail(e_); \
  } while (0)

int check_weights(const dflash2_config* c, const dflash2_weights* w) {
  if (!w) return DFLASH2_ERR_ARG;
  if (!w->prepared) return DFLASH2_ERR_LAYOUT;
  const void* ptrs[] = {w->fc, w->fc_norm, w->final_norm, w->embed, w->lm_head, w->sel_proj, w->cb_a, w->cb_b};
  for (const void* q : ptrs) {
    if (!q) return DFLASH2_ERR_ARG;
    if (!aligned16(q)) return DFLASH2_ERR_ALIGN;
  }
  for (int l = 0; l < c->layers; ++l) {
    const dflash2_layer_weights& L = w->layer[l];
    const void* lp[] = {L.wq, L.wk, L.wv, L.wo, L.wg, L.wu, L.wd, L.ln1, L.ln2, L.qn, L.kn, L.dc_w, L.dc_s0, L.dc_s1};
    for (const void* q : lp) {
      if (!q) return DFLASH2_ERR_ARG;
      if (!aligned16(q)) return DFLASH2_ERR_ALIGN;
    }
  }
  return DFLASH2_OK;
}

int check_kv(const dflash2_config* c, const dflash2_kv* kv) {
  if (!kv || !kv->page_table || !kv->seq_len || kv->max_pages < 1 || kv->num_pages < 1) return DFLASH2_ERR_ARG;
  for (int l = 0; l < c->layers; ++l) {
    if (!kv->k[l] || !kv->v[l]) return DFLASH2_ERR_ARG;
    if (!aligned16(kv->k[l]) || !aligned16(kv->v[l])) return DFLASH2_ERR_ALIGN;
  }
  return DFLASH2_OK;
}

// Scratch of the allocation-free entry point: file-scope device memory, present on every GPU
// that loads this library for the life of the process.
static __device__ __align__(256) uint8_t g_static_scratch[DFLASH2_STATIC_SCRATCH_BYTES];

// Device address of g_static_scratch on the current device, looked up once per device.  (The
// symbol's name in host code is only a host-side stand-in, not a device address.)
void* static_scratch(cudaError_t* err) {
  static std::atomic<void*> cache[kMaxDevices];
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  void* p = cache[dev].load(std::memory_order_acquire);
  if (p) return p;
  *err = cudaGetSymbolAddress(&p, g_static_scratch);
  if (*err != cudaSuccess) return nullptr;
  cache[dev].store(p, std::memory_order_release);
  return p;
}

}  // namespace

extern "C" {

size_t dflash2_workspace_size(const dflash2_config* cfg, int32_t batch) {
  if (!cfg_ok(cfg) || batch < 1) return 0;
  return make_plan(cfg, batch).total;
}

size_t dflash2_prepared_size(const dflash2_config* c) {
  if (!cfg_ok(c)) return 0;
  const size_t H = c->hidden, F = c->ffn, HQ = (size_t)c->n_q * kHeadDim, HKV = (size_t)c->n_kv * kHeadDim;
  const size_t per_layer = HQ * H + 2 * HKV * H + H * HQ + 2 * F * H + H * F;
  const size_t mats = H * c->n_taps * H + c->layers * per_layer;
  const size_t mat_bytes = (c->wfmt == 0 || c->wfmt == 2) ? mats / kUnit * 144 : mats * 2;
  const size_t dyn = (size_t)c->layers * 2 * (H / 4) * H * 2;
  const size_t head_groups = ((size_t)(c->vocab + c->rank) / 16 + kHeadTiles - 1) / kHeadTiles;
  // the head twice: the streaming kernel's records and the tensor-core operand copy
  return mat_bytes + dyn + 2 * head_groups * kHeadTiles * 16 * H * 2;
}

int dflash2_prepare_weights(const dflash2_config* c, const dflash2_weights* src, void* dst, size_t dst_bytes,
                            dflash2_weights* out, void* stream) {
  if (!cfg_ok(c)) return DFLASH2_ERR_SHAPE;
  if (!src || !out) return DFLASH2_ERR_ARG;
  dflash2_weights tmp = *src;
  tmp.prepared = 1;
  int rc = check_weights(c, &tmp);
  if (rc != DFLASH2_OK) return rc;
  if (!dst) return DFLASH2_ERR_ARG;
  if (!aligned16(dst)) return DFLASH2_ERR_ALIGN;
  if (dst_bytes < dflash2_prepared_size(c)) return DFLASH2_ERR_WORKSPACE;
  *out = *src;
  out->prepared = 1;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* d = (uint8_t*)dst;
  const int H = c->hidden, F = c->ffn, HQ = c->n_q * kHeadDim, HKV = c->n_kv * kHeadDim;
  // one matrix (or a set sharing one buffer) into group-interleaved records at d
  const int fmt = c->wfmt;
  // fmt: 0 Q4_K, 1 bf16, 2 MLX 4-bit group-64 (into the same 4-bit records), 3 Q8_0 (into bf16 records)
  auto place_fmt = [&](const void* w, int N, int K, int fmt, PrepPlace pl) {
    if (fmt == 0)
      k_q4k_prepare<<<dim3(K / kUnit, N / 16), 32, 0, s>>>((const uint8_t*)w, d, N, K, pl);
    else if (fmt == 2)
      k_mlx4_prepare<<<dim3(K / kUnit, N / 16), 32, 0, s>>>((const uint8_t*)w, d, N, K, pl);
    else if (fmt == 3)
      k_q80_prepare<<<dim3(K / 64, N / 16), 32, 0, s>>>((const uint8_t*)w, d, N, K, pl);
    else
      k_bf16_prepare<<<dim3(K / 64, N / 16), 32, 0, s>>>((const uint16_t*)w, d, N, K, pl);
  };
  auto place = [&](const void* w, int N, int K, bool q4, PrepPlace pl) { place_fmt(w, N, K, q4 ? fmt : 1, pl); };
  // bytes of one prepared matrix: q4 = "in the configured format" (4-bit records for Q4_K and MLX,
  // bf16 records for bf16 and Q8_0), else bf16
  auto bytes = [&](int N, int K, bool q4) {
    return (q4 && (fmt == 0 || fmt == 2)) ? (size_t)N * K / kUnit * 144 : (size_t)N * K * 2;
  };
  auto prep = [&](const void* w, int N, int K, bool q4) -> const void* {
    const void* r = d;
    place(w, N, K, q4, PrepPlace{0, 8, 0, 8});
    d += bytes(N, K, q4);
    return r;
  };
  const bool q4 = c->wfmt != 1;  // the layer matrices in the configured format (the W_dc generators are bf16)
  out->fc = prep(src->fc, H, c->n_taps * H, q4);
  for (int l = 0; l < c->layers; ++l) {
    const dflash2_layer_weights& S = src->layer[l];
    dflash2_layer_weights& O = out->layer[l];
    O.wq = prep(S.wq, HQ, H, q4);
    O.wk = prep(S.wk, HKV, H, q4);
    O.wv = prep(S.wv, HKV, H, q4);
    O.wo = prep(S.wo, H, HQ, q4);
    // gate and up interleaved 4 + 4 tiles per group; wu aliases the same buffer
    place(S.wg, F, H, q4, PrepPlace{0, 4, 0, 8});
    place(S.wu, F, H, q4, PrepPlace{0, 4, 4, 8});
    O.wg = O.wu = d;
    d += 2 * bytes(F, H, q4);
    O.wd = prep(S.wd, H, F, q4);
    // the convolution's gate generators a0 | a1 interleaved 4 + 4 tiles per group (both gates of a
    // channel group in one CTA's fix-up); dc_w points at the pair
    place(S.dc_w, H / 4, H, false, PrepPlace{0, 4, 0, 8});
    place(S.dc_w + (size_t)(H / 4) * H, H / 4, H, false, PrepPlace{0, 4, 4, 8});
    O.dc_w = (const uint16_t*)d;
    d += bytes(2 * (H / 4), H, false);
  }
  // the output head and the selector projection as one [V + R, H] matrix in records of 16 tiles
  // (32 KB per 64-wide step: one bulk copy feeds two 8-tile column groups), padded to whole records
  const size_t groups = ((size_t)(c->vocab + c->rank) / 16 + kHeadTiles - 1) / kHeadTiles;
  const size_t gbytes = (size_t)kHeadTiles * 16 * H * 2;
  CK(cudaMemsetAsync(d + (groups - 1) * gbytes, 0, gbytes, s));
  place(src->lm_head, c->vocab, H, false, PrepPlace{0, kHeadTiles, 0, kHeadTiles});
  place(src->sel_proj, c->rank, H, false, PrepPlace{c->vocab / 16, kHeadTiles, 0, kHeadTiles});
  out->lm_head = (const uint16_t*)d;
  out->sel_proj = (const uint16_t*)d;  // interleaved into the head's records
  // the tensor-core operand copy of the same head follows the records (see k_umma_head)
  k_head_sw_prepare<<<dim3(H / 64, (unsigned)(groups * kHeadTiles / 16)), 256, 0, s>>>(
      src->lm_head, src->sel_proj, d + groups * gbytes, c->vocab, c->rank, H);
  return fail(cudaGetLastError());
}

}  // extern "C"

namespace {

// A vocabulary shard of the output head: this rank's head rows [v0, v0 + rows) (prepared with
// dflash2_prepare_head_shard) and where its local candidates and the selector projection go.
struct HeadShard {
  const uint8_t* head;  // prepared streaming records, the tensor-core operand copy following them
  int v0, rows;
  float* out_val;
  int32_t* out_id;
  float* out_z;
};

size_t head_records(const dflash2_config* c, int rows) { return ((size_t)(rows + c->rank) / 16 + kHeadTiles - 1) / kHeadTiles; }

int draft_step_impl(const dflash2_config* c, const dflash2_weights* w, const dflash2_inputs* in, const dflash2_kv* kv,
                    int32_t batch, int32_t* out_path, float* out_scores, void* ws, size_t ws_bytes,
                    const dflash2_debug* dbg, void* stream, const HeadShard* hs) {
  if (!cfg_ok(c)) return DFLASH2_ERR_SHAPE;
  if (batch < 1 || !in || !kv || !ws || (!hs && (!out_path || !out_scores))) return DFLASH2_ERR_ARG;
  int rc = check_weights(c, w);
  if (rc) return rc;
  if (!in->taps || !in->n_new || !in->block_tokens) return DFLASH2_ERR_ARG;
  rc = check_kv(c, kv);
  if (rc) return rc;
  if (!aligned16(in->taps) || ((uintptr_t)ws & 255u)) return DFLASH2_ERR_ALIGN;
  Plan P = make_plan(c, batch);
  if (ws_bytes < P.step_bytes) return DFLASH2_ERR_WORKSPACE;
  if (hs) plan_head(P, hs->rows);  // the head's launch shape for this shard (workspace sized for the whole head)
  const uint8_t* head = hs ? hs->head : (const uint8_t*)w->lm_head;
  const int Vh = hs ? hs->rows : P.V, id0 = hs ? hs->v0 : 0;
  cudaStream_t s = (cudaStream_t)stream;
  int* err = at<int>(ws, P.off_err);
  float* h = at<float>(ws, P.off_h);
  float* xf = at<float>(ws, P.off_xf);
  uint16_t* xb = at<uint16_t>(ws, P.off_xb);
  uint16_t* yb = at<uint16_t>(ws, P.off_yb);
  uint16_t* ctx = yb + (size_t)P.Mb * P.H;
  float* part = at<float>(ws, P.off_part);
  uint16_t* qb = at<uint16_t>(ws, P.off_qb);
  uint16_t* kb = at<uint16_t>(ws, P.off_kb);
  uint16_t* vb = at<uint16_t>(ws, P.off_vb);
  uint16_t* ob = at<uint16_t>(ws, P.off_ob);
  uint16_t* act = at<uint16_t>(ws, P.off_act);
  uint16_t* hn = at<uint16_t>(ws, P.off_hn);
  float* zbuf = at<float>(ws, P.off_z);
  const int H = P.H, Mb = P.Mb;
  const size_t hbytes = (size_t)Mb * H * 4;
  AttnParams ap{};
  ap.qb = qb;
  ap.kb = kb;
  ap.vb = vb;
  ap.page_table = kv->page_table;
  ap.max_pages = kv->max_pages;
  ap.num_pages = kv->num_pages;
  ap.seq_len = kv->seq_len;
  ap.n_new = in->n_new;
  ap.Bk = P.Bk;
  ap.nq = c->n_q;
  ap.nkv = c->n_kv;
  ap.W = c->window;
  ap.NC = P.NC;
  ap.QVP = P.QVP;
  ap.part_o = at<float>(ws, P.off_ao);
  ap.part_ml = at<float>(ws, P.off_aml);
  ap.scale_log2 = (float)(1.4426950408889634 / sqrt((double)kHeadDim));
  ap.err = err;

  float* gbuf = at<float>(ws, P.off_g);
  int* ctr = at<int>(ws, P.off_ctr);
  // These two memsets are full stream barriers: every earlier operation on the stream (the host
  // round's staging kernel, the previous round's acceptance writing n_new and block tokens) has
  // finished before the step's first kernel, so the kernels below may read the step inputs before
  // their programmatic-launch wait.
  CK(cudaMemsetAsync(err, 0, 4, s));
  CK(cudaMemsetAsync(ctr, 0, P.ctr_total * 4, s));
  // A1: block rows from the shared embedding table (+ the first RMSNorm's inputs: h * ln1 and the
  // rows' sums of squares; every RMSNorm before a product is folded the same way: the residual
  // epilogues write bf16(h * w) and sums of squares, the product scales its outputs per row)
  float* ssp = at<float>(ws, P.off_ssp);
  float2* rope = at<float2>(ws, P.off_rope);
  int2* rpage = at<int2>(ws, P.off_rpage);
  RopeInit ri{kv->seq_len, in->n_new, kv->page_table, kv->max_pages, kv->num_pages, P.Bk, Mb,
              log2((double)c->rope_theta), rope, rpage};
  CK(launch_pdl(k_embed, dim3(Mb), dim3(256), 0, s, in->block_tokens, w->embed, h, H, P.V, err, xb, w->layer[0].ln1,
                ssp, Mb, ri));
  if (dbg && dbg->hidden) CK(cudaMemcpyAsync(dbg->hidden, h, hbytes, cudaMemcpyDeviceToDevice, s));

  // A2: context rows = RMSNorm_fc(W_fc . concat(taps)); fc output staged in xf
  {
    GemvSeg seg{(const uint8_t*)w->fc, H / 16, Mb, 0};
    Epi e;
    e.mode = EPI_STORE;
    e.y = xf;
    e.ldy = H;
    CK(launch_gemv(P.fc, P.q4, &seg, 1, false, in->taps, P.T * H, Mb, part, H, Mb, ctr, e, err, s));
    NormParams np{};
    np.in = xf;
    np.w = w->fc_norm;
    np.eps = c->rms_eps;
    np.H = H;
    np.out_bf = ctx;
    np.ldob = H;
    np.mode = 1;
    np.n_new = in->n_new;
    np.Bk = P.Bk;
    CK(launch_norm(np, Mb, s));
    if (dbg && dbg->ctx) CK(cudaMemcpyAsync(dbg->ctx, ctx, (size_t)Mb * H * 2, cudaMemcpyDeviceToDevice, s));
  }


  for (int l = 0; l < c->layers; ++l) {
    const dflash2_layer_weights& L = w->layer[l];
    int* lctr = ctr + P.ctr_fc + (size_t)l * P.ctr_per_layer;
    // A3a: x = RMSNorm(h; ln1), g = W_dc x (operand xb = bf16(h * ln1), outputs scaled by the row
    // scale), y = dynconv(x, g)
    {
      if (dbg && dbg->hidden && l > 0)
        CK(cudaMemcpyAsync(dbg->hidden + (size_t)l * Mb * H, h, hbytes, cudaMemcpyDeviceToDevice, s));
      // gate generators a0 | a1 paired per group; the fix-up applies the row scale, tanh and the
      // two-tap convolution of its 256 channels and writes y (bf16) for the q/k/v product
      GemvSeg segs[2] = {{(const uint8_t*)L.dc_w, (H / 4) / 16, Mb, 0}, {(const uint8_t*)L.dc_w, (H / 4) / 16, Mb, H / 4}};
      Epi e;
      e.mode = EPI_DYNCONV;
      e.rs_in = ssp;
      e.rs_glob = at<float>(ws, P.off_rsg);
      e.ssp_rows = Mb;
      e.rs_H = H;
      e.eps = c->rms_eps;
      e.dyn_h = h;
      e.dyn_w = L.ln1;
      e.dyn_s0 = L.dc_s0;
      e.dyn_s1 = L.dc_s1;
      e.dyn_y = yb;
      e.Bk = P.Bk;
      CK(launch_gemv(P.dc, false, segs, 2, true, xb, H, Mb, part, H / 2, Mb, lctr + P.ctr_layer[0], e, err, s));
    }
    // A3b+c: q from the block rows; k, v from block + context rows (stacked: each matrix read once);
    // the last CTA of each head applies q/k RMSNorm + RoPE and appends context K/V to the cache
    {
      const int ldo = P.HQ + 2 * P.HKV;
      GemvSeg segs[3] = {{(const uint8_t*)L.wq, P.HQ / 16, Mb, 0},
                         {(const uint8_t*)L.wk, P.HKV / 16, 2 * Mb, P.HQ},
                         {(const uint8_t*)L.wv, P.HKV / 16, 2 * Mb, P.HQ + P.HKV}};
      Epi e;
      e.mode = EPI_QKV;
      QkvEpi& q = e.qkv;
      q.qn = L.qn;
      q.kn = L.kn;
      q.eps = c->rms_eps;
      q.log2_theta = log2((double)c->rope_theta);
      q.Bk = P.Bk;
      q.nq = c->n_q;
      q.nkv = c->n_kv;
      q.Mb = Mb;
      q.seq_len = kv->seq_len;
      q.n_new = in->n_new;
      q.qb = qb;
      q.kb = kb;
      q.vb = vb;
      q.kc = kv->k[l];
      q.vc = kv->v[l];
      q.page_table = kv->page_table;
      q.max_pages = kv->max_pages;
      q.num_pages = kv->num_pages;
      q.rope = rope;  // positions and cache slots of this step, from the embedding kernel
      q.rpage = rpage;
      q.err = err;
      CK(launch_gemv(P.qkv, P.q4, segs, 3, false, yb, H, 2 * Mb, part, ldo, 2 * Mb, lctr + P.ctr_layer[1], e, err, s));
    }
    // A3d: sliding-window GQA attention over cache + block keys
    {
      ap.kc = kv->k[l];
      ap.vc = kv->v[l];
      if (P.attn_stream) {
        CK(launch_attn_stream(P, ap, ob, s));
      } else if (P.attn_ntk > 0) {
        if (P.MT == 1) CK(launch_attn_cluster_mt<1>(P, ap, ob, s));
        else CK(launch_attn_cluster_mt<2>(P, ap, ob, s));
      } else {
        switch (P.MT) {
          case 1: CK(launch_attn_t<1>(P, ap, s)); break;
          case 2: CK(launch_attn_t<2>(P, ap, s)); break;
          case 3: CK(launch_attn_t<3>(P, ap, s)); break;
          default: CK(launch_attn_t<4>(P, ap, s)); break;
        }
        CK(launch_pdl(k_attn_combine, dim3((P.QV + 3) / 4, c->n_kv, batch), dim3(128), 0, s, ap, ob));
      }
    }
    // A3e: h += W_o o (residual added by the last CTA of each column group)
    {
      GemvSeg seg{(const uint8_t*)L.wo, H / 16, Mb, 0};
      Epi e;
      e.mode = EPI_RESID;
      e.y = h;
      e.ldy = H;
      e.hw = xb;  // bf16(h * ln2) and sums of squares for the gate/up product
      e.hw_w = L.ln2;
      e.hw_ld = H;
      e.ssp = ssp;
      e.ssp_rows = Mb;
      CK(launch_gemv(P.o, P.q4, &seg, 1, false, ob, P.HQ, Mb, part, H, Mb, lctr + P.ctr_layer[2], e, err, s));
    }
    // A3f: h += W_d (silu(W_g x2) * W_u x2); gate and up tiles paired per CTA so the SwiGLU is fused
    {
      GemvSeg segs[2] = {{(const uint8_t*)L.wg, P.F / 16, Mb, 0}, {(const uint8_t*)L.wg, P.F / 16, Mb, P.F}};
      Epi e;
      e.mode = EPI_SWIGLU;
      e.act = act;
      e.F = P.F;
      e.rs_in = ssp;
      e.rs_glob = at<float>(ws, P.off_rsg);
      e.ssp_rows = Mb;
      e.rs_H = H;
      e.eps = c->rms_eps;
      CK(launch_gemv(P.gu, P.q4, segs, 2, true, xb, H, Mb, part, 2 * P.F, Mb, lctr + P.ctr_layer[3], e, err, s));
      GemvSeg seg{(const uint8_t*)L.wd, H / 16, Mb, 0};
      Epi e2;
      e2.mode = EPI_RESID;
      e2.y = h;
      e2.ldy = H;
      if (l + 1 < c->layers) {  // bf16(h * ln1') and sums of squares for the next layer
        e2.hw = xb;
        e2.hw_w = w->layer[l + 1].ln1;
        e2.hw_ld = H;
        e2.ssp = ssp;
        e2.ssp_rows = Mb;
      }
      CK(launch_gemv(P.dn, P.q4, &seg, 1, false, act, P.F, Mb, part, H, Mb, lctr + P.ctr_layer[4], e2, err, s));
    }
  }
  // A4: final norm of the drafted rows 1..block-1
  {
    NormParams np{};
    np.in = h;
    np.w = w->final_norm;
    np.eps = c->rms_eps;
    np.H = H;
    np.out_bf = hn;
    np.ldob = H;
    np.mode = 2;
    np.Bk = P.Bk;
    CK(launch_norm(np, Mb, s));
    if (dbg && dbg->hidden)
      CK(cudaMemcpyAsync(dbg->hidden + (size_t)c->layers * Mb * H, h, hbytes, cudaMemcpyDeviceToDevice, s));
    if (dbg && dbg->final_h)
      CK(cudaMemcpyAsync(dbg->final_h, hn, (size_t)P.lm_rows * H * 2, cudaMemcpyDeviceToDevice, s));
  }
  // A5: LM head + streaming top-16 (+ selector projection)
  {
    if (dbg && dbg->ev_lm_begin) CK(cudaEventRecord((cudaEvent_t)dbg->ev_lm_begin, s));
    if (P.lm_umma) {
      static std::atomic<int> uattr[kMaxDevices];
      CK(smem_optin(k_umma_head, kUHeadSmem, uattr));
      CUtensorMap tm;
      CK(make_act_tmap(&tm, hn, H, H, P.lm_rows));
      UHeadParams hp{};
      hp.Wsw = head + (size_t)P.lm_unrec * kHeadTiles * 16 * H * 2;  // the operand copy
      hp.V = Vh;
      hp.id0 = id0;
      hp.R = P.R;
      hp.H = H;
      hp.rows = P.lm_rows;
      hp.nrec = P.lm_unrec;
      hp.nrt = P.lm_unrt;
      hp.z = hs ? hs->out_z : zbuf;
      hp.cand_val = at<float>(ws, P.off_cv);
      hp.cand_id = at<int32_t>(ws, P.off_ci);
      hp.err = err;
      CK(launch_pdl(k_umma_head, dim3(P.lm_uP), dim3(kUHeadThreads), (size_t)kUHeadSmem, s, tm, hp));
    } else {
      static std::atomic<int> attr[kMaxDevices];
      CK(smem_optin(k_slmhead, kSmemLimit - kStaticSmem, attr));
      SLmParams lp{};
      lp.W = head;
      lp.V = Vh;
      lp.id0 = id0;
      lp.R = P.R;
      lp.H = H;
      lp.X = hn;
      lp.rows = P.lm_rows;
      lp.z = hs ? hs->out_z : zbuf;
      lp.cand_val = at<float>(ws, P.off_cv);
      lp.cand_id = at<int32_t>(ws, P.off_ci);
      lp.part = at<float>(ws, P.off_hpart);
      lp.counters = ctr + P.ctr_head;
      lp.err = err;
      lp.groups = P.lm_groups;
      CK(launch_pdl(k_slmhead, dim3(P.lm_nparts * P.lm_groups), dim3(kGemvThreads), P.lm_smem, s, lp));
    }
    if (dbg && dbg->ev_lm_end) CK(cudaEventRecord((cudaEvent_t)dbg->ev_lm_end, s));
    if (dbg && dbg->z) CK(cudaMemcpyAsync(dbg->z, zbuf, (size_t)P.lm_rows * P.R * 4, cudaMemcpyDeviceToDevice, s));
  }
  if (hs) {  // a shard: its local top-16 per row for the exchange; seq_len advanced here
    CK(launch_pdl(k_merge_rows, dim3((P.lm_rows + 3) / 4), dim3(128), 0, s, (const float*)at<float>(ws, P.off_cv),
                  (const int32_t*)at<int32_t>(ws, P.off_ci), P.sel_parts, P.lm_rows, hs->out_val, hs->out_id,
                  kv->seq_len, in->n_new, batch));
    return DFLASH2_OK;
  }
  // A6: candidates, selector scores, Viterbi path; seq_len advanced
  {
    SelParams sp{};
    sp.cand_val = at<float>(ws, P.off_cv);
    sp.cand_id = at<int32_t>(ws, P.off_ci);
    sp.nparts = P.sel_parts;
    sp.rows_total = P.lm_rows;
    sp.z = zbuf;
    sp.R = P.R;
    sp.V = P.V;
    sp.Bk = P.Bk;
    sp.cb_a = w->cb_a;
    sp.cb_b = w->cb_b;
    sp.block_tokens = in->block_tokens;
    sp.out_path = out_path;
    sp.out_scores = out_scores;
    sp.seq_len = kv->seq_len;
    sp.n_new = in->n_new;
    sp.dbg_cand = dbg ? dbg->cand : nullptr;
    sp.dbg_logit = dbg ? dbg->cand_logit : nullptr;
    sp.err = err;
    if (sp.dbg_cand && !sp.dbg_logit) sp.dbg_cand = nullptr;
    float* tau = at<float>(ws, P.off_tau);
    float* clg = at<float>(ws, P.off_cfv);
    int32_t* cdg = at<int32_t>(ws, P.off_cfi);
    // The CTAs are few and latency-bound: reserve (unused) dynamic shared memory so that each gets
    // an SM of its own instead of several landing on the first SM the output head frees.
    static std::atomic<int> sel_attr[kMaxDevices];
    CK(smem_optin(k_sel_tau, kSelSpreadSmem, sel_attr));
    CK(launch_pdl(k_sel_tau, dim3(P.D, batch), dim3(256), kSelSpreadSmem, s, sp, tau, clg, cdg, ctr + P.ctr_sel));
  }
  return DFLASH2_OK;
}

}  // namespace

extern "C" {

int dflash2_draft_step(const dflash2_config* c, const dflash2_weights* w, const dflash2_inputs* in,
                       const dflash2_kv* kv, int32_t batch, int32_t* out_path, float* out_scores, void* ws,
                       size_t ws_bytes, const dflash2_debug* dbg, void* stream) {
  return draft_step_impl(c, w, in, kv, batch, out_path, out_scores, ws, ws_bytes, dbg, stream, nullptr);
}

size_t dflash2_head_shard_size(const dflash2_config* c, int32_t rows) {
  if (!cfg_ok(c) || rows < 16 || rows % 16) return 0;
  return 2 * head_records(c, rows) * kHeadTiles * 16 * (size_t)c->hidden * 2;
}

int dflash2_prepare_head_shard(const dflash2_config* c, const uint16_t* lm_head_rows, int32_t rows,
                               const uint16_t* sel_proj, void* dst, size_t dst_bytes, void* stream) {
  if (!cfg_ok(c)) return DFLASH2_ERR_SHAPE;
  if (!lm_head_rows || !sel_proj || !dst || rows < 16 || rows % 16 || rows > c->vocab) return DFLASH2_ERR_ARG;
  if (!aligned16(dst) || !aligned16(lm_head_rows) || !aligned16(sel_proj)) return DFLASH2_ERR_ALIGN;
  if (dst_bytes < dflash2_head_shard_size(c, rows)) return DFLASH2_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const int H = c->hidden;
  const size_t groups = head_records(c, rows), gbytes = (size_t)kHeadTiles * 16 * H * 2;
  uint8_t* d = (uint8_t*)dst;
  CK(cudaMemsetAsync(d + (groups - 1) * gbytes, 0, gbytes, s));
  k_bf16_prepare<<<dim3(H / 64, rows / 16), 32, 0, s>>>(lm_head_rows, d, rows, H, PrepPlace{0, kHeadTiles, 0, kHeadTiles});
  k_bf16_prepare<<<dim3(H / 64, c->rank / 16), 32, 0, s>>>(sel_proj, d, c->rank, H,
                                                            PrepPlace{rows / 16, kHeadTiles, 0, kHeadTiles});
  k_head_sw_prepare<<<dim3(H / 64, (unsigned)groups), 256, 0, s>>>(lm_head_rows, sel_proj, d + groups * gbytes, rows,
                                                                   c->rank, H);
  return fail(cudaGetLastError());
}

int dflash2_draft_step_head_shard(const dflash2_config* c, const dflash2_weights* w, const void* head_shard,
                                  int32_t v0, int32_t rows, const dflash2_inputs* in, const dflash2_kv* kv,
                                  int32_t batch, float* out_cand_val, int32_t* out_cand_id, float* out_z, void* ws,
                                  size_t ws_bytes, void* stream) {
  if (!cfg_ok(c)) return DFLASH2_ERR_SHAPE;
  if (!head_shard || !out_cand_val || !out_cand_id || !out_z || rows < 16 || rows % 16 || v0 < 0 ||
      (long long)v0 + rows > c->vocab)
    return DFLASH2_ERR_ARG;
  if (!aligned16(head_shard) || !w) return !w ? DFLASH2_ERR_ARG : DFLASH2_ERR_ALIGN;
  // a shard rank reads neither the whole head nor the codebooks: stand their pointers in for the
  // weight checks (the step never reads them)
  dflash2_weights ws_w = *w;
  ws_w.lm_head = ws_w.sel_proj = (const uint16_t*)head_shard;
  if (!ws_w.cb_a) ws_w.cb_a = (const uint16_t*)head_shard;
  if (!ws_w.cb_b) ws_w.cb_b = (const uint16_t*)head_shard;
  const HeadShard hs{(const uint8_t*)head_shard, v0, rows, out_cand_val, out_cand_id, out_z};
  return draft_step_impl(c, &ws_w, in, kv, batch, nullptr, nullptr, ws, ws_bytes, nullptr, stream, &hs);
}

int dflash2_select(const dflash2_config* c, const dflash2_weights* w, int32_t batch, int32_t nparts,
                   const float* cand_val, const int32_t* cand_id, const float* z, const int32_t* block_tokens,
                   int32_t* out_path, float* out_scores, void* ws, size_t ws_bytes, void* stream) {
  if (!cfg_ok(c)) return DFLASH2_ERR_SHAPE;
  if (!w || !w->cb_a || !w->cb_b || !cand_val || !cand_id || !z || !block_tokens || !out_path || !out_scores || !ws ||
      batch < 1 || nparts < 1 || nparts > 256)
    return DFLASH2_ERR_ARG;
  if ((uintptr_t)ws & 255u) return DFLASH2_ERR_ALIGN;
  const Plan P = make_plan(c, batch);
  if (ws_bytes < P.step_bytes) return DFLASH2_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  int* err = at<int>(ws, P.off_err);
  int* ctr = at<int>(ws, P.off_ctr);
  CK(cudaMemsetAsync(err, 0, 4, s));
  CK(cudaMemsetAsync(ctr + P.ctr_sel, 0, (size_t)batch * 4, s));
  SelParams sp{};
  sp.cand_val = cand_val;
  sp.cand_id = cand_id;
  sp.nparts = nparts;
  sp.rows_total = P.lm_rows;
  sp.z = z;
  sp.R = P.R;
  sp.V = P.V;
  sp.Bk = P.Bk;
  sp.cb_a = w->cb_a;
  sp.cb_b = w->cb_b;
  sp.block_tokens = block_tokens;
  sp.out_path = out_path;
  sp.out_scores = out_scores;
  sp.seq_len = nullptr;  // advanced by each shard's step
  sp.err = err;
  static std::atomic<int> sel_attr[kMaxDevices];
  CK(smem_optin(k_sel_tau, kSelSpreadSmem, sel_attr));
  CK(launch_pdl(k_sel_tau, dim3(P.D, batch), dim3(256), kSelSpreadSmem, s, sp, at<float>(ws, P.off_tau),
                at<float>(ws, P.off_cfv), at<int32_t>(ws, P.off_cfi), ctr + P.ctr_sel));
  return DFLASH2_OK;
}

int dflash2_draft_step_static(const dflash2_config* c, const dflash2_weights* w, const dflash2_inputs* in,
                              const dflash2_kv* kv, int32_t batch, int32_t* out_path, float* out_scores,
                              int32_t* dev_err, const dflash2_debug* dbg, void* stream) {
  if (!cfg_ok(c)) return DFLASH2_ERR_SHAPE;
  if (batch < 1) return DFLASH2_ERR_ARG;
  if (make_plan(c, batch).step_bytes > DFLASH2_STATIC_SCRATCH_BYTES) return DFLASH2_ERR_STATIC_LIMIT;
  cudaError_t e = cudaSuccess;
  void* ws = static_scratch(&e);
  if (!ws) return fail(e == cudaSuccess ? cudaErrorUnknown : e);
  const int rc = dflash2_draft_step(c, w, in, kv, batch, out_path, out_scores, ws, DFLASH2_STATIC_SCRATCH_BYTES, dbg,
                                    stream);
  if (rc != DFLASH2_OK) return rc;
  if (dev_err)  // the error word sits at the start of the scratch
    CK(cudaMemcpyAsync(dev_err, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
  return DFLASH2_OK;
}

int dflash2_accept(const int32_t* draft, const int32_t* target, int32_t batch, int32_t block, int32_t* accepted,
                   int32_t* emitted, void* stream) {
  if (!draft || !target || !accepted || !emitted || batch < 1 || block < 2) return DFLASH2_ERR_ARG;
  k_accept<<<(batch + 127) / 128, 128, 0, (cudaStream_t)stream>>>(draft, target, batch, block, accepted, emitted);
  return fail(cudaGetLastError());
}

int dflash2_accept_sampled(const int32_t* draft, const float* p_target, const float* q_draft, const float* u_accept,
                           const uint32_t* u_sample, int32_t batch, int32_t block, int32_t vocab, int32_t* accepted,
                           int32_t* emitted, void* stream) {
  if (!draft || !p_target || !u_accept || !u_sample || !accepted || !emitted || batch < 1 || block < 2 || vocab < 1)
    return DFLASH2_ERR_ARG;
  k_accept_sampled<<<batch, kSampThreads, 0, (cudaStream_t)stream>>>(draft, p_target, q_draft, u_accept, u_sample,
                                                                     block, vocab, accepted, emitted);
  return fail(cudaGetLastError());
}

int dflash2_accept_chain(const int32_t* draft, const int32_t* target, int32_t batch, int32_t block, int32_t mask_id,
                         int32_t* accepted, int32_t* emitted, int32_t* n_new_next, int32_t* block_tokens_next,
                         void* stream) {
  if (!draft || !target || !accepted || !emitted || !n_new_next || !block_tokens_next || batch < 1 || block < 2 ||
      mask_id < 0)
    return DFLASH2_ERR_ARG;
  k_accept_chain<<<(batch + 127) / 128, 128, 0, (cudaStream_t)stream>>>(draft, target, batch, block, mask_id, accepted,
                                                                        emitted, n_new_next, block_tokens_next);
  return fail(cudaGetLastError());
}

int dflash2_spec_round(const dflash2_config* c, const dflash2_weights* w, dflash2_inputs_mut* in, const dflash2_kv* kv,
                       int32_t batch, const int32_t* prev_path, const int32_t* target, int32_t mask_id,
                       int32_t* accepted, int32_t* emitted, int32_t* out_path, float* out_scores, void* ws,
                       size_t ws_bytes, void* stream) {
  if (!cfg_ok(c)) return DFLASH2_ERR_SHAPE;
  if (!in || !in->taps || !in->n_new || !in->block_tokens || !prev_path || !target || !accepted || !emitted ||
      !out_path || !out_scores || !ws || batch < 1 || mask_id < 0 || mask_id >= c->vocab)
    return DFLASH2_ERR_ARG;
  // the step's own checks, before anything is queued
  int rc = check_weights(c, w);
  if (rc) return rc;
  rc = check_kv(c, kv);
  if (rc) return rc;
  if (!aligned16(in->taps) || ((uintptr_t)ws & 255u)) return DFLASH2_ERR_ALIGN;
  if (ws_bytes < make_plan(c, batch).step_bytes) return DFLASH2_ERR_WORKSPACE;
  rc = dflash2_accept_chain(prev_path, target, batch, c->block, mask_id, accepted, emitted, in->n_new,
                            in->block_tokens, stream);
  if (rc) return rc;
  const dflash2_inputs ci{in->taps, in->n_new, in->block_tokens};
  return dflash2_draft_step(c, w, &ci, kv, batch, out_path, out_scores, ws, ws_bytes, nullptr, stream);
}

int dflash2_spec_step_host(const dflash2_config* c, const dflash2_weights* w, const dflash2_kv* kv, int32_t batch,
                           const uint16_t* taps_h, const int32_t* n_new_h, const int32_t* block_tokens_h,
                           const int32_t* target_h, int32_t* path_h, float* scores_h, int32_t* accepted_h,
                           int32_t* emitted_h, int32_t* dev_err, void* ws, size_t ws_bytes, void* stream) {
  if (!cfg_ok(c)) return DFLASH2_ERR_SHAPE;
  if (batch < 1 || !taps_h || !n_new_h || !block_tokens_h || !target_h || !path_h || !scores_h || !accepted_h ||
      !emitted_h || !ws)
    return DFLASH2_ERR_ARG;
  // everything the step checks is checked before the first copy or launch, so a rejected call
  // leaves no queued work reading the caller's host buffers
  int rc = check_weights(c, w);
  if (rc) return rc;
  rc = check_kv(c, kv);
  if (rc) return rc;
  if ((uintptr_t)ws & 255u) return DFLASH2_ERR_ALIGN;
  const Plan P = make_plan(c, batch);
  if (ws_bytes < P.total) return DFLASH2_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t Mb = P.Mb;
  CK(cudaMemcpyAsync(at<void>(ws, P.off_s_taps), taps_h, Mb * P.T * P.H * 2, cudaMemcpyHostToDevice, s));
  // While the taps copy runs: when every small buffer is page-locked, kernels read and write them
  // in place (one gather kernel and the acceptance kernel) instead of eight small copies.
  void* const small_h[] = {(void*)n_new_h, (void*)block_tokens_h, (void*)target_h, path_h, scores_h, accepted_h,
                           emitted_h, dev_err};
  void* small_d[8] = {};
  bool direct = true;
  for (int i = 0; i < (dev_err ? 8 : 7) && direct; ++i) {
    small_d[i] = host_mapped(small_h[i]);
    direct = small_d[i] != nullptr;
  }
  if (direct) {
    k_stage_host_inputs<<<1, 256, 0, s>>>((const int32_t*)small_d[0], (const int32_t*)small_d[1],
                                         (const int32_t*)small_d[2], batch, (int)Mb, at<int32_t>(ws, P.off_s_nnew),
                                         at<int32_t>(ws, P.off_s_btok), at<int32_t>(ws, P.off_s_tgt));
    CK(cudaGetLastError());
  } else {
    CK(cudaMemcpyAsync(at<void>(ws, P.off_s_nnew), n_new_h, (size_t)batch * 4, cudaMemcpyHostToDevice, s));
    CK(cudaMemcpyAsync(at<void>(ws, P.off_s_btok), block_tokens_h, Mb * 4, cudaMemcpyHostToDevice, s));
    CK(cudaMemcpyAsync(at<void>(ws, P.off_s_tgt), target_h, Mb * 4, cudaMemcpyHostToDevice, s));
  }
  dflash2_inputs in{at<uint16_t>(ws, P.off_s_taps), at<int32_t>(ws, P.off_s_nnew), at<int32_t>(ws, P.off_s_btok)};
  rc = dflash2_draft_step(c, w, &in, kv, batch, at<int32_t>(ws, P.off_s_path), at<float>(ws, P.off_s_scores), ws,
                          ws_bytes, nullptr, stream);
  if (rc) {
    cudaStreamSynchronize(s);  // queued copies may still read the caller's host buffers
    return rc;
  }
  if (direct) {
    const int n = std::max(batch * P.D, batch);
    k_accept_to_host<<<(n + 127) / 128, 128, 0, s>>>(
        at<int32_t>(ws, P.off_s_path), at<float>(ws, P.off_s_scores), at<int32_t>(ws, P.off_s_tgt), batch, P.Bk,
        at<int>(ws, P.off_err), (int32_t*)small_d[3], (float*)small_d[4], (int32_t*)small_d[5], (int32_t*)small_d[6],
        (int32_t*)small_d[7]);
    CK(cudaGetLastError());
  } else {
    rc = dflash2_accept(at<int32_t>(ws, P.off_s_path), at<int32_t>(ws, P.off_s_tgt), batch, P.Bk,
                        at<int32_t>(ws, P.off_s_acc), at<int32_t>(ws, P.off_s_emit), stream);
    if (rc) return rc;
    CK(cudaMemcpyAsync(path_h, at<void>(ws, P.off_s_path), (size_t)batch * P.D * 4, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(scores_h, at<void>(ws, P.off_s_scores), (size_t)batch * P.D * 4, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(accepted_h, at<void>(ws, P.off_s_acc), (size_t)batch * 4, cudaMemcpyDeviceToHost, s));
    CK(cudaMemcpyAsync(emitted_h, at<void>(ws, P.off_s_emit), Mb * 4, cudaMemcpyDeviceToHost, s));
    if (dev_err) CK(cudaMemcpyAsync(dev_err, at<void>(ws, P.off_err), 4, cudaMemcpyDeviceToHost, s));
  }
  CK(cudaStreamSynchronize(s));
  return DFLASH2_OK;
}

int32_t dflash2_step_kernels(const dflash2_config* c, int32_t batch) {
  if (!cfg_ok(c) || batch < 1) return 0;
  const Plan P = make_plan(c, batch);
  // embed, fc GEMV, fc norm | per layer: W_dc GEMV (+ convolution), QKV GEMV, attention (+ a merge
  // kernel when the merge is not fused in), W_o GEMV, gate/up GEMV, W_d GEMV | final norm, LM head
  // pass(es), selector (transition scores, the last CTA of a request runs its Viterbi path)
  // (a tensor-core product is two kernels: the product and its fix-up)
  const GemvPlan* gp[6] = {&P.dc, &P.qkv, &P.o, &P.gu, &P.dn, &P.fc};
  int extra = 0;
  for (int i = 0; i < 5; ++i) extra += gp[i]->umma ? c->layers : 0;
  extra += P.fc.umma ? 1 : 0;
  return 3 + (P.attn_stream || P.attn_ntk > 0 ? 6 : 7) * c->layers + 1 + 1 + 1 + extra;
}

int dflash2_device_error(const void* ws, int32_t* out_bits, void* stream) {
  if (!ws || !out_bits) return DFLASH2_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  CK(cudaMemcpyAsync(out_bits, ws, 4, cudaMemcpyDeviceToHost, s));
  CK(cudaStreamSynchronize(s));
  return DFLASH2_OK;
}

const char* dflash2_strerror(int code) {
  switch (code) {
    case DFLASH2_OK: return "ok";
    case DFLASH2_ERR_ARG: return "null pointer or bad argument";
    case DFLASH2_ERR_SHAPE: return "configuration not supported by the kernels";
    case DFLASH2_ERR_ALIGN: return "device pointer not 16-byte aligned (workspace: 256-byte)";
    case DFLASH2_ERR_WORKSPACE: return "workspace or prepared-weight buffer too small";
    case DFLASH2_ERR_CUDA: return "CUDA launch or copy failed";
    case DFLASH2_ERR_LAYOUT: return "Q4_K weights must go through dflash2_prepare_weights";
    case DFLASH2_ERR_STATIC_LIMIT: return "request needs more scratch than the allocation-free entry point holds";
  }
  return "unknown error";
}

}  // extern "C"
