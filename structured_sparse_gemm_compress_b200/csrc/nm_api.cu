// nm_api.cu -- the C ABI of libnmspmm (declared in include/nmspmm.h):
// argument validation, handle lifetime, the per-shape launch plan (adaptive
// parallelism, "Realizable N:M Sparse Transformer Inference via Search-Kernel
// Co-Design", section 4.1 mechanism 3), activation tensor maps and the split-K
// workspace.  All arithmetic runs in the kernels of nm_pack.cu / nm_spmm.cu.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <string>

#include "nmspmm.h"
#include "nm_device.cuh"
#include "nm_internal.h"

namespace {

thread_local std::string g_err;

nm_status fail(nm_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
nm_status fail(nm_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

nm_status cuda_fail(cudaError_t e, const char* what) {
  return fail(e == cudaErrorMemoryAllocation ? NM_ERR_OOM : NM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int num_sms(int dev) {
  static int cache[64] = {0};
  if (dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

int env_int(const char* name, int dflt) {
  const char* v = getenv(name);
  return (v && *v) ? atoi(v) : dflt;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Activation X [T][k] as a 2-D tensor: inner dim k, box = 128 bytes x bn rows,
// 128-byte swizzle (the layout the MMA's K-major B descriptor expects);
// out-of-range rows and columns read as zero.
nm_status make_x_map(nm_handle* h, const void* X, int64_t T, int bn) {  // bn = token rows per box
  if (h->tm_x == X && h->tm_T == T && h->tm_bn == bn) return NM_OK;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(NM_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const int es = nm::elem_bytes(h->dt);
  CUtensorMapDataType ty = h->dt == nm::DT_I8    ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                           : h->dt == nm::DT_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cuuint64_t dims[2] = {(cuuint64_t)h->k, (cuuint64_t)T};
  cuuint64_t strides[1] = {(cuuint64_t)(h->k * es)};
  cuuint32_t box[2] = {(cuuint32_t)(128 / es), (cuuint32_t)bn};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&h->tm, ty, 2, const_cast<void*>(X), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    h->tm_x = nullptr;
    return fail(NM_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for T=%lld k=%lld", (int)r, (long long)T,
                (long long)h->k);
  }
  h->tm_x = X;
  h->tm_T = T;
  h->tm_bn = bn;
  h->tm_ld = -1;
  return NM_OK;
}

// Feature-major activation Xt [k][ldx] (only the first T columns exist) as a
// 2-D tensor whose rows are features: box = one row x 128 bytes of tokens,
// 128-byte swizzle, so a four-row gather lands as four rows of the MN-major
// operand layout; tokens beyond T read as zero.
nm_status make_xt_map(nm_handle* h, const void* Xt, int64_t ldx, int64_t T) {
  if (h->tm_x == Xt && h->tm_T == T && h->tm_ld == ldx) return NM_OK;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(NM_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const int es = nm::elem_bytes(h->dt);
  CUtensorMapDataType ty = h->dt == nm::DT_I8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  cuuint64_t dims[2] = {(cuuint64_t)T, (cuuint64_t)h->k};
  cuuint64_t strides[1] = {(cuuint64_t)(ldx * es)};
  cuuint32_t box[2] = {(cuuint32_t)(128 / es), 1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&h->tm, ty, 2, const_cast<void*>(Xt), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    h->tm_x = nullptr;
    return fail(NM_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for Xt with T=%lld ldx=%lld k=%lld", (int)r,
                (long long)T, (long long)ldx, (long long)h->k);
  }
  h->tm_x = Xt;
  h->tm_T = T;
  h->tm_ld = ldx;
  h->tm_bn = 0;
  return NM_OK;
}

// The packed operand image as a 2-D tensor of 128-byte rows, so one tensor
// copy with a box of (chunk bytes / 128) rows brings one chunk (values and
// positions together) into shared memory.
nm_status make_w_map(nm_handle* h) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(NM_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t rows = (cuuint64_t)(h->bpack_bytes / 128);
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {128, (cuuint32_t)(h->chunk / 128)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&h->tmw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, h->d_bpack, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NM_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for the packed image", (int)r);
  h->has_tmw = 1;
  return NM_OK;
}

// Output Y [T][n_out] as a 2-D tensor for the epilogue's TMA stores: box =
// 32 channels x ch tokens, no swizzle; stores outside the tensor are clipped.
// Returns false (direct stores instead) when the row pitch is not a multiple of
// 16 bytes, which TMA requires.
bool make_y_map(nm_handle* h, void* Y, int64_t T, int out_es, int out_ty, int ch, nm_status* st) {
  *st = NM_OK;
  if ((h->n_out * out_es) % 16 != 0) return false;
  const int key = out_ty * 1024 + ch;
  if (h->tmy_y == Y && h->tmy_T == T && h->tmy_out == key) return true;
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    *st = fail(NM_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    return false;
  }
  cuuint64_t dims[2] = {(cuuint64_t)h->n_out, (cuuint64_t)T};
  cuuint64_t strides[1] = {(cuuint64_t)(h->n_out * out_es)};
  cuuint32_t box[2] = {32, (cuuint32_t)ch};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&h->tmy, (CUtensorMapDataType)out_ty, 2, Y, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    h->tmy_y = nullptr;
    *st = fail(NM_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for the output", (int)r);
    return false;
  }
  h->tmy_y = Y;
  h->tmy_T = T;
  h->tmy_out = key;
  return true;
}

// Output element type and size of a launch: int32 / fp32 for INT8 (without /
// with scale), else the input's 16-bit type.
void out_type(const nm_handle* h, bool scaled, int* es, int* ty) {
  if (h->dt == nm::DT_I8) {
    *es = 4;
    *ty = scaled ? (int)CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : (int)CU_TENSOR_MAP_DATA_TYPE_INT32;
  } else {
    *es = 2;
    *ty = h->dt == nm::DT_F16 ? (int)CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : (int)CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  }
}

int out_code(const nm_handle* h, bool scaled) {
  if (h->dt == nm::DT_I8) return scaled ? nm::OUT_F32 : nm::OUT_I32;
  return h->dt == nm::DT_F16 ? nm::OUT_F16 : nm::OUT_BF16;
}

// Resident-cluster capacities the planner consults: queried from the device
// (device_capacity), or given by the caller of nm_plan_for_shape so that the
// planner's rules can be exercised without a GPU.
struct Capacity {
  int pair[3] = {0, 0, 0};                // resident CTA pairs of the two-SM kernel, token tiles 224 / 192 / 128
  int stream[nm::kMaxClusterSplit + 1] = {};  // [S]: resident clusters of S one-SM CTAs (S = 1 .. 8)
};

constexpr int kPairTiles[3] = {224, 192, 128};

int pair_slot(int bn) { return bn == 224 ? 0 : bn == 192 ? 1 : 2; }

Capacity device_capacity(const nm_handle* h, bool scaled) {
  Capacity c;
  if (!h->tile)
    for (int i = 0; i < 3; ++i) c.pair[i] = nm::pair_max_clusters(h->dt, h->img, kPairTiles[i], out_code(h, scaled));
  for (int S = 1; S <= nm::kMaxClusterSplit; ++S) c.stream[S] = nm::stream_max_clusters(S);
  return c;
}

// Small-token model of one streaming launch (us), fitted on B200 to a sweep of
// forced (token tile, split) plans over the ViT-B INT8 shapes at T = 16 .. 788
// (CUDA graphs of back-to-back launches; within ~5 % of every point):
//   waves x (start + epilogue + reduction + load), where
//   load = max(k-blocks per CTA x per-k-block time at one SM's L2 rate,
//              operand bytes of the resident tiles / aggregate L2 rate),
// the reduction (cluster launch, two cluster barriers, parked partials read
// through distributed shared memory) paid only when k is split.
struct SmallTModel {
  double start = 2.7;          // launch, first operand latency, completion
  double per_kb = 0.24;        // one k-block at one SM's L2 rate, plus per token column:
  double per_kb_tok = 0.0006;
  double epi_tok = 0.004;      // epilogue per token column
  double red = 1.2;            // on-chip reduction, plus per token column:
  double red_tok = 0.012;
  double l2_bytes_per_us = 10.0e6;  // aggregate L2 -> SM operand rate (~10 TB/s)
};

double small_t_cost(const nm_handle* h, int64_t T, int sms, int bn, int S, const Capacity& capacity) {
  const SmallTModel m;
  const int64_t tiles = (int64_t)h->n_ct * ((T + bn - 1) / bn);
  const int kbs = (h->n_kb + S - 1) / S;
  int64_t cap = sms;  // tiles resident at once: one per SM, or one per resident cluster
  if (S > 1) {
    const int c = capacity.stream[S];
    if (c <= 0) return 1e300;
    cap = c;
  }
  const int64_t waves = (tiles + cap - 1) / cap;
  const double stage = (double)nm::chunk_bytes(h->dt, h->img) + 256.0 * bn;  // packed chunk + X rows
  const double load = std::max(kbs * (m.per_kb + m.per_kb_tok * bn),
                               (double)std::min(tiles, cap) * h->n_kb * stage / m.l2_bytes_per_us);
  double t = m.start + m.epi_tok * bn + load;
  if (S > 1) t += m.red + m.red_tok * bn;
  return (double)waves * t;
}

// For a shape whose unsplit tiles leave SMs idle: keeps the streaming rule's
// token tile unsplit unless, by the model above, some (token tile, split > 1)
// is clearly faster; then sets both.  (Measured: at T <= 64 the K = 3072 ViT-B
// layer drops from 5.8 to 4.8 us with 6 splits of 32-token tiles; K = 768
// layers, whose 3 k-blocks leave nothing to split, stay unsplit.)
void choose_cluster_split(const nm_handle* h, int64_t T, int sms, int forced_bn, const Capacity& capacity, nm::Plan* p,
                          int* splits) {
  double best = small_t_cost(h, T, sms, p->bn, 1, capacity);
  for (int bn : {32, 64, 128}) {
    if (forced_bn && bn != forced_bn) continue;
    for (int S = 2; S <= std::min(nm::kMaxClusterSplit, h->n_kb); ++S) {
      const int kps = (h->n_kb + S - 1) / S;
      if ((h->n_kb + kps - 1) / kps != S) continue;  // every split owns >= 1 k-block
      const double c = small_t_cost(h, T, sms, bn, S, capacity);
      if (c < best * 0.95) {  // a clear win only
        best = c;
        p->bn = bn;
        *splits = S;
      }
    }
  }
}

// Adaptive parallelism: pick the kernel (CTA pair or single SM), the token tile
// and the split-K factor for this shape (rules and their measurements below),
// given the resident-cluster capacities.
nm::Plan plan_with(const nm_handle* h, int64_t T, int sms, const Capacity& capacity) {
  nm::Plan p;
  const int forced_bn = env_int("NMSPMM_FORCE_BN", 0);
  const int forced_split = env_int("NMSPMM_FORCE_SPLITK", 0);
  const int forced_xs = env_int("NMSPMM_FORCE_XS", -1);  // -1 auto, 0 off, 1 on when eligible
  const int forced_grid = env_int("NMSPMM_FORCE_GRID", 0);  // cap on persistent CTAs (tests, sweeps)
  if (forced_grid > 0) sms = std::min(sms, forced_grid);
  if (h->tile) {
    // Gather image (streaming kernel only): token tiles of 256 or 128, by the
    // same waves x (BN + fixed cost) model as below; split-K only when forced.
    double best = 1e300;
    for (int bn : {256, 128}) {
      if (forced_bn && bn != forced_bn) continue;
      const int64_t tiles = (int64_t)h->n_ct * ((T + bn - 1) / bn);
      const double cost = (double)((tiles + sms - 1) / sms) * (bn + 140);
      if (cost < best) {
        best = cost;
        p.bn = bn;
      }
    }
    p.n_tt = (int)((T + p.bn - 1) / p.bn);
    const int splits = std::max(1, std::min(forced_split > 0 ? forced_split : 1, h->n_kb));
    p.kb_per_split = (h->n_kb + splits - 1) / splits;
    p.splits = (h->n_kb + p.kb_per_split - 1) / p.kb_per_split;
    p.units = (int)((int64_t)h->n_ct * p.n_tt * p.splits);
    p.grid = std::min(p.units, sms);
    return p;
  }
  // CTA-pair mode (M = 256 per MMA, one issuing thread per two SMs): whenever
  // there are enough 256-channel x BN-token tiles to occupy every resident pair.
  const int forced_pair = env_int("NMSPMM_FORCE_PAIR", -1);  // -1 auto, 0 off, 1 on
  // Measured on B200 (CUDA-graph timing of both kernels, INT8 and FP16, K = 192 .. 1536,
  // n_out = 192 .. 3072, T = 6272 .. 100352): the pair is the faster kernel whenever its
  // 256-channel tiles are whole (an even number of 128-channel tiles; with an odd number the
  // last pair computes a padding tile, a quarter or more of the work at the ViT and Swin
  // widths) and there are at least as many 256 x 128 pair tiles as SMs (fewer, and the single-SM
  // kernel's smaller tiles balance better); by 5-25 % at K = 768 .. 1536, as its operand bytes
  // in flight per SM pair and its single MMA issuer outweigh the streaming kernel's shorter
  // tiles.  A long k loop (>= 2 KB of X per token) takes it regardless: per-stage issue cost
  // and X re-reads dominate there.
  const int64_t kbytes = h->k * nm::elem_bytes(h->dt);
  const bool pair_default = kbytes >= 2048 ||
                            (kbytes >= 192 && h->n_ct % 2 == 0 && (int64_t)(h->n_ct / 2) * ((T + 127) / 128) >= sms);
  if ((forced_pair == 1 || (forced_pair == -1 && pair_default)) && forced_split <= 1 && forced_xs != 1) {
    const int cands[3] = {224, 192, 128};
    double best_cost = 1e300;
    for (int bn : cands) {
      if (forced_bn && bn != forced_bn) continue;
      int clusters = capacity.pair[pair_slot(bn)];
      if (clusters <= 0) continue;
      if (forced_grid > 0) clusters = std::min(clusters, std::max(1, forced_grid / 2));
      const int64_t units = (int64_t)((h->n_ct + 1) / 2) * ((T + bn - 1) / bn);
      if (forced_pair != 1 && units < clusters) continue;
      const int64_t rounds = (units + clusters - 1) / clusters;
      const double cost = (double)rounds * (bn + 48);
      if (cost < best_cost) {
        best_cost = cost;
        p.pair = 1;
        p.bn = bn;
        p.n_tt = (int)((T + bn - 1) / bn);
        p.splits = 1;
        p.kb_per_split = h->n_kb;
        p.units = (int)units;
        p.grid = (int)std::min<int64_t>(units, clusters);
      }
    }
    if (p.pair) return p;
  }
  // X-stationary mode: INT8 with at most kXsMaxKb k-blocks, several channel tiles
  // sharing each X tile, and enough 128-token tiles to fill the SMs without split-K.
  const int64_t tt128 = (T + 127) / 128;
  const bool xs_ok = h->dt == nm::DT_I8 && h->n_kb <= nm::kXsMaxKb && (forced_bn == 0 || forced_bn == 128) &&
                     forced_split <= 1 && h->n_ct >= 2;
  if (xs_ok && forced_xs == 1) {  // measured slower than streaming by default: its write order is scattered
    p.bn = 128;
    p.xkb = h->n_kb;
    p.n_tt = (int)tt128;
    p.splits = 1;
    p.kb_per_split = h->n_kb;
    p.units = (int)(tt128 * h->n_ct);
    p.grid = std::min(p.units, sms);
    return p;
  }
  // Streaming token tile: minimise (waves of persistent CTAs) x (cost of one
  // tile).  Measured on B200 (ViT-B INT8 shapes at T = 12608 and 50432): a tile
  // costs about (BN + 140) token columns' worth -- its fixed part (weight chunk
  // loads, MMA issue per stage, epilogue start) equals ~140 columns -- and 18 %
  // more when only three pipeline stages fit in shared memory.  Tiles that
  // would leave two stages are not used.
  const int bns[4] = {192, 128, 64, 32};
  double best = 1e300;
  for (int bn : bns) {
    if (forced_bn && bn != forced_bn) continue;
    const int stage = nm::chunk_bytes(h->dt, h->img) + bn * 256;  // packed chunk + 256 B of X per token
    const int stages = std::min(8, (227 * 1024 - 1024) / stage);
    if (stages < 3 && bn > 128) continue;
    const int64_t tiles = (int64_t)h->n_ct * ((T + bn - 1) / bn);
    const int64_t waves = (tiles + sms - 1) / sms;
    const double cost = (double)waves * (bn + 140) * (stages >= 4 ? 1.0 : 1.18);
    if (cost < best) {
      best = cost;
      p.bn = bn;
    }
  }
  int splits = 1;
  if (forced_split > 0) {
    splits = forced_split;
  } else if (env_int("NMSPMM_CSPLIT", 1) != 0) {
    // Small token counts: too few tiles to occupy the SMs.  Split k over the
    // CTAs of a cluster, which sum their partials on chip (no workspace), when
    // the model below says that beats the unsplit tile.
    const int64_t tiles0 = (int64_t)h->n_ct * ((T + p.bn - 1) / p.bn);
    if (tiles0 < sms) choose_cluster_split(h, T, sms, forced_bn, capacity, &p, &splits);
  }
  p.n_tt = (int)((T + p.bn - 1) / p.bn);
  const int64_t tiles = (int64_t)h->n_ct * p.n_tt;
  splits = std::max(1, std::min(splits, h->n_kb));
  p.kb_per_split = (h->n_kb + splits - 1) / splits;
  p.splits = (h->n_kb + p.kb_per_split - 1) / p.kb_per_split;  // every split owns >= 1 k-block
  p.units = (int)(tiles * p.splits);
  p.grid = std::min(p.units, sms);
  // Splits of one tile form a cluster and reduce through distributed shared
  // memory (one unit per CTA: the grid is every unit), unless the global
  // workspace reduction is asked for (NMSPMM_SPLIT_GLOBAL=1) or the split is
  // wider than a portable cluster.
  if (p.splits > 1 && p.splits <= nm::kMaxClusterSplit && env_int("NMSPMM_SPLIT_GLOBAL", 0) == 0 &&
      capacity.stream[p.splits] > 0) {
    p.cluster = 1;
    p.grid = p.units;
  }
  return p;
}

// The plan for a call on this handle's device.
nm::Plan make_plan(const nm_handle* h, int64_t T, int sms, bool scaled) {
  return plan_with(h, T, sms, device_capacity(h, scaled));
}

nm_status check_handle(const nm_handle* h) {
  if (!h) return fail(NM_ERR_INVALID, "null handle");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device)
    return fail(NM_ERR_INVALID, "handle belongs to device %d but the current device is %d", h->device, dev);
  return NM_OK;
}

// Output stage chosen at run time (nm_spmm_ex); out_ty < 0: the fixed stage of nm_spmm.
struct EpiReq {
  int out_ty = -1;  // nm::OUT_F32 / F16 / BF16 / I8
  const float* bias = nullptr;
  int act = nm::ACT_NONE;
  float out_scale = 1.0f;
};

int out_elem_bytes(const nm_handle* h, const EpiReq* ep) {
  if (ep && ep->out_ty >= 0)
    return ep->out_ty == nm::OUT_I8 ? 1 : (ep->out_ty == nm::OUT_F32 ? 4 : 2);
  return h->dt == nm::DT_I8 ? 4 : 2;
}

// Split-K partial tiles and per-tile arrival counters of the handle, grown
// (after a device synchronisation: earlier launches may still use the old
// ones) when plan `p` needs more than the handle holds.
nm_status ensure_split_workspace(nm_handle* h, const nm::Plan& p) {
  const int tiles = h->n_ct * p.n_tt;
  const size_t need = (size_t)tiles * p.splits * p.bn * nm::kRows * 4;
  if (need <= h->ws_bytes && tiles <= h->cnt_len) return NM_OK;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "synchronise before growing the split-K workspace");
  cudaFree(h->d_ws);
  cudaFree(h->d_cnt);
  h->d_ws = nullptr;
  h->d_cnt = nullptr;
  h->ws_bytes = 0;
  h->cnt_len = 0;
  const int cl = std::max(tiles, 256);
  if ((e = cudaMalloc(&h->d_ws, need)) != cudaSuccess) return cuda_fail(e, "allocate split-K workspace");
  if ((e = cudaMalloc(&h->d_cnt, (size_t)cl * sizeof(int))) != cudaSuccess)
    return cuda_fail(e, "allocate split-K counters");
  if ((e = cudaMemset(h->d_cnt, 0, (size_t)cl * sizeof(int))) != cudaSuccess)
    return cuda_fail(e, "clear split-K counters");
  h->ws_bytes = need;
  h->cnt_len = cl;
  return NM_OK;
}

// Validates the output stage `ep` for handle `h`.  *fixed: the fixed stages
// of nm_spmm compute exactly these values (r is then unused); otherwise r is
// the runtime stage to run.
nm_status resolve_epilogue(const nm_handle* h, const nm_epilogue* ep, bool* fixed, EpiReq* r) {
  if ((int)ep->out < 0 || (int)ep->out > 5) return fail(NM_ERR_INVALID, "unknown output type %d", (int)ep->out);
  if ((int)ep->act < 0 || (int)ep->act > 1) return fail(NM_ERR_INVALID, "unknown activation %d", (int)ep->act);
  if ((ep->scale && !aligned(ep->scale, 4)) || (ep->bias && !aligned(ep->bias, 4)))
    return fail(NM_ERR_INVALID, "scale and bias must be 4-byte aligned");
  const bool plain = !ep->scale && !ep->bias && ep->act == NM_ACT_NONE;
  const bool int_in = h->dt == nm::DT_I8;
  nm_out_type out = ep->out;
  if (out == NM_OUT_DEFAULT)
    out = int_in ? (plain ? NM_OUT_INT32 : NM_OUT_FP32) : (h->dt == nm::DT_F16 ? NM_OUT_FP16 : NM_OUT_BF16);
  if (!int_in && (out == NM_OUT_INT32 || out == NM_OUT_INT8))
    return fail(NM_ERR_UNSUPPORTED, "integer outputs need an INT8 handle");
  if (out == NM_OUT_INT32 && !plain)
    return fail(NM_ERR_INVALID, "NM_OUT_INT32 is the raw accumulator: no scale, bias or activation");
  if (out == NM_OUT_INT8 && !(std::isfinite(ep->out_scale) && ep->out_scale > 0.0f))
    return fail(NM_ERR_INVALID, "out_scale must be finite and positive for NM_OUT_INT8");
  *fixed = ep->act == NM_ACT_NONE && !ep->bias &&
           ((int_in && out == NM_OUT_INT32) || (int_in && out == NM_OUT_FP32 && ep->scale) ||
            (h->dt == nm::DT_F16 && out == NM_OUT_FP16) || (h->dt == nm::DT_BF16 && out == NM_OUT_BF16));
  r->out_ty = out == NM_OUT_FP32 ? nm::OUT_F32 : out == NM_OUT_FP16 ? nm::OUT_F16 : out == NM_OUT_BF16 ? nm::OUT_BF16
                                                                                                       : nm::OUT_I8;
  r->bias = ep->bias;
  r->act = ep->act == NM_ACT_GELU ? nm::ACT_GELU : nm::ACT_NONE;
  r->out_scale = ep->out_scale;
  return NM_OK;
}

nm_status reject_tile(const nm_handle* h) {
  if (h->tile) return fail(NM_ERR_INVALID, "the handle was made by nm_compress_tile: its product is nm_spmm_gather");
  return NM_OK;
}

// Split-K scratch supplied by the caller instead of the handle's workspace
// (nm_spmm_noalloc): partial tiles and arrival counters with their capacities.
struct SplitScratch {
  void* ws = nullptr;
  size_t ws_bytes = 0;
  int* cnt = nullptr;
  int cnt_len = 0;
};

// Workspace of a global-memory split-K launch of plan `p`: the handle's (grown
// on demand) or the caller's `ext` (never grown: too small is an error).  The
// tiles' arrival counters are cleared on the stream before the launch: a
// launch that gave up a bounded wait can leave them part-counted.
nm_status split_workspace(nm_handle* h, const nm::Plan& p, const SplitScratch* ext, cudaStream_t s,
                          nm::SpmmArgs* a) {
  const int tiles = h->n_ct * p.n_tt;
  if (ext) {
    const size_t need = (size_t)tiles * p.splits * p.bn * nm::kRows * 4;
    if (need > ext->ws_bytes || tiles > ext->cnt_len)
      return fail(NM_ERR_UNSUPPORTED,
                  "this shape needs %zu bytes of split-K scratch for %d tiles; the allocation-free entry point "
                  "holds at most %zu bytes and %d tiles (use nm_spmm)",
                  need, tiles, ext->ws_bytes, ext->cnt_len);
    a->ws = ext->ws;
    a->cnt = ext->cnt;
  } else {
    nm_status st = ensure_split_workspace(h, p);
    if (st != NM_OK) return st;
    a->ws = h->d_ws;
    a->cnt = h->d_cnt;
  }
  cudaError_t e = cudaMemsetAsync(a->cnt, 0, (size_t)tiles * sizeof(int), s);
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "clear the split-K counters");
}

nm_status spmm_impl(const nm_handle* hc, const void* X, int64_t T, void* Y, const float* scale, void* stream,
                    int inject_skip, unsigned long long timeout_ns, const EpiReq* ep = nullptr,
                    const SplitScratch* ext = nullptr) {
  g_err.clear();
  nm_status st = check_handle(hc);
  if (st != NM_OK) return st;
  if ((st = reject_tile(hc)) != NM_OK) return st;
  nm_handle* h = const_cast<nm_handle*>(hc);  // only caches (tensor map, workspace) change
  if (T < 0) return fail(NM_ERR_INVALID, "T must be >= 0 (got %lld)", (long long)T);
  if (T == 0) return NM_OK;
  if (!X || !Y) return fail(NM_ERR_INVALID, "null X or Y");
  if (T > INT32_MAX) return fail(NM_ERR_UNSUPPORTED, "T above 2^31-1");
  const int es = nm::elem_bytes(h->dt);
  if (!aligned(X, 16) || !aligned(Y, 16)) return fail(NM_ERR_INVALID, "X and Y must be 16-byte aligned");
  if ((h->k * es) % 16 != 0)
    return fail(NM_ERR_UNSUPPORTED, "k * sizeof(dtype) must be a multiple of 16 bytes (k=%lld)", (long long)h->k);
  if (scale && !aligned(scale, 4)) return fail(NM_ERR_INVALID, "scale must be 4-byte aligned");
  const size_t ybytes = (size_t)T * h->n_out * out_elem_bytes(h, ep);
  const size_t xbytes = (size_t)T * h->k * es;
  const uintptr_t xs = (uintptr_t)X, ys = (uintptr_t)Y;
  if (xs < ys + ybytes && ys < xs + xbytes) return fail(NM_ERR_INVALID, "Y overlaps X");

  const int sms = num_sms(h->device);
  nm::Plan p = make_plan(h, T, sms, scale != nullptr);
  st = make_x_map(h, X, T, p.pair ? p.bn / 2 : p.bn);
  if (st != NM_OK) return st;

  nm::SpmmArgs a{};
  a.bpack = h->d_bpack;
  a.Y = Y;
  a.scale = scale;
  a.err = h->d_err;
  a.T = (int)T;
  a.n_out = (int)h->n_out;
  a.n_kb = h->n_kb;
  a.n_ct = h->n_ct;
  a.n_tt = p.n_tt;
  a.splits = p.splits;
  a.kb_per_split = p.kb_per_split;
  a.units = p.units;
  a.timeout_ns = timeout_ns;
  a.inject_skip = inject_skip;
  a.w_tma = (h->has_tmw && env_int("NMSPMM_W_BULK", 0) == 0) ? 1 : 0;
  a.out_ty = ep ? ep->out_ty : -1;
  a.bias = ep ? ep->bias : nullptr;
  a.act = ep ? ep->act : nm::ACT_NONE;
  a.out_scale = ep ? ep->out_scale : 1.0f;
#ifdef NM_TRACE
  // timeline builds only: device buffer of grid * kTraceStride int64 given as an integer address
  if (const char* tp = getenv("NMSPMM_TRACE_PTR")) a.trace = reinterpret_cast<long long*>(strtoull(tp, nullptr, 0));
#endif
  a.prefetch = std::max(0, std::min(2, env_int("NMSPMM_PREFETCH", 2)));
  if (p.cluster) {
    a.csplit = 1;  // partials summed on chip: no workspace
  } else if (p.splits > 1) {
    if ((st = split_workspace(h, p, ext, (cudaStream_t)stream, &a)) != NM_OK) return st;
  }
  int oes, oty;
  out_type(h, scale != nullptr, &oes, &oty);
  const int wcols = p.bn / nm::epw_for(false);  // token columns per epilogue warp; the TMA-store box
  const int ych = p.pair ? (wcols % 32 == 0 ? 32 : wcols % 16 == 0 ? 16 : 8)
                         : (wcols % 32 == 0 ? 32 : (wcols % 8 == 0 && wcols <= 96) ? wcols : 8);
  // Direct stores measured faster than staged TMA stores (they keep the TMA unit
  // for operand loads); the TMA-store epilogue remains selectable.
  a.tma_store = 0;
  if (env_int("NMSPMM_TMA_STORE", 0) && a.out_ty < 0 && !p.cluster)
    a.tma_store = make_y_map(h, Y, T, oes, oty, ych, &st) ? 1 : 0;
  if (st != NM_OK) return st;
  cudaError_t e = nm::launch_spmm(h, &h->tm, &h->tmy, p, a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "launch SpMM kernel");
  return NM_OK;
}

// ---- scratch of the allocation-free entry point (nm_spmm_noalloc)
//
// A fixed, file-scope device array instead of cudaMalloc: 4 MiB of split-K
// partial tiles followed by 1024 per-tile arrival counters.  Every GPU that
// loads this library holds it until the process exits.  Host code may not use
// the array's name as an address (on the host it is only a stand-in), so the
// first call on each device looks its device address up with
// cudaGetSymbolAddress while that device is current, and passes that address
// to the kernel.
constexpr size_t kNoAllocPartialBytes = size_t(4) << 20;
constexpr int kNoAllocCounters = 1024;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocPartialBytes + kNoAllocCounters * sizeof(int)];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[64] = {};

nm_status noalloc_scratch(int dev, void** out) {
  if (dev < 0 || dev >= 64) return fail(NM_ERR_UNSUPPORTED, "device index %d above 63", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "look up the device address of the static split-K scratch");
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return NM_OK;
}

// nm_spmm_gather / nm_spmm_gather_ex (defined after the exported calls that use it).
nm_status gather_impl(const nm_handle* hc, const void* Xt, int64_t ldx, int64_t T, void* Y, const float* scale,
                      void* stream, const EpiReq* ep);

}  // namespace

extern "C" {

const char* nm_last_error(void) { return g_err.c_str(); }

const char* nm_version(void) { return "nmspmm 0.1.0 (sm_100a)"; }

nm_status nm_compress(const void* W_dev, int64_t n_out, int64_t k, nm_dtype dt, int N, int M, void* stream,
                      nm_handle** out) {
  g_err.clear();
  if (!out) return fail(NM_ERR_INVALID, "null output handle pointer");
  *out = nullptr;
  if (!W_dev) return fail(NM_ERR_INVALID, "null W");
  if ((int)dt < 0 || (int)dt > 2) return fail(NM_ERR_INVALID, "unknown dtype %d", (int)dt);
  if (n_out <= 0 || k <= 0) return fail(NM_ERR_INVALID, "n_out and k must be positive");
  if (n_out > (1 << 24) || k > (1 << 24)) return fail(NM_ERR_UNSUPPORTED, "n_out and k are limited to 2^24");
  // INT8 accumulates exactly in int32: |acc| <= k * 128 * 127 must stay below 2^31.
  if (dt == NM_INT8 && k > (1 << 17))
    return fail(NM_ERR_UNSUPPORTED, "INT8 k is limited to 2^17 (int32 accumulation must not overflow)");
  if (M <= 0 || N <= 0 || N > M) return fail(NM_ERR_INVALID, "bad N:M %d:%d", N, M);
  const bool sp24 = (N == 1 && M == 4) || (N == 2 && M == 4) || (N == 2 && M == 8);
  const bool dense = (N == 4 && M == 8) || (N == M && (M == 4 || M == 8));
  if (!sp24 && !dense) return fail(NM_ERR_UNSUPPORTED, "N:M %d:%d is not supported", N, M);
  if (k % M != 0) return fail(NM_ERR_INVALID, "k=%lld is not a multiple of M=%d", (long long)k, M);
  const int es = nm::elem_bytes((int)dt);
  if (!aligned(W_dev, (size_t)es)) return fail(NM_ERR_INVALID, "W is not element aligned");

  nm_handle* h = new (std::nothrow) nm_handle();
  if (!h) return fail(NM_ERR_OOM, "host allocation failed");
  cudaGetDevice(&h->device);
  h->n_out = n_out;
  h->k = k;
  h->N = N;
  h->M = M;
  h->dt = (int)dt;
  h->img = sp24 ? nm::IMG_SP24 : nm::IMG_DENSE;
  const int KB = nm::kblock_elems(h->dt);
  h->n_kb = (int)((k + KB - 1) / KB);
  h->n_ct = (int)((n_out + nm::kRows - 1) / nm::kRows);
  h->chunk = (size_t)nm::chunk_bytes(h->dt, h->img);
  h->values_bytes = (size_t)n_out * (size_t)(k / M) * N * es;
  h->idx_pitch = ((k / M) * N + 1) / 2;
  h->idx_bytes = (size_t)n_out * (size_t)h->idx_pitch;
  h->bpack_bytes = (size_t)h->n_ct * h->n_kb * h->chunk;

  cudaError_t e;
  nm_status st = NM_OK;
  if ((e = cudaMalloc(&h->d_values, h->values_bytes)) != cudaSuccess) st = cuda_fail(e, "allocate values");
  else if ((e = cudaMalloc(&h->d_idx, h->idx_bytes)) != cudaSuccess) st = cuda_fail(e, "allocate idx");
  else if ((e = cudaMalloc(&h->d_bpack, h->bpack_bytes)) != cudaSuccess) st = cuda_fail(e, "allocate packed image");
  else if ((e = cudaMalloc(&h->d_err, sizeof(int))) != cudaSuccess) st = cuda_fail(e, "allocate error word");
  else if ((e = cudaMemsetAsync(h->d_err, 0, sizeof(int), (cudaStream_t)stream)) != cudaSuccess)
    st = cuda_fail(e, "clear error word");
  else if ((e = nm::launch_compress(h, W_dev, (cudaStream_t)stream)) != cudaSuccess)
    st = cuda_fail(e, "launch compress kernel");
  else
    st = make_w_map(h);
  if (st != NM_OK) {
    const std::string msg = g_err;
    nm_destroy(h);
    g_err = msg;
    return st;
  }
  *out = h;
  return NM_OK;
}

nm_status nm_recompress(nm_handle* h, const void* W_dev, void* stream) {
  g_err.clear();
  nm_status st = check_handle(h);
  if (st != NM_OK) return st;
  if (!W_dev) return fail(NM_ERR_INVALID, "null W");
  if (!aligned(W_dev, (size_t)nm::elem_bytes(h->dt))) return fail(NM_ERR_INVALID, "W is not element aligned");
  cudaError_t e = h->tile ? nm::launch_compress_tile(h, W_dev, (cudaStream_t)stream)
                          : nm::launch_compress(h, W_dev, (cudaStream_t)stream);
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "launch compress kernel");
}

nm_status nm_spmm(const nm_handle* h, const void* X_dev, int64_t T, void* Y_dev, const float* scale_dev,
                  void* stream) {
  return spmm_impl(h, X_dev, T, Y_dev, scale_dev, stream, -1, 1000000000ull);
}

nm_status nm_spmm_ex(const nm_handle* h, const void* X_dev, int64_t T, void* Y_dev, const nm_epilogue* ep,
                     void* stream) {
  g_err.clear();
  if (!ep) return spmm_impl(h, X_dev, T, Y_dev, nullptr, stream, -1, 1000000000ull);
  nm_status st = check_handle(h);
  if (st != NM_OK) return st;
  bool fixed = false;
  EpiReq r;
  if ((st = resolve_epilogue(h, ep, &fixed, &r)) != NM_OK) return st;
  return spmm_impl(h, X_dev, T, Y_dev, ep->scale, stream, -1, 1000000000ull, fixed ? nullptr : &r);
}

nm_status nm_test_spmm_skip_stage(const nm_handle* h, const void* X_dev, int64_t T, void* Y_dev,
                                  const float* scale_dev, void* stream, int skip_stage, int64_t timeout_ns) {
  if (timeout_ns <= 0 || timeout_ns > 2000000000ll) return fail(NM_ERR_INVALID, "timeout must be in (0, 2 s]");
  return spmm_impl(h, X_dev, T, Y_dev, scale_dev, stream, skip_stage, (unsigned long long)timeout_ns);
}

nm_status nm_compress_tile(const void* W_dev, int64_t n_out, int64_t k, nm_dtype dt, int N, int M, void* stream,
                           nm_handle** out) {
  g_err.clear();
  if (!out) return fail(NM_ERR_INVALID, "null output handle pointer");
  *out = nullptr;
  if (!W_dev) return fail(NM_ERR_INVALID, "null W");
  if ((int)dt < 0 || (int)dt > 2) return fail(NM_ERR_INVALID, "unknown dtype %d", (int)dt);
  if (dt == NM_BF16)
    return fail(NM_ERR_UNSUPPORTED, "tile-shared patterns need exact column sums: INT8 and FP16 only");
  if (n_out <= 0 || k <= 0) return fail(NM_ERR_INVALID, "n_out and k must be positive");
  if (n_out > (1 << 24) || k > (1 << 24)) return fail(NM_ERR_UNSUPPORTED, "n_out and k are limited to 2^24");
  if (dt == NM_INT8 && k > (1 << 17))
    return fail(NM_ERR_UNSUPPORTED, "INT8 k is limited to 2^17 (int32 accumulation must not overflow)");
  if (M <= 0 || N <= 0 || N > M) return fail(NM_ERR_INVALID, "bad N:M %d:%d", N, M);
  const bool ok = (N == 1 && M == 4) || (N == 2 && M == 4) || (N == 2 && M == 8) || (N == 4 && M == 8) ||
                  (N == M && (M == 4 || M == 8));
  if (!ok) return fail(NM_ERR_UNSUPPORTED, "N:M %d:%d is not supported", N, M);
  if (k % M != 0) return fail(NM_ERR_INVALID, "k=%lld is not a multiple of M=%d", (long long)k, M);
  const int es = nm::elem_bytes((int)dt);
  if (!aligned(W_dev, (size_t)es)) return fail(NM_ERR_INVALID, "W is not element aligned");

  nm_handle* h = new (std::nothrow) nm_handle();
  if (!h) return fail(NM_ERR_OOM, "host allocation failed");
  cudaGetDevice(&h->device);
  h->n_out = n_out;
  h->k = k;
  h->N = N;
  h->M = M;
  h->dt = (int)dt;
  h->tile = 1;
  h->img = nm::IMG_GATHER;
  h->kp = (k / M) * N;
  const int KBG = nm::gather_kblock_elems(h->dt);
  h->n_kb = (int)((h->kp + KBG - 1) / KBG);
  h->n_ct = (int)((n_out + nm::kRows - 1) / nm::kRows);
  h->chunk = (size_t)nm::chunk_bytes(h->dt, h->img);
  h->values_bytes = (size_t)n_out * (size_t)h->kp * es;
  h->idx_pitch = (h->kp + 1) / 2;
  h->idx_bytes = (size_t)n_out * (size_t)h->idx_pitch;
  h->bpack_bytes = (size_t)h->n_ct * h->n_kb * h->chunk;
  h->kidx_bytes = (size_t)h->n_ct * h->n_kb * KBG * sizeof(int32_t);

  cudaError_t e;
  nm_status st = NM_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if ((e = cudaMalloc(&h->d_values, h->values_bytes)) != cudaSuccess) st = cuda_fail(e, "allocate values");
  else if ((e = cudaMalloc(&h->d_idx, h->idx_bytes)) != cudaSuccess) st = cuda_fail(e, "allocate idx");
  else if ((e = cudaMalloc(&h->d_bpack, h->bpack_bytes)) != cudaSuccess) st = cuda_fail(e, "allocate packed image");
  else if ((e = cudaMalloc(&h->d_kidx, h->kidx_bytes)) != cudaSuccess) st = cuda_fail(e, "allocate kept k lists");
  else if ((e = cudaMalloc(&h->d_err, sizeof(int))) != cudaSuccess) st = cuda_fail(e, "allocate error word");
  else if ((e = cudaMemsetAsync(h->d_err, 0, sizeof(int), s)) != cudaSuccess) st = cuda_fail(e, "clear error word");
  else if ((e = cudaMemsetAsync(h->d_kidx, 0, h->kidx_bytes, s)) != cudaSuccess)  // padding slots gather row 0
    st = cuda_fail(e, "clear kept k lists");
  else if ((e = nm::launch_compress_tile(h, W_dev, s)) != cudaSuccess)
    st = cuda_fail(e, "launch compress kernels");
  else
    st = make_w_map(h);
  if (st != NM_OK) {
    const std::string msg = g_err;
    nm_destroy(h);
    g_err = msg;
    return st;
  }
  *out = h;
  return NM_OK;
}

nm_status nm_spmm_gather(const nm_handle* hc, const void* Xt, int64_t ldx, int64_t T, void* Y, const float* scale,
                         void* stream) {
  g_err.clear();
  nm_status st = check_handle(hc);
  if (st != NM_OK) return st;
  return gather_impl(hc, Xt, ldx, T, Y, scale, stream, nullptr);
}

nm_status nm_spmm_gather_ex(const nm_handle* h, const void* Xt, int64_t ldx, int64_t T, void* Y,
                            const nm_epilogue* ep, void* stream) {
  g_err.clear();
  nm_status st = check_handle(h);
  if (st != NM_OK) return st;
  if (!ep) return gather_impl(h, Xt, ldx, T, Y, nullptr, stream, nullptr);
  bool fixed = false;
  EpiReq r;
  if ((st = resolve_epilogue(h, ep, &fixed, &r)) != NM_OK) return st;
  return gather_impl(h, Xt, ldx, T, Y, ep->scale, stream, fixed ? nullptr : &r);
}

}  // extern "C"

namespace {

nm_status gather_impl(const nm_handle* hc, const void* Xt, int64_t ldx, int64_t T, void* Y, const float* scale,
                      void* stream, const EpiReq* ep) {
  nm_status st = NM_OK;
  if (!hc->tile) return fail(NM_ERR_INVALID, "nm_spmm_gather needs a handle made by nm_compress_tile");
  nm_handle* h = const_cast<nm_handle*>(hc);  // only caches (tensor map, workspace) change
  if (T < 0) return fail(NM_ERR_INVALID, "T must be >= 0 (got %lld)", (long long)T);
  if (T == 0) return NM_OK;
  if (!Xt || !Y) return fail(NM_ERR_INVALID, "null Xt or Y");
  if (T > INT32_MAX) return fail(NM_ERR_UNSUPPORTED, "T above 2^31-1");
  const int es = nm::elem_bytes(h->dt);
  if (ldx < T) return fail(NM_ERR_INVALID, "ldx=%lld is below T=%lld", (long long)ldx, (long long)T);
  if ((ldx * es) % 16 != 0)
    return fail(NM_ERR_INVALID, "ldx * sizeof(dtype) must be a multiple of 16 bytes (ldx=%lld)", (long long)ldx);
  if (!aligned(Xt, 16) || !aligned(Y, 16)) return fail(NM_ERR_INVALID, "Xt and Y must be 16-byte aligned");
  if (scale && !aligned(scale, 4)) return fail(NM_ERR_INVALID, "scale must be 4-byte aligned");
  const size_t ybytes = (size_t)T * h->n_out * out_elem_bytes(h, ep);
  const size_t xbytes = ((size_t)(h->k - 1) * ldx + T) * es;
  const uintptr_t xs = (uintptr_t)Xt, ys = (uintptr_t)Y;
  if (xs < ys + ybytes && ys < xs + xbytes) return fail(NM_ERR_INVALID, "Y overlaps Xt");

  const nm::Plan p = make_plan(h, T, num_sms(h->device), scale != nullptr);
  st = make_xt_map(h, Xt, ldx, T);
  if (st != NM_OK) return st;
  nm::SpmmArgs a{};
  a.bpack = h->d_bpack;
  a.Y = Y;
  a.scale = scale;
  a.err = h->d_err;
  a.T = (int)T;
  a.n_out = (int)h->n_out;
  a.n_kb = h->n_kb;
  a.n_ct = h->n_ct;
  a.n_tt = p.n_tt;
  a.splits = p.splits;
  a.kb_per_split = p.kb_per_split;
  a.units = p.units;
  a.timeout_ns = 1000000000ull;
  a.inject_skip = -1;
  a.w_tma = (h->has_tmw && env_int("NMSPMM_W_BULK", 0) == 0) ? 1 : 0;
  a.tma_store = 0;
  a.kidx = h->d_kidx;
  a.xt = Xt;
  a.ldx = (long long)ldx;
  // Gather warps (load/store path) by default: measured faster on B200 than
  // four-row tensor gathers, whose per-copy cost caps them near 1.3 TB/s.
  a.gather_tma = env_int("NMSPMM_GATHER_TMA", 0) ? 1 : 0;
  a.out_ty = ep ? ep->out_ty : -1;
  a.bias = ep ? ep->bias : nullptr;
  a.act = ep ? ep->act : nm::ACT_NONE;
  a.out_scale = ep ? ep->out_scale : 1.0f;
  if (p.splits > 1 && (st = split_workspace(h, p, nullptr, (cudaStream_t)stream, &a)) != NM_OK) return st;
  cudaError_t e = nm::launch_spmm(h, &h->tm, &h->tmy, p, a, (cudaStream_t)stream);
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "launch SpMM kernel");
}

}  // namespace

extern "C" {

nm_status nm_decompress(const nm_handle* h, void* W_dev_out, void* stream) {
  g_err.clear();
  nm_status st = check_handle(h);
  if (st != NM_OK) return st;
  if (!W_dev_out) return fail(NM_ERR_INVALID, "null output");
  if (!aligned(W_dev_out, 16)) return fail(NM_ERR_INVALID, "output must be 16-byte aligned");
  cudaError_t e = nm::launch_decompress(h, W_dev_out, (cudaStream_t)stream);
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "launch decompress kernel");
}

nm_status nm_export_sizes(const nm_handle* h, size_t* values_bytes, size_t* idx_bytes) {
  g_err.clear();
  if (!h) return fail(NM_ERR_INVALID, "null handle");
  if (values_bytes) *values_bytes = h->values_bytes;
  if (idx_bytes) *idx_bytes = h->idx_bytes;
  return NM_OK;
}

nm_status nm_export(const nm_handle* h, void* values_host, uint8_t* idx_host) {
  g_err.clear();
  nm_status st = check_handle(h);
  if (st != NM_OK) return st;
  if (!values_host || !idx_host) return fail(NM_ERR_INVALID, "null host buffer");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "synchronise before export");
  if ((e = cudaMemcpy(values_host, h->d_values, h->values_bytes, cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "copy values");
  if ((e = cudaMemcpy(idx_host, h->d_idx, h->idx_bytes, cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "copy idx");
  return NM_OK;
}

nm_status nm_plan_query(const nm_handle* h, int64_t T, int scaled, nm_plan_info* out) {
  g_err.clear();
  nm_status st = check_handle(h);
  if (st != NM_OK) return st;
  if (!out) return fail(NM_ERR_INVALID, "null output");
  if (T <= 0 || T > INT32_MAX) return fail(NM_ERR_INVALID, "T must be in [1, 2^31-1] (got %lld)", (long long)T);
  const nm::Plan p = make_plan(h, T, num_sms(h->device), scaled != 0);
  out->pair = p.pair;
  out->bn = p.bn;
  out->splits = p.splits;
  out->cluster = p.cluster;
  out->grid = p.grid;
  out->units = p.units;
  return NM_OK;
}

nm_status nm_plan_for_shape(nm_dtype dt, int64_t n_out, int64_t k, int N, int M, int64_t T, int sms,
                            const int* pair_clusters, const int* stream_clusters, nm_plan_info* out) {
  g_err.clear();
  if (!pair_clusters || !stream_clusters || !out) return fail(NM_ERR_INVALID, "null argument");
  if (dt != NM_INT8 && dt != NM_FP16 && dt != NM_BF16) return fail(NM_ERR_INVALID, "unknown dtype %d", (int)dt);
  if (n_out <= 0 || k <= 0 || n_out > INT32_MAX || k > INT32_MAX) return fail(NM_ERR_INVALID, "bad shape");
  const bool sp24 = (N == 1 && M == 4) || (N == 2 && M == 4) || (N == 2 && M == 8);
  const bool dense = (N == 4 && M == 8) || (N == M && (M == 4 || M == 8));
  if (!sp24 && !dense) return fail(NM_ERR_UNSUPPORTED, "N:M %d:%d is not supported", N, M);
  if (k % M != 0) return fail(NM_ERR_INVALID, "k=%lld is not a multiple of M=%d", (long long)k, M);
  if (T <= 0 || T > INT32_MAX) return fail(NM_ERR_INVALID, "T must be in [1, 2^31-1] (got %lld)", (long long)T);
  if (sms <= 0) return fail(NM_ERR_INVALID, "sms must be positive");
  nm_handle h;  // the shape fields nm_compress derives; no device memory
  h.n_out = n_out;
  h.k = k;
  h.N = N;
  h.M = M;
  h.dt = (int)dt;
  h.img = sp24 ? nm::IMG_SP24 : nm::IMG_DENSE;
  h.n_kb = (int)((k + nm::kblock_elems(h.dt) - 1) / nm::kblock_elems(h.dt));
  h.n_ct = (int)((n_out + nm::kRows - 1) / nm::kRows);
  Capacity c;
  for (int i = 0; i < 3; ++i) c.pair[i] = pair_clusters[i];
  for (int S = 1; S <= nm::kMaxClusterSplit; ++S) c.stream[S] = stream_clusters[S - 1];
  const nm::Plan p = plan_with(&h, T, sms, c);
  out->pair = p.pair;
  out->bn = p.bn;
  out->splits = p.splits;
  out->cluster = p.cluster;
  out->grid = p.grid;
  out->units = p.units;
  return NM_OK;
}

nm_status nm_query(const nm_handle* h, int64_t* n_out, int64_t* k, int* N, int* M, nm_dtype* dt) {
  g_err.clear();
  if (!h) return fail(NM_ERR_INVALID, "null handle");
  if (n_out) *n_out = h->n_out;
  if (k) *k = h->k;
  if (N) *N = h->N;
  if (M) *M = h->M;
  if (dt) *dt = (nm_dtype)h->dt;
  return NM_OK;
}

nm_status nm_device_status(const nm_handle* h) {
  g_err.clear();
  nm_status st = check_handle(h);
  if (st != NM_OK) return st;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "synchronise");
  int word = 0;
  if ((e = cudaMemcpy(&word, h->d_err, sizeof word, cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "read error word");
  if (word == 0) return NM_OK;
  cudaMemset(h->d_err, 0, sizeof(int));
  static const char* where[] = {"", "producer waiting for a free stage", "MMA waiting for a free accumulator",
                                "MMA waiting for operands", "epilogue waiting for an accumulator"};
  return fail(NM_ERR_TIMEOUT, "a kernel gave up a bounded wait (%s)", (word >= 1 && word <= 4) ? where[word] : "?");
}

nm_status nm_spmm_noalloc(const nm_handle* h, const void* X, int64_t T, void* Y, const float* scale,
                          void* stream) {
  g_err.clear();
  nm_status st = check_handle(h);
  if (st != NM_OK) return st;
  void* scratch = nullptr;
  st = noalloc_scratch(h->device, &scratch);  // first call on this device: address lookup
  if (st != NM_OK) return st;
  SplitScratch ext;
  ext.ws = scratch;
  ext.ws_bytes = kNoAllocPartialBytes;
  ext.cnt = reinterpret_cast<int*>(static_cast<unsigned char*>(scratch) + kNoAllocPartialBytes);
  ext.cnt_len = kNoAllocCounters;
  return spmm_impl(h, X, T, Y, scale, stream, -1, 1000000000ull, nullptr, &ext);
}

void nm_destroy(nm_handle* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  cudaFree(h->d_values);
  cudaFree(h->d_idx);
  cudaFree(h->d_bpack);
  cudaFree(h->d_kidx);
  cudaFree(h->d_err);
  cudaFree(h->d_ws);
  cudaFree(h->d_cnt);
  delete h;
}

}  // extern "C"
