// nm_internal.h -- declarations shared by the host-side translation units of
// libnmspmm (not part of the public ABI; see include/nmspmm.h for that).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

struct nm_handle {
  int64_t n_out = 0, k = 0;
  int N = 0, M = 0;
  int dt = 0;            // nm::DT_*
  int img = 0;           // nm::IMG_*
  int n_kb = 0;          // k-blocks in the packed image
  int n_ct = 0;          // 128-row channel tiles
  size_t chunk = 0;      // bytes per (channel tile, k-block) chunk
  int device = 0;

  void* d_values = nullptr;   // canonical values [n_out][k/M][N]
  uint8_t* d_idx = nullptr;   // canonical 4-bit positions [n_out][idx_pitch]
  size_t values_bytes = 0, idx_bytes = 0;
  int64_t idx_pitch = 0;
  uint8_t* d_bpack = nullptr; // packed operand image
  size_t bpack_bytes = 0;
  // one pattern per 128-row tile (nm_compress_tile): the image covers the kept
  // k only (kp per row) and d_kidx lists, per tile, the kept k of every
  // k-block slot (n_kb * gather_kblock_elems entries, padded with 0)
  int tile = 0;
  int64_t kp = 0;
  int32_t* d_kidx = nullptr;
  size_t kidx_bytes = 0;
  int* d_err = nullptr;       // device error word (bounded-wait timeouts)

  // split-K workspace (partials + per-tile arrival counters), grown on demand
  void* d_ws = nullptr;
  size_t ws_bytes = 0;
  int* d_cnt = nullptr;
  int cnt_len = 0;

  // cached tensor map of the last activation seen
  const void* tm_x = nullptr;
  int64_t tm_T = -1;
  int64_t tm_ld = -1;     // row pitch (elements) of a feature-major activation map
  int tm_bn = 0;
  alignas(64) CUtensorMap tm;
  // the packed image as a 2-D tensor of 128-byte rows (one box = one chunk)
  int has_tmw = 0;
  alignas(64) CUtensorMap tmw;
  // cached tensor map of the last output seen
  const void* tmy_y = nullptr;
  int64_t tmy_T = -1;
  int tmy_out = -1;
  alignas(64) CUtensorMap tmy;
};

namespace nm {

// Launch plan chosen per problem (inference-aware adaptive parallelism).
struct Plan {
  int bn = 128;       // token tile (MMA N)
  int splits = 1;     // split-K factor
  int kb_per_split = 1;
  int n_tt = 1;       // token tiles
  int units = 1;      // (tile, split) work units
  int grid = 1;       // persistent CTAs
  int xkb = 0;        // > 0: X-stationary mode holding this many k-blocks of X resident
  int pair = 0;       // 1: CTA-pair kernel (M = 256 per MMA); grid counts pairs
  int cluster = 0;    // 1: the splits of a tile are the CTAs of one cluster (grid = units, one unit
                      //    per CTA) and their partials are summed through distributed shared memory
};

// Epilogue warps per TMEM lane quarter (each owns BN / epw token columns of a
// tile): 2 for the fixed output stages, 4 for the runtime output stage, whose
// longer per-element work needs more warps to hide its latencies.  The fixed
// stages keep the smaller CTA so that other kernels (weight re-packs) can share
// the SM.
constexpr int epw_for(bool runtime_stage) { return runtime_stage ? 4 : 2; }

// Largest number of INT8 k-blocks (256 dense k each) the X-stationary mode keeps resident.
constexpr int kXsMaxKb = 3;

struct SpmmArgs {
  const uint8_t* bpack;
  void* Y;
  const float* scale;
  void* ws;
  int* cnt;
  int* err;
  int T, n_out, n_kb, n_ct, n_tt, splits, kb_per_split, units;
  unsigned long long timeout_ns;
  int tma_store;      // 1: epilogue writes Y with TMA tensor stores (tmY valid)
  int w_tma;          // 1: packed chunks arrive by 2-D tensor copy (tmW valid), else one bulk copy
  int inject_skip;    // test hook: producer omits the stage with this index (-1: never)
  // Fused output stage chosen at run time (kernels built with the runtime output
  // stage only): element type OUT_F32/F16/BF16/I8, per-channel bias (or null),
  // activation ACT_*, and the multiplier applied before int8 rounding.
  int out_ty = -1;
  const float* bias = nullptr;
  int act = 0;
  float out_scale = 1.0f;
  // Gather image only: per channel tile, n_kb * gather_kblock_elems kept k
  // (the activation rows each k-block gathers).
  const int32_t* kidx = nullptr;
  // Gather image: the feature-major activation Xt [k][ldx] read by the gather
  // warps (load/store path), and gather_tma = 1 to gather with four-row tensor
  // copies from the producer warp instead.
  const void* xt = nullptr;
  long long ldx = 0;
  int gather_tma = 0;
  long long* trace;   // timeline buffer, only written by builds compiled with NM_TRACE
  // Split-K reduced on chip (streaming kernel, splits > 1): the `splits` CTAs of
  // a cluster are the splits of one tile, one unit per CTA; ws and cnt unused.
  int csplit = 0;
  // Before waiting for the previous kernel of the stream, hint into L2 the
  // first unit's weight chunks (1) and also its activation boxes (2); 0: none.
  int prefetch = 0;
};

// Timeline trace layout (builds with NM_TRACE): per CTA kTraceStride int64
// slots: [kind][index], kinds below, kTraceMax indices each.
constexpr int kTraceMax = 64;
// TR_GT holds %globaltimer (ns, comparable across SMs) at kernel entry (0),
// after the wait on the previous kernel (1), after the producer's loop (2) and
// at exit (3), written by thread 0, and the SM clock at the same points (4..7).
enum : int { TR_P_ISSUE = 0, TR_M_FULL, TR_M_DONE, TR_M_ACCE, TR_E_START, TR_E_END, TR_GT, TR_KINDS };
constexpr int kTraceStride = TR_KINDS * kTraceMax;

cudaError_t launch_compress(const nm_handle* h, const void* W, cudaStream_t s);
cudaError_t launch_decompress(const nm_handle* h, void* Wout, cudaStream_t s);
// Tile-shared compress (nm_compress_tile): selects each tile's kept k, then packs.
cudaError_t launch_compress_tile(const nm_handle* h, const void* W, cudaStream_t s);
// Resident CTA pairs for the pair kernel of this (dtype, image, token tile, output) or <= 0.
int pair_max_clusters(int dt, int img, int bn, int out);
// Clusters of `size` one-SM streaming CTAs that can be resident at once (<= 0: none).
int stream_max_clusters(int size);
// Largest cluster the on-chip split-K uses (portable cluster size).
constexpr int kMaxClusterSplit = 8;
cudaError_t launch_spmm(const nm_handle* h, const CUtensorMap* tmX, const CUtensorMap* tmY, const Plan& p,
                        const SpmmArgs& a, cudaStream_t s);

}  // namespace nm
