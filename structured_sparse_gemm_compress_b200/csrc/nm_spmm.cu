// nm_spmm.cu -- the micro-dense N:M SpMM kernel for sm_100a.
//
// Implements the execution side of "Realizable N:M Sparse Transformer Inference
// via Search-Kernel Co-Design":
//   * section 4.2, micro-dense execution: only the kept values of every window
//     reach the tensor core, as regular dense operand tiles; the positions ride
//     along in the same packed chunk and feed the sparse MMA's metadata, so
//     the runtime compute is MMA only;
//   * section 4.1, mechanism (3), adaptive parallelism: the host picks the
//     token tile and a split-K factor per shape (nm_api.cu); split partials are
//     reduced by the last-arriving CTA of a tile, so no CTA ever waits on
//     another.
//
// Y^T tile [128 channels x BN tokens] = sum over k-blocks of
//     MMA( W_tile [128 x k-block] (sparse 2:4 image or dense),
//          X_tile [BN x k-block] (K-major) )
// accumulated in tensor memory, so TMEM lane = output channel and TMEM column
// = token; the epilogue therefore stores 32 consecutive channels of one token
// per warp instruction (128 B, coalesced) without a transpose.
//
// CTA = 2 + 4 * epw warps, one persistent CTA per SM:
//   warp 0      producer: one bulk copy of the packed weight chunk (values +
//               positions) and two 2-D tensor copies of X per stage;
//   warp 1      TMEM owner and MMA issuer (one elected lane): copies the positions
//               into TMEM (tcgen05.cp) and issues tcgen05.mma(.sp);
//   warps 2..   epilogue, epw warps per TMEM lane quarter (each owning BN/epw
//               token columns): tcgen05.ld, the output stage, then coalesced
//               direct stores (one 32-channel run of a token per instruction)
//               or, optionally, a staged tile written by a TMA tensor store.
// Two TMEM accumulators let the epilogue of one tile overlap the mainloop of
// the next.  Every wait is bounded; on a timeout the kernel records an error
// word, drains its own copies and MMAs, frees TMEM and returns.
#include "nm_device.cuh"
#include "nm_internal.h"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <type_traits>

namespace nm {


constexpr int kSmemBudget = 227 * 1024 - 1024;  // dynamic shared memory after 1 KB alignment slack

// OUT template parameter: bits 0-1 = output element (OUT_*), bit 2 = direct-store
// epilogue (no shared-memory staging, which leaves room for more pipeline stages),
// bit 3 = runtime output stage (scale, bias, activation and element type read from
// SpmmArgs; always with direct stores).
constexpr int kOutDirect = 4;
constexpr int kOutEpi = 8;
constexpr int out_bytes(int out) { return ((out & 3) == OUT_I32 || (out & 3) == OUT_F32) ? 4 : 2; }
// Epilogue warps and CTA size of a kernel with output code OUT.
constexpr int epi_warps(int out) { return 4 * epw_for((out & kOutEpi) != 0); }
constexpr int cta_threads(int out) { return 64 + 32 * epi_warps(out); }
// Gather image: warps that gather the kept activation rows (after the epilogue
// warps): 8, or 4 beside the runtime output stage's 16 epilogue warps (which
// keeps every thread within 88 registers).
__host__ __device__ constexpr int gather_warps(int out) { return (out & kOutEpi) ? 4 : 8; }
constexpr int kernel_threads(int img, int out) {
  return cta_threads(out) + (img == IMG_GATHER ? 32 * gather_warps(out) : 0);
}

// Kernel configuration.  XKB = 0: streaming mode, every stage carries a packed
// weight chunk and the matching X boxes.  XKB > 0: X-stationary mode, the
// whole X tile of a token tile (up to XKB k-blocks) stays resident in shared
// memory while the CTA walks the channel tiles of its range; stages carry only
// packed weight chunks, so X is read from L2 once per token tile instead of
// once per 128-channel tile.
//
// IMG_GATHER (one pattern per channel tile): the stage's A is one 128-byte atom
// of kept values (KB = 128 / sizeof(elem) kept k), and B is gathered from the
// feature-major activation Xt [k][T]: the KB kept rows of the tile, BN tokens
// each, land MN-major (token-contiguous 128-byte runs, 128-byte swizzle) in NB
// runs of BN tokens, run j holding tokens [j*128/es, (j+1)*128/es).
template <int DT, int IMG, int BN, int OUT, int XKB>
struct Cfg {
  static constexpr bool SP = IMG == IMG_SP24;
  static constexpr bool GA = IMG == IMG_GATHER;
  static constexpr bool XS = XKB > 0;
  static constexpr int KB = GA ? gather_kblock_elems(DT) : kblock_elems(DT);
  static constexpr int CHUNK = chunk_bytes(DT, IMG);
  static constexpr int NB = GA ? BN * elem_bytes(DT) / 128 : 0;  // gather: 128-byte token runs per row
  static constexpr int B_BOX = GA ? KB * 128 : BN * 128;  // one 128-byte-wide box of X (gather: all KB rows of one run)
  static constexpr int B_KBLK = GA ? NB * B_BOX : 2 * B_BOX;  // X bytes of one k-block
  static constexpr int STAGE = XS ? CHUNK : CHUNK + B_KBLK;  // multiple of 1024
  static constexpr int X_BYTES = XKB * B_KBLK;      // resident X region (X-stationary mode)
  static constexpr int MMAS = (SP || GA) ? 4 : 8;   // MMAs per stage (each 32 B of A per row)
  static_assert(!GA || (!XS && NB >= 1 && BN * elem_bytes(DT) % 128 == 0), "gather tiles are whole 128-byte runs");
  static constexpr int E_COLS = SP ? (DT == DT_I8 ? 8 : 4) : 0;
  static constexpr int E_COL0 = 2 * BN;             // metadata slots after the two accumulators
  static constexpr int COLS_NEEDED = 2 * BN + 2 * E_COLS;
  static constexpr int TMEM_COLS = COLS_NEEDED <= 32 ? 32 : COLS_NEEDED <= 64 ? 64 : COLS_NEEDED <= 128 ? 128
                                   : COLS_NEEDED <= 256 ? 256 : 512;
  // epilogue: each warp owns BN/epw token columns of its lane quarter, in chunks of CH
  static constexpr int EPI_WARPS = epi_warps(OUT);
  static constexpr int THREADS = kernel_threads(IMG, OUT);
  static constexpr int WCOLS = BN / (EPI_WARPS / 4);
  // chunks of 32 columns, or one chunk of the whole run when it is not a multiple of 32
  static constexpr int CH = (WCOLS % 32 == 0) ? 32 : (WCOLS % 8 == 0 && WCOLS <= 96) ? WCOLS : 8;
  static constexpr int NCH = WCOLS / CH;
  static constexpr int OES = out_bytes(OUT);
  static constexpr int EPI_BUF = CH * 32 * OES;     // one staged [CH tokens][32 channels] tile
  static constexpr int AVAIL = kSmemBudget - X_BYTES;
  // two staging buffers per warp unless that would leave fewer stages than wanted
  static constexpr int WANT = XS ? 4 : 3;
  static constexpr bool TS = (OUT & kOutDirect) == 0;   // TMA-store epilogue with staging
  static constexpr int EPI_NB = (AVAIL - 2 * EPI_WARPS * EPI_BUF) / STAGE >= WANT ? 2 : 1;
  static constexpr int EPI_BYTES = TS ? EPI_NB * EPI_WARPS * EPI_BUF : 0;
  static constexpr int STAGES_FIT = (AVAIL - EPI_BYTES) / STAGE;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int SMEM = STAGES * STAGE + X_BYTES + EPI_BYTES + 1024;
  static_assert(STAGE % 1024 == 0 && B_KBLK % 1024 == 0, "stages keep 1024-byte alignment");
  static_assert(STAGES >= 2, "need at least two stages");
  static_assert(COLS_NEEDED <= 512, "tensor memory overflow");
  static_assert(WCOLS % CH == 0 && CH % 8 == 0, "epilogue chunking");
};

// Instruction descriptor: A K-major (sparse or dense), B K-major (MN-major
// when B_MN), M = 128.
template <int DT, bool SP, int BN, int M_MMA = 128, bool B_MN = false>
__host__ __device__ constexpr uint32_t make_idesc() {
  uint32_t d = 0;
  if (SP) d |= 1u << 2;                    // sparse A
  if (B_MN) d |= 1u << 16;                 // B MN-major (token-contiguous)
  if (DT == DT_I8) {
    d |= 2u << 4;                          // D: s32
    d |= 1u << 7;                          // A: signed 8-bit
    d |= 1u << 10;                         // B: signed 8-bit
  } else {
    d |= 1u << 4;                          // D: f32
    const uint32_t f = DT == DT_BF16 ? 1u : 0u;
    d |= f << 7;                           // A: f16 / bf16
    d |= f << 10;                          // B
  }
  d |= (uint32_t)(BN >> 3) << 17;          // N
  d |= (uint32_t)(M_MMA >> 4) << 24;       // M
  return d;
}

// Optional timeline trace (compiled in only with NM_TRACE): SM clock-cycle
// stamps of pipeline events, per CTA (all roles of a CTA share one SM clock).
#ifdef NM_TRACE
#define NM_TR(kind, idx)                                                                   \
  do {                                                                                     \
    if (a.trace && (idx) < kTraceMax)                                                      \
      a.trace[(size_t)blockIdx.x * kTraceStride + (kind) * kTraceMax + (idx)] =            \
          (long long)clock64();                                                            \
  } while (0)
#define NM_TG(idx)                                                                                   \
  do {                                                                                               \
    if (a.trace && threadIdx.x == 0) {                                                               \
      long long* g_ = a.trace + (size_t)blockIdx.x * kTraceStride + TR_GT * kTraceMax;               \
      g_[(idx)] = (long long)globaltimer();                                                          \
      g_[4 + (idx)] = (long long)clock64();                                                          \
    }                                                                                                \
  } while (0)
#else
#define NM_TR(kind, idx) \
  do {                   \
  } while (0)
#define NM_TG(idx) \
  do {             \
  } while (0)
#endif

struct Unit {
  int ct, tt, z, tile, kb0, kb1;
};
__device__ __forceinline__ Unit decode_unit(int u, const SpmmArgs& a) {
  Unit w;
  w.tile = u / a.splits;
  w.z = u - w.tile * a.splits;
  w.ct = w.tile % a.n_ct;
  w.tt = w.tile / a.n_ct;
  w.kb0 = w.z * a.kb_per_split;
  w.kb1 = min(a.n_kb, w.kb0 + a.kb_per_split);
  return w;
}

// clamp(round-half-even(x), -128, 127) in one conversion instruction (NaN -> 0).
__device__ __forceinline__ int32_t rne_sat_s8(float x) {
  int32_t q;
  asm("cvt.rni.sat.s8.f32 %0, %1;" : "=r"(q) : "f"(x));
  return q;
}

// Output element from the 32-bit accumulator: int32; (float)acc * scale; or
// fp16/bf16 rounded once from the fp32 accumulator (times scale when given).
template <int OUT>
__device__ __forceinline__ auto convert_out(uint32_t acc, float s, bool has_scale) {
  if constexpr (OUT == OUT_I32) {
    return (int32_t)acc;
  } else if constexpr (OUT == OUT_F32) {
    return __fmul_rn(__int2float_rn((int32_t)acc), s);
  } else {
    float f = __uint_as_float(acc);
    if (has_scale) f = __fmul_rn(f, s);
    if constexpr (OUT == OUT_F16)
      return __float2half_rn(f);
    else
      return __float2bfloat16_rn(f);
  }
}

// The units a CTA processes.  Streaming mode: u = blockIdx.x, +gridDim.x, ...
// X-stationary mode: one contiguous range of tiles in (token tile, channel
// tile) order, so consecutive tiles share their X tile.
struct UnitRange {
  int first, end, step;
};
template <bool XS>
__device__ __forceinline__ UnitRange my_units(const SpmmArgs& a) {
  UnitRange r;
  if constexpr (XS) {
    r.first = (int)(((long long)a.units * blockIdx.x) / gridDim.x);
    r.end = (int)(((long long)a.units * (blockIdx.x + 1)) / gridDim.x);
    r.step = 1;
  } else {
    r.first = blockIdx.x;
    r.end = a.units;
    r.step = gridDim.x;
  }
  return r;
}

template <int OUT>
__device__ __forceinline__ void store_out(void* Y, size_t i, uint32_t acc, float s, bool has_scale) {
  if constexpr (OUT == OUT_I32) {
    reinterpret_cast<int32_t*>(Y)[i] = (int32_t)acc;
  } else if constexpr (OUT == OUT_F32) {
    reinterpret_cast<float*>(Y)[i] = __fmul_rn(__int2float_rn((int32_t)acc), s);
  } else {
    float f = __uint_as_float(acc);
    if (has_scale) f = __fmul_rn(f, s);
    if constexpr (OUT == OUT_F16)
      reinterpret_cast<__half*>(Y)[i] = __float2half_rn(f);
    else
      reinterpret_cast<__nv_bfloat16*>(Y)[i] = __float2bfloat16_rn(f);
  }
}

// ---- runtime output stage (OUT has kOutEpi)
//
// y = act(acc * scale[n] + bias[n]) in fp32, one rounding per step (scale and
// bias only when given), then stored as fp32, fp16 or bf16 (round to nearest
// even) or int8 (round half to even of y * out_scale, saturated to [-128, 127]).
// The GELU is the erf form x/2 (1 + erf(x / sqrt 2)), with erf evaluated by
// Abramowitz and Stegun's formula 7.1.26 (Handbook of Mathematical Functions,
// after Hastings): for u >= 0,
//   erfc(u) = (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-u^2) + e(u),
//   t = 1 / (1 + p u),  |e(u)| <= 1.5e-7,
// so that, with q = erfc(|x| / sqrt 2) / 2, GELU(x) = x (1 - q) for x >= 0 and
// x q for x < 0.  The reciprocal and the power of two are the hardware's
// approximate instructions (about 1 and 2 ulp); the whole function stays within
// |y - GELU(x)| <= 4e-7 |x| + 2e-6 |GELU(x)| of the exact value (checked by a
// dense sweep against fp64 in the tests).  Pairs of values go through the
// packed fp32 pipe (add/mul/fma .f32x2: each half is its own fp32 operation,
// rounded to nearest even), which halves the instruction count of the
// arithmetic; a single value takes the same operations in the same order, so
// both give identical results.
struct EpiCh {  // per output channel
  float s, b;
};

namespace gelu_as {
constexpr float kP = 0.2316418883f;     // p / sqrt 2, p = 0.3275911
constexpr float kB1 = 0.127414796f;     // a_i / 2
constexpr float kB2 = -0.142248368f;
constexpr float kB3 = 0.7107068705f;
constexpr float kB4 = -0.7265760135f;
constexpr float kB5 = 0.5307027145f;
constexpr float kE = -0.7213475204f;    // -log2(e) / 2: exp(-x^2 / 2) = 2^(kE x^2)
}  // namespace gelu_as

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Two fp32 values in one 64-bit register pair, and the packed operations on them.
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ float gelu1(float x) {
  using namespace gelu_as;
  const float ax = fabsf(x);
  const float t = rcp_approx(__fmaf_rn(ax, kP, 1.0f));
  float h = __fmaf_rn(t, kB5, kB4);
  h = __fmaf_rn(t, h, kB3);
  h = __fmaf_rn(t, h, kB2);
  h = __fmaf_rn(t, h, kB1);
  h = __fmul_rn(t, h);
  const float e = ex2_approx(__fmul_rn(x, __fmul_rn(x, kE)));
  const float q = __fmul_rn(h, e);
  return __fmul_rn(x, x >= 0.0f ? __fsub_rn(1.0f, q) : q);
}

// gelu1 of both halves of a pair.
__device__ __forceinline__ void gelu2(float& x0, float& x1) {
  using namespace gelu_as;
  const uint64_t x = pk2(x0, x1);
  const uint64_t d = fma2(pk2(fabsf(x0), fabsf(x1)), pk2(kP, kP), pk2(1.0f, 1.0f));
  float d0, d1;
  upk2(d, d0, d1);
  const uint64_t t = pk2(rcp_approx(d0), rcp_approx(d1));
  uint64_t h = fma2(t, pk2(kB5, kB5), pk2(kB4, kB4));
  h = fma2(t, h, pk2(kB3, kB3));
  h = fma2(t, h, pk2(kB2, kB2));
  h = fma2(t, h, pk2(kB1, kB1));
  h = mul2(t, h);
  float w0, w1;
  upk2(mul2(x, mul2(x, pk2(kE, kE))), w0, w1);
  float q0, q1;
  upk2(mul2(h, pk2(ex2_approx(w0), ex2_approx(w1))), q0, q1);
  float r0, r1;  // 1 - q (x >= 0) or q (x < 0)
  upk2(add2(pk2(1.0f, 1.0f), pk2(-q0, -q1)), r0, r1);
  upk2(mul2(x, pk2(x0 >= 0.0f ? r0 : q0, x1 >= 0.0f ? r1 : q1)), x0, x1);
}

template <int DT>
__device__ __forceinline__ float epi_value(uint32_t acc, const EpiCh& e, const SpmmArgs& a) {
  float f = DT == DT_I8 ? __int2float_rn((int32_t)acc) : __uint_as_float(acc);
  if (a.scale) f = __fmul_rn(f, e.s);
  if (a.bias) f = __fadd_rn(f, e.b);
  if (a.act == ACT_GELU) f = gelu1(f);
  return f;
}

template <int OT>
__device__ __forceinline__ void epi_put(void* Y, size_t i, float f, float out_scale) {
  if constexpr (OT == OUT_F32) {
    reinterpret_cast<float*>(Y)[i] = f;
  } else if constexpr (OT == OUT_F16) {
    reinterpret_cast<__half*>(Y)[i] = __float2half_rn(f);
  } else if constexpr (OT == OUT_BF16) {
    reinterpret_cast<__nv_bfloat16*>(Y)[i] = __float2bfloat16_rn(f);
  } else {
    reinterpret_cast<int8_t*>(Y)[i] = (int8_t)rne_sat_s8(__fmul_rn(f, out_scale));
  }
}

// One channel's run of CH consecutive tokens (row stride n_out), the first
// nvalid of them inside the output.  Two phases, so each optional step is one
// uniform branch around one short loop (the GELU's code exists once): values
// first, then one store loop per element type, unpredicated when the whole
// run is inside the output.
template <int OT, int CH>
__device__ __forceinline__ void epi_store_t(const SpmmArgs& a, float (&f)[CH], size_t base, int nvalid) {
  if constexpr (OT == OUT_F16 || OT == OUT_BF16) {
    // one paired conversion (round to nearest even each) per two tokens
    using T2 = typename std::conditional<OT == OUT_F16, __half2, __nv_bfloat162>::type;
    using T1 = typename std::conditional<OT == OUT_F16, __half, __nv_bfloat16>::type;
    T1* y = reinterpret_cast<T1*>(a.Y) + base;
    if (nvalid >= CH) {
#pragma unroll
      for (int j = 0; j < CH; j += 2) {
        T2 p;
        if constexpr (OT == OUT_F16)
          p = __floats2half2_rn(f[j], f[j + 1]);
        else
          p = __floats2bfloat162_rn(f[j], f[j + 1]);
        y[(size_t)j * a.n_out] = p.x;
        y[(size_t)(j + 1) * a.n_out] = p.y;
      }
    } else {
#pragma unroll
      for (int j = 0; j < CH; j += 2) {
        T2 p;
        if constexpr (OT == OUT_F16)
          p = __floats2half2_rn(f[j], f[j + 1]);
        else
          p = __floats2bfloat162_rn(f[j], f[j + 1]);
        if (j < nvalid) y[(size_t)j * a.n_out] = p.x;
        if (j + 1 < nvalid) y[(size_t)(j + 1) * a.n_out] = p.y;
      }
    }
  } else if constexpr (OT == OUT_I8) {
    const uint64_t os2 = pk2(a.out_scale, a.out_scale);
#pragma unroll
    for (int j = 0; j < CH; j += 2) upk2(mul2(pk2(f[j], f[j + 1]), os2), f[j], f[j + 1]);
    int8_t* y = reinterpret_cast<int8_t*>(a.Y) + base;
    if (nvalid >= CH) {
#pragma unroll
      for (int j = 0; j < CH; ++j) y[(size_t)j * a.n_out] = (int8_t)rne_sat_s8(f[j]);
    } else {
#pragma unroll
      for (int j = 0; j < CH; ++j)
        if (j < nvalid) y[(size_t)j * a.n_out] = (int8_t)rne_sat_s8(f[j]);
    }
  } else {
    float* y = reinterpret_cast<float*>(a.Y) + base;
    if (nvalid >= CH) {
#pragma unroll
      for (int j = 0; j < CH; ++j) y[(size_t)j * a.n_out] = f[j];
    } else {
#pragma unroll
      for (int j = 0; j < CH; ++j)
        if (j < nvalid) y[(size_t)j * a.n_out] = f[j];
    }
  }
}

template <int DT, int CH>
__device__ __forceinline__ void epi_run(const SpmmArgs& a, const EpiCh& e, const uint32_t (&r)[CH], size_t base,
                                        int nvalid) {
  static_assert(CH % 2 == 0, "values go in pairs");
  float f[CH];
#pragma unroll
  for (int j = 0; j < CH; ++j) f[j] = DT == DT_I8 ? __int2float_rn((int32_t)r[j]) : __uint_as_float(r[j]);
  if (a.scale) {
    const uint64_t s2 = pk2(e.s, e.s);
#pragma unroll
    for (int j = 0; j < CH; j += 2) upk2(mul2(pk2(f[j], f[j + 1]), s2), f[j], f[j + 1]);
  }
  if (a.bias) {
    const uint64_t b2 = pk2(e.b, e.b);
#pragma unroll
    for (int j = 0; j < CH; j += 2) upk2(add2(pk2(f[j], f[j + 1]), b2), f[j], f[j + 1]);
  }
  if (a.act == ACT_GELU) {
#pragma unroll
    for (int j = 0; j < CH; j += 2) gelu2(f[j], f[j + 1]);
  }
  switch (a.out_ty) {
    case OUT_F16: epi_store_t<OUT_F16, CH>(a, f, base, nvalid); break;
    case OUT_BF16: epi_store_t<OUT_BF16, CH>(a, f, base, nvalid); break;
    case OUT_I8: epi_store_t<OUT_I8, CH>(a, f, base, nvalid); break;
    default: epi_store_t<OUT_F32, CH>(a, f, base, nvalid); break;
  }
}

// A single element (split-K reduction).
template <int DT>
__device__ __forceinline__ void epi_one(const SpmmArgs& a, const EpiCh& e, size_t i, uint32_t acc) {
  const float f = epi_value<DT>(acc, e, a);
  switch (a.out_ty) {
    case OUT_F16: epi_put<OUT_F16>(a.Y, i, f, a.out_scale); break;
    case OUT_BF16: epi_put<OUT_BF16>(a.Y, i, f, a.out_scale); break;
    case OUT_I8: epi_put<OUT_I8>(a.Y, i, f, a.out_scale); break;
    default: epi_put<OUT_F32>(a.Y, i, f, a.out_scale); break;
  }
}

// Sum of split partials (int32 for INT8, fp32 otherwise), in split order.
template <int DT>
__device__ __forceinline__ uint32_t add_acc(uint32_t x, uint32_t y) {
  if constexpr (DT == DT_I8)
    return (uint32_t)((int32_t)x + (int32_t)y);
  else
    return __float_as_uint(__uint_as_float(x) + __uint_as_float(y));
}

// N consecutive 32-bit columns of this warp's 32 lanes, N a multiple of 8:
// issued as 32-, 16- and 8-column loads with no wait in between (the caller
// waits once with tmem_wait_ld).
template <int N, int OFF = 0>
__device__ __forceinline__ void tmem_ld_run(uint32_t taddr, uint32_t* r) {
  if constexpr (N - OFF >= 32) {
    tmem_ld32(taddr + OFF, *reinterpret_cast<uint32_t(*)[32]>(r + OFF));
    tmem_ld_run<N, OFF + 32>(taddr, r);
  } else if constexpr (N - OFF >= 16) {
    tmem_ld16(taddr + OFF, *reinterpret_cast<uint32_t(*)[16]>(r + OFF));
    tmem_ld_run<N, OFF + 16>(taddr, r);
  } else if constexpr (N - OFF >= 8) {
    tmem_ld8(taddr + OFF, *reinterpret_cast<uint32_t(*)[8]>(r + OFF));
    tmem_ld_run<N, OFF + 8>(taddr, r);
  }
}

template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, uint32_t (&r)[N]) {
  static_assert(N % 8 == 0 && N <= 96, "tcgen05.ld run width");
  tmem_ld_run<N>(taddr, r);
}

__device__ __forceinline__ uint32_t out_bits(int32_t v) { return (uint32_t)v; }
__device__ __forceinline__ uint32_t out_bits(float v) { return __float_as_uint(v); }
__device__ __forceinline__ uint32_t out_bits(__half v) { return (uint32_t)__half_as_ushort(v); }
__device__ __forceinline__ uint32_t out_bits(__nv_bfloat16 v) { return (uint32_t)__bfloat16_as_ushort(v); }

// On-chip split-K reduction.  The S = a.splits CTAs of a cluster computed the
// S k-ranges of one tile and parked their partial tiles in their own shared
// memory at `xb_local` ([BN token columns][128 channels], 32-bit).  This CTA
// (cluster rank w.z) finishes the token columns j with j % S == w.z: it reads
// the S partials of a column through distributed shared memory, sums them in
// split order (so fp32 sums do not depend on timing), applies the output stage
// and stores.  Each thread owns four consecutive channels, so a warp covers the
// tile's 128 channels of one token with 16-byte reads and stores.
template <int DT, int BN, int OUT, int EPI_WARPS>
__device__ __forceinline__ void csplit_reduce(const SpmmArgs& a, const Unit& w, uint32_t xb_local, int ew,
                                              int lane) {
  constexpr bool EPI = (OUT & kOutEpi) != 0;
  const int S = a.splits;
  uint32_t src[kMaxClusterSplit];
#pragma unroll
  for (int z = 0; z < kMaxClusterSplit; ++z) src[z] = z < S ? mapa_shared(xb_local, (uint32_t)z) : 0u;
  const int chl = 4 * lane;
  const int ch = w.ct * kRows + chl;
  const bool vec = (a.n_out & 3) == 0;  // whole, aligned 4-channel groups
  const bool has_scale = a.scale != nullptr;
  float sc[4], bi[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool ok = ch + i < a.n_out;
    sc[i] = (has_scale && ok) ? __ldg(a.scale + ch + i) : 1.0f;
    bi[i] = (EPI && a.bias && ok) ? __ldg(a.bias + ch + i) : 0.0f;
  }
  if (ch >= a.n_out) return;
#pragma unroll 1
  for (int j = w.z + S * ew; j < BN; j += S * EPI_WARPS) {
    const int t = w.tt * BN + j;
    if (t >= a.T) break;  // columns ascend: the rest are beyond T too
    const uint32_t off = (uint32_t)(j * kRows + chl) * 4u;
    uint4 v[kMaxClusterSplit];
#pragma unroll
    for (int z = 0; z < kMaxClusterSplit; ++z)
      if (z < S) v[z] = ld_cluster_v4(src[z] + off);
    uint32_t acc[4] = {v[0].x, v[0].y, v[0].z, v[0].w};
#pragma unroll
    for (int z = 1; z < kMaxClusterSplit; ++z) {
      if (z < S) {
        acc[0] = add_acc<DT>(acc[0], v[z].x);
        acc[1] = add_acc<DT>(acc[1], v[z].y);
        acc[2] = add_acc<DT>(acc[2], v[z].z);
        acc[3] = add_acc<DT>(acc[3], v[z].w);
      }
    }
    const size_t i0 = (size_t)t * a.n_out + ch;
    if constexpr (EPI) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (ch + i < a.n_out) epi_one<DT>(a, EpiCh{sc[i], bi[i]}, i0 + i, acc[i]);
    } else {
      using OutT = decltype(convert_out<(OUT & 3)>(0u, 1.0f, false));
      OutT o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = convert_out<(OUT & 3)>(acc[i], sc[i], has_scale);
      OutT* yp = reinterpret_cast<OutT*>(a.Y) + i0;
      if (vec) {
        if constexpr (sizeof(OutT) == 4)
          *reinterpret_cast<uint4*>(yp) = make_uint4(out_bits(o[0]), out_bits(o[1]), out_bits(o[2]), out_bits(o[3]));
        else
          *reinterpret_cast<uint2*>(yp) =
              make_uint2(out_bits(o[0]) | (out_bits(o[1]) << 16), out_bits(o[2]) | (out_bits(o[3]) << 16));
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (ch + i < a.n_out) yp[i] = o[i];
      }
    }
  }
}

template <int DT, int IMG, int BN, int OUT, int XKB>
__global__ void __launch_bounds__(kernel_threads(IMG, OUT), 1)
    spmm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                const __grid_constant__ CUtensorMap tmW, const SpmmArgs a) {
  using C = Cfg<DT, IMG, BN, OUT, XKB>;
  constexpr bool XS = C::XS;
  constexpr bool SP = C::SP;
  constexpr bool EPI = (OUT & kOutEpi) != 0;
  static_assert(!EPI || !C::TS, "the runtime output stage stores directly");
  constexpr int KIND = DT == DT_I8 ? 0 : 1;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
  __shared__ __align__(8) uint64_t accf_bar[2];
  __shared__ __align__(8) uint64_t acce_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ __align__(8) uint64_t xfull_bar;   // X-stationary: resident X tile loaded
  __shared__ __align__(8) uint64_t xempty_bar;  // X-stationary: MMAs reading it have completed
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;
  __shared__ int last_sh;
  __shared__ volatile int ep_ok_sh[2];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  NM_TG(0);

  if (threadIdx.x == 0) {
    // gather image with gather warps: the producer's arrive plus one per gather warp
    const uint32_t full_count = (C::GA && !a.gather_tma) ? 1u + gather_warps(OUT) : 1u;
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full_bar[i], full_count);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accf_bar[i], 1);
      mbar_init(&acce_bar[i], C::EPI_WARPS);
    }
    mbar_init(&drain_bar, 1);
    mbar_init(&xfull_bar, 1);
    mbar_init(&xempty_bar, 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmX);
    if (C::TS && a.tma_store) prefetch_tensormap(&tmY);
    if (a.w_tma) prefetch_tensormap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Prologue done: the next kernel may start its own; global memory is touched
  // only after the previous kernel has completed (RAW/WAW order across launches).
  pdl_launch_dependents();
  const UnitRange ur = my_units<XS>(a);
  if (a.prefetch && warp == 0 && lane == 0 && ur.first < ur.end) {
    // L2 hints for the first unit's operands while the previous kernel drains:
    // a prefetch is not a memory access in the consistency model, so it may run
    // ahead of the wait below (the copies that use the data come after it).
    const Unit w0 = decode_unit(ur.first, a);
    const int nkb = min(w0.kb1 - w0.kb0, C::STAGES);
    if (nkb > 0) {
      prefetch_l2(a.bpack + ((size_t)w0.ct * a.n_kb + w0.kb0) * C::CHUNK, (uint32_t)(nkb * C::CHUNK));
      if constexpr (!XS && !C::GA) {
        if (a.prefetch >= 2) {
          for (int kb = w0.kb0; kb < w0.kb0 + nkb; ++kb) {  // boxes that start inside k only
            prefetch_box_l2(&tmX, kb * C::KB, w0.tt * BN);
            if (kb + 1 < a.n_kb) prefetch_box_l2(&tmX, kb * C::KB + C::KB / 2, w0.tt * BN);
          }
        }
      }
    }
  }
  pdl_wait();
  NM_TG(1);
  const uint32_t tmem = tmem_base_sh;
  const uint64_t tmo = a.timeout_ns;
  uint8_t* const xregion = smem + (size_t)C::STAGES * C::STAGE;  // X-stationary mode only

  auto give_up = [&](int code) {
    abort_sh = 1;
    if (a.err) atomicExch(a.err, code);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop; one elected lane issues the copies.
    {
      const bool issuer = elect_one();
      int stage = 0, seq = 0, cur_tt = -1;
      uint32_t phase = 0, xphase = 0;
      uint32_t armed = 0, armed_par = 0;  // per stage: last use carried copies / its parity
      bool xarmed = false;
      bool ok = true;
      for (int u = ur.first; ok && u < ur.end; u += ur.step) {
        const Unit w = decode_unit(u, a);
        if (XS && w.tt != cur_tt) {
          // load the X tile of this token tile once the MMAs on the previous one have completed
          if (!mbar_wait_warp(&xempty_bar, xphase ^ 1u, &abort_sh, tmo)) {
            if (issuer) give_up(1);
            break;
          }
          if (issuer) {
            mbar_arrive_expect_tx(&xfull_bar, (uint32_t)(a.n_kb * C::B_KBLK));
            for (int kb = 0; kb < a.n_kb; ++kb) {
              uint8_t* xs = xregion + (size_t)kb * C::B_KBLK;
              tma_load_2d(xs, &tmX, &xfull_bar, kb * C::KB, w.tt * BN);
              tma_load_2d(xs + C::B_BOX, &tmX, &xfull_bar, kb * C::KB + C::KB / 2, w.tt * BN);
            }
          }
          xarmed = true;
          xphase ^= 1u;
          cur_tt = w.tt;
        }
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++seq) {
          // gather image: lanes 0 .. KB/4-1 each fetch four of the k-block's
          // kept rows (read before the wait so the load overlaps it)
          int4 grow = make_int4(0, 0, 0, 0);
          if constexpr (C::GA) {
            if (a.gather_tma && lane < C::KB / 4)
              grow = __ldg(reinterpret_cast<const int4*>(a.kidx + ((size_t)w.ct * a.n_kb + kb) * C::KB) + lane);
          }
          if (!mbar_wait_warp(&empty_bar[stage], phase ^ 1u, &abort_sh, tmo)) {
            if (issuer) give_up(1);
            ok = false;
            break;
          }
          if (issuer) NM_TR(TR_P_ISSUE, seq);
          if (seq != a.inject_skip) {
            uint8_t* st = smem + (size_t)stage * C::STAGE;
            const int wrow = (w.ct * a.n_kb + kb) * (C::CHUNK / 128);
            if (issuer) {
              // bytes the tensor copies bring (gather warps signal their part by arriving)
              const uint32_t tx = (C::GA && !a.gather_tma) ? (uint32_t)C::CHUNK : (uint32_t)C::STAGE;
              mbar_arrive_expect_tx(&full_bar[stage], tx);
              if (a.w_tma)  // the packed image as rows of 128 bytes: one box = one chunk
                tma_load_2d(st, &tmW, &full_bar[stage], 0, wrow);
              else
                bulk_load(st, a.bpack + ((size_t)w.ct * a.n_kb + kb) * C::CHUNK, (uint32_t)C::CHUNK,
                          &full_bar[stage]);
              if constexpr (!XS && !C::GA) {
                tma_load_2d(st + C::CHUNK, &tmX, &full_bar[stage], kb * C::KB, w.tt * BN);
                tma_load_2d(st + C::CHUNK + C::B_BOX, &tmX, &full_bar[stage], kb * C::KB + C::KB / 2, w.tt * BN);
              }
            }
            if constexpr (C::GA) {
              __syncwarp();  // the stage's byte count is armed before any gather lands
              if (a.gather_tma && lane < C::KB / 4) {
#pragma unroll
                for (int j = 0; j < C::NB; ++j)
                  tma_gather4(st + C::CHUNK + j * C::B_BOX + lane * 512, &tmX, &full_bar[stage],
                              w.tt * BN + j * (128 / elem_bytes(DT)), grow.x, grow.y, grow.z, grow.w);
              }
            }
            armed |= 1u << stage;
            armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          } else {
            armed &= ~(1u << stage);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: every copy this warp issued has landed before the CTA exits.
      // Earlier uses of a stage were consumed before it was re-armed, so only
      // the last armed use of each stage (and the last X tile) can still be in flight.
      for (int i = 0; i < C::STAGES; ++i)
        if ((armed >> i) & 1u) mbar_wait_warp(&full_bar[i], (armed_par >> i) & 1u, &abort_sh, tmo);
      if (xarmed) mbar_wait_warp(&xfull_bar, xphase ^ 1u, &abort_sh, tmo);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (barrier waits, descriptors); one elected
    // lane issues the tcgen05 copies, MMAs and commits.
    {
      const bool issuer = elect_one();
      constexpr uint32_t idesc = make_idesc<DT, SP, BN, 128, C::GA>();
      int stage = 0, acc = 0, eslot = 0, cur_tt = -1, mseq = 0, mtile = 0;
      uint32_t phase = 0, acc_phase = 0, xphase = 0;
      bool ok = true;
      for (int u = ur.first; ok && u < ur.end; u += ur.step) {
        const Unit w = decode_unit(u, a);
        if (XS && w.tt != cur_tt) {
          if (cur_tt >= 0 && issuer) tc_commit(&xempty_bar);  // the old X tile is free once these MMAs finish
          if (!mbar_wait_warp(&xfull_bar, xphase, &abort_sh, tmo)) {
            if (issuer) give_up(3);
            break;
          }
          xphase ^= 1u;
          cur_tt = w.tt;
        }
        if (!mbar_wait_warp(&acce_bar[acc], acc_phase ^ 1u, &abort_sh, tmo)) {
          if (issuer) give_up(2);
          break;
        }
        if (issuer) NM_TR(TR_M_ACCE, mtile);
        ++mtile;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait_warp(&full_bar[stage], phase, &abort_sh, tmo)) {
            if (issuer) give_up(3);
            ok = false;
            break;
          }
          if (issuer) NM_TR(TR_M_FULL, mseq);
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + (size_t)stage * C::STAGE);
          const uint32_t b_addr = XS ? smem_u32(xregion + (size_t)kb * C::B_KBLK) : a_addr + C::CHUNK;
          uint32_t e_tmem = 0;
          if constexpr (SP) {
            e_tmem = tmem + (uint32_t)(C::E_COL0 + eslot * C::E_COLS);
            const uint32_t e_addr = a_addr + kAtomBytes;
            if (issuer) {
              if constexpr (DT == DT_I8)
                tc_cp_128x256b(e_tmem, sdesc_rows16x2(e_addr));
              else
                tc_cp_128x128b(e_tmem, sdesc_rows16(e_addr));
            }
          }
          // descriptors differ only in the start-address field: build once, add offsets
          const uint64_t ad0 = sdesc_sw128(a_addr);
          const uint64_t bd0 = C::GA ? sdesc_sw128_mn(b_addr, (uint32_t)C::B_BOX) : sdesc_sw128(b_addr);
#pragma unroll
          for (int j = 0; j < C::MMAS; ++j) {
            const uint32_t accum = (kb > w.kb0 || j > 0) ? 1u : 0u;
            if constexpr (C::GA) {
              // MMA j: 32 bytes of each A row; the matching 32 / es kept rows of B
              const uint64_t ad = ad0 + (uint64_t)((32u * j) >> 4);
              const uint64_t bd = bd0 + (uint64_t)(((uint32_t)j * (32u / elem_bytes(DT)) * 128u) >> 4);
              if (issuer) tc_mma<KIND>(d_tmem, ad, bd, idesc, accum);
            } else if constexpr (SP) {
              const uint64_t ad = ad0 + (uint64_t)((32u * j) >> 4);
              const uint64_t bd = bd0 + (uint64_t)(((uint32_t)((j >> 1) * C::B_BOX) + 64u * (j & 1)) >> 4);
              uint32_t e_addr, id2;
              if constexpr (DT == DT_I8) {
                e_addr = e_tmem + 2u * j;
                id2 = 0;
              } else {
                e_addr = e_tmem + (uint32_t)(j & ~1);
                id2 = (uint32_t)(j & 1);
              }
              if (issuer) tc_mma_sp<KIND>(d_tmem, ad, bd, e_addr, idesc | id2, accum);
            } else {
              const uint64_t ad = ad0 + (uint64_t)(((uint32_t)((j >> 2) * kAtomBytes) + 32u * (j & 3)) >> 4);
              const uint64_t bd = bd0 + (uint64_t)(((uint32_t)((j >> 2) * C::B_BOX) + 32u * (j & 3)) >> 4);
              if (issuer) tc_mma<KIND>(d_tmem, ad, bd, idesc, accum);
            }
          }
          if (issuer) tc_commit(&empty_bar[stage]);  // frees the smem stage once these MMAs have read it
          if (issuer) NM_TR(TR_M_DONE, mseq);
          ++mseq;
          eslot ^= 1;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (issuer) tc_commit(&accf_bar[acc]);  // accumulator ready for the epilogue
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // Drain: all tcgen05 work issued by this warp completes before TMEM is freed.
      if (issuer) tc_commit(&drain_bar);
      mbar_wait_warp(&drain_bar, 0, &abort_sh, tmo);
    }
  } else if (C::GA && warp >= 2 + C::EPI_WARPS) {
    // ------------------------------------------------------------ gather warps
    // Gather image: copy the kept rows of the feature-major activation into the
    // stage's MN-major operand, 16 bytes per thread and copy (8 threads per
    // 128-byte token run, so each warp instruction reads four 128-byte rows).
    // A warp signals a stage LAG stages later, once its own copies of it have
    // landed (wait_group), after a proxy fence that makes them visible to the
    // tensor core.  Needs STAGES >= LAG + 2 (a stage is re-filled only after
    // the MMAs that read it, which need the stages signalled before it).
    if constexpr (C::GA) {
      if (!a.gather_tma) {
        constexpr int ES = elem_bytes(DT);
        constexpr int RSTEP = 32 * gather_warps(OUT) / 8;  // kept rows per pass
        constexpr int PASSES = C::KB / RSTEP;
        constexpr int TOK = 128 / ES;                 // tokens per 128-byte run
        constexpr int LAG = 2;
        static_assert(C::KB % RSTEP == 0 && C::STAGES >= LAG + 2, "gather warp schedule");
        const int gt = threadIdx.x - (64 + 32 * C::EPI_WARPS);
        const int piece = gt & 7;   // 16-byte piece of a 128-byte run
        const int rsub = gt >> 3;   // first kept row of this thread
        const uint8_t* xt = static_cast<const uint8_t*>(a.xt);
        const size_t pitch = (size_t)a.ldx * ES;
        int stage = 0, pend = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int u = ur.first; ok && u < ur.end; u += ur.step) {
          const Unit w = decode_unit(u, a);
          for (int kb = w.kb0; kb < w.kb1; ++kb) {
            // kept-row indices, loaded before the wait so their latency overlaps it
            // (not across the proxy fence below, which would wait for them)
            int rows[PASSES];
            const int32_t* kl = a.kidx + ((size_t)w.ct * a.n_kb + kb) * C::KB + rsub;
#pragma unroll
            for (int i = 0; i < PASSES; ++i) rows[i] = __ldg(kl + i * RSTEP);
            if (!mbar_wait_warp(&empty_bar[stage], phase ^ 1u, &abort_sh, tmo)) {
              if (lane == 0) give_up(1);
              ok = false;
              break;
            }
            uint8_t* bst = smem + (size_t)stage * C::STAGE + C::CHUNK;
#pragma unroll
            for (int j = 0; j < C::NB; ++j) {
              const int tok0 = w.tt * BN + j * TOK + piece * (16 / ES);
              const int rem = a.T - tok0;
              const uint32_t bytes = rem <= 0 ? 0u : rem >= 16 / ES ? 16u : (uint32_t)(rem * ES);
#pragma unroll
              for (int i = 0; i < PASSES; ++i) {
                const int row = rsub + i * RSTEP;
                const uint8_t* src = bytes ? xt + (size_t)rows[i] * pitch + (size_t)tok0 * ES : xt;
                cp_async16(bst + j * C::B_BOX + swz128((uint32_t)row, (uint32_t)piece * 16u), src, bytes);
              }
            }
            cp_async_commit();
            if (pend == LAG) {
              cp_async_wait<LAG>();  // the k-block issued LAG k-blocks ago has landed
              fence_async_smem();
              __syncwarp();
              if (lane == 0) mbar_arrive(&full_bar[(stage + C::STAGES - LAG) % C::STAGES]);
            } else {
              ++pend;
            }
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        cp_async_wait<0>();
        fence_async_smem();
        __syncwarp();
        if (lane == 0)
          for (int q = pend; q >= 1; --q) mbar_arrive(&full_bar[(stage + C::STAGES - q) % C::STAGES]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    using OutT = decltype(convert_out<(OUT & 3)>(0u, 1.0f, false));
    const int ep_tid = threadIdx.x - 64;  // 0 .. 32*EPI_WARPS-1
    const int ew = warp - 2;              // epilogue warp 0..EPI_WARPS-1
    const int lq = warp & 3;              // TMEM lane quarter this warp may access
    const int part = ew >> 2;             // which BN/epw slice of the token columns
    uint8_t* stage_buf =
        smem + (size_t)C::STAGES * C::STAGE + C::X_BYTES + (size_t)ew * C::EPI_NB * C::EPI_BUF;
    int buf = 0, acc = 0;
    uint32_t acc_phase = 0;
    // Runtime-stage kernels without split-K: each warp waits (bounded, warp
    // vote) for its tile's accumulator on its own.  Otherwise one thread waits
    // and broadcasts the outcome and every thread takes the same branch (the
    // split-K path meets at named barriers); the flag alternates between two
    // slots so a fast thread's next write cannot overtake a slow thread's read.
    int iter = 0;
    for (int u = ur.first; u < ur.end; u += ur.step, ++iter) {
      const Unit w = decode_unit(u, a);
      if (EPI && a.splits == 1) {
        // No named barrier below: each warp waits for the accumulator itself
        // (measured faster for the runtime output stage, slower for the fixed
        // fp32 stage, whose warps stay in step through the shared wait).
        if (!mbar_wait_warp(&accf_bar[acc], acc_phase, &abort_sh, tmo)) {
          if (lane == 0) give_up(4);
          break;
        }
        if (ep_tid == 0) NM_TR(TR_E_START, iter);
      } else {
        // The split-K path meets at named barriers: every warp must take the
        // same branch, so one thread decides and broadcasts.
        if (ep_tid == 0) {
          const bool got = mbar_wait(&accf_bar[acc], acc_phase, &abort_sh, tmo);
          if (!got) give_up(4);
          ep_ok_sh[iter & 1] = got ? 1 : 0;
          NM_TR(TR_E_START, iter);
        }
        named_bar_sync(1, 32 * C::EPI_WARPS);
        if (!ep_ok_sh[iter & 1]) break;
      }
      tc_fence_after();
      const int ch0 = w.ct * kRows + lq * 32;  // first channel of this warp's lane quarter
      const int ch = ch0 + lane;
      const bool ch_ok = ch < a.n_out;
      const bool has_scale = a.scale != nullptr;
      const float s = (has_scale && ch_ok) ? __ldg(a.scale + ch) : 1.0f;
      const float bch = (EPI && a.bias && ch_ok) ? __ldg(a.bias + ch) : 0.0f;
      const int col0 = part * C::WCOLS;        // first token column of this warp within the tile
      const int t0 = w.tt * BN + col0;
      const uint32_t tbase = tmem + ((uint32_t)(lq * 32) << 16) + (uint32_t)(acc * BN + col0);
      if (a.splits == 1) {
#pragma unroll 1
        for (int c = 0; c < C::NCH; ++c) {
          uint32_t r[C::CH];
          // tcgen05.ld is .sync.aligned: reconverge after the previous chunk's
          // per-lane stores (and lane 0's tensor store) before issuing it
          __syncwarp();
          tmem_ld_n<C::CH>(tbase + (uint32_t)(c * C::CH), r);
          tmem_wait_ld();
          if (c == C::NCH - 1) {  // all of this warp's columns are in registers: release the accumulator
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce_bar[acc]);
          }
          const int tc0 = t0 + c * C::CH;
          if (C::TS && a.tma_store) {
            if (lane == 0) {
              if (C::EPI_NB == 2) bulk_wait_read<1>(); else bulk_wait_read<0>();
            }
            __syncwarp();
            OutT* sb = reinterpret_cast<OutT*>(stage_buf + buf * C::EPI_BUF);
#pragma unroll
            for (int j = 0; j < C::CH; ++j) sb[j * 32 + lane] = convert_out<(OUT & 3)>(r[j], s, has_scale);
            fence_async_smem();
            __syncwarp();
            if (lane == 0 && ch0 < a.n_out && tc0 < a.T) {
              tma_store_2d(&tmY, sb, ch0, tc0);
              bulk_commit();
            }
            if (C::EPI_NB == 2) buf ^= 1;
          } else if (ch_ok) {
            if constexpr (EPI) {
              epi_run<DT, C::CH>(a, EpiCh{s, bch}, r, (size_t)tc0 * a.n_out + ch, a.T - tc0);
            } else {
              OutT* yp = reinterpret_cast<OutT*>(a.Y) + (size_t)tc0 * a.n_out + ch;
              const int nvalid = a.T - tc0;
              if (nvalid >= C::CH) {
#pragma unroll
                for (int j = 0; j < C::CH; ++j) yp[(size_t)j * a.n_out] = convert_out<(OUT & 3)>(r[j], s, has_scale);
              } else {
#pragma unroll
                for (int j = 0; j < C::CH; ++j)
                  if (j < nvalid) yp[(size_t)j * a.n_out] = convert_out<(OUT & 3)>(r[j], s, has_scale);
              }
            }
          }
        }
      } else if (a.csplit) {
        // on-chip split-K: park this split's partial tile in shared memory (the
        // pipeline stages are idle: this CTA's only unit is fully accumulated);
        // the cluster sums the partials after the role loops
        if constexpr (!XS && !C::GA) {
          uint32_t* xb = reinterpret_cast<uint32_t*>(smem);
#pragma unroll 1
          for (int c = 0; c < C::NCH; ++c) {
            uint32_t r[C::CH];
            tmem_ld_n<C::CH>(tbase + (uint32_t)(c * C::CH), r);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < C::CH; ++j) xb[(col0 + c * C::CH + j) * kRows + lq * 32 + lane] = r[j];
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acce_bar[acc]);
        }
      } else {
        // split-K: publish this split's partial tile, the last arriving split reduces
        uint32_t* part = reinterpret_cast<uint32_t*>(a.ws);
        const size_t tile_elems = (size_t)BN * kRows;
        uint32_t* mine = part + ((size_t)w.tile * a.splits + w.z) * tile_elems;
#pragma unroll 1
        for (int c = 0; c < C::NCH; ++c) {
          uint32_t r[C::CH];
          tmem_ld_n<C::CH>(tbase + (uint32_t)(c * C::CH), r);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < C::CH; ++j)
            __stcg(mine + (size_t)(col0 + c * C::CH + j) * kRows + lq * 32 + lane, r[j]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce_bar[acc]);
        __threadfence();
        named_bar_sync(1, 32 * C::EPI_WARPS);
        if (ep_tid == 0) last_sh = (atomicAdd(a.cnt + w.tile, 1) == a.splits - 1);
        named_bar_sync(1, 32 * C::EPI_WARPS);
        if (last_sh) {
          __threadfence();
          const uint32_t* tile_base = part + (size_t)w.tile * a.splits * tile_elems;
          // eight columns at a time, every split's loads in flight before any add
          constexpr int RC = C::WCOLS < 8 ? C::WCOLS : 8;
#pragma unroll 1
          for (int cb = col0; cb < col0 + C::WCOLS; cb += RC) {
            uint32_t sum[RC];
            const uint32_t* src = tile_base + (size_t)cb * kRows + lq * 32 + lane;
#pragma unroll
            for (int q = 0; q < RC; ++q) sum[q] = __ldcg(src + (size_t)q * kRows);
            for (int z = 1; z < a.splits; ++z) {
              uint32_t v[RC];
#pragma unroll
              for (int q = 0; q < RC; ++q) v[q] = __ldcg(src + z * tile_elems + (size_t)q * kRows);
#pragma unroll
              for (int q = 0; q < RC; ++q) sum[q] = add_acc<DT>(sum[q], v[q]);
            }
#pragma unroll
            for (int q = 0; q < RC; ++q) {
              const int t = w.tt * BN + cb + q;
              if (ch_ok && t < a.T) {
                if constexpr (EPI)
                  epi_one<DT>(a, EpiCh{s, bch}, (size_t)t * a.n_out + ch, sum[q]);
                else
                  store_out<(OUT & 3)>(a.Y, (size_t)t * a.n_out + ch, sum[q], s, has_scale);
              }
            }
          }
          if (ep_tid == 0) a.cnt[w.tile] = 0;  // re-arm for the next launch
        }
      }
      if (ep_tid == 0) NM_TR(TR_E_END, iter);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait<0>();  // this warp's tensor stores are complete before the CTA exits
  }

  NM_TG(2);
  if constexpr (!XS && !C::GA) {
    static_assert(C::STAGES * C::STAGE >= BN * kRows * 4, "the stages hold a parked partial tile");
    if (a.csplit) {
      // Every thread of the cluster takes both barriers, whatever its role did
      // (a bounded wait that gave up included): the first publishes the parked
      // partials, the second keeps each CTA's shared memory alive until the
      // whole cluster has read it.
      __syncwarp();
      cluster_arrive();
      cluster_wait();
      if (warp >= 2 && warp < 2 + C::EPI_WARPS)
        csplit_reduce<DT, BN, OUT, C::EPI_WARPS>(a, decode_unit(ur.first, a), smem_u32(smem), warp - 2, lane);
      __syncwarp();
      cluster_arrive();
      cluster_wait();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  NM_TG(3);
}

// ------------------------------------------------------------------ CTA-pair kernel
//
// Two CTAs on two SMs compute one 256-channel x BN-token tile with
// tcgen05.mma.cta_group::2 (M = 256: each CTA's 128 rows of the packed weight;
// N = BN: each CTA holds BN/2 token rows of X).  One thread of the pair leader
// issues every MMA for both SMs, which halves the per-SM cost of MMA issue, and
// each SM loads only half of the X tile.  Both CTAs' copies count on the
// leader's stage barrier; the leader's commits arrive on both CTAs' barriers;
// the peer's epilogue releases accumulators through its own warp 1, which
// forwards one cluster-scope arrive per release to the leader.  (A cluster-scope
// release issued by an epilogue lane would first wait for that lane's own
// output stores to become visible, holding the leader's next tile back by the
// store latency; the forwarding warp has no stores in flight.)
// No load uses cluster multicast.
template <int DT, int IMG, int BN, int OUT>
struct PairCfg {
  static constexpr bool SP = IMG == IMG_SP24;
  static constexpr int KB = kblock_elems(DT);
  static constexpr int CHUNK = chunk_bytes(DT, IMG);
  static constexpr int HB = BN / 2;                 // token rows of X held by each CTA
  static constexpr int B_BOX = HB * 128;
  static constexpr int STAGE = CHUNK + 2 * B_BOX;
  static constexpr int MMAS = SP ? 4 : 8;
  static constexpr int E_COLS = SP ? (DT == DT_I8 ? 8 : 4) : 0;
  static constexpr int E_COL0 = 2 * BN;
  static constexpr int COLS_NEEDED = 2 * BN + 2 * E_COLS;
  static constexpr int TMEM_COLS = COLS_NEEDED <= 256 ? 256 : 512;
  static constexpr int EPI_WARPS = epi_warps(OUT);
  static constexpr int THREADS = cta_threads(OUT);
  static constexpr int WCOLS = BN / (EPI_WARPS / 4);  // token columns per epilogue warp
  static constexpr bool TS = (OUT & kOutDirect) == 0;
  // Columns per tcgen05.ld run: 32, or, for the INT8 fixed output stages with
  // direct stores, half of a warp's columns when they are not a multiple of 32
  // (224-token tiles: two runs of 56 rather than seven of 16; measured 4-5 %
  // faster on the ViT-B qkv layers, and 1.5 % slower for the FP16 kernels,
  // which keep the short runs).
  static constexpr int CH = (WCOLS % 32 == 0) ? 32
                            : (DT == DT_I8 && !TS && (OUT & kOutEpi) == 0 && WCOLS <= 112 && (WCOLS / 2) % 8 == 0)
                                ? WCOLS / 2
                                : (WCOLS % 16 == 0) ? 16 : 8;
  static constexpr int NCH = WCOLS / CH;
  static constexpr int OES = out_bytes(OUT);
  static constexpr int EPI_BUF = CH * 32 * OES;
  static constexpr int EPI_NB = (kSmemBudget - 2 * EPI_WARPS * EPI_BUF) / STAGE >= 4 ? 2 : 1;
  static constexpr int EPI_BYTES = TS ? EPI_NB * EPI_WARPS * EPI_BUF : 0;
  static constexpr int STAGES_FIT = (kSmemBudget - EPI_BYTES) / STAGE;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int SMEM = STAGES * STAGE + EPI_BYTES + 1024;
  static_assert(STAGE % 1024 == 0 && B_BOX % 1024 == 0, "stages keep 1024-byte alignment");
  static_assert(STAGES >= 2, "need at least two stages");
  static_assert(COLS_NEEDED <= 512, "tensor memory overflow");
  static_assert(BN % 32 == 0 && BN <= 256, "pair MMA N");
  static_assert(WCOLS % CH == 0, "epilogue chunking");
};

template <int DT, int IMG, int BN, int OUT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(cta_threads(OUT), 1)
    spmm_pair_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                     const __grid_constant__ CUtensorMap tmW, const SpmmArgs a) {
  using C = PairCfg<DT, IMG, BN, OUT>;
  constexpr bool SP = C::SP;
  constexpr bool EPI = (OUT & kOutEpi) != 0;
  static_assert(!EPI || !C::TS, "the runtime output stage stores directly");
  constexpr int KIND = DT == DT_I8 ? 0 : 1;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
  __shared__ __align__(8) uint64_t accf_bar[2];
  __shared__ __align__(8) uint64_t acce_bar[2];
  __shared__ __align__(8) uint64_t pfree_bar[2];  // peer: its epilogue warps have read accumulator i
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  NM_TG(0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accf_bar[i], 1);
      // the leader's epilogue warps, plus one arrive forwarded by the peer for
      // all of its warps (tensor-store variant: every peer warp arrives itself)
      mbar_init(&acce_bar[i], C::TS ? 2 * C::EPI_WARPS : C::EPI_WARPS + 1);
      mbar_init(&pfree_bar[i], C::EPI_WARPS);
    }
    mbar_init(&drain_bar, 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmW);
    if (C::TS && a.tma_store) prefetch_tensormap(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_cg<2>(&tmem_base_sh, C::TMEM_COLS);
    tmem_relinquish_cg<2>();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers are initialised before any cross-CTA arrive or copy
  tc_fence_after();
  pdl_launch_dependents();
  pdl_wait();
  NM_TG(1);
  const uint32_t tmem = tmem_base_sh;
  const uint64_t tmo = a.timeout_ns;
  const uint32_t full_lead0 = mapa_shared(smem_u32(&full_bar[0]), 0);  // leader's stage barriers
  const uint32_t acce_lead0 = mapa_shared(smem_u32(&acce_bar[0]), 0);
  const int u_first = (int)cluster_id_x(), u_step = (int)nclusters_x();
  const int n_pct = (a.n_ct + 1) / 2;  // channel-tile pairs

  auto give_up = [&](int code) {
    abort_sh = 1;
    if (a.err) atomicExch(a.err, code);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    // The whole warp runs the loop; one elected lane issues the copies.
    {
      const bool issuer = elect_one();
      int stage = 0, seq = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;
      bool ok = true;
      for (int u = u_first; ok && u < a.units; u += u_step) {
        const int pt = u % n_pct, tt = u / n_pct;
        const int ct = 2 * pt + (int)rank;
        for (int kb = 0; kb < a.n_kb; ++kb, ++seq) {
          if (!mbar_wait_warp(&empty_bar[stage], phase ^ 1u, &abort_sh, tmo)) {
            if (issuer) give_up(1);
            ok = false;
            break;
          }
          if (issuer) NM_TR(TR_P_ISSUE, seq);
          if (seq != a.inject_skip) {
            uint8_t* st = smem + (size_t)stage * C::STAGE;
            const uint32_t fb = full_lead0 + 8u * (uint32_t)stage;
            const int wrow = (ct * a.n_kb + kb) * (C::CHUNK / 128);
            const int trow = tt * BN + (int)rank * C::HB;
            if (issuer) {
              if (leader) mbar_arrive_expect_tx(&full_bar[stage], (uint32_t)(2 * C::STAGE));
              tma_load_2d_pair(st, &tmW, fb, 0, wrow);
              tma_load_2d_pair(st + C::CHUNK, &tmX, fb, kb * C::KB, trow);
              tma_load_2d_pair(st + C::CHUNK + C::B_BOX, &tmX, fb, kb * C::KB + C::KB / 2, trow);
            }
            armed |= 1u << stage;
            armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          } else {
            armed &= ~(1u << stage);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: the leader's stage barriers count both CTAs' copies; the peer is
      // held by the cluster barrier below until the leader has seen them land.
      if (leader)
        for (int i = 0; i < C::STAGES; ++i)
          if ((armed >> i) & 1u) mbar_wait_warp(&full_bar[i], (armed_par >> i) & 1u, &abort_sh, tmo);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    // The leader's whole warp runs the loop; one elected lane issues.
    if (leader) {
      const bool issuer = elect_one();
      constexpr uint32_t idesc = make_idesc<DT, SP, BN, 256>();
      int stage = 0, acc = 0, eslot = 0, mseq = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int u = u_first; ok && u < a.units; u += u_step) {
        if (!mbar_wait_warp(&acce_bar[acc], acc_phase ^ 1u, &abort_sh, tmo)) {
          if (issuer) give_up(2);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        for (int kb = 0; kb < a.n_kb; ++kb) {
          if (!mbar_wait_warp(&full_bar[stage], phase, &abort_sh, tmo)) {
            if (issuer) give_up(3);
            ok = false;
            break;
          }
          if (issuer) NM_TR(TR_M_FULL, mseq);
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + (size_t)stage * C::STAGE);
          const uint32_t b_addr = a_addr + C::CHUNK;
          uint32_t e_tmem = 0;
          if constexpr (SP) {
            e_tmem = tmem + (uint32_t)(C::E_COL0 + eslot * C::E_COLS);
            const uint32_t e_addr = a_addr + kAtomBytes;
            if (issuer) {
              if constexpr (DT == DT_I8)
                tc_cp_128x256b_pair(e_tmem, sdesc_rows16x2(e_addr));
              else
                tc_cp_128x128b_pair(e_tmem, sdesc_rows16(e_addr));
            }
          }
          const uint64_t ad0 = sdesc_sw128(a_addr), bd0 = sdesc_sw128(b_addr);
#pragma unroll
          for (int j = 0; j < C::MMAS; ++j) {
            const uint32_t accum = (kb > 0 || j > 0) ? 1u : 0u;
            if constexpr (SP) {
              const uint64_t ad = ad0 + (uint64_t)((32u * j) >> 4);
              const uint64_t bd = bd0 + (uint64_t)(((uint32_t)((j >> 1) * C::B_BOX) + 64u * (j & 1)) >> 4);
              uint32_t e_addr, id2;
              if constexpr (DT == DT_I8) {
                e_addr = e_tmem + 2u * j;
                id2 = 0;
              } else {
                e_addr = e_tmem + (uint32_t)(j & ~1);
                id2 = (uint32_t)(j & 1);
              }
              if (issuer) tc_mma_sp_pair<KIND>(d_tmem, ad, bd, e_addr, idesc | id2, accum);
            } else {
              const uint64_t ad = ad0 + (uint64_t)(((uint32_t)((j >> 2) * kAtomBytes) + 32u * (j & 3)) >> 4);
              const uint64_t bd = bd0 + (uint64_t)(((uint32_t)((j >> 2) * C::B_BOX) + 32u * (j & 3)) >> 4);
              if (issuer) tc_mma_pair<KIND>(d_tmem, ad, bd, idesc, accum);
            }
          }
          if (issuer) tc_commit_pair(&empty_bar[stage], (uint16_t)3);  // frees this stage in both CTAs
          if (issuer) NM_TR(TR_M_DONE, mseq);
          ++mseq;
          eslot ^= 1;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (issuer) tc_commit_pair(&accf_bar[acc], (uint16_t)3);  // both CTAs' accumulators are ready
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (issuer) tc_commit_pair(&drain_bar, (uint16_t)3);  // every MMA of this pair has completed
      mbar_wait_warp(&drain_bar, 0, &abort_sh, tmo);
    } else {
      // Peer: forward each accumulator release of this CTA's epilogue to the
      // leader.  The epilogue warps arrive on a local barrier (no wait for
      // their own output stores to drain); this warp, with no stores of its own
      // in flight, turns each completed phase into one cluster-scope release on
      // the leader's barrier (releases are cumulative, so the epilogue's tensor
      // memory reads, fenced before its local arrives, are ordered before it).
      // The tensor-store variant's epilogue arrives on the leader itself: its
      // output leaves through asynchronous bulk copies, which a release does not
      // wait for.
      if constexpr (!C::TS) {
        const bool issuer = elect_one();
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = u_first; u < a.units; u += u_step) {
          if (!mbar_wait_warp(&pfree_bar[acc], acc_phase, &abort_sh, tmo)) {
            if (issuer) give_up(4);
            break;
          }
          if (issuer) mbar_arrive_cluster(acce_lead0 + 8u * (uint32_t)acc);
          if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1u;
          }
        }
      }
      mbar_wait_warp(&drain_bar, 0, &abort_sh, tmo);  // the leader's MMAs into this TMEM are done
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    using OutT = decltype(convert_out<(OUT & 3)>(0u, 1.0f, false));
    const int ep_tid = threadIdx.x - 64;
    const int ew = warp - 2;
    const int lq = warp & 3;
    const int part = ew >> 2;
    uint8_t* stage_buf = smem + (size_t)C::STAGES * C::STAGE + (size_t)ew * C::EPI_NB * C::EPI_BUF;
    int buf = 0, acc = 0, iter = 0;
    uint32_t acc_phase = 0;
    for (int u = u_first; u < a.units; u += u_step, ++iter) {
      const int pt = u % n_pct, tt = u / n_pct;
      const int ct = 2 * pt + (int)rank;
      // No named barrier in this loop: each warp waits for the accumulator itself.
      if (!mbar_wait_warp(&accf_bar[acc], acc_phase, &abort_sh, tmo)) {
        if (lane == 0) give_up(4);
        break;
      }
      if (ep_tid == 0) NM_TR(TR_E_START, iter);
      tc_fence_after();
      const int ch0 = ct * kRows + lq * 32;
      const int ch = ch0 + lane;
      const bool ch_ok = ch < a.n_out;
      const bool has_scale = a.scale != nullptr;
      const float s = (has_scale && ch_ok) ? __ldg(a.scale + ch) : 1.0f;
      const float bch = (EPI && a.bias && ch_ok) ? __ldg(a.bias + ch) : 0.0f;
      const int col0 = part * C::WCOLS;
      const int t0 = tt * BN + col0;
      const uint32_t tbase = tmem + ((uint32_t)(lq * 32) << 16) + (uint32_t)(acc * BN + col0);
#pragma unroll 1
      for (int c = 0; c < C::NCH; ++c) {
        uint32_t r[C::CH];
        __syncwarp();  // tcgen05.ld is .sync.aligned: reconverge after the previous chunk's stores
        tmem_ld_n<C::CH>(tbase + (uint32_t)(c * C::CH), r);
        tmem_wait_ld();
        if (c == C::NCH - 1) {  // release the accumulator (the peer's release is forwarded by its warp 1)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (leader)
              mbar_arrive(&acce_bar[acc]);
            else if constexpr (C::TS)
              mbar_arrive_cluster(acce_lead0 + 8u * (uint32_t)acc);
            else
              mbar_arrive(&pfree_bar[acc]);
          }
        }
        const int tc0 = t0 + c * C::CH;
        if (C::TS && a.tma_store) {
          if (lane == 0) {
            if (C::EPI_NB == 2) bulk_wait_read<1>(); else bulk_wait_read<0>();
          }
          __syncwarp();
          OutT* sb = reinterpret_cast<OutT*>(stage_buf + buf * C::EPI_BUF);
#pragma unroll
          for (int j = 0; j < C::CH; ++j) sb[j * 32 + lane] = convert_out<(OUT & 3)>(r[j], s, has_scale);
          fence_async_smem();
          __syncwarp();
          if (lane == 0 && ch0 < a.n_out && tc0 < a.T) {
            tma_store_2d(&tmY, sb, ch0, tc0);
            bulk_commit();
          }
          if (C::EPI_NB == 2) buf ^= 1;
        } else if (ch_ok) {
          if constexpr (EPI) {
            epi_run<DT, C::CH>(a, EpiCh{s, bch}, r, (size_t)tc0 * a.n_out + ch, a.T - tc0);
          } else {
            OutT* yp = reinterpret_cast<OutT*>(a.Y) + (size_t)tc0 * a.n_out + ch;
            const int nvalid = a.T - tc0;
            if (nvalid >= C::CH) {
#pragma unroll
              for (int j = 0; j < C::CH; ++j) yp[(size_t)j * a.n_out] = convert_out<(OUT & 3)>(r[j], s, has_scale);
            } else {
#pragma unroll
              for (int j = 0; j < C::CH; ++j)
                if (j < nvalid) yp[(size_t)j * a.n_out] = convert_out<(OUT & 3)>(r[j], s, has_scale);
            }
          }
        }
      }
      if (ep_tid == 0) NM_TR(TR_E_END, iter);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  // Teardown: every remote arrive and copy of the pair is done before either
  // CTA frees tensor memory or exits.
  NM_TG(2);
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_cg<2>(tmem, C::TMEM_COLS);
  }
  NM_TG(3);
}

// ------------------------------------------------------------------ host launch

// Launch with programmatic stream serialization, so the kernel's prologue can
// overlap the tail of the previous kernel in the stream (see pdl_wait).
// cluster > 1: launch as clusters of that many CTAs along x (grid a multiple of it).
template <typename Kern>
static cudaError_t launch_pdl(Kern kern, dim3 grid, int threads, int smem, cudaStream_t s, const CUtensorMap& tmX,
                              const CUtensorMap& tmY, const CUtensorMap& tmW, const SpmmArgs& a, int cluster = 0) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cluster > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  return cudaLaunchKernelEx(&cfg, kern, tmX, tmY, tmW, a);
}

// The dynamic shared-memory opt-in is a per-device property of a kernel: set it
// once per (kernel, device), remembered in a bit mask of device ordinals.
template <typename Kern>
static cudaError_t smem_opt_in(Kern kern, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

template <int DT, int IMG, int BN, int OUT, int XKB>
static cudaError_t launch_t(const CUtensorMap* tmX, const CUtensorMap* tmY, const CUtensorMap* tmW,
                            const Plan& p, const SpmmArgs& a, cudaStream_t s) {
  using C = Cfg<DT, IMG, BN, OUT, XKB>;
  auto kern = spmm_kernel<DT, IMG, BN, OUT, XKB>;
  static std::atomic<uint64_t> opted{0};
  cudaError_t e = smem_opt_in(kern, C::SMEM, opted);
  if (e != cudaSuccess) return e;
  if (p.cluster && (XKB > 0 || IMG == IMG_GATHER || p.splits > kMaxClusterSplit || p.grid != p.units))
    return cudaErrorInvalidValue;  // on-chip split-K: streaming kernel, one unit per CTA
  return launch_pdl(kern, dim3(p.grid), C::THREADS, C::SMEM, s, *tmX, *tmY, *tmW, a, p.cluster ? p.splits : 0);
}

template <int DT, int IMG, int BN, int OUT>
static cudaError_t launch_pair_t(const CUtensorMap* tmX, const CUtensorMap* tmY, const CUtensorMap* tmW,
                                 const Plan& p, const SpmmArgs& a, cudaStream_t s) {
  using C = PairCfg<DT, IMG, BN, OUT>;
  auto kern = spmm_pair_kernel<DT, IMG, BN, OUT>;
  static std::atomic<uint64_t> opted{0};
  cudaError_t e = smem_opt_in(kern, C::SMEM, opted);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(2 * p.grid), C::THREADS, C::SMEM, s, *tmX, *tmY, *tmW, a);  // p.grid = CTA pairs
}

int pair_max_clusters(int dt, int img, int bn, int out);

template <int DT, int IMG, int OUT>
static cudaError_t launch_bn(const CUtensorMap* tmX, const CUtensorMap* tmY, const CUtensorMap* tmW,
                             const Plan& p, const SpmmArgs& a, cudaStream_t s) {
  if (p.pair) {
    switch (p.bn) {
      case 128: return launch_pair_t<DT, IMG, 128, OUT>(tmX, tmY, tmW, p, a, s);
      case 192: return launch_pair_t<DT, IMG, 192, OUT>(tmX, tmY, tmW, p, a, s);
      case 224: return launch_pair_t<DT, IMG, 224, OUT>(tmX, tmY, tmW, p, a, s);
      default: return cudaErrorInvalidValue;
    }
  }
  if (p.xkb > 0) {  // X-stationary mode: INT8, 128-token tiles, up to kXsMaxKb k-blocks (k <= 768)
    if constexpr (DT == DT_I8) {
      if (p.bn == 128 && p.xkb <= kXsMaxKb) return launch_t<DT, IMG, 128, OUT, kXsMaxKb>(tmX, tmY, tmW, p, a, s);
    }
    return cudaErrorInvalidValue;
  }
  switch (p.bn) {
    case 32: return launch_t<DT, IMG, 32, OUT, 0>(tmX, tmY, tmW, p, a, s);
    case 64: return launch_t<DT, IMG, 64, OUT, 0>(tmX, tmY, tmW, p, a, s);
    case 128: return launch_t<DT, IMG, 128, OUT, 0>(tmX, tmY, tmW, p, a, s);
    case 192: return launch_t<DT, IMG, 192, OUT, 0>(tmX, tmY, tmW, p, a, s);
    default: return cudaErrorInvalidValue;
  }
}

// Gather image: streaming kernel only, direct-store output stages (fixed or runtime).
template <int DT, int OUT>
static cudaError_t launch_gather(const CUtensorMap* tmX, const CUtensorMap* tmY, const CUtensorMap* tmW,
                                 const Plan& p, const SpmmArgs& a, cudaStream_t s) {
  if constexpr (DT != DT_BF16 && (OUT & kOutDirect) != 0) {
    if (p.pair || p.xkb > 0) return cudaErrorInvalidValue;
    switch (p.bn) {
      case 128: return launch_t<DT, IMG_GATHER, 128, OUT, 0>(tmX, tmY, tmW, p, a, s);
      case 256: return launch_t<DT, IMG_GATHER, 256, OUT, 0>(tmX, tmY, tmW, p, a, s);
      default: return cudaErrorInvalidValue;
    }
  }
  return cudaErrorInvalidValue;
}

template <int DT, int OUT>
static cudaError_t launch_img(int img, const CUtensorMap* tmX, const CUtensorMap* tmY, const CUtensorMap* tmW,
                              const Plan& p, const SpmmArgs& a, cudaStream_t s) {
  if (img == IMG_GATHER) return launch_gather<DT, OUT>(tmX, tmY, tmW, p, a, s);
  return img == IMG_SP24 ? launch_bn<DT, IMG_SP24, OUT>(tmX, tmY, tmW, p, a, s)
                         : launch_bn<DT, IMG_DENSE, OUT>(tmX, tmY, tmW, p, a, s);
}

template <int OUT_TS>
static cudaError_t launch_dt(const nm_handle* h, const CUtensorMap* tmX, const CUtensorMap* tmY,
                             const CUtensorMap* tmW, const Plan& p, const SpmmArgs& a, cudaStream_t s) {
  constexpr int D = OUT_TS;  // 0 or kOutDirect
  if constexpr (D == kOutDirect) {
    if (a.out_ty >= 0) {  // runtime output stage
      switch (h->dt) {
        case DT_I8: return launch_img<DT_I8, kOutEpi | kOutDirect>(h->img, tmX, tmY, tmW, p, a, s);
        case DT_F16: return launch_img<DT_F16, kOutEpi | kOutDirect>(h->img, tmX, tmY, tmW, p, a, s);
        default: return launch_img<DT_BF16, kOutEpi | kOutDirect>(h->img, tmX, tmY, tmW, p, a, s);
      }
    }
  } else {
    if (a.out_ty >= 0) return cudaErrorInvalidValue;  // the runtime output stage stores directly
  }
  switch (h->dt) {
    case DT_I8:
      return a.scale ? launch_img<DT_I8, OUT_F32 | D>(h->img, tmX, tmY, tmW, p, a, s)
                     : launch_img<DT_I8, OUT_I32 | D>(h->img, tmX, tmY, tmW, p, a, s);
    case DT_F16: return launch_img<DT_F16, OUT_F16 | D>(h->img, tmX, tmY, tmW, p, a, s);
    default: return launch_img<DT_BF16, OUT_BF16 | D>(h->img, tmX, tmY, tmW, p, a, s);
  }
}

cudaError_t launch_spmm(const nm_handle* h, const CUtensorMap* tmX, const CUtensorMap* tmY, const Plan& p,
                        const SpmmArgs& a, cudaStream_t s) {
  const CUtensorMap* tmW = &h->tmw;
  return a.tma_store ? launch_dt<0>(h, tmX, tmY, tmW, p, a, s) : launch_dt<kOutDirect>(h, tmX, tmY, tmW, p, a, s);
}

// Pairs that can be resident at once for a pair-kernel configuration (cached per device).
template <int DT, int IMG, int BN, int OUT>
static int max_clusters_t() {
  static std::atomic<int> cache[64];
  static std::atomic<uint64_t> opted{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  int cached = cache[dev].load(std::memory_order_acquire);
  if (!cached) {
    using C = PairCfg<DT, IMG, BN, OUT>;
    auto kern = spmm_pair_kernel<DT, IMG, BN, OUT>;
    if (smem_opt_in(kern, C::SMEM, opted) != cudaSuccess) cudaGetLastError();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.attrs = nullptr;  // the kernel declares its cluster shape (2 CTAs) at compile time
    cfg.numAttrs = 0;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (void*)kern, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 0;
    }
    cached = n > 0 ? n : -1;
    cache[dev].store(cached, std::memory_order_release);
  }
  return cached;
}

int stream_max_clusters(int size) {
  static std::atomic<int> cache[64][kMaxClusterSplit + 1];
  static std::atomic<uint64_t> opted{0};
  int dev = 0;
  if (size < 1 || size > kMaxClusterSplit) return -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  int cached = cache[dev][size].load(std::memory_order_acquire);
  if (!cached) {
    // every streaming configuration runs one CTA per SM, so one instance answers for all
    using C = Cfg<DT_I8, IMG_SP24, 32, OUT_I32 | kOutDirect, 0>;
    auto kern = spmm_kernel<DT_I8, IMG_SP24, 32, OUT_I32 | kOutDirect, 0>;
    if (smem_opt_in(kern, C::SMEM, opted) != cudaSuccess) cudaGetLastError();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(size, 1, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = (unsigned)size;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (void*)kern, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 0;
    }
    cached = n > 0 ? n : -1;
    cache[dev][size].store(cached, std::memory_order_release);
  }
  return cached;
}

int pair_max_clusters(int dt, int img, int bn, int out) {
  // All configurations share threads and (nearly) shared memory: one query per dtype/bn suffices.
  int n = -1;
  if (dt == DT_I8) {
    const bool f32 = out == OUT_F32;
    if (img == IMG_SP24) n = bn == 224 ? (f32 ? max_clusters_t<DT_I8, IMG_SP24, 224, OUT_F32>() : max_clusters_t<DT_I8, IMG_SP24, 224, OUT_I32>())
                       : bn == 192 ? (f32 ? max_clusters_t<DT_I8, IMG_SP24, 192, OUT_F32>() : max_clusters_t<DT_I8, IMG_SP24, 192, OUT_I32>())
                                   : (f32 ? max_clusters_t<DT_I8, IMG_SP24, 128, OUT_F32>() : max_clusters_t<DT_I8, IMG_SP24, 128, OUT_I32>());
    else n = bn == 224 ? (f32 ? max_clusters_t<DT_I8, IMG_DENSE, 224, OUT_F32>() : max_clusters_t<DT_I8, IMG_DENSE, 224, OUT_I32>())
           : bn == 192 ? (f32 ? max_clusters_t<DT_I8, IMG_DENSE, 192, OUT_F32>() : max_clusters_t<DT_I8, IMG_DENSE, 192, OUT_I32>())
                       : (f32 ? max_clusters_t<DT_I8, IMG_DENSE, 128, OUT_F32>() : max_clusters_t<DT_I8, IMG_DENSE, 128, OUT_I32>());
  } else if (dt == DT_F16) {
    n = img == IMG_SP24 ? (bn == 224 ? max_clusters_t<DT_F16, IMG_SP24, 224, OUT_F16>() : bn == 192 ? max_clusters_t<DT_F16, IMG_SP24, 192, OUT_F16>() : max_clusters_t<DT_F16, IMG_SP24, 128, OUT_F16>())
                        : (bn == 224 ? max_clusters_t<DT_F16, IMG_DENSE, 224, OUT_F16>() : bn == 192 ? max_clusters_t<DT_F16, IMG_DENSE, 192, OUT_F16>() : max_clusters_t<DT_F16, IMG_DENSE, 128, OUT_F16>());
  } else {
    n = img == IMG_SP24 ? (bn == 224 ? max_clusters_t<DT_BF16, IMG_SP24, 224, OUT_BF16>() : bn == 192 ? max_clusters_t<DT_BF16, IMG_SP24, 192, OUT_BF16>() : max_clusters_t<DT_BF16, IMG_SP24, 128, OUT_BF16>())
                        : (bn == 224 ? max_clusters_t<DT_BF16, IMG_DENSE, 224, OUT_BF16>() : bn == 192 ? max_clusters_t<DT_BF16, IMG_DENSE, 192, OUT_BF16>() : max_clusters_t<DT_BF16, IMG_DENSE, 128, OUT_BF16>());
  }
  return n;
}

}  // namespace nm
