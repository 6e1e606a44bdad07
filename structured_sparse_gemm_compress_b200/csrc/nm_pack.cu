// nm_pack.cu -- weight packing for the N:M sparse GEMM ("Realizable N:M Sparse
// Transformer Inference via Search-Kernel Co-Design", section 2.1 for the N:M
// rule and section 4.2 for the packed, decode-friendly representation).
//
// One fused pass over W writes both
//   * the canonical compressed format (values in ascending in-group position,
//     4-bit positions, two per byte), and
//   * the packed operand image the SpMM kernel streams (layout in nm_device.cuh).
// Each thread owns one row and 16 consecutive dense k positions, so every
// output byte has exactly one writer and W is read once, coalesced.
#include "nm_device.cuh"
#include "nm_internal.h"

namespace nm {
namespace {

template <int DT>
struct Elem;
template <>
struct Elem<DT_I8> {
  using T = int8_t;
  __device__ static uint32_t mag(T v) { return (uint32_t)(v < 0 ? -(int)v : (int)v); }
};
template <int DT>
struct Elem {  // FP16 / BF16 as raw bits: |x| orders like the bits with the sign cleared
  using T = uint16_t;
  __device__ static uint32_t mag(T v) { return (uint32_t)(v & 0x7FFFu); }
};

// 16 bytes <-> elements, little-endian, without type punning local arrays.
template <typename T>
__device__ __forceinline__ uint4 pack16(const T* v) {
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  constexpr int per = 4 / (int)sizeof(T);
#pragma unroll
  for (int e = 0; e < 16 / (int)sizeof(T); ++e) {
    const uint32_t bits = sizeof(T) == 1 ? (uint32_t)(uint8_t)v[e] : (uint32_t)(uint16_t)v[e];
    w[e / per] |= bits << (8 * (int)sizeof(T) * (e % per));
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}
template <typename T>
__device__ __forceinline__ void unpack16(uint4 q, T* v) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  constexpr int per = 4 / (int)sizeof(T);
#pragma unroll
  for (int e = 0; e < 16 / (int)sizeof(T); ++e) {
    const uint32_t bits = w[e / per] >> (8 * (int)sizeof(T) * (e % per));
    v[e] = sizeof(T) == 1 ? (T)(int8_t)(uint8_t)bits : (T)(uint16_t)bits;
  }
}

// Kept-position mask of one group of M (compile-time N, M, fully unrolled):
// N rounds of "largest magnitude not yet taken, first position on ties".
template <int DT, int N, int M>
__device__ __forceinline__ uint32_t select_group(const typename Elem<DT>::T* v) {
  uint32_t keep = 0;
#pragma unroll
  for (int j = 0; j < N; ++j) {
    int best = 0;
    uint32_t bv = 0;
    bool found = false;
#pragma unroll
    for (int p = 0; p < M; ++p) {
      const uint32_t a = Elem<DT>::mag(v[p]);
      const bool avail = ((keep >> p) & 1u) == 0u;
      const bool better = avail && (!found || a > bv);
      best = better ? p : best;
      bv = better ? a : bv;
      found = found || avail;
    }
    keep |= 1u << best;
  }
  return keep;
}

// v[p] for a runtime p in [0, M), without indexing a register array dynamically.
template <int M, typename T>
__device__ __forceinline__ T pick(const T* v, int p) {
  T out = v[0];
#pragma unroll
  for (int q = 1; q < M; ++q) out = (p == q) ? v[q] : out;
  return out;
}

// Store `bytes` (4, 8, 16 or 32) bytes held in w[] at dst: one vector store
// when dst is aligned to it, else byte stores.
__device__ __forceinline__ void store_bytes(uint8_t* dst, const uint32_t* w, int bytes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(dst);
  if (bytes == 32 && (a & 15u) == 0) {
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  } else if (bytes == 16 && (a & 15u) == 0) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if (bytes == 8 && (a & 7u) == 0) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  } else if (bytes == 4 && (a & 3u) == 0) {
    *reinterpret_cast<uint32_t*>(dst) = w[0];
  } else {
    for (int b = 0; b < bytes; ++b) dst[b] = (uint8_t)(w[b >> 2] >> (8 * (b & 3)));
  }
}

// INT8 fast path for a full unit of 16 positions held as four 32-bit words
// (byte i of word j is position 4j + i).  The kept set comes from a rank per
// position -- how many positions of its group precede it in the order
// (|w| descending, position ascending), kept iff fewer than N -- computed by
// pairwise compares; kept values are gathered with byte permutes.
template <int N, int M>
__device__ __forceinline__ uint32_t keep_mask_i8(const uint32_t (&w)[4]) {
  if constexpr (N == M) {
    return 0xFFFFu;
  } else {
    uint32_t mag[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int v = (int)(int8_t)(uint8_t)(w[c >> 2] >> (8 * (c & 3)));
      mag[c] = (uint32_t)(v < 0 ? -v : v);
    }
    uint32_t keep = 0;
#pragma unroll
    for (int g = 0; g < 16 / M; ++g) {
      int rank[M];
#pragma unroll
      for (int i = 0; i < M; ++i) rank[i] = 0;
#pragma unroll
      for (int p = 0; p < M; ++p)
#pragma unroll
        for (int q = p + 1; q < M; ++q) {
          // q (the later position) precedes p only with a strictly larger magnitude
          const int later_first = mag[g * M + q] > mag[g * M + p] ? 1 : 0;
          rank[p] += later_first;
          rank[q] += 1 - later_first;
        }
#pragma unroll
      for (int p = 0; p < M; ++p) keep |= (rank[p] < N ? 1u : 0u) << (g * M + p);
    }
    return keep;
  }
}

// Bytes of the kept positions of bits `m` (group-relative, ascending) as a
// byte-permute selector over the group's words; also their 4-bit positions.
template <int N>
__device__ __forceinline__ void kept_selector(uint32_t m, uint32_t& sel, uint32_t& nib) {
  sel = 0x4444u;  // nibble 4..7 select bytes of the zero second operand
  nib = 0;
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const uint32_t p = (uint32_t)(__ffs(m) - 1);
    m &= m - 1u;
    sel = (sel & ~(0xFu << (4 * j))) | (p << (4 * j));
    nib |= p << (4 * j);
  }
}

template <int N, int M, int IMG>
__device__ __forceinline__ void compress_unit_i8(const uint32_t (&w)[4], int64_t r, int64_t k0, int64_t K,
                                                 int n_kb, int8_t* __restrict__ values, uint8_t* __restrict__ idx,
                                                 int64_t idx_pitch, uint8_t* __restrict__ bpack) {
  constexpr int G = 16 / M;
  constexpr int CNT = 16 * N / M;
  const uint32_t keep = keep_mask_i8<N, M>(w);

  // ---- canonical format
  uint32_t vw[(CNT + 3) / 4] = {};
  uint32_t nibw[(CNT + 7) / 8 > 0 ? (CNT + 7) / 8 : 1] = {};
  if constexpr (N == M) {  // everything kept: the values are the unit itself
#pragma unroll
    for (int i = 0; i < 4; ++i) vw[i] = w[i];
#pragma unroll
    for (int e = 0; e < 16; ++e) nibw[e / 8] |= (uint32_t)(e % M) << (4 * (e % 8));
  } else {
    static_assert(N <= 4, "one byte permute gathers at most four kept values");
#pragma unroll
    for (int g = 0; g < G; ++g) {
      uint32_t sel, nib;
      kept_selector<N>((keep >> (g * M)) & ((1u << M) - 1u), sel, nib);
      uint32_t v;
      if constexpr (M == 4)
        v = __byte_perm(w[g], 0u, sel);
      else
        v = __byte_perm(w[2 * g], w[2 * g + 1], sel & 0x7777u);  // positions 0..7 of the pair
      const int e0 = g * N;  // first kept element of this group within the unit
#pragma unroll
      for (int j = 0; j < N; ++j) {
        const int e = e0 + j;
        vw[e / 4] |= ((v >> (8 * j)) & 0xFFu) << (8 * (e % 4));
        nibw[e / 8] |= ((nib >> (4 * j)) & 0xFu) << (4 * (e % 8));
      }
    }
  }
  const int64_t kept_per_row = (K / M) * N;
  const int64_t e0 = (k0 / M) * N;
  uint8_t* vdst = reinterpret_cast<uint8_t*>(values + r * kept_per_row + e0);
  uint8_t* idst = idx + r * idx_pitch + e0 / 2;
  if constexpr (CNT >= 4) {
    store_bytes(vdst, vw, CNT);
  } else {
    for (int b = 0; b < CNT; ++b) vdst[b] = (uint8_t)(vw[0] >> (8 * b));
  }
  if constexpr (CNT / 2 >= 4) {
    store_bytes(idst, nibw, CNT / 2);
  } else {
    for (int b = 0; b < CNT / 2; ++b) idst[b] = (uint8_t)(nibw[0] >> (8 * b));
  }

  // ---- packed operand image
  const int64_t ct = r / kRows;
  const uint32_t rr = (uint32_t)(r % kRows);
  const int kb = (int)(k0 / kblock_elems(DT_I8));
  const uint32_t kk = (uint32_t)(k0 % kblock_elems(DT_I8));
  uint8_t* chunk = bpack + ((size_t)ct * n_kb + kb) * (size_t)chunk_bytes(DT_I8, IMG);
  if constexpr (IMG == IMG_SP24) {
    uint32_t comp[2] = {0u, 0u}, meta = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // groups of four: two slots each, positions ascending
      const uint32_t bits = (keep >> (4 * j)) & 0xFu;
      const int n = __popc(bits);
      const uint32_t lo = (uint32_t)(__ffs(bits) - 1);
      const uint32_t hi = (uint32_t)(31 - __clz(bits | 1u));
      uint32_t i0, i1, sel;  // slot positions; selector (4 = a zero byte)
      if (n >= 2) {
        i0 = lo; i1 = hi; sel = lo | (hi << 4);
      } else if (n == 1 && lo < 3) {
        i0 = lo; i1 = 3; sel = lo | (4u << 4);
      } else if (n == 1) {
        i0 = 0; i1 = 3; sel = 4u | (3u << 4);
      } else {
        i0 = 0; i1 = 1; sel = 4u | (4u << 4);
      }
      const uint32_t two = __byte_perm(w[j], 0u, sel | 0x4400u) & 0xFFFFu;
      comp[j >> 1] |= two << (16 * (j & 1));
      meta |= (i0 | (i1 << 2)) << (4 * j);
    }
    *reinterpret_cast<uint2*>(chunk + swz128(rr, kk / 2)) = make_uint2(comp[0], comp[1]);
    *reinterpret_cast<uint16_t*>(chunk + kAtomBytes + meta_off16(DT_I8, rr, kk)) = (uint16_t)meta;
  } else {
    uint32_t d[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t b4 = (keep >> (4 * j)) & 0xFu;  // one bit per byte of word j
      const uint32_t bytemask = ((b4 & 1u) ? 0xFFu : 0u) | ((b4 & 2u) ? 0xFF00u : 0u) |
                                ((b4 & 4u) ? 0xFF0000u : 0u) | ((b4 & 8u) ? 0xFF000000u : 0u);
      d[j] = w[j] & bytemask;
    }
    *reinterpret_cast<uint4*>(chunk + (kk >> 7) * kAtomBytes + swz128(rr, kk & 127u)) =
        make_uint4(d[0], d[1], d[2], d[3]);
  }
}

template <int DT, int N, int M>
__global__ void __launch_bounds__(256) compress_kernel(const typename Elem<DT>::T* __restrict__ W, int64_t n_out,
                                                       int64_t K, int n_kb, typename Elem<DT>::T* __restrict__ values,
                                                       uint8_t* __restrict__ idx, int64_t idx_pitch,
                                                       uint8_t* __restrict__ bpack, int64_t total_units) {
  using T = typename Elem<DT>::T;
  constexpr int KB = kblock_elems(DT);
  constexpr int ES = elem_bytes(DT);
  constexpr int IMG = (N == M || (N == 4 && M == 8)) ? IMG_DENSE : IMG_SP24;
  constexpr int G = 16 / M;            // groups of M in one 16-position unit
  constexpr int CNT = 16 * N / M;      // kept values of a full unit
  const int64_t unit = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (unit >= total_units) return;
  const int64_t units_per_row = (int64_t)n_kb * (KB / 16);
  const int64_t r = unit / units_per_row;
  const int64_t k0 = (unit - r * units_per_row) * 16;

  // ---- load 16 positions (zero beyond the row or beyond K)
  T raw[16];
  const int64_t rem = K - k0;
  const int valid = r < n_out ? (int)(rem < 0 ? 0 : (rem > 16 ? 16 : rem)) : 0;
  const T* src = W + r * K + k0;
  if constexpr (DT == DT_I8) {
    if (valid == 16 && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(src));
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
      compress_unit_i8<N, M, IMG>(w, r, k0, K, n_kb, reinterpret_cast<int8_t*>(values), idx, idx_pitch, bpack);
      return;
    }
  }
  if (valid == 16 && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
#pragma unroll
    for (int h = 0; h < ES; ++h) unpack16<T>(__ldg(reinterpret_cast<const uint4*>(src) + h), raw + h * (16 / ES));
  } else {
#pragma unroll
    for (int c = 0; c < 16; ++c) raw[c] = (c < valid) ? src[c] : (T)0;
  }

  uint32_t keep = 0;
#pragma unroll
  for (int g = 0; g < G; ++g)
    if (g * M < valid) keep |= select_group<DT, N, M>(raw + g * M) << (g * M);

  // ---- canonical format: kept values in ascending position + 4-bit positions
  if (valid > 0) {
    const int64_t kept_per_row = (K / M) * N;
    const int64_t e0 = (k0 / M) * N;
    T vals[CNT];
    uint32_t nib[CNT / 8 > 0 ? CNT / 8 : 1] = {};
#pragma unroll
    for (int g = 0; g < G; ++g) {
      uint32_t m = (keep >> (g * M)) & ((1u << M) - 1u);
#pragma unroll
      for (int j = 0; j < N; ++j) {
        const int p = __ffs(m) - 1;  // j-th kept position of the group (ascending)
        m &= m - 1u;
        const int e = g * N + j;
        vals[e] = pick<M>(raw + g * M, p < 0 ? 0 : p);
        nib[e / 8] |= (uint32_t)(p & 0xF) << (4 * (e % 8));
      }
    }
    uint8_t* vdst = reinterpret_cast<uint8_t*>(values + r * kept_per_row + e0);
    uint8_t* idst = idx + r * idx_pitch + e0 / 2;
    if (valid == 16) {
      uint32_t vw[CNT * ES / 4 > 0 ? CNT * ES / 4 : 1];
      if constexpr (CNT * ES >= 4) {
#pragma unroll
        for (int i = 0; i < CNT * ES / 4; ++i) {
          uint32_t w = 0;
#pragma unroll
          for (int b = 0; b < 4 / ES; ++b) {
            const int e = i * (4 / ES) + b;
            w |= (ES == 1 ? (uint32_t)(uint8_t)vals[e] : (uint32_t)(uint16_t)vals[e]) << (8 * ES * b);
          }
          vw[i] = w;
        }
        store_bytes(vdst, vw, CNT * ES);
      }
      if constexpr (CNT / 2 >= 4) {
        store_bytes(idst, nib, CNT / 2);
      } else {
        for (int b = 0; b < CNT / 2; ++b) idst[b] = (uint8_t)(nib[0] >> (8 * b));
      }
    } else {  // ragged end of a row: only the groups that exist
      const int cnt = (valid / M) * N;
      T* vd = values + r * kept_per_row + e0;
#pragma unroll
      for (int e = 0; e < CNT; ++e)
        if (e < cnt) vd[e] = vals[e];
      for (int b = 0; b < (cnt + 1) / 2; ++b) {
        const int e = 2 * b;
        uint8_t byte = (uint8_t)((nib[e / 8] >> (4 * (e % 8))) & 0xF);
        if (e + 1 < cnt) byte |= (uint8_t)(((nib[(e + 1) / 8] >> (4 * ((e + 1) % 8))) & 0xF) << 4);
        idst[b] = byte;
      }
    }
  }

  // ---- packed operand image
  const int64_t ct = r / kRows;
  const uint32_t rr = (uint32_t)(r % kRows);
  const int kb = (int)(k0 / KB);
  const uint32_t kk = (uint32_t)(k0 % KB);
  uint8_t* chunk = bpack + ((size_t)ct * n_kb + kb) * (size_t)chunk_bytes(DT, IMG);

  if constexpr (IMG == IMG_SP24) {
    T comp[8];
    uint32_t meta = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // groups of four: two slots each, positions ascending
      const uint32_t bits = (keep >> (4 * j)) & 0xFu;
      const int n = __popc(bits);
      const int lo = __ffs(bits) - 1;
      const int hi = 31 - __clz(bits | 1u);
      int i0, i1;
      T v0, v1;
      if (n >= 2) {
        i0 = lo; i1 = hi;
        v0 = pick<4>(raw + 4 * j, lo);
        v1 = pick<4>(raw + 4 * j, hi);
      } else if (n == 1 && lo < 3) {
        i0 = lo; i1 = 3;
        v0 = pick<4>(raw + 4 * j, lo);
        v1 = (T)0;
      } else if (n == 1) {
        i0 = 0; i1 = 3;
        v0 = (T)0;
        v1 = raw[4 * j + 3];
      } else {
        i0 = 0; i1 = 1;
        v0 = (T)0;
        v1 = (T)0;
      }
      comp[2 * j] = v0;
      comp[2 * j + 1] = v1;
      meta |= (uint32_t)(i0 | (i1 << 2)) << (4 * j);
    }
    if constexpr (ES == 1) {
      uint32_t w0 = 0, w1 = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        w0 |= (uint32_t)(uint8_t)comp[e] << (8 * e);
        w1 |= (uint32_t)(uint8_t)comp[e + 4] << (8 * e);
      }
      *reinterpret_cast<uint2*>(chunk + swz128(rr, kk / 2)) = make_uint2(w0, w1);
    } else {
      *reinterpret_cast<uint4*>(chunk + swz128(rr, kk)) = pack16<T>(comp);
    }
    *reinterpret_cast<uint16_t*>(chunk + kAtomBytes + meta_off16(DT, rr, kk)) = (uint16_t)meta;
  } else {
    T dense[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) dense[c] = ((keep >> c) & 1u) ? raw[c] : (T)0;
#pragma unroll
    for (int h = 0; h < ES; ++h) {  // 16-byte units of this thread's slice
      const uint32_t byte = kk * ES + 16u * h;
      *reinterpret_cast<uint4*>(chunk + (byte >> 7) * kAtomBytes + swz128(rr, byte & 127u)) =
          pack16<T>(dense + h * (16 / ES));
    }
  }
}

template <int DT>
__global__ void __launch_bounds__(256) decompress_kernel(const uint8_t* __restrict__ bpack, int64_t n_out,
                                                         int64_t K, int img, int n_kb,
                                                         typename Elem<DT>::T* __restrict__ Wout,
                                                         int64_t total_units) {
  using T = typename Elem<DT>::T;
  constexpr int KB = kblock_elems(DT);
  constexpr int ES = elem_bytes(DT);
  const int64_t unit = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (unit >= total_units) return;
  const int64_t units_per_row = (K + 15) / 16;
  const int64_t r = unit / units_per_row;
  const int64_t k0 = (unit - r * units_per_row) * 16;
  const int valid = (int)(K - k0 > 16 ? 16 : K - k0);
  const int64_t ct = r / kRows;
  const uint32_t rr = (uint32_t)(r % kRows);
  const int kb = (int)(k0 / KB);
  const uint32_t kk = (uint32_t)(k0 % KB);
  const uint8_t* chunk = bpack + ((size_t)ct * n_kb + kb) * (size_t)chunk_bytes(DT, img);

  T out[16];
  if (img == IMG_SP24) {
    T comp[8];
    if (ES == 1) {
      const uint64_t v = *reinterpret_cast<const uint64_t*>(chunk + swz128(rr, kk / 2));
#pragma unroll
      for (int e = 0; e < 8; ++e) comp[e] = (T)(int8_t)(uint8_t)(v >> (8 * e));
    } else {
      unpack16<T>(*reinterpret_cast<const uint4*>(chunk + swz128(rr, kk)), comp);
    }
    const uint32_t meta = *reinterpret_cast<const uint16_t*>(chunk + kAtomBytes + meta_off16(DT, rr, kk));
#pragma unroll
    for (int c = 0; c < 16; ++c) out[c] = (T)0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int nib = (meta >> (4 * j)) & 0xF;
      const int i0 = nib & 3, i1 = (nib >> 2) & 3;
      out[4 * j + i0] = comp[2 * j];
      if (i1 != i0) {
        out[4 * j + i1] = comp[2 * j + 1];
      } else if (ES == 1) {
        out[4 * j + i0] = (T)((int)comp[2 * j] + (int)comp[2 * j + 1]);
      }
      // (equal 2-byte positions only occur for all-zero padding slots)
    }
  } else {
#pragma unroll
    for (int h = 0; h < ES; ++h) {
      const uint32_t byte = kk * ES + 16u * h;
      unpack16<T>(*reinterpret_cast<const uint4*>(chunk + (byte >> 7) * kAtomBytes + swz128(rr, byte & 127u)),
                  out + h * (16 / ES));
    }
  }
  for (int c = 0; c < valid; ++c) Wout[r * K + k0 + c] = out[c];
}

// ------------------------------------------------------------------ tile-shared patterns
//
// One pattern per 128-row channel tile (nm_compress_tile): per tile and group
// of M positions, score(p) = sum over the tile's rows of |w| at p, kept = the N
// largest scores, ties to the lower position.  Scores are exact integers:
// |int8| as is, |fp16| in units of 2^-24 (every fp16 magnitude is a whole
// multiple of 2^-24 below 2^16, so a tile's sum stays below 2^47).
template <int DT>
struct TileScore;
template <>
struct TileScore<DT_I8> {
  using S = int;
  __device__ static S of(int8_t v) { return v < 0 ? -(int)v : (int)v; }
};
template <>
struct TileScore<DT_F16> {
  using S = long long;
  __device__ static S of(uint16_t bits) {
    const int e = (bits >> 10) & 0x1F;
    const long long m = bits & 0x3FF;
    return e == 0 ? m : ((m | 0x400) << (e - 1));  // (1.m) * 2^(e-15) = (m | 2^10) * 2^(e-25)
  }
};

// Block = 8 row slices x 32 groups; slice s sums rows s, s + 8, ... of the tile,
// then one thread per group combines the slices and ranks the M positions.
template <int DT, int N, int M>
__global__ void __launch_bounds__(256) tile_select_kernel(const typename Elem<DT>::T* __restrict__ W, int64_t n_out,
                                                          int64_t K, int64_t gblocks, int32_t* __restrict__ kidx,
                                                          int64_t kidx_pitch) {
  using S = typename TileScore<DT>::S;
  constexpr int G = 32, SL = 8;
  __shared__ S part[SL][G][M];
  const int gl = threadIdx.x & 31, sl = threadIdx.x >> 5;
  const int64_t ct = blockIdx.x / gblocks;
  const int64_t g = (blockIdx.x - ct * gblocks) * G + gl;
  const int64_t groups = K / M;
  S acc[M];
#pragma unroll
  for (int p = 0; p < M; ++p) acc[p] = 0;
  if (g < groups) {
#pragma unroll 4
    for (int i = sl; i < kRows; i += SL) {
      const int64_t r = ct * kRows + i;
      if (r >= n_out) break;
      const typename Elem<DT>::T* src = W + r * K + g * M;
#pragma unroll
      for (int p = 0; p < M; ++p) acc[p] += TileScore<DT>::of(src[p]);
    }
  }
#pragma unroll
  for (int p = 0; p < M; ++p) part[sl][gl][p] = acc[p];
  __syncthreads();
  if (sl != 0 || g >= groups) return;
  S sc[M];
#pragma unroll
  for (int p = 0; p < M; ++p) {
    S t = 0;
#pragma unroll
    for (int q = 0; q < SL; ++q) t += part[q][gl][p];
    sc[p] = t;
  }
  int e = 0;
#pragma unroll
  for (int p = 0; p < M; ++p) {
    int ahead = 0;
#pragma unroll
    for (int q = 0; q < M; ++q) ahead += (sc[q] > sc[p] || (sc[q] == sc[p] && q < p)) ? 1 : 0;
    if (ahead < N) kidx[ct * kidx_pitch + g * N + e++] = (int32_t)(g * M + p);
  }
}

// One thread per (row, 16 consecutive kept slots): gathers the kept values
// through the tile's kept k list and writes the canonical format (rows < n_out,
// slots < kp) and the gather image (zero beyond them).
template <int DT>
__global__ void __launch_bounds__(256) tile_pack_kernel(const typename Elem<DT>::T* __restrict__ W, int64_t n_out,
                                                        int64_t K, int64_t kp, int M, int n_kb,
                                                        const int32_t* __restrict__ kidx, int64_t kidx_pitch,
                                                        typename Elem<DT>::T* __restrict__ values,
                                                        uint8_t* __restrict__ idx, int64_t idx_pitch,
                                                        uint8_t* __restrict__ bpack, int64_t total_units) {
  using T = typename Elem<DT>::T;
  constexpr int KBG = gather_kblock_elems(DT);
  constexpr int ES = elem_bytes(DT);
  const int64_t unit = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (unit >= total_units) return;
  const int64_t units_per_row = (int64_t)n_kb * (KBG / 16);
  const int64_t r = unit / units_per_row;
  const int64_t e0 = (unit - r * units_per_row) * 16;
  const int64_t ct = r / kRows;
  int32_t kk[16];
  const int4* kl = reinterpret_cast<const int4*>(kidx + ct * kidx_pitch + e0);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int4 v = __ldg(kl + q);
    kk[4 * q] = v.x; kk[4 * q + 1] = v.y; kk[4 * q + 2] = v.z; kk[4 * q + 3] = v.w;
  }
  const bool row_ok = r < n_out;
  T v[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = (row_ok && e0 + j < kp) ? W[r * K + kk[j]] : (T)0;

  if (row_ok) {  // canonical format
    const int cnt = (int)(kp - e0 < 16 ? kp - e0 : 16);
    uint32_t nib[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < cnt) nib[j / 8] |= (uint32_t)(kk[j] % M) << (4 * (j % 8));
    if (cnt == 16) {
      const uint4 lo = pack16<T>(v);
      uint32_t vw[8] = {lo.x, lo.y, lo.z, lo.w, 0u, 0u, 0u, 0u};
      if constexpr (ES == 2) {
        const uint4 hi = pack16<T>(v + 8);
        vw[4] = hi.x; vw[5] = hi.y; vw[6] = hi.z; vw[7] = hi.w;
      }
      store_bytes(reinterpret_cast<uint8_t*>(values + r * kp + e0), vw, 16 * ES);
      store_bytes(idx + r * idx_pitch + e0 / 2, nib, 8);
    } else {
      for (int j = 0; j < cnt; ++j) values[r * kp + e0 + j] = v[j];
      for (int b = 0; b < (cnt + 1) / 2; ++b) idx[r * idx_pitch + e0 / 2 + b] = (uint8_t)(nib[b / 4] >> (8 * (b % 4)));
    }
  }

  // gather image: 16 slots = 16 * ES bytes of the tile row's 128-byte k-block row
  const uint32_t rr = (uint32_t)(r % kRows);
  const int kb = (int)(e0 / KBG);
  const uint32_t byte0 = (uint32_t)(e0 % KBG) * ES;
  uint8_t* chunk = bpack + ((size_t)ct * n_kb + kb) * (size_t)chunk_bytes(DT, IMG_GATHER);
#pragma unroll
  for (int h = 0; h < ES; ++h)
    *reinterpret_cast<uint4*>(chunk + swz128(rr, byte0 + 16u * h)) = pack16<T>(v + h * (16 / ES));
}

// Masked dense weight from the gather image and the kept k list (Wout zeroed first).
template <int DT>
__global__ void __launch_bounds__(256) tile_decompress_kernel(const uint8_t* __restrict__ bpack, int64_t n_out,
                                                              int64_t K, int64_t kp, int n_kb,
                                                              const int32_t* __restrict__ kidx, int64_t kidx_pitch,
                                                              typename Elem<DT>::T* __restrict__ Wout,
                                                              int64_t total_units) {
  using T = typename Elem<DT>::T;
  constexpr int KBG = gather_kblock_elems(DT);
  constexpr int ES = elem_bytes(DT);
  const int64_t unit = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (unit >= total_units) return;
  const int64_t units_per_row = (kp + 15) / 16;
  const int64_t r = unit / units_per_row;
  const int64_t e0 = (unit - r * units_per_row) * 16;
  const int64_t ct = r / kRows;
  const uint32_t rr = (uint32_t)(r % kRows);
  const int kb = (int)(e0 / KBG);
  const uint32_t byte0 = (uint32_t)(e0 % KBG) * ES;
  const uint8_t* chunk = bpack + ((size_t)ct * n_kb + kb) * (size_t)chunk_bytes(DT, IMG_GATHER);
  T v[16];
#pragma unroll
  for (int h = 0; h < ES; ++h)
    unpack16<T>(*reinterpret_cast<const uint4*>(chunk + swz128(rr, byte0 + 16u * h)), v + h * (16 / ES));
  const int cnt = (int)(kp - e0 < 16 ? kp - e0 : 16);
  for (int j = 0; j < cnt; ++j) Wout[r * K + kidx[ct * kidx_pitch + e0 + j]] = v[j];
}

}  // namespace

template <int DT, int N, int M>
static void launch_compress_t(const nm_handle* h, const void* W, int64_t total, cudaStream_t s) {
  using T = typename Elem<DT>::T;
  const int threads = 256;
  const unsigned blocks = (unsigned)((total + threads - 1) / threads);
  compress_kernel<DT, N, M><<<blocks, threads, 0, s>>>((const T*)W, h->n_out, h->k, h->n_kb, (T*)h->d_values,
                                                       h->d_idx, h->idx_pitch, h->d_bpack, total);
}

template <int DT>
static cudaError_t launch_compress_dt(const nm_handle* h, const void* W, int64_t total, cudaStream_t s) {
  const int nm_code = h->N * 16 + h->M;
  switch (nm_code) {
    case 1 * 16 + 4: launch_compress_t<DT, 1, 4>(h, W, total, s); break;
    case 2 * 16 + 4: launch_compress_t<DT, 2, 4>(h, W, total, s); break;
    case 2 * 16 + 8: launch_compress_t<DT, 2, 8>(h, W, total, s); break;
    case 4 * 16 + 8: launch_compress_t<DT, 4, 8>(h, W, total, s); break;
    case 4 * 16 + 4: launch_compress_t<DT, 4, 4>(h, W, total, s); break;
    case 8 * 16 + 8: launch_compress_t<DT, 8, 8>(h, W, total, s); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_compress(const nm_handle* h, const void* W, cudaStream_t s) {
  const int KB = kblock_elems(h->dt);
  const int64_t total = (int64_t)h->n_ct * kRows * ((int64_t)h->n_kb * (KB / 16));
  switch (h->dt) {
    case DT_I8: return launch_compress_dt<DT_I8>(h, W, total, s);
    case DT_F16: return launch_compress_dt<DT_F16>(h, W, total, s);
    default: return launch_compress_dt<DT_BF16>(h, W, total, s);
  }
}

template <int DT, int N, int M>
static void launch_tile_select_t(const nm_handle* h, const void* W, cudaStream_t s) {
  using T = typename Elem<DT>::T;
  const int64_t groups = h->k / M;
  const int64_t gblocks = (groups + 31) / 32;
  const int64_t kidx_pitch = (int64_t)h->n_kb * gather_kblock_elems(DT);
  tile_select_kernel<DT, N, M><<<(unsigned)(gblocks * h->n_ct), 256, 0, s>>>((const T*)W, h->n_out, h->k, gblocks,
                                                                              h->d_kidx, kidx_pitch);
}

template <int DT>
static cudaError_t launch_compress_tile_dt(const nm_handle* h, const void* W, cudaStream_t s) {
  using T = typename Elem<DT>::T;
  switch (h->N * 16 + h->M) {
    case 1 * 16 + 4: launch_tile_select_t<DT, 1, 4>(h, W, s); break;
    case 2 * 16 + 4: launch_tile_select_t<DT, 2, 4>(h, W, s); break;
    case 2 * 16 + 8: launch_tile_select_t<DT, 2, 8>(h, W, s); break;
    case 4 * 16 + 8: launch_tile_select_t<DT, 4, 8>(h, W, s); break;
    case 4 * 16 + 4: launch_tile_select_t<DT, 4, 4>(h, W, s); break;
    case 8 * 16 + 8: launch_tile_select_t<DT, 8, 8>(h, W, s); break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  constexpr int KBG = gather_kblock_elems(DT);
  const int64_t kidx_pitch = (int64_t)h->n_kb * KBG;
  const int64_t total = (int64_t)h->n_ct * kRows * ((int64_t)h->n_kb * (KBG / 16));
  const unsigned blocks = (unsigned)((total + 255) / 256);
  tile_pack_kernel<DT><<<blocks, 256, 0, s>>>((const T*)W, h->n_out, h->k, h->kp, h->M, h->n_kb, h->d_kidx,
                                             kidx_pitch, (T*)h->d_values, h->d_idx, h->idx_pitch, h->d_bpack, total);
  return cudaGetLastError();
}

cudaError_t launch_compress_tile(const nm_handle* h, const void* W, cudaStream_t s) {
  switch (h->dt) {
    case DT_I8: return launch_compress_tile_dt<DT_I8>(h, W, s);
    case DT_F16: return launch_compress_tile_dt<DT_F16>(h, W, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int DT>
static cudaError_t launch_tile_decompress_t(const nm_handle* h, void* Wout, cudaStream_t s) {
  using T = typename Elem<DT>::T;
  cudaError_t e = cudaMemsetAsync(Wout, 0, (size_t)h->n_out * (size_t)h->k * elem_bytes(DT), s);
  if (e != cudaSuccess) return e;
  const int64_t total = h->n_out * ((h->kp + 15) / 16);
  const int64_t kidx_pitch = (int64_t)h->n_kb * gather_kblock_elems(DT);
  tile_decompress_kernel<DT><<<(unsigned)((total + 255) / 256), 256, 0, s>>>(
      h->d_bpack, h->n_out, h->k, h->kp, h->n_kb, h->d_kidx, kidx_pitch, (T*)Wout, total);
  return cudaGetLastError();
}

cudaError_t launch_decompress(const nm_handle* h, void* Wout, cudaStream_t s) {
  if (h->tile) {
    switch (h->dt) {
      case DT_I8: return launch_tile_decompress_t<DT_I8>(h, Wout, s);
      case DT_F16: return launch_tile_decompress_t<DT_F16>(h, Wout, s);
      default: return cudaErrorInvalidValue;
    }
  }
  const int64_t total = h->n_out * ((h->k + 15) / 16);
  const int threads = 256;
  const unsigned blocks = (unsigned)((total + threads - 1) / threads);
  switch (h->dt) {
    case DT_I8:
      decompress_kernel<DT_I8><<<blocks, threads, 0, s>>>(h->d_bpack, h->n_out, h->k, h->img, h->n_kb,
                                                         (int8_t*)Wout, total);
      break;
    case DT_F16:
      decompress_kernel<DT_F16><<<blocks, threads, 0, s>>>(h->d_bpack, h->n_out, h->k, h->img, h->n_kb,
                                                          (uint16_t*)Wout, total);
      break;
    default:
      decompress_kernel<DT_BF16><<<blocks, threads, 0, s>>>(h->d_bpack, h->n_out, h->k, h->img, h->n_kb,
                                                           (uint16_t*)Wout, total);
      break;
  }
  return cudaGetLastError();
}

}  // namespace nm
