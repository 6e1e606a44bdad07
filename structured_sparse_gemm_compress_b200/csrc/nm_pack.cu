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

// Kept-position mask of one group of M: N rounds of "largest magnitude not yet
// taken, first position on ties".
template <int DT>
__device__ __forceinline__ uint32_t select_group(const uint32_t* a, int N, int M) {
  uint32_t keep = 0;
  for (int j = 0; j < N; ++j) {
    int best = -1;
    uint32_t bv = 0;
    for (int p = 0; p < M; ++p) {
      if ((keep >> p) & 1u) continue;
      if (best < 0 || a[p] > bv) {
        best = p;
        bv = a[p];
      }
    }
    keep |= 1u << best;
  }
  return keep;
}

template <int DT>
__global__ void __launch_bounds__(256) compress_kernel(const typename Elem<DT>::T* __restrict__ W, int64_t n_out,
                                                       int64_t K, int N, int M, int img, int n_kb,
                                                       typename Elem<DT>::T* __restrict__ values,
                                                       uint8_t* __restrict__ idx, int64_t idx_pitch,
                                                       uint8_t* __restrict__ bpack, int64_t total_units) {
  using T = typename Elem<DT>::T;
  constexpr int KB = kblock_elems(DT);
  constexpr int ES = elem_bytes(DT);
  const int64_t unit = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (unit >= total_units) return;
  const int64_t units_per_row = (int64_t)n_kb * (KB / 16);
  const int64_t r = unit / units_per_row;
  const int64_t k0 = (unit - r * units_per_row) * 16;

  T raw[16];
  uint32_t a[16];
  const bool row_ok = r < n_out;
  const int64_t rem = K - k0;
  const int valid = row_ok ? (int)(rem < 0 ? 0 : (rem > 16 ? 16 : rem)) : 0;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    raw[c] = (c < valid) ? W[r * K + k0 + c] : (T)0;
    a[c] = Elem<DT>::mag(raw[c]);
  }
  uint32_t keep = 0;
  for (int g = 0; g < valid / M; ++g) keep |= select_group<DT>(a + g * M, N, M) << (g * M);

  // ---- canonical format
  if (valid > 0) {
    const int64_t kept_per_row = (K / M) * N;
    const int64_t e0 = (k0 / M) * N;
    T* vdst = values + r * kept_per_row + e0;
    uint64_t nib = 0;
    int cnt = 0;
    for (int c = 0; c < valid; ++c) {
      if ((keep >> c) & 1u) {
        vdst[cnt] = raw[c];
        nib |= (uint64_t)(c % M) << (4 * cnt);
        ++cnt;
      }
    }
    uint8_t* idst = idx + r * idx_pitch + e0 / 2;
    for (int b = 0; b < (cnt + 1) / 2; ++b) idst[b] = (uint8_t)(nib >> (8 * b));
  }

  // ---- packed operand image
  const int64_t ct = r / kRows;
  const uint32_t rr = (uint32_t)(r % kRows);
  const int kb = (int)(k0 / KB);
  const uint32_t kk = (uint32_t)(k0 % KB);
  uint8_t* chunk = bpack + ((size_t)ct * n_kb + kb) * (size_t)chunk_bytes(DT, img);

  if (img == IMG_SP24) {
    T comp[8];
    uint32_t meta = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t bits = (keep >> (4 * j)) & 0xFu;
      int i0, i1;
      T v0, v1;
      const int n = __popc(bits);
      if (n >= 2) {
        i0 = __ffs(bits) - 1;
        i1 = __ffs(bits & (bits - 1)) - 1;
        v0 = raw[4 * j + i0];
        v1 = raw[4 * j + i1];
      } else if (n == 1) {
        const int p = __ffs(bits) - 1;
        if (p < 3) {
          i0 = p; i1 = 3; v0 = raw[4 * j + p]; v1 = (T)0;
        } else {
          i0 = 0; i1 = 3; v0 = (T)0; v1 = raw[4 * j + 3];
        }
      } else {
        i0 = 0; i1 = 1; v0 = (T)0; v1 = (T)0;
      }
      comp[2 * j] = v0;
      comp[2 * j + 1] = v1;
      meta |= (uint32_t)(i0 | (i1 << 2)) << (4 * j);
    }
    if (ES == 1) {
      uint64_t packed = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) packed |= (uint64_t)(uint8_t)comp[e] << (8 * e);
      *reinterpret_cast<uint64_t*>(chunk + swz128(rr, kk / 2)) = packed;
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

}  // namespace

cudaError_t launch_compress(const nm_handle* h, const void* W, cudaStream_t s) {
  const int KB = kblock_elems(h->dt);
  const int64_t total = (int64_t)h->n_ct * kRows * ((int64_t)h->n_kb * (KB / 16));
  const int threads = 256;
  const unsigned blocks = (unsigned)((total + threads - 1) / threads);
  switch (h->dt) {
    case DT_I8:
      compress_kernel<DT_I8><<<blocks, threads, 0, s>>>(
          (const int8_t*)W, h->n_out, h->k, h->N, h->M, h->img, h->n_kb, (int8_t*)h->d_values, h->d_idx,
          h->idx_pitch, h->d_bpack, total);
      break;
    case DT_F16:
      compress_kernel<DT_F16><<<blocks, threads, 0, s>>>(
          (const uint16_t*)W, h->n_out, h->k, h->N, h->M, h->img, h->n_kb, (uint16_t*)h->d_values, h->d_idx,
          h->idx_pitch, h->d_bpack, total);
      break;
    default:
      compress_kernel<DT_BF16><<<blocks, threads, 0, s>>>(
          (const uint16_t*)W, h->n_out, h->k, h->N, h->M, h->img, h->n_kb, (uint16_t*)h->d_values, h->d_idx,
          h->idx_pitch, h->d_bpack, total);
      break;
  }
  return cudaGetLastError();
}

cudaError_t launch_decompress(const nm_handle* h, void* Wout, cudaStream_t s) {
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
