// Device helpers shared by the TurboQuant kernels (warp reductions, the
// in-register Walsh-Hadamard butterflies and the bit-stream packer).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "tq_internal.h"

namespace tq {

constexpr unsigned kFull = 0xffffffffu;
// sqrt(pi/2): E|g| = sqrt(2/pi) for g ~ N(0,1), so sqrt(pi/2)/m * gamma * <S x, sign(S r)>
// is an unbiased estimate of <x, r>.
constexpr float kQjl = 1.2533141373155003f;

// Record row of token t of unit u under the cache addressing p (t the first token of a
// tile, which never crosses a page). A page index outside [0, n_pages) sets bit 2 of
// *err and reads page 0 instead.
__device__ __forceinline__ int64_t record_row(const Paging& p, int64_t max_len, int64_t u, int64_t t,
                                              unsigned int* err) {
  if (!p.block_table) return u * max_len + t;
  int64_t pg = __ldg(p.block_table + u * p.max_pages + t / p.page_size);
  if (pg < 0 || pg >= p.n_pages) {
    atomicOr(err, 4u);
    pg = 0;
  }
  return pg * p.page_size + t % p.page_size;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Load E consecutive elements (row[lane*E .. lane*E+E-1]) as fp32.
template <int E, typename T>
__device__ __forceinline__ void load_lane(const T* __restrict__ row, int lane, float (&x)[E]) {
  const T* p = row + lane * E;
  if constexpr (sizeof(T) == 4 && E % 4 == 0) {
#pragma unroll
    for (int e = 0; e < E; e += 4) {
      float4 f = *reinterpret_cast<const float4*>(p + e);
      x[e] = f.x; x[e + 1] = f.y; x[e + 2] = f.z; x[e + 3] = f.w;
    }
  } else if constexpr (sizeof(T) == 2 && E % 4 == 0) {
#pragma unroll
    for (int e = 0; e < E; e += 4) {
      uint2 u = *reinterpret_cast<const uint2*>(p + e);
      x[e] = __uint_as_float(u.x << 16);
      x[e + 1] = __uint_as_float(u.x & 0xffff0000u);
      x[e + 2] = __uint_as_float(u.y << 16);
      x[e + 3] = __uint_as_float(u.y & 0xffff0000u);
    }
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = to_f32<T>(p[e]);
  }
}

// Unnormalised Sylvester Walsh-Hadamard transform of a d = 32*E vector held
// E consecutive elements per lane: y_i = sum_j (-1)^popcount(i & j) x_j.
// Butterflies of stride < E stay in registers, larger strides use shuffles.
template <int E>
__device__ __forceinline__ void fwht_warp(float (&x)[E], int lane) {
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if ((e & h) == 0) {
        float a = x[e], b = x[e + h];
        x[e] = a + b;
        x[e + h] = a - b;
      }
    }
  }
#pragma unroll
  for (int lm = 1; lm < 32; lm <<= 1) {
    const bool upper = lane & lm;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float o = __shfl_xor_sync(kFull, x[e], lm);
      x[e] = upper ? (o - x[e]) : (x[e] + o);
    }
  }
}

__device__ __forceinline__ float flip_sign(float x, uint32_t bit) {
  return __uint_as_float(__float_as_uint(x) ^ (bit << 31));
}

// Cooperative packer: lane `lane` contributes `nbits` bits (value `v`) at bit
// offset lane*nbits of a little-endian stream of `nwords` 32-bit words. Returns
// the word with index == lane (lanes >= nwords get 0).
__device__ __forceinline__ uint32_t pack_stream_word(uint32_t v, int nbits, int nwords, int lane) {
  const int o = lane * nbits;
  const uint64_t wide = (uint64_t)v << (o & 31);
  const uint32_t lo = (uint32_t)wide, hi = (uint32_t)(wide >> 32);
  const int w0 = o >> 5;
  uint32_t mine = 0;
  for (int w = 0; w < nwords; ++w) {
    uint32_t c = (w == w0 ? lo : 0u) | (w == w0 + 1 ? hi : 0u);
    uint32_t word = __reduce_or_sync(kFull, c);
    if (lane == w) mine = word;
  }
  return mine;
}

// Same with the bit count per lane and the word count known at compile time.
template <int NBITS, int NWORDS>
__device__ __forceinline__ uint32_t pack_stream_word_t(uint32_t v, int lane) {
  static_assert(NBITS <= 32 && NWORDS <= 32, "stream geometry");
  const int o = lane * NBITS;
  const uint64_t wide = (uint64_t)v << (o & 31);
  const uint32_t lo = (uint32_t)wide, hi = (uint32_t)(wide >> 32);
  const int w0 = o >> 5;
  uint32_t mine = 0;
#pragma unroll
  for (int w = 0; w < NWORDS; ++w) {
    const uint32_t c = (w == w0 ? lo : 0u) | ((32 % (NBITS > 0 ? NBITS : 32) != 0 && w == w0 + 1) ? hi : 0u);
    const uint32_t word = __reduce_or_sync(kFull, c);
    if (lane == w) mine = word;
  }
  return mine;
}

// Code j (bits [b*j, b*j+b)) from a little-endian stream held in registers.
template <int B, int NW>
__device__ __forceinline__ uint32_t stream_code(const uint32_t (&w)[NW], int j) {
  const int o = j * B;
  const int wi = o >> 5, sh = o & 31;
  uint32_t v = w[wi] >> sh;
  if (sh + B > 32 && wi + 1 < NW) v |= w[wi + 1] << (32 - sh);
  return v & ((1u << B) - 1u);
}

// Parity word of the 32 three-bit codes held in three consecutive stream words: bit p is the
// parity of code (32 (p mod 3) + p) / 3.
__device__ __forceinline__ uint32_t parity_word(uint32_t x0, uint32_t x1, uint32_t x2) {
  const uint32_t X0 = x0 ^ __funnelshift_r(x0, x1, 1) ^ __funnelshift_r(x0, x1, 2);
  const uint32_t X1 = x1 ^ __funnelshift_r(x1, x2, 1) ^ __funnelshift_r(x1, x2, 2);
  const uint32_t X2 = x2 ^ (x2 >> 1) ^ (x2 >> 2);
  return (X0 & 0x49249249u) | (X1 & 0x92492492u) | (X2 & 0x24924924u);
}

}  // namespace tq
