// Decompression of packed keys and values to fp32 (debug / parity path, not
// timed). Keys: x = n Pi^T (c[idx] + sqrt(pi/2)/m * gamma * S^T s), the vector
// the decode estimator implicitly scores against; values: min + scale * code.
// One warp per vector, lane l owning coordinates [l*E, l*E+E).
#include <cuda_runtime.h>

#include "tq_device.cuh"

namespace tq {
namespace {

constexpr int kWarps = 8;

struct DecompressArgs {
  const uint8_t* k_codes;
  const uint8_t* k_signs;
  const uint16_t* k_norms;
  const uint8_t* v_codes;
  const uint16_t* v_params;
  int64_t n_vec;
  float* k_out;
  float* v_out;
  const float* S;   // [m][d]
  const float* Pi;  // [d][d], Haar only
  Codebook cb;
  int lm_bits, m, v_bits, rot;
  float inv_sqrt_d;
};

template <int D>
__device__ void decompress_key(const DecompressArgs& a, int64_t i, int lane, float* ybuf) {
  constexpr int E = D / 32;
  const int cwords = a.lm_bits * D / 32, swords = a.m / 32;
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(a.k_codes) + i * cwords;
  const uint32_t* sw = reinterpret_cast<const uint32_t*>(a.k_signs) + i * swords;
  const uint32_t nb = reinterpret_cast<const uint32_t*>(a.k_norms)[i];
  const float n = __half2float(__ushort_as_half((unsigned short)(nb & 0xffffu)));
  const float gamma = __half2float(__ushort_as_half((unsigned short)(nb >> 16)));
  float y[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int j = lane * E + e, o = j * a.lm_bits;
    uint32_t v = cw[o >> 5] >> (o & 31);
    if ((o & 31) + a.lm_bits > 32) v |= cw[(o >> 5) + 1] << (32 - (o & 31));
    const uint32_t code = v & ((1u << a.lm_bits) - 1u);
    const float cv = a.cb.c[code];
    float acc = 0.f;
    for (int w = 0; w < swords; ++w) {
      const uint32_t bits = sw[w];
      for (int bb = 0; bb < 32; ++bb) {
        const float s = a.S[(size_t)(w * 32 + bb) * D + j];
        acc += ((bits >> bb) & 1u) ? s : -s;
      }
    }
    y[e] = a.m > 0 ? cv + (kQjl / (float)a.m) * gamma * acc : cv;  // m = 0: no QJL stage
  }
  float x[E];
  if (a.rot == TQ_ROT_HADAMARD) {
    // Pi^T = diag(sigma) H / sqrt(d) (H is symmetric).
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = y[e];
    fwht_warp<E>(x, lane);
    const uint32_t sb = a.cb.sign_bits[(lane * E) / 32] >> ((lane * E) % 32);
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = flip_sign(x[e] * a.inv_sqrt_d, (sb >> e) & 1u);
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) ybuf[lane * E + e] = y[e];
    __syncwarp();
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = 0.f;
    for (int r = 0; r < D; ++r) {
      const float yr = ybuf[r];
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = fmaf(a.Pi[(size_t)r * D + lane * E + e], yr, x[e]);
    }
    __syncwarp();
  }
#pragma unroll
  for (int e = 0; e < E; ++e) a.k_out[i * D + lane * E + e] = n * x[e];
}

template <int D>
__device__ void decompress_value(const DecompressArgs& a, int64_t i, int lane) {
  constexpr int E = D / 32;
  const int cwords = a.v_bits * D / 32;
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(a.v_codes) + i * cwords;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int j = lane * E + e, o = j * a.v_bits;
    uint32_t code = cw[o >> 5] >> (o & 31);
    if ((o & 31) + a.v_bits > 32) code |= cw[(o >> 5) + 1] << (32 - (o & 31));  // 3-bit codes straddle words
    code &= (1u << a.v_bits) - 1u;
    const uint32_t par = reinterpret_cast<const uint32_t*>(a.v_params)[i * (D / kVGroup) + j / kVGroup];
    const float sc = __half2float(__ushort_as_half((unsigned short)(par & 0xffffu)));
    const float lo = __half2float(__ushort_as_half((unsigned short)(par >> 16)));
    a.v_out[i * D + j] = fmaf(sc, (float)code, lo);
  }
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32) decompress_kernel(const __grid_constant__ DecompressArgs a) {
  __shared__ float ybuf[kWarps][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t i = (int64_t)blockIdx.x * kWarps + warp; i < a.n_vec; i += (int64_t)gridDim.x * kWarps) {
    if (a.k_out) decompress_key<D>(a, i, lane, ybuf[warp]);
    if (a.v_out) decompress_value<D>(a, i, lane);
  }
}

}  // namespace

cudaError_t launch_decompress(const tq_ctx* ctx, const uint8_t* k_codes, const uint8_t* k_signs,
                              const uint16_t* k_norms, const uint8_t* v_codes, const uint16_t* v_params,
                              int64_t n_vec, float* k_out, float* v_out, cudaStream_t stream) {
  DecompressArgs a;
  a.k_codes = k_codes;
  a.k_signs = k_signs;
  a.k_norms = k_norms;
  a.v_codes = v_codes;
  a.v_params = v_params;
  a.n_vec = n_vec;
  a.k_out = k_out;
  a.v_out = v_out;
  a.S = ctx->S;
  a.Pi = ctx->Pi;
  a.cb = ctx->cb;
  a.lm_bits = ctx->shape.lm_bits;
  a.m = ctx->shape.m;
  a.v_bits = ctx->shape.v_bits;
  a.rot = ctx->shape.rot;
  a.inv_sqrt_d = (float)(1.0 / sqrt((double)ctx->shape.d));
  int64_t blocks = (n_vec + kWarps - 1) / kWarps;
  if (blocks > (int64_t)ctx->num_sms * 16) blocks = (int64_t)ctx->num_sms * 16;
  switch (ctx->shape.d) {
    case 64: decompress_kernel<64><<<(unsigned)blocks, kWarps * 32, 0, stream>>>(a); break;
    case 128: decompress_kernel<128><<<(unsigned)blocks, kWarps * 32, 0, stream>>>(a); break;
    case 256: decompress_kernel<256><<<(unsigned)blocks, kWarps * 32, 0, stream>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace tq
