// Key/value compression (prefill / append path).
//
// Keys (TurboQuantProd; "turboquant-pytorch" skill card, "Что делает"; discosf
// news item, "一句话看懂" steps 1-3): norm, rotation (sign flip + in-register
// Walsh-Hadamard butterflies, or a dense Haar matrix), Lloyd-Max bucketize,
// residual, 1-bit QJL signs of S r, bit packing, fp16 side info.
// Values (discosf step 4): min/max group quantization over 32 coordinates.
//
// One warp owns one vector; lane l holds coordinates [l*E, l*E+E), E = d/32, so
// every global load and store of a record is a contiguous warp-wide access.
#include <cuda_runtime.h>

#include "tq_device.cuh"

namespace tq {
namespace {

constexpr int kWarps = 8;

struct CompressArgs {
  const void* k;
  const void* v;
  int64_t n_vec;
  uint8_t* k_codes;
  uint8_t* k_signs;
  uint16_t* k_norms;
  uint8_t* v_codes;
  uint16_t* v_params;
  const float* St;   // [d][m]
  const float* PiT;  // [d][d], Haar only
  Codebook cb;
  int lm_bits, m, v_bits, rot;
  float inv_sqrt_d;  // 1/sqrt(d) rounded once from fp64
};

template <int D, typename T>
__device__ void compress_key(const CompressArgs& a, int64_t i, int lane, float* rbuf) {
  constexpr int E = D / 32;
  float x[E];
  load_lane<E>(static_cast<const T*>(a.k) + i * D, lane, x);

  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) ss = fmaf(x[e], x[e], ss);
  const float n = sqrtf(warp_sum(ss));

  const int cbytes = a.lm_bits * D / 8;
  uint32_t* codes_out = reinterpret_cast<uint32_t*>(a.k_codes + i * cbytes);
  uint32_t* signs_out = reinterpret_cast<uint32_t*>(a.k_signs + i * (a.m / 8));
  if (n == 0.f) {  // a zero key is stored as zero bytes
    if (lane < cbytes / 4) codes_out[lane] = 0u;
    if (lane < a.m / 32) signs_out[lane] = 0u;
    if (lane == 0) reinterpret_cast<uint32_t*>(a.k_norms)[i] = 0u;
    return;
  }
  const float inv_n = 1.0f / n;

  float y[E];
  if (a.rot == TQ_ROT_HADAMARD) {
    const uint32_t sb = a.cb.sign_bits[(lane * E) / 32] >> ((lane * E) % 32);
#pragma unroll
    for (int e = 0; e < E; ++e) y[e] = flip_sign(x[e] * inv_n, (sb >> e) & 1u);
    fwht_warp<E>(y, lane);
#pragma unroll
    for (int e = 0; e < E; ++e) y[e] *= a.inv_sqrt_d;
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) rbuf[lane * E + e] = x[e] * inv_n;
    __syncwarp();
#pragma unroll
    for (int e = 0; e < E; ++e) y[e] = 0.f;
    for (int j = 0; j < D; ++j) {
      const float uj = rbuf[j];
      const float* row = a.PiT + (size_t)j * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) y[e] = fmaf(__ldg(row + e), uj, y[e]);
    }
    __syncwarp();
  }

  // Lloyd-Max bucketize: code = #{k : y >= t_k}; residual against its centroid.
  uint32_t code_bits = 0;
  float r[E];
  float rr = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    uint32_t idx = 0;
    float cv = a.cb.c[0];
#pragma unroll
    for (int k = 0; k < kMaxLevels - 1; ++k) {
      if (k + 1 < a.cb.levels && y[e] >= a.cb.t[k]) {
        idx = k + 1;
        cv = a.cb.c[k + 1];
      }
    }
    code_bits |= idx << (e * a.lm_bits);
    r[e] = y[e] - cv;
    rr = fmaf(r[e], r[e], rr);
  }
  const float gamma = sqrtf(warp_sum(rr));

  // QJL: sign bits of S r; lane computes rows i = lane + 32*q so a ballot gives word q.
#pragma unroll
  for (int e = 0; e < E; ++e) rbuf[lane * E + e] = r[e];
  __syncwarp();
  uint32_t my_sign_word = 0;
  for (int q = 0; q < a.m / 32; ++q) {
    float acc = 0.f;
    const float* col = a.St + lane + 32 * q;
    for (int j = 0; j < D; ++j) acc = fmaf(__ldg(col + (size_t)j * a.m), rbuf[j], acc);
    const uint32_t word = __ballot_sync(kFull, acc >= 0.f);
    if (lane == q) my_sign_word = word;
  }
  __syncwarp();

  const uint32_t code_word = pack_stream_word(code_bits, E * a.lm_bits, cbytes / 4, lane);
  if (lane < cbytes / 4) codes_out[lane] = code_word;
  if (lane < a.m / 32) signs_out[lane] = my_sign_word;
  if (lane == 0) {
    const uint32_t nb = __half_as_ushort(__float2half_rn(n));
    const uint32_t gb = __half_as_ushort(__float2half_rn(gamma));
    reinterpret_cast<uint32_t*>(a.k_norms)[i] = nb | (gb << 16);
  }
}

template <int D, typename T>
__device__ void compress_value(const CompressArgs& a, int64_t i, int lane) {
  constexpr int E = D / 32;
  constexpr int W = 32 / E;  // lanes per group of 32 coordinates
  float x[E];
  load_lane<E>(static_cast<const T*>(a.v) + i * D, lane, x);
  float lo = x[0], hi = x[0];
#pragma unroll
  for (int e = 1; e < E; ++e) {
    lo = fminf(lo, x[e]);
    hi = fmaxf(hi, x[e]);
  }
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(kFull, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(kFull, hi, o));
  }
  const int levels = (1 << a.v_bits) - 1;
  // Code arithmetic in fp64 so decisions match the exact quantizer except within
  // a few fp64 ulps of a half-step.
  const double dlo = lo, span = (double)hi - dlo;
  const double scale = span / levels;
  const double inv = span > 0.0 ? levels / span : 0.0;
  uint32_t code_bits = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    double q = floor(((double)x[e] - dlo) * inv + 0.5);
    q = fmin(fmax(q, 0.0), (double)levels);
    code_bits |= (uint32_t)q << (e * a.v_bits);
  }
  const int cbytes = a.v_bits * D / 8;
  const uint32_t word = pack_stream_word(code_bits, E * a.v_bits, cbytes / 4, lane);
  if (lane < cbytes / 4) reinterpret_cast<uint32_t*>(a.v_codes + i * cbytes)[lane] = word;
  if ((lane % W) == 0) {
    const uint32_t sb = __half_as_ushort(__double2half(scale));
    const uint32_t mb = __half_as_ushort(__float2half_rn(lo));
    reinterpret_cast<uint32_t*>(a.v_params)[i * (D / kVGroup) + lane / W] = sb | (mb << 16);
  }
}

template <int D, typename T>
__global__ void __launch_bounds__(kWarps * 32) compress_kernel(const __grid_constant__ CompressArgs a) {
  __shared__ float rbuf[kWarps][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t i = (int64_t)blockIdx.x * kWarps + warp; i < a.n_vec; i += (int64_t)gridDim.x * kWarps) {
    if (a.k) compress_key<D, T>(a, i, lane, rbuf[warp]);
    if (a.v) compress_value<D, T>(a, i, lane);
  }
}

template <int D>
cudaError_t launch_d(const tq_ctx* ctx, const CompressArgs& a, int dtype, cudaStream_t s) {
  int64_t blocks = (a.n_vec + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)ctx->num_sms * 16;
  if (blocks > cap) blocks = cap;
  if (ctx->prof_start) cudaEventRecord(ctx->prof_start, s);
  if (dtype == TQ_F32)
    compress_kernel<D, float><<<(unsigned)blocks, kWarps * 32, 0, s>>>(a);
  else
    compress_kernel<D, __nv_bfloat16><<<(unsigned)blocks, kWarps * 32, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (ctx->prof_stop) cudaEventRecord(ctx->prof_stop, s);
  return e;
}

}  // namespace

cudaError_t launch_compress(const tq_ctx* ctx, const void* k, const void* v, int dtype, int64_t n_vec,
                            uint8_t* k_codes, uint8_t* k_signs, uint16_t* k_norms, uint8_t* v_codes,
                            uint16_t* v_params, cudaStream_t stream) {
  CompressArgs a;
  a.k = k;
  a.v = v;
  a.n_vec = n_vec;
  a.k_codes = k_codes;
  a.k_signs = k_signs;
  a.k_norms = k_norms;
  a.v_codes = v_codes;
  a.v_params = v_params;
  a.St = ctx->St;
  a.PiT = ctx->PiT;
  a.cb = ctx->cb;
  a.lm_bits = ctx->shape.lm_bits;
  a.m = ctx->shape.m;
  a.v_bits = ctx->shape.v_bits;
  a.rot = ctx->shape.rot;
  a.inv_sqrt_d = (float)(1.0 / sqrt((double)ctx->shape.d));
  switch (ctx->shape.d) {
    case 64: return launch_d<64>(ctx, a, dtype, stream);
    case 128: return launch_d<128>(ctx, a, dtype, stream);
    case 256: return launch_d<256>(ctx, a, dtype, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tq
