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
#include <cuda.h>  // CUtensorMap and its enums (types only: the encoder is fetched at run time)
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <vector>

#include "tq_device.cuh"
#include "tq_sm100.cuh"

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
  const uint16_t* S_sw128;  // S as f16 in the swizzled K-major operand layout (tensor-core path)
  const uint16_t* H_sw128;  // H diag(sigma) as bf16 in the same layout (tensor-core rotation)
  unsigned int* err;
  Codebook cb;
  int lm_bits, m, v_bits, rot;
  float inv_sqrt_d;  // 1/sqrt(d) rounded once from fp64
  const int64_t* slot;  // output row of each input vector (null: row i), each in [0, n_rows)
  int64_t n_rows;       // rows the output arrays hold (slot mode)
  CUtensorMap kmap;  // compress_pipe_kernel: bf16 keys [n_vec][128], 64 x 128 boxes, 128-byte swizzle
  CUtensorMap vmap;  // compress_pipe_kernel: bf16 values [n_vec][128], 64 x 64 boxes, 128-byte swizzle
};

// Output row of input vector i: slot[i] when a slot map is given, else i. A slot outside
// [0, n_rows) sets bit 2 of the error word and gives -1: that vector is not written.
__device__ __forceinline__ int64_t out_row(const CompressArgs& a, int64_t i) {
  if (!a.slot) return i;
  const int64_t o = __ldg(a.slot + i);
  if (o < 0 || o >= a.n_rows) {
    atomicOr(a.err, 4u);
    return -1;
  }
  return o;
}

// Norm, rotation, Lloyd-Max codes and residual of key i; writes the packed codes
// and (n, gamma). Returns false for a zero key (all its bytes already written as 0);
// otherwise leaves the lane's residual coordinates in r.
template <int D, typename T, int LMB = 0>
__device__ bool key_front(const CompressArgs& a, int64_t i, int64_t o, int lane, float* rbuf, float (&r)[D / 32]) {
  constexpr int E = D / 32;
  const int lmb = LMB ? LMB : a.lm_bits;       // compile-time when specialised
  const int levels = LMB ? (1 << LMB) : a.cb.levels;
  float x[E];
  load_lane<E>(static_cast<const T*>(a.k) + i * D, lane, x);

  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) ss = fmaf(x[e], x[e], ss);
  const float n = sqrtf(warp_sum(ss));

  const int cbytes = lmb * D / 8;
  uint32_t* codes_out = reinterpret_cast<uint32_t*>(a.k_codes + o * cbytes);
  uint32_t* signs_out = reinterpret_cast<uint32_t*>(a.k_signs + o * (a.m / 8));
  if (n == 0.f) {  // a zero key is stored as zero bytes
    if (lane < cbytes / 4) codes_out[lane] = 0u;
    if (lane < a.m / 32) signs_out[lane] = 0u;
    if (lane == 0) reinterpret_cast<uint32_t*>(a.k_norms)[o] = 0u;
    return false;
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
  float rr = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    uint32_t idx = 0;
    float cv;
    if constexpr (LMB == 0) {
      // any width: binary search for #{k : y >= t_k} over the power-of-two level count
      for (int s = levels >> 1; s > 0; s >>= 1)
        if (y[e] >= a.cb.t[idx + s - 1]) idx += s;
      cv = a.cb.c[idx];
    } else {
      cv = a.cb.c[0];
#pragma unroll
      for (int k = 0; k < (1 << LMB) - 1; ++k) {
        if (y[e] >= a.cb.t[k]) {
          idx = k + 1;
          cv = a.cb.c[k + 1];
        }
      }
    }
    code_bits |= idx << (e * lmb);
    r[e] = y[e] - cv;
    rr = fmaf(r[e], r[e], rr);
  }
  const float gamma = sqrtf(warp_sum(rr));
  const uint32_t code_word = LMB ? pack_stream_word_t<E * LMB, LMB * D / 32>(code_bits, lane)
                                 : pack_stream_word(code_bits, E * lmb, cbytes / 4, lane);
  if (lane < cbytes / 4) codes_out[lane] = code_word;
  if (lane == 0) {
    const uint32_t nb = __half_as_ushort(__float2half_rn(n));
    const uint32_t gb = __half_as_ushort(__float2half_rn(gamma));
    reinterpret_cast<uint32_t*>(a.k_norms)[o] = nb | (gb << 16);
  }
  return true;
}

template <int D, typename T>
__device__ void compress_key(const CompressArgs& a, int64_t i, int lane, float* rbuf) {
  constexpr int E = D / 32;
  float r[E];
  const int64_t o = out_row(a, i);  // the same in every lane
  if (o < 0 || !key_front<D, T>(a, i, o, lane, rbuf, r)) return;
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
  if (lane < a.m / 32) reinterpret_cast<uint32_t*>(a.k_signs + o * (a.m / 8))[lane] = my_sign_word;
}

template <int D, typename T, int VB = 0>
__device__ void compress_value(const CompressArgs& a, int64_t i, int lane) {
  constexpr int E = D / 32;
  constexpr int W = 32 / E;  // lanes per group of 32 coordinates
  const int vbits = VB ? VB : a.v_bits;
  const int64_t o = out_row(a, i);  // the same in every lane
  if (o < 0) return;
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
  const int levels = (1 << vbits) - 1;
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
    code_bits |= (uint32_t)q << (e * vbits);
  }
  const int cbytes = vbits * D / 8;
  const uint32_t word = VB ? pack_stream_word_t<E * VB, VB * D / 32>(code_bits, lane)
                           : pack_stream_word(code_bits, E * vbits, cbytes / 4, lane);
  if (lane < cbytes / 4) reinterpret_cast<uint32_t*>(a.v_codes + o * cbytes)[lane] = word;
  if ((lane % W) == 0) {
    const uint32_t sb = __half_as_ushort(__double2half(scale));
    const uint32_t mb = __half_as_ushort(__float2half_rn(lo));
    reinterpret_cast<uint32_t*>(a.v_params)[o * (D / kVGroup) + lane / W] = sb | (mb << 16);
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

// ---------------------------------------------------------------------------------
// Tensor-core variant (d = m = 128): the QJL projection S r of 128 keys at a time is
// one 128 x 128 x 128 MMA on the 5th-generation tensor cores. Warps 0-3 rotate and
// quantize the keys (one key per warp step, as above) and write the residuals,
// scaled by 16 and split into f16 hi + lo, to two swizzled shared-memory operand
// tiles; one thread issues 3 x 8 tcgen05.mma (residual hi and lo against S hi, residual
// hi against S lo, S being split in two f16 terms like the residual) into a 128 x 128
// fp32 accumulator in tensor memory; after
// the commit barrier each thread reads its key's 128 projections back and packs the
// sign bits. Warps 4-7 group-quantize the values of the same tile meanwhile.
constexpr int kTcRows = 128;
constexpr int kTcThreads = 256;
constexpr uint32_t kTcTileBytes = kTcRows * 128 * 2;  // one f16 operand tile, 32 KB

struct TcSmem {
  static constexpr uint32_t A_HI = 0, A_LO = kTcTileBytes, S = 2 * kTcTileBytes;  // S: hi tile, then lo tile
  static constexpr uint32_t RBUF = 4 * kTcTileBytes;         // [4 warps][128] fp32
  static constexpr uint32_t ZF = RBUF + 4 * 128 * 4;         // [128] nonzero flags
  static constexpr uint32_t BAR = ZF + 128;                  // mbarrier
  static constexpr uint32_t TMEM = BAR + 8;                  // TMEM base address
  static constexpr uint32_t BYTES = TMEM + 8;
};

__device__ __forceinline__ bool kwarps_sync_or(bool v) {
  // barrier 1 over the 128 key threads (warps 0-3), OR-reduced predicate
  uint32_t r;
  asm volatile(
      "{ .reg .pred p, q; setp.ne.u32 p, %1, 0; barrier.red.or.pred q, 1, 128, p; selp.u32 %0, 1, 0, q; }"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

template <typename T, int LMB, int VB>
__global__ void __launch_bounds__(kTcThreads, 1) compress_tc_kernel(const __grid_constant__ CompressArgs a) {
  namespace s1 = tq::sm100;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = s1::smem_u32(sm);
  float* rbuf = reinterpret_cast<float*>(sm + TcSmem::RBUF);
  uint8_t* zf = sm + TcSmem::ZF;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + TcSmem::BAR);
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(sm + TcSmem::TMEM);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (warp == 0) {
    s1::tmem_alloc(tmem_s, 128);
    s1::tmem_relinquish();
  }
  if (tid == 0) {
    s1::mbar_init(bar, 1);
    s1::mbar_init_fence();
  }
  {  // S operand tiles (hi, lo), prepacked on the host
    const uint4* src = reinterpret_cast<const uint4*>(a.S_sw128);
    uint4* dst = reinterpret_cast<uint4*>(sm + TcSmem::S);
    for (int w = tid; w < (int)(2 * kTcTileBytes / 16); w += kTcThreads) dst[w] = src[w];
  }
  s1::fence_async_smem();
  s1::fence_before_sync();
  __syncthreads();
  s1::fence_after_sync();
  const uint32_t tmem = *tmem_s;
  constexpr uint32_t idesc = s1::idesc_f16_f32(128, 128);

  uint32_t phase = 0;
  bool failed = false;
  const int64_t ntile = (a.n_vec + kTcRows - 1) / kTcRows;
  for (int64_t tile = blockIdx.x; tile < ntile; tile += gridDim.x) {
    const int64_t v0 = tile * kTcRows;
    const int nrows = (int)min((int64_t)kTcRows, a.n_vec - v0);
    if (warp < 4) {
      if (a.k) {
        for (int vv = 0; vv < 32; ++vv) {
          const int row = warp * 32 + vv;
          if (row >= nrows) break;
          float r[4] = {0.f, 0.f, 0.f, 0.f};
          const int64_t o = out_row(a, v0 + row);  // the same in every lane
          const bool nz = o >= 0 && key_front<128, T, LMB>(a, v0 + row, o, lane, rbuf + warp * 128, r);
          // residual coordinates 4 lane .. 4 lane + 3, scaled by 16 (signs unchanged)
          float x[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) x[e] = nz ? 16.f * r[e] : 0.f;
          const __half2 h01 = __floats2half2_rn(x[0], x[1]), h23 = __floats2half2_rn(x[2], x[3]);
          const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
          const __half2 l01 = __floats2half2_rn(x[0] - f01.x, x[1] - f01.y);
          const __half2 l23 = __floats2half2_rn(x[2] - f23.x, x[3] - f23.y);
          const uint32_t off = s1::sw128_offset(row, 4 * lane, kTcRows);
          uint2 hv, lv;
          hv.x = *reinterpret_cast<const uint32_t*>(&h01);
          hv.y = *reinterpret_cast<const uint32_t*>(&h23);
          lv.x = *reinterpret_cast<const uint32_t*>(&l01);
          lv.y = *reinterpret_cast<const uint32_t*>(&l23);
          *reinterpret_cast<uint2*>(sm + TcSmem::A_HI + off) = hv;
          *reinterpret_cast<uint2*>(sm + TcSmem::A_LO + off) = lv;
          if (lane == 0) zf[row] = nz ? 1 : 0;
        }
        s1::fence_async_smem();
        s1::fence_before_sync();
        kwarps_sync_or(false);
        s1::fence_after_sync();
        if (tid == 0) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            s1::umma_f16(tmem, s1::sw128_desc(sbase + TcSmem::A_HI, 16 * ks, kTcRows),
                         s1::sw128_desc(sbase + TcSmem::S, 16 * ks, 128), idesc, ks > 0 ? 1u : 0u);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            s1::umma_f16(tmem, s1::sw128_desc(sbase + TcSmem::A_LO, 16 * ks, kTcRows),
                         s1::sw128_desc(sbase + TcSmem::S, 16 * ks, 128), idesc, 1u);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            s1::umma_f16(tmem, s1::sw128_desc(sbase + TcSmem::A_HI, 16 * ks, kTcRows),
                         s1::sw128_desc(sbase + TcSmem::S + kTcTileBytes, 16 * ks, 128), idesc, 1u);
          s1::umma_commit(bar);
        }
        const bool ok = s1::mbar_wait(bar, phase);
        phase ^= 1u;
        if (kwarps_sync_or(!ok)) {
          failed = true;
          break;
        }
        s1::fence_after_sync();
        // thread = key (TMEM lane 32 warp + lane); 4 x 32 projections -> 4 sign words
        uint32_t words[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t v[32];
          s1::tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + 32 * q, v);
          s1::tmem_ld_wait();
          uint32_t bits = 0;
#pragma unroll
          for (int k = 0; k < 32; ++k) bits |= (__uint_as_float(v[k]) >= 0.f ? 1u : 0u) << k;
          words[q] = bits;
        }
        const int row = 32 * warp + lane;
        const int64_t so = row < nrows ? out_row(a, v0 + row) : -1;
        if (so >= 0) {
          const bool nz = zf[row] != 0;
          uint4 w4 = nz ? make_uint4(words[0], words[1], words[2], words[3]) : make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(a.k_signs + so * 16) = w4;
        }
        s1::fence_before_sync();
        kwarps_sync_or(false);  // TMEM and the operand tiles are free for the next tile
      }
    } else if (a.v) {
      for (int vv = 0; vv < 32; ++vv) {
        const int row = (warp - 4) * 32 + vv;
        if (row >= nrows) break;
        compress_value<128, T, VB>(a, v0 + row, lane);
      }
    }
  }
  if (failed && tid == 0) {
    atomicOr(a.err, 1u);
    s1::mbar_wait(bar, phase ^ 1u);  // bounded: let the abandoned MMA finish before TMEM is freed
  }
  s1::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    s1::fence_after_sync();
    s1::tmem_dealloc(tmem, 128);
  }
}

template <typename T, int LMB, int VB>
cudaError_t launch_tc_t(const tq_ctx* ctx, const CompressArgs& a, cudaStream_t s) {
  static bool configured = false;
  const size_t smem = TcSmem::BYTES + 1024;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(compress_tc_kernel<T, LMB, VB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  int64_t blocks = (a.n_vec + kTcRows - 1) / kTcRows;
  if (blocks > ctx->num_sms) blocks = ctx->num_sms;
  if (ctx->prof_start) cudaEventRecord(ctx->prof_start, s);
  compress_tc_kernel<T, LMB, VB><<<(unsigned)blocks, kTcThreads, smem, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (ctx->prof_stop) cudaEventRecord(ctx->prof_stop, s);
  return e;
}

template <typename T>
cudaError_t launch_tc(const tq_ctx* ctx, const CompressArgs& a, cudaStream_t s) {
  const int lmb = ctx->shape.lm_bits, vb = ctx->shape.v_bits;
  if (lmb == 1) return vb == 2 ? launch_tc_t<T, 1, 2>(ctx, a, s) : launch_tc_t<T, 1, 4>(ctx, a, s);
  if (lmb == 2) return vb == 2 ? launch_tc_t<T, 2, 2>(ctx, a, s) : launch_tc_t<T, 2, 4>(ctx, a, s);
  return vb == 2 ? launch_tc_t<T, 3, 2>(ctx, a, s) : launch_tc_t<T, 3, 4>(ctx, a, s);
}


// ---------------------------------------------------------------------------------
// Fast path (d = m = 128, randomized Hadamard rotation): four lanes
// per vector, lane q of a vector holding coordinates [32q, 32q + 32). Norm, sign flip,
// the first five Walsh-Hadamard stages, bucketize, residual and code packing are
// lane-local; the last two butterfly stages and the two norms take two shuffles
// each. A value's group of 32 coordinates is one lane, so min / max and its codes
// need no shuffles at all. 512 threads handle 128 vectors at a time: the 128
// residuals (x16, f16 hi + lo) go to two swizzled shared-memory tiles, one thread
// issues the 128 x 128 x 128 QJL projection on the tensor cores (as in
// compress_tc_kernel), the values are quantized while it runs, and one thread per key
// reads its 128 projections back from tensor memory and packs the sign bits.
constexpr int kQ4Rows = 128;
constexpr int kQ4Threads = 4 * kQ4Rows;

struct Q4Smem {
  static constexpr uint32_t A_HI = 0, A_LO = kTcTileBytes, S = 2 * kTcTileBytes;  // S: hi tile, then lo tile
  static constexpr uint32_t ZF = 4 * kTcTileBytes;  // [128] nonzero-key flags
  static constexpr uint32_t BAR = ZF + 128;         // mbarrier
  static constexpr uint32_t TMEM = BAR + 8;         // TMEM base address
  static constexpr uint32_t BYTES = TMEM + 8;
};

// 32 consecutive elements (64 or 128 bytes, 16-byte aligned) as fp32.
template <typename T>
__device__ __forceinline__ void load32(const T* __restrict__ p, float (&x)[32]) {
  if constexpr (sizeof(T) == 2) {
    const uint4* p4 = reinterpret_cast<const uint4*>(p);
    uint4 u[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) u[k] = __ldg(p4 + k);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t w[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        x[8 * k + 2 * h] = __uint_as_float(w[h] << 16);
        x[8 * k + 2 * h + 1] = __uint_as_float(w[h] & 0xffff0000u);
      }
    }
  } else {
    const float4* p4 = reinterpret_cast<const float4*>(p);
    float4 f[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) f[k] = __ldg(p4 + k);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      x[4 * k] = f[k].x;
      x[4 * k + 1] = f[k].y;
      x[4 * k + 2] = f[k].z;
      x[4 * k + 3] = f[k].w;
    }
  }
}

// Unnormalised Sylvester Walsh-Hadamard transform of 32 values held by one thread.
__device__ __forceinline__ void fwht32(float (&x)[32]) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      if ((e & h) == 0) {
        const float u = x[e], w = x[e + h];
        x[e] = u + w;
        x[e + h] = u - w;
      }
    }
  }
}

// OR `v` (NB bits) into a little-endian stream of 32-bit words at bit `o` (o and
// NB compile-time after unrolling).
template <int NB, int NW>
__device__ __forceinline__ void put_bits(uint32_t (&w)[NW], int o, uint32_t v) {
  const int wi = o >> 5, sh = o & 31;
  w[wi] += v << sh;  // the bits are still zero: add == or
  if (sh + NB > 32) w[wi + 1] += v >> (32 - sh);
}

template <typename T, int LMB, int VB>
__global__ void __launch_bounds__(kQ4Threads, 1) compress_q4_kernel(const __grid_constant__ CompressArgs a) {
  namespace s1 = tq::sm100;
  constexpr int KW = LMB;  // code words per lane (32 codes x LMB bits)
  constexpr int VW = VB;   // value code words per lane
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = s1::smem_u32(sm);
  uint8_t* zf = sm + Q4Smem::ZF;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Q4Smem::BAR);
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(sm + Q4Smem::TMEM);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int R = tid >> 2, q = tid & 3;  // vector row within the pass, quarter of the vector

  if (warp == 0) {
    s1::tmem_alloc(tmem_s, 128);
    s1::tmem_relinquish();
  }
  if (tid == 0) {
    s1::mbar_init(bar, 1);
    s1::mbar_init_fence();
  }
  if (a.k) {  // S operand tile, prepacked on the host
    const uint4* src = reinterpret_cast<const uint4*>(a.S_sw128);
    uint4* dst = reinterpret_cast<uint4*>(sm + Q4Smem::S);
    for (int w = tid; w < (int)(2 * kTcTileBytes / 16); w += kQ4Threads) dst[w] = src[w];
  }
  s1::fence_async_smem();
  s1::fence_before_sync();
  __syncthreads();
  s1::fence_after_sync();
  const uint32_t tmem = *tmem_s;
  constexpr uint32_t idesc = s1::idesc_f16_f32(128, 128);

  const uint32_t sbits = a.cb.sign_bits[q];   // Hadamard signs of this lane's coordinates
  const float up1 = (q & 1) ? -1.f : 1.f;     // butterfly across lanes q ^ 1 (stride 32)
  const float up2 = (q & 2) ? -1.f : 1.f;     // and across lanes q ^ 2 (stride 64)
  float cb_t[(1 << LMB) - 1], cb_c[1 << LMB];
#pragma unroll
  for (int k = 0; k < (1 << LMB) - 1; ++k) cb_t[k] = a.cb.t[k];
#pragma unroll
  for (int k = 0; k < (1 << LMB); ++k) cb_c[k] = a.cb.c[k];

  uint32_t phase = 0;
  bool failed = false;
  const int64_t ntile = (a.n_vec + kQ4Rows - 1) / kQ4Rows;
  for (int64_t tile = blockIdx.x; tile < ntile; tile += gridDim.x) {
    const int64_t i = tile * kQ4Rows + R;
    const bool valid = i < a.n_vec;
    const int64_t o = valid ? out_row(a, i) : -1;  // output row

    // The values' loads are issued first, so that they are in flight while the keys
    // are worked on (bf16: 4 x 16 bytes per lane).
    uint4 vraw[sizeof(T) == 2 ? 4 : 1];
    if constexpr (sizeof(T) == 2) {
      if (a.v && valid) {
        const uint4* p4 = reinterpret_cast<const uint4*>(static_cast<const T*>(a.v) + i * 128 + 32 * q);
#pragma unroll
        for (int k = 0; k < 4; ++k) vraw[k] = __ldg(p4 + k);
      }
    }

    // ---------------------------------------------------------------- keys
    if (a.k) {
      float x[32];
      if (valid) {
        load32<T>(static_cast<const T*>(a.k) + i * 128 + 32 * q, x);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = 0.f;
      }
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) ss = fmaf(x[e], x[e], ss);
      ss += __shfl_xor_sync(kFull, ss, 1);
      ss += __shfl_xor_sync(kFull, ss, 2);
      const float n = sqrtf(ss);
      const bool nz = n > 0.f;
      // y = H diag(sigma) (k / n) / sqrt(d): sign flip, butterflies, one scale at the end
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] = flip_sign(x[e], (sbits >> e) & 1u);
      fwht32(x);
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] = fmaf(up1, x[e], __shfl_xor_sync(kFull, x[e], 1));
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] = fmaf(up2, x[e], __shfl_xor_sync(kFull, x[e], 2));
      const float sc = nz ? (1.0f / n) * a.inv_sqrt_d : 0.f;
      // Lloyd-Max bucketize: code = #{k : y >= t_k}; residual against its centroid.
      uint32_t cw[KW];
#pragma unroll
      for (int w = 0; w < KW; ++w) cw[w] = 0u;
      float rr = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float y = x[e] * sc;
        uint32_t idx = 0;
        float cv = cb_c[0];
#pragma unroll
        for (int k = 0; k < (1 << LMB) - 1; ++k) {
          if (y >= cb_t[k]) {
            idx = k + 1;
            cv = cb_c[k + 1];
          }
        }
        put_bits<LMB, KW>(cw, LMB * e, idx);
        x[e] = y - cv;
        rr = fmaf(x[e], x[e], rr);
      }
      rr += __shfl_xor_sync(kFull, rr, 1);
      rr += __shfl_xor_sync(kFull, rr, 2);
      const float gamma = sqrtf(rr);
      if (o >= 0) {
        uint32_t* co = reinterpret_cast<uint32_t*>(a.k_codes + o * (LMB * 16) + q * (LMB * 4));
#pragma unroll
        for (int w = 0; w < KW; ++w) co[w] = nz ? cw[w] : 0u;
        if (q == 0) {
          const uint32_t nb = __half_as_ushort(__float2half_rn(n));
          const uint32_t gb = __half_as_ushort(__float2half_rn(gamma));
          reinterpret_cast<uint32_t*>(a.k_norms)[o] = nz ? (nb | (gb << 16)) : 0u;
        }
      }
      // Residual x16 (signs unchanged) as f16 hi + lo into the operand tiles (the
      // previous pass's projection is complete: every thread waited for it).
      const bool use = valid && nz;
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {  // 8 coordinates = one 16-byte chunk of each tile
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float f0 = use ? 16.f * x[8 * c8 + 2 * p] : 0.f, f1 = use ? 16.f * x[8 * c8 + 2 * p + 1] : 0.f;
          const __half2 h = __floats2half2_rn(f0, f1);
          const float2 hf = __half22float2(h);
          const __half2 l = __floats2half2_rn(f0 - hf.x, f1 - hf.y);
          hw[p] = *reinterpret_cast<const uint32_t*>(&h);
          lw[p] = *reinterpret_cast<const uint32_t*>(&l);
        }
        const uint32_t off = s1::sw128_offset(R, 32 * q + 8 * c8, kQ4Rows);
        *reinterpret_cast<uint4*>(sm + Q4Smem::A_HI + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(sm + Q4Smem::A_LO + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      if (q == 0) zf[R] = use ? 1 : 0;
      s1::fence_async_smem();
      s1::fence_before_sync();
      __syncthreads();
      s1::fence_after_sync();
      if (tid == 0) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          s1::umma_f16(tmem, s1::sw128_desc(sbase + Q4Smem::A_HI, 16 * ks, kQ4Rows),
                       s1::sw128_desc(sbase + Q4Smem::S, 16 * ks, 128), idesc, ks > 0 ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          s1::umma_f16(tmem, s1::sw128_desc(sbase + Q4Smem::A_LO, 16 * ks, kQ4Rows),
                       s1::sw128_desc(sbase + Q4Smem::S, 16 * ks, 128), idesc, 1u);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          s1::umma_f16(tmem, s1::sw128_desc(sbase + Q4Smem::A_HI, 16 * ks, kQ4Rows),
                       s1::sw128_desc(sbase + Q4Smem::S + kTcTileBytes, 16 * ks, 128), idesc, 1u);
        s1::umma_commit(bar);
      }
    }

    // ---------------------------------------------------------------- values
    if (a.v && o >= 0) {
      float x[32];
      if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t w[4] = {vraw[k].x, vraw[k].y, vraw[k].z, vraw[k].w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            x[8 * k + 2 * h] = __uint_as_float(w[h] << 16);
            x[8 * k + 2 * h + 1] = __uint_as_float(w[h] & 0xffff0000u);
          }
        }
      } else {
        load32<T>(static_cast<const T*>(a.v) + i * 128 + 32 * q, x);
      }
      float lo = x[0], hi = x[0];
#pragma unroll
      for (int e = 1; e < 32; ++e) {
        lo = fminf(lo, x[e]);
        hi = fmaxf(hi, x[e]);
      }
      constexpr int levels = (1 << VB) - 1;
      // scale in fp64 as the reference quantizer. Codes: t = (v - min) / scale in fp32,
      // rounded to nearest by adding 1.5 * 2^23 (t is in [0, levels]; the integer lands
      // in the low mantissa bits); within 1e-5 of a half step the decision is redone
      // in fp64 with the reference's floor(t + 1/2).
      const double dlo = lo, span = (double)hi - dlo;
      const float inv = span > 0.0 ? (float)(levels / span) : 0.f;
      uint32_t vw[VW];
#pragma unroll
      for (int w = 0; w < VW; ++w) vw[w] = 0u;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float t = (x[e] - lo) * inv;
        const float tr = t + 12582912.0f;
        uint32_t qv = __float_as_uint(tr) & 0xffu;
        if (fabsf(t - (tr - 12582912.0f)) > 0.5f - 1e-5f)
          qv = (uint32_t)floor(((double)x[e] - dlo) * (levels / span) + 0.5);
        qv = min(qv, (uint32_t)levels);
        put_bits<VB, VW>(vw, VB * e, qv);
      }
      uint32_t* vo = reinterpret_cast<uint32_t*>(a.v_codes + o * (VB * 16) + q * (VB * 4));
#pragma unroll
      for (int w = 0; w < VW; ++w) vo[w] = vw[w];
      const uint32_t sb = __half_as_ushort(__double2half(span / levels));
      const uint32_t mb = __half_as_ushort(__float2half_rn(lo));
      reinterpret_cast<uint32_t*>(a.v_params)[o * 4 + q] = sb | (mb << 16);
    }

    // ---------------------------------------------------------------- QJL signs
    if (a.k) {
      const bool ok = s1::mbar_wait(bar, phase);
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      phase ^= 1u;
      s1::fence_after_sync();
      if (warp < 4) {
        // thread = key (TMEM lane 32 warp + lane); 4 x 32 projections -> 4 sign words
        uint32_t words[4];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t v[32];
          s1::tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + 32 * c4, v);
          s1::tmem_ld_wait();
          uint32_t bits = 0;
#pragma unroll
          for (int k = 31; k >= 0; --k) bits = __funnelshift_l(v[k] ^ 0x80000000u, bits, 1);
          words[c4] = bits;
        }
        const int row = 32 * warp + lane;
        const int64_t ik = tile * kQ4Rows + row;
        const int64_t so = ik < a.n_vec ? out_row(a, ik) : -1;
        if (so >= 0) {
          const bool nzk = zf[row] != 0;
          const uint4 w4 = nzk ? make_uint4(words[0], words[1], words[2], words[3]) : make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(a.k_signs + so * 16) = w4;
        }
      }
      s1::fence_before_sync();
    }
  }
  if (failed && tid == 0) {
    atomicOr(a.err, 1u);
    s1::mbar_wait(bar, phase);  // bounded: let an abandoned MMA finish before TMEM is freed
  }
  s1::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    s1::fence_after_sync();
    s1::tmem_dealloc(tmem, 128);
  }
}

template <typename T, int LMB, int VB>
cudaError_t launch_q4_t(const tq_ctx* ctx, const CompressArgs& a, cudaStream_t s) {
  static bool configured = false;
  const size_t smem = Q4Smem::BYTES + 1024;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(compress_q4_kernel<T, LMB, VB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  int64_t blocks = (a.n_vec + kQ4Rows - 1) / kQ4Rows;
  if (blocks > ctx->num_sms) blocks = ctx->num_sms;
  if (ctx->prof_start) cudaEventRecord(ctx->prof_start, s);
  compress_q4_kernel<T, LMB, VB><<<(unsigned)blocks, kQ4Threads, smem, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (ctx->prof_stop) cudaEventRecord(ctx->prof_stop, s);
  return e;
}

template <typename T>
cudaError_t launch_q4(const tq_ctx* ctx, const CompressArgs& a, cudaStream_t s) {
  const int lmb = ctx->shape.lm_bits, vb = ctx->shape.v_bits;
  if (lmb == 1) return vb == 2 ? launch_q4_t<T, 1, 2>(ctx, a, s) : launch_q4_t<T, 1, 4>(ctx, a, s);
  if (lmb == 2) return vb == 2 ? launch_q4_t<T, 2, 2>(ctx, a, s) : launch_q4_t<T, 2, 4>(ctx, a, s);
  return vb == 2 ? launch_q4_t<T, 3, 2>(ctx, a, s) : launch_q4_t<T, 3, 4>(ctx, a, s);
}


// ---------------------------------------------------------------------------------
// bf16 keys, randomized Hadamard rotation, d = m = 128: the rotation runs on the
// tensor cores too. The keys are bf16 and H diag(sigma) is +-1, both exact in bf16, so
// Y = K (H diag(sigma))^T is one bf16 x bf16 -> fp32 MMA per 128 keys with exact
// products (fp32 sums, like the butterflies). As Pi = H diag(sigma) / sqrt(d) is
// orthogonal, ||k|| = ||Y|| / sqrt(d) and y = Pi k / ||k|| = Y / ||Y||: the norm comes
// out of Y as well. Eight key warps read Y back from tensor memory (a warp reaches
// the 32 lanes of its sub-partition, so two warps share each row, one per half of
// the columns), bucketize, pack the codes and stage the residual for the QJL MMA;
// eight value warps quantize the 128 values meanwhile.
constexpr int kRotThreads = 512;
constexpr int kRotKeyThreads = 256;

// Shared memory of compress_rot_kernel. The Haar rotation needs three bf16 tiles of Pi
// (its 24-bit split), so that variant loads keys and values straight from global
// memory instead of staging raw rows.
template <bool HAAR>
struct RotSmem {
  static constexpr uint32_t NT = HAAR ? 3 : 1;               // bf16 terms of the rotation
  static constexpr uint32_t KT = 0;                          // keys, bf16 operand tile
  static constexpr uint32_t HB = kTcTileBytes;               // rotation, NT bf16 operand tiles
  static constexpr uint32_t S = (1 + NT) * kTcTileBytes;     // QJL matrix, f16 hi and lo operand tiles
  static constexpr uint32_t KR = (3 + NT) * kTcTileBytes;    // Hadamard: next pass's raw key rows
  static constexpr uint32_t VR = (4 + NT) * kTcTileBytes;    // Hadamard: next pass's raw value rows
  static constexpr uint32_t XS = (HAAR ? 3 + NT : 5 + NT) * kTcTileBytes;  // [2][128] half-row sums
  static constexpr uint32_t ZF = XS + 2 * 128 * 4;           // [128] nonzero-key flags
  static constexpr uint32_t BAR = ZF + 128;                  // four mbarriers
  static constexpr uint32_t TMEM = BAR + 32;                 // TMEM base address
  static constexpr uint32_t BYTES = TMEM + 8;
  static_assert(BYTES + 1024 <= 227 * 1024, "compress_rot_kernel shared memory");
};

__device__ __forceinline__ void key_warps_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kRotKeyThreads) : "memory");
}

// Instruction descriptor, kind::f16 with bf16 operands, f32 accumulate, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return sm100::idesc_f16_f32(M, N) | (1u << 7) | (1u << 10);
}

template <int LMB, int VB, bool HAAR>
__global__ void __launch_bounds__(kRotThreads, 1) compress_rot_kernel(const __grid_constant__ CompressArgs a) {
  using RS = RotSmem<HAAR>;
  namespace s1 = tq::sm100;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = s1::smem_u32(sm);
  float* xs = reinterpret_cast<float*>(sm + RS::XS);
  uint8_t* zf = sm + RS::ZF;
  uint64_t* bar1 = reinterpret_cast<uint64_t*>(sm + RS::BAR);  // rotation MMA done
  uint64_t* bar2 = bar1 + 1;                                         // projection MMA done
  uint64_t* bar3 = bar1 + 2;                                         // raw key rows landed
  uint64_t* bar4 = bar1 + 3;                                         // raw value rows landed
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(sm + RS::TMEM);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool key_warp = warp < 8;
  const int sp = warp & 3, ch = (warp >> 2) & 1;  // key warps: sub-partition, column half
  const int R = 32 * sp + lane;                    // key warps: row = key within the pass

  if (warp == 0) {
    s1::tmem_alloc(tmem_s, 512);
    s1::tmem_relinquish();
  }
  if (tid == 0) {
    s1::mbar_init(bar1, 1);
    s1::mbar_init(bar2, 1);
    s1::mbar_init(bar3, 1);
    s1::mbar_init(bar4, 1);
    s1::mbar_init_fence();
  }
  {  // H diag(sigma) and S operand tiles, prepacked on the host
    const uint4* hsrc = reinterpret_cast<const uint4*>(a.H_sw128);
    const uint4* ssrc = reinterpret_cast<const uint4*>(a.S_sw128);
    uint4* hdst = reinterpret_cast<uint4*>(sm + RS::HB);
    uint4* sdst = reinterpret_cast<uint4*>(sm + RS::S);
    for (int w = tid; w < (int)(2 * kTcTileBytes / 16); w += kRotThreads) sdst[w] = ssrc[w];
    for (int w = tid; w < (int)(RS::NT * kTcTileBytes / 16); w += kRotThreads) hdst[w] = hsrc[w];
  }
  s1::fence_async_smem();
  s1::fence_before_sync();
  __syncthreads();
  s1::fence_after_sync();
  const uint32_t tmem = *tmem_s;
  // columns 0..127: Y, 128..255: S r, 256..383: the residual operand (hi: 64 columns of
  // f16 pairs, then lo)
  const uint32_t tmem_y = tmem, tmem_p = tmem + 128, tmem_a = tmem + 256;
  const uint32_t lane_base = (uint32_t)(32 * sp) << 16;
  float cb_t[(1 << LMB) - 1], cb_c[1 << LMB];
#pragma unroll
  for (int k = 0; k < (1 << LMB) - 1; ++k) cb_t[k] = a.cb.t[k];
#pragma unroll
  for (int k = 0; k < (1 << LMB); ++k) cb_c[k] = a.cb.c[k];

  uint32_t phase = 0;
  bool failed = false;
  const int64_t ntile = (a.n_vec + kQ4Rows - 1) / kQ4Rows;
  // One thread: bring the raw rows of pass `tile` (contiguous in memory) into KR.
  auto fetch_keys = [&](int64_t tile) {
    const int64_t v0 = tile * kQ4Rows;
    const uint32_t bytes = (uint32_t)(min((int64_t)kQ4Rows, a.n_vec - v0) * 256);
    s1::mbar_expect_tx(bar3, bytes);
    s1::bulk_g2s(sm + RS::KR, static_cast<const __nv_bfloat16*>(a.k) + v0 * 128, bytes, bar3);
  };
  // One thread: bring the raw value rows of pass `tile` into VR.
  auto fetch_vals = [&](int64_t tile) {
    const int64_t v0 = tile * kQ4Rows;
    const uint32_t bytes = (uint32_t)(min((int64_t)kQ4Rows, a.n_vec - v0) * 256);
    s1::mbar_expect_tx(bar4, bytes);
    s1::bulk_g2s(sm + RS::VR, static_cast<const __nv_bfloat16*>(a.v) + v0 * 128, bytes, bar4);
  };
  if (!HAAR && a.k && tid == 0 && blockIdx.x < ntile) fetch_keys(blockIdx.x);
  if (!HAAR && a.v && tid == 0 && blockIdx.x < ntile) fetch_vals(blockIdx.x);
  for (int64_t tile = blockIdx.x; tile < ntile; tile += gridDim.x, phase ^= 1u) {
    const int64_t v0 = tile * kQ4Rows;
    // ---- stage the 128 keys: raw rows -> swizzled operand tile, once they landed and
    // the previous pass's rotation MMA has finished reading the tile.
    if (a.k && tile != blockIdx.x && !failed && !s1::mbar_wait(bar1, phase ^ 1u)) failed = true;
    if (!HAAR && a.k && !failed && !s1::mbar_wait(bar3, phase)) failed = true;
    if (__syncthreads_or(failed)) break;
    if (a.k) {
      const int nrows = (int)min((int64_t)kQ4Rows, a.n_vec - v0);
      uint4 kv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int id = tid + kRotThreads * u, row = id >> 4;
        if constexpr (HAAR)
          kv[u] = row < nrows ? __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.k) + v0 * 128) + id)
                              : make_uint4(0u, 0u, 0u, 0u);
        else
          kv[u] = row < nrows ? reinterpret_cast<const uint4*>(sm + RS::KR)[id] : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int id = tid + kRotThreads * u, row = id >> 4, c16 = id & 15;
        *reinterpret_cast<uint4*>(sm + RS::KT + s1::sw128_offset(row, 8 * c16, kQ4Rows)) = kv[u];
      }
      s1::fence_async_smem();
      s1::fence_before_sync();
      __syncthreads();
      s1::fence_after_sync();
      if (tid == 0) {
        constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
#pragma unroll
        for (int t = 0; t < (int)RS::NT; ++t)
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            s1::umma_f16(tmem_y, s1::sw128_desc(sbase + RS::KT, 16 * ks, kQ4Rows),
                         s1::sw128_desc(sbase + RS::HB + t * kTcTileBytes, 16 * ks, 128), idesc,
                         (t > 0 || ks > 0) ? 1u : 0u);
        s1::umma_commit(bar1);
        // KR has been read by every thread (the barrier above): fetch the next pass.
        if (!HAAR && tile + gridDim.x < ntile) {
          s1::fence_async_smem();
          fetch_keys(tile + gridDim.x);
        }
      }
    }

    if (key_warp && a.k) {
      // ---------------------------------------------------------------- keys
      const int64_t i = v0 + R;
      const bool valid = i < a.n_vec;
      const int64_t o = valid ? out_row(a, i) : -1;  // output row
      if (!failed && !s1::mbar_wait(bar1, phase)) failed = true;
      s1::fence_after_sync();
      // Two 32-column chunks per thread: a first pass for the norm, a second one (a loop
      // that is not unrolled, to keep the code small) for codes, residual and operands.
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t v[32];
        s1::tmem_ld32(tmem_y + lane_base + 64 * ch + 32 * h, v);
        s1::tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float yv = __uint_as_float(v[e]);
          s4[e & 3] = fmaf(yv, yv, s4[e & 3]);
        }
      }
      xs[ch * 128 + R] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
      key_warps_sync();
      const float tot = xs[R] + xs[128 + R];  // ||Y||^2 = d ||k||^2 (Hadamard), ||k||^2 (Haar)
      key_warps_sync();                      // both halves read before xs is reused
      const bool nz = tot > 0.f;
      const float sc = nz ? 1.0f / sqrtf(tot) : 0.f;
      const bool use = valid && nz;
      constexpr int CW = LMB;  // code words of a 32-column chunk
      float r4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t v[32];
        s1::tmem_ld32(tmem_y + lane_base + 64 * ch + 32 * h, v);
        s1::tmem_ld_wait();
        uint32_t cw[CW], cw2[CW];  // even / odd codes: two independent insert chains per word
#pragma unroll
        for (int w = 0; w < CW; ++w) cw[w] = cw2[w] = 0u;
        float r[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float yy = __uint_as_float(v[e]) * sc;
          uint32_t idx = 0;
          float cv = cb_c[0];
#pragma unroll
          for (int k = 0; k < (1 << LMB) - 1; ++k) {
            if (yy >= cb_t[k]) {
              idx = k + 1;
              cv = cb_c[k + 1];
            }
          }
          if (e & 1)
            put_bits<LMB, CW>(cw2, LMB * e, idx);
          else
            put_bits<LMB, CW>(cw, LMB * e, idx);
          r[e] = yy - cv;
          r4[e & 3] = fmaf(r[e], r[e], r4[e & 3]);
        }
        if (o >= 0) {
          uint32_t* co = reinterpret_cast<uint32_t*>(a.k_codes + o * (LMB * 16) + ch * (LMB * 8) + h * (LMB * 4));
#pragma unroll
          for (int w = 0; w < CW; ++w) co[w] = nz ? (cw[w] | cw2[w]) : 0u;
        }
        // residual x16 as f16 hi + lo into tensor memory, row R, one f16 pair per column
        // (the previous projection finished: it was waited for)
#pragma unroll
        for (int c16 = 0; c16 < 2; ++c16) {
          uint32_t hw[8], lw[8];
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            const float f0 = use ? 16.f * r[16 * c16 + 2 * p] : 0.f, f1 = use ? 16.f * r[16 * c16 + 2 * p + 1] : 0.f;
            const __half2 hh = __floats2half2_rn(f0, f1);
            const float2 hf = __half22float2(hh);
            const __half2 ll = __floats2half2_rn(f0 - hf.x, f1 - hf.y);
            hw[p] = *reinterpret_cast<const uint32_t*>(&hh);
            lw[p] = *reinterpret_cast<const uint32_t*>(&ll);
          }
          const uint32_t col = 32 * ch + 16 * h + 8 * c16;  // coordinates 2 col .. 2 col + 15
          s1::tmem_st8(tmem_a + lane_base + col, hw);
          s1::tmem_st8(tmem_a + 64 + lane_base + col, lw);
        }
      }
      xs[ch * 128 + R] = (r4[0] + r4[1]) + (r4[2] + r4[3]);
      key_warps_sync();
      const float gamma = sqrtf(xs[R] + xs[128 + R]);
      if (o >= 0 && ch == 0) {
        const float n = HAAR ? sqrtf(tot) : sqrtf(tot * (1.0f / 128.f));
        const uint32_t nb = __half_as_ushort(__float2half_rn(n));
        const uint32_t gb = __half_as_ushort(__float2half_rn(gamma));
        reinterpret_cast<uint32_t*>(a.k_norms)[o] = nz ? (nb | (gb << 16)) : 0u;
      }
      if (ch == 0) zf[R] = use ? 1 : 0;
      s1::tmem_st_wait();
      s1::fence_before_sync();
      key_warps_sync();
      s1::fence_after_sync();
      if (tid == 0) {
        // S r = (A_hi + A_lo) S_hi^T + A_hi S_lo^T, A from tensor memory (the A_lo S_lo
        // term, about 2^-22 of the product, is left out)
        constexpr uint32_t idesc = s1::idesc_f16_f32(128, 128);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          s1::umma_f16_ts(tmem_p, tmem_a + 8 * ks, s1::sw128_desc(sbase + RS::S, 16 * ks, 128), idesc,
                          ks > 0 ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          s1::umma_f16_ts(tmem_p, tmem_a + 64 + 8 * ks, s1::sw128_desc(sbase + RS::S, 16 * ks, 128), idesc, 1u);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          s1::umma_f16_ts(tmem_p, tmem_a + 8 * ks, s1::sw128_desc(sbase + RS::S + kTcTileBytes, 16 * ks, 128),
                          idesc, 1u);
        s1::umma_commit(bar2);
      }
      // ---- QJL signs of this thread's 64 projections
      if (!failed && !s1::mbar_wait(bar2, phase)) failed = true;
      s1::fence_after_sync();
      const bool nzk = zf[R] != 0;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t v[32];
        s1::tmem_ld32(tmem_p + lane_base + 64 * ch + 32 * h, v);
        s1::tmem_ld_wait();
        uint32_t b4[4] = {0u, 0u, 0u, 0u};  // four independent 8-bit chains
#pragma unroll
        for (int k = 7; k >= 0; --k)
#pragma unroll
          for (int g = 0; g < 4; ++g) b4[g] = __funnelshift_l(v[8 * g + k] ^ 0x80000000u, b4[g], 1);
        const uint32_t word = b4[0] | (b4[1] << 8) | (b4[2] << 16) | (b4[3] << 24);
        if (o >= 0) reinterpret_cast<uint32_t*>(a.k_signs + o * 16 + 8 * ch)[h] = nzk ? word : 0u;
      }
      s1::fence_before_sync();
    } else if (!key_warp && a.v) {
      // ---------------------------------------------------------------- values
      const int vt = tid - kRotKeyThreads, q = vt & 3;
      // Hadamard: the pass's value rows were bulk-copied into VR one pass ahead.
      // Haar: both rounds' rows are loaded before either is worked on.
      uint4 raw[HAAR ? 2 : 1][4];
      if constexpr (HAAR) {
#pragma unroll
        for (int round = 0; round < 2; ++round) {
          const int64_t i = v0 + (vt >> 2) + 64 * round;
          if (i < a.n_vec) {
            const uint4* g4 = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.v) + i * 128 + 32 * q);
#pragma unroll
            for (int k = 0; k < 4; ++k) raw[round][k] = __ldg(g4 + k);
          }
        }
      } else {
        if (!failed && !s1::mbar_wait(bar4, phase)) failed = true;
      }
#pragma unroll(HAAR ? 2 : 1)
      for (int round = 0; round < 2; ++round) {
        const int row = (vt >> 2) + 64 * round;
        const int64_t i = v0 + row;
        if (i >= a.n_vec || failed) break;
        const int64_t o = out_row(a, i);
        if (o < 0) continue;
        float x[32];
        const uint4* p4 = reinterpret_cast<const uint4*>(sm + RS::VR + row * 256 + 64 * q);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 rv = HAAR ? raw[HAAR ? round : 0][k] : p4[k];
          const uint32_t w[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            x[8 * k + 2 * h] = __uint_as_float(w[h] << 16);
            x[8 * k + 2 * h + 1] = __uint_as_float(w[h] & 0xffff0000u);
          }
        }
        // min / max as four independent chains
        float lo4[4] = {x[0], x[1], x[2], x[3]}, hi4[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
        for (int e = 4; e < 32; ++e) {
          lo4[e & 3] = fminf(lo4[e & 3], x[e]);
          hi4[e & 3] = fmaxf(hi4[e & 3], x[e]);
        }
        const float lo = fminf(fminf(lo4[0], lo4[1]), fminf(lo4[2], lo4[3]));
        const float hi = fmaxf(fmaxf(hi4[0], hi4[1]), fmaxf(hi4[2], hi4[3]));
        constexpr int levels = (1 << VB) - 1;
        // scale in fp64 as the reference quantizer; codes rounded to nearest by adding
        // 1.5 * 2^23, redone in fp64 with floor(t + 1/2) within 1e-5 of a half step.
        const double dlo = lo, span = (double)hi - dlo;
        const float inv = span > 0.0 ? (float)(levels / span) : 0.f;
        uint32_t vw[VB], vw2[VB];  // even / odd codes: two independent insert chains per word
#pragma unroll
        for (int w = 0; w < VB; ++w) vw[w] = vw2[w] = 0u;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float t = (x[e] - lo) * inv;
          const float tr = t + 12582912.0f;
          uint32_t qv = __float_as_uint(tr) & 0xffu;
          if (fabsf(t - (tr - 12582912.0f)) > 0.5f - 1e-5f)
            qv = (uint32_t)floor(((double)x[e] - dlo) * (levels / span) + 0.5);
          qv = min(qv, (uint32_t)levels);
          if (e & 1)
            put_bits<VB, VB>(vw2, VB * e, qv);
          else
            put_bits<VB, VB>(vw, VB * e, qv);
        }
#pragma unroll
        for (int w = 0; w < VB; ++w) vw[w] |= vw2[w];
        uint32_t* vo = reinterpret_cast<uint32_t*>(a.v_codes + o * (VB * 16) + q * (VB * 4));
#pragma unroll
        for (int w = 0; w < VB; ++w) vo[w] = vw[w];
        const uint32_t sb = __half_as_ushort(__double2half(span / levels));
        const uint32_t mb = __half_as_ushort(__float2half_rn(lo));
        reinterpret_cast<uint32_t*>(a.v_params)[o * 4 + q] = sb | (mb << 16);
      }
      if constexpr (!HAAR) {
        // every value thread has read VR: fetch the next pass's values
        asm volatile("bar.sync 2, %0;" ::"n"(kRotThreads - kRotKeyThreads) : "memory");
        if (tid == kRotKeyThreads && tile + gridDim.x < ntile) {
          s1::fence_async_smem();
          fetch_vals(tile + gridDim.x);
        }
      }
    }
  }
  if (__syncthreads_or(failed) && tid == 0) {
    atomicOr(a.err, 1u);
    // bounded: let abandoned MMAs (the last ones issued completed phase ^ 1) finish
    // before TMEM is freed
    s1::mbar_wait(bar1, phase ^ 1u);
    s1::mbar_wait(bar2, phase ^ 1u);
    if (!HAAR) {
      s1::mbar_wait(bar3, phase);  // key / value fetches issued for the pass that never ran
      s1::mbar_wait(bar4, phase);
    }
  }
  s1::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    s1::fence_after_sync();
    s1::tmem_dealloc(tmem, 512);
  }
}

template <int LMB, int VB, bool HAAR>
cudaError_t launch_rot_t(const tq_ctx* ctx, const CompressArgs& a, cudaStream_t s) {
  static bool configured = false;
  const size_t smem = RotSmem<HAAR>::BYTES + 1024;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(compress_rot_kernel<LMB, VB, HAAR>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  int64_t blocks = (a.n_vec + kQ4Rows - 1) / kQ4Rows;
  if (blocks > ctx->num_sms) blocks = ctx->num_sms;
  if (ctx->prof_start) cudaEventRecord(ctx->prof_start, s);
  compress_rot_kernel<LMB, VB, HAAR><<<(unsigned)blocks, kRotThreads, smem, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (ctx->prof_stop) cudaEventRecord(ctx->prof_stop, s);
  return e;
}

template <bool HAAR>
cudaError_t launch_rot(const tq_ctx* ctx, const CompressArgs& a, cudaStream_t s) {
  const int lmb = ctx->shape.lm_bits, vb = ctx->shape.v_bits;
  if (lmb == 1) return vb == 2 ? launch_rot_t<1, 2, HAAR>(ctx, a, s) : launch_rot_t<1, 4, HAAR>(ctx, a, s);
  if (lmb == 2) return vb == 2 ? launch_rot_t<2, 2, HAAR>(ctx, a, s) : launch_rot_t<2, 4, HAAR>(ctx, a, s);
  return vb == 2 ? launch_rot_t<3, 2, HAAR>(ctx, a, s) : launch_rot_t<3, 4, HAAR>(ctx, a, s);
}

// ---------------------------------------------------------------------------------
// bf16 keys, randomized Hadamard rotation, d = m = 128, and a codebook symmetric about
// zero (c[L-1-k] = -c[k], t[L-2-k] = -t[k]; the sphere Lloyd-Max codebook is). The
// arithmetic is that of compress_rot_kernel; the organisation lets consecutive passes
// of 128 vectors overlap and keeps the tensor cores' shared-memory reads low:
//  * one producer thread (warp 16) issues every key TMA and every MMA, so that no
//    compute warp waits while the tensor core takes the instructions;
//  * the key rows arrive by TMA straight into one of two swizzled operand tiles, and the
//    rotation MMA of pass i+2 (into the half of a double-buffered Y in tensor memory
//    that pass i has just released) runs while the key warps work on pass i+1;
//  * the residual's f16 hi / lo operand goes to tensor memory (tcgen05.st), so the
//    projection MMA reads only S from shared memory; it runs while the key warps start
//    on the next pass, which reads its signs out before overwriting the operand;
//  * the value warps run a loop of their own over the same passes, with the value rows
//    in four half buffers (two passes of two halves; TMA, 128-byte swizzle, so that the
//    four threads of a row and the eight rows of a warp read distinct banks), each
//    refilled two passes ahead.
// Both threads of a key row compute ||Y||^2 over all 128 columns (no exchange); the
// residual's squared norm is exchanged through shared memory at the one key-warp
// barrier of a pass. With the symmetric codebook a coordinate is bucketized on its
// magnitude and the code's bits follow from its sign; everything is scaled by 16 (an
// exact power of two) so that the residual comes out as the x16 operand directly.
constexpr int kPipeThreads = 640;  // warps 0-7 keys, 8-15 values, 16 producer (17-19 idle)

// NT: bf16 terms of the rotation, 1 for H diag(sigma) (exact), 3 for the Haar matrix (about
// 24 bits; keys only: its tiles take the space of the value rows).
template <int NT>
struct PipeSmem {
  static constexpr uint32_t KT = 0;                         // [2] key operand tiles (TMA, 128B swizzle)
  static constexpr uint32_t HB = 2 * kTcTileBytes;          // the rotation, NT bf16 operand tiles
  static constexpr uint32_t S = (2 + NT) * kTcTileBytes;    // QJL matrix, f16 hi and lo operand tiles
  static constexpr uint32_t VR = (4 + NT) * kTcTileBytes;   // [2 passes][2 halves] value rows (NT = 1)
  static constexpr uint32_t XR = 7 * kTcTileBytes;          // [2 passes][128] second-half sums of r^2
  static constexpr uint32_t BAR = XR + 2 * 128 * 4;         // eleven mbarriers
  static constexpr uint32_t TMEM = BAR + 88;                // TMEM base address
  static constexpr uint32_t BYTES = TMEM + 8;
  static_assert(BYTES + 1024 <= 227 * 1024, "compress_pipe_kernel shared memory");
};
// Tensor memory (512 columns): Y[2] at 0 and 128, S r at 256, the residual operand at
// 384 (hi: 64 columns of f16 pairs, then lo).
constexpr uint32_t kTmY = 0, kTmP = 256, kTmA = 384;

// Adds the NB-bit field v at bit offset o of the words w (fields start zero, so add
// acts as or, and compiles to one integer multiply-add).
template <int NB, int NW>
__device__ __forceinline__ void add_field(uint32_t (&w)[NW], int o, uint32_t v) {
  const int wi = o >> 5, sh = o & 31;
  w[wi] += v << sh;
  if (sh + NB > 32) w[wi + 1] += v >> (32 - sh);
}

// Bucketize y (x16 domain) with a symmetric codebook: magnitude thresholds tm and
// levels cm (the upper half of t and c, x16). Returns the centroid and sets the code.
template <int LMB>
__device__ __forceinline__ float bucket_sym(float y, const float* tm, const float* cm, uint32_t& code) {
  constexpr int L = 1 << LMB, HL = L / 2;
  const float a = fabsf(y);
  uint32_t im = HL;
  float mag = cm[0];
#pragma unroll
  for (int j = 0; j < HL - 1; ++j) {
    if (a >= tm[j]) {
      im = HL + j + 1;
      mag = cm[j + 1];
    }
  }
  const uint32_t yb = __float_as_uint(y);
  const uint32_t neg = (uint32_t)((int32_t)yb >> 31);  // all ones for a negative y
  code = im ^ (neg & (uint32_t)(L - 1));               // lower half: L - 1 - im
  return __uint_as_float(__float_as_uint(mag) | (yb & 0x80000000u));
}

// span / L rounded to nearest in fp64 without a division (Markstein's correction step:
// q0 = span * RN(1/L) is within an ulp of the quotient, the remainder span - L q0 is exact
// with an FMA, and q0 + remainder * RN(1/L) rounds to the quotient).
template <int L>
__device__ __forceinline__ double div_levels(double span) {
  constexpr double inv = 1.0 / L;
  const double q0 = span * inv;
  return fma(fma(-(double)L, q0, span), inv, q0);
}

// QJL: the QJL stage is on (m = 128); without it (m = 0) the S tiles, the residual operand,
// the projection and the sign readout are left out, and gamma = ||r|| is stored as before.
template <int LMB, int VB, int NT, bool QJL>
__global__ void __launch_bounds__(kPipeThreads, 1) compress_pipe_kernel(const __grid_constant__ CompressArgs a) {
  using PS = PipeSmem<NT>;
  namespace s1 = tq::sm100;
  constexpr int L = 1 << LMB, HL = L / 2;
  extern __shared__ unsigned char smem_pipe[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(((uintptr_t)smem_pipe + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = s1::smem_u32(sm);
  float* xr = reinterpret_cast<float*>(sm + PS::XR);
  uint64_t* kfull = reinterpret_cast<uint64_t*>(sm + PS::BAR);  // [2] key tile landed
  uint64_t* rotd = kfull + 2;                                        // [2] rotation into Y[b] done
  uint64_t* projd = kfull + 4;                                       // projection done
  uint64_t* vfull = kfull + 5;                                       // [4] value half landed
  uint64_t* aready = kfull + 9;                                      // key warps done with a pass (8 arrivals)
  uint64_t* fin = kfull + 10;                                        // failure path: MMAs drained
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(sm + PS::TMEM);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t ntile = (a.n_vec + 127) / 128, g = gridDim.x;

  if (warp == 0) {
    s1::tmem_alloc(tmem_s, 512);
    s1::tmem_relinquish();
  }
  if (tid == 0) {
    for (int k = 0; k < 9; ++k) s1::mbar_init(kfull + k, 1);
    s1::mbar_init(aready, 8);
    s1::mbar_init(fin, 1);
    s1::mbar_init_fence();
  }
  {  // H diag(sigma) and S operand tiles, prepacked on the host
    const uint4* hsrc = reinterpret_cast<const uint4*>(a.H_sw128);
    const uint4* ssrc = reinterpret_cast<const uint4*>(a.S_sw128);
    uint4* hdst = reinterpret_cast<uint4*>(sm + PS::HB);
    uint4* sdst = reinterpret_cast<uint4*>(sm + PS::S);
    for (int w = tid; a.k && w < (int)(kTcTileBytes / 16); w += kPipeThreads) {  // values alone: none
      if constexpr (QJL) {
        sdst[w] = ssrc[w];
        sdst[w + kTcTileBytes / 16] = ssrc[w + kTcTileBytes / 16];
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) hdst[w + t * (kTcTileBytes / 16)] = hsrc[w + t * (kTcTileBytes / 16)];
    }
  }
  s1::fence_async_smem();
  s1::fence_before_sync();
  __syncthreads();
  s1::fence_after_sync();
  const uint32_t tmem = *tmem_s;
  bool failed = false;

  if (warp < 8) {
    // ================================================================ keys
    if (a.k) {
      const int sp = warp & 3, ch = warp >> 2;  // TMEM sub-partition, column half
      const int R = 32 * sp + lane;             // key (row) within the pass
      const uint32_t lane_base = (uint32_t)(32 * sp) << 16;
      float tm[HL > 1 ? HL - 1 : 1], cm[HL];
#pragma unroll
      for (int j = 0; j < HL - 1; ++j) tm[j] = 16.f * a.cb.t[HL + j];
#pragma unroll
      for (int j = 0; j < HL; ++j) cm[j] = 16.f * a.cb.c[HL + j];
      // Sign readout of a pass whose projection has completed: bit j set <=> (S r)_j >= 0.
      auto read_signs = [&](int64_t po, bool nzk) {  // po: the row's output row, or -1
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          uint32_t v[32];
          s1::tmem_ld32(tmem + kTmP + lane_base + 64 * ch + 32 * h, v);
          s1::tmem_ld_wait();
          uint32_t b4[4] = {0u, 0u, 0u, 0u};  // sign bits, four independent 8-bit chains
#pragma unroll
          for (int k = 7; k >= 0; --k)
#pragma unroll
            for (int q = 0; q < 4; ++q) b4[q] = __funnelshift_l(v[8 * q + k], b4[q], 1);
          const uint32_t word = ~(b4[0] | (b4[1] << 8) | (b4[2] << 16) | (b4[3] << 24));
          if (po >= 0) reinterpret_cast<uint32_t*>(a.k_signs + po * 16 + 8 * ch)[h] = nzk ? word : 0u;
        }
      };
      int it = 0;
      int64_t prev_o = -1;   // the previous pass's output row of this row's key (-1: none)
      bool prev_nz = false;  // and whether it was stored as nonzero
      for (int64_t tile = blockIdx.x; tile < ntile; tile += g, ++it) {
        const int b = it & 1;
        const int64_t v0 = tile * 128, i = v0 + R;
        const int64_t o = i < a.n_vec ? out_row(a, i) : -1;  // output row
        if (!failed && !s1::mbar_wait(rotd + b, (uint32_t)(it >> 1) & 1u)) failed = true;
        s1::fence_after_sync();
        // ||Y||^2 over the row's 128 columns, as two 64-column halves of four chains each
        float hs[2];
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          float2 s01 = make_float2(0.f, 0.f), s23 = make_float2(0.f, 0.f);
#pragma unroll 1
          for (int h = 0; h < 2; ++h) {
            uint32_t v[32];
            s1::tmem_ld32(tmem + kTmY + 128 * b + lane_base + 64 * c2 + 32 * h, v);
            s1::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float2 y01 = make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
              const float2 y23 = make_float2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
              s01 = s1::fma2(y01, y01, s01);
              s23 = s1::fma2(y23, y23, s23);
            }
          }
          hs[c2] = (s01.x + s01.y) + (s23.x + s23.y);
        }
        const float tot = hs[0] + hs[1];  // ||Y||^2: d ||k||^2 with H diag(sigma), ||k||^2 with Haar
        const bool nz = tot > 0.f;
        const float sc16 = nz ? 16.f * (1.0f / sqrtf(tot)) : 0.f;
        const float2 sc2 = make_float2(sc16, sc16);
        // the previous projection has finished: its S r is readable and the operand free
        if (QJL && it > 0) {
          if (!failed && !s1::mbar_wait(projd, (uint32_t)(it - 1) & 1u)) failed = true;
          s1::fence_after_sync();
          read_signs(prev_o, prev_nz);
        }
        float2 ra = make_float2(0.f, 0.f), rb = make_float2(0.f, 0.f);  // r^2 chains (0,1), (2,3)
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          uint32_t v[32];
          s1::tmem_ld32(tmem + kTmY + 128 * b + lane_base + 64 * ch + 32 * h, v);
          s1::tmem_ld_wait();
          uint32_t cw[LMB], cw2[LMB];  // even / odd codes: two independent chains per word
#pragma unroll
          for (int w = 0; w < LMB; ++w) cw[w] = cw2[w] = 0u;
#pragma unroll
          for (int o8 = 0; o8 < 2; ++o8) {
            uint32_t hw[8], lw[8];  // residual x16 as f16 pairs: hi, lo
#pragma unroll
            for (int pp = 0; pp < 8; ++pp) {
              const int p = 8 * o8 + pp, e = 2 * p;
              const float2 yy = s1::mul2(make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), sc2);
              uint32_t q0, q1;
              const float c0 = bucket_sym<LMB>(yy.x, tm, cm, q0);
              const float c1 = bucket_sym<LMB>(yy.y, tm, cm, q1);
              add_field<LMB, LMB>(cw, LMB * e, q0);
              add_field<LMB, LMB>(cw2, LMB * (e + 1), q1);
              const float2 r = s1::sub2(yy, make_float2(c0, c1));  // residual x16
              if (p & 1) rb = s1::fma2(r, r, rb);
              else ra = s1::fma2(r, r, ra);
              const __half2 hh = __floats2half2_rn(r.x, r.y);
              const float2 lo = s1::sub2(r, __half22float2(hh));
              const __half2 ll = __floats2half2_rn(lo.x, lo.y);
              hw[pp] = *reinterpret_cast<const uint32_t*>(&hh);
              lw[pp] = *reinterpret_cast<const uint32_t*>(&ll);
            }
            // row R's coordinates 64ch + 32h + 16o8 .. + 15: 8 columns of hi and of lo
            const uint32_t col = 32 * ch + 16 * h + 8 * o8;
            if constexpr (QJL) {
              s1::tmem_st8(tmem + kTmA + lane_base + col, hw);
              s1::tmem_st8(tmem + kTmA + 64 + lane_base + col, lw);
            }
          }
          if (o >= 0) {
            uint32_t* co = reinterpret_cast<uint32_t*>(a.k_codes + o * (LMB * 16) + ch * (LMB * 8) + h * (LMB * 4));
#pragma unroll
            for (int w = 0; w < LMB; ++w) co[w] = nz ? (cw[w] | cw2[w]) : 0u;
          }
        }
        const float rsum = (ra.x + ra.y) + (rb.x + rb.y);  // this half's sum of r^2
        if (ch == 1) xr[b * 128 + R] = rsum;
        // Y[b] read, S r read, operand written: hand the pass to the producer
        s1::tmem_st_wait();
        s1::fence_before_sync();
        __syncwarp();
        if (lane == 0) s1::mbar_arrive(aready);
        failed = s1::bar_sync_or<1, 256>(failed);
        if (failed) break;
        if (ch == 0 && o >= 0) {
          const float gamma = sqrtf(rsum + xr[b * 128 + R]) * (1.f / 16.f);
          // ||Y|| = sqrt(d) ||k|| with H diag(sigma); ||k|| with the orthonormal Haar matrix
          const uint32_t nb = __half_as_ushort(__float2half_rn(NT == 1 ? sqrtf(tot * (1.0f / 128.f)) : sqrtf(tot)));
          const uint32_t gb = __half_as_ushort(__float2half_rn(gamma));
          reinterpret_cast<uint32_t*>(a.k_norms)[o] = nz ? (nb | (gb << 16)) : 0u;
        }
        prev_o = o;
        prev_nz = nz;
      }
      // the last pass's signs
      if (QJL && !failed && it > 0) {
        if (!s1::mbar_wait(projd, (uint32_t)(it - 1) & 1u)) {
          failed = true;
        } else {
          s1::fence_after_sync();
          read_signs(prev_o, prev_nz);
        }
      }
    }
  } else if (warp < 16) {
    // ================================================================ values
    if (NT == 1 && a.v) {
    const int vt = tid - 256, q = vt & 3, vrow = vt >> 2;  // 4 threads per value, 64 per half
    const bool leader = vt == 0;
    uint32_t vpar = 0u, vpend = 0u;  // bit f for value half buffer f: next parity, copy outstanding
    // half h of a pass into buffer f: rows 64h..64h+63 as two panels of 64 rows x 128 bytes
    auto fetch_half = [&](int64_t tile, int h, int f) {
      const int64_t r0 = tile * 128 + 64 * h;
      if (r0 >= a.n_vec) return;
      unsigned char* dst = sm + PS::VR + f * (kTcTileBytes / 2);
      s1::mbar_expect_tx(vfull + f, 64u * 128u * 2u);
      s1::tma_load_2d(dst, &a.vmap, 0, (int)r0, vfull + f);
      s1::tma_load_2d(dst + kTcTileBytes / 4, &a.vmap, 64, (int)r0, vfull + f);
      vpend |= 1u << f;
    };
    // byte offset, within a half buffer, of this thread's 16-byte chunk k (coordinates 32q + 8k ..)
    const int vsw = vrow & 7;
    auto chunk_off = [&](int k) -> uint32_t {
      return (uint32_t)((q >> 1) * (kTcTileBytes / 4) + vrow * 128 + (((4 * (q & 1) + k) ^ vsw) << 4));
    };
    if (leader && (int64_t)blockIdx.x < ntile) {
      fetch_half(blockIdx.x, 0, 0);
      fetch_half(blockIdx.x, 1, 1);
      if (blockIdx.x + g < ntile) {
        fetch_half(blockIdx.x + g, 0, 2);
        fetch_half(blockIdx.x + g, 1, 3);
      }
    }
    constexpr int levels = (1 << VB) - 1;
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: adding it rounds to an integer
    // sum over a word's fields of the magic constant's bits shifted into place (mod 2^32)
    uint32_t magic_sum = 0u;
#pragma unroll
    for (int f = 0; f < 32 / VB; ++f) magic_sum += __float_as_uint(kMagic) << (VB * f);
    int it = 0;
    for (int64_t tile = blockIdx.x; tile < ntile && !failed; tile += g, ++it) {
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int f = 2 * (it & 1) + h;
        const int64_t r0 = tile * 128 + 64 * h;
        if (r0 >= a.n_vec) break;  // the same for every value thread
        if (!failed) {
          if (s1::mbar_wait(vfull + f, (vpar >> f) & 1u)) {
            vpar ^= 1u << f;
            vpend &= ~(1u << f);
          } else {
            failed = true;
          }
        }
        const int64_t i = r0 + vrow;
        const int64_t o = i < a.n_vec ? out_row(a, i) : -1;  // output row
        if (!failed && o >= 0) {
          const unsigned char* half = sm + PS::VR + f * (kTcTileBytes / 2);
          uint32_t w[16];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 u = *reinterpret_cast<const uint4*>(half + chunk_off(k));
            w[4 * k] = u.x;
            w[4 * k + 1] = u.y;
            w[4 * k + 2] = u.z;
            w[4 * k + 3] = u.w;
          }
          // min / max on the packed bf16 pairs (exact: bf16 -> fp32 is monotone), as trees
          __nv_bfloat162 mn[8], mx[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const __nv_bfloat162 x0 = *reinterpret_cast<const __nv_bfloat162*>(&w[k]);
            const __nv_bfloat162 x1 = *reinterpret_cast<const __nv_bfloat162*>(&w[k + 8]);
            mn[k] = __hmin2(x0, x1);
            mx[k] = __hmax2(x0, x1);
          }
#pragma unroll
          for (int s = 4; s >= 1; s >>= 1)
#pragma unroll
            for (int k = 0; k < s; ++k) {
              mn[k] = __hmin2(mn[k], mn[k + s]);
              mx[k] = __hmax2(mx[k], mx[k + s]);
            }
          const float lo = fminf(__low2float(mn[0]), __high2float(mn[0]));
          const float hi = fmaxf(__low2float(mx[0]), __high2float(mx[0]));
          // Codes rounded to nearest by adding 1.5 * 2^23 to t = (v - min) * levels / span.
          // Four roundings (span, levels / span, v - min, the product) put the fp32 t within
          // levels * 2.4e-7 of the exact value, so it gives the reference's floor(t + 1/2)
          // except at most that close to a half step (an exact tie, or within rounding of
          // one), where the code may be the other neighbour. For 2-bit codes that band is
          // narrower than 1e-6; for 4-bit codes the coordinates within 5e-6 of a half step
          // are redone in fp64 as floor(t + 1/2).
          constexpr bool kRedoNearHalf = VB > 2;
          const double dlo = lo, span = (double)hi - dlo;
          const float span32 = hi - lo;
          const float inv = span32 > 0.f ? __fdiv_rn((float)levels, span32) : 0.f;
          const float2 lo2 = make_float2(lo, lo), inv2 = make_float2(inv, inv), mg2 = make_float2(kMagic, kMagic);
          uint32_t vw[VB], vw2[VB];
#pragma unroll
          for (int k = 0; k < VB; ++k) vw[k] = vw2[k] = 0u;
          uint32_t near = 0u;  // bit e: coordinate e within 1e-5 of a half step
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float2 x = make_float2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xffff0000u));
            const float2 t = s1::mul2(s1::sub2(x, lo2), inv2);
            const float2 tr = s1::add2(t, mg2);
            const float2 e = s1::sub2(t, s1::sub2(tr, mg2));
            if (kRedoNearHalf) {
              if (fabsf(e.x) > 0.5f - 5e-6f) near |= 1u << (2 * k);
              if (fabsf(e.y) > 0.5f - 5e-6f) near |= 2u << (2 * k);
            }
            if constexpr (VB == 3) {
              // 3-bit fields straddle words: the code alone, masked out of tr's low bits
              add_field<VB, VB>(vw, VB * 2 * k, __float_as_uint(tr.x) & 7u);
              add_field<VB, VB>(vw2, VB * (2 * k + 1), __float_as_uint(tr.y) & 7u);
            } else {
              // tr's bits are those of the magic constant plus the code
              add_field<VB, VB>(vw, VB * 2 * k, __float_as_uint(tr.x));
              add_field<VB, VB>(vw2, VB * (2 * k + 1), __float_as_uint(tr.y));
            }
          }
#pragma unroll
          for (int k = 0; k < VB; ++k) vw[k] = vw[k] + vw2[k] - (VB == 3 ? 0u : magic_sum);
          if (kRedoNearHalf && near) {
            // Some coordinate lies within 5e-6 of a half step (with bf16 inputs a ratio of
            // small integers lands exactly on one in about one group of twenty): redo only
            // those in fp64.
            uint32_t mask = near;
            const double r64 = levels / span;
            while (mask) {
              const int e = __ffs(mask) - 1;
              mask &= mask - 1u;
              const float xe = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                  half + chunk_off(e >> 3) + 2 * (e & 7)));
              const uint32_t qv = min((uint32_t)floor(((double)xe - dlo) * r64 + 0.5), (uint32_t)levels);
              const int wi = (VB * e) >> 5, sh = (VB * e) & 31;
#pragma unroll
              for (int k = 0; k < VB; ++k) {  // replace the field in place (static indices)
                const uint32_t sel = (wi == k) ? 0xffffffffu : 0u;
                const uint32_t old = (vw[k] >> sh) & (uint32_t)levels;
                vw[k] ^= ((old ^ qv) << sh) & sel;
                if (VB == 3 && sh > 29) {  // the field's high bits, at the bottom of the next word
                  const uint32_t selh = (wi + 1 == k) ? 0xffffffffu : 0u;
                  const uint32_t mh = (1u << (sh - 29)) - 1u;
                  vw[k] ^= ((vw[k] & mh) ^ (qv >> (32 - sh))) & selh;
                }
              }
            }
          }
          uint32_t* vo = reinterpret_cast<uint32_t*>(a.v_codes + o * (VB * 16) + q * (VB * 4));
#pragma unroll
          for (int k = 0; k < VB; ++k) vo[k] = vw[k];
          const uint32_t sb = __half_as_ushort(__double2half(div_levels<levels>(span)));
          const uint32_t mb = __half_as_ushort(__float2half_rn(lo));
          reinterpret_cast<uint32_t*>(a.v_params)[o * 4 + q] = sb | (mb << 16);
        }
        // every value thread is done with this half: refill it two passes ahead
        failed = s1::bar_sync_or<2, 256>(failed);
        if (failed) break;
        if (leader && tile + 2 * g < ntile) {
          s1::fence_async_smem();
          fetch_half(tile + 2 * g, h, f);
        }
      }
    }
    if (failed && leader)
      for (int f = 0; f < 4; ++f)
        if ((vpend >> f) & 1u) s1::mbar_wait(vfull + f, (vpar >> f) & 1u);  // bounded
    }
  } else if (warp == 16 && lane == 0 && a.k && (int64_t)blockIdx.x < ntile) {
    // ================================================================ producer
    const int64_t n_my = (ntile - blockIdx.x + g - 1) / g;  // passes of this CTA
    auto tile_of = [&](int64_t j) { return (int64_t)blockIdx.x + j * g; };
    uint32_t kpar = 0u, kpend = 0u;  // bit b for key buffer b: next parity, load outstanding
    auto load_keys = [&](int b, int64_t tile) {
      s1::mbar_expect_tx(kfull + b, 2u * 128u * 128u);
      s1::tma_load_2d(sm + PS::KT + b * kTcTileBytes, &a.kmap, 0, (int)(tile * 128), kfull + b);
      s1::tma_load_2d(sm + PS::KT + b * kTcTileBytes + kTcTileBytes / 2, &a.kmap, 64, (int)(tile * 128), kfull + b);
      kpend |= 1u << b;
    };
    auto wait_keys = [&](int b) -> bool {
      if (!s1::mbar_wait(kfull + b, (kpar >> b) & 1u)) return false;
      kpar ^= 1u << b;
      kpend &= ~(1u << b);
      return true;
    };
    auto rotation = [&](int b) {  // Y[b] = KT[b] R^T, R = H diag(sigma) or the Haar matrix's NT terms
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          s1::umma_f16(tmem + kTmY + 128 * b, s1::sw128_desc(sbase + PS::KT + b * kTcTileBytes, 16 * ks, 128),
                       s1::sw128_desc(sbase + PS::HB + t * kTcTileBytes, 16 * ks, 128), idesc,
                       (t > 0 || ks > 0) ? 1u : 0u);
      s1::umma_commit(rotd + b);
    };
    auto projection = [&]() {  // S r = (A_hi + A_lo) S_hi^T + A_hi S_lo^T, A in tensor memory
      constexpr uint32_t idesc = s1::idesc_f16_f32(128, 128);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        s1::umma_f16_ts(tmem + kTmP, tmem + kTmA + 8 * ks, s1::sw128_desc(sbase + PS::S, 16 * ks, 128), idesc,
                        ks > 0 ? 1u : 0u);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        s1::umma_f16_ts(tmem + kTmP, tmem + kTmA + 64 + 8 * ks, s1::sw128_desc(sbase + PS::S, 16 * ks, 128), idesc,
                        1u);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        s1::umma_f16_ts(tmem + kTmP, tmem + kTmA + 8 * ks,
                        s1::sw128_desc(sbase + PS::S + kTcTileBytes, 16 * ks, 128), idesc, 1u);
      s1::umma_commit(projd);
    };
    // Prologue: passes 0 and 1 loaded and rotated, pass 2's keys on their way.
    load_keys(0, tile_of(0));
    if (n_my > 1) load_keys(1, tile_of(1));
    if (!wait_keys(0)) failed = true;
    else rotation(0);
    if (!failed && n_my > 1) {
      if (!wait_keys(1)) failed = true;
      else rotation(1);
    }
    if (!failed && n_my > 2) {
      if (!s1::mbar_wait(rotd, 0u)) failed = true;
      else load_keys(0, tile_of(2));
    }
    for (int64_t j = 0; j < n_my && !failed; ++j) {
      const int b = (int)(j & 1);
      // KT[b^1] holds pass j+1, whose rotation was issued: once it has completed, refill
      // that buffer with pass j+3
      if (j + 3 < n_my) {
        if (!s1::mbar_wait(rotd + (b ^ 1), (uint32_t)((j + 1) >> 1) & 1u)) {
          failed = true;
          break;
        }
        load_keys(b ^ 1, tile_of(j + 3));
      }
      // pass j's residual operand is in tensor memory (and its S r slot read out): project
      if (!s1::mbar_wait(aready, (uint32_t)j & 1u)) {
        failed = true;
        break;
      }
      s1::fence_after_sync();
      if constexpr (QJL) projection();
      // Y[b] is free again: rotate pass j+2 once its keys have landed
      if (j + 2 < n_my) {
        if (!wait_keys(b)) {
          failed = true;
          break;
        }
        rotation(b);
      }
    }
    if (failed) {
      // bounded: drain the issued MMAs and the outstanding key loads before the shared
      // and tensor memory they use is released
      s1::umma_commit(fin);
      s1::mbar_wait(fin, 0u);
      for (int b = 0; b < 2; ++b)
        if ((kpend >> b) & 1u) s1::mbar_wait(kfull + b, (kpar >> b) & 1u);
    }
  }
  if (__syncthreads_or(failed) && tid == 0) atomicOr(a.err, 1u);
  s1::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    s1::fence_after_sync();
    s1::tmem_dealloc(tmem, 512);
  }
}

// cuTensorMapEncodeTiled, fetched once from the driver through the runtime.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// A tensor map of compress_pipe_kernel: [n_vec][128] bf16 rows, boxes of 64 columns x
// box_rows rows (one 128-byte-swizzled panel each). False if it cannot be made.
bool encode_rows_map(CUtensorMap* map, const void* k, int64_t n_vec, uint32_t box_rows, int cols = 128) {
  const EncodeTiledFn enc = tensor_map_encoder();
  if (!enc || n_vec <= 0 || n_vec >= ((int64_t)1 << 31)) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)n_vec};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(k), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// c[L-1-k] == -c[k] and t[L-2-k] == -t[k] exactly.
bool codebook_symmetric(const Codebook& cb, int lm_bits) {
  const int L = 1 << lm_bits;
  for (int k = 0; k < L; ++k)
    if (cb.c[L - 1 - k] != -cb.c[k]) return false;
  for (int k = 0; k < L - 1; ++k)
    if (cb.t[L - 2 - k] != -cb.t[k]) return false;
  return true;
}

template <int LMB, int VB, int NT, bool QJL = true>
cudaError_t launch_pipe_t(const tq_ctx* ctx, const CompressArgs& a, cudaStream_t s) {
  static bool configured = false;
  const size_t smem = PipeSmem<NT>::BYTES + 1024;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(compress_pipe_kernel<LMB, VB, NT, QJL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  int64_t blocks = (a.n_vec + 127) / 128;
  if (blocks > ctx->num_sms) blocks = ctx->num_sms;
  if (ctx->prof_start) cudaEventRecord(ctx->prof_start, s);
  compress_pipe_kernel<LMB, VB, NT, QJL><<<(unsigned)blocks, kPipeThreads, smem, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (ctx->prof_stop) cudaEventRecord(ctx->prof_stop, s);
  return e;
}

template <int VB>
cudaError_t launch_pipe_vb(const tq_ctx* ctx, const CompressArgs& a, cudaStream_t s) {
  const int lmb = ctx->shape.lm_bits;
  if (lmb == 1) return launch_pipe_t<1, VB, 1>(ctx, a, s);
  if (lmb == 2) return launch_pipe_t<2, VB, 1>(ctx, a, s);
  return launch_pipe_t<3, VB, 1>(ctx, a, s);
}

cudaError_t launch_pipe(const tq_ctx* ctx, const CompressArgs& a, cudaStream_t s) {
  const int vb = ctx->shape.v_bits;
  return vb == 2 ? launch_pipe_vb<2>(ctx, a, s) : vb == 3 ? launch_pipe_vb<3>(ctx, a, s) : launch_pipe_vb<4>(ctx, a, s);
}

// Keys without the QJL stage (m = 0; either rotation), or values alone, on the same kernel.
cudaError_t launch_pipe_nq(const tq_ctx* ctx, const CompressArgs& a, cudaStream_t s) {
  const int lmb = ctx->shape.lm_bits, vb = ctx->shape.v_bits;
  if (a.k && ctx->shape.rot == TQ_ROT_HAAR) {  // keys only: the Haar tiles take the value rows
    if (lmb == 1) return launch_pipe_t<1, 2, 3, false>(ctx, a, s);
    if (lmb == 2) return launch_pipe_t<2, 2, 3, false>(ctx, a, s);
    return launch_pipe_t<3, 2, 3, false>(ctx, a, s);
  }
  if (!a.k)  // values alone: the key settings do not matter
    return vb == 2 ? launch_pipe_t<1, 2, 1, false>(ctx, a, s)
           : vb == 3 ? launch_pipe_t<1, 3, 1, false>(ctx, a, s) : launch_pipe_t<1, 4, 1, false>(ctx, a, s);
  if (lmb == 1) return launch_pipe_t<1, 2, 1, false>(ctx, a, s);
  if (lmb == 2) return launch_pipe_t<2, 2, 1, false>(ctx, a, s);
  return launch_pipe_t<3, 2, 1, false>(ctx, a, s);
}

// Keys only with the Haar rotation (its three operand tiles in place of the value rows).
cudaError_t launch_pipe_haar(const tq_ctx* ctx, const CompressArgs& a, cudaStream_t s) {
  const int lmb = ctx->shape.lm_bits;
  if (lmb == 1) return launch_pipe_t<1, 2, 3>(ctx, a, s);
  if (lmb == 2) return launch_pipe_t<2, 2, 3>(ctx, a, s);
  return launch_pipe_t<3, 2, 3>(ctx, a, s);
}

// ---------------------------------------------------------------------------------
// bf16 keys at d = 64 or 256 on the tensor cores, with either rotation (the keys only; a
// call with values runs them through the warp-per-vector kernel). The rotation R is held
// as NT bf16 terms: H diag(sigma) (+-1, exact, NT = 1) or the Haar matrix split in three
// terms (NT = 3, about 24 bits); Y = K R^T is exact in its products and accumulates in
// fp32, then the key work is that of compress_rot_kernel, then S r = (A_hi + A_lo) S_hi^T +
// A_hi S_lo^T with A, the residual x16 in f16 hi + lo, in tensor memory. 128 keys per pass,
// one pass at a time; two threads per key (TMEM lane = key, each thread half of the
// columns). The operand tiles (NW x NW, NW = 64 at d = 64, 128 at d = 256) are prepacked
// on the host in the swizzled K-major layout: at d = 64 all of them stay in shared memory;
// at d = 256 (12 or 20 tiles of 32 KB per pass) they stream from global memory (L2-resident)
// through a ring of three slots, each refilled as soon as the MMAs that read it complete.
constexpr int kDenseThreads = 288;  // warps 0-7 keys (lane quadrant w % 4, column half w / 4), warp 8 producer

template <int D, int NT>
struct DenseSmem {
  static constexpr int NW = D == 256 ? 128 : 64;    // chunk width (N and K) of an operand tile
  static constexpr int NCH = D / NW;                 // N chunks = K chunks
  static constexpr uint32_t TILE = (uint32_t)NW * NW * 2;
  static constexpr int NROT = NCH * NCH * NT;        // rotation tiles per pass
  static constexpr int NOPS = NROT + NCH * NCH * 2;  // + S hi / lo tiles
  static constexpr bool STREAM = D == 256;
  static constexpr int SLOTS = STREAM ? 3 : NOPS;
  static constexpr uint32_t KT = 0;                              // key tile [128][D] bf16, D/64 panels
  static constexpr uint32_t OPS = (uint32_t)128 * D * 2;         // operand tiles (ring or resident)
  static constexpr uint32_t XS = OPS + SLOTS * TILE;             // [2][128] half-row sums
  static constexpr uint32_t ZF = XS + 2 * 128 * 4;               // [128] nonzero-key flags
  static constexpr uint32_t BAR = ZF + 128;  // kfull, rotd, aready, projd, pdone, ofull[3], oempty[3], fin
  static constexpr uint32_t TMEM = BAR + 8 * 12;
  static constexpr uint32_t BYTES = TMEM + 8;
  static_assert(BYTES + 1024 <= 227 * 1024, "compress_dense_kernel shared memory");
};
// Tensor memory: Y (then S r) at columns [0, D), the residual operand's hi at A and lo at
// A + D/2 (one f16 pair per column). At d = 64 a CTA takes 256 columns (A = 128), so two CTAs
// share an SM and one's MMAs and bulk copies run under the other's key work; at d = 256 one
// CTA takes all 512 (A = 256).
template <int D>
struct DenseTmem {
  static constexpr uint32_t A = D == 64 ? 128 : 256;
  static constexpr uint32_t COLS = D == 64 ? 256 : 512;
  static constexpr int CTAS_PER_SM = D == 64 ? 2 : 1;
};

__device__ __forceinline__ void dense_key_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(256) : "memory");
}

template <int D, int LMB, int NT>
__global__ void __launch_bounds__(kDenseThreads, DenseTmem<D>::CTAS_PER_SM)
    compress_dense_kernel(const __grid_constant__ CompressArgs a, const uint16_t* __restrict__ ops) {
  using DS = DenseSmem<D, NT>;
  constexpr uint32_t kDnA = DenseTmem<D>::A;
  namespace s1 = tq::sm100;
  constexpr int NW = DS::NW, NCH = DS::NCH;
  constexpr int HALF = D / 2;  // columns per thread
  extern __shared__ unsigned char smem_dense[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(((uintptr_t)smem_dense + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = s1::smem_u32(sm);
  float* xs = reinterpret_cast<float*>(sm + DS::XS);
  uint8_t* zf = sm + DS::ZF;
  uint64_t* kfull = reinterpret_cast<uint64_t*>(sm + DS::BAR);  // key tile landed
  uint64_t* rotd = kfull + 1;     // rotation MMAs done
  uint64_t* aready = kfull + 2;   // key warps wrote the residual operand (8 arrivals)
  uint64_t* projd = kfull + 3;    // projection MMAs done
  uint64_t* pdone = kfull + 4;    // key warps read S r (8 arrivals)
  uint64_t* ofull = kfull + 5;    // [3] operand slot landed
  uint64_t* oempty = kfull + 8;   // [3] operand slot read by its MMAs
  uint64_t* fin = kfull + 11;     // every MMA issued has completed
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(sm + DS::TMEM);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t ntile = (a.n_vec + 127) / 128, g = gridDim.x;

  if (warp == 0) {
    s1::tmem_alloc(tmem_s, DenseTmem<D>::COLS);
    s1::tmem_relinquish();
  }
  if (tid == 0) {
    s1::mbar_init(kfull, 1);
    s1::mbar_init(rotd, 1);
    s1::mbar_init(aready, 8);
    s1::mbar_init(projd, 1);
    s1::mbar_init(pdone, 8);
    s1::mbar_init(fin, 1);
    for (int k = 0; k < 3; ++k) {
      s1::mbar_init(ofull + k, 1);
      s1::mbar_init(oempty + k, 1);
    }
    s1::mbar_init_fence();
  }
  if constexpr (!DS::STREAM) {  // every operand tile stays resident
    const uint4* src = reinterpret_cast<const uint4*>(ops);
    uint4* dst = reinterpret_cast<uint4*>(sm + DS::OPS);
    for (int w = tid; w < (int)(DS::NOPS * DS::TILE / 16); w += kDenseThreads) dst[w] = src[w];
  }
  s1::fence_async_smem();
  s1::fence_before_sync();
  __syncthreads();
  s1::fence_after_sync();
  const uint32_t tmem = *tmem_s;
  bool failed = false;

  if (warp < 8) {
    // ================================================================ keys
    const int sp = warp & 3, ch = warp >> 2;
    const int R = 32 * sp + lane;
    const uint32_t lane_base = (uint32_t)(32 * sp) << 16;
    float cb_t[(1 << LMB) - 1], cb_c[1 << LMB];
#pragma unroll
    for (int k = 0; k < (1 << LMB) - 1; ++k) cb_t[k] = a.cb.t[k];
#pragma unroll
    for (int k = 0; k < (1 << LMB); ++k) cb_c[k] = a.cb.c[k];
    // ||Y|| = sqrt(d) ||k|| for H diag(sigma) (not normalised), ||k|| for Haar
    const float ninv = NT == 1 ? rsqrtf((float)D) : 1.f;
    int it = 0;
    for (int64_t tile = blockIdx.x; tile < ntile; tile += g, ++it) {
      const uint32_t ph = (uint32_t)it & 1u;
      const int64_t i = tile * 128 + R;
      const bool valid = i < a.n_vec;
      const int64_t o = valid ? out_row(a, i) : -1;
      if (!failed && !s1::mbar_wait(rotd, ph)) failed = true;
      if (s1::bar_sync_or<1, 256>(failed)) {
        failed = true;
        break;
      }
      s1::fence_after_sync();
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
      for (int h = 0; h < HALF / 32; ++h) {
        uint32_t v[32];
        s1::tmem_ld32(tmem + lane_base + HALF * ch + 32 * h, v);
        s1::tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float yv = __uint_as_float(v[e]);
          s4[e & 3] = fmaf(yv, yv, s4[e & 3]);
        }
      }
      xs[ch * 128 + R] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
      dense_key_sync();
      const float tot = xs[R] + xs[128 + R];
      dense_key_sync();
      const bool nz = tot > 0.f;
      const float sc = nz ? 1.0f / sqrtf(tot) : 0.f;
      const bool use = valid && nz;
      float r4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
      for (int h = 0; h < HALF / 32; ++h) {
        uint32_t v[32];
        s1::tmem_ld32(tmem + lane_base + HALF * ch + 32 * h, v);
        s1::tmem_ld_wait();
        uint32_t cw[LMB], cw2[LMB];
#pragma unroll
        for (int w = 0; w < LMB; ++w) cw[w] = cw2[w] = 0u;
        float r[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float yy = __uint_as_float(v[e]) * sc;
          uint32_t idx = 0;
          float cv = cb_c[0];
#pragma unroll
          for (int k = 0; k < (1 << LMB) - 1; ++k) {
            if (yy >= cb_t[k]) {
              idx = k + 1;
              cv = cb_c[k + 1];
            }
          }
          if (e & 1)
            put_bits<LMB, LMB>(cw2, LMB * e, idx);
          else
            put_bits<LMB, LMB>(cw, LMB * e, idx);
          r[e] = yy - cv;
          r4[e & 3] = fmaf(r[e], r[e], r4[e & 3]);
        }
        if (o >= 0) {
          uint32_t* co = reinterpret_cast<uint32_t*>(a.k_codes + o * (LMB * D / 8) + (HALF * ch + 32 * h) * LMB / 8);
#pragma unroll
          for (int w = 0; w < LMB; ++w) co[w] = nz ? (cw[w] | cw2[w]) : 0u;
        }
#pragma unroll
        for (int c16 = 0; c16 < 2; ++c16) {
          uint32_t hw[8], lw[8];
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            const float f0 = use ? 16.f * r[16 * c16 + 2 * p] : 0.f, f1 = use ? 16.f * r[16 * c16 + 2 * p + 1] : 0.f;
            const __half2 hh = __floats2half2_rn(f0, f1);
            const float2 hf = __half22float2(hh);
            const __half2 ll = __floats2half2_rn(f0 - hf.x, f1 - hf.y);
            hw[p] = *reinterpret_cast<const uint32_t*>(&hh);
            lw[p] = *reinterpret_cast<const uint32_t*>(&ll);
          }
          const uint32_t col = (HALF * ch + 32 * h + 16 * c16) / 2;
          s1::tmem_st8(tmem + kDnA + lane_base + col, hw);
          s1::tmem_st8(tmem + kDnA + HALF + lane_base + col, lw);
        }
      }
      xs[ch * 128 + R] = (r4[0] + r4[1]) + (r4[2] + r4[3]);
      dense_key_sync();
      const float gamma = sqrtf(xs[R] + xs[128 + R]);
      if (o >= 0 && ch == 0) {
        const uint32_t nb = __half_as_ushort(__float2half_rn(sqrtf(tot) * ninv));
        const uint32_t gb = __half_as_ushort(__float2half_rn(gamma));
        reinterpret_cast<uint32_t*>(a.k_norms)[o] = nz ? (nb | (gb << 16)) : 0u;
      }
      if (ch == 0) zf[R] = use ? 1 : 0;
      s1::tmem_st_wait();
      s1::fence_before_sync();
      __syncwarp();
      if (lane == 0) s1::mbar_arrive(aready);
      // ---- QJL signs of this thread's projections
      if (!failed && !s1::mbar_wait(projd, ph)) failed = true;
      dense_key_sync();  // zf of both halves written (and read below)
      s1::fence_after_sync();
      const bool nzk = zf[R] != 0;
#pragma unroll 1
      for (int h = 0; h < HALF / 32; ++h) {
        uint32_t v[32];
        s1::tmem_ld32(tmem + lane_base + HALF * ch + 32 * h, v);
        s1::tmem_ld_wait();
        uint32_t b4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int k = 7; k >= 0; --k)
#pragma unroll
          for (int q = 0; q < 4; ++q) b4[q] = __funnelshift_l(v[8 * q + k] ^ 0x80000000u, b4[q], 1);
        const uint32_t word = b4[0] | (b4[1] << 8) | (b4[2] << 16) | (b4[3] << 24);
        if (o >= 0 && !failed)
          reinterpret_cast<uint32_t*>(a.k_signs + o * (D / 8) + (HALF * ch + 32 * h) / 8)[0] = nzk ? word : 0u;
      }
      s1::fence_before_sync();
      __syncwarp();
      if (lane == 0) s1::mbar_arrive(pdone);
    }
  } else if (warp == 8 && lane == 0 && (int64_t)blockIdx.x < ntile) {
    // ================================================================ producer (TMA and MMA)
    constexpr uint32_t idesc_rot = s1::idesc_f16_f32(128, NW) | (1u << 7) | (1u << 10);  // bf16 x bf16
    constexpr uint32_t idesc_prj = s1::idesc_f16_f32(128, NW);                           // f16 x f16
    const int64_t n_my = (ntile - blockIdx.x + g - 1) / g;
    int kloads = 0;  // key-tile loads issued (phase kloads - 1 is the last one)
    auto load_keys = [&](int64_t tile) {
      ++kloads;
      s1::mbar_expect_tx(kfull, (uint32_t)128 * D * 2);
#pragma unroll
      for (int p = 0; p < D / 64; ++p)
        s1::tma_load_2d(sm + DS::KT + p * 128 * 128, &a.kmap, 64 * p, (int)(tile * 128), kfull);
    };
    // streamed operand q (0 .. n_my * NOPS - 1): tile q % NOPS of the pass sequence, slot q % 3
    int64_t issued = 0, used = 0;
    auto issue_op = [&]() {
      const int slot = (int)(issued % 3);
      s1::mbar_expect_tx(ofull + slot, DS::TILE);
      s1::bulk_g2s(sm + DS::OPS + slot * DS::TILE, ops + (size_t)(issued % DS::NOPS) * (DS::TILE / 2), DS::TILE,
                   ofull + slot);
      ++issued;
    };
    const int64_t n_ops = n_my * DS::NOPS;
    // the operand tile of sequence number q: its shared-memory address (waits for it to land)
    auto op_addr = [&](int64_t q, bool& ok) -> uint32_t {
      if constexpr (!DS::STREAM) {
        return sbase + DS::OPS + (uint32_t)(q % DS::NOPS) * DS::TILE;
      } else {
        const int slot = (int)(q % 3);
        if (!s1::mbar_wait(ofull + slot, (uint32_t)(q / 3) & 1u)) ok = false;
        return sbase + DS::OPS + slot * DS::TILE;
      }
    };
    // after the MMAs of operand q are issued: release its slot, refill the slot of q - 1
    auto done_op = [&](int64_t q, bool& ok) {
      if constexpr (DS::STREAM) {
        s1::umma_commit(oempty + (int)(q % 3));
        ++used;
        if (q >= 1 && issued < n_ops) {
          // the slot of q - 1 is the slot of q + 2
          if (!s1::mbar_wait(oempty + (int)((q - 1) % 3), (uint32_t)((q - 1) / 3) & 1u)) ok = false;
          else issue_op();
        }
      }
    };
    if constexpr (DS::STREAM) {
      for (int k = 0; k < 3 && issued < n_ops; ++k) issue_op();
    }
    load_keys(blockIdx.x);
    int64_t q = 0;  // operand sequence number
    for (int64_t j = 0; j < n_my && !failed; ++j) {
      const uint32_t ph = (uint32_t)j & 1u;
      bool ok = s1::mbar_wait(kfull, ph);
      if (ok && j > 0) ok = s1::mbar_wait(pdone, ph ^ 1u);  // S r of the previous pass read: TMEM free
      if (!ok) {
        failed = true;
        break;
      }
      s1::fence_after_sync();
      // rotation: Y[:, nc] = sum over kc, t of K[:, kc] R_t[nc, kc]^T
      for (int nc = 0; nc < NCH && ok; ++nc)
        for (int kc = 0; kc < NCH && ok; ++kc)
          for (int t = 0; t < NT && ok; ++t, ++q) {
            const uint32_t b = op_addr(q, ok);
            if (!ok) break;
#pragma unroll
            for (int ks = 0; ks < NW / 16; ++ks)
              s1::umma_f16(tmem + nc * NW, s1::sw128_desc(sbase + DS::KT, kc * NW + 16 * ks, 128),
                           s1::sw128_desc(b, 16 * ks, NW), idesc_rot, (kc > 0 || t > 0 || ks > 0) ? 1u : 0u);
            done_op(q, ok);
          }
      if (!ok) {
        failed = true;
        break;
      }
      s1::umma_commit(rotd);
      // the key tile is free once the rotation has completed: fetch the next pass's
      if (j + 1 < n_my) {
        if (!s1::mbar_wait(rotd, ph)) {
          failed = true;
          break;
        }
        load_keys(blockIdx.x + (j + 1) * g);
      }
      if (!s1::mbar_wait(aready, ph)) {
        failed = true;
        break;
      }
      s1::fence_after_sync();
      // projection: S r[:, nc] = sum over kc of (A_hi + A_lo)[:, kc] S_hi[nc, kc]^T + A_hi S_lo^T
      for (int nc = 0; nc < NCH && ok; ++nc)
        for (int kc = 0; kc < NCH && ok; ++kc) {
          const uint32_t bh = op_addr(q, ok);
          if (!ok) break;
#pragma unroll
          for (int ks = 0; ks < NW / 16; ++ks) {
            const uint32_t ac = (uint32_t)(kc * NW + 16 * ks) / 2;
            s1::umma_f16_ts(tmem + nc * NW, tmem + kDnA + ac, s1::sw128_desc(bh, 16 * ks, NW), idesc_prj,
                            (kc > 0 || ks > 0) ? 1u : 0u);
            s1::umma_f16_ts(tmem + nc * NW, tmem + kDnA + HALF + ac, s1::sw128_desc(bh, 16 * ks, NW), idesc_prj, 1u);
          }
          done_op(q, ok);
          ++q;
          const uint32_t bl = op_addr(q, ok);
          if (!ok) break;
#pragma unroll
          for (int ks = 0; ks < NW / 16; ++ks) {
            const uint32_t ac = (uint32_t)(kc * NW + 16 * ks) / 2;
            s1::umma_f16_ts(tmem + nc * NW, tmem + kDnA + ac, s1::sw128_desc(bl, 16 * ks, NW), idesc_prj, 1u);
          }
          done_op(q, ok);
          ++q;
        }
      if (!ok) {
        failed = true;
        break;
      }
      s1::umma_commit(projd);
    }
    if (failed) atomicOr(a.err, 1u);
    // every MMA issued and every copy issued completes before the CTA's memory goes away
    s1::umma_commit(fin);
    s1::mbar_wait(fin, 0u);
    if (kloads > 0) s1::mbar_wait(kfull, (uint32_t)(kloads - 1) & 1u);
    if constexpr (DS::STREAM) {
      // the operand copies issued ahead of use land before the CTA exits
      for (int64_t qq = used; qq < issued; ++qq) s1::mbar_wait(ofull + (int)(qq % 3), (uint32_t)(qq / 3) & 1u);
    }
  }
  s1::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    s1::fence_after_sync();
    s1::tmem_dealloc(tmem, DenseTmem<D>::COLS);
  }
}

template <int D, int LMB, int NT>
cudaError_t launch_dense_t(const tq_ctx* ctx, const CompressArgs& a, const uint16_t* ops, cudaStream_t s) {
  using DS = DenseSmem<D, NT>;
  static bool configured = false;
  // Shared memory padded so that an SM holds no more CTAs than tensor memory takes: at least
  // 120 KB at d = 256 (one CTA, all 512 columns), 80 KB at d = 64 (two CTAs of 256 columns).
  constexpr size_t kFloor = DenseTmem<D>::CTAS_PER_SM == 2 ? 80 * 1024 : 120 * 1024;
  static_assert(DenseTmem<D>::CTAS_PER_SM == 1 || DS::BYTES + 1024 <= kFloor, "two CTAs per SM at d = 64");
  const size_t smem = DS::BYTES + 1024 > kFloor ? DS::BYTES + 1024 : kFloor;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(compress_dense_kernel<D, LMB, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  int64_t blocks = (a.n_vec + 127) / 128;
  if (blocks > (int64_t)DenseTmem<D>::CTAS_PER_SM * ctx->num_sms) blocks = (int64_t)DenseTmem<D>::CTAS_PER_SM * ctx->num_sms;
  if (ctx->prof_start) cudaEventRecord(ctx->prof_start, s);
  compress_dense_kernel<D, LMB, NT><<<(unsigned)blocks, kDenseThreads, smem, s>>>(a, ops);
  cudaError_t e = cudaGetLastError();
  if (ctx->prof_stop) cudaEventRecord(ctx->prof_stop, s);
  return e;
}

template <int D, int NT>
cudaError_t launch_dense_l(const tq_ctx* ctx, const CompressArgs& a, const uint16_t* ops, cudaStream_t s) {
  switch (ctx->shape.lm_bits) {
    case 1: return launch_dense_t<D, 1, NT>(ctx, a, ops, s);
    case 2: return launch_dense_t<D, 2, NT>(ctx, a, ops, s);
    case 3: return launch_dense_t<D, 3, NT>(ctx, a, ops, s);
  }
  return cudaErrorInvalidValue;
}

// The dense tensor-core kernel for bf16 keys at d = 64 or 256 (keys only).
cudaError_t launch_dense(const tq_ctx* ctx, const CompressArgs& a, cudaStream_t s) {
  const bool haar = ctx->shape.rot == TQ_ROT_HAAR;
  if (ctx->shape.d == 64)
    return haar ? launch_dense_l<64, 3>(ctx, a, ctx->dense_ops, s) : launch_dense_l<64, 1>(ctx, a, ctx->dense_ops, s);
  return haar ? launch_dense_l<256, 3>(ctx, a, ctx->dense_ops, s) : launch_dense_l<256, 1>(ctx, a, ctx->dense_ops, s);
}

}  // namespace

// S split in two f16 terms, hi = S rounded to f16 and lo = the remainder S - hi rounded
// to f16 (about 22 bits of each fp32 value together; an absolute error below 2^-25 where
// lo falls in the f16 subnormal range), as two tiles (hi, then lo) in the swizzled K-major
// operand layout of the compression kernels. False if S holds a value that is not finite
// or lies beyond the f16 range (the tensor-core kernels are then not used).
bool pack_qjl_operand(const float* S, int m, int d, uint16_t* out) {
  if (m != 128 || d != 128) return false;
  constexpr size_t kTile = 128 * 128;
  for (int i = 0; i < m; ++i)
    for (int j = 0; j < d; ++j) {
      const float v = S[(size_t)i * d + j];
      if (!(std::fabs(v) <= 65504.f)) return false;
      const __half h = __float2half_rn(v);
      const __half l = __float2half_rn(v - __half2float(h));  // v - hi is exact in fp32
      const size_t off = tq::sm100::sw128_offset(i, j, 128) / 2;
      out[off] = __half_as_ushort(h);
      out[kTile + off] = __half_as_ushort(l);
    }
  return true;
}

// H diag(sigma) (Sylvester H[n][j] = (-1)^popcount(n & j), sigma_j = -1 where sign bit j is
// set) as bf16 +-1 in the swizzled K-major operand layout of compress_rot_kernel:
// element (n, j) multiplies key coordinate j into rotated coordinate n.
void pack_hadamard_operand(const uint32_t* sign_bits, uint16_t* out) {
  for (int n = 0; n < 128; ++n)
    for (int j = 0; j < 128; ++j) {
      bool neg = (__builtin_popcount((unsigned)(n & j)) & 1) != 0;
      if ((sign_bits[j / 32] >> (j % 32)) & 1u) neg = !neg;
      out[tq::sm100::sw128_offset(n, j, 128) / 2] = neg ? 0xBF80u : 0x3F80u;  // bf16 -1, +1
    }
}

namespace {
uint16_t bf16_rn(float x) {  // round to nearest even (finite inputs)
  uint32_t u;
  std::memcpy(&u, &x, 4);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}
float bf16_value(uint16_t h) {
  const uint32_t u = (uint32_t)h << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}
}  // namespace

// Operand tiles of compress_dense_kernel (d = 64 or 256, m = d): the rotation R as NT bf16
// terms (H diag(sigma) exact, NT = 1; the Haar matrix as three rounded remainders, NT = 3)
// and S as f16 hi + lo, cut into NW x NW tiles (NW = 64 at d = 64, 128 at d = 256) in the
// swizzled K-major layout: rotation tiles in (row chunk, column chunk, term) order, then S
// tiles in (row chunk, column chunk, hi / lo) order. Element (n, k) of a rotation tile
// multiplies key coordinate k into rotated coordinate n; of an S tile, residual coordinate k
// into projection n. False if S is not finite or beyond the f16 range.
bool pack_dense_operands(int d, int rot, const uint32_t* sign_bits, const double* haar, const float* S,
                         std::vector<uint16_t>& out) {
  if (d != 64 && d != 256) return false;
  const int NW = d == 256 ? 128 : 64, NCH = d / NW, NT = rot == TQ_ROT_HAAR ? 3 : 1;
  const size_t tile = (size_t)NW * NW;
  out.assign((size_t)NCH * NCH * (NT + 2) * tile, 0);
  size_t t_idx = 0;
  for (int nc = 0; nc < NCH; ++nc)
    for (int kc = 0; kc < NCH; ++kc)
      for (int t = 0; t < NT; ++t, ++t_idx)
        for (int n = 0; n < NW; ++n)
          for (int k = 0; k < NW; ++k) {
            const int gn = nc * NW + n, gk = kc * NW + k;
            uint16_t v;
            if (rot == TQ_ROT_HAAR) {
              double rem = haar[(size_t)gn * d + gk];
              uint16_t h = 0;
              for (int tt = 0; tt <= t; ++tt) {
                h = bf16_rn((float)rem);
                rem -= (double)bf16_value(h);
              }
              v = h;
            } else {
              bool neg = (__builtin_popcount((unsigned)(gn & gk)) & 1) != 0;
              if ((sign_bits[gk / 32] >> (gk % 32)) & 1u) neg = !neg;
              v = neg ? 0xBF80u : 0x3F80u;
            }
            out[t_idx * tile + tq::sm100::sw128_offset(n, k, NW) / 2] = v;
          }
  for (int nc = 0; nc < NCH; ++nc)
    for (int kc = 0; kc < NCH; ++kc, t_idx += 2)
      for (int n = 0; n < NW; ++n)
        for (int k = 0; k < NW; ++k) {
          const float v = S[(size_t)(nc * NW + n) * d + kc * NW + k];
          if (!(std::fabs(v) <= 65504.f)) return false;
          const __half h = __float2half_rn(v);
          const __half l = __float2half_rn(v - __half2float(h));
          const size_t off = tq::sm100::sw128_offset(n, k, NW) / 2;
          out[t_idx * tile + off] = __half_as_ushort(h);
          out[(t_idx + 1) * tile + off] = __half_as_ushort(l);
        }
  return true;
}

// Pi (fp64, row-major, d = 128) as three bf16 terms Pi ~ P1 + P2 + P3 (each the rounded
// remainder of the previous ones, about 24 bits together), three tiles in the swizzled
// K-major operand layout of compress_rot_kernel: element (n, j) multiplies key
// coordinate j into rotated coordinate n.
void pack_haar_operand(const double* pi, uint16_t* out) {
  for (int n = 0; n < 128; ++n)
    for (int j = 0; j < 128; ++j) {
      double rem = pi[(size_t)n * 128 + j];
      for (int t = 0; t < 3; ++t) {
        const uint16_t h = bf16_rn((float)rem);
        out[(size_t)t * 128 * 128 + tq::sm100::sw128_offset(n, j, 128) / 2] = h;
        rem -= (double)bf16_value(h);
      }
    }
}

cudaError_t launch_compress(const tq_ctx* ctx, const void* k, const void* v, int dtype, int64_t n_vec,
                            const int64_t* slot, int64_t n_rows, uint8_t* k_codes, uint8_t* k_signs,
                            uint16_t* k_norms, uint8_t* v_codes, uint16_t* v_params, cudaStream_t stream) {
  CompressArgs a;
  a.k = k;
  a.v = v;
  a.n_vec = n_vec;
  a.slot = slot;
  a.n_rows = n_rows;
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
  a.S_sw128 = ctx->S_sw128;
  a.H_sw128 = ctx->H_sw128;
  a.err = ctx->d_err;
  auto generic = [&](const CompressArgs& g) -> cudaError_t {
    switch (ctx->shape.d) {
      case 64: return launch_d<64>(ctx, g, dtype, stream);
      case 128: return launch_d<128>(ctx, g, dtype, stream);
      case 256: return launch_d<256>(ctx, g, dtype, stream);
    }
    return cudaErrorInvalidValue;
  };
  if (ctx->shape.lm_bits > 3) return generic(a);  // the tensor-core kernels take 1-3 Lloyd-Max bits
  if (ctx->dense_ops && (ctx->shape.d == 64 || ctx->shape.d == 256) && ctx->shape.m == ctx->shape.d &&
      dtype == TQ_BF16 && k) {
    // keys on the dense tensor-core kernel; values (if any) on the warp-per-vector kernel
    CompressArgs ka = a;
    ka.v = nullptr;
    if (!encode_rows_map(&ka.kmap, k, n_vec, 128, ctx->shape.d)) return generic(a);
    const cudaError_t e = launch_dense(ctx, ka, stream);
    if (e != cudaSuccess || !v) return e;
    CompressArgs va = a;
    va.k = nullptr;
    return generic(va);
  }
  // d = 128, bf16, a symmetric codebook, with the QJL stage (S on its operand tiles) or
  // without it: the pipelined tensor-core kernel. Values (value coding does not depend on the
  // keys' settings) run on its value warps, 2 to 4 bits, in the same launch as the keys with the
  // QJL stage and the Hadamard rotation, in a launch of their own otherwise; the records are the
  // same either way.
  const bool pipe_shape = ctx->shape.d == 128 && dtype == TQ_BF16 && codebook_symmetric(ctx->cb, ctx->shape.lm_bits) &&
                          ((ctx->shape.m == 128 && ctx->S_sw128) || ctx->shape.m == 0);
  const uint16_t* rot_tiles = ctx->shape.rot == TQ_ROT_HAAR ? ctx->Pi_sw128 : ctx->H_sw128;
  if (pipe_shape && rot_tiles && (!k || encode_rows_map(&a.kmap, k, n_vec, 128))) {
    a.H_sw128 = rot_tiles;
    const bool vmap_ok = v && encode_rows_map(&a.vmap, v, n_vec, 64);
    auto values_alone = [&]() -> cudaError_t {
      CompressArgs va = a;
      va.k = nullptr;
      return vmap_ok ? launch_pipe_nq(ctx, va, stream) : generic(va);
    };
    if (!k) return values_alone();
    if (ctx->shape.m == 128 && ctx->shape.rot == TQ_ROT_HADAMARD && (!v || vmap_ok))
      return launch_pipe(ctx, a, stream);  // keys and values in one launch
    CompressArgs ka = a;
    ka.v = nullptr;
    const cudaError_t e = ctx->shape.m == 0 ? launch_pipe_nq(ctx, ka, stream)
                          : ctx->shape.rot == TQ_ROT_HAAR ? launch_pipe_haar(ctx, ka, stream)
                                                          : launch_pipe(ctx, ka, stream);
    if (e != cudaSuccess || !v) return e;
    return values_alone();
  }
  if (ctx->shape.v_bits == 3 && k && v && ctx->S_sw128) {
    // 3-bit values on the warp-per-vector kernel, the keys alone on the tensor-core kernels
    CompressArgs vv = a;
    vv.k = nullptr;
    const cudaError_t e = launch_compress(ctx, k, nullptr, dtype, n_vec, slot, n_rows, k_codes, k_signs, k_norms,
                                          nullptr, nullptr, stream);
    return e != cudaSuccess ? e : generic(vv);
  }
  if (ctx->S_sw128 && ctx->shape.d == 128 && ctx->shape.m == 128 && !(ctx->shape.v_bits == 3 && v)) {
    // fp32 keys, a codebook that is not symmetric, or rows no tensor map takes
    if (ctx->shape.rot == TQ_ROT_HADAMARD && dtype == TQ_BF16 && ctx->H_sw128) return launch_rot<false>(ctx, a, stream);
    if (ctx->shape.rot == TQ_ROT_HAAR && dtype == TQ_BF16 && ctx->Pi_sw128) {
      a.H_sw128 = ctx->Pi_sw128;
      return launch_rot<true>(ctx, a, stream);
    }
    if (ctx->shape.rot == TQ_ROT_HADAMARD)
      return dtype == TQ_F32 ? launch_q4<float>(ctx, a, stream) : launch_q4<__nv_bfloat16>(ctx, a, stream);
    return dtype == TQ_F32 ? launch_tc<float>(ctx, a, stream) : launch_tc<__nv_bfloat16>(ctx, a, stream);
  }
  return generic(a);
}

}  // namespace tq
