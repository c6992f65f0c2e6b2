// Decode attention over the packed cache (one new query token per sequence).
//
// The pages describe decode as scoring every cached key directly from its
// compressed form ("turboquant-pytorch" skill card, "Что делает": asymmetric
// scores from compressed keys) inside fused kernels (discosf news item, the
// three fused decode kernels). Here:
//   1. qprep_kernel   qr = Pi q (sign flip + Walsh-Hadamard, or dense Haar),
//                     sq = S qr, once per query head;
//   2. decode_kernel  one CTA per (sequence x KV head, chunk of the cache):
//                     logits from the codebook inner products plus the QJL
//                     correction, online softmax, accumulation of the group-
//                     dequantized values; writes a partial (max, sum, acc);
//   3. combine_kernel log-sum-exp merge of the chunk partials (split-K).
// No kernel waits on another kernel's progress inside a launch.
#include <cuda_runtime.h>
#include <math.h>

#include "tq_device.cuh"

namespace tq {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 64;        // tokens per tile
constexpr int kSlices = kThreads / kTile;
constexpr int kMaxQ = 32;        // value accumulators per thread
constexpr int kPartPad = 4;      // floats before acc[] in a partial record

struct QPrepArgs {
  const void* q;
  int q_dtype;
  int d, m, rot;
  float inv_sqrt_d;
  const float* St;
  const float* PiT;
  Codebook cb;
  float* ws_q;
  int q_stride;
};

__global__ void __launch_bounds__(kThreads) qprep_kernel(const __grid_constant__ QPrepArgs a) {
  __shared__ float xs[kMaxD];
  __shared__ float qr[kMaxD];
  const int row = blockIdx.x, tid = threadIdx.x, d = a.d;
  if (tid < d) {
    float v = a.q_dtype == TQ_F32 ? static_cast<const float*>(a.q)[(size_t)row * d + tid]
                                  : __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[(size_t)row * d + tid]);
    if (a.rot == TQ_ROT_HADAMARD) v = flip_sign(v, (a.cb.sign_bits[tid / 32] >> (tid % 32)) & 1u);
    xs[tid] = v;
  }
  __syncthreads();
  if (a.rot == TQ_ROT_HADAMARD) {
    for (int h = 1; h < d; h <<= 1) {
      if (tid < d / 2) {
        const int i = (tid / h) * 2 * h + (tid % h);
        const float x0 = xs[i], x1 = xs[i + h];
        xs[i] = x0 + x1;
        xs[i + h] = x0 - x1;
      }
      __syncthreads();
    }
    if (tid < d) qr[tid] = xs[tid] * a.inv_sqrt_d;
  } else {
    if (tid < d) {
      float acc = 0.f;
      for (int j = 0; j < d; ++j) acc = fmaf(a.PiT[(size_t)j * d + tid], xs[j], acc);
      qr[tid] = acc;
    }
  }
  __syncthreads();
  float* out = a.ws_q + (size_t)row * a.q_stride;
  if (tid < d) out[tid] = qr[tid];
  if (tid < a.m) {
    float acc = 0.f;
    for (int j = 0; j < d; ++j) acc = fmaf(a.St[(size_t)j * a.m + tid], qr[j], acc);
    out[d + tid] = acc;
  }
}

struct DecodeArgs {
  const float* ws_q;
  int q_stride;
  const uint8_t* k_codes;
  const uint8_t* k_signs;
  const uint16_t* k_norms;
  const uint8_t* v_codes;
  const uint16_t* v_params;
  const int32_t* seq_lens;
  int64_t max_len;
  Paging pg;           // contiguous or paged cache addressing
  unsigned int* err;   // device error word (bit 2: a page index out of range)
  int hq, hkv, G, m;
  int n_chunks;
  int64_t chunk_len;
  float scale;
  float* scores;
  float* ws_part;
  int part_stride;
  Codebook cb;
};

template <int D, int LMB, int VB>
__global__ void __launch_bounds__(kThreads) decode_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int KW = LMB * D / 32;   // code words per key
  static_assert(KW % LMB == 0, "a key holds whole 32-code groups");
  constexpr int VW = VB * D / 32;    // code words per value
  constexpr int NG = D / kVGroup;    // value groups
  constexpr int HS = kThreads / D;   // head slices in the value phase
  const int G = a.G, M = a.m, SW = M / 32;

  extern __shared__ float smem[];
  float* qr_s = smem;                       // [D][G]
  float* sq_s = qr_s + D * G;               // [M][G]
  float* score_s = sq_s + M * G;            // [G][kTile]
  float* m_s = score_s + G * kTile;         // [G]
  float* l_s = m_s + G;                     // [G]
  float* corr_s = l_s + G;                  // [G]
  float* sqsum_s = corr_s + G;              // [G]
  uint32_t* vcode_s = reinterpret_cast<uint32_t*>(sqsum_s + G);  // [kTile][VW]
  uint32_t* vpar_s = vcode_s + kTile * VW;                         // [kTile][NG]
  float* cb_s = reinterpret_cast<float*>(vpar_s + kTile * NG);     // [2^LMB] centroids (LMB >= 4)

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = blockIdx.x, unit = blockIdx.y;
  const int b = unit / a.hkv, kvh = unit % a.hkv;
  int64_t len = a.max_len;
  if (a.seq_lens) len = min((int64_t)max(a.seq_lens[b], 0), a.max_len);
  const int64_t t0 = (int64_t)chunk * a.chunk_len;
  const int64_t t1 = min(t0 + a.chunk_len, len);
  const int qrow0 = b * a.hq + kvh * G;

  for (int idx = tid; idx < G * D; idx += kThreads) {
    const int h = idx / D, j = idx % D;
    qr_s[j * G + h] = a.ws_q[(size_t)(qrow0 + h) * a.q_stride + j];
  }
  for (int idx = tid; idx < G * M; idx += kThreads) {
    const int h = idx / M, i = idx % M;
    sq_s[i * G + h] = a.ws_q[(size_t)(qrow0 + h) * a.q_stride + D + i];
  }
  if constexpr (LMB >= 4)
    for (int k = tid; k < (1 << LMB); k += kThreads) cb_s[k] = a.cb.c[k];
  for (int h = tid; h < G; h += kThreads) {
    m_s[h] = -INFINITY;
    l_s[h] = 0.f;
  }
  __syncthreads();
  for (int h = warp; h < G; h += kThreads / 32) {
    float s = 0.f;
    for (int i = lane; i < M; i += 32) s += sq_s[i * G + h];
    s = warp_sum(s);
    if (lane == 0) sqsum_s[h] = s;
  }
  __syncthreads();

  const int vj = tid % D, vhs = tid / D;
  const int nq = (G - vhs + HS - 1) / HS;
  float acc[kMaxQ];
#pragma unroll
  for (int q = 0; q < kMaxQ; ++q) acc[q] = 0.f;

  const float qjl = M > 0 ? kQjl / (float)M : 0.f;  // M = 0: no QJL stage
  for (int64_t tt = t0; tt < t1; tt += kTile) {
    const int nt = (int)min((int64_t)kTile, t1 - tt);
    const int64_t row0 = record_row(a.pg, a.max_len, unit, tt, a.err);  // the tile's first record
    // Stage this tile's value codes and (scale, min) pairs.
    const uint32_t* vsrc = reinterpret_cast<const uint32_t*>(a.v_codes + row0 * (VW * 4));
    for (int w = tid; w < nt * VW; w += kThreads) vcode_s[w] = vsrc[w];
    const uint32_t* psrc = reinterpret_cast<const uint32_t*>(a.v_params) + row0 * NG;
    for (int w = tid; w < nt * NG; w += kThreads) vpar_s[w] = psrc[w];

    // Logits: thread (token tl, slice sl) scores heads sl, sl + kSlices, ...
    const int tl = tid % kTile, sl = tid / kTile;
    if (tl < nt) {
      const int64_t vec = row0 + tl;
      const uint32_t* ksrc = reinterpret_cast<const uint32_t*>(a.k_codes + vec * (KW * 4));
      uint32_t sw[kMaxM / 32];
      const uint32_t* ssrc = reinterpret_cast<const uint32_t*>(a.k_signs + vec * (M / 8));
#pragma unroll
      for (int w = 0; w < kMaxM / 32; ++w) sw[w] = w < SW ? ssrc[w] : 0u;
      const uint32_t nb = reinterpret_cast<const uint32_t*>(a.k_norms)[vec];
      const float n = __half2float(__ushort_as_half((unsigned short)(nb & 0xffffu)));
      const float gamma = __half2float(__ushort_as_half((unsigned short)(nb >> 16)));
      for (int h0 = sl; h0 < G; h0 += 4 * kSlices) {
        float al[4] = {0.f, 0.f, 0.f, 0.f}, as[4] = {0.f, 0.f, 0.f, 0.f};
        // 32 consecutive codes occupy exactly LMB words; walk the key 32 codes at a time.
        for (int g32 = 0; g32 < D / 32; ++g32) {
          uint32_t kw[LMB];
#pragma unroll
          for (int w = 0; w < LMB; ++w) kw[w] = ksrc[g32 * LMB + w];
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const uint32_t code = stream_code<LMB>(kw, jj);
            float cv;
            if constexpr (LMB >= 4) {
              cv = cb_s[code];  // many levels: a table in shared memory
            } else {
              cv = a.cb.c[0];
#pragma unroll
              for (int k = 1; k < (1 << LMB); ++k) cv = (code == (uint32_t)k) ? a.cb.c[k] : cv;
            }
            const float* qrow = qr_s + (g32 * 32 + jj) * G;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int h = h0 + u * kSlices;
              if (h < G) al[u] = fmaf(qrow[h], cv, al[u]);
            }
          }
        }
#pragma unroll
        for (int w = 0; w < kMaxM / 32; ++w) {
          if (w < SW) {
            const uint32_t bits = sw[w];
#pragma unroll 4
            for (int bb = 0; bb < 32; ++bb) {
              if ((bits >> bb) & 1u) {
                const float* row = sq_s + (w * 32 + bb) * G;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const int h = h0 + u * kSlices;
                  if (h < G) as[u] += row[h];
                }
              }
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int h = h0 + u * kSlices;
          if (h < G) {
            const float l = a.scale * n * (al[u] + qjl * gamma * (2.f * as[u] - sqsum_s[h]));
            score_s[h * kTile + tl] = l;
            if (a.scores) a.scores[(size_t)(qrow0 + h) * a.max_len + tt + tl] = l;
          }
        }
      }
    } else {
      for (int h = sl; h < G; h += kSlices) score_s[h * kTile + tl] = -INFINITY;
    }
    __syncthreads();

    // Online softmax over the tile, one warp per head.
    for (int h = warp; h < G; h += kThreads / 32) {
      const float v0 = score_s[h * kTile + lane], v1 = score_s[h * kTile + lane + 32];
      const float tmax = warp_max(fmaxf(v0, v1));
      const float m_old = m_s[h];
      const float m_new = fmaxf(m_old, tmax);
      const float corr = (m_old == -INFINITY) ? 0.f : expf(m_old - m_new);
      const float p0 = expf(v0 - m_new), p1 = expf(v1 - m_new);
      score_s[h * kTile + lane] = p0;
      score_s[h * kTile + lane + 32] = p1;
      const float ps = warp_sum(p0 + p1);
      if (lane == 0) {
        l_s[h] = l_s[h] * corr + ps;
        m_s[h] = m_new;
        corr_s[h] = corr;
      }
    }
    __syncthreads();

    // Values: thread (coordinate vj, head slice vhs).
#pragma unroll
    for (int q = 0; q < kMaxQ; ++q)
      if (q < nq) acc[q] *= corr_s[vhs + q * HS];
    const int g = vj / kVGroup;
    const int wsel = (vj * VB) >> 5, shift = (vj * VB) & 31;
    for (int t = 0; t < nt; ++t) {
      uint32_t code = vcode_s[t * VW + wsel] >> shift;
      if (VB == 3 && shift > 29) code |= vcode_s[t * VW + wsel + 1] << (32 - shift);  // straddles two words
      code &= (1u << VB) - 1u;
      const uint32_t par = vpar_s[t * NG + g];
      const float sc = __half2float(__ushort_as_half((unsigned short)(par & 0xffffu)));
      const float lo = __half2float(__ushort_as_half((unsigned short)(par >> 16)));
      const float val = fmaf(sc, (float)code, lo);
#pragma unroll
      for (int q = 0; q < kMaxQ; ++q)
        if (q < nq) acc[q] = fmaf(score_s[(vhs + q * HS) * kTile + t], val, acc[q]);
    }
    __syncthreads();
  }

  // Partial record per (unit, chunk, head): [m, l, -, -, acc[0..D)].
#pragma unroll
  for (int q = 0; q < kMaxQ; ++q) {
    if (q < nq) {
      const int h = vhs + q * HS;
      float* part = a.ws_part + ((size_t)(unit * a.n_chunks + chunk) * G + h) * a.part_stride;
      part[kPartPad + vj] = acc[q];
      if (vj == 0) {
        part[0] = m_s[h];
        part[1] = l_s[h];
      }
    }
  }
}

struct CombineArgs {
  const float* ws_part;
  int part_stride, n_chunks, G, hq, hkv, d;
  float* out;
  float* lse;  // null, or the log of each row's softmax denominator
};

__global__ void __launch_bounds__(kThreads) combine_kernel(const __grid_constant__ CombineArgs a) {
  const int row = blockIdx.x;  // b * hq + query head
  const int b = row / a.hq, hg = row % a.hq;
  const int unit = b * a.hkv + hg / a.G, h = hg % a.G;
  const float* base = a.ws_part + ((size_t)unit * a.n_chunks * a.G + h) * a.part_stride;
  const size_t cstride = (size_t)a.G * a.part_stride;
  float mx = -INFINITY;
  for (int c = 0; c < a.n_chunks; ++c) mx = fmaxf(mx, base[c * cstride]);
  for (int j = threadIdx.x; j < a.d; j += blockDim.x) {
    float num = 0.f, den = 0.f;
    if (mx != -INFINITY) {
      for (int c = 0; c < a.n_chunks; ++c) {
        const float* p = base + c * cstride;
        const float w = (p[0] == -INFINITY) ? 0.f : expf(p[0] - mx);
        den = fmaf(w, p[1], den);
        num = fmaf(w, p[kPartPad + j], num);
      }
    }
    a.out[(size_t)row * a.d + j] = den > 0.f ? num / den : 0.f;
    if (a.lse && j == 0) a.lse[row] = den > 0.f ? mx + logf(den) : -INFINITY;
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t decode_smem_bytes(int d, int m, int G, int vbits) {
  const int vw = vbits * d / 32, ng = d / kVGroup;
  return sizeof(float) * ((size_t)d * G + (size_t)m * G + (size_t)G * kTile + 4 * (size_t)G) +
         sizeof(uint32_t) * ((size_t)kTile * vw + (size_t)kTile * ng) + sizeof(float) * kMaxLevels;
}

template <int D, int LMB, int VB>
cudaError_t launch_main(const DecodeArgs& a, dim3 grid, size_t smem, cudaStream_t s) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, LMB, VB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  decode_kernel<D, LMB, VB><<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <int D, int LMB>
cudaError_t dispatch_vb(const DecodeArgs& a, int vb, dim3 grid, size_t smem, cudaStream_t s) {
  if (vb == 3) return launch_main<D, LMB, 3>(a, grid, smem, s);
  return vb == 2 ? launch_main<D, LMB, 2>(a, grid, smem, s) : launch_main<D, LMB, 4>(a, grid, smem, s);
}

template <int D>
cudaError_t dispatch_lmb(const DecodeArgs& a, int lmb, int vb, dim3 grid, size_t smem, cudaStream_t s) {
  switch (lmb) {
    case 1: return dispatch_vb<D, 1>(a, vb, grid, smem, s);
    case 2: return dispatch_vb<D, 2>(a, vb, grid, smem, s);
    case 3: return dispatch_vb<D, 3>(a, vb, grid, smem, s);
    case 4: return dispatch_vb<D, 4>(a, vb, grid, smem, s);
  }
  if constexpr (D <= 128) {  // more bits than 32 / (D / 32) do not fit a lane's code word at D = 256
    switch (lmb) {
      case 5: return dispatch_vb<D, 5>(a, vb, grid, smem, s);
      case 6: return dispatch_vb<D, 6>(a, vb, grid, smem, s);
      case 7: return dispatch_vb<D, 7>(a, vb, grid, smem, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace

DecodePlan plan_decode(const tq_ctx* ctx, int batch, int hq, int hkv, int64_t max_len) {
  DecodePlan p{};
  const int d = ctx->shape.d, m = ctx->shape.m, G = hq / hkv;
  // TQ_DECODE_AUTO: mma.sync where it applies (1- to 3-bit codes with the QJL stage, the
  // faster of the two tensor-core kernels on those shapes), then tcgen05 (keys without the
  // QJL stage), then the generic kernels. A family selected explicitly runs or the call is
  // refused.
  const bool tc_ok = tc_decode_supported(ctx, G), mma_ok = mma_decode_supported(ctx, G);
  p.supported = true;
  switch (ctx->decode_kernel) {
    case TQ_DECODE_TCGEN05: p.tc = tc_ok; p.supported = tc_ok; break;
    case TQ_DECODE_MMA: p.mma = mma_ok; p.supported = mma_ok; break;
    case TQ_DECODE_CUDA_CORE: break;
    default: p.mma = mma_ok; p.tc = !mma_ok && tc_ok; break;
  }
  p.family = p.tc ? TQ_DECODE_TCGEN05 : p.mma ? TQ_DECODE_MMA : TQ_DECODE_CUDA_CORE;
  if (!p.supported) return p;
  const int64_t units = (int64_t)batch * hkv;
  const int64_t sms = ctx->num_sms > 0 ? ctx->num_sms : 148;
  if (p.tc) {
    // As below, with 128-token tiles (the MMA's M) and one CTA per SM.
    const int64_t tile = 128;
    const int64_t Tu = max_len > 0 ? (max_len + tile - 1) / tile : 1;
    const int64_t Tt = units * Tu;
    const int64_t P = Tt < sms ? Tt : sms;
    p.n_ctas = (int)P;
    p.tiles_per_unit = Tu;
    p.total_tiles = Tt;
    int64_t s_max = 1;
    for (int64_t u = 0; u < units; ++u) {
      const int64_t first = ((u * Tu + 1) * P - 1) / Tt, last = ((u + 1) * Tu * P - 1) / Tt;
      if (last - first + 1 > s_max) s_max = last - first + 1;
    }
    p.s_max = (int)s_max;
    // one partial per warp group of every CTA that shares a unit
    p.ws_part_bytes = align256((size_t)units * s_max * tc_groups(ctx, G) * G * (d + kPartPad) * sizeof(float));
    p.off_frag = 0;
    p.off_part = align256((size_t)units * tc_operand_bytes(ctx, G));
    p.off_cnt = p.off_part + p.ws_part_bytes;
    p.total_bytes = p.off_cnt;
    return p;
  }
  if (p.mma) {
    // Every unit (sequence x KV head) is cut into tiles; the tiles that hold tokens, of all
    // units laid end to end, are split evenly over one wave of resident CTAs (one per SM),
    // by the kernel itself from the lengths on the device. A CTA's range may cross unit
    // boundaries; each unit is merged from the partials of the CTAs that share it, CTA k's
    // partial of unit u in slot u + k (at most units + CTAs slots). The grid is sized for
    // every sequence at max_len.
    const int64_t tile = mma_tile_tokens(G);
    const int64_t Tu = max_len > 0 ? (max_len + tile - 1) / tile : 1;
    const int64_t Tt = units * Tu;
    const int64_t slots = (int64_t)mma_ctas_per_sm(ctx->shape.lm_bits, ctx->shape.v_bits, G) * sms;
    const int64_t P = Tt < slots ? Tt : slots;
    p.n_ctas = (int)P;
    p.tiles_per_unit = Tu;
    p.total_tiles = Tt;
    p.s_max = 0;
    p.n_chunks = 0;
    p.chunk_len = 0;
    p.ws_q_bytes = 0;
    p.ws_part_bytes = align256((size_t)(units + P) * G * (d + kPartPad) * sizeof(float));
    p.off_frag = 0;
    p.off_part = align256((size_t)units * mma_frag_bytes(ctx->shape.lm_bits, G));
    // then, for calls with lengths, each sequence's first tile in the split order and the
    // total ([batch + 1] int64, written by the decode grid for the combine kernel)
    p.off_cnt = p.off_part + p.ws_part_bytes;
    p.total_bytes = p.off_cnt + align256((size_t)(batch + 1) * sizeof(int64_t));
    return p;
  }
  const int64_t tiles = max_len > 0 ? (max_len + kTile - 1) / kTile : 1;
  const int64_t target = 4 * sms;  // a few waves of resident CTAs
  int64_t chunks = units > 0 ? (target + units - 1) / units : 1;
  if (chunks > tiles) chunks = tiles;
  if (chunks < 1) chunks = 1;
  const int64_t tiles_per_chunk = (tiles + chunks - 1) / chunks;
  p.chunk_len = tiles_per_chunk * kTile;
  p.n_chunks = (int)((tiles + tiles_per_chunk - 1) / tiles_per_chunk);
  p.ws_part_bytes = align256((size_t)units * p.n_chunks * G * (d + kPartPad) * sizeof(float));
  const int q_stride = d + m;
  p.ws_q_bytes = align256((size_t)batch * hq * q_stride * sizeof(float));
  p.total_bytes = p.ws_q_bytes + p.ws_part_bytes;
  return p;
}

cudaError_t launch_decode(const tq_ctx* ctx, const DecodePlan& plan, const void* q, int q_dtype, int batch,
                          int hq, int hkv, const int32_t* seq_lens, int64_t max_len, const Paging& pg,
                          const uint8_t* k_codes,
                          const uint8_t* k_signs, const uint16_t* k_norms, const uint8_t* v_codes,
                          const uint16_t* v_params, float scale, float* scores, float* out, float* lse,
                          void* workspace, cudaStream_t stream) {
  const int d = ctx->shape.d, m = ctx->shape.m, G = hq / hkv;
  if (plan.tc)
    return launch_decode_tc(ctx, plan, q, q_dtype, batch, hq, hkv, seq_lens, max_len, pg, k_codes, k_signs,
                            k_norms, v_codes, v_params, scale, scores, out, lse, workspace, stream);
  if (plan.mma)
    return launch_decode_mma(ctx, plan, q, q_dtype, batch, hq, hkv, seq_lens, max_len, pg, k_codes, k_signs,
                             k_norms, v_codes, v_params, scale, scores, out, lse, workspace, stream);
  if ((G + (kThreads / d) - 1) / (kThreads / d) > kMaxQ) return cudaErrorInvalidValue;
  float* ws_q = static_cast<float*>(workspace);
  float* ws_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + plan.ws_q_bytes);

  QPrepArgs qa;
  qa.q = q;
  qa.q_dtype = q_dtype;
  qa.d = d;
  qa.m = m;
  qa.rot = ctx->shape.rot;
  qa.inv_sqrt_d = (float)(1.0 / sqrt((double)d));
  qa.St = ctx->St;
  qa.PiT = ctx->PiT;
  qa.cb = ctx->cb;
  qa.ws_q = ws_q;
  qa.q_stride = d + m;
  qprep_kernel<<<batch * hq, kThreads, 0, stream>>>(qa);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  DecodeArgs a;
  a.ws_q = ws_q;
  a.q_stride = d + m;
  a.k_codes = k_codes;
  a.k_signs = k_signs;
  a.k_norms = k_norms;
  a.v_codes = v_codes;
  a.v_params = v_params;
  a.seq_lens = seq_lens;
  a.max_len = max_len;
  a.pg = pg;
  a.err = ctx->d_err;
  a.hq = hq;
  a.hkv = hkv;
  a.G = G;
  a.m = m;
  a.n_chunks = plan.n_chunks;
  a.chunk_len = plan.chunk_len;
  a.scale = scale;
  a.scores = scores;
  a.ws_part = ws_part;
  a.part_stride = d + kPartPad;
  a.cb = ctx->cb;
  const dim3 grid(plan.n_chunks, batch * hkv);
  const size_t smem = decode_smem_bytes(d, m, G, ctx->shape.v_bits);
  if (ctx->prof_start) cudaEventRecord(ctx->prof_start, stream);
  switch (d) {
    case 64: e = dispatch_lmb<64>(a, ctx->shape.lm_bits, ctx->shape.v_bits, grid, smem, stream); break;
    case 128: e = dispatch_lmb<128>(a, ctx->shape.lm_bits, ctx->shape.v_bits, grid, smem, stream); break;
    case 256: e = dispatch_lmb<256>(a, ctx->shape.lm_bits, ctx->shape.v_bits, grid, smem, stream); break;
    default: return cudaErrorInvalidValue;
  }
  if (ctx->prof_stop) cudaEventRecord(ctx->prof_stop, stream);
  if (e != cudaSuccess) return e;

  CombineArgs ca;
  ca.ws_part = ws_part;
  ca.part_stride = d + kPartPad;
  ca.n_chunks = plan.n_chunks;
  ca.G = G;
  ca.hq = hq;
  ca.hkv = hkv;
  ca.d = d;
  ca.out = out;
  ca.lse = lse;
  combine_kernel<<<batch * hq, d, 0, stream>>>(ca);
  return cudaGetLastError();
}

}  // namespace tq
