// Tensor-core decode attention over the packed cache (d = m = 128, up to 8 query
// heads per KV head, 1- to 3-bit Lloyd-Max keys of a symmetric codebook, 2- to 4-bit values).
//
// Same mathematics as decode_kernel (the skill card "turboquant-pytorch", "Что
// делает": scores straight from the compressed keys; the discosf news item:
// fused decode kernels): logit = scale * n * (<qr, c[idx]> + sqrt(pi/2)/m * gamma *
// <sq, s>), online softmax, sum of p * (min + scale * code). What changes is how
// the per-token work is spread: with G query heads sharing a KV head, the three
// contractions (key bits x query, signs x S q, value codes x probabilities) are
// small dense products over a tile of tokens, so they run on the tensor cores
// (warp-level mma.sync) instead of G scalar loops.
//
// Scores (mma.sync m16n8k32, u8 x s8 -> s32): rows = 16 tokens, columns = 2 query heads x 4
// signed 8-bit digits of each key bit's weight (31 bits together, as fine as the fp32 weights;
// the int32 sums are exact and recombined in fp32), so 4 heads take two n-blocks.
//  * A symmetric codebook is affine in the code's bits: c[b0 + 2 b1] = c0 + (c1 - c0) b0 +
//    (c2 - c0) b1 at 2 bits; at 3 bits the odd part also holds the product of the three signs,
//    affine in the parity b0 ^ b1 ^ b2 (one parity word per 32 codes, built by each lane from
//    three stream words). So <qr, c[idx]> = kappa sum(qr) + sum over bits of (beta_plane *
//    qr_j) * bit: every packed bit, codes, parities and signs alike, is one operand element.
//  * Mask q of a packed word keeps bit q mod 4 of each of its four bytes (of the word shifted
//    right by 4 for q >= 4): four u8 elements worth 2^(q mod 4) or 0 in one AND; the weights
//    are divided by that power of two.
// Values (mma.sync m16n8k16, f16 operands, fp32 accumulation): rows = 16 value coordinates,
// K = 16 tokens, columns = 4 query heads x (hi, lo), the two f16 halves of p * scale.
//  * A value code placed in the mantissa bits of an f16 is a subnormal equal to
//    code * 2^(pos - 24), so a byte permute, a shift and a mask yield two exact
//    operands; the power of two is undone once at the end. The codes sit at bit 4 or
//    higher (6 and up at 2 and 3 bits): products of codes at the lowest positions with
//    the small low parts of p * scale lost about 1e-4 of the output on the tensor cores.
//
// Kernels:
//  * prep_mma_kernel, one CTA per (sequence, KV head): rotates the G queries
//    (sign flip + Walsh-Hadamard butterflies, or the dense Haar matrix), forms
//    S qr, and writes that KV head's query operand fragments once.
//  * decode_mma_kernel, one 16-warp CTA per SM, launched with programmatic
//    dependent launch: the tiles that hold tokens, of all (sequence, KV head) units
//    laid end to end, are split evenly over the CTAs (each CTA finds its range from
//    the sequence lengths on the device), so a CTA's range may start and end inside a
//    unit and may span several, and a batch of varied lengths costs the tokens it
//    holds. It starts streaming its cache tiles (cp.async.bulk
//    into a ring of stages, mbarrier completion) while the prep kernel finishes,
//    then waits for the fragments of its first units (two operand buffers, refilled
//    by bulk copy at each unit boundary). Each warp owns 16 or 32 consecutive tokens
//    of each tile: it scores them, runs the online softmax for its heads and
//    accumulates their values. At a unit boundary the 16 warps merge their partials
//    in a fixed order and the CTA writes one partial (m, l, acc) of the unit.
//  * combine_mma_kernel, a programmatic dependent of the decode grid: merges the
//    partials of the CTAs that shared a unit (log-sum-exp) and writes the output
//    rows (and, for a partial decode, each row's log-partition).
// Every wait is bounded; a timeout sets the context's error word and ends the CTA.
#include <cuda_runtime.h>
#include <math.h>

#include "tq_device.cuh"

namespace tq {
namespace {

constexpr int kD = 128;
constexpr int kM = 128;
constexpr int kWarpsMma = 16;  // warps per decode CTA (one CTA per SM)
constexpr int kThreadsMma = kWarpsMma * 32;
constexpr int kPartPadMma = 4;
constexpr int kPrepThreads = 256;
// Base-2 slack of the lazy online-softmax rescale: probabilities stay below 2^kSlack,
// so p * scale fits fp16 for any value-group scale below 65504 / 2^kSlack = 16376.
constexpr float kSlack = 2.f;
constexpr uint32_t kWaitLimit = 1u << 24;                 // polls of one mbarrier phase
constexpr unsigned long long kWaitNs = 2000000000ull;    // and at most 2 s of wall time

// 32-bit words of key bits per token (code stream, then signs). The score MMAs
// (m16n8k32, u8 x s8) take one k-step of 32 elements per word and lane column: lane column
// c of k-step s holds masks 2 (s mod 4) and 2 (s mod 4) + 1 of word c + 4 (s / 4).
__host__ __device__ constexpr int code_words(int lmb) { return 4 * lmb; }
__host__ __device__ constexpr int par_words(int lmb) { return lmb == 3 ? 4 : 0; }  // parities of 3-bit codes
__host__ __device__ constexpr int key_words(int lmb) { return code_words(lmb) + par_words(lmb) + kM / 32; }
__host__ __device__ constexpr int key_steps(int lmb) { return 2 * key_words(lmb); }  // k-steps x 2 n-blocks
// n-blocks of 8 operand columns (4 heads x hi/lo) for G query heads.
__host__ __device__ constexpr int n_blocks(int G) { return G <= 4 ? 1 : 2; }
// 16-token row blocks per warp and tile (fewer when two n-blocks need the registers).
__host__ __device__ constexpr int m_blocks(int nb) { return nb == 1 ? 2 : 1; }
__host__ __device__ constexpr int tile_tokens(int nb) { return 16 * kWarpsMma * m_blocks(nb); }
// Per (sequence, KV head): query operand words [k-step][digit n-block][32 lanes][2] (two
// digit n-blocks per block of 4 heads), then [8 heads][4] logit constants (k1..k4 of the
// decode kernel).
__host__ __device__ constexpr int frag_words(int lmb, int nb) { return key_steps(lmb) * nb * 64 + 32; }

struct PrepArgs {
  const void* q;
  int q_dtype;
  int hq, hkv, G, rot;
  float inv_sqrt_d;
  const float* St;   // [d][m]
  const float* PiT;  // [d][d] (Haar)
  Codebook cb;
  float kappa;       // c[idx] = kappa + sum_p beta[p] bit_p (bit 3: the parity of 3-bit codes)
  float beta[4];
  float sl2;         // softmax scale * log2(e)
  int nb;            // n-blocks of the query operand
  uint32_t* frag;    // [units][frag_words]
};

struct MmaArgs {
  const uint32_t* frag;
  const uint8_t* k_codes;
  const uint8_t* k_signs;
  const uint16_t* k_norms;
  const uint8_t* v_codes;
  const uint16_t* v_params;
  const int32_t* seq_lens;
  int64_t max_len;
  Paging pg;               // contiguous or paged cache addressing
  int batch, hq, hkv, G;
  float* scores;
  float* out;
  float* ws_part;          // [units + CTAs][G][kPartPadMma + d]: CTA k's partial of unit u in slot u + k
  int64_t* seq_first;      // with lengths: [batch + 1] first tile of each sequence, then Tv (CTA 0 writes)
  int use_tma;             // 1 when every record array offset is 16-byte aligned
  unsigned int* err;       // device error word of the context
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on an mbarrier phase (poll count and wall time). Returns false if
// the phase did not complete within the bound.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  unsigned long long start = 0;
  for (uint32_t it = 0; it < kWaitLimit; ++it) {
    uint32_t done;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
    if (it == 0) start = global_ns();
    else if ((it & 255) == 0 && global_ns() - start > kWaitNs) return false;
  }
  return false;
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

// D (s32) += A (u8) x B (s8), m16n8k32, A row-major, B column-major.
__device__ __forceinline__ void mma_i8(int (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float2 unpack_h2(uint32_t w) {
  return __half22float2(*reinterpret_cast<const __half2*>(&w));
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<const uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t w) { return *reinterpret_cast<const __half2*>(&w); }

// 2^x with the hardware approximation (relative error about 2^-22); 2^-inf = 0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------------ prep kernel

// Copy a 128 x 128 fp32 matrix to shared memory: all 16 loads of a thread are
// issued before any store, so their latencies overlap.
__device__ __forceinline__ void stage_matrix(float* dst, const float* src, int tid) {
  constexpr int kPer = kD * kM / 4 / kPrepThreads;  // 16 float4 per thread
  const float4* s4 = reinterpret_cast<const float4*>(src);
  float4* d4 = reinterpret_cast<float4*>(dst);
  float4 v[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) v[u] = __ldg(s4 + tid + u * kPrepThreads);
#pragma unroll
  for (int u = 0; u < kPer; ++u) d4[tid + u * kPrepThreads] = v[u];
}

// HS: query-head slots worked on (4 for one n-block of heads, 8 for two).
template <int LMB, int HS>
__global__ void __launch_bounds__(kPrepThreads) prep_mma_kernel(const __grid_constant__ PrepArgs a) {
  // Let the dependent decode grid start streaming its cache tiles right away.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(16) float st_s[];  // [d][m] staged S^T (or Pi^T), 64 KB
  __shared__ float x_s[8 * kD];
  __shared__ float qr_s[8 * kD];
  __shared__ float sq_s[8 * kM];
  __shared__ float head_s[32];
  __shared__ float inv_s[16];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int unit = blockIdx.x;
  const int b = unit / a.hkv, kvh = unit % a.hkv, G = a.G;
  const int qrow0 = b * a.hq + kvh * G;

  {
    float v[HS * kD / kPrepThreads];
#pragma unroll
    for (int u = 0; u < HS * kD / kPrepThreads; ++u) {
      const int idx = tid + u * kPrepThreads, h = idx / kD, j = idx % kD;
      const size_t off = (size_t)(qrow0 + h) * kD + j;
      v[u] = 0.f;
      if (h < G)
        v[u] = a.q_dtype == TQ_F32 ? __ldg(static_cast<const float*>(a.q) + off)
                                   : __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[off]);
    }
#pragma unroll
    for (int u = 0; u < HS * kD / kPrepThreads; ++u) {
      const int idx = tid + u * kPrepThreads, j = idx % kD;
      float x = v[u];
      if (a.rot == TQ_ROT_HADAMARD) x = flip_sign(x, (a.cb.sign_bits[j / 32] >> (j % 32)) & 1u);
      x_s[idx] = x;
    }
  }
  __syncthreads();
  if (a.rot == TQ_ROT_HADAMARD) {
    for (int hs = 1; hs < kD; hs <<= 1) {
      for (int p = tid; p < HS * (kD / 2); p += kPrepThreads) {
        const int h = p / (kD / 2), i = p % (kD / 2);
        const int i0 = h * kD + (i / hs) * 2 * hs + (i % hs);
        const float u = x_s[i0], w = x_s[i0 + hs];
        x_s[i0] = u + w;
        x_s[i0 + hs] = u - w;
      }
      __syncthreads();
    }
    for (int idx = tid; idx < HS * kD; idx += kPrepThreads) qr_s[idx] = x_s[idx] * a.inv_sqrt_d;
  } else {
    stage_matrix(st_s, a.PiT, tid);
    __syncthreads();
    const int i = tid % kD, half = tid / kD;
    float acc[HS];
#pragma unroll
    for (int h = 0; h < HS; ++h) acc[h] = 0.f;
#pragma unroll 8
    for (int j = half * (kD / 2); j < (half + 1) * (kD / 2); ++j) {
      const float pv = st_s[j * kD + i];
#pragma unroll
      for (int h = 0; h < HS; ++h) acc[h] = fmaf(pv, x_s[h * kD + j], acc[h]);
    }
    if (half == 1)
#pragma unroll
      for (int h = 0; h < HS; ++h) sq_s[h * kD + i] = acc[h];  // scratch
    __syncthreads();
    if (half == 0)
#pragma unroll
      for (int h = 0; h < HS; ++h) qr_s[h * kD + i] = acc[h] + sq_s[h * kD + i];
    __syncthreads();  // st_s is reused for S^T below
  }
  __syncthreads();
  {
    // sq = S qr for the HS head slots at once. S^T is staged in shared memory with
    // independent 16-byte loads (its 64 KB would otherwise be read at L2 latency,
    // one dependent load per step); thread (i, half) then runs over half of j.
    stage_matrix(st_s, a.St, tid);
    __syncthreads();
    const int i = tid % kM, half = tid / kM;
    float acc[HS];
#pragma unroll
    for (int h = 0; h < HS; ++h) acc[h] = 0.f;
#pragma unroll 8
    for (int j = half * (kD / 2); j < (half + 1) * (kD / 2); ++j) {
      const float sv = st_s[j * kM + i];
#pragma unroll
      for (int h = 0; h < HS; ++h) acc[h] = fmaf(sv, qr_s[h * kD + j], acc[h]);
    }
    if (half == 1)
#pragma unroll
      for (int h = 0; h < HS; ++h) x_s[h * kM + i] = acc[h];
    __syncthreads();
    if (half == 0)
#pragma unroll
      for (int h = 0; h < HS; ++h) sq_s[h * kM + i] = acc[h] + x_s[h * kM + i];
  }
  __syncthreads();
  if (warp >= HS) {  // slots past HS: constants of an empty head (never read)
    if (lane < 4) head_s[warp * 4 + lane] = 0.f;
  } else {
    const int h = warp;  // one warp per head slot
    float qsum = 0.f, ssum = 0.f, qmax = 0.f, smax = 0.f;
    for (int j = lane; j < kD; j += 32) {
      qsum += qr_s[h * kD + j];
      ssum += sq_s[h * kM + j];
      qmax = fmaxf(qmax, fabsf(qr_s[h * kD + j]));
      smax = fmaxf(smax, fabsf(sq_s[h * kM + j]));
    }
    qsum = warp_sum(qsum);
    ssum = warp_sum(ssum);
    qmax = warp_max(qmax);
    smax = warp_max(smax);
    if (lane == 0) {
      const float bmax = fmaxf(fmaxf(fabsf(a.beta[0]), fabsf(a.beta[1])), fmaxf(fabsf(a.beta[2]), fabsf(a.beta[3])));
      const float qs = qmax * bmax > 0.f ? qmax * bmax : 1.f;  // LM operand scale
      const float ss = smax > 0.f ? smax : 1.f;                // sign operand scale
      // logit (base 2) = n * (k1 + k2 * lm + gamma * (k3 * sg - k4)), lm and sg being the
      // decode kernel's raw tensor-core sums over the normalised operands.
      constexpr float kSignW = kQjl / (float)kM;
      head_s[h * 4 + 0] = a.sl2 * a.kappa * qsum;
      head_s[h * 4 + 1] = a.sl2 * qs * (1.f / 1073741824.f);
      head_s[h * 4 + 2] = a.sl2 * kSignW * 2.f * ss * (1.f / 1073741824.f);
      head_s[h * 4 + 3] = a.sl2 * kSignW * ssum;
      inv_s[h * 2 + 0] = 1.f / qs;
      inv_s[h * 2 + 1] = 1.f / ss;
    }
  }
  __syncthreads();
  const int nb = a.nb;
  uint32_t* frag = a.frag + (size_t)unit * frag_words(LMB, nb);
  // Word (k-step s, digit n-block nbi, lane (r, c), register reg) holds four signed 8-bit B
  // elements of the m16n8k32 fragment: column r = head 4 (nbi / 2) + r / 2, digit 2 (nbi mod
  // 2) + r mod 2; rows 4c + i (register 0) or 4c + 16 + i (register 1). Row 4c + i of
  // register reg stands for bit 8i + q of key word c + 4 (s / 4), q = 2 (s mod 4) + reg,
  // which the decode lane's mask q turns into an element worth 2^(q mod 4). The weight of
  // that bit, normalised to [-1, 1] and divided by 2^(q mod 4), is Q = round(w 2^30) as four
  // balanced 8-bit digits (Q = d0 + 2^8 d1 + 2^16 d2 + 2^24 d3); column digit d carries d_d.
  const int nbi_n = 2 * nb;
  const int nwords = key_words(LMB) * nbi_n * 64;
  for (int w = tid; w < nwords; w += kPrepThreads) {
    const int reg = w & 1, ln = (w >> 1) & 31, blk = w >> 6;
    const int nbi = blk % nbi_n, kstep = blk / nbi_n;
    const int rr = ln >> 2, cc = ln & 3;
    const int head = 4 * (nbi >> 1) + (rr >> 1);
    const int digit = 2 * (nbi & 1) + (rr & 1);
    const int wi = cc + 4 * (kstep >> 2), q = 2 * (kstep & 3) + reg;
    uint32_t word = 0u;
    if (head < G) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int o = 8 * i + q;  // bit of the 32-bit key word
        float x;
        if (wi < code_words(LMB)) {
          const int sbit = 32 * wi + o;  // bit of the code stream: code sbit / LMB, plane sbit % LMB
          const int j = sbit / LMB, plane = sbit % LMB;
          x = qr_s[head * kD + j] * (a.beta[plane] * inv_s[head * 2 + 0]);
        } else if (wi < code_words(LMB) + par_words(LMB)) {
          // parity word pw, bit o: the parity of code 32 pw + (32 (o mod 3) + o) / 3
          const int j = 32 * (wi - code_words(LMB)) + (32 * (o % 3) + o) / 3;
          x = qr_s[head * kD + j] * (a.beta[3] * inv_s[head * 2 + 0]);
        } else {
          x = sq_s[head * kM + 32 * (wi - code_words(LMB) - par_words(LMB)) + o] * inv_s[head * 2 + 1];
        }
        const int Q = __float2int_rn(x * (1073741824.f / (float)(1 << (q & 3))));
        const int d0 = ((Q + 128) & 255) - 128;
        const int Q1 = (Q - d0) >> 8;
        const int d1 = ((Q1 + 128) & 255) - 128;
        const int Q2 = (Q1 - d1) >> 8;
        const int d2 = ((Q2 + 128) & 255) - 128;
        const int d3 = (Q2 - d2) >> 8;
        const int dd = digit == 0 ? d0 : digit == 1 ? d1 : digit == 2 ? d2 : d3;
        word |= ((uint32_t)dd & 0xffu) << (8 * i);
      }
    }
    frag[w] = word;
  }
  if (tid < 32) reinterpret_cast<float*>(frag)[nwords + tid] = head_s[tid];
}

// ------------------------------------------------------------------ decode kernel

template <int LMB, int VB, int NB>
struct Layout {
  static constexpr int MB = m_blocks(NB);
  static constexpr int TILE = tile_tokens(NB);
  static constexpr int KCB = LMB * kD / 8;  // key code bytes per token
  static constexpr int SB = kM / 8;         // sign bytes
  static constexpr int VCB = VB * kD / 8;   // value code bytes
  static constexpr int PB = (kD / kVGroup) * 4;
  static constexpr int REC = KCB + SB + 4 + VCB + PB;
  static constexpr int STAGE = TILE * REC;
  static constexpr int FRAG_BYTES = frag_words(LMB, NB) * 4;
  // As many stages (2..4) as fit in shared memory next to the two operand buffers and
  // the reduction area (one CTA per SM).
  static constexpr int RED_BYTES = (kWarpsMma * kD + 2 * kWarpsMma * 8 + 8) * 4;
  static constexpr int BUDGET = 227 * 1024 - 2 * FRAG_BYTES - RED_BYTES - 512;
  static constexpr int STAGES = 4 * STAGE <= BUDGET ? 4 : 3 * STAGE <= BUDGET ? 3 : 2;
  static constexpr int OFF_KC = 0;
  static constexpr int OFF_KS = OFF_KC + TILE * KCB;
  static constexpr int OFF_KN = OFF_KS + TILE * SB;
  static constexpr int OFF_VC = OFF_KN + TILE * 4;
  static constexpr int OFF_VP = OFF_VC + TILE * VCB;
  static constexpr int KS = key_steps(LMB);
  static constexpr int RING = STAGES * STAGE;
  static constexpr int OFF_FRAG = RING;                        // two query-operand buffers
  static constexpr int OFF_BAR = OFF_FRAG + 2 * FRAG_BYTES;    // STAGES + 2 mbarriers
  static constexpr int OFF_CNT = OFF_BAR + 8 * (STAGES + 2);   // arrive / issue counters
  static constexpr int OFF_PROD = OFF_CNT + 4 * (2 * STAGES + 4);  // the producer thread's unit walk
  static constexpr int OFF_RED = OFF_PROD + 48;                      // unit-boundary reduction
  static constexpr size_t SMEM = (size_t)OFF_RED + RED_BYTES;
  static_assert(STAGE % 16 == 0 && FRAG_BYTES % 16 == 0, "16-byte aligned stages and fragments");
  static_assert(SMEM <= 227 * 1024, "fits one CTA per SM");
};

__device__ __forceinline__ uint32_t word_of(const uint4& w, int i) {
  return i == 0 ? w.x : i == 1 ? w.y : i == 2 ? w.z : w.w;
}

// CTA owning global tile g when CTA k takes tiles [k T / P, (k + 1) T / P).
__device__ __forceinline__ int64_t tile_owner(int64_t g, int64_t P, int64_t T) { return ((g + 1) * P - 1) / T; }

// VARLEN: lengths given (seq_lens); otherwise every sequence holds max_len tokens, and the
// split below reduces to plain arithmetic on the tile index.
template <int LMB, int VB, int NB, bool VARLEN>
__global__ void __launch_bounds__(kThreadsMma, 1) decode_mma_kernel(const __grid_constant__ MmaArgs a) {
  using L = Layout<LMB, VB, NB>;
  constexpr int MB = L::MB, TILE = L::TILE, NST = L::STAGES;
  constexpr int RS = kPartPadMma + kD;
  constexpr float kLn2 = 0.6931471805599453f;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* stage_base = smem;
  unsigned char* frag_base = smem + L::OFF_FRAG;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);  // [NST] stages
  uint64_t* fbars = bars + NST;                                      // [2] query operands
  int* arrive_s = reinterpret_cast<int*>(smem + L::OFF_CNT);  // [NST] warps done with the stage's tile
  int* issued_s = arrive_s + NST;   // [NST] bulk-copy batches issued into the stage
  int* fissued_s = issued_s + NST;  // [2] copies issued into the operand buffer
  float* red_s = reinterpret_cast<float*>(smem + L::OFF_RED);  // [warps][d] one head's rescaled sums
  // Thread 0's walk over the units whose query operands it fetches: the last unit issued,
  // its tile 0 in the global order and its tiles, the CTA's range end, the units issued.
  struct ProducerWalk {
    int64_t fpre, fn, g1, pre0;
    int fu, fj;
    int cur_u;  // the unit whose partials the warps are accumulating
  };
  ProducerWalk* pw = reinterpret_cast<ProducerWalk*>(smem + L::OFF_PROD);
  float* rm_s = red_s + kWarpsMma * kD;                          // [warps][8] warp maxima
  float* rwl_s = rm_s + kWarpsMma * 8;                           // [warps][8] warp sums of p
  float* rM_s = rwl_s + kWarpsMma * 8;                           // [8] CTA maxima

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = lane >> 2, c = lane & 3;
  const int G = a.G, hkv = a.hkv;
  const int units = a.batch * hkv;
  const int64_t P = gridDim.x, kcta = blockIdx.x;

  if (tid == 0) {
    for (int s = 0; s < NST + 2; ++s) mbar_init(&bars[s], 1);
    for (int s = 0; s < 2 * NST + 4; ++s) arrive_s[s] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }

  const int64_t Tu = (a.max_len + TILE - 1) / TILE;  // tiles of a sequence at max_len
  auto seq_len = [&](int b) -> int64_t {
    if constexpr (VARLEN) return min((int64_t)max(a.seq_lens[b], 0), a.max_len);
    return a.max_len;
  };
  auto unit_len = [&](int u) -> int64_t { return seq_len(u / hkv); };
  auto unit_tiles = [&](int u) -> int {
    if constexpr (VARLEN) return (int)((unit_len(u) + TILE - 1) / TILE);
    return (int)Tu;
  };
  auto next_unit = [&](int u) -> int {  // the next unit after u that holds a token (or units)
    if constexpr (VARLEN) {
      do {
        ++u;
      } while (u < units && unit_tiles(u) == 0);
      return u;
    } else {
      return u + 1;
    }
  };
  // Split by the tokens present: the tiles that hold at least one token, of every unit (a
  // unit = one sequence x KV head) laid end to end, are split evenly over the CTAs, so a
  // batch of short and long sequences costs what its tokens cost. CTA k takes the tiles
  // [k Tv / P, (k + 1) Tv / P); its range may start and end inside a unit and span several.
  // Every CTA finds Tv and its first (unit, tile) from the lengths: a block-wide scan of
  // the per-sequence tile counts (the reduction area is free until the first unit ends).
  int64_t* scan_s = reinterpret_cast<int64_t*>(red_s);
  if constexpr (!VARLEN) {
    if (tid == 0) {
      const int64_t Tv = (int64_t)units * Tu, g0 = kcta * Tv / P, g1 = (kcta + 1) * Tv / P;
      scan_s[2 * kWarpsMma] = Tv;
      scan_s[2 * kWarpsMma + 4] = g1;
      if (g0 < g1) {
        scan_s[2 * kWarpsMma + 1] = g0 / Tu;
        scan_s[2 * kWarpsMma + 2] = g0 % Tu;
        scan_s[2 * kWarpsMma + 3] = g0 - g0 % Tu;
        scan_s[2 * kWarpsMma + 5] = a.max_len;
      }
    }
    __syncthreads();
  } else {
    const int per = (a.batch + kThreadsMma - 1) / kThreadsMma;
    const int b_lo = min(a.batch, tid * per), b_hi = min(a.batch, b_lo + per);
    int64_t mine = 0, len_lo = 0;  // len_lo: the length of sequence b_lo (kept: no L1 for reloads)
    for (int b = b_lo; b < b_hi; ++b) {
      const int64_t len = seq_len(b);
      if (b == b_lo) len_lo = len;
      mine += (len + TILE - 1) / TILE;
    }
    mine *= hkv;
    int64_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t t = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) scan_s[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int64_t w = lane < kWarpsMma ? scan_s[lane] : 0;
      int64_t wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t t = __shfl_up_sync(kFull, wi, o);
        if (lane >= o) wi += t;
      }
      if (lane < kWarpsMma) scan_s[kWarpsMma + lane] = wi - w;
      if (lane == 31) scan_s[2 * kWarpsMma] = wi;
    }
    __syncthreads();
    const int64_t Tv = scan_s[2 * kWarpsMma];
    const int64_t g0 = kcta * Tv / P, g1 = (kcta + 1) * Tv / P;
    const int64_t before = scan_s[kWarpsMma + warp] + incl - mine;  // tiles before sequence b_lo
    if (kcta == 0) {  // for the combine kernel: each sequence's first tile, and Tv
      int64_t acc = before;
      for (int b = b_lo; b < b_hi; ++b) {
        a.seq_first[b] = acc;
        acc += hkv * ((seq_len(b) + TILE - 1) / TILE);
      }
      if (tid == 0) a.seq_first[a.batch] = Tv;
    }
    if (g0 < g1 && before <= g0 && g0 < before + mine) {
      int64_t pre = before, len = len_lo;
      int b = b_lo;
      for (;;) {
        const int64_t t = hkv * ((len + TILE - 1) / TILE);
        if (g0 < pre + t) break;
        pre += t;
        len = seq_len(++b);
      }
      const int64_t nb_t = (len + TILE - 1) / TILE, off = g0 - pre;
      scan_s[2 * kWarpsMma + 1] = (int64_t)b * hkv + off / nb_t;         // first unit
      scan_s[2 * kWarpsMma + 2] = off % nb_t;                            // its first tile here
      scan_s[2 * kWarpsMma + 3] = pre + (off / nb_t) * nb_t;             // its tile 0, globally
      scan_s[2 * kWarpsMma + 5] = len;                                   // its length
    }
    scan_s[2 * kWarpsMma + 4] = g1;
    __syncthreads();
  }
  const int64_t Tv_all = scan_s[2 * kWarpsMma], g1 = scan_s[2 * kWarpsMma + 4];
  const int64_t g0 = kcta * Tv_all / P;
  const int ntl = (int)(g1 - g0);
  const int u0 = ntl > 0 ? (int)scan_s[2 * kWarpsMma + 1] : 0;
  const int tl0 = ntl > 0 ? (int)scan_s[2 * kWarpsMma + 2] : 0;
  const int64_t len0 = ntl > 0 ? scan_s[2 * kWarpsMma + 5] : 0;  // tokens of unit u0
  if (tid == 0) {
    pw->pre0 = ntl > 0 ? scan_s[2 * kWarpsMma + 3] : 0;
    pw->g1 = g1;
    pw->fj = 0;
  }
  __syncthreads();  // the reduction area is free again
  // One thread: start tile i. Every tile completes one phase of its stage's barrier:
  // a tile with 16-byte aligned records through its bulk copies, any other tile (and one
  // wholly past its sequence's end) through a plain arrival (its warps then copy it
  // themselves). The last tile of a sequence copies its valid records rounded up to a
  // multiple of 4 (16-byte sizes): with max_len a multiple of 4, and pages a multiple of
  // the tile, those records still lie in the unit's rows or page; the rows past the
  // sequence's end are masked by the warps.
  // The tile after (u, tl) in this CTA's order (len: the tokens of unit u).
  auto advance = [&](int& u, int& tl, int64_t& len) {
    if constexpr (!VARLEN) {
      if (++tl == (int)Tu) {
        ++u;
        tl = 0;
      }
      return;
    }
    if (++tl == (int)((len + TILE - 1) / TILE)) {
      u = next_unit(u);
      tl = 0;
      len = u < units ? unit_len(u) : 0;
    }
  };
  // Tile i of this CTA is tile tl of unit u: the first NST are issued by thread 0 at the
  // start, each later one by the warp that frees its stage, NST tiles after the one it
  // has just finished (every thread walks the same tiles).
  auto issue = [&](int i, int u, int tl, int64_t len) {
    const int64_t tok0 = (int64_t)tl * TILE;
    uint64_t* bar = &bars[i % NST];
    const int64_t nv = min((int64_t)TILE, len - tok0);
    if (!a.use_tma || nv <= 0) {
      mbar_arrive(bar);
      return;
    }
    const uint32_t n = (uint32_t)((nv + 3) & ~(int64_t)3);  // <= TILE
    unsigned char* st = stage_base + (i % NST) * L::STAGE;
    const int64_t v = record_row(a.pg, a.max_len, u, tok0, a.err);
    issued_s[i % NST] += 1;
    mbar_expect_tx(bar, n * (uint32_t)L::REC);
    bulk_g2s(st + L::OFF_KC, a.k_codes + v * L::KCB, n * L::KCB, bar);
    bulk_g2s(st + L::OFF_KS, a.k_signs + v * L::SB, n * L::SB, bar);
    bulk_g2s(st + L::OFF_KN, reinterpret_cast<const uint8_t*>(a.k_norms) + v * 4, n * 4, bar);
    bulk_g2s(st + L::OFF_VC, a.v_codes + v * L::VCB, n * L::VCB, bar);
    bulk_g2s(st + L::OFF_VP, reinterpret_cast<const uint8_t*>(a.v_params) + v * L::PB, n * L::PB, bar);
  };
  // One thread: the query operands of this CTA's next unit (local index fj) into buffer
  // fj % 2, if that unit starts before the CTA's range ends. fu: the last unit issued, fpre
  // its tile 0 in the global order, fn its tiles.
  auto issue_frag = [&]() {
    const int fj = pw->fj;
    int u = u0;
    int64_t pre = pw->pre0;
    if (fj > 0) {
      u = next_unit(pw->fu);
      pre = pw->fpre + pw->fn;
      if (u >= units || pre >= pw->g1) return;
    }
    pw->fu = u;
    pw->fpre = pre;
    pw->fn = unit_tiles(u);
    uint64_t* bar = &fbars[fj & 1];
    fissued_s[fj & 1] += 1;
    mbar_expect_tx(bar, (uint32_t)L::FRAG_BYTES);
    bulk_g2s(frag_base + (fj & 1) * L::FRAG_BYTES, a.frag + (size_t)u * frag_words(LMB, NB), L::FRAG_BYTES,
             bar);
    pw->fj = fj + 1;
  };
  // The packed cache does not depend on the prep kernel: start streaming it now.
  if (tid == 0) {
    int pu = u0, ptl = tl0;
    int64_t plen = len0;
    for (int i = 0; i < NST && i < ntl; ++i) {
      issue(i, pu, ptl, plen);
      advance(pu, ptl, plen);
    }
  }
  // Wait for the prep kernel (programmatic dependent launch), then fetch the query
  // operands of this CTA's first two units.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0 && ntl > 0) {
    issue_frag();
    issue_frag();
  }
  // The combine kernel may launch now; it waits for this grid to finish.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // Value-side B column of this lane: head 4 nb + hsel, part (hi / lo). Its tokens,
  // in K order, are (c, c + 8) and (c + 4, c + 12) of a 16-token block, whose
  // probabilities the lanes srcA and srcB hold after the score step.
  const int part = r & 1, hsel = r >> 1;
  const int srcA = 4 * c + hsel, srcB = 4 * (c + 4) + hsel;

  float m_run[NB], l_run[NB];
  float dmin[NB][4];       // rows g < 4: sum_t p * min(t, g); columns: heads x (hi, lo)
  float dv[4][2][NB][4];   // [group][half of the group][n-block]: rows = coordinates
  int cur = -1;            // local index of the unit being accumulated
  int qrow0 = 0;
  bool failed = false;

  // End of local unit j (every warp calls this at the same tile): the 16 warps' partials
  // are merged into this CTA's partial (m, l, acc) of the unit, in a fixed order (warp 0
  // first) so that the result does not depend on how the warps were scheduled; one head
  // at a time, each warp rescales its sums to the CTA maximum and stores them in
  // red_s[warp][coordinate], then one thread per coordinate adds the 16 rows in order.
  // combine_mma_kernel merges the partials of the CTAs that shared the unit. Then buffer
  // j % 2 is refilled with the operands of local unit j + 2.
  auto finish_unit = [&](int j) {
    __syncthreads();  // every warp has left the previous boundary's reduction
    float* part = a.ws_part + ((size_t)pw->cur_u + (size_t)kcta) * G * RS;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      float l = l_run[nb];
      l += __shfl_xor_sync(kFull, l, 4);
      l += __shfl_xor_sync(kFull, l, 8);
      l += __shfl_xor_sync(kFull, l, 16);
      if (r == 0) {
        rm_s[warp * 8 + c + 4 * nb] = failed ? -INFINITY : m_run[nb];
        rwl_s[warp * 8 + c + 4 * nb] = failed ? 0.f : l;
      }
    }
    __syncthreads();
    if (tid < 8) {
      float M = -INFINITY;
      for (int w = 0; w < kWarpsMma; ++w) M = fmaxf(M, rm_s[w * 8 + tid]);
      float L = 0.f;
      for (int w = 0; w < kWarpsMma; ++w) {
        const float mw = rm_s[w * 8 + tid];
        if (mw != -INFINITY) L = fmaf(ex2(mw - M), rwl_s[w * 8 + tid], L);
      }
      rM_s[tid] = M;
      if (tid < G) {
        part[tid * RS + 0] = M;
        part[tid * RS + 1] = L;
      }
    }
    __syncthreads();
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      // lane (g, c), g < 4, holds sum_t p * min(t, g) for head c + 4 nb in dmin[0] + dmin[1]
      const float own = dmin[nb][0] + dmin[nb][1];
      float mt[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) mt[g] = __shfl_sync(kFull, own, 4 * g + c);
      const float M = rM_s[c + 4 * nb];
      const float wsc = (failed || m_run[nb] == -INFINITY) ? 0.f : ex2(m_run[nb] - M);
      float* red = red_s + warp * kD;
      for (int c4 = 0; c4 < 4; ++c4) {
        const int h = 4 * nb + c4;
        if (h >= G) break;  // uniform
        if (c == c4) {  // the 8 lanes holding head h: 16 coordinates each
#pragma unroll
          for (int g = 0; g < 4; ++g)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const float* d = dv[g][hf][nb];
              int j0;
              float v0, v1;
              if (VB == 2) {
                j0 = 4 * (8 * g + r) + 2 * hf;  // code at mantissa bits 6 (row r), 8 (row r + 8)
                v0 = (d[0] + d[1]) * 262144.f + mt[g];
                v1 = (d[2] + d[3]) * 65536.f + mt[g];
              } else if (VB == 3) {
                j0 = 32 * g + 4 * r + 2 * hf;  // codes at mantissa bit 6
                v0 = (d[0] + d[1]) * 262144.f + mt[g];
                v1 = (d[2] + d[3]) * 262144.f + mt[g];
              } else {
                j0 = 2 * (16 * g + 8 * hf + r);  // low nibble (row r), high nibble (row r + 8), both at bit 4
                v0 = (d[0] + d[1]) * 1048576.f + mt[g];
                v1 = (d[2] + d[3]) * 1048576.f + mt[g];
              }
              red[j0] = wsc != 0.f ? wsc * v0 : 0.f;
              red[j0 + 1] = wsc != 0.f ? wsc * v1 : 0.f;
            }
        }
        __syncthreads();
        if (tid < kD) {
          float acc = 0.f;
#pragma unroll
          for (int w = 0; w < kWarpsMma; ++w) acc += red_s[w * kD + tid];
          part[h * RS + kPartPadMma + tid] = acc;
        }
        __syncthreads();
      }
    }
    if (tid == 0 && pw->fj == j + 2) {
      // every warp is past unit j: its operand buffer may be refilled
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue_frag();
    }
  };

  // ulen: the tokens of unit u when lengths are given (read once per unit: the lengths are
  // not in L1, which the shared memory takes); max_len otherwise.
  int u = u0, tl = tl0;
  int64_t ulen = len0;
  auto cur_len = [&]() -> int64_t {
    if constexpr (VARLEN) return ulen;
    return a.max_len;
  };
  for (int i = 0; i < ntl; ++i) {
    bool enter = i == 0;
    if (i > 0 && ++tl == (VARLEN ? (int)((cur_len() + TILE - 1) / TILE) : (int)Tu)) {  // u < units
      u = next_unit(u);
      tl = 0;
      if constexpr (VARLEN) ulen = unit_len(u);
      enter = true;
    }
    const int j = enter ? cur + 1 : cur;
    if (enter) {
      if (cur >= 0) finish_unit(cur);
      cur = j;
      if (tid == 0) pw->cur_u = u;  // read in finish_unit, after its first barrier
      // Wait for the unit's query operands; after a timeout the warp keeps the loop's
      // structure (arrivals, barriers) but does no more work.
      if (!failed && !mbar_wait(&fbars[j & 1], (uint32_t)((j >> 1) & 1))) failed = true;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        m_run[nb] = -INFINITY;
        l_run[nb] = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) dmin[nb][e] = 0.f;
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int e = 0; e < 4; ++e) dv[g][hf][nb][e] = 0.f;
      }
      const int b = u / a.hkv, kvh = u - b * a.hkv;
      qrow0 = b * a.hq + kvh * G;
    }
    const uint2* bq = reinterpret_cast<const uint2*>(frag_base + (j & 1) * L::FRAG_BYTES);
    const int64_t tok0 = (int64_t)tl * TILE;
    const int nt = (int)max((int64_t)0, min((int64_t)TILE, cur_len() - tok0));

    unsigned char* st = stage_base + (i % NST) * L::STAGE;
    // Warps run ahead of one another; each waits only for the tile it needs.
    if (!failed && !mbar_wait(&bars[i % NST], (uint32_t)((i / NST) & 1))) failed = true;
    if (!a.use_tma && nt > 0) {
      // Unaligned records: plain 4-byte copies (all record sizes are multiples of 4),
      // after every warp has left the tile that used this stage before.
      __syncthreads();
      const int64_t v = record_row(a.pg, a.max_len, u, tok0, a.err);
      auto copy = [&](int off, const void* src, int bytes_per_tok) {
        const uint32_t* s32 =
            reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(src) + v * bytes_per_tok);
        uint32_t* d32 = reinterpret_cast<uint32_t*>(st + off);
        for (int w = tid; w < nt * bytes_per_tok / 4; w += kThreadsMma) d32[w] = s32[w];
      };
      copy(L::OFF_KC, a.k_codes, L::KCB);
      copy(L::OFF_KS, a.k_signs, L::SB);
      copy(L::OFF_KN, a.k_norms, 4);
      copy(L::OFF_VC, a.v_codes, L::VCB);
      copy(L::OFF_VP, a.v_params, L::PB);
      __syncthreads();
    }

    const int wbase = 16 * MB * warp;  // this warp's first token within the tile
    if (wbase < nt && !failed) {
      const uint4* kc4 = reinterpret_cast<const uint4*>(st + L::OFF_KC);
      const uint4* ks4 = reinterpret_cast<const uint4*>(st + L::OFF_KS);
      const uint32_t* kn = reinterpret_cast<const uint32_t*>(st + L::OFF_KN);
      const uint32_t* vc = reinterpret_cast<const uint32_t*>(st + L::OFF_VC);
      const uint4* vp = reinterpret_cast<const uint4*>(st + L::OFF_VP);
      const uint32_t* vpw = reinterpret_cast<const uint32_t*>(st + L::OFF_VP);

      // ---- scores: D[token rows][(head, digit) columns] over all key bits ---------
      // Rows r and r + 8 of block mb are tokens wbase + 16 mb + r (+ 8). Lane column c takes
      // words c, c + 4, ... of each token: mask q of a word keeps bit q mod 4 of each byte
      // (of the word shifted right by 4 for q >= 4), four u8 elements in one AND.
      int dl[MB][2 * NB][4], ds[MB][2 * NB][4];
#pragma unroll
      for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int nb = 0; nb < 2 * NB; ++nb)
#pragma unroll
          for (int e = 0; e < 4; ++e) dl[mb][nb][e] = ds[mb][nb][e] = 0;
      const uint32_t* kcw = reinterpret_cast<const uint32_t*>(st + L::OFF_KC);
      const uint32_t* ksw = reinterpret_cast<const uint32_t*>(st + L::OFF_KS);
      constexpr int NWG = key_words(LMB) / 4;  // word groups: code words, parity words, signs
#pragma unroll
      for (int wg = 0; wg < NWG; ++wg) {  // lane column c takes word 4 wg + c of each token
        uint32_t w0[MB], w1[MB];
#pragma unroll
        for (int mb = 0; mb < MB; ++mb) {
          const int tok = wbase + 16 * mb + r;
          if (wg < LMB) {
            w0[mb] = kcw[tok * (4 * LMB) + 4 * wg + c];
            w1[mb] = kcw[(tok + 8) * (4 * LMB) + 4 * wg + c];
          } else if (wg == NWG - 1) {
            w0[mb] = ksw[tok * 4 + c];
            w1[mb] = ksw[(tok + 8) * 4 + c];
          } else {  // parity word c: from the three code words 3c .. 3c + 2 of the token
            const uint32_t* p0 = kcw + tok * (4 * LMB) + 3 * c;
            const uint32_t* p1 = kcw + (tok + 8) * (4 * LMB) + 3 * c;
            w0[mb] = parity_word(p0[0], p0[1], p0[2]);
            w1[mb] = parity_word(p1[0], p1[1], p1[2]);
          }
        }
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {
          const int kstep = 4 * wg + s4;
          uint2 bf[2 * NB];
#pragma unroll
          for (int nb = 0; nb < 2 * NB; ++nb) bf[nb] = bq[(kstep * 2 * NB + nb) * 32 + lane];
#pragma unroll
          for (int mb = 0; mb < MB; ++mb) {
            // masks 2 s4 and 2 s4 + 1: bits 2 s4, 2 s4 + 1 of each byte (of the word >> 4 past 3)
            const uint32_t x0 = s4 < 2 ? w0[mb] : w0[mb] >> 4, x1 = s4 < 2 ? w1[mb] : w1[mb] >> 4;
            const uint32_t m0 = 0x01010101u << (2 * (s4 & 1)), m1 = 0x02020202u << (2 * (s4 & 1));
            uint4 af;
            af.x = x0 & m0;
            af.y = x1 & m0;
            af.z = x0 & m1;
            af.w = x1 & m1;
#pragma unroll
            for (int nb = 0; nb < 2 * NB; ++nb) {
              if (wg < NWG - 1)
                mma_i8(dl[mb][nb], af, bf[nb].x, bf[nb].y);
              else
                mma_i8(ds[mb][nb], af, bf[nb].x, bf[nb].y);
            }
          }
        }
      }

#pragma unroll
      for (int mb = 0; mb < MB; ++mb) {
        const int tb = wbase + 16 * mb;
        if (tb >= nt) break;  // warp-uniform
        const int nv = nt - tb;  // valid tokens from tb on (rows past it hold stale bytes)

        // ---- logits and online softmax: lane (r, c) has tokens tb + r, tb + r + 8 ----
        const float2 ng0 = unpack_h2(kn[tb + r]), ng1 = unpack_h2(kn[tb + r + 8]);  // (n, gamma)
        float lg[NB][2];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          // lane (r, c) holds digits 0, 1 (n-block 2 nb) and 2, 3 (2 nb + 1) of head c + 4 nb
          const int* L0 = dl[mb][2 * nb];
          const int* L1 = dl[mb][2 * nb + 1];
          const int* S0 = ds[mb][2 * nb];
          const int* S1 = ds[mb][2 * nb + 1];
          const float lm0 = fmaf(65536.f, (float)(L1[0] + (L1[1] << 8)), (float)(L0[0] + (L0[1] << 8)));
          const float lm1 = fmaf(65536.f, (float)(L1[2] + (L1[3] << 8)), (float)(L0[2] + (L0[3] << 8)));
          const float sg0 = fmaf(65536.f, (float)(S1[0] + (S1[1] << 8)), (float)(S0[0] + (S0[1] << 8)));
          const float sg1 = fmaf(65536.f, (float)(S1[2] + (S1[3] << 8)), (float)(S0[2] + (S0[3] << 8)));
          // logit constants of head c + 4 nb (after the operand words of the buffer)
          const float4 kk = reinterpret_cast<const float4*>(bq + L::KS * NB * 32)[c + 4 * nb];
          lg[nb][0] = ng0.x * fmaf(ng0.y, fmaf(kk.z, sg0, -kk.w), fmaf(kk.y, lm0, kk.x));
          lg[nb][1] = ng1.x * fmaf(ng1.y, fmaf(kk.z, sg1, -kk.w), fmaf(kk.y, lm1, kk.x));
          if (nv < 16) {
            if (r >= nv) lg[nb][0] = -INFINITY;
            if (r + 8 >= nv) lg[nb][1] = -INFINITY;
          }
        }
        if (a.scores) {
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const int h = c + 4 * nb;
            if (h < G) {
              float* srow = a.scores + (size_t)(qrow0 + h) * a.max_len + (tok0 + tb);
              if (r < nv) srow[r] = lg[nb][0] * kLn2;
              if (r + 8 < nv) srow[r + 8] = lg[nb][1] * kLn2;
            }
          }
        }
        uint32_t ph[NB], pl[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          float cm = fmaxf(lg[nb][0], lg[nb][1]);
          cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 4));
          cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 8));
          cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 16));
          // Lazy rescaling: the reference maximum moves only when a logit exceeds it by
          // more than kSlack (base 2), so p stays below 2^kSlack and the accumulators
          // are rescaled a handful of times per CTA.
          if (cm > m_run[nb] + kSlack) {
            if (m_run[nb] != -INFINITY) {
              const float corr = ex2(m_run[nb] - cm);
              l_run[nb] *= corr;
#pragma unroll
              for (int e = 0; e < 4; ++e) dmin[nb][e] *= corr;
#pragma unroll
              for (int g = 0; g < 4; ++g)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                  for (int e = 0; e < 4; ++e) dv[g][hf][nb][e] *= corr;
            }
            m_run[nb] = cm;
          }
          const float p0 = ex2(lg[nb][0] - m_run[nb]), p1 = ex2(lg[nb][1] - m_run[nb]);
          l_run[nb] += p0 + p1;
          const __half2 hp = __floats2half2_rn(p0, p1);
          const float2 hpf = __half22float2(hp);
          ph[nb] = h2_bits(hp);
          pl[nb] = h2_bits(__floats2half2_rn(p0 - hpf.x, p1 - hpf.y));
        }

        // ---- values: D[coordinate rows][head columns] += codes x P' -----------------
        // B element (token t, head h, part) = p(t, h) * scale(t, g) split in f16 hi + lo:
        // hi = p_hi*s (rounded), err = fma(p_hi, s, -hi) (exact), lo = fma(p_lo, s, err).
        // The group minima enter through one more MMA: sum_t p_t * min(t, g).
        uint32_t phA[NB], plA[NB], phB[NB], plB[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          phA[nb] = __shfl_sync(kFull, ph[nb], srcA);
          plA[nb] = __shfl_sync(kFull, pl[nb], srcA);
          phB[nb] = __shfl_sync(kFull, ph[nb], srcB);
          plB[nb] = __shfl_sync(kFull, pl[nb], srcB);
        }
        const int tA0 = tb + c, tA1 = tA0 + 8, tB0 = tA0 + 4, tB1 = tA0 + 12;
        uint4 pA0 = vp[tA0], pA1 = vp[tA1], pB0 = vp[tB0], pB1 = vp[tB1];
        uint32_t mA0 = 0u, mA1 = 0u, mB0 = 0u, mB1 = 0u;
        if (r < 4) {
          mA0 = vpw[tA0 * 4 + r];
          mA1 = vpw[tA1 * 4 + r];
          mB0 = vpw[tB0 * 4 + r];
          mB1 = vpw[tB1 * 4 + r];
        }
        if (nv < 16) {  // tokens past the end: weight 0 and params 0 (their bytes are stale)
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
          if (c >= nv) { pA0 = z; mA0 = 0u; }
          if (c + 8 >= nv) { pA1 = z; mA1 = 0u; }
          if (c + 4 >= nv) { pB0 = z; mB0 = 0u; }
          if (c + 12 >= nv) { pB1 = z; mB1 = 0u; }
        }
        {
          uint4 am;  // rows g < 4: (min(t, g) of the two tokens of each K pair); rows 4.. zero
          am.x = __byte_perm(mA0, mA1, 0x7632);
          am.y = 0u;
          am.z = __byte_perm(mB0, mB1, 0x7632);
          am.w = 0u;
#pragma unroll
          for (int nb = 0; nb < NB; ++nb)
            mma16816(dmin[nb], am, part ? plA[nb] : phA[nb], part ? plB[nb] : phB[nb]);
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const __half2 sA = bits_h2(__byte_perm(word_of(pA0, g), word_of(pA1, g), 0x5410));
          const __half2 sB = bits_h2(__byte_perm(word_of(pB0, g), word_of(pB1, g), 0x5410));
          uint32_t bA[NB], bB[NB];
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const __half2 hA = __hmul2(bits_h2(phA[nb]), sA), hB = __hmul2(bits_h2(phB[nb]), sB);
            const __half2 eA = __hfma2(bits_h2(phA[nb]), sA, __hneg2(hA));
            const __half2 eB = __hfma2(bits_h2(phB[nb]), sB, __hneg2(hB));
            bA[nb] = part ? h2_bits(__hfma2(bits_h2(plA[nb]), sA, eA)) : h2_bits(hA);
            bB[nb] = part ? h2_bits(__hfma2(bits_h2(plB[nb]), sB, eB)) : h2_bits(hB);
          }
          // Row r of block (g, hf) is one byte of the group's codes; the codes of the
          // two tokens of a K pair go to the low byte of each f16 half.
          const uint32_t sel = (uint32_t)(r & 3) | ((uint32_t)(4 + (r & 3)) << 8);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            uint32_t xA, xB;
            uint4 av;
            if (VB == 2) {
              // byte 8g + r: rows r -> coordinate 4(8g + r) + 2hf, rows r + 8 -> + 1; codes moved
              // to mantissa bits 6 (rows r) and 8 (rows r + 8)
              constexpr int WPT = L::VCB / 4;
              const int wv = 2 * g + (r >> 2);
              if (hf == 0) {
                xA = __byte_perm(vc[tA0 * WPT + wv], vc[tA1 * WPT + wv], sel);
                xB = __byte_perm(vc[tB0 * WPT + wv], vc[tB1 * WPT + wv], sel);
              }
              const uint32_t yA = xA << (6 - 4 * hf), yB = xB << (6 - 4 * hf);
              av = make_uint4(yA & 0x00C000C0u, yA & 0x03000300u, yB & 0x00C000C0u, yB & 0x03000300u);
            } else if (VB == 3) {
              // Lane row r takes coordinates 32g + 4r .. + 3: the 12 bits at bit 12r of the
              // group's 96 (one funnel shift per token), two tokens' windows in the f16 halves.
              // Rows r -> coordinate 32g + 4r + 2hf, rows r + 8 -> + 1: every code moved to
              // mantissa bits 6..8.
              constexpr int WPT = L::VCB / 4;
              if (hf == 0) {
                const int bo = 12 * r, wi = 3 * g + (bo >> 5), wj = 3 * g + min((bo >> 5) + 1, 2), sh = bo & 31;
                auto win = [&](int t) { return __funnelshift_r(vc[t * WPT + wi], vc[t * WPT + wj], sh); };
                xA = __byte_perm(win(tA0), win(tA1), 0x5410);
                xB = __byte_perm(win(tB0), win(tB1), 0x5410);
                av = make_uint4((xA << 6) & 0x01C001C0u, (xA << 3) & 0x01C001C0u, (xB << 6) & 0x01C001C0u,
                                (xB << 3) & 0x01C001C0u);
              } else {
                av = make_uint4(xA & 0x01C001C0u, (xA >> 3) & 0x01C001C0u, xB & 0x01C001C0u,
                                (xB >> 3) & 0x01C001C0u);
              }
            } else {
              // byte 16g + 8hf + r: rows r -> coordinate 2(16g + 8hf + r), rows r + 8 -> + 1
              constexpr int WPT = L::VCB / 4;
              const int wv = 4 * g + 2 * hf + (r >> 2);
              xA = __byte_perm(vc[tA0 * WPT + wv], vc[tA1 * WPT + wv], sel);
              xB = __byte_perm(vc[tB0 * WPT + wv], vc[tB1 * WPT + wv], sel);
              // both nibbles at mantissa bits 4-7 (the low one shifted up)
              av = make_uint4((xA << 4) & 0x00F000F0u, xA & 0x00F000F0u, (xB << 4) & 0x00F000F0u,
                              xB & 0x00F000F0u);
            }
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) mma16816(dv[g][hf][nb], av, bA[nb], bB[nb]);
          }
        }
      }
    }
    // The last warp to finish with this stage refills it with tile i + NST.
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      const int prev = atomicAdd(&arrive_s[i % NST], 1);
      if (prev == kWarpsMma - 1) {
        arrive_s[i % NST] = 0;
        if (i + NST < ntl) {
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          int nu = u, ntl_ = tl;
          int64_t nlen = cur_len();
          for (int k = 0; k < NST; ++k) advance(nu, ntl_, nlen);
          issue(i + NST, nu, ntl_, nlen);
        }
      }
    }
  }
  if (cur >= 0) finish_unit(cur);

  if (__syncthreads_or(failed)) {
    // A copy did not complete in time: flag it, then wait (bounded again) for every
    // copy this CTA may still have in flight before its shared memory goes away.
    if (failed && lane == 0) atomicOr(a.err, 1u);
    if (tid == 0) {
      // Phases of one mbarrier complete in order: waiting for the last batch issued
      // into each stage (and operand buffer) covers every copy still in flight.
      for (int s = 0; s < NST; ++s)
        if (issued_s[s] > 0) mbar_wait(&bars[s], (uint32_t)((issued_s[s] - 1) & 1));
      for (int s = 0; s < 2; ++s)
        if (fissued_s[s] > 0) mbar_wait(&fbars[s], (uint32_t)((fissued_s[s] - 1) & 1));
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ combine kernel

struct CombineArgs {
  const float* ws_part;
  float* out;
  float* lse;  // null, or the log of each row's softmax denominator
  int batch, hq, hkv, G, s_max;
  int ppc;     // partials per CTA and unit (consecutive slots)
  int64_t tiles_per_unit, total_tiles, n_ctas;
  // Split by the tokens present (decode_mma_kernel): tile_tokens > 0, the lengths as there
  // (and with them each sequence's first tile and Tv, as the decode grid wrote them), and CTA
  // k's partial of unit u in slot u + k.
  int tile_tokens;
  const int32_t* seq_lens;
  const int64_t* seq_first;
  int64_t max_len;
};

// One CTA per (unit, query head), one thread per coordinate: log-sum-exp merge of the
// partials of the CTAs that shared the unit, launched as a programmatic dependent of
// the decode grid.
__global__ void __launch_bounds__(kD) combine_mma_kernel(const __grid_constant__ CombineArgs a) {
  constexpr int RS = kPartPadMma + kD;
  __shared__ float w_s[kD];
  __shared__ float red_s[2][kD / 32];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int u = blockIdx.x / a.G, h = blockIdx.x - u * a.G;
  const size_t pstride = (size_t)a.G * RS;  // partial p of head h at base + p * pstride
  int n_part;
  const float* base;
  // Partial p comes from CTA first + p; with fewer tiles than CTAs some CTAs between the
  // unit's first and last own no tile (and wrote nothing): they are skipped.
  int64_t k_first = 0, Tv = 0, pre = 0, nu = 0;
  auto live = [&](int p) -> bool {
    if (a.tile_tokens == 0) return true;
    const int64_t k = k_first + p;
    return max(k * Tv / a.n_ctas, pre) < min((k + 1) * Tv / a.n_ctas, pre + nu);
  };
  if (a.tile_tokens > 0) {
    // The decode kernel's split: the tiles holding tokens, all units end to end, Tv in all.
    const int64_t T = a.tile_tokens;
    auto tiles = [&](int b) -> int64_t {
      const int64_t len = a.seq_lens ? min((int64_t)max(a.seq_lens[b], 0), a.max_len) : a.max_len;
      return (len + T - 1) / T;
    };
    const int b = u / a.hkv, kvh = u - b * a.hkv;
    nu = tiles(b);
    if (a.seq_lens) {
      Tv = a.seq_first[a.batch];
      pre = a.seq_first[b] + kvh * nu;
    } else {
      Tv = (int64_t)a.batch * a.hkv * nu;
      pre = (int64_t)u * nu;
    }
    if (nu == 0) {  // no token: no partial
      const int row = b * a.hq + kvh * a.G + h;
      a.out[(size_t)row * kD + tid] = 0.f;
      if (a.lse && tid == 0) a.lse[row] = -INFINITY;
      return;
    }
    k_first = tile_owner(pre, a.n_ctas, Tv);
    n_part = (int)(tile_owner(pre + nu - 1, a.n_ctas, Tv) - k_first + 1);
    base = a.ws_part + ((size_t)u + (size_t)k_first) * pstride + (size_t)h * RS;
  } else {
    const int64_t Tu = a.tiles_per_unit;
    const int64_t first = tile_owner((int64_t)u * Tu, a.n_ctas, a.total_tiles);
    n_part = a.ppc * (int)(tile_owner((int64_t)(u + 1) * Tu - 1, a.n_ctas, a.total_tiles) - first + 1);
    base = a.ws_part + (size_t)u * a.s_max * a.ppc * pstride + (size_t)h * RS;
  }

  float M = -INFINITY;
  for (int p = tid; p < n_part; p += kD)
    if (live(p)) M = fmaxf(M, base[p * pstride]);
  M = warp_max(M);
  if (lane == 0) red_s[0][warp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(red_s[0][0], red_s[0][1]), fmaxf(red_s[0][2], red_s[0][3]));
  float den = 0.f, num0 = 0.f, num1 = 0.f;
  for (int p0 = 0; p0 < n_part; p0 += kD) {
    const int p = p0 + tid;
    float w = 0.f;
    if (p < n_part && live(p)) {
      const float mp = base[p * pstride];
      w = mp == -INFINITY ? 0.f : exp2f(mp - M);
      if (w != 0.f) den = fmaf(w, base[p * pstride + 1], den);
    }
    __syncthreads();  // the previous chunk's weights are consumed
    w_s[tid] = w;
    __syncthreads();
    const int np = min(kD, n_part - p0);
    const float* acc = base + (size_t)p0 * pstride + kPartPadMma + tid;
    int q = 0;
    // a partial of weight 0 (no valid token) is skipped: its sums need not be written
    for (; q + 2 <= np; q += 2) {
      if (w_s[q] != 0.f) num0 = fmaf(w_s[q], acc[q * pstride], num0);
      if (w_s[q + 1] != 0.f) num1 = fmaf(w_s[q + 1], acc[(q + 1) * pstride], num1);
    }
    if (q < np && w_s[q] != 0.f) num0 = fmaf(w_s[q], acc[q * pstride], num0);
  }
  den = warp_sum(den);
  if (lane == 0) red_s[1][warp] = den;
  __syncthreads();
  den = (red_s[1][0] + red_s[1][1]) + (red_s[1][2] + red_s[1][3]);
  const int b = u / a.hkv, kvh = u - b * a.hkv;
  const int row = b * a.hq + kvh * a.G + h;
  a.out[(size_t)row * kD + tid] = den > 0.f ? (num0 + num1) / den : 0.f;
  // The partial maxima and sums are in base 2 (logits times log2(e)): back to natural log.
  if (a.lse && tid == 0) a.lse[row] = den > 0.f ? (M + log2f(den)) * 0.6931471805599453f : -INFINITY;
}

template <int LMB, int VB, int NB, bool VARLEN>
cudaError_t configure_mma_t() {
  using L = Layout<LMB, VB, NB>;
  static cudaError_t status = cudaFuncSetAttribute(decode_mma_kernel<LMB, VB, NB, VARLEN>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::SMEM);
  return status;
}

template <int LMB, int VB, int NB>
int ctas_per_sm_t() {
  using L = Layout<LMB, VB, NB>;
  static int n = [] {
    int blocks = 0;
    if (configure_mma_t<LMB, VB, NB, false>() != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, decode_mma_kernel<LMB, VB, NB, false>, kThreadsMma,
                                                      L::SMEM) != cudaSuccess ||
        blocks < 1) {
      cudaGetLastError();
      blocks = 1;
    }
    return blocks;
  }();
  return n;
}

template <int LMB, int VB, int NB, bool VARLEN>
cudaError_t launch_mma_t(const MmaArgs& a, dim3 grid, cudaStream_t s) {
  using L = Layout<LMB, VB, NB>;
  cudaError_t e = configure_mma_t<LMB, VB, NB, VARLEN>();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreadsMma);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_mma_kernel<LMB, VB, NB, VARLEN>, a);
}

template <int LMB, int VB>
cudaError_t launch_mma_nb(const MmaArgs& a, int nb, dim3 grid, cudaStream_t s) {
  if (a.seq_lens)
    return nb == 1 ? launch_mma_t<LMB, VB, 1, true>(a, grid, s) : launch_mma_t<LMB, VB, 2, true>(a, grid, s);
  return nb == 1 ? launch_mma_t<LMB, VB, 1, false>(a, grid, s) : launch_mma_t<LMB, VB, 2, false>(a, grid, s);
}

}  // namespace

bool mma_decode_supported(const tq_ctx* ctx, int G) {
  const Shape& sh = ctx->shape;
  if (sh.d != kD || sh.m != kM || G < 1 || G > 8) return false;
  if (sh.lm_bits < 1 || sh.lm_bits > 3) return false;
  if (sh.v_bits < 2 || sh.v_bits > 4) return false;
  // the codebook must be affine in its bits (and the parity at 3 bits): true for a symmetric one
  float kappa, beta[4];
  return codebook_bits(ctx->cb, sh.lm_bits, kappa, beta);
}

template <int LMB>
int ctas_per_sm_l(int v_bits, int nb) {
  if (v_bits == 2) return nb == 1 ? ctas_per_sm_t<LMB, 2, 1>() : ctas_per_sm_t<LMB, 2, 2>();
  if (v_bits == 3) return nb == 1 ? ctas_per_sm_t<LMB, 3, 1>() : ctas_per_sm_t<LMB, 3, 2>();
  return nb == 1 ? ctas_per_sm_t<LMB, 4, 1>() : ctas_per_sm_t<LMB, 4, 2>();
}

int mma_ctas_per_sm(int lm_bits, int v_bits, int G) {
  const int nb = n_blocks(G);
  return lm_bits == 1 ? ctas_per_sm_l<1>(v_bits, nb) : lm_bits == 2 ? ctas_per_sm_l<2>(v_bits, nb)
                                                                  : ctas_per_sm_l<3>(v_bits, nb);
}

size_t mma_frag_bytes(int lm_bits, int G) { return (size_t)frag_words(lm_bits, n_blocks(G)) * 4; }

int mma_tile_tokens(int G) { return tile_tokens(n_blocks(G)); }

cudaError_t launch_decode_mma(const tq_ctx* ctx, const DecodePlan& plan, const void* q, int q_dtype, int batch,
                              int hq, int hkv, const int32_t* seq_lens, int64_t max_len, const Paging& pg,
                              const uint8_t* k_codes,
                              const uint8_t* k_signs, const uint16_t* k_norms, const uint8_t* v_codes,
                              const uint16_t* v_params, float scale, float* scores, float* out, float* lse,
                              void* workspace, cudaStream_t stream) {
  char* ws = static_cast<char*>(workspace);
  uint32_t* frag = reinterpret_cast<uint32_t*>(ws + plan.off_frag);
  float* part = reinterpret_cast<float*>(ws + plan.off_part);
  int64_t* seq_first = reinterpret_cast<int64_t*>(ws + plan.off_cnt);
  const int G = hq / hkv, lmb = ctx->shape.lm_bits, vb = ctx->shape.v_bits, nb = n_blocks(G);
  if (plan.n_ctas < 1 || plan.tiles_per_unit < 1) return cudaErrorInvalidValue;

  PrepArgs pa;
  pa.q = q;
  pa.q_dtype = q_dtype;
  pa.hq = hq;
  pa.hkv = hkv;
  pa.G = G;
  pa.rot = ctx->shape.rot;
  pa.inv_sqrt_d = (float)(1.0 / sqrt((double)kD));
  pa.St = ctx->St;
  pa.PiT = ctx->PiT;
  pa.cb = ctx->cb;
  if (!codebook_bits(ctx->cb, lmb, pa.kappa, pa.beta)) return cudaErrorInvalidValue;
  pa.sl2 = scale * 1.4426950408889634f;
  pa.nb = nb;
  pa.frag = frag;
  const size_t prep_smem = sizeof(float) * kD * kM;
  static bool prep_configured = false;
  if (!prep_configured) {
    const void* kernels[6] = {(const void*)prep_mma_kernel<1, 4>, (const void*)prep_mma_kernel<2, 4>,
                              (const void*)prep_mma_kernel<3, 4>, (const void*)prep_mma_kernel<1, 8>,
                              (const void*)prep_mma_kernel<2, 8>, (const void*)prep_mma_kernel<3, 8>};
    for (const void* k : kernels) {
      const cudaError_t ce = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem);
      if (ce != cudaSuccess) return ce;
    }
    prep_configured = true;
  }
  const unsigned prep_grid = (unsigned)(batch * hkv);
  if (nb == 1) {
    if (lmb == 1) prep_mma_kernel<1, 4><<<prep_grid, kPrepThreads, prep_smem, stream>>>(pa);
    else if (lmb == 2) prep_mma_kernel<2, 4><<<prep_grid, kPrepThreads, prep_smem, stream>>>(pa);
    else prep_mma_kernel<3, 4><<<prep_grid, kPrepThreads, prep_smem, stream>>>(pa);
  } else {
    if (lmb == 1) prep_mma_kernel<1, 8><<<prep_grid, kPrepThreads, prep_smem, stream>>>(pa);
    else if (lmb == 2) prep_mma_kernel<2, 8><<<prep_grid, kPrepThreads, prep_smem, stream>>>(pa);
    else prep_mma_kernel<3, 8><<<prep_grid, kPrepThreads, prep_smem, stream>>>(pa);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  MmaArgs a;
  a.frag = frag;
  a.k_codes = k_codes;
  a.k_signs = k_signs;
  a.k_norms = k_norms;
  a.v_codes = v_codes;
  a.v_params = v_params;
  a.seq_lens = seq_lens;
  a.max_len = max_len;
  a.pg = pg;
  a.batch = batch;
  a.hq = hq;
  a.hkv = hkv;
  a.G = G;
  a.scores = scores;
  a.out = out;
  a.ws_part = part;
  a.seq_first = seq_first;
  a.use_tma = (max_len % 4 == 0) ? 1 : 0;
  a.err = ctx->d_err;
  const dim3 grid((unsigned)plan.n_ctas);
  if (ctx->prof_start) cudaEventRecord(ctx->prof_start, stream);
  if (lmb == 1)
    e = vb == 2 ? launch_mma_nb<1, 2>(a, nb, grid, stream)
        : vb == 3 ? launch_mma_nb<1, 3>(a, nb, grid, stream) : launch_mma_nb<1, 4>(a, nb, grid, stream);
  else if (lmb == 2)
    e = vb == 2 ? launch_mma_nb<2, 2>(a, nb, grid, stream)
        : vb == 3 ? launch_mma_nb<2, 3>(a, nb, grid, stream) : launch_mma_nb<2, 4>(a, nb, grid, stream);
  else
    e = vb == 2 ? launch_mma_nb<3, 2>(a, nb, grid, stream)
        : vb == 3 ? launch_mma_nb<3, 3>(a, nb, grid, stream) : launch_mma_nb<3, 4>(a, nb, grid, stream);
  if (ctx->prof_stop) cudaEventRecord(ctx->prof_stop, stream);
  if (e != cudaSuccess) return e;

  return launch_combine_partials(part, out, lse, batch, hq, hkv, G, plan.s_max, 1, plan.tiles_per_unit,
                                 plan.total_tiles, plan.n_ctas, stream, mma_tile_tokens(G), seq_lens, seq_first,
                                 max_len);
}

cudaError_t launch_combine_partials(const float* part, float* out, float* lse, int batch, int hq, int hkv, int G,
                                    int s_max, int ppc, int64_t tiles_per_unit, int64_t total_tiles, int n_ctas,
                                    cudaStream_t stream, int tile_tokens, const int32_t* seq_lens,
                                    const int64_t* seq_first, int64_t max_len) {
  CombineArgs ca;
  ca.batch = batch;
  ca.tile_tokens = tile_tokens;
  ca.seq_lens = seq_lens;
  ca.seq_first = seq_first;
  ca.max_len = max_len;
  ca.ppc = ppc;
  ca.ws_part = part;
  ca.out = out;
  ca.lse = lse;
  ca.hq = hq;
  ca.hkv = hkv;
  ca.G = G;
  ca.s_max = s_max;
  ca.tiles_per_unit = tiles_per_unit;
  ca.total_tiles = total_tiles;
  ca.n_ctas = n_ctas;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((int64_t)batch * hkv * G));
  cfg.blockDim = dim3(kD);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_mma_kernel, ca);
}

}  // namespace tq
