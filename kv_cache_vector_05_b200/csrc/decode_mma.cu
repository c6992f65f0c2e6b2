// Tensor-core decode attention over the packed cache (d = m = 128, up to 8 query
// heads per KV head, 1- or 2-bit Lloyd-Max keys, 2- or 4-bit values).
//
// Same mathematics as decode_kernel (the skill card "turboquant-pytorch", "Что
// делает": scores straight from the compressed keys; the discosf news item:
// fused decode kernels): logit = scale * n * (<qr, c[idx]> + sqrt(pi/2)/m * gamma *
// <sq, s>), online softmax, sum of p * (min + scale * code). What changes is how
// the per-token work is spread: with G query heads sharing a KV head, the three
// contractions (codes x qr, signs x sq, probabilities x value codes) are small
// dense products over a tile of tokens, so they run on the tensor cores
// (mma.sync m16n8k16, f16 operands, fp32 accumulation) instead of G scalar loops.
//
// Operand construction (no unpacking loops):
//  * A 2-bit code with a symmetric codebook is affine in its two bits:
//    c[b0 + 2 b1] = c0 + (c1 - c0) b0 + (c2 - c0) b1. So <qr, c[idx]> =
//    c0 sum(qr) + sum over stream bits of (beta_plane * qr_j) * bit. Every packed
//    bit, keys and signs alike, becomes one MMA operand element.
//  * Masking one bit per 16-bit half of a word yields an f16 that is 0 or a power
//    of two (2^-15 .. 2 for bit positions 9..14); the query side is pre-divided by
//    that power, so one LOP3 turns two bits into two exact operand elements.
//  * A value code placed in the low mantissa bits of an f16 is a subnormal equal
//    to code * 2^(pos - 24), so a byte permute plus a mask yields two exact
//    operands; the power of two is undone once at the end.
//  * Query and probability operands are split hi + lo in f16 (about 22 bits), the
//    two halves occupying rows h and h + 8 of the 16-row tile.
//
// Kernels:
//  * prep_mma_kernel, one CTA per (sequence, KV head): rotates the G queries
//    (sign flip + Walsh-Hadamard butterflies, or the dense Haar matrix), forms
//    S qr, and writes the query operand fragments of that KV head once.
//  * decode_mma_kernel, one CTA per (sequence x KV head, chunk of the cache),
//    launched with programmatic dependent launch: it starts streaming its cache
//    tiles (cp.async.bulk into a 4-deep ring, mbarrier completion) while the prep
//    kernel finishes, then waits for the fragments. Each warp owns 16 tokens of
//    each 64-token tile. The last CTA of a (sequence, KV head) to finish - decided
//    by an atomic ticket, nobody waits - merges the chunk partials (log-sum-exp)
//    and writes the output rows.
// Every wait is bounded; a timeout sets the context's error word and ends the CTA.
#include <cuda_runtime.h>
#include <math.h>

#include "tq_device.cuh"

namespace tq {
namespace {

constexpr int kD = 128;
constexpr int kM = 128;
constexpr int kWarpsMma = 4;
constexpr int kThreadsMma = kWarpsMma * 32;
constexpr int kTileMma = 64;  // tokens per stage: 16 per warp
constexpr int kStages = 4;
constexpr int kPartPadMma = 4;
constexpr int kPrepThreads = 256;
// Base-2 slack of the lazy online-softmax rescale: probabilities stay below 2^kSlack,
// so p * scale fits fp16 for any value-group scale below 65504 / 2^kSlack = 16376.
constexpr float kSlack = 2.f;
constexpr uint32_t kWaitLimit = 1u << 24;                 // polls of one mbarrier phase
constexpr unsigned long long kWaitNs = 2000000000ull;    // and at most 2 s of wall time

__host__ __device__ constexpr int frag_chunks(int lmb) { return 8 * (lmb + 1); }
// Per (sequence, KV head): A fragments [chunks][32 lanes] uint4, then [8 heads][4] floats
// (sum of qr, sum of sq, LM scale, sign scale).
__host__ __device__ constexpr int frag_words(int lmb) { return frag_chunks(lmb) * 32 * 4 + 32; }

struct PrepArgs {
  const void* q;
  int q_dtype;
  int hq, hkv, G, rot;
  float inv_sqrt_d;
  const float* St;   // [d][m]
  const float* PiT;  // [d][d] (Haar)
  Codebook cb;
  float beta0, beta1;
  uint32_t* frag;    // [units][frag_words]
  unsigned int* cnt; // [units] completion tickets, zeroed here
  const uint16_t* table;  // [frag_chunks * 32 * 4 * 2] operand sources (frag_source)
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
  int hq, hkv, G;
  int n_chunks;
  int64_t chunk_len;
  float scale;
  float* scores;
  float* out;
  float* ws_part;
  unsigned int* cnt;
  float c0;
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

__device__ __forceinline__ uint32_t pack_h2(float lo_half, float hi_half) {
  const __half2 h = __floats2half2_rn(lo_half, hi_half);
  return *reinterpret_cast<const uint32_t*>(&h);
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

// Register rho (0..15) of a key word: which shifted copy of the word it masks,
// which bit position p of each 16-bit half it keeps, and which original bit o.
//   rho 0..5   : word       , p = 9 + rho   , o = 9 + rho
//   rho 6..11  : word << 6  , p = 3 + rho   , o = rho - 3
//   rho 12..14 : word << 12 , p = rho       , o = rho - 12
//   rho 15     : word >> 6  , p = 9         , o = 15
__host__ __device__ constexpr int key_variant(int rho) { return rho < 6 ? 0 : rho < 12 ? 1 : rho < 15 ? 2 : 3; }
__host__ __device__ constexpr int key_pos(int rho) { return rho < 6 ? 9 + rho : rho < 12 ? 3 + rho : rho < 15 ? rho : 9; }
__host__ __device__ constexpr int key_orig(int rho) { return rho < 6 ? 9 + rho : rho < 12 ? rho - 3 : rho < 15 ? rho - 12 : 15; }

// log2 of the f16 value of a lone bit at position p (0..14) of a half.
__host__ __device__ constexpr int lone_bit_log2(int p) { return p <= 9 ? p - 24 : (1 << (p - 10)) - 15; }

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

template <int LMB>
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
    float v[8 * kD / kPrepThreads];
#pragma unroll
    for (int u = 0; u < 8 * kD / kPrepThreads; ++u) {
      const int idx = tid + u * kPrepThreads, h = idx / kD, j = idx % kD;
      const size_t off = (size_t)(qrow0 + h) * kD + j;
      v[u] = 0.f;
      if (h < G)
        v[u] = a.q_dtype == TQ_F32 ? __ldg(static_cast<const float*>(a.q) + off)
                                   : __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[off]);
    }
#pragma unroll
    for (int u = 0; u < 8 * kD / kPrepThreads; ++u) {
      const int idx = tid + u * kPrepThreads, j = idx % kD;
      float x = v[u];
      if (a.rot == TQ_ROT_HADAMARD) x = flip_sign(x, (a.cb.sign_bits[j / 32] >> (j % 32)) & 1u);
      x_s[idx] = x;
    }
  }
  __syncthreads();
  if (a.rot == TQ_ROT_HADAMARD) {
    for (int hs = 1; hs < kD; hs <<= 1) {
      for (int p = tid; p < 8 * (kD / 2); p += kPrepThreads) {
        const int h = p / (kD / 2), i = p % (kD / 2);
        const int i0 = h * kD + (i / hs) * 2 * hs + (i % hs);
        const float u = x_s[i0], w = x_s[i0 + hs];
        x_s[i0] = u + w;
        x_s[i0 + hs] = u - w;
      }
      __syncthreads();
    }
    for (int idx = tid; idx < 8 * kD; idx += kPrepThreads) qr_s[idx] = x_s[idx] * a.inv_sqrt_d;
  } else {
    stage_matrix(st_s, a.PiT, tid);
    __syncthreads();
    const int i = tid % kD, half = tid / kD;
    float acc[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) acc[h] = 0.f;
#pragma unroll 8
    for (int j = half * (kD / 2); j < (half + 1) * (kD / 2); ++j) {
      const float pv = st_s[j * kD + i];
#pragma unroll
      for (int h = 0; h < 8; ++h) acc[h] = fmaf(pv, x_s[h * kD + j], acc[h]);
    }
    if (half == 1)
#pragma unroll
      for (int h = 0; h < 8; ++h) sq_s[h * kD + i] = acc[h];  // scratch
    __syncthreads();
    if (half == 0)
#pragma unroll
      for (int h = 0; h < 8; ++h) qr_s[h * kD + i] = acc[h] + sq_s[h * kD + i];
    __syncthreads();  // st_s is reused for S^T below
  }
  __syncthreads();
  {
    // sq = S qr for the 8 head slots at once. S^T is staged in shared memory with
    // independent 16-byte loads (its 64 KB would otherwise be read at L2 latency,
    // one dependent load per step); thread (i, half) then runs over half of j.
    stage_matrix(st_s, a.St, tid);
    __syncthreads();
    const int i = tid % kM, half = tid / kM;
    float acc[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) acc[h] = 0.f;
#pragma unroll 8
    for (int j = half * (kD / 2); j < (half + 1) * (kD / 2); ++j) {
      const float sv = st_s[j * kM + i];
#pragma unroll
      for (int h = 0; h < 8; ++h) acc[h] = fmaf(sv, qr_s[h * kD + j], acc[h]);
    }
    if (half == 1)
#pragma unroll
      for (int h = 0; h < 8; ++h) x_s[h * kM + i] = acc[h];
    __syncthreads();
    if (half == 0)
#pragma unroll
      for (int h = 0; h < 8; ++h) sq_s[h * kM + i] = acc[h] + x_s[h * kM + i];
  }
  __syncthreads();
  {
    const int h = warp;  // 8 warps, one per head slot
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
      const float bmax = fmaxf(fabsf(a.beta0), LMB > 1 ? fabsf(a.beta1) : 0.f);
      const float qs = qmax * bmax;
      head_s[h * 4 + 0] = qsum;
      head_s[h * 4 + 1] = ssum;
      head_s[h * 4 + 2] = qs > 0.f ? qs : 1.f;
      head_s[h * 4 + 3] = smax > 0.f ? smax : 1.f;
      inv_s[h * 2 + 0] = 1.f / head_s[h * 4 + 2];
      inv_s[h * 2 + 1] = 1.f / head_s[h * 4 + 3];
    }
  }
  __syncthreads();
  uint32_t* frag = a.frag + (size_t)unit * frag_words(LMB);
  // A fragment word (chunk k, lane l, register q = a0..a3) holds two f16 (row, slot)
  // values: a0/a2 rows r (hi part), a1/a3 rows r + 8 (lo part). Where each value
  // comes from is fixed by the layout and precomputed (see frag_source).
  const uint32_t* tab = reinterpret_cast<const uint32_t*>(a.table);
  constexpr int kPerT = frag_chunks(LMB) * 32 * 4 / kPrepThreads;  // 6 or 12 words per thread
  uint32_t ents[kPerT];
#pragma unroll
  for (int u = 0; u < kPerT; ++u) ents[u] = __ldg(tab + tid + u * kPrepThreads);
#pragma unroll
  for (int u = 0; u < kPerT; ++u) {
    const int idx = tid + u * kPrepThreads;
    const int q = idx & 3, l = (idx >> 2) & 31;
    const int row_head = l >> 2;
    const bool lo_part = (q & 1) != 0;
    const uint32_t ent2 = ents[u];
    float v2[2] = {0.f, 0.f};
    if (row_head < G) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const uint32_t ent = (ent2 >> (16 * e)) & 0xffffu;
        const int src = ent & 0xff, plane = (ent >> 8) & 1, ex = (int)((ent >> 9) & 31) - 16;
        const float pw2 = __int_as_float((ex + 127) << 23);
        float x;
        if (src < kD)
          x = qr_s[row_head * kD + src] * ((plane ? a.beta1 : a.beta0) * inv_s[row_head * 2 + 0] * pw2);
        else
          x = sq_s[row_head * kM + (src - kD)] * (inv_s[row_head * 2 + 1] * pw2);
        const float hi = __half2float(__float2half_rn(x));
        v2[e] = lo_part ? (x - hi) : hi;
      }
    }
    frag[idx] = pack_h2(v2[0], v2[1]);
  }
  if (tid < 32) reinterpret_cast<float*>(frag)[frag_chunks(LMB) * 32 * 4 + tid] = head_s[tid];
  if (tid == 0) a.cnt[unit] = 0u;
}

// ------------------------------------------------------------------ decode kernel

template <int LMB, int VB>
struct Layout {
  static constexpr int KCB = LMB * kD / 8;  // key code bytes per token
  static constexpr int SB = kM / 8;         // sign bytes
  static constexpr int VCB = VB * kD / 8;   // value code bytes
  static constexpr int PB = (kD / kVGroup) * 4;
  static constexpr int REC = KCB + SB + 4 + VCB + PB;
  static constexpr int STAGE = kTileMma * REC;
  static constexpr int OFF_KC = 0;
  static constexpr int OFF_KS = OFF_KC + kTileMma * KCB;
  static constexpr int OFF_KN = OFF_KS + kTileMma * SB;
  static constexpr int OFF_VC = OFF_KN + kTileMma * 4;
  static constexpr int OFF_VP = OFF_VC + kTileMma * VCB;
  static constexpr int KCHUNKS = frag_chunks(LMB);
  static constexpr int FRAG_BYTES = frag_words(LMB) * 4;
  static constexpr int RED_BYTES = kWarpsMma * 8 * (kPartPadMma + kD) * 4;  // per-warp partials
  static constexpr int RING = kStages * STAGE > RED_BYTES ? kStages * STAGE : RED_BYTES;
  static constexpr size_t SMEM = (size_t)RING + FRAG_BYTES + 8 * kStages + 4 * (1 + 2 * kStages) + 16;
};

template <int LMB, int VB>
__global__ void __launch_bounds__(kThreadsMma, 4) decode_mma_kernel(const __grid_constant__ MmaArgs a) {
  using L = Layout<LMB, VB>;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* stage_base = smem;                                     // ring, later per-warp partials
  uint4* afrag = reinterpret_cast<uint4*>(smem + L::RING);             // [KCHUNKS][32], then head consts
  const float* head_s = reinterpret_cast<const float*>(afrag + L::KCHUNKS * 32);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::RING + L::FRAG_BYTES);
  int* last_s = reinterpret_cast<int*>(bars + kStages);
  int* arrive_s = last_s + 1;        // [kStages] warps done with the stage's current tile
  int* issued_s = arrive_s + kStages; // [kStages] bulk-copy batches issued into the stage

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = lane >> 2, c = lane & 3;
  const int G = a.G;
  const int chunk = blockIdx.x, unit = blockIdx.y;
  const int b = unit / a.hkv, kvh = unit % a.hkv;
  int64_t len = a.max_len;
  if (a.seq_lens) len = min((int64_t)max(a.seq_lens[b], 0), a.max_len);
  const int64_t t0 = (int64_t)chunk * a.chunk_len;
  const int64_t t1 = min(t0 + a.chunk_len, len);
  const int qrow0 = b * a.hq + kvh * G;
  const int64_t vec0 = (int64_t)unit * a.max_len;
  const int span = t1 > t0 ? (int)(t1 - t0) : 0;  // tokens of this chunk (< 2^31)
  const int ntiles = (span + kTileMma - 1) / kTileMma;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[s], 1);
      arrive_s[s] = 0;
      issued_s[s] = 0;
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  auto tile_full = [&](int i) -> bool { return (i + 1) * kTileMma <= span; };
  auto issue = [&](int i) {  // one thread: bulk-copy tile i into its stage
    unsigned char* st = stage_base + (i % kStages) * L::STAGE;
    const int64_t v = vec0 + t0 + (int64_t)i * kTileMma;
    uint64_t* bar = &bars[i % kStages];
    issued_s[i % kStages] += 1;
    mbar_expect_tx(bar, (uint32_t)L::STAGE);
    bulk_g2s(st + L::OFF_KC, a.k_codes + v * L::KCB, kTileMma * L::KCB, bar);
    bulk_g2s(st + L::OFF_KS, a.k_signs + v * L::SB, kTileMma * L::SB, bar);
    bulk_g2s(st + L::OFF_KN, reinterpret_cast<const uint8_t*>(a.k_norms) + v * 4, kTileMma * 4, bar);
    bulk_g2s(st + L::OFF_VC, a.v_codes + v * L::VCB, kTileMma * L::VCB, bar);
    bulk_g2s(st + L::OFF_VP, reinterpret_cast<const uint8_t*>(a.v_params) + v * L::PB, kTileMma * L::PB, bar);
  };
  // The packed cache does not depend on the prep kernel: start streaming it now.
  if (tid == 0 && a.use_tma) {
    for (int i = 0; i < kStages && i < ntiles; ++i)
      if (tile_full(i)) issue(i);
  }

  // Wait for the prep kernel (programmatic dependent launch), then fetch this KV
  // head's query fragments and constants.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.frag + (size_t)unit * frag_words(LMB));
    for (int w = tid; w < L::FRAG_BYTES / 16; w += kThreadsMma) afrag[w] = src[w];
  }
  __syncthreads();

  const bool head_ok = r < G;
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr float kLn2 = 0.6931471805599453f;
  // logit (base-2 units) = n * (k1 + k2 * lm + gamma * (k3 * sg - k4)), with lm, sg the raw
  // tensor-core dot products and every per-head constant folded in once.
  const float sl2 = a.scale * kLog2e;
  const float k1 = sl2 * a.c0 * head_s[r * 4 + 0];
  const float k2 = sl2 * head_s[r * 4 + 2];
  const float k3 = sl2 * (kQjl / (float)kM) * 2.f * head_s[r * 4 + 3];
  const float k4 = sl2 * (kQjl / (float)kM) * head_s[r * 4 + 1];

  float m_run = -INFINITY, l_run = 0.f;
  float dmin[4] = {0.f, 0.f, 0.f, 0.f};  // sum_t p * min(t, g): rows (head, hi/lo), cols = groups
  float dv[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) dv[i][0] = dv[i][1] = dv[i][2] = dv[i][3] = 0.f;

  bool failed = false;
  for (int i = 0; i < ntiles; ++i) {
    unsigned char* st = stage_base + (i % kStages) * L::STAGE;
    const int nt = min(kTileMma, span - i * kTileMma);
    if (a.use_tma && tile_full(i)) {
      // Warps run ahead of one another; each waits only for the tile it needs. After
      // a timeout a warp keeps the loop's structure (arrivals, barriers) but does no
      // more work, so every warp of the CTA reaches the same barriers.
      if (!failed && !mbar_wait(&bars[i % kStages], (uint32_t)((i / kStages) & 1))) failed = true;
    } else {
      // Ragged or unaligned tile: plain 4-byte copies (all record sizes are multiples
      // of 4), after every warp has left the tile that used this stage before.
      __syncthreads();
      const int64_t v = vec0 + t0 + (int64_t)i * kTileMma;
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

    const int tb = 16 * warp;  // this warp's 16 tokens within the tile
    if (tb < nt && !failed) {
      const uint32_t* kc = reinterpret_cast<const uint32_t*>(st + L::OFF_KC);
      const uint32_t* ks = reinterpret_cast<const uint32_t*>(st + L::OFF_KS);
      const uint32_t* kn = reinterpret_cast<const uint32_t*>(st + L::OFF_KN);
      const uint32_t* vc = reinterpret_cast<const uint32_t*>(st + L::OFF_VC);
      const uint4* vp = reinterpret_cast<const uint4*>(st + L::OFF_VP);

      // ---- logits: D[head hi/lo rows][token columns] ---------------------------
      float dl[2][4], ds[2][4];
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) dl[nb][e] = ds[nb][e] = 0.f;
      uint32_t kw[2][LMB + 1];
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        const int tok = tb + 8 * nb + (r >> 1) + 4 * (r & 1);  // token of B column r
#pragma unroll
        for (int wi = 0; wi < LMB; ++wi) kw[nb][wi] = kc[tok * (L::KCB / 4) + c + 4 * wi];
        kw[nb][LMB] = ks[tok * (L::SB / 4) + c];
      }
#pragma unroll
      for (int wi = 0; wi <= LMB; ++wi) {
        uint32_t var[2][4];
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
          const uint32_t w = kw[nb][wi];
          var[nb][0] = w;
          var[nb][1] = w << 6;
          var[nb][2] = w << 12;
          var[nb][3] = w >> 6;
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint4 af = afrag[(8 * wi + kk) * 32 + lane];
          const int r0 = 2 * kk, r1 = 2 * kk + 1;
          const uint32_t m0 = (1u << key_pos(r0)) | (1u << (key_pos(r0) + 16));
          const uint32_t m1 = (1u << key_pos(r1)) | (1u << (key_pos(r1) + 16));
#pragma unroll
          for (int nb = 0; nb < 2; ++nb) {
            const uint32_t b0 = var[nb][key_variant(r0)] & m0;
            const uint32_t b1 = var[nb][key_variant(r1)] & m1;
            if (wi < LMB)
              mma16816(dl[nb], af, b0, b1);
            else
              mma16816(ds[nb], af, b0, b1);
          }
        }
      }

      // ---- logits epilogue and online softmax (thread: head r, 4 tokens) ---------
      // token order of the thread's four values: c, c + 4, c + 8, c + 12. Rows of
      // absent heads (r >= G) carry zero query operands, so their values stay finite
      // and are simply never written out.
      float lg[4];
      bool tv[4] = {true, true, true, true};
      const bool ragged = nt - tb < 16;  // warp-uniform
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int nb = e >> 1, col = e & 1;
        const float2 ng = unpack_h2(kn[tb + c + 4 * e]);  // (n, gamma)
        const float lm = dl[nb][col] + dl[nb][col + 2];
        const float sg = ds[nb][col] + ds[nb][col + 2];
        lg[e] = ng.x * fmaf(ng.y, fmaf(k3, sg, -k4), fmaf(k2, lm, k1));
      }
      if (ragged) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          tv[e] = c + 4 * e < nt - tb;
          if (!tv[e]) lg[e] = -INFINITY;  // stale bytes past the end of the cache
        }
      }
      if (a.scores && head_ok) {
        float* srow = a.scores + (size_t)(qrow0 + r) * a.max_len + (t0 + (int64_t)i * kTileMma + tb);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (tv[e]) srow[c + 4 * e] = lg[e] * kLn2;
      }
      float cmax = fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3]));
      cmax = fmaxf(cmax, __shfl_xor_sync(kFull, cmax, 1));
      cmax = fmaxf(cmax, __shfl_xor_sync(kFull, cmax, 2));
      // Lazy rescaling: the reference maximum moves only when a logit exceeds it by
      // more than kSlack (base 2), so p stays below 2^kSlack and the accumulators are
      // rescaled a handful of times per CTA instead of at most chunks.
      if (cmax > m_run + kSlack) {
        if (m_run != -INFINITY) {
          const float corr = ex2(m_run - cmax);
          l_run *= corr;
#pragma unroll
          for (int e = 0; e < 4; ++e) dmin[e] *= corr;
#pragma unroll
          for (int nbk = 0; nbk < 16; ++nbk)
#pragma unroll
            for (int e = 0; e < 4; ++e) dv[nbk][e] *= corr;
        }
        m_run = cmax;
      }
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        p[e] = ex2(lg[e] - m_run);
        l_run += p[e];
      }

      // ---- values: D[head hi/lo rows][coordinate columns] += P' x codes ----------
      // p is split once into f16 hi + lo; for each value group g the operand
      // P'_g = p * scale_g is formed in half2 arithmetic as an exact product split:
      // hi = p_hi*s (rounded), err = fma(p_hi, s, -hi) (exact), lo = fma(p_lo, s, err).
      // The group minima enter through one more MMA: sum_t p_t * min(t, g).
      // Tokens past the end of a ragged tile carry stale bytes: weight 0, params 0.
      uint4 par[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) par[e] = vp[tb + c + 4 * e];
      if (ragged) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (!tv[e]) par[e] = make_uint4(0u, 0u, 0u, 0u);
      }
      const __half2 ph01 = __floats2half2_rn(p[0], p[1]);
      const __half2 ph23 = __floats2half2_rn(p[2], p[3]);
      const float2 pf01 = __half22float2(ph01), pf23 = __half22float2(ph23);
      const __half2 pl01 = __floats2half2_rn(p[0] - pf01.x, p[1] - pf01.y);
      const __half2 pl23 = __floats2half2_rn(p[2] - pf23.x, p[3] - pf23.y);
      {
        // group minima: B[token][group] = min (high half of word g); rows r < 4 are the groups
        const int gsel = r & 3;
        auto word = [&](const uint4& w) { return gsel == 0 ? w.x : gsel == 1 ? w.y : gsel == 2 ? w.z : w.w; };
        const uint32_t m01 = r < 4 ? __byte_perm(word(par[0]), word(par[1]), 0x7632) : 0u;
        const uint32_t m23 = r < 4 ? __byte_perm(word(par[2]), word(par[3]), 0x7632) : 0u;
        uint4 ap;
        ap.x = h2_bits(ph01);
        ap.y = h2_bits(pl01);
        ap.z = h2_bits(ph23);
        ap.w = h2_bits(pl23);
        mma16816(dmin, ap, m01, m23);
      }
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const uint32_t w0 = g == 0 ? par[0].x : g == 1 ? par[0].y : g == 2 ? par[0].z : par[0].w;
        const uint32_t w1 = g == 0 ? par[1].x : g == 1 ? par[1].y : g == 2 ? par[1].z : par[1].w;
        const uint32_t w2 = g == 0 ? par[2].x : g == 1 ? par[2].y : g == 2 ? par[2].z : par[2].w;
        const uint32_t w3 = g == 0 ? par[3].x : g == 1 ? par[3].y : g == 2 ? par[3].z : par[3].w;
        const __half2 s01 = bits_h2(__byte_perm(w0, w1, 0x5410));  // (scale of token c, of c + 4)
        const __half2 s23 = bits_h2(__byte_perm(w2, w3, 0x5410));
        const __half2 hi01 = __hmul2(ph01, s01), hi23 = __hmul2(ph23, s23);
        const __half2 er01 = __hfma2(ph01, s01, __hneg2(hi01)), er23 = __hfma2(ph23, s23, __hneg2(hi23));
        const __half2 lo01 = __hfma2(pl01, s01, er01), lo23 = __hfma2(pl23, s23, er23);
        uint4 av;
        av.x = h2_bits(hi01);
        av.y = h2_bits(lo01);
        av.z = h2_bits(hi23);
        av.w = h2_bits(lo23);
        // codes of coordinate 32g + 4r + sigma for the 4 tokens
        uint32_t w4[4];
        constexpr int WPT = L::VCB / 4;  // value code words per token
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tok = tb + c + 4 * e;
          w4[e] = VB == 2 ? vc[tok * WPT + 2 * g + (r >> 2)] : vc[tok * WPT + 4 * g + (r >> 1)];
        }
        if (VB == 2) {
          const uint32_t byte = r & 3;
          const uint32_t sel = byte | ((4 + byte) << 8);
          const uint32_t x01 = __byte_perm(w4[0], w4[1], sel);
          const uint32_t x23 = __byte_perm(w4[2], w4[3], sel);
#pragma unroll
          for (int sg = 0; sg < 4; ++sg) {
            const uint32_t m = (3u << (2 * sg)) | (3u << (16 + 2 * sg));
            mma16816(dv[4 * g + sg], av, x01 & m, x23 & m);
          }
        } else {
          const uint32_t byte0 = 2 * (r & 1);
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            const uint32_t bt = byte0 + hb;
            const uint32_t sel = bt | ((4 + bt) << 8);
            const uint32_t x01 = __byte_perm(w4[0], w4[1], sel);
            const uint32_t x23 = __byte_perm(w4[2], w4[3], sel);
#pragma unroll
            for (int nib = 0; nib < 2; ++nib) {
              const uint32_t m = (15u << (4 * nib)) | (15u << (16 + 4 * nib));
              mma16816(dv[4 * g + 2 * hb + nib], av, x01 & m, x23 & m);
            }
          }
        }
      }
    }
    // The last warp to finish with this stage refills it with tile i + kStages.
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      const int prev = atomicAdd(&arrive_s[i % kStages], 1);
      if (prev == kWarpsMma - 1) {
        arrive_s[i % kStages] = 0;
        if (a.use_tma && i + kStages < ntiles && tile_full(i + kStages)) {
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          issue(i + kStages);
        }
      }
    }
  }

  if (__syncthreads_or(failed)) {
    // A bulk copy did not complete in time: flag it, then wait (bounded again) for
    // every copy this CTA may still have in flight before its shared memory goes away.
    if (failed && lane == 0) atomicOr(a.err, 1u);
    if (tid == 0) {
      // Phases of one mbarrier complete in order: waiting for the last batch issued
      // into each stage covers every copy still in flight.
      for (int st = 0; st < kStages; ++st)
        if (issued_s[st] > 0) mbar_wait(&bars[st], (uint32_t)((issued_s[st] - 1) & 1));
    }
    __syncthreads();
    return;
  }

  // ---- per-warp results -> CTA partial ---------------------------------------------
  l_run += __shfl_xor_sync(kFull, l_run, 1);
  l_run += __shfl_xor_sync(kFull, l_run, 2);
  // thread (r, c) holds sum p*min for groups 2c, 2c+1 (c < 2) in dmin[0] + dmin[2], dmin[1] + dmin[3]
  float lo_acc[4];
  {
    const float own0 = dmin[0] + dmin[2], own1 = dmin[1] + dmin[3];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const float v = __shfl_sync(kFull, (g & 1) ? own1 : own0, (lane & ~3) | (g >> 1));
      lo_acc[g] = v;
    }
  }
  float* red = reinterpret_cast<float*>(stage_base);  // [warp][head][kPartPadMma + d]
  constexpr int RS = kPartPadMma + kD;
  float* mine = red + (warp * 8 + r) * RS;
  if (c == 0) {
    mine[0] = m_run;
    mine[1] = l_run;
  }
#pragma unroll
  for (int nbk = 0; nbk < 16; ++nbk) {
    const int g = nbk >> 2, sg = nbk & 3;
    // n-block (g, sg): column n is coordinate 32g + 4n + sg; the code sat at mantissa
    // bit 2 sg (2-bit) or 4 (sg & 1) (4-bit) of the f16 operand.
    const int shift = VB == 2 ? 2 * sg : 4 * (sg & 1);
    const float unscale = ldexpf(1.f, 24 - shift);
#pragma unroll
    for (int col = 0; col < 2; ++col) {
      const int j = 32 * g + 4 * (2 * c + col) + sg;
      mine[kPartPadMma + j] = (dv[nbk][col] + dv[nbk][col + 2]) * unscale + lo_acc[g];
    }
  }
  __syncthreads();
  float* ws_base = a.ws_part + (size_t)unit * a.n_chunks * G * RS;
  for (int idx = tid; idx < G * kD; idx += kThreadsMma) {
    const int h = idx / kD, j = idx % kD;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarpsMma; ++w) mx = fmaxf(mx, red[(w * 8 + h) * RS]);
    float num = 0.f, den = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarpsMma; ++w) {
        const float* pw = red + (w * 8 + h) * RS;
        const float wt = pw[0] == -INFINITY ? 0.f : exp2f(pw[0] - mx);
        num = fmaf(wt, pw[kPartPadMma + j], num);
        den = fmaf(wt, pw[1], den);
      }
    }
    float* part = ws_base + ((size_t)chunk * G + h) * RS;
    part[kPartPadMma + j] = num;
    if (j == 0) {
      part[0] = mx;
      part[1] = den;
    }
  }

  // ---- the last CTA of this (sequence, KV head) merges the chunk partials -----------
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned int prev = atomicAdd(&a.cnt[unit], 1u);
    *last_s = (prev == (unsigned int)(a.n_chunks - 1)) ? 1 : 0;
  }
  __syncthreads();
  if (*last_s) {
    __threadfence();
    // Chunk weights per head first (m, l of every chunk), then one independent
    // weighted sum per output; the ring is free again and holds the weights.
    const size_t cs = (size_t)G * RS;
    const int nwt = a.n_chunks * 8;
    float* wts = red;        // [n_chunks][8] chunk weights
    float* hsum = red + nwt; // [8] running max per head, then [8] 1 / sum
    const bool fits = (size_t)(nwt + 16) * 4 <= (size_t)L::RING;
    __syncthreads();
    if (fits) {
      if (tid < 8) {
        float mx = -INFINITY;
        if (tid < G)
          for (int ch = 0; ch < a.n_chunks; ++ch) mx = fmaxf(mx, __ldcg(ws_base + ch * cs + (size_t)tid * RS));
        hsum[tid] = mx;
      }
      __syncthreads();
      for (int idx = tid; idx < nwt; idx += kThreadsMma) {
        const int ch = idx >> 3, h = idx & 7;
        float wt = 0.f;
        if (h < G) {
          const float mc = __ldcg(ws_base + ch * cs + (size_t)h * RS);
          wt = (mc == -INFINITY || hsum[h] == -INFINITY) ? 0.f : exp2f(mc - hsum[h]);
        }
        wts[idx] = wt;
      }
      __syncthreads();
      if (tid < 8) {
        float den = 0.f;
        if (tid < G)
          for (int ch = 0; ch < a.n_chunks; ++ch)
            den = fmaf(wts[ch * 8 + tid], __ldcg(ws_base + ch * cs + (size_t)tid * RS + 1), den);
        hsum[8 + tid] = den > 0.f ? 1.f / den : 0.f;
      }
      __syncthreads();
      for (int idx = tid; idx < G * kD; idx += kThreadsMma) {
        const int h = idx / kD, j = idx % kD;
        const float* base = ws_base + (size_t)h * RS + kPartPadMma + j;
        float num0 = 0.f, num1 = 0.f, num2 = 0.f, num3 = 0.f;
        int ch = 0;
        for (; ch + 4 <= a.n_chunks; ch += 4) {
          num0 = fmaf(wts[(ch + 0) * 8 + h], __ldcg(base + (ch + 0) * cs), num0);
          num1 = fmaf(wts[(ch + 1) * 8 + h], __ldcg(base + (ch + 1) * cs), num1);
          num2 = fmaf(wts[(ch + 2) * 8 + h], __ldcg(base + (ch + 2) * cs), num2);
          num3 = fmaf(wts[(ch + 3) * 8 + h], __ldcg(base + (ch + 3) * cs), num3);
        }
        for (; ch < a.n_chunks; ++ch) num0 = fmaf(wts[ch * 8 + h], __ldcg(base + ch * cs), num0);
        a.out[(size_t)(qrow0 + h) * kD + j] = ((num0 + num1) + (num2 + num3)) * hsum[8 + h];
      }
    } else {
      for (int idx = tid; idx < G * kD; idx += kThreadsMma) {
        const int h = idx / kD, j = idx % kD;
        const float* base = ws_base + (size_t)h * RS;
        float mx = -INFINITY;
        for (int ch = 0; ch < a.n_chunks; ++ch) mx = fmaxf(mx, __ldcg(base + ch * cs));
        float num = 0.f, den = 0.f;
        if (mx != -INFINITY) {
          for (int ch = 0; ch < a.n_chunks; ++ch) {
            const float* pp = base + ch * cs;
            const float mc = __ldcg(pp);
            const float wt = mc == -INFINITY ? 0.f : exp2f(mc - mx);
            den = fmaf(wt, __ldcg(pp + 1), den);
            num = fmaf(wt, __ldcg(pp + kPartPadMma + j), num);
          }
        }
        a.out[(size_t)(qrow0 + h) * kD + j] = den > 0.f ? num / den : 0.f;
      }
    }
    if (tid == 0) a.cnt[unit] = 0u;
  }
}

template <int LMB, int VB>
cudaError_t launch_mma_t(const MmaArgs& a, dim3 grid, cudaStream_t s) {
  using L = Layout<LMB, VB>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel<LMB, VB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
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
  return cudaLaunchKernelEx(&cfg, decode_mma_kernel<LMB, VB>, a);
}

}  // namespace

// For every operand element of the query fragments (chunk k, lane l, register q,
// half e) the layout fixes which query coordinate it scales and by which power of
// two (the inverse of the lone-bit f16 value its key bit becomes). Encoded per
// element as src (8 bits: 0..127 = qr index, 128..255 = 128 + sq index), code plane
// (1 bit), exponent + 16 (5 bits).
void build_frag_table(int lmb, uint16_t* table) {
  const int n = frag_chunks(lmb) * 32 * 4;
  for (int idx = 0; idx < n; ++idx) {
    const int q = idx & 3, l = (idx >> 2) & 31, k = idx >> 7;
    const int slot0 = 2 * (l & 3) + ((q & 2) ? 8 : 0);
    for (int e = 0; e < 2; ++e) {
      const int s = slot0 + e;
      const int cs = (s & 7) >> 1, half = s & 1;
      const int rho = 2 * (k & 7) + (s >> 3), wi = k >> 3;
      const int o = key_orig(rho) + 16 * half;
      const int ex = -lone_bit_log2(key_pos(rho));
      int src, plane = 0;
      if (wi < lmb) {
        const int sbit = 32 * (cs + 4 * wi) + o;  // bit of the key's code stream
        src = sbit / lmb;
        plane = sbit % lmb;
      } else {
        src = kD + 32 * cs + o;
      }
      table[2 * idx + e] = (uint16_t)(src | (plane << 8) | ((ex + 16) << 9));
    }
  }
}

size_t frag_table_entries(int lmb) { return (size_t)frag_chunks(lmb) * 32 * 4 * 2; }

bool mma_decode_supported(const tq_ctx* ctx, int G) {
  const Shape& sh = ctx->shape;
  if (sh.d != kD || sh.m != kM || G < 1 || G > 8 || !ctx->frag_table) return false;
  if (sh.lm_bits < 1 || sh.lm_bits > 2) return false;
  if (sh.lm_bits == 2) {
    // the codebook must be affine in its two bits (true for a symmetric codebook)
    const float* cc = ctx->cb.c;
    const float scale = fmaxf(fabsf(cc[0]), fabsf(cc[3]));
    if (fabsf((cc[3] - cc[0]) - ((cc[1] - cc[0]) + (cc[2] - cc[0]))) > 1e-6f * scale) return false;
  }
  return sh.v_bits == 2 || sh.v_bits == 4;
}

size_t mma_frag_bytes(int lm_bits) { return (size_t)frag_words(lm_bits) * 4; }

cudaError_t launch_decode_mma(const tq_ctx* ctx, const DecodePlan& plan, const void* q, int q_dtype, int batch,
                              int hq, int hkv, const int32_t* seq_lens, int64_t max_len, const uint8_t* k_codes,
                              const uint8_t* k_signs, const uint16_t* k_norms, const uint8_t* v_codes,
                              const uint16_t* v_params, float scale, float* scores, float* out, void* workspace,
                              cudaStream_t stream) {
  char* ws = static_cast<char*>(workspace);
  uint32_t* frag = reinterpret_cast<uint32_t*>(ws + plan.off_frag);
  float* part = reinterpret_cast<float*>(ws + plan.off_part);
  unsigned int* cnt = reinterpret_cast<unsigned int*>(ws + plan.off_cnt);
  const int G = hq / hkv, lmb = ctx->shape.lm_bits, vb = ctx->shape.v_bits;
  const float* cc = ctx->cb.c;

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
  pa.beta0 = cc[1] - cc[0];
  pa.beta1 = lmb > 1 ? cc[2] - cc[0] : 0.f;
  pa.frag = frag;
  pa.cnt = cnt;
  pa.table = ctx->frag_table;
  const size_t prep_smem = sizeof(float) * kD * kM;
  static bool prep_configured = false;
  if (!prep_configured) {
    cudaError_t ce = cudaFuncSetAttribute(prep_mma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem);
    if (ce == cudaSuccess)
      ce = cudaFuncSetAttribute(prep_mma_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem);
    if (ce != cudaSuccess) return ce;
    prep_configured = true;
  }
  if (lmb == 1)
    prep_mma_kernel<1><<<batch * hkv, kPrepThreads, prep_smem, stream>>>(pa);
  else
    prep_mma_kernel<2><<<batch * hkv, kPrepThreads, prep_smem, stream>>>(pa);
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
  a.hq = hq;
  a.hkv = hkv;
  a.G = G;
  a.n_chunks = plan.n_chunks;
  a.chunk_len = plan.chunk_len;
  a.scale = scale;
  a.scores = scores;
  a.out = out;
  a.ws_part = part;
  a.cnt = cnt;
  a.c0 = cc[0];
  a.use_tma = (max_len % 4 == 0) ? 1 : 0;
  a.err = ctx->d_err;
  const dim3 grid(plan.n_chunks, batch * hkv);
  if (ctx->prof_start) cudaEventRecord(ctx->prof_start, stream);
  if (lmb == 1)
    e = vb == 2 ? launch_mma_t<1, 2>(a, grid, stream) : launch_mma_t<1, 4>(a, grid, stream);
  else
    e = vb == 2 ? launch_mma_t<2, 2>(a, grid, stream) : launch_mma_t<2, 4>(a, grid, stream);
  if (ctx->prof_stop) cudaEventRecord(ctx->prof_stop, stream);
  return e;
}

}  // namespace tq
