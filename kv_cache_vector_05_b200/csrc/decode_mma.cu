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
// The cache is staged into shared memory by cp.async.bulk copies completing on
// mbarriers (4-deep ring of 64-token tiles); every wait is bounded and a timeout
// sets the context's error word and ends the CTA.
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
constexpr uint32_t kWaitLimit = 1u << 24;                 // polls of one mbarrier phase
constexpr unsigned long long kWaitNs = 2000000000ull;    // and at most 2 s of wall time

struct MmaArgs {
  const float* ws_q;  // [batch*hq][d+m]: qr then sq
  int q_stride;
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
  float* ws_part;
  int part_stride;
  float c0, beta0, beta1;  // affine form of the codebook
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
__device__ __forceinline__ int lone_bit_log2(int p) { return p <= 9 ? p - 24 : (1 << (p - 10)) - 15; }

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
  static constexpr int KCHUNKS = 8 * (LMB + 1);  // k16 chunks: 8 per key word per thread
};

template <int LMB, int VB>
__global__ void __launch_bounds__(kThreadsMma, 3) decode_mma_kernel(const __grid_constant__ MmaArgs a) {
  using L = Layout<LMB, VB>;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* stage_base = smem;                                                // kStages * STAGE
  uint4* afrag = reinterpret_cast<uint4*>(smem + kStages * L::STAGE);             // [KCHUNKS][32]
  float* qr_s = reinterpret_cast<float*>(afrag + L::KCHUNKS * 32);                // [8][128]
  float* sq_s = qr_s + 8 * kD;                                                     // [8][128]
  float* head_s = sq_s + 8 * kM;                                                   // [8][4]: Q, Sq, qs, ss
  uint64_t* bars = reinterpret_cast<uint64_t*>(head_s + 32);                       // [kStages]
  int* flag_s = reinterpret_cast<int*>(bars + kStages);

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
  const int ntiles = t1 > t0 ? (int)((t1 - t0 + kTileMma - 1) / kTileMma) : 0;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    *flag_s = 0;
  }
  __syncthreads();

  auto tile_full = [&](int i) -> bool { return t0 + (int64_t)(i + 1) * kTileMma <= t1; };
  auto issue = [&](int i) {  // one thread: bulk-copy tile i into its stage
    unsigned char* st = stage_base + (i % kStages) * L::STAGE;
    const int64_t v = vec0 + t0 + (int64_t)i * kTileMma;
    uint64_t* bar = &bars[i % kStages];
    mbar_expect_tx(bar, (uint32_t)L::STAGE);
    bulk_g2s(st + L::OFF_KC, a.k_codes + v * L::KCB, kTileMma * L::KCB, bar);
    bulk_g2s(st + L::OFF_KS, a.k_signs + v * L::SB, kTileMma * L::SB, bar);
    bulk_g2s(st + L::OFF_KN, reinterpret_cast<const uint8_t*>(a.k_norms) + v * 4, kTileMma * 4, bar);
    bulk_g2s(st + L::OFF_VC, a.v_codes + v * L::VCB, kTileMma * L::VCB, bar);
    bulk_g2s(st + L::OFF_VP, reinterpret_cast<const uint8_t*>(a.v_params) + v * L::PB, kTileMma * L::PB, bar);
  };
  if (tid == 0 && a.use_tma) {
    for (int i = 0; i < kStages && i < ntiles; ++i)
      if (tile_full(i)) issue(i);
  }

  // ---- per-CTA query operands -------------------------------------------------
  for (int idx = tid; idx < 8 * kD; idx += kThreadsMma) {
    const int h = idx / kD, j = idx % kD;
    qr_s[idx] = h < G ? a.ws_q[(size_t)(qrow0 + h) * a.q_stride + j] : 0.f;
    sq_s[idx] = h < G ? a.ws_q[(size_t)(qrow0 + h) * a.q_stride + kD + j] : 0.f;
  }
  __syncthreads();
  for (int h = warp; h < 8; h += kWarpsMma) {
    float qsum = 0.f, ssum = 0.f, qmax = 0.f, smax = 0.f;
    for (int j = lane; j < kD; j += 32) {
      qsum += qr_s[h * kD + j];
      ssum += sq_s[h * kD + j];
      qmax = fmaxf(qmax, fabsf(qr_s[h * kD + j]));
      smax = fmaxf(smax, fabsf(sq_s[h * kD + j]));
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
    }
  }
  __syncthreads();
  // A fragments: chunk k, lane l, register q (a0..a3) -> two f16 (row, slot) values.
  for (int idx = tid; idx < L::KCHUNKS * 32 * 4; idx += kThreadsMma) {
    const int q = idx & 3, l = (idx >> 2) & 31, k = idx >> 7;
    const int row_head = l >> 2;             // head of rows r and r + 8
    const bool lo_part = (q & 1) != 0;       // a1, a3: rows r + 8 hold the lo halves
    const int slot0 = 2 * (l & 3) + ((q & 2) ? 8 : 0);
    float v2[2] = {0.f, 0.f};
    if (row_head < G) {
      for (int e = 0; e < 2; ++e) {
        const int s = slot0 + e;
        const int cs = (s & 7) >> 1, half = s & 1;
        const int rho = 2 * (k & 7) + (s >> 3), wi = k >> 3;
        const int o = key_orig(rho) + 16 * half;
        const float inv = ldexpf(1.f, -lone_bit_log2(key_pos(rho)));
        float x;
        if (wi < LMB) {
          const int sb = 32 * (cs + 4 * wi) + o;
          const int j = sb / LMB, plane = sb % LMB;
          const float beta = plane == 0 ? a.beta0 : a.beta1;
          x = beta * qr_s[row_head * kD + j] / head_s[row_head * 4 + 2];
        } else {
          x = sq_s[row_head * kD + 32 * cs + o] / head_s[row_head * 4 + 3];
        }
        x *= inv;
        const float hi = __half2float(__float2half_rn(x));
        v2[e] = lo_part ? (x - hi) : hi;
      }
    }
    reinterpret_cast<uint32_t*>(afrag)[idx] = pack_h2(v2[0], v2[1]);
  }
  __syncthreads();

  // Per-thread head constants (row r = head r).
  const bool head_ok = r < G;
  const float Qr = head_s[r * 4 + 0], Sqr = head_s[r * 4 + 1];
  const float qs = head_s[r * 4 + 2], ss = head_s[r * 4 + 3];
  const float qjl = kQjl / (float)kM;
  constexpr float kLog2e = 1.4426950408889634f;

  float m_run = -INFINITY, l_run = 0.f;
  float lo_acc[4] = {0.f, 0.f, 0.f, 0.f};
  float dv[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) dv[i][0] = dv[i][1] = dv[i][2] = dv[i][3] = 0.f;

  bool failed = false;
  int fail_tile = 0;
  for (int i = 0; i < ntiles; ++i) {
    unsigned char* st = stage_base + (i % kStages) * L::STAGE;
    const int nt = (int)min((int64_t)kTileMma, t1 - t0 - (int64_t)i * kTileMma);
    if (a.use_tma && tile_full(i)) {
      const bool ok = mbar_wait(&bars[i % kStages], (uint32_t)((i / kStages) & 1));
      if (__syncthreads_or(!ok)) {
        failed = true;
        fail_tile = i;
        break;
      }
    } else {
      // Ragged or unaligned tile: plain 4-byte copies (all record sizes are multiples of 4).
      const int64_t v = vec0 + t0 + (int64_t)i * kTileMma;
      auto copy = [&](int off, const void* src, int bytes_per_tok) {
        const uint32_t* s32 = reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(src) + v * bytes_per_tok);
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
    if (tb < nt) {
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
      // token order of the thread's four values: c, c + 4, c + 8, c + 12
      float lg[4];
      const int64_t tok_abs0 = t0 + (int64_t)i * kTileMma + tb;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int nb = e >> 1, col = e & 1;
        const int tok = tb + c + 4 * e;
        const uint32_t nw = kn[tok];
        const float n = __half2float(__ushort_as_half((unsigned short)(nw & 0xffffu)));
        const float gamma = __half2float(__ushort_as_half((unsigned short)(nw >> 16)));
        const float lm = (dl[nb][col] + dl[nb][col + 2]) * qs;
        const float sg = (ds[nb][col] + ds[nb][col + 2]) * ss;
        const float lgt = a.scale * n * (a.c0 * Qr + lm + qjl * gamma * (2.f * sg - Sqr));
        const bool valid = head_ok && (c + 4 * e < nt - tb);
        lg[e] = valid ? lgt : -INFINITY;
        if (valid && a.scores) a.scores[(size_t)(qrow0 + r) * a.max_len + tok_abs0 + c + 4 * e] = lgt;
      }
      float cmax = fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3]));
      cmax = fmaxf(cmax, __shfl_xor_sync(kFull, cmax, 1));
      cmax = fmaxf(cmax, __shfl_xor_sync(kFull, cmax, 2));
      if (cmax > m_run) {
        const float corr = (m_run == -INFINITY) ? 0.f : exp2f((m_run - cmax) * kLog2e);
        l_run *= corr;
#pragma unroll
        for (int g = 0; g < 4; ++g) lo_acc[g] *= corr;
#pragma unroll
        for (int nbk = 0; nbk < 16; ++nbk)
#pragma unroll
          for (int e = 0; e < 4; ++e) dv[nbk][e] *= corr;
        m_run = cmax;
      }
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        p[e] = (lg[e] == -INFINITY) ? 0.f : exp2f((lg[e] - m_run) * kLog2e);
        l_run += p[e];
      }

      // ---- values: D[head hi/lo rows][coordinate columns] += P' x codes ----------
      // value params of the thread's 4 tokens: word g = (scale, min) of group g.
      // Tokens past the end of a ragged tile carry stale bytes: weight them by 0 and
      // keep their (scale, min) out of every product.
      uint4 par[4];
      bool tv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        tv[e] = c + 4 * e < nt - tb;
        par[e] = tv[e] ? vp[tb + c + 4 * e] : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float pw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t pr = g == 0 ? par[e].x : g == 1 ? par[e].y : g == 2 ? par[e].z : par[e].w;
          const float sc = __half2float(__ushort_as_half((unsigned short)(pr & 0xffffu)));
          const float mn = __half2float(__ushort_as_half((unsigned short)(pr >> 16)));
          lo_acc[g] = fmaf(p[e], mn, lo_acc[g]);
          pw[e] = p[e] * sc;
        }
        const __half2 h01 = __floats2half2_rn(pw[0], pw[1]);
        const __half2 h23 = __floats2half2_rn(pw[2], pw[3]);
        const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
        uint4 av;
        av.x = *reinterpret_cast<const uint32_t*>(&h01);
        av.y = pack_h2(pw[0] - f01.x, pw[1] - f01.y);
        av.z = *reinterpret_cast<const uint32_t*>(&h23);
        av.w = pack_h2(pw[2] - f23.x, pw[3] - f23.y);
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
    __syncthreads();  // every warp is done with this stage
    if (tid == 0 && a.use_tma && i + kStages < ntiles && tile_full(i + kStages)) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(i + kStages);
    }
  }

  if (failed) {
    // A bulk copy did not complete in time: flag it, then wait (bounded again) for
    // every copy this CTA may still have in flight before its shared memory goes away.
    if (tid == 0) {
      atomicOr(a.err, 1u);
      for (int j = fail_tile; j < ntiles && j < fail_tile + kStages; ++j)
        if (tile_full(j)) mbar_wait(&bars[j % kStages], (uint32_t)((j / kStages) & 1));
    }
    return;
  }

  // ---- per-warp results -> CTA partial ---------------------------------------------
  l_run += __shfl_xor_sync(kFull, l_run, 1);
  l_run += __shfl_xor_sync(kFull, l_run, 2);
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    lo_acc[g] += __shfl_xor_sync(kFull, lo_acc[g], 1);
    lo_acc[g] += __shfl_xor_sync(kFull, lo_acc[g], 2);
  }
  // Reuse the stage ring: [warp][head][kPartPadMma + d] floats.
  float* red = reinterpret_cast<float*>(stage_base);
  constexpr int RS = kPartPadMma + kD;
  float* mine = red + (warp * 8 + r) * RS;
  if (c == 0) {
    mine[0] = m_run;
    mine[1] = l_run;
  }
#pragma unroll
  for (int nbk = 0; nbk < 16; ++nbk) {
    const int g = nbk >> 2, sg = nbk & 3;
    int pos, shift;  // coordinate offset within the group and mantissa position of the code
    if (VB == 2) {
      pos = sg;
      shift = 2 * sg;
    } else {
      pos = sg;  // nibble nib of byte 2(r&1)+hb -> coordinate 32g + 4r + 2hb + nib
      shift = 4 * (sg & 1);
    }
    const float unscale = ldexpf(1.f, 24 - shift);
#pragma unroll
    for (int col = 0; col < 2; ++col) {
      const int n = 2 * c + col;  // D column = coordinate 32g + 4n + pos
      const int j = 32 * g + 4 * n + pos;
      mine[kPartPadMma + j] = (dv[nbk][col] + dv[nbk][col + 2]) * unscale + lo_acc[g];
    }
  }
  __syncthreads();
  // Merge the warps' partials of each head and write one partial per (chunk, head).
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
        const float wt = pw[0] == -INFINITY ? 0.f : exp2f((pw[0] - mx) * kLog2e);
        num = fmaf(wt, pw[kPartPadMma + j], num);
        den = fmaf(wt, pw[1], den);
      }
    }
    float* part = a.ws_part + ((size_t)(unit * a.n_chunks + chunk) * G + h) * a.part_stride;
    part[kPartPadMma + j] = num;
    if (j == 0) {
      part[0] = mx;
      part[1] = den;
    }
  }
}

template <int LMB, int VB>
size_t mma_smem_bytes() {
  using L = Layout<LMB, VB>;
  return (size_t)kStages * L::STAGE + sizeof(uint4) * L::KCHUNKS * 32 + sizeof(float) * (16 * kD + 32) +
         sizeof(uint64_t) * kStages + 16;
}

template <int LMB, int VB>
cudaError_t launch_mma_t(const MmaArgs& a, dim3 grid, cudaStream_t s) {
  static bool configured = false;
  const size_t smem = mma_smem_bytes<LMB, VB>();
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel<LMB, VB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  decode_mma_kernel<LMB, VB><<<grid, kThreadsMma, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

bool mma_decode_supported(const tq_ctx* ctx, int G) {
  const Shape& sh = ctx->shape;
  if (sh.d != kD || sh.m != kM || G < 1 || G > 8) return false;
  if (sh.lm_bits < 1 || sh.lm_bits > 2) return false;
  if (sh.lm_bits == 2) {
    // the codebook must be affine in its two bits (true for a symmetric codebook)
    const float* cc = ctx->cb.c;
    const float scale = fmaxf(fabsf(cc[0]), fabsf(cc[3]));
    if (fabsf((cc[3] - cc[0]) - ((cc[1] - cc[0]) + (cc[2] - cc[0]))) > 1e-6f * scale) return false;
  }
  return sh.v_bits == 2 || sh.v_bits == 4;
}

cudaError_t launch_decode_mma(const tq_ctx* ctx, const DecodePlan& plan, const float* ws_q, int q_stride,
                              float* ws_part, int part_stride, int batch, int hq, int hkv,
                              const int32_t* seq_lens, int64_t max_len, const uint8_t* k_codes,
                              const uint8_t* k_signs, const uint16_t* k_norms, const uint8_t* v_codes,
                              const uint16_t* v_params, float scale, float* scores, cudaStream_t stream) {
  MmaArgs a;
  a.ws_q = ws_q;
  a.q_stride = q_stride;
  a.k_codes = k_codes;
  a.k_signs = k_signs;
  a.k_norms = k_norms;
  a.v_codes = v_codes;
  a.v_params = v_params;
  a.seq_lens = seq_lens;
  a.max_len = max_len;
  a.hq = hq;
  a.hkv = hkv;
  a.G = hq / hkv;
  a.n_chunks = plan.n_chunks;
  a.chunk_len = plan.chunk_len;
  a.scale = scale;
  a.scores = scores;
  a.ws_part = ws_part;
  a.part_stride = part_stride;
  const float* cc = ctx->cb.c;
  a.c0 = cc[0];
  a.beta0 = cc[1] - cc[0];
  a.beta1 = ctx->shape.lm_bits > 1 ? cc[2] - cc[0] : 0.f;
  a.use_tma = (max_len % 4 == 0) ? 1 : 0;
  a.err = ctx->d_err;
  const dim3 grid(plan.n_chunks, batch * hkv);
  const int lmb = ctx->shape.lm_bits, vb = ctx->shape.v_bits;
  if (lmb == 1) return vb == 2 ? launch_mma_t<1, 2>(a, grid, stream) : launch_mma_t<1, 4>(a, grid, stream);
  return vb == 2 ? launch_mma_t<2, 2>(a, grid, stream) : launch_mma_t<2, 4>(a, grid, stream);
}

}  // namespace tq
