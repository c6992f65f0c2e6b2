// Decode attention with the key scores on the 5th-generation tensor cores (d = 128; keys of
// 1- to 3-bit Lloyd-Max codes from a codebook symmetric about zero, with the 128-bit QJL
// sketch or without it; 2- or 4-bit values; up to 8 query heads per KV head).
//
// Same mathematics as decode_kernel and decode_mma_kernel (the skill card "turboquant-
// pytorch", "Что делает": attention scores straight from the compressed keys; the discosf
// news item, "一句话看懂": fused decode kernels on the compressed cache): logit = scale * n *
// (<qr, c[idx]> + sqrt(pi/2)/m * gamma * <sq, s>), online softmax, sum of p * (min + scale *
// code). What changes is where the work runs.
//
// Scores. A tile is 128 tokens of one (sequence, KV head) unit, the M dimension of one
// tcgen05.mma. Row t of the A operand holds every packed key bit of token t as one unsigned
// 8-bit element: the code bits, for 3-bit codes one parity bit per code, and the QJL sign
// bits. Column n of the B operand holds, for one query head, one signed 8-bit digit of each
// bit's weight (four digits, 31 bits together, as four columns: as fine as the fp32 weights
// themselves); the int32 sums of kind::i8 are exact, and the digits are recombined in fp32
// afterwards.
//  * A symmetric codebook is an odd function of the code's bits taken as +-1, so it is
//    affine in them: c[b0 + 2 b1] = c0 + (c1 - c0) b0 + (c2 - c0) b1 at two bits, and at
//    three bits the odd part also holds the product of the three signs, which is affine in
//    the parity b0 ^ b1 ^ b2: c[idx] = kappa + beta0 b0 + beta1 b1 + beta2 b2 + beta3 par.
//    So <qr, c[idx]> = kappa sum(qr) + sum over bits of (beta_plane qr_j) * bit.
//  * A packed word becomes elements by one AND: mask q keeps bit q of each of its four bytes
//    (of the word shifted right by four for q >= 4), giving bytes worth 2^(q mod 4) or 0;
//    the weights in B are divided by that power of two. Eight masks of a word are one K-step
//    (32 elements) of the MMA, eight tensor-memory columns of the token's row.
//  * The parities of a group of 32 three-bit codes (three words) fit one word: with X the
//    96-bit stream XORed with itself shifted by one and by two, bit 3j of X is code j's
//    parity, and the bits 3j fall on distinct positions of the three 32-bit words (0, 1, 2
//    mod 3), so one word keeps them all: bit p holds code (32 (p mod 3) + p) / 3.
// Values. out = sum_t p_t (min + scale * code): the warps of the value role run mma.sync
// m16n8k16 with rows = value coordinates, k = tokens, columns = 4 query heads x (hi, lo):
// a 2- or 4-bit code in the low mantissa bits of an f16 is an exact subnormal (the power of
// two is undone at the end), and p * scale arrives as an f16 hi + lo pair (an exact
// TwoProduct) computed once per token by the softmax role; the group minima enter through
// one more MMA with p itself.
// Online softmax in base 2 with one reference maximum per query head for the whole CTA,
// moved only when a logit exceeds it by more than 2 (p < 4, so p * scale stays finite in f16
// for value scales below 16376); when it moves, the value role rescales its sums.
//
// Roles (512 threads, one CTA per SM, the units' tiles laid end to end and split evenly
// over the CTAs as in decode_mma_kernel):
//   warp 0      streams the packed tiles into a ring of shared-memory stages (bulk copies;
//               warp-wide plain copies for a ragged or unaligned tile);
//   warp 1      one thread issues every MMA;
//   warp 2      one thread loads each unit's query operand (digits + logit constants);
//   warps 4-7   one token per thread: expand the key bits into tensor memory;
//   warps 8-11  one token per thread: read the scores back, logits, online softmax, write
//               the value weights (p * scale, hi + lo) to shared memory;
//   warps 12-15 32 tokens each: accumulate the values.
// Tensor memory holds two A buffers (key elements) and two D buffers (digit sums), so the
// expansion of tile i + 1 and the softmax of tile i - 1 overlap the MMA of tile i.
// Every wait is bounded: on a timeout the CTA raises an abort flag that every role polls,
// sets the context's error word, drains the copies and MMAs it issued and returns.
#include <cuda_runtime.h>
#include <math.h>

#include "tq_device.cuh"
#include "tq_sm100.cuh"

namespace tq {
namespace {

namespace s1 = tq::sm100;

constexpr int kD = 128;
constexpr int kM = 128;
constexpr int kTileTc = 128;       // tokens per tile = MMA rows
constexpr int kThreadsTc = 512;
constexpr int kPairStride = 68;    // words per (group, head, part) row of the value weights: 64 token pairs + 4
constexpr int kPrepTcThreads = 256;
constexpr float kSlackTc = 2.f;
constexpr uint32_t kWaitPolls = 1u << 24;
constexpr unsigned long long kWaitNs = 2000000000ull;
// |Q| <= 2^30 keeps the top one of four balanced 8-bit digits in [-64, 64]
constexpr float kQmax = 1073741824.f;
constexpr int kDigits = 4;

// Named barriers: 1 = softmax warps, 2 = value warps (0 is __syncthreads).
constexpr int kBarSm = 1, kBarV = 2;

template <int LMB, bool QJL, int VB, int NB>
struct TcLayout {
  static constexpr int HG = 4 * NB;                    // query-head slots
  static constexpr int CW = 4 * LMB;                   // code words per token
  static constexpr int PW = LMB == 3 ? 4 : 0;          // parity words
  static constexpr int SW = QJL ? 4 : 0;               // sign words
  static constexpr int KSC = CW + PW;                  // K-steps of the code bits
  static constexpr int EW = KSC + SW;                  // K-steps = element words per token
  static constexpr int KB = 32 * EW;                   // bytes of one B row
  static constexpr int NC = kDigits * HG;              // code columns (4 digits per head)
  static constexpr int N = ((NC + (QJL ? NC : 0)) + 15) / 16 * 16;
  static constexpr int TA = 8 * EW;                    // tensor-memory columns of one A buffer
  static constexpr int TM_D = 2 * TA;                  // D[b] at TM_D + b * N
  static_assert(2 * TA + 2 * N <= 512, "tensor memory");
  static constexpr int KCB = LMB * 16, SB = QJL ? 16 : 0, VCB = VB * 16, PB = 16;
  static constexpr int REC = KCB + SB + 4 + VCB + PB;
  static constexpr int STAGE = kTileTc * REC;
  static constexpr int OFF_KC = 0, OFF_KS = kTileTc * KCB, OFF_KN = OFF_KS + kTileTc * SB;
  static constexpr int OFF_VC = OFF_KN + kTileTc * 4, OFF_VP = OFF_VC + kTileTc * VCB;
  static constexpr int BOP = N * KB;                   // digits, K-major, 128-byte swizzle
  static constexpr int BBUF = BOP + HG * 16;           // + logit constants (float4 per head)
  static constexpr int BBUF_AL = (BBUF + 1023) / 1024 * 1024;
  static constexpr int PPW = 4 * HG * 2 * kPairStride + 16;  // value weights p * scale [group][head][part][pair]
  static constexpr int PMW = HG * 2 * kPairStride;     // p [head][part][pair] for the minima
  static constexpr int PHDR = 16;                      // flag, rescale factors [HG]
  static constexpr int PBUF = (PPW + PMW + PHDR) * 4;
  static constexpr int SM_B = 0;
  static constexpr int SM_P = 2 * BBUF_AL;
  static constexpr int SM_VR = SM_P + 2 * PBUF;        // [4 value warps][HG][d] unit-end sums
  static constexpr int SM_LR = SM_VR + 4 * HG * kD * 4;   // [HG][128] unit-end sums of p
  static constexpr int SM_TMX = SM_LR + HG * kTileTc * 4; // [4 softmax warps][HG] tile maxima
  static constexpr int SM_BAR = SM_TMX + 4 * HG * 4;
  static constexpr int NBAR_FIXED = 16;
  static constexpr int SM_MISC = SM_BAR + 8 * (NBAR_FIXED + 2 * 12);  // TMEM address, abort flag
  static constexpr int SM_RING = (SM_MISC + 16 + 127) / 128 * 128;
  static constexpr int BUDGET = 227 * 1024 - 1024 - SM_RING;
  static constexpr int NST = BUDGET / STAGE > 8 ? 8 : BUDGET / STAGE;
  static_assert(NST >= 3 && NST <= 12, "stages");
  static constexpr size_t SMEM = (size_t)SM_RING + (size_t)NST * STAGE + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(STAGE % 16 == 0 && BBUF % 16 == 0, "16-byte bulk copies");
};

struct TcArgs {
  const uint8_t* bop;       // [units][BBUF] query operand of each unit (prep_tc_kernel)
  const uint8_t* k_codes;
  const uint8_t* k_signs;
  const uint16_t* k_norms;
  const uint8_t* v_codes;
  const uint16_t* v_params;
  const int32_t* seq_lens;
  int64_t max_len;
  Paging pg;
  int hq, hkv, G;
  int64_t tiles_per_unit;
  int64_t total_tiles;
  int s_max;
  float* scores;
  float* ws_part;           // [units][s_max][G][4 + d]
  int use_tma;
  unsigned int* err;
};

// ------------------------------------------------------------------ small helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return s1::smem_u32(p); }

// Bounded wait on an mbarrier phase that also gives up as soon as another role raised the
// CTA's abort flag. Returns false on a timeout or an abort.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, const volatile int* abort_flag) {
  const uint32_t a = smem_addr(bar);
  unsigned long long start = 0;
  for (uint32_t it = 0; it < kWaitPolls; ++it) {
    uint32_t done;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
        : "=r"(done)
        : "r"(a), "r"(parity), "r"(20000u)
        : "memory");
    if (done) return true;
    if (*abort_flag) return false;
    if (it == 0) start = s1::global_ns();
    else if ((it & 63) == 0 && s1::global_ns() - start > kWaitNs) return false;
  }
  return false;
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag) { *abort_flag = 1; }

// D[tmem] (+)= A[tmem] x B[smem], kind::i8 (u8 x s8 -> s32), one CTA.
__device__ __forceinline__ void umma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::i8: u8 A x s8 B -> s32 D, K-major operands.
__host__ __device__ constexpr uint32_t idesc_u8s8_s32(int M, int N) {
  return (2u << 4)                       // D format s32
         | (0u << 7)                     // A format u8
         | (1u << 10)                    // B format s8
         | ((uint32_t)(N >> 3) << 17)    // N / 8
         | ((uint32_t)(M >> 4) << 24);   // M / 16
}

// Warp-wide load of 16 consecutive 32-bit columns of the warp's 32 lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

__device__ __forceinline__ void mma16816_tc(float (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t hbits(__half2 h) { return *reinterpret_cast<const uint32_t*>(&h); }
__device__ __forceinline__ __half2 h2of(uint32_t w) { return *reinterpret_cast<const __half2*>(&w); }

__device__ __forceinline__ void named_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ bool named_sync_or(int id, int count, bool p) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred q, o; setp.ne.u32 q, %1, 0; bar.red.or.pred o, %2, %3, q; selp.u32 %0, 1, 0, o; }"
      : "=r"(r)
      : "r"((uint32_t)p), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// Mask q of a packed word: bit q of each byte (bit q - 4 of each byte of w >> 4 for q >= 4),
// in place, so byte i holds 2^(q mod 4) * bit(8 i + q).
template <int Q>
__device__ __forceinline__ uint32_t bitmask_el(uint32_t w, uint32_t w4) {
  return (Q < 4 ? w : w4) & (0x01010101u << (Q & 3));
}

// Parity word of the 32 three-bit codes held in three consecutive stream words: bit p is the
// parity of code (32 (p mod 3) + p) / 3.
__device__ __forceinline__ uint32_t parity_word(uint32_t x0, uint32_t x1, uint32_t x2) {
  const uint32_t X0 = x0 ^ __funnelshift_r(x0, x1, 1) ^ __funnelshift_r(x0, x1, 2);
  const uint32_t X1 = x1 ^ __funnelshift_r(x1, x2, 1) ^ __funnelshift_r(x1, x2, 2);
  const uint32_t X2 = x2 ^ (x2 >> 1) ^ (x2 >> 2);
  return (X0 & 0x49249249u) | (X1 & 0x92492492u) | (X2 & 0x24924924u);
}

// Word offset of the value-weight row (group g, head h, part) in a P buffer; groups 2-3 sit
// 16 words further so that the even and odd threads of a token pair write distinct banks.
__device__ __forceinline__ int prow(int g, int h, int part, int HG) {
  return ((g * HG + h) * 2 + part) * kPairStride + (g >> 1) * 16;
}

// CTA owning global tile g when CTA k takes tiles [k T / P, (k + 1) T / P).
__device__ __forceinline__ int64_t owner_tc(int64_t g, int64_t P, int64_t T) { return ((g + 1) * P - 1) / T; }

// ------------------------------------------------------------------ prep kernel

struct PrepTcArgs {
  const void* q;
  int q_dtype;
  int hq, hkv, G, rot;
  float inv_sqrt_d;
  const float* St;   // [d][m]
  const float* PiT;  // [d][d] (Haar)
  Codebook cb;
  float kappa;       // constant term of the codebook's bit expansion
  float beta[4];     // weights of the code bits (and of the parity at 3 bits)
  float sl2;         // softmax scale * log2(e)
  uint8_t* bop;      // [units][BBUF]
};

// One CTA per (sequence, KV head): rotate the G queries, form S qr, then write the unit's
// B operand (the digits of every key bit's weight, swizzled K-major rows of N columns)
// and the per-head logit constants.
template <int LMB, bool QJL, int VB, int NB>
__global__ void __launch_bounds__(kPrepTcThreads) prep_tc_kernel(const __grid_constant__ PrepTcArgs a) {
  using L = TcLayout<LMB, QJL, VB, NB>;
  constexpr int HG = L::HG;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(16) float stp_s[];  // [d][m] staged S^T (or Pi^T), 64 KB
  __shared__ float x_s[HG * kD];
  __shared__ float qr_s[HG * kD];
  __shared__ float sq_s[HG * kM];
  __shared__ float ec_s[HG], es_s[HG];  // 2^E of the code and sign digits
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int unit = blockIdx.x;
  const int b = unit / a.hkv, kvh = unit % a.hkv, G = a.G;
  const int qrow0 = b * a.hq + kvh * G;
  for (int idx = tid; idx < HG * kD; idx += kPrepTcThreads) {
    const int h = idx / kD, j = idx % kD;
    float x = 0.f;
    if (h < G) {
      const size_t off = (size_t)(qrow0 + h) * kD + j;
      x = a.q_dtype == TQ_F32 ? __ldg(static_cast<const float*>(a.q) + off)
                              : __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[off]);
    }
    if (a.rot == TQ_ROT_HADAMARD) x = flip_sign(x, (a.cb.sign_bits[j / 32] >> (j % 32)) & 1u);
    x_s[idx] = x;
  }
  __syncthreads();
  if (a.rot == TQ_ROT_HADAMARD) {
    for (int hs = 1; hs < kD; hs <<= 1) {
      for (int p = tid; p < HG * (kD / 2); p += kPrepTcThreads) {
        const int h = p / (kD / 2), i = p % (kD / 2);
        const int i0 = h * kD + (i / hs) * 2 * hs + (i % hs);
        const float u = x_s[i0], w = x_s[i0 + hs];
        x_s[i0] = u + w;
        x_s[i0 + hs] = u - w;
      }
      __syncthreads();
    }
    for (int idx = tid; idx < HG * kD; idx += kPrepTcThreads) qr_s[idx] = x_s[idx] * a.inv_sqrt_d;
  } else {
    for (int w = tid; w < kD * kD / 4; w += kPrepTcThreads)
      reinterpret_cast<float4*>(stp_s)[w] = __ldg(reinterpret_cast<const float4*>(a.PiT) + w);
    __syncthreads();
    for (int idx = tid; idx < HG * kD; idx += kPrepTcThreads) {
      const int h = idx / kD, i = idx % kD;
      float acc = 0.f;
      for (int j = 0; j < kD; ++j) acc = fmaf(stp_s[j * kD + i], x_s[h * kD + j], acc);
      qr_s[idx] = acc;
    }
    __syncthreads();
  }
  __syncthreads();
  if constexpr (QJL) {
    for (int w = tid; w < kD * kM / 4; w += kPrepTcThreads)
      reinterpret_cast<float4*>(stp_s)[w] = __ldg(reinterpret_cast<const float4*>(a.St) + w);
    __syncthreads();
    for (int idx = tid; idx < HG * kM; idx += kPrepTcThreads) {
      const int h = idx / kM, i = idx % kM;
      float acc = 0.f;
      for (int j = 0; j < kD; ++j) acc = fmaf(stp_s[j * kM + i], qr_s[h * kD + j], acc);
      sq_s[idx] = acc;
    }
    __syncthreads();
  }
  float* kconst = reinterpret_cast<float*>(a.bop + (size_t)unit * L::BBUF + L::BOP);
  if (warp < HG) {
    const int h = warp;
    float qsum = 0.f, ssum = 0.f, qmax = 0.f, smax = 0.f;
    for (int j = lane; j < kD; j += 32) {
      qsum += qr_s[h * kD + j];
      qmax = fmaxf(qmax, fabsf(qr_s[h * kD + j]));
      if (QJL) {
        ssum += sq_s[h * kM + j];
        smax = fmaxf(smax, fabsf(sq_s[h * kM + j]));
      }
    }
    qsum = warp_sum(qsum);
    ssum = warp_sum(ssum);
    qmax = warp_max(qmax);
    smax = warp_max(smax);
    if (lane == 0) {
      float bmax = 0.f;
#pragma unroll
      for (int p = 0; p < 4; ++p) bmax = fmaxf(bmax, fabsf(a.beta[p]));
      const float wc = qmax * bmax, ws = smax;
      // 2^E with E = floor(log2(kQmax / max |weight|)): every digit set stays in range
      const int ec = wc > 0.f ? min((int)floorf(log2f(kQmax / wc)), 100) : 0;
      const int es = ws > 0.f ? min((int)floorf(log2f(kQmax / ws)), 100) : 0;
      ec_s[h] = ldexpf(1.f, ec);
      es_s[h] = ldexpf(1.f, es);
      constexpr float kSignW = kQjl / (float)kM;
      // logit (base 2) = n * (k1 + k2 * code + gamma * (k3 * sign - k4)), code and sign the
      // decode kernel's recombined digit sums
      kconst[h * 4 + 0] = a.sl2 * a.kappa * qsum;
      kconst[h * 4 + 1] = a.sl2 * ldexpf(1.f, -ec);
      kconst[h * 4 + 2] = QJL ? a.sl2 * kSignW * 2.f * ldexpf(1.f, -es) : 0.f;
      kconst[h * 4 + 3] = QJL ? a.sl2 * kSignW * ssum : 0.f;
    }
  }
  __syncthreads();
  // The B operand: row n (a column of D), byte k = 32 ks + 4 q + i: element i of mask q of
  // element word ks. Code columns n = 4 h + digit, sign columns NC + 4 h + digit.
  uint8_t* bop = a.bop + (size_t)unit * L::BBUF;
  constexpr int WPR = L::KB / 4;  // 32-bit words per row
  for (int w = tid; w < L::N * WPR; w += kPrepTcThreads) {
    const int n = w / WPR, kw = w % WPR;
    const int ks = kw / 8, q = kw % 8;
    const bool code_col = n < L::NC, sign_col = QJL && n >= L::NC && n < 2 * L::NC;
    const int h = code_col ? n / kDigits : (n - L::NC) / kDigits;
    const int dg = code_col ? n % kDigits : (n - L::NC) % kDigits;
    const bool live = (code_col && ks < L::KSC) || (sign_col && ks >= L::KSC);
    uint32_t packed = 0;
    if (live && h < G) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float wgt, e2;
        if (code_col) {
          int j, plane;
          if (ks < L::CW) {
            const int sbit = 32 * ks + 8 * i + q;  // bit of the code stream
            j = sbit / LMB;
            plane = sbit % LMB;
          } else {  // parity word ks - CW, bit p: code 32 (ks - CW) + (32 (p mod 3) + p) / 3
            const int p = 8 * i + q;
            j = 32 * (ks - L::CW) + (32 * (p % 3) + p) / 3;
            plane = 3;
          }
          wgt = a.beta[plane] * qr_s[h * kD + j];
          e2 = ec_s[h];
        } else {
          wgt = sq_s[h * kM + 32 * (ks - L::KSC) + 8 * i + q];
          e2 = es_s[h];
        }
        // Q = round(weight * 2^E / 2^(q mod 4)) as balanced digits d0 + 2^8 d1 + 2^16 d2 + 2^24 d3
        const int Q = __float2int_rn(wgt * e2 * (1.f / (float)(1 << (q & 3))));
        const int d0 = ((Q + 128) & 255) - 128;
        const int Q1 = (Q - d0) >> 8;
        const int d1 = ((Q1 + 128) & 255) - 128;
        const int Q2 = (Q1 - d1) >> 8;
        const int d2 = ((Q2 + 128) & 255) - 128;
        const int d3 = (Q2 - d2) >> 8;
        const int dig = dg == 0 ? d0 : dg == 1 ? d1 : dg == 2 ? d2 : d3;
        packed |= ((uint32_t)dig & 0xffu) << (8 * i);
      }
    }
    *reinterpret_cast<uint32_t*>(bop + s1::sw128_offset(n, 2 * kw, L::N)) = packed;
  }
}

// ------------------------------------------------------------------ decode kernel

template <int LMB, bool QJL, int VB, int NB>
__global__ void __launch_bounds__(kThreadsTc, 1) decode_tc_kernel(const __grid_constant__ TcArgs a) {
  using L = TcLayout<LMB, QJL, VB, NB>;
  constexpr int HG = L::HG, NST = L::NST;
  constexpr int RS = 4 + kD;  // partial row: m, l, pad, pad, acc[d]
  constexpr float kLn2 = 0.6931471805599453f;
  extern __shared__ unsigned char smem_tc_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(((uintptr_t)smem_tc_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::SM_BAR);
  uint64_t* full = bars;                 // [NST] stage landed
  uint64_t* empty = bars + NST;          // [NST] stage consumed (12 warps)
  uint64_t* afull = bars + 2 * NST;      // [2] key elements written (4 warps)
  uint64_t* mmad = afull + 2;            // [2] MMA of the tile done (commit)
  uint64_t* dempty = mmad + 2;           // [2] digit sums read (4 warps)
  uint64_t* pfull = dempty + 2;          // [2] value weights written (4 warps)
  uint64_t* pempty = pfull + 2;          // [2] value weights consumed (4 warps)
  uint64_t* fbfull = pempty + 2;         // [2] query operand landed
  uint64_t* fbempty = fbfull + 2;        // [2] query operand released (MMA commit + 4 softmax warps)
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(sm + L::SM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::SM_MISC + 4);
  int* issued_s = reinterpret_cast<int*>(sm + L::SM_MISC + 8);  // bulk batches into stages (unused slot)
  (void)issued_s;
  unsigned char* ring = sm + L::SM_RING;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.G;
  const int64_t P = gridDim.x, kcta = blockIdx.x;
  const int64_t Tu = a.tiles_per_unit, Tt = a.total_tiles;
  const int64_t g0 = kcta * Tt / P, g1 = (kcta + 1) * Tt / P;
  const int ntl = (int)(g1 - g0);
  const int u_first = ntl > 0 ? (int)(g0 / Tu) : 0;
  const int n_units = ntl > 0 ? (int)((g1 - 1) / Tu) - u_first + 1 : 0;

  if (warp == 0) {
    s1::tmem_alloc(tmem_s, 512);
    s1::tmem_relinquish();
  }
  if (tid == 32) {
    for (int s = 0; s < NST; ++s) {
      s1::mbar_init(&full[s], 1);
      s1::mbar_init(&empty[s], 12);
    }
    for (int b = 0; b < 2; ++b) {
      s1::mbar_init(&afull[b], 4);
      s1::mbar_init(&mmad[b], 1);
      s1::mbar_init(&dempty[b], 4);
      s1::mbar_init(&pfull[b], 4);
      s1::mbar_init(&pempty[b], 4);
      s1::mbar_init(&fbfull[b], 1);
      s1::mbar_init(&fbempty[b], 5);
    }
    *abort_flag = 0;
    s1::mbar_init_fence();
  }
  s1::fence_before_sync();
  __syncthreads();
  s1::fence_after_sync();
  const uint32_t tmem = *tmem_s;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // Per tile i of this CTA: its unit, its first token and its valid token count.
  auto unit_len = [&](int u) -> int64_t {
    int64_t len = a.max_len;
    if (a.seq_lens) len = min((int64_t)max(a.seq_lens[u / a.hkv], 0), a.max_len);
    return len;
  };
  auto tile_info = [&](int i, int& u, int64_t& tok0, int& nt) {
    const int64_t g = g0 + i;
    u = (int)(g / Tu);
    tok0 = (g - (int64_t)u * Tu) * kTileTc;
    nt = (int)max((int64_t)0, min((int64_t)kTileTc, unit_len(u) - tok0));
  };
  auto last_of_unit = [&](int i) -> bool {
    const int64_t g = g0 + i;
    return i == ntl - 1 || (g + 1) % Tu == 0;
  };

  bool failed = false;
  if (warp == 0) {
    // ============================================================ producer: packed tiles
    int bulk_issued[12] = {};  // bulk batches issued per stage (for the failure drain)
    int uses[12] = {};         // phases started per stage
    for (int i = 0; i < ntl && !failed; ++i) {
      const int s = i % NST;
      if (i >= NST) {
        bool ok = true;
        if (lane == 0) ok = wait_phase(&empty[s], (uint32_t)((i / NST) - 1) & 1u, abort_flag);
        ok = __shfl_sync(kFull, ok, 0);
        if (!ok) {
          failed = true;
          break;
        }
      }
      int u, nt;
      int64_t tok0;
      tile_info(i, u, tok0, nt);
      unsigned char* st = ring + s * L::STAGE;
      uses[s] += 1;
      if (a.use_tma && nt == kTileTc) {
        if (lane == 0) {
          // the consumers' generic reads of the stage are ordered before the async-proxy writes
          s1::fence_async_smem();
          const int64_t v = record_row(a.pg, a.max_len, u, tok0, a.err);
          s1::mbar_expect_tx(&full[s], (uint32_t)L::STAGE);
          s1::bulk_g2s(st + L::OFF_KC, a.k_codes + v * L::KCB, kTileTc * L::KCB, &full[s]);
          if constexpr (QJL) s1::bulk_g2s(st + L::OFF_KS, a.k_signs + v * L::SB, kTileTc * L::SB, &full[s]);
          s1::bulk_g2s(st + L::OFF_KN, reinterpret_cast<const uint8_t*>(a.k_norms) + v * 4, kTileTc * 4, &full[s]);
          s1::bulk_g2s(st + L::OFF_VC, a.v_codes + v * L::VCB, kTileTc * L::VCB, &full[s]);
          s1::bulk_g2s(st + L::OFF_VP, reinterpret_cast<const uint8_t*>(a.v_params) + v * L::PB, kTileTc * L::PB,
                       &full[s]);
          bulk_issued[s] += 1;
        }
      } else {
        // ragged or unaligned tile: the warp copies the valid records with 4-byte loads
        if (nt > 0) {
          const int64_t v = record_row(a.pg, a.max_len, u, tok0, a.err);
          auto copy = [&](int off, const void* src, int bpt) {
            const uint32_t* s32 = reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(src) + v * bpt);
            uint32_t* d32 = reinterpret_cast<uint32_t*>(st + off);
            for (int w = lane; w < nt * bpt / 4; w += 32) d32[w] = s32[w];
          };
          copy(L::OFF_KC, a.k_codes, L::KCB);
          if constexpr (QJL) copy(L::OFF_KS, a.k_signs, L::SB);
          copy(L::OFF_KN, a.k_norms, 4);
          copy(L::OFF_VC, a.v_codes, L::VCB);
          copy(L::OFF_VP, a.v_params, L::PB);
        }
        __syncwarp();
        if (lane == 0) s1::mbar_arrive(&full[s]);
      }
    }
    if (failed && lane == 0) raise_abort(abort_flag);
    __syncwarp();
    if (lane == 0 && *abort_flag) {
      // Consumers may have left before waiting for every stage: let each stage's last batch
      // land before the shared memory goes away (the phases of one stage complete in order,
      // and the producer never runs more than one phase ahead of a stage's consumers).
      for (int s = 0; s < NST; ++s)
        if (bulk_issued[s] > 0) s1::mbar_wait(&full[s], (uint32_t)(uses[s] - 1) & 1u);
    }
  } else if (warp == 1) {
    // ============================================================ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_u8s8_s32(kTileTc, L::N);
      int cur = -1;
      int committed = 0;  // MMA batches committed to mmad (for the drain)
      for (int i = 0; i < ntl; ++i) {
        const int b = i & 1;
        const int j = (int)((g0 + i) / Tu) - u_first;
        if (j != cur) {
          cur = j;
          if (!wait_phase(&fbfull[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag)) {
            failed = true;
            break;
          }
        }
        if (!wait_phase(&afull[b], (uint32_t)(i >> 1) & 1u, abort_flag)) {
          failed = true;
          break;
        }
        if (i >= 2 && !wait_phase(&dempty[b], (uint32_t)((i >> 1) - 1) & 1u, abort_flag)) {
          failed = true;
          break;
        }
        s1::fence_after_sync();
        const uint32_t bbase = smem_addr(sm + L::SM_B + (j & 1) * L::BBUF_AL);
#pragma unroll
        for (int ks = 0; ks < L::EW; ++ks)
          umma_i8_ts(tmem + L::TM_D + b * L::N, tmem + b * L::TA + 8 * ks, s1::sw128_desc(bbase, 16 * ks, L::N),
                     idesc, ks > 0 ? 1u : 0u);
        s1::umma_commit(&mmad[b]);
        ++committed;
        if (last_of_unit(i)) s1::umma_commit(&fbempty[j & 1]);
      }
      if (failed) raise_abort(abort_flag);
      // the last committed MMAs complete before the tensor memory is freed
      if (committed > 0) {
        const int il = committed - 1;
        s1::mbar_wait(&mmad[il & 1], (uint32_t)(il >> 1) & 1u);
      }
    }
  } else if (warp == 2) {
    // ============================================================ query operands
    if (lane == 0) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int issued = 0;
      for (int j = 0; j < n_units; ++j) {
        if (j >= 2 && !wait_phase(&fbempty[j & 1], (uint32_t)((j >> 1) - 1) & 1u, abort_flag)) {
          failed = true;
          break;
        }
        s1::fence_async_smem();  // generic reads of the buffer's constants come first
        s1::mbar_expect_tx(&fbfull[j & 1], (uint32_t)L::BBUF);
        s1::bulk_g2s(sm + L::SM_B + (j & 1) * L::BBUF_AL, a.bop + (size_t)(u_first + j) * L::BBUF, L::BBUF,
                     &fbfull[j & 1]);
        ++issued;
      }
      if (failed) raise_abort(abort_flag);
      // drain: the copies issued land before the shared memory goes away
      for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j)
        s1::mbar_wait(&fbfull[j & 1], (uint32_t)(j >> 1) & 1u);
    }
  } else if (warp >= 4 && warp < 8) {
    // ============================================================ key bits -> tensor memory
    const int kw = warp - 4, R = 32 * kw + lane;
    const uint32_t lane_base = (uint32_t)(32 * kw) << 16;
    for (int i = 0; i < ntl; ++i) {
      const int s = i % NST, b = i & 1;
      if (!wait_phase(&full[s], (uint32_t)(i / NST) & 1u, abort_flag)) {
        failed = true;
        break;
      }
      if (i >= 2 && !wait_phase(&mmad[b], (uint32_t)((i >> 1) - 1) & 1u, abort_flag)) {
        failed = true;
        break;
      }
      s1::fence_after_sync();
      const unsigned char* st = ring + s * L::STAGE;
      uint32_t w[L::EW];
      {
        const uint4* kc = reinterpret_cast<const uint4*>(st + L::OFF_KC + R * L::KCB);
#pragma unroll
        for (int c = 0; c < LMB; ++c) {
          const uint4 v = kc[c];
          w[4 * c] = v.x;
          w[4 * c + 1] = v.y;
          w[4 * c + 2] = v.z;
          w[4 * c + 3] = v.w;
        }
        if constexpr (QJL) {
          const uint4 v = *reinterpret_cast<const uint4*>(st + L::OFF_KS + R * L::SB);
          w[L::KSC] = v.x;
          w[L::KSC + 1] = v.y;
          w[L::KSC + 2] = v.z;
          w[L::KSC + 3] = v.w;
        }
      }
      __syncwarp();
      if (lane == 0) s1::mbar_arrive(&empty[s]);  // the stage's key bytes are in registers
      if constexpr (LMB == 3) {
#pragma unroll
        for (int gq = 0; gq < 4; ++gq) w[L::CW + gq] = parity_word(w[3 * gq], w[3 * gq + 1], w[3 * gq + 2]);
      }
      const uint32_t abase = tmem + b * L::TA + lane_base;
#pragma unroll
      for (int e = 0; e < L::EW; ++e) {
        const uint32_t x = w[e], x4 = x >> 4;
        uint32_t m[8];
        m[0] = bitmask_el<0>(x, x4);
        m[1] = bitmask_el<1>(x, x4);
        m[2] = bitmask_el<2>(x, x4);
        m[3] = bitmask_el<3>(x, x4);
        m[4] = bitmask_el<4>(x, x4);
        m[5] = bitmask_el<5>(x, x4);
        m[6] = bitmask_el<6>(x, x4);
        m[7] = bitmask_el<7>(x, x4);
        s1::tmem_st8(abase + 8 * e, m);
      }
      s1::tmem_st_wait();
      s1::fence_before_sync();
      __syncwarp();
      if (lane == 0) s1::mbar_arrive(&afull[b]);
    }
    if (failed && lane == 0) raise_abort(abort_flag);
  } else if (warp >= 8 && warp < 12) {
    // ============================================================ scores, online softmax
    const int sw = warp - 8, R = 32 * sw + lane;
    const uint32_t lane_base = (uint32_t)(32 * sw) << 16;
    float* lred = reinterpret_cast<float*>(sm + L::SM_LR);   // [HG][128]
    float* tmx = reinterpret_cast<float*>(sm + L::SM_TMX);   // [4][HG]
    float Mref[HG], lsum[HG];
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      Mref[h] = -INFINITY;
      lsum[h] = 0.f;
    }
    int cur = -1, qrow0 = 0;
    // End of local unit j: the CTA's (m, l) of each query head, l summed over the 128
    // threads in a fixed order; then the unit's query operand is released.
    auto finish_sm = [&](int j) {
      const int u = u_first + j;
      const int seg = (int)(kcta - owner_tc((int64_t)u * Tu, P, Tt));
      float* part = a.ws_part + ((size_t)u * a.s_max + seg) * G * RS;
#pragma unroll
      for (int h = 0; h < HG; ++h) lred[h * kTileTc + R] = lsum[h];
      named_sync(kBarSm, 128);
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        if (R == h && h < G) {
          float l = 0.f;
          for (int t = 0; t < kTileTc; ++t) l += lred[h * kTileTc + t];
          part[h * RS + 0] = failed ? -INFINITY : Mref[h];
          part[h * RS + 1] = failed ? 0.f : l;
        }
      }
      named_sync(kBarSm, 128);
      __syncwarp();
      if (lane == 0) s1::mbar_arrive(&fbempty[j & 1]);
    };
    for (int i = 0; i < ntl; ++i) {
      const int s = i % NST, b = i & 1, pb = i & 1;
      int u, nt;
      int64_t tok0;
      tile_info(i, u, tok0, nt);
      const int j = u - u_first;
      if (j != cur) {
        cur = j;
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          Mref[h] = -INFINITY;
          lsum[h] = 0.f;
        }
        const int bq = u / a.hkv, kvh = u - bq * a.hkv;
        qrow0 = bq * a.hq + kvh * G;
        if (!failed && !wait_phase(&fbfull[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag)) failed = true;
      }
      if (!failed && !wait_phase(&mmad[b], (uint32_t)(i >> 1) & 1u, abort_flag)) failed = true;
      if (!failed && !wait_phase(&full[s], (uint32_t)(i / NST) & 1u, abort_flag)) failed = true;
      if (!failed && i >= 2 && !wait_phase(&pempty[pb], (uint32_t)((i >> 1) - 1) & 1u, abort_flag)) failed = true;
      // the four softmax warps share named barriers: they leave together or not at all
      if (named_sync_or(kBarSm, 128, failed)) {
        failed = true;
        break;
      }
      s1::fence_after_sync();
      uint32_t dsum[L::N];
#pragma unroll
      for (int c = 0; c < L::N; c += 16) tmem_ld16(tmem + L::TM_D + b * L::N + c + lane_base, dsum + c);
      s1::tmem_ld_wait();
      s1::fence_before_sync();
      __syncwarp();
      if (lane == 0) s1::mbar_arrive(&dempty[b]);
      const unsigned char* st = ring + s * L::STAGE;
      const bool valid = R < nt;
      const uint32_t ngw = *reinterpret_cast<const uint32_t*>(st + L::OFF_KN + 4 * R);
      const uint4 vpar = *reinterpret_cast<const uint4*>(st + L::OFF_VP + 16 * R);
      __syncwarp();
      if (lane == 0) s1::mbar_arrive(&empty[s]);
      const float2 ng = __half22float2(h2of(ngw));  // (n, gamma)
      const float4* kc = reinterpret_cast<const float4*>(sm + L::SM_B + (j & 1) * L::BBUF_AL + L::BOP);
      float lg[HG];
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const float4 k = kc[h];
        // digit sums recombined: (s0 + 2^8 s1) + 2^16 (s2 + 2^8 s3), each part an exact int
        const int c0 = kDigits * h;
        const float code = (float)((int)dsum[c0] + ((int)dsum[c0 + 1] << 8)) +
                           65536.f * (float)((int)dsum[c0 + 2] + ((int)dsum[c0 + 3] << 8));
        float sg = 0.f;
        if constexpr (QJL) {
          const int c1 = L::NC + kDigits * h;
          sg = (float)((int)dsum[c1] + ((int)dsum[c1 + 1] << 8)) +
               65536.f * (float)((int)dsum[c1 + 2] + ((int)dsum[c1 + 3] << 8));
        }
        const float l = ng.x * fmaf(ng.y, fmaf(k.z, sg, -k.w), fmaf(k.y, code, k.x));
        lg[h] = (valid && h < G) ? l : -INFINITY;
      }
      if (a.scores && valid) {
#pragma unroll
        for (int h = 0; h < HG; ++h)
          if (h < G) a.scores[(size_t)(qrow0 + h) * a.max_len + tok0 + R] = lg[h] * kLn2;
      }
      // Lazy rescale: the reference maxima move only when a logit exceeds them by more than
      // the slack; all 128 softmax threads take the same decision.
      bool need = false;
#pragma unroll
      for (int h = 0; h < HG; ++h) need |= lg[h] > Mref[h] + kSlackTc;
      need = named_sync_or(kBarSm, 128, need);
      float corr[HG];
#pragma unroll
      for (int h = 0; h < HG; ++h) corr[h] = 1.f;
      if (need) {
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          const float m = warp_max(lg[h]);
          if (lane == 0) tmx[sw * HG + h] = m;
        }
        named_sync(kBarSm, 128);
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          const float tm = fmaxf(fmaxf(tmx[h], tmx[HG + h]), fmaxf(tmx[2 * HG + h], tmx[3 * HG + h]));
          const float Mn = fmaxf(Mref[h], tm);
          if (Mn > Mref[h]) {
            corr[h] = Mref[h] == -INFINITY ? 0.f : ex2f(Mref[h] - Mn);
            lsum[h] *= corr[h];
            Mref[h] = Mn;
          }
        }
      }
      // p of this token per head, split in f16 hi + lo
      uint32_t own[HG];  // (p_hi, p_lo) of this token
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const float p = lg[h] == -INFINITY ? 0.f : ex2f(lg[h] - Mref[h]);
        lsum[h] += p;
        const __half hi = __float2half_rn(p);
        const __half lo = __float2half_rn(p - __half2float(hi));
        own[h] = (uint32_t)__half_as_ushort(hi) | ((uint32_t)__half_as_ushort(lo) << 16);
      }
      // value weights of the token pair (t even, t odd): the even thread writes groups 0-1,
      // the odd thread groups 2-3 (and the minima's p of the first / second half of the heads)
      const bool odd = (lane & 1) != 0;
      uint32_t par[HG];
#pragma unroll
      for (int h = 0; h < HG; ++h) par[h] = __shfl_xor_sync(kFull, own[h], 1);
      const uint32_t sc[4] = {valid ? vpar.x : 0u, valid ? vpar.y : 0u, valid ? vpar.z : 0u, valid ? vpar.w : 0u};
      // send the partner the (scale, min) words of its two groups, receive ours
      const uint32_t send0 = odd ? sc[0] : sc[2], send1 = odd ? sc[1] : sc[3];
      const uint32_t got0 = __shfl_xor_sync(kFull, send0, 1), got1 = __shfl_xor_sync(kFull, send1, 1);
      uint32_t* pw = reinterpret_cast<uint32_t*>(sm + L::SM_P + pb * L::PBUF);
      const int pair = R >> 1;
#pragma unroll
      for (int gg = 0; gg < 2; ++gg) {
        const int g = odd ? 2 + gg : gg;
        const uint32_t mine = odd ? sc[2 + gg] : sc[gg];
        const uint32_t other = gg == 0 ? got0 : got1;
        // scales (low halves) of the even and the odd token
        const uint32_t s2w = odd ? __byte_perm(other, mine, 0x5410) : __byte_perm(mine, other, 0x5410);
        const __half2 s2 = h2of(s2w);
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          const uint32_t ev = odd ? par[h] : own[h], ov = odd ? own[h] : par[h];
          const __half2 ph = h2of(__byte_perm(ev, ov, 0x5410));  // p_hi of (even, odd)
          const __half2 pl = h2of(__byte_perm(ev, ov, 0x7632));  // p_lo of (even, odd)
          const __half2 hi = __hmul2(ph, s2);
          const __half2 err = __hfma2(ph, s2, __hneg2(hi));
          const __half2 lo = __hfma2(pl, s2, err);
          pw[prow(g, h, 0, HG) + pair] = hbits(hi);
          pw[prow(g, h, 1, HG) + pair] = hbits(lo);
        }
      }
      uint32_t* pmw = pw + L::PPW;
#pragma unroll
      for (int hh = 0; hh < HG / 2; ++hh) {
        const int h = odd ? HG / 2 + hh : hh;
        const uint32_t ev = odd ? par[h] : own[h], ov = odd ? own[h] : par[h];
        pmw[(h * 2 + 0) * kPairStride + pair] = __byte_perm(ev, ov, 0x5410);
        pmw[(h * 2 + 1) * kPairStride + pair] = __byte_perm(ev, ov, 0x7632);
      }
      if (R == 0) {
        float* hdr = reinterpret_cast<float*>(pw + L::PPW + L::PMW);
        hdr[0] = need ? 1.f : 0.f;
#pragma unroll
        for (int h = 0; h < HG; ++h) hdr[1 + h] = corr[h];
      }
      __syncwarp();
      if (lane == 0) s1::mbar_arrive(&pfull[pb]);
      if (last_of_unit(i)) finish_sm(j);
    }
    if (failed) {
      if (lane == 0) raise_abort(abort_flag);
    }
  } else if (warp >= 12) {
    // ============================================================ values
    const int vw = warp - 12;
    const int r = lane >> 2, c = lane & 3;
    const int part = r & 1, hsel = r >> 1;
    float* vred = reinterpret_cast<float*>(sm + L::SM_VR);  // [4][HG][d]
    float dmin[NB][4];
    float dv[4][2][NB][4];
    auto reset = [&]() {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
        for (int e = 0; e < 4; ++e) dmin[nb][e] = 0.f;
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int e = 0; e < 4; ++e) dv[g][hf][nb][e] = 0.f;
      }
    };
    reset();
    int cur = -1;
    // End of local unit j: the four value warps' sums, added in warp order, are the CTA's
    // acc of each head (all warps share the softmax role's reference maxima).
    auto finish_v = [&](int j) {
      const int u = u_first + j;
      const int seg = (int)(kcta - owner_tc((int64_t)u * Tu, P, Tt));
      float* partp = a.ws_part + ((size_t)u * a.s_max + seg) * G * RS;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const float own = dmin[nb][0] + dmin[nb][1];
        float mt[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) mt[g] = __shfl_sync(kFull, own, 4 * g + c);
        float* red = vred + (vw * HG + c + 4 * nb) * kD;
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const float* d = dv[g][hf][nb];
            int j0;
            float v0, v1;
            if (VB == 2) {
              j0 = 4 * (8 * g + r) + 2 * hf;
              v0 = (d[0] + d[1]) * ldexpf(1.f, 24 - 4 * hf) + mt[g];
              v1 = (d[2] + d[3]) * ldexpf(1.f, 22 - 4 * hf) + mt[g];
            } else {
              j0 = 2 * (16 * g + 8 * hf + r);
              v0 = (d[0] + d[1]) * 16777216.f + mt[g];
              v1 = (d[2] + d[3]) * 1048576.f + mt[g];
            }
            red[j0] = failed ? 0.f : v0;
            red[j0 + 1] = failed ? 0.f : v1;
          }
      }
      named_sync(kBarV, 128);
      const int t = tid - 12 * 32;  // 0..127: one coordinate per thread
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        if (h < G) {
          const float acc = ((vred[(0 * HG + h) * kD + t] + vred[(1 * HG + h) * kD + t]) +
                             vred[(2 * HG + h) * kD + t]) + vred[(3 * HG + h) * kD + t];
          partp[h * RS + 4 + t] = acc;
        }
      }
      named_sync(kBarV, 128);
      reset();
    };
    for (int i = 0; i < ntl; ++i) {
      const int s = i % NST, pb = i & 1;
      int u, nt;
      int64_t tok0;
      tile_info(i, u, tok0, nt);
      const int j = u - u_first;
      if (j != cur) cur = j;
      if (!failed && !wait_phase(&pfull[pb], (uint32_t)(i >> 1) & 1u, abort_flag)) failed = true;
      if (!failed && !wait_phase(&full[s], (uint32_t)(i / NST) & 1u, abort_flag)) failed = true;
      // the four value warps share named barriers: they leave together or not at all
      if (named_sync_or(kBarV, 128, failed)) {
        failed = true;
        break;
      }
      const uint32_t* pw = reinterpret_cast<const uint32_t*>(sm + L::SM_P + pb * L::PBUF);
      const uint32_t* pmw = pw + L::PPW;
      const float* hdr = reinterpret_cast<const float*>(pw + L::PPW + L::PMW);
      if (hdr[0] != 0.f) {
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          const float cf = hdr[1 + c + 4 * nb];
#pragma unroll
          for (int e = 0; e < 4; ++e) dmin[nb][e] *= cf;
#pragma unroll
          for (int g = 0; g < 4; ++g)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
              for (int e = 0; e < 4; ++e) dv[g][hf][nb][e] *= cf;
        }
      }
      const unsigned char* st = ring + s * L::STAGE;
      const uint32_t* vc = reinterpret_cast<const uint32_t*>(st + L::OFF_VC);
      const uint32_t* vpw = reinterpret_cast<const uint32_t*>(st + L::OFF_VP);
#pragma unroll
      for (int mb = 0; mb < 2; ++mb) {
        const int tb = 32 * vw + 16 * mb;  // first token of the block within the tile
        if (tb >= nt) break;              // warp-uniform
        const int nv = nt - tb;
        // k = token - tb: lane (r, c) holds tokens tb + 2c, 2c + 1 (a0/a1) and tb + 2c + 8, 2c + 9 (a2/a3)
        const int tA0 = tb + 2 * c, tA1 = tA0 + 1, tB0 = tA0 + 8, tB1 = tA0 + 9;
        const int pA = (tb >> 1) + c, pB = pA + 4;  // token pairs of b0 and b1
        // ---- minima: rows g < 4 = group minima of the k tokens; B = p (hi / lo)
        {
          uint32_t mA0 = 0u, mA1 = 0u, mB0 = 0u, mB1 = 0u;
          if (r < 4) {
            if (2 * c < nv) mA0 = vpw[tA0 * 4 + r];
            if (2 * c + 1 < nv) mA1 = vpw[tA1 * 4 + r];
            if (2 * c + 8 < nv) mB0 = vpw[tB0 * 4 + r];
            if (2 * c + 9 < nv) mB1 = vpw[tB1 * 4 + r];
          }
          uint4 am;
          am.x = __byte_perm(mA0, mA1, 0x7632);
          am.y = 0u;
          am.z = __byte_perm(mB0, mB1, 0x7632);
          am.w = 0u;
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const int row = ((4 * nb + hsel) * 2 + part) * kPairStride;
            mma16816_tc(dmin[nb], am, pmw[row + pA], pmw[row + pB]);
          }
        }
        const uint32_t sel = (uint32_t)(r & 3) | ((uint32_t)(4 + (r & 3)) << 8);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t bA[NB], bB[NB];
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const int row = prow(g, 4 * nb + hsel, part, HG);
            bA[nb] = pw[row + pA];
            bB[nb] = pw[row + pB];
          }
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            uint32_t xA, xB;
            uint4 av;
            constexpr int WPT = L::VCB / 4;
            if (VB == 2) {
              const int wv = 2 * g + (r >> 2);
              if (hf == 0) {
                xA = __byte_perm(vc[tA0 * WPT + wv], vc[tA1 * WPT + wv], sel);
                xB = __byte_perm(vc[tB0 * WPT + wv], vc[tB1 * WPT + wv], sel);
              }
              const uint32_t m0 = 0x00030003u << (4 * hf), m1 = 0x00030003u << (4 * hf + 2);
              av = make_uint4(xA & m0, xA & m1, xB & m0, xB & m1);
            } else {
              const int wv = 4 * g + 2 * hf + (r >> 2);
              xA = __byte_perm(vc[tA0 * WPT + wv], vc[tA1 * WPT + wv], sel);
              xB = __byte_perm(vc[tB0 * WPT + wv], vc[tB1 * WPT + wv], sel);
              av = make_uint4(xA & 0x000F000Fu, xA & 0x00F000F0u, xB & 0x000F000Fu, xB & 0x00F000F0u);
            }
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) mma16816_tc(dv[g][hf][nb], av, bA[nb], bB[nb]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        s1::mbar_arrive(&pempty[pb]);
        s1::mbar_arrive(&empty[s]);
      }
      if (last_of_unit(i)) finish_v(j);
    }
    if (failed && lane == 0) raise_abort(abort_flag);
  }

  // ---------------------------------------------------------------- end
  __syncthreads();
  if (*abort_flag) {
    if (tid == 0) atomicOr(a.err, 1u);
  }
  s1::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    s1::fence_after_sync();
    s1::tmem_dealloc(tmem, 512);
  }
}

template <int LMB, bool QJL, int VB, int NB>
cudaError_t launch_tc_t(const tq_ctx* ctx, const PrepTcArgs& pa, int units, const TcArgs& a, int n_ctas,
                        cudaStream_t s) {
  using L = TcLayout<LMB, QJL, VB, NB>;
  static cudaError_t cfg_err = [] {
    cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<LMB, QJL, VB, NB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(prep_tc_kernel<LMB, QJL, VB, NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(sizeof(float) * kD * kM));
    return e;
  }();
  if (cfg_err != cudaSuccess) return cfg_err;
  prep_tc_kernel<LMB, QJL, VB, NB><<<units, kPrepTcThreads, sizeof(float) * kD * kM, s>>>(pa);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)n_ctas);
  cfg.blockDim = dim3(kThreadsTc);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (ctx->prof_start) cudaEventRecord(ctx->prof_start, s);
  e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<LMB, QJL, VB, NB>, a);
  if (ctx->prof_stop) cudaEventRecord(ctx->prof_stop, s);
  return e;
}

template <int LMB, bool QJL, int VB>
cudaError_t launch_tc_nb(const tq_ctx* ctx, const PrepTcArgs& pa, int units, const TcArgs& a, int n_ctas, int nb,
                         cudaStream_t s) {
  return nb == 1 ? launch_tc_t<LMB, QJL, VB, 1>(ctx, pa, units, a, n_ctas, s)
                 : launch_tc_t<LMB, QJL, VB, 2>(ctx, pa, units, a, n_ctas, s);
}

template <int LMB, bool QJL>
cudaError_t launch_tc_vb(const tq_ctx* ctx, const PrepTcArgs& pa, int units, const TcArgs& a, int n_ctas, int nb,
                         int vb, cudaStream_t s) {
  return vb == 2 ? launch_tc_nb<LMB, QJL, 2>(ctx, pa, units, a, n_ctas, nb, s)
                 : launch_tc_nb<LMB, QJL, 4>(ctx, pa, units, a, n_ctas, nb, s);
}

template <int LMB, bool QJL>
size_t tc_bbuf_t(int nb, int vb) {
  if (vb == 2) return nb == 1 ? TcLayout<LMB, QJL, 2, 1>::BBUF : TcLayout<LMB, QJL, 2, 2>::BBUF;
  return nb == 1 ? TcLayout<LMB, QJL, 4, 1>::BBUF : TcLayout<LMB, QJL, 4, 2>::BBUF;
}

// Bit expansion of a symmetric codebook: c[idx] = kappa + sum_p beta_p bit_p (bit 3 = the
// parity of the three code bits at 3 bits). False if the codebook is not of that form.
bool codebook_bits(const Codebook& cb, int lmb, float& kappa, float beta[4]) {
  const float* c = cb.c;
  for (int p = 0; p < 4; ++p) beta[p] = 0.f;
  kappa = c[0];
  const int L = 1 << lmb;
  float scale = 0.f;
  for (int k = 0; k < L; ++k) scale = fmaxf(scale, fabsf(c[k]));
  for (int k = 0; k < L; ++k)
    if (fabsf(c[k] + c[L - 1 - k]) > 1e-6f * scale) return false;  // symmetric about zero
  if (lmb == 1) {
    beta[0] = c[1] - c[0];
  } else if (lmb == 2) {
    beta[0] = c[1] - c[0];
    beta[1] = c[2] - c[0];
  } else if (lmb == 3) {
    const double c0 = c[0], c1 = c[1], c2 = c[2], c4 = c[4], c7 = c[7];
    const double b3 = 0.5 * (c1 + c2 + c4 - 2.0 * c0 - c7);
    beta[3] = (float)b3;
    beta[0] = (float)(c1 - c0 - b3);
    beta[1] = (float)(c2 - c0 - b3);
    beta[2] = (float)(c4 - c0 - b3);
  } else {
    return false;
  }
  // every level is reproduced by the expansion
  for (int k = 0; k < L; ++k) {
    const int b0 = k & 1, b1 = (k >> 1) & 1, b2 = (k >> 2) & 1;
    const double v = (double)kappa + beta[0] * b0 + beta[1] * b1 + beta[2] * b2 + beta[3] * ((b0 ^ b1 ^ b2) & 1);
    if (fabs(v - (double)c[k]) > 1e-6 * scale) return false;
  }
  return true;
}

}  // namespace

bool tc_decode_supported(const tq_ctx* ctx, int G) {
  const Shape& sh = ctx->shape;
  if (sh.d != kD || !(sh.m == kM || sh.m == 0) || G < 1 || G > 8) return false;
  if (sh.lm_bits < 1 || sh.lm_bits > 3) return false;
  if (!(sh.v_bits == 2 || sh.v_bits == 4)) return false;
  float kappa, beta[4];
  return codebook_bits(ctx->cb, sh.lm_bits, kappa, beta);
}

size_t tc_operand_bytes(const tq_ctx* ctx, int G) {
  const int nb = G <= 4 ? 1 : 2, vb = ctx->shape.v_bits;
  const bool qjl = ctx->shape.m > 0;
  switch (ctx->shape.lm_bits) {
    case 1: return qjl ? tc_bbuf_t<1, true>(nb, vb) : tc_bbuf_t<1, false>(nb, vb);
    case 2: return qjl ? tc_bbuf_t<2, true>(nb, vb) : tc_bbuf_t<2, false>(nb, vb);
    default: return qjl ? tc_bbuf_t<3, true>(nb, vb) : tc_bbuf_t<3, false>(nb, vb);
  }
}

cudaError_t launch_decode_tc(const tq_ctx* ctx, const DecodePlan& plan, const void* q, int q_dtype, int batch,
                             int hq, int hkv, const int32_t* seq_lens, int64_t max_len, const Paging& pg,
                             const uint8_t* k_codes, const uint8_t* k_signs, const uint16_t* k_norms,
                             const uint8_t* v_codes, const uint16_t* v_params, float scale, float* scores,
                             float* out, float* lse, void* workspace, cudaStream_t stream) {
  char* ws = static_cast<char*>(workspace);
  uint8_t* bop = reinterpret_cast<uint8_t*>(ws + plan.off_frag);
  float* part = reinterpret_cast<float*>(ws + plan.off_part);
  const int G = hq / hkv, lmb = ctx->shape.lm_bits, vb = ctx->shape.v_bits, nb = G <= 4 ? 1 : 2;
  const bool qjl = ctx->shape.m > 0;
  if (plan.n_ctas < 1 || plan.tiles_per_unit < 1) return cudaErrorInvalidValue;
  PrepTcArgs pa;
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
  pa.bop = bop;
  TcArgs a;
  a.bop = bop;
  a.k_codes = k_codes;
  a.k_signs = k_signs;
  a.k_norms = k_norms;
  a.v_codes = v_codes;
  a.v_params = v_params;
  a.seq_lens = seq_lens;
  a.max_len = max_len;
  a.pg = pg;
  a.hq = hq;
  a.hkv = hkv;
  a.G = G;
  a.tiles_per_unit = plan.tiles_per_unit;
  a.total_tiles = plan.total_tiles;
  a.s_max = plan.s_max;
  a.scores = scores;
  a.ws_part = part;
  a.use_tma = (max_len % 4 == 0) ? 1 : 0;
  a.err = ctx->d_err;
  const int units = batch * hkv;
  cudaError_t e;
  switch (lmb) {
    case 1:
      e = qjl ? launch_tc_vb<1, true>(ctx, pa, units, a, plan.n_ctas, nb, vb, stream)
              : launch_tc_vb<1, false>(ctx, pa, units, a, plan.n_ctas, nb, vb, stream);
      break;
    case 2:
      e = qjl ? launch_tc_vb<2, true>(ctx, pa, units, a, plan.n_ctas, nb, vb, stream)
              : launch_tc_vb<2, false>(ctx, pa, units, a, plan.n_ctas, nb, vb, stream);
      break;
    default:
      e = qjl ? launch_tc_vb<3, true>(ctx, pa, units, a, plan.n_ctas, nb, vb, stream)
              : launch_tc_vb<3, false>(ctx, pa, units, a, plan.n_ctas, nb, vb, stream);
  }
  if (e != cudaSuccess) return e;
  return launch_combine_partials(part, out, lse, batch, hq, hkv, G, plan.s_max, plan.tiles_per_unit,
                                 plan.total_tiles, plan.n_ctas, stream);
}

}  // namespace tq
