// Decode attention with the key scores on the 5th-generation tensor cores (d = 128; keys of
// 1- to 3-bit Lloyd-Max codes from a codebook symmetric about zero, with the 128-bit QJL
// sketch or without it; 2- or 4-bit values; up to 8 query heads per KV head).
//
// Same mathematics as decode_kernel (the skill card "turboquant-
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
// Values. out = sum_t p_t (min + scale * code) on warp-level tensor-core MMAs (mma.sync
// m16n8k16, f16 operands built in registers, fp32 sums in registers): rows = 16 value
// coordinates, K = 16 tokens, columns = 4 query heads x (high, low part of p * scale). A 2- or
// 4-bit code masked into the low mantissa bits of an f16 is an exact subnormal, code *
// 2^(position - 24): a byte permute pairs the same code byte of two tokens and one AND makes
// two elements; the power of two depends only on the row and is undone at the end. p * scale
// is an exact TwoProduct in half2 (high part rounded, low part = the rounding error plus
// p_low * scale). The group minima, sum_t p_t min_t, go through one more MMA (rows = value
// groups, columns = p's high and low parts). (Value
// operands staged in shared memory for tcgen05 cost 512 bytes of shared-memory traffic per
// token; in registers they cost none.)
// Online softmax in base 2 with one reference maximum per query head for a group of warps,
// moved only when a logit exceeds it by more than 2 (p < 4, so p * scale stays finite in f16
// for value scales below 16376); when it moves, the sums so far are rescaled in place.
//
// Work split (one CTA per SM; the units' tiles laid end to end and split evenly over the
// CTAs, so a CTA's range may start and end inside a unit and span several):
//   one producer warp streams the packed records into a ring of two-tile stages (one bulk
//   copy per array and stage; a ragged or unaligned tile is copied by the warp) and loads
//   each unit's query operand (digits + logit constants) when the unit's first tile goes;
//   groups of four compute warps take the tiles in turn, one token per thread: a group waits
//   for tile k's digit sums, reads them and forms the logits, writes tile k + 1's key
//   elements into its tensor-memory A operand, and only then runs tile k's online softmax
//   and value MMAs, so that tile k + 1's score MMAs overlap them;
//   one MMA warp per group issues the group's score MMAs as soon as a tile's key elements
//   are written (a tcgen05.mma holds its issuing warp for tens of nanoseconds; no compute
//   warp waits on that). At the end of a unit each group writes one partial (m, l, acc) per
//   query head; combine_partials merges them in a fixed order.
// Every wait is bounded: on a timeout the CTA raises an abort flag that every warp polls,
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
constexpr int kPrepTcThreads = 256;
constexpr float kSlackTc = 2.f;
constexpr uint32_t kWaitPolls = 1u << 24;
// Suspend-time hint of one mbarrier poll in ns: a waiting warp sleeps until the phase
// completes (or this long) instead of spinning, and leaves the issue slots to the others.
constexpr uint32_t kTryWaitNs = 100000;
constexpr unsigned long long kWaitNs = 2000000000ull;
// |Q| <= 2^30 keeps the top one of four balanced 8-bit digits in [-64, 64]
constexpr float kQmax = 1073741824.f;
constexpr int kDigits = 4;


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
  static constexpr int TA = 8 * EW;                    // tensor-memory columns: key elements
  static constexpr int TG = TA + N;                    // per group: key elements, digit sums
  // Groups of four compute warps, one tile each: as many as tensor memory holds, at most 3 (at
  // most 2 with two head blocks, whose value sums take twice the registers).
  static constexpr int NG_MAX = NB == 1 ? 3 : 2;
  static constexpr int NG = 512 / TG >= NG_MAX ? NG_MAX : 512 / TG;
  static_assert(NG >= 2, "tensor memory for two groups");
  // A stage holds two tiles (256 tokens): each array of the pair arrives with one bulk copy,
  // [kc 256 x KCB][ks 256 x SB][kn 256 x 4][vc 256 x VCB][vp 256 x PB]; tile k of the pair sits
  // 128 k records into each region. (Copies of 128 records streamed at under 60% of the HBM
  // bandwidth; one thread issues every copy, and fewer, larger copies keep up with HBM.)
  static constexpr int KCB = LMB * 16, SB = QJL ? 16 : 0, VCB = VB * 16, PB = 16;
  static constexpr int REC = KCB + SB + 4 + VCB + PB;
  static constexpr int STAGE = 2 * kTileTc * REC;
  static constexpr int OFF_KC = 0, OFF_KS = 2 * kTileTc * KCB, OFF_KN = OFF_KS + 2 * kTileTc * SB;
  static constexpr int OFF_VC = OFF_KN + 2 * kTileTc * 4, OFF_VP = OFF_VC + 2 * kTileTc * VCB;
  static constexpr int BOP = N * KB;                   // digits, K-major, 128-byte swizzle
  static constexpr int BBUF = BOP + HG * 16;           // + logit constants (float4 per head)
  static constexpr int BBUF_AL = (BBUF + 1023) / 1024 * 1024;
  static constexpr int NBUF = 2;                       // query-operand buffers (next unit's loads)
  static constexpr int NCW = 4 * NG;                   // compute warps
  static constexpr int THREADS = 32 * (NCW + 1 + NG);  // + the producer warp + one MMA warp per group
  // Per compute warp: the probabilities of its 32 tokens as f16 high and low parts, [2][HG][32],
  // read back in the B-fragment layout of the value MMAs.
  static constexpr int PT = 2 * HG * 32 * 2;
  static constexpr int RED_F = 5 * HG;                 // per warp: minima sums [HG][4], sums of p [HG]
  static constexpr int NBAR = 2 * 6 + 3 + 3 + 2;       // full, empty [<= 6]; afull, mmad [<= 3]; fbfull [2]
  static constexpr int SM_B = 0;                                   // [NBUF] query operands
  static constexpr int SM_PT = NBUF * BBUF_AL;                     // [NCW] probability parts
  static constexpr int SM_RED = SM_PT + NCW * PT;                  // [NG][4 warps][128] value sums of a head
  static constexpr int SM_REDF = SM_RED + NG * 4 * kD * 4;         // [NG][4 warps][RED_F]
  static constexpr int SM_RM = SM_REDF + NG * 4 * RED_F * 4;       // [NG][4 warps][8] warp maxima
  static constexpr int SM_BAR = SM_RM + NG * 4 * 8 * 4;
  static constexpr int SM_MISC = SM_BAR + 8 * NBAR;                // TMEM address, abort flag, grp_unit[NG]
  static constexpr int SM_RING = (SM_MISC + 8 + 4 * NG + 127) / 128 * 128;
  static constexpr int FIT = (227 * 1024 - 1024 - SM_RING) / STAGE > 6 ? 6 : (227 * 1024 - 1024 - SM_RING) / STAGE;
  // Group g consumes tiles g, g + NG, ...; tile i sits in stage (i / 2) mod NST. With 2 NST a
  // multiple of NG, the previous use of a group's stage held a tile of the same group, so the
  // phase a group waits for can never be confused with the one two uses back.
  static constexpr int NST = NG == 3 ? FIT / 3 * 3 : FIT;
  static_assert(NST >= 2 && NST <= 6, "stages");
  static constexpr size_t SMEM = (size_t)SM_RING + (size_t)NST * STAGE + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(STAGE % 16 == 0 && BBUF % 16 == 0 && SM_PT % 16 == 0, "alignment");
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
    if constexpr (kTryWaitNs > 0)
      asm volatile(
          "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
          : "=r"(done)
          : "r"(a), "r"(parity), "r"(kTryWaitNs)
          : "memory");
    else
      asm volatile(
          "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
          : "=r"(done)
          : "r"(a), "r"(parity)
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

// Warp-wide store of 32 consecutive 32-bit columns of the warp's 32 lanes.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
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


// Walks a CTA's tiles in order without dividing: the unit, the tile within it, the unit's
// valid length.
struct TileWalk {
  int64_t Tu, max_len;
  const int32_t* seq_lens;
  int hkv;
  int u;
  int64_t tl, len;
  __device__ __forceinline__ int64_t unit_len(int uu) const {
    int64_t l = max_len;
    if (seq_lens) l = min((int64_t)max(seq_lens[uu / hkv], 0), max_len);
    return l;
  }
  __device__ __forceinline__ void start(int64_t g0) {
    u = (int)(g0 / Tu);
    tl = g0 - (int64_t)u * Tu;
    len = unit_len(u);
  }
  __device__ __forceinline__ void next() {
    if (++tl == Tu) {
      tl = 0;
      ++u;
      len = unit_len(u);
    }
  }
  __device__ __forceinline__ int64_t tok0() const { return tl * kTileTc; }
  __device__ __forceinline__ int nt() const {
    return (int)max((int64_t)0, min((int64_t)kTileTc, len - tl * kTileTc));
  }
};

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
  // element word ks. Code columns n = 4 h + digit, sign columns NC + 4 h + digit. One thread
  // per (head, element word, mask): the four weights of the word's bytes are quantized once
  // and their digits stored as one 32-bit word in each of the four digit columns.
  uint8_t* bop = a.bop + (size_t)unit * L::BBUF;
  constexpr int WPR = L::KB / 4;  // 32-bit words per row
  auto put = [&](int n, int kw, uint32_t word) {
    *reinterpret_cast<uint32_t*>(bop + s1::sw128_offset(n, 2 * kw, L::N)) = word;
  };
  for (int it = tid; it < HG * L::EW * 8; it += kPrepTcThreads) {
    const int h = it / (L::EW * 8), ks = (it / 8) % L::EW, q = it % 8;
    const bool code = ks < L::KSC;
    uint32_t dw[kDigits] = {0u, 0u, 0u, 0u};
    if (h < G) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float wgt, e2;
        if (code) {
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
        dw[0] |= ((uint32_t)d0 & 0xffu) << (8 * i);
        dw[1] |= ((uint32_t)d1 & 0xffu) << (8 * i);
        dw[2] |= ((uint32_t)d2 & 0xffu) << (8 * i);
        dw[3] |= ((uint32_t)d3 & 0xffu) << (8 * i);
      }
    }
    const int kw = 8 * ks + q;
    const int n_live = (code ? 0 : L::NC) + kDigits * h;  // this word's four columns
    const int n_dead = (code ? L::NC : 0) + kDigits * h;  // the other kind's columns: zero
#pragma unroll
    for (int dgt = 0; dgt < kDigits; ++dgt) {
      put(n_live + dgt, kw, dw[dgt]);
      if (QJL) put(n_dead + dgt, kw, 0u);
    }
  }
  // padding columns beyond the code and sign columns
  constexpr int NUSED = QJL ? 2 * L::NC : L::NC;
  for (int w = tid; w < (L::N - NUSED) * WPR; w += kPrepTcThreads) put(NUSED + w / WPR, w % WPR, 0u);
}

// ------------------------------------------------------------------ decode kernel

// D (fp32) += A (f16) x B (f16), m16n8k16, A row-major, B column-major (warp-level MMA).
__device__ __forceinline__ void mma16816(float (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t word_of(const uint4& w, int i) {
  return i == 0 ? w.x : i == 1 ? w.y : i == 2 ? w.z : w.w;
}

template <int LMB, bool QJL, int VB, int NB>
__global__ void __launch_bounds__(TcLayout<LMB, QJL, VB, NB>::THREADS, 1)
    decode_tc_kernel(const __grid_constant__ TcArgs a) {
  using L = TcLayout<LMB, QJL, VB, NB>;
  constexpr int HG = L::HG, NST = L::NST, NG = L::NG, NBUF = L::NBUF;
  constexpr int RS = 4 + kD;  // partial row: m, l, pad, pad, acc[d]
  constexpr float kLn2 = 0.6931471805599453f;
  extern __shared__ unsigned char smem_tc_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(((uintptr_t)smem_tc_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::SM_BAR);
  uint64_t* full = bars;           // [NST] stage landed
  uint64_t* empty = bars + 6;      // [NST] both tiles of the stage read (2 x 4 warps)
  uint64_t* afull = bars + 12;     // [NG] the group's key elements of its next tile written (4 warps)
  uint64_t* mmad = bars + 15;      // [NG] the group's score MMAs done (commit)
  uint64_t* fbfull = bars + 18;    // [NBUF] query operand landed
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(sm + L::SM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::SM_MISC + 4);
  volatile int* grp_unit = reinterpret_cast<volatile int*>(sm + L::SM_MISC + 8);  // [NG]
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
      s1::mbar_init(&empty[s], 8);  // two tiles x four warps
    }
    for (int g = 0; g < NG; ++g) {
      s1::mbar_init(&afull[g], 4);  // four warps
      s1::mbar_init(&mmad[g], 1);
      grp_unit[g] = -1;
    }
    for (int b = 0; b < NBUF; ++b) s1::mbar_init(&fbfull[b], 1);
    *abort_flag = 0;
    s1::mbar_init_fence();
  }
  s1::fence_before_sync();
  __syncthreads();
  s1::fence_after_sync();
  const uint32_t tmem = *tmem_s;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  TileWalk walk;
  walk.Tu = Tu;
  walk.max_len = a.max_len;
  walk.seq_lens = a.seq_lens;
  walk.hkv = a.hkv;
  walk.start(g0);

  bool failed = false;
  if (warp == L::NCW) {
    // ============================================================ producer
    int bulk_issued[6] = {};  // bulk batches issued per stage (for the failure drain)
    int uses[6] = {};         // phases started per stage
    int b_issued = 0;         // query operands issued (units in order)
    // The query operand of local unit j is loaded when the unit's first tile is, into buffer
    // j mod NBUF, once every group has moved past the unit that buffer held (its MMAs done,
    // its constants read).
    auto load_operand = [&](int u) -> bool {
      const int j = u - u_first;
      if (j != b_issued) return true;
      bool ok = true;
      if (lane == 0) {
        if (b_issued == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
        if (j >= NBUF) {
          const unsigned long long t0 = s1::global_ns();
          for (uint32_t it = 0;; ++it) {
            int mn = 0x7fffffff;
            for (int g = 0; g < NG; ++g) mn = min(mn, grp_unit[g]);
            if (mn >= j - NBUF + 1) break;
            if (*abort_flag || ((it & 63) == 63 && s1::global_ns() - t0 > kWaitNs)) {
              ok = false;
              break;
            }
            __nanosleep(64);
          }
          asm volatile("fence.acq_rel.cta;" ::: "memory");
        }
        if (ok) {
          s1::fence_async_smem();
          s1::mbar_expect_tx(&fbfull[j % NBUF], (uint32_t)L::BBUF);
          s1::bulk_g2s(sm + L::SM_B + (j % NBUF) * L::BBUF_AL, a.bop + (size_t)(u_first + j) * L::BBUF, L::BBUF,
                       &fbfull[j % NBUF]);
        }
      }
      ok = __shfl_sync(kFull, ok, 0);
      if (ok) ++b_issued;
      return ok;
    };
    const int npairs = (ntl + 1) / 2;
    for (int pi = 0; pi < npairs && !failed; ++pi) {
      const int s = pi % NST;
      if (pi >= NST) {
        bool ok = true;
        if (lane == 0) ok = wait_phase(&empty[s], (uint32_t)((pi / NST) - 1) & 1u, abort_flag);
        if (!__shfl_sync(kFull, ok, 0)) {
          failed = true;
          break;
        }
      }
      // the pair's tiles: k = 0, 1 (the second may be past the CTA's range)
      int tu[2], tn[2];
      int64_t tt[2], tv[2];
      const int ntiles = min(2, ntl - 2 * pi);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        tu[k] = u_first;
        tn[k] = 0;
        tt[k] = 0;
        tv[k] = 0;
        if (k >= ntiles) continue;
        tu[k] = walk.u;
        tn[k] = walk.nt();
        tt[k] = walk.tok0();
        walk.next();
        tv[k] = tn[k] > 0 ? record_row(a.pg, a.max_len, tu[k], tt[k], a.err) : 0;
      }
      unsigned char* st = ring + s * L::STAGE;
      uses[s] += 1;
      const bool bulk0 = a.use_tma && tn[0] == kTileTc;
      const bool bulk1 = ntiles == 2 && a.use_tma && tn[1] == kTileTc;
      const bool one_copy = bulk0 && bulk1 && tv[1] == tv[0] + kTileTc;  // contiguous records
      // ragged or unaligned tiles first: the warp copies their valid records with 4-byte loads
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        if (k >= ntiles || (k == 0 ? bulk0 : bulk1) || tn[k] == 0) continue;
        const int64_t v = tv[k];
        const int nt = tn[k];
        auto copy = [&](int off, const void* src, int bpt) {
          const uint32_t* s32 = reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(src) + v * bpt);
          uint32_t* d32 = reinterpret_cast<uint32_t*>(st + off + k * kTileTc * bpt);
          for (int w = lane; w < nt * bpt / 4; w += 32) d32[w] = s32[w];
        };
        copy(L::OFF_KC, a.k_codes, L::KCB);
        if constexpr (QJL) copy(L::OFF_KS, a.k_signs, L::SB);
        copy(L::OFF_KN, a.k_norms, 4);
        copy(L::OFF_VC, a.v_codes, L::VCB);
        copy(L::OFF_VP, a.v_params, L::PB);
      }
      __syncwarp();
      if (lane == 0) {
        // then the bulk copies, after the arrival that announces their bytes
        const uint32_t tile_bytes = (uint32_t)(L::STAGE / 2);
        s1::fence_async_smem();  // the consumers' generic reads come before the async writes
        s1::mbar_expect_tx(&full[s], (bulk0 ? tile_bytes : 0u) + (bulk1 ? tile_bytes : 0u));
        auto issue = [&](int k, int64_t v, int nrec) {
          const int o = k * kTileTc;
          s1::bulk_g2s(st + L::OFF_KC + o * L::KCB, a.k_codes + v * L::KCB, nrec * L::KCB, &full[s]);
          if constexpr (QJL) s1::bulk_g2s(st + L::OFF_KS + o * L::SB, a.k_signs + v * L::SB, nrec * L::SB, &full[s]);
          s1::bulk_g2s(st + L::OFF_KN + o * 4, reinterpret_cast<const uint8_t*>(a.k_norms) + v * 4, nrec * 4,
                       &full[s]);
          s1::bulk_g2s(st + L::OFF_VC + o * L::VCB, a.v_codes + v * L::VCB, nrec * L::VCB, &full[s]);
          s1::bulk_g2s(st + L::OFF_VP + o * L::PB, reinterpret_cast<const uint8_t*>(a.v_params) + v * L::PB,
                       nrec * L::PB, &full[s]);
        };
        if (one_copy) {
          issue(0, tv[0], 2 * kTileTc);
        } else {
          if (bulk0) issue(0, tv[0], kTileTc);
          if (bulk1) issue(1, tv[1], kTileTc);
        }
        if (bulk0 || bulk1) bulk_issued[s] += 1;
      }
#pragma unroll
      for (int k = 0; k < 2; ++k)
        if (k < ntiles && !failed && !load_operand(tu[k])) failed = true;
    }
    if (failed && lane == 0) raise_abort(abort_flag);
    __syncwarp();
    if (lane == 0) {
      // copies still in flight land before the shared memory goes away (phases of one
      // barrier complete in order; at most one phase per stage runs ahead of its consumers)
      if (*abort_flag)
        for (int s = 0; s < NST; ++s)
          if (bulk_issued[s] > 0) s1::mbar_wait(&full[s], (uint32_t)(uses[s] - 1) & 1u);
      for (int jj = (b_issued > NBUF ? b_issued - NBUF : 0); jj < b_issued; ++jj)
        s1::mbar_wait(&fbfull[jj % NBUF], (uint32_t)(jj / NBUF) & 1u);
    }
  } else if (warp > L::NCW) {
    // ============================================================ MMA warps
    // Warp NCW + 1 + g issues the score MMAs of group g's tiles, in order: once the group's
    // four warps have written a tile's key elements (afull), D = A x B over the tile's element
    // words, committed to mmad. The query operand of each unit is waited for in unit order
    // (every unit's phase, also of units the group has no tile of, so that no phase of a
    // buffer is skipped).
    const int gi = warp - L::NCW - 1;
    const uint32_t tgrp = tmem + gi * L::TG;
    int cur = -1, kt = 0, issued = 0;
    for (int k = 0; k < gi; ++k) walk.next();
    for (int i = gi; i < ntl; i += NG, ++kt) {
      const int j = walk.u - u_first;
      for (int k = 0; k < NG; ++k) walk.next();
      if (lane == 0 && !failed) {
        for (int jj = cur + 1; jj <= j && !failed; ++jj)
          if (!wait_phase(&fbfull[jj % NBUF], (uint32_t)(jj / NBUF) & 1u, abort_flag)) failed = true;
        cur = j;
        if (!failed && !wait_phase(&afull[gi], (uint32_t)kt & 1u, abort_flag)) failed = true;
        if (!failed) {
          s1::fence_after_sync();
          constexpr uint32_t idesc = idesc_u8s8_s32(kTileTc, L::N);
          const uint32_t bbase = smem_addr(sm + L::SM_B + (j % NBUF) * L::BBUF_AL);
          const uint32_t d_tm = tgrp + L::TA;
#pragma unroll
          for (int ks = 0; ks < L::EW; ++ks)
            umma_i8_ts(d_tm, tgrp + 8 * ks, s1::sw128_desc(bbase, 16 * ks, L::N), idesc, ks > 0 ? 1u : 0u);
          s1::umma_commit(&mmad[gi]);
          ++issued;
        }
      }
    }
    if (lane == 0) {
      if (failed) raise_abort(abort_flag);
      // the last commit lands before the tensor memory goes away
      if (issued > 0) s1::mbar_wait(&mmad[gi], (uint32_t)(issued - 1) & 1u);
    }
    __syncwarp();
  } else {
    // ============================================================ compute warps
    // Group gi (warps 4 gi .. 4 gi + 3) takes tiles gi, gi + NG, ...; warp q of the group owns
    // tokens 32 q .. 32 q + 31 of each tile (tensor-memory lanes 32 q ..), one token per thread
    // for the key elements, the logits and the online softmax. Tile k + 1's key elements are
    // written while the MMA warp still works on tile k: the loop waits for tile k's digit sums,
    // reads them, writes tile k + 1's elements (the MMA warp then issues its MMAs), and only
    // then runs tile k's softmax and value sums, so the score MMAs overlap that work.
    // Value sums run on warp-level MMAs (mma.sync m16n8k16, f16 operands from registers,
    // fp32 sums in registers): rows = 16 value coordinates, K = 16 tokens, columns = 4 query
    // heads x (high, low part of p * scale). Lane (r, c) holds rows r and r + 8 of each of the
    // eight row blocks, for head 4 nb + c.
    const int gi = warp >> 2, q = warp & 3;
    const int R = 32 * q + lane;
    const int r = lane >> 2, c = lane & 3;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const uint32_t tgrp = tmem + gi * L::TG;
    const uint32_t tA = tgrp + lane_base, tD = tgrp + L::TA + lane_base;
    const int bar_id = 1 + gi;
    const bool leader = q == 0 && lane == 0;
    float* red = reinterpret_cast<float*>(sm + L::SM_RED) + gi * 4 * kD;             // [4][128]
    float* redf = reinterpret_cast<float*>(sm + L::SM_REDF) + gi * 4 * L::RED_F;      // [4][RED_F]
    float* rm = reinterpret_cast<float*>(sm + L::SM_RM) + gi * 32;                     // [4][8]
    __half* pt = reinterpret_cast<__half*>(sm + L::SM_PT + warp * L::PT);             // [2][HG][32]

    // Per thread: the group's reference maxima, this token's share of the sums of p; per lane
    // the value sums and the sums of p * min (fragment layout: rows g < 4 of the minima MMA are
    // value group g).
    float Mref[HG], lsum[HG];
    float dv[4][2][NB][4];  // [value group][half of the group][n-block][fragment]
    float dmin[NB][4];
    auto reset = [&]() {
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        Mref[h] = -INFINITY;
        lsum[h] = 0.f;
      }
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) dmin[nb][e] = 0.f;
#pragma unroll
      for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int e = 0; e < 4; ++e) dv[g][hf][nb][e] = 0.f;
    };
    auto part_ptr = [&](int j) -> float* {
      const int u = u_first + j;
      const int seg = (int)(kcta - owner_tc((int64_t)u * Tu, P, Tt));
      return a.ws_part + (((size_t)u * a.s_max + seg) * NG + gi) * G * RS;
    };
    // a local unit this group has no tile of: an empty partial (m = -inf, l = 0)
    auto mark_empty = [&](int j) {
      if (q == 0 && lane < G) {
        float* pp = part_ptr(j);
        pp[lane * RS + 0] = -INFINITY;
        pp[lane * RS + 1] = 0.f;
      }
    };
    // End of local unit j: the group's partial (m, l, acc) of the unit. The reference maxima
    // are the group's; the sums of p, of p * min and the value sums are added over the
    // group's four warps in a fixed order (warp 0 first).
    auto finish = [&](int j) {
      float* pp = part_ptr(j);
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const float l = warp_sum(lsum[h]);
        if (lane == 0) redf[q * L::RED_F + 4 * HG + h] = l;
      }
      // lane (g, c), g < 4: sum_t p * min(t, g) of head 4 nb + c in dmin[nb][0] + dmin[nb][1]
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
        if (r < 4) redf[q * L::RED_F + 4 * (4 * nb + c) + r] = dmin[nb][0] + dmin[nb][1];
      named_sync(bar_id, 128);
      for (int h = 0; h < G; ++h) {
        const int nb = h >> 2;
        if (c == (h & 3)) {  // the 8 lanes holding head h: 16 coordinates each
#pragma unroll
          for (int g = 0; g < 4; ++g)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
              for (int nbb = 0; nbb < NB; ++nbb) {
                if (nbb != nb) continue;
                const float* d = dv[g][hf][nbb];
                int j0;
                float v0, v1;
                // element = code * 2^(bit - 24): bit 6 (row r) and bit 8 (row r + 8) at 2 bits,
                // bit 6 for both at 4 bits
                if (VB == 2) {
                  j0 = 4 * (8 * g + r) + 2 * hf;
                  v0 = (d[0] + d[1]) * 262144.f;
                  v1 = (d[2] + d[3]) * 65536.f;
                } else if (VB == 3) {  // coordinates 32g + 4r + 2hf (+ 1), codes at bit 6
                  j0 = 32 * g + 4 * r + 2 * hf;
                  v0 = (d[0] + d[1]) * 262144.f;
                  v1 = (d[2] + d[3]) * 262144.f;
                } else {
                  j0 = 2 * (16 * g + 8 * hf + r);
                  v0 = (d[0] + d[1]) * 262144.f;
                  v1 = (d[2] + d[3]) * 262144.f;
                }
                red[q * kD + j0] = v0;
                red[q * kD + j0 + 1] = v1;
              }
        }
        named_sync(bar_id, 128);
        {
          const int gq = R >> 5;  // value group of coordinate R
          const float msum = ((redf[4 * h + gq] + redf[L::RED_F + 4 * h + gq]) + redf[2 * L::RED_F + 4 * h + gq]) +
                             redf[3 * L::RED_F + 4 * h + gq];
          const float acc = ((red[R] + red[kD + R]) + red[2 * kD + R]) + red[3 * kD + R];
          pp[h * RS + 4 + R] = failed ? 0.f : acc + msum;
        }
        named_sync(bar_id, 128);
      }
      if (q == 0 && lane < G) {
        const int h = lane;
        const float Ls = ((redf[4 * HG + h] + redf[L::RED_F + 4 * HG + h]) + redf[2 * L::RED_F + 4 * HG + h]) +
                         redf[3 * L::RED_F + 4 * HG + h];
        pp[h * RS + 0] = failed ? -INFINITY : Mref[h];
        pp[h * RS + 1] = failed ? 0.f : Ls;
      }
      named_sync(bar_id, 128);  // redf is reused by the next unit
    };

    // Key bits -> unsigned 8-bit elements in tensor memory (row R of the A operand) of the
    // tile in slot `slot` of stage `st`.
    auto expand_keys = [&](const unsigned char* st, int slot) {
      uint32_t w[L::EW];
      const uint4* kc = reinterpret_cast<const uint4*>(st + L::OFF_KC + (slot * kTileTc + R) * L::KCB);
#pragma unroll
      for (int cc = 0; cc < LMB; ++cc) {
        const uint4 v = kc[cc];
        w[4 * cc] = v.x;
        w[4 * cc + 1] = v.y;
        w[4 * cc + 2] = v.z;
        w[4 * cc + 3] = v.w;
      }
      if constexpr (QJL) {
        const uint4 v = *reinterpret_cast<const uint4*>(st + L::OFF_KS + (slot * kTileTc + R) * L::SB);
        w[L::KSC] = v.x;
        w[L::KSC + 1] = v.y;
        w[L::KSC + 2] = v.z;
        w[L::KSC + 3] = v.w;
      }
      if constexpr (LMB == 3) {
#pragma unroll
        for (int gq = 0; gq < 4; ++gq) w[L::CW + gq] = parity_word(w[3 * gq], w[3 * gq + 1], w[3 * gq + 2]);
      }
      static_assert(L::EW % 4 == 0, "element words in groups of four");
#pragma unroll
      for (int e4 = 0; e4 < L::EW / 4; ++e4) {
        uint32_t m[32];  // four element words x eight masks: 32 tensor-memory columns
#pragma unroll
        for (int ee = 0; ee < 4; ++ee) {
          const uint32_t x = w[4 * e4 + ee], x4 = x >> 4;
          m[8 * ee + 0] = bitmask_el<0>(x, x4);
          m[8 * ee + 1] = bitmask_el<1>(x, x4);
          m[8 * ee + 2] = bitmask_el<2>(x, x4);
          m[8 * ee + 3] = bitmask_el<3>(x, x4);
          m[8 * ee + 4] = bitmask_el<4>(x, x4);
          m[8 * ee + 5] = bitmask_el<5>(x, x4);
          m[8 * ee + 6] = bitmask_el<6>(x, x4);
          m[8 * ee + 7] = bitmask_el<7>(x, x4);
        }
        tmem_st32(tA + 32 * e4, m);
      }
      s1::tmem_st_wait();
    };
    // Writes the key elements of the group's tile i (if it exists) and signals the MMA warp;
    // every warp arrives, also without work, so that the phases stay in step.
    auto stage_keys = [&](int i) {
      if (i >= ntl) return;
      const int s = (i >> 1) % NST, slot = i & 1;
      if (!failed && !wait_phase(&full[s], (uint32_t)((i >> 1) / NST) & 1u, abort_flag)) failed = true;
      if (!failed) expand_keys(ring + s * L::STAGE, slot);
      s1::fence_before_sync();
      __syncwarp();
      if (lane == 0) s1::mbar_arrive(&afull[gi]);
    };

    // Moves the group from local unit `from` (finished) to local unit `to` (n_units: none):
    // units in between get empty partials; the leader steps through their operand phases in
    // order, releasing each before waiting for the next, so that a buffer's phases are never
    // skipped and no parity wait can match the phase of two loads back; then the group waits
    // for the operand of unit `to`. Every warp of the group is past unit `from` here, so its
    // operand buffer may be reloaded.
    int cur = -1, qrow0 = 0;
    auto enter_unit = [&](int from, int to) {
      for (int jj = from + 1; jj < to; ++jj) mark_empty(jj);
      if (leader) {
        asm volatile("fence.acq_rel.cta;" ::: "memory");
        for (int jj = from + 1; jj < to && !failed; ++jj) {
          grp_unit[gi] = jj;
          if (!wait_phase(&fbfull[jj % NBUF], (uint32_t)(jj / NBUF) & 1u, abort_flag)) failed = true;
        }
        grp_unit[gi] = to;
        if (failed) raise_abort(abort_flag);
      }
      named_sync(bar_id, 128);
      cur = to;
      reset();
      if (to < n_units) {
        const int u = u_first + to;
        const int bq = u / a.hkv, kvh = u - bq * a.hkv;
        qrow0 = bq * a.hq + kvh * G;
        if (!failed && !wait_phase(&fbfull[to % NBUF], (uint32_t)(to / NBUF) & 1u, abort_flag)) failed = true;
      }
    };

    for (int k = 0; k < gi; ++k) walk.next();
    if (gi < ntl) {
      stage_keys(gi);
      enter_unit(-1, walk.u - u_first);
    }
    int kt = 0;  // tiles of this group so far
    for (int i = gi; i < ntl; i += NG, ++kt) {
      const int s = (i >> 1) % NST, slot = i & 1;
      const int nt = walk.nt();
      const int64_t tok0 = walk.tok0();
      for (int k = 0; k < NG; ++k) walk.next();
      const int j = cur;
      const unsigned char* st = ring + s * L::STAGE;
      // ---- tile i's digit sums (its MMAs done: the A operand is free again), logits
      if (!failed && !wait_phase(&mmad[gi], (uint32_t)kt & 1u, abort_flag)) failed = true;
      s1::fence_after_sync();
      const bool valid = R < nt && !failed;
      float lg[HG];
      {
        // digit sums recombined: (s0 + 2^8 s1) + 2^16 (s2 + 2^8 s3), each part an exact int;
        // the code columns first, then the sign columns (fewer live registers)
        float code[HG], sg[HG];
        {
          uint32_t ds[L::NC];
#pragma unroll
          for (int cc = 0; cc < L::NC; cc += 16) tmem_ld16(tD + cc, ds + cc);
          s1::tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < HG; ++h)
            code[h] = (float)((int)ds[4 * h] + ((int)ds[4 * h + 1] << 8)) +
                      65536.f * (float)((int)ds[4 * h + 2] + ((int)ds[4 * h + 3] << 8));
        }
#pragma unroll
        for (int h = 0; h < HG; ++h) sg[h] = 0.f;
        if constexpr (QJL) {
          uint32_t ds[L::NC];
#pragma unroll
          for (int cc = 0; cc < L::NC; cc += 16) tmem_ld16(tD + L::NC + cc, ds + cc);
          s1::tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < HG; ++h)
            sg[h] = (float)((int)ds[4 * h] + ((int)ds[4 * h + 1] << 8)) +
                    65536.f * (float)((int)ds[4 * h + 2] + ((int)ds[4 * h + 3] << 8));
        }
        const uint32_t ngw = *reinterpret_cast<const uint32_t*>(st + L::OFF_KN + (slot * kTileTc + R) * 4);
        const float2 ng = __half22float2(h2of(ngw));  // (n, gamma)
        const float4* kc4 = reinterpret_cast<const float4*>(sm + L::SM_B + (j % NBUF) * L::BBUF_AL + L::BOP);
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          const float4 k = kc4[h];
          const float l = ng.x * fmaf(ng.y, fmaf(k.z, sg[h], -k.w), fmaf(k.y, code[h], k.x));
          lg[h] = (valid && h < G) ? l : -INFINITY;
        }
      }
      s1::fence_before_sync();
      // ---- the next tile's key elements: its MMAs overlap the rest of this tile
      stage_keys(i + NG);
      if (a.scores && valid) {
#pragma unroll
        for (int h = 0; h < HG; ++h)
          if (h < G) a.scores[(size_t)(qrow0 + h) * a.max_len + tok0 + R] = lg[h] * kLn2;
      }
      // ---- online softmax with the group's reference maxima, moved only when a logit exceeds
      // them by more than the slack; the sums so far are rescaled then
      bool need = false;
#pragma unroll
      for (int h = 0; h < HG; ++h) need |= lg[h] > Mref[h] + kSlackTc;
      if (named_sync_or(bar_id, 128, need)) {
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          const float wm = warp_max(lg[h]);
          if (lane == 0) rm[q * 8 + h] = wm;
        }
        named_sync(bar_id, 128);
        float corr[HG];
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          const float Mn = fmaxf(fmaxf(fmaxf(Mref[h], rm[h]), fmaxf(rm[8 + h], rm[16 + h])), rm[24 + h]);
          corr[h] = 1.f;
          if (Mn > Mref[h]) {
            corr[h] = Mref[h] == -INFINITY ? 0.f : ex2f(Mref[h] - Mn);
            Mref[h] = Mn;
          }
          lsum[h] *= corr[h];
        }
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          const float cf = corr[4 * nb + c];  // this lane's value sums are of head 4 nb + c
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
      // ---- p per head, as f16 high and low parts for the value MMAs
      {
        float p[HG];
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          p[h] = lg[h] == -INFINITY ? 0.f : ex2f(lg[h] - Mref[h]);
          lsum[h] += p[h];
        }
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          const __half hi = __float2half_rn(p[h]);
          const __half lo = __float2half_rn(p[h] - __half2float(hi));
          pt[h * 32 + lane] = hi;
          pt[(HG + h) * 32 + lane] = lo;
        }
      }
      __syncwarp();
      // ---- value sums of the warp's tokens: two K blocks of 16 tokens
      {
        const unsigned char* vcb = st + L::OFF_VC + (slot * kTileTc + 32 * q) * L::VCB;
        const unsigned char* vpb = st + L::OFF_VP + (slot * kTileTc + 32 * q) * L::PB;
        const int part = r & 1, hsel = r >> 1;
        const uint32_t sel = (uint32_t)(r & 3) | ((uint32_t)(4 + (r & 3)) << 8);
        const int nvw = nt - 32 * q;  // valid tokens of this warp (may be <= 0 or >= 32)
        const bool wfail = __any_sync(kFull, failed);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          if (wfail || nvw <= 16 * kb) break;  // warp-uniform
          // K order of the block: rows 2c, 2c + 1 (register 0) and 2c + 8, 2c + 9 (register 1)
          // are tokens 16 kb + 2c, + 1, + 8, + 9 of the warp
          const int tA0 = 16 * kb + 2 * c, tA1 = tA0 + 1, tB0 = tA0 + 8, tB1 = tA0 + 9;
          uint32_t phA[NB], plA[NB], phB[NB], plB[NB];
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const int h = 4 * nb + hsel;
            phA[nb] = *reinterpret_cast<const uint32_t*>(pt + h * 32 + tA0);
            plA[nb] = *reinterpret_cast<const uint32_t*>(pt + (HG + h) * 32 + tA0);
            phB[nb] = *reinterpret_cast<const uint32_t*>(pt + h * 32 + tB0);
            plB[nb] = *reinterpret_cast<const uint32_t*>(pt + (HG + h) * 32 + tB0);
          }
          uint4 pA0 = *reinterpret_cast<const uint4*>(vpb + tA0 * L::PB);
          uint4 pA1 = *reinterpret_cast<const uint4*>(vpb + tA1 * L::PB);
          uint4 pB0 = *reinterpret_cast<const uint4*>(vpb + tB0 * L::PB);
          uint4 pB1 = *reinterpret_cast<const uint4*>(vpb + tB1 * L::PB);
          if (nvw < 16 * kb + 16) {  // tokens past the end: scale 0 (their bytes are stale)
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
            if (tA0 >= nvw) pA0 = z;
            if (tA1 >= nvw) pA1 = z;
            if (tB0 >= nvw) pB0 = z;
            if (tB1 >= nvw) pB1 = z;
          }
          {
            // the group minima through one more MMA: rows g < 4 = min(token, g) of the K pairs,
            // columns = p (high, low) of the heads
            uint4 am = make_uint4(0u, 0u, 0u, 0u);
            if (r < 4) {
              am.x = __byte_perm(word_of(pA0, r), word_of(pA1, r), 0x7632);
              am.z = __byte_perm(word_of(pB0, r), word_of(pB1, r), 0x7632);
            }
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
              mma16816(dmin[nb], am, part ? plA[nb] : phA[nb], part ? plB[nb] : phB[nb]);
          }
          const uint32_t* vA0 = reinterpret_cast<const uint32_t*>(vcb + tA0 * L::VCB);
          const uint32_t* vA1 = reinterpret_cast<const uint32_t*>(vcb + tA1 * L::VCB);
          const uint32_t* vB0 = reinterpret_cast<const uint32_t*>(vcb + tB0 * L::VCB);
          const uint32_t* vB1 = reinterpret_cast<const uint32_t*>(vcb + tB1 * L::VCB);
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            // B element (token, head, part) = p * scale(token, g) in f16 hi + lo:
            // hi = p_hi * s (rounded), err = fma(p_hi, s, -hi) (exact), lo = fma(p_lo, s, err)
            const __half2 sA = h2of(__byte_perm(word_of(pA0, g), word_of(pA1, g), 0x5410));
            const __half2 sB = h2of(__byte_perm(word_of(pB0, g), word_of(pB1, g), 0x5410));
            uint32_t bA[NB], bB[NB];
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
              const __half2 hA = __hmul2(h2of(phA[nb]), sA), hB = __hmul2(h2of(phB[nb]), sB);
              const __half2 eA = __hfma2(h2of(phA[nb]), sA, __hneg2(hA));
              const __half2 eB = __hfma2(h2of(phB[nb]), sB, __hneg2(hB));
              bA[nb] = part ? hbits(__hfma2(h2of(plA[nb]), sA, eA)) : hbits(hA);
              bB[nb] = part ? hbits(__hfma2(h2of(plB[nb]), sB, eB)) : hbits(hB);
            }
            // Row r of block (g, hf) is one byte of the group's codes; the codes of the two
            // tokens of a K pair go to the low byte of each f16 half.
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              uint32_t xA, xB;
              uint4 av;
              // Every code ends in mantissa bits 6..9 of its f16, the largest subnormals: the
              // tensor cores resolve products with small subnormal elements less finely
              // (strongly peaked attention showed errors near 1e-4 with codes in bits 0..3).
              if (VB == 2) {
                // byte 8g + r: rows r -> coordinate 4(8g + r) + 2hf (bits 4hf.. of the byte,
                // to bits 6, 7), rows r + 8 -> + 1 (to bits 8, 9)
                const int wv = 2 * g + (r >> 2);
                xA = __byte_perm(vA0[wv], vA1[wv], sel) << (6 - 4 * hf);
                xB = __byte_perm(vB0[wv], vB1[wv], sel) << (6 - 4 * hf);
                av = make_uint4(xA & 0x00C000C0u, xA & 0x03000300u, xB & 0x00C000C0u, xB & 0x03000300u);
              } else if (VB == 3) {
                // 3-bit fields straddle bytes: row r takes coordinates 32g + 4r .. + 3, the 12 bits
                // at bit 12r of the group's 96 (one funnel shift per token); rows r -> coordinate
                // 32g + 4r + 2hf, rows r + 8 -> + 1, every code moved to bits 6..8
                if (hf == 0) {
                  const int bo = 12 * r, wi = 3 * g + (bo >> 5), wj = 3 * g + min((bo >> 5) + 1, 2), sh = bo & 31;
                  xA = __byte_perm(__funnelshift_r(vA0[wi], vA0[wj], sh), __funnelshift_r(vA1[wi], vA1[wj], sh), 0x5410);
                  xB = __byte_perm(__funnelshift_r(vB0[wi], vB0[wj], sh), __funnelshift_r(vB1[wi], vB1[wj], sh), 0x5410);
                  av = make_uint4((xA << 6) & 0x01C001C0u, (xA << 3) & 0x01C001C0u, (xB << 6) & 0x01C001C0u,
                                  (xB << 3) & 0x01C001C0u);
                } else {
                  av = make_uint4(xA & 0x01C001C0u, (xA >> 3) & 0x01C001C0u, xB & 0x01C001C0u,
                                  (xB >> 3) & 0x01C001C0u);
                }
              } else {
                // byte 16g + 8hf + r: rows r -> coordinate 2(16g + 8hf + r) (low nibble), rows
                // r + 8 -> + 1 (high nibble), both to bits 6..9
                const int wv = 4 * g + 2 * hf + (r >> 2);
                xA = __byte_perm(vA0[wv], vA1[wv], sel);
                xB = __byte_perm(vB0[wv], vB1[wv], sel);
                av = make_uint4((xA << 6) & 0x03C003C0u, (xA << 2) & 0x03C003C0u, (xB << 6) & 0x03C003C0u,
                                (xB << 2) & 0x03C003C0u);
              }
#pragma unroll
              for (int nb = 0; nb < NB; ++nb) mma16816(dv[g][hf][nb], av, bA[nb], bB[nb]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) s1::mbar_arrive(&empty[s]);  // the stage is no longer read by this warp
      // ---- unit boundary: the group's next tile (walk) belongs to another unit, or there is none
      const int jn = i + NG < ntl ? walk.u - u_first : n_units;
      if (jn != cur) {
        finish(cur);
        enter_unit(cur, jn);
      }
    }
    if (gi >= ntl)
      for (int jj = 0; jj < n_units; ++jj) mark_empty(jj);
    if (leader) grp_unit[gi] = 0x7fffffff;  // done: the producer may reload any buffer
    if (failed && lane == 0) raise_abort(abort_flag);
  }

  // ---------------------------------------------------------------- end
  __syncthreads();
  if (tid == 0 && *abort_flag) atomicOr(a.err, 1u);
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
  cfg.blockDim = dim3(L::THREADS);
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
  return vb == 2   ? launch_tc_nb<LMB, QJL, 2>(ctx, pa, units, a, n_ctas, nb, s)
         : vb == 3 ? launch_tc_nb<LMB, QJL, 3>(ctx, pa, units, a, n_ctas, nb, s)
                   : launch_tc_nb<LMB, QJL, 4>(ctx, pa, units, a, n_ctas, nb, s);
}

template <int LMB, bool QJL>
int tc_groups_t(int nb, int vb) {
  if (vb == 2) return nb == 1 ? TcLayout<LMB, QJL, 2, 1>::NG : TcLayout<LMB, QJL, 2, 2>::NG;
  if (vb == 3) return nb == 1 ? TcLayout<LMB, QJL, 3, 1>::NG : TcLayout<LMB, QJL, 3, 2>::NG;
  return nb == 1 ? TcLayout<LMB, QJL, 4, 1>::NG : TcLayout<LMB, QJL, 4, 2>::NG;
}

template <int LMB, bool QJL>
size_t tc_bbuf_t(int nb, int vb) {
  if (vb == 2) return nb == 1 ? TcLayout<LMB, QJL, 2, 1>::BBUF : TcLayout<LMB, QJL, 2, 2>::BBUF;
  if (vb == 3) return nb == 1 ? TcLayout<LMB, QJL, 3, 1>::BBUF : TcLayout<LMB, QJL, 3, 2>::BBUF;
  return nb == 1 ? TcLayout<LMB, QJL, 4, 1>::BBUF : TcLayout<LMB, QJL, 4, 2>::BBUF;
}

}  // namespace

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


bool tc_decode_supported(const tq_ctx* ctx, int G) {
  const Shape& sh = ctx->shape;
  if (sh.d != kD || !(sh.m == kM || sh.m == 0) || G < 1 || G > 8) return false;
  if (sh.lm_bits < 1 || sh.lm_bits > 3) return false;
  if (sh.v_bits < 2 || sh.v_bits > 4) return false;
  float kappa, beta[4];
  return codebook_bits(ctx->cb, sh.lm_bits, kappa, beta);
}

int tc_groups(const tq_ctx* ctx, int G) {
  const int nb = G <= 4 ? 1 : 2, vb = ctx->shape.v_bits;
  const bool qjl = ctx->shape.m > 0;
  switch (ctx->shape.lm_bits) {
    case 1: return qjl ? tc_groups_t<1, true>(nb, vb) : tc_groups_t<1, false>(nb, vb);
    case 2: return qjl ? tc_groups_t<2, true>(nb, vb) : tc_groups_t<2, false>(nb, vb);
    default: return qjl ? tc_groups_t<3, true>(nb, vb) : tc_groups_t<3, false>(nb, vb);
  }
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
  return launch_combine_partials(part, out, lse, batch, hq, hkv, G, plan.s_max, tc_groups(ctx, G),
                                 plan.tiles_per_unit, plan.total_tiles, plan.n_ctas, stream);
}

}  // namespace tq
