// Internal declarations shared by the C-ABI layer and the CUDA kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/tq.h"

namespace tq {

constexpr int kMaxLmBits = 7;  // 1-3 on the tensor-core kernels, 4-7 on the CUDA-core ones
constexpr int kMaxLevels = 1 << kMaxLmBits;
constexpr int kMaxD = 256;
constexpr int kMaxM = 256;
constexpr int kVGroup = 32;

// Small method tables passed by value to every kernel (parameter space, uniform
// across the warp, no global loads).
struct Codebook {
  float c[kMaxLevels];      // centroids, ascending
  float t[kMaxLevels - 1];  // boundaries, ascending
  int levels;               // 2^lm_bits
  uint32_t sign_bits[kMaxD / 32];  // Hadamard sign diagonal: bit j set <=> sigma_j = -1
};

struct Shape {
  int d;
  int lm_bits;
  int m;
  int v_bits;
  int rot;  // tq_rot
};

// Cache addressing of the decode kernels. Contiguous (block_table null): token t of unit
// u = (sequence, KV head) is record row u * max_len + t. Paged: it is row
// block_table[u * max_pages + t / page_size] * page_size + t % page_size, page_size a
// multiple of every kernel's tile so that a tile never crosses a page.
struct Paging {
  const int32_t* block_table;
  int64_t page_size, max_pages, n_pages;
};

}  // namespace tq

struct tq_ctx {
  tq::Shape shape;
  tq::Codebook cb;
  int device;
  int num_sms;
  float* S;        // device [m][d] fp32 row-major
  float* St;       // device [d][m] fp32 (transpose of S)
  float* Pi;       // device [d][d] fp32 row-major (Haar only)
  float* PiT;      // device [d][d] fp32 transpose (Haar only)
  int decode_kernel;       // tq_decode_kernel selected by tq_set_decode_kernel
  cudaEvent_t prof_start;  // optional events around the main kernel of each call
  cudaEvent_t prof_stop;
  unsigned int* d_err;     // device error word: bit 0 = a bounded wait in a kernel timed out,
                           // bit 2 = a slot or page index outside the caller's arrays
  uint16_t* S_sw128;       // tensor-core compression: S as f16 hi and lo operand tiles (d = m = 128)
  uint16_t* H_sw128;       // tensor-core compression: H diag(sigma) as a bf16 operand tile (d = 128, Hadamard)
  uint16_t* Pi_sw128;      // tensor-core compression: Haar Pi as three bf16 operand tiles (d = 128)
  uint16_t* dense_ops;     // tensor-core compression at d = 64 / 256 (m = d): rotation and S operand tiles
};

namespace tq {

// Launchers (defined in the .cu files). Return cudaSuccess or the launch error.
// slot: null (vector i -> row i) or the output row of each vector, checked against n_rows.
cudaError_t launch_compress(const tq_ctx* ctx, const void* k, const void* v, int dtype,
                            int64_t n_vec, const int64_t* slot, int64_t n_rows, uint8_t* k_codes,
                            uint8_t* k_signs, uint16_t* k_norms, uint8_t* v_codes, uint16_t* v_params,
                            cudaStream_t stream);

struct DecodePlan {
  bool supported;    // false: the context's selected kernel family does not take the shape
  int family;        // tq_decode_kernel that runs (never TQ_DECODE_AUTO)
  bool tc;           // tcgen05 score kernels (decode_tc.cu)
  bool mma;          // mma.sync kernels (decode_mma.cu) instead of the generic ones
  int n_chunks;      // split-K chunks per (sequence, KV head)
  int64_t chunk_len; // tokens per chunk (multiple of the tile)
  size_t ws_q_bytes;     // generic path: prepared queries
  size_t ws_part_bytes;  // partial (m, l, acc) per chunk and query head
  size_t off_frag, off_part, off_cnt;  // tensor-core path: byte offsets in the workspace
  // tensor-core path: the units' tiles are split evenly over n_ctas resident CTAs
  int n_ctas;
  int64_t tiles_per_unit, total_tiles;
  int s_max;         // most CTAs that share one unit (partial slots per unit)
  size_t total_bytes;
};

DecodePlan plan_decode(const tq_ctx* ctx, int batch, int hq, int hkv, int64_t max_len);

cudaError_t launch_decode(const tq_ctx* ctx, const DecodePlan& plan, const void* q, int q_dtype,
                          int batch, int hq, int hkv, const int32_t* seq_lens, int64_t max_len,
                          const Paging& pg, const uint8_t* k_codes, const uint8_t* k_signs,
                          const uint16_t* k_norms, const uint8_t* v_codes, const uint16_t* v_params,
                          float scale, float* scores, float* out, float* lse, void* workspace,
                          cudaStream_t stream);

bool mma_decode_supported(const tq_ctx* ctx, int G);
// Bit expansion of a symmetric 1- to 3-bit codebook (decode_tc.cu): c[idx] = kappa + sum_p
// beta_p bit_p, with bit 3 the parity of the three code bits at 3 bits; false otherwise.
bool codebook_bits(const Codebook& cb, int lmb, float& kappa, float beta[4]);
bool tc_decode_supported(const tq_ctx* ctx, int G);
size_t tc_operand_bytes(const tq_ctx* ctx, int G);  // query operand bytes per (sequence, KV head)
int tc_groups(const tq_ctx* ctx, int G);            // warp groups (partials per CTA and unit)

cudaError_t launch_decode_tc(const tq_ctx* ctx, const DecodePlan& plan, const void* q, int q_dtype, int batch,
                             int hq, int hkv, const int32_t* seq_lens, int64_t max_len, const Paging& pg,
                             const uint8_t* k_codes, const uint8_t* k_signs, const uint16_t* k_norms,
                             const uint8_t* v_codes, const uint16_t* v_params, float scale, float* scores,
                             float* out, float* lse, void* workspace, cudaStream_t stream);

// Log-sum-exp merge of the partials (m, l in base 2, acc) of the tile-split decode kernels
// into out (and lse), launched as a programmatic dependent of the decode grid (decode_mma.cu).
// With tile_tokens = 0 the layout is [units][s_max][ppc][G][4 + 128] (ppc partials per CTA,
// tiles split by max_len); with tile_tokens > 0 it is decode_mma_kernel's split by the tokens
// present (tiles of tile_tokens, lengths from seq_lens and max_len; with lengths, seq_first
// holds each sequence's first tile in that order and the total, as the decode grid wrote
// them): CTA k's partial of unit u in slot u + k of [units + n_ctas][G][4 + 128]. A partial with m = -inf carries no token and
// its sums are not read.
cudaError_t launch_combine_partials(const float* part, float* out, float* lse, int batch, int hq, int hkv, int G,
                                    int s_max, int ppc, int64_t tiles_per_unit, int64_t total_tiles, int n_ctas,
                                    cudaStream_t stream, int tile_tokens = 0, const int32_t* seq_lens = nullptr,
                                    const int64_t* seq_first = nullptr, int64_t max_len = 0);

size_t mma_frag_bytes(int lm_bits, int G);  // query operand bytes per (sequence, KV head)
int mma_tile_tokens(int G);                  // tokens per tile of the tensor-core decode
int mma_ctas_per_sm(int lm_bits, int v_bits, int G);  // resident CTAs per SM of the tensor-core decode
bool pack_qjl_operand(const float* S, int m, int d, uint16_t* out);
void pack_hadamard_operand(const uint32_t* sign_bits, uint16_t* out);  // d = 128
void pack_haar_operand(const double* pi, uint16_t* out);                // d = 128, 3 tiles
bool pack_dense_operands(int d, int rot, const uint32_t* sign_bits, const double* haar, const float* S,
                         std::vector<uint16_t>& out);                   // d = 64 / 256

cudaError_t launch_decode_mma(const tq_ctx* ctx, const DecodePlan& plan, const void* q, int q_dtype, int batch,
                              int hq, int hkv, const int32_t* seq_lens, int64_t max_len, const Paging& pg,
                              const uint8_t* k_codes,
                              const uint8_t* k_signs, const uint16_t* k_norms, const uint8_t* v_codes,
                              const uint16_t* v_params, float scale, float* scores, float* out, float* lse,
                              void* workspace, cudaStream_t stream);

// Log-sum-exp merge of n_parts attention outputs of disjoint token ranges (merge.cu).
cudaError_t launch_merge(const float* outs, int64_t outs_stride, const float* lses, int64_t lses_stride,
                         int n_parts, int64_t rows, int d, float* out, float* lse, cudaStream_t stream);

cudaError_t launch_decompress(const tq_ctx* ctx, const uint8_t* k_codes, const uint8_t* k_signs,
                              const uint16_t* k_norms, const uint8_t* v_codes,
                              const uint16_t* v_params, int64_t n_vec, float* k_out, float* v_out,
                              cudaStream_t stream);

// Records the message tq_last_error() returns on this thread (tq_api.cpp).
void set_last_error(const char* msg);

// Host math (tq_host_math.cpp).
int lloyd_max_sphere(int d, int bits, double* centroids, double* boundaries);
int haar_from_gaussian(int d, const double* g, double* q);

}  // namespace tq
