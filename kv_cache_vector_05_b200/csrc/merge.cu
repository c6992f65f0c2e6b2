// Merge of attention outputs computed over disjoint token ranges of the same
// sequences (one range per GPU when a long sequence's cache is split over GPUs).
//
// Each range r gives, per row (sequence, query head), its normalized output o_r
// and the log of its softmax denominator lse_r. The softmax over all tokens is
// then sum_r exp(lse_r) o_r / sum_r exp(lse_r) exactly; the weights are taken
// relative to the largest lse_r so nothing overflows. This is the same
// log-sum-exp merge the split-K decode applies to its chunks, one level up.
//
// Traffic: n_parts * rows * (d + 1) floats read, rows * d (+ rows) written; a few
// KB per decode step for one long sequence, so the kernel is launch-bound and
// kept simple: one CTA per row, one thread per output coordinate.
#include "tq_internal.h"

#include <cuda_runtime.h>

namespace tq {
namespace {

constexpr int kMergeThreads = 128;

struct MergeArgs {
  const float* outs;
  const float* lses;
  int64_t outs_stride, lses_stride;  // floats between consecutive parts
  int n_parts, d;
  float* out;
  float* lse;  // null, or the merged log-partition of each row
};

__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const __grid_constant__ MergeArgs a) {
  const int64_t row = blockIdx.x;
  float M = -INFINITY;
  for (int r = 0; r < a.n_parts; ++r) M = fmaxf(M, a.lses[r * a.lses_stride + row]);
  float den = 0.f;
  if (M != -INFINITY)
    for (int r = 0; r < a.n_parts; ++r) {
      const float l = a.lses[r * a.lses_stride + row];
      den += l == -INFINITY ? 0.f : expf(l - M);
    }
  for (int j = threadIdx.x; j < a.d; j += blockDim.x) {
    float num = 0.f;
    if (den > 0.f)
      for (int r = 0; r < a.n_parts; ++r) {
        const float l = a.lses[r * a.lses_stride + row];
        if (l != -INFINITY) num = fmaf(expf(l - M), a.outs[r * a.outs_stride + row * a.d + j], num);
      }
    a.out[row * a.d + j] = den > 0.f ? num / den : 0.f;
  }
  if (a.lse && threadIdx.x == 0) a.lse[row] = den > 0.f ? M + logf(den) : -INFINITY;
}

}  // namespace

cudaError_t launch_merge(const float* outs, int64_t outs_stride, const float* lses, int64_t lses_stride,
                         int n_parts, int64_t rows, int d, float* out, float* lse, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  // n_parts = 0 writes the empty merge (zero outputs, lse -inf) without reading outs or lses.
  if (rows > 0x7fffffff || n_parts < 0 || d <= 0) return cudaErrorInvalidValue;
  MergeArgs a;
  a.outs = outs;
  a.lses = lses;
  a.outs_stride = outs_stride;
  a.lses_stride = lses_stride;
  a.n_parts = n_parts;
  a.d = d;
  a.out = out;
  a.lse = lse;
  merge_kernel<<<(unsigned)rows, kMergeThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace tq
