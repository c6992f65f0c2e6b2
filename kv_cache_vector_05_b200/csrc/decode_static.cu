// Decode attention whose scratch lives in a fixed device array of this library,
// for callers that cannot allocate device memory themselves.
//
// tq_decode_attention needs a caller-provided workspace (prepared queries and the
// split-K partials). Some callers cannot provide one: code that runs where no
// device allocator is reachable (a plugin handed only input and output pointers
// by its host application), serving loops that must not call cudaMalloc once
// they are running (it can synchronize the device and stall other streams), or
// small runtimes without a caching allocator. tq_decode_attention_static runs
// the same kernels with the workspace placed in `g_decode_scratch` below.
#include <cuda_runtime.h>

#include <cstdio>

#include "tq_internal.h"

namespace {

// Fixed scratch, one copy per device that loads the library, held until the
// process exits. 32 MiB covers, e.g., 72 (sequence, KV head) pairs x 8192 tokens
// x 16 query heads at d = 128 (about 13 MB) or 256 pairs x 32768 tokens x 32
// query heads (about 10 MB).
constexpr size_t kStaticScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

}  // namespace

extern "C" {

size_t tq_decode_static_scratch_capacity(void) { return kStaticScratchBytes; }

tq_status tq_decode_attention_static(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int batch,
                                     int hq, int hkv, const int32_t* seq_lens, int64_t max_len,
                                     const uint8_t* k_codes, const uint8_t* k_signs,
                                     const uint16_t* k_norms, const uint8_t* v_codes,
                                     const uint16_t* v_params, float softmax_scale, float* scores,
                                     float* out, void* stream) {
  if (!ctx || batch < 0 || hq <= 0 || hkv <= 0 || hq % hkv || max_len < 0) {
    tq::set_last_error("tq_decode_attention_static: NULL context or bad batch/head/length arguments");
    return TQ_EINVAL;
  }
  const size_t need = tq_decode_workspace_bytes(ctx, batch, hq, hkv, max_len);
  if (need > kStaticScratchBytes) {
    char msg[256];
    std::snprintf(msg, sizeof(msg),
                  "tq_decode_attention_static: this shape needs %zu bytes of scratch, the static "
                  "buffer holds %zu; use tq_decode_attention with a workspace",
                  need, kStaticScratchBytes);
    tq::set_last_error(msg);
    return TQ_EUNSUPPORTED;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    tq::set_last_error("tq_decode_attention_static: no usable current device");
    return TQ_ECUDA;
  }
  if (dev != ctx->device) {
    tq::set_last_error("tq_decode_attention_static: the context belongs to another device");
    return TQ_EINVAL;
  }
  // The host-side name of a __device__ array is not a device address, so ask the
  // runtime for it, with the caller's device current. The address belongs to the
  // module loaded in the current CUDA context; it is looked up on every call (a host
  // table lookup once the module is loaded) rather than cached, so that a context
  // created after a device reset, or a context the caller made current itself, gets
  // its own copy's address. The first call in a context loads the module: make it
  // before any stream capture.
  void* ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
  if (e != cudaSuccess || !ptr) {
    char msg[256];
    std::snprintf(msg, sizeof(msg), "tq_decode_attention_static: cudaGetSymbolAddress failed: %s",
                  cudaGetErrorString(e));
    tq::set_last_error(msg);
    return TQ_ECUDA;
  }
  // Everything the kernels read from the scratch is written earlier in the same
  // call (prepared queries, then every split-K partial), so nothing needs clearing.
  return tq_decode_attention(ctx, q, q_dtype, batch, hq, hkv, seq_lens, max_len, k_codes, k_signs,
                             k_norms, v_codes, v_params, softmax_scale, scores, out, ptr,
                             kStaticScratchBytes, stream);
}

}  // extern "C"
