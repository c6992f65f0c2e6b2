// C ABI entry points: argument validation, context management and dispatch to
// the kernel launchers. No exception crosses this boundary.
#include <cmath>
#include <string>
#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include "tq_internal.h"

namespace {

thread_local char g_last_error[512] = "";

tq_status fail(tq_status st, const char* msg) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s", msg);
  return st;
}
tq_status fail(tq_status st, const std::string& msg) { return fail(st, msg.c_str()); }

tq_status fail_cuda(cudaError_t e, const char* where) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorName(e),
                cudaGetErrorString(e));
  return TQ_ECUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

void free_tables(tq_ctx* c) {
  if (!c) return;
  cudaFree(c->S);
  cudaFree(c->St);
  cudaFree(c->Pi);
  cudaFree(c->PiT);
  cudaFree(c->d_err);
  cudaFree(c->S_sw128);
  cudaFree(c->H_sw128);
  cudaFree(c->Pi_sw128);
  cudaFree(c->dense_ops);
}

}  // namespace

namespace tq {
void set_last_error(const char* msg) { std::snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }
}  // namespace tq

extern "C" {

const char* tq_status_string(tq_status s) {
  switch (s) {
    case TQ_OK: return "TQ_OK";
    case TQ_EINVAL: return "TQ_EINVAL: invalid argument";
    case TQ_EUNSUPPORTED: return "TQ_EUNSUPPORTED: unsupported size or bit width";
    case TQ_ECUDA: return "TQ_ECUDA: CUDA error";
    case TQ_ENOMEM: return "TQ_ENOMEM: out of memory";
  }
  return "TQ_UNKNOWN";
}

const char* tq_last_error(void) { return g_last_error; }

tq_status tq_lloyd_max_codebook(int d, int bits, float* centroids, float* boundaries) {
  if (!centroids || !boundaries) return fail(TQ_EINVAL, "tq_lloyd_max_codebook: NULL output");
  if (d < 4 || d > 4096 || bits < 1 || bits > 7)
    return fail(TQ_EINVAL, "tq_lloyd_max_codebook: d must be in [4,4096], bits in [1,7]");
  double c[128], t[127];  // up to 7 bits
  if (tq::lloyd_max_sphere(d, bits, c, t) != 0)
    return fail(TQ_EINVAL, "tq_lloyd_max_codebook: iteration did not converge");
  for (int k = 0; k < (1 << bits); ++k) centroids[k] = (float)c[k];
  for (int k = 0; k + 1 < (1 << bits); ++k) boundaries[k] = (float)t[k];
  return TQ_OK;
}

tq_status tq_haar_from_gaussian(int d, const double* gaussian, double* pi_out) {
  if (!gaussian || !pi_out) return fail(TQ_EINVAL, "tq_haar_from_gaussian: NULL pointer");
  if (d < 1 || d > 1024) return fail(TQ_EINVAL, "tq_haar_from_gaussian: d must be in [1,1024]");
  if (tq::haar_from_gaussian(d, gaussian, pi_out) != 0)
    return fail(TQ_EINVAL, "tq_haar_from_gaussian: input is rank deficient");
  return TQ_OK;
}

tq_status tq_codebook_load(const tq_params* p, void* stream, tq_ctx** out) {
  if (!p || !out) return fail(TQ_EINVAL, "tq_codebook_load: NULL params or out");
  *out = nullptr;
  const int d = p->d, b = p->k_lm_bits, m = p->qjl_m;
  if (!(d == 64 || d == 128 || d == 256))
    return fail(TQ_EUNSUPPORTED, "tq_codebook_load: d must be 64, 128 or 256");
  if (b < 1 || b > tq::kMaxLmBits)
    return fail(TQ_EUNSUPPORTED, "tq_codebook_load: k_lm_bits must be in [1, 7]");
  if (b * (d / 32) > 32)
    return fail(TQ_EUNSUPPORTED, "tq_codebook_load: k_lm_bits * d / 32 must be at most 32 (d = 256: 4 bits)");
  if (m < 0 || m > tq::kMaxM || m % 32)
    return fail(TQ_EUNSUPPORTED, "tq_codebook_load: qjl_m must be 0 (no QJL stage) or a multiple of 32 up to 256");
  if (!(p->v_bits == 2 || p->v_bits == 3 || p->v_bits == 4))
    return fail(TQ_EUNSUPPORTED, "tq_codebook_load: v_bits must be 2, 3 or 4");
  if (p->v_group != tq::kVGroup)
    return fail(TQ_EUNSUPPORTED, "tq_codebook_load: v_group must be 32");
  if (p->rot != TQ_ROT_HADAMARD && p->rot != TQ_ROT_HAAR)
    return fail(TQ_EINVAL, "tq_codebook_load: unknown rotation");
  if (!p->centroids || !p->boundaries || (m > 0 && !p->qjl_S))
    return fail(TQ_EINVAL, "tq_codebook_load: NULL codebook or QJL matrix");
  if (p->rot == TQ_ROT_HADAMARD && !p->hadamard_signs)
    return fail(TQ_EINVAL, "tq_codebook_load: NULL Hadamard signs");
  if (p->rot == TQ_ROT_HAAR && !p->haar) return fail(TQ_EINVAL, "tq_codebook_load: NULL Haar matrix");

  const int L = 1 << b;
  for (int k = 0; k + 1 < L; ++k)
    if (!(p->centroids[k] < p->centroids[k + 1]))
      return fail(TQ_EINVAL, "tq_codebook_load: centroids must be strictly ascending");
  for (int k = 0; k + 2 < L; ++k)
    if (!(p->boundaries[k] < p->boundaries[k + 1]))
      return fail(TQ_EINVAL, "tq_codebook_load: boundaries must be strictly ascending");
  for (int k = 0; k < L; ++k)
    if (!std::isfinite(p->centroids[k])) return fail(TQ_EINVAL, "tq_codebook_load: non-finite centroid");
  if (p->rot == TQ_ROT_HADAMARD)
    for (int j = 0; j < d; ++j)
      if (p->hadamard_signs[j] != 1 && p->hadamard_signs[j] != -1)
        return fail(TQ_EINVAL, "tq_codebook_load: Hadamard signs must be +1 or -1");

  tq_ctx* c = new (std::nothrow) tq_ctx();
  if (!c) return fail(TQ_ENOMEM, "tq_codebook_load: host allocation failed");
  std::memset(c, 0, sizeof(*c));
  c->shape = {d, b, m, p->v_bits, (int)p->rot};
  c->cb.levels = L;
  for (int k = 0; k < tq::kMaxLevels; ++k) c->cb.c[k] = k < L ? p->centroids[k] : 0.f;
  for (int k = 0; k < tq::kMaxLevels - 1; ++k) c->cb.t[k] = k + 1 < L ? p->boundaries[k] : INFINITY;
  if (p->rot == TQ_ROT_HADAMARD)
    for (int j = 0; j < d; ++j)
      if (p->hadamard_signs[j] < 0) c->cb.sign_bits[j / 32] |= 1u << (j % 32);

  cudaError_t e = cudaGetDevice(&c->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
  if (e != cudaSuccess) {
    delete c;
    return fail_cuda(e, "tq_codebook_load: device query");
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::vector<float> S((size_t)m * d), St((size_t)d * m);
  for (int i = 0; i < m; ++i)
    for (int j = 0; j < d; ++j) {
      S[(size_t)i * d + j] = p->qjl_S[(size_t)i * d + j];
      St[(size_t)j * m + i] = p->qjl_S[(size_t)i * d + j];
    }
  std::vector<float> Pi, PiT;
  if (p->rot == TQ_ROT_HAAR) {
    Pi.resize((size_t)d * d);
    PiT.resize((size_t)d * d);
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < d; ++j) {
        Pi[(size_t)i * d + j] = (float)p->haar[(size_t)i * d + j];
        PiT[(size_t)j * d + i] = (float)p->haar[(size_t)i * d + j];
      }
  }
  auto alloc = [&](float** dst, size_t n) -> cudaError_t { return cudaMalloc((void**)dst, n * sizeof(float)); };
  if (m > 0) e = alloc(&c->S, S.size());  // m = 0: no QJL stage, no S
  if (e == cudaSuccess && m > 0) e = alloc(&c->St, St.size());
  if (e == cudaSuccess && !Pi.empty()) e = alloc(&c->Pi, Pi.size());
  if (e == cudaSuccess && !Pi.empty()) e = alloc(&c->PiT, PiT.size());
  if (e == cudaSuccess) e = cudaMalloc((void**)&c->d_err, sizeof(unsigned int));
  std::vector<uint16_t> s_op;
  if (d == 128 && m == 128) {
    s_op.assign((size_t)2 * m * d, 0);  // hi and lo tiles
    if (!tq::pack_qjl_operand(p->qjl_S, m, d, s_op.data())) s_op.clear();
    if (e == cudaSuccess && !s_op.empty()) e = cudaMalloc((void**)&c->S_sw128, s_op.size() * sizeof(uint16_t));
  }
  std::vector<uint16_t> h_op;
  // the rotation operand of the pipelined compression kernel: with the QJL stage when S fits
  // its operand tiles, and for keys without it (m = 0)
  const bool pipe_rot = d == 128 && ((m == 128 && !s_op.empty()) || m == 0);
  if (pipe_rot && p->rot == TQ_ROT_HADAMARD) {
    h_op.assign((size_t)d * d, 0);
    tq::pack_hadamard_operand(c->cb.sign_bits, h_op.data());
    if (e == cudaSuccess) e = cudaMalloc((void**)&c->H_sw128, h_op.size() * sizeof(uint16_t));
  }
  std::vector<uint16_t> dense_op;
  if ((d == 64 || d == 256) && m == d && b <= 3) {
    if (!tq::pack_dense_operands(d, p->rot, c->cb.sign_bits, p->haar, p->qjl_S, dense_op)) dense_op.clear();
    if (e == cudaSuccess && !dense_op.empty())
      e = cudaMalloc((void**)&c->dense_ops, dense_op.size() * sizeof(uint16_t));
  }
  std::vector<uint16_t> pi_op;
  if (pipe_rot && p->rot == TQ_ROT_HAAR) {
    pi_op.assign((size_t)3 * d * d, 0);
    tq::pack_haar_operand(p->haar, pi_op.data());
    if (e == cudaSuccess) e = cudaMalloc((void**)&c->Pi_sw128, pi_op.size() * sizeof(uint16_t));
  }
  if (e != cudaSuccess) {
    free_tables(c);
    delete c;
    cudaGetLastError();
    return e == cudaErrorMemoryAllocation ? fail(TQ_ENOMEM, "tq_codebook_load: cudaMalloc failed")
                                          : fail_cuda(e, "tq_codebook_load: cudaMalloc");
  }
  if (m > 0) e = cudaMemcpyAsync(c->S, S.data(), S.size() * sizeof(float), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && m > 0)
    e = cudaMemcpyAsync(c->St, St.data(), St.size() * sizeof(float), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !Pi.empty())
    e = cudaMemcpyAsync(c->Pi, Pi.data(), Pi.size() * sizeof(float), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !Pi.empty())
    e = cudaMemcpyAsync(c->PiT, PiT.data(), PiT.size() * sizeof(float), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->d_err, 0, sizeof(unsigned int), s);
  if (e == cudaSuccess && !s_op.empty())
    e = cudaMemcpyAsync(c->S_sw128, s_op.data(), s_op.size() * sizeof(uint16_t), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !h_op.empty())
    e = cudaMemcpyAsync(c->H_sw128, h_op.data(), h_op.size() * sizeof(uint16_t), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !pi_op.empty())
    e = cudaMemcpyAsync(c->Pi_sw128, pi_op.data(), pi_op.size() * sizeof(uint16_t), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !dense_op.empty())
    e = cudaMemcpyAsync(c->dense_ops, dense_op.data(), dense_op.size() * sizeof(uint16_t), cudaMemcpyHostToDevice,
                        s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    free_tables(c);
    delete c;
    return fail_cuda(e, "tq_codebook_load: upload");
  }
  *out = c;
  return TQ_OK;
}

tq_status tq_set_profile_events(tq_ctx* c, void* start, void* stop) {
  if (!c) return fail(TQ_EINVAL, "tq_set_profile_events: NULL context");
  if ((start == nullptr) != (stop == nullptr))
    return fail(TQ_EINVAL, "tq_set_profile_events: give both events or neither");
  c->prof_start = static_cast<cudaEvent_t>(start);
  c->prof_stop = static_cast<cudaEvent_t>(stop);
  return TQ_OK;
}

tq_status tq_set_decode_kernel(tq_ctx* c, tq_decode_kernel k) {
  if (!c) return fail(TQ_EINVAL, "tq_set_decode_kernel: NULL context");
  if (k < TQ_DECODE_AUTO || k > TQ_DECODE_CUDA_CORE) return fail(TQ_EINVAL, "tq_set_decode_kernel: unknown kernel");
  c->decode_kernel = (int)k;
  return TQ_OK;
}

int tq_decode_kernel_for(const tq_ctx* c, int hq, int hkv) {
  if (!c || hq <= 0 || hkv <= 0 || hq % hkv) return -1;
  const tq::DecodePlan p = tq::plan_decode(c, 1, hq, hkv, 1);
  return p.supported ? p.family : -1;
}

tq_status tq_check_device(const tq_ctx* c, void* stream) {
  if (!c) return fail(TQ_EINVAL, "tq_check_device: NULL context");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int flag = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&flag, c->d_err, sizeof(flag), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && flag) e = cudaMemset(c->d_err, 0, sizeof(flag));
  if (e != cudaSuccess) return fail_cuda(e, "tq_check_device");
  if (flag & 1u) return fail(TQ_ECUDA, "tq_check_device: a bounded wait for a bulk copy timed out; results of that call are invalid");
  if (flag & 4u)
    return fail(TQ_EINVAL, "tq_check_device: a slot or page index was outside the caller's arrays; those vectors "
                           "were not written (compression) or read as page 0 (decode)");
  return TQ_OK;
}

void tq_free(tq_ctx* c) {
  if (!c) return;
  free_tables(c);
  delete c;
}

namespace {
// Shared by tq_compress_kv (slot = NULL: vector i to row i) and tq_compress_kv_slots.
tq_status compress_impl(const char* name, const tq_ctx* c, const void* k, const void* v, tq_dtype dtype,
                        int64_t n_vec, const int64_t* slot, int64_t n_rows, uint8_t* k_codes, uint8_t* k_signs,
                        uint16_t* k_norms, uint8_t* v_codes, uint16_t* v_params, void* stream) {
  const std::string nm(name);
  if (!c) return fail(TQ_EINVAL, nm + ": NULL context");
  if (n_vec < 0) return fail(TQ_EINVAL, nm + ": negative n_vec");
  if (n_vec == 0) return TQ_OK;
  if (dtype != TQ_F32 && dtype != TQ_BF16) return fail(TQ_EINVAL, nm + ": bad dtype");
  if (!k && !v) return fail(TQ_EINVAL, nm + ": both k and v are NULL");
  if (k && (!k_codes || (c->shape.m > 0 && !k_signs) || !k_norms)) return fail(TQ_EINVAL, nm + ": NULL key output");
  if (v && (!v_codes || !v_params)) return fail(TQ_EINVAL, nm + ": NULL value output");
  if (k && !(aligned16(k) && aligned16(k_codes) && aligned16(k_signs) && aligned16(k_norms)))
    return fail(TQ_EINVAL, nm + ": key pointers must be 16-byte aligned");
  if (v && !(aligned16(v) && aligned16(v_codes) && aligned16(v_params)))
    return fail(TQ_EINVAL, nm + ": value pointers must be 16-byte aligned");
  if (slot && ((reinterpret_cast<uintptr_t>(slot) & 7u) || n_rows <= 0))
    return fail(TQ_EINVAL, nm + ": the slot map must be 8-byte aligned and n_rows positive");
  if (n_vec > (int64_t(1) << 40)) return fail(TQ_EINVAL, nm + ": n_vec too large");
  cudaError_t e = tq::launch_compress(c, k, v, (int)dtype, n_vec, slot, n_rows, k_codes, k_signs, k_norms,
                                      v_codes, v_params, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, name);
  return TQ_OK;
}
}  // namespace

tq_status tq_compress_kv(const tq_ctx* c, const void* k, const void* v, tq_dtype dtype, int64_t n_vec,
                         uint8_t* k_codes, uint8_t* k_signs, uint16_t* k_norms, uint8_t* v_codes,
                         uint16_t* v_params, void* stream) {
  return compress_impl("tq_compress_kv", c, k, v, dtype, n_vec, nullptr, 0, k_codes, k_signs, k_norms, v_codes,
                       v_params, stream);
}

tq_status tq_compress_kv_slots(const tq_ctx* c, const void* k, const void* v, tq_dtype dtype, int64_t n_vec,
                               const int64_t* slot, int64_t n_rows, uint8_t* k_codes, uint8_t* k_signs,
                               uint16_t* k_norms, uint8_t* v_codes, uint16_t* v_params, void* stream) {
  if (!slot) return fail(TQ_EINVAL, "tq_compress_kv_slots: NULL slot map");
  return compress_impl("tq_compress_kv_slots", c, k, v, dtype, n_vec, slot, n_rows, k_codes, k_signs, k_norms,
                       v_codes, v_params, stream);
}

size_t tq_decode_workspace_bytes(const tq_ctx* c, int batch, int hq, int hkv, int64_t max_len) {
  if (!c || batch < 0 || hq <= 0 || hkv <= 0 || hq % hkv || max_len < 0) return 0;
  return tq::plan_decode(c, batch, hq, hkv, max_len).total_bytes;
}

namespace {
// Shared by tq_decode_attention (contiguous cache) and tq_decode_attention_paged.
tq_status decode_impl(const char* name, const tq_ctx* c, const void* q, tq_dtype q_dtype, int batch, int hq,
                      int hkv, const int32_t* seq_lens, int64_t max_len, const tq::Paging& pg,
                      const uint8_t* k_codes, const uint8_t* k_signs, const uint16_t* k_norms,
                      const uint8_t* v_codes, const uint16_t* v_params, float softmax_scale, float* scores,
                      float* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  const std::string nm(name);
  if (!c) return fail(TQ_EINVAL, nm + ": NULL context");
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return fail(TQ_EINVAL, nm + ": bad dtype");
  if (batch < 0 || hq <= 0 || hkv <= 0 || hq % hkv || max_len < 0)
    return fail(TQ_EINVAL, nm + ": bad batch/head/length arguments");
  if (hq / hkv > 64 || (c->shape.d == 256 && hq / hkv > 32))
    return fail(TQ_EUNSUPPORTED, nm + ": too many query heads per KV head (max 64; 32 at d=256)");
  if (!std::isfinite(softmax_scale) || softmax_scale < 0.f)
    return fail(TQ_EINVAL, nm + ": softmax_scale must be finite and >= 0");
  if (batch == 0) return TQ_OK;
  if (!q || !out) return fail(TQ_EINVAL, nm + ": NULL q or out");
  if (lse && reinterpret_cast<uintptr_t>(lse) % alignof(float))
    return fail(TQ_EINVAL, nm + ": lse not aligned to a float");
  if (max_len > 0 && (!k_codes || (c->shape.m > 0 && !k_signs) || !k_norms || !v_codes || !v_params))
    return fail(TQ_EINVAL, nm + ": NULL packed cache");
  const void* ptrs[] = {q, out, k_codes, k_signs, k_norms, v_codes, v_params, workspace, scores, seq_lens};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return fail(TQ_EINVAL, nm + ": pointers must be 16-byte aligned");
  if (max_len > (int64_t(1) << 31)) return fail(TQ_EINVAL, nm + ": max_len too large");
  tq::DecodePlan plan = tq::plan_decode(c, batch, hq, hkv, max_len);
  if (!plan.supported) return fail(TQ_EUNSUPPORTED, nm + ": the selected decode kernel does not support this shape");
  if (!workspace || workspace_bytes < plan.total_bytes)
    return fail(TQ_EINVAL, nm + ": workspace missing or too small");
  float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)c->shape.d);
  if (max_len == 0) {  // no tokens anywhere: zero outputs, log-partitions -inf (a merge of no parts)
    cudaError_t e = tq::launch_merge(nullptr, 0, nullptr, 0, 0, (int64_t)batch * hq, c->shape.d, out, lse,
                                     static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail_cuda(e, name);
    return TQ_OK;
  }
  cudaError_t e = tq::launch_decode(c, plan, q, (int)q_dtype, batch, hq, hkv, seq_lens, max_len, pg, k_codes,
                                    k_signs, k_norms, v_codes, v_params, scale, scores, out, lse, workspace,
                                    static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, name);
  return TQ_OK;
}
}  // namespace

tq_status tq_decode_attention(const tq_ctx* c, const void* q, tq_dtype q_dtype, int batch, int hq,
                              int hkv, const int32_t* seq_lens, int64_t max_len,
                              const uint8_t* k_codes, const uint8_t* k_signs,
                              const uint16_t* k_norms, const uint8_t* v_codes,
                              const uint16_t* v_params, float softmax_scale, float* scores,
                              float* out, void* workspace, size_t workspace_bytes, void* stream) {
  const tq::Paging contiguous{nullptr, 0, 0, 0};
  return decode_impl("tq_decode_attention", c, q, q_dtype, batch, hq, hkv, seq_lens, max_len, contiguous,
                     k_codes, k_signs, k_norms, v_codes, v_params, softmax_scale, scores, out, nullptr, workspace,
                     workspace_bytes, stream);
}

tq_status tq_decode_attention_partial(const tq_ctx* c, const void* q, tq_dtype q_dtype, int batch, int hq,
                                      int hkv, const int32_t* seq_lens, int64_t max_len,
                                      const uint8_t* k_codes, const uint8_t* k_signs,
                                      const uint16_t* k_norms, const uint8_t* v_codes,
                                      const uint16_t* v_params, float softmax_scale, float* scores,
                                      float* out, float* lse, void* workspace, size_t workspace_bytes,
                                      void* stream) {
  if (batch > 0 && !lse) return fail(TQ_EINVAL, "tq_decode_attention_partial: NULL lse");
  const tq::Paging contiguous{nullptr, 0, 0, 0};
  return decode_impl("tq_decode_attention_partial", c, q, q_dtype, batch, hq, hkv, seq_lens, max_len,
                     contiguous, k_codes, k_signs, k_norms, v_codes, v_params, softmax_scale, scores, out, lse,
                     workspace, workspace_bytes, stream);
}

tq_status tq_merge_attention(const float* outs, int64_t outs_stride, const float* lses, int64_t lses_stride,
                             int n_parts, int64_t rows, int d, float* out, float* lse, void* stream) {
  if (n_parts <= 0 || rows < 0 || d <= 0)
    return fail(TQ_EINVAL, "tq_merge_attention: n_parts and d must be positive, rows >= 0");
  if (rows > 0x7fffffff) return fail(TQ_EINVAL, "tq_merge_attention: more than 2^31 - 1 rows");
  if (outs_stride < rows * d || lses_stride < rows)
    return fail(TQ_EINVAL, "tq_merge_attention: a part's stride is below its size");
  if (rows == 0) return TQ_OK;
  if (!outs || !lses || !out) return fail(TQ_EINVAL, "tq_merge_attention: NULL outs, lses or out");
  const void* ptrs[] = {outs, lses, out, lse};
  for (const void* ptr : ptrs)
    if (ptr && reinterpret_cast<uintptr_t>(ptr) % alignof(float))
      return fail(TQ_EINVAL, "tq_merge_attention: pointers must be aligned to a float");
  cudaError_t e = tq::launch_merge(outs, outs_stride, lses, lses_stride, n_parts, rows, d, out, lse,
                                   static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "tq_merge_attention");
  return TQ_OK;
}

tq_status tq_decode_attention_paged(const tq_ctx* c, const void* q, tq_dtype q_dtype, int batch, int hq,
                                    int hkv, const int32_t* seq_lens, int64_t max_len,
                                    const int32_t* block_table, int64_t page_size, int64_t max_pages,
                                    int64_t n_pages, const uint8_t* k_codes, const uint8_t* k_signs,
                                    const uint16_t* k_norms, const uint8_t* v_codes, const uint16_t* v_params,
                                    float softmax_scale, float* scores, float* out, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (!block_table || !aligned16(block_table))
    return fail(TQ_EINVAL, "tq_decode_attention_paged: block_table NULL or not 16-byte aligned");
  if (page_size <= 0 || page_size % 512)
    return fail(TQ_EINVAL, "tq_decode_attention_paged: page_size must be a positive multiple of 512");
  if (max_len < 0 || max_pages < (max_len + page_size - 1) / page_size || n_pages <= 0)
    return fail(TQ_EINVAL, "tq_decode_attention_paged: max_pages below ceil(max_len / page_size), or no pages");
  const tq::Paging paged{block_table, page_size, max_pages, n_pages};
  return decode_impl("tq_decode_attention_paged", c, q, q_dtype, batch, hq, hkv, seq_lens, max_len, paged, k_codes,
                     k_signs, k_norms, v_codes, v_params, softmax_scale, scores, out, nullptr, workspace,
                     workspace_bytes, stream);
}

tq_status tq_decompress(const tq_ctx* c, const uint8_t* k_codes, const uint8_t* k_signs,
                        const uint16_t* k_norms, const uint8_t* v_codes, const uint16_t* v_params,
                        int64_t n_vec, float* k_out, float* v_out, void* stream) {
  if (!c) return fail(TQ_EINVAL, "tq_decompress: NULL context");
  if (n_vec < 0) return fail(TQ_EINVAL, "tq_decompress: negative n_vec");
  if (n_vec == 0) return TQ_OK;
  if (!k_out && !v_out) return fail(TQ_EINVAL, "tq_decompress: both outputs NULL");
  if (k_out && (!k_codes || (c->shape.m > 0 && !k_signs) || !k_norms))
    return fail(TQ_EINVAL, "tq_decompress: NULL key input");
  if (v_out && (!v_codes || !v_params)) return fail(TQ_EINVAL, "tq_decompress: NULL value input");
  const void* ptrs[] = {k_codes, k_signs, k_norms, v_codes, v_params, k_out, v_out};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return fail(TQ_EINVAL, "tq_decompress: pointers must be 16-byte aligned");
  if (n_vec == 0) return TQ_OK;
  cudaError_t e = tq::launch_decompress(c, k_out ? k_codes : nullptr, k_signs, k_norms,
                                        v_out ? v_codes : nullptr, v_params, n_vec, k_out, v_out,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "tq_decompress");
  return TQ_OK;
}

}  // extern "C"
