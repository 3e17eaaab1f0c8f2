// The C ABI of libmqa: argument checks, the choice of kernel path and CTA
// count, and the launches.  No allocation, no synchronisation, no exceptions.
#include <atomic>
#include <cmath>
#include <cstdint>

#include "common.cuh"

namespace {

using namespace mqa;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
int elem_bytes(mqa_dtype_t dt) { return dt == MQA_F32 ? 4 : 2; }
bool valid_dtype(int dt) { return dt == MQA_F32 || dt == MQA_BF16; }

// SM count of the current device, cached per device.
int sm_count() {
  static std::atomic<int> cache[64];   // 0 = not yet known; every thread computes the same value
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

}  // namespace

extern "C" {

const char* mqa_status_string(mqa_status_t s) {
  switch (s) {
    case MQA_OK: return "MQA_OK";
    case MQA_ERR_INVALID_ARG: return "MQA_ERR_INVALID_ARG";
    case MQA_ERR_UNSUPPORTED: return "MQA_ERR_UNSUPPORTED";
    case MQA_ERR_CUDA: return "MQA_ERR_CUDA";
  }
  return "MQA_STATUS_UNKNOWN";
}

mqa_status_t mqa_kv_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new, const int32_t* pos,
                           int b, int m_max, int g, int d_k, int d_v, mqa_dtype_t dtype, int32_t* status_flags,
                           cudaStream_t stream) {
  if (b < 0 || m_max < 1 || g < 1 || d_k < 1 || d_v < 1 || !valid_dtype(dtype)) return MQA_ERR_INVALID_ARG;
  if (b == 0) return MQA_OK;
  if (!k_cache || !v_cache || !k_new || !v_new || !pos) return MQA_ERR_INVALID_ARG;
  const int64_t row_k = int64_t(g) * d_k * elem_bytes(dtype), row_v = int64_t(g) * d_v * elem_bytes(dtype);
  if (row_k % 16 != 0 || row_v % 16 != 0 || row_k > (int64_t(1) << 30) || row_v > (int64_t(1) << 30))
    return MQA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(pos))
    return MQA_ERR_INVALID_ARG;
  if (launch_append(k_cache, v_cache, k_new, v_new, pos, b, m_max, g, int(row_k), int(row_v), status_flags,
                    stream) != cudaSuccess)
    return MQA_ERR_CUDA;
  return MQA_OK;
}

size_t mqa_decode_workspace_size(int b, int h, int g, int d_v) {
  if (b < 0 || h < 1 || g < 1 || h % g != 0 || d_v < 1) return 0;
  return workspace_bytes(b, g, h / g, d_v);
}

}  // extern "C"

namespace {

// mqa_decode_ex, and with k_new/v_new the fused append + decode.
mqa_status_t decode_impl(void* o, const void* q, const void* k_cache, const void* v_cache, const void* k_new,
                         const void* v_new, const int32_t* lens, int b, int h, int g, int m_max, int d_k, int d_v,
                         float scale, mqa_dtype_t dtype, void* workspace, size_t workspace_bytes_given,
                         int32_t* status_flags, const mqa_decode_opts_t* opts, cudaStream_t stream) {
  if (b < 0 || h < 1 || g < 1 || h % g != 0 || m_max < 1 || d_k < 1 || d_v < 1 || !valid_dtype(dtype) ||
      !std::isfinite(scale))
    return MQA_ERR_INVALID_ARG;
  const int path = opts ? opts->path : MQA_PATH_AUTO;
  if (path < MQA_PATH_AUTO || path > MQA_PATH_TCGEN05) return MQA_ERR_INVALID_ARG;
  if (opts && (opts->num_ctas < 0 || opts->num_ctas > kMaxCtas || opts->window < 0)) return MQA_ERR_INVALID_ARG;
  if (b == 0) return MQA_OK;
  if (!o || !q || !k_cache || !v_cache || !lens || !workspace) return MQA_ERR_INVALID_ARG;
  if ((k_new == nullptr) != (v_new == nullptr)) return MQA_ERR_INVALID_ARG;
  if (k_new && (!aligned16(k_new) || !aligned16(v_new))) return MQA_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(lens) ||
      !aligned256(workspace))
    return MQA_ERR_INVALID_ARG;
  if (int64_t(b) * g > (int64_t(1) << 30) || int64_t(b) * m_max * g > (int64_t(1) << 40))
    return MQA_ERR_INVALID_ARG;
  const int hq = h / g;
  if (workspace_bytes_given < workspace_bytes(b, g, hq, d_v)) return MQA_ERR_INVALID_ARG;
  if ((d_k != 32 && d_k != 64 && d_k != 128) || (d_v != 32 && d_v != 64 && d_v != 128)) return MQA_ERR_UNSUPPORTED;

  const bool tc_ok = dtype == MQA_BF16 && tc_supported(d_k, d_v, hq);
  const bool simt_ok = int64_t(hq) * d_k <= 4096 && int64_t(hq) * d_v <= 4096;
  bool use_tc;
  if (path == MQA_PATH_TCGEN05) {
    if (!tc_ok) return MQA_ERR_UNSUPPORTED;
    use_tc = true;
  } else if (path == MQA_PATH_SIMT) {
    if (!simt_ok) return MQA_ERR_UNSUPPORTED;
    use_tc = false;
  } else {
    use_tc = tc_ok;
    if (!use_tc && !simt_ok) return MQA_ERR_UNSUPPORTED;
  }

  const int sms = sm_count();
  if (sms <= 0) return MQA_ERR_CUDA;
  DecodeArgs a;
  a.o = o;
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.k_new = k_new;
  a.v_new = v_new;
  a.lens = lens;
  a.b = b;
  a.h = h;
  a.g = g;
  a.m_max = m_max;
  a.d = d_v;
  a.dk = d_k;
  a.hq = hq;
  a.window = opts ? opts->window : 0;
  a.q_beams = 0;
  a.q_group_heads = hq;
  a.sk = nullptr;
  a.sv = nullptr;
  a.slens = nullptr;
  a.m_s = 0;
  // When no sequence spans more than one tile no segment is ever split, so
  // every output row is final when the decode kernel ends: the merge is left out.
  const int span_max = a.window > 0 && a.window < m_max ? a.window : m_max;
  a.no_merge = span_max <= (use_tc ? tc_tile_rows() : simt_tile_rows());
  a.scale = scale;
  a.ws = carve_workspace(workspace, b, g, hq);
  a.flags = status_flags;
  int grid = opts && opts->num_ctas > 0 ? opts->num_ctas
                                         : sms * (use_tc ? tc_ctas_per_sm(hq) : simt_ctas_per_sm(dtype, d_k, d_v, hq));
  a.grid = grid < 1 ? 1 : (grid > kMaxCtas ? kMaxCtas : grid);

  cudaError_t e = use_tc ? launch_decode_tc(a, stream) : launch_decode_simt(a, d_k, dtype, stream);
  if (e != cudaSuccess) return MQA_ERR_CUDA;
  if (!a.no_merge) e = launch_merge(a, dtype, stream);
  if (e != cudaSuccess) return MQA_ERR_CUDA;
  return MQA_OK;
}

}  // namespace

extern "C" {

mqa_status_t mqa_decode_ex(void* o, const void* q, const void* k_cache, const void* v_cache, const int32_t* lens,
                           int b, int h, int g, int m_max, int d_k, int d_v, float scale, mqa_dtype_t dtype,
                           void* workspace, size_t workspace_bytes_given, int32_t* status_flags,
                           const mqa_decode_opts_t* opts, cudaStream_t stream) {
  return decode_impl(o, q, k_cache, v_cache, nullptr, nullptr, lens, b, h, g, m_max, d_k, d_v, scale, dtype,
                     workspace, workspace_bytes_given, status_flags, opts, stream);
}

size_t mqa_decode_beam_workspace_size(int b, int W, int h, int g, int d_v) {
  if (b < 0 || W < 1 || h < 1 || g < 1 || h % g != 0 || d_v < 1) return 0;
  return workspace_bytes(b, g, W * (h / g), d_v);
}

mqa_status_t mqa_decode_beam(void* o, const void* q, const void* prefix_k, const void* prefix_v,
                             const int32_t* prefix_lens, const void* suffix_k, const void* suffix_v,
                             const int32_t* suffix_lens, int b, int W, int h, int g, int m_p, int m_s, int d_k,
                             int d_v, float scale, mqa_dtype_t dtype, void* workspace, size_t workspace_bytes_given,
                             int32_t* status_flags, cudaStream_t stream) {
  if (b < 0 || W < 1 || h < 1 || g < 1 || h % g != 0 || m_p < 1 || m_s < 1 || d_k < 1 || d_v < 1 ||
      !valid_dtype(dtype) || !std::isfinite(scale))
    return MQA_ERR_INVALID_ARG;
  if (b == 0) return MQA_OK;
  if (!o || !q || !prefix_k || !prefix_v || !prefix_lens || !suffix_k || !suffix_v || !suffix_lens || !workspace)
    return MQA_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(q) || !aligned16(prefix_k) || !aligned16(prefix_v) || !aligned16(prefix_lens) ||
      !aligned16(suffix_k) || !aligned16(suffix_v) || !aligned16(suffix_lens) || !aligned256(workspace))
    return MQA_ERR_INVALID_ARG;
  if (int64_t(b) * W * g > (int64_t(1) << 30) || int64_t(b) * m_p * g > (int64_t(1) << 40) ||
      int64_t(b) * W * m_s * g > (int64_t(1) << 40) || int64_t(b) * W * h >= (int64_t(1) << 31))
    return MQA_ERR_INVALID_ARG;
  const int hq = h / g;
  if (workspace_bytes_given < mqa_decode_beam_workspace_size(b, W, h, g, d_v)) return MQA_ERR_INVALID_ARG;
  if (dtype != MQA_BF16 || d_k != 128 || d_v != 128 || !tc_supported(d_k, d_v, W * hq)) return MQA_ERR_UNSUPPORTED;
  const int sms = sm_count();
  if (sms <= 0) return MQA_ERR_CUDA;
  // One pass: segment (s, j) reads sequence s's prefix once for the W beams'
  // heads of group j (a 3-D box gathers their query rows), then each beam's
  // suffix rows, which count for that beam's heads only.
  DecodeArgs a;
  a.o = o;
  a.q = q;
  a.k = prefix_k;
  a.v = prefix_v;
  a.k_new = nullptr;
  a.v_new = nullptr;
  a.lens = prefix_lens;
  a.b = b;
  a.h = h;
  a.g = g;
  a.m_max = m_p;
  a.d = d_v;
  a.dk = d_k;
  a.hq = W * hq;
  a.window = 0;
  a.no_merge = 0;
  a.q_beams = W;
  a.q_group_heads = hq;
  a.sk = suffix_k;
  a.sv = suffix_v;
  a.slens = suffix_lens;
  a.m_s = m_s;
  a.scale = scale;
  a.ws = carve_workspace(workspace, b, g, W * hq);
  a.flags = status_flags;
  a.grid = sms * tc_ctas_per_sm(W * hq);
  if (launch_decode_tc(a, stream) != cudaSuccess || launch_merge(a, dtype, stream) != cudaSuccess)
    return MQA_ERR_CUDA;
  return MQA_OK;
}

mqa_status_t mqa_prefill(void* o, const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int b,
                         int total, int max_seqlen, int h, int g, int d_k, int d_v, float scale, int causal,
                         mqa_dtype_t dtype, int32_t* status_flags, cudaStream_t stream) {
  if (b < 0 || total < 0 || max_seqlen < 0 || h < 1 || g < 1 || h % g != 0 || d_k < 1 || d_v < 1 ||
      !valid_dtype(dtype) || !std::isfinite(scale) || (causal != 0 && causal != 1))
    return MQA_ERR_INVALID_ARG;
  if (b == 0 || total == 0 || max_seqlen == 0) return MQA_OK;
  if (!o || !q || !k || !v || !cu_seqlens) return MQA_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(cu_seqlens))
    return MQA_ERR_INVALID_ARG;
  if (dtype != MQA_BF16 || d_k != d_v || !prefill_tc_supported(d_k, h / g)) return MQA_ERR_UNSUPPORTED;
  const cudaError_t e = launch_prefill_tc(o, q, k, v, cu_seqlens, b, total, h, g, max_seqlen, scale, causal,
                                          status_flags, stream);
  if (e == cudaErrorInvalidValue) return MQA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? MQA_OK : MQA_ERR_CUDA;
}

mqa_status_t mqa_decode(void* o, const void* q, const void* k_cache, const void* v_cache, const int32_t* lens, int b,
                        int h, int g, int m_max, int d_k, int d_v, float scale, mqa_dtype_t dtype, void* workspace,
                        size_t workspace_bytes_given, int32_t* status_flags, cudaStream_t stream) {
  return decode_impl(o, q, k_cache, v_cache, nullptr, nullptr, lens, b, h, g, m_max, d_k, d_v, scale, dtype,
                     workspace, workspace_bytes_given, status_flags, nullptr, stream);
}

mqa_status_t mqa_decode_append(void* o, const void* q, void* k_cache, void* v_cache, const void* k_new,
                               const void* v_new, const int32_t* lens, int b, int h, int g, int m_max, int d_k,
                               int d_v, float scale, mqa_dtype_t dtype, void* workspace,
                               size_t workspace_bytes_given, int32_t* status_flags, const mqa_decode_opts_t* opts,
                               cudaStream_t stream) {
  if (b > 0 && (k_new == nullptr || v_new == nullptr)) return MQA_ERR_INVALID_ARG;
  return decode_impl(o, q, k_cache, v_cache, k_new, v_new, lens, b, h, g, m_max, d_k, d_v, scale, dtype, workspace,
                     workspace_bytes_given, status_flags, opts, stream);
}

}  // extern "C"
