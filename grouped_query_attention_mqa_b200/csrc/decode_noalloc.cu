// mqa_decode_noalloc: the decode with its scratch in a fixed device array.
//
// Some callers cannot hand the library a workspace: code that runs where no
// allocator is reachable (a plugin inside a host application that owns every
// allocation, a custom runtime whose memory pool is fixed at start-up, or a
// call site that may not allocate because allocating could synchronise the
// device or fail at a point where failure is not allowed).  For them this
// entry point keeps the split-KV partials in a file-scope device array of
// MQA_NOALLOC_SCRATCH_BYTES that every GPU which loads the library holds
// until the process exits.  It calls no allocator of any kind.
//
// The array's host-side name is only a stand-in for the symbol, not a device
// address, so the host looks the address up once per device with
// cudaGetSymbolAddress (with that device current) and passes it to the
// kernels like any other workspace pointer.
#include <atomic>
#include <cmath>
#include <cstdint>

#include "common.cuh"

namespace mqa {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MQA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on the current device, looked up on
// the first call per device.  Returns nullptr if the lookup fails.  Host
// threads may make their first calls concurrently: each slot is an atomic,
// and two threads that both look the address up store the same value.
void* scratch_address() {
  static std::atomic<void*> addr[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* cached = addr[dev].load(std::memory_order_acquire);
  if (cached != nullptr) return cached;
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
  addr[dev].store(ptr, std::memory_order_release);
  return ptr;
}

int sm_count_current() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// Scratch bytes for `slots` partials: the same three regions as the regular
// workspace, sized for exactly the slots this call can use.
size_t scratch_bytes(int b, int g, int hq, int d_v, size_t slots) {
  return align256(sizeof(int2) * size_t(b) * size_t(g)) + align256(sizeof(float) * slots * hq) +
         align256(sizeof(float) * slots * hq * size_t(d_v));
}

Workspace carve(void* base, int b, int g, int hq, size_t slots) {
  char* p = static_cast<char*>(base);
  Workspace w;
  w.seg_info = reinterpret_cast<int2*>(p);
  p += align256(sizeof(int2) * size_t(b) * size_t(g));
  w.part_lse = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * slots * hq);
  w.part_o = reinterpret_cast<float*>(p);
  return w;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace mqa

extern "C" mqa_status_t mqa_decode_noalloc(void* o, const void* q, const void* k_cache, const void* v_cache,
                                           const int32_t* lens, int b, int h, int g, int m_max, int d_k, int d_v,
                                           float scale, mqa_dtype_t dtype, int32_t* status_flags,
                                           cudaStream_t stream) {
  using namespace mqa;
  if (b < 0 || h < 1 || g < 1 || h % g != 0 || m_max < 1 || d_k < 1 || d_v < 1 ||
      (dtype != MQA_F32 && dtype != MQA_BF16) || !std::isfinite(scale))
    return MQA_ERR_INVALID_ARG;
  if (b == 0) return MQA_OK;
  if (!o || !q || !k_cache || !v_cache || !lens) return MQA_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(lens))
    return MQA_ERR_INVALID_ARG;
  if (int64_t(b) * g > (int64_t(1) << 30) || int64_t(b) * m_max * g > (int64_t(1) << 40))
    return MQA_ERR_INVALID_ARG;
  if ((d_k != 32 && d_k != 64 && d_k != 128) || (d_v != 32 && d_v != 64 && d_v != 128)) return MQA_ERR_UNSUPPORTED;
  const int hq = h / g;
  const bool use_tc = dtype == MQA_BF16 && tc_supported(d_k, d_v, hq);
  if (!use_tc && (int64_t(hq) * d_k > 4096 || int64_t(hq) * d_v > 4096)) return MQA_ERR_UNSUPPORTED;

  // Largest CTA count whose partials fit the array; reject when even one CTA
  // does not fit.
  const size_t segs = size_t(b) * size_t(g);
  if (scratch_bytes(b, g, hq, d_v, segs + 1) > size_t(MQA_NOALLOC_SCRATCH_BYTES)) return MQA_ERR_INVALID_ARG;
  const int sms = sm_count_current();
  if (sms <= 0) return MQA_ERR_CUDA;
  int grid = sms * (use_tc ? tc_ctas_per_sm(hq) : simt_ctas_per_sm(dtype, d_k, d_v, hq));
  if (grid > kMaxCtas) grid = kMaxCtas;
  while (grid > 1 && scratch_bytes(b, g, hq, d_v, segs + size_t(grid)) > size_t(MQA_NOALLOC_SCRATCH_BYTES)) {
    const int step = grid / 8 > 0 ? grid / 8 : 1;
    grid -= step;
  }
  if (grid < 1) grid = 1;

  void* scratch = scratch_address();
  if (scratch == nullptr) return MQA_ERR_CUDA;

  DecodeArgs a;
  a.o = o;
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.k_new = nullptr;
  a.v_new = nullptr;
  a.lens = lens;
  a.b = b;
  a.h = h;
  a.g = g;
  a.m_max = m_max;
  a.d = d_v;
  a.dk = d_k;
  a.hq = hq;
  a.window = 0;
  a.q_beams = 0;
  a.q_group_heads = hq;
  // As in mqa_decode: when no sequence can span two tiles no segment is split,
  // the decode writes every output row itself and the merge is not launched.
  a.no_merge = m_max <= (use_tc ? tc_tile_rows() : simt_tile_rows());
  a.sk = nullptr;
  a.sv = nullptr;
  a.slens = nullptr;
  a.m_s = 0;
  a.scale = scale;
  a.ws = carve(scratch, b, g, hq, segs + size_t(grid));
  a.flags = status_flags;
  a.grid = grid;
  cudaError_t e = use_tc ? launch_decode_tc(a, stream) : launch_decode_simt(a, d_k, dtype, stream);
  if (e != cudaSuccess) return MQA_ERR_CUDA;
  if (!a.no_merge && launch_merge(a, dtype, stream) != cudaSuccess) return MQA_ERR_CUDA;
  return MQA_OK;
}
