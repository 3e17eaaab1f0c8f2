// K/V append: the step's "one write-head".
//
// "Fast Transformer Decoding" (velog paper review), §3: every step writes one
// K and one V row per sequence, new_K = concat(prev_K, k_new).  With a cache of
// fixed size [b, m_max, g, d] that is a bitwise copy of k_new[b] (g*d
// elements, contiguous in both places) to row pos[b].  The g K/V heads of a row
// sit next to each other in the cache, so one sequence is two contiguous
// copies, done here with 16-byte loads and stores.
#include "common.cuh"

namespace mqa {

namespace {

constexpr int kAppendThreads = 128;

__global__ void __launch_bounds__(kAppendThreads)
append_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache, const uint4* __restrict__ k_new,
              const uint4* __restrict__ v_new, const int32_t* __restrict__ pos, int m_max, int row_k16,
              int row_v16, int32_t* flags) {
  // The cache may be read by the kernel that ran before on this stream; with
  // programmatic dependent launch the wait below orders this kernel's writes
  // after it.  Without PDL it returns at once.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // The decode that usually follows may start its set-up now; it waits for
  // this grid's writes before it reads the cache.
  asm volatile("griddepcontrol.launch_dependents;");
  const int b = blockIdx.x;
  const int p = __ldg(pos + b);
  if (p < 0 || p >= m_max) {
    if (threadIdx.x == 0) set_flag(flags, MQA_FLAG_POS_SKIPPED);
    return;
  }
  const int64_t dst_k = (int64_t(b) * m_max + p) * row_k16;
  const int64_t dst_v = (int64_t(b) * m_max + p) * row_v16;
  for (int i = threadIdx.x; i < row_k16; i += kAppendThreads)
    k_cache[dst_k + i] = __ldg(k_new + int64_t(b) * row_k16 + i);
  for (int i = threadIdx.x; i < row_v16; i += kAppendThreads)
    v_cache[dst_v + i] = __ldg(v_new + int64_t(b) * row_v16 + i);
}

}  // namespace

cudaError_t launch_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new, const int32_t* pos,
                          int b, int m_max, int g, int row_k_bytes, int row_v_bytes, int32_t* flags,
                          cudaStream_t stream) {
  // row_*_bytes is the size of one cache row (all g heads), a multiple of 16.
  (void)g;
  append_kernel<<<b, kAppendThreads, 0, stream>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), static_cast<const uint4*>(k_new),
      static_cast<const uint4*>(v_new), pos, m_max, row_k_bytes / 16, row_v_bytes / 16, flags);
  return cudaGetLastError();
}

}  // namespace mqa
