// Log-sum-exp merge of split-KV partial outputs.
//
// A segment (sequence b, K/V head j) whose rows were split between CTAs left,
// per CTA k, a normalised partial o_k (softmax over its rows only) and
// lse_k = log2 sum_t 2^{s_t} over those rows (logits in log2 units).  The
// softmax over all rows is then
//   o = sum_k 2^{lse_k - LSE} o_k,   LSE = log2 sum_k 2^{lse_k},
// evaluated here with a running maximum so no exponent overflows.  Segments
// handled whole by one CTA were written by the decode kernel directly; empty
// sequences (length 0 after clamping) get an all-zero output row here.
#include "common.cuh"

namespace mqa {

namespace {

constexpr int kMergeThreads = 128;

template <typename T>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const DecodeArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t s = blockIdx.x;
  const int seq = int(s / a.g), head = int(s - int64_t(seq) * a.g);
  const int hq = a.hq, D = a.d;
  T* O = static_cast<T*>(a.o) + (int64_t(seq) * a.h + int64_t(head) * hq) * D;
  const int len = clamp_len(__ldg(a.lens + seq), a.m_max, nullptr, false);
  if (len == 0) {
    for (int f = threadIdx.x; f < hq * D; f += kMergeThreads) O[f] = from_f32<T>(0.f);
    return;
  }
  const int2 info = a.ws.seg_info[s];
  if (info.x == info.y) return;
  for (int f = threadIdx.x; f < hq * D; f += kMergeThreads) {
    const int i = f / D;
    float m = -INFINITY, wsum = 0.f, acc = 0.f;
    for (int k = info.x; k <= info.y; ++k) {
      const int64_t slot = partial_slot(k, s);
      const float lse = a.ws.part_lse[slot * hq + i];
      const float v = a.ws.part_o[slot * hq * D + f];
      if (lse > m) {
        const float c = exp2f(m - lse);
        acc = acc * c + v;
        wsum = wsum * c + 1.f;
        m = lse;
      } else {
        const float w = exp2f(lse - m);
        acc = fmaf(w, v, acc);
        wsum += w;
      }
    }
    O[f] = from_f32<T>(acc / wsum);
  }
}

}  // namespace

cudaError_t launch_merge(const DecodeArgs& a, mqa_dtype_t dtype, cudaStream_t stream) {
  const int64_t segs = int64_t(a.b) * a.g;
  if (segs > 0x7fffffff) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(segs));
  cfg.blockDim = dim3(kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (dtype == MQA_BF16) return cudaLaunchKernelEx(&cfg, merge_kernel<__nv_bfloat16>, a);
  return cudaLaunchKernelEx(&cfg, merge_kernel<float>, a);
}

}  // namespace mqa
