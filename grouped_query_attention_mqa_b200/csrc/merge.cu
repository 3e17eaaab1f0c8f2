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

// One CTA per (segment, group of heads); each thread merges four consecutive
// output columns of one head, so the few partial loads of every output are
// issued by many threads at once instead of walked serially.
template <typename T>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const DecodeArgs a, int heads_per_cta) {
  const int hq = a.hq, D = a.d;
  const int chunks = (hq + heads_per_cta - 1) / heads_per_cta;
  const int64_t s = blockIdx.x / chunks;
  const int hc = int(blockIdx.x - s * chunks);
  const int tph = D / 4;                                    // threads per head
  const int i = hc * heads_per_cta + int(threadIdx.x) / tph;
  const int c4 = (int(threadIdx.x) % tph) * 4;
  const bool active = threadIdx.x < heads_per_cta * tph && i < hq;
  const int seq = int(s / a.g), head = int(s - int64_t(seq) * a.g);
  // lens is an input of the call, never written by the decode kernel this
  // merge follows, so it is read before waiting for that kernel.
  const int len = active ? clamp_len(__ldg(a.lens + seq), a.m_max, nullptr, false) : 0;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // The next step's decode may launch and set up while the merge runs.
  asm volatile("griddepcontrol.launch_dependents;");
  if (!active) return;
  T* O = static_cast<T*>(a.o) + (int64_t(seq) * a.h + int64_t(head) * hq + i) * D + c4;
  if (len == 0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) O[k] = from_f32<T>(0.f);
    return;
  }
  const int2 info = a.ws.seg_info[s];
  if (info.x == info.y) return;
  // The loads of the first kParts partials go out together (one L2 round
  // trip), then they are combined; a segment split more ways takes the rest
  // one by one.
  constexpr int kParts = 4;
  const int nparts = info.y - info.x + 1;
  float lse[kParts];
  float4 v[kParts];
#pragma unroll
  for (int k = 0; k < kParts; ++k) {
    lse[k] = -INFINITY;
    v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (k < nparts) {
      const int64_t slot = partial_slot(info.x + k, s);
      lse[k] = __ldcg(a.ws.part_lse + slot * hq + i);
      v[k] = __ldcg(reinterpret_cast<const float4*>(a.ws.part_o + (slot * hq + i) * D + c4));
    }
  }
  float m = lse[0];
#pragma unroll
  for (int k = 1; k < kParts; ++k) m = fmaxf(m, lse[k]);
  float wsum = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int k = 0; k < kParts; ++k) {
    const float w = exp2f(lse[k] - m);   // 0 for the absent parts (lse = -inf)
    acc.x += w * v[k].x;
    acc.y += w * v[k].y;
    acc.z += w * v[k].z;
    acc.w += w * v[k].w;
    wsum += w;
  }
  for (int k = info.x + kParts; k <= info.y; ++k) {
    const int64_t slot = partial_slot(k, s);
    const float l = __ldcg(a.ws.part_lse + slot * hq + i);
    const float4 u = __ldcg(reinterpret_cast<const float4*>(a.ws.part_o + (slot * hq + i) * D + c4));
    const float mn = fmaxf(m, l);
    const float cold = exp2f(m - mn), cnew = exp2f(l - mn);
    acc.x = acc.x * cold + cnew * u.x;
    acc.y = acc.y * cold + cnew * u.y;
    acc.z = acc.z * cold + cnew * u.z;
    acc.w = acc.w * cold + cnew * u.w;
    wsum = wsum * cold + cnew;
    m = mn;
  }
  const float inv = 1.f / wsum;
  O[0] = from_f32<T>(acc.x * inv);
  O[1] = from_f32<T>(acc.y * inv);
  O[2] = from_f32<T>(acc.z * inv);
  O[3] = from_f32<T>(acc.w * inv);
}

// Beams sharing a prefix: output (sequence s, beam w, head j*hq+i) combines
// the partials of the prefix pass (segment s*g+j, query column w*hq+i of its
// W*hq) and of the suffix pass (segment (s*W+w)*g+j, column i) with the same
// log-sum-exp weights; either part may be empty.  One thread per four output
// columns of one head.
__global__ void __launch_bounds__(kMergeThreads) beam_combine_kernel(const BeamCombineArgs c, int heads_per_cta) {
  const int hq = c.hq, D = c.d, Whq = c.W * hq;
  const int chunks = (hq + heads_per_cta - 1) / heads_per_cta;
  const int64_t u = blockIdx.x / chunks;                      // (s, w, j)
  const int hc = int(blockIdx.x - u * chunks);
  const int tph = D / 4;
  const int i = hc * heads_per_cta + int(threadIdx.x) / tph;
  const int c4 = (int(threadIdx.x) % tph) * 4;
  const bool active = threadIdx.x < heads_per_cta * tph && i < hq;
  const int j = int(u % c.g);
  const int64_t sw = u / c.g;                                 // s * W + w
  const int s = int(sw / c.W), w = int(sw % c.W);
  // the lengths are inputs of the call, never written by the decodes before
  const int lp = active ? clamp_len(__ldg(c.plens + s), c.m_p, nullptr, false) : 0;
  const int ls = active ? clamp_len(__ldg(c.slens + sw), c.m_s, nullptr, false) : 0;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  if (!active) return;
  float m = -INFINITY, wsum = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  auto add = [&](float l, float4 v) {
    const float mn = fmaxf(m, l);
    const float cold = exp2f(m - mn), cnew = exp2f(l - mn);
    acc.x = acc.x * cold + cnew * v.x;
    acc.y = acc.y * cold + cnew * v.y;
    acc.z = acc.z * cold + cnew * v.z;
    acc.w = acc.w * cold + cnew * v.w;
    wsum = wsum * cold + cnew;
    m = mn;
  };
  if (lp > 0) {
    const int64_t seg = int64_t(s) * c.g + j;
    const int2 info = c.pre.seg_info[seg];
    for (int k = info.x; k <= info.y; ++k) {
      const int64_t col = partial_slot(k, seg) * Whq + w * hq + i;
      add(__ldcg(c.pre.part_lse + col), __ldcg(reinterpret_cast<const float4*>(c.pre.part_o + col * D + c4)));
    }
  }
  if (ls > 0) {
    const int64_t seg = sw * c.g + j;
    const int2 info = c.suf.seg_info[seg];
    for (int k = info.x; k <= info.y; ++k) {
      const int64_t col = partial_slot(k, seg) * hq + i;
      add(__ldcg(c.suf.part_lse + col), __ldcg(reinterpret_cast<const float4*>(c.suf.part_o + col * D + c4)));
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* O = static_cast<__nv_bfloat16*>(c.o) + (sw * c.h + int64_t(j) * hq + i) * D + c4;
  O[0] = __float2bfloat16_rn(acc.x * inv);
  O[1] = __float2bfloat16_rn(acc.y * inv);
  O[2] = __float2bfloat16_rn(acc.z * inv);
  O[3] = __float2bfloat16_rn(acc.w * inv);
}

}  // namespace

cudaError_t launch_beam_combine(const BeamCombineArgs& c, cudaStream_t stream) {
  const int heads_per_cta = kMergeThreads / (c.d / 4);
  const int64_t ctas = int64_t(c.b) * c.W * c.g * ((c.hq + heads_per_cta - 1) / heads_per_cta);
  if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(ctas));
  cfg.blockDim = dim3(kMergeThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, beam_combine_kernel, c, heads_per_cta);
}

cudaError_t launch_merge(const DecodeArgs& a, mqa_dtype_t dtype, cudaStream_t stream) {
  const int heads_per_cta = kMergeThreads / (a.d / 4);
  const int64_t ctas = int64_t(a.b) * a.g * ((a.hq + heads_per_cta - 1) / heads_per_cta);
  if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(ctas));
  cfg.blockDim = dim3(kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (dtype == MQA_BF16) return cudaLaunchKernelEx(&cfg, merge_kernel<__nv_bfloat16>, a, heads_per_cta);
  return cudaLaunchKernelEx(&cfg, merge_kernel<float>, a, heads_per_cta);
}

}  // namespace mqa
