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
//
// Beams sharing a prefix in one pass: a segment's query columns are its W
// beams' heads of the group (column w*hq_b + i is head i of beam w, written to
// output row s*W + w), and a sequence is empty only when its prefix and every
// suffix are.  A column with no rows in any partial (a beam with neither
// prefix nor suffix) has lse = -inf everywhere and gets a zero row.
#include "common.cuh"

namespace mqa {

namespace {

constexpr int kMergeThreads = 128;

// What the merge reads of a decode's arguments (a small parameter block).
struct MergeArgs {
  void* o;
  const int32_t* lens;
  const int32_t* slens;
  Workspace ws;
  int h, g, hq, d, m_max, q_beams, q_group_heads, m_s;
};

// One CTA per (segment, group of heads); each thread merges four consecutive
// output columns of one head, so the few partial loads of every output are
// issued by many threads at once instead of walked serially.
template <typename T, bool kBeams>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const MergeArgs a, int heads_per_cta) {
  const int hq = a.hq, D = a.d;
  const int chunks = (hq + heads_per_cta - 1) / heads_per_cta;
  const int64_t s = blockIdx.x / chunks;
  const int hc = int(blockIdx.x - s * chunks);
  const int tph = D / 4;                                    // threads per head
  const int i = hc * heads_per_cta + int(threadIdx.x) / tph;
  const int c4 = (int(threadIdx.x) % tph) * 4;
  const bool active = threadIdx.x < heads_per_cta * tph && i < hq;
  const int seq = int(s / a.g), head = int(s - int64_t(seq) * a.g);
  // The lengths are inputs of the call, never written by the decode kernel
  // this merge follows, so they are read before waiting for that kernel.
  int len = active ? clamp_len(__ldg(a.lens + seq), a.m_max, nullptr, false) : 0;
  if (kBeams && active)
    for (int w = 0; w < a.q_beams; ++w)
      len += clamp_len(__ldg(a.slens + int64_t(seq) * a.q_beams + w), a.m_s, nullptr, false);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // The next step's decode may launch and set up while the merge runs.
  asm volatile("griddepcontrol.launch_dependents;");
  if (!active) return;
  T* O;
  if constexpr (kBeams) {
    const int qgh = a.q_group_heads, bw = i / qgh, bi = i - bw * qgh;
    O = static_cast<T*>(a.o) + ((int64_t(seq) * a.q_beams + bw) * a.h + int64_t(head) * qgh + bi) * D + c4;
  } else {
    O = static_cast<T*>(a.o) + (int64_t(seq) * a.h + int64_t(head) * hq + i) * D + c4;
  }
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
    // 0 for the absent parts (lse = -inf); with beams also for parts without rows for the column
    const float w = kBeams && lse[k] == -INFINITY ? 0.f : exp2f(lse[k] - m);
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
    if (kBeams && l == -INFINITY) continue;   // a part without rows for this column
    const float mn = fmaxf(m, l);
    const float cold = kBeams && m == -INFINITY ? 0.f : exp2f(m - mn), cnew = exp2f(l - mn);
    acc.x = acc.x * cold + cnew * u.x;
    acc.y = acc.y * cold + cnew * u.y;
    acc.z = acc.z * cold + cnew * u.z;
    acc.w = acc.w * cold + cnew * u.w;
    wsum = wsum * cold + cnew;
    m = mn;
  }
  const float inv = kBeams ? (wsum > 0.f ? 1.f / wsum : 0.f) : 1.f / wsum;
  O[0] = from_f32<T>(acc.x * inv);
  O[1] = from_f32<T>(acc.y * inv);
  O[2] = from_f32<T>(acc.z * inv);
  O[3] = from_f32<T>(acc.w * inv);
}

}  // namespace

cudaError_t launch_merge(const DecodeArgs& da, mqa_dtype_t dtype, cudaStream_t stream) {
  MergeArgs a;
  a.o = da.o;
  a.lens = da.lens;
  a.slens = da.slens;
  a.ws = da.ws;
  a.h = da.h;
  a.g = da.g;
  a.hq = da.hq;
  a.d = da.d;
  a.m_max = da.m_max;
  a.q_beams = da.q_beams;
  a.q_group_heads = da.q_group_heads;
  a.m_s = da.m_s;
  const int b = da.b;
  const bool beams = da.sk != nullptr;
  const int heads_per_cta = kMergeThreads / (a.d / 4);
  const int64_t ctas = int64_t(b) * a.g * ((a.hq + heads_per_cta - 1) / heads_per_cta);
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
  if (beams) return cudaLaunchKernelEx(&cfg, merge_kernel<__nv_bfloat16, true>, a, heads_per_cta);
  if (dtype == MQA_BF16) return cudaLaunchKernelEx(&cfg, merge_kernel<__nv_bfloat16, false>, a, heads_per_cta);
  return cudaLaunchKernelEx(&cfg, merge_kernel<float, false>, a, heads_per_cta);
}

}  // namespace mqa
