// Batched (prefill) MQA / GQA attention on the 5th-generation tensor cores.
//
// Computation (paper review of "Fast Transformer Decoding", §2.3 batched
// attention and §3 multi-query attention; study notes §1 and §10): every
// position t of a sequence attends to the keys of the same sequence, under a
// causal mask (keys 0..t) or none, with the h/g query heads of a group sharing
// one K/V head.  Sequences are packed: q, o [T, h, d]; k, v [T, g, d]; rows
// cu_seqlens[s] .. cu_seqlens[s+1]-1 belong to sequence s.
//
// A CTA takes one 128-row query tile of one (sequence, K/V group): rows are
// (position, head) pairs, 128 / (h/g) positions times the h/g heads of the
// group, so every K/V tile it loads feeds all heads of the group (the MQA
// saving, here in the reuse of each staged tile).  Per 64-key tile:
//   S = Q K^T      M = 128 rows, N = 64 keys, K = d = 128    (tensor memory)
//   O += P V       M = 128 rows, N = d = 128, K = 64 keys    (tensor memory)
// Two CTAs share each SM (112 KB of shared memory and 256 tensor-memory
// columns each): a tile's chain of product, softmax and product costs about
// the same at 64 keys as at 128, so two independent chains per SM do more.
// One softmax thread per row holds the tile's 64 logits in registers; its
// reference max is moved only when a logit exceeds it by more than 8 (log2
// units), and only then is its row of O rescaled in tensor memory.
//
// Roles: warp 0 lane 0 loads Q and the K ring, warp 6 lane 0 the V ring (a
// warp of its own), warp 1 lane 0 issues the products, warps 2-5 are the
// softmax and epilogue (one row per thread).  Tensor-memory loads and stores
// are warp-collective (.sync.aligned), so every decision that guards one is
// made per warp: a lane whose row needs nothing runs them all the same.
// Every wait is bounded (one second); on expiry the kernel sets
// MQA_FLAG_PIPE_TIMEOUT and returns.
//
// Query tiles are launched longest first (the causal tiles near the end of a
// sequence carry the most keys), one CTA each.
#include <atomic>
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace mqa {

namespace {

using namespace sm100;

constexpr int kRows = 128;                     // query rows per tile (the MMA M)
constexpr int kKeys = 64;                      // keys per K/V tile
constexpr int kD = 128;                        // head size
constexpr int kSK = 2, kSV = 2;                // K and V ring stages
constexpr int kThreads = 224;                  // 7 warps
constexpr int kCtasPerSm = 2;                  // two query tiles' pipelines share each SM
constexpr int kVWarp = 6;
constexpr uint32_t kHalf = kRows * 128;        // one 64-column half of the 128-row Q tile
constexpr uint32_t kHalfKV = kKeys * 128;      // one 64-column half of a K or V tile
constexpr uint32_t kQBytes = 2 * kHalf, kKVBytes = 2 * kHalfKV;
constexpr uint32_t kPBytes = kRows * kKeys * 2;   // 128 rows x 64 keys (bf16): one 128-byte swizzle column
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr float kRescaleThreshold = 8.f;       // log2 units
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kTmemCols = 256;            // S double buffer at [0, 128), O at [128, 256)
constexpr uint32_t kOCol = 2 * kKeys;

struct Cfg {
  // barriers
  static constexpr int kQFull = 0, kKFull = 1, kKEmpty = kKFull + kSK, kVFull = kKEmpty + kSK,
                       kVEmpty = kVFull + kSV, kSFull = kVEmpty + kSV, kPFull = kSFull + 2, kOFull = kPFull + 1,
                       kDone = kOFull + 1, kNumBars = kDone + 1;
  // shared memory (1024-byte aligned base)
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kQBytes;
  static constexpr uint32_t kV = kK + kSK * kKVBytes;
  static constexpr uint32_t kP = kV + kSV * kKVBytes;
  static constexpr uint32_t kBar = kP + kPBytes;
  static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
  static constexpr uint32_t kAbort = kTmemSlot + 4;
  static constexpr uint32_t kEnd = kAbort + 4;
  // No room to align the base at run time: two CTAs per SM leave each at most
  // (228 KB - 2 x 1 KB reserved) / 2.  The kernel checks that the base it gets
  // is 1024-byte aligned and refuses to run otherwise.
  static constexpr uint32_t kAlloc = kEnd;
  static_assert(kK % 1024 == 0 && kV % 1024 == 0 && kP % 1024 == 0, "swizzle atoms need 1024-byte alignment");
  static_assert(kAlloc <= (233472 - kCtasPerSm * 1024) / kCtasPerSm, "shared memory budget for two CTAs per SM");
};

struct PrefillArgs {
  void* o;
  const int32_t* cu;     // [b+1] cumulative sequence lengths
  int b, h, g, hq;
  int total, max_seqlen; // rows of the packed arrays; longest sequence the grid covers
  int causal;
  float scale;
  int32_t* flags;
};

__device__ __forceinline__ void set_timeout(volatile int* abort, int32_t* flags) {
  *abort = 1;
  if (flags != nullptr) atomicOr(flags, MQA_FLAG_PIPE_TIMEOUT);
}

__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    prefill_tc_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  using C = Cfg;
  const int seq = blockIdx.x, grp = blockIdx.y;
  const int per = kRows / a.hq;                                        // positions per tile
  const int qb = int(gridDim.z) - 1 - int(blockIdx.z);                 // longest tiles first
  // The lengths are read on the device: a sequence is cut to max_seqlen and to
  // the end of the packed arrays (flagged), so no row outside them is touched.
  const int tok0 = __ldg(a.cu + seq);
  int n = __ldg(a.cu + seq + 1) - tok0;
  if (tok0 < 0 || tok0 > a.total || n < 0) n = 0;
  if (n > a.max_seqlen || tok0 + n > a.total) {
    n = min(a.max_seqlen, a.total - tok0);
    if (a.flags != nullptr && qb == 0 && threadIdx.x == 0) atomicOr(a.flags, MQA_FLAG_LEN_CLAMPED);
  }
  const int p0 = qb * per;
  if (p0 >= n) return;                                                 // the whole CTA leaves together
  const int pos_last = min(p0 + per, n) - 1;
  const int nk = a.causal ? pos_last / kKeys + 1 : (n + kKeys - 1) / kKeys;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  if (raw & 1023u) {   // the swizzled tiles need a 1024-byte aligned base (uniform across the CTA)
    if (a.flags != nullptr && threadIdx.x == 0) atomicOr(a.flags, MQA_FLAG_PIPE_TIMEOUT);
    return;
  }
  unsigned char* smem = smem_raw;
  const uint32_t sbase = raw;
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kAbort);
  auto bar = [&](int id) { return sbase + C::kBar + 8u * id; };
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(bar(C::kQFull), 1);
    for (int s = 0; s < kSK; ++s) {
      mbar_init(bar(C::kKFull + s), 1);
      mbar_init(bar(C::kKEmpty + s), 1);
    }
    for (int s = 0; s < kSV; ++s) {
      mbar_init(bar(C::kVFull + s), 1);
      mbar_init(bar(C::kVEmpty + s), 1);
    }
    mbar_init(bar(C::kSFull), 1);
    mbar_init(bar(C::kSFull + 1), 1);
    mbar_init(bar(C::kPFull), kRows);
    mbar_init(bar(C::kOFull), 1);
    mbar_init(bar(C::kDone), 1);
    *abort = 0;
    mbar_fence_init();
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(sbase + C::kTmemSlot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + C::kTmemSlot);

  if (warp == 0 || warp == kVWarp) {
    // ---------------------------------------------------------- producers
    if (lane == 0) {
      const bool is_k = warp == 0;
      const uint64_t pol = l2_evict_last_policy();   // K/V tiles are read again by the sequence's other tiles
      if (is_k) {
        mbar_expect_tx(bar(C::kQFull), kQBytes);
        tma_load_3d(sbase + C::kQ, &tm_q, bar(C::kQFull), 0, grp * a.hq, tok0 + p0, l2_evict_first_policy());
        tma_load_3d(sbase + C::kQ + kHalf, &tm_q, bar(C::kQFull), 64, grp * a.hq, tok0 + p0,
                    l2_evict_first_policy());
      }
      const int S = is_k ? kSK : kSV;
      const int full = is_k ? C::kKFull : C::kVFull, empty = is_k ? C::kKEmpty : C::kVEmpty;
      const uint32_t ring = is_k ? C::kK : C::kV;
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      int k = 0;
      for (; k < nk; ++k) {
        const int st = k % S;
        if (k >= S && !mbar_wait(bar(empty + st), uint32_t(k / S - 1) & 1, kTimeoutNs)) {
          set_timeout(abort, a.flags);
          break;
        }
        if (*abort) break;
        const uint32_t dst = sbase + ring + st * kKVBytes;
        mbar_expect_tx(bar(full + st), kKVBytes);
        tma_load_3d(dst, map, bar(full + st), 0, grp, tok0 + k * kKeys, pol);
        tma_load_3d(dst + kHalfKV, map, bar(full + st), 64, grp, tok0 + k * kKeys, pol);
      }
      // every copy issued has landed before the CTA may exit
      for (int j = (k - S > 0 ? k - S : 0); j < k; ++j) mbar_wait(bar(full + j % S), uint32_t(j / S) & 1, kTimeoutNs);
      if (is_k) mbar_wait(bar(C::kQFull), 0, kTimeoutNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kRows, kKeys, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kRows, kD, 0, 1);
      const uint64_t qdesc = smem_desc_sw128(sbase + C::kQ, 16, 1024);        // K-major Q
      const uint64_t kdesc0 = smem_desc_sw128(sbase + C::kK, 16, 1024);       // K-major K (N = keys)
      const uint64_t pdesc = smem_desc_sw128(sbase + C::kP, 16, 1024);        // K-major P (K = keys)
      const uint64_t vdesc0 = smem_desc_sw128(sbase + C::kV, kHalfKV, 1024);  // MN-major V (N = d)
      int iq = 0, ip = 0;
      bool q_ready = false;
      uint32_t idle = 0;
      uint64_t idle_since = 0;
      while (ip < nk) {
        bool progressed = false;
        if (iq < nk && iq <= ip + 1) {   // S buffer iq&1 is free once P(iq-2) has been consumed
          const int st = iq % kSK;
          if (!q_ready) q_ready = mbar_test(bar(C::kQFull), 0);
          if (q_ready && mbar_test(bar(C::kKFull + st), uint32_t(iq / kSK) & 1)) {
            tc_fence_after();
            const uint64_t ka = kdesc0 + ((st * kKVBytes) >> 4);
            const uint32_t d = tmem + uint32_t(iq & 1) * kKeys;
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
              const uint32_t qoff = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
              const uint32_t koff = ((kk >> 2) * kHalfKV + (kk & 3) * 32) >> 4;
              mma_bf16_ss(d, qdesc + qoff, ka + koff, idesc_qk, kk > 0);
            }
            mma_commit(bar(C::kSFull + (iq & 1)));
            mma_commit(bar(C::kKEmpty + st));
            ++iq;
            progressed = true;
          }
        }
        if (ip < iq) {
          const int st = ip % kSV;
          if (mbar_test(bar(C::kPFull), uint32_t(ip & 1)) &&
              mbar_test(bar(C::kVFull + st), uint32_t(ip / kSV) & 1)) {
            tc_fence_after();
            const uint64_t va = vdesc0 + ((st * kKVBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < kKeys / 16; ++kk) {
              const uint32_t poff = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;   // one 64-key column: kk < 4
              mma_bf16_ss(tmem + kOCol, pdesc + poff, va + ((kk * 2048) >> 4), idesc_pv, (ip > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(bar(C::kOFull));
            mma_commit(bar(C::kVEmpty + st));
            ++ip;
            progressed = true;
          }
        }
        if (progressed) {
          idle = 0;
        } else if ((++idle & 1023u) == 0) {
          const uint64_t now = globaltimer_ns();
          if (idle == 1024) {
            idle_since = now;
          } else if (now - idle_since > kTimeoutNs || *abort) {
            set_timeout(abort, a.flags);
            break;
          }
        }
      }
      mma_commit(bar(C::kDone));
      mbar_wait(bar(C::kDone), 0, kTimeoutNs);
    }
  } else {
    // ---------------------------------------------------------- softmax and epilogue, one row per thread
    const int q4 = warp & 3;
    const int row = 32 * q4 + lane;
    const uint32_t t_lane = tmem + (uint32_t(32 * q4) << 16);
    const int pos = p0 + row / a.hq;                 // position of this row in its sequence
    const int head = grp * a.hq + row % a.hq;
    const bool row_valid = pos < n;
    const int key_end = a.causal ? min(pos + 1, n) : n;   // keys [0, key_end) are attended
    const float c = a.scale * kLog2e;
    float m_ref = 0.f, l = 0.f;
    bool failed = false;
    unsigned char* prow = smem + C::kP + (row >> 3) * 1024 + (row & 7) * 128;
    for (int k = 0; k < nk; ++k) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar(C::kSFull + (k & 1)), uint32_t(k >> 1) & 1, kTimeoutNs))) {
        failed = true;   // the whole warp leaves: its tensor-memory accesses stay collective
        break;
      }
      tc_fence_after();
      float s[kKeys];
#pragma unroll
      for (int ch = 0; ch < kKeys / 32; ++ch) {
        float w[32];
        tmem_ld32(t_lane + uint32_t(k & 1) * kKeys + ch * 32, w);
#pragma unroll
        for (int x = 0; x < 32; ++x) s[ch * 32 + x] = w[x] * c;
      }
      const int kb = k * kKeys;
      if (kb + kKeys > key_end) {   // this tile reaches past the row's last key
#pragma unroll
        for (int x = 0; x < kKeys; ++x)
          if (kb + x >= key_end) s[x] = -INFINITY;
      }
      float mt = s[0];
#pragma unroll
      for (int x = 1; x < kKeys; ++x) mt = fmaxf(mt, s[x]);
      float alpha = 1.f;
      bool rescale = false;
      if (k == 0) {
        m_ref = mt == -INFINITY ? 0.f : mt;
      } else if (mt > m_ref + kRescaleThreshold) {
        alpha = ex2_approx(m_ref - mt);
        m_ref = mt;
        l *= alpha;
        rescale = true;
      }
      // P(k) overwrites the P buffer and O may be rescaled: P.V(k-1) must be done
      if (k > 0 && !__all_sync(0xffffffffu, mbar_wait(bar(C::kOFull), uint32_t(k - 1) & 1, kTimeoutNs))) {
        failed = true;
        break;
      }
      tc_fence_after();
      if (__any_sync(0xffffffffu, rescale)) {   // collective for the warp; alpha = 1 in rows that keep their max
#pragma unroll
        for (int ch = 0; ch < kD / 32; ++ch) {
          float w[32];
          tmem_ld32(t_lane + kOCol + ch * 32, w);
#pragma unroll
          for (int x = 0; x < 32; ++x) w[x] *= alpha;
          float w0[16], w1[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            w0[x] = w[x];
            w1[x] = w[16 + x];
          }
          tmem_st16(t_lane + kOCol + ch * 32, w0);
          tmem_st16(t_lane + kOCol + ch * 32 + 16, w1);
        }
        tmem_wait_st();
      }
      // P = exp2(s - m_ref) in bf16, K-major with the 128-byte swizzle
#pragma unroll
      for (int ch = 0; ch < kKeys / 8; ++ch) {
        uint32_t packed[4];
#pragma unroll
        for (int x2 = 0; x2 < 4; ++x2) {
          const float e0 = ex2_approx(s[ch * 8 + 2 * x2] - m_ref);
          const float e1 = ex2_approx(s[ch * 8 + 2 * x2 + 1] - m_ref);
          __nv_bfloat162 b2 = __floats2bfloat162_rn(e0, e1);
          const float2 rounded = __bfloat1622float2(b2);   // the sum uses the P the product sees
          l += rounded.x + rounded.y;
          packed[x2] = *reinterpret_cast<uint32_t*>(&b2);
        }
        const int half = ch >> 3, c16 = ch & 7;
        *reinterpret_cast<uint4*>(prow + half * kHalf + ((c16 ^ (row & 7)) << 4)) =
            make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(C::kPFull));
    }
    if (!failed && !__all_sync(0xffffffffu, mbar_wait(bar(C::kOFull), uint32_t(nk - 1) & 1, kTimeoutNs)))
      failed = true;
    if (!failed) {
      tc_fence_after();
      // every lane loads its row of O (collective); rows past the sequence are not stored
      const float inv = l > 0.f ? rcp_approx(l) : 0.f;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) +
                                            (int64_t(tok0 + (row_valid ? pos : 0)) * a.h + head) * kD);
#pragma unroll
      for (int ch = 0; ch < kD / 32; ++ch) {
        float w[32];
        tmem_ld32(t_lane + kOCol + ch * 32, w);
#pragma unroll
        for (int x8 = 0; x8 < 4; ++x8) {
          uint32_t packed[4];
#pragma unroll
          for (int x2 = 0; x2 < 4; ++x2) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(w[x8 * 8 + 2 * x2] * inv, w[x8 * 8 + 2 * x2 + 1] * inv);
            packed[x2] = *reinterpret_cast<uint32_t*>(&b2);
          }
          if (row_valid) dst[ch * 4 + x8] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
      }
    } else {
      set_timeout(abort, a.flags);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ host

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Rows of `heads` heads of d bf16 each, one row per token: map (d, heads, T),
// box (64, box_heads, box_tokens), 128-byte swizzle.
bool encode_rows(CUtensorMap* m, const void* base, int64_t tokens, int heads, int box_heads, int box_tokens) {
  const cuuint64_t dims[3] = {cuuint64_t(kD), cuuint64_t(heads), cuuint64_t(tokens)};
  const cuuint64_t strides[2] = {cuuint64_t(kD) * 2, cuuint64_t(heads) * kD * 2};
  const cuuint32_t box[3] = {64, cuuint32_t(box_heads), cuuint32_t(box_tokens)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool prefill_tc_supported(int d, int hq) { return d == kD && hq >= 1 && hq <= kRows && kRows % hq == 0; }

cudaError_t launch_prefill_tc(void* o, const void* q, const void* k, const void* v, const int32_t* cu, int b,
                              int64_t total, int h, int g, int max_seqlen, float scale, int causal, int32_t* flags,
                              cudaStream_t stream) {
  const int hq = h / g;
  if (!prefill_tc_supported(kD, hq) || total >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  static std::atomic<bool> attr_set[64];   // per device; setting it twice is harmless
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_relaxed)) {
    e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(Cfg::kAlloc));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_relaxed);
  }
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  CUtensorMap tq, tk, tv;
  const int per = kRows / hq;
  if (!encode_rows(&tq, q, total, h, hq, per) || !encode_rows(&tk, k, total, g, 1, kKeys) ||
      !encode_rows(&tv, v, total, g, 1, kKeys))
    return cudaErrorInvalidValue;
  PrefillArgs a;
  a.o = o;
  a.cu = cu;
  a.b = b;
  a.h = h;
  a.g = g;
  a.hq = hq;
  a.causal = causal;
  a.scale = scale;
  a.total = int(total);
  a.max_seqlen = max_seqlen;
  a.flags = flags;
  const int64_t tiles = (int64_t(max_seqlen) + per - 1) / per;
  if (tiles > 65535 || b > 0x7fffffff || g > 65535) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(b), static_cast<unsigned>(g), static_cast<unsigned>(tiles));
  prefill_tc_kernel<<<grid, kThreads, Cfg::kAlloc, stream>>>(a, tq, tk, tv);
  return cudaGetLastError();
}

}  // namespace mqa
