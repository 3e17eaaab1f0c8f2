// Split-KV decode attention on CUDA cores (FFMA), for any element type and
// small query-head groups.
//
// Computation ("Fast Transformer Decoding", velog paper review §3 and §2.4):
// for each sequence b and K/V head j, the h/g query heads of the group attend
// over the rows t < L_b of that head's cache,
//   s_{i,t} = scale * q_i . K_t,  w = softmax_t(s),  o_i = sum_t w_{i,t} V_t.
// The logits never leave the SM: each tile of TILE rows is staged once in
// shared memory with cp.async (double buffered, 16-byte copies), every query
// head of the group reads it from there (the MQA point: one K/V read serves
// all heads of the group), and an online softmax keeps a running max m and sum
// l per head.  Exponentials are exp2 of log2(e)-prescaled logits.
//
// The arithmetic is h/g FLOP per cache byte in bf16, so this kernel keeps up
// with HBM only for small groups; bf16 with d = 128 is served by the
// tensor-core kernel, and this one takes fp32, head sizes 32 and 64, and keys
// and values of different widths (d_k for q and K, d_v for V and o), as the
// paper's per-head dimensions k and v allow (velog paper review §2.4, §3).
#include <atomic>
#include "common.cuh"

namespace mqa {

namespace {

constexpr int kThreads = 128;
constexpr int kTile = 64;
constexpr int kMaxOutPairs = 16;   // column pairs per thread: h/g * d <= 4096

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Shared memory: reduction scratch, q [hq][DK] fp32, logits [hq][kTile],
// m/l/alpha [hq], then two K stages of kTile rows of DK and two V stages of
// kTile rows of DV (K0 K1 V0 V1).
template <typename T, int DK, int DV>
struct SimtLayout {
  static constexpr int kRowBytesK = DK * int(sizeof(T)) + 16;   // +16: rows land on rotating banks
  static constexpr int kRowBytesV = DV * int(sizeof(T)) + 16;
  static constexpr int kChunksK = DK * int(sizeof(T)) / 16;     // 16-byte pieces per row
  static constexpr int kChunksV = DV * int(sizeof(T)) / 16;
  static constexpr int kStageK = kTile * kRowBytesK;
  static constexpr int kStageV = kTile * kRowBytesV;
  static constexpr int kRedBytes = ((kThreads / 32 + kThreads + 2) * 8 + 15) / 16 * 16;
  static __host__ __device__ size_t bytes(int hq) {
    return size_t(kRedBytes) + size_t(hq) * DK * 4 + size_t(hq) * kTile * 4 + (size_t(3 * hq) * 4 + 15) / 16 * 16 +
           size_t(2) * (kStageK + kStageV);
  }
};

// Stage `rows` rows of one cache (D elements each, row r at element
// (row_base + r*g) * D) at a pitch of kRowBytes; row `new_row`, if any, comes
// from `src_new` and is also written into the cache.
template <typename T, int D, int kRowBytes>
__device__ __forceinline__ void stage_rows(unsigned char* st, const T* __restrict__ C, int64_t row_base, int g,
                                           int rows, int new_row, const T* __restrict__ src_new) {
  constexpr int kChunks = D * int(sizeof(T)) / 16;
  const int n = rows * kChunks;
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const int r = i / kChunks, c = i - r * kChunks;
    const int64_t off = (row_base + int64_t(r) * g) * D;
    if (r == new_row) {
      const uint4 x = reinterpret_cast<const uint4*>(src_new)[c];
      reinterpret_cast<uint4*>(const_cast<T*>(C) + off)[c] = x;
      *reinterpret_cast<uint4*>(st + r * kRowBytes + c * 16) = x;
    } else {
      cp_async16(st + r * kRowBytes + c * 16, reinterpret_cast<const unsigned char*>(C + off) + c * 16);
    }
  }
}

// Stage the valid rows of a tile.  With the fused append (knew != nullptr)
// the sequence's last tile holds its newest row: that row is taken from
// knew/vnew, written into the cache and into the stage directly.
template <typename T, int DK, int DV>
__device__ __forceinline__ void load_tile(unsigned char* ks, unsigned char* vs, const T* __restrict__ K,
                                          const T* __restrict__ V, const TileCoord& tc, int g, int m_max,
                                          const T* __restrict__ knew, const T* __restrict__ vnew) {
  using L = SimtLayout<T, DK, DV>;
  const int64_t row_base = (int64_t(tc.seq) * m_max + tc.row0) * g + tc.head;
  const int new_row = (knew != nullptr && tc.k == tc.nb - 1) ? tc.rows - 1 : -1;
  if constexpr (DK != DV) {
    const int64_t src = int64_t(tc.seq) * g + tc.head;   // row of k_new / v_new
    stage_rows<T, DK, L::kRowBytesK>(ks, K, row_base, g, tc.rows, new_row, knew ? knew + src * DK : nullptr);
    stage_rows<T, DV, L::kRowBytesV>(vs, V, row_base, g, tc.rows, new_row, vnew ? vnew + src * DV : nullptr);
  } else {
    constexpr int D = DK;   // equal widths: one pass stages a K and a V piece per index
    const int n = tc.rows * L::kChunksK;
    for (int i = threadIdx.x; i < n; i += kThreads) {
      const int r = i / L::kChunksK, c = i - r * L::kChunksK;
      const int64_t off = (row_base + int64_t(r) * g) * D;        // element offset of the row
      if (r == new_row) {
        const int64_t src = (int64_t(tc.seq) * g + tc.head) * D;
        const uint4 kv = reinterpret_cast<const uint4*>(knew + src)[c];
        const uint4 vv = reinterpret_cast<const uint4*>(vnew + src)[c];
        reinterpret_cast<uint4*>(const_cast<T*>(K) + off)[c] = kv;
        reinterpret_cast<uint4*>(const_cast<T*>(V) + off)[c] = vv;
        *reinterpret_cast<uint4*>(ks + r * L::kRowBytesK + c * 16) = kv;
        *reinterpret_cast<uint4*>(vs + r * L::kRowBytesV + c * 16) = vv;
      } else {
        cp_async16(ks + r * L::kRowBytesK + c * 16, reinterpret_cast<const unsigned char*>(K + off) + c * 16);
        cp_async16(vs + r * L::kRowBytesV + c * 16, reinterpret_cast<const unsigned char*>(V + off) + c * 16);
      }
    }
  }
}

// Dot product of a prescaled query (fp32, shared) with `n` elements of a staged
// row, 16 bytes at a time.
template <typename T>
__device__ __forceinline__ float dot_row(const float* __restrict__ q, const unsigned char* row, int e0, int n);

template <>
__device__ __forceinline__ float dot_row<__nv_bfloat16>(const float* __restrict__ q, const unsigned char* row,
                                                         int e0, int n) {
  float acc = 0.f;
  for (int e = e0; e < e0 + n; e += 8) {
    const uint4 w = *reinterpret_cast<const uint4*>(row + e * 2);
    const float4 qa = *reinterpret_cast<const float4*>(q + e);
    const float4 qb = *reinterpret_cast<const float4*>(q + e + 4);
    float2 k0 = bf16x2_to_f32x2(w.x), k1 = bf16x2_to_f32x2(w.y), k2 = bf16x2_to_f32x2(w.z),
           k3 = bf16x2_to_f32x2(w.w);
    acc = fmaf(qa.x, k0.x, acc);
    acc = fmaf(qa.y, k0.y, acc);
    acc = fmaf(qa.z, k1.x, acc);
    acc = fmaf(qa.w, k1.y, acc);
    acc = fmaf(qb.x, k2.x, acc);
    acc = fmaf(qb.y, k2.y, acc);
    acc = fmaf(qb.z, k3.x, acc);
    acc = fmaf(qb.w, k3.y, acc);
  }
  return acc;
}

template <>
__device__ __forceinline__ float dot_row<float>(const float* __restrict__ q, const unsigned char* row, int e0,
                                                int n) {
  float acc = 0.f;
  for (int e = e0; e < e0 + n; e += 4) {
    const float4 k = *reinterpret_cast<const float4*>(row + e * 4);
    const float4 qa = *reinterpret_cast<const float4*>(q + e);
    acc = fmaf(qa.x, k.x, acc);
    acc = fmaf(qa.y, k.y, acc);
    acc = fmaf(qa.z, k.z, acc);
    acc = fmaf(qa.w, k.w, acc);
  }
  return acc;
}

__device__ __forceinline__ float2 load_v_pair(const unsigned char* row, int c2, __nv_bfloat16*) {
  return bf16x2_to_f32x2(*reinterpret_cast<const uint32_t*>(row + c2 * 4));
}
__device__ __forceinline__ float2 load_v_pair(const unsigned char* row, int c2, float*) {
  return *reinterpret_cast<const float2*>(row + c2 * 8);
}

__device__ __forceinline__ void store_pair(__nv_bfloat16* p, float2 v) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v.x, v.y);
}
__device__ __forceinline__ void store_pair(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kThreads) decode_simt_kernel(const DecodeArgs a) {
  using L = SimtLayout<T, DK, DV>;
  extern __shared__ __align__(16) unsigned char smem[];
  int64_t* red = reinterpret_cast<int64_t*>(smem);
  float* q_s = reinterpret_cast<float*>(smem + L::kRedBytes);
  float* p_s = q_s + a.hq * DK;
  float* m_s = p_s + a.hq * kTile;
  float* l_s = m_s + a.hq;
  float* al_s = l_s + a.hq;
  unsigned char* stage = reinterpret_cast<unsigned char*>(m_s) + (size_t(3 * a.hq) * 4 + 15) / 16 * 16;
  // stage s: K at stage + s*kStageK, V at stage + 2*kStageK + s*kStageV
  unsigned char* const kst = stage;
  unsigned char* const vst = stage + 2 * L::kStageK;

  const T* __restrict__ Q = static_cast<const T*>(a.q);
  const T* __restrict__ K = static_cast<const T*>(a.k);
  const T* __restrict__ V = static_cast<const T*>(a.v);
  const T* __restrict__ KN = static_cast<const T*>(a.k_new);
  const T* __restrict__ VN = static_cast<const T*>(a.v_new);
  T* __restrict__ O = static_cast<T*>(a.o);
  const int hq = a.hq, g = a.g;
  const float qscale = a.scale * kLog2e;

  // Inputs may come from the kernel before this one on the stream (the append).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const Sched sc = make_schedule<kThreads>(a.lens, a.b, g, a.m_max, a.window, kTile, a.grid, blockIdx.x, a.flags, red);
  if (a.no_merge) {   // no merge follows: empty sequences get their zero rows here
    for (int s = blockIdx.x; s < a.b; s += gridDim.x) {
      if (clamp_len(__ldg(a.lens + s), a.m_max, nullptr, false) == 0) {
        T* o = static_cast<T*>(a.o) + int64_t(s) * a.h * DV;
        for (int k = threadIdx.x; k < a.h * DV; k += kThreads) o[k] = from_f32<T>(0.f);
      }
    }
  }
  if (sc.t_begin >= sc.t_end) {
    asm volatile("griddepcontrol.launch_dependents;");
    return;
  }

  Cursor cur = cursor_at(a.lens, a.m_max, a.window, kTile, sc.seq, sc.seq_base);
  Cursor nxt = cur;
  cursor_seek(cur, a.lens, g, a.m_max, a.window, kTile, sc.t_begin);
  {
    const TileCoord t0 = tile_coord(cur, g, kTile, sc.t_begin);
    load_tile<T, DK, DV>(kst, vst, K, V, t0, g, a.m_max, KN, VN);
    cp_async_commit();
  }

  const int pairs_out = hq * (DV / 2);
  float2 acc[kMaxOutPairs];
#pragma unroll
  for (int r = 0; r < kMaxOutPairs; ++r) acc[r] = make_float2(0.f, 0.f);

  const int lg_pairs = hq * kTile;
  const int split = lg_pairs < kThreads ? kThreads / lg_pairs : 1;   // threads per (head, row)
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  for (int64_t t = sc.t_begin; t < sc.t_end; ++t) {
    const int st = int((t - sc.t_begin) & 1);
    cursor_seek(cur, a.lens, g, a.m_max, a.window, kTile, t);
    const TileCoord tc = tile_coord(cur, g, kTile, t);

    if (t == sc.t_begin || tc.k == 0) {   // a new segment starts: its queries, fresh state
      const T* qg = Q + (int64_t(tc.seq) * a.h + int64_t(tc.head) * hq) * DK;
      for (int i = threadIdx.x; i < hq * DK; i += kThreads) q_s[i] = to_f32(qg[i]) * qscale;
      for (int i = threadIdx.x; i < hq; i += kThreads) {
        m_s[i] = -INFINITY;
        l_s[i] = 0.f;
      }
#pragma unroll
      for (int r = 0; r < kMaxOutPairs; ++r) acc[r] = make_float2(0.f, 0.f);
    }
    if (t + 1 < sc.t_end) {
      cursor_seek(nxt, a.lens, g, a.m_max, a.window, kTile, t + 1);
      const TileCoord tn = tile_coord(nxt, g, kTile, t + 1);
      load_tile<T, DK, DV>(kst + (st ^ 1) * L::kStageK, vst + (st ^ 1) * L::kStageV, K, V, tn, g, a.m_max, KN,
                           VN);
    }
    cp_async_commit();
    cp_async_wait1();
    __syncthreads();

    // logits, prescaled by scale*log2(e); rows past the valid count are -inf
    for (int p = threadIdx.x / split; p < lg_pairs; p += kThreads / split) {
      const int i = p / kTile, r = p - i * kTile;
      const int part = threadIdx.x % split;
      float s = 0.f;
      if (r < tc.rows)
        s = dot_row<T>(q_s + i * DK, kst + st * L::kStageK + r * L::kRowBytesK, part * (DK / split), DK / split);
      for (int o = split / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (part == 0) p_s[i * kTile + r] = r < tc.rows ? s : -INFINITY;
    }
    __syncthreads();

    // online softmax, one warp per head
    for (int i = warp; i < hq; i += kThreads / 32) {
      const float s0 = p_s[i * kTile + lane], s1 = p_s[i * kTile + lane + 32];
      float mx = fmaxf(s0, s1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = m_s[i];
      const float m_new = fmaxf(m_old, mx);
      const float p0 = exp2f(s0 - m_new), p1 = exp2f(s1 - m_new);
      p_s[i * kTile + lane] = p0;
      p_s[i * kTile + lane + 32] = p1;
      float sum = p0 + p1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        const float alpha = exp2f(m_old - m_new);
        al_s[i] = alpha;
        l_s[i] = l_s[i] * alpha + sum;
        m_s[i] = m_new;
      }
    }
    __syncthreads();

    // weighted V: thread owns column pairs (head i, columns 2c2, 2c2+1)
#pragma unroll
    for (int r = 0; r < kMaxOutPairs; ++r) {
      const int f = threadIdx.x + r * kThreads;
      if (f < pairs_out) {
        const int i = f / (DV / 2), c2 = f - i * (DV / 2);
        const float alpha = al_s[i];
        float2 o2 = make_float2(acc[r].x * alpha, acc[r].y * alpha);
        const float* pw = p_s + i * kTile;
        const unsigned char* vrow = vst + st * L::kStageV;
        for (int row = 0; row < tc.rows; ++row) {
          const float w = pw[row];
          const float2 v = load_v_pair(vrow + row * L::kRowBytesV, c2, static_cast<T*>(nullptr));
          o2.x = fmaf(w, v.x, o2.x);
          o2.y = fmaf(w, v.y, o2.y);
        }
        acc[r] = o2;
      }
    }

    const bool seg_last = (tc.k == tc.nb - 1) || (t + 1 == sc.t_end);
    if (seg_last) {
      const bool owns_first = tc.seg_t0 >= sc.t_begin;
      const bool whole = owns_first && (tc.seg_t0 + tc.nb <= sc.t_end);
      const int64_t slot = partial_slot(blockIdx.x, tc.seg);
#pragma unroll
      for (int r = 0; r < kMaxOutPairs; ++r) {
        const int f = threadIdx.x + r * kThreads;
        if (f < pairs_out) {
          const int i = f / (DV / 2), c2 = f - i * (DV / 2);
          const float inv = 1.f / l_s[i];
          const float2 v = make_float2(acc[r].x * inv, acc[r].y * inv);
          if (whole) {
            store_pair(O + (int64_t(tc.seq) * a.h + int64_t(tc.head) * hq + i) * DV + 2 * c2, v);
          } else {
            *reinterpret_cast<float2*>(a.ws.part_o + (slot * hq + i) * DV + 2 * c2) = v;
          }
        }
      }
      if (!whole)
        for (int i = threadIdx.x; i < hq; i += kThreads) a.ws.part_lse[slot * hq + i] = m_s[i] + log2f(l_s[i]);
      if (owns_first && threadIdx.x == 0)
        a.ws.seg_info[tc.seg] =
            make_int2(blockIdx.x, cta_of_tile(tc.seg_t0 + tc.nb - 1, sc.total, sc.active));
    }
    __syncthreads();
  }
  asm volatile("griddepcontrol.launch_dependents;");
}

// Opt the kernel into large dynamic shared memory once per device.
template <typename T, int DK, int DV>
cudaError_t ensure_smem_attr() {
  static std::atomic<bool> done[64];   // per device; any thread may set it (the call is idempotent)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(decode_simt_kernel<T, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev].store(true, std::memory_order_relaxed);
  return e;
}

template <typename T, int DK, int DV>
cudaError_t launch_t(const DecodeArgs& a, cudaStream_t stream) {
  const size_t smem = SimtLayout<T, DK, DV>::bytes(a.hq);
  cudaError_t e = ensure_smem_attr<T, DK, DV>();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(a.grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_simt_kernel<T, DK, DV>, a);
}

// Resident CTAs per SM for this shared-memory size, cached per (device, h/g).
template <typename T, int DK, int DV>
int occupancy_t(int hq) {
  static std::atomic<int> cache[64][129];   // 0 = not yet known; every thread computes the same value
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  const bool cacheable = dev >= 0 && dev < 64 && hq >= 1 && hq <= 128;
  if (cacheable) {
    const int c = cache[dev][hq].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  const size_t smem = SimtLayout<T, DK, DV>::bytes(hq);
  if (ensure_smem_attr<T, DK, DV>() != cudaSuccess) return 1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_simt_kernel<T, DK, DV>, kThreads, smem) !=
          cudaSuccess ||
      n < 1)
    n = 1;
  if (cacheable) cache[dev][hq].store(n, std::memory_order_relaxed);
  return n;
}

// The built widths: d_k, d_v in {32, 64, 128}, any pairing.
template <typename T, int DK>
cudaError_t launch_dk(const DecodeArgs& a, int d_v, cudaStream_t stream) {
  switch (d_v) {
    case 32: return launch_t<T, DK, 32>(a, stream);
    case 64: return launch_t<T, DK, 64>(a, stream);
    case 128: return launch_t<T, DK, 128>(a, stream);
  }
  return cudaErrorInvalidValue;
}
template <typename T>
cudaError_t launch_typed(const DecodeArgs& a, int d_k, int d_v, cudaStream_t stream) {
  switch (d_k) {
    case 32: return launch_dk<T, 32>(a, d_v, stream);
    case 64: return launch_dk<T, 64>(a, d_v, stream);
    case 128: return launch_dk<T, 128>(a, d_v, stream);
  }
  return cudaErrorInvalidValue;
}

template <typename T, int DK>
int occupancy_dk(int d_v, int hq) {
  switch (d_v) {
    case 32: return occupancy_t<T, DK, 32>(hq);
    case 64: return occupancy_t<T, DK, 64>(hq);
    case 128: return occupancy_t<T, DK, 128>(hq);
  }
  return 1;
}
template <typename T>
int occupancy_typed(int d_k, int d_v, int hq) {
  switch (d_k) {
    case 32: return occupancy_dk<T, 32>(d_v, hq);
    case 64: return occupancy_dk<T, 64>(d_v, hq);
    case 128: return occupancy_dk<T, 128>(d_v, hq);
  }
  return 1;
}

}  // namespace

cudaError_t launch_decode_simt(const DecodeArgs& a, int d_k, mqa_dtype_t dtype, cudaStream_t stream) {
  return dtype == MQA_BF16 ? launch_typed<__nv_bfloat16>(a, d_k, a.d, stream) : launch_typed<float>(a, d_k, a.d, stream);
}

int simt_tile_rows() { return kTile; }

int simt_ctas_per_sm(mqa_dtype_t dtype, int d_k, int d_v, int hq) {
  return dtype == MQA_BF16 ? occupancy_typed<__nv_bfloat16>(d_k, d_v, hq) : occupancy_typed<float>(d_k, d_v, hq);
}

}  // namespace mqa
