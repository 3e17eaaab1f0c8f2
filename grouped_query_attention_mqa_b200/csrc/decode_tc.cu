// Split-KV decode attention on the 5th-generation tensor cores (tcgen05),
// for bf16 caches with head size 128 and up to 64 query heads per K/V head.
//
// Computation ("Fast Transformer Decoding", velog paper review §3; GQA blog
// "第三站: GQA"): for sequence b and K/V head j the h/g query heads of the
// group attend over the rows t < L_b of that head's cache.  With h/g = 32 the
// two contractions are 32 FLOP per cache byte, more than CUDA cores can feed
// at HBM speed, so both run on tensor cores:
//
//   S^T[t, i] = K[t, :] . q_i        M = 128 cache rows, N = heads, K = 128
//   O^T[c, i] += sum_t V[t, c] P[t, i] M = 128 columns of V, N = 64, K = 128 rows
//
// Cache rows are the M dimension of both products, so a 128-row tile of K
// (and of V) is one MMA operand exactly as TMA lands it, and every query head
// of the group reads the same staged tile — the bandwidth saving MQA is for.
// S and O live in tensor memory; O accumulates over all tiles of a segment.
//
// Roles (one CTA per SM, persistent over an even share of all tiles):
//   warp 0, one thread  TMA producer: Q of each segment, K and V tiles into a
//                       two-stage ring (64 KB per stage), L2 evict-first.
//   warp 1, one thread  MMA issuer: S(i+1) = K Q^T while P(i) is being made,
//                       then O += V^T P(i); completions signalled with
//                       tcgen05.commit on mbarriers.
//   warps 2-5           softmax and epilogue, one cache row (then one output
//                       column) per thread: column maxima over the tile by a
//                       warp transpose-reduction, P = exp2(s - m) in bf16 to
//                       shared memory, per-head sums kept in registers.  The
//                       running max is only moved when a head's tile max
//                       exceeds it by more than 8 (a factor 256), so O in
//                       tensor memory rarely needs rescaling.
// Every wait is bounded (one second); on expiry the kernel sets
// MQA_FLAG_PIPE_TIMEOUT, drains its own copies and MMAs, frees its tensor
// memory and returns.
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace mqa {

namespace {

using namespace sm100;

constexpr int kTile = 128;                   // cache rows per tile (the MMA M)
constexpr int kD = 128;                      // head size
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr int kNpv = 64;                     // N of the P.V product (P padded with zero columns)
constexpr uint32_t kHalfBytes = kTile * 128; // 128 rows x 64 bf16, one 128-byte swizzle column
constexpr uint32_t kTileBytes = 2 * kHalfBytes;
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr float kRescaleThreshold = 8.f;     // log2 units
constexpr uint32_t kTmemCols = 256;          // S double buffer at [0, 2*NP), O double buffer at [128, 256)
constexpr uint32_t kOCol = 128;

enum Bar {
  B_KFULL = 0, B_VFULL = 2, B_KVEMPTY = 4, B_SFULL = 6, B_PFULL = 8, B_OFULL = 10, B_QFULL = 12, B_QEMPTY = 14,
  B_OFREE = 16, B_DONE = 18, B_COUNT = 19
};

template <int NP>
struct TcLayout {
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kStages * kTileBytes;
  static constexpr uint32_t kQ = kV + kStages * kTileBytes;
  static constexpr uint32_t kQBytes = NP * 256;                // two 64-column halves of NP rows
  static constexpr uint32_t kP = kQ + 2 * kQBytes;
  static constexpr uint32_t kPBytes = kTile * 128;             // 128 rows x 64 heads (bf16)
  static constexpr uint32_t kBar = kP + 2 * kPBytes;
  static constexpr uint32_t kTmemSlot = kBar + B_COUNT * 8;
  static constexpr uint32_t kFlag = kTmemSlot + 4;
  static constexpr uint32_t kAbort = kFlag + 4;
  static constexpr uint32_t kRed = (kAbort + 4 + 15) / 16 * 16;  // [4][64] f32
  static constexpr uint32_t kMref = kRed + 4 * 64 * 4;
  static constexpr uint32_t kAlpha = kMref + 64 * 4;
  static constexpr uint32_t kLsum = kAlpha + 64 * 4;
  static constexpr uint32_t kSched = kLsum + 64 * 4;
  static constexpr uint32_t kEnd = kSched + (kThreads / 32 + kThreads + 2) * 8;
  static constexpr uint32_t kAlloc = kEnd + 1024;             // room to align the base to 1024 bytes
  static_assert(kQ % 1024 == 0 && kP % 1024 == 0 && kQBytes % 1024 == 0, "swizzle atoms need 1024-byte alignment");
};

__device__ __forceinline__ void named_barrier_softmax() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// After a transpose-reduction over the 32 lanes, lane l holds the result for
// column (l % W) of the W columns that every lane contributed.
template <int W, bool kMax>
__device__ __forceinline__ float transpose_reduce(float (&v)[W], int lane) {
#pragma unroll
  for (int o = W / 2; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int k = 0; k < o; ++k) {
      const float send = upper ? v[k] : v[k + o];
      const float keep = upper ? v[k + o] : v[k];
      const float recv = __shfl_xor_sync(0xffffffffu, send, o);
      v[k] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  float r = v[0];
#pragma unroll
  for (int o = W; o < 32; o <<= 1) {
    const float other = __shfl_xor_sync(0xffffffffu, r, o);
    r = kMax ? fmaxf(r, other) : r + other;
  }
  return r;
}

struct Roles {
  uint32_t sbase;            // shared address of the aligned base
  unsigned char* smem;
  uint32_t tmem;
  volatile int* abort;
  int32_t* flags;
};

__device__ __forceinline__ bool wait_bar(const Roles& r, uint32_t bar, uint32_t parity) {
  if (mbar_wait(bar, parity, kTimeoutNs)) return true;
  *r.abort = 1;
  set_flag(r.flags, MQA_FLAG_PIPE_TIMEOUT);
  return false;
}

// Walks the CTA's tiles in order and tells each role what a tile is.
struct TileWalk {
  Cursor cu;
  int64_t t;
  int sidx;                  // segment number within this CTA
  TileCoord tc;
  bool first, last;
  __device__ TileWalk(const DecodeArgs& a, const Sched& sc) : t(sc.t_begin - 1), sidx(-1) {
    cu = cursor_at(a.lens, a.m_max, kTile, sc.seq, sc.seq_base);
  }
  __device__ void next(const DecodeArgs& a, const Sched& sc) {
    ++t;
    cursor_seek(cu, a.lens, a.g, a.m_max, kTile, t);
    tc = tile_coord(cu, a.g, kTile, t);
    first = (t == sc.t_begin) || tc.k == 0;
    last = (tc.k == tc.nb - 1) || (t + 1 == sc.t_end);
    if (first) ++sidx;
  }
};

template <int NP>
__device__ void producer(const DecodeArgs& a, const Sched& sc, const Roles& r, const CUtensorMap* tm_k,
                         const CUtensorMap* tm_v, const CUtensorMap* tm_q) {
  using L = TcLayout<NP>;
  auto bar = [&](int id) { return r.sbase + L::kBar + 8u * id; };
  const uint64_t pol = l2_evict_first_policy();
  TileWalk w(a, sc);
  const int64_t n = sc.t_end - sc.t_begin;
  int64_t i = 0;
  for (; i < n; ++i) {
    w.next(a, sc);
    if (*r.abort) break;
    if (w.first) {
      const int qb = w.sidx & 1;
      if (w.sidx >= 2 && !wait_bar(r, bar(B_QEMPTY + qb), ((w.sidx >> 1) - 1) & 1)) break;
      mbar_expect_tx(bar(B_QFULL + qb), 2 * NP * 128);
      const int qrow = w.tc.seq * a.h + w.tc.head * a.hq;
      const uint32_t qdst = r.sbase + L::kQ + qb * L::kQBytes;
      tma_load_2d(qdst, tm_q, bar(B_QFULL + qb), 0, qrow);
      tma_load_2d(qdst + NP * 128, tm_q, bar(B_QFULL + qb), 64, qrow);
    }
    const int st = int(i % kStages);
    if (i >= kStages && !wait_bar(r, bar(B_KVEMPTY + st), uint32_t((i / kStages) - 1) & 1)) break;
    const int row = w.tc.seq * a.m_max + w.tc.row0;
    const uint32_t kdst = r.sbase + L::kK + st * kTileBytes;
    const uint32_t vdst = r.sbase + L::kV + st * kTileBytes;
    mbar_expect_tx(bar(B_KFULL + st), kTileBytes);
    tma_load_3d(kdst, tm_k, bar(B_KFULL + st), 0, w.tc.head, row, pol);
    tma_load_3d(kdst + kHalfBytes, tm_k, bar(B_KFULL + st), 64, w.tc.head, row, pol);
    mbar_expect_tx(bar(B_VFULL + st), kTileBytes);
    tma_load_3d(vdst, tm_v, bar(B_VFULL + st), 0, w.tc.head, row, pol);
    tma_load_3d(vdst + kHalfBytes, tm_v, bar(B_VFULL + st), 64, w.tc.head, row, pol);
  }
  // Drain: every copy this thread issued has landed before the CTA can exit.
  for (int64_t j = (i - kStages > 0 ? i - kStages : 0); j < i; ++j) {
    const int st = int(j % kStages);
    mbar_wait(bar(B_KFULL + st), uint32_t(j / kStages) & 1, kTimeoutNs);
    mbar_wait(bar(B_VFULL + st), uint32_t(j / kStages) & 1, kTimeoutNs);
  }
  if (w.sidx >= 0) mbar_wait(bar(B_QFULL + (w.sidx & 1)), uint32_t(w.sidx >> 1) & 1, kTimeoutNs);
  if (w.sidx >= 1) mbar_wait(bar(B_QFULL + ((w.sidx - 1) & 1)), uint32_t((w.sidx - 1) >> 1) & 1, kTimeoutNs);
}

template <int NP>
__device__ void mma_issuer(const DecodeArgs& a, const Sched& sc, const Roles& r) {
  using L = TcLayout<NP>;
  auto bar = [&](int id) { return r.sbase + L::kBar + 8u * id; };
  constexpr uint32_t idesc_qk = idesc_bf16_f32(kTile, NP, 0, 0);
  constexpr uint32_t idesc_pv = idesc_bf16_f32(kTile, kNpv, 1, 1);
  const int64_t n = sc.t_end - sc.t_begin;
  TileWalk wq(a, sc), wp(a, sc);   // look-ahead walker for S, trailing walker for O

  auto issue_qk = [&](int64_t i) -> bool {
    wq.next(a, sc);
    const int st = int(i % kStages);
    const int qb = wq.sidx & 1;
    if (wq.first && !wait_bar(r, bar(B_QFULL + qb), uint32_t(wq.sidx >> 1) & 1)) return false;
    if (!wait_bar(r, bar(B_KFULL + st), uint32_t(i / kStages) & 1)) return false;
    tc_fence_after();
    const uint32_t kbase = r.sbase + L::kK + st * kTileBytes;
    const uint32_t qbase = r.sbase + L::kQ + qb * L::kQBytes;
    const uint32_t d = r.tmem + uint32_t(i & 1) * NP;
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
      const uint32_t koff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
      const uint32_t qoff = (kk >> 2) * (NP * 128) + (kk & 3) * 32;
      mma_bf16_ss(d, smem_desc_sw128(kbase + koff, 16, 1024), smem_desc_sw128(qbase + qoff, 16, 1024), idesc_qk,
                  kk > 0);
    }
    mma_commit(bar(B_SFULL + (i & 1)));
    if (wq.last) mma_commit(bar(B_QEMPTY + qb));
    return true;
  };
  auto issue_pv = [&](int64_t i) -> bool {
    wp.next(a, sc);
    const int st = int(i % kStages);
    const int ob = wp.sidx & 1;
    if (!wait_bar(r, bar(B_PFULL + (i & 1)), uint32_t(i >> 1) & 1)) return false;
    if (!wait_bar(r, bar(B_VFULL + st), uint32_t(i / kStages) & 1)) return false;
    if (wp.first && wp.sidx >= 2 && !wait_bar(r, bar(B_OFREE + ob), uint32_t((wp.sidx >> 1) - 1) & 1)) return false;
    tc_fence_after();
    const uint32_t vbase = r.sbase + L::kV + st * kTileBytes;
    const uint32_t pbase = r.sbase + L::kP + uint32_t(i & 1) * L::kPBytes;
    const uint32_t d = r.tmem + kOCol + uint32_t(ob) * kNpv;
#pragma unroll
    for (int kk = 0; kk < kTile / 16; ++kk) {
      mma_bf16_ss(d, smem_desc_sw128(vbase + kk * 2048, kHalfBytes, 1024),
                  smem_desc_sw128(pbase + kk * 2048, kHalfBytes, 1024), idesc_pv, (kk > 0 || !wp.first) ? 1u : 0u);
    }
    mma_commit(bar(B_OFULL + (i & 1)));
    mma_commit(bar(B_KVEMPTY + st));
    return true;
  };

  if (n > 0 && issue_qk(0)) {
    for (int64_t i = 0; i < n; ++i) {
      if (*r.abort) break;
      if (i + 1 < n && !issue_qk(i + 1)) break;
      if (!issue_pv(i)) break;
    }
  }
  // every MMA issued above has completed before tensor memory is released
  mma_commit(bar(B_DONE));
  mbar_wait(bar(B_DONE), 0, kTimeoutNs);
}

// Barrier of the four softmax warps that also ANDs a per-thread flag, so that
// every thread takes the same branch after a bounded wait (a thread that gave
// up alone would otherwise leave the others blocked at the next barrier).
__device__ __forceinline__ bool softmax_barrier_and(bool ok) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, 1, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(out)
      : "r"(uint32_t(ok))
      : "memory");
  return out != 0;
}

template <int NP>
__device__ void softmax_epilogue(const DecodeArgs& a, const Sched& sc, const Roles& r, int warp, int lane) {
  using L = TcLayout<NP>;
  auto bar = [&](int id) { return r.sbase + L::kBar + 8u * id; };
  auto wait = [&](int id, uint32_t parity) { return mbar_wait(bar(id), parity, kTimeoutNs); };
  constexpr int NCH = NP / 16;
  const int q4 = warp & 3;                         // TMEM lane quarter this warp may access
  const int sw = warp - 2;                         // index within the softmax group
  const int row = 32 * q4 + lane;                  // cache row of the tile (S), output column (O)
  const uint32_t t_lane = r.tmem + (uint32_t(32 * q4) << 16);
  float* red = reinterpret_cast<float*>(r.smem + L::kRed);
  float* mref = reinterpret_cast<float*>(r.smem + L::kMref);
  float* alpha = reinterpret_cast<float*>(r.smem + L::kAlpha);
  float* lsum = reinterpret_cast<float*>(r.smem + L::kLsum);
  volatile int* flag = reinterpret_cast<volatile int*>(r.smem + L::kFlag);
  const float c = a.scale * kLog2e;
  const int hq = a.hq;
  float lpart[NP];
  float sv[NP];
  TileWalk w(a, sc);
  const int64_t n = sc.t_end - sc.t_begin;
  int64_t pv_waited = -1;
  bool failed = false;
  for (int64_t i = 0; i < n; ++i) {
    w.next(a, sc);
    if (w.first) {
#pragma unroll
      for (int k = 0; k < NP; ++k) lpart[k] = 0.f;
    }
    bool ok = wait(B_SFULL + (i & 1), uint32_t(i >> 1) & 1);
    tc_fence_after();
    const bool valid = row < w.tc.rows;
    // scaled logits (log2 units) of this thread's row, and the tile's column maxima
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
      float v[16];
      tmem_ld16(t_lane + uint32_t(i & 1) * NP + ch * 16, v);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        sv[ch * 16 + k] = valid ? v[k] * c : -INFINITY;
        v[k] = sv[ch * 16 + k];
      }
      const float mx = transpose_reduce<16, true>(v, lane);
      if (lane < 16) red[sw * 64 + ch * 16 + lane] = mx;
    }
    if (!softmax_barrier_and(ok)) { failed = true; break; }
    if (sw == 0) {
      int resc = 0;
      for (int col = lane; col < NP; col += 32) {
        const float mt = fmaxf(fmaxf(red[col], red[64 + col]), fmaxf(red[128 + col], red[192 + col]));
        float mn = mt, al = 1.f;
        if (!w.first) {
          const float mo = mref[col];
          if (mt > mo + kRescaleThreshold) {
            al = exp2f(mo - mt);
            resc |= col < hq;
          } else {
            mn = mo;
          }
        }
        mref[col] = mn;
        alpha[col] = al;
      }
      resc = __any_sync(0xffffffffu, resc);
      if (lane == 0) *flag = resc;
    }
    named_barrier_softmax();
    const bool resc = *flag != 0;
    // O(i-1) must be complete before O is rescaled and before P(i) overwrites
    // the buffer P(i-2) used; a ragged tile needs its V rows landed before the
    // rows past the sequence end are zeroed.
    ok = true;
    if (i > 0 && pv_waited < i - 1) {
      ok = wait(B_OFULL + ((i - 1) & 1), uint32_t((i - 1) >> 1) & 1);
      pv_waited = i - 1;
    }
    const int st = int(i % kStages);
    if (w.tc.rows < kTile) ok = wait(B_VFULL + st, uint32_t(i / kStages) & 1) && ok;
    if (!softmax_barrier_and(ok)) { failed = true; break; }
    tc_fence_after();
    if (resc) {
#pragma unroll
      for (int k = 0; k < NP; ++k) lpart[k] *= alpha[k];
      if (!w.first) {   // rescale the O accumulated so far (thread = output column)
        const uint32_t oc = t_lane + kOCol + uint32_t(w.sidx & 1) * kNpv;
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          float v[16];
          tmem_ld16(oc + ch * 16, v);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 16; ++k) v[k] *= alpha[ch * 16 + k];
          tmem_st16(oc + ch * 16, v);
        }
        tmem_wait_st();
      }
    }
    // P = exp2(s - m), bf16, into the MN-major 128-byte-swizzled P buffer
    unsigned char* prow = r.smem + L::kP + uint32_t(i & 1) * L::kPBytes + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
    for (int c8 = 0; c8 < NP / 8; ++c8) {
      uint32_t packed[4];
#pragma unroll
      for (int k2 = 0; k2 < 4; ++k2) {
        const int col = c8 * 8 + k2 * 2;
        const float p0 = (valid && col < hq) ? exp2f(sv[col] - mref[col]) : 0.f;
        const float p1 = (valid && col + 1 < hq) ? exp2f(sv[col + 1] - mref[col + 1]) : 0.f;
        lpart[col] += p0;
        lpart[col + 1] += p1;
        __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
        packed[k2] = *reinterpret_cast<uint32_t*>(&b2);
      }
      *reinterpret_cast<uint4*>(prow + ((c8 ^ (row & 7)) << 4)) =
          make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
    if (!valid) {
      // rows past the sequence end were loaded too; zero them in V so that
      // P = 0 times whatever they hold contributes exactly 0
      unsigned char* v0 = r.smem + L::kV + st * kTileBytes + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16) {
        *reinterpret_cast<uint4*>(v0 + c16 * 16) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(v0 + kHalfBytes + c16 * 16) = make_uint4(0, 0, 0, 0);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(bar(B_PFULL + (i & 1)));

    if (w.last) {
      ok = wait(B_OFULL + (i & 1), uint32_t(i >> 1) & 1);
      pv_waited = i;
      // per-head sums over the 128 rows
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        float v[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = lpart[ch * 16 + k];
        const float s = transpose_reduce<16, false>(v, lane);
        if (lane < 16) red[sw * 64 + ch * 16 + lane] = s;
      }
      if (!softmax_barrier_and(ok)) { failed = true; break; }
      tc_fence_after();
      if (sw == 0)
        for (int col = lane; col < NP; col += 32)
          lsum[col] = red[col] + red[64 + col] + red[128 + col] + red[192 + col];
      named_barrier_softmax();
      const bool owns_first = w.tc.seg_t0 >= sc.t_begin;
      const bool whole = owns_first && (w.tc.seg_t0 + w.tc.nb <= sc.t_end);
      const int64_t slot = partial_slot(blockIdx.x, w.tc.seg);
      const uint32_t oc = t_lane + kOCol + uint32_t(w.sidx & 1) * kNpv;
      const int64_t obase = (int64_t(w.tc.seq) * a.h + int64_t(w.tc.head) * hq) * kD;
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        float v[16];
        tmem_ld16(oc + ch * 16, v);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int col = ch * 16 + k;
          if (col < hq) {
            const float val = v[k] / lsum[col];
            if (whole)
              static_cast<__nv_bfloat16*>(a.o)[obase + int64_t(col) * kD + row] = __float2bfloat16_rn(val);
            else
              a.ws.part_o[(slot * hq + col) * kD + row] = val;
          }
        }
      }
      if (sw == 0) {
        if (!whole)
          for (int col = lane; col < hq; col += 32) a.ws.part_lse[slot * hq + col] = mref[col] + log2f(lsum[col]);
        if (owns_first && lane == 0)
          a.ws.seg_info[w.tc.seg] =
              make_int2(blockIdx.x, cta_of_tile(w.tc.seg_t0 + w.tc.nb - 1, sc.total, sc.active));
      }
      tc_fence_before();
      mbar_arrive(bar(B_OFREE + (w.sidx & 1)));
    }
  }
  if (failed && threadIdx.x == 64) {
    *r.abort = 1;
    set_flag(r.flags, MQA_FLAG_PIPE_TIMEOUT);
  }
}

template <int NP>
__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q) {
  using L = TcLayout<NP>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  Roles r;
  r.smem = smem_raw + pad;
  r.sbase = raw + pad;
  r.abort = reinterpret_cast<volatile int*>(r.smem + L::kAbort);
  r.flags = a.flags;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  auto bar = [&](int id) { return r.sbase + L::kBar + 8u * id; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_KVEMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_SFULL + s), 1);
      mbar_init(bar(B_PFULL + s), 128);
      mbar_init(bar(B_OFULL + s), 1);
      mbar_init(bar(B_QFULL + s), 1);
      mbar_init(bar(B_QEMPTY + s), 1);
      mbar_init(bar(B_OFREE + s), 128);
    }
    mbar_init(bar(B_DONE), 1);
    *r.abort = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_q);
  }
  if (warp == 1) {
    tmem_alloc(r.sbase + L::kTmemSlot, kTmemCols);
    tmem_relinquish();
  }
  if (warp >= 2) {   // zero both P buffers: the pad columns (heads >= NP) stay zero
    uint4* p = reinterpret_cast<uint4*>(r.smem + L::kP);
    for (int k = threadIdx.x - 64; k < int(2 * L::kPBytes / 16); k += 128) p[k] = make_uint4(0, 0, 0, 0);
  }
  // Inputs may come from the kernel before this one on the stream (the append).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const Sched sc = make_schedule<kThreads>(a.lens, a.b, a.g, a.m_max, kTile, a.grid, blockIdx.x, a.flags,
                                           reinterpret_cast<int64_t*>(r.smem + L::kSched));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  r.tmem = *reinterpret_cast<volatile uint32_t*>(r.smem + L::kTmemSlot);

  if (sc.t_begin < sc.t_end) {
    if (warp == 0) {
      if (lane == 0) producer<NP>(a, sc, r, &tm_k, &tm_v, &tm_q);
    } else if (warp == 1) {
      if (lane == 0) mma_issuer<NP>(a, sc, r);
    } else {
      softmax_epilogue<NP>(a, sc, r, warp, lane);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(r.tmem, kTmemCols);
  asm volatile("griddepcontrol.launch_dependents;");
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

// Cache [b, m_max, g, 128] bf16 as a 3-D tensor (d, g, b*m_max); a box is 64
// columns of one K/V head over 128 consecutive rows, 128-byte swizzled.
bool encode_cache(CUtensorMap* m, const void* base, int b, int m_max, int g) {
  const cuuint64_t dims[3] = {cuuint64_t(kD), cuuint64_t(g), cuuint64_t(b) * cuuint64_t(m_max)};
  const cuuint64_t strides[2] = {cuuint64_t(kD) * 2, cuuint64_t(g) * kD * 2};
  const cuuint32_t box[3] = {64, 1, kTile};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q [b*h, 128] bf16; a box is 64 columns of NP consecutive heads.
bool encode_q(CUtensorMap* m, const void* base, int rows, int np) {
  const cuuint64_t dims[2] = {cuuint64_t(kD), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(kD) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(np)};
  const cuuint32_t estr[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NP>
cudaError_t launch_np(const DecodeArgs& a, cudaStream_t stream) {
  using L = TcLayout<NP>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(decode_tc_kernel<NP>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(L::kAlloc));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  CUtensorMap tk, tv, tq;
  if (!encode_cache(&tk, a.k, a.b, a.m_max, a.g) || !encode_cache(&tv, a.v, a.b, a.m_max, a.g) ||
      !encode_q(&tq, a.q, a.b * a.h, NP))
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(a.grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_tc_kernel<NP>, a, tk, tv, tq);
}

}  // namespace

bool tc_supported(int d, int hq) { return d == kD && hq >= 1 && hq <= 64; }

int tc_ctas_per_sm(int) { return 1; }

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream) {
  if (int64_t(a.b) * a.m_max >= (int64_t(1) << 31) || int64_t(a.b) * a.h >= (int64_t(1) << 31))
    return cudaErrorInvalidValue;
  if (a.hq <= 16) return launch_np<16>(a, stream);
  if (a.hq <= 32) return launch_np<32>(a, stream);
  if (a.hq <= 64) return launch_np<64>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace mqa
