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
//   warp 0, lane 0      TMA producer of Q (per segment) and of K tiles into a
//                       ring of SK stages; a K stage is released as soon as
//                       the S product that reads it has completed.
//   warp 0, lane 1      TMA producer of V tiles into a ring of SV stages,
//                       released when the P.V product has completed.  Both
//                       rings use L2 evict-first: each byte is read once.
//   warp 1, lane 0      MMA issuer: S(i+1) = K Q^T while P(i) is being made,
//                       then O += V^T P(i); completions are signalled with
//                       tcgen05.commit on mbarriers.
//   warps 2-5           softmax and epilogue, one cache row (then one output
//                       column) per thread.  The reference max per head is set
//                       from the first tile of a segment and only moved when
//                       some logit exceeds it by more than 8 (a factor 256 in
//                       exp2); only then do the warps reduce column maxima and
//                       rescale O in tensor memory.  P = exp2(s - m) goes to
//                       shared memory in bf16, per-head sums stay in registers.
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
constexpr int kThreads = 192;
constexpr int kNpv = 64;                     // N of the P.V product (P padded with zero columns)
constexpr uint32_t kHalfBytes = kTile * 128; // 128 rows x 64 bf16, one 128-byte swizzle column
constexpr uint32_t kTileBytes = 2 * kHalfBytes;
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr float kRescaleThreshold = 8.f;     // log2 units
constexpr uint32_t kTmemCols = 256;          // S double buffer at [0, 2*NP), O double buffer at [128, 256)
constexpr uint32_t kOCol = 128;
constexpr uint32_t kMaxDynSmem = 232448;     // 227 KB opt-in limit per CTA

template <int NP, int SK, int SV>
struct TcCfg {
  // barriers
  static constexpr int kKFull = 0, kKEmpty = SK, kVFull = 2 * SK, kVEmpty = 2 * SK + SV, kSFull = 2 * SK + 2 * SV,
                       kPFull = kSFull + 2, kOFull = kPFull + 1, kQFull = kOFull + 1, kQEmpty = kQFull + 2,
                       kOFree = kQEmpty + 2, kDone = kOFree + 2, kNumBars = kDone + 1;
  // shared memory
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + SK * kTileBytes;
  static constexpr uint32_t kQ = kV + SV * kTileBytes;
  static constexpr uint32_t kQBytes = NP * 256;                // two 64-column halves of NP rows
  static constexpr uint32_t kP = kQ + 2 * kQBytes;
  static constexpr uint32_t kPBytes = kTile * 128;             // 128 rows x 64 heads (bf16)
  static constexpr uint32_t kBar = kP + kPBytes;
  static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
  static constexpr uint32_t kFlag = kTmemSlot + 4;
  static constexpr uint32_t kAbort = kFlag + 4;
  static constexpr uint32_t kRed = (kAbort + 4 + 15) / 16 * 16;  // [4][NP] f32
  static constexpr uint32_t kMref = kRed + 4 * NP * 4;
  static constexpr uint32_t kAlpha = kMref + NP * 4;
  static constexpr uint32_t kLsum = kAlpha + NP * 4;
  static constexpr uint32_t kEnd = kLsum + NP * 4;
  static constexpr uint32_t kAlloc = kEnd + 1024;             // room to align the base to 1024 bytes
  static constexpr uint32_t kSched = kP;                      // start-up scratch, before P is zeroed
  static_assert(kQ % 1024 == 0 && kP % 1024 == 0 && kQBytes % 1024 == 0, "swizzle atoms need 1024-byte alignment");
  static_assert(kAlloc <= kMaxDynSmem, "shared memory budget");
  static_assert((kThreads / 32 + kThreads + 2) * 8 <= kPBytes, "schedule scratch fits in P");
};

__device__ __forceinline__ void named_barrier_softmax() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Barriers of the four softmax warps that also reduce a per-thread flag, so
// that every thread takes the same branch afterwards (a thread that gave up a
// bounded wait alone would otherwise leave the others blocked).
__device__ __forceinline__ bool softmax_barrier_and(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, 1, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(out)
      : "r"(uint32_t(v))
      : "memory");
  return out != 0;
}
__device__ __forceinline__ bool softmax_barrier_or(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, 1, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(out)
      : "r"(uint32_t(v))
      : "memory");
  return out != 0;
}

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

// Walks the CTA's tiles in order and tells each role what a tile is.  Only
// the first step divides; later steps count (tile, head, sequence) forward.
struct TileWalk {
  int64_t t;                 // current tile number
  int64_t base;              // first tile of the current sequence
  int seq, head, k, nb, len;
  int sidx;                  // segment number within this CTA
  TileCoord tc;
  bool first, last;
  __device__ TileWalk(const DecodeArgs& a, const Sched& sc) : t(sc.t_begin - 1), sidx(-1) {
    Cursor cu = cursor_at(a.lens, a.m_max, kTile, sc.seq, sc.seq_base);
    cursor_seek(cu, a.lens, a.g, a.m_max, kTile, sc.t_begin);
    seq = cu.seq;
    base = cu.base;
    nb = cu.nb;
    len = cu.len;
    const int64_t rel = sc.t_begin - cu.base;
    head = int(rel / cu.nb);
    k = int(rel - int64_t(head) * cu.nb) - 1;   // next() advances to the first tile
  }
  __device__ void next(const DecodeArgs& a, const Sched& sc) {
    ++t;
    if (++k == nb) {
      k = 0;
      if (++head == a.g) {
        head = 0;
        base += int64_t(a.g) * nb;
        do {
          ++seq;
          len = clamp_len(__ldg(a.lens + seq), a.m_max, nullptr, false);
          nb = tiles_of(len, kTile);
        } while (nb == 0);
      }
    }
    tc.seq = seq;
    tc.head = head;
    tc.k = k;
    tc.row0 = k * kTile;
    tc.rows = min(kTile, len - tc.row0);
    tc.seg = int64_t(seq) * a.g + head;
    tc.nb = nb;
    tc.seg_t0 = base + int64_t(head) * nb;
    first = (t == sc.t_begin) || k == 0;
    last = (k == nb - 1) || (t + 1 == sc.t_end);
    if (first) ++sidx;
  }
};

// K ring and the per-segment Q (kIsK), or the V ring.
template <int NP, int SK, int SV, bool kIsK>
__device__ void producer(const DecodeArgs& a, const Sched& sc, const Roles& r, const CUtensorMap* tm_kv,
                         const CUtensorMap* tm_q) {
  using C = TcCfg<NP, SK, SV>;
  constexpr int S = kIsK ? SK : SV;
  constexpr int kFull = kIsK ? C::kKFull : C::kVFull;
  constexpr int kEmpty = kIsK ? C::kKEmpty : C::kVEmpty;
  constexpr uint32_t kRing = kIsK ? C::kK : C::kV;
  auto bar = [&](int id) { return r.sbase + C::kBar + 8u * id; };
  const uint64_t pol = l2_evict_first_policy();
  TileWalk w(a, sc);
  const int64_t n = sc.t_end - sc.t_begin;
  int64_t i = 0;
  int q_issued = -1;
  for (; i < n; ++i) {
    w.next(a, sc);
    if (*r.abort) break;
    if (kIsK && w.first) {
      const int qb = w.sidx & 1;
      if (w.sidx >= 2 && !wait_bar(r, bar(C::kQEmpty + qb), ((w.sidx >> 1) - 1) & 1)) break;
      mbar_expect_tx(bar(C::kQFull + qb), 2 * NP * 128);
      const int qrow = w.tc.seq * a.h + w.tc.head * a.hq;
      const uint32_t qdst = r.sbase + C::kQ + qb * C::kQBytes;
      tma_load_2d(qdst, tm_q, bar(C::kQFull + qb), 0, qrow);
      tma_load_2d(qdst + NP * 128, tm_q, bar(C::kQFull + qb), 64, qrow);
      q_issued = w.sidx;
    }
    const int st = int(i % S);
    if (i >= S && !wait_bar(r, bar(kEmpty + st), uint32_t((i / S) - 1) & 1)) break;
    const int row = w.tc.seq * a.m_max + w.tc.row0;
    const uint32_t dst = r.sbase + kRing + st * kTileBytes;
    mbar_expect_tx(bar(kFull + st), kTileBytes);
    tma_load_3d(dst, tm_kv, bar(kFull + st), 0, w.tc.head, row, pol);
    tma_load_3d(dst + kHalfBytes, tm_kv, bar(kFull + st), 64, w.tc.head, row, pol);
  }
  // Drain: every copy this thread issued has landed before the CTA can exit.
  for (int64_t j = (i - S > 0 ? i - S : 0); j < i; ++j)
    mbar_wait(bar(kFull + int(j % S)), uint32_t(j / S) & 1, kTimeoutNs);
  if (kIsK)
    for (int sq = (q_issued - 1 > 0 ? q_issued - 1 : 0); sq <= q_issued; ++sq)
      mbar_wait(bar(C::kQFull + (sq & 1)), uint32_t(sq >> 1) & 1, kTimeoutNs);
}

template <int NP, int SK, int SV>
__device__ void mma_issuer(const DecodeArgs& a, const Sched& sc, const Roles& r) {
  using C = TcCfg<NP, SK, SV>;
  auto bar = [&](int id) { return r.sbase + C::kBar + 8u * id; };
  constexpr uint32_t idesc_qk = idesc_bf16_f32(kTile, NP, 0, 0);
  constexpr uint32_t idesc_pv = idesc_bf16_f32(kTile, kNpv, 1, 1);
  const int64_t n = sc.t_end - sc.t_begin;
  TileWalk wq(a, sc), wp(a, sc);   // look-ahead walker for S, trailing walker for O

  auto issue_qk = [&](int64_t i) -> bool {
    wq.next(a, sc);
    const int st = int(i % SK);
    const int qb = wq.sidx & 1;
    if (wq.first && !wait_bar(r, bar(C::kQFull + qb), uint32_t(wq.sidx >> 1) & 1)) return false;
    if (!wait_bar(r, bar(C::kKFull + st), uint32_t(i / SK) & 1)) return false;
    tc_fence_after();
    const uint32_t kbase = r.sbase + C::kK + st * kTileBytes;
    const uint32_t qbase = r.sbase + C::kQ + qb * C::kQBytes;
    const uint32_t d = r.tmem + uint32_t(i & 1) * NP;
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
      const uint32_t koff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
      const uint32_t qoff = (kk >> 2) * (NP * 128) + (kk & 3) * 32;
      mma_bf16_ss(d, smem_desc_sw128(kbase + koff, 16, 1024), smem_desc_sw128(qbase + qoff, 16, 1024), idesc_qk,
                  kk > 0);
    }
    mma_commit(bar(C::kSFull + (i & 1)));
    mma_commit(bar(C::kKEmpty + st));
    if (wq.last) mma_commit(bar(C::kQEmpty + qb));
    return true;
  };
  auto issue_pv = [&](int64_t i) -> bool {
    wp.next(a, sc);
    const int st = int(i % SV);
    const int ob = wp.sidx & 1;
    if (!wait_bar(r, bar(C::kPFull), uint32_t(i & 1))) return false;
    if (!wait_bar(r, bar(C::kVFull + st), uint32_t(i / SV) & 1)) return false;
    if (wp.first && wp.sidx >= 2 && !wait_bar(r, bar(C::kOFree + ob), uint32_t((wp.sidx >> 1) - 1) & 1))
      return false;
    tc_fence_after();
    const uint32_t vbase = r.sbase + C::kV + st * kTileBytes;
    const uint32_t pbase = r.sbase + C::kP;
    const uint32_t d = r.tmem + kOCol + uint32_t(ob) * kNpv;
#pragma unroll
    for (int kk = 0; kk < kTile / 16; ++kk) {
      mma_bf16_ss(d, smem_desc_sw128(vbase + kk * 2048, kHalfBytes, 1024),
                  smem_desc_sw128(pbase + kk * 2048, kHalfBytes, 1024), idesc_pv, (kk > 0 || !wp.first) ? 1u : 0u);
    }
    mma_commit(bar(C::kOFull));
    mma_commit(bar(C::kVEmpty + st));
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
  mma_commit(bar(C::kDone));
  mbar_wait(bar(C::kDone), 0, kTimeoutNs);
}

template <int NP, int SK, int SV>
__device__ void softmax_epilogue(const DecodeArgs& a, const Sched& sc, const Roles& r, int warp, int lane) {
  using C = TcCfg<NP, SK, SV>;
  auto bar = [&](int id) { return r.sbase + C::kBar + 8u * id; };
  auto wait = [&](int id, uint32_t parity) { return mbar_wait(bar(id), parity, kTimeoutNs); };
  constexpr int NCH = NP / 16;
  const int q4 = warp & 3;                         // TMEM lane quarter this warp may access
  const int sw = warp - 2;                         // index within the softmax group
  const int row = 32 * q4 + lane;                  // cache row of the tile (S), output column (O)
  const uint32_t t_lane = r.tmem + (uint32_t(32 * q4) << 16);
  float* red = reinterpret_cast<float*>(r.smem + C::kRed);
  float* mref = reinterpret_cast<float*>(r.smem + C::kMref);
  float* alpha = reinterpret_cast<float*>(r.smem + C::kAlpha);
  float* lsum = reinterpret_cast<float*>(r.smem + C::kLsum);
  const float c = a.scale * kLog2e;
  const int hq = a.hq;
  float lpart[NP];
  float sv[NP];
  // reference max per head (log2 units): mirrored in registers when they suffice
  constexpr bool kMrRegs = NP <= 32;
  float mr[kMrRegs ? NP : 1];
  auto mref_of = [&](int k) -> float {
    if constexpr (kMrRegs) return mr[k];
    else return mref[k];
  };
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
    bool ok = wait(C::kSFull + (i & 1), uint32_t(i >> 1) & 1);
    tc_fence_after();
    const bool valid = row < w.tc.rows;
    // scaled logits (log2 units) of this thread's row
#pragma unroll
    for (int ch = 0; ch < NP / 32; ++ch) {
      float v[32];
      tmem_ld32(t_lane + uint32_t(i & 1) * NP + ch * 32, v);
#pragma unroll
      for (int k = 0; k < 32; ++k) sv[ch * 32 + k] = v[k];
    }
    if constexpr (NP % 32 != 0) {
      float v[16];
      tmem_ld16(t_lane + uint32_t(i & 1) * NP + (NP / 32) * 32, v);
#pragma unroll
      for (int k = 0; k < 16; ++k) sv[(NP / 32) * 32 + k] = v[k];
    }
#pragma unroll
    for (int k = 0; k < NP; ++k) sv[k] = valid ? sv[k] * c : -INFINITY;
    // Does any logit of a real head exceed the reference max by the threshold?
    bool exceed = false;
    if (!w.first) {
#pragma unroll
      for (int k = 0; k < NP; ++k) exceed |= (k < hq) && (sv[k] > mref_of(k) + kRescaleThreshold);
    }
    const bool full = w.first || softmax_barrier_or(exceed);
    if (full) {   // column maxima of the tile and the new reference max
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        float v[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = sv[ch * 16 + k];
        const float mx = transpose_reduce<16, true>(v, lane);
        if (lane < 16) red[sw * NP + ch * 16 + lane] = mx;
      }
      named_barrier_softmax();
      if (sw == 0) {
        for (int col = lane; col < NP; col += 32) {
          const float mt = fmaxf(fmaxf(red[col], red[NP + col]), fmaxf(red[2 * NP + col], red[3 * NP + col]));
          float mn = mt, al = 1.f;
          if (!w.first) {
            const float mo = mref[col];
            if (mt > mo + kRescaleThreshold) {
              al = ex2_approx(mo - mt);
            } else {
              mn = mo;
            }
          }
          mref[col] = mn;
          alpha[col] = al;
        }
      }
      named_barrier_softmax();
      if constexpr (kMrRegs) {
#pragma unroll
        for (int k = 0; k < NP; ++k) mr[k] = mref[k];
      }
    }
    // O(i-1) must be complete before O is rescaled and before P(i) overwrites
    // the P buffer it read; a ragged tile needs its V rows landed before the
    // rows past the sequence end are zeroed.
    bool ok2 = true;
    if (i > 0 && pv_waited < i - 1) {
      ok2 = wait(C::kOFull, uint32_t(i - 1) & 1);
      pv_waited = i - 1;
    }
    const int st = int(i % SV);
    if (w.tc.rows < kTile) ok2 = wait(C::kVFull + st, uint32_t(i / SV) & 1) && ok2;
    if (!softmax_barrier_and(ok && ok2)) { failed = true; break; }
    tc_fence_after();
    if (full && !w.first) {
#pragma unroll
      for (int k = 0; k < NP; ++k) lpart[k] *= alpha[k];
      // rescale the O accumulated so far (thread = output column)
      const uint32_t oc = t_lane + kOCol + uint32_t(w.sidx & 1) * kNpv;
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        float v[16];
        tmem_ld16(oc + ch * 16, v);
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] *= alpha[ch * 16 + k];
        tmem_st16(oc + ch * 16, v);
      }
      tmem_wait_st();
    }
    // P = exp2(s - m), bf16, into the MN-major 128-byte-swizzled P buffer
    unsigned char* prow = r.smem + C::kP + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
    for (int c8 = 0; c8 < NP / 8; ++c8) {
      uint32_t packed[4];
#pragma unroll
      for (int k2 = 0; k2 < 4; ++k2) {
        const int col = c8 * 8 + k2 * 2;
        const float p0 = col < hq ? ex2_approx(sv[col] - mref_of(col)) : 0.f;
        const float p1 = col + 1 < hq ? ex2_approx(sv[col + 1] - mref_of(col + 1)) : 0.f;
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
      unsigned char* v0 = r.smem + C::kV + st * kTileBytes + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16) {
        *reinterpret_cast<uint4*>(v0 + c16 * 16) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(v0 + kHalfBytes + c16 * 16) = make_uint4(0, 0, 0, 0);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(bar(C::kPFull));

    if (w.last) {
      ok = wait(C::kOFull, uint32_t(i) & 1);
      pv_waited = i;
      // per-head sums over the 128 rows
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        float v[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = lpart[ch * 16 + k];
        const float s = transpose_reduce<16, false>(v, lane);
        if (lane < 16) red[sw * NP + ch * 16 + lane] = s;
      }
      if (!softmax_barrier_and(ok)) { failed = true; break; }
      tc_fence_after();
      if (sw == 0)
        for (int col = lane; col < NP; col += 32)
          lsum[col] = red[col] + red[NP + col] + red[2 * NP + col] + red[3 * NP + col];
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
      mbar_arrive(bar(C::kOFree + (w.sidx & 1)));
    }
  }
  if (failed && threadIdx.x == 64) {
    *r.abort = 1;
    set_flag(r.flags, MQA_FLAG_PIPE_TIMEOUT);
  }
}

template <int NP, int SK, int SV>
__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q) {
  using C = TcCfg<NP, SK, SV>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  Roles r;
  r.smem = smem_raw + pad;
  r.sbase = raw + pad;
  r.abort = reinterpret_cast<volatile int*>(r.smem + C::kAbort);
  r.flags = a.flags;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  auto bar = [&](int id) { return r.sbase + C::kBar + 8u * id; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < SK; ++s) {
      mbar_init(bar(C::kKFull + s), 1);
      mbar_init(bar(C::kKEmpty + s), 1);
    }
    for (int s = 0; s < SV; ++s) {
      mbar_init(bar(C::kVFull + s), 1);
      mbar_init(bar(C::kVEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(C::kSFull + s), 1);
      mbar_init(bar(C::kQFull + s), 1);
      mbar_init(bar(C::kQEmpty + s), 1);
      mbar_init(bar(C::kOFree + s), 128);
    }
    mbar_init(bar(C::kPFull), 128);
    mbar_init(bar(C::kOFull), 1);
    mbar_init(bar(C::kDone), 1);
    *r.abort = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_q);
  }
  if (warp == 1) {
    tmem_alloc(r.sbase + C::kTmemSlot, kTmemCols);
    tmem_relinquish();
  }
  // Inputs may come from the kernel before this one on the stream (the append).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const Sched sc = make_schedule<kThreads>(a.lens, a.b, a.g, a.m_max, kTile, a.grid, blockIdx.x, a.flags,
                                           reinterpret_cast<int64_t*>(r.smem + C::kSched));
  __syncthreads();
  if (warp >= 2) {   // zero the P buffer (it held the schedule scratch): pad columns stay zero
    uint4* p = reinterpret_cast<uint4*>(r.smem + C::kP);
    for (int k = threadIdx.x - 64; k < int(C::kPBytes / 16); k += 128) p[k] = make_uint4(0, 0, 0, 0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  r.tmem = *reinterpret_cast<volatile uint32_t*>(r.smem + C::kTmemSlot);

  if (sc.t_begin < sc.t_end) {
    if (warp == 0) {
      if (lane == 0) producer<NP, SK, SV, true>(a, sc, r, &tm_k, &tm_q);
      else if (lane == 1) producer<NP, SK, SV, false>(a, sc, r, &tm_v, &tm_q);
    } else if (warp == 1) {
      if (lane == 0) mma_issuer<NP, SK, SV>(a, sc, r);
    } else {
      softmax_epilogue<NP, SK, SV>(a, sc, r, warp, lane);
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

template <int NP, int SK, int SV>
cudaError_t launch_np(const DecodeArgs& a, cudaStream_t stream) {
  using L = TcCfg<NP, SK, SV>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(decode_tc_kernel<NP, SK, SV>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(L::kAlloc));
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
  return cudaLaunchKernelEx(&cfg, decode_tc_kernel<NP, SK, SV>, a, tk, tv, tq);
}

}  // namespace

bool tc_supported(int d, int hq) { return d == kD && hq >= 1 && hq <= 64; }

int tc_ctas_per_sm(int) { return 1; }

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream) {
  if (int64_t(a.b) * a.m_max >= (int64_t(1) << 31) || int64_t(a.b) * a.h >= (int64_t(1) << 31))
    return cudaErrorInvalidValue;
  if (a.hq <= 16) return launch_np<16, 3, 3>(a, stream);
  if (a.hq <= 32) return launch_np<32, 3, 3>(a, stream);
  if (a.hq <= 64) return launch_np<64, 2, 3>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace mqa
