// Split-KV decode attention on the 5th-generation tensor cores (tcgen05),
// for bf16 caches with key and value head sizes of 64 or 128 and up to 64
// query heads per K/V head.
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
// With the fused append (k_new/v_new given) the producer that owns a
// sequence's last tile first writes the step's new K (or V) row into the cache
// at row lens-1 and then loads the tile, so the row is both stored for later
// steps and attended to now.
//
// Work: one CTA per SM, persistent over a contiguous run of all segments'
// tiles; runs are balanced in quarter tiles with a segment's entry weighted
// as a whole tile.  The thread of the schedule that finds a CTA's first tile
// issues its first Q, K and V loads itself (start-up code runs at
// instruction-fetch speed; a separate role would reach them much later).
// A segment split between CTAs leaves normalised partials with their
// log-sum-exp for the merge kernel; a whole one is written directly.  With a
// local window the partition counts only the window's rows.  Beams sharing a
// prefix: with q_beams the W beams' heads of a group form the segment's query
// rows (a 3-D box gathers them), and every segment leaves a partial.
//
// Roles:
//   warp 0, lane 0      TMA producer of Q (per segment) and of K tiles into a
//                       ring of SK stages; a K stage is released as soon as
//                       the S product that reads it has completed.
//   warp 10, lane 0     TMA producer of V tiles into a ring of SV stages,
//                       released when the P.V product has completed; it
//                       never runs ahead of the K producer.  Both rings use
//                       L2 evict-first: each byte is read once.  The two
//                       producers sit in different warps because the waits of
//                       two diverged threads of one warp are serialised.
//   warp 1, lane 0      S issuer: S(i) = K Q^T into a double buffer in tensor
//                       memory, as soon as K(i) has landed and the softmax
//                       warps hold S(i-2) in registers.
//   warp 11, lane 0     P.V issuer: O += V^T P(i) once P(i) is written; the two
//                       issuers' completions are signalled with
//                       tcgen05.commit on mbarriers.
//   warps 2-9           softmax and epilogue in two column groups of four
//                       warps: one cache row (then one output column) and
//                       half of the heads per thread.  The reference max per
//                       head is set from the first tile of a segment and only
//                       moved when some logit exceeds it by more than 8 (a
//                       factor 256 in exp2); only then do the warps reduce
//                       column maxima and rescale O in tensor memory.
//                       P = exp2(s - m) goes to shared memory in bf16, per-head
//                       sums stay in registers; a finished segment's O is
//                       stored straight from the tensor-memory registers.
// Every wait is bounded (one second); on expiry the kernel sets
// MQA_FLAG_PIPE_TIMEOUT, drains its own copies and MMAs, frees its tensor
// memory and returns.
#include <atomic>
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace mqa {

namespace {

using namespace sm100;

constexpr int kTile = 128;                   // cache rows per tile (the MMA M)
constexpr int kThreads = 384;                // warp 0 K/Q loads, warp 1 S products, warps 2-9 softmax, warp 10 V loads,
                                             // warp 11 P.V products
constexpr int kVWarp = 10;
constexpr int kPvWarp = 11;
constexpr int kNpv = 64;                     // N of the P.V product (P padded with zero columns)
constexpr uint32_t kHalfBytes = kTile * 128; // 128 rows x 64 bf16, one 128-byte swizzle column
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr float kRescaleThreshold = 8.f;     // log2 units
constexpr int kSegUnits = 4;                 // cost of entering a segment, in quarter tiles (partition weight)
constexpr int kLensCache = kThreads;         // clamped lengths kept in shared memory (all of them when b <= kThreads)
constexpr uint32_t kTmemCols = 256;          // S double buffer at [0, 2*NP), O double buffer at [128, 256)
constexpr uint32_t kOCol = 128;
constexpr uint32_t kMaxDynSmem = 232448;     // 227 KB opt-in limit per CTA

template <int NP, int SK, int SV, int DK, int DV>
struct TcCfg {
  // barriers
  static constexpr int kKFull = 0, kKEmpty = SK, kVFull = 2 * SK, kVEmpty = 2 * SK + SV, kSFull = 2 * SK + 2 * SV,
                       kSEmpty = kSFull + 2, kPFull = kSEmpty + 2, kOFull = kPFull + 1, kQFull = kOFull + 1,
                       kQEmpty = kQFull + 2, kOFree = kQEmpty + 2, kDone = kOFree + 2, kNumBars = kDone + 1;
  // head sizes: keys of DK and values of DV columns, each 64 or 128, stored as
  // one or two 64-column halves of 128-byte swizzled rows
  static_assert((DK == 64 || DK == 128) && (DV == 64 || DV == 128), "head sizes 64 and 128");
  static constexpr int kKHalves = DK / 64, kVHalves = DV / 64;
  // Head size 64 with at most 32 heads per group: a tile is 256 rows, two
  // 128-row halves.  Both halves' S products land side by side in tensor
  // memory (the second at column kNpv/2), their P rows share the P buffer's
  // lines, and one P.V product takes V's two row halves as the two 64-row
  // halves of its M = 128, so a 256-row tile costs the MMAs of a 128-row tile
  // at head size 128.  The second half's output is in lanes 64-127 at columns
  // kNpv/2 + head and is added to the first's in the epilogue.
  static constexpr bool kPair = DK == 64 && DV == 64 && NP <= kNpv / 2;
  static constexpr int kRowHalves = kPair ? 2 : 1;
  static constexpr int kRows = kRowHalves * kTile;             // cache rows per tile
  static constexpr uint32_t kSStride = kPair ? kNpv : NP;      // tensor-memory columns per S buffer
  static constexpr uint32_t kKTileBytes = kRowHalves * kKHalves * kHalfBytes,
                            kVTileBytes = kRowHalves * kVHalves * kHalfBytes;
  // shared memory
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + SK * kKTileBytes;
  static constexpr uint32_t kQ = kV + SV * kVTileBytes;
  static constexpr uint32_t kQBytes = NP * 128 * kKHalves;    // DK/64 64-column halves of NP rows
  static constexpr uint32_t kP = kQ + 2 * kQBytes;
  static constexpr uint32_t kPBytes = kTile * 128;             // 128 rows x 64 heads (bf16)
  static constexpr uint32_t kBar = kP + kPBytes;
  static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
  static constexpr uint32_t kFlag = kTmemSlot + 4;
  static constexpr uint32_t kAbort = kFlag + 4;
  static constexpr uint32_t kRed = (kAbort + 4 + 15) / 16 * 16;  // [4][NP] f32
  static constexpr uint32_t kMref = kRed + 4 * NP * 4;
  static constexpr uint32_t kAlpha = kMref + NP * 4;
  static constexpr uint32_t kRedL = kAlpha + NP * 4;             // [4][NP] f32: per-warp head sums
  static constexpr uint32_t kLinv = kRedL + 4 * NP * 4;          // [2][NP]: 1 / l per segment parity
  static constexpr uint32_t kLse = kLinv + 2 * NP * 4;           // [2][NP]: log2-sum-exp per segment parity
  static constexpr uint32_t kLens = kLse + 2 * NP * 4;          // [kLensCache] clamped lengths from seq0
  static constexpr uint32_t kKIssued = kLens + kLensCache * 4;   // K tiles issued so far (V producer trails it)
  static constexpr uint32_t kSched = kKIssued + 16;            // start-up scratch of the schedule
  static constexpr uint32_t kNsuf = kSched + 256;              // [kLensCache] beams: suffix tiles per sequence
  static constexpr uint32_t kX = kNsuf + kLensCache * 4;       // [NP][64] f32: second row half's output
  static constexpr uint32_t kEnd = kX + (kPair ? NP * 64 * 4 : 0);
  static constexpr uint32_t kAlloc = kEnd + 1024;             // room to align the base to 1024 bytes
  static_assert(kQ % 1024 == 0 && kP % 1024 == 0 && kQBytes % 1024 == 0, "swizzle atoms need 1024-byte alignment");
  static_assert(kAlloc <= kMaxDynSmem, "shared memory budget");
  static_assert((2 * (kThreads / 32) + 8) * 8 <= 256, "schedule scratch");
  static_assert(kSched % 8 == 0, "schedule scratch alignment");
  static_assert(kLens % 4 == 0, "lens table alignment");
};

__device__ __forceinline__ void named_barrier_softmax() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Barriers of the four softmax warps that also reduce a per-thread flag, so
// that every thread takes the same branch afterwards (a thread that gave up a
// bounded wait alone would otherwise leave the others blocked).
__device__ __forceinline__ bool softmax_barrier_and(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, 1, 256, pi;\n\t"
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
      "bar.red.or.pred po, 1, 256, pi;\n\t"
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
  const int* lens_s;         // clamped lens[seq0 + i], i < kLensCache (global memory beyond that)
  const int* nsuf_s;         // beams: suffix tiles of sequence i < kLensCache, or nullptr
  int seq0;                  // 0 when the whole batch is in the table
};

// Clamped length of sequence s: from shared memory (the whole batch when it
// has at most kLensCache sequences, else the CTA's first ones).  Under the
// start-up flood of TMA loads a dependent global load here would stall the
// role that needs it for thousands of cycles.
__device__ __forceinline__ int seq_len(const DecodeArgs& a, const Roles& r, int s) {
  const int i = s - r.seq0;
  if (i >= 0 && i < kLensCache) return r.lens_s[i];
  return clamp_len(__ldg(a.lens + s), a.m_max, nullptr, false);
}

__device__ __forceinline__ bool wait_bar(const Roles& r, uint32_t bar, uint32_t parity) {
  if (mbar_wait(bar, parity, kTimeoutNs)) return true;
  *r.abort = 1;
  set_flag(r.flags, MQA_FLAG_PIPE_TIMEOUT);
  return false;
}

// Beams sharing a prefix in one pass: the suffixes of the segment's sequence.
__device__ __forceinline__ BeamSuffixes beam_suffixes(const DecodeArgs& a) {
  BeamSuffixes bs;
  bs.slens = a.slens;
  bs.W = a.q_beams;
  bs.m_s = a.m_s;
  return bs;
}

// Cache rows of tile k of sequence seq: tile k of its attended span (k < nbp),
// or, with beams sharing a prefix (kFB), a tile of one beam's suffix, the
// beams' suffixes following the prefix in beam order.
template <bool kFB>
__device__ __forceinline__ void locate_tile(const DecodeArgs& a, int seq, int k, int len, int lo, int nbp,
                                            TileCoord& tc) {
  if (!kFB || k < nbp) {
    tc.beam = -1;
    tc.row0 = lo + k * kTile;
    tc.rows = min(kTile, len - tc.row0);
    tc.src_row = seq * a.m_max + tc.row0;
    return;
  }
  int kk = k - nbp;
  for (int w = 0; w < a.q_beams; ++w) {
    const int ls = clamp_len(__ldg(a.slens + seq * a.q_beams + w), a.m_s, nullptr, false);
    const int t = tiles_of(ls, kTile);
    if (kk < t) {
      tc.beam = w;
      tc.row0 = kk * kTile;
      tc.rows = min(kTile, ls - tc.row0);
      tc.src_row = (seq * a.q_beams + w) * a.m_s + tc.row0;
      return;
    }
    kk -= t;
  }
  tc.beam = 0;   // k beyond the segment: not reached
  tc.row0 = 0;
  tc.rows = 0;
  tc.src_row = 0;
}

// Walks the CTA's tiles in order and tells each role what a tile is.  Only
// the first step divides; later steps count (tile, head, sequence) forward.
// It also tracks the partition units, so that the owner of any tile can be
// computed.
template <bool kFB, int R>
struct TileWalk {
  int64_t t;                 // current tile number
  int64_t base;              // first tile of the current sequence
  int64_t ubase;             // first partition unit of the current sequence
  int seq, head, k, nb, len;
  int lo;                    // first attended row of the sequence (len - span)
  int nbp;                   // tiles of the attended span (the prefix, with beams)
  int sidx;                  // segment number within this CTA
  TileCoord tc;
  bool first, last;
  const Roles* rr;
  __device__ TileWalk(const DecodeArgs& a, const WSched& ws, const Roles& r) : t(ws.s.t_begin - 1), sidx(-1), rr(&r) {
    seq = ws.s.seq;
    base = ws.s.seq_base;
    ubase = ws.seq_ubase;
    set_seq(a, r, seq);
    while (ws.s.t_begin >= base + int64_t(a.g) * nb) {   // the first tile may lie in a later sequence
      base += int64_t(a.g) * nb;
      ubase += seq_units(nb, a.g, kSegUnits);
      set_seq(a, r, seq + 1);
    }
    const int rel = int(ws.s.t_begin - base);   // < g * nb
    head = rel / nb;
    k = rel - head * nb - 1;                     // next() advances to the first tile
  }
  __device__ void set_seq(const DecodeArgs& a, const Roles& r, int s) {
    seq = s;
    len = seq_len(a, r, s);
    lo = len - span_of(len, a.window);
    nb = tiles_of(len - lo, R);
    if constexpr (kFB) {
      nbp = nb;
      nb += r.nsuf_s != nullptr && s < kLensCache ? r.nsuf_s[s]
                                                 : suffix_tiles(beam_suffixes(a), s, kTile, nullptr, false);
    }
  }
  __device__ void next(const DecodeArgs& a, const Sched& sc) {
    ++t;
    if (++k == nb) {
      k = 0;
      if (++head == a.g) {
        head = 0;
        base += int64_t(a.g) * nb;
        ubase += seq_units(nb, a.g, kSegUnits);
        do {
          set_seq(a, *rr, seq + 1);
        } while (nb == 0);
      }
    }
    tc.seq = seq;
    tc.head = head;
    tc.k = k;
    if constexpr (kFB) {
      locate_tile<kFB>(a, seq, k, len, lo, nbp, tc);
    } else {
      tc.row0 = lo + k * R;
      tc.rows = min(R, len - tc.row0);
    }
    tc.seg = int64_t(seq) * a.g + head;
    tc.nb = nb;
    tc.seg_t0 = base + int64_t(head) * nb;
    first = (t == sc.t_begin) || k == 0;
    last = (k == nb - 1) || (t + 1 == sc.t_end);
    if (first) ++sidx;
  }
  // partition unit where the current segment's last tile starts
  __device__ int64_t seg_last_unit() const {
    return ubase + int64_t(head) * (kSegUnits + 4 * int64_t(nb)) + kSegUnits + 4 * int64_t(nb - 1);
  }
};

// Q of segment (seq, head) into a Q buffer (two 64-column halves of NP rows):
// rows seq*h + head*hq.. of the 2-D map (d, b*h), or with beams the W beams'
// q_group_heads heads of the group through the 3-D map (d, h, b*W).
template <int DK>
__device__ __forceinline__ void load_q(const DecodeArgs& a, const CUtensorMap* tm_q, uint32_t qdst, uint32_t bar,
                                       int seq, int head, int np) {
  constexpr int kHalves = DK / 64;
  if (a.q_beams > 0) {
    const uint64_t pol = l2_evict_first_policy();
    mbar_expect_tx(bar, uint32_t(kHalves) * uint32_t(a.hq) * 128u);
#pragma unroll
    for (int hf = 0; hf < kHalves; ++hf)
      tma_load_3d(qdst + hf * np * 128, tm_q, bar, 64 * hf, head * a.q_group_heads, seq * a.q_beams, pol);
  } else {
    mbar_expect_tx(bar, uint32_t(kHalves) * uint32_t(np) * 128u);
    const int qrow = seq * a.h + head * a.hq;
#pragma unroll
    for (int hf = 0; hf < kHalves; ++hf) tma_load_2d(qdst + hf * np * 128, tm_q, bar, 64 * hf, qrow);
  }
}

// One K or V tile: RH x W/64 boxes of 64 columns x 128 rows, one per row
// half and column half, row half major.
template <int W, int RH>
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar, int head, int row,
                                          uint64_t pol) {
  mbar_expect_tx(bar, uint32_t(RH * (W / 64)) * kHalfBytes);
#pragma unroll
  for (int rh = 0; rh < RH; ++rh)
#pragma unroll
    for (int hf = 0; hf < W / 64; ++hf)
      tma_load_3d(dst + (rh * (W / 64) + hf) * kHalfBytes, map, bar, 64 * hf, head, row + rh * kTile, pol);
}

// Fused append: write the step's new row of (sequence, K/V head) into the
// cache at row len-1, then order that store before the tensor-memory-access
// read of the same row.
template <int D>
__device__ __forceinline__ void append_new_row(const DecodeArgs& a, bool is_k, int seq, int head, int len) {
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(is_k ? a.k_new : a.v_new) +
                                                    (int64_t(seq) * a.g + head) * D);
  uint4* cache = reinterpret_cast<uint4*>(const_cast<__nv_bfloat16*>(
      static_cast<const __nv_bfloat16*>(is_k ? a.k : a.v) + ((int64_t(seq) * a.m_max + (len - 1)) * a.g + head) * D));
  uint4 tmp[D / 8];
#pragma unroll
  for (int c = 0; c < D / 8; ++c) tmp[c] = __ldg(src + c);
#pragma unroll
  for (int c = 0; c < D / 8; ++c) cache[c] = tmp[c];
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Loads of the CTA's first tiles, issued by the schedule thread that finds
// them: Q of the segment into Q buffer 0 and the first min(2, own) K and V
// tiles into stages 0 and 1 (K before V, as the producers order them).
// Returns the number of tiles started; the producers skip those.
template <int NP, int SK, int SV, int DK, int DV, bool kFB>
__device__ int pre_issue(const DecodeArgs& a, const Roles& r, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                         const CUtensorMap* tm_q, const CUtensorMap* tm_sk, const CUtensorMap* tm_sv, int seq,
                         int head, int k0, int own, int len, int nb) {
  using C = TcCfg<NP, SK, SV, DK, DV>;
  static_assert(SK >= 2 && SV >= 2, "two stages of each ring");
  auto bar = [&](int id) { return r.sbase + C::kBar + 8u * id; };
  const uint64_t pol = l2_evict_first_policy();
  load_q<DK>(a, tm_q, r.sbase + C::kQ, bar(C::kQFull), seq, head, NP);
  const int npre = own < 2 ? own : 2;
  for (int i = 0; i < npre; ++i) {
    const int k = k0 + i;
    if (a.k_new != nullptr && k == nb - 1) {
      append_new_row<DK>(a, true, seq, head, len);
      append_new_row<DV>(a, false, seq, head, len);
    }
    int row;
    const CUtensorMap* mk = tm_k;
    const CUtensorMap* mv = tm_v;
    if constexpr (kFB) {
      const int lo = len - span_of(len, a.window);
      TileCoord tc;
      locate_tile<kFB>(a, seq, k, len, lo, tiles_of(len - lo, kTile), tc);
      row = tc.src_row;
      if (tc.beam >= 0) {
        mk = tm_sk;
        mv = tm_sv;
      }
    } else {
      row = seq * a.m_max + len - span_of(len, a.window) + k * C::kRows;
    }
    load_tile<DK, C::kRowHalves>(r.sbase + C::kK + i * C::kKTileBytes, mk, bar(C::kKFull + i), head, row, pol);
    load_tile<DV, C::kRowHalves>(r.sbase + C::kV + i * C::kVTileBytes, mv, bar(C::kVFull + i), head, row, pol);
  }
  return npre;
}

// K ring and the per-segment Q (kIsK), or the V ring.
template <int NP, int SK, int SV, int DK, int DV, bool kIsK, bool kFB>
__device__ void producer(const DecodeArgs& a, const WSched& ws, const Roles& r, const CUtensorMap* tm_kv,
                         const CUtensorMap* tm_q, const CUtensorMap* tm_skv) {
  using C = TcCfg<NP, SK, SV, DK, DV>;
  const Sched& sc = ws.s;
  constexpr int S = kIsK ? SK : SV;
  constexpr int kFull = kIsK ? C::kKFull : C::kVFull;
  constexpr int kEmpty = kIsK ? C::kKEmpty : C::kVEmpty;
  constexpr uint32_t kRing = kIsK ? C::kK : C::kV;
  auto bar = [&](int id) { return r.sbase + C::kBar + 8u * id; };
  const uint64_t pol = l2_evict_first_policy();
  TileWalk<kFB, C::kRows> w(a, ws, r);
  const int64_t n = sc.t_end - sc.t_begin;
  int64_t i = 0;
  int q_issued = -1;
  const int64_t pre = ws.pre;   // tiles (and the first Q) the schedule already loads
  for (; i < n; ++i) {
    w.next(a, sc);
    if (*r.abort) break;
    if (i < pre) {
      if (kIsK) {
        q_issued = 0;
        *reinterpret_cast<volatile int*>(r.smem + C::kKIssued) = int(i + 1);
      }
      continue;
    }
    if (kIsK && w.first) {
      const int qb = w.sidx & 1;
      if (w.sidx >= 2 && !wait_bar(r, bar(C::kQEmpty + qb), ((w.sidx >> 1) - 1) & 1)) break;
      load_q<DK>(a, tm_q, r.sbase + C::kQ + qb * C::kQBytes, bar(C::kQFull + qb), w.tc.seq, w.tc.head, NP);
      q_issued = w.sidx;
    }
    const int st = int(i % S);
    if (i >= S && !wait_bar(r, bar(kEmpty + st), uint32_t((i / S) - 1) & 1)) break;
    if (!kIsK) {   // never run ahead of the K producer: the loads go out K(0), V(0), K(1), ...
      volatile int* k_issued = reinterpret_cast<volatile int*>(r.smem + C::kKIssued);
      uint32_t polls = 0;
      while (*k_issued <= i && !*r.abort) {
        if ((++polls & 1023u) == 0 && polls > (1u << 24)) break;   // cannot stall for good: K gives up on abort
      }
    }
    int row;
    const CUtensorMap* map = tm_kv;
    if constexpr (kFB) {
      row = w.tc.src_row;
      if (w.tc.beam >= 0) map = tm_skv;
    } else {
      row = w.tc.seq * a.m_max + w.tc.row0;
    }
    constexpr int kW = kIsK ? DK : DV;
    const uint32_t dst = r.sbase + kRing + st * (kIsK ? C::kKTileBytes : C::kVTileBytes);
    if (a.k_new != nullptr && w.tc.k == w.tc.nb - 1)   // this tile holds the sequence's newest row
      append_new_row<kW>(a, kIsK, w.tc.seq, w.tc.head, w.len);
    load_tile<kW, C::kRowHalves>(dst, map, bar(kFull + st), w.tc.head, row, pol);
    if (kIsK) *reinterpret_cast<volatile int*>(r.smem + C::kKIssued) = int(i + 1);
  }
  // Drain: every copy this thread issued has landed before the CTA can exit.
  for (int64_t j = (i - S > 0 ? i - S : 0); j < i; ++j)
    mbar_wait(bar(kFull + int(j % S)), uint32_t(j / S) & 1, kTimeoutNs);
  if (kIsK)
    for (int sq = (q_issued - 1 > 0 ? q_issued - 1 : 0); sq <= q_issued; ++sq)
      mbar_wait(bar(C::kQFull + (sq & 1)), uint32_t(sq >> 1) & 1, kTimeoutNs);
}

// Two threads issue the tensor-core products, each in a warp of its own: one
// the S = K Q^T stream, one the O += V^T P stream.  A thread issuing
// tcgen05.mma spends tens of cycles on each instruction and more on noticing
// the event that enables it, so one thread serving both streams set the tile
// period by itself; split, the P.V chain the softmax waits on only carries its
// own products.  tcgen05.commit tracks the products of the committing thread,
// so each stream releases its own ring stages.
//
// S(j) needs K(j) landed, for a segment's first tile its Q, and S buffer j&1
// free: the softmax warps arrive on SEmpty once they hold S(j-2) in registers.
template <int NP, int SK, int SV, int DK, int DV, bool kFB>
__device__ void s_issuer(const DecodeArgs& a, const WSched& ws, const Roles& r) {
  using C = TcCfg<NP, SK, SV, DK, DV>;
  const Sched& sc = ws.s;
  constexpr uint32_t idesc_qk = idesc_bf16_f32(kTile, NP, 0, 0);
  const int n = int(sc.t_end - sc.t_begin);   // tiles of this CTA (fewer than 2^31)
  TileWalk<kFB, C::kRows> w(a, ws, r);
  const uint64_t kdesc0 = smem_desc_sw128(r.sbase + C::kK, 16, 1024);   // K-major, rows of 128 B
  const uint64_t qdesc0 = smem_desc_sw128(r.sbase + C::kQ, 16, 1024);
  const uint32_t bar0 = r.sbase + C::kBar;
  auto bar = [&](int id) { return bar0 + 8u * uint32_t(id); };
  int kst = 0;
  uint32_t kph = 0;   // ring stage of K(i) and the parity of its full barrier
  for (int i = 0; i < n; ++i) {
    w.next(a, sc);
    const int qb = w.sidx & 1;
    if (w.first && !wait_bar(r, bar(C::kQFull + qb), uint32_t(w.sidx >> 1) & 1)) break;
    if (!wait_bar(r, bar(C::kKFull + kst), kph)) break;
    if (i >= 2 && !wait_bar(r, bar(C::kSEmpty + (i & 1)), uint32_t((i >> 1) - 1) & 1)) break;
    tc_fence_after();
    // descriptors differ only in their start address (bits 0-13, 16-byte units)
    const uint64_t ka = kdesc0 + uint64_t((uint32_t(kst) * C::kKTileBytes) >> 4);
    const uint64_t qa = qdesc0 + uint64_t((uint32_t(qb) * C::kQBytes) >> 4);
    const uint32_t d = r.tmem + uint32_t(i & 1) * C::kSStride;
#pragma unroll
    for (int rh = 0; rh < C::kRowHalves; ++rh)
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk) {
        const uint32_t koff = ((rh * C::kKHalves + (kk >> 2)) * kHalfBytes + (kk & 3) * 32) >> 4;
        const uint32_t qoff = ((kk >> 2) * (NP * 128) + (kk & 3) * 32) >> 4;
        mma_bf16_ss(d + uint32_t(rh) * (kNpv / 2), ka + koff, qa + qoff, idesc_qk, kk > 0);
      }
    mma_commit(bar(C::kSFull + (i & 1)));
    mma_commit(bar(C::kKEmpty + kst));
    if (w.last) mma_commit(bar(C::kQEmpty + qb));
    if (++kst == SK) {
      kst = 0;
      kph ^= 1u;
    }
  }
  // every product issued above has completed before tensor memory is released
  mma_commit(bar(C::kDone));
  mbar_wait(bar(C::kDone), 0, kTimeoutNs);
}

// O += V^T P(j) needs P(j) written, V(j) landed and, for a segment's first
// tile, its O buffer released by the epilogue of the segment two back.
template <int NP, int SK, int SV, int DK, int DV, bool kFB>
__device__ void pv_issuer(const DecodeArgs& a, const WSched& ws, const Roles& r) {
  using C = TcCfg<NP, SK, SV, DK, DV>;
  const Sched& sc = ws.s;
  constexpr uint32_t idesc_pv = idesc_bf16_f32(kTile, kNpv, 1, 1);
  const int n = int(sc.t_end - sc.t_begin);
  TileWalk<kFB, C::kRows> w(a, ws, r);
  // MN-major V^T; its M (V columns) is always 128: with DV = 64 the second
  // 64-column atom points back at the first (leading offset 0), and the
  // duplicated half of O is never written out; with 256-row tiles it is the
  // second row half instead.
  const uint64_t vdesc0 = smem_desc_sw128(r.sbase + C::kV, DV == 128 || C::kPair ? kHalfBytes : 0u, 1024);
  const uint64_t pdesc0 = smem_desc_sw128(r.sbase + C::kP, kHalfBytes, 1024);   // MN-major P
  const uint32_t bar0 = r.sbase + C::kBar;
  auto bar = [&](int id) { return bar0 + 8u * uint32_t(id); };
  int vst = 0;
  uint32_t vph = 0;   // ring stage of V(i) and the parity of its full barrier
  for (int i = 0; i < n; ++i) {
    w.next(a, sc);
    const int ob = w.sidx & 1;
    if (!wait_bar(r, bar(C::kPFull), uint32_t(i & 1))) break;
    if (!wait_bar(r, bar(C::kVFull + vst), vph)) break;
    if (w.first && w.sidx >= 2 && !wait_bar(r, bar(C::kOFree + ob), uint32_t((w.sidx >> 1) - 1) & 1)) break;
    tc_fence_after();
    const uint64_t va = vdesc0 + uint64_t((uint32_t(vst) * C::kVTileBytes) >> 4);
    const uint32_t d = r.tmem + kOCol + uint32_t(ob) * kNpv;
    const uint32_t acc0 = w.first ? 0u : 1u;
#pragma unroll
    for (int kk = 0; kk < kTile / 16; ++kk)
      mma_bf16_ss(d, va + ((kk * 2048) >> 4), pdesc0 + ((kk * 2048) >> 4), idesc_pv, kk > 0 ? 1u : acc0);
    mma_commit(bar(C::kOFull));
    mma_commit(bar(C::kVEmpty + vst));
    if (++vst == SV) {
      vst = 0;
      vph ^= 1u;
    }
  }
  mma_commit(bar(C::kDone));
  mbar_wait(bar(C::kDone), 0, kTimeoutNs);
}

// The beam kernel keeps one thread for both streams: S(j) = K Q^T once K(j)
// (and a segment's Q) has landed and P(j-2) has been consumed (j <= i + 1),
// O += V^T P(i) once P(i) and V(i) are there; it polls both and issues
// whichever is ready, P.V first (the softmax waits on it before it can store
// the next P), with ring stages and phase parities advanced by increments.  (Its walker reads the suffix lengths of every beam; a copy per
// stream measured slower than one thread serving both.)
template <int NP, int SK, int SV, int DK, int DV, bool kFB>
__device__ void mma_issuer(const DecodeArgs& a, const WSched& ws, const Roles& r) {
  using C = TcCfg<NP, SK, SV, DK, DV>;
  const Sched& sc = ws.s;
  constexpr uint32_t idesc_qk = idesc_bf16_f32(kTile, NP, 0, 0);
  constexpr uint32_t idesc_pv = idesc_bf16_f32(kTile, kNpv, 1, 1);
  const int n = int(sc.t_end - sc.t_begin);
  static_assert(!(C::kPair && kFB), "one issuer: 128-row tiles");
  TileWalk<kFB, C::kRows> wq(a, ws, r), wp(a, ws, r);
  const uint64_t kdesc0 = smem_desc_sw128(r.sbase + C::kK, 16, 1024);
  const uint64_t qdesc0 = smem_desc_sw128(r.sbase + C::kQ, 16, 1024);
  const uint64_t vdesc0 = smem_desc_sw128(r.sbase + C::kV, DV == 128 ? kHalfBytes : 0u, 1024);
  const uint64_t pdesc0 = smem_desc_sw128(r.sbase + C::kP, kHalfBytes, 1024);
  const uint32_t bar0 = r.sbase + C::kBar;
  auto bar = [&](int id) { return bar0 + 8u * uint32_t(id); };
  int iq = 0, ip = 0, kst = 0, vst = 0;
  uint32_t kph = 0, vph = 0;
  if (n > 0) {
    wq.next(a, sc);
    wp.next(a, sc);
  }
  uint64_t idle_since = 0;
  uint32_t idle_polls = 0;
  while (ip < n) {
    bool progressed = false;
    if (ip < iq) {
      const int ob = wp.sidx & 1;
      if (mbar_test(bar(C::kPFull), uint32_t(ip & 1)) && mbar_test(bar(C::kVFull + vst), vph) &&
          (!wp.first || wp.sidx < 2 || mbar_test(bar(C::kOFree + ob), uint32_t((wp.sidx >> 1) - 1) & 1))) {
        tc_fence_after();
        const uint64_t va = vdesc0 + uint64_t((uint32_t(vst) * C::kVTileBytes) >> 4);
        const uint32_t d = r.tmem + kOCol + uint32_t(ob) * kNpv;
        const uint32_t acc0 = wp.first ? 0u : 1u;
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_bf16_ss(d, va + ((kk * 2048) >> 4), pdesc0 + ((kk * 2048) >> 4), idesc_pv, kk > 0 ? 1u : acc0);
        mma_commit(bar(C::kOFull));
        mma_commit(bar(C::kVEmpty + vst));
        ++ip;
        if (++vst == SV) {
          vst = 0;
          vph ^= 1u;
        }
        if (ip < n) wp.next(a, sc);
        progressed = true;
      }
    }
    if (iq < n && iq <= ip + 1) {
      const int qb = wq.sidx & 1;
      if ((!wq.first || mbar_test(bar(C::kQFull + qb), uint32_t(wq.sidx >> 1) & 1)) &&
          mbar_test(bar(C::kKFull + kst), kph)) {
        tc_fence_after();
        const uint64_t ka = kdesc0 + uint64_t((uint32_t(kst) * C::kKTileBytes) >> 4);
        const uint64_t qa = qdesc0 + uint64_t((uint32_t(qb) * C::kQBytes) >> 4);
        const uint32_t d = r.tmem + uint32_t(iq & 1) * NP;
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint32_t koff = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
          const uint32_t qoff = ((kk >> 2) * (NP * 128) + (kk & 3) * 32) >> 4;
          mma_bf16_ss(d, ka + koff, qa + qoff, idesc_qk, kk > 0);
        }
        mma_commit(bar(C::kSFull + (iq & 1)));
        mma_commit(bar(C::kKEmpty + kst));
        if (wq.last) mma_commit(bar(C::kQEmpty + qb));
        ++iq;
        if (++kst == SK) {
          kst = 0;
          kph ^= 1u;
        }
        if (iq < n) wq.next(a, sc);
        progressed = true;
      }
    }
    if (progressed) {
      idle_polls = 0;
    } else if ((++idle_polls & 1023u) == 0) {   // bounded: give up after the timeout without progress
      const uint64_t now = globaltimer_ns();
      if (idle_polls == 1024) {
        idle_since = now;
      } else if (now - idle_since > kTimeoutNs || *r.abort) {
        *r.abort = 1;
        set_flag(r.flags, MQA_FLAG_PIPE_TIMEOUT);
        break;
      }
    }
  }
  mma_commit(bar(C::kDone));
  mbar_wait(bar(C::kDone), 0, kTimeoutNs);
}

template <int NP, int SK, int SV, int DK, int DV, bool kFB>
__device__ void softmax_epilogue(const DecodeArgs& a, const WSched& ws, const Roles& r, int warp, int lane) {
  using C = TcCfg<NP, SK, SV, DK, DV>;
  const Sched& sc = ws.s;
  auto bar = [&](int id) { return r.sbase + C::kBar + 8u * id; };
  auto wait = [&](int id, uint32_t parity) { return mbar_wait(bar(id), parity, kTimeoutNs); };
  constexpr int CPT = NP / 2;                      // heads per thread: two warps share each row
  constexpr int W = CPT < 16 ? CPT : 16;           // transpose-reduction width
  const int q4 = warp & 3;                         // TMEM lane quarter this warp may access
  const int grp = (warp - 2) >> 2;                 // column group: heads [grp*CPT, grp*CPT + CPT)
  const int gw = (warp - 2) & 3;                   // warp index within the column group
  const int col0 = grp * CPT;
  const int tid = threadIdx.x - 64;                // 0..255 over the softmax warps
  const int row = 32 * q4 + lane;                  // cache row of the tile (S), output column (O)
  const uint32_t t_lane = r.tmem + (uint32_t(32 * q4) << 16);
  float* red = reinterpret_cast<float*>(r.smem + C::kRed);      // [4][NP]
  float* mref = reinterpret_cast<float*>(r.smem + C::kMref);
  float* alpha = reinterpret_cast<float*>(r.smem + C::kAlpha);
  float* redl = reinterpret_cast<float*>(r.smem + C::kRedL);    // [4][NP]
  float* linv = reinterpret_cast<float*>(r.smem + C::kLinv);
  float* lse2 = reinterpret_cast<float*>(r.smem + C::kLse);
  const float c = a.scale * kLog2e;
  const int hq = a.hq;
  constexpr bool kPair = C::kPair;                 // 256-row tiles: this thread also takes row `row` + 128
  const uint32_t o_col = kOCol + (kPair && q4 >= 2 ? kNpv / 2 : 0);   // this lane's block of O
  float lpart[CPT];                                // this row's share of the per-head sums
  float sv[CPT];                                   // this row's scaled logits (log2 units)
  float sv2[CPT];                                  // the same for row `row` + 128 (256-row tiles)
  float mr[CPT];                                   // reference max per head, mirrored from smem
  {   // zero the P buffer: its pad columns must read as zero
    uint4* p = reinterpret_cast<uint4*>(r.smem + C::kP);
    for (int k = tid; k < int(C::kPBytes / 16); k += 256) p[k] = make_uint4(0, 0, 0, 0);
    named_barrier_softmax();
  }
  TileWalk<kFB, C::kRows> w(a, ws, r);
  const int64_t n = sc.t_end - sc.t_begin;
  int64_t pv_waited = -1;
  bool failed = false;

  // A finished segment whose output is written one tile later, once the P.V
  // product of its last tile is known to have completed.
  struct Pending {
    bool on;
    int sidx, seq, head;
    int64_t seg;
    bool whole, owns_first;
    int64_t seg_last_unit;   // partition unit where the segment's last tile starts
  } pend;
  pend.on = false;

  // Write a finished segment: O^T from tensor memory times 1/l.  Thread `row`
  // holds output column `row` of its CPT heads, so for each head the 32 lanes
  // of a warp store 32 consecutive columns (128 bytes of fp32 partial, 64 of
  // bf16 output) straight from registers; then the O buffer is released.
  auto epilogue = [&](const Pending& e) {
    const int pb = e.sidx & 1;
    const int64_t slot = partial_slot(blockIdx.x, e.seg);
    float v[CPT];
    tmem_ld<CPT>(t_lane + o_col + uint32_t(pb) * kNpv + col0, v);
    if constexpr (kPair) {   // add the second row half's product (lanes 64-127) to the first's
      float* xb = reinterpret_cast<float*>(r.smem + C::kX);   // [NP][64]
      if (row >= 64)
#pragma unroll
        for (int k = 0; k < CPT; ++k) xb[(col0 + k) * 64 + row - 64] = v[k];
      named_barrier_softmax();
      if (row < 64)
#pragma unroll
        for (int k = 0; k < CPT; ++k) v[k] += xb[(col0 + k) * 64 + row];
    }
    if (row >= DV) {
      // columns past DV only repeat the first ones (see the P.V descriptor)
    } else if (e.whole) {
      if constexpr (kFB) {   // column (w, i) of the segment is head i of the group in beam w's output row
        const int qgh = a.q_group_heads;
        int bw = col0 / qgh, bi = col0 - bw * qgh;
#pragma unroll
        for (int k = 0; k < CPT; ++k) {
          if (col0 + k < hq)
            static_cast<__nv_bfloat16*>(a.o)[((int64_t(e.seq) * a.q_beams + bw) * a.h + int64_t(e.head) * qgh + bi) *
                                                 DV + row] = __float2bfloat16_rn(v[k] * linv[pb * NP + col0 + k]);
          if (++bi == qgh) {
            bi = 0;
            ++bw;
          }
        }
      } else {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.o) +
                             (int64_t(e.seq) * a.h + int64_t(e.head) * hq + col0) * DV + row;
#pragma unroll
        for (int k = 0; k < CPT; ++k)
          if (col0 + k < hq) dst[k * DV] = __float2bfloat16_rn(v[k] * linv[pb * NP + col0 + k]);
      }
    } else {
      float* dst = a.ws.part_o + (slot * hq + col0) * DV + row;
#pragma unroll
      for (int k = 0; k < CPT; ++k)
        if (col0 + k < hq) dst[k * DV] = v[k] * linv[pb * NP + col0 + k];
    }
    if (warp == 2) {
      if (!e.whole)   // every partial carries its log-sum-exp
        for (int col = lane; col < hq; col += 32) a.ws.part_lse[slot * hq + col] = lse2[pb * NP + col];
      if (e.owns_first && lane == 0)
        a.ws.seg_info[e.seg] = make_int2(blockIdx.x, cta_of_unit(e.seg_last_unit, ws.wtotal, sc.active));
    }
    tc_fence_before();
    mbar_arrive(bar(C::kOFree + pb));
  };

  for (int64_t i = 0; i < n; ++i) {
    w.next(a, sc);
    if (w.first) {
#pragma unroll
      for (int k = 0; k < CPT; ++k) lpart[k] = 0.f;
    }
    bool ok = wait(C::kSFull + (i & 1), uint32_t(i >> 1) & 1);
    tc_fence_after();
    const bool valid = row < w.tc.rows;
    if constexpr (kPair)
      tmem_ld_two<CPT>(t_lane + uint32_t(i & 1) * C::kSStride + col0,
                       t_lane + uint32_t(i & 1) * C::kSStride + kNpv / 2 + col0, sv, sv2);
    else
      tmem_ld<CPT>(t_lane + uint32_t(i & 1) * NP + col0, sv);
    tc_fence_before();
    mbar_arrive(bar(C::kSEmpty + (i & 1)));   // S buffer i&1 may take S(i+2)
#pragma unroll
    for (int k = 0; k < CPT; ++k) sv[k] = valid ? sv[k] * c : -INFINITY;
    if constexpr (kPair) {
      const bool valid2 = row + kTile < w.tc.rows;
#pragma unroll
      for (int k = 0; k < CPT; ++k) sv2[k] = valid2 ? sv2[k] * c : -INFINITY;
    }
    if constexpr (kFB) {
      if (w.tc.beam >= 0) {   // a beam's suffix tile counts for that beam's query columns only
        const int cb0 = w.tc.beam * a.q_group_heads, cb1 = cb0 + a.q_group_heads;
#pragma unroll
        for (int k = 0; k < CPT; ++k)
          if (col0 + k < cb0 || col0 + k >= cb1) sv[k] = -INFINITY;
      }
    }
    // Does any logit of a real head exceed the reference max by the threshold?
    bool exceed = false;
    if (!w.first) {
      float d[CPT];
#pragma unroll
      for (int k = 0; k < CPT; ++k) d[k] = (col0 + k < hq) ? (kPair ? fmaxf(sv[k], sv2[k]) : sv[k]) - mr[k] : -INFINITY;
#pragma unroll
      for (int span = CPT / 2; span >= 1; span >>= 1)
#pragma unroll
        for (int k = 0; k < span; ++k) d[k] = fmaxf(d[k], d[k + span]);
      exceed = d[0] > kRescaleThreshold;
    }
    const bool full = w.first || softmax_barrier_or(exceed);
    if (full) {   // column maxima of the tile and the new reference max
#pragma unroll
      for (int ch = 0; ch < CPT / W; ++ch) {
        float v[W];
#pragma unroll
        for (int k = 0; k < W; ++k) v[k] = kPair ? fmaxf(sv[ch * W + k], sv2[ch * W + k]) : sv[ch * W + k];
        const float mx = transpose_reduce<W, true>(v, lane);
        if (lane < W) red[gw * NP + col0 + ch * W + lane] = mx;
      }
      named_barrier_softmax();
      if (gw == 0) {   // one warp per column group decides for its heads
        for (int col = col0 + lane; col < col0 + CPT; col += 32) {
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
          // With beams a column may have no row yet: a finite floor keeps exp2(s - m) at 0
          // (s = -inf) instead of NaN, and the first real logit then exceeds it.
          mref[col] = kFB ? fmaxf(mn, -1e30f) : mn;
          alpha[col] = al;
        }
      }
      named_barrier_softmax();
#pragma unroll
      for (int k = 0; k < CPT; ++k) mr[k] = mref[col0 + k];
    }
    // P = exp2(s - m) in bf16, into registers before waiting for the previous
    // product: only the shared-memory store has to follow that wait.
    if (full && !w.first) {
#pragma unroll
      for (int k = 0; k < CPT; ++k) lpart[k] *= alpha[col0 + k];
    }
    uint32_t packed[CPT / 2], packed2[CPT / 2];
#pragma unroll
    for (int k2 = 0; k2 < CPT / 2; ++k2) {
      const int k = 2 * k2;
      const float p0 = col0 + k < hq ? ex2_approx(sv[k] - mr[k]) : 0.f;
      const float p1 = col0 + k + 1 < hq ? ex2_approx(sv[k + 1] - mr[k + 1]) : 0.f;
      lpart[k] += p0;
      lpart[k + 1] += p1;
      __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
      packed[k2] = *reinterpret_cast<uint32_t*>(&b2);
      if constexpr (kPair) {
        const float q0 = col0 + k < hq ? ex2_approx(sv2[k] - mr[k]) : 0.f;
        const float q1 = col0 + k + 1 < hq ? ex2_approx(sv2[k + 1] - mr[k + 1]) : 0.f;
        lpart[k] += q0;
        lpart[k + 1] += q1;
        __nv_bfloat162 c2 = __floats2bfloat162_rn(q0, q1);
        packed2[k2] = *reinterpret_cast<uint32_t*>(&c2);
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
    if (w.tc.rows < C::kRows) ok2 = wait(C::kVFull + st, uint32_t(i / SV) & 1) && ok2;
    if (!softmax_barrier_and(ok && ok2)) { failed = true; break; }
    tc_fence_after();
    if (full && !w.first) {
      // rescale the O accumulated so far (thread = output column, its heads)
      const uint32_t oc = t_lane + o_col + uint32_t(w.sidx & 1) * kNpv + col0;
      float v[CPT];
      tmem_ld<CPT>(oc, v);
#pragma unroll
      for (int k = 0; k < CPT; ++k) v[k] *= alpha[col0 + k];
      tmem_st<CPT>(oc, v);
      tmem_wait_st();
    }
    // P into the MN-major 128-byte-swizzled P buffer
    unsigned char* prow = r.smem + C::kP + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
    for (int c8 = 0; c8 < CPT / 8; ++c8) {
      const int chunk = col0 / 8 + c8;
      *reinterpret_cast<uint4*>(prow + ((chunk ^ (row & 7)) << 4)) =
          make_uint4(packed[c8 * 4], packed[c8 * 4 + 1], packed[c8 * 4 + 2], packed[c8 * 4 + 3]);
      if constexpr (kPair) {   // row + 128's P in the same line, kNpv/2 columns on
        const int chunk2 = (kNpv / 2 + col0) / 8 + c8;
        *reinterpret_cast<uint4*>(prow + ((chunk2 ^ (row & 7)) << 4)) =
            make_uint4(packed2[c8 * 4], packed2[c8 * 4 + 1], packed2[c8 * 4 + 2], packed2[c8 * 4 + 3]);
      }
    }
    if (w.tc.rows < C::kRows) {
      // rows past the sequence end were loaded too; zero them in V so that
      // P = 0 times whatever they hold contributes exactly 0.  Consecutive
      // threads take consecutive 16-byte pieces of a row (no bank conflicts).
      // A stage is [row half][column half][128 rows][128 bytes].
      unsigned char* vst = r.smem + C::kV + st * C::kVTileBytes;
      const int nchunks = (C::kRows - w.tc.rows) * 8 * C::kVHalves;
      for (int k = tid; k < nchunks; k += 256) {
        const int vr = w.tc.rows + k / (8 * C::kVHalves), half = (k >> 3) & (C::kVHalves - 1), c16 = k & 7;
        if constexpr (kPair) {
          const int vh = vr >> 7, vl = vr & 127;
          *reinterpret_cast<uint4*>(vst + vh * kHalfBytes + (vl >> 3) * 1024 + (vl & 7) * 128 + c16 * 16) =
              make_uint4(0, 0, 0, 0);
        } else {
          *reinterpret_cast<uint4*>(vst + half * kHalfBytes + (vr >> 3) * 1024 + (vr & 7) * 128 + c16 * 16) =
              make_uint4(0, 0, 0, 0);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(bar(C::kPFull));
    // The previous segment's output, now off the path to the next product: its
    // O buffer is final (its last product completed before the wait above) and
    // P.V(i) accumulates into the other buffer.
    if (pend.on) {
      epilogue(pend);
      pend.on = false;
    }

    if (w.last) {
      // per-head sums over the 128 rows; the output follows one tile later
#pragma unroll
      for (int ch = 0; ch < CPT / W; ++ch) {
        float v[W];
#pragma unroll
        for (int k = 0; k < W; ++k) v[k] = lpart[ch * W + k];
        const float sum = transpose_reduce<W, false>(v, lane);
        if (lane < W) redl[gw * NP + col0 + ch * W + lane] = sum;
      }
      named_barrier_softmax();
      const int pb = w.sidx & 1;
      if (gw == 0)
        for (int col = col0 + lane; col < col0 + CPT; col += 32) {
          const float l = redl[col] + redl[NP + col] + redl[2 * NP + col] + redl[3 * NP + col];
          linv[pb * NP + col] = kFB && !(l > 0.f) ? 0.f : rcp_approx(l);   // a beam with no rows here: o = 0
          lse2[pb * NP + col] = mref[col] + lg2_approx(l);
        }
      pend.on = true;
      pend.sidx = w.sidx;
      pend.seq = w.tc.seq;
      pend.head = w.tc.head;
      pend.seg = w.tc.seg;
      pend.owns_first = w.tc.seg_t0 >= sc.t_begin;
      pend.whole = pend.owns_first && (w.tc.seg_t0 + w.tc.nb <= sc.t_end);
      pend.seg_last_unit = w.seg_last_unit();
    }
  }
  if (!failed && pend.on) {   // the CTA's last segment: wait for its final P.V, then write it
    bool ok = true;
    if (pv_waited < n - 1) ok = wait(C::kOFull, uint32_t(n - 1) & 1);
    if (softmax_barrier_and(ok)) {
      tc_fence_after();
      epilogue(pend);
    } else {
      failed = true;
    }
  }
  if (failed && tid == 0) {
    *r.abort = 1;
    set_flag(r.flags, MQA_FLAG_PIPE_TIMEOUT);
  }
}

// One CTA per SM.  The warps of a CTA are spread over the SM's four
// sub-partitions of 16K registers each; with 12 warps three share one, which
// caps a thread at 168 registers.
template <int NP, int SK, int SV, int DK, int DV, bool kFB, bool kOne>
__device__ __forceinline__ void decode_tc_body(const DecodeArgs& a, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                               const CUtensorMap& tm_q, const CUtensorMap& tm_sk,
                                               const CUtensorMap& tm_sv) {
  using C = TcCfg<NP, SK, SV, DK, DV>;
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
      mbar_init(bar(C::kSEmpty + s), 256);
      mbar_init(bar(C::kQFull + s), 1);
      mbar_init(bar(C::kQEmpty + s), 1);
      mbar_init(bar(C::kOFree + s), 256);
    }
    mbar_init(bar(C::kPFull), 256);
    mbar_init(bar(C::kOFull), 1);
    mbar_init(bar(C::kDone), kFB ? 1 : 2);   // one commit from each issuing thread
    *r.abort = 0;
    *reinterpret_cast<int*>(r.smem + C::kKIssued) = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_q);
    if constexpr (kFB) {
      prefetch_tensormap(&tm_sk);
      prefetch_tensormap(&tm_sv);
    }
  }
  if (warp == 1) {
    tmem_alloc(r.sbase + C::kTmemSlot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();   // the block barriers of the schedule publish the slot
  }
  // Inputs may come from the kernel before this one on the stream (the append).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  int* lens_tab = reinterpret_cast<int*>(r.smem + C::kLens);
  r.lens_s = lens_tab;
  r.nsuf_s = nullptr;
  int64_t* sched_red = reinterpret_cast<int64_t*>(r.smem + C::kSched);
  WSched ws;
  BeamSuffixes bs;
  if constexpr (kFB) {
    bs = beam_suffixes(a);
  } else {
    bs.slens = nullptr;
    bs.W = 0;
    bs.m_s = 0;
  }
  if constexpr (kOne) {
    // Every attended span fits one tile and there are no more (sequence,
    // K/V head) segments than CTAs: CTA c takes segment c whole, its only
    // tile.  No scan: one length load, then at once the loads of the
    // segment's Q, K and V.
    const int c = blockIdx.x, nseg = a.b * a.g;
    const int seq = c < nseg ? c / a.g : 0, head = c < nseg ? c - seq * a.g : 0;
    if (threadIdx.x == 0) {
      const int len = c < nseg ? clamp_len(__ldg(a.lens + seq), a.m_max, a.flags, head == 0) : 0;
      lens_tab[0] = len;
      sched_red[0] = len > 0 ? pre_issue<NP, SK, SV, DK, DV, kFB>(a, r, &tm_k, &tm_v, &tm_q, &tm_sk, &tm_sv, seq, head,
                                                                 0, 1, len, 1)
                             : 0;
    }
    __syncthreads();
    const bool work = lens_tab[0] > 0;
    ws.s.total = nseg;
    ws.s.active = a.grid;
    ws.s.t_begin = work ? c : 0;   // numbered per sequence: segment (seq, head) is tile seq*g + head
    ws.s.t_end = work ? c + 1 : 0;
    ws.s.seq = seq;
    ws.s.seq_base = int64_t(seq) * a.g;
    ws.wtotal = 1;
    ws.seq_ubase = 0;
    ws.pre = int(sched_red[0]);
    r.seq0 = seq;   // lens_tab[0] holds this sequence's length
  } else if (small_schedule_fits(a.b, a.g, a.m_max, C::kRows, kThreads, kSegUnits,
                                 kFB ? int64_t(a.q_beams) * tiles_of(a.m_s, kTile) : 0)) {
    ws = make_schedule_small<kThreads>(
        a.lens, a.b, a.g, a.m_max, a.window, C::kRows, a.grid, blockIdx.x, a.flags, sched_red, kSegUnits, lens_tab, bs,
        kFB ? reinterpret_cast<int*>(r.smem + C::kNsuf) : nullptr,
        [&](int seq, int head, int k0, int own, int len, int nb) {
          return pre_issue<NP, SK, SV, DK, DV, kFB>(a, r, &tm_k, &tm_v, &tm_q, &tm_sk, &tm_sv, seq, head, k0, own, len, nb);
        });
    r.seq0 = 0;
    if (kFB) r.nsuf_s = reinterpret_cast<const int*>(r.smem + C::kNsuf);
  } else {
    ws = make_schedule_weighted<kThreads>(a.lens, a.b, a.g, a.m_max, a.window, C::kRows, a.grid, blockIdx.x, a.flags, sched_red,
                                          kSegUnits, bs);
    r.seq0 = ws.s.seq;
    if (threadIdx.x < kLensCache && ws.s.seq + int(threadIdx.x) < a.b)   // L1-resident: the schedule just read them
      lens_tab[threadIdx.x] = clamp_len(__ldg(a.lens + ws.s.seq + threadIdx.x), a.m_max, nullptr, false);
    __syncthreads();
  }
  const Sched& sc = ws.s;
  tc_fence_after();
  r.tmem = *reinterpret_cast<volatile uint32_t*>(r.smem + C::kTmemSlot);
  if (a.no_merge && warp >= 2 && warp < kVWarp) {   // no merge follows: empty sequences get their zero rows here
    for (int s = blockIdx.x; s < a.b; s += gridDim.x) {
      if (clamp_len(__ldg(a.lens + s), a.m_max, nullptr, false) == 0) {
        uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + int64_t(s) * a.h * DV);
        for (int k = int(threadIdx.x) - 64; k < a.h * DV / 8; k += 256) o[k] = make_uint4(0, 0, 0, 0);
      }
    }
  }

  if (sc.t_begin < sc.t_end) {
    if (warp == 0) {
      if (lane == 0) producer<NP, SK, SV, DK, DV, true, kFB>(a, ws, r, &tm_k, &tm_q, &tm_sk);
    } else if (warp == 1) {
      if (lane == 0) {
        if constexpr (kFB) mma_issuer<NP, SK, SV, DK, DV, kFB>(a, ws, r);
        else s_issuer<NP, SK, SV, DK, DV, kFB>(a, ws, r);
      }
    } else if (warp == kPvWarp) {
      if (!kFB && lane == 0) pv_issuer<NP, SK, SV, DK, DV, kFB>(a, ws, r);
    } else if (warp == kVWarp) {
      // V loads from a warp of their own: sharing one with the K loads would
      // serialise the two threads' waits
      if (lane == 0) producer<NP, SK, SV, DK, DV, false, kFB>(a, ws, r, &tm_v, &tm_q, &tm_sv);
    } else {
      softmax_epilogue<NP, SK, SV, DK, DV, kFB>(a, ws, r, warp, lane);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(r.tmem, kTmemCols);
  // The merge kernel may launch now (launching it earlier, to wait beside this
  // grid, measured slower).
  asm volatile("griddepcontrol.launch_dependents;");
}

template <int NP, int SK, int SV, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q) {
  decode_tc_body<NP, SK, SV, DK, DV, false, false>(a, tm_k, tm_v, tm_q, tm_k, tm_v);
}

// Single-tile spans with no more segments than CTAs: one segment per CTA.  A
// kernel of its own, so that the general kernel carries none of its code.
template <int NP, int SK, int SV, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_one_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q) {
  decode_tc_body<NP, SK, SV, DK, DV, false, true>(a, tm_k, tm_v, tm_q, tm_k, tm_v);
}

// Beams sharing a prefix in one pass: the suffix caches' maps as well.
template <int NP, int SK, int SV, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_beam_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_sk, const __grid_constant__ CUtensorMap tm_sv) {
  decode_tc_body<NP, SK, SV, DK, DV, true, false>(a, tm_k, tm_v, tm_q, tm_sk, tm_sv);
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

// Cache [b, m_max, g, d] bf16 (d = 64 or 128) as a 3-D tensor (d, g, b*m_max);
// a box is 64 columns of one K/V head over 128 consecutive rows, 128-byte
// swizzled.
bool encode_cache(CUtensorMap* m, const void* base, int b, int m_max, int g, int d) {
  const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(g), cuuint64_t(b) * cuuint64_t(m_max)};
  const cuuint64_t strides[2] = {cuuint64_t(d) * 2, cuuint64_t(g) * cuuint64_t(d) * 2};
  const cuuint32_t box[3] = {64, 1, kTile};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q [b*h, d_k] bf16; a box is 64 columns of NP consecutive heads.
// Beam queries [b*W, h, d] as (d, h, b*W) with boxes of 64 x heads x W.
bool encode_q_beams(CUtensorMap* m, const void* base, int h, int rows, int heads, int beams, int d) {
  const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(h), cuuint64_t(rows)};
  const cuuint64_t strides[2] = {cuuint64_t(d) * 2, cuuint64_t(h) * cuuint64_t(d) * 2};
  const cuuint32_t box[3] = {64, cuuint32_t(heads), cuuint32_t(beams)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_q(CUtensorMap* m, const void* base, int rows, int np, int d) {
  const cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(d) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(np)};
  const cuuint32_t estr[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NP, int SK, int SV, int DK, int DV, bool kFB>
cudaError_t launch_np(const DecodeArgs& a, cudaStream_t stream) {
  using L = TcCfg<NP, SK, SV, DK, DV>;
  const bool one = !kFB && a.no_merge && int64_t(a.b) * a.g <= a.grid;
  static std::atomic<bool> attr_set[2][64];   // per kernel and device; setting it twice is harmless
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[one][dev].load(std::memory_order_relaxed)) {
    if constexpr (kFB)
      e = cudaFuncSetAttribute(decode_tc_beam_kernel<NP, SK, SV, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(L::kAlloc));
    else
      e = one ? cudaFuncSetAttribute(decode_tc_one_kernel<NP, SK, SV, DK, DV>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, int(L::kAlloc))
              : cudaFuncSetAttribute(decode_tc_kernel<NP, SK, SV, DK, DV>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, int(L::kAlloc));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[one][dev].store(true, std::memory_order_relaxed);
  }
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  CUtensorMap tk, tv, tq, tsk, tsv;
  if (!encode_cache(&tk, a.k, a.b, a.m_max, a.g, DK) || !encode_cache(&tv, a.v, a.b, a.m_max, a.g, DV) ||
      !(a.q_beams > 0 ? encode_q_beams(&tq, a.q, a.h, a.b * a.q_beams, a.q_group_heads, a.q_beams, DK)
                      : encode_q(&tq, a.q, a.b * a.h, NP, DK)))
    return cudaErrorInvalidValue;
  if (kFB && (!encode_cache(&tsk, a.sk, a.b * a.q_beams, a.m_s, a.g, DK) ||
              !encode_cache(&tsv, a.sv, a.b * a.q_beams, a.m_s, a.g, DV)))
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
  if constexpr (kFB) return cudaLaunchKernelEx(&cfg, decode_tc_beam_kernel<NP, SK, SV, DK, DV>, a, tk, tv, tq, tsk, tsv);
  if (one) {   // one CTA per segment, none idle
    DecodeArgs a1 = a;
    a1.grid = a.b * a.g;
    cfg.gridDim = dim3(unsigned(a1.grid));
    return cudaLaunchKernelEx(&cfg, decode_tc_one_kernel<NP, SK, SV, DK, DV>, a1, tk, tv, tq);
  }
  return cudaLaunchKernelEx(&cfg, decode_tc_kernel<NP, SK, SV, DK, DV>, a, tk, tv, tq);
}

template <int SK, int SV, int DK, int DV>
cudaError_t launch_hq(const DecodeArgs& a, cudaStream_t stream) {
  if (a.hq <= 16) return launch_np<16, SK, SV, DK, DV, false>(a, stream);
  if (a.hq <= 32) return launch_np<32, SK, SV, DK, DV, false>(a, stream);
  if (a.hq <= 64) return launch_np<64, SK, SV, DK, DV, false>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

bool tc_supported(int d_k, int d_v, int hq) {
  return (d_k == 64 || d_k == 128) && (d_v == 64 || d_v == 128) && hq >= 1 && hq <= 64;
}

int tc_ctas_per_sm(int) { return 1; }

int tc_tile_rows() { return kTile; }

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream) {
  // (row coordinates of a tile's second half reach 256 rows past a tile start)
  if (int64_t(a.b) * a.m_max >= (int64_t(1) << 31) - 256 || int64_t(a.b) * a.h >= (int64_t(1) << 31))
    return cudaErrorInvalidValue;
  if (a.sk != nullptr) {   // beams sharing a prefix, one pass (head size 128)
    if (a.q_beams < 1 || int64_t(a.b) * a.q_beams * a.m_s >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
    if (a.dk != 128 || a.d != 128) return cudaErrorInvalidValue;
    if (a.hq <= 16) return launch_np<16, 2, 3, 128, 128, true>(a, stream);
    if (a.hq <= 32) return launch_np<32, 2, 3, 128, 128, true>(a, stream);
    if (a.hq <= 64) return launch_np<64, 2, 3, 128, 128, true>(a, stream);
    return cudaErrorInvalidValue;
  }
  // Ring stages: about 64 KB of K and 96 KB of V tiles whatever the head sizes.
  if (a.dk == 128 && a.d == 128) return launch_hq<2, 3, 128, 128>(a, stream);
  if (a.dk == 64 && a.d == 64) {   // up to 32 heads per group: 256-row tiles of 32 KB, as at head size 128
    if (a.hq <= 16) return launch_np<16, 2, 3, 64, 64, false>(a, stream);
    if (a.hq <= 32) return launch_np<32, 2, 3, 64, 64, false>(a, stream);
    if (a.hq <= 64) return launch_np<64, 4, 6, 64, 64, false>(a, stream);
    return cudaErrorInvalidValue;
  }
  if (a.dk == 128 && a.d == 64) return launch_hq<2, 6, 128, 64>(a, stream);
  if (a.dk == 64 && a.d == 128) return launch_hq<4, 3, 64, 128>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace mqa
