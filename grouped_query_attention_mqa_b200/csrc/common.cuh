// Shared device-side pieces of libmqa: element types, the work partition of a
// decode across persistent CTAs, and the workspace layout.
//
// Work partition.  A decode touches, for every sequence b and K/V head j, the
// valid rows t < L_b of the cache.  Rows are cut into tiles of TILE rows; the
// tiles of all (b, j) "segments" are numbered in (b, j, tile) order, and the G
// persistent CTAs each take one contiguous run of that numbering,
// CTA c owning tiles [floor(c*T/G), floor((c+1)*T/G)).  Every CTA therefore
// moves the same number of bytes (up to one tile) whatever the length mix, and
// a segment split between CTAs leaves one normalised partial output plus its
// log-sum-exp per CTA, combined afterwards by the merge kernel.  This split is
// exact: softmax over a union of row sets is the log-sum-exp weighted mix of
// the softmaxes over the parts.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "mqa.h"

namespace mqa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxCtas = MQA_MAX_CTAS;

// ------------------------------------------------------------ element access

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Two bf16 packed in a 32-bit word -> two floats (exact: bf16 is the top half
// of an fp32).
__device__ __forceinline__ float2 bf16x2_to_f32x2(uint32_t w) {
  float2 r;
  r.x = __uint_as_float(w << 16);
  r.y = __uint_as_float(w & 0xffff0000u);
  return r;
}

__device__ __forceinline__ void set_flag(int32_t* flags, int bit) {
  if (flags) atomicOr(flags, bit);
}

// Clamp a device-provided length to [0, m_max]; report values outside
// [1, m_max].
__device__ __forceinline__ int clamp_len(int len, int m_max, int32_t* flags, bool report) {
  if (len < 1 || len > m_max) {
    if (report) set_flag(flags, MQA_FLAG_LEN_CLAMPED);
    len = len < 0 ? 0 : (len > m_max ? m_max : len);
  }
  return len;
}

// ------------------------------------------------------------ workspace

struct Workspace {
  int2* seg_info;   // [b*g]: first and last CTA that touched the segment
  float* part_lse;  // [slots][hq]: log2-domain log-sum-exp of each partial
  float* part_o;    // [slots][hq][d_v]: normalised partial outputs
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline size_t workspace_slots(int b, int g) {
  return size_t(kMaxCtas) + size_t(b) * size_t(g);
}

__host__ __device__ inline size_t workspace_bytes(int b, int g, int hq, int d_v) {
  size_t slots = workspace_slots(b, g);
  return align256(sizeof(int2) * size_t(b) * size_t(g)) + align256(sizeof(float) * slots * hq) +
         align256(sizeof(float) * slots * hq * size_t(d_v));
}

__host__ __device__ inline Workspace carve_workspace(void* base, int b, int g, int hq) {
  char* p = static_cast<char*>(base);
  Workspace w;
  w.seg_info = reinterpret_cast<int2*>(p);
  p += align256(sizeof(int2) * size_t(b) * size_t(g));
  w.part_lse = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * workspace_slots(b, g) * hq);
  w.part_o = reinterpret_cast<float*>(p);
  return w;
}

// Slot of the partial that CTA c leaves for segment s.  For consecutive
// segments the CTA ranges only meet at one shared CTA, so c + s never
// collides, and slots < G + b*g.
__device__ __forceinline__ int64_t partial_slot(int c, int64_t s) { return int64_t(c) + s; }

// ------------------------------------------------------------ work partition

struct Sched {
  int64_t total;     // T: tiles over all segments
  int active;        // G_eff = min(G, T): CTAs that get work
  int64_t t_begin;   // this CTA's first tile
  int64_t t_end;     // one past its last tile
  int seq;           // sequence of t_begin (valid when t_begin < t_end)
  int64_t seq_base;  // first tile number of that sequence
};

__device__ __forceinline__ int tiles_of(int len, int tile) { return (len + tile - 1) / tile; }

// Rows of a sequence of length len that a decode attends to: all of them, or
// with a local window w > 0 the newest min(len, w) ("Fast Transformer
// Decoding" study notes §6.1, §6.4).  Partitions count tiles of the span;
// tile k of a segment starts at cache row (len - span) + k * tile.
__device__ __forceinline__ int span_of(int len, int window) { return window > 0 && len > window ? window : len; }

// Beams sharing a prefix in one pass: sequence s owns, after its prefix rows,
// the suffix rows of its W beams (beam w's cache row block is s*W + w), each
// beam's rows starting at a tile edge.  slens == nullptr: no suffixes.
struct BeamSuffixes {
  const int32_t* slens;   // [b*W] suffix lengths (clamped to [0, m_s])
  int W;
  int m_s;
};

__device__ __forceinline__ int suffix_tiles(const BeamSuffixes& bs, int s, int tile, int32_t* flags, bool report) {
  if (bs.slens == nullptr) return 0;
  int n = 0;
#pragma unroll 4
  for (int w = 0; w < bs.W; ++w)   // unrolled: the length loads go out together
    n += tiles_of(clamp_len(__ldg(bs.slens + int64_t(s) * bs.W + w), bs.m_s, flags, report), tile);
  return n;
}

__device__ __forceinline__ int64_t range_start(int64_t c, int64_t total, int active) {
  return (c * total) / active;
}

// Last CTA whose range starts at or before tile t (the owner of t).
__device__ __forceinline__ int cta_of_tile(int64_t t, int64_t total, int active) {
  return int(((t + 1) * int64_t(active) - 1) / total);
}

// Every CTA derives the same partition from lens.  Thread i sums the tiles of
// a contiguous block of sequences; a warp shuffle scan plus a scan of the warp
// totals gives T and this thread's exclusive prefix; the thread whose block
// holds this CTA's first tile walks its block to find the sequence.
// Cost: O(b / NT) loads per thread and three block barriers.
// `red` needs NT/32 + 2 int64 of shared memory.
template <int NT>
__device__ Sched make_schedule(const int32_t* __restrict__ lens, int b, int g, int m_max, int window, int tile,
                               int grid, int cta, int32_t* flags, int64_t* red) {
  static_assert(NT % 32 == 0, "whole warps");
  const int per = (b + NT - 1) / NT;
  const int s0 = min(b, int(threadIdx.x) * per);
  const int s1 = min(b, s0 + per);
  int64_t mine = 0;
  for (int s = s0; s < s1; ++s)
    mine += int64_t(g) * tiles_of(span_of(clamp_len(__ldg(lens + s), m_max, flags, cta == 0), window), tile);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t x = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  int64_t* wtot = red;
  int64_t* out = red + NT / 32;
  __syncthreads();
  if (lane == 31) wtot[warp] = x;
  __syncthreads();
  int64_t total = 0, before = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const int64_t v = wtot[w];
    total += v;
    if (w < warp) before += v;
  }
  const int64_t excl = before + x - mine;
  Sched sc;
  sc.total = total;
  sc.active = int(total < grid ? total : int64_t(grid));
  sc.t_begin = sc.t_end = 0;
  sc.seq = 0;
  sc.seq_base = 0;
  if (cta >= sc.active) return sc;   // uniform across the CTA
  sc.t_begin = range_start(cta, total, sc.active);
  sc.t_end = range_start(int64_t(cta) + 1, total, sc.active);
  if (sc.t_begin >= excl && sc.t_begin < excl + mine) {
    int64_t base = excl;
    for (int s = s0; s < s1; ++s) {
      int64_t n = int64_t(g) * tiles_of(span_of(clamp_len(__ldg(lens + s), m_max, nullptr, false), window), tile);
      if (sc.t_begin < base + n) {
        out[0] = s;
        out[1] = base;
        break;
      }
      base += n;
    }
  }
  __syncthreads();
  sc.seq = int(out[0]);
  sc.seq_base = out[1];
  return sc;
}

// Weighted partition (tensor-core path).  Positions are counted in units of a
// quarter tile, and every segment starts with `xw` extra units that stand for
// the fixed cost a CTA pays to enter a segment (its queries, a full max
// reduction, writing the output).  Segment s of sequence b spans
// xw + 4*nb units; tile k of it starts xw + 4*k units after the segment does.
// CTA c owns the tiles whose start unit lies in [c*W/A, (c+1)*W/A), so a CTA
// whose range crosses segment starts gets correspondingly fewer tiles.  With
// A <= W / (xw + 4) every range holds at least one tile start.
struct WSched {
  Sched s;
  int64_t wtotal;     // W: units over all segments
  int64_t seq_ubase;  // first unit of sequence s.seq
  int pre;            // leading tiles whose loads the schedule already issued
};

__device__ __forceinline__ int64_t seq_units(int nb, int g, int xw) {
  return nb > 0 ? int64_t(g) * (xw + 4 * int64_t(nb)) : 0;
}

// CTA whose unit range holds unit u.
__device__ __forceinline__ int cta_of_unit(int64_t u, int64_t wtotal, int active) {
  return int(((u + 1) * int64_t(active) - 1) / wtotal);
}

template <int NT>
__device__ WSched make_schedule_weighted(const int32_t* __restrict__ lens, int b, int g, int m_max, int window,
                                         int tile, int grid, int cta, int32_t* flags, int64_t* red, int xw,
                                         const BeamSuffixes& bs) {
  static_assert(NT % 32 == 0, "whole warps");
  const int per = (b + NT - 1) / NT;
  const int s0 = min(b, int(threadIdx.x) * per);
  const int s1 = min(b, s0 + per);
  int64_t my_t = 0, my_u = 0;
  for (int s = s0; s < s1; ++s) {
    const int nb = tiles_of(span_of(clamp_len(__ldg(lens + s), m_max, flags, cta == 0), window), tile) +
                   suffix_tiles(bs, s, tile, flags, cta == 0);
    my_t += int64_t(g) * nb;
    my_u += seq_units(nb, g, xw);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t xt = my_t, xu = my_u;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t yt = __shfl_up_sync(0xffffffffu, xt, o);
    const int64_t yu = __shfl_up_sync(0xffffffffu, xu, o);
    if (lane >= o) {
      xt += yt;
      xu += yu;
    }
  }
  int64_t* wt = red;                 // [NT/32] warp tile totals
  int64_t* wu = red + NT / 32;       // [NT/32] warp unit totals
  int64_t* out = red + 2 * (NT / 32);
  __syncthreads();
  if (lane == 31) {
    wt[warp] = xt;
    wu[warp] = xu;
  }
  __syncthreads();
  int64_t T = 0, W = 0, bt = 0, bu = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const int64_t vt = wt[w], vu = wu[w];
    T += vt;
    W += vu;
    if (w < warp) {
      bt += vt;
      bu += vu;
    }
  }
  const int64_t excl_t = bt + xt - my_t, excl_u = bu + xu - my_u;
  WSched ws;
  ws.s.total = T;
  ws.wtotal = W;
  const int64_t cap = W / (xw + 4);
  ws.s.active = int(cap < grid ? cap : int64_t(grid));
  ws.s.t_begin = ws.s.t_end = 0;
  ws.s.seq = 0;
  ws.s.seq_base = 0;
  ws.seq_ubase = 0;
  ws.pre = 0;
  if (cta >= ws.s.active) return ws;   // uniform across the CTA
  const int64_t u0 = (int64_t(cta) * W) / ws.s.active;
  const int64_t u1 = ((int64_t(cta) + 1) * W) / ws.s.active;
  // Tiles whose start unit is below u (< W), computed by the thread whose
  // block of sequences holds u; also the sequence holding u and its bases.
  auto locate = [&](int64_t u, int64_t* dst, bool with_seq) {
    if (!(u >= excl_u && u < excl_u + my_u)) return;
    int64_t tb = excl_t, ub = excl_u;
    for (int s = s0; s < s1; ++s) {
      const int nb = tiles_of(span_of(clamp_len(__ldg(lens + s), m_max, nullptr, false), window), tile) +
                     suffix_tiles(bs, s, tile, nullptr, false);
      const int64_t su = seq_units(nb, g, xw);
      if (u < ub + su) {
        const int64_t seglen = xw + 4 * int64_t(nb);
        const int64_t rel = u - ub;
        const int64_t j = rel / seglen, off = rel - j * seglen;
        const int64_t cnt = off <= xw ? 0 : (off - xw + 3) / 4;
        dst[0] = tb + j * nb + cnt;
        if (with_seq) {
          dst[1] = s;
          dst[2] = tb;
          dst[3] = ub;
        }
        return;
      }
      tb += int64_t(g) * nb;
      ub += su;
    }
  };
  locate(u0, out, true);
  if (u1 < W) locate(u1, out + 4, false);
  __syncthreads();
  ws.s.t_begin = out[0];
  ws.s.seq = int(out[1]);
  ws.s.seq_base = out[2];
  ws.seq_ubase = out[3];
  ws.s.t_end = u1 == W ? T : out[4];
  ws.pre = 0;
  return ws;
}

// The same weighted partition when every sequence has a thread (b <= NT) and
// the unit total stays below 2^31 (checked by small_schedule_fits): each thread
// loads one length, which it also leaves in lens_tab[s] (clamped) for the rest
// of the kernel; the tile and unit counts are scanned together as one 64-bit
// word (high and low halves, neither can carry), and the range ends are found
// with 32-bit arithmetic.  Two block barriers.  `red` needs NT/32 + 8 int64.
// The thread that finds the CTA's first tile calls
// on_first(seq, head, k, own, len, nb) at once, with `own` >= 1 tiles of that
// segment from tile k on belonging to the CTA; it returns how many of them it
// has started to load (WSched::pre).  Code that runs once per launch executes
// at instruction-fetch speed, so this gets the first loads out well before a
// separate role would reach them.
__device__ __forceinline__ bool small_schedule_fits(int b, int g, int m_max, int tile, int nt, int xw,
                                                    int64_t suffix_tiles_max = 0) {
  return b <= nt && int64_t(b) * g * (xw + 4 * ((int64_t(m_max) + tile - 1) / tile + suffix_tiles_max)) <
                        (int64_t(1) << 31);
}

template <int NT, typename OnFirst>
__device__ WSched make_schedule_small(const int32_t* __restrict__ lens, int b, int g, int m_max, int window, int tile,
                                      int grid, int cta, int32_t* flags, int64_t* red, int xw, int* lens_tab,
                                      const BeamSuffixes& bs, int* nsuf_tab, OnFirst&& on_first) {
  static_assert(NT % 32 == 0, "whole warps");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int len = 0, nsuf = 0;
  if (tid < b) {
    len = clamp_len(__ldg(lens + tid), m_max, flags, cta == 0);
    lens_tab[tid] = len;
    nsuf = suffix_tiles(bs, tid, tile, flags, cta == 0);
    if (nsuf_tab != nullptr) nsuf_tab[tid] = nsuf;
  }
  const int nb = tiles_of(span_of(len, window), tile) + nsuf;
  const int my_t = g * nb;
  const int my_u = nb > 0 ? g * (xw + 4 * nb) : 0;
  uint64_t x = (uint64_t(uint32_t(my_t)) << 32) | uint32_t(my_u);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  uint64_t* wsum = reinterpret_cast<uint64_t*>(red);   // [NT/32]
  int64_t* out = red + NT / 32;
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  uint64_t tot = 0, before = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const uint64_t v = wsum[w];
    tot += v;
    if (w < warp) before += v;
  }
  const uint64_t incl = before + x;
  const int T = int(tot >> 32), W = int(uint32_t(tot));
  const int excl_t = int(incl >> 32) - my_t, excl_u = int(uint32_t(incl)) - my_u;
  WSched ws;
  ws.s.total = T;
  ws.wtotal = W;
  const int cap = W / (xw + 4);
  ws.s.active = cap < grid ? cap : grid;
  ws.s.t_begin = ws.s.t_end = 0;
  ws.s.seq = 0;
  ws.s.seq_base = 0;
  ws.seq_ubase = 0;
  ws.pre = 0;
  if (cta >= ws.s.active) return ws;   // uniform across the CTA
  // c*W/A without a 64-bit product: W = q*A + rm and c*rm < A*A
  const int q = W / ws.s.active, rm = W - q * ws.s.active;
  const int u0 = cta * q + (cta * rm) / ws.s.active;
  const int u1 = (cta + 1) * q + ((cta + 1) * rm) / ws.s.active;
  const int seglen = xw + 4 * nb;
  auto first_tile = [&](int u) {   // tiles of this thread's sequence whose start unit is below u
    const int rel = u - excl_u;
    const int j = rel / seglen, off = rel - j * seglen;
    return excl_t + j * nb + (off <= xw ? 0 : (off - xw + 3) / 4);
  };
  if (u1 < W && u1 >= excl_u && u1 < excl_u + my_u) out[4] = first_tile(u1);
  if (u0 >= excl_u && u0 < excl_u + my_u) {
    const int rel = u0 - excl_u;
    const int j = rel / seglen, off = rel - j * seglen;
    const int k = off <= xw ? 0 : (off - xw + 3) / 4;
    out[0] = excl_t + j * nb + k;
    out[1] = tid;
    out[2] = excl_t;
    out[3] = excl_u;
    int started = 0;
    if (k < nb) {   // tile k of segment j exists; the CTA owns its tiles whose start unit is below u1
      const int lim = u1 - (excl_u + j * seglen + xw);
      const int kend = min(nb, lim <= 0 ? 0 : (lim + 3) / 4);
      if (kend > k) started = on_first(tid, j, k, kend - k, len, nb);
    }
    out[5] = started;
  }
  __syncthreads();
  ws.s.t_begin = out[0];
  ws.s.seq = int(out[1]);
  ws.s.seq_base = out[2];
  ws.seq_ubase = out[3];
  ws.s.t_end = u1 == W ? T : out[4];
  ws.pre = int(out[5]);
  return ws;
}

// Walks the tile numbering forward from a known sequence.
struct Cursor {
  int seq;          // sequence of the current tile
  int64_t base;     // first tile of that sequence
  int nb;           // tiles per segment of that sequence
  int len;          // clamped length of that sequence
  int lo;           // first attended row (len - span)
};

__device__ __forceinline__ Cursor cursor_at(const int32_t* __restrict__ lens, int m_max, int window, int tile,
                                            int seq, int64_t base) {
  Cursor cu;
  cu.seq = seq;
  cu.base = base;
  cu.len = clamp_len(__ldg(lens + seq), m_max, nullptr, false);
  cu.lo = cu.len - span_of(cu.len, window);
  cu.nb = tiles_of(cu.len - cu.lo, tile);
  return cu;
}

// Advance the cursor until tile t lies in its sequence.
__device__ __forceinline__ void cursor_seek(Cursor& cu, const int32_t* __restrict__ lens, int g, int m_max,
                                            int window, int tile, int64_t t) {
  while (t >= cu.base + int64_t(g) * cu.nb) {
    cu.base += int64_t(g) * cu.nb;
    cu.seq += 1;
    cu.len = clamp_len(__ldg(lens + cu.seq), m_max, nullptr, false);
    cu.lo = cu.len - span_of(cu.len, window);
    cu.nb = tiles_of(cu.len - cu.lo, tile);
  }
}

struct TileCoord {
  int seq, head, k;   // sequence, K/V head, tile index within the segment
  int row0, rows;     // first cache row and number of valid rows in the tile
  int beam;           // beams sharing a prefix: the beam whose suffix the tile is, -1 for a prefix tile
  int src_row;        // row of the tile's first row in its cache viewed as (rows, g, d)
  int64_t seg;        // segment number seq*g + head
  int64_t seg_t0;     // global number of the segment's first tile
  int nb;             // tiles in the segment
};

__device__ __forceinline__ TileCoord tile_coord(const Cursor& cu, int g, int tile, int64_t t) {
  TileCoord tc;
  const int64_t rel = t - cu.base;
  tc.seq = cu.seq;
  tc.head = int(rel / cu.nb);
  tc.k = int(rel - int64_t(tc.head) * cu.nb);
  tc.row0 = cu.lo + tc.k * tile;
  tc.rows = min(tile, cu.len - tc.row0);
  tc.beam = -1;
  tc.src_row = 0;   // not used by the SIMT path
  tc.seg = int64_t(cu.seq) * g + tc.head;
  tc.nb = cu.nb;
  tc.seg_t0 = cu.base + int64_t(tc.head) * cu.nb;
  return tc;
}

// ------------------------------------------------------------ launchers

struct DecodeArgs {
  void* o;
  const void* q;
  const void* k;
  const void* v;
  // Fused append: when non-null, k_new/v_new [b, g, d] are written at row
  // lens[b]-1 of the caches by the CTA that loads that row, before it loads it.
  const void* k_new;
  const void* v_new;
  const int32_t* lens;
  int b, h, g, m_max, d;   // d: value head size d_v
  int dk;                 // key head size d_k (q and K rows)
  int hq;
  int window;          // local attention: the newest `window` rows (0 = all rows)
  int no_merge;        // no segment spans two tiles: the decode writes every output row
                       // itself (zero rows for empty sequences) and no merge follows
  int q_beams;         // 0: q is [b, h, d]; W > 0: q is [b, W, h, d] and a segment's query rows
                       // are the W beams' q_group_heads heads of its group (hq = W * q_group_heads)
  int q_group_heads;   // query heads per K/V head in q
  float scale;
  Workspace ws;
  int32_t* flags;
  int grid;
  // Beams sharing a prefix in one pass (q_beams = W > 0 and sk != nullptr): segment (b, j) walks
  // sequence b's prefix rows (k, v, lens, m_max), then each beam's own suffix rows (sk, sv,
  // slens [b*W], m_s; beam w's rows at cache row block b*W + w).  A suffix tile of beam w counts
  // for that beam's q_group_heads query columns only; o is [b, W, h, d].
  const void* sk;
  const void* sv;
  const int32_t* slens;
  int m_s;
};

cudaError_t launch_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new, const int32_t* pos,
                          int b, int m_max, int g, int row_k_bytes, int row_v_bytes, int32_t* flags,
                          cudaStream_t stream);
// The CUDA-core decode: q and K rows of d_k elements, V and o rows of a.d = d_v.
cudaError_t launch_decode_simt(const DecodeArgs& a, int d_k, mqa_dtype_t dtype, cudaStream_t stream);
int simt_ctas_per_sm(mqa_dtype_t dtype, int d_k, int d_v, int hq);
cudaError_t launch_merge(const DecodeArgs& a, mqa_dtype_t dtype, cudaStream_t stream);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream);
bool prefill_tc_supported(int d, int hq);
cudaError_t launch_prefill_tc(void* o, const void* q, const void* k, const void* v, const int32_t* cu, int b,
                              int64_t total, int h, int g, int max_seqlen, float scale, int causal, int32_t* flags,
                              cudaStream_t stream);
int tc_ctas_per_sm(int hq);
int tc_tile_rows();
int simt_tile_rows();
bool tc_supported(int d_k, int d_v, int hq);

}  // namespace mqa
