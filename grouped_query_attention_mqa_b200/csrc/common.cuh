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

__device__ __forceinline__ int64_t range_start(int64_t c, int64_t total, int active) {
  return (c * total) / active;
}

// Last CTA whose range starts at or before tile t (the owner of t).
__device__ __forceinline__ int cta_of_tile(int64_t t, int64_t total, int active) {
  return int(((t + 1) * int64_t(active) - 1) / total);
}

template <int NT>
__device__ __forceinline__ int64_t block_sum_i64(int64_t v, int64_t* red) {
  static_assert(NT % 32 == 0, "whole warps");
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  int64_t s = 0;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) s += red[i];
  return s;
}

// Every CTA derives the same partition from lens.  Thread i sums the tiles of
// a contiguous block of sequences, a block-wide sum gives T, an exclusive scan
// of the per-thread sums locates this CTA's first tile, and the thread holding
// it walks its block to find the sequence.  Cost: O(b / NT) loads per thread.
// `red` needs NT/32 + NT + 2 int64 of shared memory.
template <int NT>
__device__ Sched make_schedule(const int32_t* __restrict__ lens, int b, int g, int m_max, int tile,
                               int grid, int cta, int32_t* flags, int64_t* red) {
  const int per = (b + NT - 1) / NT;
  const int s0 = min(b, int(threadIdx.x) * per);
  const int s1 = min(b, s0 + per);
  int64_t mine = 0;
  for (int s = s0; s < s1; ++s)
    mine += int64_t(g) * tiles_of(clamp_len(__ldg(lens + s), m_max, flags, cta == 0), tile);
  int64_t* warp_red = red;
  int64_t* incl = red + NT / 32;
  int64_t* out = incl + NT;
  const int64_t total = block_sum_i64<NT>(mine, warp_red);
  Sched sc;
  sc.total = total;
  sc.active = int(total < grid ? total : int64_t(grid));
  sc.t_begin = sc.t_end = 0;
  sc.seq = 0;
  sc.seq_base = 0;
  if (cta >= sc.active) return sc;
  sc.t_begin = range_start(cta, total, sc.active);
  sc.t_end = range_start(int64_t(cta) + 1, total, sc.active);
  // inclusive scan of per-thread tile sums (NT is small: a plain two-pass scan
  // through shared memory is enough)
  incl[threadIdx.x] = mine;
  __syncthreads();
  for (int off = 1; off < NT; off <<= 1) {
    int64_t add = threadIdx.x >= off ? incl[threadIdx.x - off] : 0;
    __syncthreads();
    incl[threadIdx.x] += add;
    __syncthreads();
  }
  const int64_t excl = incl[threadIdx.x] - mine;
  if (sc.t_begin >= excl && sc.t_begin < excl + mine) {
    int64_t base = excl;
    for (int s = s0; s < s1; ++s) {
      int64_t n = int64_t(g) * tiles_of(clamp_len(__ldg(lens + s), m_max, nullptr, false), tile);
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

// Walks the tile numbering forward from a known sequence.
struct Cursor {
  int seq;          // sequence of the current tile
  int64_t base;     // first tile of that sequence
  int nb;           // tiles per segment of that sequence
  int len;          // clamped length of that sequence
};

__device__ __forceinline__ Cursor cursor_at(const int32_t* __restrict__ lens, int m_max, int tile, int seq,
                                            int64_t base) {
  Cursor cu;
  cu.seq = seq;
  cu.base = base;
  cu.len = clamp_len(__ldg(lens + seq), m_max, nullptr, false);
  cu.nb = tiles_of(cu.len, tile);
  return cu;
}

// Advance the cursor until tile t lies in its sequence.
__device__ __forceinline__ void cursor_seek(Cursor& cu, const int32_t* __restrict__ lens, int g, int m_max,
                                            int tile, int64_t t) {
  while (t >= cu.base + int64_t(g) * cu.nb) {
    cu.base += int64_t(g) * cu.nb;
    cu.seq += 1;
    cu.len = clamp_len(__ldg(lens + cu.seq), m_max, nullptr, false);
    cu.nb = tiles_of(cu.len, tile);
  }
}

struct TileCoord {
  int seq, head, k;   // sequence, K/V head, tile index within the segment
  int row0, rows;     // first cache row and number of valid rows in the tile
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
  tc.row0 = tc.k * tile;
  tc.rows = min(tile, cu.len - tc.row0);
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
  const int32_t* lens;
  int b, h, g, m_max, d;
  int hq;
  float scale;
  Workspace ws;
  int32_t* flags;
  int grid;
};

cudaError_t launch_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new, const int32_t* pos,
                          int b, int m_max, int g, int row_k_bytes, int row_v_bytes, int32_t* flags,
                          cudaStream_t stream);
cudaError_t launch_decode_simt(const DecodeArgs& a, mqa_dtype_t dtype, cudaStream_t stream);
int simt_ctas_per_sm(mqa_dtype_t dtype, int d, int hq);
cudaError_t launch_merge(const DecodeArgs& a, mqa_dtype_t dtype, cudaStream_t stream);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream);
int tc_ctas_per_sm(int hq);
bool tc_supported(int d, int hq);

}  // namespace mqa
