// pkv_kernels.cuh -- sm_100a kernels of the paged KV cache:
//   pkv_append_kernel   scatter of new K/V rows into their slots
//   pkv_copy_blocks_kernel  whole-block copies for copy-on-write
//   pkv_append_i8_kernel    quantising append into the INT8 cache
//   pkv_decode_kernel   persistent split-KV paged decode attention, with the
//                       log-sum-exp merge of split contexts after a grid-wide
//                       barrier
//
// Decode design (one launch for every sequence, head group and context split):
//
// * Work is counted in tiles: one tile is one 16-token physical block of one kv
//   head (a contiguous 16 x head_dim run of the pool).  A segment is the whole
//   context of one sequence for one group of `gp` query heads that share a kv
//   head; it has ceil(ctx / 16) tiles.  The tiles of all segments, in the order
//   (sequence, head group, logical block), are split into `num_units` equal
//   contiguous ranges (stream-K style).  A unit is one consumer warp, so every
//   warp gets the same number of tiles whatever the length mix; a segment that
//   straddles unit boundaries is a split context whose partial softmax states
//   are merged, after a grid-wide barrier of the cooperative launch, by the
//   unit that holds its first piece.
// * Each CTA runs 10 consumer warps (units) and one producer warp.  Lane w of
//   the producer walks unit w's tiles, reads the physical block id from the
//   block table one tile ahead and issues TMA tensor loads of the K and V tile
//   into unit w's ring of `stages` shared-memory slots (mbarrier full/empty
//   pairs).  The tensor map views the pool as [block][kv head][token][dim] and
//   loads 128-byte-wide boxes with the 128B swizzle, so that the consumers'
//   shared-memory reads are free of bank conflicts.
// * Consumers: grouped query heads (2..16 of them on one kv head, 16-bit
//   data) use mma.sync m16n8k16 with fp32 accumulation: S = Q K^T with the
//   query heads as the M rows, then O += P V with P taken from the S
//   registers.  When a group has at most 8 heads the unused M rows 8..15 carry
//   the rounding residual of P (P - round16(P)), so that P enters the product
//   with about 16 significant bits.  A single query head per kv head, or fp32
//   data, runs on CUDA cores (8 tokens x 4 dim-slices per warp).  Both keep an
//   fp32 online softmax (running max and sum, exp2 with log2(e) folded into
//   the scale) reduced with warp shuffles.
// * The reduction order depends only on logical positions and on the split,
//   never on where blocks sit in the pool, so the result is bit-identical
//   under any block placement and with shared or private prefix blocks.
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "pkv_device.cuh"

namespace pkv {

constexpr int kBlockTokens = 16;
constexpr int kConsumerWarps = 10;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr int kBoxBytes = 16 * 128;  // one TMA box: 16 tokens x 128 bytes
constexpr uint64_t kWaitLimitNs = 2000000000ull;
// Tiles before a chunk's end at which its producer lane claims the next chunk.
constexpr int kClaimAhead = 3;

enum DType { kF32 = 0, kF16 = 1, kBF16 = 2 };

template <int DT>
struct DTypeInfo;
template <>
struct DTypeInfo<kF32> {
  using T = float;
  static constexpr int kBytes = 4;
};
template <>
struct DTypeInfo<kF16> {
  using T = __half;
  static constexpr int kBytes = 2;
};
template <>
struct DTypeInfo<kBF16> {
  using T = __nv_bfloat16;
  static constexpr int kBytes = 2;
};

// ---------------------------------------------------------------------------
// Append
// ---------------------------------------------------------------------------
struct AppendParams {
  const uint8_t* k;
  const uint8_t* v;
  const int64_t* slot_mapping;
  uint8_t* k_cache;
  uint8_t* v_cache;
  int64_t num_slots;  // num_blocks * block_size
  int64_t total;      // num_tokens * n_kv_heads * row_chunks
  int32_t n_kv_heads;
  int32_t row_chunks;  // 16-byte chunks per head row
};

// Chunks idx = start, start + stride, ... of the append: one 16-byte chunk
// of one head row of one token per index.  Four chunks' loads (slot, k, v)
// go out before their stores, so that the loop does not wait for one load
// round trip per chunk (the stores might alias the next loads otherwise).
__device__ __forceinline__ void append_range(const AppendParams& p, int64_t start, int64_t stride) {
  constexpr int kU = 4;
  for (int64_t base = start; base < p.total; base += kU * stride) {
    int4 kv[kU], vv[kU];
    int64_t dst[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t idx = base + u * stride;
      dst[u] = -1;
      if (idx >= p.total) continue;
      const int c = static_cast<int>(idx % p.row_chunks);
      const int64_t th = idx / p.row_chunks;  // token * n_kv + head
      const int h = static_cast<int>(th % p.n_kv_heads);
      const int64_t i = th / p.n_kv_heads;
      const int64_t sl = __ldg(p.slot_mapping + i);
      const int64_t src = (th * p.row_chunks + c) * 16;
      kv[u] = __ldg(reinterpret_cast<const int4*>(p.k + src));
      vv[u] = __ldg(reinterpret_cast<const int4*>(p.v + src));
      if (sl < 0) continue;  // padding token
      if (sl >= p.num_slots) {
        if (h == 0 && c == 0) flag_error(PKV_DEVERR_SLOT);
        continue;
      }
      const int64_t blk = sl / kBlockTokens, off = sl % kBlockTokens;
      dst[u] = (((blk * p.n_kv_heads + h) * kBlockTokens + off) * p.row_chunks + c) * 16;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (dst[u] < 0) continue;
      *reinterpret_cast<int4*>(p.k_cache + dst[u]) = kv[u];
      *reinterpret_cast<int4*>(p.v_cache + dst[u]) = vv[u];
    }
  }
}

// The fused append of the decode kernel's first phase: every thread writes its
// share of the new rows, makes them visible to the TMA reads that follow the
// grid barrier (fence.proxy.async: generic-proxy writes, async-proxy reads)
// and arrives on that barrier.  Out of line, so that it stays out of the
// decode loop's register allocation.
__device__ __noinline__ unsigned int fused_append_arrive(const AppendParams& p, int64_t start, int64_t stride) {
  append_range(p, start, stride);
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return cooperative_groups::this_grid().barrier_arrive();
}

__global__ void __launch_bounds__(256) pkv_append_kernel(const AppendParams p) {
  append_range(p, blockIdx.x * (int64_t)blockDim.x + threadIdx.x, (int64_t)gridDim.x * blockDim.x);
}

// ---------------------------------------------------------------------------
// Block copy (copy-on-write of shared blocks)
// ---------------------------------------------------------------------------
struct CopyParams {
  uint8_t* k_cache;
  uint8_t* v_cache;
  const int32_t* src;
  const int32_t* dst;
  int32_t n_pairs;
  int32_t num_blocks;
  int32_t chunks;  // 16-byte chunks per block of one cache
};

// CTAs stride over the pairs; the threads of a CTA stream one block of K and
// one of V, four 16-byte loads in flight per thread before the stores.
__global__ void __launch_bounds__(256) pkv_copy_blocks_kernel(const CopyParams p) {
  for (int pair = blockIdx.x; pair < p.n_pairs; pair += gridDim.x) {
    const int32_t s = __ldg(p.src + pair), d = __ldg(p.dst + pair);
    if (s < 0 || s >= p.num_blocks || d < 0 || d >= p.num_blocks) {
      if (threadIdx.x == 0) flag_error(PKV_DEVERR_BLOCK_ID);
      continue;
    }
    const int64_t so = static_cast<int64_t>(s) * p.chunks, dof = static_cast<int64_t>(d) * p.chunks;
    const int4* ks = reinterpret_cast<const int4*>(p.k_cache) + so;
    const int4* vs = reinterpret_cast<const int4*>(p.v_cache) + so;
    int4* kd = reinterpret_cast<int4*>(p.k_cache) + dof;
    int4* vd = reinterpret_cast<int4*>(p.v_cache) + dof;
    for (int c0 = threadIdx.x; c0 < p.chunks; c0 += 2 * blockDim.x) {
      const int c1 = c0 + blockDim.x;
      const bool two = c1 < p.chunks;
      const int4 a = ks[c0], b = vs[c0];
      int4 e = make_int4(0, 0, 0, 0), f = e;
      if (two) {
        e = ks[c1];
        f = vs[c1];
      }
      kd[c0] = a;
      vd[c0] = b;
      if (two) {
        kd[c1] = e;
        vd[c1] = f;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// INT8 cache append (quantised KV)
// ---------------------------------------------------------------------------
// Byte position of block offset j in a transposed V row: the four tokens a
// tensor-core lane t needs for one P V step (2t, 2t + 1, 2t + 8, 2t + 9) are
// bytes 4t .. 4t + 3.
__host__ __device__ __forceinline__ int vpos_i8(int j) { return 4 * ((j & 7) >> 1) + 2 * (j >> 3) + (j & 1); }

// One record per (block, kv head) of the INT8 cache, head dim D: K codes
// (16 rows of D bytes, 16-byte chunk c of row j stored at chunk c ^ (j %
// min(8, D / 16))), transposed V codes (D rows of 16 bytes, token order
// vpos_i8), 16 fp32 K scales, 16 fp32 V scales.
__host__ __device__ constexpr int i8_record_bytes(int D) { return 32 * D + 128; }

struct AppendI8Params {
  const void* k;
  const void* v;
  const int64_t* slot_mapping;
  uint8_t* cache;  // [num_blocks][n_kv][i8_record_bytes(D)]
  int64_t num_slots;
  int32_t num_tokens;
  int32_t n_kv_heads;
};

// Symmetric quantisation of one row held D / 32 elements per lane (lane owns
// dims [lane * EPL, lane * EPL + EPL)): scale = amax / 127, codes
// rint(x / scale), both in binary32 (IEEE division: the build uses no fast
// math).
template <int EPL>
__device__ __forceinline__ float quantise_row(const float (&x)[EPL], int8_t (&c)[EPL]) {
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float scale = amax / 127.0f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    float q = amax == 0.f ? 0.f : rintf(x[e] / scale);
    q = fminf(fmaxf(q, -127.f), 127.f);
    c[e] = static_cast<int8_t>(q);
  }
  return scale;
}

template <int DT, int D>
__global__ void __launch_bounds__(256) pkv_append_i8_kernel(const AppendI8Params p) {
  using T = typename DTypeInfo<DT>::T;
  constexpr int EPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t n_rows = static_cast<int64_t>(p.num_tokens) * p.n_kv_heads;
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < n_rows;
       r += (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) {
    const int64_t i = r / p.n_kv_heads;
    const int h = static_cast<int>(r % p.n_kv_heads);
    const int64_t s = __ldg(p.slot_mapping + i);
    if (s < 0) continue;  // padding token
    if (s >= p.num_slots) {
      if (lane == 0 && h == 0) flag_error(PKV_DEVERR_SLOT);
      continue;
    }
    const int64_t blk = s / kBlockTokens;
    const int off = static_cast<int>(s % kBlockTokens);
    uint8_t* rec = p.cache + (static_cast<size_t>(blk) * p.n_kv_heads + h) * i8_record_bytes(D);
    const size_t src = static_cast<size_t>(r) * D + lane * EPL;
    float xk[EPL], xv[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      if constexpr (DT == kF32) {
        xk[e] = __ldg(static_cast<const float*>(p.k) + src + e);
        xv[e] = __ldg(static_cast<const float*>(p.v) + src + e);
      } else {
        const uint16_t bk = __ldg(reinterpret_cast<const unsigned short*>(p.k) + src + e);
        const uint16_t bv = __ldg(reinterpret_cast<const unsigned short*>(p.v) + src + e);
        float lo, hi;
        unpack2<DT == kBF16>(static_cast<uint32_t>(bk) | (static_cast<uint32_t>(bv) << 16), lo, hi);
        xk[e] = lo;
        xv[e] = hi;
      }
    }
    int8_t ck[EPL], cv[EPL];
    const float sk = quantise_row<EPL>(xk, ck);
    const float sv = quantise_row<EPL>(xv, cv);
    // This lane's EPL dims sit inside one 16-byte chunk of the K row.
    constexpr int kSwz = (D / 16) < 8 ? (D / 16) : 8;
    const int c = (lane * EPL) / 16;
    uint8_t* krow = rec + off * D + ((c ^ (off % kSwz)) * 16) + (lane * EPL) % 16;
#pragma unroll
    for (int e = 0; e < EPL; ++e) krow[e] = static_cast<uint8_t>(ck[e]);
    const int vp = vpos_i8(off);
#pragma unroll
    for (int e = 0; e < EPL; ++e) rec[16 * D + (lane * EPL + e) * kBlockTokens + vp] = static_cast<uint8_t>(cv[e]);
    if (lane == 0) {
      reinterpret_cast<float*>(rec + 32 * D)[off] = sk;
      reinterpret_cast<float*>(rec + 32 * D + 64)[off] = sv;
    }
  }
}

// ---------------------------------------------------------------------------
// Decode
// ---------------------------------------------------------------------------
struct DecodeParams {
  const void* q;
  void* out;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* records;  // [chunks][2][rec_floats]: O[gp][D], m[gp], l[gp]
  const uint8_t* kv_i8;  // INT8 cache only: one record per (block, kv head)
  int32_t n_kv_heads;
  int4* meta;      // [chunks]: split segment whose first piece the chunk holds
  int* sched;      // [0]: claim counter of the balancing chunks (0 between launches)
  // Optional initial softmax state per (sequence, query head) -- the shared
  // prefix part of a cascade decode: O [batch][n_q][D] unnormalised, then
  // m [batch][n_q] (log2 units), then l [batch][n_q].  Used for sequences with
  // seq_group[b] >= 0 when `init` is not null.
  const float* init;
  const int32_t* seq_group;
  int32_t n_groups;
  int32_t max_blocks_per_seq;
  int32_t batch;
  int32_t num_blocks;
  int32_t n_q_heads;
  int32_t group;       // query heads per kv head
  int32_t gp;          // query heads per segment
  int32_t ng;          // segments per sequence (n_q_heads / gp)
  int32_t num_units;
  int32_t sub_chunks;      // balancing chunks cut from the end of each unit's range (0..4)
  int32_t static_permille; // share of each unit's range that the unit keeps
  int32_t stages;      // ring slots per consumer warp
  int32_t rec_floats;  // floats per partial record: rows * (head_dim + 2), rounded up to 4
  int32_t q_len;       // queries per sequence (the last q_len tokens of its context)
  int32_t rows;        // rows per segment: q_len * gp
  int32_t head_dim;
  float scale_log2;    // scale * log2(e)
  uint64_t wait_limit_ns;  // bound of every in-kernel wait
  int32_t withhold_unit;   // test hook: this unit's producer lane issues nothing (-1: none)
  // Fused append (paged_kv_append_and_decode): the new tokens' K and V are
  // written into their slots by every CTA before any tile is read (app.total
  // = 0: none).
  AppendParams app;
};

// Row `row` of segment (b, hg) -- query row / gp, head hg * gp + row % gp
// -- as an index into [batch][q_len][n_q] (q, out; [batch][n_q] when q_len
// is 1).
__device__ __forceinline__ size_t out_row(const DecodeParams& p, int b, int hg, int row) {
  const int qi = row / p.gp;
  return (static_cast<size_t>(b) * p.q_len + qi) * p.n_q_heads + hg * p.gp + (row - qi * p.gp);
}

// Position of a warp in its unit's tile range.
struct Walk {
  int b, hg, j, nb, ctx;
  int k, k_end;
};

// Does sequence b continue from an initial state?  A group id outside
// [0, n_groups) is flagged and ignored (its state was never computed).
__device__ __forceinline__ bool has_init(const DecodeParams& p, int b) {
  const int gi = __ldg(p.seq_group + b);
  if (gi < 0) return false;
  if (gi >= p.n_groups) {
    flag_error(PKV_DEVERR_CONTEXT);
    return false;
  }
  return true;
}

__device__ __forceinline__ int clamp_ctx(int c, int max_ctx) { return c < 0 ? 0 : (c > max_ctx ? max_ctx : c); }

__device__ __forceinline__ bool walk_begin(Walk& w, const int* prefix, const int* ctxs, int B, int k0, int k1) {
  w.k = k0;
  w.k_end = k1;
  if (k0 >= k1) return false;
  int lo = 0, hi = B;  // prefix[lo] <= k0 < prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= k0) lo = mid; else hi = mid;
  }
  w.b = lo;
  w.ctx = ctxs[lo];
  w.nb = (w.ctx + kBlockTokens - 1) / kBlockTokens;
  const int local = k0 - prefix[lo];
  w.hg = local / w.nb;
  w.j = local - w.hg * w.nb;
  return true;
}

__device__ __forceinline__ void walk_next(Walk& w, const int* prefix, const int* ctxs, int B, int ng) {
  ++w.k;
  if (++w.j == w.nb) {
    w.j = 0;
    if (++w.hg == ng) {
      w.hg = 0;
      do {
        ++w.b;
      } while (w.b < B && prefix[w.b + 1] == prefix[w.b]);
      if (w.b < B) {
        w.ctx = ctxs[w.b];
        w.nb = (w.ctx + kBlockTokens - 1) / kBlockTokens;
      }
    }
  }
}

// Work partition.  The T tiles are cut into U units of Lq = T / U tiles,
// the first r = T % U of them one tile longer, so that the boundaries need no
// division.  Unit u's range [a, a + L) is cut into chunk u * (M + 1) (its
// first S = L * static_permille / 1000 tiles, run by unit u's own warp) and M
// balancing chunks that split the other D = L - S tiles in the ratio
// M : M-1 : ... : 1.  Balancing chunks are claimed at run time through an
// atomic counter, largest first over all units, by the producer lanes whose
// warps run out of work first.  Chunk boundaries depend only on (T, U, M, S),
// so the result does not depend on which warp runs a chunk.  Chunk ids
// follow tile order.
struct Sched {
  int U, M, Lq, r;
  int Sq, Dq, Sr, Dr;  // S and D of units of Lq tiles and of Lq + 1 tiles
};

__device__ __forceinline__ int sub_cum(int i, int M) { return i * (2 * M + 1 - i) / 2; }

// x / (M (M + 1) / 2) with a constant divisor per case.
__device__ __forceinline__ int div_sub_weight(int64_t x, int M) {
  switch (M) {
    case 1: return static_cast<int>(x);
    case 2: return static_cast<int>(x / 3);
    case 3: return static_cast<int>(x / 6);
    default: return static_cast<int>(x / 10);
  }
}

__device__ __forceinline__ int div_small(int x, int d) {  // d in 1..5
  switch (d) {
    case 1: return x;
    case 2: return x / 2;
    case 3: return x / 3;
    case 4: return x / 4;
    default: return x / 5;
  }
}

__device__ __forceinline__ Sched make_sched(int T, int num_units, int M, int fpm) {
  Sched sc;
  sc.U = min(num_units, max(T, 1));  // at most one unit per tile: no unit is empty
  sc.Lq = T / sc.U;
  sc.r = T - sc.Lq * sc.U;
  sc.Sq = static_cast<int>(static_cast<int64_t>(sc.Lq) * fpm / 1000);
  sc.Dq = sc.Lq - sc.Sq;
  sc.Sr = static_cast<int>(static_cast<int64_t>(sc.Lq + 1) * fpm / 1000);
  sc.Dr = sc.Lq + 1 - sc.Sr;
  // Balancing chunks only when every chunk of every unit gets a tile.
  sc.M = (M > 0 && sc.Sq >= 1 && sc.Dq >= M * (M + 1) / 2) ? M : 0;
  return sc;
}

__device__ __forceinline__ int unit_begin(const Sched& sc, int u) { return u * sc.Lq + min(u, sc.r); }

__device__ __forceinline__ int unit_of_tile(const Sched& sc, int k) {
  const int edge = sc.r * (sc.Lq + 1);
  return k < edge ? k / (sc.Lq + 1) : sc.r + (k - edge) / sc.Lq;
}

__device__ __forceinline__ void chunk_bounds(const Sched& sc, int c, int& k0, int& k1) {
  const int u = div_small(c, sc.M + 1), i = c - u * (sc.M + 1);
  const int a = unit_begin(sc, u);
  const bool longer = u < sc.r;
  if (sc.M == 0) {
    k0 = a;
    k1 = a + sc.Lq + longer;
    return;
  }
  const int S = longer ? sc.Sr : sc.Sq, D = longer ? sc.Dr : sc.Dq;
  if (i == 0) {
    k0 = a;
    k1 = a + S;
  } else {
    k0 = a + S + div_sub_weight(static_cast<int64_t>(D) * sub_cum(i - 1, sc.M), sc.M);
    k1 = a + S + div_sub_weight(static_cast<int64_t>(D) * sub_cum(i, sc.M), sc.M);
  }
}

__device__ __forceinline__ int chunk_of_tile(const Sched& sc, int k) {
  const int u = unit_of_tile(sc, k);
  if (sc.M == 0) return u;
  const int a = unit_begin(sc, u);
  const bool longer = u < sc.r;
  const int S = longer ? sc.Sr : sc.Sq, D = longer ? sc.Dr : sc.Dq;
  int i = 0;
  if (k >= a + S) {
    i = 1;
    while (i < sc.M && k >= a + S + div_sub_weight(static_cast<int64_t>(D) * sub_cum(i, sc.M), sc.M)) ++i;
  }
  return u * (sc.M + 1) + i;
}

// Byte offset of (token, dim) inside one K or V tile in shared memory: boxes of
// 16 rows x 128 bytes, one box per 128 bytes of head dim, 16-byte chunks
// swizzled by row (the TMA 128B swizzle).
template <int ES>
__device__ __forceinline__ uint32_t tile_offset(int tok, int dim) {
  constexpr int X = 128 / ES;
  const int y = dim / X;
  const int xb = (dim % X) * ES;
  return static_cast<uint32_t>(y * kBoxBytes + tok * 128 + ((((xb >> 4) ^ (tok & 7))) << 4) + (xb & 15));
}

// ---- tensor-core consumer (16-bit data, 2..16 query heads per kv head) ----
// kMQ: several queries per sequence (rows = query x head); query qi sees the
// context up to its own position, ctx - q_len + qi, so that in the tile that
// holds the sequence's last tokens each row has its own causal limit.
template <int DT, int D, int GPAD, bool kMQ = false>
struct MmaConsumer {
  static constexpr bool kBf16 = (DT == kBF16);
  static constexpr int ES = 2;
  using T = typename DTypeInfo<DT>::T;
  static constexpr int KS = D / 16;  // k-steps of QK
  static constexpr int NT = D / 8;   // n-tiles of PV

  uint32_t qa[KS][4];
  float o[NT][4];
  float m[2], l[2];
  int mq_gp = 1, mq_len = 1;  // kMQ: heads per query row block, queries per sequence

  __device__ __forceinline__ void set_mq(int gp, int q_len) {
    mq_gp = gp;
    mq_len = q_len;
  }

  // Q of the segment's gp heads from the warp's shared buffer ([gp][D]).
  __device__ __forceinline__ void begin(const uint8_t* qbuf, int gp, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const T* qb = reinterpret_cast<const T*>(qbuf);
    const bool r0 = g < gp;
    const bool r1 = (GPAD == 16) && (g + 8 < gp);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int c = ks * 16 + 2 * t;
      qa[ks][0] = r0 ? *reinterpret_cast<const uint32_t*>(qb + g * D + c) : 0u;
      qa[ks][2] = r0 ? *reinterpret_cast<const uint32_t*>(qb + g * D + c + 8) : 0u;
      qa[ks][1] = r1 ? *reinterpret_cast<const uint32_t*>(qb + (g + 8) * D + c) : 0u;
      qa[ks][3] = r1 ? *reinterpret_cast<const uint32_t*>(qb + (g + 8) * D + c + 8) : 0u;
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
  }

  // Continue from a given partial state (the segment's first piece only).
  __device__ __forceinline__ void load_init(const DecodeParams& p, int b, int hg, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const size_t nqb = static_cast<size_t>(p.batch) * p.n_q_heads;
    constexpr int kRows = (GPAD == 16) ? 2 : 1;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int row = g + 8 * r;
      if (row >= p.gp) continue;
      const size_t rowi = static_cast<size_t>(b) * p.n_q_heads + hg * p.gp + row;
      const float* oi = p.init + rowi * D;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const float2 x = __ldg(reinterpret_cast<const float2*>(oi + n * 8 + 2 * t));
        o[n][2 * r] = x.x;
        o[n][2 * r + 1] = x.y;
      }
      m[r] = __ldg(p.init + nqb * D + rowi);
      l[r] = t == 0 ? __ldg(p.init + nqb * D + nqb + rowi) : 0.f;
    }
  }

  __device__ __forceinline__ void tile(uint32_t kbase, uint32_t vbase, int nv, float scale_log2, int lane) {
    const int t = lane & 3;
    const int mi = lane >> 3, rr = lane & 7;

    // S = Q K^T: rows = query heads (g, g + 8), columns = tokens.
    float s[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk) {
      const int dim = (2 * kk + (mi >> 1)) * 16 + (mi & 1) * 8;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbase + tile_offset<ES>(nt * 8 + rr, dim), b0, b1, b2, b3);
        mma_16816<kBf16>(s[nt], qa[2 * kk][0], qa[2 * kk][1], qa[2 * kk][2], qa[2 * kk][3], b0, b1);
        mma_16816<kBf16>(s[nt], qa[2 * kk + 1][0], qa[2 * kk + 1][1], qa[2 * kk + 1][2], qa[2 * kk + 1][3],
                         b2, b3);
      }
    }

    // Online softmax.  Thread holds tokens nt*8 + 2t + e for rows g (s[.][0..1])
    // and g + 8 (s[.][2..3]).
    constexpr int kRows = (GPAD == 16) ? 2 : 1;
    float pr[2][2][2];  // [row][nt][e]
    bool grow = false;
    float alpha[2] = {1.f, 1.f};
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      // Tokens this row sees in the tile (kMQ: `nv` is the count of context
      // tokens from the tile's start on, unclamped; query qi stops
      // q_len - 1 - qi tokens before the context's end).
      const int nvr = kMQ ? min(kBlockTokens, nv - (mq_len - 1 - (lane / 4 + 8 * r) / mq_gp)) : nv;
      float x[2][2];
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int tok = nt * 8 + 2 * t + e;
          x[nt][e] = (tok < nvr) ? s[nt][2 * r + e] * scale_log2 : -INFINITY;
          mx = fmaxf(mx, x[nt][e]);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mn = fmaxf(m[r], mx);
      if (mn > m[r]) {
        grow = true;
        // kMQ: a row may have seen no token yet (m = -inf; O and l are 0).
        alpha[r] = (kMQ && m[r] == -INFINITY) ? 0.f : exp2f(m[r] - mn);
      }
      float sum = 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          // kMQ: a row with no token so far in this piece has mn = -inf.
          pr[r][nt][e] = (kMQ && x[nt][e] == -INFINITY) ? 0.f : exp2f(x[nt][e] - mn);
          sum += pr[r][nt][e];
        }
      l[r] = l[r] * alpha[r] + sum;
      m[r] = mn;
    }
    if (__any_sync(0xffffffffu, grow)) {
      const float a_lo = alpha[0];
      const float a_hi = (GPAD == 16) ? alpha[1] : alpha[0];
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        o[n][0] *= a_lo;
        o[n][1] *= a_lo;
        o[n][2] *= a_hi;
        o[n][3] *= a_hi;
      }
    }

    // P as the A operand of P V: a0/a2 = row g, tokens 2t.. / 8+2t..; a1/a3 =
    // row g + 8 (the next 8 heads, or the residual of row g).
    uint32_t pa0 = pack2<kBf16>(pr[0][0][0], pr[0][0][1]);
    uint32_t pa2 = pack2<kBf16>(pr[0][1][0], pr[0][1][1]);
    uint32_t pa1, pa3;
    if constexpr (GPAD == 16) {
      pa1 = pack2<kBf16>(pr[1][0][0], pr[1][0][1]);
      pa3 = pack2<kBf16>(pr[1][1][0], pr[1][1][1]);
    } else {
      float h00, h01, h10, h11;
      unpack2<kBf16>(pa0, h00, h01);
      unpack2<kBf16>(pa2, h10, h11);
      pa1 = pack2<kBf16>(pr[0][0][0] - h00, pr[0][0][1] - h01);
      pa3 = pack2<kBf16>(pr[0][1][0] - h10, pr[0][1][1] - h11);
    }

    // Rows of V past the context may hold anything (NaN included): zero them.
    const int nvt = kMQ ? min(nv, kBlockTokens) : nv;
    uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;
    if (nvt < kBlockTokens) {
      vm0 = ((2 * t < nvt) ? 0x0000ffffu : 0u) | ((2 * t + 1 < nvt) ? 0xffff0000u : 0u);
      vm1 = ((2 * t + 8 < nvt) ? 0x0000ffffu : 0u) | ((2 * t + 9 < nvt) ? 0xffff0000u : 0u);
    }
#pragma unroll
    for (int nd2 = 0; nd2 < D / 16; ++nd2) {
      const int tok = (mi & 1) * 8 + rr;
      const int dim = (2 * nd2 + (mi >> 1)) * 8;
      uint32_t v0, v1, v2, v3;
      ldsm_x4_trans(vbase + tile_offset<ES>(tok, dim), v0, v1, v2, v3);
      v0 &= vm0;
      v2 &= vm0;
      v1 &= vm1;
      v3 &= vm1;
      mma_16816<kBf16>(o[2 * nd2], pa0, pa1, pa2, pa3, v0, v1);
      mma_16816<kBf16>(o[2 * nd2 + 1], pa0, pa1, pa2, pa3, v2, v3);
    }
  }

  // Write either the normalised output rows or an unnormalised partial record.
  __device__ __forceinline__ void finish(const DecodeParams& p, int b, int hg, float* rec, int lane) {
    const int g = lane >> 2, t = lane & 3;
    float lt[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float x = l[r];
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      lt[r] = x;
    }
    constexpr int kRows = (GPAD == 16) ? 2 : 1;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int row = g + 8 * r;
      if (row >= p.rows) continue;
      if (rec == nullptr) {
        T* ob = static_cast<T*>(p.out) + out_row(p, b, hg, row) * D;
        // lt is 0 only when every tile of the row was skipped (bad block ids): a zero row.
        const float inv = lt[r] > 0.f ? 1.f / lt[r] : 0.f;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          float a0, a1;
          if constexpr (GPAD == 16) {
            a0 = o[n][2 * r];
            a1 = o[n][2 * r + 1];
          } else {
            a0 = o[n][0] + o[n][2];
            a1 = o[n][1] + o[n][3];
          }
          *reinterpret_cast<uint32_t*>(ob + n * 8 + 2 * t) = pack2<kBf16>(a0 * inv, a1 * inv);
        }
      } else {
        if (t == 0) {
          rec[p.rows * D + row] = m[r];
          rec[p.rows * D + p.rows + row] = lt[r];
        }
        float* ro = rec + row * D;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          float a0, a1;
          if constexpr (GPAD == 16) {
            a0 = o[n][2 * r];
            a1 = o[n][2 * r + 1];
          } else {
            a0 = o[n][0] + o[n][2];
            a1 = o[n][1] + o[n][3];
          }
          *reinterpret_cast<float2*>(ro + n * 8 + 2 * t) = make_float2(a0, a1);
        }
      }
    }
  }
};

// ---- CUDA-core consumer (one query head per segment; any dtype) ----
template <int DT, int D>
struct SimtConsumer {
  static constexpr int ES = DTypeInfo<DT>::kBytes;
  using T = typename DTypeInfo<DT>::T;
  static constexpr int DL = D / 4;        // dims per lane
  static constexpr int EPC = 16 / ES;     // elements per 16-byte chunk
  static constexpr int NCH = DL / EPC;    // chunks per lane row slice
  static constexpr int DO = DL / 8;       // output dims per lane after the reduce-scatter

  float qs[DL];
  float o[DL];
  float m, l;

  __device__ __forceinline__ static void widen16(const uint4& c, float* f) {
    if constexpr (DT == kF32) {
      f[0] = __uint_as_float(c.x);
      f[1] = __uint_as_float(c.y);
      f[2] = __uint_as_float(c.z);
      f[3] = __uint_as_float(c.w);
    } else {
      constexpr bool kB = (DT == kBF16);
      unpack2<kB>(c.x, f[0], f[1]);
      unpack2<kB>(c.y, f[2], f[3]);
      unpack2<kB>(c.z, f[4], f[5]);
      unpack2<kB>(c.w, f[6], f[7]);
    }
  }

  // This lane's dim slice of the segment's one query head, from the warp's
  // shared buffer.
  __device__ __forceinline__ void begin(const uint8_t* qbuf, int /*gp*/, int lane) {
    const int sub = lane >> 3;
    const uint4* qb = reinterpret_cast<const uint4*>(qbuf + sub * DL * ES);
#pragma unroll
    for (int c = 0; c < NCH; ++c) widen16(qb[c], qs + c * EPC);
#pragma unroll
    for (int i = 0; i < DL; ++i) o[i] = 0.f;
    m = -INFINITY;
    l = 0.f;
  }

  // Continue from a given partial state (the segment's first piece only):
  // the token lanes' partial sums are added up at the end, so lane tp == 0
  // carries the initial O and l.
  __device__ __forceinline__ void load_init(const DecodeParams& p, int b, int hg, int lane) {
    const int tp = lane & 7, sub = lane >> 3;
    const size_t nqb = static_cast<size_t>(p.batch) * p.n_q_heads;
    const size_t rowi = static_cast<size_t>(b) * p.n_q_heads + hg;
    const float* oi = p.init + rowi * D + sub * DL;
#pragma unroll
    for (int i = 0; i < DL; ++i) o[i] = tp == 0 ? __ldg(oi + i) : 0.f;
    m = __ldg(p.init + nqb * D + rowi);
    l = tp == 0 ? __ldg(p.init + nqb * D + nqb + rowi) : 0.f;
  }

  __device__ __forceinline__ void tile(uint32_t kbase, uint32_t vbase, int nv, float scale_log2, int lane) {
    const int tp = lane & 7, sub = lane >> 3;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int dim = sub * DL + c * EPC;
      uint4 k0, k1;
      asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(k0.x), "=r"(k0.y), "=r"(k0.z), "=r"(k0.w)
                   : "r"(kbase + tile_offset<ES>(tp, dim)));
      asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(k1.x), "=r"(k1.y), "=r"(k1.z), "=r"(k1.w)
                   : "r"(kbase + tile_offset<ES>(tp + 8, dim)));
      float f0[EPC], f1[EPC];
      widen16(k0, f0);
      widen16(k1, f1);
#pragma unroll
      for (int e = 0; e < EPC; ++e) {
        s0 = fmaf(qs[c * EPC + e], f0[e], s0);
        s1 = fmaf(qs[c * EPC + e], f1[e], s1);
      }
    }
    s0 += __shfl_xor_sync(0xffffffffu, s0, 8);
    s0 += __shfl_xor_sync(0xffffffffu, s0, 16);
    s1 += __shfl_xor_sync(0xffffffffu, s1, 8);
    s1 += __shfl_xor_sync(0xffffffffu, s1, 16);
    const bool ok0 = tp < nv, ok1 = tp + 8 < nv;
    const float x0 = ok0 ? s0 * scale_log2 : -INFINITY;
    const float x1 = ok1 ? s1 * scale_log2 : -INFINITY;
    float mx = fmaxf(x0, x1);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    const float mn = fmaxf(m, mx);
    if (mn > m) {  // warp-uniform: m and mx are the same in every lane
      const float alpha = exp2f(m - mn);
      l *= alpha;
#pragma unroll
      for (int i = 0; i < DL; ++i) o[i] *= alpha;
      m = mn;
    }
    const float p0 = exp2f(x0 - mn), p1 = exp2f(x1 - mn);
    l += p0 + p1;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int dim = sub * DL + c * EPC;
      float f[EPC];
      if (ok0) {
        uint4 v0;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(v0.x), "=r"(v0.y), "=r"(v0.z), "=r"(v0.w)
                     : "r"(vbase + tile_offset<ES>(tp, dim)));
        widen16(v0, f);
#pragma unroll
        for (int e = 0; e < EPC; ++e) o[c * EPC + e] = fmaf(p0, f[e], o[c * EPC + e]);
      }
      if (ok1) {
        uint4 v1;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(v1.x), "=r"(v1.y), "=r"(v1.z), "=r"(v1.w)
                     : "r"(vbase + tile_offset<ES>(tp + 8, dim)));
        widen16(v1, f);
#pragma unroll
        for (int e = 0; e < EPC; ++e) o[c * EPC + e] = fmaf(p1, f[e], o[c * EPC + e]);
      }
    }
  }

  __device__ __forceinline__ void finish(const DecodeParams& p, int b, int hg, float* rec, int lane) {
    const int tp = lane & 7, sub = lane >> 3;
    float lt = l;
    lt += __shfl_xor_sync(0xffffffffu, lt, 1);
    lt += __shfl_xor_sync(0xffffffffu, lt, 2);
    lt += __shfl_xor_sync(0xffffffffu, lt, 4);
    // Reduce-scatter of o over the 8 token lanes: after the three steps lane
    // tp holds dims [tp * DO, tp * DO + DO) of its slice, summed.
#pragma unroll
    for (int step = 0; step < 3; ++step) {
      const int mask = 4 >> step;
      const int half = DL >> (step + 1);
      const bool upper = (tp & mask) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send = upper ? o[i] : o[i + half];
        const float keep = upper ? o[i + half] : o[i];
        o[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
      }
    }
    const int d0 = sub * DL + tp * DO;
    if (rec == nullptr) {
      T* ob = static_cast<T*>(p.out) + (static_cast<size_t>(b) * p.n_q_heads + hg) * D + d0;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;  // 0: every tile skipped
      if constexpr (DT == kF32) {
#pragma unroll
        for (int i = 0; i < DO; ++i) ob[i] = o[i] * inv;
      } else {
#pragma unroll
        for (int i = 0; i < DO; i += 2)
          *reinterpret_cast<uint32_t*>(ob + i) = pack2<DT == kBF16>(o[i] * inv, o[i + 1] * inv);
      }
    } else {
      if (lane == 0) {
        rec[D] = m;
        rec[D + 1] = lt;
      }
#pragma unroll
      for (int i = 0; i < DO; ++i) rec[d0 + i] = o[i];
    }
  }
};

// ---- tensor-core consumer over the INT8 cache (head_dim 128) ----
// K tile: 16 rows of 128 one-byte codes, TMA 128B swizzle (16-byte chunk c of
// row r at chunk c ^ (r % 8)).  V tile: 128 rows (dims) of 16 bytes (tokens,
// in vpos_i8 order).  Then 16 fp32 K scales and 16 V scales (token order).
//
// S = Q K^T runs on the integer tensor-core path (mma m16n8k32 s8): each Q
// row is put on a 14-bit grid once per segment, q ~ sq * (128 hi + lo) with
// sq = max|q| / 8191 and hi, lo signed 8-bit, so that S = sq * sk * (128
// (hi . k) + (lo . k)) with exact int32 dot products over the K codes (the
// grid's rounding, at most sq / 2 per element, is the only approximation).
// The dot product over the head dim does not depend on the order of the
// dims, so lane t owns dims [32t, 32t + 32): k-step kk takes dims 32t + 8kk
// + [0, 4) as the fragment's columns 4t.. and 32t + 8kk + [4, 8) as columns
// 16 + 4t.., for Q and K alike; a lane's K codes of one row are two 16-byte
// loads that the swizzle keeps free of bank conflicts.
//
// O += P V runs in f16 with V codes turned into exact f16 values.  The V
// scale of token t enters through the probabilities, p * vs_t / c, where c
// is the largest V scale seen so far by the warp: the factors stay in [0, 1]
// (f16 range), O is rescaled when c grows, and O * c is the true sum.
template <int DT, int GPAD>
struct MmaConsumerI8 : MmaConsumer<DT, 128, GPAD> {
  using Base = MmaConsumer<DT, 128, GPAD>;
  using T = typename Base::T;
  static constexpr bool kBf16 = Base::kBf16;
  static constexpr int D = 128;
  static constexpr int NT = D / 8;
  using Base::l;
  using Base::m;
  using Base::o;
  using Base::qa;  // qa[kk] = hi, qa[4 + kk] = lo, k-steps kk = 0..3
  float qs[2];     // grid step of rows g and g + 8
  float cv;        // largest V scale seen (0 before the first tile)
  float inv_cv;    // 1 / cv (0 while cv is 0)

  // Q row `row` (this lane's 32 dims) on the 14-bit grid.
  __device__ __forceinline__ void split_row(const T* qr, bool live, int t, int slot) {
    float x[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t w = live ? *reinterpret_cast<const uint32_t*>(qr + 32 * t + 2 * i) : 0u;
      unpack2<kBf16>(w, x[2 * i], x[2 * i + 1]);
    }
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) mx = fmaxf(mx, fabsf(x[i]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float inv = mx > 0.f ? 8191.f / mx : 0.f;
    qs[slot] = mx / 8191.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t h[2] = {0u, 0u}, lo[2] = {0u, 0u};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int qi = __float2int_rn(x[8 * kk + j] * inv);  // |qi| <= 8191
        const int hi = (qi + 64) >> 7;                        // [-64, 64]
        const int lw = qi - (hi << 7);                        // [-64, 63]
        h[j >> 2] |= (static_cast<uint32_t>(hi) & 0xffu) << (8 * (j & 3));
        lo[j >> 2] |= (static_cast<uint32_t>(lw) & 0xffu) << (8 * (j & 3));
      }
      // a0 / a2 carry row g (columns 4t.. and 16 + 4t..); a1 / a3 row g + 8.
      qa[kk][slot] = h[0];
      qa[kk][2 + slot] = h[1];
      qa[4 + kk][slot] = lo[0];
      qa[4 + kk][2 + slot] = lo[1];
    }
  }

  __device__ __forceinline__ void begin(const uint8_t* qbuf, int gp, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const T* qb = reinterpret_cast<const T*>(qbuf);
    split_row(qb + g * D, g < gp, t, 0);
    if constexpr (GPAD == 16) {
      split_row(qb + (g + 8) * D, g + 8 < gp, t, 1);
    } else {
      qs[1] = 0.f;
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
    cv = 0.f;
    inv_cv = 0.f;
  }

  __device__ __forceinline__ void tile(uint32_t kbase, uint32_t vbase, int nv, float scale_log2, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const uint32_t sbase = vbase + D * kBlockTokens;  // K scales, then V scales

    // Integer S for tokens g (n-tile 0) and g + 8 (n-tile 1).
    float s[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int row = nt * 8 + g;
      uint4 c0, c1;
      asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(c0.x), "=r"(c0.y), "=r"(c0.z), "=r"(c0.w)
                   : "r"(kbase + row * 128 + (((2 * t) ^ (row & 7)) << 4)));
      asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(c1.x), "=r"(c1.y), "=r"(c1.z), "=r"(c1.w)
                   : "r"(kbase + row * 128 + (((2 * t + 1) ^ (row & 7)) << 4)));
      const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      if constexpr (GPAD == 16) {
        int ah[4] = {0, 0, 0, 0}, al[4] = {0, 0, 0, 0};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          mma_16832_s8(ah, qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], w[2 * kk], w[2 * kk + 1]);
          mma_16832_s8(al, qa[4 + kk][0], qa[4 + kk][1], qa[4 + kk][2], qa[4 + kk][3], w[2 * kk], w[2 * kk + 1]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = static_cast<float>(ah[e] * 128 + al[e]);
      } else {
        // At most 8 rows: the high parts of Q go in A's rows 0-7 and the low
        // parts in rows 8-15, so that one MMA per k-step gives both dot
        // products, in the same lane (c0, c1: high; c2, c3: low).
        int a[4] = {0, 0, 0, 0};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_16832_s8(a, qa[kk][0], qa[4 + kk][0], qa[kk][2], qa[4 + kk][2], w[2 * kk], w[2 * kk + 1]);
        s[nt][0] = static_cast<float>(a[0] * 128 + a[2]);
        s[nt][1] = static_cast<float>(a[1] * 128 + a[3]);
        s[nt][2] = s[nt][3] = 0.f;  // rows 8-15: none
      }
    }
    // Scales: the row's grid step and the K scale of this lane's columns
    // (tokens 2t, 2t + 1 and 2t + 8, 2t + 9).
    float2 ks0, ks1;
    asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(ks0.x), "=f"(ks0.y) : "r"(sbase + 8 * t));
    asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(ks1.x), "=f"(ks1.y) : "r"(sbase + 32 + 8 * t));
    s[0][0] *= qs[0] * ks0.x;
    s[0][1] *= qs[0] * ks0.y;
    s[0][2] *= qs[1] * ks0.x;
    s[0][3] *= qs[1] * ks0.y;
    s[1][0] *= qs[0] * ks1.x;
    s[1][1] *= qs[0] * ks1.y;
    s[1][2] *= qs[1] * ks1.x;
    s[1][3] *= qs[1] * ks1.y;

    // Online softmax (as in the 16-bit consumer).
    constexpr int kRows = (GPAD == 16) ? 2 : 1;
    float pr[2][2][2];
    bool grow = false;
    float alpha[2] = {1.f, 1.f};
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      float x[2][2];
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int tok = nt * 8 + 2 * t + e;
          x[nt][e] = (tok < nv) ? s[nt][2 * r + e] * scale_log2 : -INFINITY;
          mx = fmaxf(mx, x[nt][e]);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mn = fmaxf(m[r], mx);
      if (mn > m[r]) {
        grow = true;
        alpha[r] = exp2f(m[r] - mn);
      }
      float sum = 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          pr[r][nt][e] = exp2f(x[nt][e] - mn);
          sum += pr[r][nt][e];
        }
      l[r] = l[r] * alpha[r] + sum;
      m[r] = mn;
    }

    // V scales of this lane's tokens; the largest over the tile's live tokens
    // (scales past the context may be anything, NaN included).
    float2 vs0, vs1;
    asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(vs0.x), "=f"(vs0.y) : "r"(sbase + 64 + 8 * t));
    asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(vs1.x), "=f"(vs1.y) : "r"(sbase + 96 + 8 * t));
    float vsc[2][2] = {{vs0.x, vs0.y}, {vs1.x, vs1.y}};
    float vmax = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool live = nt * 8 + 2 * t + e < nv;
        vsc[nt][e] = live ? vsc[nt][e] : 0.f;
        vmax = fmaxf(vmax, vsc[nt][e]);
      }
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 1));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 2));
    const float cn = fmaxf(cv, vmax);
    const bool cgrow = cn > cv;  // warp-uniform (cv, vmax are)
    float rc = 1.f;
    if (cgrow) {
      rc = cv / cn;  // 0 on the first tile (O is 0 then)
      inv_cv = 1.f / cn;
      cv = cn;
    }
    if (__any_sync(0xffffffffu, grow || cgrow)) {
      const float a_lo = alpha[0] * rc;
      const float a_hi = ((GPAD == 16) ? alpha[1] : alpha[0]) * rc;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        o[n][0] *= a_lo;
        o[n][1] *= a_lo;
        o[n][2] *= a_hi;
        o[n][3] *= a_hi;
      }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) vsc[nt][e] *= inv_cv;
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) pr[r][nt][e] *= vsc[nt][e];

    uint32_t pa0 = pack2<false>(pr[0][0][0], pr[0][0][1]);
    uint32_t pa2 = pack2<false>(pr[0][1][0], pr[0][1][1]);
    uint32_t pa1, pa3;
    if constexpr (GPAD == 16) {
      pa1 = pack2<false>(pr[1][0][0], pr[1][0][1]);
      pa3 = pack2<false>(pr[1][1][0], pr[1][1][1]);
    } else {
      float h00, h01, h10, h11;
      unpack2<false>(pa0, h00, h01);
      unpack2<false>(pa2, h10, h11);
      pa1 = pack2<false>(pr[0][0][0] - h00, pr[0][0][1] - h01);
      pa3 = pack2<false>(pr[0][1][0] - h10, pr[0][1][1] - h11);
    }

    // O += P V in f16: V^T row 8n + g holds dim 8n + g of all 16 tokens; bytes
    // 4t .. 4t + 3 are tokens 2t, 2t + 1, 2t + 8, 2t + 9 (codes are finite, so
    // the rows past the context need no mask: their factors are 0).
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      uint32_t w;
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w) : "r"(vbase + (8 * n + g) * kBlockTokens + 4 * t));
      mma_16816<false>(o[n], pa0, pa1, pa2, pa3, i8x2_to_16x2<false>(w, 0), i8x2_to_16x2<false>(w, 1));
    }
  }

  // O in true units (times c) before the 16-bit consumer's epilogue.
  __device__ __forceinline__ void finish(const DecodeParams& p, int b, int hg, float* rec, int lane) {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      o[n][0] *= cv;
      o[n][1] *= cv;
      o[n][2] *= cv;
      o[n][3] *= cv;
    }
    Base::finish(p, b, hg, rec, lane);
  }
};

template <int DT, int D, int GPAD, bool kI8 = false, bool kMQ = false>
struct ConsumerFor {
  using type = MmaConsumer<DT, D, GPAD, kMQ>;
};
template <int DT, int D>
struct ConsumerFor<DT, D, 0, false, false> {
  using type = SimtConsumer<DT, D>;
};
template <int DT, int GPAD>
struct ConsumerFor<DT, 128, GPAD, true, false> {
  using type = MmaConsumerI8<DT, GPAD>;
};

// Four fp32 values rounded to the output dtype and stored together.
template <int DT>
__device__ __forceinline__ void store4(typename DTypeInfo<DT>::T* dst, float a, float b, float c, float d) {
  if constexpr (DT == kF32) {
    *reinterpret_cast<float4*>(dst) = make_float4(a, b, c, d);
  } else {
    uint2 v;
    v.x = pack2<DT == kBF16>(a, b);
    v.y = pack2<DT == kBF16>(c, d);
    *reinterpret_cast<uint2*>(dst) = v;
  }
}

// Prefetch this CTA's 1/gridDim share of a buffer of `bytes` (a multiple of
// 16, 16-byte aligned) into L2.
__device__ __forceinline__ void prefetch_slice_l2(const void* base, size_t bytes) {
  const size_t slice = ((bytes / gridDim.x) + 15) & ~static_cast<size_t>(15);
  const size_t off = slice * blockIdx.x;
  if (slice > 0 && off < bytes) {
    const size_t n = bytes - off < slice ? bytes - off : slice;
    bulk_prefetch_l2(static_cast<const uint8_t*>(base) + off, static_cast<uint32_t>(n));
  }
}

// Copy the rows x head_dim Q rows of segment (b, hg) into a warp's shared
// buffer with 16-byte cp.async (completion: cp_async_wait_all + __syncwarp).
template <int ES, int D>
__device__ __forceinline__ void q_fetch(uint8_t* qbuf, const DecodeParams& p, int b, int hg, int lane) {
  constexpr int kRowChunks = D * ES / 16;
  const uint8_t* q = static_cast<const uint8_t*>(p.q);
  for (int c = lane; c < p.rows * kRowChunks; c += 32) {
    const int row = c / kRowChunks, w = c - row * kRowChunks;
    cp_async_16(qbuf + c * 16, q + (out_row(p, b, hg, row) * D * ES) + w * 16);
  }
  cp_async_commit();
}

// Where the partial records of one split segment are: piece 0 in chunk u1,
// record slot z (0: the segment is the chunk's first, 1: its last); piece j
// >= 1 in chunk base + j * step, slot 0 (the segment continues there from
// the previous chunk).  n pieces in all.
struct MergeSrc {
  int u1, z, n, base, step;
};

// Combines dims [d0, d0 + 32 DPL) of row g of segment (b, hg) from its
// pieces, in piece order, as an online merge over batches of 8 pieces:
//   M = max_i m_i,  w_i = 2^(m_i - M),  O = sum_i w_i O_i,  l = sum_i w_i l_i
// (the running O and l are rescaled by 2^(M_old - M_new) when a batch raises
// the maximum).  With to_rec null the result is normalised and written to
// `out` (rounded to nearest even); otherwise the unnormalised state (O, M, l)
// is written into the record `to_rec` (piece 0's own record: every load
// comes before the stores).  Each lane owns DPL dims of O.  A batch's loads
// (m, l and the lane's O slice of 8 pieces) go out together, in program order
// (ld.global.cg: other SMs, or other warps of this CTA, wrote the records
// before a barrier), so that a batch costs one round trip to L2.
template <int DT, int D, int DPL>
__device__ __forceinline__ void merge_rows(const DecodeParams& p, const MergeSrc& src, int b, int hg, int g, int d0,
                                           int lane, float* to_rec) {
  using T = typename DTypeInfo<DT>::T;
  constexpr int kBatch = DPL == 1 ? 16 : 8;  // pieces per round: 3 kBatch + kBatch DPL registers
  const int n = src.n;
  const int mo = p.rows * D + g, lo = p.rows * D + p.rows + g, oo = g * D + d0 + lane * DPL;
  float M = -INFINITY, L = 0.f, acc[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
  for (int j0 = 0; j0 < n; j0 += kBatch) {
    float mj[kBatch], lj[kBatch], o[kBatch][DPL];
#pragma unroll
    for (int jj = 0; jj < kBatch; ++jj) {
      const int j = min(j0 + jj, n - 1);
      const int chunk = j == 0 ? src.u1 : src.base + j * src.step;
      const float* r = p.records + (static_cast<size_t>(chunk) * 2 + (j == 0 ? src.z : 0)) * p.rec_floats;
      mj[jj] = ld_cg(r + mo);
      lj[jj] = ld_cg(r + lo);
      if constexpr (DPL == 8) {
        const float4 v = ld_cg4(r + oo), w = ld_cg4(r + oo + 4);
        o[jj][0] = v.x; o[jj][1] = v.y; o[jj][2] = v.z; o[jj][3] = v.w;
        o[jj][4] = w.x; o[jj][5] = w.y; o[jj][6] = w.z; o[jj][7] = w.w;
      } else if constexpr (DPL == 4) {
        const float4 v = ld_cg4(r + oo);
        o[jj][0] = v.x; o[jj][1] = v.y; o[jj][2] = v.z; o[jj][3] = v.w;
      } else if constexpr (DPL == 2) {
        const float2 v = ld_cg2(r + oo);
        o[jj][0] = v.x; o[jj][1] = v.y;
      } else {
        o[jj][0] = ld_cg(r + oo);
      }
    }
    float Mb = M;
#pragma unroll
    for (int jj = 0; jj < kBatch; ++jj)
      if (j0 + jj < n) Mb = fmaxf(Mb, mj[jj]);
    // M (and Mb) stay -inf only while every piece so far skipped all its
    // tiles (bad block ids): those weights are 0 and the state stays empty.
    const float alpha = M == -INFINITY ? 0.f : exp2f(M - Mb);
    L *= alpha;
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] *= alpha;
#pragma unroll
    for (int jj = 0; jj < kBatch; ++jj) {
      const float w = (j0 + jj < n && Mb != -INFINITY) ? exp2f(mj[jj] - Mb) : 0.f;
      L = fmaf(w, lj[jj], L);
#pragma unroll
      for (int i = 0; i < DPL; ++i) acc[i] = fmaf(w, o[jj][i], acc[i]);
    }
    M = Mb;
  }
  if (to_rec != nullptr) {
    float* ro = to_rec + oo;
#pragma unroll
    for (int i = 0; i < DPL; ++i) ro[i] = acc[i];
    if (lane == 0 && d0 == 0) {
      to_rec[mo] = M;
      to_rec[lo] = L;
    }
    return;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;  // L is 0 only when every piece skipped all its tiles
  T* const ob = static_cast<T*>(p.out) + out_row(p, b, hg, g) * D + d0 + lane * DPL;
  if constexpr (DPL == 8) {
    store4<DT>(ob, acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    store4<DT>(ob + 4, acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
  } else if constexpr (DPL == 4) {
    store4<DT>(ob, acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  } else if constexpr (DT == kF32) {
#pragma unroll
    for (int i = 0; i < DPL; ++i) ob[i] = acc[i] * inv;
  } else if constexpr (DPL == 2) {
    *reinterpret_cast<uint32_t*>(ob) = pack2<DT == kBF16>(acc[0] * inv, acc[1] * inv);
  } else {
    ob[0] = static_cast<T>(acc[0] * inv);  // round to nearest even
  }
}

// Tile range [start, end) of segment (b, hg) from the block-wide prefix sums.
__device__ __forceinline__ void segment_tiles(const int* prefix, const int* ctxs, int b, int hg, int& start,
                                              int& end) {
  const int nb = (ctxs[b] + kBlockTokens - 1) / kBlockTokens;
  start = prefix[b] + hg * nb;
  end = start + nb;
}

// kFused: the launch first writes the new tokens of p.app into the cache
// (paged_kv_append_and_decode); a separate instantiation, so that the plain
// decode's register allocation does not carry the fused prologue.
template <int DT, int D, int GPAD, bool kI8, bool kMQ, bool kFused = false>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    pkv_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const DecodeParams p) {
  constexpr int ES = DTypeInfo<DT>::kBytes;
  constexpr int X = 128 / ES;                      // elements per swizzle row
  constexpr int Y = D / X;                         // boxes per tile
  constexpr int kTileBytes = Y * kBoxBytes;
  // Ring slots (1 KiB aligned for the swizzle; INT8 records on 128-byte
  // multiples, which keeps their pre-swizzled K rows conflict-free).
  constexpr int kRingStride = kI8 ? i8_record_bytes(D) : 2 * kTileBytes;
  constexpr int kStageBytes = kRingStride;  // bytes landing per slot
  constexpr int kQBufBytes = (GPAD == 0 ? 1 : GPAD) * D * ES;
  using Consumer = typename ConsumerFor<DT, D, GPAD, kI8, kMQ>::type;
  using OutT = typename DTypeInfo<DT>::T;
  static_assert(!kI8 || (D == 128 && GPAD != 0), "INT8 cache: head_dim 128, tensor-core consumer");
  static_assert(!kMQ || (GPAD != 0 && !kI8), "several queries: 16-bit cache, tensor-core consumer");

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* ring = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int n_slots = kConsumerWarps * p.stages;
  uint8_t* qbufs = ring + static_cast<size_t>(n_slots) * kRingStride;  // [warps][kQBufBytes]
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(qbufs + kConsumerWarps * kQBufBytes);
  uint64_t* empty_bar = full_bar + n_slots;
  int4* slot_info = reinterpret_cast<int4*>(empty_bar + n_slots);  // [n_slots]: next chunk, from the producer
  volatile int* abort_flag = reinterpret_cast<volatile int*>(slot_info + n_slots);
  int* prefix = const_cast<int*>(reinterpret_cast<volatile int*>(abort_flag + 4));  // [batch + 1]
  int* ctxs = prefix + p.batch + 1;                                                    // [batch]
  __shared__ int warp_sums[kConsumerWarps + 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = p.batch;
  const int max_ctx = p.max_blocks_per_seq * kBlockTokens;

  if (threadIdx.x == 0) {
    for (int i = 0; i < n_slots; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
    // Bring this CTA's slices of q and of the block table into L2: the
    // consumers' Q copies and the producers' block-id loads then hit L2.
    prefetch_slice_l2(p.q, static_cast<size_t>(B) * p.n_q_heads * D * ES);
    if ((reinterpret_cast<uintptr_t>(p.block_tables) & 15u) == 0)
      prefetch_slice_l2(p.block_tables, static_cast<size_t>(B) * p.max_blocks_per_seq * sizeof(int32_t) & ~size_t(15));
  }
  if (!kI8 && warp == kConsumerWarps && lane == 0) {  // the INT8 cache uses no tensor map
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }

  // Fused append: every thread of the grid writes its share of the new
  // tokens' rows, then arrives on the grid barrier; the wait comes after the
  // scan below, before any tile is read.  The proxy fence makes the rows,
  // written through the generic proxy, visible to the TMA reads (async
  // proxy) that follow the barrier.
  constexpr bool fused_append = kFused;
  [[maybe_unused]] unsigned int app_token = 0;
  const int scan_per = (B + kDecodeThreads - 1) / kDecodeThreads;
  const int scan_lo = min(B, static_cast<int>(threadIdx.x) * scan_per), scan_hi = min(B, scan_lo + scan_per);
  // Fused: this thread's first context length is read before the append, so
  // that the two reads overlap.
  [[maybe_unused]] int ctx_first = 0;
  if constexpr (fused_append) {
    if (scan_lo < scan_hi) ctx_first = __ldg(p.context_lens + scan_lo);
    app_token = fused_append_arrive(p.app, blockIdx.x * static_cast<int64_t>(kDecodeThreads) + threadIdx.x,
                                    static_cast<int64_t>(gridDim.x) * kDecodeThreads);
  }

  // Tiles per sequence -> exclusive prefix sums (block-wide scan).
  {
    const int lo = scan_lo, hi = scan_hi;
    int local = 0;
    for (int b = lo; b < hi; ++b) {
      int c0;
      if constexpr (fused_append)
        c0 = b == lo ? ctx_first : __ldg(p.context_lens + b);
      else
        c0 = __ldg(p.context_lens + b);
      int c = clamp_ctx(c0, max_ctx);
      if (c > 0 && c < p.q_len) c = 0;  // fewer tokens than queries: flagged, no output but zeros
      if (c != c0) flag_error(PKV_DEVERR_CONTEXT);
      ctxs[b] = c;
      local += ((c + kBlockTokens - 1) / kBlockTokens) * p.ng;
    }
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_sums[w];
    int run = base + incl - local;
    for (int b = lo; b < hi; ++b) {
      prefix[b] = run;
      run += ((ctxs[b] + kBlockTokens - 1) / kBlockTokens) * p.ng;
    }
    if (threadIdx.x == kDecodeThreads - 1) prefix[B] = base + incl;
  }
  if constexpr (fused_append)
    cooperative_groups::this_grid().barrier_wait(static_cast<unsigned int&&>(app_token));  // ends with a CTA barrier
  else
    __syncthreads();

  const int T = prefix[B];
  const Sched sc = make_sched(T, p.num_units, p.sub_chunks, p.static_permille);
  const int U = sc.U, M = sc.M;
  const int n_chunks = U * (M + 1);

  if (warp == kConsumerWarps) {
    // ---------------- producer ----------------
    // Lane w feeds consumer warp w: first its unit's own chunk, then the
    // balancing chunks it claims.  Lanes never wait for each other: each polls
    // its own next ring slot (non-blocking test of the empty barrier) and
    // issues the TMA loads when the slot is free.  The next two tiles are
    // resolved ahead.  Nothing fetched from global memory is used in the
    // iteration that fetches it: a physical block id is checked when its tile
    // is issued, and the claim of the next chunk is sent kClaimAhead tiles
    // before the current chunk's end and read at its last tile, so the warp
    // (whose lanes run in step) never waits on an L2 round trip.
    if constexpr (fused_append) asm volatile("fence.proxy.async.global;" ::: "memory");
    const uint64_t kv_policy = l2_policy_evict_first();  // each K/V tile is read once
    const int u = blockIdx.x * kConsumerWarps + lane;
    // Test hook: the lane of the withheld unit never issues, so that its
    // consumer's bounded wait runs out (no copy is then in flight for it).
    const bool withheld = u == p.withhold_unit;
    Walk wn;
    bool walking = false;
    if (lane < kConsumerWarps && u < U) {
      int k0, k1;
      chunk_bounds(sc, u * (M + 1), k0, k1);
      walking = walk_begin(wn, prefix, ctxs, B, k0, k1);
    }
    int ticket = -1;
    bool claimed = false;
    struct Ahead {
      int phys, kvh;
      int4 info;  // {next chunk, its first tile, its end, 0} on a chunk's last tile, else next chunk -2
      bool valid;
    };
    auto resolve = [&](Ahead& t) {
      t.valid = walking;
      if (!walking) return;
      t.phys = __ldg(p.block_tables + static_cast<size_t>(wn.b) * p.max_blocks_per_seq + wn.j);
      t.kvh = (wn.hg * p.gp) / p.group;
      t.info = make_int4(-2, 0, 0, 0);
      if (M > 0 && !claimed && wn.k + kClaimAhead >= wn.k_end) {
        ticket = atomicAdd(p.sched, 1);
        claimed = true;
      }
      if (wn.k + 1 < wn.k_end) {
        walk_next(wn, prefix, ctxs, B, p.ng);
        return;
      }
      walking = false;
      t.info.x = -1;
      if (claimed && ticket >= 0 && ticket < U * M) {
        // All units' largest balancing chunks first.
        const int c = (ticket % U) * (M + 1) + 1 + ticket / U;
        int k0, k1;
        chunk_bounds(sc, c, k0, k1);
        t.info = make_int4(c, k0, k1, 0);
        walking = walk_begin(wn, prefix, ctxs, B, k0, k1);
      }
      claimed = false;
    };
    Ahead t0, t1;
    resolve(t0);
    resolve(t1);
    int stage = 0, issued = 0;
    uint32_t phase = 0;
    uint64_t idle_since = 0;
    while (__any_sync(0xffffffffu, t0.valid)) {
      bool progressed = false;
      if (t0.valid && !withheld) {
        const int slot = lane * p.stages + stage;
        if (mbar_test_wait(&empty_bar[slot], phase ^ 1u)) {
          const int ph = t0.phys;
          // A block id outside the pool: nothing is copied, the slot is
          // marked (info.w) and its consumer leaves the tile's tokens out.
          const int bad = (ph < 0 || ph >= p.num_blocks) ? 1 : 0;
          if (bad) flag_error(PKV_DEVERR_BLOCK_ID);
          asm volatile("st.shared.v4.s32 [%0], {%1,%2,%3,%4};" ::"r"(smem_u32(&slot_info[slot])), "r"(t0.info.x),
                       "r"(t0.info.y), "r"(t0.info.z), "r"(bad)
                       : "memory");  // published to the consumer by the arrive below
          uint8_t* sk = ring + static_cast<size_t>(slot) * kRingStride;
          if (bad) {
            mbar_arrive(&full_bar[slot]);  // completes the phase with no bytes in flight
          } else if constexpr (kI8) {
            mbar_arrive_expect_tx(&full_bar[slot], kStageBytes);
            // The whole record in one contiguous request.
            const size_t bh = static_cast<size_t>(ph) * p.n_kv_heads + t0.kvh;
            bulk_load_hint(sk, p.kv_i8 + bh * kRingStride, kRingStride, &full_bar[slot], kv_policy);
          } else {
            // One request for the whole K tile and one for V: the number
            // of requests per tile, not their bytes, sets the pace of the
            // copy engine.
            mbar_arrive_expect_tx(&full_bar[slot], kStageBytes);
            tma_load_5d_hint(sk, &tm_k, &full_bar[slot], t0.kvh, ph, kv_policy);
            tma_load_5d_hint(sk + kTileBytes, &tm_v, &full_bar[slot], t0.kvh, ph, kv_policy);
          }
          ++issued;
          if (++stage == p.stages) {
            stage = 0;
            phase ^= 1u;
          }
          t0 = t1;
          resolve(t1);
          progressed = true;
        }
      }
      // Bounded: give up (warp-uniformly) after the wait limit without progress.
      if (__any_sync(0xffffffffu, progressed)) {
        idle_since = 0;
      } else {
        const uint64_t now = global_timer_ns();
        if (idle_since == 0) idle_since = now;
        const bool give_up = __shfl_sync(0xffffffffu, (*abort_flag != 0) || (now - idle_since > p.wait_limit_ns), 0);
        if (give_up) {
          if (lane == 0 && *abort_flag == 0) {
            *abort_flag = 1;
            flag_error(kDevErrTimeout);
          }
          break;
        }
      }
    }
    // Do not leave while copies issued by this lane may still be landing.
    if (lane < kConsumerWarps) {
      for (int s = 0; s < p.stages && s < issued; ++s) {
        const int cnt = (issued - s + p.stages - 1) / p.stages;
        const uint32_t par = static_cast<uint32_t>((cnt - 1) & 1);
        const uint64_t t0s = global_timer_ns();
        while (!mbar_try_wait(&full_bar[lane * p.stages + s], par)) {
          if (global_timer_ns() - t0s > p.wait_limit_ns) {
            flag_error(kDevErrTimeout);
            break;
          }
        }
      }
    }
  } else {
    // ---------------- consumers ----------------
    const int u = blockIdx.x * kConsumerWarps + warp;
    if (u < U) {
      uint8_t* qbuf = qbufs + warp * kQBufBytes;
      int chunk = u * (M + 1);
      int k0, k1;
      chunk_bounds(sc, chunk, k0, k1);
      Walk wk;
      bool have = walk_begin(wk, prefix, ctxs, B, k0, k1);
      Consumer cs;
      int first_seg = -1, cur_seg = -1, cur_b = 0, cur_hg = 0, seg_start = 0, seg_end = 0;
      int4 my_meta = make_int4(-1, 0, 0, 0);  // split segment whose first piece this chunk holds
      int stage = 0;
      uint32_t phase = 0;
      bool aborted = false;
      bool q_ready = false;  // qbuf holds the next segment's Q (copy in flight)

      auto finish_segment = [&]() {
        const bool starts_here = seg_start >= k0, ends_here = seg_end <= k1;
        if (starts_here && ends_here) {
          cs.finish(p, cur_b, cur_hg, nullptr, lane);
        } else {
          const int slot_idx = (cur_seg == first_seg) ? 0 : 1;
          float* rec = p.records + (static_cast<size_t>(chunk) * 2 + slot_idx) * p.rec_floats;
          cs.finish(p, cur_b, cur_hg, rec, lane);
          if (starts_here) my_meta = make_int4(cur_seg, chunk_of_tile(sc, seg_end - 1), slot_idx, 0);
        }
      };

      while (have) {
        const int seg = wk.b * p.ng + wk.hg;
        if (seg != cur_seg) {
          if (cur_seg >= 0) finish_segment();
          cur_seg = seg;
          if (first_seg < 0) first_seg = seg;
          cur_b = wk.b;
          cur_hg = wk.hg;
          seg_start = prefix[wk.b] + wk.hg * wk.nb;
          seg_end = seg_start + wk.nb;
          if (!q_ready) q_fetch<ES, D>(qbuf, p, wk.b, wk.hg, lane);
          cp_async_wait_all();
          __syncwarp();
          cs.begin(qbuf, p.rows, lane);
          if constexpr (kMQ) cs.set_mq(p.gp, p.q_len);
          if (p.init != nullptr && wk.j == 0 && has_init(p, wk.b)) cs.load_init(p, wk.b, wk.hg, lane);
          __syncwarp();
          q_ready = false;
        }
        const bool last = wk.k + 1 >= wk.k_end;
        // The last tile of a segment, with more tiles to come in this chunk:
        // start copying the next segment's Q now, so that it is in place when
        // it is needed.
        if (wk.j == wk.nb - 1 && !last) {
          Walk nx = wk;
          walk_next(nx, prefix, ctxs, B, p.ng);
          q_fetch<ES, D>(qbuf, p, nx.b, nx.hg, lane);
          q_ready = true;
        }
        const int slot = warp * p.stages + stage;
        if (!mbar_wait_bounded(&full_bar[slot], phase, abort_flag, p.wait_limit_ns)) {
          aborted = true;
          break;
        }
        // From the producer: the next chunk (on a chunk's last tile) and
        // whether the tile's block id was out of range (info.w).
        int4 info;
        asm volatile("ld.shared.v4.s32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(info.x), "=r"(info.y), "=r"(info.z), "=r"(info.w)
                     : "r"(smem_u32(&slot_info[slot])));
        int next_chunk = -1, n0 = 0, n1 = 0;
        if (last) {
          // The chunk this warp runs next, as claimed by its producer lane:
          // start copying the Q of its first segment.
          next_chunk = info.x;
          n0 = info.y;
          n1 = info.z;
          Walk nw;
          if (next_chunk >= 0 && walk_begin(nw, prefix, ctxs, B, n0, n1)) {
            q_fetch<ES, D>(qbuf, p, nw.b, nw.hg, lane);
            q_ready = true;
          } else {
            next_chunk = -1;
          }
        }
        // Context tokens from this tile's start on (the tile holds at most 16).
        const int rem = wk.ctx - wk.j * kBlockTokens;
        const int nv = kMQ ? rem : min(kBlockTokens, rem);
        const uint32_t kaddr = smem_u32(ring + static_cast<size_t>(slot) * kRingStride);
        const uint32_t vaddr = kI8 ? kaddr + D * kBlockTokens : kaddr + kTileBytes;
        if (info.w == 0) cs.tile(kaddr, vaddr, nv, p.scale_log2, lane);  // a bad block's tokens are left out
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[slot]);
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1u;
        }
        if (!last) {
          walk_next(wk, prefix, ctxs, B, p.ng);
          continue;
        }
        // End of a chunk: close its open segment and publish its metadata.
        finish_segment();
        if (lane == 0) p.meta[chunk] = my_meta;
        have = next_chunk >= 0;
        if (have) {
          chunk = next_chunk;
          k0 = n0;
          k1 = n1;
          walk_begin(wk, prefix, ctxs, B, k0, k1);
          first_seg = cur_seg = -1;
          my_meta = make_int4(-1, 0, 0, 0);
        }
      }
      cp_async_wait_all();
      if (aborted && lane == 0) p.meta[chunk] = make_int4(-1, 0, 0, 0);
    }
  }

  // ---------------- phase 2: merge split segments ----------------
  cooperative_groups::this_grid().sync();
  {
    constexpr int kWarps = kConsumerWarps + 1;
    const int gw = blockIdx.x * kWarps + warp, n_warps = gridDim.x * kWarps;
    const int n_segs = B * p.ng;
    constexpr int kSlices = D / 32;
    if (M == 0) {
      // Static schedule.  A split segment is merged from its pieces, one
      // record per unit it spans; its first piece lies in the unit where it
      // starts, and a unit starts at most one segment that continues past its
      // end (its last one).  The items are (segment, row[, dim slice]) or
      // (unit, row[, dim slice]), whichever set is smaller -- every segment,
      // and every unit, yields at most one merge per row -- taken by every
      // warp of the grid in turn, so that the merges spread evenly.  When
      // segments span many units (long contexts: few merges, many pieces),
      // D / 32 warps share a row, one dim per lane, so that more warps take
      // part.  (The schedule is recomputed from shared memory rather than
      // held in registers through phase 1.)
      const int T2 = prefix[B];
      const Sched s2 = make_sched(T2, p.num_units, 0, p.static_permille);
      const int n_units = T2 > 0 ? s2.U : 0;
      const bool by_segment = n_segs <= n_units;
      const bool sliced = T2 / max(1, n_segs) >= 8 * max(1, s2.Lq);
      const int per_item = sliced ? p.rows * kSlices : p.rows;
      const int items = (by_segment ? n_segs : n_units) * per_item;
      // Item i's segment (b, hg), row and source pieces; false when it needs
      // no merge (written in phase 1, or taken from another item).
      auto item = [&](int i, int& b, int& hg, int& rem, MergeSrc& src) {
        const int x = i / per_item;
        rem = i - x * per_item;
        int st, en, u1;
        if (by_segment) {
          b = x / p.ng;
          hg = x - b * p.ng;
          if (ctxs[b] == 0) return false;
          segment_tiles(prefix, ctxs, b, hg, st, en);
          u1 = unit_of_tile(s2, st);
          if (en <= unit_begin(s2, u1 + 1)) return false;  // the whole segment in one unit: written in phase 1
        } else {
          u1 = x;
          const int a = unit_begin(s2, u1), e = unit_begin(s2, u1 + 1);
          Walk wl;
          walk_begin(wl, prefix, ctxs, B, e - 1, e);  // the segment of the unit's last tile
          b = wl.b;
          hg = wl.hg;
          segment_tiles(prefix, ctxs, b, hg, st, en);
          if (st < a || en <= e) return false;  // started in an earlier unit, or ends in this one
        }
        src = {u1, st == unit_begin(s2, u1) ? 0 : 1, unit_of_tile(s2, en - 1) - u1 + 1, u1, 1};
        return true;
      };
      if (sliced) {
        for (int i = gw; i < items; i += n_warps) {
          int b, hg, rem;
          MergeSrc src;
          if (item(i, b, hg, rem, src))
            merge_rows<DT, D, 1>(p, src, b, hg, rem / kSlices, (rem % kSlices) * 32, lane, nullptr);
        }
      } else {
        // Each half-warp takes items of its own (16 lanes, D / 16 dims per
        // lane): a merge is a round trip or two of loads, so that two in
        // flight per warp halve the rounds of phase 2.
        const int half = lane >> 4;
        for (int i = 2 * gw + half; i < items; i += 2 * n_warps) {
          int b, hg, rem;
          MergeSrc src;
          if (item(i, b, hg, rem, src)) merge_rows<DT, D, D / 16>(p, src, b, hg, rem, 0, lane & 15, nullptr);
        }
      }
    } else {
      // Balancing chunks: the chunk that holds a split segment's first piece
      // publishes it in meta; every warp takes (chunk, row) items and merges
      // the pieces of consecutive chunks.  Item metadata is loaded 32 items
      // at a time, lane t for the round's t-th item of this warp.
      const int items = n_chunks * p.rows;
      for (int base = gw; base < items; base += 32 * n_warps) {
        int4 my_item = make_int4(-1, 0, 0, 0);
        const int i_lane = base + lane * n_warps;
        if (i_lane < items) my_item = __ldcg(p.meta + i_lane / p.rows);
        for (int t = 0; t < 32 && base + t * n_warps < items; ++t) {
          const int i = base + t * n_warps;
          const int c = i / p.rows;
          int4 mt;
          mt.x = __shfl_sync(0xffffffffu, my_item.x, t);
          mt.y = __shfl_sync(0xffffffffu, my_item.y, t);
          mt.z = __shfl_sync(0xffffffffu, my_item.z, t);
          // Entries of chunks that an aborted launch never reached may be
          // stale: only well-formed ones are merged.
          if (mt.x >= 0 && mt.x < n_segs && mt.y > c && mt.y < n_chunks && (mt.z == 0 || mt.z == 1)) {
            const MergeSrc src = {c, mt.z, mt.y - c + 1, c, 1};
            merge_rows<DT, D, D / 32>(p, src, mt.x / p.ng, mt.x % p.ng, i - c * p.rows, 0, lane, nullptr);
          }
        }
      }
    }
    // The claim counter must have seen every balancing chunk plus one failed
    // claim per unit; anything else means it was not zero at launch (the
    // workspace was not cleared before its first use).  Leave it at zero.
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      const int expect = M > 0 ? U * M + U : 0;
      const int seen = *reinterpret_cast<volatile int*>(p.sched);
      if (seen != expect && (*reinterpret_cast<volatile uint32_t*>(&g_device_error) & kDevErrTimeout) == 0)
        flag_error(PKV_DEVERR_SCHEDULE);
      if (seen != 0) *reinterpret_cast<volatile int*>(p.sched) = 0;
    }
    // Sequences with no tokens get a zero output row, or, when an initial
    // state is given for them, that state normalised.
    const int total = B * p.ng;
    const size_t nqb = static_cast<size_t>(B) * p.n_q_heads;
    for (int sgi = gw; sgi < total; sgi += n_warps) {
      const int b = sgi / p.ng, hg = sgi % p.ng;
      if (ctxs[b] != 0) continue;
      const bool with_init = p.init != nullptr && has_init(p, b);
      for (int e = lane; e < p.rows * (D / 4); e += 32) {
        const int g = e / (D / 4), d4 = (e % (D / 4)) * 4;
        const size_t rowi = out_row(p, b, hg, g);  // the initial state is given for q_len 1 only
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        float inv = 0.f;
        if (with_init) {
          x = __ldg(reinterpret_cast<const float4*>(p.init + rowi * D + d4));
          const float li = __ldg(p.init + nqb * D + nqb + rowi);
          inv = li > 0.f ? 1.f / li : 0.f;
        }
        store4<DT>(static_cast<OutT*>(p.out) + rowi * D + d4, x.x * inv, x.y * inv, x.z * inv, x.w * inv);
      }
    }
  }
}

}  // namespace pkv
