// pkv_prefix.cuh -- attention over shared prefix blocks for cascade decode.
//
// Sequences that share prefix blocks (refcounted sharing of the block table:
// "Transformer anatomy" ch. 15 §15.6, prefix caching; "LLM Primer VI" ch. 8
// §8.1/§8.3, block sharing and prefix caching) read the same keys and values
// for their first prefix_len tokens.  Instead of every sequence streaming them
// again, this kernel treats the prefix as one dense attention problem per
// (group, kv head): the query rows are every (member sequence, query head of
// that kv head) pair, the keys are the group's prefix tokens, read once per
// CTA through the group's prefix block table.  Each row's unnormalised partial
// softmax state (O, m, l) -- with m in log2 units of the scaled scores -- is
// the initial state from which the decode kernel continues over the
// sequence's private suffix blocks, so that the result equals attention over
// the whole context.
//
// CTA: four consumer warps of 16 query rows each (a 64-row tile) and one
// producer warp.  Each stage brings 64 prefix tokens (four 16-token blocks) of
// K and V into shared memory with TMA tensor loads (the decode kernel's tensor
// maps and swizzled tile layout); the warps compute S = Q K^T and O += P V
// with mma.sync m16n8k16 (fp32 accumulation) and keep an fp32 online softmax
// per row.
#pragma once

#include "pkv_kernels.cuh"

namespace pkv {

constexpr int kPrefixWarps = 4;
constexpr int kPrefixThreads = (kPrefixWarps + 1) * 32;
constexpr int kPrefixRows = 16 * kPrefixWarps;  // query rows per CTA
constexpr int kPrefixBlocks = 4;                // 16-token blocks per stage

struct PrefixParams {
  const void* q;                 // [batch][n_q][D]
  const int32_t* prefix_tables;  // [n_groups][max_prefix_blocks]
  const int32_t* prefix_lens;    // [n_groups], multiples of 16
  const int32_t* seq_group;      // [batch], -1 = no shared prefix
  float* init;                   // O [batch][n_q][D], then m [batch][n_q], then l [batch][n_q]
  int32_t batch;
  int32_t n_groups;
  int32_t max_prefix_blocks;
  int32_t num_blocks;
  int32_t n_q_heads;
  int32_t group;   // query heads per kv head
  int32_t stages;  // ring slots
  float scale_log2;
};

template <int DT, int D>
__global__ void __launch_bounds__(kPrefixThreads, 1)
    pkv_prefix_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const PrefixParams p) {
  constexpr bool kBf16 = (DT == kBF16);
  constexpr int ES = 2;
  constexpr int X = 128 / ES;
  constexpr int Y = D / X;
  constexpr int kTileBytes = Y * kBoxBytes;              // one block's K (or V) tile
  constexpr int kHalf = kPrefixBlocks * kTileBytes;      // K (or V) of one stage
  constexpr int kStageBytes = 2 * kHalf;
  constexpr int KS = D / 16;
  constexpr int NT = D / 8;
  using T = typename DTypeInfo<DT>::T;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* ring = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(ring + static_cast<size_t>(p.stages) * kStageBytes);
  uint64_t* empty_bar = full_bar + p.stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty_bar + p.stages);
  int* members = const_cast<int*>(reinterpret_cast<volatile int*>(abort_flag + 4));  // [batch]
  __shared__ int warp_counts[kPrefixWarps + 1];
  __shared__ int n_members;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, kvh = blockIdx.y, grp = blockIdx.z;
  const int G = p.group;

  // Members of this group, in increasing sequence order (block-wide compaction).
  {
    const int per = (p.batch + kPrefixThreads - 1) / kPrefixThreads;
    const int lo = min(p.batch, static_cast<int>(threadIdx.x) * per), hi = min(p.batch, lo + per);
    int cnt = 0;
    for (int b = lo; b < hi; ++b) cnt += (__ldg(p.seq_group + b) == grp);
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) warp_counts[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_counts[w];
    int pos = base + incl - cnt;
    for (int b = lo; b < hi; ++b)
      if (__ldg(p.seq_group + b) == grp) members[pos++] = b;
    if (threadIdx.x == kPrefixThreads - 1) n_members = base + incl;
  }
  __syncthreads();
  const int R = n_members * G;
  const int row0 = tile * kPrefixRows;
  if (row0 >= R) return;  // uniform over the CTA: no barrier has been used yet

  int plen = __ldg(p.prefix_lens + grp);
  if (plen < 0 || plen > p.max_prefix_blocks * kBlockTokens || (plen % kBlockTokens) != 0) {
    flag_error(PKV_DEVERR_CONTEXT);
    plen = plen < 0 ? 0 : min(plen - plen % kBlockTokens, p.max_prefix_blocks * kBlockTokens);
  }
  const int n_stages = (plen + kPrefixBlocks * kBlockTokens - 1) / (kPrefixBlocks * kBlockTokens);

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kPrefixWarps);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == kPrefixWarps) {
    // ---------------- producer (lane 0) ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int32_t* tab = p.prefix_tables + static_cast<size_t>(grp) * p.max_prefix_blocks;
      int slot = 0, issued = 0;
      uint32_t phase = 0;
      for (int s = 0; s < n_stages; ++s) {
        if (!mbar_wait_bounded(&empty_bar[slot], phase ^ 1u, abort_flag, kWaitLimitNs)) break;
        mbar_arrive_expect_tx(&full_bar[slot], kStageBytes);
        uint8_t* st = ring + static_cast<size_t>(slot) * kStageBytes;
        for (int i = 0; i < kPrefixBlocks; ++i) {
          const int j = s * kPrefixBlocks + i;
          int phys = 0;
          if (j * kBlockTokens < plen) {
            phys = __ldg(tab + j);
            if (phys < 0 || phys >= p.num_blocks) {  // copied from block 0; the consumers mask its keys
              flag_error(PKV_DEVERR_BLOCK_ID);
              phys = 0;
            }
          }
#pragma unroll
          for (int y = 0; y < Y; ++y) {
            tma_load_4d(st + i * kTileBytes + y * kBoxBytes, &tm_k, &full_bar[slot], y * X, 0, kvh, phys);
            tma_load_4d(st + kHalf + i * kTileBytes + y * kBoxBytes, &tm_v, &full_bar[slot], y * X, 0, kvh, phys);
          }
        }
        ++issued;
        if (++slot == p.stages) {
          slot = 0;
          phase ^= 1u;
        }
      }
      // Do not leave while copies may still be landing.
      for (int s = 0; s < p.stages && s < issued; ++s) {
        const int cnt = (issued - s + p.stages - 1) / p.stages;
        const uint32_t par = static_cast<uint32_t>((cnt - 1) & 1);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&full_bar[s], par)) {
          if (global_timer_ns() - t0 > kWaitLimitNs) {
            flag_error(kDevErrTimeout);
            break;
          }
        }
      }
    }
    return;
  }

  // ---------------- consumers: 16 query rows per warp ----------------
  const int g = lane >> 2, t = lane & 3, mi = lane >> 3, rr = lane & 7;
  int row_b[2], row_h[2];
  bool row_ok[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = row0 + warp * 16 + g + 8 * r;
    row_ok[r] = row < R;
    const int m_i = row_ok[r] ? row / G : 0;
    row_b[r] = row_ok[r] ? members[m_i] : 0;
    row_h[r] = kvh * G + (row_ok[r] ? row % G : 0);
  }
  uint32_t qa[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const T* qr = static_cast<const T*>(p.q) + (static_cast<size_t>(row_b[r]) * p.n_q_heads + row_h[r]) * D;
      const int c = ks * 16 + 2 * t;
      qa[ks][r] = row_ok[r] ? __ldg(reinterpret_cast<const uint32_t*>(qr + c)) : 0u;
      qa[ks][2 + r] = row_ok[r] ? __ldg(reinterpret_cast<const uint32_t*>(qr + c + 8)) : 0u;
    }
  }
  float o[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

  // Block ids of the stage's blocks, read one stage ahead by lanes 0..3: a
  // block whose id is outside the pool contributes no key (bit i of `bad`).
  const int32_t* ctab = p.prefix_tables + static_cast<size_t>(grp) * p.max_prefix_blocks;
  const int n_prefix_blocks = plen / kBlockTokens;
  auto stage_id = [&](int s) {
    const int j = s * kPrefixBlocks + lane;
    return (lane < kPrefixBlocks && j < n_prefix_blocks) ? __ldg(ctab + j) : 0;
  };
  int id_next = n_stages > 0 ? stage_id(0) : 0;
  int slot = 0;
  uint32_t phase = 0;
  for (int s = 0; s < n_stages; ++s) {
    const int id = id_next;
    if (s + 1 < n_stages) id_next = stage_id(s + 1);
    const uint32_t bad = __ballot_sync(0xffffffffu, id < 0 || id >= p.num_blocks) & ((1u << kPrefixBlocks) - 1u);
    if (!mbar_wait_bounded(&full_bar[slot], phase, abort_flag, kWaitLimitNs)) break;
    const uint32_t kb = smem_u32(ring + static_cast<size_t>(slot) * kStageBytes);
    const uint32_t vb = kb + kHalf;
    const int nv = min(kPrefixBlocks * kBlockTokens, plen - s * kPrefixBlocks * kBlockTokens);

    // S = Q K^T over the stage's 64 tokens: 8 n-tiles of 8 tokens.
    float sc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const uint32_t tb = kb + (nt >> 1) * kTileBytes;
      const int tok = (nt & 1) * 8 + rr;
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk) {
        const int dim = (2 * kk + (mi >> 1)) * 16 + (mi & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(tb + tile_offset<ES>(tok, dim), b0, b1, b2, b3);
        mma_16816<kBf16>(sc[nt], qa[2 * kk][0], qa[2 * kk][1], qa[2 * kk][2], qa[2 * kk][3], b0, b1);
        mma_16816<kBf16>(sc[nt], qa[2 * kk + 1][0], qa[2 * kk + 1][1], qa[2 * kk + 1][2], qa[2 * kk + 1][3], b2,
                         b3);
      }
    }
    // Online softmax; rows g (sc[.][0..1]) and g + 8 (sc[.][2..3]); the
    // probabilities replace the scores in place.
    float alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int tok = nt * 8 + 2 * t + e;
          const float x = (tok < nv && !((bad >> (nt >> 1)) & 1u)) ? sc[nt][2 * r + e] * p.scale_log2 : -INFINITY;
          sc[nt][2 * r + e] = x;
          mx = fmaxf(mx, x);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mn = fmaxf(m_run[r], mx);
      // -inf only while every key so far was masked (bad block ids): then
      // every weight is 0 and the state stays empty.
      const float mb = mn == -INFINITY ? 0.f : mn;
      alpha[r] = exp2f(m_run[r] - mb);
      float sum = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          sc[nt][2 * r + e] = exp2f(sc[nt][2 * r + e] - mb);
          sum += sc[nt][2 * r + e];
        }
      l_run[r] = l_run[r] * alpha[r] + sum;
      m_run[r] = mn;
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      o[n][0] *= alpha[0];
      o[n][1] *= alpha[0];
      o[n][2] *= alpha[1];
      o[n][3] *= alpha[1];
    }
    // O += P V, one 16-token block (k-step) at a time.
#pragma unroll
    for (int blk = 0; blk < kPrefixBlocks; ++blk) {
      const uint32_t pa0 = pack2<kBf16>(sc[2 * blk][0], sc[2 * blk][1]);
      const uint32_t pa1 = pack2<kBf16>(sc[2 * blk][2], sc[2 * blk][3]);
      const uint32_t pa2 = pack2<kBf16>(sc[2 * blk + 1][0], sc[2 * blk + 1][1]);
      const uint32_t pa3 = pack2<kBf16>(sc[2 * blk + 1][2], sc[2 * blk + 1][3]);
      const uint32_t tv = vb + blk * kTileBytes;
      // Whole blocks only (plen % 16 == 0); a bad block holds no token either.
      const bool live = blk * kBlockTokens < nv && !((bad >> blk) & 1u);
#pragma unroll
      for (int nd2 = 0; nd2 < D / 16; ++nd2) {
        const int tok = (mi & 1) * 8 + rr;
        const int dim = (2 * nd2 + (mi >> 1)) * 8;
        uint32_t v0, v1, v2, v3;
        ldsm_x4_trans(tv + tile_offset<ES>(tok, dim), v0, v1, v2, v3);
        if (!live) v0 = v1 = v2 = v3 = 0u;  // blocks past the prefix hold no token
        mma_16816<kBf16>(o[2 * nd2], pa0, pa1, pa2, pa3, v0, v1);
        mma_16816<kBf16>(o[2 * nd2 + 1], pa0, pa1, pa2, pa3, v2, v3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[slot]);
    if (++slot == p.stages) {
      slot = 0;
      phase ^= 1u;
    }
  }

  // Per-row partial state: O unnormalised, m, l (l summed over the four lanes of a row).
  const size_t nqb = static_cast<size_t>(p.batch) * p.n_q_heads;
  float* init_m = p.init + nqb * D;
  float* init_l = init_m + nqb;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float lt = l_run[r];
    lt += __shfl_xor_sync(0xffffffffu, lt, 1);
    lt += __shfl_xor_sync(0xffffffffu, lt, 2);
    if (!row_ok[r]) continue;
    const size_t rowi = static_cast<size_t>(row_b[r]) * p.n_q_heads + row_h[r];
    float* ob = p.init + rowi * D;
#pragma unroll
    for (int n = 0; n < NT; ++n)
      *reinterpret_cast<float2*>(ob + n * 8 + 2 * t) = make_float2(o[n][2 * r], o[n][2 * r + 1]);
    if (t == 0) {
      init_m[rowi] = m_run[r];
      init_l[rowi] = lt;
    }
  }
}

}  // namespace pkv
