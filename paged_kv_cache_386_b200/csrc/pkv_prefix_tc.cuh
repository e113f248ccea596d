// pkv_prefix_tc.cuh -- the shared-prefix attention of cascade decode on the
// fifth-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// Same problem and output as pkv_prefix_kernel (pkv_prefix.cuh): for every
// (group, kv head), the query rows are the (member sequence, query head of
// that kv head) pairs and the keys are the group's shared prefix tokens
// ("Transformer anatomy" ch. 15 §15.6, prefix sharing; "LLM Primer VI" ch. 8
// §8.1/§8.3).  Each row's unnormalised (O, m, l), m in log2 units of the
// scaled scores, is the state from which the decode kernel continues over the
// sequence's private suffix.
//
// A cluster of 1-4 CTAs per 128-row tile of one (group, kv head), head dim
// 128; CTA k of the cluster takes the k-th share of the prefix stages, so that
// a few tiles still fill the SMs.  After its last stage each CTA of rank > 0
// leaves its partial (O, m, l) in its own shared memory; rank 0 reads them
// through distributed shared memory, merges them with its own (each term
// scaled by 2^(m_k - max m)) and writes the row's state.  192 threads:
//   warps 0-3  softmax: thread r owns row r (tensor-memory lane r);
//   warp 4     producer: TMA loads of 64 prefix tokens (4 blocks) of K and V
//              per stage into a 4-stage ring;
//   warp 5     allocates the tensor memory; its lane 0 issues every MMA.
// Per stage s:  S_s = Q K_s^T (M 128, N 64 keys, K 128) into one of two S
// buffers in tensor memory; the softmax warps read their S row, turn it into
// probabilities P_s (16-bit, shared memory) and the MMA thread accumulates
// O += P_s V_s (M 128, N 128 dims, K 64 keys) in tensor memory.  S of the
// next stage is issued before O += P V of this one, so that the softmax of a
// stage overlaps the tensor cores; P is double-buffered, so that the softmax
// of stage s + 1 does not wait for O += P V of stage s.  The running maximum
// is only moved (and O,
// l rescaled) when a row's maximum grows by more than 2^8, so that O rarely
// makes a round trip through registers; P stays below 2^8.
//
// Shared-memory operands use the 128-byte swizzle (16-byte chunk c of a
// 128-byte row r at chunk c ^ (r % 8)), in 1 KiB atoms of 8 rows:
//   Q     K-major A operand:  [64-dim block][128 rows][128 B];
//   P     K-major A operand:  [128 rows][128 B] (64 keys);
//   K     K-major B operand:  [64-dim block][64 tokens][128 B];
//   V     MN-major B operand: [64-dim block][64 tokens][128 B].
// The K and V blocks land there from the decode kernel's tensor maps (one
// 16-row x 128-byte box per block and 64-dim block).
#pragma once

#include "pkv_prefix.cuh"

namespace pkv {

constexpr int kTcRows = 128;                  // query rows per CTA (M)
constexpr int kTcKeys = 64;                   // prefix tokens per stage (N of S, K of P V)
constexpr int kTcBlocks = kTcKeys / kBlockTokens;
constexpr int kTcThreads = 192;
constexpr int kTcQBytes = kTcRows * 128 * 2;        // Q: 128 rows x 128 dims, 32 KiB
constexpr int kTcQHalf = kTcQBytes / 2;             // one 64-dim block of Q: 16 KiB
constexpr int kTcPBytes = kTcRows * kTcKeys * 2;    // P: 128 rows x 64 keys, 16 KiB
constexpr int kTcKVBytes = kTcKeys * 128 * 2;       // K (or V) of one stage: 64 tokens x 128 dims, 16 KiB
constexpr int kTcKVHalf = kTcKVBytes / 2;           // one 64-dim block: 8 KiB
constexpr int kTcStageBytes = 2 * kTcKVBytes;       // K and V of one stage
constexpr int kTcStages = 4;
constexpr int kTcSmemBytes = kTcQBytes + 2 * kTcPBytes + kTcStages * kTcStageBytes;  // 192 KiB
constexpr uint32_t kTcTmemCols = 256;  // S0 [0,64), S1 [64,128), O [128,256)
constexpr uint32_t kTcOCol = 2 * kTcKeys;
constexpr int kTcMaxSplit = 4;          // CTAs per cluster (prefix shares per tile)
constexpr int kTcPartStride = 128 + 4;  // floats per row of a partial O in shared memory (float4 accesses
                                        // of 8 consecutive rows fall in distinct bank groups)
static_assert(kTcRows * kTcPartStride * 4 + 2 * kTcRows * 4 <= kTcStages * kTcStageBytes,
              "a partial state fits in the drained K/V ring");

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// Every thread of every CTA of the cluster; writes before it are visible to
// distributed-shared-memory reads after it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// The address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_cluster(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_cluster4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// Shared-memory matrix descriptor (tcgen05): start address, leading and
// stride byte offsets (16-byte units), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulate, A and B both f16 or
// both bf16, A K-major, B K-major or MN-major, M = 128, N = n.
template <bool kBf16>
__host__ __device__ constexpr uint32_t tc_idesc(bool b_mn_major, uint32_t n) {
  return (1u << 4) | ((kBf16 ? 1u : 0u) << 7) | ((kBf16 ? 1u : 0u) << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this warp's 32 tensor-memory lanes (one row
// per thread).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
      "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]),
      "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]),
      "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]),
      "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31]));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Byte offset of the 16-byte chunk c of row r in a swizzled 128-row operand
// ([64-column block][128 rows][128 B]).
__device__ __forceinline__ uint32_t tc_chunk(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * kTcQHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <int DT>
__global__ void __launch_bounds__(kTcThreads, 1)
    pkv_prefix_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const PrefixParams p) {
  constexpr bool kBf16 = (DT == kBF16);
  constexpr int D = 128;
  constexpr int X = 64;  // 16-bit elements per 128-byte row

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* q_s = base;                               // [2][128 rows][128 B]
  uint8_t* p_s = base + kTcQBytes;                   // two P buffers, each [128 rows][128 B]
  uint8_t* ring = p_s + 2 * kTcPBytes;               // [stage]{K, V}, each [2][64 tokens][128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + kTcStages * kTcStageBytes);
  uint64_t* kv_full = bars;                // [kTcStages]
  uint64_t* kv_empty = bars + kTcStages;   // [kTcStages]
  uint64_t* s_full = bars + 2 * kTcStages; // [2]
  uint64_t* s_free = s_full + 2;           // [2]
  uint64_t* p_full = s_full + 4;
  uint64_t* o_done = s_full + 5;           // [2]: P V of stages with that parity (P buffer free, O updated)
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(s_full + 7);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* members = const_cast<int*>(reinterpret_cast<volatile int*>(abort_flag + 2));  // [batch]
  __shared__ int warp_counts[kTcThreads / 32];
  __shared__ int n_members;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_rank(), csize = cluster_size();
  const int tile = blockIdx.x / csize, kvh = blockIdx.y, grp = blockIdx.z;
  const int G = p.group;

  // Members of this group, in increasing sequence order (block-wide compaction).
  {
    const int per = (p.batch + kTcThreads - 1) / kTcThreads;
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
    int wbase = 0;
    for (int w = 0; w < warp; ++w) wbase += warp_counts[w];
    int pos = wbase + incl - cnt;
    for (int b = lo; b < hi; ++b)
      if (__ldg(p.seq_group + b) == grp) members[pos++] = b;
    if (threadIdx.x == kTcThreads - 1) n_members = wbase + incl;
  }
  __syncthreads();
  const int R = n_members * G;
  const int row0 = tile * kTcRows;
  if (row0 >= R) return;  // uniform over the cluster: no barrier or tensor memory is in use yet

  int plen = __ldg(p.prefix_lens + grp);
  if (plen < 0 || plen > p.max_prefix_blocks * kBlockTokens || (plen % kBlockTokens) != 0) {
    flag_error(PKV_DEVERR_CONTEXT);
    plen = plen < 0 ? 0 : min(plen - plen % kBlockTokens, p.max_prefix_blocks * kBlockTokens);
  }
  // This CTA's share of the prefix: stages [s_begin, s_begin + n_stages).
  const int n_total = (plen + kTcKeys - 1) / kTcKeys;
  const int s_begin = n_total * static_cast<int>(crank) / static_cast<int>(csize);
  const int n_stages = n_total * static_cast<int>(crank + 1) / static_cast<int>(csize) - s_begin;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(&o_done[0], 1);
    mbar_init(&o_done[1], 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(const_cast<uint32_t*>(tmem_slot))),
                 "r"(kTcTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // Q rows into the swizzled A operand (zero rows past R).
  if (warp < 4) {
    const int r = threadIdx.x;
    const int row = row0 + r;
    const uint4* src = nullptr;
    if (row < R) {
      const int b = members[row / G], h = kvh * G + row % G;
      src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.q) +
                                           (static_cast<size_t>(b) * p.n_q_heads + h) * D * 2);
    }
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const uint4 v = src ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(q_s + tc_chunk(r, c)) = v;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);  // softmax warps' lanes
  float* part_o = reinterpret_cast<float*>(ring);  // a rank > 0 CTA's partial O: [128 rows][kTcPartStride]
  float* part_ml = part_o + kTcRows * kTcPartStride;  // its m [128], then l [128]
  float m_ref = -INFINITY, l_sum = 0.f;  // the softmax thread's row state
  bool row_ok = true;

  if (warp == 4) {
    // ---------------- producer: 16 TMA requests per stage, one per lane ----------------
    const int32_t* tab = p.prefix_tables + static_cast<size_t>(grp) * p.max_prefix_blocks;
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    const int blk = (lane >> 2) & 3, isv = (lane >> 1) & 1, y = lane & 1;
    const bool active = lane < 4 * kTcBlocks;
    int issued = 0;
    for (int s = 0; s < n_stages; ++s) {
      const int slot = s % kTcStages;
      if (!mbar_wait_bounded(&kv_empty[slot], ((s / kTcStages) & 1) ^ 1u, abort_flag, kWaitLimitNs)) break;
      const int j = (s_begin + s) * kTcBlocks + blk;
      // Blocks past the prefix reload block 0 of the prefix (finite values;
      // their probabilities are 0).
      int phys = __ldg(tab + (j * kBlockTokens < plen ? j : 0));
      if (phys < 0 || phys >= p.num_blocks) {
        flag_error(PKV_DEVERR_BLOCK_ID);
        phys = 0;
      }
      if (lane == 0) mbar_arrive_expect_tx(&kv_full[slot], kTcStageBytes);
      __syncwarp();
      uint8_t* dst = ring + slot * kTcStageBytes + isv * kTcKVBytes + y * kTcKVHalf + blk * (kBlockTokens * 128);
      if (active) tma_load_4d(dst, isv ? &tm_v : &tm_k, &kv_full[slot], y * X, 0, kvh, phys);
      ++issued;
    }
    // Do not leave while copies may still be landing.
    if (lane == 0) {
      for (int s = max(0, issued - kTcStages); s < issued; ++s) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&kv_full[s % kTcStages], (s / kTcStages) & 1)) {
          if (global_timer_ns() - t0 > kWaitLimitNs) {
            flag_error(kDevErrTimeout);
            break;
          }
        }
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issue (one thread) ----------------
    if (lane == 0 && n_stages > 0) {
      constexpr uint32_t kIdS = tc_idesc<kBf16>(false, kTcKeys), kIdPV = tc_idesc<kBf16>(true, D);
      const uint32_t qa = smem_u32(q_s), pa = smem_u32(p_s), ra = smem_u32(ring);
      auto issue_s = [&](int s) {
        const uint32_t ka = ra + (s % kTcStages) * kTcStageBytes;
        const uint32_t d = tmem + (s & 1) * kTcKeys;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          tc_mma(d, smem_desc_sw128(qa + (kk >> 2) * kTcQHalf + (kk & 3) * 32, 16, 1024),
                 smem_desc_sw128(ka + (kk >> 2) * kTcKVHalf + (kk & 3) * 32, 16, 1024), kIdS, kk > 0);
        }
        tc_commit(&s_full[s & 1]);
      };
      bool ok = mbar_wait_bounded(&kv_full[0], 0, abort_flag, kWaitLimitNs);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int s = 0; ok && s < n_stages; ++s) {
        if (s + 1 < n_stages) {
          ok = mbar_wait_bounded(&kv_full[(s + 1) % kTcStages], ((s + 1) / kTcStages) & 1, abort_flag, kWaitLimitNs);
          // The S buffer of stage s + 1 was last read by the softmax of stage s - 1.
          if (ok && s >= 1) ok = mbar_wait_bounded(&s_free[(s + 1) & 1], ((s - 1) >> 1) & 1, abort_flag, kWaitLimitNs);
          if (!ok) break;
          tc_fence_after();
          issue_s(s + 1);
        }
        if (!mbar_wait_bounded(p_full, s & 1, abort_flag, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t va = ra + (s % kTcStages) * kTcStageBytes + kTcKVBytes;
        const uint32_t pb = pa + (s & 1) * kTcPBytes;
#pragma unroll
        for (int kt = 0; kt < kTcKeys / 16; ++kt) {
          tc_mma(tmem + kTcOCol, smem_desc_sw128(pb + kt * 32, 16, 1024),
                 smem_desc_sw128(va + kt * 16 * 128, kTcKVHalf, 1024), kIdPV, s > 0 || kt > 0);
        }
        tc_commit(&o_done[s & 1]);
        tc_commit(&kv_empty[s % kTcStages]);
      }
      // Before the tensor memory is freed, every MMA issued must have completed.
      if (!ok) mbar_wait_bounded(&o_done[(n_stages - 1) & 1], ((n_stages - 1) >> 1) & 1, abort_flag, kWaitLimitNs);
    }
  } else {
    // ---------------- softmax: thread r owns row r ----------------
    const int r = threadIdx.x;
    // Every tensor-memory access below is warp-converged (.sync.aligned):
    // waits and decisions are made warp-uniform first.
    bool ok = true;
    for (int s = 0; s < n_stages; ++s) {
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_full[s & 1], (s >> 1) & 1, abort_flag, kWaitLimitNs));
      if (!ok) break;
      tc_fence_after();
      float x[kTcKeys];
#pragma unroll
      for (int c = 0; c < kTcKeys / 32; ++c) {
        float v[32];
        tmem_ld32(lane_base + (s & 1) * kTcKeys + c * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[c * 32 + i] = v[i];
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[s & 1]);

      const int live = min(kTcKeys, plen - (s_begin + s) * kTcKeys);
      float mx8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) mx8[j] = -INFINITY;
#pragma unroll
      for (int i = 0; i < kTcKeys; ++i) {
        x[i] = i < live ? x[i] * p.scale_log2 : -INFINITY;
        mx8[i & 7] = fmaxf(mx8[i & 7], x[i]);  // eight independent chains
      }
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      // P buffer s % 2 is free once P V of stage s - 2 is done.
      if (s >= 2) {
        ok = __all_sync(0xffffffffu,
                        mbar_wait_bounded(&o_done[s & 1], ((s - 2) >> 1) & 1, abort_flag, kWaitLimitNs));
        if (!ok) break;
        tc_fence_after();
      }
      // Move the reference maximum only when it grows by more than 2^8 (so
      // that O rarely makes the round trip); when any row of the warp moves,
      // the whole warp takes the round trip, with factor 1 for the others.
      // O is stable once P V of stage s - 1 is done.
      const bool move = mx > m_ref + 8.f;
      if (s > 0 && __any_sync(0xffffffffu, move)) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&o_done[(s - 1) & 1], ((s - 1) >> 1) & 1, abort_flag,
                                                       kWaitLimitNs));
        if (!ok) break;
        tc_fence_after();
        const float alpha = move ? exp2f(m_ref - mx) : 1.f;
        l_sum *= alpha;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float v[32];
          tmem_ld32(lane_base + kTcOCol + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= alpha;
          tmem_st32(lane_base + kTcOCol + c * 32, v);
        }
        tmem_wait_st();
      }
      if (move) m_ref = mx;
      float sum8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) sum8[j] = 0.f;
#pragma unroll
      for (int c = 0; c < kTcKeys / 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float a = exp2f(x[8 * c + 2 * k] - m_ref), b = exp2f(x[8 * c + 2 * k + 1] - m_ref);
          sum8[2 * k] += a;
          sum8[2 * k + 1] += b;
          w[k] = pack2<kBf16>(a, b);
        }
        *reinterpret_cast<uint4*>(p_s + (s & 1) * kTcPBytes + tc_chunk(r, c)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      l_sum += ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && n_stages > 0)
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&o_done[(n_stages - 1) & 1], ((n_stages - 1) >> 1) & 1,
                                                      abort_flag, kWaitLimitNs));
    tc_fence_after();
    row_ok = ok;
    if (crank > 0) {
      // Partial state into the drained ring (every copy into it has been
      // consumed by an MMA that has completed); l = NaN marks a failed row.
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
        if (ok && n_stages > 0) {
          tmem_ld32(lane_base + kTcOCol + c * 32, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(part_o + r * kTcPartStride + c * 32 + i) =
              make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      }
      part_ml[r] = m_ref;
      part_ml[kTcRows + r] = ok ? l_sum : __int_as_float(0x7fc00000);
    }
  }
  tc_fence_before();
  cluster_sync();  // partial states written
  tc_fence_after();
  if (warp < 4 && crank == 0) {
    // The row's state: O (unnormalised), m, l, merged over the cluster.
    const int r = threadIdx.x;
    const int row = row0 + r;
    float m_all = m_ref;
    float mk[kTcMaxSplit], lk[kTcMaxSplit];
    bool valid = row_ok;
    const uint32_t ml_addr = smem_u32(part_ml);
#pragma unroll
    for (int k = 1; k < kTcMaxSplit; ++k) {
      mk[k] = -INFINITY;
      lk[k] = 0.f;
      if (k < static_cast<int>(csize)) {
        mk[k] = ld_cluster(cluster_map(ml_addr + r * 4, k));
        lk[k] = ld_cluster(cluster_map(ml_addr + (kTcRows + r) * 4, k));
        valid = valid && !isnan(lk[k]);
        m_all = fmaxf(m_all, mk[k]);
      }
    }
    // Weight of each share: 2^(m_k - max m), 0 for a share with no keys.
    const float a0 = m_ref == -INFINITY ? 0.f : exp2f(m_ref - m_all);
    float l_all = a0 * l_sum;
#pragma unroll
    for (int k = 1; k < kTcMaxSplit; ++k) {
      mk[k] = mk[k] == -INFINITY ? 0.f : exp2f(mk[k] - m_all);  // now the weight
      l_all += mk[k] * lk[k];
    }
    const bool mine = row < R && valid;
    size_t rowi = 0;
    if (mine) rowi = static_cast<size_t>(members[row / G]) * p.n_q_heads + kvh * G + row % G;
    float* ob = p.init + rowi * D;
    const uint32_t po_addr = smem_u32(part_o) + r * kTcPartStride * 4;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float v[32];
      if (row_ok && n_stages > 0) {
        tmem_ld32(lane_base + kTcOCol + c * 32, v);  // every lane of the warp
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= a0;
#pragma unroll
      for (int k = 1; k < kTcMaxSplit; ++k) {
        if (k >= static_cast<int>(csize)) break;
        const uint32_t src = cluster_map(po_addr + c * 128, k);
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 t = ld_cluster4(src + i * 4);
          v[i] += mk[k] * t.x;
          v[i + 1] += mk[k] * t.y;
          v[i + 2] += mk[k] * t.z;
          v[i + 3] += mk[k] * t.w;
        }
      }
      if (mine) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(ob + c * 32 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      }
    }
    if (mine) {
      const size_t nqb = static_cast<size_t>(p.batch) * p.n_q_heads;
      p.init[nqb * D + rowi] = m_all;
      p.init[nqb * D + nqb + rowi] = l_all;
    }
  }
  tc_fence_before();
  cluster_sync();  // the other CTAs' shared memory stays in place until rank 0 has read it
  if (warp == 5) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols));
  }
}

}  // namespace pkv
