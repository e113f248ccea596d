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
// a few tiles still fill the SMs.  After its last stage each CTA leaves the
// partial (O, m, l) of the rows it does not own in its own shared memory; the
// owner of a row group (rank lg * size / 4) reads the other shares through
// distributed shared memory, weights each by 2^(m_k - max m), and writes the
// row's state with coalesced stores.  320 threads:
//   warps 0-7  softmax, two sets of four: set t = warp / 4 takes the stages
//              s = t, t + 2, t + 4, ... of this CTA's share, warp lg = warp % 4
//              of a set the rows 32 lg .. 32 lg + 31 (its tensor-memory lanes)
//              and all 64 scores of each of its stages;
//   warp 8     producer: TMA loads of 64 prefix tokens (4 blocks) of K and V
//              per stage into a 5-stage ring, from the kernel's start on;
//   warp 9     allocates the tensor memory and issues every MMA (the warp
//              runs the issue loop converged, one elected lane issues).
// Per stage s:  S_s = Q K_s^T (M 128, N 64 keys, K 128) into S buffer s % 4
// of tensor memory; the softmax warps of set s % 2 read their S row, turn it
// into probabilities P_s (16-bit, written over the first half of the same S
// buffer) and the MMA thread accumulates O_t += P_s V_s (M 128, N 128 dims,
// K 64 keys) into the set's own accumulator O_t.  The two sets keep separate
// running maxima, sums and accumulators, so that the softmax of stage s + 1
// runs while that of stage s is still in flight; they are combined, like the
// shares of a cluster, after the last stage.  The running maximum is only
// moved (and O_t, l rescaled) when a row's maximum grows by more than 2^8, so
// that O_t rarely makes a round trip through registers; P stays below 2^8.
//
// P, the A operand of P V, lives in tensor memory (lane = row).  Q, the A
// operand of S, and the B operands are in shared memory with the 128-byte
// swizzle (16-byte chunk c of a 128-byte row r at chunk c ^ (r % 8)), in 1 KiB
// atoms of 8 rows:
//   Q     K-major A operand:  [64-dim half][128 rows][128 B];
//   K     K-major B operand:  [block][8-token group][64-dim half][8 tokens][128 B],
//         so that the 8-token atoms of one dim half lie 2 KiB apart;
//   V     MN-major B operand: [block][64-dim half][16 tokens][128 B].
// Each lands as one TMA request per block: K through a 5-D map whose
// dimensions are (64 dims, 8 tokens, dim half, token group, block x kv head),
// V through a 5-D map whose box is a block's whole tile.
#pragma once

#include "pkv_prefix.cuh"

namespace pkv {

constexpr int kTcRows = 128;                  // query rows per CTA (M)
constexpr int kTcKeys = 64;                   // prefix tokens per stage (N of S, K of P V)
constexpr int kTcBlocks = kTcKeys / kBlockTokens;
constexpr int kTcSoftmaxWarps = 8;           // two sets of four: even and odd stages
constexpr int kTcSetWarps = 4;
constexpr int kTcProducerWarp = 8;
constexpr int kTcMmaWarp = 9;
constexpr int kTcThreads = 320;
constexpr int kTcKVBytes = kTcKeys * 128 * 2;       // K (or V) of one stage: 64 tokens x 128 dims, 16 KiB
constexpr int kTcBlockBytes = kTcKVBytes / kTcBlocks;  // one block's K (or V): 4 KiB
constexpr int kTcStageBytes = 2 * kTcKVBytes;       // K and V of one stage
constexpr int kTcStages = 5;
constexpr int kTcRingBytes = kTcStages * kTcStageBytes;  // the K/V ring, 160 KiB
constexpr int kTcQBytes = kTcRows * 128 * 2;             // Q: [64-dim half][128 rows][128 B], 32 KiB
constexpr int kTcSmemBytes = kTcRingBytes + kTcQBytes;
constexpr int kTcSBufs = 4;             // S buffers in tensor memory (P of a stage overwrites its S)
// Tensor-memory columns (one fp32 or one pair of 16-bit values each): S
// buffer i at [64 i, 64 i + 64) for i < 4, O_0 [256,384) and O_1 [384,512).
// P_s, the A operand of P V, takes the first 32 columns of S buffer s % 4;
// Q, the A operand of S, is in shared memory.  S of stage s + 4 waits for P V
// of stage s, so that the issuing warp rarely waits for a P V to complete.
constexpr uint32_t kTcTmemCols = 512;
constexpr uint32_t kTcOCol = 256;       // O_t at kTcOCol + 128 t
constexpr int kTcMaxSplit = 4;          // CTAs per cluster (prefix shares per tile)
constexpr int kTcPartStride = 128 + 4;  // floats per row of a partial O in shared memory (float4 accesses
                                        // of 8 consecutive rows fall in distinct bank groups)
static_assert(kTcRows * kTcPartStride * 4 + 2 * kTcRows * 4 <= kTcRingBytes,
              "a partial state fits in the drained K/V ring");
// After the last stage the drained ring holds a CTA's partial state for the
// rows it does not own (from byte 0) and the output rows it owns (from
// kTcOutOffset).
constexpr int kTcOutOffset = 68 * 1024;
static_assert(kTcRows * kTcPartStride * 4 + 2 * kTcRows * 4 <= kTcOutOffset, "partial state before the output rows");
static_assert(kTcOutOffset + kTcRows * 512 <= kTcRingBytes, "output rows fit in the drained ring");
// Barriers (K/V full and empty per ring slot; S full, S buffer free and P
// full per S buffer; one to drain the MMAs on an abort), the tensor-memory
// slot and the abort flag, then the exchange arrays of the set merge (maxima
// [2][128], sums [2][128]).
constexpr int kTcBarBytes = (2 * kTcStages + 3 * kTcSBufs + 1) * 8 + 16;
constexpr int kTcExchBytes = (2 * kTcRows + 2 * kTcRows) * 4;

// Softmax arithmetic with fewer issue slots: two fp32 lanes per packed FMA /
// add (sm_100), two new values per three-input max, and the hardware base-2
// exponential with flush to zero (the probabilities become 16-bit anyway).
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

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
// Ordered after the cluster barrier by that barrier's memory clobber; no
// clobber here, so that a batch of them is in flight at once.
__device__ __forceinline__ float4 ld_cluster4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
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

// D (+)= A B on the tensor cores (kind::f16, fp32 accumulate in tensor
// memory), A (M x 16, 16-bit) in tensor memory (lane = row, each 32-bit
// column a pair of consecutive K elements), B from a shared-memory
// descriptor.
// Executed by a whole converged warp: the operands are the same in every
// lane and one elected lane issues the MMA (so that the warp's control flow
// and operand arithmetic stay uniform).
__device__ __forceinline__ void tc_mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t idesc,
                                          bool accumulate) {
  asm volatile(
      "{\n .reg .pred p, e;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

// The same with A from a shared-memory descriptor as well.
__device__ __forceinline__ void tc_mma_ss(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n .reg .pred p, e;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

// The mbarrier tracks the completion of every MMA the elected lane (the
// same lane as in tc_mma_ts) has issued; executed by the whole warp.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(smem_u32(bar))
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

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

template <int DT>
__global__ void __launch_bounds__(kTcThreads, 1)
    pkv_prefix_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const PrefixParams p) {
  constexpr bool kBf16 = (DT == kBF16);
  constexpr int D = 128;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* ring = base;                     // [stage]{K, V}: K [4 blocks][2][2][8][128 B], V [4 blocks][2][16][128 B]
  uint8_t* out_s = ring + kTcOutOffset;     // after the last stage: the merged output rows, [128 rows][512 B]
  uint8_t* q_s = ring + kTcRingBytes;     // Q, the K-major A operand of S: [half][128 rows][128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(q_s + kTcQBytes);
  uint64_t* kv_full = bars;                // [kTcStages]
  uint64_t* kv_empty = bars + kTcStages;   // [kTcStages]
  uint64_t* s_full = bars + 2 * kTcStages; // [kTcSBufs]: S written
  uint64_t* s_free = s_full + kTcSBufs;    // [kTcSBufs]: P V of the buffer's stage done (buffer free)
  uint64_t* p_full = s_free + kTcSBufs;    // [kTcSBufs]: P written by the four warps of the stage's set
  uint64_t* mma_drain = p_full + kTcSBufs; // every MMA issued done (abort path)
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(mma_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red_max = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + kTcBarBytes);  // [2][128]
  float* red_l = red_max + 2 * kTcRows;                                                     // [2][128]
  int* members = reinterpret_cast<int*>(red_l + 2 * kTcRows);                               // [batch]
  __shared__ int warp_counts[kTcThreads / 32];
  __shared__ int set_ok[2][kTcSetWarps];
  __shared__ int n_members;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_rank(), csize = cluster_size();
  const int tile = blockIdx.x / csize, kvh = blockIdx.y, grp = blockIdx.z;
  const int G = p.group;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < kTcSBufs; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 1);
      mbar_init(&p_full[i], kTcSetWarps);
    }
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  int plen = __ldg(p.prefix_lens + grp);
  const bool plen_bad = plen < 0 || plen > p.max_prefix_blocks * kBlockTokens || (plen % kBlockTokens) != 0;
  if (plen_bad) plen = plen < 0 ? 0 : min(plen - plen % kBlockTokens, p.max_prefix_blocks * kBlockTokens);
  // This CTA's share of the prefix: stages [s_begin, s_begin + n_stages).
  const int n_total = (plen + kTcKeys - 1) / kTcKeys;
  const int s_begin = n_total * static_cast<int>(crank) / static_cast<int>(csize);
  const int n_stages = n_total * static_cast<int>(crank + 1) / static_cast<int>(csize) - s_begin;
  // The producer reads the block table a window of 32 entries (8 stages) at
  // a time, one window ahead, lane l holding entry l of the window; the first
  // two windows are in flight during the member scan.  Entries past the
  // prefix read as entry 0 (finite values whose probabilities are 0).
  const int32_t* tab = p.prefix_tables + static_cast<size_t>(grp) * p.max_prefix_blocks;
  const int n_prefix_blocks = plen / kBlockTokens;
  auto tab_entry = [&](int j) { return __ldg(tab + (j < n_prefix_blocks ? j : 0)); };
  int tab_cur = 0, tab_next = 0;
  if (warp == kTcProducerWarp) {
    tab_cur = tab_entry(s_begin * kTcBlocks + lane);
    tab_next = tab_entry(s_begin * kTcBlocks + 32 + lane);
  }

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
  if (row0 >= R) return;  // uniform over the cluster: no copy, MMA or tensor memory is in use yet

  if (plen_bad && threadIdx.x == 0) flag_error(PKV_DEVERR_CONTEXT);

  // Softmax-warp geometry: row group lg (tensor-memory lanes 32 lg ..) and
  // set hf (stages of parity hf); after the last stage, warp (lg, hf) also
  // takes the dims [64 hf, 64 hf + 64) of its rows.
  const int lg = warp & 3, hf = (warp >> 2) & 1;
  const int r = lg * 32 + lane;
  const uint32_t owner = static_cast<uint32_t>(lg) * csize / 4;  // cluster rank that writes these rows
  float m_ref = -INFINITY, l_row = 0.f;                           // the softmax thread's row state
  float set_w[2] = {0.f, 0.f};                                    // weights of O_0, O_1 in the row's O
  bool ok = true;
  uint32_t tmem = 0;
  // Columns [64 hf + 32 c, + 32) of this row's O, the two sets' accumulators
  // combined (an accumulator of a set with no stage is never read).
  auto load_o = [&](int c, float (&t)[32]) {
#pragma unroll
    for (int i = 0; i < 32; ++i) t[i] = 0.f;
    if (!ok) return;
    const uint32_t col = tmem + (static_cast<uint32_t>(lg * 32) << 16) + kTcOCol + hf * 64 + c * 32;
#pragma unroll
    for (int st = 0; st < 2; ++st) {
      if (n_stages > st) {
        float u[32];
        tmem_ld32(col + st * D, u);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) t[i] = fmaf(set_w[st], u[i], t[i]);
      }
    }
  };

  if (warp == kTcProducerWarp) {
    // ---------------- producer: 8 TMA requests per stage ----------------
    // Lanes 0-3: K of block `lane`, lanes 4-7: V of block lane - 4, each one
    // box of the block's whole 16-token x 128-dim tile.  Starts at once: the
    // copies of the first stages overlap the Q load.
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    const int n_kv = p.n_q_heads / G;
    const bool is_k = lane < kTcBlocks, is_v = !is_k && lane < 2 * kTcBlocks;
    const int blk = is_k ? lane : is_v ? lane - kTcBlocks : 0;
    int issued = 0;
    for (int s = 0; s < n_stages; ++s) {
      const int slot = s % kTcStages;
      if (!__all_sync(0xffffffffu,
                      mbar_wait_bounded(&kv_empty[slot], ((s / kTcStages) & 1) ^ 1u, abort_flag, kWaitLimitNs)))
        break;  // warp-uniform, so that the shuffles below stay converged
      if (s > 0 && (s & 7) == 0) {
        tab_cur = tab_next;
        tab_next = tab_entry((s_begin + s + 8) * kTcBlocks + lane);
      }
      int phys = __shfl_sync(0xffffffffu, tab_cur, (s & 7) * kTcBlocks + blk);
      if (phys < 0 || phys >= p.num_blocks) {  // copied from block 0; the softmax masks its keys
        flag_error(PKV_DEVERR_BLOCK_ID);
        phys = 0;
      }
      if (lane == 0) mbar_arrive_expect_tx(&kv_full[slot], kTcStageBytes);
      __syncwarp();
      uint8_t* stage = ring + slot * kTcStageBytes;
      if (is_k) tma_load_5d(stage + blk * kTcBlockBytes, &tm_k, &kv_full[slot], 0, 0, 0, 0, phys * n_kv + kvh);
      if (is_v) tma_load_5d(stage + kTcKVBytes + blk * kTcBlockBytes, &tm_v, &kv_full[slot], 0, 0, 0, kvh, phys);
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
  } else {
    if (warp == kTcMmaWarp) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(const_cast<uint32_t*>(tmem_slot))),
                   "r"(kTcTmemCols));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    } else {
      // Q rows into shared memory (zero rows past R): softmax warp (lg, hf)
      // writes dims [64 hf, 64 hf + 64) of its 32 rows (lanes), 16-byte
      // chunk c of row r at chunk c ^ (r % 8) (the 128-byte swizzle).
      // A negative scale is taken as |scale| on -Q (exact), so that the
      // softmax can take its maximum over the raw scores.
      const uint32_t flip = p.scale_log2 < 0.f ? 0x80008000u : 0u;
      const int qr = lg * 32 + lane, c0 = hf * 8;
      const int row = row0 + qr;
      const uint4* src = nullptr;
      if (row < R) {
        const int b = members[row / G], h = kvh * G + row % G;
        src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.q) +
                                             (static_cast<size_t>(b) * p.n_q_heads + h) * D * 2);
      }
      uint4 v[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) v[c] = src ? __ldg(src + c0 + c) : make_uint4(0u, 0u, 0u, 0u);
      uint8_t* qrow = q_s + hf * (kTcRows * 128) + qr * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(qrow + ((c ^ (qr & 7)) * 16)) =
            make_uint4(v[c].x ^ flip, v[c].y ^ flip, v[c].z ^ flip, v[c].w ^ flip);
      // Generic-proxy writes, read by the tensor cores (async proxy).
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    tc_fence_before();
    named_bar_sync(1, (kTcSoftmaxWarps + 1) * 32);  // tensor memory allocated, Q in shared memory
    tc_fence_after();
    tmem = *tmem_slot;

    if (warp == kTcMmaWarp) {
      // ---------------- MMA issue (the whole warp, one elected lane) ----------------
      // S of a stage is issued as soon as its K has landed and its S buffer
      // is free (P V of the stage four back done), O_t += P V as soon as
      // its P is written; the warp polls both and issues in stage order
      // within each kind.  Decisions are taken from lane 0, so that the
      // warp stays converged.
      if (n_stages > 0) {
        constexpr uint32_t kIdS = tc_idesc<kBf16>(false, kTcKeys), kIdPV = tc_idesc<kBf16>(true, D);
        const uint32_t ra = smem_u32(ring);
        // Descriptors of ring slot 0's K (dims 0-15) and V (block 0); the
        // other operands add a start-address offset (16-byte units).
        const uint64_t dk0 = smem_desc_sw128(ra, 16, 2048);
        const uint64_t dq0 = smem_desc_sw128(smem_u32(q_s), 16, 1024);
        const uint64_t dv0 = smem_desc_sw128(ra + kTcKVBytes, kBlockTokens * 128, 1024);
        int ns = 0, np = 0;  // next stage whose S, whose P V is to be issued
        uint64_t t0 = 0;
        uint32_t idle = 0;
        bool mok = true;
        while (np < n_stages) {
          bool progress = false;
          // The buffer's previous P V must have been issued before its
          // barrier's parity says anything about it.
          bool go = ns < n_stages && (ns < kTcSBufs || np > ns - kTcSBufs) &&
                    mbar_test_wait(&kv_full[ns % kTcStages], (ns / kTcStages) & 1) &&
                    (ns < kTcSBufs || mbar_test_wait(&s_free[ns % kTcSBufs], ((ns - kTcSBufs) / kTcSBufs) & 1));
          if (__shfl_sync(0xffffffffu, go, 0)) {
            tc_fence_after();
            const uint64_t dk = dk0 + static_cast<uint64_t>(((ns % kTcStages) * kTcStageBytes) >> 4);
            const uint32_t d = tmem + (ns % kTcSBufs) * kTcKeys;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              // Dims 16 kk ..: dim half kk / 4, 32-byte step kk % 4 of its
              // 128-byte rows; the 8-token atoms of the half lie 2 KiB apart.
              tc_mma_ss(d, dq0 + static_cast<uint64_t>(((kk >> 2) * (kTcRows * 128) + (kk & 3) * 32) >> 4),
                        dk + static_cast<uint64_t>(((kk >> 2) * 1024 + (kk & 3) * 32) >> 4), kIdS, kk > 0);
            }
            tc_commit(&s_full[ns % kTcSBufs]);
            ++ns;
            progress = true;
          }
          go = np < ns && mbar_test_wait(&p_full[np % kTcSBufs], (np / kTcSBufs) & 1);
          if (__shfl_sync(0xffffffffu, go, 0)) {
            tc_fence_after();
            const uint64_t dv = dv0 + static_cast<uint64_t>(((np % kTcStages) * kTcStageBytes) >> 4);
            const uint32_t pa = tmem + (np % kTcSBufs) * kTcKeys;
#pragma unroll
            for (int kt = 0; kt < kTcKeys / 16; ++kt) {
              // V of block kt: [half][16 tokens][128 B], halves 2 KiB apart.
              tc_mma_ts(tmem + kTcOCol + (np & 1) * D, pa + kt * 8,
                        dv + static_cast<uint64_t>((kt * kTcBlockBytes) >> 4), kIdPV, np > 1 || kt > 0);
            }
            tc_commit(&s_free[np % kTcSBufs]);
            tc_commit(&kv_empty[np % kTcStages]);
            ++np;
            progress = true;
          }
          int st = 0;  // 0 go on, 1 another warp gave up, 2 the limit passed
          if (progress) {
            idle = 0;
          } else if ((++idle & 1023u) == 0) {
            // The clock is read once per 1024 idle polls: the first read
            // after progress starts the limit, later ones test it.
            const uint64_t now = global_timer_ns();
            if (idle == 1024u) t0 = now;
            st = *abort_flag ? 1 : (now - t0 > kWaitLimitNs) ? 2 : 0;
          }
          st = __shfl_sync(0xffffffffu, st, 0);
          if (st != 0) {
            if (st == 2 && lane == 0) {
              *abort_flag = 1;
              flag_error(kDevErrTimeout);
            }
            mok = false;
            break;
          }
        }
        // Before the tensor memory is freed, every MMA issued must have completed.
        if (!mok && ns > 0) {
          tc_commit(mma_drain);
          if (lane == 0) {
            const uint64_t t1 = global_timer_ns();
            while (!mbar_try_wait(mma_drain, 0) && global_timer_ns() - t1 < kWaitLimitNs) {
            }
          }
          __syncwarp();
        }
      }
    } else {
      // ---------------- softmax: set hf, rows 32 lg .. 32 lg + 31 ----------------
      // Every tensor-memory access is warp-converged (.sync.aligned): waits
      // and decisions are made warp-uniform first.  After a failed wait the
      // warp still arrives on every P barrier, so that nothing waits for it
      // in vain.
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(lg * 32) << 16);
      const uint32_t o_col = kTcOCol + hf * D;
      const float sc = fabsf(p.scale_log2);
      float l_set = 0.f;
      // Block ids of a stage's four blocks, read one own stage ahead: a block
      // whose id is outside the pool contributes no key (its copy read block
      // 0, whose scores are masked here).
      auto bad_mask = [&](int s) {
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < kTcBlocks; ++i) {
          const int j = (s_begin + s) * kTcBlocks + i;
          const int id = j < n_prefix_blocks ? __ldg(tab + j) : 0;
          if (id < 0 || id >= p.num_blocks) m |= 1u << i;
        }
        return m;
      };
      uint32_t bad_next = hf < n_stages ? bad_mask(hf) : 0u;
      int k = 0;  // this set's stage count so far
      for (int s = hf; s < n_stages; s += 2, ++k) {
        const uint32_t bad = bad_next;
        if (s + 2 < n_stages) bad_next = bad_mask(s + 2);
        const int sb = s % kTcSBufs;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_full[sb], (s / kTcSBufs) & 1, abort_flag,
                                                                kWaitLimitNs));
        float x[64];
        if (ok) {
          tc_fence_after();
          float xa[32], xb[32];
          tmem_ld32(lane_base + sb * kTcKeys, xa);
          tmem_ld32(lane_base + sb * kTcKeys + 32, xb);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            x[i] = xa[i];
            x[32 + i] = xb[i];
          }
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) x[i] = 0.f;
        }

        // Scores past the prefix (only in the last stage) and those of a bad
        // block are masked: bit i of keep[h] is score 32 h + i.
        const int live = min(kTcKeys, plen - (s_begin + s) * kTcKeys);
        uint32_t keep[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int lv = live - 32 * h;
          keep[h] = lv >= 32 ? 0xffffffffu : lv <= 0 ? 0u : (1u << lv) - 1u;
          if (bad & (1u << (2 * h))) keep[h] &= 0xffff0000u;
          if (bad & (2u << (2 * h))) keep[h] &= 0x0000ffffu;
        }
        const bool masked = (keep[0] & keep[1]) != 0xffffffffu;
        if (masked) {
#pragma unroll
          for (int i = 0; i < 64; ++i) x[i] = ((keep[i >> 5] >> (i & 31)) & 1u) ? x[i] : -INFINITY;
        }
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < 64; i += 2) mx4[(i >> 1) & 3] = max3f(mx4[(i >> 1) & 3], x[i], x[i + 1]);
        float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        mx = (keep[0] | keep[1]) != 0u ? mx * sc : -INFINITY;  // the maximum of the scaled scores (sc >= 0)
        // Move the reference maximum only when it grows by more than 2^8 (so
        // that O_t rarely makes the round trip); when any row of the warp
        // moves, the warp takes the round trip for its 128 columns of O_t,
        // with factor 1 for the rows that stay.  O_t is stable once the set's
        // previous P V (stage s - 2) is done: the free barrier of its S
        // buffer, whose earlier use (stage s - 2 - kTcSBufs) completed before
        // S of stage s - 2 was issued, so that its parity is unambiguous.
        const bool move = mx > m_ref + 8.f;
        if (ok && k > 0 && __any_sync(0xffffffffu, move)) {
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_free[(s - 2) % kTcSBufs], ((s - 2) / kTcSBufs) & 1,
                                                         abort_flag, kWaitLimitNs));
          if (ok) {
            tc_fence_after();
            const float alpha = move ? exp2f(m_ref - mx) : 1.f;
            l_set *= alpha;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              float v[32];
              tmem_ld32(lane_base + o_col + c * 32, v);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] *= alpha;
              tmem_st32(lane_base + o_col + c * 32, v);
            }
            tmem_wait_st();
          }
        }
        if (move) m_ref = mx;
        {
          const uint64_t sc2 = f2_pack(sc, sc), nm2 = f2_pack(-m_ref, -m_ref);
#pragma unroll
          for (int i = 0; i < 64; i += 2) f2_unpack(f2_fma(f2_pack(x[i], x[i + 1]), sc2, nm2), x[i], x[i + 1]);
        }
        if (masked) {
#pragma unroll
          for (int i = 0; i < 64; ++i) x[i] = ((keep[i >> 5] >> (i & 31)) & 1u) ? x[i] : -INFINITY;
        }
        uint64_t sum2[2] = {0ull, 0ull};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pw[16];  // 32 probabilities as 16-bit pairs
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float a = ex2_ftz(x[32 * h + 2 * j]), b = ex2_ftz(x[32 * h + 2 * j + 1]);
            sum2[j & 1] = f2_add(sum2[j & 1], f2_pack(a, b));
            pw[j] = pack2<kBf16>(a, b);
          }
          // P over the first half of the stage's S buffer (its scores are in registers).
          if (ok) tmem_st16(lane_base + sb * kTcKeys + h * 16, pw);
        }
        if (ok) tmem_wait_st();
        {
          float a0, a1, b0, b1;
          f2_unpack(sum2[0], a0, a1);
          f2_unpack(sum2[1], b0, b1);
          l_set += (a0 + a1) + (b0 + b1);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[sb]);
      }
      // Both sets' accumulators are final once each set's last P V is done
      // (and with it every earlier MMA).  Its S buffer's free barrier is
      // waited on, not a per-set counter: when the set's P V two stages
      // back is still in flight, a per-set barrier would be two phases
      // behind and its parity would read as done.
      if (ok && k > 0) {
        const int s_last = hf + 2 * (k - 1);
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_free[s_last % kTcSBufs], (s_last / kTcSBufs) & 1,
                                                        abort_flag, kWaitLimitNs));
      }
      // The two sets' states of each row, combined: weights 2^(m_t - max m),
      // 0 for a set with no keys; NaN in the sum marks a row whose pipeline
      // failed.
      red_max[hf * kTcRows + r] = m_ref;
      red_l[hf * kTcRows + r] = l_set;
      if (lane == 0) set_ok[hf][lg] = ok ? 1 : 0;
      tc_fence_before();
      named_bar_sync(2 + lg, 64);
      tc_fence_after();
      ok = ok && set_ok[hf ^ 1][lg] != 0;  // warp-uniform
      {
        const float m_o = red_max[(hf ^ 1) * kTcRows + r], l_o = red_l[(hf ^ 1) * kTcRows + r];
        const float m_c = fmaxf(m_ref, m_o);
        const float a_me = m_ref == -INFINITY ? 0.f : exp2f(m_ref - m_c);
        const float a_o = m_o == -INFINITY ? 0.f : exp2f(m_o - m_c);
        l_row = ok ? a_me * l_set + a_o * l_o : __int_as_float(0x7fc00000);
        set_w[0] = hf == 0 ? a_me : a_o;  // selects, not a dynamic index (which would live on the stack)
        set_w[1] = hf == 0 ? a_o : a_me;
        m_ref = m_c;
      }
      if (owner != crank) {
        // Partial state for the owner of these rows, in the drained ring
        // (every copy into it has been consumed by an MMA that has completed).
        float* part_o = reinterpret_cast<float*>(ring);  // [128 rows][kTcPartStride]
        float* part_ml = part_o + kTcRows * kTcPartStride;  // m [128], l [128]
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float v[32];
          load_o(c, v);
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(part_o + r * kTcPartStride + hf * 64 + c * 32 + i) =
                make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
        if (hf == 0) {
          part_ml[r] = m_ref;
          part_ml[kTcRows + r] = l_row;
        }
      } else {
        // This warp's 64 columns of its own share of O, not yet weighted, into
        // [128 rows][512 B] (16-byte chunk c of row r at c ^ (r % 8)); done
        // before the cluster barrier, so that it overlaps the other CTAs'
        // partial writes.
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float t[32];
          load_o(c, t);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int chunk = (hf * 16 + c * 8 + i) ^ (r & 7);
            *reinterpret_cast<float4*>(out_s + r * 512 + chunk * 16) =
                make_float4(t[4 * i], t[4 * i + 1], t[4 * i + 2], t[4 * i + 3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  cluster_sync();  // partial states and own shares written
  tc_fence_after();
  if (warp < kTcSoftmaxWarps && owner == crank) {
    // The row's state, merged over the cluster: O (unnormalised), m, l.
    // Rows out, coalesced: warp (lg, hf) takes rows 32 lg + 16 hf .. + 15,
    // lane l the 16-byte chunk l of each; the other shares of the same chunk
    // come from their CTAs' shared memory, one 512-byte row per warp-wide
    // load, weighted with the factors of the lane that holds the row's state
    // (lane 16 hf + j for row 32 lg + 16 hf + j).  The first other share's
    // rows are requested together with every share's m and l.
    const uint32_t part_o_addr = smem_u32(ring);
    const uint32_t part_ml_addr = part_o_addr + kTcRows * kTcPartStride * 4;
    const int rbase = lg * 32 + hf * 16;
    const uint32_t first = crank == 0 ? 1u : 0u;  // the first other CTA of the cluster
    float m_all = m_ref;
    float wk[kTcMaxSplit], lk[kTcMaxSplit];
    bool valid = !isnan(l_row);
#pragma unroll
    for (int k = 0; k < kTcMaxSplit; ++k) {
      wk[k] = -INFINITY;
      lk[k] = 0.f;
      if (k < static_cast<int>(csize) && k != static_cast<int>(crank)) {
        wk[k] = ld_cluster(cluster_map(part_ml_addr + r * 4, k));
        lk[k] = ld_cluster(cluster_map(part_ml_addr + (kTcRows + r) * 4, k));
      }
    }
    float4 t[16];
    if (csize > 1) {
      const uint32_t src = cluster_map(part_o_addr + (rbase * kTcPartStride + lane * 4) * 4, first);
#pragma unroll
      for (int j = 0; j < 16; ++j) t[j] = ld_cluster4(src + j * kTcPartStride * 4);
    }
    float4 o[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int rr = rbase + j;
      o[j] = *reinterpret_cast<const float4*>(out_s + rr * 512 + ((lane ^ (rr & 7)) * 16));
    }
#pragma unroll
    for (int k = 0; k < kTcMaxSplit; ++k) {
      if (k < static_cast<int>(csize) && k != static_cast<int>(crank)) {
        valid = valid && !isnan(lk[k]);
        m_all = fmaxf(m_all, wk[k]);
      }
    }
    // Weight of each share: 2^(m_k - max m), 0 for a share with no keys.
    const float a_self = m_ref == -INFINITY ? 0.f : exp2f(m_ref - m_all);
    float l_all = a_self * l_row;
#pragma unroll
    for (int k = 0; k < kTcMaxSplit; ++k) {
      wk[k] = wk[k] == -INFINITY ? 0.f : exp2f(wk[k] - m_all);
      l_all += wk[k] * lk[k];
    }
    const int row = row0 + r;
    int dst = -1;  // this lane's row's destination (-1: none)
    if (row < R && valid) {
      dst = members[row / G] * p.n_q_heads + kvh * G + row % G;
      if (hf == 0) {
        const size_t nqb = static_cast<size_t>(p.batch) * p.n_q_heads;
        p.init[nqb * D + dst] = m_all;
        p.init[nqb * D + nqb + dst] = l_all;
      }
    }
    float w_first = 0.f;
#pragma unroll
    for (int k = 0; k < kTcMaxSplit; ++k) w_first = k == static_cast<int>(first) ? wk[k] : w_first;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float ws = __shfl_sync(0xffffffffu, a_self, hf * 16 + j);
      o[j].x *= ws;
      o[j].y *= ws;
      o[j].z *= ws;
      o[j].w *= ws;
    }
    if (csize > 1) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float w = __shfl_sync(0xffffffffu, w_first, hf * 16 + j);
        o[j].x += w * t[j].x;
        o[j].y += w * t[j].y;
        o[j].z += w * t[j].z;
        o[j].w += w * t[j].w;
      }
    }
#pragma unroll
    for (int k = 0; k < kTcMaxSplit; ++k) {
      if (k < static_cast<int>(csize) && k != static_cast<int>(crank) && k != static_cast<int>(first)) {
        const uint32_t src = cluster_map(part_o_addr + (rbase * kTcPartStride + lane * 4) * 4, k);
#pragma unroll
        for (int j = 0; j < 16; ++j) t[j] = ld_cluster4(src + j * kTcPartStride * 4);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float w = __shfl_sync(0xffffffffu, wk[k], hf * 16 + j);
          o[j].x += w * t[j].x;
          o[j].y += w * t[j].y;
          o[j].z += w * t[j].z;
          o[j].w += w * t[j].w;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int d = __shfl_sync(0xffffffffu, dst, hf * 16 + j);
      if (d >= 0) *reinterpret_cast<float4*>(p.init + static_cast<size_t>(d) * D + lane * 4) = o[j];
    }
  }
  tc_fence_before();
  cluster_sync();  // the other CTAs' shared memory stays in place until every owner has read it
  if (warp == kTcMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols));
  }
}

}  // namespace pkv
