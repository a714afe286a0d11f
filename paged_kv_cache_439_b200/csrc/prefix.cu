// Shared-prefix (cascade) pass of paged decode attention, bf16 caches, on the
// fifth-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// Prefix caching ("生产级 LLM 推理的 KV 缓存优化" (GPUYard), the serving-flags
// section: --enable-prefix-caching avoids recomputing shared prompt prefixes;
// "LLM推理显存优化KV Cache管理3大策略" §2: blocks carry a ref_count so that
// sequences can share them) lets many sequences point at the same physical
// blocks for their common first tokens.  A per-sequence decode reads those
// blocks once per sequence.  This pass reads them once per KV head for all
// sequences: for KV head h and a slice of the prefix it computes, for every
// (sequence, q head of h's group) row, the attention of that q row over the
// slice, and writes the normalised partial (o, log2-sum-exp) into the split
// workspace.  The per-sequence suffix runs through the split decode kernel
// from token prefix_len on, and the merge kernel combines both exactly.
//
// The rows of one KV head form a dense contraction, so one CTA takes 128 / group
// whole sequences, up to 128 rows (the M of one tcgen05.mma), and walks its
// slice in 64-token tiles:
//   S = Q K^T      tcgen05.mma, A = Q and B = K from shared memory (K-major,
//                  128-byte swizzle), D = S in tensor memory (128 lanes x 64
//                  fp32 columns, one of two score buffers);
//   softmax        thread r owns row r: tcgen05.ld of its 64 scores, fp32
//                  online softmax, P written back over S in the same buffer
//                  as bf16 hi + lo halves (about 16 significant bits of P);
//   O += P V       tcgen05.mma with A = P from tensor memory and B = V from
//                  shared memory (head_dim-major), D = O in tensor memory.
// The running maximum is only moved when a tile's maximum exceeds it by more
// than 2^8 (then O is rescaled in tensor memory): exponentials stay below 256,
// and the final normalisation uses the same maximum as every P, so the result
// is the same softmax.  Two more warps feed the tensor cores: one lane of a
// copy warp issues every TMA copy, one lane of an MMA warp every tcgen05.mma;
// copies, tcgen05.commit (S ready, P V done, and per ring stage "K/V stage
// free") and the softmax warps' hand-offs (S read, P written) arrive on
// mbarriers, each wait bounded.  Q, K and V move by
// TMA (cp.async.bulk.tensor) straight into the 128-byte-swizzled layout the
// MMAs read: Q as a (sequences x heads x 64 columns) box, the K and V tiles
// as one box per paged block (or 64-token piece of one) and column block, a
// bad block being read from past the end of the cache (zero fill).  K and V
// have two-stage rings of their own.  With two score buffers the softmax of
// tile j never waits for an MMA other than its own S: P_j goes over S_j, S of
// tile j + 1 is already in the other buffer, and S of tile j + 2 is issued
// into buffer j % 2 once P V of tile j has read P_j there (it runs during
// tile j + 1's softmax).  K tile j + 2 is fetched once S of tile j is done, V
// tile j + 1 once P V of tile j - 1 is done.  Two CTAs share an SM (half of
// its tensor memory each, at most 168 registers a thread so that both fit),
// so one CTA's softmax overlaps the other's MMAs.  The softmax keeps eight
// independent max and sum chains per row.
#include <math_constants.h>

#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "decode.cuh"

namespace pkv {

namespace {

constexpr int kTcSoftmaxWarps = 4;  // thread r owns row r; warp w reads TMEM lanes 32w..32w+31
constexpr int kTcThreads = (kTcSoftmaxWarps + 2) * 32;  // plus a copy warp and an MMA warp
constexpr int kTcRows = 128;     // rows per CTA (MMA M)
constexpr int kTcTok = kPrefixTokens;  // tokens per tile (MMA N of Q K^T)
constexpr int kTcStages = 2;
constexpr float kRescaleLog2 = 8.f;  // move the running max only past 2^8
constexpr uint64_t kWaitNs = 2000000000ull;  // a wait gives up after 2 s
constexpr int kOTile = kTcRows * 128;            // staged partial: 128 rows x 32 fp32 columns
constexpr int kTailBarBytes = 128;               // mbarriers, tensor-memory address, failure word
constexpr int kTailBytes = kTailBarBytes + kTcRows * 8;  // then one workspace row per row

static_assert(kTcTok == 64, "the score row is read as two 32-column loads");

template <int HD>
struct TcCfg {
  static constexpr int DB = HD / 64;                      // 128-byte column blocks of head_dim
  static constexpr int Q_DB = kTcRows * 128;              // bytes of one Q column block
  static constexpr int KV_DB = kTcTok * 128;              // bytes of one K (or V) column block
  static constexpr int Q_BYTES = DB * Q_DB;
  static constexpr int KV_BYTES = DB * KV_DB;            // one K (or V) tile
  // tensor-memory columns: two score buffers, S_j in buffer j % 2 (64 fp32
  // columns) and P_j over it (bf16 hi + lo pairs: 32 columns each), then O
  static __device__ __forceinline__ uint32_t s_col(int j) { return (uint32_t)((j & 1) * kTcTok); }
  static constexpr int O_COL = 2 * kTcTok;
  static constexpr int COLS_USED = O_COL + HD;
  static constexpr int TMEM_COLS = COLS_USED <= 128 ? 128 : (COLS_USED <= 256 ? 256 : 512);
  // dynamic shared memory: 1 KB alignment slack, Q, the stages, then the
  // block-table slice, the mbarriers, the tensor-memory address and failure
  // word, and the workspace row of each of the 128 rows
  static constexpr int BODY = Q_BYTES + 2 * kTcStages * KV_BYTES;
  static_assert(HD == 64 || HD == 128, "head_dim 64 or 128");
};

// Shared-memory matrix descriptor (tcgen05): start address, leading and
// stride byte offsets (all >> 4), version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B,
// A K-major, B K-major (b_mn = 0) or N-major (b_mn = 1), M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits for the mbarrier phase with the given parity; false once kWaitNs have
// passed (the caller records the failure and stops issuing work).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
    if (i == 0) t0 = global_ns();
    else if ((i & 15) == 0 && global_ns() - t0 > kWaitNs) return false;
  }
}

// One lane per warp polls while the others wait at the warp barrier, so that
// waiting warps do not flood the shared-memory pipe that the copies and the
// tensor-memory loads go through.  Every lane gets the result.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// 32 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Arrives on `bar` (count 1) and adds `bytes` of expected copy transactions.
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
// Adds `bytes` of expected copy transactions without arriving.
__device__ __forceinline__ void mbar_add_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// One box of a 3-D tensor map into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// One box of a 4-D tensor map from shared to global memory, in this thread's
// bulk group.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int x, int y,
                                             int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::
          "l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}
// Waits until this thread's bulk stores have completed.
__device__ __forceinline__ void bulk_store_wait() {
  asm volatile("cp.async.bulk.commit_group;\n cp.async.bulk.wait_group 0;" ::: "memory");
}

// Max of 64 values in 8 independent chains.
__device__ __forceinline__ float max64(const float (&v)[kTcTok]) {
  float m[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) m[c] = v[c];
#pragma unroll
  for (int i = 8; i < kTcTok; i += 8)
#pragma unroll
    for (int c = 0; c < 8; ++c) m[c] = fmaxf(m[c], v[i + c]);
  return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])),
               fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Bounded wait for the phase that tile `last` completed on a two-stage ring's
// barrier pair (tile j: stage j % 2, phase j / 2), and, when both stages were
// used, for the other stage's last tile.  True when nothing was issued.
__device__ __forceinline__ bool drain_last(uint32_t bar_pair, int last) {
  bool done = true;
  for (int j = last; j >= 0 && j >= last - 1; --j)
    done = done && mbar_wait(bar_pair + 8 * (j % 2), (uint32_t)((j / 2) & 1));
  return done;
}

// Bits of the CTA's failure word: a wait gave up; a drain gave up as well.
constexpr int kFailWait = 1, kFailDrain = 2;

template <int HD>
__global__ void __maxnreg__(168)  // 2 CTAs x 6 warps per SM: 3 warps x 168 regs per SM partition
    prefix_kernel(const DecodeParams p, const PrefixParams pp,
                  const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o) {
  using Cfg = TcCfg<HD>;
  pdl_trigger();  // the split merge may be scheduled once every CTA has started
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // swizzle atoms need 1024-byte alignment
  uint8_t* const gbase = smem_raw + (base - raw);
  const uint32_t q_sm = base;
  const uint32_t k_ring = base + Cfg::Q_BYTES;
  const uint32_t v_ring = k_ring + kTcStages * Cfg::KV_BYTES;
  int* const s_phys = reinterpret_cast<int*>(gbase + Cfg::BODY);
  uint8_t* const tail = gbase + Cfg::BODY + pp.phys_bytes;
  // Each barrier's waiters must never fall two phases behind it (try_wait.parity
  // would then match the incomplete phase two ahead): every waiter polls a
  // barrier whose next phase cannot complete before that waiter's own next step.
  // Tile j uses score buffer j % 2 and the phase j / 2 of that buffer's pair.
  const uint32_t bar_sfull = smem_u32(tail);        // [2]: S of a tile is in tensor memory
  const uint32_t bar_pfull = smem_u32(tail + 16);   // [2]: every row has written P (4 warps)
  const uint32_t bar_odone = smem_u32(tail + 32);   // a tile's P V has been accumulated (MMA)
  // Every MMA the CTA issued has completed: one commit after the last issue,
  // waited once (phase 0), so no later phase can alias it.  The final waits
  // use it rather than odone, whose last two phases may both have completed
  // before a waiter polls (the parity of phase n would then match n - 2).
  const uint32_t bar_done = smem_u32(tail + 40);
  const uint32_t bar_k = smem_u32(tail + 48);       // [2]: K tile (and, first, Q) landed
  const uint32_t bar_v = smem_u32(tail + 64);       // [2]: V tile landed
  const uint32_t bar_kfree = smem_u32(tail + 80);   // [2]: S of the stage's K tile is done
  const uint32_t bar_vfree = smem_u32(tail + 96);   // [2]: P V of the stage's V tile is done
  volatile uint32_t* const s_tmem = reinterpret_cast<volatile uint32_t*>(tail + 112);
  volatile int* const s_fail = reinterpret_cast<volatile int*>(tail + 116);
  long long* const s_roff = reinterpret_cast<long long*>(tail + kTailBarBytes);  // [kTcRows]

  const int kvh = blockIdx.x, split = blockIdx.y, rg = blockIdx.z;
  const int tid = threadIdx.x, warp = tid / kWarp, lane = tid % kWarp;
  const bool copier = warp == kTcSoftmaxWarps, mma_warp = warp == kTcSoftmaxWarps + 1;
  const int G = p.group;
  const int spc = kTcRows / G;  // sequences per CTA; rows (seq, head) = spc * G <= 128
  const int t0 = split * pp.pchunk;
  const int t1 = min(pp.prefix_len, t0 + pp.pchunk);
  const int bs = p.block_size;
  const int blk0 = t0 >> p.log2_bs;
  const int ntiles = (t1 - t0 + kTcTok - 1) / kTcTok;

  // ---- set-up.  The copy lane initialises the barriers and starts the Q load
  // at once (it needs no block-table entry); then the block-table slice, the
  // tensor memory and the zeroed Q padding, all before one CTA barrier.
  if (copier && lane == 0) {
    mbar_init(bar_sfull, 1);
    mbar_init(bar_sfull + 8, 1);
    mbar_init(bar_pfull, kTcSoftmaxWarps);
    mbar_init(bar_pfull + 8, kTcSoftmaxWarps);
    mbar_init(bar_odone, 1);
    mbar_init(bar_done, 1);
    mbar_init(bar_kfree, 1);
    mbar_init(bar_kfree + 8, 1);
    mbar_init(bar_vfree, 1);
    mbar_init(bar_vfree + 8, 1);
    mbar_init(bar_k, 1);
    mbar_init(bar_k + 8, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_v + 8, 1);
    *s_fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    // Q (rows spc * G of this CTA's sequences) completes on K0's barrier
    // together with K0; the K0 load adds the arrival
    mbar_add_tx(bar_k, (uint32_t)(Cfg::DB * spc * G * 128));
#pragma unroll
    for (int db = 0; db < Cfg::DB; ++db)
      tma_load_3d(q_sm + (uint32_t)(db * Cfg::Q_DB), &tm_q, db * 64, kvh * G, rg * spc, bar_k);
  }
  {
    const int nphys = ((t1 - 1) >> p.log2_bs) - blk0 + 1;
    for (int i = tid; i < nphys; i += kTcThreads) {
      int b = p.block_tables[blk0 + i];
      if (b < 0 || b >= p.num_blocks) {
        set_flag(p.err_flag, PKV_FLAG_BAD_BLOCK);
        b = -1;
      }
      s_phys[i] = b;
    }
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32((const void*)s_tmem)),
                 "r"(Cfg::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // Q rows past spc * G (when G does not divide 128) are never loaded: zero them
  for (int rr = spc * G + tid / 8; rr < kTcRows; rr += kTcThreads / 8)
#pragma unroll
    for (int db = 0; db < Cfg::DB; ++db)
      *reinterpret_cast<uint4*>(gbase + db * Cfg::Q_DB + rr * 128 + (tid % 8) * 16) =
          make_uint4(0, 0, 0, 0);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();  // s_phys, barriers, tensor-memory address, zeroed Q rows
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  bool ok = true;

  if (copier) {
    // ================= copy warp: one lane issues every TMA copy =============
    // It waits only on per-stage "free" barriers: the next phase of each needs
    // the tile this warp loads after the wait, so the warp can never be two
    // phases behind one (which would alias the parity it polls).
    if (lane == 0) {
      const int R = bs < kTcTok ? bs : kTcTok;  // token rows per box
      const int nbox = kTcTok / R;
      const int oob = p.num_blocks * bs;
      // K or V tile j as boxes of R token rows x 64 head_dim columns, one per
      // (block piece, column block); a bad block, or rows past the slice, load
      // from past the end of the cache: zeros
      auto load_tile = [&](const CUtensorMap* map, uint32_t stage, int j, uint32_t bar) {
        const int tt = t0 + j * kTcTok;
        constexpr int kMaxBox = kTcTok / 8;  // block_size >= 8
        int z[kMaxBox];
#pragma unroll
        for (int b = 0; b < kMaxBox; ++b) {
          const int t = tt + b * R;
          const int phys = (b < nbox && t < t1) ? s_phys[(t >> p.log2_bs) - blk0] : -1;
          z[b] = phys >= 0 ? phys * bs + (t & (bs - 1)) : oob;
        }
        mbar_expect_tx(bar, Cfg::KV_BYTES);
#pragma unroll
        for (int b = 0; b < kMaxBox; ++b)
          if (b < nbox)
#pragma unroll
            for (int db = 0; db < Cfg::DB; ++db)
              tma_load_3d(stage + (uint32_t)(db * Cfg::KV_DB + b * R * 128), map, db * 64, kvh,
                          z[b], bar);
      };
      auto kstage = [&](int j) { return k_ring + (uint32_t)((j % kTcStages) * Cfg::KV_BYTES); };
      auto vstage = [&](int j) { return v_ring + (uint32_t)((j % kTcStages) * Cfg::KV_BYTES); };
      int k_last = -1, v_last = -1;  // last K and V tile issued
      // K0 first (S of tile 0 waits for it and Q), then V0, K1, V1
      load_tile(&tm_k, kstage(0), 0, bar_k);
      load_tile(&tm_v, vstage(0), 0, bar_v);
      k_last = v_last = 0;
      if (ntiles > 1) {
        load_tile(&tm_k, kstage(1), 1, bar_k + 8);
        load_tile(&tm_v, vstage(1), 1, bar_v + 8);
        k_last = v_last = 1;
      }
      for (int j = 0; ok && j < ntiles; ++j) {
        // S of tile j is done: K tile j's stage takes tile j + 2
        if (j + 2 < ntiles) {
          ok = mbar_wait(bar_kfree + 8 * (j % 2), (uint32_t)((j / 2) & 1));
          if (ok) {
            load_tile(&tm_k, kstage(j), j + 2, bar_k + 8 * (j % 2));
            k_last = j + 2;
          }
        }
        // P V of tile j - 1 is done: its V stage takes tile j + 1
        if (ok && j > 0 && j + 1 < ntiles) {
          ok = mbar_wait(bar_vfree + 8 * ((j - 1) % 2), (uint32_t)(((j - 1) / 2) & 1));
          if (ok) {
            load_tile(&tm_v, vstage(j + 1), j + 1, bar_v + 8 * ((j + 1) % 2));
            v_last = j + 1;
          }
        }
      }
      if (!ok) atomicOr(const_cast<int*>(s_fail), kFailWait);
      // Drain: every copy this lane issued lands before the CTA can exit, also
      // after a wait gave up.  Tile j of a ring completes phase j / 2 of its
      // stage's barrier, and only this lane's loads arrive there, so waiting
      // on the parity of the last tile issued per stage cannot alias.
      if (!drain_last(bar_k, k_last) || !drain_last(bar_v, v_last))
        atomicOr(const_cast<int*>(s_fail), kFailDrain);
    }
  } else if (mma_warp) {
    // ================= MMA warp: one lane issues every tcgen05.mma ============
    if (lane == 0) {
      // descriptors of the operand bases; an MMA adds its offset (>> 4) to the
      // start-address field, which never carries out (shared addresses < 256 KB)
      const uint64_t dq = smem_desc(q_sm, 16, 1024);
      const uint64_t dk = smem_desc(k_ring, 16, 1024);
      const uint64_t dv = smem_desc(v_ring, Cfg::KV_DB, 1024);
      constexpr uint32_t kIdQK = idesc_bf16(kTcRows, kTcTok, 0);
      constexpr uint32_t kIdPV = idesc_bf16(kTcRows, HD, 1);
      auto issue_qk = [&](int j) {  // S = Q K^T of tile j into score buffer j % 2
        const uint64_t kb0 = dk + (uint64_t)(((j % kTcStages) * Cfg::KV_BYTES) >> 4);
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
          const uint32_t koff = (uint32_t)((ks >> 2) * Cfg::KV_DB + (ks & 3) * 32) >> 4;
          const uint32_t qoff = (uint32_t)((ks >> 2) * Cfg::Q_DB + (ks & 3) * 32) >> 4;
          mma_ss(tmem + Cfg::s_col(j), dq + qoff, kb0 + koff, kIdQK, ks > 0);
        }
        mma_commit(bar_sfull + 8 * (j % 2));
        mma_commit(bar_kfree + 8 * (j % 2));
      };
      auto issue_pv = [&](int j) {  // O += P V of tile j, P (bf16 hi + lo) over S_j
        const uint64_t vb0 = dv + (uint64_t)(((j % kTcStages) * Cfg::KV_BYTES) >> 4);
        const uint32_t ph = tmem + Cfg::s_col(j), pl = ph + kTcTok / 2;
#pragma unroll
        for (int kk = 0; kk < kTcTok / 16; ++kk) {
          const uint64_t bd = vb0 + (uint64_t)((kk * 16 * 128) >> 4);
          mma_ts(tmem + Cfg::O_COL, ph + kk * 8, bd, kIdPV, (j > 0 || kk > 0));
          mma_ts(tmem + Cfg::O_COL, pl + kk * 8, bd, kIdPV, 1u);
        }
        mma_commit(bar_odone);
        mma_commit(bar_vfree + 8 * (j % 2));
      };
      int n_qk = 0, n_pv = 0;  // tiles whose S = Q K^T / O += P V were issued
      // S of tiles 0 and 1 (one per score buffer)
      for (int j = 0; ok && j < 2 && j < ntiles; ++j) {
        ok = mbar_wait(bar_k + 8 * j, 0u);
        tc_fence_after();
        if (ok) {
          issue_qk(j);
          n_qk = j + 1;
        }
      }
      for (int j = 0; ok && j < ntiles; ++j) {
        // every row has written P_j, V_j has landed: O += P_j V_j
        ok = mbar_wait(bar_pfull + 8 * (j % 2), (uint32_t)((j / 2) & 1));
        if (ok) ok = mbar_wait(bar_v + 8 * (j % 2), (uint32_t)((j / 2) & 1));
        tc_fence_after();
        if (!ok) break;
        issue_pv(j);
        n_pv = j + 1;
        // S of tile j + 2 goes into buffer j % 2 once P V of tile j has read
        // P_j there and K tile j + 2 has landed; it runs during tile j + 1's
        // softmax
        if (j + 2 < ntiles) {
          ok = mbar_wait(bar_odone, (uint32_t)(j & 1));
          if (ok) ok = mbar_wait(bar_k + 8 * (j % 2), (uint32_t)(((j + 2) / 2) & 1));
          tc_fence_after();
          if (ok) {
            issue_qk(j + 2);
            n_qk = j + 3;
          }
        }
      }
      if (!ok) atomicOr(const_cast<int*>(s_fail), kFailWait);
      // every MMA issued so far, also after a wait gave up
      mma_commit(bar_done);
      // Drain: bar_done completes once every issued MMA has; then the last
      // phase committed on each ring barrier (its earlier phases were waited
      // by the softmax or the copy warp, so none of these waits can alias).
      // Only this lane commits to these barriers.
      bool drained = mbar_wait(bar_done, 0u) && drain_last(bar_sfull, n_qk - 1) &&
                     drain_last(bar_kfree, n_qk - 1) && drain_last(bar_vfree, n_pv - 1);
      if (!drained) atomicOr(const_cast<int*>(s_fail), kFailDrain);
    }
  } else {
    // ================= softmax: thread r owns row r ==========================
    const int row = tid;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int seq = rg * spc + row / G;
    const bool rvalid = row < spc * G && seq < p.num_seqs;
    const size_t qrow = (size_t)(rvalid ? seq : 0) * p.num_q_heads + kvh * G + row % G;
    s_roff[row] = rvalid ? (long long)(qrow * p.ws_slots + split) : -1ll;  // workspace row
    int lim = 0;  // tokens of the prefix this row attends to
    if (rvalid) {
      int ctx = p.context_lens[seq];
      ctx = ctx < 0 ? 0 : ctx;
      lim = min(ctx, pp.prefix_len);
    }
    float m_ref = -CUDART_INF_F;  // reference maximum of this row (scaled, log2 units)
    float l_run = 0.f;
    const float sc = p.scale_log2;
    for (int j = 0; j < ntiles; ++j) {
      const int tt = t0 + j * kTcTok;
      const uint32_t sbuf = tmem + lane_base + Cfg::s_col(j);
      // ---- scores of tile j
      ok = ok && warp_wait(bar_sfull + 8 * (j % 2), (uint32_t)((j / 2) & 1));
      tc_fence_after();
      float s[kTcTok];
      {
        float a[32], b[32];
        tmem_ld32(sbuf, a);
        tmem_ld32(sbuf + 32, b);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = a[i];
          s[32 + i] = b[i];
        }
      }
      // valid tokens of this row: inside the slice, below the row's limit, in a good block
      const int nval = max(0, min(t1, lim) - tt);
      bool bad = false;
      for (int b = (tt >> p.log2_bs) - blk0; b <= ((min(tt + kTcTok, t1) - 1) >> p.log2_bs) - blk0;
           ++b)
        bad |= s_phys[b] < 0;
      if (nval < kTcTok || bad || sc <= 0.f) {  // masked tile (or an unusual scale)
#pragma unroll
        for (int i = 0; i < kTcTok; ++i) {
          bool v = i < nval;
          if (bad) v = v && s_phys[((tt + i) >> p.log2_bs) - blk0] >= 0;
          s[i] = v ? s[i] * sc : -CUDART_INF_F;
        }
      } else {
#pragma unroll
        for (int i = 0; i < kTcTok; ++i) s[i] *= sc;
      }
      const float mt = max64(s);
      const bool move = mt > m_ref + kRescaleLog2;  // also true for the first valid tile
      const float m_new = move ? mt : m_ref;
      const float alpha = move ? fast_exp2(m_ref - m_new) : 1.f;  // 0 when m_ref = -inf

      // rare: rescale O in place, once the previous tile's P V is done (P_j
      // goes over S_j in its own buffer, so no other step waits for it).
      // tcgen05.ld/st are warp-collective, so the whole warp takes this path
      // when any of its rows needs it (alpha = 1 for the rest).
      const bool need = move && j > 0 && m_ref != -CUDART_INF_F;
      if (__any_sync(0xffffffffu, need)) {
        ok = ok && warp_wait(bar_odone, (uint32_t)((j - 1) & 1));
        tc_fence_after();
        const float a_row = need ? alpha : 1.f;
#pragma unroll 1
        for (int c = 0; c < HD; c += 32) {
          float o[32];
          tmem_ld32(tmem + lane_base + Cfg::O_COL + c, o);
          tmem_wait_ld();
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(o[i] * a_row);
          tmem_st32(tmem + lane_base + Cfg::O_COL + c, w);
          tmem_wait_st();
        }
      }
      l_run *= alpha;
      m_ref = m_new;
      const float m_use = m_ref == -CUDART_INF_F ? 0.f : m_ref;

      // ---- P = 2^(s - m) as bf16 hi + lo over S_j (8 partial sums)
      {
        uint32_t hi[32], lo[32];
        float rs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x0 = fast_exp2(s[2 * i] - m_use), x1 = fast_exp2(s[2 * i + 1] - m_use);
          rs[i & 7] += x0 + x1;
          const uint32_t h = pack_bf16(x0, x1);
          const float2 f = unpack_bf16(h);
          hi[i] = h;
          lo[i] = pack_bf16(x0 - f.x, x1 - f.y);
        }
        l_run += ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
        tmem_st32(sbuf, hi);
        tmem_st32(sbuf + kTcTok / 2, lo);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_pfull + 8 * (j % 2));
      if (!ok) break;
    }
    // ---- every MMA, the last P V included, is done
    ok = ok && warp_wait(bar_done, 0u);
    tc_fence_after();
    if (!ok && lane == 0) atomicOr(const_cast<int*>(s_fail), kFailWait);
    // ---- normalise this slice's partial into shared memory (the K/V rings,
    // idle once the last P V is done): one 128-byte-swizzled tile of 128 rows
    // x 32 columns per column block, the layout of the tensor store below
    if (ok) {
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll 1
      for (int c = 0; c < HD; c += 64) {
        float o0[32], o1[32];
        tmem_ld32(tmem + lane_base + Cfg::O_COL + c, o0);
        tmem_ld32(tmem + lane_base + Cfg::O_COL + c + 32, o1);
        tmem_wait_ld();
        float4* t0 = reinterpret_cast<float4*>(gbase + Cfg::Q_BYTES + (c / 32) * kOTile + row * 128);
        float4* t1 = t0 + kOTile / 16;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          t0[i ^ (row & 7)] = make_float4(o0[4 * i] * inv, o0[4 * i + 1] * inv,
                                          o0[4 * i + 2] * inv, o0[4 * i + 3] * inv);
          t1[i ^ (row & 7)] = make_float4(o1[4 * i] * inv, o1[4 * i + 1] * inv,
                                          o1[4 * i + 2] * inv, o1[4 * i + 3] * inv);
        }
      }
      if (rvalid)
        p.ws_lse[qrow * p.ws_slots + split] = l_run > 0.f ? m_ref + log2f(l_run) : -CUDART_INF_F;
    }
  }

  fence_async_smem();  // the staged partial, to the tensor store
  tc_fence_before();
  const bool failed = __syncthreads_or(!ok || *s_fail != 0);
  if (failed) {
    // A slice that gave up writes a defined partial instead (o = 0, log2-sum-exp
    // = -inf): the merge then gives it weight 0 and the output stays finite.
    if (warp < kTcSoftmaxWarps) {
      const int row = tid;
#pragma unroll 1
      for (int cb = 0; cb < HD / 32; ++cb)
#pragma unroll
        for (int i = 0; i < 8; ++i)
          reinterpret_cast<float4*>(gbase + Cfg::Q_BYTES + cb * kOTile + row * 128)[i] =
              make_float4(0.f, 0.f, 0.f, 0.f);
      const long long slot = s_roff[row];
      if (slot >= 0) p.ws_lse[slot] = -CUDART_INF_F;
    }
    fence_async_smem();
    __syncthreads();
  }
  // The partial rows of this slice, (sequence, q head) rows x head_dim, as one
  // tensor box per 32-column block: workspace dims (head_dim, slot, q head,
  // sequence); rows of sequences past num_seqs fall outside and are dropped.
  if (copier && lane == 0) {
#pragma unroll
    for (int cb = 0; cb < HD / 32; ++cb)
      tma_store_4d(&tm_o, smem_u32(gbase + Cfg::Q_BYTES + cb * kOTile), cb * 32, split, kvh * G,
                   rg * spc);
    bulk_store_wait();
  }
  if (failed && tid == 0) set_flag(p.err_flag, PKV_FLAG_TIMEOUT);
  // Tensor memory is freed after the bounded drains above, also when one of
  // them gave up: tcgen05.alloc waits without a bound for free columns, so
  // memory left allocated could stall a later CTA on this SM indefinitely.
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(Cfg::TMEM_COLS)
                 : "memory");
  }
  // Launched behind the suffix decode (see launch_prefix), this grid may start
  // before that one ends; it completes only after it, so the merge, which
  // waits for this grid, also sees every suffix partial.
  pdl_wait();
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// bf16 tensor [d2][d1][d0] (d0 innermost, contiguous rows) with 128-byte
// swizzled boxes of 64 x b1 x b2 elements.
cudaError_t bf16_map(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                     uint32_t b1, uint32_t b2) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  const cuuint32_t box[3] = {64u, b1, b2};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The workspace partials as fp32 [num_seqs][num_q_heads][slots][head_dim],
// stored through 128-byte-swizzled boxes of 32 columns x 1 slot x group heads x
// sequences-per-CTA.
cudaError_t ws_map(CUtensorMap* map, float* base, uint64_t hd, uint64_t slots, uint64_t nqh,
                   uint64_t nseq, uint32_t group, uint32_t spc) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[4] = {hd, slots, nqh, nseq};
  const cuuint64_t strides[3] = {hd * 4, hd * 4 * slots, hd * 4 * slots * nqh};
  const cuuint32_t box[4] = {32u, 1u, group, spc};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int HD>
int smem_bytes(const PrefixParams& pp) {
  return 1024 + TcCfg<HD>::BODY + pp.phys_bytes + kTailBytes;
}

// Once per device: the kernel's dynamic shared-memory limit.
template <int HD>
cudaError_t prepare(int dev) {
  static std::atomic<uint64_t> ready{0};
  const uint64_t bit = 1ull << (dev & 63);
  if (ready.load() & bit) return cudaSuccess;
  int max_optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(prefix_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           max_optin);
  if (e != cudaSuccess) return e;
  ready.fetch_or(bit);
  return cudaSuccess;
}

template <int HD>
cudaError_t launch(const DecodeParams& p, const PrefixParams& pp, bool behind, cudaStream_t st) {
  const int smem = smem_bytes<HD>(pp);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = prepare<HD>(dev);
  if (e != cudaSuccess) return e;
  const int G = p.group;
  const int spc = kTcRows / G;
  const int rows_box = p.block_size < kTcTok ? p.block_size : kTcTok;
  const uint64_t cache_rows = (uint64_t)p.num_blocks * p.block_size;
  CUtensorMap tq, tk, tv, to;
  e = bf16_map(&tq, p.q, HD, p.num_q_heads, p.num_seqs, (uint32_t)G, (uint32_t)spc);
  if (e == cudaSuccess)
    e = bf16_map(&tk, p.k_cache, HD, p.num_kv_heads, cache_rows, 1u, (uint32_t)rows_box);
  if (e == cudaSuccess)
    e = bf16_map(&tv, p.v_cache, HD, p.num_kv_heads, cache_rows, 1u, (uint32_t)rows_box);
  if (e == cudaSuccess)
    e = ws_map(&to, p.ws_o, HD, p.ws_slots, p.num_q_heads, p.num_seqs, (uint32_t)G, (uint32_t)spc);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.num_kv_heads, pp.prefix_splits, (p.num_seqs + spc - 1) / spc);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = behind ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, prefix_kernel<HD>, p, pp, tq, tk, tv, to);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int prefix_row_groups(int num_seqs, int group) {
  const int spc = kTcRows / group;
  return (num_seqs + spc - 1) / spc;
}

cudaError_t launch_prefix(const DecodeParams& p, const PrefixParams& pp, int head_dim,
                          bool behind_decode, cudaStream_t st) {
  if (head_dim == 128) return launch<128>(p, pp, behind_decode, st);
  return launch<64>(p, pp, behind_decode, st);
}

}  // namespace pkv
