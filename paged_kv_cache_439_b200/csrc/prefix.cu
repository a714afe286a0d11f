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
// The rows of one KV head form a dense contraction, so one CTA takes 128 rows
// (the M of one tcgen05.mma) and walks its slice in 64-token tiles:
//   S = Q K^T      tcgen05.mma, A = Q and B = K from shared memory (K-major,
//                  128-byte swizzle), D = S in tensor memory (128 lanes x 64
//                  fp32 columns);
//   softmax        thread r owns row r: tcgen05.ld of its 64 scores, fp32
//                  online softmax, P written back to tensor memory as bf16
//                  hi + lo halves (about 16 significant bits of P);
//   O += P V       tcgen05.mma with A = P from tensor memory and B = V from
//                  shared memory (head_dim-major), D = O in tensor memory.
// The running maximum is only moved when a tile's maximum exceeds it by more
// than 2^8 (then O is rescaled in tensor memory): exponentials stay below 256,
// and the final normalisation uses the same maximum as every P, so the result
// is the same softmax.  One thread issues the MMAs; tcgen05.commit arrives on
// an mbarrier the other threads wait on, each wait bounded.  K and V tiles are
// gathered from the paged blocks with cp.async into two-stage rings of their
// own: K tile j + 2 is fetched as soon as S of tile j is in tensor memory, V
// tile j + 1 as soon as P V of tile j - 1 is done, so every copy has a whole
// tile of work to land behind.  Two CTAs share an SM (half of its tensor
// memory each), so one CTA's softmax overlaps the other's MMAs.
#include <math_constants.h>

#include <atomic>

#include "common.cuh"
#include "decode.cuh"

namespace pkv {

namespace {

constexpr int kTcThreads = 128;  // one thread per row; warp w reads TMEM lanes 32w..32w+31
constexpr int kTcRows = 128;     // rows per CTA (MMA M)
constexpr int kTcTok = kPrefixTokens;  // tokens per tile (MMA N of Q K^T)
constexpr int kTcStages = 2;
constexpr float kRescaleLog2 = 8.f;  // move the running max only past 2^8
constexpr uint64_t kWaitNs = 2000000000ull;  // a wait gives up after 2 s

static_assert(kTcTok == 64, "the score row is read as two 32-column loads");

template <int HD>
struct TcCfg {
  static constexpr int DB = HD / 64;                      // 128-byte column blocks of head_dim
  static constexpr int Q_DB = kTcRows * 128;              // bytes of one Q column block
  static constexpr int KV_DB = kTcTok * 128;              // bytes of one K (or V) column block
  static constexpr int Q_BYTES = DB * Q_DB;
  static constexpr int KV_BYTES = DB * KV_DB;            // one K (or V) tile
  static constexpr int S_COL = 0;                         // tensor-memory columns
  static constexpr int PH_COL = kTcTok;                   // P hi: 2 bf16 per column
  static constexpr int PL_COL = kTcTok + kTcTok / 2;      // P lo
  static constexpr int O_COL = 2 * kTcTok;
  static constexpr int COLS_USED = O_COL + HD;
  static constexpr int TMEM_COLS = COLS_USED <= 128 ? 128 : (COLS_USED <= 256 ? 256 : 512);
  // dynamic shared memory: 1 KB alignment slack, Q, the stages, then the
  // block-table slice, two mbarriers and the tensor-memory address
  static constexpr int BODY = Q_BYTES + 2 * kTcStages * KV_BYTES;
  static_assert(HD == 64 || HD == 128, "head_dim 64 or 128");
};

// 128-byte swizzle: 16-byte chunk c of the 128-byte row r of a 1024-byte
// aligned atom lives at chunk c ^ (r & 7).
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

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
    else if ((i & 63) == 0 && global_ns() - t0 > kWaitNs) return false;
  }
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

template <int HD>
__global__ void __launch_bounds__(kTcThreads)
    prefix_kernel(const DecodeParams p, const PrefixParams pp) {
  using Cfg = TcCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // swizzle atoms need 1024-byte alignment
  uint8_t* const gbase = smem_raw + (base - raw);
  const uint32_t q_sm = base;
  const uint32_t k_ring = base + Cfg::Q_BYTES;
  const uint32_t v_ring = k_ring + kTcStages * Cfg::KV_BYTES;
  int* const s_phys = reinterpret_cast<int*>(gbase + Cfg::BODY);
  uint8_t* const tail = gbase + Cfg::BODY + pp.phys_bytes;
  const uint32_t bar_s = smem_u32(tail);       // S of a tile is in tensor memory
  const uint32_t bar_o = smem_u32(tail + 8);   // a tile's P V has been accumulated
  volatile uint32_t* const s_tmem = reinterpret_cast<volatile uint32_t*>(tail + 16);

  const int kvh = blockIdx.x, split = blockIdx.y, rg = blockIdx.z;
  const int tid = threadIdx.x, warp = tid / kWarp;
  const int G = p.group;
  const int t0 = split * pp.pchunk;
  const int t1 = min(pp.prefix_len, t0 + pp.pchunk);
  const int bs = p.block_size;
  const int blk0 = t0 >> p.log2_bs;

  // ---- set-up: block-table slice, barriers, tensor memory
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
  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32((const void*)s_tmem)),
                 "r"(Cfg::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }

  // ---- this thread's row
  const int row = tid;
  const int r = rg * kTcRows + row;
  const bool rvalid = r < pp.rows;
  const int seq = rvalid ? r / G : 0;
  const size_t qrow = (size_t)seq * p.num_q_heads + kvh * G + (rvalid ? r % G : 0);
  int lim = 0;  // tokens of the prefix this row attends to
  if (rvalid) {
    int ctx = p.context_lens[seq];
    ctx = ctx < 0 ? 0 : ctx;
    lim = min(ctx, pp.prefix_len);
  }

  // ---- copies: Q (once) and the K/V tiles, into the swizzled column blocks
  const uint8_t* kb = static_cast<const uint8_t*>(p.k_cache);
  const uint8_t* vb = static_cast<const uint8_t*>(p.v_cache);
  const size_t tok_stride = (size_t)p.num_kv_heads * HD * 2;
  __syncthreads();  // s_phys
  {
    const uint8_t* qb = static_cast<const uint8_t*>(p.q);
    constexpr int CH = HD / 8;  // 16-byte chunks per row
#pragma unroll 4
    for (int i = tid; i < kTcRows * CH; i += kTcThreads) {
      const int rr = i / CH, c = i % CH;
      const int gr = rg * kTcRows + rr;
      const bool ok = gr < pp.rows;
      const size_t qr = ok ? (size_t)(gr / G) * p.num_q_heads + kvh * G + gr % G : 0;
      cp_async_16(q_sm + (uint32_t)((c >> 3) * Cfg::Q_DB) + sw128(rr, c & 7),
                  qb + qr * HD * 2 + (size_t)c * 16, ok ? 16 : 0);
    }
  }
  const int ntiles = (t1 - t0 + kTcTok - 1) / kTcTok;
  // copies of K (or V) tile j into its ring stage; rows past the slice or in a
  // bad block are zero-filled
  auto copy_tile = [&](const uint8_t* src, uint32_t ring_base, int j) {
    constexpr int CH = HD / 8;
    const int tt = t0 + j * kTcTok;
    const uint32_t st = ring_base + (uint32_t)((j % kTcStages) * Cfg::KV_BYTES);
#pragma unroll 4
    for (int i = tid; i < kTcTok * CH; i += kTcThreads) {
      const int rr = i / CH, c = i % CH;
      const int t = tt + rr;
      const int phys = t < t1 ? s_phys[(t >> p.log2_bs) - blk0] : -1;
      size_t off = 0;
      int n = 0;
      if (phys >= 0) {
        off = ((size_t)phys * bs + (t & (bs - 1))) * tok_stride + (size_t)kvh * HD * 2 +
              (size_t)c * 16;
        n = 16;
      }
      cp_async_16(st + (uint32_t)((c >> 3) * Cfg::KV_DB) + sw128(rr, c & 7), src + off, n);
    }
  };
  // one commit group per call (empty past the last tile, to keep the count)
  auto issue_tile = [&](const uint8_t* src, uint32_t ring_base, int j) {
    if (j < ntiles) copy_tile(src, ring_base, j);
    cp_async_commit();
  };
  // groups in commit order: {Q, V0, K0}, {K1}, then per tile j: {K j+2}, {V j+1}
  copy_tile(vb, v_ring, 0);
  issue_tile(kb, k_ring, 0);
  issue_tile(kb, k_ring, 1);

  tc_fence_before();
  __syncthreads();  // barriers initialised, tensor-memory address written
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  constexpr uint32_t kIdQK = idesc_bf16(kTcRows, kTcTok, 0);
  constexpr uint32_t kIdPV = idesc_bf16(kTcRows, HD, 1);
  auto issue_qk = [&](int j) {  // S = Q K^T of tile j (thread 0)
    const uint32_t kS = k_ring + (uint32_t)((j % kTcStages) * Cfg::KV_BYTES);
#pragma unroll
    for (int ks = 0; ks < HD / 16; ++ks) {
      const uint32_t koff = (uint32_t)((ks >> 2) * Cfg::KV_DB + (ks & 3) * 32);
      const uint32_t qoff = (uint32_t)((ks >> 2) * Cfg::Q_DB + (ks & 3) * 32);
      mma_ss(tmem + Cfg::S_COL, smem_desc(q_sm + qoff, 16, 1024), smem_desc(kS + koff, 16, 1024),
             kIdQK, ks > 0);
    }
    mma_commit(bar_s);
  };
  auto issue_pv = [&](int j) {  // O += P V of tile j (thread 0)
    const uint32_t vS = v_ring + (uint32_t)((j % kTcStages) * Cfg::KV_BYTES);
#pragma unroll
    for (int kk = 0; kk < kTcTok / 16; ++kk) {
      const uint64_t bd = smem_desc(vS + (uint32_t)(kk * 16 * 128), Cfg::KV_DB, 1024);
      mma_ts(tmem + Cfg::O_COL, tmem + Cfg::PH_COL + kk * 8, bd, kIdPV, (j > 0 || kk > 0));
      mma_ts(tmem + Cfg::O_COL, tmem + Cfg::PL_COL + kk * 8, bd, kIdPV, 1u);
    }
    mma_commit(bar_o);
  };

  // first tile: data (and Q) landed -> visible to the tensor cores -> S_0
  cp_async_wait<1>();
  fence_async_smem();
  __syncthreads();
  if (tid == 0) {
    tc_fence_after();
    issue_qk(0);
  }

  float m_ref = -CUDART_INF_F;  // reference maximum of this row (log2 units)
  float l_run = 0.f;
  bool failed = false;
  for (int j = 0; j < ntiles; ++j) {
    const int tt = t0 + j * kTcTok;
    // ---- scores of tile j
    bool ok = mbar_wait(bar_s, (uint32_t)(j & 1));
    tc_fence_after();
    issue_tile(kb, k_ring, j + 2);  // K tile j has been consumed
    float s[kTcTok];
    {
      float a[32], b[32];
      tmem_ld32(tmem + lane_base + Cfg::S_COL, a);
      tmem_ld32(tmem + lane_base + Cfg::S_COL + 32, b);
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
    float mt = -CUDART_INF_F;
#pragma unroll
    for (int i = 0; i < kTcTok; ++i) {
      bool v = i < nval;
      if (bad) v = v && s_phys[((tt + i) >> p.log2_bs) - blk0] >= 0;
      s[i] = v ? s[i] * p.scale_log2 : -CUDART_INF_F;
      mt = fmaxf(mt, s[i]);
    }
    const bool move = mt > m_ref + kRescaleLog2;  // also true for the first valid tile
    const float m_new = move ? mt : m_ref;
    const float alpha = move ? fast_exp2(m_ref - m_new) : 1.f;  // 0 when m_ref = -inf

    // ---- the previous tile's P V must be done: P is overwritten, O may be
    // rescaled, and its V stage takes tile j + 1
    if (j > 0) {
      ok &= mbar_wait(bar_o, (uint32_t)((j - 1) & 1));
      tc_fence_after();
    }
    issue_tile(vb, v_ring, j + 1);
    // rare: rescale O in place.  tcgen05.ld/st are warp-collective, so the whole
    // warp takes this path when any of its rows needs it (alpha = 1 for the rest).
    const bool need = move && j > 0 && m_ref != -CUDART_INF_F;
    if (__any_sync(0xffffffffu, need)) {
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

    // ---- P = 2^(s - m) as bf16 hi + lo, into tensor memory
    {
      uint32_t hi[32], lo[32];
      float rs = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float x0 = fast_exp2(s[2 * i] - m_use), x1 = fast_exp2(s[2 * i + 1] - m_use);
        rs += x0 + x1;
        const uint32_t h = pack_bf16(x0, x1);
        const float2 f = unpack_bf16(h);
        hi[i] = h;
        lo[i] = pack_bf16(x0 - f.x, x1 - f.y);
      }
      l_run += rs;
      tmem_st32(tmem + lane_base + Cfg::PH_COL, hi);
      tmem_st32(tmem + lane_base + Cfg::PL_COL, lo);
      tmem_wait_st();
    }
    // ---- V tile j and K tile j + 1 landed (the two groups of this tile may still fly)
    cp_async_wait<2>();
    fence_async_smem();
    tc_fence_before();
    failed = __syncthreads_or(!ok);
    if (failed) break;
    if (tid == 0) {
      tc_fence_after();
      issue_pv(j);
      if (j + 1 < ntiles) issue_qk(j + 1);
    }
  }

  // ---- the last P V, then normalise and write this slice's partial
  if (!failed) {
    const bool ok = mbar_wait(bar_o, (uint32_t)((ntiles - 1) & 1));
    tc_fence_after();
    failed = !ok;
    const size_t slot = qrow * p.ws_slots + split;
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
    for (int c = 0; c < HD; c += 32) {
      float o[32];
      tmem_ld32(tmem + lane_base + Cfg::O_COL + c, o);
      tmem_wait_ld();
      if (rvalid && ok) {
        float4* dst = reinterpret_cast<float4*>(p.ws_o + slot * HD + c);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv,
                               o[4 * i + 3] * inv);
      }
    }
    if (rvalid && ok)
      p.ws_lse[slot] = l_run > 0.f ? m_ref + log2f(l_run) : -CUDART_INF_F;
  }
  cp_async_wait<0>();
  tc_fence_before();
  failed = __syncthreads_or(failed);
  if (failed && tid == 0) set_flag(p.err_flag, PKV_FLAG_TIMEOUT);
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(Cfg::TMEM_COLS)
                 : "memory");
  }
}

template <int HD>
int smem_bytes(const PrefixParams& pp) {
  return 1024 + TcCfg<HD>::BODY + pp.phys_bytes + 32;
}

template <int HD>
cudaError_t launch(const DecodeParams& p, const PrefixParams& pp, cudaStream_t st) {
  const int smem = smem_bytes<HD>(pp);
  auto k = prefix_kernel<HD>;
  // opt in to the largest dynamic shared memory once per device
  static std::atomic<uint64_t> ready{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(ready.load() & bit)) {
    int max_optin = 0;
    e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, max_optin);
    if (e != cudaSuccess) return e;
    ready.fetch_or(bit);
  }
  const dim3 grid(p.num_kv_heads, pp.prefix_splits, (pp.rows + kTcRows - 1) / kTcRows);
  k<<<grid, kTcThreads, smem, st>>>(p, pp);
  return cudaGetLastError();
}

}  // namespace

int prefix_rows_per_cta() { return kTcRows; }

cudaError_t launch_prefix(const DecodeParams& p, const PrefixParams& pp, int head_dim,
                          cudaStream_t st) {
  if (head_dim == 128) return launch<128>(p, pp, st);
  return launch<64>(p, pp, st);
}

}  // namespace pkv
