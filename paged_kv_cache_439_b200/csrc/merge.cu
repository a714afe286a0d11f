// Split merge of paged decode attention (sm_100a): combines the normalised
// partials (o_k, log2-sum-exp_k) that the split decode kernels and the
// shared-prefix pass write into the workspace, out = sum_k 2^{lse_k} o_k /
// sum_k 2^{lse_k}.  Split-K is not on the pages; the merge is its exact
// combination step.
#include "common.cuh"
#include "decode.cuh"
#include "decode_common.cuh"

namespace pkv {

namespace {

// Split merge: out = sum_k 2^{lse_k} o_k / sum_k 2^{lse_k} over the partials
// of one (sequence, q head): the shared-prefix slots [0, ws_base) and the
// splits that hold tokens (every one of them was written, so all are finite).
// One warp per (q head, sequence); lane l sums head_dim columns 4l..4l+3 of the
// weighted partials with 16-byte loads.  The first kMergeBatch partial rows are
// loaded before the weights are known, so their latency overlaps the
// log-sum-exp reads (with up to 16 partials, one memory round trip in all);
// the weights are held one per lane and broadcast with shuffles, 32 slots per
// round.
constexpr int kMergeWarps = 4;

template <int HD>
__global__ void __launch_bounds__(kMergeWarps* kWarp) merge_kernel(const DecodeParams p) {
  pdl_wait();  // the decode grid's partials are complete and visible past this point
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int qh = blockIdx.x * kMergeWarps + warp, seq = blockIdx.y;
  if (qh >= p.num_q_heads) return;
  const int ctx = effective_ctx(p, seq, false);
  const int rest = ctx > p.t_start ? ctx - p.t_start : 0;
  const int n = p.ws_base + (rest + p.chunk - 1) / p.chunk;
  const size_t r = ((size_t)seq * p.num_q_heads + qh) * p.ws_slots;
  const bool cols = lane * 4 < HD;
  const float4* src = reinterpret_cast<const float4*>(p.ws_o + r * HD) + lane;
  constexpr int kRow = HD / 4;  // float4 per partial row

  float4 v[kMergeBatch];
#pragma unroll
  for (int i = 0; i < kMergeBatch; ++i)
    if (cols && i < n) v[i] = src[(size_t)i * kRow];
  float M = -CUDART_INF_F;
  for (int k = lane; k < n; k += kWarp) M = fmaxf(M, p.ws_lse[r + k]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float L = 0.f;
  if (M != -CUDART_INF_F) {
    for (int base = 0; base < n; base += kWarp) {
      const int cnt = min(n - base, kWarp);
      const float lse = lane < cnt ? p.ws_lse[r + base + lane] : -CUDART_INF_F;
      const float w = lse == -CUDART_INF_F ? 0.f : exp2f(lse - M);
      float ws = w;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, off);
      L += ws;
      for (int k0 = 0; k0 < cnt; k0 += kMergeBatch) {
        if (base + k0 >= kMergeBatch) {  // the first batch is already in registers
#pragma unroll
          for (int i = 0; i < kMergeBatch; ++i)
            if (cols && k0 + i < cnt) v[i] = src[(size_t)(base + k0 + i) * kRow];
        }
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i) {
          const float wk = __shfl_sync(0xffffffffu, w, (k0 + i) & (kWarp - 1));
          if (k0 + i < cnt) {
            acc[0] += wk * v[i].x;
            acc[1] += wk * v[i].y;
            acc[2] += wk * v[i].z;
            acc[3] += wk * v[i].w;
          }
        }
      }
    }
  }
  if (!cols) return;
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const size_t o = ((size_t)seq * p.num_q_heads + qh) * HD + lane * 4;
  if (p.out_f32) {
    *reinterpret_cast<float4*>(static_cast<float*>(p.out) + o) =
        make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  } else {
    __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(p.out) + o;
    *reinterpret_cast<uint2*>(ob) =
        make_uint2(pack_bf16(acc[0] * inv, acc[1] * inv), pack_bf16(acc[2] * inv, acc[3] * inv));
  }
}

}  // namespace

// The merge is launched with programmatic stream serialization: its CTAs
// may become resident while the decode grid's last CTAs run (every decode CTA
// signals at its start), and each waits in pdl_wait for the decode grid to
// complete, so the launch latency hides behind the decode's tail.
cudaError_t launch_merge(const DecodeParams& p, int head_dim, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.num_q_heads + kMergeWarps - 1) / kMergeWarps, p.num_seqs);
  cfg.blockDim = dim3(kMergeWarps * kWarp);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = head_dim == 128 ? cudaLaunchKernelEx(&cfg, merge_kernel<128>, p)
                                  : cudaLaunchKernelEx(&cfg, merge_kernel<64>, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pkv
