// Device helpers shared by the pkv kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pkv.h"

namespace pkv {

constexpr int kWarp = 32;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global->shared copy that bypasses L1; src_bytes = 0 zero-fills the
// destination without reading the source.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

// Returns `addr`, computed from `dep` inside an asm block: a copy whose
// destination is derived from the result cannot issue before the instructions
// producing `dep` have their inputs (used to refill a stage only after every
// ldmatrix that read it has returned its data).  Applied once to a stage's
// base address, it orders every copy into that stage.
__device__ __forceinline__ uint32_t after_dep(uint32_t addr, uint32_t dep) {
  uint32_t r;
  asm volatile("{\n .reg .b32 z;\n and.b32 z, %2, 0;\n add.u32 %0, z, %1;\n}\n"
               : "=r"(r)
               : "r"(addr), "r"(dep));
  return r;
}

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                            uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Transpose of one 8x8 matrix of 16-bit elements held in the standard
// fragment layout (thread i: row i/4, columns 2*(i%4), 2*(i%4)+1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// D = A * B + D, m16n8k16, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A * B + D, m16n8k32, signed 8-bit A and B, 32-bit integer accumulate.
__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Round-to-nearest-even packs of two fp32 values (lo in bits 0..15).
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t v) {
  return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}
__device__ __forceinline__ float2 unpack_f16(uint32_t v) {
  __half2 h = *reinterpret_cast<__half2*>(&v);
  return __half22float2(h);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Two bytes of `biased` (each b + 128) -> two exact fp16 values b + 1152
// (0x64uu is 1024 + u).  The caller removes the constant 1152 analytically.
template <uint32_t SEL>
__device__ __forceinline__ uint32_t i8pair_to_f16x2_biased(uint32_t biased) {
  return prmt(biased, 0x64646464u, SEL);
}

// Two E4M3 codes -> two exact fp16 values (every E4M3 value is an fp16 value).
// SEL (prmt selector) puts the first code's byte in bits 0-7 and the second's
// in bits 8-15; the first lands in the low half of the result.
template <uint32_t SEL>
__device__ __forceinline__ uint32_t e4m3pair_to_f16x2(uint32_t x) {
  const uint32_t pair = prmt(x, 0u, SEL);
  uint32_t r;
  asm("{\n .reg .b16 t;\n cvt.u16.u32 t, %1;\n cvt.rn.f16x2.e4m3x2 %0, t;\n}\n"
      : "=r"(r)
      : "r"(pair));
  return r;
}

// The E4M3 codes in the low (LO) or high half of x -> two exact fp16 values,
// the lower byte in the low half of the result.
template <bool LO>
__device__ __forceinline__ uint32_t e4m3half_to_f16x2(uint32_t x) {
  uint32_t r;
  if constexpr (LO)
    asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %1;\n cvt.rn.f16x2.e4m3x2 %0, lo;\n}\n"
        : "=r"(r)
        : "r"(x));
  else
    asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %1;\n cvt.rn.f16x2.e4m3x2 %0, hi;\n}\n"
        : "=r"(r)
        : "r"(x));
  return r;
}

// Two fp32 values -> two E4M3 codes (round to nearest even, saturated to
// +-448); `lo` lands in bits 0-7.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;\n" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Row quantisers of the cache append rule, for one warp per (token, head) row:
// lane l holds the row's elements E*l .. E*l+E-1 (E = head_dim / 32) as fp32.
// Both return the lane's codes packed into the low 8*E bits (first element in
// the lowest byte) and leave the row's scale in *scale.
// INT8 (the mlqm page, §4 quantize_tensor): scale = 127 / max|x| over the row,
// code = clamp(rint(x * scale), -128, 127), division and product correctly
// rounded and unfused; an all-zero row gives codes 0 and scale 1.
template <int E>
__device__ __forceinline__ uint32_t quant_row_int8(const float (&x)[E], float* scale) {
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float s = (amax > 0.f) ? __fdiv_rn(127.0f, amax) : 1.0f;
  uint32_t packed = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    float r = rintf(__fmul_rn(x[e], s));
    r = fminf(fmaxf(r, -128.f), 127.f);
    const int qv = (amax > 0.f) ? (int)r : 0;
    packed |= (uint32_t)(qv & 0xff) << (8 * e);
  }
  *scale = s;
  return packed;
}

// FP8 (E4M3) form of the same rule: scale = 448 / max|x|, codes E4M3(x * scale)
// rounded to nearest even and saturated; an all-zero row gives codes 0, scale 1.
template <int E>
__device__ __forceinline__ uint32_t quant_row_fp8(const float (&x)[E], float* scale) {
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float s = (amax > 0.f) ? __fdiv_rn(448.0f, amax) : 1.0f;
  uint32_t packed = 0;
  if (amax > 0.f) {
#pragma unroll
    for (int e = 0; e < E; e += 2)
      packed |= f32x2_to_e4m3x2(__fmul_rn(x[e], s), __fmul_rn(x[e + 1], s)) << (8 * e);
  }
  *scale = s;
  return packed;
}

__device__ __forceinline__ float fast_rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Programmatic dependent launch (PDL).  A kernel whose successor may start
// early signals it with launch_dependents; the successor, launched with
// programmatic stream serialization, calls wait before it touches anything
// the predecessor wrote (it returns once the predecessor grid has completed
// and its memory is visible).  Both are no-ops without such a launch.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void set_flag(int* err, int bit) {
  if (err) atomicOr(err, bit);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Smem index of the 16-byte chunk `ch` of tile row `row` (rows of CH chunks).
// XOR-swizzle so that the 8 rows an ldmatrix phase reads hit 8 distinct bank
// groups.
template <int CH>
__device__ __forceinline__ int swz(int row, int ch) {
  if constexpr (CH >= 8) {
    return row * CH + (ch ^ (row & 7));
  } else {
    static_assert(CH == 4, "rows of 4 or a multiple of 8 chunks");
    return row * CH + (ch ^ ((row >> 1) & 3));
  }
}

}  // namespace pkv
