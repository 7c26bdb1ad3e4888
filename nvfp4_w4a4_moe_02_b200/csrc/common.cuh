// Device-side building blocks of the NVFP4 W4A4 + RAC library (sm_100a).
//
// NVFP4 = E2M1 element codes, one E4M3 scale per 16 elements, one FP32 tensor scale
// ("QUADS ..." Abstract: fine-grained scaling + native W4A4 FP4 GEMMs; "Why 4-bit RL
// rollout collapses ..." The failure mode: 8 E2M1 magnitudes per sign).  The block
// quantiser below is the single routine behind activation quantisation, the residual
// pass, the rollout weight pack and the trainer fake-quant (the shared QDQ path).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4 {

enum : int32_t {
  kOk = 0,
  kErrInvalid = 1,
  kErrShape = 2,
  kErrAlign = 3,
  kErrRange = 4,
  kErrCuda = 5,
  kErrTimeout = 6,
};

// 6 * 448: largest E2M1 magnitude times largest E4M3 scale.
constexpr float kScaleDenom = 2688.0f;

__device__ __forceinline__ void report_status(int32_t* st, int32_t code) {
  if (st != nullptr) atomicCAS(st, 0, code);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// ----------------------------------------------------------------------------------------
// codecs (hardware conversions, round-to-nearest-even with saturation to the largest finite)
// ----------------------------------------------------------------------------------------

// Eight floats -> eight E2M1 codes in one 32-bit word, element i in nibble i.
__device__ __forceinline__ uint32_t e2m1_encode8(const float v[8]) {
  uint32_t out;
  asm("{\n\t"
      ".reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t"
      "}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

// Two E2M1 codes (one byte, zero-extended in a 32-bit register) -> two exact halves, the low
// nibble into the low half; a negative zero code gives -0.  The byte is narrowed inside the asm
// block, so the conversion sees exactly the byte (fed with bytes unpacked from a word by a
// vector move it returned wrong values).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.u8.u32 t, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(r)
      : "r"(byte));
  return r;
}

// Eight E2M1 codes (nibble i = element i) -> their values, exact (halves widen exactly).
__device__ __forceinline__ void e2m1_decode8(uint32_t codes, float out[8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t h = e2m1x2_to_f16x2((codes >> (8 * i)) & 0xFFu);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}

// Non-negative float -> E4M3 code (RNE, saturating at 448).
__device__ __forceinline__ uint32_t e4m3_encode(float raw) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(raw));
  return r & 0xFFu;
}

// E4M3 code -> value, exact.
__device__ __forceinline__ float e4m3_decode(uint32_t code) {
  uint32_t h;
  uint16_t c = (uint16_t)code;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(c));
  return __low2float(*reinterpret_cast<__half2*>(&h));
}

// ----------------------------------------------------------------------------------------
// the block quantiser (binary32, explicit round-to-nearest operations, no contraction)
// ----------------------------------------------------------------------------------------
struct BlockScale {
  uint32_t S;   // E4M3 code
  float d;      // S * s_g
  float inv;    // 1 / d  (unused when S == 0)
};

// b: max |x| over the 16-block; t6 = RN(6 * s_g); s_g == 0 -> S = 0.
__device__ __forceinline__ BlockScale block_scale(float b, float s_g, float t6) {
  BlockScale bs;
  bs.S = 0;
  if (s_g > 0.0f) bs.S = e4m3_encode(__fdiv_rn(b, t6));
  bs.d = __fmul_rn(e4m3_decode(bs.S), s_g);
  bs.inv = (bs.S != 0) ? __frcp_rn(bs.d) : 0.0f;
  return bs;
}

// Quantise 8 elements of a block: codes (nibble i = element i) and dequantised values.
__device__ __forceinline__ uint32_t quant8(const float x[8], const BlockScale& bs, float dq[8]) {
  if (bs.S == 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) dq[i] = 0.0f;
    return 0u;
  }
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 p = __fmul2_rn(make_float2(x[i], x[i + 1]), make_float2(bs.inv, bs.inv));
    v[i] = p.x;
    v[i + 1] = p.y;
  }
  uint32_t c = e2m1_encode8(v);
  float e[8];
  e2m1_decode8(c, e);
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 p = __fmul2_rn(make_float2(e[i], e[i + 1]), make_float2(bs.d, bs.d));
    dq[i] = p.x;
    dq[i + 1] = p.y;
  }
  return c;
}

__device__ __forceinline__ uint32_t quant8_codes(const float x[8], const BlockScale& bs) {
  if (bs.S == 0) return 0u;
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 p = __fmul2_rn(make_float2(x[i], x[i + 1]), make_float2(bs.inv, bs.inv));
    v[i] = p.x;
    v[i + 1] = p.y;
  }
  return e2m1_encode8(v);
}

// s_g from amax, with the range contract (nonzero amax within [2^-100, 2^100], finite).
__device__ __forceinline__ float scale_from_amax(float amax, int32_t* status) {
  if (!(amax <= 1.2676506e30f) || (amax > 0.0f && amax < 7.888609e-31f)) {
    report_status(status, kErrRange);
  }
  return __fdiv_rn(amax, kScaleDenom);
}

// Byte offset of the scale of (row, 16-column block kb) inside a scale-atom array whose
// rows hold `k64` groups of 64 columns.
__device__ __forceinline__ int64_t sf_offset(int64_t row, int64_t kb, int64_t k64) {
  return ((row >> 7) * k64 + (kb >> 2)) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4 + (kb & 3);
}
// The same for the 16-row slab layout of decode activations: slab row / 16 owns one atom per 64
// columns and uses its first 16 atom rows (row % 16 at i = 0).
__device__ __forceinline__ int64_t sf_offset_slab16(int64_t row, int64_t kb, int64_t k64) {
  return ((row >> 4) * k64 + (kb >> 2)) * 512 + (row & 15) * 16 + (kb & 3);
}
__device__ __forceinline__ int64_t sf_offset_any(int64_t row, int64_t kb, int64_t k64, bool slab16) {
  return slab16 ? sf_offset_slab16(row, kb, k64) : sf_offset(row, kb, k64);
}

// ----------------------------------------------------------------------------------------
// warp reductions
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

}  // namespace nvfp4
