// Device helpers shared by the sm_100a kernels of the bf16 x NVFP4 library.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "fi_nvfp4.h"

namespace fi {

// ------------------------------------------------------------------ global loads

// 16-byte streaming load through the non-coherent path, not kept in L1, with a 256-byte
// L2 prefetch hint: the weights are read exactly once per call.
__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ldg_stream_u16(const void* p) {
  unsigned short v;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ldg_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ldg_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ------------------------------------------------------------ format conversions

// Two E2M1 codes (one byte: low nibble = element 2j, high nibble = element 2j+1) to an
// f16x2 whose low half is element 2j. Exact: every E2M1 value is an f16.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte_in_low8) {
  uint32_t h;
  asm("{\n .reg .b8 b;\n cvt.u8.u32 b, %1;\n cvt.rn.f16x2.e2m1x2 %0, b;\n}"
      : "=r"(h)
      : "r"(byte_in_low8));
  return h;
}

// Byte `i` (0..3) of a 32-bit word as an f16x2 of its two E2M1 codes.
template <int I>
__device__ __forceinline__ uint32_t e2m1x2_byte_to_f16x2(uint32_t w) {
  uint32_t h;
  if constexpr (I == 0) {
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %1;\n cvt.rn.f16x2.e2m1x2 %0, b0;\n}" : "=r"(h) : "r"(w));
  } else if constexpr (I == 1) {
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %1;\n cvt.rn.f16x2.e2m1x2 %0, b1;\n}" : "=r"(h) : "r"(w));
  } else if constexpr (I == 2) {
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %1;\n cvt.rn.f16x2.e2m1x2 %0, b2;\n}" : "=r"(h) : "r"(w));
  } else {
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %1;\n cvt.rn.f16x2.e2m1x2 %0, b3;\n}" : "=r"(h) : "r"(w));
  }
  return h;
}

// Two E4M3 codes (low 16 bits: low byte = first) to f16x2 (low half = first). Exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
  uint32_t h;
  asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %1;\n cvt.rn.f16x2.e4m3x2 %0, lo;\n}"
      : "=r"(h)
      : "r"(two_bytes));
  return h;
}

__device__ __forceinline__ float f16_lo_to_f32(uint32_t h2) {
  float f;
  asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %1;\n cvt.f32.f16 %0, lo;\n}" : "=f"(f) : "r"(h2));
  return f;
}

__device__ __forceinline__ float f16_hi_to_f32(uint32_t h2) {
  float f;
  asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %1;\n cvt.f32.f16 %0, hi;\n}" : "=f"(f) : "r"(h2));
  return f;
}

// fp32 pair -> E2M1x2 byte, round to nearest even, saturating; `lo` lands in bits 0-3.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n .reg .b8 b;\n cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n cvt.u32.u8 %0, b;\n}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r & 0xFFu;
}

// fp32 -> E4M3 code, round to nearest even, saturating to +-448.
__device__ __forceinline__ uint32_t f32_to_e4m3(float x) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return (uint32_t)r & 0xFFu;
}

// f32 pair -> f16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ------------------------------------------------------------------- output rounding

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float x) {
  unsigned short r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

// fp32 -> IEEE binary16 bits, round to nearest even (the optional f16 output).
__device__ __forceinline__ uint16_t f32_to_f16_rn(float x) {
  unsigned short r;
  asm("cvt.rn.f16.f32 %0, %1;" : "=h"(r) : "f"(x));
  return r;
}

// The output element's bits: bf16 (f16 == false) or f16, round to nearest even.
__device__ __forceinline__ uint16_t f32_to_out(float x, bool f16) { return f16 ? f32_to_f16_rn(x) : f32_to_bf16_rn(x); }

// ---------------------------------------------------- programmatic dependent launch

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace fi
