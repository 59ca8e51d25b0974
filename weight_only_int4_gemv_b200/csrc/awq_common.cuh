// Shared device helpers and host-side validation for libawq_b200.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "awq.h"

namespace awq {

constexpr int kGroup = 128;          // weights per (row, group); the only group size built
constexpr int kWordsPerGroup = kGroup / 8;

// ---------------------------------------------------------------------------
// host-side argument checks (no CUDA calls)
// ---------------------------------------------------------------------------
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline awq_status_t check_cfg(awq_qconfig_t cfg) {
  if (cfg.group_size != kGroup) return AWQ_ERR_UNSUPPORTED;
  if (cfg.zero_point != 0 && cfg.zero_point != 1) return AWQ_ERR_UNSUPPORTED;
  return AWQ_OK;
}

// K must hold whole groups; N >= 0. Sizes are bounded so that every row
// offset fits comfortably in 64 bits and every per-row count in 32 bits.
inline awq_status_t check_nk(int64_t N, int64_t K) {
  if (N < 0 || K <= 0) return AWQ_ERR_SHAPE;
  if (K % kGroup) return AWQ_ERR_SHAPE;
  if (N > (int64_t(1) << 31) - 1 || K > (int64_t(1) << 30)) return AWQ_ERR_SHAPE;
  return AWQ_OK;
}

inline awq_status_t launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {
  // (a & b) | c
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Streaming 16-byte load that does not allocate in L1 (packed codes are read once).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Read-only 16-byte load through L1 (activations are shared by many warps).
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint16_t ld_nc_u16(const uint16_t* p) {
  uint16_t v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ float half_bits_to_float(uint16_t b) {
  return __half2float(__ushort_as_half(b));
}

// Codes of one packed word as four fp16 pairs (q - z) for the consecutive k
// pairs (0,1), (2,3), (4,5), (6,7) of the word.
//
// Nibble slot i holds k offset {0,2,4,6,1,3,5,7}[i], so the pair (2j, 2j+1)
// sits in slots j (low half) and 4+j (high half). OR-ing a 4-bit field into
// the mantissa of an fp16 power of two gives an exact small integer:
//   0x6400 | q        = 1024 + q      (fp16 ulp 1 at 1024)
//   0x5400 | (q << 4) = 64 + q        (fp16 ulp 1/16 at 64)
// and subtracting 1024 + z or 64 + z (exact in fp16) leaves q - z exactly.
// zb1024 = (1024 + z) in both halves, zb64 = (64 + z) in both halves.
__device__ __forceinline__ void decode_word_qz(uint32_t w, uint32_t zb1024, uint32_t zb64,
                                               uint32_t (&p)[4]) {
  const uint32_t w8 = w >> 8;
  p[0] = hsub2_u32(lop3_and_or(w, 0x000F000Fu, 0x64006400u), zb1024);
  p[1] = hsub2_u32(lop3_and_or(w, 0x00F000F0u, 0x54005400u), zb64);
  p[2] = hsub2_u32(lop3_and_or(w8, 0x000F000Fu, 0x64006400u), zb1024);
  p[3] = hsub2_u32(lop3_and_or(w8, 0x00F000F0u, 0x54005400u), zb64);
}

// (1024 + z) and (64 + z) in both fp16 halves for an integer zero point z.
__device__ __forceinline__ void zero_bias_pairs(float z, uint32_t& zb1024, uint32_t& zb64) {
  const uint32_t a = __half_as_ushort(__float2half_rn(1024.0f + z));
  const uint32_t b = __half_as_ushort(__float2half_rn(64.0f + z));
  zb1024 = a | (a << 16);
  zb64 = b | (b << 16);
}

}  // namespace awq
