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

// packed_zeros: the entry point reads AWQ_FLAG_PACKED_ZEROS zero points
// (the others reject the flag).
inline awq_status_t check_cfg(awq_qconfig_t cfg, bool packed_zeros = false) {
  if (cfg.group_size != kGroup) return AWQ_ERR_UNSUPPORTED;
  if (cfg.zero_point != 0 && cfg.zero_point != 1) return AWQ_ERR_UNSUPPORTED;
  const uint32_t known = AWQ_FLAG_WEIGHTS_STATIC | AWQ_FLAG_SILU_MUL | (packed_zeros ? AWQ_FLAG_PACKED_ZEROS : 0u);
  if (cfg.flags & ~known) return AWQ_ERR_UNSUPPORTED;
  if ((cfg.flags & AWQ_FLAG_PACKED_ZEROS) && !cfg.zero_point) return AWQ_ERR_UNSUPPORTED;
  return AWQ_OK;
}

// 0 symmetric, 1 fp16 zero points, 2 packed zero points (after check_cfg).
inline int zero_mode(awq_qconfig_t cfg) {
  return cfg.zero_point ? ((cfg.flags & AWQ_FLAG_PACKED_ZEROS) ? 2 : 1) : 0;
}

// Group quantization parameters, one warp per (row, group), four weights per
// lane in any lane order ("AutoAWQ" code tour, "The Quantization Flow Up
// Close": each group is rounded against its scale and zero point). IEEE fp32
// with explicit round-to-nearest intrinsics, so the bits do not depend on
// contraction flags:
//   asymmetric: s = fp16(max((max w - min w) / 15, 1e-5)), z = clamp(-rint(min w / s), 0, 15)
//   symmetric:  s = fp16(max(max|w| / 7, 1e-5)), z = 8
// sf is the fp32 value of the fp16 scale.
template <bool ZP>
__device__ __forceinline__ void group_quant_params(const float (&w)[4], float& sf, float& zf) {
  if (ZP) {
    float mx = fmaxf(fmaxf(w[0], w[1]), fmaxf(w[2], w[3]));
    float mn = fminf(fminf(w[0], w[1]), fminf(w[2], w[3]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    const float s32 = fmaxf(__fdiv_rn(__fsub_rn(mx, mn), 15.0f), 1e-5f);
    sf = __half2float(__float2half_rn(s32));
    zf = fminf(fmaxf(-rintf(__fdiv_rn(mn, sf)), 0.0f), 15.0f);
  } else {
    float a = fmaxf(fmaxf(fabsf(w[0]), fabsf(w[1])), fmaxf(fabsf(w[2]), fabsf(w[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const float s32 = fmaxf(__fdiv_rn(a, 7.0f), 1e-5f);
    sf = __half2float(__float2half_rn(s32));
    zf = 8.0f;
  }
}

// The code of one weight under (sf, zf): clamp(rint(w / s) + z, 0, 15)
// (symmetric: clamp(rint(w / s), -8, 7) + 8, the same value with z = 8).
template <bool ZP>
__device__ __forceinline__ int group_quant_code(float w, float sf, float zf) {
  if (ZP) return int(fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(w, sf)), zf), 0.0f), 15.0f));
  return int(fminf(fmaxf(rintf(__fdiv_rn(w, sf)), -8.0f), 7.0f)) + 8;
}

// SiLU in fp32 for the fused gate/up epilogues: v / (1 + e^-v) with the
// fast exponential and division intrinsics (relative error a few fp32 ulp,
// far below the fp16 rounding of the output; large negative v gives 0, NaN
// stays NaN). The exact library forms cost tens of instructions and enough
// registers to spill the GEMM's epilogue warps.
__device__ __forceinline__ float silu_f32(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

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

// Codes of one packed word as four fp16 pairs without the zero point: the
// pairs (0,1) and (4,5) come out as 1024 + q, the pairs (2,3) and (6,7) as
// 64 + q (same masks and magic numbers as decode_word_qz). The offsets are
// removed later in fp32, once per group, by the caller.
__device__ __forceinline__ void decode_word_magic(uint32_t w, uint32_t (&p)[4]) {
  const uint32_t w8 = w >> 8;
  p[0] = lop3_and_or(w, 0x000F000Fu, 0x64006400u);
  p[1] = lop3_and_or(w, 0x00F000F0u, 0x54005400u);
  p[2] = lop3_and_or(w8, 0x000F000Fu, 0x64006400u);
  p[3] = lop3_and_or(w8, 0x00F000F0u, 0x54005400u);
}

// (1024 + z) and (64 + z) in both fp16 halves for an integer zero point z.
__device__ __forceinline__ void zero_bias_pairs(float z, uint32_t& zb1024, uint32_t& zb64) {
  const uint32_t a = __half_as_ushort(__float2half_rn(1024.0f + z));
  const uint32_t b = __half_as_ushort(__float2half_rn(64.0f + z));
  zb1024 = a | (a << 16);
  zb64 = b | (b << 16);
}

// ---------------------------------------------------------------------------
// mbarrier / TMA wrappers (PTX ISA: mbarrier, cp.async.bulk(.tensor))
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s for any single wait

// Wait for the phase of `parity` to complete. Gives up (returns false) when
// *abort is set by another thread or the wait passes kWaitLimitNs, in which
// case it sets *abort and ORs `err_bit` into *err.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort,
                                             uint32_t* err, uint32_t err_bit) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0) {
      if (*abort) return false;
      if (now_ns() - t0 > kWaitLimitNs) {
        *abort = 1;
        atomicOr(err, err_bit);
        return false;
      }
    }
  }
}

// Bounded wait with no abort protocol (teardown of copies already issued).
__device__ __forceinline__ void wait_teardown(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = now_ns();
  while (!mbar_try_wait(bar, parity) && now_ns() - t0 < kWaitLimitNs) {
  }
}

// mbarrier.try_wait with a suspend-time hint: a thread whose phase is not yet
// complete sleeps until it completes (or the 1 ms hint runs out) instead of
// re-polling, so waiting warps do not take issue slots from the warps that
// share their scheduler.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}

// wait_bounded built on the sleeping try_wait (same limit, abort flag and
// error bit).
__device__ __forceinline__ bool wait_sleep(uint64_t* bar, uint32_t parity, volatile int* abort,
                                           uint32_t* err, uint32_t err_bit) {
  if (mbar_try_wait_sleep(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if (*abort) return false;
    if (now_ns() - t0 > kWaitLimitNs) {
      *abort = 1;
      atomicOr(err, err_bit);
      return false;
    }
  }
}

__device__ __forceinline__ void wait_sleep_teardown(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = now_ns();
  while (!mbar_try_wait_sleep(bar, parity) && now_ns() - t0 < kWaitLimitNs) {
  }
}

// 2-D tiled TMA load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tensor_map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tensor_map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 3-D tiled TMA load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tensor_map, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tensor_map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// 4-D tiled TMA load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_4d(void* dst, const void* tensor_map, int x, int y, int z, int w,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tensor_map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
      : "memory");
}

// Prefetch one 3-D box of a tensor from global memory into L2.
__device__ __forceinline__ void tma_prefetch_l2_3d(const void* tensor_map, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(tensor_map)),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}

// Prefetch one 2-D box of a tensor from global memory into L2 (no data
// reaches shared memory; no barrier is involved).
__device__ __forceinline__ void tma_prefetch_l2_2d(const void* tensor_map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(tensor_map)),
               "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace awq
