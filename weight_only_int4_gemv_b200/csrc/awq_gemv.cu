// W4A16 small-batch product y[M][N] = x[M][K] . W'^T, 1 <= M <= 16, for sm_100a.
//
// ("AutoAWQ" code tour, "The big picture": the GEMV kernel for single-token
// decoding; "AutoAWQ" capability page: INT4 weights are decoded inside the
// matmul and never written back as fp16.)
//
// The layer is bound by HBM: every packed code byte is read once and feeds
// only M multiply-adds, so the kernel is built around keeping enough bytes
// in flight on every SM.
//
// * Work unit = (row block of 16*RT output channels, one group of 128 k).
//   Units are ordered block-major and split evenly over every warp of a grid
//   sized to the resident capacity of the GPU (a stream-K split): all SMs
//   stream the same number of bytes whatever N and K are.
// * Each warp owns an S-stage ring in shared memory and fills it with 16-byte
//   cp.async copies S-1 units ahead of the arithmetic: the unit's packed
//   codes (lane (g, t) copies 16 bytes of rows g and g+8 of each 16-row
//   tile, the bytes it will decode itself), the 16-row runs of scales and
//   zero points (group-major metadata makes them contiguous), and the
//   unit's slice of x (128 k of every batch row, 16-byte chunks swizzled so
//   the fragment reads are free of bank conflicts).
// * Decode: the packed nibble order puts consecutive k pairs in the low and
//   high halves of a word, so one LOP3 turns a word into two fp16 values
//   1024+q (or 64+q) and one HSUB2 subtracts 1024+z (64+z), leaving q - z
//   exactly.
// * Multiply: the decoded 16x16 weight tile is the A operand of
//   mma.m16n8k16 straight from registers; x is the B operand (batch in the
//   n dimension, two n8 tiles for M > 8). The k positions inside an MMA are
//   a permutation of the word's k (each lane owns whole words), matched by
//   reading x[m][8w .. 8w+7] for the same words: one 16-byte read covers two
//   MMAs. Accumulation is fp32.
// * The scale is applied once per group: sum_k x (q - z) s = s * sum_k x (q - z).
// * A row block split between warps is finished by the last warp to arrive
//   (arrival counter per block): it sums the contributors' fp32 partials in
//   a fixed order, so results do not depend on timing, and resets the
//   counter for the next call. No warp ever waits on another.

#include <atomic>

#include "awq_common.cuh"

namespace awq {
namespace {

constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = kGemvWarps * 32;

struct GemvParams {
  const uint16_t* x;
  const int32_t* qweight;
  const uint16_t* scales;
  const uint16_t* zeros;
  uint16_t* y;
  float* partials;       // [total_warps][2][slot floats]
  uint32_t* counters;    // [nb]
  int64_t units;         // nb * G
  int M, N, K, G, nb, total_warps;
  int stage_bytes;       // codes + metadata + x slice of one unit
  int x_offset;          // offset of the x slice inside a stage
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte async copy global -> shared; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ uint16_t lds16(const uint8_t* p) { return *reinterpret_cast<const uint16_t*>(p); }

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// (1024 + z, 1024 + z) and (64 + z, 64 + z) from the fp16 bits of an
// integer zero point z in 0..15: both sums are exact in fp16.
__device__ __forceinline__ void zero_bias_from_bits(uint16_t zbits, uint32_t& zb1024, uint32_t& zb64) {
  const uint32_t zz = uint32_t(zbits) | (uint32_t(zbits) << 16);
  uint32_t a, b;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(a) : "r"(zz), "r"(0x64006400u));
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(b) : "r"(zz), "r"(0x54005400u));
  zb1024 = a;
  zb64 = b;
}

// Position of 16-byte chunk c (0..15) of batch row m inside a stage's x
// slice: spreads the 8 lanes of each quarter-warp fragment read over all
// 32 banks.
__device__ __forceinline__ int x_chunk_pos(int m, int c) { return c ^ ((c >> 3) & 1) ^ ((m & 1) << 1); }

// First unit of warp w in the even split of `units` over `warps`.
__device__ __forceinline__ int64_t warp_start(int64_t units, int64_t w, int64_t warps) {
  return units * w / warps;
}

template <int MT, int RT>
__device__ __forceinline__ void store_y(const GemvParams& p, int64_t row0, int g, int t,
                                        const float (&acc)[RT][MT][4]) {
#pragma unroll
  for (int rt = 0; rt < RT; ++rt) {
    const int64_t r_lo = row0 + 16 * rt + g;
    const int64_t r_hi = r_lo + 8;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int m0 = 8 * mt + 2 * t;
      if (m0 < p.M) {
        if (r_lo < p.N) p.y[int64_t(m0) * p.N + r_lo] = __half_as_ushort(__float2half_rn(acc[rt][mt][0]));
        if (r_hi < p.N) p.y[int64_t(m0) * p.N + r_hi] = __half_as_ushort(__float2half_rn(acc[rt][mt][2]));
      }
      if (m0 + 1 < p.M) {
        if (r_lo < p.N) p.y[int64_t(m0 + 1) * p.N + r_lo] = __half_as_ushort(__float2half_rn(acc[rt][mt][1]));
        if (r_hi < p.N) p.y[int64_t(m0 + 1) * p.N + r_hi] = __half_as_ushort(__float2half_rn(acc[rt][mt][3]));
      }
    }
  }
}

// Finish row block b after this warp summed groups [j0, j1) of it.
template <int MT, int RT>
__device__ __forceinline__ void finish_block(const GemvParams& p, int64_t b, int j0, int j1, int64_t gw,
                                             int64_t first_block, int lane, int g, int t,
                                             const float (&acc)[RT][MT][4]) {
  const int64_t row0 = b * (16 * RT);
  const int64_t G = p.G;
  if (j0 == 0 && j1 == G) {
    store_y<MT, RT>(p, row0, g, t, acc);
    return;
  }
  // Partial block: publish this warp's fp32 sums, count its groups in.
  constexpr int kSlot = RT * MT * 4 * 32;
  const int slot = (b == first_block) ? 0 : 1;
  float* sp = p.partials + (gw * 2 + slot) * kSlot;
  int idx = 0;
#pragma unroll
  for (int rt = 0; rt < RT; ++rt)
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i, ++idx) __stcg(sp + idx * 32 + lane, acc[rt][mt][i]);
  __threadfence();
  __syncwarp();
  uint32_t last = 0;
  if (lane == 0) {
    const uint32_t mine = uint32_t(j1 - j0);
    const uint32_t old = atomicAdd(p.counters + b, mine);
    last = (old + mine == uint32_t(G)) ? 1u : 0u;
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __threadfence();
  // contributors: every non-empty warp range overlapping block b, in warp order
  const int64_t W = p.total_warps;
  const int64_t w_first = ((b * G + 1) * W - 1) / p.units;
  const int64_t w_last = ((b * G + G) * W - 1) / p.units;
  float tot[RT][MT][4];
#pragma unroll
  for (int rt = 0; rt < RT; ++rt)
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) tot[rt][mt][i] = 0.0f;
  for (int64_t w = w_first; w <= w_last; ++w) {
    const int64_t ws = warp_start(p.units, w, W);
    if (ws >= warp_start(p.units, w + 1, W)) continue;   // empty range
    const int s = (ws / G == b) ? 0 : 1;
    const float* rp = p.partials + (w * 2 + s) * kSlot;
    int k = 0;
#pragma unroll
    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i, ++k) tot[rt][mt][i] += __ldcg(rp + k * 32 + lane);
  }
  store_y<MT, RT>(p, row0, g, t, tot);
  if (lane == 0) p.counters[b] = 0u;
}

template <int MT, int RT, bool ZP, int S>
__global__ void __launch_bounds__(kGemvThreads)
gemv_kernel(const GemvParams p) {
  extern __shared__ __align__(16) uint8_t gemv_smem[];
  constexpr int kCodeBytes = RT * 2 * 32 * 16;   // [rt][row half][lane] x 16 B
  constexpr int kMetaBytes = RT * 16 * 2;         // one fp16 per row of the block
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int wi = threadIdx.x >> 5;
  const int64_t gw = int64_t(blockIdx.x) * kGemvWarps + wi;
  const int64_t W = p.total_warps;
  const int64_t G = p.G;
  const int64_t u_begin = warp_start(p.units, gw, W);
  const int64_t u_end = warp_start(p.units, gw + 1, W);
  if (u_begin >= u_end) return;
  const int stage_bytes = p.stage_bytes;
  uint8_t* ring = gemv_smem + int64_t(wi) * S * stage_bytes;
  const uint32_t ring_s = smem_addr(ring);
  const int64_t words_per_row = p.K / 8;
  const int x_chunks = p.M * 16;

  auto issue = [&](int64_t u, int slot) {
    if (u < u_end) {
      const int64_t b = u / G;
      const int64_t j = u - b * G;
      const int64_t r0 = b * (16 * RT);
      const uint32_t st = ring_s + uint32_t(slot * stage_bytes);
#pragma unroll
      for (int rt = 0; rt < RT; ++rt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int64_t row = r0 + 16 * rt + 8 * h + g;
          const bool v = row < p.N;
          const int32_t* src = p.qweight + (v ? row : 0) * words_per_row + j * kWordsPerGroup + t * 4;
          cp_async_16(st + uint32_t(((rt * 2 + h) * 32 + lane) * 16), src, v ? 16u : 0u);
        }
      constexpr int kMetaLanes = 2 * RT * (ZP ? 2 : 1);
      if (lane < kMetaLanes) {   // runs of 8 rows: N % 8 == 0 makes each run all in or all out
        const int which = lane / (2 * RT);   // 0 scales, 1 zero points
        const int rt = (lane >> 1) % RT;
        const int h = lane & 1;
        const int64_t rowc = r0 + 16 * rt + 8 * h;
        const bool v = rowc < p.N;
        const uint16_t* src = (which ? p.zeros : p.scales) + j * p.N + (v ? rowc : 0);
        cp_async_16(st + uint32_t(kCodeBytes + which * kMetaBytes + (rt * 16 + 8 * h) * 2), src, v ? 16u : 0u);
      }
      for (int c = lane; c < x_chunks; c += 32) {
        const int m = c >> 4;
        const int cc = c & 15;
        const uint16_t* src = p.x + int64_t(m) * p.K + j * kGroup + cc * 8;
        cp_async_16(st + uint32_t(p.x_offset + m * 256 + x_chunk_pos(m, cc) * 16), src, 16u);
      }
    }
    cp_async_commit();   // one group per unit, empty past the range, so counts stay uniform
  };

#pragma unroll
  for (int i = 0; i < S - 1; ++i) issue(u_begin + i, i);

  const int64_t first_block = u_begin / G;
  int64_t cur_b = first_block;
  int jstart = int(u_begin - cur_b * G);
  float acc[RT][MT][4];
#pragma unroll
  for (int rt = 0; rt < RT; ++rt)
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[rt][mt][i] = 0.0f;

  int slot = 0;
  for (int64_t u = u_begin; u < u_end; ++u) {
    issue(u + S - 1, slot == 0 ? S - 1 : slot - 1);
    cp_async_wait<S - 1>();
    __syncwarp();   // metadata and x were copied by other lanes
    const int64_t b = u / G;
    if (b != cur_b) {
      finish_block<MT, RT>(p, cur_b, jstart, int(G), gw, first_block, lane, g, t, acc);
      cur_b = b;
      jstart = 0;
#pragma unroll
      for (int rt = 0; rt < RT; ++rt)
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[rt][mt][i] = 0.0f;
    }
    const uint8_t* st = ring + slot * stage_bytes;

    uint4 xf[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int m = 8 * mt + g;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
        xf[mt][jj] = m < p.M ? lds128(st + p.x_offset + m * 256 + x_chunk_pos(m, 4 * t + jj) * 16)
                             : make_uint4(0, 0, 0, 0);
    }

#pragma unroll
    for (int rt = 0; rt < RT; ++rt) {
      const uint4 c_lo = lds128(st + ((rt * 2 + 0) * 32 + lane) * 16);
      const uint4 c_hi = lds128(st + ((rt * 2 + 1) * 32 + lane) * 16);
      const float s_lo = half_bits_to_float(lds16(st + kCodeBytes + (rt * 16 + g) * 2));
      const float s_hi = half_bits_to_float(lds16(st + kCodeBytes + (rt * 16 + 8 + g) * 2));
      uint32_t zl1024, zl64, zh1024, zh64;
      if (ZP) {
        zero_bias_from_bits(lds16(st + kCodeBytes + kMetaBytes + (rt * 16 + g) * 2), zl1024, zl64);
        zero_bias_from_bits(lds16(st + kCodeBytes + kMetaBytes + (rt * 16 + 8 + g) * 2), zh1024, zh64);
      } else {
        zl1024 = zh1024 = 0x64086408u;   // 1032 = 1024 + 8
        zl64 = zh64 = 0x54805480u;       // 72 = 64 + 8
      }
      float grp[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) grp[mt][i] = 0.0f;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        uint32_t plo[4], phi[4];
        decode_word_qz(word_of(c_lo, jj), zl1024, zl64, plo);
        decode_word_qz(word_of(c_hi, jj), zh1024, zh64, phi);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          mma_16816(grp[mt], plo[0], phi[0], plo[1], phi[1], xf[mt][jj].x, xf[mt][jj].y);
          mma_16816(grp[mt], plo[2], phi[2], plo[3], phi[3], xf[mt][jj].z, xf[mt][jj].w);
        }
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        acc[rt][mt][0] = fmaf(s_lo, grp[mt][0], acc[rt][mt][0]);
        acc[rt][mt][1] = fmaf(s_lo, grp[mt][1], acc[rt][mt][1]);
        acc[rt][mt][2] = fmaf(s_hi, grp[mt][2], acc[rt][mt][2]);
        acc[rt][mt][3] = fmaf(s_hi, grp[mt][3], acc[rt][mt][3]);
      }
    }
    __syncwarp();   // every lane is done with the slot before it is refilled
    slot = (slot + 1 == S) ? 0 : slot + 1;
  }
  finish_block<MT, RT>(p, cur_b, jstart, int(u_end - cur_b * G), gw, first_block, lane, g, t, acc);
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// host side: plan (variant, grid, workspace) for a shape
// ---------------------------------------------------------------------------
using KernelFn = void (*)(const GemvParams);

struct Variant {
  KernelFn fn;
  int mt, rt, stages, id;
};

constexpr int kNumVariants = 4;

Variant pick_variant(int64_t M, bool zp) {
  if (M <= 8)
    return zp ? Variant{gemv_kernel<1, 2, true, 4>, 1, 2, 4, 0} : Variant{gemv_kernel<1, 2, false, 4>, 1, 2, 4, 1};
  return zp ? Variant{gemv_kernel<2, 2, true, 3>, 2, 2, 3, 2} : Variant{gemv_kernel<2, 2, false, 3>, 2, 2, 3, 3};
}

int stage_bytes_for(const Variant& v, int64_t M, bool zp) {
  return v.rt * 2 * 32 * 16 + v.rt * 16 * 2 * (zp ? 2 : 1) + int(M) * 256;
}

struct Plan {
  Variant v;
  int grid;
  int nb;
  int smem;
  int stage_bytes;
  int64_t units;
  size_t counter_bytes;
  size_t partial_bytes;
};

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<int> g_smem_attr[kMaxDevices][kNumVariants];
std::atomic<int> g_occ[kMaxDevices][kNumVariants][17];   // by M

awq_status_t make_plan(int64_t M, int64_t N, int64_t K, bool zp, Plan& pl) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return AWQ_ERR_UNSUPPORTED;
  pl.v = pick_variant(M, zp);
  pl.stage_bytes = stage_bytes_for(pl.v, M, zp);
  pl.smem = kGemvWarps * pl.v.stages * pl.stage_bytes;
  int sms = g_sm_count[dev].load(std::memory_order_relaxed);
  if (sms == 0) {
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return AWQ_ERR_CUDA;
    g_sm_count[dev].store(sms, std::memory_order_relaxed);
  }
  if (!g_smem_attr[dev][pl.v.id].load(std::memory_order_acquire)) {
    // the largest ring any M asks of this variant
    const int most = kGemvWarps * pl.v.stages * stage_bytes_for(pl.v, pl.v.mt * 8, zp);
    if (cudaFuncSetAttribute(pl.v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, most) != cudaSuccess)
      return AWQ_ERR_CUDA;
    g_smem_attr[dev][pl.v.id].store(1, std::memory_order_release);
  }
  int occ = g_occ[dev][pl.v.id][M].load(std::memory_order_relaxed);
  if (occ == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, pl.v.fn, kGemvThreads, pl.smem) != cudaSuccess)
      return AWQ_ERR_CUDA;
    if (occ < 1) return AWQ_ERR_UNSUPPORTED;
    g_occ[dev][pl.v.id][M].store(occ, std::memory_order_relaxed);
  }
  const int64_t rows_per_block = 16 * pl.v.rt;
  const int64_t G = K / kGroup;
  pl.nb = int((N + rows_per_block - 1) / rows_per_block);
  pl.units = int64_t(pl.nb) * G;
  const int64_t want = (pl.units + kGemvWarps - 1) / kGemvWarps;
  const int64_t cap = int64_t(sms) * occ;
  pl.grid = int(want < cap ? (want > 0 ? want : 1) : cap);
  const int64_t total_warps = int64_t(pl.grid) * kGemvWarps;
  // units * warps must fit the kernel's 64-bit split arithmetic
  if (pl.units > 0 && total_warps > (int64_t(1) << 62) / pl.units) return AWQ_ERR_SHAPE;
  const size_t slot_floats = size_t(pl.v.rt) * pl.v.mt * 4 * 32;
  pl.counter_bytes = ((size_t(pl.nb) * 4 + 255) / 256) * 256;
  // With one group per row (G == 1) every unit is a whole block and no
  // block is ever split; otherwise warps may share blocks. A warp holds at
  // most two partial blocks: the first and the last of its range.
  pl.partial_bytes = G > 1 ? size_t(total_warps) * 2 * slot_floats * 4 : 0;
  return AWQ_OK;
}

awq_status_t check_gemv_args(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                             const uint16_t* zeros, int64_t M, int64_t N, int64_t K,
                             awq_qconfig_t cfg, uint16_t* y) {
  awq_status_t st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if ((st = check_nk(N, K)) != AWQ_OK) return st;
  if (M < 1 || M > 16) return AWQ_ERR_SHAPE;
  if (N % 8) return AWQ_ERR_SHAPE;
  if (N == 0) return AWQ_OK;
  if (!x || !qweight || !scales || !y) return AWQ_ERR_NULL;
  if (cfg.zero_point && !zeros) return AWQ_ERR_NULL;
  if (!cfg.zero_point && zeros) return AWQ_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(qweight) || !aligned16(scales) || !aligned16(y) ||
      (zeros && !aligned16(zeros)))
    return AWQ_ERR_ALIGN;
  return AWQ_OK;
}

}  // namespace

// Workspace bytes of the GEMV for (M, N, K); used by awq_workspace_bytes.
awq_status_t gemv_workspace_bytes(int64_t M, int64_t N, int64_t K, bool zp, size_t* bytes) {
  if (N == 0) { *bytes = 0; return AWQ_OK; }
  Plan pl;
  awq_status_t st = make_plan(M, N, K, zp, pl);
  if (st != AWQ_OK) return st;
  *bytes = pl.partial_bytes ? pl.counter_bytes + pl.partial_bytes : 0;
  return AWQ_OK;
}

}  // namespace awq

using namespace awq;

extern "C" awq_status_t awq_gemv(const uint16_t* x, const int32_t* qweight,
                                 const uint16_t* scales, const uint16_t* zeros, int64_t M,
                                 int64_t N, int64_t K, awq_qconfig_t cfg, uint16_t* y,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  awq_status_t st = check_gemv_args(x, qweight, scales, zeros, M, N, K, cfg, y);
  if (st != AWQ_OK || N == 0) return st;
  Plan pl;
  if ((st = make_plan(M, N, K, cfg.zero_point != 0, pl)) != AWQ_OK) return st;
  GemvParams p;
  p.x = x;
  p.qweight = qweight;
  p.scales = scales;
  p.zeros = zeros;
  p.y = y;
  p.counters = nullptr;
  p.partials = nullptr;
  if (pl.partial_bytes) {
    if (!workspace || workspace_bytes < pl.counter_bytes + pl.partial_bytes) return AWQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return AWQ_ERR_ALIGN;
    p.counters = static_cast<uint32_t*>(workspace);
    p.partials = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.counter_bytes);
  }
  p.units = pl.units;
  p.M = int(M);
  p.N = int(N);
  p.K = int(K);
  p.G = int(K / kGroup);
  p.nb = pl.nb;
  p.total_warps = pl.grid * kGemvWarps;
  p.stage_bytes = pl.stage_bytes;
  p.x_offset = pl.v.rt * 2 * 32 * 16 + pl.v.rt * 16 * 2 * (cfg.zero_point ? 2 : 1);
  pl.v.fn<<<pl.grid, kGemvThreads, pl.smem, static_cast<cudaStream_t>(stream)>>>(p);
  return launch_status();
}
