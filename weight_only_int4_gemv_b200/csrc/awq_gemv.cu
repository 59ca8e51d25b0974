// W4A16 small-batch product y[M][N] = x[M][K] . W'^T, 1 <= M <= 16, for sm_100a.
//
// ("AutoAWQ" code tour, "The big picture": the GEMV kernel for single-token
// decoding; "AutoAWQ" capability page: INT4 weights are decoded inside the
// matmul and never written back as fp16.)
//
// The layer is bound by HBM: every packed code byte is read once and feeds
// only M multiply-adds. Design:
//
// * Work unit = (row block of 16*RT output channels, one group of 128 k).
//   Units are ordered block-major and split evenly over every warp of a grid
//   sized to the resident capacity of the GPU (a stream-K split): all SMs
//   stream the same number of bytes whatever N and K are.
// * Each warp owns an S-stage ring in shared memory. Lane 0 fills a stage
//   with TMA: one 2-D box of packed codes (16*RT rows x 64 bytes), one box
//   of x (M rows x 128 k), and the 16*RT-long runs of scales and zero points
//   (group-major metadata makes them contiguous), all completing on the
//   stage's mbarrier. Units S-1 ahead of the arithmetic stay in flight
//   without holding registers or L1 request slots.
// * Decode: the packed nibble order puts consecutive k pairs in the low and
//   high halves of a word, so one LOP3 turns a word into two exact fp16
//   integers, 1024+q for the pairs (0,1), (4,5) and 64+q for (2,3), (6,7):
//   five instructions per eight weights.
// * Multiply: the decoded 16x16 weight tile is the A operand of
//   mma.m16n8k16 straight from registers; x is the B operand (batch in the
//   n dimension, two n8 tiles for M > 8). The k positions inside an MMA are
//   a permutation of the word's k (each lane owns whole words), matched by
//   reading x[m][8w .. 8w+7] for the same words: one 16-byte read covers two
//   MMAs. Products are exact and accumulation is fp32. The RT row tiles are
//   independent accumulator chains, interleaved.
// * Offsets and scale, once per group and batch row, in fp32:
//   sum_k x (q - z) = raw - C(m) - z S(m), with raw the MMA sum over the
//   magic-offset values, C(m) = 1024 sum_{k: 1024 pairs} x + 64 sum_{k: 64
//   pairs} x and S(m) = sum_k x. C and S come from two more MMAs against a
//   constant tile (rows 0 and 1), shared by all rows of the unit. Then
//   acc += s (raw - C - z S): the scale multiplies the group's partial sum.
// * A row block split between warps is finished by the last warp to arrive
//   (arrival counter per block): it sums the contributors' fp32 partials in
//   a fixed order, so results do not depend on timing, and resets the
//   counter for the next call. No warp ever waits on another.
// * Programmatic dependent launch: every CTA lets the next kernel launch as
//   soon as it runs, and prefetches its first weight units from HBM into L2
//   before waiting for the previous kernel (griddepcontrol.wait); loads into
//   shared memory, workspace accesses and y stores come after the wait.
//   Back-to-back layers overlap their launch and HBM ramp-up with the
//   previous layer's tail. The L2 prefetch runs kPrefetchUnits ahead.
// * Every mbarrier wait is bounded (2 s); a warp that gives up records bit 1
//   of the device error word, waits (bounded) for its copies in flight and
//   leaves its rows unwritten.

#include <atomic>

#include "awq_common.cuh"
#include "awq_tma_host.h"

namespace awq {

__device__ uint32_t g_awq_gemv_error = 0;

namespace {

constexpr int kMaxConsumers = 12;
constexpr int kMaxStages = 8;
constexpr int kBarRegion = 2 * kMaxConsumers * kMaxStages * 8;   // full + empty mbarriers
constexpr int kPrefetchUnits = 1;  // L2 prefetch distance, in units, per consumer

struct GemvParams {
  uint16_t* y;
  float* partials;       // [total consumers][2][16*RT*M] floats, [row][m]
  uint32_t* counters;    // [nb]
  int64_t units;         // nb * G
  int M, N, K, G, nb;
  int consumers;         // consumer warps per CTA
  int total_consumers;   // grid * consumers
  int stages;            // ring stages per consumer
  int stage_bytes;       // codes + metadata + x slice of one unit (multiple of 128)
  int x_offset;          // offset of the x slice inside a stage
  uint32_t tx_bytes;     // bytes the TMA copies of one unit deliver
};

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

// First unit of consumer w in the even split of `units` over `consumers`.
__device__ __forceinline__ int64_t range_start(int64_t units, int64_t w, int64_t consumers) {
  return units * w / consumers;
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

// Finish row block b after consumer gc summed groups [j0, j1) of it.
// A split block's partial sums are stored compactly (the block's 16*RT rows
// x M batch rows, [row][m]); the consumer that completes the block's group
// count sums every contributor's values in consumer order (reproducible
// bits), loading many contributors at once.
template <int MT, int RT>
__device__ __forceinline__ void finish_block(const GemvParams& p, int64_t b, int j0, int j1, int64_t gc,
                                             int64_t first_block, int lane, int g, int t,
                                             const float (&acc)[RT][MT][4]) {
  const int64_t row0 = b * (16 * RT);
  const int64_t G = p.G;
  if (j0 == 0 && j1 == G) {
    store_y<MT, RT>(p, row0, g, t, acc);
    return;
  }
  const int M = p.M;
  const int V = 16 * RT * M;                     // values of one partial
  const int slot = (b == first_block) ? 0 : 1;
  float* sp = p.partials + (gc * 2 + slot) * int64_t(V);
#pragma unroll
  for (int rt = 0; rt < RT; ++rt)
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int m0 = 8 * mt + 2 * t;
      const int r_lo = 16 * rt + g, r_hi = r_lo + 8;
      if (m0 < M) {
        __stcg(sp + r_lo * M + m0, acc[rt][mt][0]);
        __stcg(sp + r_hi * M + m0, acc[rt][mt][2]);
      }
      if (m0 + 1 < M) {
        __stcg(sp + r_lo * M + m0 + 1, acc[rt][mt][1]);
        __stcg(sp + r_hi * M + m0 + 1, acc[rt][mt][3]);
      }
    }
  __syncwarp();   // every lane's stores happen before lane 0's release below
  uint32_t last = 0;
  if (lane == 0) {
    const uint32_t mine = uint32_t(j1 - j0);
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
                 : "=r"(old) : "l"(p.counters + b), "r"(mine) : "memory");
    last = (old + mine == uint32_t(G)) ? 1u : 0u;
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  // Contributors: every non-empty consumer range overlapping block b, in
  // consumer order. Range starts floor(units * w / W) advance by
  // floor(units / W) plus a carry, so no division happens per contributor.
  const int64_t W = p.total_consumers;
  const int64_t w_first = ((b * G + 1) * W - 1) / p.units;
  const int64_t w_last = ((b * G + G) * W - 1) / p.units;
  const int64_t q_step = p.units / W, r_step = p.units % W;
  const int64_t bG = b * G;
  constexpr int kChunk = 16;                     // contributors loaded at once
  const int nv = V / 32;                         // values per lane (V = 64 M), two per pass
  for (int v0 = 0; v0 < nv; v0 += 2) {
    int64_t ws = range_start(p.units, w_first, W);
    int64_t rem = (p.units * w_first) % W;
    float acc2[2] = {0.0f, 0.0f};
    for (int64_t w0 = w_first; w0 <= w_last; w0 += kChunk) {
      float part[kChunk][2];
#pragma unroll
      for (int c = 0; c < kChunk; ++c) {
        const int64_t w = w0 + c;
        int64_t we = ws + q_step;                // start of range w + 1
        int64_t rem2 = rem + r_step;
        if (rem2 >= W) { rem2 -= W; ++we; }
        const bool live = w <= w_last && ws < we;
        const int s = ws >= bG ? 0 : 1;          // block b is the range's first block, or its last
        const float* src = p.partials + (w * 2 + s) * int64_t(V);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int v = lane + 32 * (v0 + e);
          part[c][e] = (live && v < V) ? __ldcg(src + v) : 0.0f;
        }
        ws = we;
        rem = rem2;
      }
#pragma unroll
      for (int c = 0; c < kChunk; ++c) {
        acc2[0] += part[c][0];
        acc2[1] += part[c][1];
      }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int v = lane + 32 * (v0 + e);
      if (v < V) {
        const int row = v / M, m = v - row * M;
        if (row0 + row < p.N)
          p.y[int64_t(m) * p.N + row0 + row] = __half_as_ushort(__float2half_rn(acc2[e]));
      }
    }
  }
  if (lane == 0) p.counters[b] = 0u;
}

// A fragment of the constant 16x16 tile that turns two extra MMAs into the
// per-batch-row sums the decode offsets need: row 0 holds 1024 at the k
// slots fed by (1024 + q) pairs and 64 at the slots fed by (64 + q) pairs,
// row 1 holds 1; every other row is 0. Lane (g, t) owns rows g and g+8.
__device__ __forceinline__ void offset_tile(int g, uint32_t& a0, uint32_t& a2) {
  a0 = g == 0 ? 0x64006400u : (g == 1 ? 0x3C003C00u : 0u);
  a2 = g == 0 ? 0x54005400u : (g == 1 ? 0x3C003C00u : 0u);
}

template <int RT>
struct StageLayout {
  static constexpr int kCodeBytes = 16 * RT * 64;   // [16*RT rows][16 words]
  static constexpr int kMetaBytes = 16 * RT * 2;    // one fp16 per row of the block
  static constexpr int kMetaStride = (kMetaBytes + 127) / 128 * 128;
};

// Consumer warps per CTA: 7, plus the producer, so each SM sub-partition's
// quarter of the register file holds a whole number of warps. With one n8
// batch tile a CTA is built to take half an SM (<= 128 registers per thread,
// <= 113 KB of shared memory): one CTA per SM streams this layer while the
// other half hosts the next kernel's CTA, which starts prefetching its
// weights before this one finishes. With two batch tiles a CTA takes the
// whole SM (255 registers per thread).
template <int MT>
struct Consumers {
  static constexpr int value = 7;
  static constexpr int ctas_per_sm = MT == 1 ? 2 : 1;
};

template <int MT, int RT, bool ZP>
__global__ void __launch_bounds__(32 * (1 + Consumers<MT>::value), Consumers<MT>::ctas_per_sm)
gemv_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_x,
            const __grid_constant__ CUtensorMap tmap_s, const __grid_constant__ CUtensorMap tmap_z,
            const GemvParams p) {
  extern __shared__ __align__(1024) uint8_t gemv_smem[];
  using L = StageLayout<RT>;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int C = p.consumers;
  const int S = p.stages;
  const int64_t W = p.total_consumers;
  const int64_t G = p.G;
  const int stage_bytes = p.stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(gemv_smem);            // [consumer][stage]
  uint64_t* empty = full + kMaxConsumers * kMaxStages;                // [consumer][stage]
  uint8_t* rings = gemv_smem + kBarRegion;                            // consumer c: c * S stages
  // Let the next kernel in the stream (if launched as a programmatic
  // dependent) start as soon as every CTA of this one is running; it waits
  // for this grid's completion before it reads anything this grid writes.
  asm volatile("griddepcontrol.launch_dependents;");

  if (threadIdx.x == 0) {
    for (int i = 0; i < C * S; ++i) {
      mbar_init(&full[(i / S) * kMaxStages + i % S], 1);
      mbar_init(&empty[(i / S) * kMaxStages + i % S], 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Lane c feeds consumer c. All lanes step through their rounds together,
    // so round r of every consumer is issued before round r+1 and data
    // returns roughly in the order it is consumed.
    if (lane >= C) return;
    const int64_t gc = int64_t(blockIdx.x) * C + lane;
    const int64_t ub = range_start(p.units, gc, W);
    const int64_t n = range_start(p.units, gc + 1, W) - ub;
    if (n <= 0) return;
    // (block, group) of the consumer's first unit; later units advance by one group
    int64_t b0 = ub / G;
    int j0 = int(ub - b0 * G);
    // Before the dependency wait only L2 prefetches: they are safe even
    // while an earlier kernel may still be writing these bytes.
    {
      int64_t b = b0;
      int j = j0;
      for (int64_t r = 0; r < n && r < kPrefetchUnits; ++r) {
        const int r0 = int(b * (16 * RT));
        tma_prefetch_l2_2d(&tmap_q, j * kWordsPerGroup, r0);
        tma_prefetch_l2_2d(&tmap_s, r0, j);
        if (ZP) tma_prefetch_l2_2d(&tmap_z, r0, j);
        if (++j == G) { j = 0; ++b; }
      }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    uint64_t* fb0 = &full[lane * kMaxStages];
    uint64_t* eb0 = &empty[lane * kMaxStages];
    uint8_t* ring = rings + lane * S * stage_bytes;
    volatile int abort_flag = 0;
    int64_t b = b0;
    int j = j0;
    int slot = 0;
    uint32_t ephase = 1;   // parity of the empty phase to wait for in the slot's next reuse
    int64_t r = 0;
    for (; r < n; ++r) {
      if (r >= S && !wait_bounded(&eb0[slot], ephase, &abort_flag, &g_awq_gemv_error, 2u)) break;
      const int r0 = int(b * (16 * RT));
      uint8_t* st = ring + slot * stage_bytes;
      mbar_arrive_expect_tx(&fb0[slot], p.tx_bytes);
      tma_load_2d(st, &tmap_q, j * kWordsPerGroup, r0, &fb0[slot]);
      tma_load_2d(st + p.x_offset, &tmap_x, j * kGroup, 0, &fb0[slot]);
      tma_load_2d(st + L::kCodeBytes, &tmap_s, r0, j, &fb0[slot]);
      if (ZP) tma_load_2d(st + L::kCodeBytes + L::kMetaStride, &tmap_z, r0, j, &fb0[slot]);
      if (++j == G) { j = 0; ++b; }
      if (++slot == S) { slot = 0; ephase ^= 1u; }
    }
    // Gave up: the copies already issued (the last S rounds before r) land
    // before the CTA's shared memory can be reused.
    if (r < n) {
      for (int64_t q = r - S > 0 ? r - S : 0; q < r; ++q)
        wait_teardown(&fb0[int(q % S)], uint32_t((q / S) & 1));
    }
    return;
  }

  // -------------------------------------------------------------- consumer
  const int cw = warp - 1;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int64_t gc = int64_t(blockIdx.x) * C + cw;
  const int64_t u_begin = range_start(p.units, gc, W);
  const int64_t u_end = range_start(p.units, gc + 1, W);
  if (u_begin >= u_end) return;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  uint8_t* ring = rings + cw * S * stage_bytes;

  // x fragment offsets inside a stage: batch row m = 8 mt + g, chunk 4t + jj
  int xoff[MT];
  bool xok[MT];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int m = 8 * mt + g;
    xok[mt] = m < p.M;
    xoff[mt] = p.x_offset + m * 256 + t * 64;
  }
  uint32_t ca0, ca2;
  offset_tile(g, ca0, ca2);
  volatile int abort_flag = 0;

  const int64_t first_block = u_begin / G;
  int64_t cur_b = first_block;
  int jstart = int(u_begin - cur_b * G);
  int64_t ub_ = cur_b;   // block of the unit being consumed
  int jg = jstart;       // its group
  float acc[RT][MT][4];
#pragma unroll
  for (int rt = 0; rt < RT; ++rt)
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[rt][mt][i] = 0.0f;

  int slot = 0;
  uint32_t phase = 0;
  for (int64_t u = u_begin; u < u_end; ++u) {
    const bool got = wait_bounded(&full[cw * kMaxStages + slot], phase, &abort_flag, &g_awq_gemv_error, 2u);
    if (!__all_sync(0xffffffffu, got)) return;   // producer gave up or timed out: rows stay unwritten
    const int64_t b = ub_;
    if (++jg == G) { jg = 0; ++ub_; }
    if (b != cur_b) {
      finish_block<MT, RT>(p, cur_b, jstart, int(G), gc, first_block, lane, g, t, acc);
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

    // x fragments and packed codes of the unit
    uint4 xf[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) xf[mt][jj] = xok[mt] ? lds128(st + xoff[mt] + jj * 16) : make_uint4(0, 0, 0, 0);
    uint4 c_lo[RT], c_hi[RT];
#pragma unroll
    for (int rt = 0; rt < RT; ++rt) {
      c_lo[rt] = lds128(st + (16 * rt + g) * 64 + t * 16);
      c_hi[rt] = lds128(st + (16 * rt + 8 + g) * 64 + t * 16);
    }
    float grp[RT][MT][4];
    float cs[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        cs[mt][i] = 0.0f;
#pragma unroll
        for (int rt = 0; rt < RT; ++rt) grp[rt][mt][i] = 0.0f;
      }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        mma_16816(cs[mt], ca0, 0u, ca2, 0u, xf[mt][jj].x, xf[mt][jj].y);
        mma_16816(cs[mt], ca0, 0u, ca2, 0u, xf[mt][jj].z, xf[mt][jj].w);
      }
#pragma unroll
      for (int rt = 0; rt < RT; ++rt) {
        uint32_t plo[4], phi[4];
        decode_word_magic(word_of(c_lo[rt], jj), plo);
        decode_word_magic(word_of(c_hi[rt], jj), phi);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          mma_16816(grp[rt][mt], plo[0], phi[0], plo[1], phi[1], xf[mt][jj].x, xf[mt][jj].y);
          mma_16816(grp[rt][mt], plo[2], phi[2], plo[3], phi[3], xf[mt][jj].z, xf[mt][jj].w);
        }
      }
    }
    // row 0 of the constant tile (lanes 0..3) holds C, row 1 (lanes 4..7) holds S
    float cm[MT][2], sm[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      cm[mt][0] = __shfl_sync(0xffffffffu, cs[mt][0], t);
      cm[mt][1] = __shfl_sync(0xffffffffu, cs[mt][1], t);
      sm[mt][0] = __shfl_sync(0xffffffffu, cs[mt][0], 4 + t);
      sm[mt][1] = __shfl_sync(0xffffffffu, cs[mt][1], 4 + t);
    }
    float s_lo[RT], s_hi[RT], z_lo[RT], z_hi[RT];
#pragma unroll
    for (int rt = 0; rt < RT; ++rt) {
      s_lo[rt] = half_bits_to_float(lds16(st + L::kCodeBytes + (16 * rt + g) * 2));
      s_hi[rt] = half_bits_to_float(lds16(st + L::kCodeBytes + (16 * rt + 8 + g) * 2));
      z_lo[rt] = ZP ? half_bits_to_float(lds16(st + L::kCodeBytes + L::kMetaStride + (16 * rt + g) * 2)) : 8.0f;
      z_hi[rt] = ZP ? half_bits_to_float(lds16(st + L::kCodeBytes + L::kMetaStride + (16 * rt + 8 + g) * 2)) : 8.0f;
    }
    // everything the unit needs is in registers: release the slot
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[cw * kMaxStages + slot]);
    if (++slot == S) {
      slot = 0;
      phase ^= 1u;
    }
    // sum_k x (q - z) = raw - C(m) - z S(m); then the group's scale
#pragma unroll
    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        acc[rt][mt][0] = fmaf(s_lo[rt], fmaf(-z_lo[rt], sm[mt][0], grp[rt][mt][0] - cm[mt][0]), acc[rt][mt][0]);
        acc[rt][mt][1] = fmaf(s_lo[rt], fmaf(-z_lo[rt], sm[mt][1], grp[rt][mt][1] - cm[mt][1]), acc[rt][mt][1]);
        acc[rt][mt][2] = fmaf(s_hi[rt], fmaf(-z_hi[rt], sm[mt][0], grp[rt][mt][2] - cm[mt][0]), acc[rt][mt][2]);
        acc[rt][mt][3] = fmaf(s_hi[rt], fmaf(-z_hi[rt], sm[mt][1], grp[rt][mt][3] - cm[mt][1]), acc[rt][mt][3]);
      }
  }
  finish_block<MT, RT>(p, cur_b, jstart, int(u_end - cur_b * G), gc, first_block, lane, g, t, acc);
}

// ---------------------------------------------------------------------------
// host side: plan (variant, grid, workspace) for a shape
// ---------------------------------------------------------------------------
using KernelFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                          const GemvParams);

struct Variant {
  KernelFn fn;
  int mt, rt, consumers, id;
};

constexpr int kNumVariants = 4;
constexpr int kRT = 4;
constexpr int kSmemBudget = 232448;   // largest dynamic shared memory of one sm_100 CTA
constexpr int kHalfSmBudget = 115712; // half of an SM's 228 KB, less the 1 KB reserved per CTA

int smem_budget(const Variant& v);

Variant pick_variant(int64_t M, bool zp) {
  if (M <= 8)
    return zp ? Variant{gemv_kernel<1, kRT, true>, 1, kRT, Consumers<1>::value, 0}
              : Variant{gemv_kernel<1, kRT, false>, 1, kRT, Consumers<1>::value, 1};
  return zp ? Variant{gemv_kernel<2, kRT, true>, 2, kRT, Consumers<2>::value, 2}
            : Variant{gemv_kernel<2, kRT, false>, 2, kRT, Consumers<2>::value, 3};
}

int round128(int v) { return (v + 127) / 128 * 128; }

struct StageGeometry {
  int code_bytes, meta_stride, x_offset, stage_bytes, stages;
  uint32_t tx_bytes;
};

StageGeometry stage_geometry(const Variant& v, int64_t M, bool zp) {
  StageGeometry sg;
  sg.code_bytes = 16 * v.rt * 64;
  sg.meta_stride = round128(16 * v.rt * 2);
  sg.x_offset = sg.code_bytes + sg.meta_stride * (zp ? 2 : 1);
  sg.stage_bytes = round128(sg.x_offset + int(M) * 256);
  sg.tx_bytes = uint32_t(sg.code_bytes + 16 * v.rt * 2 * (zp ? 2 : 1) + int(M) * 256);
  int st = (smem_budget(v) - kBarRegion) / (v.consumers * sg.stage_bytes);
  sg.stages = st > kMaxStages ? kMaxStages : st;
  return sg;
}

int smem_budget(const Variant& v) { return v.mt == 1 ? kHalfSmBudget : kSmemBudget; }

struct Plan {
  Variant v;
  StageGeometry sg;
  int grid;
  int nb;
  int smem;
  int64_t units;
  size_t counter_bytes;
  size_t partial_bytes;
};

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<int> g_smem_attr[kMaxDevices][kNumVariants];

awq_status_t make_plan(int64_t M, int64_t N, int64_t K, bool zp, Plan& pl) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return AWQ_ERR_UNSUPPORTED;
  pl.v = pick_variant(M, zp);
  pl.sg = stage_geometry(pl.v, M, zp);
  if (pl.sg.stages < 2) return AWQ_ERR_UNSUPPORTED;
  pl.smem = kBarRegion + pl.v.consumers * pl.sg.stages * pl.sg.stage_bytes;
  int sms = g_sm_count[dev].load(std::memory_order_relaxed);
  if (sms == 0) {
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return AWQ_ERR_CUDA;
    g_sm_count[dev].store(sms, std::memory_order_relaxed);
  }
  if (!g_smem_attr[dev][pl.v.id].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(pl.v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_budget(pl.v)) != cudaSuccess)
      return AWQ_ERR_CUDA;
    g_smem_attr[dev][pl.v.id].store(1, std::memory_order_release);
  }
  const int64_t rows_per_block = 16 * pl.v.rt;
  const int64_t G = K / kGroup;
  pl.nb = int((N + rows_per_block - 1) / rows_per_block);
  pl.units = int64_t(pl.nb) * G;
  // one CTA per SM (for one batch tile it takes half the SM, leaving the
  // other half to the next kernel); fewer when there are fewer units than
  // consumers
  const int64_t want = (pl.units + pl.v.consumers - 1) / pl.v.consumers;
  pl.grid = int(want < sms ? (want > 0 ? want : 1) : sms);
  const int64_t total = int64_t(pl.grid) * pl.v.consumers;
  // units * consumers must fit the kernel's 64-bit split arithmetic
  if (pl.units > 0 && total > (int64_t(1) << 62) / pl.units) return AWQ_ERR_SHAPE;
  pl.counter_bytes = ((size_t(pl.nb) * 4 + 255) / 256) * 256;
  // With one group per row (G == 1) every unit is a whole block and no
  // block is ever split; otherwise consumers may share blocks. A consumer
  // holds at most two partial blocks: the first and the last of its range,
  // each 16*RT rows x M values.
  pl.partial_bytes = G > 1 ? size_t(total) * 2 * size_t(16 * pl.v.rt) * size_t(M) * 4 : 0;
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

// Read and clear this file's device error word (stream-ordered).
awq_status_t gemv_take_error(uint32_t* word, cudaStream_t s) {
  uint32_t zero = 0;
  if (cudaMemcpyFromSymbolAsync(word, g_awq_gemv_error, sizeof(uint32_t), 0, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return AWQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return AWQ_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(g_awq_gemv_error, &zero, sizeof(uint32_t), 0, cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return AWQ_ERR_CUDA;
  return cudaStreamSynchronize(s) == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

}  // namespace awq

using namespace awq;

extern "C" awq_status_t awq_gemv(const uint16_t* x, const int32_t* qweight,
                                 const uint16_t* scales, const uint16_t* zeros, int64_t M,
                                 int64_t N, int64_t K, awq_qconfig_t cfg, uint16_t* y,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  awq_status_t st = check_gemv_args(x, qweight, scales, zeros, M, N, K, cfg, y);
  if (st != AWQ_OK || N == 0) return st;
  const bool zp = cfg.zero_point != 0;
  Plan pl;
  if ((st = make_plan(M, N, K, zp, pl)) != AWQ_OK) return st;
  GemvParams p;
  p.y = y;
  p.counters = nullptr;
  p.partials = nullptr;
  if (pl.partial_bytes) {
    if (!workspace || workspace_bytes < pl.counter_bytes + pl.partial_bytes) return AWQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return AWQ_ERR_ALIGN;
    p.counters = static_cast<uint32_t*>(workspace);
    p.partials = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.counter_bytes);
  }
  const int G = int(K / kGroup);
  // codes: int32 [N][K/8], box 16 words (one group) x 16*RT rows
  // x: fp16 [M][K], box 128 k x M rows; scales / zeros: fp16 [G][N], box 16*RT x 1
  CUtensorMap tq, tx, ts, tz;
  const uint32_t rows = uint32_t(16 * pl.v.rt);
  if (!make_tensor_map_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_INT32, qweight, uint64_t(K / 8), uint64_t(N),
                          uint64_t(K / 8) * 4, kWordsPerGroup, rows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tensor_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, uint64_t(K), uint64_t(M),
                          uint64_t(K) * 2, kGroup, uint32_t(M), CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tensor_map_2d(&ts, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, scales, uint64_t(N), uint64_t(G),
                          uint64_t(N) * 2, rows, 1, CU_TENSOR_MAP_SWIZZLE_NONE))
    return AWQ_ERR_CUDA;
  if (zp) {
    if (!make_tensor_map_2d(&tz, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, zeros, uint64_t(N), uint64_t(G),
                            uint64_t(N) * 2, rows, 1, CU_TENSOR_MAP_SWIZZLE_NONE))
      return AWQ_ERR_CUDA;
  } else {
    tz = ts;   // never read by the symmetric kernels
  }
  p.units = pl.units;
  p.M = int(M);
  p.N = int(N);
  p.K = int(K);
  p.G = G;
  p.nb = pl.nb;
  p.consumers = pl.v.consumers;
  p.total_consumers = pl.grid * pl.v.consumers;
  p.stages = pl.sg.stages;
  p.stage_bytes = pl.sg.stage_bytes;
  p.x_offset = pl.sg.x_offset;
  p.tx_bytes = pl.sg.tx_bytes;
  // Programmatic dependent launch: this grid may start while the previous
  // kernel in the stream finishes; the kernel waits for it (griddepcontrol)
  // before any load into shared memory, workspace access or store.
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(pl.grid);
  lc.blockDim = dim3(32 * (1 + pl.v.consumers));
  lc.dynamicSmemBytes = size_t(pl.smem);
  lc.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  if (cudaLaunchKernelEx(&lc, pl.v.fn, tq, tx, ts, tz, p) != cudaSuccess) return AWQ_ERR_CUDA;
  return launch_status();
}

// ---------------------------------------------------------------------------
// awq_gemv_noalloc: awq_gemv with its scratch in a fixed array of this
// library instead of caller memory. The AWQ pages have no counterpart; it
// exists for callers that cannot allocate device memory at the point of
// the call (see awq.h).
// ---------------------------------------------------------------------------
namespace awq {
namespace {

constexpr size_t kStaticScratchBytes = AWQ_GEMV_STATIC_WORKSPACE_BYTES;

// Split-K partials and arrival counters of awq_gemv_noalloc. Every GPU that
// loads the library holds this array until the process exits; all calls on
// a device share it.
static __device__ __align__(256) uint8_t g_gemv_scratch[kStaticScratchBytes];

std::atomic<uintptr_t> g_scratch_addr[kMaxDevices];

// Device address of g_gemv_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
awq_status_t scratch_address(int dev, void** out) {
  uintptr_t a = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (a == 0) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gemv_scratch) != cudaSuccess || p == nullptr) return AWQ_ERR_CUDA;
    a = reinterpret_cast<uintptr_t>(p);
    g_scratch_addr[dev].store(a, std::memory_order_release);
  }
  *out = reinterpret_cast<void*>(a);
  return AWQ_OK;
}

}  // namespace
}  // namespace awq

extern "C" awq_status_t awq_gemv_noalloc(const uint16_t* x, const int32_t* qweight,
                                         const uint16_t* scales, const uint16_t* zeros, int64_t M,
                                         int64_t N, int64_t K, awq_qconfig_t cfg, uint16_t* y,
                                         void* stream) {
  awq_status_t st = check_gemv_args(x, qweight, scales, zeros, M, N, K, cfg, y);
  if (st != AWQ_OK || N == 0) return st;
  Plan pl;
  if ((st = make_plan(M, N, K, cfg.zero_point != 0, pl)) != AWQ_OK) return st;
  const size_t need = pl.partial_bytes ? pl.counter_bytes + pl.partial_bytes : 0;
  if (need > kStaticScratchBytes) return AWQ_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
  void* scratch = nullptr;
  if ((st = scratch_address(dev, &scratch)) != AWQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The arrival counters must start at zero. A completed call leaves them at
  // zero, but one that gave up part-way may not, so clear them every call.
  if (need && cudaMemsetAsync(scratch, 0, pl.counter_bytes, s) != cudaSuccess) return AWQ_ERR_CUDA;
  return awq_gemv(x, qweight, scales, zeros, M, N, K, cfg, y, scratch, kStaticScratchBytes, stream);
}
