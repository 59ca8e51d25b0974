// W4A16 small-batch product y[M][N] = x[M][K] . W'^T, 1 <= M <= 16, for sm_100a.
//
// ("AutoAWQ" code tour, "The big picture": the GEMV kernel for single-token
// decoding; "AutoAWQ" capability page: INT4 weights are decoded inside the
// matmul and never written back as fp16.)
//
// The layer is bound by HBM: every packed code byte is read once and feeds
// only M multiply-adds. Design:
//
// * Output channels come in tiles of 16 (one MMA tile). Each CTA owns a
//   contiguous run of whole tiles over the whole of K, so no partial sum
//   ever leaves the SM: the CTA's 8 warps split K between them and reduce
//   through shared memory. Tiles are spread evenly (at most one tile of
//   difference) over two half-SM CTAs per SM for M <= 8 (16 warps hide the
//   latency of the decode and MMA chains better than 8), one otherwise.
//   Only when there are fewer tiles than CTAs is K also cut into slices
//   handled by different CTAs; their fp32 partials meet in a workspace and
//   the last CTA to arrive on a tile sums them in slice order.
// * A CTA walks its tiles in chunks of up to four (64 channels). Within a
//   chunk, the K range goes by in stages of 8 groups, one group per warp: a
//   unit of work is (chunk, group), 16 words x up to 64 rows of codes.
// * The stages form one ring per CTA in shared memory, filled by TMA with a
//   few large boxes per stage: the codes through a 3-D view of qweight that
//   lands them group-major ([group][16 rows][16 words] per tile, so a warp's
//   16-byte reads hit distinct banks), the 64 x 8 blocks of scales and zero
//   points (group-major metadata), and x as [m][group][128 k]. A TMA issue
//   can hold its thread for hundreds of cycles, so few, large copies keep
//   that cost off the arithmetic. Each warp takes its group of a stage into
//   registers and counts itself out of the stage; the last of the 8 warps
//   refills the stage with the one S ahead, so no warp ever waits for
//   another.
// * Decode: the packed nibble order puts consecutive k pairs in the low and
//   high halves of a word, so one LOP3 turns a word into two exact fp16
//   integers, 1024+q for the pairs (0,1), (4,5) and 64+q for (2,3), (6,7):
//   five instructions per eight weights.
// * Multiply: the decoded 16x16 weight tile is the A operand of
//   mma.m16n8k16 straight from registers; x is the B operand (batch in the
//   n dimension, two n8 tiles for M > 8). The k positions inside an MMA are
//   a permutation of the word's k (each lane owns whole words), matched by
//   reading x[m][8w .. 8w+7] for the same words: one 16-byte read covers two
//   MMAs. Products are exact and accumulation is fp32.
// * Offsets and scale, once per group and batch row, in fp32:
//   sum_k x (q - z) = raw - C(m) - z S(m), with raw the MMA sum over the
//   magic-offset values, C(m) = 1024 sum_{k: 1024 pairs} x + 64 sum_{k: 64
//   pairs} x and S(m) = sum_k x. C and S come from two more MMAs against a
//   constant tile (rows 0 and 1). Then acc += s (raw - C - z S).
// * Programmatic dependent launch: every CTA lets the next kernel launch as
//   soon as it runs. Before waiting for the previous kernel
//   (griddepcontrol.wait) a CTA only prefetches its first code box into L2
//   (always safe), or, when the caller declares the weights static
//   (AWQ_FLAG_WEIGHTS_STATIC), already loads the codes, scales and zero
//   points of its first S stages into its ring; x, the workspace and y are
//   touched only after the wait; the next layer's CTAs take an SM's place as
//   soon as this layer's CTAs there have finished.
// * Every mbarrier wait is bounded (2 s); a warp that gives up records bit 1
//   of the device error word, stops waiting and stops releasing stages,
//   still takes part in its CTA's reductions (so no CTA barrier can hang),
//   and before the CTA exits thread 0 waits (bounded) for the fills still in
//   flight. The output is then incomplete.

#include <atomic>
#include <mutex>

#include "awq_common.cuh"
#include "awq_tma_host.h"

namespace awq {

__device__ uint32_t g_awq_gemv_error = 0;

namespace {

constexpr int kWarps = 8;                      // warps per CTA, each with its own ring
constexpr int kThreads = 32 * kWarps;
constexpr int kTile = 16;                      // output channels per MMA tile
constexpr int kChunkTiles = 4;                 // tiles accumulated together
constexpr int kChunkRows = kTile * kChunkTiles;
constexpr int kMaxStages = 8;
constexpr int kRingOffset = 1024;              // mbarriers and counters live below the ring
// One stage = one chunk x kWarps groups (one group per warp):
constexpr int kTileStageBytes = kWarps * kTile * 64;    // codes of one tile: [group][16 rows][16 words]
constexpr int kMetaStageBytes = kWarps * kChunkRows * 2;  // [group][64 rows] fp16 scales (or zeros)
constexpr int kXStageBytesPerRow = kWarps * 128 * 2;      // x: [m][group][128 k] fp16
// Packed zero points (AWQ_FLAG_PACKED_ZEROS): a stage holds, per group, the
// 8 qzeros words of a 4-tile chunk from a 16-byte-aligned start word (2 words
// before an odd first tile), rounded up to whole 16-byte runs: 12 words.
constexpr int kPackedZeroWords = 12;
constexpr int kPackedZeroStageBytes = kWarps * kPackedZeroWords * 4;
static_assert(kPackedZeroStageBytes % 128 == 0, "x must stay 128-byte aligned in a stage");
constexpr int kReduceBarrier = 1;              // named barrier of the chunk reductions
static_assert(kMaxStages * (8 + 4 + 4) + 4 <= kRingOffset, "stage bookkeeping overflows its region");

struct GemvParams {
  uint16_t* y;
  float* partials;       // [ks][T * 16][M] fp32, only when ks > 1
  uint32_t* counters;    // [T], only when ks > 1
  int M, N, G;
  int T;                 // tiles of 16 output channels
  int tpu;               // tiles per work unit: 1, or 2 (a gate tile and its up tile, AWQ_FLAG_SILU_MUL)
  int units;             // T / tpu work units per K slice
  int ks;                // K slices (1: every CTA covers all of K)
  int items;             // units * ks, slice-major: item i is unit i % units of slice i / units
  int stages;            // ring stages per warp
  int stage_bytes;       // codes + metadata + x slice of one unit (multiple of 128)
  int x_offset;          // offset of the x slice inside a stage
  int pbuf_offset;       // shared-memory partial sums of the chunk reductions
  int scale_offset;      // offset of the scales inside a stage (TC tiles of codes before it)
  int early;             // weights may be read before the previous kernel completes
  int codes4d;           // stage codes as one 4-D box (N % 16 == 0)
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

__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// A fragment of the constant 16x16 tile that turns two extra MMAs into the
// per-batch-row sums the decode offsets need: row 0 holds 1024 at the k
// slots fed by (1024 + q) pairs and 64 at the slots fed by (64 + q) pairs,
// row 1 holds 1; every other row is 0. Lane (g, t) owns rows g and g+8.
__device__ __forceinline__ void offset_tile(int g, uint32_t& a0, uint32_t& a2) {
  a0 = g == 0 ? 0x64006400u : (g == 1 ? 0x3C003C00u : 0u);
  a2 = g == 0 ? 0x54005400u : (g == 1 ? 0x3C003C00u : 0u);
}

// A run of up to kChunkTiles consecutive tiles (whole units) of one K slice
// inside a CTA's item range, with the slice's groups [gb, ge).
struct Chunk {
  int i;       // first item
  int nu;      // items (units)
  int tc;      // tiles
  int t0;      // first tile
  int s;       // slice
  int gb, ge;  // groups of the slice
};

// ct: most tiles per chunk; tpu: tiles per unit (a compile-time constant at every call)
__device__ __forceinline__ void load_chunk(const GemvParams& p, int ct, int tpu, int i, int i_end, Chunk& c) {
  c.i = i;
  c.s = i / p.units;
  const int u0 = i - c.s * p.units;
  int nu = i_end - i;
  if (nu > ct / tpu) nu = ct / tpu;
  if (nu > p.units - u0) nu = p.units - u0;
  c.nu = nu;
  c.t0 = u0 * tpu;
  c.tc = nu * tpu;
  c.gb = int(int64_t(p.G) * c.s / p.ks);
  c.ge = int(int64_t(p.G) * (c.s + 1) / p.ks);
}

// The CTA's sequence of stages: for each chunk, its groups in blocks of
// kWarps. Every warp walks the same sequence; lane 0 of each warp also keeps
// a second cursor S stages ahead, for the refill it may have to issue.
// gbase < 0 once the sequence is exhausted.
struct StageCursor {
  Chunk c;
  int gbase;   // first group of the stage
  __device__ __forceinline__ bool done() const { return gbase < 0; }
};

__device__ __forceinline__ void cursor_init(const GemvParams& p, int ct, int tpu, int i0, int i1, StageCursor& u) {
  load_chunk(p, ct, tpu, i0, i1, u.c);
  u.gbase = u.c.gb;
}

__device__ __forceinline__ void cursor_next(const GemvParams& p, int ct, int tpu, int i_end, StageCursor& u) {
  u.gbase += kWarps;
  if (u.gbase >= u.c.ge) {
    const int ni = u.c.i + u.c.nu;
    if (ni >= i_end) {
      u.gbase = -1;
    } else {
      load_chunk(p, ct, tpu, ni, i_end, u.c);
      u.gbase = u.c.gb;
    }
  }
}

template <bool ZP, bool PZ>
__device__ __forceinline__ uint32_t stage_tx_bytes(const GemvParams& p, int tc) {
  return uint32_t(tc * kTileStageBytes + kMetaStageBytes + (ZP ? (PZ ? kPackedZeroStageBytes : kMetaStageBytes) : 0) +
                  p.M * kXStageBytesPerRow);
}

// Two integers 0..15 in the halves of v -> the same two values as fp16:
// 0x6400 | q is exactly 1024 + q, less 1024.
__device__ __forceinline__ uint32_t small_ints_to_half2(uint32_t v) {
  uint32_t r;
  asm("sub.f16x2 %0, %1, %2;" : "=r"(r) : "r"(v | 0x64006400u), "r"(0x64006400u));
  return r;
}

__device__ __forceinline__ uint2 lds64(const uint8_t* p) { return *reinterpret_cast<const uint2*>(p); }

// The codes of a stage as one 4-D box per tile count: a view of qweight as
// {16 words, 16 rows, G groups, N/16 tiles} whose boxes of 16 x 16 x 8 x tc
// land tile-major then group-major, the same layout as tc boxes of the 3-D
// view. Used when N is a multiple of 16 (the view then covers exactly the
// array).
struct CodeMaps {
  CUtensorMap by_tiles[kChunkTiles];   // box of 1, 2, 3, 4 tiles
};

// Copies of the weight part of a stage: the codes of its tiles (one 4-D box,
// or one 3-D box of 16 words x 16 rows x 8 groups per tile, landing
// group-major), and the 64-row runs of scales and zero points of the 8 groups
// (packed zero points: 12 words x 8 groups from word 2 t0 rounded down to a
// multiple of 4, so the box starts on a 16-byte boundary).
template <bool ZP, bool PZ>
__device__ __forceinline__ void issue_weights(const StageCursor& u, uint8_t* st, uint64_t* bar,
                                              const CUtensorMap* tq, const CUtensorMap* ts,
                                              const CUtensorMap* tz, int p_scale_offset, const CodeMaps* cq) {
  const int r0 = u.c.t0 * kTile;
  if (cq) {
    tma_load_4d(st, &cq->by_tiles[u.c.tc - 1], 0, 0, u.gbase, u.c.t0, bar);
  } else {
    for (int r = 0; r < u.c.tc; ++r) tma_load_3d(st + r * kTileStageBytes, tq, 0, r0 + r * kTile, u.gbase, bar);
  }
  tma_load_2d(st + p_scale_offset, ts, r0, u.gbase, bar);
  if (ZP) {
    if (PZ) tma_load_2d(st + p_scale_offset + kMetaStageBytes, tz, (2 * u.c.t0) & ~3, u.gbase, bar);
    else tma_load_2d(st + p_scale_offset + kMetaStageBytes, tz, r0, u.gbase, bar);
  }
}

// Per-warp state of the stage pipeline.
template <int MT>
struct Pipe {
  uint8_t* ring;
  uint64_t* full;
  uint32_t* released;
  uint32_t* fills;
  uint32_t* failed;
  const CUtensorMap* tq;
  const CUtensorMap* tx;
  const CUtensorMap* ts;
  const CUtensorMap* tz;
  const CodeMaps* cq;  // null: per-tile 3-D boxes
  StageCursor pc;      // lane 0: the stage S ahead of the arithmetic
  int slot;
  uint32_t phase;
  bool ok;
  int S, i1;
  int lane, w, g, t;
  int zsh;             // 4 g: this lane's nibble in a packed zero-point word
  int xoff[MT];
  bool xok[MT];
  uint32_t ca0, ca2;
};

// The stages of one chunk: wait for a stage, take this warp's group into
// registers, release the stage (the last warp refills it), then decode and
// multiply into acc. All TC tile slots are computed, so the unrolled loops
// carry no branches; in a chunk with fewer tiles the extra slots hold stale
// shared memory and their rows are never stored.
template <int MT, bool ZP, bool PZ, int TC, int TPU>
__device__ __forceinline__ void chunk_stages(const GemvParams& p, Pipe<MT>& pp, const Chunk& cc,
                                             float (&acc)[kChunkTiles][MT][4], volatile int* abort_flag) {
    for (int gbase = cc.gb; gbase < cc.ge; gbase += kWarps) {
      if (pp.ok) {
        pp.ok = __all_sync(0xffffffffu, wait_bounded(&pp.full[pp.slot], pp.phase, abort_flag, &g_awq_gemv_error, 2u));
        if (!pp.ok && pp.lane == 0) atomicOr(pp.failed, 1u);
      }
      const uint8_t* st = pp.ring + pp.slot * p.stage_bytes;
      const bool has = pp.ok && gbase + pp.w < cc.ge;   // this warp's group of the stage
      uint4 xf[MT][4];
      uint4 c_lo[kChunkTiles], c_hi[kChunkTiles];
      uint32_t s2[kChunkTiles], z2[kChunkTiles];
      if (has) {
        // the unit's data, into registers: codes of rows g and g+8 of each
        // tile; scales and zero points of the same two rows as fp16 pairs
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) xf[mt][jj] = pp.xok[mt] ? lds128(st + pp.xoff[mt] + jj * 16) : make_uint4(0, 0, 0, 0);
        const uint8_t* cw = st + pp.w * (kTile * 64) + pp.g * 64 + pp.t * 16;
        const uint8_t* sw = st + p.scale_offset + pp.w * 128 + pp.g * 2;
        // packed zero points: rows g and g + 8 of tile rt are nibble g of
        // words 2 rt and 2 rt + 1 past the chunk's first word
        const uint8_t* zw = st + p.scale_offset + kMetaStageBytes + pp.w * (kPackedZeroWords * 4) + (cc.t0 & 1) * 8;
#pragma unroll
        for (int rt = 0; rt < TC; ++rt) {
          c_lo[rt] = lds128(cw + rt * kTileStageBytes);
          c_hi[rt] = lds128(cw + rt * kTileStageBytes + 8 * 64);
          s2[rt] = uint32_t(lds16(sw + rt * 32)) | (uint32_t(lds16(sw + rt * 32 + 16)) << 16);
          if constexpr (PZ) {
            const uint2 zz = lds64(zw + rt * 8);
            z2[rt] = small_ints_to_half2(((zz.x >> pp.zsh) & 0xFu) | (((zz.y >> pp.zsh) & 0xFu) << 16));
          } else {
            z2[rt] = ZP ? (uint32_t(lds16(sw + kMetaStageBytes + rt * 32)) |
                           (uint32_t(lds16(sw + kMetaStageBytes + rt * 32 + 16)) << 16))
                        : 0x48004800u;   // 8.0 in both halves
          }
        }
      }
      // Release the stage; the last of the CTA's warps to do so refills it
      // with the stage S ahead.
      __syncwarp();
      if (pp.lane == 0 && pp.ok) {
        uint32_t before;
        asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;"
                     : "=r"(before) : "r"(smem_u32(&pp.released[pp.slot])) : "memory");
        if (before == kWarps - 1) {
          pp.released[pp.slot] = 0u;
          if (!pp.pc.done()) {
            fence_proxy_async_smem();
            uint8_t* dst = pp.ring + pp.slot * p.stage_bytes;
            mbar_arrive_expect_tx(&pp.full[pp.slot], stage_tx_bytes<ZP, PZ>(p, pp.pc.c.tc));
            issue_weights<ZP, PZ>(pp.pc, dst, &pp.full[pp.slot], pp.tq, pp.ts, pp.tz, p.scale_offset, pp.cq);
            tma_load_3d(dst + p.x_offset, pp.tx, 0, pp.pc.gbase, 0, &pp.full[pp.slot]);
            pp.fills[pp.slot] += 1u;
          }
        }
        cursor_next(p, TC, TPU, pp.i1, pp.pc);
      }

      if (has) {
        float grp[kChunkTiles][MT][4];
        float cs[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            cs[mt][i] = 0.0f;
#pragma unroll
            for (int rt = 0; rt < TC; ++rt) grp[rt][mt][i] = 0.0f;
          }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            mma_16816(cs[mt], pp.ca0, 0u, pp.ca2, 0u, xf[mt][jj].x, xf[mt][jj].y);
            mma_16816(cs[mt], pp.ca0, 0u, pp.ca2, 0u, xf[mt][jj].z, xf[mt][jj].w);
          }
#pragma unroll
          for (int rt = 0; rt < TC; ++rt) {
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
          cm[mt][0] = __shfl_sync(0xffffffffu, cs[mt][0], pp.t);
          cm[mt][1] = __shfl_sync(0xffffffffu, cs[mt][1], pp.t);
          sm[mt][0] = __shfl_sync(0xffffffffu, cs[mt][0], 4 + pp.t);
          sm[mt][1] = __shfl_sync(0xffffffffu, cs[mt][1], 4 + pp.t);
        }
        // sum_k x (q - z) = raw - C(m) - z S(m); then the group's scale
#pragma unroll
        for (int rt = 0; rt < TC; ++rt) {
          const float s_lo = half_bits_to_float(uint16_t(s2[rt])), s_hi = half_bits_to_float(uint16_t(s2[rt] >> 16));
          const float z_lo = half_bits_to_float(uint16_t(z2[rt])), z_hi = half_bits_to_float(uint16_t(z2[rt] >> 16));
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            acc[rt][mt][0] = fmaf(s_lo, fmaf(-z_lo, sm[mt][0], grp[rt][mt][0] - cm[mt][0]), acc[rt][mt][0]);
            acc[rt][mt][1] = fmaf(s_lo, fmaf(-z_lo, sm[mt][1], grp[rt][mt][1] - cm[mt][1]), acc[rt][mt][1]);
            acc[rt][mt][2] = fmaf(s_hi, fmaf(-z_hi, sm[mt][0], grp[rt][mt][2] - cm[mt][0]), acc[rt][mt][2]);
            acc[rt][mt][3] = fmaf(s_hi, fmaf(-z_hi, sm[mt][1], grp[rt][mt][3] - cm[mt][1]), acc[rt][mt][3]);
          }
        }
      }
      if (++pp.slot == pp.S) {
        pp.slot = 0;
        pp.phase ^= 1u;
      }
    }

}

// One CTA's work: items [i0, i1) in chunks of at most TC tiles. SILU: the
// fused gate/up epilogue (AWQ_FLAG_SILU_MUL; units are tile pairs). PZ:
// packed zero points (AWQ_FLAG_PACKED_ZEROS, asymmetric only).
template <int MT, bool ZP, bool PZ, int TC, bool SILU>
__device__ __forceinline__ void gemv_cta(const CUtensorMap& tmap_q, const CUtensorMap& tmap_x,
                                         const CUtensorMap& tmap_s, const CUtensorMap& tmap_z,
                                         const CodeMaps& code_maps, const GemvParams& p, const int i0,
                                         const int i1) {
  extern __shared__ __align__(1024) uint8_t gemv_smem[];
  constexpr int TPU = SILU ? 2 : 1;   // tiles per work unit

  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int S = p.stages;
  const int M = p.M;
  uint64_t* full = reinterpret_cast<uint64_t*>(gemv_smem);                        // [S]
  uint32_t* released = reinterpret_cast<uint32_t*>(gemv_smem + kMaxStages * 8);   // [S] warps done with a fill
  uint32_t* fills = released + kMaxStages;                                        // [S] fills issued
  uint32_t* failed = fills + kMaxStages;                                          // a warp gave up
  uint8_t* ring = gemv_smem + kRingOffset;
  float* pbuf = reinterpret_cast<float*>(gemv_smem + p.pbuf_offset);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      released[s] = 0u;
      fills[s] = 0u;
    }
    *failed = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
  }
  __syncthreads();

  // ---- the first S stages (weights possibly before the dependency wait)
  StageCursor pc;   // lane 0 of every warp: the stage S ahead of the arithmetic
  if (lane == 0) cursor_init(p, TC, TPU, i0, i1, pc);
  if (threadIdx.x == 0) {
    if (p.early) {
      StageCursor u = pc;
      for (int s = 0; s < S && !u.done(); ++s) {
        mbar_arrive_expect_tx(&full[s], stage_tx_bytes<ZP, PZ>(p, u.c.tc));
        issue_weights<ZP, PZ>(u, ring + s * p.stage_bytes, &full[s], &tmap_q, &tmap_s, &tmap_z, p.scale_offset, p.codes4d ? &code_maps : nullptr);
        cursor_next(p, TC, TPU, i1, u);
      }
    } else {
      tma_prefetch_l2_3d(&tmap_q, 0, pc.c.t0 * kTile, pc.gbase);
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (lane == 0) {
    for (int s = 0; s < S && !pc.done(); ++s) {
      if (w == 0) {
        uint8_t* st = ring + s * p.stage_bytes;
        if (!p.early) {
          mbar_arrive_expect_tx(&full[s], stage_tx_bytes<ZP, PZ>(p, pc.c.tc));
          issue_weights<ZP, PZ>(pc, st, &full[s], &tmap_q, &tmap_s, &tmap_z, p.scale_offset, p.codes4d ? &code_maps : nullptr);
        }
        tma_load_3d(st + p.x_offset, &tmap_x, 0, pc.gbase, 0, &full[s]);
        fills[s] = 1u;
      }
      cursor_next(p, TC, TPU, i1, pc);
    }
  }

  volatile int abort_flag = 0;
  Pipe<MT> pp;
  pp.ring = ring;
  pp.full = full;
  pp.released = released;
  pp.fills = fills;
  pp.failed = failed;
  pp.tq = &tmap_q;
  pp.tx = &tmap_x;
  pp.ts = &tmap_s;
  pp.tz = &tmap_z;
  pp.cq = p.codes4d ? &code_maps : nullptr;
  pp.pc = pc;
  pp.slot = 0;
  pp.phase = 0;
  pp.ok = true;
  pp.S = S;
  pp.i1 = i1;
  pp.lane = lane;
  pp.w = w;
  pp.g = g;
  pp.t = t;
  pp.zsh = 4 * g;
  // x fragment offsets inside a stage ([m][8 groups][128 k]): batch row
  // m = 8 mt + g, this warp's group, chunk 4t + jj
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int m = 8 * mt + g;
    pp.xok[mt] = m < M;
    pp.xoff[mt] = p.x_offset + (m * kWarps + w) * 256 + t * 64;
  }
  offset_tile(g, pp.ca0, pp.ca2);

  Chunk cc;
  load_chunk(p, TC, TPU, i0, i1, cc);
  for (int chunk = 0;; ++chunk) {
    const int tc = cc.tc;
    float acc[kChunkTiles][MT][4];
#pragma unroll
    for (int rt = 0; rt < kChunkTiles; ++rt)
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[rt][mt][i] = 0.0f;

    chunk_stages<MT, ZP, PZ, TC, TPU>(p, pp, cc, acc, &abort_flag);

    // ---- chunk reduction: the 8 warps' partial sums meet in shared memory
    // ([warp][row][m], double-buffered by chunk parity) and are summed in
    // warp order, so the result does not depend on timing.
    float* pw = pbuf + ((chunk & 1) * kWarps + w) * (kChunkRows * M);
#pragma unroll
    for (int rt = 0; rt < kChunkTiles; ++rt)
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int m0 = 8 * mt + 2 * t;
        const int r_lo = 16 * rt + g, r_hi = r_lo + 8;
        if (rt < tc) {
          if (m0 < M) {
            pw[r_lo * M + m0] = acc[rt][mt][0];
            pw[r_hi * M + m0] = acc[rt][mt][2];
          }
          if (m0 + 1 < M) {
            pw[r_lo * M + m0 + 1] = acc[rt][mt][1];
            pw[r_hi * M + m0 + 1] = acc[rt][mt][3];
          }
        }
      }
    named_barrier_sync(kReduceBarrier, kThreads);
    const float* pb0 = pbuf + (chunk & 1) * kWarps * (kChunkRows * M);
    const int64_t row0 = int64_t(cc.t0) * kTile;
    if (TPU == 1 || p.ks > 1) {
      const int V = kTile * tc * M;
      for (int v = threadIdx.x; v < V; v += kThreads) {
        float sum = 0.0f;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) sum += pb0[ww * (kChunkRows * M) + v];
        const int row = v / M;
        const int m = v - row * M;
        if (p.ks == 1) {
          if (row0 + row < p.N) p.y[int64_t(m) * p.N + row0 + row] = __half_as_ushort(__float2half_rn(sum));
        } else {
          __stcg(p.partials + ((int64_t(cc.s) * p.T * kTile + row0 + row) * M + m), sum);
        }
      }
    } else if constexpr (SILU) {
      // fused gate/up: tile 2q of the chunk holds gate rows, tile 2q + 1 the
      // matching up rows; y has N / 2 columns
      const int V = kTile * (tc / 2) * M;
      for (int v = threadIdx.x; v < V; v += kThreads) {
        const int q = v / (kTile * M);
        const int rem = v - q * (kTile * M);   // row * M + m inside the pair
        const int vg = 2 * q * kTile * M + rem;
        float g = 0.0f, u = 0.0f;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) {
          g += pb0[ww * (kChunkRows * M) + vg];
          u += pb0[ww * (kChunkRows * M) + vg + kTile * M];
        }
        const int row = rem / M;
        const int m = rem - row * M;
        p.y[int64_t(m) * (p.N / 2) + row0 / 2 + q * kTile + row] =
            __half_as_ushort(__float2half_rn(silu_f32(g) * u));
      }
    }
    if (p.ks > 1) {
      // Slices of a unit meet in the workspace: the CTA that brings a unit's
      // arrival count to ks sums the ks partials in slice order.
      __threadfence();
      named_barrier_sync(kReduceBarrier, kThreads);
      if (w < cc.nu) {
        const int unit = cc.t0 / TPU + w;
        uint32_t last = 0;
        if (lane == 0) {
          uint32_t old;
          asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                       : "=r"(old) : "l"(p.counters + unit) : "memory");
          last = (old + 1 == uint32_t(p.ks)) ? 1u : 0u;
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        __syncwarp();   // lane 0's acquire orders the warp's partial reads
        if (last) {
          const int64_t trow = int64_t(unit) * TPU * kTile;
          if constexpr (TPU == 1) {
            for (int v = lane; v < kTile * M; v += 32) {
              float sum = 0.0f;
              for (int s = 0; s < p.ks; ++s)
                sum += __ldcg(p.partials + ((int64_t(s) * p.T * kTile + trow) * M + v));
              const int row = v / M;
              const int m = v - row * M;
              if (trow + row < p.N) p.y[int64_t(m) * p.N + trow + row] = __half_as_ushort(__float2half_rn(sum));
            }
          } else if constexpr (SILU) {
            for (int v = lane; v < kTile * M; v += 32) {
              float g = 0.0f, u = 0.0f;
              for (int s = 0; s < p.ks; ++s) {
                const float* ps = p.partials + (int64_t(s) * p.T * kTile + trow) * M;
                g += __ldcg(ps + v);
                u += __ldcg(ps + kTile * M + v);
              }
              const int row = v / M;
              const int m = v - row * M;
              p.y[int64_t(m) * (p.N / 2) + trow / 2 + row] = __half_as_ushort(__float2half_rn(silu_f32(g) * u));
            }
          }
          if (lane == 0) p.counters[unit] = 0u;
        }
      }
    }
    const int ni = cc.i + cc.nu;
    if (ni >= i1) break;
    load_chunk(p, TC, TPU, ni, i1, cc);
  }

  // If a warp gave up, copies may still be in flight: a slot is refilled
  // only after every warp has taken its previous fill, so at most its latest
  // fill is pending; thread 0 waits (bounded) for it before the CTA exits.
  __syncthreads();
  if (threadIdx.x == 0 && *reinterpret_cast<volatile uint32_t*>(failed)) {
    for (int s = 0; s < S; ++s)
      if (fills[s] > 0u) wait_teardown(&full[s], (fills[s] - 1u) & 1u);
  }
}

template <int MT, bool ZP, bool PZ, int TC, bool SILU>
__global__ void __launch_bounds__(kThreads, MT == 1 ? 2 : 1)
gemv_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_x,
            const __grid_constant__ CUtensorMap tmap_s, const __grid_constant__ CUtensorMap tmap_z,
            const __grid_constant__ CodeMaps code_maps, const GemvParams p) {
  // Let the next kernel in the stream (if launched as a programmatic
  // dependent) start as soon as every CTA of this one is running; it waits
  // for this grid's completion before it reads anything this grid writes.
  asm volatile("griddepcontrol.launch_dependents;");
  const int i0 = int(int64_t(p.items) * blockIdx.x / gridDim.x);
  const int i1 = int(int64_t(p.items) * (blockIdx.x + 1) / gridDim.x);
  // A CTA with exactly 3 items of one K slice runs 3-tile chunks instead of
  // padding a 4-tile chunk (896 tiles on 296 CTAs: 288 CTAs hold 3). The
  // arithmetic of the stream phase is the limit, and the two CTAs of an SM
  // share it, so an SM with 3 + 4 tiles finishes sooner than with 4 + 4.
  if constexpr (TC == 4 && !SILU) {
    if (i1 - i0 == 3 && i0 / p.units == (i1 - 1) / p.units) {
      gemv_cta<MT, ZP, PZ, 3, false>(tmap_q, tmap_x, tmap_s, tmap_z, code_maps, p, i0, i1);
      return;
    }
  }
  gemv_cta<MT, ZP, PZ, TC, SILU>(tmap_q, tmap_x, tmap_s, tmap_z, code_maps, p, i0, i1);
}

// ---------------------------------------------------------------------------
// host side: plan (variant, decomposition, ring geometry, workspace) for a shape
// ---------------------------------------------------------------------------
using KernelFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                          const CodeMaps, const GemvParams);

struct Variant {
  KernelFn fn;
  int mt, id;
};

constexpr int kNumVariants = 24;
constexpr int kSmemBudget = 232448;   // largest dynamic shared memory of one sm_100 CTA
constexpr int kHalfSmBudget = 115712; // half of an SM's 228 KB, less the 1 KB reserved per CTA

// zp: 0 symmetric, 1 fp16 zero points, 2 packed zero points
Variant pick_variant(int64_t M, int zp, int tc, bool silu) {
  static const Variant table[kNumVariants] = {
      {gemv_kernel<1, true, false, 4, false>, 1, 0},  {gemv_kernel<1, false, false, 4, false>, 1, 1},
      {gemv_kernel<2, true, false, 4, false>, 2, 2},  {gemv_kernel<2, false, false, 4, false>, 2, 3},
      {gemv_kernel<1, true, false, 2, false>, 1, 4},  {gemv_kernel<1, false, false, 2, false>, 1, 5},
      {gemv_kernel<2, true, false, 2, false>, 2, 6},  {gemv_kernel<2, false, false, 2, false>, 2, 7},
      {gemv_kernel<1, true, false, 4, true>, 1, 8},   {gemv_kernel<1, false, false, 4, true>, 1, 9},
      {gemv_kernel<2, true, false, 4, true>, 2, 10},  {gemv_kernel<2, false, false, 4, true>, 2, 11},
      {gemv_kernel<1, true, false, 2, true>, 1, 12},  {gemv_kernel<1, false, false, 2, true>, 1, 13},
      {gemv_kernel<2, true, false, 2, true>, 2, 14},  {gemv_kernel<2, false, false, 2, true>, 2, 15},
      {gemv_kernel<1, true, true, 4, false>, 1, 16},  {gemv_kernel<2, true, true, 4, false>, 2, 17},
      {gemv_kernel<1, true, true, 2, false>, 1, 18},  {gemv_kernel<2, true, true, 2, false>, 2, 19},
      {gemv_kernel<1, true, true, 4, true>, 1, 20},   {gemv_kernel<2, true, true, 4, true>, 2, 21},
      {gemv_kernel<1, true, true, 2, true>, 1, 22},   {gemv_kernel<2, true, true, 2, true>, 2, 23}};
  if (zp == 2) return table[16 + (silu ? 4 : 0) + (tc == 2 ? 2 : 0) + (M <= 8 ? 0 : 1)];
  return table[(silu ? 8 : 0) + (tc == 2 ? 4 : 0) + (M <= 8 ? 0 : 2) + (zp ? 0 : 1)];
}

int round128(int v) { return (v + 127) / 128 * 128; }

struct Plan {
  Variant v;
  int grid, T, tpu, units, ks, items, tc, scale_offset;
  int stages, stage_bytes, x_offset, pbuf_offset, smem;
  size_t counter_bytes, partial_bytes;
};

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<int> g_smem_attr[kMaxDevices][kNumVariants];

// zp: 0 symmetric, 1 fp16 zero points, 2 packed zero points
awq_status_t make_plan(int64_t M, int64_t N, int64_t K, int zp, bool silu, Plan& pl) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return AWQ_ERR_UNSUPPORTED;
  int sms = g_sm_count[dev].load(std::memory_order_relaxed);
  if (sms == 0) {
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return AWQ_ERR_CUDA;
    g_sm_count[dev].store(sms, std::memory_order_relaxed);
  }
  // Decomposition: whole tiles per CTA over all of K, with as many CTAs as
  // fill the GPU: two half-SM CTAs per SM for M <= 8 (16 warps hide more
  // latency), one otherwise, or when half an SM cannot hold two stages. K is
  // cut into slices only when there are fewer tiles than CTAs.
  const int64_t G = K / kGroup;
  const int64_t T = (N + kTile - 1) / kTile;
  const int tpu = silu ? 2 : 1;          // a fused gate/up unit is a gate tile and its up tile
  const int64_t U = T / tpu;
  const int pbuf_bytes = 2 * kWarps * kChunkRows * int(M) * 4;
  for (int per_sm = M <= 8 ? 2 : 1;; --per_sm) {
    const int64_t want = int64_t(per_sm) * sms;
    int64_t ks = 1;
    if (U < want) {
      ks = (want + U - 1) / U;
      if (ks > G) ks = G;
    }
    pl.T = int(T);
    pl.tpu = tpu;
    pl.units = int(U);
    pl.ks = int(ks);
    pl.items = int(U * ks);
    pl.grid = int(pl.items < want ? pl.items : want);
    // Chunks of 4 tiles, or of 2 when no CTA has more than 2 items: the CTA
    // with the most items sets the kernel's time, and it then wastes no slot.
    const int64_t most = (int64_t(pl.items) + pl.grid - 1) / pl.grid;
    pl.tc = most * tpu <= 2 ? 2 : kChunkTiles;
    // Ring geometry: as many stages as the budget holds after the reduction buffers.
    pl.scale_offset = pl.tc * kTileStageBytes;
    pl.x_offset = pl.scale_offset + kMetaStageBytes + (zp == 2 ? kPackedZeroStageBytes : zp ? kMetaStageBytes : 0);
    pl.stage_bytes = round128(pl.x_offset + int(M) * kXStageBytesPerRow);
    const int budget = per_sm == 2 ? kHalfSmBudget : kSmemBudget;
    const int st = (budget - kRingOffset - pbuf_bytes) / pl.stage_bytes;
    pl.stages = st > kMaxStages ? kMaxStages : st;
    if (pl.stages >= 2 || per_sm == 1) break;
  }
  if (pl.stages < 2) return AWQ_ERR_UNSUPPORTED;
  pl.v = pick_variant(M, zp, pl.tc, silu);
  if (!g_smem_attr[dev][pl.v.id].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(pl.v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget) != cudaSuccess)
      return AWQ_ERR_CUDA;
    g_smem_attr[dev][pl.v.id].store(1, std::memory_order_release);
  }
  pl.pbuf_offset = kRingOffset + pl.stages * pl.stage_bytes;
  pl.smem = pl.pbuf_offset + pbuf_bytes;
  pl.counter_bytes = pl.ks > 1 ? ((size_t(T) * 4 + 255) / 256) * 256 : 0;
  pl.partial_bytes = pl.ks > 1 ? size_t(pl.ks) * size_t(T) * kTile * size_t(M) * 4 : 0;
  return AWQ_OK;
}

awq_status_t check_gemv_args(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                             const uint16_t* zeros, int64_t M, int64_t N, int64_t K,
                             awq_qconfig_t cfg, uint16_t* y) {
  awq_status_t st = check_cfg(cfg, true);
  if (st != AWQ_OK) return st;
  if ((st = check_nk(N, K)) != AWQ_OK) return st;
  if (M < 1 || M > 16) return AWQ_ERR_SHAPE;
  if (N % 8) return AWQ_ERR_SHAPE;
  if ((cfg.flags & AWQ_FLAG_SILU_MUL) && N % 32) return AWQ_ERR_SHAPE;
  if (cfg.flags & AWQ_FLAG_PACKED_ZEROS) {
    if (!cfg.zero_point) return AWQ_ERR_UNSUPPORTED;
    if (N % 32) return AWQ_ERR_SHAPE;   // a group row of qzeros is N/2 bytes, whole 16-byte runs
  }
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
awq_status_t gemv_workspace_bytes(int64_t M, int64_t N, int64_t K, int zp, bool silu, size_t* bytes) {
  if (N == 0) { *bytes = 0; return AWQ_OK; }
  Plan pl;
  awq_status_t st = make_plan(M, N, K, zp, silu, pl);
  if (st != AWQ_OK) return st;
  *bytes = pl.counter_bytes + pl.partial_bytes;
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
  const int zp = zero_mode(cfg);
  Plan pl;
  if ((st = make_plan(M, N, K, zp, (cfg.flags & AWQ_FLAG_SILU_MUL) != 0, pl)) != AWQ_OK) return st;
  GemvParams p;
  p.y = y;
  p.counters = nullptr;
  p.partials = nullptr;
  if (pl.ks > 1) {
    if (!workspace || workspace_bytes < pl.counter_bytes + pl.partial_bytes) return AWQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return AWQ_ERR_ALIGN;
    p.counters = static_cast<uint32_t*>(workspace);
    p.partials = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.counter_bytes);
  }
  const int G = int(K / kGroup);
  // codes: int32 [N][K/8] viewed as {16 words, N rows, G groups} (a group
  // steps 64 bytes, a row K/2 bytes), boxes of 16 x 16 x 8 that land
  // group-major; x: fp16 [M][K] viewed as {128 k, G groups, M rows}, boxes of
  // 128 x 8 x M; scales / zeros: fp16 [G][N], boxes of 64 rows x 8 groups;
  // packed zero points: int32 [G][N/8], boxes of 12 words x 8 groups.
  CUtensorMap tq, tx, ts, tz;
  if (!make_tensor_map_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_INT32, qweight, kWordsPerGroup, uint64_t(N),
                          uint64_t(G), uint64_t(K / 8) * 4, kWordsPerGroup * 4, kWordsPerGroup, kTile, kWarps) ||
      !make_tensor_map_3d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, kGroup, uint64_t(G), uint64_t(M),
                          kGroup * 2, uint64_t(K) * 2, kGroup, kWarps, uint32_t(M)) ||
      !make_tensor_map_2d(&ts, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, scales, uint64_t(N), uint64_t(G),
                          uint64_t(N) * 2, kChunkRows, kWarps, CU_TENSOR_MAP_SWIZZLE_NONE))
    return AWQ_ERR_CUDA;
  if (zp == 2) {
    if (!make_tensor_map_2d(&tz, CU_TENSOR_MAP_DATA_TYPE_INT32, zeros, uint64_t(N / 8), uint64_t(G),
                            uint64_t(N) / 2, kPackedZeroWords, kWarps, CU_TENSOR_MAP_SWIZZLE_NONE))
      return AWQ_ERR_CUDA;
  } else if (zp) {
    if (!make_tensor_map_2d(&tz, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, zeros, uint64_t(N), uint64_t(G),
                            uint64_t(N) * 2, kChunkRows, kWarps, CU_TENSOR_MAP_SWIZZLE_NONE))
      return AWQ_ERR_CUDA;
  } else {
    tz = ts;   // never read by the symmetric kernels
  }
  CodeMaps cq;
  p.codes4d = (N % kTile) == 0 ? 1 : 0;
  for (int tc = 1; tc <= kChunkTiles; ++tc) {
    if (p.codes4d) {
      const uint64_t row = uint64_t(K / 8) * 4;
      if (!make_tensor_map_4d(&cq.by_tiles[tc - 1], CU_TENSOR_MAP_DATA_TYPE_INT32, qweight, kWordsPerGroup,
                              kTile, uint64_t(G), uint64_t(N / kTile), row, kWordsPerGroup * 4, row * kTile,
                              kWordsPerGroup, kTile, kWarps, uint32_t(tc)))
        return AWQ_ERR_CUDA;
    } else {
      cq.by_tiles[tc - 1] = tq;   // never read
    }
  }
  p.M = int(M);
  p.N = int(N);
  p.G = G;
  p.T = pl.T;
  p.tpu = pl.tpu;
  p.units = pl.units;
  p.ks = pl.ks;
  p.items = pl.items;
  p.stages = pl.stages;
  p.stage_bytes = pl.stage_bytes;
  p.x_offset = pl.x_offset;
  p.pbuf_offset = pl.pbuf_offset;
  p.scale_offset = pl.scale_offset;
  p.early = (cfg.flags & AWQ_FLAG_WEIGHTS_STATIC) ? 1 : 0;
  // Programmatic dependent launch: this grid may start while the previous
  // kernel in the stream finishes; the kernel waits for it (griddepcontrol)
  // before it touches x, the workspace or y.
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(pl.grid);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = size_t(pl.smem);
  lc.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  if (cudaLaunchKernelEx(&lc, pl.v.fn, tq, tx, ts, tz, cq, p) != cudaSuccess) return AWQ_ERR_CUDA;
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

// The cached device address of g_gemv_scratch per device, with the context it
// was looked up in: a context that is torn down and created again (for
// example after cudaDeviceReset) maps the array elsewhere.
struct ScratchCache {
  std::mutex lock;
  CUcontext ctx = nullptr;
  uintptr_t addr = 0;
};
ScratchCache g_scratch[kMaxDevices];

PFN_cuCtxGetCurrent_v4000 ctx_getter() {
  static PFN_cuCtxGetCurrent_v4000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_cuCtxGetCurrent_v4000>(nullptr);
    return reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
  }();
  return fn;
}

// Device address of g_gemv_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up
// (with that device current) and cached per device and context.
awq_status_t scratch_address(int dev, void** out) {
  PFN_cuCtxGetCurrent_v4000 get = ctx_getter();
  CUcontext ctx = nullptr;
  if (!get || get(&ctx) != CUDA_SUCCESS) return AWQ_ERR_CUDA;
  ScratchCache& c = g_scratch[dev];
  std::lock_guard<std::mutex> g(c.lock);
  if (ctx == nullptr || c.addr == 0 || c.ctx != ctx) {
    // the lookup also makes the device's primary context current if it was not
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gemv_scratch) != cudaSuccess || p == nullptr) return AWQ_ERR_CUDA;
    if (get(&ctx) != CUDA_SUCCESS || ctx == nullptr) return AWQ_ERR_CUDA;
    c.addr = reinterpret_cast<uintptr_t>(p);
    c.ctx = ctx;
  }
  *out = reinterpret_cast<void*>(c.addr);
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
  if ((st = make_plan(M, N, K, zero_mode(cfg), (cfg.flags & AWQ_FLAG_SILU_MUL) != 0, pl)) != AWQ_OK)
    return st;
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
