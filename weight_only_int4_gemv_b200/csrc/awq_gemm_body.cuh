// Body of the W4A16 prefill GEMM for one output-channel tile width,
// included by awq_gemm.cu once per width with AWQ_GEMM_BN defined (256 or
// 128) inside its own namespace: constants, kernel, and the planner /
// launcher `run`. See awq_gemm.cu for the design.
// (no include guard: included twice on purpose)

#ifndef AWQ_GEMM_BN
#error "define AWQ_GEMM_BN (256 or 128) before including awq_gemm_body.cuh"
#endif

namespace {

#ifndef AWQ_GEMM_BM
#define AWQ_GEMM_BM 256
#endif
constexpr int BM = AWQ_GEMM_BM;         // rows of x per tile: 256 (two MMAs of M = 128) or 128
constexpr int BMH = 128;                // rows of one MMA
constexpr int BN = AWQ_GEMM_BN;         // output channels per tile (MMA N): 256 or 128
constexpr int BK = 64;                  // k per stage (one 128-byte swizzle row of fp16)
constexpr int kStages = BN == 256 ? 3 : (BM == 256 ? 4 : 6);
constexpr int kDecodeWarps = BN / 16;   // 2 threads per weight row
constexpr int kEpiWarp0 = kDecodeWarps; // 4 epilogue warps
constexpr int kTmaWarp = kEpiWarp0 + 4;
constexpr int kMmaWarp = kTmaWarp + 1;
constexpr int kGemmThreads = (kMmaWarp + 1) * 32;
constexpr int kAccCols = 2 * BN;        // one accumulator pair (two M halves)
constexpr int kAccBufs = 1;             // the pair fills tensor memory
constexpr int kTmemCols = kAccBufs * kAccCols;
static_assert(kDecodeWarps * 32 == 2 * BN, "two decode threads per weight row");
constexpr int kPartStride = BN + 4;
constexpr int kMaxSlices = 8;           // cluster size limit of the K-split path     // fp32 per row of a K-slice partial (16-byte pad: no bank conflicts)

constexpr int kABytes = BM * BK * 2;        // 32 KB of x
constexpr int kBBytes = BN * BK * 2;        // decoded W'
constexpr int kCBytes = BN * (BK / 8) * 4;  // packed codes
constexpr int kSmemTiles = kStages * (kABytes + kBBytes + kCBytes);
constexpr int kSmemBytes = kSmemTiles + 1024 /*barriers*/ + 1024 /*alignment*/;

// instruction descriptor: F16 x F16 -> F32, both K-major, M = 128, N = BN
constexpr uint32_t kIdesc = (1u << 4) | (uint32_t(BN >> 3) << 17) | (uint32_t(BMH >> 4) << 24);

struct SmemLayout {
  // offsets from the 1024-aligned base
  static constexpr int a(int s) { return s * kABytes; }
  static constexpr int b(int s) { return kStages * kABytes + s * kBBytes; }
  static constexpr int c(int s) { return kStages * (kABytes + kBBytes) + s * kCBytes; }
  static constexpr int bar = kSmemTiles;
};

struct Bars {
  uint64_t full_a[kStages];    // TMA bytes of x + codes landed
  uint64_t full_b[kStages];    // decoded W' tile written (8 warp arrivals)
  uint64_t empty[kStages];     // MMAs that read the stage finished
  uint64_t tmem_full[kAccBufs];    // accumulator complete
  uint64_t tmem_empty[kAccBufs];   // accumulator drained (4 warp arrivals)
  uint64_t mma_done;           // final commit before teardown
  uint32_t tmem_base;
  int abort;
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 8 consecutive fp32 columns
__device__ __forceinline__ void tc_ld_32x32b_x8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive fp32 columns
__device__ __forceinline__ void tc_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// 16 bytes of CTA `rank`'s shared memory at the offset `saddr` has in this CTA
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t saddr, int rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(saddr), "r"(rank));
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a) : "memory");
  return v;
}

// Sum of the float4 at shared-memory offset `saddr` over CTAs 0 .. S-1 of
// the cluster: all S loads in flight at once, then added in slice order (so
// the bits do not depend on timing).
__device__ __forceinline__ float4 sum_slices_dsmem(uint32_t saddr, int S) {
  float4 v[kMaxSlices];
#pragma unroll
  for (int sl = 0; sl < kMaxSlices; ++sl)
    if (sl < S) v[sl] = ld_dsmem_f4(saddr, sl);
  float4 acc = v[0];
#pragma unroll
  for (int sl = 1; sl < kMaxSlices; ++sl)
    if (sl < S) {
      acc.x += v[sl].x;
      acc.y += v[sl].y;
      acc.z += v[sl].z;
      acc.w += v[sl].w;
    }
  return acc;
}

// Two such sums at once (the gate and up values of the fused epilogue), in
// the same slice order, two slices per step so that no more than eight
// float4 loads are live (all slices of both at once would spill).
__device__ __forceinline__ void sum_slices_dsmem2(uint32_t sa, uint32_t sb, int S, float4& a, float4& b) {
  a = ld_dsmem_f4(sa, 0);
  b = ld_dsmem_f4(sb, 0);
#pragma unroll 1
  for (int sl = 1; sl < S; sl += 2) {
    const float4 a1 = ld_dsmem_f4(sa, sl), b1 = ld_dsmem_f4(sb, sl);
    float4 a2 = make_float4(0.f, 0.f, 0.f, 0.f), b2 = a2;
    if (sl + 1 < S) {
      a2 = ld_dsmem_f4(sa, sl + 1);
      b2 = ld_dsmem_f4(sb, sl + 1);
    }
    a.x += a1.x; a.y += a1.y; a.z += a1.z; a.w += a1.w;
    b.x += b1.x; b.y += b1.y; b.z += b1.z; b.w += b1.w;
    if (sl + 1 < S) {
      a.x += a2.x; a.y += a2.y; a.z += a2.z; a.w += a2.w;
      b.x += b2.x; b.y += b2.y; b.z += b2.z; b.w += b2.w;
    }
  }
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), sm100 descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return uint64_t((saddr >> 4) & 0x3FFF) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Scale and zero point of one weight row, loaded kMetaAhead groups before
// their use through a register shift chain: the global-load latency (over a
// microsecond under load) stays off the k loop, which otherwise waits for it
// at every group.
constexpr int kMetaAhead = 4;

template <bool ZP>
struct MetaChain {
  const uint16_t* scol;
  const uint16_t* zcol;
  int64_t N;
  int G;
  bool valid;
  uint16_t s0, s1, s2, s3, z0, z1, z2, z3;   // groups g .. g + 3

  __device__ __forceinline__ uint16_t load(const uint16_t* col, int g) const {
    return (valid && g < G) ? ld_nc_u16(col + int64_t(g) * N) : uint16_t(0);
  }
  __device__ __forceinline__ void start(int g0) {
    s0 = load(scol, g0);
    s1 = load(scol, g0 + 1);
    s2 = load(scol, g0 + 2);
    s3 = load(scol, g0 + 3);
    if (ZP) {
      z0 = load(zcol, g0);
      z1 = load(zcol, g0 + 1);
      z2 = load(zcol, g0 + 2);
      z3 = load(zcol, g0 + 3);
    } else {
      z0 = z1 = z2 = z3 = 0;
    }
  }
  // group g's scale and zero bits; group g + kMetaAhead is requested
  __device__ __forceinline__ void next(int g, uint16_t& sb, uint16_t& zb) {
    sb = s0;
    zb = z0;
    s0 = s1;
    s1 = s2;
    s2 = s3;
    s3 = load(scol, g + kMetaAhead);
    if (ZP) {
      z0 = z1;
      z1 = z2;
      z2 = z3;
      z3 = load(zcol, g + kMetaAhead);
    }
  }
};

struct GemmParams {
  uint16_t* y;
  const uint16_t* scales;
  const uint16_t* zeros;
  int M, N, K, G;
  int m_tiles, n_tiles, k_blocks;
  int tile0, num_tiles;   // this launch takes tiles tile0 .. tile0 + num_tiles - 1
  int silu;               // AWQ_FLAG_SILU_MUL: 16-channel tiles alternate gate, up; y has N / 2 columns
  int S;            // K slices per tile: 1 = persistent CTAs over whole tiles; 2, 4, 8 = one
                    // cluster of S CTAs per tile, CTA r of the cluster taking slice r
  int kb_per_unit;  // k blocks one CTA multiplies per tile (k_blocks / S)
};

template <bool ZP, bool SILU>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_q,
            const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + SmemLayout::bar);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = p.num_tiles;   // tile indices below are relative to p.tile0
  // work of this CTA: tiles t_first, t_first + t_step, ..., k blocks [kb0, kb1) of each
  const bool split = p.S > 1;
  const int t_first = split ? int(blockIdx.x) / p.S : int(blockIdx.x);
  const int t_step = split ? num_tiles : int(gridDim.x);
  const int kb0 = split ? (int(blockIdx.x) % p.S) * p.kb_per_unit : 0;
  const int kb1 = kb0 + p.kb_per_unit;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full_a[s], 1);
      mbar_init(&bars->full_b[s], kDecodeWarps);
      mbar_init(&bars->empty[s], 1);
    }
    for (int a = 0; a < kAccBufs; ++a) {
      mbar_init(&bars->tmem_full[a], 1);
      mbar_init(&bars->tmem_empty[a], 4);
    }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;

  if (warp < kDecodeWarps) {
    // ------------------------------------------------------------ decode
    const int i = threadIdx.x >> 1;  // row of the weight tile
    const int h = threadIdx.x & 1;   // which 32 k of the k block (words 4h .. 4h+3)
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int tile = t_first; tile < num_tiles && ok; tile += t_step) {
      const int n0 = ((tile + p.tile0) / p.m_tiles) * BN;
      const int64_t row = int64_t(n0) + i;
      const bool valid = row < p.N;
      // group-major metadata: consecutive threads read consecutive rows
      MetaChain<ZP> meta;
      meta.scol = p.scales + (valid ? row : 0);
      meta.zcol = ZP ? p.zeros + (valid ? row : 0) : nullptr;
      meta.N = p.N;
      meta.G = p.G;
      meta.valid = valid;
      meta.start(kb0 >> 1);   // kb0 is even: slices hold whole groups
      uint32_t zb1024 = 0, zb64 = 0, sc2 = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if ((kb & 1) == 0) {  // new group of 128 k
          uint16_t sb, zbits;
          meta.next(kb >> 1, sb, zbits);
          const float z = ZP ? half_bits_to_float(zbits) : 8.0f;
          zero_bias_pairs(z, zb1024, zb64);
          sc2 = uint32_t(sb) | (uint32_t(sb) << 16);
        }
        if (!wait_sleep(&bars->full_a[s], ph, abort, &g_awq_error_word, 1u)) { ok = false; break; }
        // codes of row i: 32 bytes, 16-byte halves swapped on rows with bit 2 set
        // (32B swizzle); this thread decodes half h
        const uint8_t* crow = smem + SmemLayout::c(s) + i * 32;
        const int sw = (i >> 2) & 1;
        const uint4 c = *reinterpret_cast<const uint4*>(crow + ((h ^ sw) << 4));
        uint8_t* brow = smem + SmemLayout::b(s) + i * 128;
        const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          uint32_t pq[4];
          decode_word_qz(words[w], zb1024, zb64, pq);
          uint4 v;
          v.x = hmul2_u32(pq[0], sc2);
          v.y = hmul2_u32(pq[1], sc2);
          v.z = hmul2_u32(pq[2], sc2);
          v.w = hmul2_u32(pq[3], sc2);
          *reinterpret_cast<uint4*>(brow + (((4 * h + w) ^ (i & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->full_b[s]);
        if (++s == kStages) { s = 0; ph ^= 1; }
      }
    }
  } else if (warp < kEpiWarp0 + 4) {
    // ------------------------------------------------------------ epilogue (whole tiles)
    const int q = warp - kEpiWarp0;            // TMEM lane quadrant (warp % 4)
    int it = 0;
    for (int tile = t_first; tile < num_tiles && !split; tile += t_step, ++it) {
      const int m0 = ((tile + p.tile0) % p.m_tiles) * BM;
      const int n0 = ((tile + p.tile0) / p.m_tiles) * BN;
      const int acc = it % kAccBufs;
      const uint32_t aph = (it / kAccBufs) & 1;
      if (!wait_sleep(&bars->tmem_full[acc], aph, abort, &g_awq_error_word, 1u)) break;
      tc_fence_after();
      const int halves = BM > BMH && m0 + BMH < p.M ? 2 : 1;   // the MMAs skip an upper half with no rows
#pragma unroll 1
      for (int c8 = 0; c8 < halves * (BN / 32); ++c8) {
        const int hm = c8 / (BN / 32);      // which 128 rows of x
        const int c = c8 % (BN / 32);       // which 32 output channels
        const int64_t m = int64_t(m0) + hm * BMH + q * 32 + lane;
        uint16_t* yrow = p.y + m * p.N;
        const uint32_t tcol = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * kAccCols + hm * BN + c * 32);
        const int nc = n0 + c * 32;
        if constexpr (SILU) {
          // columns nc .. nc+15: gate rows, nc+16 .. nc+31: the matching up
          // rows; eight of each at a time (fewer live registers)
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t gr[8], ur[8];
            tc_ld_32x32b_x8(tcol + hh * 8, gr);
            tc_ld_32x32b_x8(tcol + 16 + hh * 8, ur);
            if (m < p.M && nc < p.N) {
              uint32_t h[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float a = silu_f32(__uint_as_float(gr[2 * e])) * __uint_as_float(ur[2 * e]);
                const float b = silu_f32(__uint_as_float(gr[2 * e + 1])) * __uint_as_float(ur[2 * e + 1]);
                h[e] = uint32_t(__half_as_ushort(__float2half_rn(a))) |
                       (uint32_t(__half_as_ushort(__float2half_rn(b))) << 16);
              }
              reinterpret_cast<uint4*>(p.y + m * (p.N / 2) + nc / 2)[hh] = make_uint4(h[0], h[1], h[2], h[3]);
            }
          }
        } else {
          // (tcgen05.ld is warp-collective: every lane loads, whatever its row)
          uint32_t r[32];
          tc_ld_32x32b_x32(tcol, r);
          if (m < p.M && nc < p.N) {
            uint32_t h[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const uint32_t lo = __half_as_ushort(__float2half_rn(__uint_as_float(r[2 * e])));
              const uint32_t hi = __half_as_ushort(__float2half_rn(__uint_as_float(r[2 * e + 1])));
              h[e] = lo | (hi << 16);
            }
            if (nc + 32 <= p.N && (p.N & 7) == 0) {
              uint4* dst = reinterpret_cast<uint4*>(yrow + nc);
#pragma unroll
              for (int v = 0; v < 4; ++v) dst[v] = make_uint4(h[4 * v], h[4 * v + 1], h[4 * v + 2], h[4 * v + 3]);
            } else {
              for (int e = 0; e < 32 && nc + e < p.N; ++e)
                yrow[nc + e] = uint16_t((h[e >> 1] >> ((e & 1) * 16)) & 0xFFFF);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->tmem_empty[acc]);
    }
  } else if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      bool issued[kStages] = {};
      uint32_t issued_ph[kStages] = {};
      for (int tile = t_first; tile < num_tiles && ok; tile += t_step) {
        const int m0 = ((tile + p.tile0) % p.m_tiles) * BM;
        const int n0 = ((tile + p.tile0) / p.m_tiles) * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_sleep(&bars->empty[s], ph ^ 1, abort, &g_awq_error_word, 1u)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars->full_a[s], kABytes + kCBytes);
          tma_load_2d(smem + SmemLayout::a(s), &tmap_x, kb * BK, m0, &bars->full_a[s]);
          tma_load_2d(smem + SmemLayout::c(s), &tmap_q, kb * (BK / 8), n0, &bars->full_a[s]);
          issued[s] = true;
          issued_ph[s] = ph;
          if (++s == kStages) { s = 0; ph ^= 1; }
        }
      }
      // The copies still in flight land before the CTA's shared memory goes away.
      for (int t = 0; t < kStages; ++t)
        if (issued[t]) wait_teardown(&bars->full_a[t], issued_ph[t]);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      bool ok = true;
      for (int tile = t_first; tile < num_tiles && ok; tile += t_step, ++it) {
        const int acc = it % kAccBufs;
        const uint32_t aph = (it / kAccBufs) & 1;
        if (!wait_sleep(&bars->tmem_empty[acc], aph ^ 1, abort, &g_awq_error_word, 1u)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * kAccCols);
        const bool upper = BM > BMH && ((tile + p.tile0) % p.m_tiles) * BM + BMH < p.M;   // rows of x in the upper half
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_sleep(&bars->full_a[s], ph, abort, &g_awq_error_word, 1u) ||
              !wait_sleep(&bars->full_b[s], ph, abort, &g_awq_error_word, 1u)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + SmemLayout::a(s));
          const uint32_t b_addr = smem_u32(smem + SmemLayout::b(s));
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t bd = sw128_desc(b_addr + k * 32);
            const uint32_t accum = (kb > kb0 || k > 0) ? 1u : 0u;
            tc_mma_f16(d_tmem, sw128_desc(a_addr + k * 32), bd, kIdesc, accum);
            if (upper) tc_mma_f16(d_tmem + BN, sw128_desc(a_addr + BMH * 128 + k * 32), bd, kIdesc, accum);
          }
          tc_commit(&bars->empty[s]);
          if (++s == kStages) { s = 0; ph ^= 1; }
        }
        if (ok) tc_commit(&bars->tmem_full[acc]);
      }
      // every MMA this thread issued completes before tensor memory is freed
      tc_commit(&bars->mma_done);
      wait_teardown(&bars->mma_done, 0);
    }
  }

  if (split) {
    // ------------------------------------------------------------ K-slice reduction (all warps)
    // Each CTA of the cluster holds the fp32 partial of its K slice for the
    // tile. Per half of x: the epilogue warps copy the partial from tensor
    // memory into this CTA's shared memory (the stage area, idle once the
    // accumulator is complete); after a cluster barrier CTA r sums rows
    // [r 128/S, (r+1) 128/S) of every slice's partial, in slice order (so
    // the bits do not depend on timing), and stores them as fp16; a second
    // barrier keeps every partial in place until all CTAs have read it.
    const int tile = t_first;
    const int m0 = ((tile + p.tile0) % p.m_tiles) * BM;
    const int n0 = ((tile + p.tile0) / p.m_tiles) * BN;
    const int halves = BM > BMH && m0 + BMH < p.M ? 2 : 1;
    const int rank = int(blockIdx.x) % p.S;
    float* part = reinterpret_cast<float*>(smem);
    const bool epi = warp >= kEpiWarp0 && warp < kEpiWarp0 + 4;
    bool have = false;
    if (epi) {
      have = wait_sleep(&bars->tmem_full[0], 0u, abort, &g_awq_error_word, 1u);
      tc_fence_after();
    }
    const int rows_per = BMH / p.S;
    for (int hm = 0; hm < halves; ++hm) {
      if (epi && have) {
        const int q = warp - kEpiWarp0;
        const int r = q * 32 + lane;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tc_ld_32x32b_x32(tmem_base + (uint32_t(q * 32) << 16) + uint32_t(hm * BN + c * 32), v);
          float4* dst = reinterpret_cast<float4*>(part + r * kPartStride + c * 32);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                 __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        }
      }
      cluster_sync_all();
      if constexpr (SILU) {
        // output quad j of a row: pair q = j / 4 (gate columns 32q .. 32q+15,
        // up columns 32q+16 .. 32q+31 of the tile), columns 4 (j % 4) .. + 3
        for (int idx = threadIdx.x; idx < rows_per * (BN / 8); idx += kGemmThreads) {
          const int r = rank * rows_per + idx / (BN / 8);
          const int j = idx % (BN / 8);
          const int gc = 32 * (j >> 2) + 4 * (j & 3);
          const int64_t m = int64_t(m0) + hm * BMH + r;
          if (m >= p.M || n0 + gc >= p.N) continue;
          const uint32_t offg = smem_u32(part + r * kPartStride + gc);
          float4 g, u;
          sum_slices_dsmem2(offg, offg + 16 * 4, p.S, g, u);
          const uint32_t lo = uint32_t(__half_as_ushort(__float2half_rn(silu_f32(g.x) * u.x))) |
                              (uint32_t(__half_as_ushort(__float2half_rn(silu_f32(g.y) * u.y))) << 16);
          const uint32_t hi = uint32_t(__half_as_ushort(__float2half_rn(silu_f32(g.z) * u.z))) |
                              (uint32_t(__half_as_ushort(__float2half_rn(silu_f32(g.w) * u.w))) << 16);
          *reinterpret_cast<uint2*>(p.y + m * (p.N / 2) + n0 / 2 + 16 * (j >> 2) + 4 * (j & 3)) =
              make_uint2(lo, hi);
        }
      } else {
      for (int idx = threadIdx.x; idx < rows_per * (BN / 4); idx += kGemmThreads) {
        const int r = rank * rows_per + idx / (BN / 4);
        const int c4 = idx % (BN / 4);
        const int64_t m = int64_t(m0) + hm * BMH + r;
        const int n = n0 + 4 * c4;
        if (m >= p.M || n >= p.N) continue;
        const float4 acc = sum_slices_dsmem(smem_u32(part + r * kPartStride + 4 * c4), p.S);
        const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
        uint16_t* yrow = p.y + m * p.N;
        if (n + 4 <= p.N && (p.N & 3) == 0) {
          const uint32_t lo = uint32_t(__half_as_ushort(__float2half_rn(a4[0]))) |
                              (uint32_t(__half_as_ushort(__float2half_rn(a4[1]))) << 16);
          const uint32_t hi = uint32_t(__half_as_ushort(__float2half_rn(a4[2]))) |
                              (uint32_t(__half_as_ushort(__float2half_rn(a4[3]))) << 16);
          *reinterpret_cast<uint2*>(yrow + n) = make_uint2(lo, hi);
        } else {
          for (int e = 0; e < 4 && n + e < p.N; ++e) yrow[n + e] = __half_as_ushort(__float2half_rn(a4[e]));
        }
      }
      }
      cluster_sync_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols));
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
constexpr int kMaxDevices = 64;
// Cost model of the plan, fitted to B200 measurements of every tile shape
// at M = 32 .. 512 (SM cycles at 1.965 GHz): a CTA's k block takes about
// 1150 cycles when its x tile holds up to 128 rows and 2010 with 256 (the
// stage pipeline's latency, not the MMA issue, sets it at these sizes,
// whatever the tile shape); a launch on whole tiles pays about 3 us of
// pipeline fill and epilogue, one that sums K slices across a cluster about
// 12 us with 256-channel tiles and 7 us with 128-channel ones.
constexpr int64_t kKbCycles1 = 1150, kKbCycles2 = 2010;
constexpr int64_t kFixedCycles = 5900, kSplitFixedCycles = BN == 256 ? 23600 : 13800;
std::atomic<int> g_sms[kMaxDevices];
std::atomic<int> g_attr_set[kMaxDevices][4];   // [zero point + 2 * fused]
// clusters of 2, 4, 8 CTAs that fit at once: 0 = not queried yet, -1 = none, else the count
std::atomic<int> g_clusters[kMaxDevices][4][3];


// Plan (dry: estimate only, in SM cycles, into *cost) or launch the product
// with this tile width. The arguments were validated by the caller.
awq_status_t run(const uint16_t* x, const int32_t* qweight, const uint16_t* scales, const uint16_t* zeros,
                 int64_t M, int64_t N, int64_t K, awq_qconfig_t cfg, uint16_t* y, void* stream, bool dry,
                 int64_t* cost) {
  awq_status_t st = AWQ_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return AWQ_ERR_UNSUPPORTED;
  int sms = g_sms[dev].load(std::memory_order_relaxed);
  if (sms == 0) {
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return AWQ_ERR_CUDA;
    g_sms[dev].store(sms, std::memory_order_relaxed);
  }
  const bool silu = (cfg.flags & AWQ_FLAG_SILU_MUL) != 0;
  auto kernel = cfg.zero_point ? (silu ? gemm_kernel<true, true> : gemm_kernel<true, false>)
                               : (silu ? gemm_kernel<false, true> : gemm_kernel<false, false>);
  const int zi = (cfg.zero_point ? 1 : 0) + (silu ? 2 : 0);
  if (!g_attr_set[dev][zi].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
        cudaSuccess)
      return AWQ_ERR_CUDA;
    g_attr_set[dev][zi].store(1, std::memory_order_release);
  }

  // x: fp16 [M][K], box 64 (k) x 256 (rows), 128-byte swizzle; rows past M read as 0.
  // codes: int32 [N][K/8], box 8 words x BN rows, 32-byte swizzle; rows past N read as 0.
  CUtensorMap tmap_x, tmap_q;
  if (!dry && (!make_tensor_map_2d(&tmap_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, uint64_t(K), uint64_t(M),
                                   uint64_t(K) * 2, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
               !make_tensor_map_2d(&tmap_q, CU_TENSOR_MAP_DATA_TYPE_INT32, qweight, uint64_t(K / 8),
                                   uint64_t(N), uint64_t(K / 8) * 4, BK / 8, BN, CU_TENSOR_MAP_SWIZZLE_32B)))
    return AWQ_ERR_CUDA;
  GemmParams p;
  p.y = y;
  p.silu = (cfg.flags & AWQ_FLAG_SILU_MUL) ? 1 : 0;
  p.scales = scales;
  p.zeros = zeros;
  p.M = int(M);
  p.N = int(N);
  p.K = int(K);
  p.G = int(K / kGroup);
  p.m_tiles = int((M + BM - 1) / BM);
  p.n_tiles = int((N + BN - 1) / BN);
  p.k_blocks = int(K / BK);
  const int64_t tiles = int64_t(p.m_tiles) * p.n_tiles;
  if (tiles > (int64_t(1) << 31) - 1) return AWQ_ERR_SHAPE;
  // One launch takes tiles tile0 .. tile0 + count - 1. Few tiles: split K
  // over a cluster of S CTAs per tile (whole groups per slice, at least 4 k
  // blocks each). S is chosen to minimise the estimated time
  //   waves(S) x (k blocks per slice) x (cycles of one k block) + fixed(S),
  // waves(S) = ceil(count / clusters of S that fit at once) (S = 1: the
  // persistent grid of one CTA per SM), a k block = 4 MMAs per 128 rows of x
  // (kMmaCycles each), fixed = pipeline fill and epilogue (more with the
  // cross-CTA slice reduction). The estimate also chooses the tile width.
  const int64_t kb_cycles = BM > BMH && M > BMH ? kKbCycles2 : kKbCycles1;
  auto part_cost = [&](int64_t count, int S, int fit) -> int64_t {
    const int64_t slots = S == 1 ? sms : fit;
    return ((count + slots - 1) / slots) * (p.k_blocks / S) * kb_cycles + (S == 1 ? kFixedCycles : kSplitFixedCycles);
  };
  auto launch_part = [&](int64_t tile0, int64_t count, bool dry, int64_t* cost) -> awq_status_t {
    GemmParams q = p;
    q.tile0 = int(tile0);
    q.num_tiles = int(count);
    q.S = 1;
    int64_t best = part_cost(count, 1, 0);
    if (2 * count <= sms) {
      const int cands[3] = {2, 4, 8};
      for (int ci = 0; ci < 3; ++ci) {
        const int S = cands[ci];
        if (q.G % S != 0 || q.k_blocks / S < 4) continue;
        int fit = g_clusters[dev][zi][ci].load(std::memory_order_acquire);
        if (fit == 0) {
          cudaLaunchConfig_t qc = {};
          qc.gridDim = dim3(unsigned(S));
          qc.blockDim = dim3(kGemmThreads);
          qc.dynamicSmemBytes = kSmemBytes;
          cudaLaunchAttribute qa[1];
          qa[0].id = cudaLaunchAttributeClusterDimension;
          qa[0].val.clusterDim.x = unsigned(S);
          qa[0].val.clusterDim.y = 1;
          qa[0].val.clusterDim.z = 1;
          qc.attrs = qa;
          qc.numAttrs = 1;
          int n = 0;
          if (cudaOccupancyMaxActiveClusters(&n, kernel, &qc) != cudaSuccess) {
            (void)cudaGetLastError();
            n = 0;
          }
          fit = n > 0 ? n : -1;
          g_clusters[dev][zi][ci].store(fit, std::memory_order_release);
        }
        if (fit <= 0) continue;
        const int64_t c = part_cost(count, S, fit);
        if (c < best) {
          best = c;
          q.S = S;
        }
      }
    }
    *cost += best;
    if (dry) return AWQ_OK;
    q.kb_per_unit = q.k_blocks / q.S;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(unsigned(q.S > 1 ? count * q.S : (count < sms ? count : sms)));
    lc.blockDim = dim3(kGemmThreads);
    lc.dynamicSmemBytes = kSmemBytes;
    lc.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(q.S);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.attrs = attr;
    lc.numAttrs = q.S > 1 ? 1 : 0;
    if (cudaLaunchKernelEx(&lc, kernel, tmap_x, tmap_q, q) != cudaSuccess) return AWQ_ERR_CUDA;
    return launch_status();
  };
  // Whole waves of one tile per SM stay on the persistent grid. A last partial
  // wave of at most half the SMs goes to a second launch, where its few tiles
  // split K over clusters instead of leaving the other SMs idle while they
  // finish (448 tiles on 148 SMs: 3 waves + 4 tiles). The launches write
  // disjoint tiles of y.
  const int64_t rem = tiles % sms;
  int64_t total = 0;
  if (tiles > sms && rem > 0 && 2 * rem <= sms) {
    const awq_status_t st1 = launch_part(0, tiles - rem, dry, &total);
    if (st1 != AWQ_OK) return st1;
    st = launch_part(tiles - rem, rem, dry, &total);
  } else {
    st = launch_part(0, tiles, dry, &total);
  }
  if (cost) *cost = total;
  return st;
}

}  // namespace
