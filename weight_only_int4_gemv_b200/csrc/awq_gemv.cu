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
//   The units are ordered block-major and split evenly over every warp of a
//   grid sized to the resident capacity of the GPU (a stream-K split), so all
//   148 SMs stream the same number of bytes whatever N and K are.
// * Each lane streams its codes with 16-byte non-allocating loads, one group
//   ahead of the arithmetic: lane (g, t) of a warp reads 16 bytes (32 codes)
//   of rows g and g+8 of each 16-row tile; the four lanes of a quad cover one
//   whole group of a row.
// * Decode: the packed nibble order puts consecutive k pairs in the low and
//   high halves of a word, so one LOP3 turns a word into two fp16 values
//   1024+q (or 64+q) and one HSUB2 subtracts 1024+z, leaving q - z exactly.
// * Multiply: the decoded 16x16 weight tile is the A operand of
//   mma.m16n8k16 straight from registers; x is the B operand (batch in the
//   n dimension, two n8 tiles for M > 8). The k positions inside an MMA are
//   a permutation of the word's k (each lane owns whole words), matched by
//   loading x[m][8w .. 8w+7] for the same words, which is one 16-byte load
//   covering two MMAs. Accumulation is fp32.
// * The scale is applied once per group: sum_k x (q - z) s = s * sum_k x (q - z),
//   the group's fp32 partial is multiplied by s and added to the fp32 total.
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
};

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

template <int RT>
struct Stage {
  uint4 c_lo[RT], c_hi[RT];
  uint16_t s_lo[RT], s_hi[RT], z_lo[RT], z_hi[RT];
};

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

template <int MT, int RT, bool ZP>
__global__ void __launch_bounds__(kGemvThreads)
gemv_kernel(const GemvParams p) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int64_t gw = int64_t(blockIdx.x) * kGemvWarps + (threadIdx.x >> 5);
  const int64_t W = p.total_warps;
  const int64_t G = p.G;
  const int64_t u_begin = warp_start(p.units, gw, W);
  const int64_t u_end = warp_start(p.units, gw + 1, W);
  if (u_begin >= u_end) return;
  const int64_t first_block = u_begin / G;
  const int64_t row_vec = p.K / 32;       // 16-byte vectors per packed row
  const uint4* qv = reinterpret_cast<const uint4*>(p.qweight);

  // activation rows served by this lane (batch index m = 8 mt + g)
  const uint16_t* xrow[MT];
  bool xok[MT];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int m = 8 * mt + g;
    xok[mt] = m < p.M;
    xrow[mt] = p.x + int64_t(xok[mt] ? m : 0) * p.K + 32 * t;
  }

  for (int64_t u = u_begin; u < u_end;) {
    const int64_t b = u / G;
    const int j0 = int(u - b * G);
    const int j1 = int(u_end - b * G < G ? u_end - b * G : G);
    const int64_t row0 = b * (16 * RT);

    const uint4* cp_lo[RT];
    const uint4* cp_hi[RT];
    const uint16_t* sp_lo[RT];
    const uint16_t* sp_hi[RT];
    bool ok_lo[RT], ok_hi[RT];
#pragma unroll
    for (int rt = 0; rt < RT; ++rt) {
      const int64_t r_lo = row0 + 16 * rt + g;
      const int64_t r_hi = r_lo + 8;
      ok_lo[rt] = r_lo < p.N;
      ok_hi[rt] = r_hi < p.N;
      cp_lo[rt] = qv + (ok_lo[rt] ? r_lo : 0) * row_vec + t;
      cp_hi[rt] = qv + (ok_hi[rt] ? r_hi : 0) * row_vec + t;
      sp_lo[rt] = p.scales + (ok_lo[rt] ? r_lo : 0) * G;
      sp_hi[rt] = p.scales + (ok_hi[rt] ? r_hi : 0) * G;
    }

    auto load_stage = [&](Stage<RT>& s, int j) {
#pragma unroll
      for (int rt = 0; rt < RT; ++rt) {
        s.c_lo[rt] = ok_lo[rt] ? ld_stream_v4(cp_lo[rt] + 4 * j) : make_uint4(0, 0, 0, 0);
        s.c_hi[rt] = ok_hi[rt] ? ld_stream_v4(cp_hi[rt] + 4 * j) : make_uint4(0, 0, 0, 0);
        s.s_lo[rt] = ok_lo[rt] ? ld_nc_u16(sp_lo[rt] + j) : uint16_t(0);
        s.s_hi[rt] = ok_hi[rt] ? ld_nc_u16(sp_hi[rt] + j) : uint16_t(0);
        if (ZP) {
          s.z_lo[rt] = ok_lo[rt] ? ld_nc_u16(p.zeros + (sp_lo[rt] - p.scales) + j) : uint16_t(0);
          s.z_hi[rt] = ok_hi[rt] ? ld_nc_u16(p.zeros + (sp_hi[rt] - p.scales) + j) : uint16_t(0);
        }
      }
    };

    float acc[RT][MT][4];
#pragma unroll
    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[rt][mt][i] = 0.0f;

    Stage<RT> cur;
    load_stage(cur, j0);
    for (int j = j0; j < j1; ++j) {
      Stage<RT> nxt;
      if (j + 1 < j1) load_stage(nxt, j + 1);

      uint4 xf[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          xf[mt][jj] = xok[mt] ? ld_nc_v4(xrow[mt] + int64_t(j) * kGroup + 8 * jj) : make_uint4(0, 0, 0, 0);

#pragma unroll
      for (int rt = 0; rt < RT; ++rt) {
        uint32_t zl1024, zl64, zh1024, zh64;
        if (ZP) {
          zero_bias_pairs(half_bits_to_float(cur.z_lo[rt]), zl1024, zl64);
          zero_bias_pairs(half_bits_to_float(cur.z_hi[rt]), zh1024, zh64);
        } else {
          zero_bias_pairs(8.0f, zl1024, zl64);
          zh1024 = zl1024;
          zh64 = zl64;
        }
        float grp[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) grp[mt][i] = 0.0f;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          uint32_t plo[4], phi[4];
          decode_word_qz(word_of(cur.c_lo[rt], jj), zl1024, zl64, plo);
          decode_word_qz(word_of(cur.c_hi[rt], jj), zh1024, zh64, phi);
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            mma_16816(grp[mt], plo[0], phi[0], plo[1], phi[1], xf[mt][jj].x, xf[mt][jj].y);
            mma_16816(grp[mt], plo[2], phi[2], plo[3], phi[3], xf[mt][jj].z, xf[mt][jj].w);
          }
        }
        const float s_lo = half_bits_to_float(cur.s_lo[rt]);
        const float s_hi = half_bits_to_float(cur.s_hi[rt]);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          acc[rt][mt][0] = fmaf(s_lo, grp[mt][0], acc[rt][mt][0]);
          acc[rt][mt][1] = fmaf(s_lo, grp[mt][1], acc[rt][mt][1]);
          acc[rt][mt][2] = fmaf(s_hi, grp[mt][2], acc[rt][mt][2]);
          acc[rt][mt][3] = fmaf(s_hi, grp[mt][3], acc[rt][mt][3]);
        }
      }
      cur = nxt;
    }

    if (j0 == 0 && j1 == G) {
      store_y<MT, RT>(p, row0, g, t, acc);
    } else {
      // Partial block: publish this warp's fp32 sums, count the groups in.
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
      if (last) {
        __threadfence();
        // contributors: every non-empty warp range that overlaps block b,
        // summed in warp order
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
    }
    u = b * G + j1;
  }
}

// ---------------------------------------------------------------------------
// host side: plan (variant, grid, workspace) for a shape
// ---------------------------------------------------------------------------
using KernelFn = void (*)(const GemvParams);

struct Variant {
  KernelFn fn;
  int mt, rt;
};

Variant pick_variant(int64_t M, bool zp) {
  // x fragments cost MT*256 bytes of L1 traffic per 16x128 weight tile; a
  // 32-row block halves that, so two row tiles per warp.
  if (M <= 8) return zp ? Variant{gemv_kernel<1, 2, true>, 1, 2} : Variant{gemv_kernel<1, 2, false>, 1, 2};
  return zp ? Variant{gemv_kernel<2, 2, true>, 2, 2} : Variant{gemv_kernel<2, 2, false>, 2, 2};
}

struct Plan {
  Variant v;
  int grid;
  int nb;
  int64_t units;
  size_t counter_bytes;
  size_t partial_bytes;
};

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<int> g_occ[kMaxDevices][4];

int variant_index(const Variant& v, bool zp) { return (v.mt - 1) * 2 + (zp ? 1 : 0); }

awq_status_t make_plan(int64_t M, int64_t N, int64_t K, bool zp, Plan& pl) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return AWQ_ERR_UNSUPPORTED;
  pl.v = pick_variant(M, zp);
  int sms = g_sm_count[dev].load(std::memory_order_relaxed);
  if (sms == 0) {
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return AWQ_ERR_CUDA;
    g_sm_count[dev].store(sms, std::memory_order_relaxed);
  }
  const int vi = variant_index(pl.v, zp);
  int occ = g_occ[dev][vi].load(std::memory_order_relaxed);
  if (occ == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, pl.v.fn, kGemvThreads, 0) != cudaSuccess)
      return AWQ_ERR_CUDA;
    if (occ < 1) occ = 1;
    g_occ[dev][vi].store(occ, std::memory_order_relaxed);
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
  pl.v.fn<<<pl.grid, kGemvThreads, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return launch_status();
}
