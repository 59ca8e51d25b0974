// A chain of W4A16 small-batch products in one launch, for sm_100a:
// y_l[M][N_l] = x_l[M][K_l] . W_l'^T for l = 0 .. n-1, 1 <= M <= 16, where a
// layer's x may be the y of an earlier layer of the same call.
//
// ("AutoAWQ" code tour, "The big picture": the GEMV kernel for single-token
// decoding; "AutoAWQ" capability page, WQLinear paragraph: INT4 weights are
// decoded inside the matmul, and the layer is bound by memory at small
// batch; same page, fused-blocks paragraph: fusing a block's projections
// saves launches.)
//
// A decode step runs a few quantized layers back to back, each 8-125 MB of
// packed weights. Launched one by one, every layer pays a fill (its first
// weights arrive only after the previous layer is done) and a drain (its
// last stages compute while HBM idles). The weights do not depend on the
// activations, so one persistent launch can stream them continuously: the
// weights of layer l+1 flow into shared memory while layer l finishes, and
// only the activations wait for the layer that produces them.
//
// * Grid: every CTA resident at once (one or two per SM, from the occupancy
//   of the launch). Each CTA walks every layer in order and takes a
//   contiguous run of its 16-channel tiles (whole tiles over all of K; K
//   cut into slices only when a layer has fewer tiles than CTAs), exactly
//   as a one-layer launch would. Layers that do not depend on one another
//   rotate the CTA order so that their leftover tiles land on different
//   CTAs.
// * Warp roles: one producer warp (one thread) issues every TMA copy; eight
//   consumer warps decode and multiply; one release warp (one thread)
//   publishes the CTA's completed layers, so that no consumer waits for the
//   acknowledgement of its stores. A stage of the ring is one chunk of
//   up to four tiles x eight groups (one group per consumer warp): codes,
//   scales, zero points and the matching slice of x. Consumers wait on the
//   stage's "full" barrier, compute, and arrive on its "empty" barrier; the
//   producer refills a slot once its empty barrier completes.
// * Dependencies: a layer whose x is the y of layer d has its weight copies
//   issued as soon as a slot frees up, but the copy of its x only once every
//   CTA has counted itself done with layer d (a per-layer counter, released
//   after the CTA's y stores and acquired by the producer before the copy).
// * Schedule: each CTA's share of every layer (items, K slice, groups) and
//   the layer fields the loops read are computed once at kernel start into a
//   table in shared memory; the kernel parameters hold the tensor maps.
// * Arithmetic (per consumer warp, one group of every tile of the stage):
//   the packed nibble order puts consecutive k pairs in the low and high
//   halves of a word, so one LOP3 with an fp16 magic number yields two exact
//   fp16 values 1024+q (pairs (0,1), (4,5)) or 64+q (pairs (2,3), (6,7)).
//   The decoded 16x16 tile is the A operand of mma.m16n8k16, x the B operand
//   (batch in n). The offsets, zero point and scale are removed per (row,
//   batch row, group) in fp32: sum_k x (q - z) = raw - C - z S with
//   C = 1024 sum_{1024 slots} x + 64 sum_{64 slots} x and S = sum_k x, both
//   from two MMAs per k16 against a constant tile whose rows 0-7 hold the
//   magic weights and rows 8-15 ones, so that every lane receives C and S
//   of its own batch columns. Then acc += s (raw - C - z S).
// * Every wait is bounded. A wait that gives up records bit 2 of the device
//   error word and raises the CTA's abort flag; the CTA then walks the rest
//   of its schedule without waiting or computing (so every named barrier,
//   arrival counter and done counter is still reached), the producer issues
//   the activation copies still missing from stages whose weights it issued
//   (so every armed phase completes) and waits, bounded, for all copies in
//   flight before the CTA exits. The output is then incomplete.

#include "awq_common.cuh"
#include "awq_tma_host.h"

#include <atomic>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

namespace awq {

__device__ uint32_t g_awq_chain_error = 0;
// Limit of the pipeline waits (consumer stage waits, producer slot and
// dependency waits). The waits for copies already in flight always use the
// full kWaitLimitNs.
__device__ unsigned long long g_awq_chain_wait_limit_ns = kWaitLimitNs;

namespace {

constexpr int kCW = 8;                          // consumer warps
constexpr int kProducerWarp = kCW;
constexpr int kReleaseWarp = kCW + 1;
constexpr int kThreads = (kCW + 2) * 32;        // + the producer and release warps
constexpr int kTile = 16;                       // output channels per MMA tile
constexpr int kMaxTC = 4;                       // tiles per chunk
constexpr int kMaxLayers = AWQ_CHAIN_MAX_LAYERS;
constexpr int kMaxStages = 8;
constexpr int kMaxHeader = 2048;                // barriers, flags and the layer table below the ring
constexpr int kFlagsOff = kMaxStages * 16;      // abort flag, then the count of layers the consumers finished
constexpr int kTableOff = 256;                  // LayerRun[n_layers]
constexpr int kTileBytes = kCW * 1024;          // codes of one tile: [group][16 rows][16 words]
constexpr int kScaleOff = kMaxTC * kTileBytes;  // scales: [group][64 rows] fp16
constexpr int kMetaBytes = kCW * 64 * 2;
constexpr int kZeroOff = kScaleOff + kMetaBytes;  // zero points: [group][64] fp16 or [group][12 words]
constexpr int kPackedZeroWords = 12;
constexpr int kXOff = kZeroOff + kMetaBytes;    // x: [m][group][128] fp16
constexpr int kXRowBytes = kCW * 256;
constexpr int kConsumerBarrier = 1;             // named barrier of the consumer warps
constexpr uint32_t kErrBit = 4u;
constexpr uint32_t kCodesBoxBytes = kTileBytes;

static_assert(kFlagsOff + 8 <= kTableOff, "stage bookkeeping overflows its region");
static_assert(kXOff % 1024 == 0, "x must start 1024-aligned inside a stage");

struct alignas(64) LayerDesc {
  CUtensorMap tq;      // codes: {16 words, N rows, G groups}, box {16, 16, kCW}
  CUtensorMap tx;      // x: {128, G, M}, box {128, kCW, M}
  CUtensorMap ts;      // scales: {N, G}, box {64, kCW}
  CUtensorMap tz;      // zeros: {N, G} box {64, kCW}, or packed {N/8 words, G} box {12, kCW}
  uint16_t* y;
  float* partials;     // [ks][T * 16][M], only when ks > 1
  uint32_t* counters;  // [units], only when ks > 1
  int N, G, T;
  int tpu;             // tiles per unit: 1, or 2 (gate tile + up tile, fused SiLU epilogue)
  int units;           // T / tpu
  int ks;              // K slices
  int items;           // units * ks, slice-major
  int x_from;          // -1: x is ready at launch; else the layer whose y x is
  int rot;             // CTA rotation of this layer's item ranges
  int silu;
};

// This CTA's share of one layer and the layer fields its loops read, filled
// at kernel start (kernel parameters are read through the constant cache,
// which misses for a table of 32 layer descriptors; shared memory does not).
struct LayerRun {
  int i0, i1;          // items of the CTA
  int s;               // their K slice (a CTA never straddles two)
  int gb, ge;          // the slice's groups
  int units;
  int N;
  int info;            // tpu (bits 0-1), silu (bit 2), ks (bits 8-15), x_from + 1 (bits 16-23)
  uint16_t* y;
  float* partials;
  uint32_t* counters;
};
static_assert(sizeof(LayerRun) == 56, "layer table entry");
static_assert(kTableOff + kMaxLayers * sizeof(LayerRun) <= kMaxHeader, "layer table overflows the header");

// Bytes below the ring: the table of n layers, rounded up to the ring's 1024-byte alignment.
__host__ __device__ constexpr int header_bytes(int n) {
  return (kTableOff + n * int(sizeof(LayerRun)) + 1023) / 1024 * 1024;
}

__host__ __device__ __forceinline__ int run_tpu(const LayerRun& r) { return r.info & 3; }
__host__ __device__ __forceinline__ int run_silu(const LayerRun& r) { return (r.info >> 2) & 1; }
__host__ __device__ __forceinline__ int run_ks(const LayerRun& r) { return (r.info >> 8) & 0xff; }
__host__ __device__ __forceinline__ int run_x_from(const LayerRun& r) { return ((r.info >> 16) & 0xff) - 1; }

struct ChainParams {
  LayerDesc layer[kMaxLayers];
  uint32_t* done;      // [n_layers] CTAs done with each layer; done[kMaxLayers]: CTAs done with the call
  int n_layers, M, stages, stage_bytes, pbuf_offset, early;
};

// ---------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds_half(uint32_t a) {
  unsigned short h;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h) : "r"(a));
  return __half2float(__ushort_as_half(h));
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync %0, %1;" ::"r"(kConsumerBarrier), "r"(kCW * 32) : "memory");
}

__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_try_wait_u32(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: a thread whose phase is not complete
// sleeps until it completes or the hint (ns) runs out, instead of spinning
// and taking issue slots from the warps that share its scheduler.
__device__ __forceinline__ bool mbar_sleep_wait(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void tma_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// ---------------------------------------------------------------------------
// the schedule: layers, then the CTA's chunks of each layer, then stages of
// kCW groups. Producer and consumers walk the same sequence.
// ---------------------------------------------------------------------------
struct Chunk {
  int i, nu, tc, t0, s, gb, ge;
};

// The items (units of one K slice) of a layer that CTA position b (of
// `grid`) takes. Without K slices: q = units / grid each, one more for the
// first units % grid positions. With ks slices: slice s goes to positions
// [ceil(s grid / ks), ceil((s + 1) grid / ks)), which share its units the
// same way, so that no CTA straddles two slices. Items are slice-major
// (item = slice * units + unit). The same arithmetic runs on the host.
__host__ __device__ __forceinline__ void split_items(int units, int ks, int grid, int b, int& i0, int& i1) {
  // grid <= 2048 CTAs and ks <= 32 slices: the products fit in 32 bits
  int s = 0, b0 = 0, n = grid;
  if (ks > 1) {
    s = b * ks / grid;
    b0 = (s * grid + ks - 1) / ks;
    n = ((s + 1) * grid + ks - 1) / ks - b0;
  }
  const int j = b - b0;
  const int q = units / n, r = units - q * n;
  const int u0 = j * q + (j < r ? j : r);
  i0 = s * units + u0;
  i1 = i0 + q + (j < r ? 1 : 0);
}

// The CTA's items of a layer, its position rotated by `rot` so that
// consecutive independent layers hand their leftover items to different CTAs.
__device__ __forceinline__ void item_range(const LayerDesc& L, int& i0, int& i1) {
  const int grid = int(gridDim.x);
  int b = int(blockIdx.x) - L.rot;
  if (b < 0) b += grid;
  split_items(L.units, L.ks, grid, b, i0, i1);
}

// The CTA's share of layer l (thread-parallel at kernel start).
__device__ __forceinline__ void fill_run(const LayerDesc& L, LayerRun& r) {
  item_range(L, r.i0, r.i1);
  r.s = r.i0 < r.i1 ? r.i0 / L.units : 0;
  r.gb = L.G * r.s / L.ks;            // G < 2^25, ks <= 32
  r.ge = L.G * (r.s + 1) / L.ks;
  r.units = L.units;
  r.N = L.N;
  r.info = L.tpu | (L.silu << 2) | (L.ks << 8) | ((L.x_from + 1) << 16);
  r.y = L.y;
  r.partials = L.partials;
  r.counters = L.counters;
}

__device__ __forceinline__ void load_chunk(const LayerRun& R, int i, Chunk& c) {
  const int tpu = run_tpu(R);
  c.i = i;
  c.s = R.s;
  const int u0 = i - R.s * R.units;
  int nu = R.i1 - i;
  const int cap = kMaxTC / tpu;
  if (nu > cap) nu = cap;
  if (nu > R.units - u0) nu = R.units - u0;
  c.nu = nu;
  c.t0 = u0 * tpu;
  c.tc = nu * tpu;
  c.gb = R.gb;
  c.ge = R.ge;
}

// Flat cursor over (layer, chunk, stage) for the producer.
struct Cursor {
  int l;
  Chunk c;
  int gbase;
  __device__ __forceinline__ bool done(int n) const { return l >= n; }
};

__device__ __forceinline__ void cursor_layer(const ChainParams& p, const LayerRun* runs, Cursor& u) {
  // from layer u.l on, the first layer with items for this CTA
  for (; u.l < p.n_layers; ++u.l) {
    const LayerRun& R = runs[u.l];
    if (R.i0 < R.i1) {
      load_chunk(R, R.i0, u.c);
      u.gbase = u.c.gb;
      return;
    }
  }
}

__device__ __forceinline__ void cursor_init(const ChainParams& p, const LayerRun* runs, Cursor& u) {
  u.l = 0;
  cursor_layer(p, runs, u);
}

__device__ __forceinline__ void cursor_next(const ChainParams& p, const LayerRun* runs, Cursor& u) {
  u.gbase += kCW;
  if (u.gbase < u.c.ge) return;
  const int ni = u.c.i + u.c.nu;
  if (ni < runs[u.l].i1) {
    load_chunk(runs[u.l], ni, u.c);
    u.gbase = u.c.gb;
    return;
  }
  ++u.l;
  cursor_layer(p, runs, u);
}

template <int ZM>
__device__ __forceinline__ uint32_t weight_bytes(int tc) {
  return uint32_t(tc * kCodesBoxBytes + kMetaBytes +
                  (ZM == 2 ? kCW * kPackedZeroWords * 4 : ZM == 1 ? kMetaBytes : 0));
}

// Arm stage `slot` for the chunk stage at u (weights + x bytes) and issue
// the weight copies: codes tile by tile, the 64-row runs of scales and zero
// points (packed: 12 words from word 2 t0 rounded down to a multiple of 4,
// a 16-byte boundary).
template <int ZM>
__device__ __forceinline__ void issue_weights(const ChainParams& p, const Cursor& u, uint32_t st, uint32_t bar) {
  const LayerDesc& L = p.layer[u.l];
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(weight_bytes<ZM>(u.c.tc) + uint32_t(p.M) * kXRowBytes)
               : "memory");
  const int r0 = u.c.t0 * kTile;
  for (int r = 0; r < u.c.tc; ++r) tma_3d(st + r * kTileBytes, &L.tq, 0, r0 + r * kTile, u.gbase, bar);
  tma_2d(st + kScaleOff, &L.ts, r0, u.gbase, bar);
  if (ZM == 2) tma_2d(st + kZeroOff, &L.tz, (2 * u.c.t0) & ~3, u.gbase, bar);
  if (ZM == 1) tma_2d(st + kZeroOff, &L.tz, r0, u.gbase, bar);
}

__device__ __forceinline__ void issue_x(const ChainParams& p, const Cursor& u, uint32_t st, uint32_t bar) {
  tma_3d(st + kXOff, &p.layer[u.l].tx, 0, u.gbase, 0, bar);
}

// ---------------------------------------------------------------------------
// consumer: one stage of one warp (group w of up to four tiles)
// ---------------------------------------------------------------------------
template <int MB, int ZM>
__device__ __forceinline__ void stage_compute(uint32_t st, int w, int g, int t, int tc, int M, int zoff,
                                              float (&acc)[kMaxTC][MB > 8 ? 2 : 1][4]) {
  constexpr int MT = MB > 8 ? 2 : 1;
  constexpr bool ODD = MB > 1;        // batch columns 2t + 1 exist
  // x fragments: batch row m = 8 mt + g, this warp's group, k = 32 t .. 32 t + 31
  uint4 xf[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int m = 8 * mt + g;
    const uint32_t xa = st + kXOff + uint32_t(m) * kXRowBytes + w * 256 + t * 64;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) xf[mt][jj] = (MB == 1 ? g == 0 : m < M) ? lds128(xa + jj * 16) : make_uint4(0, 0, 0, 0);
  }
  // C and S of every batch column: rows 0-7 of the constant tile weigh the
  // 1024-offset slots by 1024 and the 64-offset slots by 64, rows 8-15 weigh
  // every slot by 1, so cs = {C(2t), C(2t+1), S(2t), S(2t+1)} in every lane.
  float cs[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int i = 0; i < 4; ++i) cs[mt][i] = 0.0f;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      mma_16816(cs[mt], 0x64006400u, 0x3C003C00u, 0x54005400u, 0x3C003C00u, xf[mt][jj].x, xf[mt][jj].y);
      mma_16816(cs[mt], 0x64006400u, 0x3C003C00u, 0x54005400u, 0x3C003C00u, xf[mt][jj].z, xf[mt][jj].w);
    }
  }
  const uint32_t cbase = st + w * 1024 + g * 64 + t * 16;
  const uint32_t sbase = st + kScaleOff + w * 128 + g * 2;
#pragma unroll
  for (int rt = 0; rt < kMaxTC; ++rt) {
    if (rt < tc) {
      const uint4 c_lo = lds128(cbase + rt * kTileBytes);
      const uint4 c_hi = lds128(cbase + rt * kTileBytes + 512);
      float grp[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) grp[mt][i] = 0.0f;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        uint32_t plo[4], phi[4];
        decode_word_magic(word_of(c_lo, jj), plo);
        decode_word_magic(word_of(c_hi, jj), phi);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          mma_16816(grp[mt], plo[0], phi[0], plo[1], phi[1], xf[mt][jj].x, xf[mt][jj].y);
          mma_16816(grp[mt], plo[2], phi[2], plo[3], phi[3], xf[mt][jj].z, xf[mt][jj].w);
        }
      }
      const float s_lo = lds_half(sbase + rt * 32), s_hi = lds_half(sbase + rt * 32 + 16);
      float z_lo, z_hi;
      if constexpr (ZM == 1) {
        z_lo = lds_half(sbase + kMetaBytes + rt * 32);
        z_hi = lds_half(sbase + kMetaBytes + rt * 32 + 16);
      } else if constexpr (ZM == 2) {
        // rows g and g + 8 of tile rt: nibble g of words 2 rt and 2 rt + 1
        // past the chunk's first word (zoff: 8 bytes when t0 is odd)
        const uint2 zz = lds64(st + kZeroOff + w * (kPackedZeroWords * 4) + zoff + rt * 8);
        z_lo = float((zz.x >> (4 * g)) & 0xFu);
        z_hi = float((zz.y >> (4 * g)) & 0xFu);
      } else {
        z_lo = 8.0f;
        z_hi = 8.0f;
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        acc[rt][mt][0] = fmaf(s_lo, fmaf(-z_lo, cs[mt][2], grp[mt][0] - cs[mt][0]), acc[rt][mt][0]);
        acc[rt][mt][2] = fmaf(s_hi, fmaf(-z_hi, cs[mt][2], grp[mt][2] - cs[mt][0]), acc[rt][mt][2]);
        if (ODD) {
          acc[rt][mt][1] = fmaf(s_lo, fmaf(-z_lo, cs[mt][3], grp[mt][1] - cs[mt][1]), acc[rt][mt][1]);
          acc[rt][mt][3] = fmaf(s_hi, fmaf(-z_hi, cs[mt][3], grp[mt][3] - cs[mt][1]), acc[rt][mt][3]);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int MB, int ZM>
__global__ void __launch_bounds__(kThreads, MB == 1 ? 2 : 1)
chain_kernel(const __grid_constant__ ChainParams p) {
  constexpr int MT = MB > 8 ? 2 : 1;
  asm volatile("griddepcontrol.launch_dependents;");
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const uint32_t full0 = sbase;                        // [S] mbarriers
  const uint32_t empty0 = sbase + kMaxStages * 8;      // [S] mbarriers
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kFlagsOff);
  // layers the consumers have finished (written by consumer thread 0, read by the release warp)
  const uint32_t layers_done = sbase + kFlagsOff + 4;
  LayerRun* runs = reinterpret_cast<LayerRun*>(smem + kTableOff);
  const uint32_t ring = sbase + header_bytes(p.n_layers);
  const int S = p.stages;
  const int warp = int(threadIdx.x) >> 5;
  const int lane = int(threadIdx.x) & 31;
  const unsigned long long limit = g_awq_chain_wait_limit_ns;
  const uint32_t hint = limit < 20000ull ? uint32_t(limit) : 20000u;   // sleep of one wait step, ns

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(full0 + 8 * s), "r"(1));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty0 + 8 * s), "r"(kCW));
    }
    *abort_flag = 0;
    asm volatile("st.shared.u32 [%0], 0;" ::"r"(layers_done) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
  }
  for (int l = int(threadIdx.x); l < p.n_layers; l += int(blockDim.x)) fill_run(p.layer[l], runs[l]);
  __syncthreads();

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      Cursor cw, cx;
      cursor_init(p, runs, cw);
      cx = cw;
      int sw = 0, sx = 0;           // stages whose weights / x have been issued
      uint32_t ready = 0;           // layers whose x may be read
      for (int l = 0; l < p.n_layers; ++l)
        if (p.layer[l].x_from < 0) ready |= 1u << l;
      if (p.early) {
        for (; sw < S && !cw.done(p.n_layers); ++sw) {
          issue_weights<ZM>(p, cw, ring + sw * p.stage_bytes, full0 + 8 * sw);
          cursor_next(p, runs, cw);
        }
      }
      asm volatile("griddepcontrol.wait;" ::: "memory");
      const uint32_t target = gridDim.x;
      // Starts of the two waits the producer can be in (0: not waiting): for
      // the layer that the next x copy comes from, and for a free slot. A
      // wait longer than the limit gives up.
      uint64_t t_x = 0, t_slot = 0;
      bool gave_up = false;
      while (!cx.done(p.n_layers)) {
        bool progress = false, slot_busy = false, x_blocked = false;
        if (!cw.done(p.n_layers)) {
          const int slot = sw % S;
          if (sw < S || mbar_test_wait(empty0 + 8 * slot, uint32_t((sw / S) + 1) & 1u)) {
            issue_weights<ZM>(p, cw, ring + slot * p.stage_bytes, full0 + 8 * slot);
            cursor_next(p, runs, cw);
            ++sw;
            progress = true;
          } else {
            slot_busy = true;
          }
        }
        if (sx < sw) {
          const int l = cx.l;
          if (!((ready >> l) & 1u)) {
            if (ld_acquire_gpu(p.done + run_x_from(runs[l])) >= target) {
              asm volatile("fence.proxy.async.global;" ::: "memory");
              ready |= 1u << l;
            }
          }
          if ((ready >> l) & 1u) {
            const int slot = sx % S;
            issue_x(p, cx, ring + slot * p.stage_bytes, full0 + 8 * slot);
            cursor_next(p, runs, cx);
            ++sx;
            progress = true;
          } else {
            x_blocked = true;
          }
        }
        if (!progress && sx == sw && slot_busy) {
          // nothing to do until the next slot frees: sleep on its barrier
          const int slot = sw % S;
          mbar_sleep_wait(empty0 + 8 * slot, uint32_t((sw / S) + 1) & 1u, hint);
        }
        if (*abort_flag) {
          gave_up = true;
          break;
        }
        const uint64_t now = now_ns();
        if (!x_blocked) t_x = 0;
        else if (t_x == 0) t_x = now;
        if (!slot_busy) t_slot = 0;
        else if (t_slot == 0) t_slot = now;
        if ((t_x && now - t_x > limit) || (t_slot && now - t_slot > limit)) {
          *abort_flag = 1;
          atomicOr(&g_awq_chain_error, kErrBit);
          gave_up = true;
          break;
        }
      }
      if (gave_up) {
        // every armed stage still missing its x gets it (from wherever x
        // points now) so that every armed phase completes
        for (; sx < sw; ++sx) {
          const int slot = sx % S;
          issue_x(p, cx, ring + slot * p.stage_bytes, full0 + 8 * slot);
          cursor_next(p, runs, cx);
        }
      }
      // every copy issued must land before the CTA exits: the last phase
      // armed on each slot (earlier ones completed before the slot was
      // re-armed)
      for (int slot = 0; slot < S && slot < sw; ++slot) {
        const int last = slot + ((sw - 1 - slot) / S) * S;
        const uint32_t par = uint32_t(last / S) & 1u;
        const uint64_t t0 = now_ns();
        while (!mbar_try_wait_u32(full0 + 8 * slot, par) && now_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
    __syncwarp();
  } else if (warp == kReleaseWarp) {
    // ------------------------------------------------------------ release
    // Publishes each layer once the consumers have finished it: their
    // stores are ordered before consumer thread 0's release of the count
    // (named barrier), this thread acquires the count, and its gpu-scope
    // release of the layer's done counter covers them.
    if (lane == 0) {
      // the previous launch's last CTA resets the counters: wait for it
      asm volatile("griddepcontrol.wait;" ::: "memory");
      uint64_t t0 = 0;
      for (int l = 0; l < p.n_layers;) {
        uint32_t n;
        asm volatile("ld.acquire.cta.shared.u32 %0, [%1];" : "=r"(n) : "r"(layers_done) : "memory");
        if (n > uint32_t(l)) {
          for (; l < int(n); ++l) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p.done + l) : "memory");
          t0 = 0;
          continue;
        }
        const uint64_t now = now_ns();
        if (t0 == 0) {
          t0 = now;
        } else if (now - t0 > kWaitLimitNs) {
          // the consumers count every layer even after giving up, so this
          // is reached only if they stopped: let the others give up too
          *abort_flag = 1;
          atomicOr(&g_awq_chain_error, kErrBit);
          break;
        }
        __nanosleep(64);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ consumers
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int w = warp;
    const int g = lane >> 2;
    const int t = lane & 3;
    const int M = p.M;
    const uint32_t pbuf = sbase + p.pbuf_offset;       // [warp][64 rows][M] fp32
    int slot = 0;
    uint32_t phase = 0;
    bool live = true;
    for (int l = 0; l < p.n_layers; ++l) {
      const LayerRun& R = runs[l];
      const int i1 = R.i1;
      const int ks = run_ks(R), tpu = run_tpu(R), silu = run_silu(R), N = R.N;
      const int T = R.units * tpu;
      uint16_t* const y = R.y;
      for (int i = R.i0; i < i1;) {
        Chunk cc;
        load_chunk(R, i, cc);
        float acc[kMaxTC][MT][4];
#pragma unroll
        for (int rt = 0; rt < kMaxTC; ++rt)
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[rt][mt][k] = 0.0f;
        for (int gbase = cc.gb; gbase < cc.ge; gbase += kCW) {
          const uint32_t full = full0 + 8 * slot;
          if (live) {
            bool ok = mbar_sleep_wait(full, phase, hint);
            if (!ok) {
              const uint64_t t0 = now_ns();
              while (!ok) {
                ok = mbar_sleep_wait(full, phase, hint);
                if (!ok) {
                  if (*abort_flag) break;
                  if (now_ns() - t0 > limit) {
                    *abort_flag = 1;
                    atomicOr(&g_awq_chain_error, kErrBit);
                    break;
                  }
                }
              }
            }
            live = __all_sync(0xffffffffu, ok);
          }
          if (live) {
            if (gbase + w < cc.ge)
              stage_compute<MB, ZM>(ring + slot * p.stage_bytes, w, g, t, cc.tc, M, (cc.t0 & 1) * 8, acc);
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty0 + 8 * slot) : "memory");
          }
          if (++slot == S) {
            slot = 0;
            phase ^= 1u;
          }
        }
        // ---- chunk reduction: the warps' partial sums meet in shared memory
        // ([warp][row][m]) and are summed in warp order (deterministic)
        const uint32_t pw = pbuf + uint32_t(w * 64 * M) * 4;
#pragma unroll
        for (int rt = 0; rt < kMaxTC; ++rt) {
          if (rt < cc.tc) {
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              const int m0 = 8 * mt + 2 * t;
              const int r_lo = 16 * rt + g, r_hi = r_lo + 8;
              if (m0 < M) {
                sts_f32(pw + uint32_t(r_lo * M + m0) * 4, acc[rt][mt][0]);
                sts_f32(pw + uint32_t(r_hi * M + m0) * 4, acc[rt][mt][2]);
              }
              if (m0 + 1 < M) {
                sts_f32(pw + uint32_t(r_lo * M + m0 + 1) * 4, acc[rt][mt][1]);
                sts_f32(pw + uint32_t(r_hi * M + m0 + 1) * 4, acc[rt][mt][3]);
              }
            }
          }
        }
        consumer_sync();
        const int64_t row0 = int64_t(cc.t0) * kTile;
        const int tid = int(threadIdx.x);
        if (!silu || ks > 1) {
          const int V = kTile * cc.tc * M;
          for (int v = tid; v < V; v += kCW * 32) {
            float sum = 0.0f;
#pragma unroll
            for (int ww = 0; ww < kCW; ++ww) sum += lds_f32(pbuf + uint32_t(ww * 64 * M + v) * 4);
            const int row = v / M;
            const int m = v - row * M;
            if (ks == 1) {
              if (row0 + row < N) y[int64_t(m) * N + row0 + row] = __half_as_ushort(__float2half_rn(sum));
            } else {
              __stcg(R.partials + ((int64_t(cc.s) * T * kTile + row0 + row) * M + m), sum);
            }
          }
        } else {
          // fused gate/up: tile 2q of the chunk holds gate rows, 2q + 1 the up rows
          const int V = kTile * (cc.tc / 2) * M;
          for (int v = tid; v < V; v += kCW * 32) {
            const int q = v / (kTile * M);
            const int rem = v - q * (kTile * M);
            const int vg = 2 * q * kTile * M + rem;
            float gs = 0.0f, us = 0.0f;
#pragma unroll
            for (int ww = 0; ww < kCW; ++ww) {
              gs += lds_f32(pbuf + uint32_t(ww * 64 * M + vg) * 4);
              us += lds_f32(pbuf + uint32_t(ww * 64 * M + vg + kTile * M) * 4);
            }
            const int row = rem / M;
            const int m = rem - row * M;
            y[int64_t(m) * (N / 2) + row0 / 2 + q * kTile + row] =
                __half_as_ushort(__float2half_rn(silu_f32(gs) * us));
          }
        }
        if (ks > 1) {
          // slices of a unit meet in the workspace: the CTA whose arrival
          // brings a unit's count to ks sums the ks partials in slice order.
          // The barrier orders every consumer's partial stores before the
          // arrivals, whose release makes them visible at GPU scope.
          consumer_sync();
          if (w < cc.nu) {
            const int unit = cc.t0 / tpu + w;
            uint32_t last = 0;
            if (lane == 0) {
              uint32_t old;
              asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                           : "=r"(old) : "l"(R.counters + unit) : "memory");
              last = (old + 1 == uint32_t(ks)) ? 1u : 0u;
            }
            last = __shfl_sync(0xffffffffu, last, 0);
            __syncwarp();   // lane 0's acquire orders the warp's partial reads
            if (last) {
              const int64_t trow = int64_t(unit) * tpu * kTile;
              if (tpu == 1) {
                for (int v = lane; v < kTile * M; v += 32) {
                  float sum = 0.0f;
                  for (int s = 0; s < ks; ++s) sum += __ldcg(R.partials + ((int64_t(s) * T * kTile + trow) * M + v));
                  const int row = v / M;
                  const int m = v - row * M;
                  if (trow + row < N) y[int64_t(m) * N + trow + row] = __half_as_ushort(__float2half_rn(sum));
                }
              } else {
                for (int v = lane; v < kTile * M; v += 32) {
                  float gs = 0.0f, us = 0.0f;
                  for (int s = 0; s < ks; ++s) {
                    const float* ps = R.partials + (int64_t(s) * T * kTile + trow) * M;
                    gs += __ldcg(ps + v);
                    us += __ldcg(ps + kTile * M + v);
                  }
                  const int row = v / M;
                  const int m = v - row * M;
                  y[int64_t(m) * (N / 2) + trow / 2 + row] = __half_as_ushort(__float2half_rn(silu_f32(gs) * us));
                }
              }
              if (lane == 0) R.counters[unit] = 0u;
            }
          }
        }
        consumer_sync();   // pbuf is reused by the next chunk; the layer's stores are done
        i += cc.nu;
      }
      // This CTA is done with layer l (the chunk's last barrier ordered every
      // consumer's stores before this point): the release warp publishes it.
      if (threadIdx.x == 0) asm volatile("st.release.cta.shared.u32 [%0], %1;" ::"r"(layers_done), "r"(l + 1) : "memory");
    }
  }
  __syncthreads();
  // The last CTA out resets the per-layer counters for the next call.
  if (threadIdx.x == 0) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                 : "=r"(old) : "l"(p.done + kMaxLayers) : "memory");
    if (old + 1 == gridDim.x) {
      for (int l = 0; l < p.n_layers; ++l) p.done[l] = 0u;
      p.done[kMaxLayers] = 0u;
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
using ChainFn = void (*)(const ChainParams);

constexpr int kNumVariants = 9;     // batch tile {1, 8, 16} x zero points {sym, fp16, packed}
constexpr int kSmemBudget = 232448;
constexpr int kHalfSmBudget = 115712;
constexpr int kMaxDevices = 64;

ChainFn pick(int64_t M, int zm, int& id) {
  static const ChainFn table[kNumVariants] = {
      chain_kernel<1, 0>, chain_kernel<1, 1>, chain_kernel<1, 2>,
      chain_kernel<8, 0>, chain_kernel<8, 1>, chain_kernel<8, 2>,
      chain_kernel<16, 0>, chain_kernel<16, 1>, chain_kernel<16, 2>};
  const int mb = M == 1 ? 0 : M <= 8 ? 1 : 2;
  id = mb * 3 + zm;
  return table[id];
}

std::atomic<int> g_sms[kMaxDevices];
std::atomic<int> g_attr_set[kMaxDevices][kNumVariants];

struct LayerPlan {
  int T, tpu, units, ks, items, rot;
  size_t counter_off, partial_off;   // workspace offsets (ks > 1)
};

struct ChainPlan {
  ChainFn fn;
  int id, grid, stages, stage_bytes, pbuf_offset, smem;
  LayerPlan lp[kMaxLayers];
  size_t ws_bytes;
};

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

awq_status_t check_layer(const awq_gemv_layer_t* L, int l, const awq_gemv_layer_t* layers, int64_t M, int zm) {
  awq_status_t st = check_cfg(L->cfg, true);
  if (st != AWQ_OK) return st;
  if (zero_mode(L->cfg) != zm) return AWQ_ERR_UNSUPPORTED;   // one zero-point form per call
  if ((st = check_nk(L->N, L->K)) != AWQ_OK) return st;
  if (L->N == 0 || L->N % 8) return AWQ_ERR_SHAPE;
  if ((L->cfg.flags & AWQ_FLAG_SILU_MUL) && L->N % 32) return AWQ_ERR_SHAPE;
  if ((L->cfg.flags & AWQ_FLAG_PACKED_ZEROS) && L->N % 32) return AWQ_ERR_SHAPE;
  if (L->K / kGroup > (int64_t(1) << 24)) return AWQ_ERR_SHAPE;
  if (!L->x || !L->qweight || !L->scales || !L->y) return AWQ_ERR_NULL;
  if (L->cfg.zero_point && !L->zeros) return AWQ_ERR_NULL;
  if (!L->cfg.zero_point && L->zeros) return AWQ_ERR_SHAPE;
  if (!aligned16(L->x) || !aligned16(L->qweight) || !aligned16(L->scales) || !aligned16(L->y) ||
      (L->zeros && !aligned16(L->zeros)))
    return AWQ_ERR_ALIGN;
  if (L->x_from < -1 || L->x_from >= l) return AWQ_ERR_SHAPE;
  if (L->x_from >= 0) {
    const awq_gemv_layer_t& D = layers[L->x_from];
    const int64_t cols = (D.cfg.flags & AWQ_FLAG_SILU_MUL) ? D.N / 2 : D.N;
    if (L->x != D.y || L->K != cols) return AWQ_ERR_SHAPE;
  }
  (void)M;
  return AWQ_OK;
}

// Cost of the busiest CTA when a layer of `units` units (tpu tiles each) and
// G groups is cut into ks K slices over `grid` CTAs, in tile-group units: each
// stage of kCW groups costs its tiles x groups, but never less than that of
// three tiles (a stage of one or two tiles has too little independent work
// to hide the latency of its decode-and-multiply chains), plus a fixed cost
// per stage, per chunk (the reduction) and per chunk of a split layer
// (partials and the arrival).
int64_t split_cost(int units, int tpu, int G, int ks, int grid) {
  constexpr int64_t kMinTiles = 3, kStageCost = 2, kChunkCost = 4, kSplitCost = 6;
  int64_t worst = 0;
  for (int b = 0; b < grid; ++b) {
    int i0, i1;
    split_items(units, ks, grid, b, i0, i1);
    int64_t c = 0;
    for (int i = i0; i < i1;) {
      const int sl = i / units, u0 = i - sl * units;
      int nu = i1 - i;
      if (nu > kMaxTC / tpu) nu = kMaxTC / tpu;
      if (nu > units - u0) nu = units - u0;
      const int64_t g = int64_t(G) * (sl + 1) / ks - int64_t(G) * sl / ks;
      const int64_t tc = nu * tpu;
      // a stage takes as long as a full one whatever its group count (one group per warp)
      c += ((g + kCW - 1) / kCW) * ((tc > kMinTiles ? tc : kMinTiles) * kCW + kStageCost) + kChunkCost +
           (ks > 1 ? kSplitCost : 0);
      i += nu;
    }
    if (c > worst) worst = c;
  }
  return worst;
}

// K slices for a layer: the candidate whose busiest CTA costs least (ties:
// fewer slices). Cached per (units, tpu, G, grid): the choice is a few
// hundred thousand steps of host arithmetic.
int pick_ks(int units, int tpu, int G, int grid) {
  struct Key {
    int units, tpu, G, grid;
  };
  static std::mutex lock;
  static std::vector<std::pair<Key, int>> cache;
  {
    std::lock_guard<std::mutex> g(lock);
    for (const auto& e : cache)
      if (e.first.units == units && e.first.tpu == tpu && e.first.G == G && e.first.grid == grid) return e.second;
  }
  int best = 1;
  int64_t best_cost = split_cost(units, tpu, G, 1, grid);
  const int cands[] = {2, 3, 4, 5, 6, 7, 8, 10, 12, 14, 16, 24, 32};
  for (int ks : cands) {
    if (ks > G || ks > grid) break;
    const int64_t c = split_cost(units, tpu, G, ks, grid);
    if (c < best_cost) {
      best_cost = c;
      best = ks;
    }
  }
  std::lock_guard<std::mutex> g(lock);
  if (cache.size() < 4096) cache.push_back({Key{units, tpu, G, grid}, best});
  return best;
}

awq_status_t make_chain_plan(const awq_gemv_layer_t* layers, int n, int64_t M, ChainPlan& pl) {
  if (!layers) return AWQ_ERR_NULL;
  if (n < 1 || n > kMaxLayers) return AWQ_ERR_SHAPE;
  if (M < 1 || M > 16) return AWQ_ERR_SHAPE;
  const int zm = zero_mode(layers[0].cfg);
  for (int l = 0; l < n; ++l) {
    awq_status_t st = check_layer(&layers[l], l, layers, M, zm);
    if (st != AWQ_OK) return st;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return AWQ_ERR_UNSUPPORTED;
  int sms = g_sms[dev].load(std::memory_order_relaxed);
  if (sms == 0) {
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return AWQ_ERR_CUDA;
    g_sms[dev].store(sms, std::memory_order_relaxed);
  }
  pl.fn = pick(M, zm, pl.id);
  if (!g_attr_set[dev][pl.id].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(pl.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget) != cudaSuccess)
      return AWQ_ERR_CUDA;
    g_attr_set[dev][pl.id].store(1, std::memory_order_release);
  }
  // Ring geometry: two CTAs per SM when each still holds three stages,
  // else one CTA per SM with the whole shared memory.
  pl.stage_bytes = kXOff + int(M) * kXRowBytes;
  const int pbuf_bytes = kCW * 64 * int(M) * 4;
  int per_sm = 2;
  for (;; --per_sm) {
    const int budget = per_sm == 2 ? kHalfSmBudget : kSmemBudget;
    int st = (budget - header_bytes(n) - pbuf_bytes) / pl.stage_bytes;
    if (st > kMaxStages) st = kMaxStages;
    pl.stages = st;
    if (st >= 3 || per_sm == 1) break;
  }
  if (pl.stages < 2) return AWQ_ERR_UNSUPPORTED;
  pl.pbuf_offset = header_bytes(n) + pl.stages * pl.stage_bytes;
  pl.smem = pl.pbuf_offset + pbuf_bytes;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, pl.fn, kThreads, size_t(pl.smem)) != cudaSuccess)
    return AWQ_ERR_CUDA;
  if (occ < 1) return AWQ_ERR_UNSUPPORTED;
  if (per_sm > occ) per_sm = occ;
  pl.grid = per_sm * sms;
  // Per layer: whole tiles per CTA over all of K, K slices only when a
  // layer has fewer units than CTAs (as a one-layer launch would).
  size_t off = align256(size_t(kMaxLayers + 1) * 4);   // per-layer done counters + the exit counter
  int level_start = 0;
  int64_t extra = 0;
  for (int l = 0; l < n; ++l) {
    const awq_gemv_layer_t& L = layers[l];
    LayerPlan& lp = pl.lp[l];
    const int64_t G = L.K / kGroup;
    lp.T = int((L.N + kTile - 1) / kTile);
    lp.tpu = (L.cfg.flags & AWQ_FLAG_SILU_MUL) ? 2 : 1;
    lp.units = lp.T / lp.tpu;
    const int ks = pick_ks(lp.units, lp.tpu, int(G), pl.grid);
    lp.ks = ks;
    lp.items = lp.units * ks;
    // A layer that reads the output of a layer of the current level starts a
    // new level. Within a level, each layer's leftover items go to the CTAs
    // after those that took the previous layers' leftovers.
    if (L.x_from >= level_start) {
      level_start = l;
      extra = 0;
    }
    lp.rot = int(extra % pl.grid);
    if (lp.ks == 1) extra += lp.units % pl.grid;
    if (lp.ks > 1) {
      lp.counter_off = off;
      off += align256(size_t(lp.units) * 4);
      lp.partial_off = off;
      off += align256(size_t(lp.ks) * size_t(lp.T) * kTile * size_t(M) * 4);
    } else {
      lp.counter_off = lp.partial_off = 0;
    }
  }
  pl.ws_bytes = off;
  return AWQ_OK;
}

}  // namespace

awq_status_t chain_take_error(uint32_t* word, cudaStream_t s) {
  uint32_t zero = 0;
  if (cudaMemcpyFromSymbolAsync(word, g_awq_chain_error, sizeof(uint32_t), 0, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return AWQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return AWQ_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(g_awq_chain_error, &zero, sizeof(uint32_t), 0, cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return AWQ_ERR_CUDA;
  return cudaStreamSynchronize(s) == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

}  // namespace awq

using namespace awq;

extern "C" awq_status_t awq_gemv_chain_workspace_bytes(const awq_gemv_layer_t* layers, int n_layers, int64_t M,
                                                       size_t* bytes) {
  if (!bytes) return AWQ_ERR_NULL;
  ChainPlan pl;
  awq_status_t st = make_chain_plan(layers, n_layers, M, pl);
  if (st != AWQ_OK) return st;
  *bytes = pl.ws_bytes;
  return AWQ_OK;
}

extern "C" awq_status_t awq_gemv_chain(const awq_gemv_layer_t* layers, int n_layers, int64_t M, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  ChainPlan pl;
  awq_status_t st = make_chain_plan(layers, n_layers, M, pl);
  if (st != AWQ_OK) return st;
  if (!workspace) return AWQ_ERR_WORKSPACE;
  if (workspace_bytes < pl.ws_bytes) return AWQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return AWQ_ERR_ALIGN;
  char* ws = static_cast<char*>(workspace);
  ChainParams p;
  std::memset(&p, 0, sizeof(p));
  bool early = true;
  for (int l = 0; l < n_layers; ++l) {
    const awq_gemv_layer_t& A = layers[l];
    const LayerPlan& lp = pl.lp[l];
    LayerDesc& D = p.layer[l];
    const int zm = zero_mode(A.cfg);
    const uint64_t G = uint64_t(A.K / kGroup);
    if (!make_tensor_map_3d(&D.tq, CU_TENSOR_MAP_DATA_TYPE_INT32, A.qweight, kWordsPerGroup, uint64_t(A.N), G,
                            uint64_t(A.K / 8) * 4, kWordsPerGroup * 4, kWordsPerGroup, kTile, kCW) ||
        !make_tensor_map_3d(&D.tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, A.x, kGroup, G, uint64_t(M), kGroup * 2,
                            uint64_t(A.K) * 2, kGroup, kCW, uint32_t(M)) ||
        !make_tensor_map_2d(&D.ts, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, A.scales, uint64_t(A.N), G, uint64_t(A.N) * 2,
                            64, kCW, CU_TENSOR_MAP_SWIZZLE_NONE))
      return AWQ_ERR_CUDA;
    if (zm == 2) {
      if (!make_tensor_map_2d(&D.tz, CU_TENSOR_MAP_DATA_TYPE_INT32, A.zeros, uint64_t(A.N / 8), G, uint64_t(A.N) / 2,
                              kPackedZeroWords, kCW, CU_TENSOR_MAP_SWIZZLE_NONE))
        return AWQ_ERR_CUDA;
    } else if (zm == 1) {
      if (!make_tensor_map_2d(&D.tz, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, A.zeros, uint64_t(A.N), G, uint64_t(A.N) * 2,
                              64, kCW, CU_TENSOR_MAP_SWIZZLE_NONE))
        return AWQ_ERR_CUDA;
    } else {
      D.tz = D.ts;   // never read
    }
    D.y = A.y;
    D.partials = lp.ks > 1 ? reinterpret_cast<float*>(ws + lp.partial_off) : nullptr;
    D.counters = lp.ks > 1 ? reinterpret_cast<uint32_t*>(ws + lp.counter_off) : nullptr;
    D.N = int(A.N);
    D.G = int(G);
    D.T = lp.T;
    D.tpu = lp.tpu;
    D.units = lp.units;
    D.ks = lp.ks;
    D.items = lp.items;
    D.x_from = A.x_from;
    D.rot = lp.rot;
    D.silu = (A.cfg.flags & AWQ_FLAG_SILU_MUL) ? 1 : 0;
    early = early && (A.cfg.flags & AWQ_FLAG_WEIGHTS_STATIC);
  }
  p.done = reinterpret_cast<uint32_t*>(ws);
  p.n_layers = n_layers;
  p.M = int(M);
  p.stages = pl.stages;
  p.stage_bytes = pl.stage_bytes;
  p.pbuf_offset = pl.pbuf_offset;
  p.early = early ? 1 : 0;
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
  if (cudaLaunchKernelEx(&lc, pl.fn, p) != cudaSuccess) return AWQ_ERR_CUDA;
  return launch_status();
}

extern "C" awq_status_t awq_debug_set_wait_limit_ns(uint64_t ns, void* stream) {
  if (ns == 0) ns = kWaitLimitNs;
  if (ns > kWaitLimitNs) return AWQ_ERR_SHAPE;
  const unsigned long long v = ns;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyToSymbolAsync(g_awq_chain_wait_limit_ns, &v, sizeof(v), 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return AWQ_ERR_CUDA;
  return cudaStreamSynchronize(s) == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}
