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
//   consumer warps decode and multiply. A stage of the ring is one chunk of
//   up to four tiles x eight groups (one group per consumer warp): codes,
//   scales, zero points and the matching slice of x. Consumers wait on the
//   stage's "full" barrier, compute, and arrive on its "empty" barrier; the
//   producer refills a slot once its empty barrier completes.
// * Dependencies: a layer whose x is the y of layer d has its weight copies
//   issued as soon as a slot frees up; its x comes from an exchange copy of
//   d's output in the workspace, in which every 16-bit value is stored as
//   its bit pattern plus one, so that 0 means "not written by this launch".
//   Each consumer warp loads its own group of x one stage ahead (plain loads
//   into registers), and before the stage checks that no value is 0,
//   reloading until all are written; it then stores the decoded values into
//   the stage's x region. No counter, fence or flag sits between the last
//   store of layer d and the first use of its values. The exchange region
//   has two halves used by alternate launches (the parity of a launch count
//   kept in the workspace); each launch zeroes its share of the half the
//   previous launch used.
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
//   of its schedule without waiting or computing (so every named barrier and
//   arrival counter is still reached, and every output is still written),
//   and the producer waits, bounded, for all copies in flight before the
//   CTA exits. The output is then incomplete.

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
constexpr int kThreads = (kCW + 1) * 32;        // + one producer warp
constexpr int kTile = 16;                       // output channels per MMA tile
constexpr int kMaxTC = 4;                       // tiles per chunk
constexpr int kMaxLayers = AWQ_CHAIN_MAX_LAYERS;
constexpr int kMaxStages = 8;
constexpr int kMaxHeader = 2048;                // barriers, flags and the layer table below the ring
constexpr int kFlagsOff = kMaxStages * 16;      // abort flag
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

// Stage geometry for chunks of up to TCAP tiles: codes [TCAP][group][16 rows]
// [16 words], then scales, zero points and x. The batch tiles of 2 and 4
// rows use two-tile stages, so that two CTAs of at least three stages share
// an SM; the others use four-tile stages (the constants above).
template <int TCAP> __host__ __device__ constexpr uint32_t scale_off() { return uint32_t(TCAP * kTileBytes); }
template <int TCAP> __host__ __device__ constexpr uint32_t zero_off() { return scale_off<TCAP>() + kMetaBytes; }
template <int TCAP> __host__ __device__ constexpr uint32_t x_off() { return zero_off<TCAP>() + kMetaBytes; }
template <int MB> __host__ __device__ constexpr int tile_cap() { return MB == 2 || MB == 4 ? 2 : kMaxTC; }
static_assert(x_off<2>() % 1024 == 0 && x_off<kMaxTC>() == uint32_t(kXOff), "stage geometry");

struct alignas(64) LayerDesc {
  CUtensorMap tq;      // codes: {16 words, N rows, G groups}, box {16, 16, kCW}
  CUtensorMap tx;      // x: {128, G, M}, box {128, kCW, M}
  CUtensorMap ts;      // scales: {N, G}, box {64, kCW}
  CUtensorMap tz;      // zeros: {N, G} box {64, kCW}, or packed {N/8 words, G} box {12, kCW}
  uint16_t* y;
  uint32_t partial_off;  // workspace offset of the tagged partials [ks - 1][T * 16][M] (ks > 1)
  uint32_t ll_off;       // offset of the exchange copy [M][N or N/2] in each half (source layers)
  int source;            // a later layer reads this layer's output
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
  int i0, i1;          // items of the CTA (all in one K slice)
  int gb, ge;          // the slice's groups
  int units;
  int N;
  int G;
  int info;            // tpu (bits 0-1), silu (bit 2), source (bit 3), ks (bits 8-15), x_from + 1 (bits 16-23)
  uint16_t* y;
  uint32_t partial_off, ll_off;
  int next;            // the next layer with items for this CTA (n_layers: none)
  int pad;
};
static_assert(sizeof(LayerRun) == 56, "layer table entry");
static_assert(kTableOff + kMaxLayers * sizeof(LayerRun) <= kMaxHeader, "layer table overflows the header");

// Bytes below the ring: the table of n layers, rounded up to the ring's 1024-byte alignment.
__host__ __device__ constexpr int header_bytes(int n) {
  return (kTableOff + n * int(sizeof(LayerRun)) + 1023) / 1024 * 1024;
}

__host__ __device__ __forceinline__ int run_tpu(const LayerRun& r) { return r.info & 3; }
__host__ __device__ __forceinline__ int run_silu(const LayerRun& r) { return (r.info >> 2) & 1; }
__host__ __device__ __forceinline__ int run_source(const LayerRun& r) { return (r.info >> 3) & 1; }
__host__ __device__ __forceinline__ int run_ks(const LayerRun& r) { return (r.info >> 8) & 0xff; }
__host__ __device__ __forceinline__ int run_x_from(const LayerRun& r) { return ((r.info >> 16) & 0xff) - 1; }

// Control words at the start of the workspace.
constexpr int kExitWord = 0;     // CTAs done with the call (the last one resets it)
constexpr int kEpochWord = 1;    // launches completed on this workspace: its parity picks the exchange half
constexpr int kControlBytes = 256;

struct ChainParams {
  LayerDesc layer[kMaxLayers];
  char* ws;            // workspace: control words, split-K partials, the exchange region
  uint32_t ll_base;    // offset of the exchange region (two halves of ll_half bytes)
  uint32_t ll_half;
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

// The exchange copy of a layer's output: each fp16 value v is stored as
// v + 1 (the pattern 0xFFFF, a NaN that the conversion never produces, is
// first replaced by the canonical NaN 0x7FFF), so that 0 marks a value not
// written by this launch. Stores and loads are relaxed at gpu scope: a value
// is either 0 or complete (16-bit accesses are single-copy atomic), so a
// reader needs no ordering, only to see every value of its slice non-zero.
__device__ __forceinline__ void ll_put(char* base, int64_t idx, uint16_t h) {
  const uint16_t e = uint16_t((h == 0xFFFFu ? 0x7FFFu : h) + 1u);
  asm volatile("st.relaxed.gpu.global.u16 [%0], %1;" ::"l"(base + idx * 2), "h"(e) : "memory");
}
__device__ __forceinline__ uint2 ll_get2(const char* a) {
  uint2 v;
  asm volatile("ld.relaxed.gpu.global.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(a) : "memory");
  return v;
}
__device__ __forceinline__ bool ll_complete(uint2 v) { return (__vcmpeq2(v.x, 0u) | __vcmpeq2(v.y, 0u)) == 0u; }
__device__ __forceinline__ uint2 ll_decode(uint2 v) {
  return make_uint2(__vsub2(v.x, 0x00010001u), __vsub2(v.y, 0x00010001u));
}
// Partial sums of the K slices of a unit: 64-bit relaxed stores of (a tag,
// the float's bits), the tag being the launch count plus one (a zero-filled
// workspace holds tag 0), so that a reader sees a value of this launch whole
// or not at all, with no fence between store and use.
__device__ __forceinline__ void put_tagged(unsigned long long* a, uint32_t tag, float v) {
  const unsigned long long x = (static_cast<unsigned long long>(tag) << 32) | __float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(a), "l"(x) : "memory");
}
__device__ __forceinline__ unsigned long long get_tagged(const unsigned long long* a) {
  unsigned long long x;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(x) : "l"(a) : "memory");
  return x;
}

// The sum over the K slices of one value of a unit: the tagged partials of
// slices 0 .. ks-2 (stride ss apart), each waited for (bounded) until it
// carries this launch's tag, in slice order, then the caller's own sum (the
// last slice). Loads are issued four at a time. Kept out of line: it runs
// once per value at the end of a chunk, and inlined it would take registers
// from the stage loop.
__device__ __noinline__ float slice_sum(const unsigned long long* partials, int64_t ss, int ks, int64_t idx,
                                        uint32_t tag, float own, volatile int* abort_flag,
                                        unsigned long long limit) {
  float sum = 0.0f;
  for (int s0 = 0; s0 < ks - 1; s0 += 4) {
    unsigned long long x[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (s0 + j < ks - 1) x[j] = get_tagged(partials + (int64_t(s0 + j) * ss + idx));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (s0 + j < ks - 1) {
        if (uint32_t(x[j] >> 32) != tag) {
          const unsigned long long* a = partials + (int64_t(s0 + j) * ss + idx);
          const uint64_t t0 = now_ns();
          for (;;) {
            x[j] = get_tagged(a);
            if (uint32_t(x[j] >> 32) == tag || *abort_flag) break;
            if (now_ns() - t0 > limit) {
              *abort_flag = 1;
              atomicOr(&g_awq_chain_error, kErrBit);
              break;
            }
          }
        }
        sum += __uint_as_float(uint32_t(x[j]));
      }
    }
  }
  return sum + own;
}

__device__ __forceinline__ void sts64(uint32_t a, uint2 v) {
  asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(a), "r"(v.x), "r"(v.y) : "memory");
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
  const int s = r.i0 < r.i1 ? r.i0 / L.units : 0;
  r.gb = L.G * s / L.ks;            // G < 2^25, ks <= 32
  r.ge = L.G * (s + 1) / L.ks;
  r.units = L.units;
  r.N = L.N;
  r.G = L.G;
  r.info = L.tpu | (L.silu << 2) | (L.source << 3) | (L.ks << 8) | ((L.x_from + 1) << 16);
  r.y = L.y;
  r.partial_off = L.partial_off;
  r.ll_off = L.ll_off;
}

template <int TCAP>
__device__ __forceinline__ void load_chunk(const LayerRun& R, int i, Chunk& c) {
  const int tpu = run_tpu(R);
  c.i = i;
  c.s = i / R.units;
  const int u0 = i - c.s * R.units;
  int nu = R.i1 - i;
  const int cap = TCAP / tpu;
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

template <int TCAP>
__device__ __forceinline__ void cursor_layer(const ChainParams& p, const LayerRun* runs, Cursor& u) {
  // from layer u.l on, the first layer with items for this CTA
  for (; u.l < p.n_layers; ++u.l) {
    const LayerRun& R = runs[u.l];
    if (R.i0 < R.i1) {
      load_chunk<TCAP>(R, R.i0, u.c);
      u.gbase = u.c.gb;
      return;
    }
  }
}

template <int TCAP>
__device__ __forceinline__ void cursor_init(const ChainParams& p, const LayerRun* runs, Cursor& u) {
  u.l = 0;
  cursor_layer<TCAP>(p, runs, u);
}

template <int TCAP>
__device__ __forceinline__ void cursor_next(const ChainParams& p, const LayerRun* runs, Cursor& u) {
  u.gbase += kCW;
  if (u.gbase < u.c.ge) return;
  const int ni = u.c.i + u.c.nu;
  if (ni < runs[u.l].i1) {
    load_chunk<TCAP>(runs[u.l], ni, u.c);
    u.gbase = u.c.gb;
    return;
  }
  ++u.l;
  cursor_layer<TCAP>(p, runs, u);
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
template <int ZM, int TCAP>
__device__ __forceinline__ void issue_weights(const ChainParams& p, const LayerRun* runs, const Cursor& u, uint32_t st,
                                              uint32_t bar) {
  const LayerDesc& L = p.layer[u.l];
  // the x of a layer that reads an earlier layer's output comes from the
  // consumers, not from a copy
  const uint32_t xb = run_x_from(runs[u.l]) < 0 ? uint32_t(p.M) * kXRowBytes : 0u;
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(weight_bytes<ZM>(u.c.tc) + xb)
               : "memory");
  const int r0 = u.c.t0 * kTile;
  for (int r = 0; r < u.c.tc; ++r) tma_3d(st + r * kTileBytes, &L.tq, 0, r0 + r * kTile, u.gbase, bar);
  tma_2d(st + scale_off<TCAP>(), &L.ts, r0, u.gbase, bar);
  if (ZM == 2) tma_2d(st + zero_off<TCAP>(), &L.tz, (2 * u.c.t0) & ~3, u.gbase, bar);
  if (ZM == 1) tma_2d(st + zero_off<TCAP>(), &L.tz, r0, u.gbase, bar);
}

template <int TCAP>
__device__ __forceinline__ void issue_x(const ChainParams& p, const Cursor& u, uint32_t st, uint32_t bar) {
  tma_3d(st + x_off<TCAP>(), &p.layer[u.l].tx, 0, u.gbase, 0, bar);
}

// ---------------------------------------------------------------------------
// consumer: x of a layer that reads an earlier layer's output (this warp's
// group of the stage, 4 values per lane of each batch row, from the exchange
// copy [M][K] of the source layer, K = this layer's input width)
// ---------------------------------------------------------------------------
template <int MB>
__device__ __forceinline__ void load_x(uint2 (&px)[MB], const LayerRun* runs, const char* xch, int l, int gbase,
                                       int w, int lane, int M) {
  const size_t K = size_t(runs[l].G) * kGroup;
  const char* a = xch + runs[run_x_from(runs[l])].ll_off + (size_t(gbase + w) * kGroup + 4 * lane) * 2;
#pragma unroll
  for (int m = 0; m < MB; ++m)
    if (m < M) px[m] = ll_get2(a + size_t(m) * K * 2);
}

template <int MB>
__device__ __forceinline__ bool x_complete(const uint2 (&px)[MB], int M) {
  bool got = true;
#pragma unroll
  for (int m = 0; m < MB; ++m)
    if (m < M) got = got && ll_complete(px[m]);
  return __all_sync(0xffffffffu, got);
}

// Whether this warp needs exchange x for the stage of layer l starting at group gbase.
__device__ __forceinline__ bool x_needed(const ChainParams& p, const LayerRun* runs, int l, int gbase, int w) {
  return l < p.n_layers && run_x_from(runs[l]) >= 0 && gbase + w < runs[l].ge;
}

// ---------------------------------------------------------------------------
// consumer: one stage of one warp (group w of up to four tiles)
// ---------------------------------------------------------------------------
template <int MB, int ZM>
__device__ __forceinline__ void stage_compute(uint32_t st, int w, int g, int t, int tc, int M, int zoff,
                                              float (&acc)[tile_cap<MB>()][MB > 8 ? 2 : 1][4]) {
  constexpr int TCAP = tile_cap<MB>();
  constexpr int MT = MB > 8 ? 2 : 1;
  constexpr bool ODD = MB > 1;        // batch columns 2t + 1 exist
  // x fragments: batch row m = 8 mt + g, this warp's group, k = 32 t .. 32 t + 31
  uint4 xf[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int m = 8 * mt + g;
    const uint32_t xa = st + x_off<TCAP>() + uint32_t(m) * kXRowBytes + w * 256 + t * 64;
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
  const uint32_t sbase = st + scale_off<TCAP>() + w * 128 + g * 2;
#pragma unroll
  for (int rt = 0; rt < TCAP; ++rt) {
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
        const uint2 zz = lds64(st + zero_off<TCAP>() + w * (kPackedZeroWords * 4) + zoff + rt * 8);
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
__global__ void __launch_bounds__(kThreads, MB <= 4 ? 2 : 1)
chain_kernel(const __grid_constant__ ChainParams p) {
  constexpr int MT = MB > 8 ? 2 : 1;
  constexpr int TCAP = tile_cap<MB>();
  asm volatile("griddepcontrol.launch_dependents;");
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const uint32_t full0 = sbase;                        // [S] mbarriers
  const uint32_t empty0 = sbase + kMaxStages * 8;      // [S] mbarriers
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kFlagsOff);
  LayerRun* runs = reinterpret_cast<LayerRun*>(smem + kTableOff);
  const uint32_t ring = sbase + header_bytes(p.n_layers);
  const int S = p.stages;
  const int warp = int(threadIdx.x) >> 5;
  const int lane = int(threadIdx.x) & 31;
  const unsigned long long limit = g_awq_chain_wait_limit_ns;
  const uint32_t hint = limit < 20000ull ? uint32_t(limit) : 20000u;   // sleep of one wait step, ns
  uint32_t* const ctl = reinterpret_cast<uint32_t*>(p.ws);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(full0 + 8 * s), "r"(1));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty0 + 8 * s), "r"(kCW));
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
  }
  for (int l = int(threadIdx.x); l < p.n_layers; l += int(blockDim.x)) fill_run(p.layer[l], runs[l]);
  __syncthreads();
  for (int l = int(threadIdx.x); l < p.n_layers; l += int(blockDim.x)) {
    int n = l + 1;
    while (n < p.n_layers && runs[n].i0 >= runs[n].i1) ++n;
    runs[l].next = n;
  }
  __syncthreads();

  if (warp == kCW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      Cursor cw;
      cursor_init<TCAP>(p, runs, cw);
      Cursor cx = cw;               // stages whose weights were issued before the wait
      int sw = 0;                   // stages issued
      if (p.early) {
        for (; sw < S && !cw.done(p.n_layers); ++sw) {
          issue_weights<ZM, TCAP>(p, runs, cw, ring + sw * p.stage_bytes, full0 + 8 * sw);
          cursor_next<TCAP>(p, runs, cw);
        }
      }
      asm volatile("griddepcontrol.wait;" ::: "memory");
      // x of those stages (layers whose x is an input of the call)
      for (int j = 0; j < sw; ++j) {
        if (run_x_from(runs[cx.l]) < 0) issue_x<TCAP>(p, cx, ring + j * p.stage_bytes, full0 + 8 * j);
        cursor_next<TCAP>(p, runs, cx);
      }
      uint64_t t_slot = 0;          // start of the wait for a free slot (0: not waiting)
      while (!cw.done(p.n_layers)) {
        const int slot = sw % S;
        if (sw < S || mbar_test_wait(empty0 + 8 * slot, uint32_t((sw / S) + 1) & 1u)) {
          const uint32_t st = ring + slot * p.stage_bytes;
          issue_weights<ZM, TCAP>(p, runs, cw, st, full0 + 8 * slot);
          if (run_x_from(runs[cw.l]) < 0) issue_x<TCAP>(p, cw, st, full0 + 8 * slot);
          cursor_next<TCAP>(p, runs, cw);
          ++sw;
          t_slot = 0;
          continue;
        }
        // nothing to do until the slot frees: sleep on its barrier
        mbar_sleep_wait(empty0 + 8 * slot, uint32_t((sw / S) + 1) & 1u, hint);
        if (*abort_flag) break;
        const uint64_t now = now_ns();
        if (t_slot == 0) {
          t_slot = now;
        } else if (now - t_slot > limit) {
          *abort_flag = 1;
          atomicOr(&g_awq_chain_error, kErrBit);
          break;
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
  } else {
    // ------------------------------------------------------------ consumers
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int w = warp;
    const int g = lane >> 2;
    const int t = lane & 3;
    const int M = p.M;
    const uint32_t pbuf = sbase + p.pbuf_offset;       // [warp][64 rows][M] fp32
    // The exchange half of this launch, and this CTA's share of the other
    // half to zero for the next launch (the previous launch, which used it,
    // has completed: griddepcontrol.wait above).
    const uint32_t epoch = ctl[kEpochWord];
    const uint32_t parity = epoch & 1u;
    const uint32_t tag = epoch + 1u;    // of this launch's partials (a zero-filled workspace holds tag 0)
    char* const xch = p.ws + p.ll_base + size_t(parity) * p.ll_half;
    {
      uint4* o = reinterpret_cast<uint4*>(p.ws + p.ll_base + size_t(parity ^ 1u) * p.ll_half);
      const uint32_t n16 = p.ll_half / 16;
      const uint32_t per = (n16 + gridDim.x - 1) / gridDim.x;
      const uint32_t b = blockIdx.x * per;
      const uint32_t e = b + per < n16 ? b + per : n16;
      for (uint32_t k = b + threadIdx.x; k < e; k += kCW * 32) o[k] = make_uint4(0u, 0u, 0u, 0u);
    }
    // x of a stage that reads an earlier layer's output: this warp's group,
    // 4 values per lane of each batch row, loaded one stage ahead
    uint2 px[MB];
    {
      // the first stage's x
      int l0 = 0;
      while (l0 < p.n_layers && runs[l0].i0 >= runs[l0].i1) ++l0;
      if (x_needed(p, runs, l0, runs[l0 < p.n_layers ? l0 : 0].gb, w))
        load_x<MB>(px, runs, xch, l0, runs[l0].gb, w, lane, M);
    }
    int slot = 0;
    uint32_t phase = 0;
    bool live = true;
    for (int l = 0; l < p.n_layers; ++l) {
      const LayerRun& R = runs[l];
      const int i1 = R.i1;
      const bool dep = run_x_from(R) >= 0;
      for (int i = R.i0; i < i1;) {
        Chunk cc;
        load_chunk<TCAP>(R, i, cc);
        float acc[TCAP][MT][4];
#pragma unroll
        for (int rt = 0; rt < TCAP; ++rt)
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[rt][mt][k] = 0.0f;
        for (int gbase = cc.gb; gbase < cc.ge; gbase += kCW) {
          const uint32_t st = ring + slot * p.stage_bytes;
          const uint32_t full = full0 + 8 * slot;
          const bool mine = gbase + w < cc.ge;
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
            if (live && dep && mine) {
              // the layer's x: every value written by this launch, else
              // reload until it is (bounded; the decisions are warp-uniform)
              if (!x_complete<MB>(px, M)) {
                const uint64_t t0 = now_ns();
                for (;;) {
                  load_x<MB>(px, runs, xch, l, gbase, w, lane, M);
                  if (x_complete<MB>(px, M)) break;
                  const bool late = now_ns() - t0 > limit;
                  if (__any_sync(0xffffffffu, late || *abort_flag != 0)) {
                    if (lane == 0 && late) {
                      *abort_flag = 1;
                      atomicOr(&g_awq_chain_error, kErrBit);
                    }
                    live = false;
                    break;
                  }
                }
              }
              if (live) {
#pragma unroll
                for (int m = 0; m < MB; ++m)
                  if (m < M) sts64(st + x_off<TCAP>() + uint32_t(m) * kXRowBytes + w * 256 + lane * 8, ll_decode(px[m]));
                __syncwarp();
              }
            }
          }
          if (live) {
            // the next stage's x: the next groups of this chunk, the next
            // chunk of this layer (same slice, so the same first group), or
            // the first stage of the next layer with items
            int nl = l, ng = gbase + kCW;
            if (ng >= cc.ge) {
              ng = cc.gb;
              if (i + cc.nu >= i1) {
                nl = R.next;
                ng = nl < p.n_layers ? runs[nl].gb : 0;
              }
            }
            if (x_needed(p, runs, nl, ng, w)) load_x<MB>(px, runs, xch, nl, ng, w, lane, M);
            if (mine) stage_compute<MB, ZM>(st, w, g, t, cc.tc, M, (cc.t0 & 1) * 8, acc);
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
        for (int rt = 0; rt < TCAP; ++rt) {
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
        // the layer's fields, read here (from the table) rather than kept in
        // registers through the stage loop
        const int ks = run_ks(R), tpu = run_tpu(R), silu = run_silu(R), N = R.N;
        const int T = R.units * tpu;
        const bool src = run_source(R) != 0;
        const int W = silu ? N / 2 : N;        // output columns
        uint16_t* const y = R.y;
        char* const xout = xch + R.ll_off;
        unsigned long long* const partials = reinterpret_cast<unsigned long long*>(p.ws + R.partial_off);
        const int64_t row0 = int64_t(cc.t0) * kTile;
        const int tid = int(threadIdx.x);
        // With K slices, every slice but the last stores its sums tagged
        // with the launch count; the CTA of the last slice waits for each
        // to carry this launch's tag and adds them in slice order, its own
        // sum last (the order of a sum over the slices from 0).
        const bool reducer = ks > 1 && cc.s == ks - 1;
        if (ks > 1 && !reducer) {
          const int V = kTile * cc.tc * M;
          for (int v = tid; v < V; v += kCW * 32) {
            float own = 0.0f;
#pragma unroll
            for (int ww = 0; ww < kCW; ++ww) own += lds_f32(pbuf + uint32_t(ww * 64 * M + v) * 4);
            put_tagged(partials + ((int64_t(cc.s) * T * kTile + row0) * M + v), tag, own);
          }
        } else if (!silu) {
          const int V = kTile * cc.tc * M;
          for (int v = tid; v < V; v += kCW * 32) {
            float sum = 0.0f;
#pragma unroll
            for (int ww = 0; ww < kCW; ++ww) sum += lds_f32(pbuf + uint32_t(ww * 64 * M + v) * 4);
            const int row = v / M;
            const int m = v - row * M;
            if (reducer) sum = slice_sum(partials, int64_t(T) * kTile * M, ks, (row0 + row) * M + m, tag, sum, abort_flag, limit);
            if (row0 + row < N) {
              const uint16_t h = __half_as_ushort(__float2half_rn(sum));
              y[int64_t(m) * N + row0 + row] = h;
              if (src) ll_put(xout, int64_t(m) * W + row0 + row, h);
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
            if (reducer) {
              const int64_t ss = int64_t(T) * kTile * M;
              gs = slice_sum(partials, ss, ks, (row0 + 2 * q * kTile) * M + rem, tag, gs, abort_flag, limit);
              us = slice_sum(partials, ss, ks, (row0 + (2 * q + 1) * kTile) * M + rem, tag, us, abort_flag, limit);
            }
            const int row = rem / M;
            const int m = rem - row * M;
            const uint16_t h = __half_as_ushort(__float2half_rn(silu_f32(gs) * us));
            y[int64_t(m) * W + row0 / 2 + q * kTile + row] = h;
            if (src) ll_put(xout, int64_t(m) * W + row0 / 2 + q * kTile + row, h);
          }
        }
        consumer_sync();   // pbuf is reused by the next chunk
        i += cc.nu;
      }
    }
  }
  __syncthreads();
  // The last CTA out resets the exit counter and counts the launch (the
  // parity of the count picks the exchange half of the next launch).
  if (threadIdx.x == 0) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(ctl + kExitWord) : "memory");
    if (old + 1 == gridDim.x) {
      ctl[kExitWord] = 0u;
      ctl[kEpochWord] += 1u;
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
using ChainFn = void (*)(const ChainParams);

constexpr int kNumVariants = 15;    // batch tile {1, 2, 4, 8, 16} x zero points {sym, fp16, packed}
constexpr int kSmemBudget = 232448;
constexpr int kHalfSmBudget = 115712;
constexpr int kMaxDevices = 64;

ChainFn pick(int64_t M, int zm, int& id) {
  static const ChainFn table[kNumVariants] = {
      chain_kernel<1, 0>, chain_kernel<1, 1>, chain_kernel<1, 2>,
      chain_kernel<8, 0>, chain_kernel<8, 1>, chain_kernel<8, 2>,
      chain_kernel<16, 0>, chain_kernel<16, 1>, chain_kernel<16, 2>,
      chain_kernel<2, 0>,  chain_kernel<2, 1>,  chain_kernel<2, 2>,
      chain_kernel<4, 0>,  chain_kernel<4, 1>,  chain_kernel<4, 2>};
  const int mb = M == 1 ? 0 : M == 2 ? 3 : M <= 4 ? 4 : M <= 8 ? 1 : 2;
  id = mb * 3 + zm;
  return table[id];
}

std::atomic<int> g_sms[kMaxDevices];
std::atomic<int> g_attr_set[kMaxDevices][kNumVariants];

struct LayerPlan {
  int T, tpu, units, ks, items, rot;
  size_t partial_off;                // workspace offset (ks > 1)
  int source;                        // a later layer reads this layer's output
  size_t ll_off;                     // its exchange copy, within each half
};

struct ChainPlan {
  ChainFn fn;
  int id, grid, stages, stage_bytes, pbuf_offset, smem, tcap;
  LayerPlan lp[kMaxLayers];
  size_t ll_base, ll_half;           // the exchange region: two halves
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
// per stage (waits, barriers), per chunk (the reduction through shared
// memory, the output stores) and per chunk of a split layer (the tagged
// partials). The constants are fitted to B200 timings of the Llama-3-8B
// decode step (4 slices for its 4096-row layers, none for the 14336-row
// ones).
int64_t split_cost(int units, int tpu, int G, int ks, int grid, int tcap) {
  constexpr int64_t kMinTiles = 3, kStageCost = 10, kChunkCost = 20, kSplitCost = 6;
  int64_t worst = 0;
  for (int b = 0; b < grid; ++b) {
    int i0, i1;
    split_items(units, ks, grid, b, i0, i1);
    int64_t c = 0;
    for (int i = i0; i < i1;) {
      const int sl = i / units, u0 = i - sl * units;
      int nu = i1 - i;
      if (nu > tcap / tpu) nu = tcap / tpu;
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
int pick_ks(int units, int tpu, int G, int grid, int tcap) {
  struct Key {
    int units, tpu, G, grid, tcap;
  };
  static std::mutex lock;
  static std::vector<std::pair<Key, int>> cache;
  {
    std::lock_guard<std::mutex> g(lock);
    for (const auto& e : cache)
      if (e.first.units == units && e.first.tpu == tpu && e.first.G == G && e.first.grid == grid &&
          e.first.tcap == tcap)
        return e.second;
  }
  int best = 1;
  int64_t best_cost = split_cost(units, tpu, G, 1, grid, tcap);
  const int cands[] = {2, 3, 4, 5, 6, 7, 8, 10, 12, 14, 16, 24, 32};
  for (int ks : cands) {
    if (ks > G || ks > grid) break;
    const int64_t c = split_cost(units, tpu, G, ks, grid, tcap);
    if (c < best_cost) {
      best_cost = c;
      best = ks;
    }
  }
  std::lock_guard<std::mutex> g(lock);
  if (cache.size() < 4096) cache.push_back({Key{units, tpu, G, grid, tcap}, best});
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
  // batch tiles of 2 and 4 rows: two-tile stages (see tile_cap)
  pl.tcap = (M == 2 || M == 3 || M == 4) ? tile_cap<2>() : kMaxTC;
  pl.stage_bytes = int(pl.tcap == 2 ? x_off<2>() : x_off<kMaxTC>()) + int(M) * kXRowBytes;
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
  size_t off = kControlBytes;   // exit counter, launch count
  int level_start = 0;
  int64_t extra = 0;
  for (int l = 0; l < n; ++l) {
    const awq_gemv_layer_t& L = layers[l];
    LayerPlan& lp = pl.lp[l];
    const int64_t G = L.K / kGroup;
    lp.T = int((L.N + kTile - 1) / kTile);
    lp.tpu = (L.cfg.flags & AWQ_FLAG_SILU_MUL) ? 2 : 1;
    lp.units = lp.T / lp.tpu;
    const int ks = pick_ks(lp.units, lp.tpu, int(G), pl.grid, pl.tcap);
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
      lp.partial_off = off;
      off += align256(size_t(lp.ks - 1) * size_t(lp.T) * kTile * size_t(M) * 8);
    } else {
      lp.partial_off = 0;
    }
    lp.source = 0;
    lp.ll_off = 0;
  }
  // The exchange region: a copy of the output of every layer that a later
  // layer reads, in each of two halves.
  size_t half = 0;
  for (int l = 0; l < n; ++l)
    if (layers[l].x_from >= 0) pl.lp[layers[l].x_from].source = 1;
  for (int l = 0; l < n; ++l) {
    if (!pl.lp[l].source) continue;
    const int64_t W = (layers[l].cfg.flags & AWQ_FLAG_SILU_MUL) ? layers[l].N / 2 : layers[l].N;
    pl.lp[l].ll_off = half;
    half += align256(size_t(M) * size_t(W) * 2);
  }
  pl.ll_base = off;
  pl.ll_half = half;
  off += 2 * half;
  pl.ws_bytes = off;
  // offsets travel to the kernel as 32-bit values
  if (pl.ws_bytes > size_t(0xFFFFFFFFu)) return AWQ_ERR_SHAPE;
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
    D.partial_off = uint32_t(lp.partial_off);
    D.ll_off = uint32_t(lp.ll_off);
    D.source = lp.source;
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
  p.ws = ws;
  p.ll_base = uint32_t(pl.ll_base);
  p.ll_half = uint32_t(pl.ll_half);
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
