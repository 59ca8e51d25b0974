// Activation-aware scale search and scale application.
//
// ("AutoAWQ" code tour, "The Quantization Flow Up Close": the search takes a
// per-channel mean of normalized weights and a float32 mean of activations,
// runs the fp16 module once as the reference and keeps the candidate scaling
// with the lowest output error; "From Install to Your First Model":
// duo_scaling uses both statistics; "The big picture": x / s against
// W diag(s) leaves the layer's output unchanged, so the scale only moves
// quantization error between channels.)
//
// For every grid point alpha = i / n_grid the candidate
//   s = max(mean|x|^alpha / (mean|w^|^(1 - alpha) + 1e-4), 1e-4)   (duo)
//   s = max(mean|x|^alpha, 1e-4)                                  (no duo)
// is divided by sqrt(max s * min s); W diag(s) (rounded to fp16) is quantized
// by the quantizer of awq_pseudo_quantize_pack reading W and s directly, (x /
// s) is multiplied by it with awq_gemv / awq_gemm, and the loss is the mean
// of (y_ref - y)^2 over the outputs, y_ref = fp16(x . W^T) on the tensor
// cores. Every step runs on the device in stream order; the best
// grid point (first minimum) is picked on the device too, so the call makes
// no host synchronization. Sums are taken in a fixed order: same inputs, same
// bits.

#include <cuda_fp16.h>

#include <atomic>

#include "awq_common.cuh"


namespace awq {

// the quantizer with a per-input-channel factor (awq_quant.cu)
awq_status_t quantize_pack_scaled(const uint16_t* W, const float* colscale, int64_t N, int64_t K, awq_qconfig_t cfg,
                                  int32_t* qweight, uint16_t* scales, uint16_t* zeros, void* stream);

namespace {

constexpr float kScaleEps = 1e-4f;
constexpr int kLossBlocks = 256;
constexpr int kWRowSplit = 16;       // row slices of the weight statistic
constexpr int kMaxGrid = 64;

__device__ __forceinline__ float h2f(uint16_t b) { return __half2float(__ushort_as_half(b)); }
__device__ __forceinline__ uint16_t f2h(float v) { return __half_as_ushort(__float2half_rn(v)); }

// mean over rows of |x[m][k]|: one thread per column, rows summed in order.
__global__ void act_mean_abs_kernel(const uint16_t* __restrict__ X, int64_t Ms, int64_t K, float* __restrict__ out) {
  const int64_t k = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k >= K) return;
  float sum = 0.0f;
  for (int64_t m = 0; m < Ms; ++m) sum += fabsf(h2f(X[m * K + k]));
  out[k] = sum / float(Ms);
}

// Partial sums over a slice of rows of |w[n][k]| / max |w[n][group of k]|.
// Block = one group of 128 columns x one row slice; thread = column.
__global__ void __launch_bounds__(128) weight_norm_partial_kernel(const uint16_t* __restrict__ W, int64_t N,
                                                                  int64_t K, float* __restrict__ partial) {
  __shared__ float wmax[4];
  const int k = blockIdx.x * 128 + threadIdx.x;
  const int slice = blockIdx.y;
  const int64_t n0 = N * slice / kWRowSplit, n1 = N * (slice + 1) / kWRowSplit;
  float sum = 0.0f;
  for (int64_t n = n0; n < n1; ++n) {
    const float a = fabsf(h2f(W[n * K + k]));
    float mx = a;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
    __syncthreads();
    sum += mx > 0.0f ? a / mx : 0.0f;
  }
  partial[int64_t(slice) * K + k] = sum;
}

__global__ void weight_norm_finish_kernel(const float* __restrict__ partial, int64_t N, int64_t K,
                                          float* __restrict__ out) {
  const int64_t k = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k >= K) return;
  float sum = 0.0f;
  for (int s = 0; s < kWRowSplit; ++s) sum += partial[int64_t(s) * K + k];
  out[k] = sum / float(N);
}

// y_ref[m][n] = fp16(sum_k x[m][k] w[n][k]) with fp32 accumulation on the
// tensor cores (mma.sync m16n8k16, fp16 operands): 128 x 128 output tiles,
// 8 warps of 64 (m) x 32 (n), k in steps of 32 through a two-stage
// cp.async ring. Shared rows are 64 bytes (32 halves); the 16-byte chunk c of
// row r sits at chunk c ^ ((r >> 1) & 3), so that the eight rows an ldmatrix
// reads fall in eight different bank groups. Rows past Ms or N are read as
// zeros (cp.async with no source bytes).
constexpr int kRefBM = 128, kRefBN = 128, kRefBK = 32, kRefThreads = 256;

__device__ __forceinline__ uint32_t ref_swz(int row, int chunk) {
  return uint32_t(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(a));
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kRefThreads) reference_product_kernel(const uint16_t* __restrict__ X,
                                                                        const uint16_t* __restrict__ W, int64_t Ms,
                                                                        int64_t N, int64_t K,
                                                                        uint16_t* __restrict__ y) {
  __shared__ __align__(128) uint8_t sm[2][2][kRefBM * kRefBK * 2];   // [stage][x, w][128 rows x 64 B]
  const int tid = int(threadIdx.x), lane = tid & 31, warp = tid >> 5;
  const int wm = warp >> 2, wn = warp & 3;            // warp tile: rows 64 wm.., columns 32 wn..
  const int64_t m0 = int64_t(blockIdx.y) * kRefBM, n0 = int64_t(blockIdx.x) * kRefBN;
  const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(sm));
  constexpr uint32_t kTileBytes = kRefBM * kRefBK * 2;

  // one stage: 128 rows x 4 chunks of x and of w, two chunks of each per thread
  auto load = [&](int stage, int64_t k0) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int idx = tid + e * kRefThreads, row = idx >> 2, chunk = idx & 3;
      const int64_t xm = m0 + row, wn_ = n0 + row;
      const uint32_t sx = base + uint32_t(stage) * 2 * kTileBytes + ref_swz(row, chunk);
      cp_async16(sx, X + (xm < Ms ? xm : 0) * K + k0 + chunk * 8, xm < Ms);
      cp_async16(sx + kTileBytes, W + (wn_ < N ? wn_ : 0) * K + k0 + chunk * 8, wn_ < N);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float acc[4][4][4] = {};
  const int nk = int(K / kRefBK);
  load(0, 0);
  for (int kb = 0; kb < nk; ++kb) {
    if (kb + 1 < nk) {
      load((kb + 1) & 1, int64_t(kb + 1) * kRefBK);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const uint32_t sx = base + uint32_t(kb & 1) * 2 * kTileBytes, sw = sx + kTileBytes;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {           // two k16 steps per stage
      uint32_t a[4][4], b[4][2];
#pragma unroll
      for (int i = 0; i < 4; ++i) {            // A: rows 64 wm + 16 i + (lane % 16), k half lane / 16
        const int row = wm * 64 + i * 16 + (lane & 15);
        ldsm_x4(sx + ref_swz(row, kk * 2 + (lane >> 4)), a[i][0], a[i][1], a[i][2], a[i][3]);
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {            // B: two n8 tiles per ldmatrix.x4
        const int row = wn * 32 + j * 16 + (lane & 7) + ((lane >> 4) << 3);
        ldsm_x4(sw + ref_swz(row, kk * 2 + ((lane >> 3) & 1)), b[2 * j][0], b[2 * j][1], b[2 * j + 1][0],
                b[2 * j + 1][1]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jn = 0; jn < 4; ++jn) mma16816(acc[i][jn], a[i], b[jn][0], b[jn][1]);
    }
    __syncthreads();
  }
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int jn = 0; jn < 4; ++jn) {
      const int64_t n = n0 + wn * 32 + jn * 8 + 2 * t;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t m = m0 + wm * 64 + i * 16 + g + 8 * h;
        if (m < Ms && n < N)   // N % 8 == 0: n + 1 < N too
          *reinterpret_cast<uint32_t*>(y + m * N + n) =
              uint32_t(f2h(acc[i][jn][2 * h])) | (uint32_t(f2h(acc[i][jn][2 * h + 1])) << 16);
      }
    }
}

// The candidate scales of grid point `idx` (idx < 0: the first minimum of
// losses[0 .. n_grid)), normalised by sqrt(max * min). One block.
__global__ void __launch_bounds__(1024) candidate_kernel(const float* __restrict__ x_mean,
                                                         const float* __restrict__ w_mean, int64_t K, int n_grid,
                                                         int idx, const float* __restrict__ losses, int duo,
                                                         float* __restrict__ s) {
  __shared__ float red_max[32], red_min[32];
  __shared__ int pick;
  if (threadIdx.x == 0) {
    int best = idx;
    if (best < 0) {
      best = 0;
      for (int i = 1; i < n_grid; ++i)
        if (losses[i] < losses[best]) best = i;
    }
    pick = best;
  }
  __syncthreads();
  const float a = float(pick) / float(n_grid);
  float mx = 0.0f, mn = 3.0e38f;
  for (int64_t k = threadIdx.x; k < K; k += blockDim.x) {
    float v = powf(x_mean[k], a);
    if (duo) v = v / (powf(w_mean[k], 1.0f - a) + kScaleEps);
    v = fmaxf(v, kScaleEps);
    s[k] = v;
    mx = fmaxf(mx, v);
    mn = fminf(mn, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  if ((threadIdx.x & 31) == 0) {
    red_max[threadIdx.x >> 5] = mx;
    red_min[threadIdx.x >> 5] = mn;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int nw = blockDim.x >> 5;
    mx = threadIdx.x < nw ? red_max[threadIdx.x] : 0.0f;
    mn = threadIdx.x < nw ? red_min[threadIdx.x] : 3.0e38f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    if (threadIdx.x == 0) {
      red_max[0] = mx;
      red_min[0] = mn;
    }
  }
  __syncthreads();
  const float norm = sqrtf(red_max[0] * red_min[0]);
  for (int64_t k = threadIdx.x; k < K; k += blockDim.x) s[k] = s[k] / norm;
}

// out[r][k] = fp16(in[r][k] * s[k]) (mul = 1) or fp16(in[r][k] / s[k]) (mul = 0),
// eight consecutive values (one 16-byte load and store) per thread; K % 8 == 0.
__global__ void scale_columns_kernel(const uint16_t* __restrict__ in, const float* __restrict__ s, int64_t rows,
                                     int64_t K, int mul, uint16_t* __restrict__ out) {
  const int64_t vecs = rows * K / 8;
  for (int64_t v = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; v < vecs; v += int64_t(gridDim.x) * blockDim.x) {
    const int64_t k0 = (v * 8) % K;
    const uint4 raw = reinterpret_cast<const uint4*>(in)[v];
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = h2f(uint16_t(w[e] & 0xFFFF)), b = h2f(uint16_t(w[e] >> 16));
      const float sa = s[k0 + 2 * e], sb = s[k0 + 2 * e + 1];
      o[e] = uint32_t(f2h(mul ? a * sa : a / sa)) | (uint32_t(f2h(mul ? b * sb : b / sb)) << 16);
    }
    reinterpret_cast<uint4*>(out)[v] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Squared differences summed per block in a fixed order (fp64), then the
// block sums in order; loss = total / count.
__global__ void __launch_bounds__(256) loss_partial_kernel(const uint16_t* __restrict__ a,
                                                           const uint16_t* __restrict__ b, int64_t count,
                                                           double* __restrict__ partial) {
  __shared__ double red[256];
  const int64_t per = (count + kLossBlocks - 1) / kLossBlocks;
  const int64_t i0 = per * blockIdx.x, i1 = i0 + per < count ? i0 + per : count;
  double sum = 0.0;
  for (int64_t i = i0 + threadIdx.x; i < i1; i += 256) {
    const double d = double(h2f(a[i])) - double(h2f(b[i]));
    sum += d * d;
  }
  red[threadIdx.x] = sum;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) partial[blockIdx.x] = red[0];
}

__global__ void loss_finish_kernel(const double* __restrict__ partial, int64_t count, float* __restrict__ loss) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    double sum = 0.0;
    for (int b = 0; b < kLossBlocks; ++b) sum += partial[b];
    *loss = float(sum / double(count));
  }
}

// ---------------------------------------------------------------------------
// Clip search ("AutoAWQ" code tour, "The Quantization Flow Up Close": the
// clipping pass shrinks extreme weights group by group where that lowers the
// output error). For row n and group j, grid point i tries the ratio
// r = 1 - max_shrink * i / n_grid: the group is clipped to [-t, t], t = r *
// max|w| (fp32), the clipped values rounded to fp16 and quantized as by
// awq_pseudo_quantize_pack; the error is d^T G_j d, d = w - w' and G_j =
// X_j^T X_j the Gram matrix of the calibration inputs over the group's 128
// input channels. The first ratio with the lowest error wins.
// ---------------------------------------------------------------------------
constexpr int kGramPad = kGroup + 1;   // row stride of a Gram matrix in shared memory (no bank conflicts)
constexpr int kClipRowsPerBlock = 64;

// G_j[a][b] = sum_m x[m][128 j + a] x[m][128 j + b] in fp32, rows of x in
// order. One block per group; thread (a, half) owns 64 entries of row a.
__global__ void __launch_bounds__(256) gram_kernel(const uint16_t* __restrict__ X, int64_t Ms, int64_t K,
                                                   float* __restrict__ gram) {
  __shared__ float xs[32][kGroup + 1];
  const int j = blockIdx.x;
  const int a = threadIdx.x >> 1;
  const int b0 = (threadIdx.x & 1) * 64;
  float acc[64];
#pragma unroll
  for (int b = 0; b < 64; ++b) acc[b] = 0.0f;
  for (int64_t m0 = 0; m0 < Ms; m0 += 32) {
    for (int i = threadIdx.x; i < 32 * kGroup; i += 256) {
      const int r = i >> 7, c = i & 127;
      xs[r][c] = (m0 + r < Ms) ? h2f(X[(m0 + r) * K + int64_t(j) * kGroup + c]) : 0.0f;
    }
    __syncthreads();
    for (int r = 0; r < 32; ++r) {
      const float xa = xs[r][a];
#pragma unroll
      for (int b = 0; b < 64; ++b) acc[b] = fmaf(xa, xs[r][b0 + b], acc[b]);
    }
    __syncthreads();
  }
  float* out = gram + (int64_t(j) * kGroup + a) * kGroup + b0;
#pragma unroll
  for (int b = 0; b < 64; ++b) out[b] = acc[b];
}

__device__ __forceinline__ float clip_ratio(int i, int n_grid, float max_shrink) {
  return __fsub_rn(1.0f, __fdiv_rn(__fmul_rn(max_shrink, float(i)), float(n_grid)));
}

// Block: one group j (its Gram matrix in shared memory) x 64 rows; warp: one
// row at a time, lane l holding k = l + 32 i of the group.
template <bool ZP>
__global__ void __launch_bounds__(256) clip_search_kernel(const uint16_t* __restrict__ W, int64_t N, int64_t K,
                                                          const float* __restrict__ gram, int n_grid,
                                                          float max_shrink, float* __restrict__ ratios) {
  extern __shared__ float clip_smem[];
  float* gs = clip_smem;                                          // [128][129]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* dbuf = clip_smem + kGroup * kGramPad + warp * kGroup;    // [128] per warp
  const int j = blockIdx.x;
  for (int i = threadIdx.x; i < kGroup * kGroup; i += 256)
    gs[(i >> 7) * kGramPad + (i & 127)] = gram[int64_t(j) * kGroup * kGroup + i];
  __syncthreads();
  const int64_t n_end = (int64_t(blockIdx.y) + 1) * kClipRowsPerBlock < N ? (int64_t(blockIdx.y) + 1) * kClipRowsPerBlock : N;
  for (int64_t n = int64_t(blockIdx.y) * kClipRowsPerBlock + warp; n < n_end; n += 8) {
    float w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = h2f(W[n * K + int64_t(j) * kGroup + lane + 32 * i]);
    float amax = fmaxf(fmaxf(fabsf(w[0]), fabsf(w[1])), fmaxf(fabsf(w[2]), fabsf(w[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float best_err = 0.0f;
    int best = 0;
    for (int it = 0; it < n_grid; ++it) {
      const float t = __fmul_rn(amax, clip_ratio(it, n_grid, max_shrink));
      float wc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) wc[i] = h2f(f2h(fminf(fmaxf(w[i], -t), t)));
      float sf, zf;
      group_quant_params<ZP>(wc, sf, zf);
      float d[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int q = group_quant_code<ZP>(wc[i], sf, zf);
        const float wq = h2f(f2h(__fmul_rn(__fsub_rn(float(q), zf), sf)));
        d[i] = __fsub_rn(w[i], wq);
        dbuf[lane + 32 * i] = d[i];
      }
      __syncwarp();
      float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      for (int b = 0; b < kGroup; ++b) {
        const float db = dbuf[b];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = fmaf(gs[(lane + 32 * i) * kGramPad + b], db, v[i]);
      }
      float e = d[0] * v[0] + d[1] * v[1] + d[2] * v[2] + d[3] * v[3];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
      e = __shfl_sync(0xffffffffu, e, 0);   // one value for the whole warp
      if (it == 0 || e < best_err) {
        best_err = e;
        best = it;
      }
      __syncwarp();
    }
    if (lane == 0) ratios[int64_t(j) * N + n] = clip_ratio(best, n_grid, max_shrink);
  }
}

// W_out = W clipped per (row, group) to [-t, t], t = ratio[j][n] * max|w|,
// values rounded to fp16. One warp per (row, group), four weights per lane.
__global__ void __launch_bounds__(256) apply_clip_kernel(const uint16_t* __restrict__ W,
                                                         const float* __restrict__ ratios, int64_t N, int64_t K,
                                                         uint16_t* __restrict__ W_out) {
  const int lane = threadIdx.x & 31;
  const int64_t G = K / kGroup, units = N * G;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t u = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; u < units; u += nwarps) {
    const int64_t n = u / G, j = u - n * G;
    const int64_t base = n * K + j * kGroup + lane * 4;
    float w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = h2f(W[base + i]);
    float amax = fmaxf(fmaxf(fabsf(w[0]), fabsf(w[1])), fmaxf(fabsf(w[2]), fabsf(w[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float t = __fmul_rn(amax, ratios[j * N + n]);
#pragma unroll
    for (int i = 0; i < 4; ++i) W_out[base + i] = f2h(fminf(fmaxf(w[i], -t), t));
  }
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

struct SearchLayout {
  size_t x_mean, w_mean, w_part, s, loss_part, y_ref, y_q, x_s, qweight, scales, zeros, prod_ws, total;
};

awq_status_t search_layout(int64_t N, int64_t K, int64_t Ms, awq_qconfig_t cfg, SearchLayout& L) {
  awq_qconfig_t plain = cfg;
  plain.flags = 0;
  size_t prod = 0;
  awq_status_t st = awq_workspace_bytes(Ms, N, K, plain, &prod);
  if (st != AWQ_OK) return st;
  const size_t G = size_t(K / kGroup);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  L.x_mean = take(size_t(K) * 4);
  L.w_mean = take(size_t(K) * 4);
  L.w_part = take(size_t(kWRowSplit) * size_t(K) * 4);
  L.s = take(size_t(K) * 4);
  L.loss_part = take(size_t(kLossBlocks) * 8);
  L.y_ref = take(size_t(Ms) * size_t(N) * 2);
  L.y_q = take(size_t(Ms) * size_t(N) * 2);
  L.x_s = take(size_t(Ms) * size_t(K) * 2);
  L.qweight = take(size_t(N) * size_t(K / 8) * 4);
  L.scales = take(G * size_t(N) * 2);
  L.zeros = take(cfg.zero_point ? G * size_t(N) * 2 : 0);
  L.prod_ws = take(prod);
  L.total = off;
  return AWQ_OK;
}

// SM count of the current device (cached per device; 148 on B200 if the query fails).
int device_sms() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) return 148;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

awq_status_t check_search_args(int64_t N, int64_t K, int64_t Ms, awq_qconfig_t cfg) {
  awq_status_t st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if (cfg.flags != 0) return AWQ_ERR_UNSUPPORTED;
  if ((st = check_nk(N, K)) != AWQ_OK) return st;
  if (N < 1 || N % 8 || Ms < 1 || Ms > (int64_t(1) << 24)) return AWQ_ERR_SHAPE;
  return AWQ_OK;
}

}  // namespace
}  // namespace awq

using namespace awq;

extern "C" awq_status_t awq_search_scale_workspace_bytes(int64_t N, int64_t K, int64_t Ms, awq_qconfig_t cfg,
                                                         size_t* bytes) {
  if (!bytes) return AWQ_ERR_NULL;
  awq_status_t st = check_search_args(N, K, Ms, cfg);
  if (st != AWQ_OK) return st;
  SearchLayout L;
  if ((st = search_layout(N, K, Ms, cfg, L)) != AWQ_OK) return st;
  *bytes = L.total;
  return AWQ_OK;
}

extern "C" awq_status_t awq_search_scale(const uint16_t* W, int64_t N, int64_t K, const uint16_t* X, int64_t Ms,
                                         awq_qconfig_t cfg, int n_grid, int duo, float* scales_out,
                                         float* losses_out, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  awq_status_t st = check_search_args(N, K, Ms, cfg);
  if (st != AWQ_OK) return st;
  if (n_grid < 1 || n_grid > kMaxGrid) return AWQ_ERR_SHAPE;
  if (!W || !X || !scales_out || !losses_out || !workspace) return AWQ_ERR_NULL;
  if (!aligned16(W) || !aligned16(X) || !aligned16(workspace) || !aligned16(scales_out)) return AWQ_ERR_ALIGN;
  SearchLayout L;
  if ((st = search_layout(N, K, Ms, cfg, L)) != AWQ_OK) return st;
  if (workspace_bytes < L.total) return AWQ_ERR_WORKSPACE;
  char* ws = static_cast<char*>(workspace);
  float* x_mean = reinterpret_cast<float*>(ws + L.x_mean);
  float* w_mean = reinterpret_cast<float*>(ws + L.w_mean);
  float* w_part = reinterpret_cast<float*>(ws + L.w_part);
  float* s = reinterpret_cast<float*>(ws + L.s);
  double* loss_part = reinterpret_cast<double*>(ws + L.loss_part);
  uint16_t* y_ref = reinterpret_cast<uint16_t*>(ws + L.y_ref);
  uint16_t* y_q = reinterpret_cast<uint16_t*>(ws + L.y_q);
  uint16_t* x_s = reinterpret_cast<uint16_t*>(ws + L.x_s);
  int32_t* qweight = reinterpret_cast<int32_t*>(ws + L.qweight);
  uint16_t* qscales = reinterpret_cast<uint16_t*>(ws + L.scales);
  uint16_t* qzeros = cfg.zero_point ? reinterpret_cast<uint16_t*>(ws + L.zeros) : nullptr;
  void* prod_ws = ws + L.prod_ws;
  const size_t prod_bytes = L.total - L.prod_ws;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);

  // the product's workspace must start zero-filled
  if (prod_bytes && cudaMemsetAsync(prod_ws, 0, prod_bytes, cs) != cudaSuccess) return AWQ_ERR_CUDA;
  const int kb = int((K + 255) / 256);
  act_mean_abs_kernel<<<kb, 256, 0, cs>>>(X, Ms, K, x_mean);
  weight_norm_partial_kernel<<<dim3(unsigned(K / 128), kWRowSplit), 128, 0, cs>>>(W, N, K, w_part);
  weight_norm_finish_kernel<<<kb, 256, 0, cs>>>(w_part, N, K, w_mean);
  reference_product_kernel<<<dim3(unsigned((N + kRefBN - 1) / kRefBN), unsigned((Ms + kRefBM - 1) / kRefBM)),
                             kRefThreads, 0, cs>>>(X, W, Ms, N, K, y_ref);
  if ((st = launch_status()) != AWQ_OK) return st;
  const int64_t outs = Ms * N;
  const int sgrid = device_sms() * 8;   // grid-stride column scaling: eight CTAs per SM
  for (int i = 0; i < n_grid; ++i) {
    candidate_kernel<<<1, 1024, 0, cs>>>(x_mean, w_mean, K, n_grid, i, losses_out, duo, s);
    scale_columns_kernel<<<sgrid, 256, 0, cs>>>(X, s, Ms, K, 0, x_s);
    if ((st = launch_status()) != AWQ_OK) return st;
    // W diag(s) is quantized straight from W (never stored)
    if ((st = quantize_pack_scaled(W, s, N, K, cfg, qweight, qscales, qzeros, stream)) != AWQ_OK) return st;
    st = Ms <= 16 ? awq_gemv(x_s, qweight, qscales, qzeros, Ms, N, K, cfg, y_q, prod_ws, prod_bytes, stream)
                  : awq_gemm(x_s, qweight, qscales, qzeros, Ms, N, K, cfg, y_q, prod_ws, prod_bytes, stream);
    if (st != AWQ_OK) return st;
    loss_partial_kernel<<<kLossBlocks, 256, 0, cs>>>(y_ref, y_q, outs, loss_part);
    loss_finish_kernel<<<1, 32, 0, cs>>>(loss_part, outs, losses_out + i);
  }
  candidate_kernel<<<1, 1024, 0, cs>>>(x_mean, w_mean, K, n_grid, -1, losses_out, duo, scales_out);
  return launch_status();
}

extern "C" awq_status_t awq_apply_scale(const uint16_t* W, const float* s, int64_t N, int64_t K, uint16_t* W_out,
                                        void* stream) {
  if (N < 0 || K <= 0) return AWQ_ERR_SHAPE;
  if (N == 0) return AWQ_OK;
  if (K % 8) return AWQ_ERR_SHAPE;
  if (!W || !s || !W_out) return AWQ_ERR_NULL;
  if (!aligned16(W) || !aligned16(W_out)) return AWQ_ERR_ALIGN;
  scale_columns_kernel<<<device_sms() * 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(W, s, N, K, 1, W_out);
  return launch_status();
}

extern "C" awq_status_t awq_search_clip_workspace_bytes(int64_t K, size_t* bytes) {
  if (!bytes) return AWQ_ERR_NULL;
  if (K <= 0 || K % kGroup) return AWQ_ERR_SHAPE;
  *bytes = size_t(K / kGroup) * kGroup * kGroup * 4;
  return AWQ_OK;
}

extern "C" awq_status_t awq_search_clip(const uint16_t* W, int64_t N, int64_t K, const uint16_t* X, int64_t Ms,
                                        awq_qconfig_t cfg, int n_grid, float max_shrink, float* ratios_out,
                                        void* workspace, size_t workspace_bytes, void* stream) {
  awq_status_t st = check_search_args(N, K, Ms, cfg);
  if (st != AWQ_OK) return st;
  if (n_grid < 1 || n_grid > kMaxGrid || !(max_shrink >= 0.0f && max_shrink < 1.0f)) return AWQ_ERR_SHAPE;
  if (!W || !X || !ratios_out || !workspace) return AWQ_ERR_NULL;
  if (!aligned16(workspace)) return AWQ_ERR_ALIGN;
  const size_t need = size_t(K / kGroup) * kGroup * kGroup * 4;
  if (workspace_bytes < need) return AWQ_ERR_WORKSPACE;
  float* gram = static_cast<float*>(workspace);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const unsigned G = unsigned(K / kGroup);
  gram_kernel<<<G, 256, 0, cs>>>(X, Ms, K, gram);
  const size_t smem = size_t(kGroup * kGramPad + 8 * kGroup) * 4;
  const dim3 grid(G, unsigned((N + kClipRowsPerBlock - 1) / kClipRowsPerBlock));
  if (cfg.zero_point) {
    if (cudaFuncSetAttribute(clip_search_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
        cudaSuccess)
      return AWQ_ERR_CUDA;
    clip_search_kernel<true><<<grid, 256, smem, cs>>>(W, N, K, gram, n_grid, max_shrink, ratios_out);
  } else {
    if (cudaFuncSetAttribute(clip_search_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
        cudaSuccess)
      return AWQ_ERR_CUDA;
    clip_search_kernel<false><<<grid, 256, smem, cs>>>(W, N, K, gram, n_grid, max_shrink, ratios_out);
  }
  return launch_status();
}

extern "C" awq_status_t awq_apply_clip(const uint16_t* W, const float* ratios, int64_t N, int64_t K,
                                       uint16_t* W_out, void* stream) {
  if (N < 0 || K <= 0 || K % kGroup) return AWQ_ERR_SHAPE;
  if (N == 0) return AWQ_OK;
  if (!W || !ratios || !W_out) return AWQ_ERR_NULL;
  if (!aligned16(W) || !aligned16(W_out)) return AWQ_ERR_ALIGN;
  const int64_t units = N * (K / kGroup);
  const int64_t blocks = (units + 7) / 8;
  const int64_t cap = int64_t(device_sms()) * 16;
  apply_clip_kernel<<<unsigned(blocks < cap ? blocks : cap), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      W, ratios, N, K, W_out);
  return launch_status();
}
