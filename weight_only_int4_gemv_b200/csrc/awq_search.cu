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
// is divided by sqrt(max s * min s); W diag(s) is quantized by
// awq_pseudo_quantize_pack, (x / s) is multiplied by it with awq_gemv /
// awq_gemm, and the loss is the mean of (y_ref - y)^2 over the outputs, y_ref
// = fp16(x . W^T). Every step runs on the device in stream order; the best
// grid point (first minimum) is picked on the device too, so the call makes
// no host synchronization. Sums are taken in a fixed order: same inputs, same
// bits.

#include <cuda_fp16.h>

#include "awq_common.cuh"


namespace awq {
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

// y_ref[m][n] = fp16(sum_k x[m][k] w[n][k]) in fp32: 64 x 64 output tiles,
// 256 threads of 4 x 4 outputs, k in steps of 32 through shared memory.
__global__ void __launch_bounds__(256) reference_product_kernel(const uint16_t* __restrict__ X,
                                                                const uint16_t* __restrict__ W, int64_t Ms,
                                                                int64_t N, int64_t K, uint16_t* __restrict__ y) {
  __shared__ float xs[64][33];
  __shared__ float ws[64][33];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t m0 = int64_t(blockIdx.y) * 64, n0 = int64_t(blockIdx.x) * 64;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < K; k0 += 32) {
    for (int i = threadIdx.x; i < 64 * 32; i += 256) {
      const int r = i >> 5, c = i & 31;
      xs[r][c] = (m0 + r < Ms) ? h2f(X[(m0 + r) * K + k0 + c]) : 0.0f;
      ws[r][c] = (n0 + r < N) ? h2f(W[(n0 + r) * K + k0 + c]) : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < 32; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = xs[ty * 4 + i][c];
        b[i] = ws[tx * 4 + i][c];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < Ms && n < N) y[m * N + n] = f2h(acc[i][j]);
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

// out[r][k] = fp16(in[r][k] * s[k]) (mul = 1) or fp16(in[r][k] / s[k]) (mul = 0)
__global__ void scale_columns_kernel(const uint16_t* __restrict__ in, const float* __restrict__ s, int64_t rows,
                                     int64_t K, int mul, uint16_t* __restrict__ out) {
  const int64_t total = rows * K;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
    const float v = h2f(in[i]);
    const float sk = s[i % K];
    out[i] = f2h(mul ? v * sk : v / sk);
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

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

struct SearchLayout {
  size_t x_mean, w_mean, w_part, s, loss_part, y_ref, y_q, w_s, x_s, qweight, scales, zeros, prod_ws, total;
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
  L.w_s = take(size_t(N) * size_t(K) * 2);
  L.x_s = take(size_t(Ms) * size_t(K) * 2);
  L.qweight = take(size_t(N) * size_t(K / 8) * 4);
  L.scales = take(G * size_t(N) * 2);
  L.zeros = take(cfg.zero_point ? G * size_t(N) * 2 : 0);
  L.prod_ws = take(prod);
  L.total = off;
  return AWQ_OK;
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
  uint16_t* w_s = reinterpret_cast<uint16_t*>(ws + L.w_s);
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
  reference_product_kernel<<<dim3(unsigned((N + 63) / 64), unsigned((Ms + 63) / 64)), 256, 0, cs>>>(X, W, Ms, N, K,
                                                                                                   y_ref);
  if ((st = launch_status()) != AWQ_OK) return st;
  const int64_t outs = Ms * N;
  const int sgrid = 148 * 8;
  for (int i = 0; i < n_grid; ++i) {
    candidate_kernel<<<1, 1024, 0, cs>>>(x_mean, w_mean, K, n_grid, i, losses_out, duo, s);
    scale_columns_kernel<<<sgrid, 256, 0, cs>>>(W, s, N, K, 1, w_s);
    scale_columns_kernel<<<sgrid, 256, 0, cs>>>(X, s, Ms, K, 0, x_s);
    if ((st = launch_status()) != AWQ_OK) return st;
    if ((st = awq_pseudo_quantize_pack(w_s, N, K, cfg, qweight, qscales, qzeros, stream)) != AWQ_OK) return st;
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
  if (!W || !s || !W_out) return AWQ_ERR_NULL;
  scale_columns_kernel<<<148 * 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(W, s, N, K, 1, W_out);
  return launch_status();
}
