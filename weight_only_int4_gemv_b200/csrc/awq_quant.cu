// Group-wise INT4 quantize + pack, and dequant, for sm_100a.
//
// Quantization rule ("AutoAWQ" code tour, "The Quantization Flow Up Close":
// each group of weights is rounded to integer levels against its scale and
// zero point; symmetric decode from "AWQ Quantization Support", section
// "Dequantization Formula"): per (row n, group j), IEEE fp32 arithmetic with
// round to nearest even,
//   asymmetric: s = fp16(max((max - min) / 15, 1e-5)), z = clamp(-rint(min / s), 0, 15),
//               q = clamp(rint(w / s) + z, 0, 15)
//   symmetric:  s = fp16(max(max|w| / 7, 1e-5)),        q = clamp(rint(w / s), -8, 7) + 8
// The explicit _rn intrinsics keep every operation a single IEEE rounding,
// so the codes are bit-exact whatever contraction flags the file is built with.

#include "awq_common.cuh"

namespace awq {
namespace {

constexpr int kQuantThreads = 256;

// One warp per (row, group) unit. Lane l holds k = 4l .. 4l+3 of the group:
// a coalesced 256-byte read per warp, min/max by butterfly shuffles, and
// the packed word of k = 8w .. 8w+7 assembled from lanes 2w and 2w+1. A warp
// reads the groups of kUnitsAhead units before working on the first (1:
// reading 2 or 4 ahead measured 10 % slower on B200, the grid already keeps
// enough reads in flight). SCALED: the weights are first multiplied by a
// per-input-channel factor and rounded to fp16, exactly as awq_apply_scale
// writes them (the scale search quantizes W diag(s) without storing it).
constexpr int kUnitsAhead = 1;

template <bool ZP, bool SCALED>
__global__ void __launch_bounds__(kQuantThreads)
quantize_pack_kernel(const uint16_t* __restrict__ W, const float* __restrict__ colscale, int64_t N, int64_t K,
                     int32_t* __restrict__ qweight, uint16_t* __restrict__ scales,
                     uint16_t* __restrict__ zeros) {
  const int lane = threadIdx.x & 31;
  const int64_t G = K / kGroup;
  const int64_t units = N * G;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t u0 = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; u0 < units; u0 += kUnitsAhead * nwarps) {
  uint2 raws[kUnitsAhead];
#pragma unroll
  for (int a = 0; a < kUnitsAhead; ++a) {
    const int64_t u = u0 + a * nwarps;
    if (u < units) {
      const int64_t n = u / G, j = u - n * G;
      raws[a] = *reinterpret_cast<const uint2*>(W + n * K + j * kGroup + lane * 4);
    }
  }
#pragma unroll
  for (int a = 0; a < kUnitsAhead; ++a) {
    const int64_t u = u0 + a * nwarps;
    if (u >= units) break;
    const int64_t n = u / G;
    const int64_t j = u - n * G;
    const uint2 raw = raws[a];
    float w[4];
    w[0] = half_bits_to_float(uint16_t(raw.x & 0xFFFF));
    w[1] = half_bits_to_float(uint16_t(raw.x >> 16));
    w[2] = half_bits_to_float(uint16_t(raw.y & 0xFFFF));
    w[3] = half_bits_to_float(uint16_t(raw.y >> 16));
    if (SCALED) {
      const float4 cs = *reinterpret_cast<const float4*>(colscale + j * kGroup + lane * 4);
      w[0] = half_bits_to_float(__half_as_ushort(__float2half_rn(__fmul_rn(w[0], cs.x))));
      w[1] = half_bits_to_float(__half_as_ushort(__float2half_rn(__fmul_rn(w[1], cs.y))));
      w[2] = half_bits_to_float(__half_as_ushort(__float2half_rn(__fmul_rn(w[2], cs.z))));
      w[3] = half_bits_to_float(__half_as_ushort(__float2half_rn(__fmul_rn(w[3], cs.w))));
    }

    int q[4];
    float sf, zf;
    group_quant_params<ZP>(w, sf, zf);
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = group_quant_code<ZP>(w[i], sf, zf);

    // k offset o of the word goes to slot (o even ? o/2 : 4 + o/2).
    // Even lane: offsets 0..3 -> slots 0,4,1,5; odd lane: offsets 4..7 -> slots 2,6,3,7.
    uint32_t part;
    if ((lane & 1) == 0)
      part = uint32_t(q[0]) | (uint32_t(q[1]) << 16) | (uint32_t(q[2]) << 4) | (uint32_t(q[3]) << 20);
    else
      part = (uint32_t(q[0]) << 8) | (uint32_t(q[1]) << 24) | (uint32_t(q[2]) << 12) |
             (uint32_t(q[3]) << 28);
    const uint32_t other = __shfl_xor_sync(0xffffffffu, part, 1);
    if ((lane & 1) == 0)
      qweight[n * (K / 8) + j * kWordsPerGroup + (lane >> 1)] = int32_t(part | other);
    if (lane == 0) {  // metadata is group-major: [j][n]
      scales[j * N + n] = __half_as_ushort(__float2half_rn(sf));
      if (ZP) zeros[j * N + n] = __half_as_ushort(__int2half_rn(int(zf)));
    }
  }
  }
}

// Zero points fp16 [G][N] <-> packed int32 [G][N/8]: word i holds the values
// 8i .. 8i+7 of the flat array, value 8i + c in bits 4c .. 4c+3. Packing
// rounds to the nearest integer (ties to even) and clamps to 0..15 (NaN -> 0).
__global__ void __launch_bounds__(256)
pack_zeros_kernel(const uint16_t* __restrict__ zeros, int64_t words, int32_t* __restrict__ qzeros) {
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < words; i += stride) {
    const uint4 v = *reinterpret_cast<const uint4*>(zeros + i * 8);
    const uint32_t h[4] = {v.x, v.y, v.z, v.w};
    uint32_t word = 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float f = half_bits_to_float(uint16_t(h[c >> 1] >> (16 * (c & 1))));
      const float q = fminf(fmaxf(rintf(f), 0.0f), 15.0f);   // fmaxf(NaN, 0) = 0
      word |= uint32_t(q) << (4 * c);
    }
    qzeros[i] = int32_t(word);
  }
}

__global__ void __launch_bounds__(256)
unpack_zeros_kernel(const int32_t* __restrict__ qzeros, int64_t words, uint16_t* __restrict__ zeros) {
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < words; i += stride) {
    const uint32_t word = uint32_t(qzeros[i]);
    uint32_t h[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) h[c] = __half_as_ushort(__uint2half_rn((word >> (4 * c)) & 0xFu));
    uint4 v;
    v.x = h[0] | (h[1] << 16);
    v.y = h[2] | (h[3] << 16);
    v.z = h[4] | (h[5] << 16);
    v.w = h[6] | (h[7] << 16);
    *reinterpret_cast<uint4*>(zeros + i * 8) = v;
  }
}

// One thread per packed word: eight fp16 outputs written as one 16-byte store.
// w' = fp16((q - z) * s): the fp32 product is exact, so one rounding.
// ZP: 0 symmetric (z = 8), 1 fp16 zero points [G][N], 2 packed zero points
// int32 [G][N/8] (channel n in bits 4 (n % 8) of word n / 8).
template <int ZP>
__global__ void __launch_bounds__(256)
dequant_kernel(const int32_t* __restrict__ qweight, const uint16_t* __restrict__ scales,
               const void* __restrict__ zeros, int64_t N, int64_t K,
               uint16_t* __restrict__ out) {
  const int64_t wpr = K / 8;
  const int64_t words = N * wpr;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < words; i += stride) {
    const int64_t n = i / wpr;
    const int64_t wi = i - n * wpr;
    const int64_t j = (wi * 8) / kGroup;
    const int64_t g = j * N + n;   // group-major metadata
    const float sf = half_bits_to_float(scales[g]);
    float zf = 8.0f;
    if (ZP == 1) zf = half_bits_to_float(static_cast<const uint16_t*>(zeros)[g]);
    if (ZP == 2)
      zf = float((uint32_t(static_cast<const int32_t*>(zeros)[j * (N / 8) + n / 8]) >> (4 * (n % 8))) & 0xFu);
    const uint32_t word = uint32_t(qweight[i]);
    uint32_t h[8];
#pragma unroll
    for (int o = 0; o < 8; ++o) {
      const int slot = (o & 1) ? 4 + (o >> 1) : (o >> 1);
      const float q = float((word >> (4 * slot)) & 0xFu);
      h[o] = __half_as_ushort(__float2half_rn(__fmul_rn(__fsub_rn(q, zf), sf)));
    }
    uint4 v;
    v.x = h[0] | (h[1] << 16);
    v.y = h[2] | (h[3] << 16);
    v.z = h[4] | (h[5] << 16);
    v.w = h[6] | (h[7] << 16);
    *reinterpret_cast<uint4*>(out + i * 8) = v;
  }
}

int grid_for(int64_t work_items, int threads_per_item, int threads_per_block) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (work_items * threads_per_item + threads_per_block - 1) / threads_per_block;
  const int64_t cap = int64_t(sms) * 8;
  return int(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

// W diag(colscale) (colscale null: W) quantized and packed as by
// awq_pseudo_quantize_pack; arguments already checked by the caller.
awq_status_t quantize_pack_scaled(const uint16_t* W, const float* colscale, int64_t N, int64_t K, awq_qconfig_t cfg,
                                  int32_t* qweight, uint16_t* scales, uint16_t* zeros, void* stream) {
  const int64_t units = N * (K / kGroup);
  if (units == 0) return AWQ_OK;
  const int grid = grid_for((units + kUnitsAhead - 1) / kUnitsAhead, 32, kQuantThreads);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (colscale) {
    if (cfg.zero_point)
      quantize_pack_kernel<true, true><<<grid, kQuantThreads, 0, s>>>(W, colscale, N, K, qweight, scales, zeros);
    else
      quantize_pack_kernel<false, true><<<grid, kQuantThreads, 0, s>>>(W, colscale, N, K, qweight, scales, nullptr);
  } else {
    if (cfg.zero_point)
      quantize_pack_kernel<true, false><<<grid, kQuantThreads, 0, s>>>(W, nullptr, N, K, qweight, scales, zeros);
    else
      quantize_pack_kernel<false, false><<<grid, kQuantThreads, 0, s>>>(W, nullptr, N, K, qweight, scales, nullptr);
  }
  return launch_status();
}

}  // namespace awq

using namespace awq;

extern "C" awq_status_t awq_pseudo_quantize_pack(const uint16_t* W, int64_t N, int64_t K,
                                                 awq_qconfig_t cfg, int32_t* qweight,
                                                 uint16_t* scales, uint16_t* zeros,
                                                 void* stream) {
  awq_status_t st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if ((st = check_nk(N, K)) != AWQ_OK) return st;
  if (N == 0) return AWQ_OK;
  if (!W || !qweight || !scales) return AWQ_ERR_NULL;
  if (cfg.zero_point && !zeros) return AWQ_ERR_NULL;
  if (!cfg.zero_point && zeros) return AWQ_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(qweight) || !aligned16(scales) || (zeros && !aligned16(zeros)))
    return AWQ_ERR_ALIGN;
  return quantize_pack_scaled(W, nullptr, N, K, cfg, qweight, scales, zeros, stream);
}

extern "C" awq_status_t awq_dequant(const int32_t* qweight, const uint16_t* scales,
                                    const uint16_t* zeros, int64_t N, int64_t K,
                                    awq_qconfig_t cfg, uint16_t* W_out, void* stream) {
  awq_status_t st = check_cfg(cfg, true);
  if (st != AWQ_OK) return st;
  if ((st = check_nk(N, K)) != AWQ_OK) return st;
  if ((cfg.flags & AWQ_FLAG_PACKED_ZEROS) && N % 8) return AWQ_ERR_SHAPE;
  if (N == 0) return AWQ_OK;
  if (!qweight || !scales || !W_out) return AWQ_ERR_NULL;
  if (cfg.zero_point && !zeros) return AWQ_ERR_NULL;
  if (!cfg.zero_point && zeros) return AWQ_ERR_SHAPE;
  if (!aligned16(qweight) || !aligned16(scales) || !aligned16(W_out) || (zeros && !aligned16(zeros)))
    return AWQ_ERR_ALIGN;
  const int64_t words = N * (K / 8);
  const int grid = grid_for(words, 1, 256);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (zero_mode(cfg)) {
    case 2: dequant_kernel<2><<<grid, 256, 0, s>>>(qweight, scales, zeros, N, K, W_out); break;
    case 1: dequant_kernel<1><<<grid, 256, 0, s>>>(qweight, scales, zeros, N, K, W_out); break;
    default: dequant_kernel<0><<<grid, 256, 0, s>>>(qweight, scales, nullptr, N, K, W_out); break;
  }
  return launch_status();
}

extern "C" awq_status_t awq_pack_zeros(const uint16_t* zeros, int64_t G, int64_t N, int32_t* qzeros,
                                       void* stream) {
  if (G < 0 || N < 0 || N % 8 || G > (int64_t(1) << 30) || N > (int64_t(1) << 31) - 1) return AWQ_ERR_SHAPE;
  if (G == 0 || N == 0) return AWQ_OK;
  if (!zeros || !qzeros) return AWQ_ERR_NULL;
  if (!aligned16(zeros) || !aligned16(qzeros)) return AWQ_ERR_ALIGN;
  const int64_t words = G * (N / 8);
  pack_zeros_kernel<<<grid_for(words, 1, 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(zeros, words, qzeros);
  return launch_status();
}

extern "C" awq_status_t awq_unpack_zeros(const int32_t* qzeros, int64_t G, int64_t N, uint16_t* zeros,
                                         void* stream) {
  if (G < 0 || N < 0 || N % 8 || G > (int64_t(1) << 30) || N > (int64_t(1) << 31) - 1) return AWQ_ERR_SHAPE;
  if (G == 0 || N == 0) return AWQ_OK;
  if (!zeros || !qzeros) return AWQ_ERR_NULL;
  if (!aligned16(zeros) || !aligned16(qzeros)) return AWQ_ERR_ALIGN;
  const int64_t words = G * (N / 8);
  unpack_zeros_kernel<<<grid_for(words, 1, 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(qzeros, words, zeros);
  return launch_status();
}

// The AWQ_FLAG_SILU_MUL layout from a gate and an up projection: 16-row tiles
// alternating gate, up, in qweight rows and in the N columns of the
// group-major scales and zero points ("AutoAWQ" code tour, "The Quantization
// Flow Up Close": gate and up merged into one MLP block). Plain 2-D copies.
extern "C" awq_status_t awq_interleave_gate_up(const int32_t* qweight_gate, const uint16_t* scales_gate,
                                               const uint16_t* zeros_gate, const int32_t* qweight_up,
                                               const uint16_t* scales_up, const uint16_t* zeros_up, int64_t N,
                                               int64_t K, awq_qconfig_t cfg, int32_t* qweight_out,
                                               uint16_t* scales_out, uint16_t* zeros_out, void* stream) {
  awq_status_t st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if ((st = check_nk(N, K)) != AWQ_OK) return st;
  if (N % 16) return AWQ_ERR_SHAPE;
  if (N == 0) return AWQ_OK;
  if (!qweight_gate || !scales_gate || !qweight_up || !scales_up || !qweight_out || !scales_out)
    return AWQ_ERR_NULL;
  if (cfg.zero_point && (!zeros_gate || !zeros_up || !zeros_out)) return AWQ_ERR_NULL;
  if (!cfg.zero_point && (zeros_gate || zeros_up || zeros_out)) return AWQ_ERR_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t tile_bytes = size_t(16) * size_t(K / 8) * 4;   // one 16-row tile of qweight
  const size_t tiles = size_t(N / 16);
  const size_t runs = size_t(K / kGroup) * tiles;               // 16-value runs of a [G][N] array
  char* qo = reinterpret_cast<char*>(qweight_out);
  if (cudaMemcpy2DAsync(qo, 2 * tile_bytes, qweight_gate, tile_bytes, tile_bytes, tiles,
                        cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
      cudaMemcpy2DAsync(qo + tile_bytes, 2 * tile_bytes, qweight_up, tile_bytes, tile_bytes, tiles,
                        cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return AWQ_ERR_CUDA;
  const uint16_t* src_g[2] = {scales_gate, zeros_gate};
  const uint16_t* src_u[2] = {scales_up, zeros_up};
  uint16_t* dst[2] = {scales_out, zeros_out};
  for (int a = 0; a < (cfg.zero_point ? 2 : 1); ++a) {
    char* d = reinterpret_cast<char*>(dst[a]);
    if (cudaMemcpy2DAsync(d, 64, src_g[a], 32, 32, runs, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
        cudaMemcpy2DAsync(d + 32, 64, src_u[a], 32, 32, runs, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return AWQ_ERR_CUDA;
  }
  return launch_status();
}

// Projections sharing K concatenated along N (the fuser's fuse_qkv, "AutoAWQ"
// code tour, "The Quantization Flow Up Close"). Plain 2-D copies.
extern "C" awq_status_t awq_concat_rows(int parts, const int32_t* const* qweights, const uint16_t* const* scales,
                                        const uint16_t* const* zeros, const int64_t* Ns, int64_t K,
                                        awq_qconfig_t cfg, int32_t* qweight_out, uint16_t* scales_out,
                                        uint16_t* zeros_out, void* stream) {
  awq_status_t st = check_cfg(cfg);
  if (st != AWQ_OK) return st;
  if (parts < 1 || parts > 16) return AWQ_ERR_SHAPE;
  if (!qweights || !scales || !Ns || (cfg.zero_point && !zeros)) return AWQ_ERR_NULL;
  int64_t total = 0;
  for (int i = 0; i < parts; ++i) {
    if ((st = check_nk(Ns[i], K)) != AWQ_OK) return st;
    total += Ns[i];
  }
  if ((st = check_nk(total, K)) != AWQ_OK) return st;
  if (total == 0) return AWQ_OK;
  if (!qweight_out || !scales_out) return AWQ_ERR_NULL;
  if (cfg.zero_point && !zeros_out) return AWQ_ERR_NULL;
  if (!cfg.zero_point && zeros_out) return AWQ_ERR_SHAPE;
  for (int i = 0; i < parts; ++i) {
    if (Ns[i] == 0) continue;
    if (!qweights[i] || !scales[i]) return AWQ_ERR_NULL;
    if (cfg.zero_point && !zeros[i]) return AWQ_ERR_NULL;
    if (!cfg.zero_point && zeros && zeros[i]) return AWQ_ERR_SHAPE;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t row_bytes = size_t(K / 8) * 4;
  const size_t G = size_t(K / kGroup);
  int64_t off = 0;
  for (int i = 0; i < parts; ++i) {
    const int64_t n = Ns[i];
    if (n == 0) continue;
    if (cudaMemcpyAsync(reinterpret_cast<char*>(qweight_out) + size_t(off) * row_bytes, qweights[i],
                        size_t(n) * row_bytes, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return AWQ_ERR_CUDA;
    for (int a = 0; a < (cfg.zero_point ? 2 : 1); ++a) {
      const uint16_t* src = a == 0 ? scales[i] : zeros[i];
      uint16_t* dst = (a == 0 ? scales_out : zeros_out) + off;
      if (cudaMemcpy2DAsync(dst, size_t(total) * 2, src, size_t(n) * 2, size_t(n) * 2, G,
                            cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return AWQ_ERR_CUDA;
    }
    off += n;
  }
  return launch_status();
}
