// W4A16 prefill product y[M][N] = x[M][K] . W'^T on the sm_100a tensor cores.
//
// ("AutoAWQ" code tour, "The big picture": WQLinear_GEMM serves batched
// requests; "AutoAWQ" capability page: the weights stay INT4 in memory and
// are decoded inside the fused matmul.)
//
// For M beyond a few tens the layer is a dense contraction, so W' tiles are
// decoded into shared memory and multiplied by tcgen05.mma with fp32
// accumulators in tensor memory. One persistent CTA per SM walks output tiles
// of 256 (rows of x) x 256 (output channels); K advances in blocks of 64.
// Each decoded 256 x 64 weight block feeds two M = 128, N = 256 MMAs (the two
// halves of the 256 rows of x). A tcgen05.mma costs about the same issue
// time whatever its N, so the widest N (256) gives the most work per
// instruction.
//
// Warp roles (704 threads):
//   warps 0-15  decode: threads 2r and 2r+1 own row r of the 256-row weight
//               tile, 32 k each; a thread reads its 16 code bytes of the k
//               block from shared memory, decodes w' = (q - z) * s exactly as
//               awq_dequant does (HSUB2 gives q - z exactly, HMUL2 rounds the
//               product once), and writes 64 bytes in the 128-byte-swizzled
//               K-major layout the tensor core reads.
//   warps 16-19 epilogue: tcgen05.ld of the fp32 accumulators (lane = row of
//               x), fp16 conversion, stores to y.
//   warp 20     TMA: x tile (256 x 64 fp16, 128B swizzle) and code tile
//               (256 rows x 32 bytes, 32B swizzle) per k block.
//   warp 21     MMA: one thread issues 2 x 4 tcgen05.mma (M=128, N=256,
//               K=16) per k block (the upper half is skipped when it holds
//               no rows of x), commits stage release and accumulator-ready
//               barriers. Warp 21 also allocates and frees tensor memory.
// Pipelines: 3 shared-memory stages (x + codes in, decoded W' out) and one
// accumulator pair (all 512 TMEM columns): the epilogue of a tile runs
// before the next tile's first MMA.
//
// Every mbarrier wait is bounded by a wall-clock limit. When a wait runs
// out, the CTA records bit 0 in the device error word, every role leaves its
// loop, in-flight copies and MMAs are waited for (again bounded), and tensor
// memory is freed before the kernel returns.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>

#include "awq_common.cuh"
#include "awq_tma_host.h"

namespace awq {

__device__ uint32_t g_awq_error_word = 0;

}  // namespace awq

// The kernel body twice: 256-channel tiles (two N = 256 MMAs per k step for
// large batches) and 128-channel tiles (twice the tiles for small batches,
// where 256-channel tiles leave SMs idle or need the cross-CTA K split).
namespace awq {
namespace gemm256 {
#define AWQ_GEMM_BN 256
#include "awq_gemm_body.cuh"
#undef AWQ_GEMM_BN
}  // namespace gemm256
namespace gemm128 {
#define AWQ_GEMM_BN 128
#include "awq_gemm_body.cuh"
#undef AWQ_GEMM_BN
}  // namespace gemm128
namespace gemm128s {   // 128-channel tiles and 128-row x tiles, for M <= 128
#define AWQ_GEMM_BN 128
#define AWQ_GEMM_BM 128
#include "awq_gemm_body.cuh"
#undef AWQ_GEMM_BM
#undef AWQ_GEMM_BN
}  // namespace gemm128s

awq_status_t gemv_take_error(uint32_t* word, cudaStream_t s);
awq_status_t chain_take_error(uint32_t* word, cudaStream_t s);

awq_status_t gemm_workspace_bytes(int64_t, int64_t, int64_t, bool, size_t* bytes) {
  *bytes = 0;
  return AWQ_OK;
}

}  // namespace awq

using namespace awq;

extern "C" awq_status_t awq_gemm(const uint16_t* x, const int32_t* qweight,
                                 const uint16_t* scales, const uint16_t* zeros, int64_t M,
                                 int64_t N, int64_t K, awq_qconfig_t cfg, uint16_t* y,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  awq_status_t st = check_cfg(cfg, true);
  if (st != AWQ_OK) return st;
  if ((st = check_nk(N, K)) != AWQ_OK) return st;
  if (M < 0 || M > (int64_t(1) << 31) - 1) return AWQ_ERR_SHAPE;
  if ((cfg.flags & AWQ_FLAG_SILU_MUL) && N % 32) return AWQ_ERR_SHAPE;
  const bool packed = (cfg.flags & AWQ_FLAG_PACKED_ZEROS) != 0;
  if (packed && N % 32) return AWQ_ERR_SHAPE;
  if (M == 0 || N == 0) return AWQ_OK;
  if (!x || !qweight || !scales || !y) return AWQ_ERR_NULL;
  if (cfg.zero_point && !zeros) return AWQ_ERR_NULL;
  if (!cfg.zero_point && zeros) return AWQ_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(qweight) || !aligned16(scales) || !aligned16(y) ||
      (zeros && !aligned16(zeros)))
    return AWQ_ERR_ALIGN;
  if (packed) {
    // Packed zero points: unpacked into the workspace (fp16 [K/128][N], the
    // values the fp16 form holds), then the same product as with that form.
    const int64_t G = K / kGroup;
    const size_t need = size_t(G) * size_t(N) * 2;
    if (!workspace || workspace_bytes < need) return AWQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return AWQ_ERR_ALIGN;
    uint16_t* z16 = static_cast<uint16_t*>(workspace);
    if ((st = awq_unpack_zeros(reinterpret_cast<const int32_t*>(zeros), G, N, z16, stream)) != AWQ_OK) return st;
    zeros = z16;
    cfg.flags &= ~AWQ_FLAG_PACKED_ZEROS;
  }

  // The tile shape with the lowest estimated time (ties: the wider tiles).
  // Beyond 256 rows of x the 256-channel tiles always win (measured).
  if (M > 256) return gemm256::run(x, qweight, scales, zeros, M, N, K, cfg, y, stream, false, nullptr);
  int64_t c256 = 0, c128 = 0, c128s = INT64_MAX;
  if ((st = gemm256::run(x, qweight, scales, zeros, M, N, K, cfg, y, stream, true, &c256)) != AWQ_OK) return st;
  if ((st = gemm128::run(x, qweight, scales, zeros, M, N, K, cfg, y, stream, true, &c128)) != AWQ_OK) return st;
  if (M <= 128 && (st = gemm128s::run(x, qweight, scales, zeros, M, N, K, cfg, y, stream, true, &c128s)) != AWQ_OK)
    return st;
  if (c128s <= c128 && c128s < c256)   // 128-row x tiles: same k blocks, half the bytes per stage
    return gemm128s::run(x, qweight, scales, zeros, M, N, K, cfg, y, stream, false, nullptr);
  if (c128 < c256) return gemm128::run(x, qweight, scales, zeros, M, N, K, cfg, y, stream, false, nullptr);
  return gemm256::run(x, qweight, scales, zeros, M, N, K, cfg, y, stream, false, nullptr);
}

extern "C" awq_status_t awq_device_error(uint32_t* error_word, void* stream) {
  if (!error_word) return AWQ_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t gemm_word = 0, gemv_word = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&gemm_word, g_awq_error_word, sizeof(uint32_t), 0,
                                cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return AWQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return AWQ_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(g_awq_error_word, &zero, sizeof(uint32_t), 0, cudaMemcpyHostToDevice,
                              s) != cudaSuccess)
    return AWQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return AWQ_ERR_CUDA;
  awq_status_t st = gemv_take_error(&gemv_word, s);
  if (st != AWQ_OK) return st;
  uint32_t chain_word = 0;
  if ((st = chain_take_error(&chain_word, s)) != AWQ_OK) return st;
  *error_word = gemm_word | gemv_word | chain_word;
  return AWQ_OK;
}
