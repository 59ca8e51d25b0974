// C ABI entry points that are not tied to one kernel: version, status text,
// workspace sizing.

#include "awq_common.cuh"

namespace awq {
awq_status_t gemv_workspace_bytes(int64_t M, int64_t N, int64_t K, int zp, bool silu, size_t* bytes);
awq_status_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, bool zp, size_t* bytes);
}  // namespace awq

extern "C" int awq_abi_version(void) { return AWQ_ABI_VERSION; }

extern "C" const char* awq_status_string(awq_status_t status) {
  switch (status) {
    case AWQ_OK: return "ok";
    case AWQ_ERR_NULL: return "a required pointer is NULL";
    case AWQ_ERR_SHAPE: return "a size is out of range or inconsistent";
    case AWQ_ERR_ALIGN: return "a device pointer is not 16-byte aligned";
    case AWQ_ERR_UNSUPPORTED:
      return "configuration not supported (group size other than 128, zero_point not 0 or 1, an undefined "
             "flag, or a flag this entry point does not take)";
    case AWQ_ERR_CUDA: return "the CUDA runtime reported an error";
    case AWQ_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

extern "C" awq_status_t awq_workspace_bytes(int64_t M, int64_t N, int64_t K, awq_qconfig_t cfg,
                                            size_t* bytes) {
  using namespace awq;
  if (!bytes) return AWQ_ERR_NULL;
  awq_status_t st = check_cfg(cfg, true);
  if (st != AWQ_OK) return st;
  if ((st = check_nk(N, K)) != AWQ_OK) return st;
  if (M < 0) return AWQ_ERR_SHAPE;
  *bytes = 0;
  if (M == 0 || N == 0) return AWQ_OK;
  if ((cfg.flags & AWQ_FLAG_SILU_MUL) && N % 32) return AWQ_ERR_SHAPE;
  if ((cfg.flags & AWQ_FLAG_PACKED_ZEROS) && N % 32) return AWQ_ERR_SHAPE;
  if (M <= 16) return gemv_workspace_bytes(M, N, K, zero_mode(cfg), (cfg.flags & AWQ_FLAG_SILU_MUL) != 0, bytes);
  if ((st = gemm_workspace_bytes(M, N, K, cfg.zero_point != 0, bytes)) != AWQ_OK) return st;
  // the GEMM reads packed zero points through an fp16 copy in the workspace
  if (cfg.flags & AWQ_FLAG_PACKED_ZEROS) *bytes += size_t(K / kGroup) * size_t(N) * 2;
  return AWQ_OK;
}
