// Library-wide entry points of libdfsattn: status text, device error word,
// version.
#include "common.cuh"

extern "C" const char* dfs_status_string(int status) {
  switch (status) {
    case DFS_OK: return "ok";
    case DFS_ERR_INVALID_ARG: return "invalid argument";
    case DFS_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case DFS_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case DFS_ERR_CUDA: return "CUDA launch or runtime error";
    case DFS_ERR_TIMEOUT: return "device wait timed out";
    case DFS_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

extern "C" int dfs_get_error_flags(uint32_t* flags, int clear) {
  if (!flags) return DFS_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return DFS_ERR_CUDA;
  uint32_t v = 0;
  int st;
  if ((st = dfs_detail_flags_perm(&v, clear)) != DFS_OK) return st;
  if ((st = dfs_detail_flags_score(&v, clear)) != DFS_OK) return st;
  if ((st = dfs_detail_flags_select(&v, clear)) != DFS_OK) return st;
  if ((st = dfs_detail_flags_attn(&v, clear)) != DFS_OK) return st;
  if ((st = dfs_detail_flags_bwd(&v, clear)) != DFS_OK) return st;
  *flags = v;
  return DFS_OK;
}

extern "C" int dfs_version(void) { return 100; }
