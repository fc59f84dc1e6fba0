// Host-side launchers of the library's kernels (called from mp_api.cu after
// argument validation).  All launch asynchronously on `st`.
#pragma once

#include "mp_common.cuh"

namespace mp {

cudaError_t launch_hash_keys(const Shape &s, const uint16_t *keys, const uint16_t *W, const int32_t *seq_lens,
                             int n_tokens, void *codes, cudaStream_t st);
cudaError_t launch_hash_queries(const Shape &s, const uint16_t *q, const uint16_t *W, uint16_t *qcodes,
                                cudaStream_t st);
cudaError_t launch_append(const Shape &s, const uint16_t *k_new, const uint16_t *v_new, const uint16_t *W,
                          uint16_t *kc, uint16_t *vc, void *codes, int32_t *seq_lens, int32_t *status,
                          cudaStream_t st);
cudaError_t launch_decode(const Shape &s, const uint16_t *q, const uint16_t *W, const void *codes,
                          const uint16_t *kc, const uint16_t *vc, const int32_t *seq_lens, int max_len,
                          float *out, float *lse, int32_t *n_sampled, void *workspace,
                          const mp_decode_debug *dbg, cudaStream_t st);
size_t decode_workspace_bytes(const Shape &s, int max_len);

// Raises the dynamic shared-memory limit of `func` on the current device once.
cudaError_t ensure_smem(const void *func, int bytes);

}  // namespace mp
