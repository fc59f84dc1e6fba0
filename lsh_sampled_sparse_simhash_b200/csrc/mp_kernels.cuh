// Host-side launchers of the library's kernels (called from mp_api.cu after
// argument validation).  All launch asynchronously on `st`.
#pragma once

#include <cuda.h>

#include <initializer_list>

#include "mp_common.cuh"
#include "mp_logu.cuh"

namespace mp {

// Host-side argument checks shared by the C entry points (mp_api.cu).
int validate_shape(const mp_shape *in, Shape &s);
bool aligned16(const void *p);
int check_ptrs(std::initializer_list<const void *> ptrs);
int cuda_status(cudaError_t e);

// Hashes tokens [tok0, tok0 + n_tokens) of every unit (tok0 a multiple of 128;
// with seq_lens, unit (b, .) stops at seq_lens[b]).
cudaError_t launch_hash_keys_tc(const Shape &s, const uint16_t *keys, const uint16_t *W, const int32_t *seq_lens,
                                int tok0, int n_tokens, void *codes, int32_t *status, cudaStream_t st);
cudaError_t launch_hash_queries(const Shape &s, const uint16_t *q, const uint16_t *W, uint16_t *qcodes,
                                cudaStream_t st);
// k8 (nullable): also write the int8 rows of the new keys (mp_kquant.cuh).
cudaError_t launch_append(const Shape &s, const uint16_t *k_new, const uint16_t *v_new, const uint16_t *W,
                          uint16_t *kc, uint16_t *vc, void *codes, int32_t *seq_lens, int32_t *status,
                          int8_t *k8, cudaStream_t st);
// With k8 (non-null) the attention gathers the int8 key rows (values and
// {scale, squared norm} record) instead of kc (the two-kernel path only).
cudaError_t launch_decode(const Shape &s, const uint16_t *q, const uint16_t *W, const void *codes,
                          const uint16_t *kc, const uint16_t *vc, const int32_t *seq_lens, int max_len,
                          float *out, float *lse, int32_t *n_sampled, void *workspace,
                          const mp_decode_debug *dbg, cudaStream_t st, const int8_t *k8 = nullptr);
// int8 copy of the keys of tokens [tok0, tok0 + n_tokens) of every unit (with
// seq_lens, unit (b, .) stops at seq_lens[b]).
cudaError_t launch_quantize_keys(const Shape &s, const uint16_t *kc, const int32_t *seq_lens, int tok0, int n_tokens,
                                 int8_t *k8, cudaStream_t st);
size_t decode_workspace_bytes(const Shape &s, int max_len);

// Sampled attention on the tensor cores (mp_attend_tc.cu): every work item of
// the split plan (units x nsplit; split nsplit - 1 of a unit is its exact set
// D) leaves one (m, l, acc) partial per query head in pm / pl / pacc
// [B*Hq][nsplit] (acc: [..][128]); m and l are in log2 units.  work_counter
// must be 0 when the kernel starts (the query hash clears it).
struct AttendTcArgs {
    Shape s;
    const uint16_t *q, *kc, *vc;
    const int32_t *seq_lens;
    int max_len, nchunk, span, subs, nsplit, chunk_tokens;
    const uint32_t *cand;  // [B*Hkv][nchunk][chunk_tokens] token | headmask << 24
    const int32_t *cnt;    // [B*Hkv][nchunk][16], [0] = candidates of the chunk
    int32_t *work_counter;
    int32_t *status;
    float *pm, *pl, *pacc;
    LogU lu;
    float scale;  // 1 / sqrt(d)
};
cudaError_t launch_attend_tc(const AttendTcArgs &a, cudaStream_t st);
size_t attend_tc_smem_bytes();

// A tiled TMA descriptor for a rank-`rank` tensor (dims and box innermost
// first, byte strides of dims 1..rank-1), no interleave, zero fill out of
// bounds.  False if the driver rejects it.
bool encode_tensor_map(CUtensorMap *m, CUtensorMapDataType type, int rank, const void *ptr, const uint64_t *dims,
                       const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle swizzle);

// Raises the dynamic shared-memory limit of `func` on the current device once.
cudaError_t ensure_smem(const void *func, int bytes);

// Launches with programmatic stream serialization: the kernel may be
// scheduled while its predecessor in the stream is still running.  Every
// kernel of this library waits for its predecessor (griddepcontrol.wait)
// before it reads anything the predecessor writes and before it writes global
// memory, and lets its own successor launch only after that wait, so ordering
// is unchanged and only launch latency is hidden (see grid_wait()).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace mp
