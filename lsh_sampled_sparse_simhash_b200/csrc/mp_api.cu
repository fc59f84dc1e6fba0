// C ABI of the library (declared in include/magicpig.h): argument validation,
// shape checks and kernel launches.  No allocation, no global state except the
// per-device record of raised shared-memory limits.
#include <stdint.h>

#include <mutex>

#include "magicpig.h"
#include "mp_common.cuh"
#include "mp_kernels.cuh"

namespace mp {

int validate_shape(const mp_shape *in, Shape &s)
{
    if (!in) return MP_ERR_ARG;
    s.B = in->batch;
    s.Hq = in->n_q_heads;
    s.Hkv = in->n_kv_heads;
    s.d = in->head_dim;
    s.Ncap = in->capacity;
    s.K = in->k_bits;
    s.L = in->n_tables;
    s.sink = in->sink;
    s.window = in->window;
    if (in->code_layout == MP_CODES_AUTO)  // bit planes unless a K = 8 problem is small (see the header)
        s.planes = in->k_bits != 8 ||
                   (int64_t)in->batch * in->n_kv_heads * in->capacity >= MP_CODES_AUTO_PLANES_MIN;
    else if (in->code_layout == MP_CODES_BYTES)
        s.planes = 0;
    else if (in->code_layout == MP_CODES_PLANES)
        s.planes = 1;
    else
        return MP_ERR_SHAPE;
    if (s.B < 1 || s.Hq < 1 || s.Hkv < 1 || s.sink < 0 || s.window < 0) return MP_ERR_SHAPE;
    if (s.d != kHeadDim) return MP_ERR_SHAPE;
    if (s.K != 8 && s.K != 10) return MP_ERR_SHAPE;
    if (!s.planes && s.K != 8) return MP_ERR_SHAPE;
    if (s.L < 2 || s.L > 255 || s.L * s.K > 2048) return MP_ERR_SHAPE;
    if (s.Hq % s.Hkv != 0) return MP_ERR_SHAPE;
    s.G = s.Hq / s.Hkv;
    if (s.G != 1 && s.G != 2 && s.G != 4 && s.G != 8) return MP_ERR_SHAPE;
    if (s.Ncap < 128 || s.Ncap % 128 != 0 || s.Ncap >= (1 << 24)) return MP_ERR_SHAPE;
    if ((int64_t)s.B * s.Hkv > 65535) return MP_ERR_SHAPE;
    s.LK = s.L * s.K;
    return MP_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_ptrs(std::initializer_list<const void *> ptrs)
{
    for (const void *p : ptrs) {
        if (!p) return MP_ERR_ARG;
        if (!aligned16(p)) return MP_ERR_ALIGN;
    }
    return MP_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MP_OK : MP_ERR_CUDA; }

static size_t codes_bytes(const Shape &s) { return (size_t)s.B * s.Hkv * s.L * s.K * (size_t)s.Ncap / 8; }

cudaError_t ensure_smem(const void *func, int bytes)
{
    static std::mutex mu;
    static const void *done_func[256];
    static int done_dev[256], done_bytes[256], n_done = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n_done; i++)
        if (done_func[i] == func && done_dev[i] == dev && done_bytes[i] >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && n_done < 256) {
        done_func[n_done] = func;
        done_dev[n_done] = dev;
        done_bytes[n_done] = bytes;
        n_done++;
    }
    return e;
}

}  // namespace mp

using namespace mp;

extern "C" {

int mp_codes_bytes(const mp_shape *shape, size_t *bytes)
{
    Shape s;
    int r = validate_shape(shape, s);
    if (r) return r;
    if (!bytes) return MP_ERR_ARG;
    *bytes = codes_bytes(s);
    return MP_OK;
}

int mp_hash_keys(const mp_shape *shape, const void *keys, const void *W, const int32_t *seq_lens,
                 int32_t n_tokens, void *codes, int32_t *status, void *stream)
{
    Shape s;
    int r = validate_shape(shape, s);
    if (r) return r;
    if ((r = check_ptrs({keys, W, codes}))) return r;
    if (seq_lens && (reinterpret_cast<uintptr_t>(seq_lens) & 3u)) return MP_ERR_ALIGN;
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return MP_ERR_ALIGN;
    if (n_tokens < 0 || n_tokens > s.Ncap) return MP_ERR_CAPACITY;
    return cuda_status(launch_hash_keys_tc(s, static_cast<const uint16_t *>(keys), static_cast<const uint16_t *>(W),
                                           seq_lens, 0, n_tokens, codes, status, static_cast<cudaStream_t>(stream)));
}

int mp_hash_keys_range(const mp_shape *shape, const void *keys, const void *W, int32_t first_token,
                       int32_t n_tokens, void *codes, int32_t *status, void *stream)
{
    Shape s;
    int r = validate_shape(shape, s);
    if (r) return r;
    if ((r = check_ptrs({keys, W, codes}))) return r;
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return MP_ERR_ALIGN;
    if (first_token < 0 || n_tokens < 0 || (int64_t)first_token + n_tokens > s.Ncap) return MP_ERR_CAPACITY;
    if (first_token % 128 != 0) return MP_ERR_ALIGN;
    return cuda_status(launch_hash_keys_tc(s, static_cast<const uint16_t *>(keys), static_cast<const uint16_t *>(W),
                                           nullptr, first_token, n_tokens, codes, status,
                                           static_cast<cudaStream_t>(stream)));
}

int mp_hash_queries(const mp_shape *shape, const void *q, const void *W, uint16_t *qcodes, void *stream)
{
    Shape s;
    int r = validate_shape(shape, s);
    if (r) return r;
    if ((r = check_ptrs({q, W, qcodes}))) return r;
    return cuda_status(launch_hash_queries(s, static_cast<const uint16_t *>(q), static_cast<const uint16_t *>(W),
                                           qcodes, static_cast<cudaStream_t>(stream)));
}

int mp_append_token(const mp_shape *shape, const void *k_new, const void *v_new, const void *W, void *k_cache,
                    void *v_cache, void *codes, int32_t *seq_lens, int32_t *status, void *stream)
{
    Shape s;
    int r = validate_shape(shape, s);
    if (r) return r;
    if ((r = check_ptrs({k_new, v_new, W, k_cache, v_cache, codes, seq_lens}))) return r;
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return MP_ERR_ALIGN;
    return cuda_status(launch_append(s, static_cast<const uint16_t *>(k_new), static_cast<const uint16_t *>(v_new),
                                     static_cast<const uint16_t *>(W), static_cast<uint16_t *>(k_cache),
                                     static_cast<uint16_t *>(v_cache), codes, seq_lens, status, nullptr,
                                     static_cast<cudaStream_t>(stream)));
}

int mp_quantize_keys(const mp_shape *shape, const void *k_cache, const int32_t *seq_lens, int32_t first_token,
                     int32_t n_tokens, int8_t *k8, void *stream)
{
    Shape s;
    int r = validate_shape(shape, s);
    if (r) return r;
    if ((r = check_ptrs({k_cache, k8}))) return r;
    if (seq_lens && (reinterpret_cast<uintptr_t>(seq_lens) & 3u)) return MP_ERR_ALIGN;
    if (first_token < 0 || n_tokens < 0 || (int64_t)first_token + n_tokens > s.Ncap) return MP_ERR_CAPACITY;
    return cuda_status(launch_quantize_keys(s, static_cast<const uint16_t *>(k_cache), seq_lens, first_token,
                                            n_tokens, k8, static_cast<cudaStream_t>(stream)));
}

int mp_append_token_q8(const mp_shape *shape, const void *k_new, const void *v_new, const void *W, void *k_cache,
                       void *v_cache, void *codes, int32_t *seq_lens, int8_t *k8, int32_t *status,
                       void *stream)
{
    Shape s;
    int r = validate_shape(shape, s);
    if (r) return r;
    if ((r = check_ptrs({k_new, v_new, W, v_cache, codes, seq_lens, k8}))) return r;
    if (k_cache && !aligned16(k_cache)) return MP_ERR_ALIGN;  // null: the int8 copy is the only key cache
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return MP_ERR_ALIGN;
    return cuda_status(launch_append(s, static_cast<const uint16_t *>(k_new), static_cast<const uint16_t *>(v_new),
                                     static_cast<const uint16_t *>(W), static_cast<uint16_t *>(k_cache),
                                     static_cast<uint16_t *>(v_cache), codes, seq_lens, status, k8,
                                     static_cast<cudaStream_t>(stream)));
}

int mp_decode_workspace_bytes(const mp_shape *shape, int32_t max_len, size_t *bytes)
{
    Shape s;
    int r = validate_shape(shape, s);
    if (r) return r;
    if (!bytes) return MP_ERR_ARG;
    if (max_len < 0 || max_len > s.Ncap) return MP_ERR_CAPACITY;
    *bytes = decode_workspace_bytes(s, max_len);
    return MP_OK;
}

int mp_decode_attend(const mp_shape *shape, const void *q, const void *W, const void *codes, const void *k_cache,
                     const void *v_cache, const int32_t *seq_lens, int32_t max_len, float *out, float *lse,
                     int32_t *n_sampled, void *workspace, size_t workspace_bytes, const mp_decode_debug *debug,
                     void *stream)
{
    Shape s;
    int r = validate_shape(shape, s);
    if (r) return r;
    if ((r = check_ptrs({q, W, codes, k_cache, v_cache, seq_lens, out, lse, n_sampled, workspace}))) return r;
    if (max_len < 0 || max_len > s.Ncap) return MP_ERR_CAPACITY;
    if (workspace_bytes < decode_workspace_bytes(s, max_len)) return MP_ERR_WORKSPACE;
    if (debug) {
        if ((debug->qcodes_in && !aligned16(debug->qcodes_in)) || (debug->qcodes_out && !aligned16(debug->qcodes_out)))
            return MP_ERR_ALIGN;
        if (debug->path < MP_PATH_AUTO || debug->path > MP_PATH_TC) return MP_ERR_ARG;
        if (debug->path == MP_PATH_FUSED && (!s.planes || s.G > 4)) return MP_ERR_SHAPE;
        if (debug->skip_scan && debug->path != MP_PATH_AUTO && debug->path != MP_PATH_SPLIT) return MP_ERR_ARG;
    }
    return cuda_status(launch_decode(s, static_cast<const uint16_t *>(q), static_cast<const uint16_t *>(W), codes,
                                     static_cast<const uint16_t *>(k_cache), static_cast<const uint16_t *>(v_cache),
                                     seq_lens, max_len, out, lse, n_sampled, workspace, debug,
                                     static_cast<cudaStream_t>(stream)));
}

int mp_decode_attend_q8(const mp_shape *shape, const void *q, const void *W, const void *codes, const int8_t *k8,
                        const void *v_cache, const int32_t *seq_lens, int32_t max_len,
                        float *out, float *lse, int32_t *n_sampled, void *workspace, size_t workspace_bytes,
                        const mp_decode_debug *debug, void *stream)
{
    Shape s;
    int r = validate_shape(shape, s);
    if (r) return r;
    if ((r = check_ptrs({q, W, codes, k8, v_cache, seq_lens, out, lse, n_sampled, workspace}))) return r;
    if (max_len < 0 || max_len > s.Ncap) return MP_ERR_CAPACITY;
    if (workspace_bytes < decode_workspace_bytes(s, max_len)) return MP_ERR_WORKSPACE;
    if (debug) {
        if ((debug->qcodes_in && !aligned16(debug->qcodes_in)) || (debug->qcodes_out && !aligned16(debug->qcodes_out)))
            return MP_ERR_ALIGN;
        if (debug->path < MP_PATH_AUTO || debug->path > MP_PATH_TC) return MP_ERR_ARG;
        if (debug->path == MP_PATH_FUSED || debug->path == MP_PATH_TC) return MP_ERR_SHAPE;
    }
    return cuda_status(launch_decode(s, static_cast<const uint16_t *>(q), static_cast<const uint16_t *>(W), codes,
                                     nullptr, static_cast<const uint16_t *>(v_cache), seq_lens, max_len, out, lse,
                                     n_sampled, workspace, debug, static_cast<cudaStream_t>(stream), k8));
}

int mp_read_status(const void *workspace, int32_t *status, void *stream)
{
    if (!workspace || !status) return MP_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return MP_ERR_CUDA;
    if (cudaMemcpy(status, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess) return MP_ERR_CUDA;
    return MP_OK;
}

const char *mp_status_string(int code)
{
    switch (code) {
    case MP_OK: return "MP_OK";
    case MP_ERR_ARG: return "MP_ERR_ARG: null pointer or invalid argument";
    case MP_ERR_SHAPE: return "MP_ERR_SHAPE: unsupported shape";
    case MP_ERR_ALIGN: return "MP_ERR_ALIGN: pointer not 16-byte aligned";
    case MP_ERR_CAPACITY: return "MP_ERR_CAPACITY: length exceeds capacity or max_len";
    case MP_ERR_WORKSPACE: return "MP_ERR_WORKSPACE: workspace too small";
    case MP_ERR_CUDA: return "MP_ERR_CUDA: CUDA runtime error";
    case MP_ERR_TOO_LARGE: return "MP_ERR_TOO_LARGE: problem needs more scratch than the fixed array of mp_decode_attend_noalloc";
    default: return "MP_ERR_UNKNOWN";
    }
}

}  // extern "C"
