// Decode entry point that needs no caller-provided workspace.
//
// mp_decode_attend takes a device workspace that the caller allocates.  Some
// callers cannot allocate device memory at the point where they decode:
// runtimes whose memory pools are sealed after start-up, and plugins that only
// ever receive tensors from a host framework and may not call cudaMalloc
// themselves.  mp_decode_attend_noalloc serves them: its scratch space is a
// fixed, file-scope device array compiled into the library.
//
// The array is kNoAllocScratchBytes (16 MiB) on every GPU that loads the
// library, for the life of the process.  Host code cannot use the array's name
// as a device address, so the first call on each device (with that device
// current) looks the address up with cudaGetSymbolAddress and caches it; make
// that first call before any stream capture begins.  The cached address is
// that of the device's current context: after cudaDeviceReset it is stale and
// the library has to be reloaded before this entry point is used again on
// that device.  All calls share the one
// array: calls whose executions overlap on the GPU (two streams, or two host
// threads on the same device) race on it and must be serialised by the caller.
// Nothing in the array has to start at zero: the first kernel of every call
// resets the status word and every other region is written before it is read.
#include <stdint.h>

#include <mutex>

#include "magicpig.h"
#include "mp_common.cuh"
#include "mp_kernels.cuh"

namespace mp {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device (looked up once).
static cudaError_t scratch_address(void **out)
{
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace mp

extern "C" int mp_decode_attend_noalloc(const mp_shape *shape, const void *q, const void *W, const void *codes,
                                        const void *k_cache, const void *v_cache, const int32_t *seq_lens,
                                        int32_t max_len, float *out, float *lse, int32_t *n_sampled,
                                        int32_t *status, void *stream)
{
    using namespace mp;
    Shape s;
    int r = validate_shape(shape, s);
    if (r) return r;
    if ((r = check_ptrs({q, W, codes, k_cache, v_cache, seq_lens, out, lse, n_sampled}))) return r;
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return MP_ERR_ALIGN;
    if (max_len < 0 || max_len > s.Ncap) return MP_ERR_CAPACITY;
    if (decode_workspace_bytes(s, max_len) > kNoAllocScratchBytes) return MP_ERR_TOO_LARGE;
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return MP_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_decode(s, static_cast<const uint16_t *>(q), static_cast<const uint16_t *>(W), codes,
                                  static_cast<const uint16_t *>(k_cache), static_cast<const uint16_t *>(v_cache),
                                  seq_lens, max_len, out, lse, n_sampled, scratch, nullptr, st);
    if (e == cudaSuccess && status) e = cudaMemcpyAsync(status, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, st);
    return cuda_status(e);
}
