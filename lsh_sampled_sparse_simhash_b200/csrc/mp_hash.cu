// Decode-time append: one new token per sequence (MagicPIG, Chen et al. 2024;
// the gitdiagram page's "LSH Sampling" component: LSH kernel behind an LSH
// interface).  The bulk key hash is the tensor-core kernel in mp_hash_tc.cu.
//
// Code layouts (table-major, exactly L*K/8 bytes per token):
//   bytes : uint8  [unit][L][Ncap], bit b of the byte = bit b of the code.
//   planes: uint32 [unit][L][Ncap/32][K], bit t of word (w, b) = bit b of the
//           code of token 32 w + t.
#include "mp_common.cuh"
#include "mp_kernels.cuh"
#include "mp_kquant.cuh"

namespace mp {

constexpr int kAppendCluster = 8;  // blocks per sequence (one thread-block cluster)
constexpr int kAppendThreads = 1024;

// --------------------------------------------------------------- append ----
// grid (kAppendCluster, B): one cluster of kAppendCluster blocks per sequence.
// Block r takes tables [r T, r T + T) (T = ceil(L / kAppendCluster)) of all
// Hkv kv heads of the sequence: its (column, head) pairs, head-minor, are
// dealt to groups of four lanes (the heads of one column sit in neighbouring
// lane groups and share the W row through L1); each lane sums 32 exact bf16
// products in fp32, and two shuffles add the quarters (bits can differ from the
// tensor-core hash only where the projection is within fp32 rounding of
// zero).  Every block reads the position seq_lens[b] first and then arrives
// on the cluster barrier; block 0 waits on it before writing seq_lens[b] + 1,
// so the length moves only after every block of the sequence has read it.
__global__ void __launch_bounds__(kAppendThreads) append_kernel(Shape s, const uint16_t *__restrict__ k_new,
                                                                const uint16_t *__restrict__ v_new,
                                                                const uint16_t *__restrict__ W, uint16_t *kc,
                                                                uint16_t *vc, void *codes, int32_t *seq_lens,
                                                                int32_t *status, int8_t *k8)
{
    // shared: this block's W rows [T K][kHeadDim] bf16, the new keys
    // [Hkv][kHeadDim + 4] fp32 (element d at d + d / 32), the bits [Hkv][T K]
    extern __shared__ __align__(16) uint8_t sm_raw[];
    const int tid = threadIdx.x;
    const int r = blockIdx.x, b = blockIdx.y;
    const int T = (s.L + kAppendCluster - 1) / kAppendCluster;
    const int l0 = min(s.L, r * T), l1 = min(s.L, l0 + T);
    const int c_begin = l0 * s.K, ncol = (l1 - l0) * s.K;
    uint16_t *wsm = reinterpret_cast<uint16_t *>(sm_raw);
    float *xs = reinterpret_cast<float *>(sm_raw + (size_t)T * s.K * kHeadDim * 2);
    uint8_t *bits = reinterpret_cast<uint8_t *>(xs + s.Hkv * (kHeadDim + 4));
    // the block's W rows into shared memory first: no kernel writes W, so the
    // copies go out before the wait for the predecessor
    for (int i = tid; i < ncol * (kHeadDim / 8); i += blockDim.x)
        cp_async_16(wsm + (size_t)i * 8, W + (size_t)c_begin * kHeadDim + (size_t)i * 8, 16);
    cp_async_commit();
    grid_dependency_wait();
    const int pos = seq_lens[b];
    asm volatile("barrier.cluster.arrive.aligned;" ::: "memory");  // (release) this block has read pos
    const bool ok = pos >= 0 && pos < s.Ncap;
    if (!ok) {
        if (r == 0 && tid == 0) set_status(status, MP_ERR_CAPACITY);
    } else {
        const size_t unit0 = (size_t)b * s.Hkv;
        if (r == 0) {  // the K and V rows, 16 bytes per thread (no K row without a bf16 key cache)
            for (int i = tid; i < s.Hkv * 32; i += blockDim.x) {
                const int h = i >> 5, isv = (i >> 4) & 1, e = i & 15;
                if (!isv && !kc) continue;
                const uint4 *src = reinterpret_cast<const uint4 *>((isv ? v_new : k_new) + (unit0 + h) * kHeadDim);
                uint4 *dst = reinterpret_cast<uint4 *>((isv ? vc : kc) + ((unit0 + h) * s.Ncap + pos) * kHeadDim);
                dst[e] = src[e];
            }
        } else if (r == 1 && k8) {  // the int8 copy of the new keys, a warp per kv head
            for (int h = tid >> 5; h < s.Hkv; h += blockDim.x >> 5) {
                const size_t row = (unit0 + h) * s.Ncap + pos;
                quantize_key_row(k_new + (unit0 + h) * kHeadDim, k8 + row * kQ8RowBytes, tid & 31);
            }
        }
        for (int i = tid; i < s.Hkv * kHeadDim; i += blockDim.x) {
            const int h = i / kHeadDim, d = i % kHeadDim;
            xs[h * (kHeadDim + 4) + d + (d >> 5)] = bf16_to_f32(k_new[(unit0 + h) * kHeadDim + d]);
        }
        cp_async_wait<0>();
        __syncthreads();
        const int part = tid & 3;  // quarter of the dims
        constexpr int kSlots = kAppendThreads / 4;
        const int npairs = ncol * s.Hkv;
        // this lane's quarter of its head's key, in registers: the slot
        // stride is a multiple of Hkv whenever Hkv divides kSlots, and then
        // the head of a lane never changes between its pairs
        float kx[32];
        int hcur = -1;
        for (int pi = tid >> 2; pi < (npairs + kSlots - 1) / kSlots * kSlots; pi += kSlots) {
            const bool valid = pi < npairs;
            const int cl = valid ? pi / s.Hkv : 0, h = valid ? pi - cl * s.Hkv : 0;
            if (valid && h != hcur) {
                const float *xp = xs + h * (kHeadDim + 4) + part * 33;
#pragma unroll
                for (int i = 0; i < 32; i++) kx[i] = xp[i];
                hcur = h;
            }
            float dot = 0.f;
            if (valid) {
                const uint4 *wr = reinterpret_cast<const uint4 *>(wsm + (size_t)cl * kHeadDim + part * 32);
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    const uint4 w = wr[j];
                    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        dot = fmaf(kx[j * 8 + 2 * e], bf16_lo(wv[e]), dot);
                        dot = fmaf(kx[j * 8 + 2 * e + 1], bf16_hi(wv[e]), dot);
                    }
                }
            }
            dot += __shfl_xor_sync(0xffffffffu, dot, 1);
            dot += __shfl_xor_sync(0xffffffffu, dot, 2);
            if (valid && part == 0) bits[h * T * s.K + cl] = dot > 0.f;
        }
        __syncthreads();
        if (!s.planes) {
            for (int i = tid; i < s.Hkv * (l1 - l0); i += blockDim.x) {
                const int h = i / (l1 - l0), lt = i % (l1 - l0);
                unsigned code = 0;
                for (int bb = 0; bb < 8; bb++) code |= (unsigned)bits[h * T * s.K + lt * 8 + bb] << bb;
                static_cast<uint8_t *>(codes)[((unit0 + h) * s.L + l0 + lt) * s.Ncap + pos] = (uint8_t)code;
            }
        } else {
            const unsigned int m = 1u << (pos & 31);
            for (int i = tid; i < s.Hkv * ncol; i += blockDim.x) {
                const int h = i / ncol, cl = i % ncol;
                const int c = c_begin + cl, l = c / s.K, bb = c - l * s.K;
                unsigned int *word = static_cast<unsigned int *>(codes) +
                                     (((unit0 + h) * s.L + l) * (s.Ncap >> 5) + (pos >> 5)) * s.K + bb;
                if (bits[h * T * s.K + cl])
                    atomicOr(word, m);
                else
                    atomicAnd(word, ~m);
            }
        }
    }
    cp_async_wait<0>();  // (the error path leaves no copy in flight either)
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");  // (acquire) every block has read pos
    if (ok && r == 0 && tid == 0) seq_lens[b] = pos + 1;
}

cudaError_t launch_append(const Shape &s, const uint16_t *k_new, const uint16_t *v_new, const uint16_t *W,
                          uint16_t *kc, uint16_t *vc, void *codes, int32_t *seq_lens, int32_t *status,
                          int8_t *k8, cudaStream_t st)
{
    const int T = (s.L + kAppendCluster - 1) / kAppendCluster;
    const size_t smem = (size_t)T * s.K * kHeadDim * 2 + (size_t)s.Hkv * (kHeadDim + 4) * sizeof(float) +
                        (size_t)s.Hkv * T * s.K;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(append_kernel), (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kAppendCluster, s.B);
    cfg.blockDim = dim3(kAppendThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kAppendCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, append_kernel, s, k_new, v_new, W, kc, vc, codes, seq_lens, status, k8);
}

}  // namespace mp
