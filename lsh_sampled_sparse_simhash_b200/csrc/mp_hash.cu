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

namespace mp {

constexpr int kAppendCols = 64;  // hyperplane columns per append block (4 lanes each)

// --------------------------------------------------------------- append ----
// grid (ceil(L / TB), B * Hkv), 256 threads: 4 lanes per hyperplane column
// of a block of TB = 64 / K whole tables; each lane sums 32 exact bf16
// products in fp32 and two shuffles add the quarters (bits can differ from
// the tensor-core hash only where the projection is within fp32 rounding of
// zero).
__global__ void __launch_bounds__(256) append_kernel(Shape s, const uint16_t *__restrict__ k_new,
                                                     const uint16_t *__restrict__ v_new,
                                                     const uint16_t *__restrict__ W, uint16_t *kc, uint16_t *vc,
                                                     void *codes, const int32_t *__restrict__ seq_lens,
                                                     int32_t *status)
{
    __shared__ float xs[kHeadDim];
    __shared__ uint8_t bits[kAppendCols];
    const int tid = threadIdx.x;
    const int unit = blockIdx.y;
    const int b = unit / s.Hkv;
    grid_dependency_wait();
    const int pos = seq_lens[b];
    if (pos < 0 || pos >= s.Ncap) {
        if (blockIdx.x == 0 && unit % s.Hkv == 0 && tid == 0) set_status(status, MP_ERR_CAPACITY);
        return;
    }
    const uint16_t *kn = k_new + (size_t)unit * kHeadDim;
    if (blockIdx.x == 0 && tid < 32) {
        const bool isv = tid >= 16;
        const uint4 *src = reinterpret_cast<const uint4 *>((isv ? v_new : k_new) + (size_t)unit * kHeadDim);
        uint4 *dst = reinterpret_cast<uint4 *>((isv ? vc : kc) + ((size_t)unit * s.Ncap + pos) * kHeadDim);
        dst[tid & 15] = src[tid & 15];
    }
    if (tid < kHeadDim) xs[tid] = bf16_to_f32(kn[tid]);
    __syncthreads();
    const int TB = kAppendCols / s.K;
    const int l0 = blockIdx.x * TB;
    const int col = tid >> 2, part = tid & 3;  // column of the block, quarter of the dims
    const int c = l0 * s.K + col;
    const bool valid = col < TB * s.K && c < s.LK;
    float dot = 0.f;
    if (valid) {
        const uint4 *wr = reinterpret_cast<const uint4 *>(W + (size_t)c * kHeadDim + part * 32);
        const float *xp = xs + part * 32;
#pragma unroll
        for (int j8 = 0; j8 < 4; j8++) {
            const uint4 w = __ldg(wr + j8);
            dot = fmaf(xp[j8 * 8 + 0], bf16_lo(w.x), dot);
            dot = fmaf(xp[j8 * 8 + 1], bf16_hi(w.x), dot);
            dot = fmaf(xp[j8 * 8 + 2], bf16_lo(w.y), dot);
            dot = fmaf(xp[j8 * 8 + 3], bf16_hi(w.y), dot);
            dot = fmaf(xp[j8 * 8 + 4], bf16_lo(w.z), dot);
            dot = fmaf(xp[j8 * 8 + 5], bf16_hi(w.z), dot);
            dot = fmaf(xp[j8 * 8 + 6], bf16_lo(w.w), dot);
            dot = fmaf(xp[j8 * 8 + 7], bf16_hi(w.w), dot);
        }
    }
    dot += __shfl_xor_sync(0xffffffffu, dot, 1);
    dot += __shfl_xor_sync(0xffffffffu, dot, 2);
    const bool bit = valid && dot > 0.f;
    if (!s.planes) {
        if (part == 0) bits[col] = bit;
        __syncthreads();
        if (tid < TB && l0 + tid < s.L) {
            unsigned code = 0;
            for (int bb = 0; bb < 8; bb++) code |= (unsigned)bits[tid * 8 + bb] << bb;
            static_cast<uint8_t *>(codes)[((size_t)unit * s.L + l0 + tid) * s.Ncap + pos] = (uint8_t)code;
        }
    } else if (valid && part == 0) {
        const int l = c / s.K, bb = c - l * s.K;
        unsigned int *word =
            static_cast<unsigned int *>(codes) + (((size_t)unit * s.L + l) * (s.Ncap >> 5) + (pos >> 5)) * s.K + bb;
        const unsigned int m = 1u << (pos & 31);
        if (bit)
            atomicOr(word, m);
        else
            atomicAnd(word, ~m);
    }
}

__global__ void bump_lengths_kernel(int B, int Ncap, int32_t *seq_lens)
{
    grid_dependency_wait();
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
        const int p = seq_lens[b];
        if (p >= 0 && p < Ncap) seq_lens[b] = p + 1;
    }
}

cudaError_t launch_append(const Shape &s, const uint16_t *k_new, const uint16_t *v_new, const uint16_t *W,
                          uint16_t *kc, uint16_t *vc, void *codes, int32_t *seq_lens, int32_t *status,
                          cudaStream_t st)
{
    const int TB = kAppendCols / s.K;
    dim3 grid((s.L + TB - 1) / TB, s.B * s.Hkv);
    cudaError_t e = launch_pdl(append_kernel, grid, dim3(256), 0, st, s, k_new, v_new, W, kc, vc, codes,
                               (const int32_t *)seq_lens, status);
    if (e != cudaSuccess) return e;
    return launch_pdl(bump_lengths_kernel, dim3(1), dim3(256), 0, st, s.B, s.Ncap, seq_lens);
}

}  // namespace mp
