// int8 copy of the cached keys for the reduced-precision attention gather
// (opt-in; the bf16 keys stay the reference).  The format is described in
// mp_kquant.cuh.
#include "mp_kernels.cuh"
#include "mp_kquant.cuh"

namespace mp {

constexpr int kQuantRowsPerWarp = 8;  // two rows per pass (a half-warp each), four passes
constexpr int kQuantRowsPerBlock = 8 * kQuantRowsPerWarp;

// grid (ceil(n_tokens / 64), B * Hkv), 256 threads.  A streaming kernel: each
// half-warp takes a row (16 bytes = 8 values per lane) and a warp loads all
// four of its row pairs before it reduces any, so that 2 KB per warp are in
// flight.  Token range [tok0, tok0 + n_tokens) of one unit; with seq_lens,
// unit (b, .) stops at seq_lens[b].
__global__ void __launch_bounds__(256) quantize_keys_kernel(Shape s, const uint16_t *__restrict__ kc,
                                                            const int32_t *__restrict__ seq_lens, int tok0,
                                                            int n_tokens, int8_t *k8)
{
    grid_dependency_wait();
    const int unit = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = lane >> 4, hl = lane & 15;
    int end = tok0 + n_tokens;
    if (seq_lens) end = min(end, max(seq_lens[unit / s.Hkv], 0));
    const int t0 = tok0 + blockIdx.x * kQuantRowsPerBlock + warp * kQuantRowsPerWarp;
    if (t0 >= end) return;  // whole warps leave together
    const size_t row0 = (size_t)unit * s.Ncap;
    uint4 v[kQuantRowsPerWarp / 2];
#pragma unroll
    for (int p = 0; p < kQuantRowsPerWarp / 2; p++) {
        const int t = t0 + 2 * p + half;
        v[p] = t < end ? reinterpret_cast<const uint4 *>(kc + (row0 + t) * kHeadDim)[hl] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int p = 0; p < kQuantRowsPerWarp / 2; p++) {
        const int t = t0 + 2 * p + half;
        const float x[8] = {bf16_lo(v[p].x), bf16_hi(v[p].x), bf16_lo(v[p].y), bf16_hi(v[p].y),
                            bf16_lo(v[p].z), bf16_hi(v[p].z), bf16_lo(v[p].w), bf16_hi(v[p].w)};
        uint32_t packed[2];
        float sc, n2;
        quantize_values<8, 16>(x, packed, sc, n2);  // every lane takes part (the shuffles span the warp)
        if (t < end) {
            int8_t *rowp = k8 + (row0 + t) * kQ8RowBytes;
            reinterpret_cast<uint2 *>(rowp)[hl] = make_uint2(packed[0], packed[1]);
            if (hl == 0) *reinterpret_cast<float4 *>(rowp + kHeadDim) = make_float4(sc, n2, 0.f, 0.f);
        }
    }
}

cudaError_t launch_quantize_keys(const Shape &s, const uint16_t *kc, const int32_t *seq_lens, int tok0, int n_tokens,
                                 int8_t *k8, cudaStream_t st)
{
    if (n_tokens == 0) return cudaSuccess;
    dim3 grid((n_tokens + kQuantRowsPerBlock - 1) / kQuantRowsPerBlock, s.B * s.Hkv);
    return launch_pdl(quantize_keys_kernel, grid, dim3(256), 0, st, s, kc, seq_lens, tok0, n_tokens, k8);
}

}  // namespace mp
