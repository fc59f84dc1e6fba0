// int8 keys for the reduced-precision attention gather (opt-in).
//
// A cached key row k (128 bf16 values) is stored as q = rint(k / s), int8 in
// [-127, 127], with one power-of-two scale per row, s = 2^e the smallest power
// of two with 127 s >= max_j |k_j| (s = 0 for a zero row).  Because s is a
// power of two, k / s and s q are exact in fp32, the rounding is the only
// error (|k - s q| <= s / 2 <= max|k| / 127), and s q is exactly a bf16 value
// (at most 8 significant bits), so the keys the attention kernel effectively
// uses can be written back as bf16 and checked against the fp64 oracle.
//
// The int8 values are followed, in the same 144-byte row, by a 16-byte
// record {s, |s q|^2, 0, 0} (fp32): the gather fetches row and record as one
// contiguous piece, and the stored squared norm saves the attention kernel
// the K K^T products it would otherwise need for the collision probability.
// sum_j q_j^2 <= 128 * 127^2 < 2^24 is an exact fp32 integer and s^2 a power
// of two, so the stored norm is exact.
#pragma once

#include <math.h>

#include "mp_common.cuh"

namespace mp {

constexpr int kQ8RowBytes = kHeadDim + 16;  // 128 int8 values, then the record

// Quantises one row spread over W lanes (aligned groups of W lanes of the
// warp; every lane of the warp calls this), each holding E consecutive values
// x[0..E): fills packed[E / 4] (bytes in value order) and returns the row's
// scale and squared norm in every lane of the group.
template <int E, int W>
__device__ __forceinline__ void quantize_values(const float (&x)[E], uint32_t (&packed)[E / 4], float &scale,
                                                float &norm2)
{
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < E; i++) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
    for (int o = W / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
#pragma unroll
    for (int i = 0; i < E / 4; i++) packed[i] = 0u;
    int sq = 0;
    float s = 0.f;
    if (amax > 0.f) {
        int E2;
        frexpf(amax, &E2);  // amax = m 2^E2, m in [0.5, 1)
        int e = E2 - 7;     // 127 * 2^(E2-7) is just below 2^E2 ...
        if (127.f * ldexpf(1.f, e) < amax) e++;  // ... so at most one step up
        s = ldexpf(1.f, e);
#pragma unroll
        for (int i = 0; i < E; i++) {
            const int qi = __float2int_rn(ldexpf(x[i], -e));  // exact scaling, then round to nearest even
            packed[i >> 2] |= (uint32_t)(qi & 0xFF) << (8 * (i & 3));
            sq += qi * qi;
        }
    }
#pragma unroll
    for (int o = W / 2; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    scale = s;
    norm2 = (float)sq * s * s;
}

// One warp quantises one row into q8row (kQ8RowBytes): lane l takes dims
// 4 l .. 4 l + 3.
__device__ __forceinline__ void quantize_key_row(const uint16_t *k, int8_t *q8row, int lane)
{
    const uint2 v = reinterpret_cast<const uint2 *>(k)[lane];
    const float x[4] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y)};
    uint32_t packed[1];
    float s, n2;
    quantize_values<4, 32>(x, packed, s, n2);
    reinterpret_cast<uint32_t *>(q8row)[lane] = packed[0];
    if (lane == 0) *reinterpret_cast<float4 *>(q8row + kHeadDim) = make_float4(s, n2, 0.f, 0.f);
}

}  // namespace mp
