// LSH-sampled decode attention for one layer (MagicPIG, Chen et al. 2024), sm_100a.
//
// Four kernels run back to back on one stream for every mp_decode_attend call:
//   qhash   SimHash codes of the query heads (fp32 projection of bf16 q onto W).
//   scan    streams the table-major key codes of a context chunk with 16-byte
//           loads, counts per token and per query head the tables whose code
//           equals the query's (saturating at 2, bit-sliced), excludes the exact
//           set D and compacts the sampled tokens (token id | head mask) with a
//           warp-ballot / block prefix sum.
//   attend  gathers the compacted K/V rows of a chunk into a cp.async shared
//           memory ring, computes q.k for all query heads of the GQA group from
//           one row load (bf16 mma.sync, fp32 accumulate), applies the -log u
//           importance correction and runs an online softmax; one extra split
//           per (b, kv head) handles D exactly (weight exp(s), no correction).
//   merge   log-sum-exp merge of the per-split partials into out / lse, plus
//           n_sampled.
#include <math.h>

#include <algorithm>

#include "mp_common.cuh"
#include "mp_kernels.cuh"

namespace mp {

// ------------------------------------------------------------------ qhash ---
// grid (ceil(L / TB), B * Hkv), 256 threads; thread = one hyperplane column of
// a table-aligned block of TB = 256 / K tables; the G query heads of one kv
// head share the W row loads.
template <int G>
__global__ void __launch_bounds__(256) qhash_kernel(Shape s, const uint16_t *__restrict__ q,
                                                    const uint16_t *__restrict__ W,
                                                    const uint16_t *__restrict__ qcodes_in,
                                                    uint16_t *__restrict__ qcodes, int32_t *status)
{
    __shared__ float qs[G][kHeadDim];
    __shared__ uint8_t bits[G][256];
    const int tid = threadIdx.x;
    const int unit = blockIdx.y;
    const int b = unit / s.Hkv, kvh = unit % s.Hkv;
    const int TB = 256 / s.K;
    const int l0 = blockIdx.x * TB;
    const size_t vec0 = (size_t)b * s.Hq + (size_t)kvh * G;

    grid_dependency_wait();
    if (status && blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) *status = 0;

    if (qcodes_in) {
        for (int i = tid; i < G * TB; i += blockDim.x) {
            int g = i / TB, l = l0 + i % TB;
            if (l < s.L) qcodes[(vec0 + g) * s.L + l] = qcodes_in[(vec0 + g) * s.L + l];
        }
        return;
    }
    for (int i = tid; i < G * kHeadDim; i += blockDim.x)
        qs[i / kHeadDim][i % kHeadDim] = bf16_to_f32(q[(vec0 + i / kHeadDim) * kHeadDim + i % kHeadDim]);
    __syncthreads();

    const int c = l0 * s.K + tid;
    const bool valid = tid < TB * s.K && c < s.LK;
    float acc[G];
#pragma unroll
    for (int g = 0; g < G; g++) acc[g] = 0.f;
    if (valid) {
        const uint4 *wr = reinterpret_cast<const uint4 *>(W + (size_t)c * kHeadDim);
#pragma unroll 4
        for (int j8 = 0; j8 < kHeadDim / 8; j8++) {
            uint4 w = __ldg(wr + j8);
            uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; e++) {
                float w0 = bf16_lo(wv[e]), w1 = bf16_hi(wv[e]);
#pragma unroll
                for (int g = 0; g < G; g++) {
                    acc[g] = fmaf(w0, qs[g][j8 * 8 + 2 * e], acc[g]);
                    acc[g] = fmaf(w1, qs[g][j8 * 8 + 2 * e + 1], acc[g]);
                }
            }
        }
    }
#pragma unroll
    for (int g = 0; g < G; g++) bits[g][tid] = valid && acc[g] > 0.f;
    __syncthreads();
    if (tid < G * TB) {
        const int g = tid / TB, tl = tid % TB, l = l0 + tl;
        if (l < s.L) {
            unsigned code = 0;
            for (int bb = 0; bb < s.K; bb++) code |= (unsigned)bits[g][tl * s.K + bb] << bb;
            qcodes[(vec0 + g) * s.L + l] = (uint16_t)code;
        }
    }
}

// ------------------------------------------------------- scan helpers -------
__device__ __forceinline__ int clamp_len(const int32_t *seq_lens, int b, int max_len, int32_t *status,
                                         bool report)
{
    int n = seq_lens[b];
    if (n < 0 || n > max_len) {
        if (report) set_status(status, MP_ERR_CAPACITY);
        n = n < 0 ? 0 : max_len;
    }
    return n;
}

// Block-wide exclusive prefix sum over blockDim.x <= 1024 threads.
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_tot, int &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = (blockDim.x + 31) >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int off = 0;
    total = 0;
    for (int w = 0; w < nwarp; w++) {
        int t = warp_tot[w];
        if (w < warp) off += t;
        total += t;
    }
    return off + incl - v;
}

__device__ __forceinline__ int block_sum(int v, int *scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = (blockDim.x + 31) >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    int t = 0;
    for (int w = 0; w < nwarp; w++) t += scratch[w];
    return t;
}

// Streaming 16-byte load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream_16(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

struct ScanOut {
    uint32_t *cand;      // [B*Hkv][nchunk][chunk] token | headmask << 24
    int32_t *cnt;        // [B*Hkv][nchunk][16]: [0] union count, [1+g] per-head count
    uint8_t *member_out; // nullable [B][Hq][Ncap]
    int32_t *status;
};

// Bits [lo - base, hi - base) of a `width`-bit token word starting at token `base`.
__device__ __forceinline__ uint32_t range_mask(int base, int lo, int hi, int width)
{
    const int a = max(lo - base, 0), e = min(hi - base, width);
    if (a >= e) return 0u;
    const uint32_t upto = e >= 32 ? 0xFFFFFFFFu : ((1u << e) - 1u);
    return upto & ~((1u << a) - 1u);
}

// Compacts one thread's sampled tokens.  hm[g][w] bit i = token t0 + 32 w + i
// is in S_g (NW words of WIDTH tokens; tokens outside [lo, hi) are masked).
// Entries keep token order: thread-major, then word, then bit.
template <int G, int NW, int WIDTH>
__device__ __forceinline__ void compact_and_store(const Shape &s, int unit, int chunk, int nchunk,
                                                  int chunk_tokens, int t0, int N, int lo, int hi,
                                                  uint32_t (&hm)[G][NW], bool owner, const ScanOut &o,
                                                  int *smem_scratch)
{
    uint32_t any[NW];
    int mine = 0;
#pragma unroll
    for (int w = 0; w < NW; w++) {
        const uint32_t v = range_mask(t0 + 32 * w, lo, hi, WIDTH);
        any[w] = 0u;
#pragma unroll
        for (int g = 0; g < G; g++) {
            hm[g][w] &= v;
            any[w] |= hm[g][w];
        }
        mine += __popc(any[w]);
    }
    int total;
    int off = block_exclusive_scan(mine, smem_scratch, total);
    uint32_t *dst = o.cand + ((size_t)unit * nchunk + chunk) * chunk_tokens;
#pragma unroll
    for (int w = 0; w < NW; w++) {
        uint32_t m = any[w];
        while (m) {
            const int bit = __ffs(m) - 1;
            m &= m - 1u;
            uint32_t heads = 0u;
#pragma unroll
            for (int g = 0; g < G; g++) heads |= ((hm[g][w] >> bit) & 1u) << g;
            dst[off++] = (uint32_t)(t0 + 32 * w + bit) | (heads << 24);
        }
    }
    int32_t *cnt = o.cnt + ((size_t)unit * nchunk + chunk) * 16;
    if (threadIdx.x == 0) cnt[0] = total;
#pragma unroll
    for (int g = 0; g < G; g++) {
        int c = 0;
#pragma unroll
        for (int w = 0; w < NW; w++) c += __popc(hm[g][w]);
        c = block_sum(c, smem_scratch + 32);
        if (threadIdx.x == 0) cnt[1 + g] = c;
    }
    if (o.member_out && owner) {
        const int b = unit / s.Hkv, kvh = unit % s.Hkv;
#pragma unroll
        for (int w = 0; w < NW; w++) {
            for (int i = 0; i < WIDTH; i++) {
                const int tok = t0 + 32 * w + i;
                if (tok >= N) break;
#pragma unroll
                for (int g = 0; g < G; g++)
                    o.member_out[((size_t)b * s.Hq + kvh * G + g) * s.Ncap + tok] = (hm[g][w] >> i) & 1u;
            }
        }
    }
}

// Table-split partial counters: thread (ts, tg) with ts > 0 leaves its two
// bit-sliced counters (seen >= 1, seen >= 2) for its token group in shared
// memory; the ts == 0 thread of the same group folds them in:
//   s2 = s2 | s2' | (s1 & s1'),  s1 = s1 | s1'.
template <int G, int NW>
__device__ __forceinline__ void combine_splits(uint32_t (&s1)[G][NW], uint32_t (&s2)[G][NW], uint32_t *part, int ts,
                                               int tg)
{
    constexpr int TG = kScanThreads / kScanSplits;
    if (ts > 0) {
#pragma unroll
        for (int g = 0; g < G; g++)
#pragma unroll
            for (int j = 0; j < NW; j++) {
                part[((g * NW + j) * 2 + 0) * kScanThreads + threadIdx.x] = s1[g][j];
                part[((g * NW + j) * 2 + 1) * kScanThreads + threadIdx.x] = s2[g][j];
            }
    }
    __syncthreads();
    if (ts == 0) {
#pragma unroll 1
        for (int t = 1; t < kScanSplits; t++) {
#pragma unroll
            for (int g = 0; g < G; g++)
#pragma unroll
                for (int j = 0; j < NW; j++) {
                    const uint32_t a1 = part[((g * NW + j) * 2 + 0) * kScanThreads + t * TG + tg];
                    const uint32_t a2 = part[((g * NW + j) * 2 + 1) * kScanThreads + t * TG + tg];
                    s2[g][j] |= a2 | (s1[g][j] & a1);
                    s1[g][j] |= a1;
                }
        }
    }
}

// ---------------------------------------------------------- scan, K = 8 ----
// Byte codes [unit][L][Ncap].  A 1024-token chunk per block of 256 threads:
// 64 token groups of 16 tokens (one 16-byte load per table) x 4 table splits
// (tables ts, ts + 4, ...), merged in shared memory.  Per 4-token word and
// head: x = codes ^ (qcode * 0x01010101); a byte of x is zero iff that token
// matches.  Zero bytes are found exactly with ((x & 0x7f..) + 0x7f..) | x,
// whose byte top bit is 1 iff the byte is non-zero.  Two bit-sliced counters
// (seen >= 1, seen >= 2) live in the byte top bits.
template <int G>
__global__ void __launch_bounds__(kScanThreads) scan_k8_kernel(
    Shape s, const uint8_t *__restrict__ codes, const uint16_t *__restrict__ qcodes,
    const int32_t *__restrict__ seq_lens, int max_len, int nchunk, ScanOut o)
{
    extern __shared__ uint32_t dyn[];  // rep [L][G] (query code in 4 bytes), then split partials
    uint32_t *rep = dyn;
    uint32_t *part = dyn + ((s.L * G + 3) & ~3);
    __shared__ int scratch[64];
    constexpr int TG = kScanThreads / kScanSplits;
    const int ts = threadIdx.x / TG, tg = threadIdx.x % TG;
    const int unit = blockIdx.y, chunk = blockIdx.x;
    const int b = unit / s.Hkv, kvh = unit % s.Hkv;
    grid_dependency_wait();
    const int N = clamp_len(seq_lens, b, max_len, o.status, chunk == 0 && kvh == 0 && threadIdx.x == 0);
    const int c0 = chunk * kChunkK8;
    if (c0 >= N) return;
    for (int i = threadIdx.x; i < s.L * G; i += blockDim.x) {
        const int l = i / G, g = i % G;
        rep[i] = (qcodes[((size_t)b * s.Hq + kvh * G + g) * s.L + l] & 0xFFu) * 0x01010101u;
    }
    __syncthreads();

    const int t0 = c0 + tg * 16;
    uint32_t s1[G][4], s2[G][4];
#pragma unroll
    for (int g = 0; g < G; g++)
#pragma unroll
        for (int j = 0; j < 4; j++) s1[g][j] = s2[g][j] = 0u;

    if (t0 < N) {
        const uint8_t *base = codes + (size_t)unit * s.L * s.Ncap + t0;
#pragma unroll 4
        for (int l = ts; l < s.L; l += kScanSplits) {
            const uint4 w4 = ld_stream_16(base + (size_t)l * s.Ncap);
            const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int g = 0; g < G; g++) {
                const uint32_t r = rep[l * G + g];
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    const uint32_t x = w[j] ^ r;
                    const uint32_t nz = ((x & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | x;
                    s2[g][j] |= s1[g][j] & ~nz;
                    s1[g][j] |= ~nz;
                }
            }
        }
    }
    combine_splits<G, 4>(s1, s2, part, ts, tg);
    // Per-head 16-bit token masks from the byte top bits of the >= 2 counter.
    uint32_t hm[G][1];
#pragma unroll
    for (int g = 0; g < G; g++) {
        uint32_t m = 0u;
#pragma unroll
        for (int i = 0; i < 16; i++) m |= ((s2[g][i >> 2] >> (8 * (i & 3) + 7)) & 1u) << i;
        hm[g][0] = ts == 0 ? m : 0u;
    }
    // Tokens eligible for S: [sink, N - window) and below N.
    compact_and_store<G, 1, 16>(s, unit, chunk, nchunk, kChunkK8, t0, N, s.sink, min(N - s.window, N), hm,
                                ts == 0, o, scratch);
}

// --------------------------------------------------------- scan, K = 10 ----
// Bit-plane codes [unit][L][K][Ncap/32] (uint32).  An 8192-token chunk per
// block of 256 threads: 64 token groups of 128 tokens (one 16-byte load per
// plane) x 4 table splits.  A token mismatches table l for head h iff some
// plane differs from the query bit: mis = OR_b (plane_b ^ qmask_b), with
// qmask_b = 0 or ~0 from shared memory.
template <int G>
__global__ void __launch_bounds__(kScanThreads) scan_k10_kernel(
    Shape s, const uint32_t *__restrict__ codes, const uint16_t *__restrict__ qcodes,
    const int32_t *__restrict__ seq_lens, int max_len, int nchunk, ScanOut o)
{
    extern __shared__ uint32_t dyn[];  // qm [L][G][12] (qmask of the 10 planes, padded), then split partials
    uint32_t *qm = dyn;
    uint32_t *part = dyn + s.L * G * 12;
    __shared__ int scratch[64];
    constexpr int KB = 10;
    constexpr int TG = kScanThreads / kScanSplits;
    const int ts = threadIdx.x / TG, tg = threadIdx.x % TG;
    const int unit = blockIdx.y, chunk = blockIdx.x;
    const int b = unit / s.Hkv, kvh = unit % s.Hkv;
    grid_dependency_wait();
    const int N = clamp_len(seq_lens, b, max_len, o.status, chunk == 0 && kvh == 0 && threadIdx.x == 0);
    const int c0 = chunk * kChunkK10;
    if (c0 >= N) return;
    for (int i = threadIdx.x; i < s.L * G * 12; i += blockDim.x) {
        const int l = i / (G * 12), g = (i / 12) % G, bb = i % 12;
        const unsigned code = qcodes[((size_t)b * s.Hq + kvh * G + g) * s.L + l];
        qm[i] = bb < KB ? 0u - ((code >> bb) & 1u) : 0u;
    }
    __syncthreads();

    const int t0 = c0 + tg * 128;
    const int words = s.Ncap >> 5;
    uint32_t s1[G][4], s2[G][4];
#pragma unroll
    for (int g = 0; g < G; g++)
#pragma unroll
        for (int j = 0; j < 4; j++) s1[g][j] = s2[g][j] = 0u;

    if (t0 < N) {
        const uint32_t *base = codes + (size_t)unit * s.L * KB * words + (t0 >> 5);
#pragma unroll 1
        for (int l = ts; l < s.L; l += kScanSplits) {
            uint4 pl[KB];
#pragma unroll
            for (int bb = 0; bb < KB; bb++) pl[bb] = ld_stream_16(base + ((size_t)l * KB + bb) * words);
#pragma unroll
            for (int g = 0; g < G; g++) {
                const uint4 *m4 = reinterpret_cast<const uint4 *>(qm + (l * G + g) * 12);
                const uint4 ma = m4[0], mb = m4[1], mc = m4[2];
                const uint32_t msk[KB] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w, mc.x, mc.y};
                uint32_t mis[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int bb = 0; bb < KB; bb++) {
                    mis[0] |= pl[bb].x ^ msk[bb];
                    mis[1] |= pl[bb].y ^ msk[bb];
                    mis[2] |= pl[bb].z ^ msk[bb];
                    mis[3] |= pl[bb].w ^ msk[bb];
                }
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    s2[g][j] |= s1[g][j] & ~mis[j];
                    s1[g][j] |= ~mis[j];
                }
            }
        }
    }
    combine_splits<G, 4>(s1, s2, part, ts, tg);
    if (ts != 0) {
#pragma unroll
        for (int g = 0; g < G; g++)
#pragma unroll
            for (int j = 0; j < 4; j++) s2[g][j] = 0u;
    }
    compact_and_store<G, 4, 32>(s, unit, chunk, nchunk, kChunkK10, t0, N, s.sink, min(N - s.window, N), s2,
                                ts == 0, o, scratch);
}

// ---------------------------------------------------------------- attend ----
// log u for the at-least-2-of-L rule, u = P[Binomial(L, x) >= 2], x = p^K,
// p = 1 - arccos(c)/pi.  Small x: u = C(L,2) x^2 (1-x)^(L-2) * (1 + a3 r (1 +
// a4 r (1 + a5 r))) with r = x / (1-x), a_j = (L-j+1)/j (binomial ratios),
// truncated after j = 5 (relative error < 2e-6 for x < 1e-3, L <= 255).
// Otherwise u = 1 - exp(y), y = (L-1) log1p(-x) + log1p((L-1) x) (the closed
// form 1 - (1-x)^L - L x (1-x)^(L-1) rearranged so that expm1 keeps u's
// relative precision).
struct LogU {
    float K, L, lnC2, a3, a4, a5;
};

__device__ __forceinline__ float log_sampling_prob(float c, const LogU &u)
{
    c = fminf(1.f, fmaxf(-1.f, c));
    float p = 1.f - acosf(c) * 0.318309886183790671538f;
    p = fmaxf(p, 1e-30f);
    const float lx = u.K * logf(p);
    const float x = expf(lx);
    if (x < 1e-3f) {
        const float r = x / (1.f - x);
        const float tail = u.a3 * r * (1.f + u.a4 * r * (1.f + u.a5 * r));
        return u.lnC2 + 2.f * lx + (u.L - 2.f) * log1pf(-x) + log1pf(tail);
    }
    const float y = (u.L - 1.f) * log1pf(-x) + log1pf((u.L - 1.f) * x);
    return logf(-expm1f(y));
}

constexpr int kAttThreads = 128;
constexpr int kAttRows = 64;                // rows per tile (4 warps x 16)
constexpr int kAttStages = 3;               // cp.async ring depth
constexpr int kRowBytes = kHeadDim * 2;     // 256
constexpr int kRowStride = kRowBytes + 16;  // padded: conflict-free ldmatrix / 8-byte reads
constexpr int kStageBytes = kAttRows * kRowStride * 2;  // K rows then V rows

struct AttendArgs {
    Shape s;
    const uint16_t *q;
    const uint16_t *kc;
    const uint16_t *vc;
    const int32_t *seq_lens;
    int max_len;
    int nchunk;
    int subs;   // blocks per scan chunk (each takes an equal share of its candidate list)
    int chunk_tokens;
    const uint32_t *cand;
    const int32_t *cnt;
    float *pm, *pl, *pacc;  // [B*Hq][nchunk*subs+1], [..][..][128]
    LogU lu;
    float scale;  // 1/sqrt(d)
};

template <int G>
__global__ void __launch_bounds__(kAttThreads, 2) attend_kernel(AttendArgs a)
{
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ float sc[4][16][G];        // per warp: raw scores, then t, then p
    __shared__ float nrm[4][16];          // per warp: |k|^2
    __shared__ uint32_t meta[kAttStages][kAttRows];  // headmask | exact << 8
    __shared__ float qinv[G];
    __shared__ uint8_t upairs[4][16 * G];             // per warp: (row, head) pairs that need log u

    const Shape &s = a.s;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int unit = blockIdx.y, split = blockIdx.x;
    const int b = unit / s.Hkv, kvh = unit % s.Hkv;
    grid_dependency_wait();
    int N = a.seq_lens[b];
    N = N < 0 ? 0 : (N > a.max_len ? a.max_len : N);
    const bool dsplit = split == a.nchunk * a.subs;
    const int chunk = split / a.subs, sub = split % a.subs;
    if (!dsplit && chunk * a.chunk_tokens >= N) return;

    // Rows of this block: its share of a chunk's compacted candidates, or the
    // exact set D.
    const int n_sink = min(s.sink, N);
    const int win0 = max(n_sink, N - s.window);
    int nrows;
    const uint32_t *list = nullptr;
    if (dsplit) {
        nrows = n_sink + (N - win0);
    } else {
        const int total = a.cnt[((size_t)unit * a.nchunk + chunk) * 16];
        const int per = (total + a.subs - 1) / a.subs;
        const int e0 = min(total, sub * per);
        nrows = min(total, e0 + per) - e0;
        list = a.cand + ((size_t)unit * a.nchunk + chunk) * a.chunk_tokens + e0;
    }
    auto row_of = [&](int e, uint32_t &m) -> int {
        if (dsplit) {
            m = ((1u << G) - 1u) | 0x100u;
            return e < n_sink ? e : win0 + (e - n_sink);
        }
        const uint32_t v = list[e];
        m = v >> 24;
        return (int)(v & 0xFFFFFFu);
    };

    const size_t vec0 = (size_t)b * s.Hq + (size_t)kvh * G;
    // B fragments of Q^T (k = head_dim, n = head), 8 k-steps x 2 registers.
    uint32_t qb[8][2];
    {
        const int gq = lane >> 2, t = lane & 3;
#pragma unroll
        for (int ks = 0; ks < 8; ks++) {
            if (gq < G) {
                const uint32_t *qp = reinterpret_cast<const uint32_t *>(a.q + (vec0 + gq) * kHeadDim);
                qb[ks][0] = qp[(ks * 16 + 2 * t) >> 1];
                qb[ks][1] = qp[(ks * 16 + 2 * t + 8) >> 1];
            } else {
                qb[ks][0] = qb[ks][1] = 0u;
            }
        }
    }
    if (tid < G) {
        float qq = 0.f;
        const uint16_t *qp = a.q + (vec0 + tid) * kHeadDim;
        for (int j = 0; j < kHeadDim; j++) {
            float v = bf16_to_f32(qp[j]);
            qq = fmaf(v, v, qq);
        }
        qinv[tid] = qq > 0.f ? rsqrtf(qq) : 0.f;
    }

    const uint16_t *kbase = a.kc + (size_t)unit * s.Ncap * kHeadDim;
    const uint16_t *vbase = a.vc + (size_t)unit * s.Ncap * kHeadDim;
    const int ntiles = (nrows + kAttRows - 1) / kAttRows;

    // Tile loader: thread = 16-byte column (tid % 16) of rows tid/16 + 8 i.
    auto load_tile = [&](int tile, int stage) {
        uint8_t *ks_ = smem + stage * kStageBytes;
        uint8_t *vs_ = ks_ + kAttRows * kRowStride;
        const int col = tid & 15;
#pragma unroll
        for (int i = 0; i < kAttRows / 8; i++) {
            const int r = (tid >> 4) + 8 * i;
            const int e = tile * kAttRows + r;
            uint32_t m = 0;
            int tok = 0;
            const bool ok = e < nrows;
            if (ok) tok = row_of(e, m);
            const size_t off = (size_t)tok * kHeadDim + col * 8;
            cp_async_16(ks_ + r * kRowStride + col * 16, kbase + off, ok ? 16 : 0);
            cp_async_16(vs_ + r * kRowStride + col * 16, vbase + off, ok ? 16 : 0);
            if (col == 0) meta[stage][r] = ok ? m : 0u;
        }
    };

    float m_run[G], l_run[G], acc[G][4];
#pragma unroll
    for (int g = 0; g < G; g++) {
        m_run[g] = -INFINITY;
        l_run[g] = 0.f;
#pragma unroll
        for (int e = 0; e < 4; e++) acc[g][e] = 0.f;
    }

#pragma unroll
    for (int st = 0; st < kAttStages - 1; st++) {
        if (st < ntiles) load_tile(st, st);
        cp_async_commit();
    }
    __syncthreads();  // qinv

    for (int tile = 0; tile < ntiles; tile++) {
        {
            const int nt = tile + kAttStages - 1;
            if (nt < ntiles) load_tile(nt, nt % kAttStages);
            cp_async_commit();
        }
        cp_async_wait<kAttStages - 1>();
        __syncthreads();
        const int stage = tile % kAttStages;
        const uint8_t *ks_ = smem + stage * kStageBytes;
        const uint8_t *vs_ = ks_ + kAttRows * kRowStride;

        // ---- S^T (16 rows x 8 heads) = K rows . Q^T, plus |k|^2 ----
        float c0 = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f, na = 0.f, nb = 0.f;
        {
            const uint8_t *arow = ks_ + (warp * 16 + (lane & 15)) * kRowStride + (lane >> 4) * 16;
#pragma unroll
            for (int kst = 0; kst < 8; kst++) {
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4(a0, a1, a2, a3, arow + kst * 32);
                mma_bf16_16816(c0, c1, c2, c3, a0, a1, a2, a3, qb[kst][0], qb[kst][1]);
                float x;
                x = bf16_lo(a0); na = fmaf(x, x, na);
                x = bf16_hi(a0); na = fmaf(x, x, na);
                x = bf16_lo(a2); na = fmaf(x, x, na);
                x = bf16_hi(a2); na = fmaf(x, x, na);
                x = bf16_lo(a1); nb = fmaf(x, x, nb);
                x = bf16_hi(a1); nb = fmaf(x, x, nb);
                x = bf16_lo(a3); nb = fmaf(x, x, nb);
                x = bf16_hi(a3); nb = fmaf(x, x, nb);
            }
            na += __shfl_xor_sync(0xffffffffu, na, 1);
            na += __shfl_xor_sync(0xffffffffu, na, 2);
            nb += __shfl_xor_sync(0xffffffffu, nb, 1);
            nb += __shfl_xor_sync(0xffffffffu, nb, 2);
            const int gr = lane >> 2, t = lane & 3;
            if (2 * t < G) {
                sc[warp][gr][2 * t] = c0;
                sc[warp][gr + 8][2 * t] = c2;
            }
            if (2 * t + 1 < G) {
                sc[warp][gr][2 * t + 1] = c1;
                sc[warp][gr + 8][2 * t + 1] = c3;
            }
            if (t == 0) {
                nrm[warp][gr] = na;
                nrm[warp][gr + 8] = nb;
            }
        }
        __syncwarp();

        // ---- log-weights t = s (exact) or s - log u (sampled), -inf if absent ----
        // The (row, head) pairs that need log u are compacted first so that the
        // transcendental work runs on sampled pairs only.
        int nu = 0;
        for (int p0 = 0; p0 < 16 * G; p0 += 32) {
            const int p = p0 + lane;
            bool need = false;
            if (p < 16 * G) {
                const int r = p / G, h = p % G;
                const uint32_t m = meta[stage][warp * 16 + r];
                const bool mem = (m >> h) & 1u;
                need = mem && !(m & 0x100u);
                sc[warp][r][h] = mem ? sc[warp][r][h] * a.scale : -INFINITY;
            }
            const uint32_t bal = __ballot_sync(0xffffffffu, need);
            if (need) upairs[warp][nu + __popc(bal & ((1u << lane) - 1u))] = (uint8_t)p;
            nu += __popc(bal);
        }
        __syncwarp();
        for (int j = lane; j < nu; j += 32) {
            const int p = upairs[warp][j];
            const int r = p / G, h = p % G;
            const float kk = nrm[warp][r];
            const float sv = sc[warp][r][h];  // already scaled by 1/sqrt(d)
            const float cosv = kk > 0.f ? sv * (1.f / a.scale) * qinv[h] * rsqrtf(kk) : 0.f;
            sc[warp][r][h] = sv - log_sampling_prob(cosv, a.lu);
        }
        __syncwarp();

        // ---- online softmax update (per warp state) ----
        float alpha[G], mnew[G];
#pragma unroll
        for (int g = 0; g < G; g++) {
            float mt = -INFINITY;
#pragma unroll
            for (int r = 0; r < 16; r++) mt = fmaxf(mt, sc[warp][r][g]);
            mnew[g] = fmaxf(m_run[g], mt);
            alpha[g] = mnew[g] == -INFINITY ? 1.f : expf(m_run[g] - mnew[g]);
        }
        __syncwarp();
        for (int p = lane; p < 16 * G; p += 32) {
            const int r = p / G, h = p % G;
            const float tv = sc[warp][r][h];
            sc[warp][r][h] = tv == -INFINITY ? 0.f : expf(tv - mnew[h]);
        }
        __syncwarp();
        float lsum[G];
#pragma unroll
        for (int g = 0; g < G; g++) {
            lsum[g] = 0.f;
#pragma unroll
            for (int e = 0; e < 4; e++) acc[g][e] *= alpha[g];
        }
#pragma unroll 4
        for (int r = 0; r < 16; r++) {
            const uint2 vv = *reinterpret_cast<const uint2 *>(vs_ + (warp * 16 + r) * kRowStride + lane * 8);
            const float v0 = bf16_lo(vv.x), v1 = bf16_hi(vv.x), v2 = bf16_lo(vv.y), v3 = bf16_hi(vv.y);
#pragma unroll
            for (int g = 0; g < G; g++) {
                const float pw = sc[warp][r][g];
                lsum[g] += pw;
                acc[g][0] = fmaf(pw, v0, acc[g][0]);
                acc[g][1] = fmaf(pw, v1, acc[g][1]);
                acc[g][2] = fmaf(pw, v2, acc[g][2]);
                acc[g][3] = fmaf(pw, v3, acc[g][3]);
            }
        }
#pragma unroll
        for (int g = 0; g < G; g++) {
            l_run[g] = l_run[g] * alpha[g] + lsum[g];
            m_run[g] = mnew[g];
        }
        __syncthreads();  // stage may be refilled next iteration
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---- merge the 4 warps' states, write this split's partial ----
    float *red = reinterpret_cast<float *>(smem);  // [4][G][128] acc, then m, l
    float *redm = red + 4 * G * kHeadDim;
    float *redl = redm + 4 * G;
#pragma unroll
    for (int g = 0; g < G; g++) {
#pragma unroll
        for (int e = 0; e < 4; e++) red[(warp * G + g) * kHeadDim + lane * 4 + e] = acc[g][e];
        if (lane == 0) {
            redm[warp * G + g] = m_run[g];
            redl[warp * G + g] = l_run[g];
        }
    }
    __syncthreads();
    const int dim = tid;  // 128 threads = head_dim
    for (int g = 0; g < G; g++) {
        float M = -INFINITY;
        for (int w = 0; w < 4; w++) M = fmaxf(M, redm[w * G + g]);
        float Ls = 0.f, A = 0.f;
        if (M != -INFINITY) {
            for (int w = 0; w < 4; w++) {
                const float mw = redm[w * G + g];
                if (mw == -INFINITY) continue;
                const float f = expf(mw - M);
                Ls += redl[w * G + g] * f;
                A += red[(w * G + g) * kHeadDim + dim] * f;
            }
        }
        const size_t bh = vec0 + g;
        const size_t pidx = bh * ((size_t)a.nchunk * a.subs + 1) + split;
        a.pacc[pidx * kHeadDim + dim] = A;
        if (dim == 0) {
            a.pm[pidx] = M;
            a.pl[pidx] = Ls;
        }
    }
}

// ----------------------------------------------------------------- merge ----
template <int G>
__global__ void __launch_bounds__(kHeadDim) merge_kernel(Shape s, const int32_t *__restrict__ seq_lens,
                                                         int max_len, int nchunk, int subs, int chunk_tokens,
                                                         const float *__restrict__ pm,
                                                         const float *__restrict__ pl,
                                                         const float *__restrict__ pacc,
                                                         const int32_t *__restrict__ cnt, float *out,
                                                         float *lse, int32_t *n_sampled)
{
    const int bh = blockIdx.x;
    const int b = bh / s.Hq, h = bh % s.Hq, kvh = h / G, g = h % G;
    const int unit = b * s.Hkv + kvh;
    grid_dependency_wait();
    int N = seq_lens[b];
    N = N < 0 ? 0 : (N > max_len ? max_len : N);
    const int nsp = ((N + chunk_tokens - 1) / chunk_tokens) * subs;  // live chunk splits
    const int dsp = nchunk * subs;                                    // the exact-set split
    const int dim = threadIdx.x;
    const size_t base = (size_t)bh * (dsp + 1);
    float M = pm[base + dsp];
    for (int j = 0; j < nsp; j++) M = fmaxf(M, pm[base + j]);
    float Ls = 0.f, A = 0.f;
    if (M != -INFINITY) {
        auto add = [&](int j) {
            const float mj = pm[base + j];
            if (mj == -INFINITY) return;
            const float f = expf(mj - M);
            Ls += pl[base + j] * f;
            A += pacc[(base + j) * kHeadDim + dim] * f;
        };
        for (int j = 0; j < nsp; j++) add(j);
        add(dsp);
    }
    out[(size_t)bh * kHeadDim + dim] = Ls > 0.f ? A / Ls : 0.f;
    if (dim == 0) {
        lse[bh] = Ls > 0.f ? M + logf(Ls) : -INFINITY;
        int ns = 0;
        for (int j = 0; j < nsp / subs; j++) ns += cnt[((size_t)unit * nchunk + j) * 16 + 1 + g];
        n_sampled[bh] = ns;
    }
}

// ---------------------------------------------------------------- launch ----
struct Workspace {
    int32_t *status;
    uint16_t *qcodes;
    uint32_t *cand;
    int32_t *cnt;
    float *pm, *pl, *pacc;
    size_t bytes;
};

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Attention blocks per scan chunk: enough blocks for two waves on 148 SMs
// (a fixed count, so the workspace size does not depend on the device).
static int attend_subs(const Shape &s, int nchunk)
{
    const int blocks = nchunk * s.B * s.Hkv;
    if (blocks == 0) return 1;
    return std::max(1, std::min(8, (296 + blocks - 1) / blocks));
}

Workspace workspace_layout(const Shape &s, int max_len, void *base)
{
    const int C = chunk_tokens(s.K);
    const int nchunk = (max_len + C - 1) / C;
    const size_t nsplit = (size_t)nchunk * attend_subs(s, nchunk) + 1;
    const size_t units = (size_t)s.B * s.Hkv, bh = (size_t)s.B * s.Hq;
    size_t off = 0;
    Workspace w{};
    uint8_t *p = static_cast<uint8_t *>(base);
    auto take = [&](size_t bytes) {
        uint8_t *r = p ? p + off : nullptr;
        off += align256(bytes);
        return r;
    };
    w.status = reinterpret_cast<int32_t *>(take(16));
    w.qcodes = reinterpret_cast<uint16_t *>(take(bh * s.L * sizeof(uint16_t)));
    w.cand = reinterpret_cast<uint32_t *>(take(units * nchunk * (size_t)C * sizeof(uint32_t)));
    w.cnt = reinterpret_cast<int32_t *>(take(units * nchunk * 16 * sizeof(int32_t)));
    w.pm = reinterpret_cast<float *>(take(bh * nsplit * sizeof(float)));
    w.pl = reinterpret_cast<float *>(take(bh * nsplit * sizeof(float)));
    w.pacc = reinterpret_cast<float *>(take(bh * nsplit * kHeadDim * sizeof(float)));
    w.bytes = off;
    return w;
}

size_t decode_workspace_bytes(const Shape &s, int max_len) { return workspace_layout(s, max_len, nullptr).bytes; }

static LogU make_logu(const Shape &s)
{
    LogU u;
    const double L = s.L;
    u.K = (float)s.K;
    u.L = (float)L;
    u.lnC2 = (float)log(L * (L - 1.0) / 2.0);
    u.a3 = (float)((L - 2.0) / 3.0);
    u.a4 = (float)((L - 3.0) / 4.0);
    u.a5 = (float)((L - 4.0) / 5.0);
    return u;
}

template <int G>
static cudaError_t launch_decode_g(const Shape &s, const uint16_t *q, const uint16_t *W, const void *codes,
                                   const uint16_t *kc, const uint16_t *vc, const int32_t *seq_lens,
                                   int max_len, float *out, float *lse, int32_t *n_sampled,
                                   const Workspace &ws, const mp_decode_debug *dbg, cudaStream_t st)
{
    const int C = chunk_tokens(s.K);
    const int nchunk = (max_len + C - 1) / C;
    const int subs = attend_subs(s, nchunk);
    const int units = s.B * s.Hkv;
    cudaError_t e;
    {
        dim3 grid((s.L + 256 / s.K - 1) / (256 / s.K), units);
        e = launch_pdl(qhash_kernel<G>, grid, dim3(256), 0, st, s, q, W,
                       (const uint16_t *)(dbg ? dbg->qcodes_in : nullptr), ws.qcodes, ws.status);
        if (e != cudaSuccess) return e;
    }
    ScanOut so{ws.cand, ws.cnt, dbg ? dbg->member_out : nullptr, ws.status};
    if (nchunk > 0) {
        dim3 grid(nchunk, units);
        const size_t part = (size_t)2 * G * 4 * kScanThreads * sizeof(uint32_t);
        if (s.K == 8) {
            const size_t sm = (size_t)((s.L * G + 3) & ~3) * sizeof(uint32_t) + part;
            if ((e = ensure_smem(reinterpret_cast<const void *>(scan_k8_kernel<G>), (int)sm)) != cudaSuccess) return e;
            e = launch_pdl(scan_k8_kernel<G>, grid, dim3(kScanThreads), sm, st, s,
                           static_cast<const uint8_t *>(codes), (const uint16_t *)ws.qcodes, seq_lens, max_len,
                           nchunk, so);
        } else {
            const size_t sm = (size_t)s.L * G * 12 * sizeof(uint32_t) + part;
            if ((e = ensure_smem(reinterpret_cast<const void *>(scan_k10_kernel<G>), (int)sm)) != cudaSuccess) return e;
            e = launch_pdl(scan_k10_kernel<G>, grid, dim3(kScanThreads), sm, st, s,
                           static_cast<const uint32_t *>(codes), (const uint16_t *)ws.qcodes, seq_lens, max_len,
                           nchunk, so);
        }
        if (e != cudaSuccess) return e;
    }
    AttendArgs aa;
    aa.s = s;
    aa.q = q;
    aa.kc = kc;
    aa.vc = vc;
    aa.seq_lens = seq_lens;
    aa.max_len = max_len;
    aa.nchunk = nchunk;
    aa.subs = subs;
    aa.chunk_tokens = C;
    aa.cand = ws.cand;
    aa.cnt = ws.cnt;
    aa.pm = ws.pm;
    aa.pl = ws.pl;
    aa.pacc = ws.pacc;
    aa.lu = make_logu(s);
    aa.scale = 1.0f / sqrtf((float)s.d);
    {
        const int sm = kAttStages * kStageBytes;
        if ((e = ensure_smem(reinterpret_cast<const void *>(attend_kernel<G>), sm)) != cudaSuccess) return e;
        dim3 grid(nchunk * subs + 1, units);
        if ((e = launch_pdl(attend_kernel<G>, grid, dim3(kAttThreads), sm, st, aa)) != cudaSuccess) return e;
    }
    e = launch_pdl(merge_kernel<G>, dim3(s.B * s.Hq), dim3(kHeadDim), 0, st, s, seq_lens, max_len, nchunk, subs, C,
                   (const float *)ws.pm, (const float *)ws.pl, (const float *)ws.pacc, (const int32_t *)ws.cnt, out,
                   lse, n_sampled);
    if (e != cudaSuccess) return e;
    if (dbg && dbg->qcodes_out)
        e = cudaMemcpyAsync(dbg->qcodes_out, ws.qcodes, (size_t)s.B * s.Hq * s.L * sizeof(uint16_t),
                            cudaMemcpyDeviceToDevice, st);
    return e;
}

cudaError_t launch_decode(const Shape &s, const uint16_t *q, const uint16_t *W, const void *codes,
                          const uint16_t *kc, const uint16_t *vc, const int32_t *seq_lens, int max_len,
                          float *out, float *lse, int32_t *n_sampled, void *workspace,
                          const mp_decode_debug *dbg, cudaStream_t st)
{
    const Workspace ws = workspace_layout(s, max_len, workspace);
    switch (s.G) {
    case 1: return launch_decode_g<1>(s, q, W, codes, kc, vc, seq_lens, max_len, out, lse, n_sampled, ws, dbg, st);
    case 2: return launch_decode_g<2>(s, q, W, codes, kc, vc, seq_lens, max_len, out, lse, n_sampled, ws, dbg, st);
    case 4: return launch_decode_g<4>(s, q, W, codes, kc, vc, seq_lens, max_len, out, lse, n_sampled, ws, dbg, st);
    case 8: return launch_decode_g<8>(s, q, W, codes, kc, vc, seq_lens, max_len, out, lse, n_sampled, ws, dbg, st);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_hash_queries(const Shape &s, const uint16_t *q, const uint16_t *W, uint16_t *qcodes,
                                cudaStream_t st)
{
    dim3 grid((s.L + 256 / s.K - 1) / (256 / s.K), s.B * s.Hkv);
    const uint16_t *none = nullptr;
    int32_t *no_status = nullptr;
    switch (s.G) {
    case 1: return launch_pdl(qhash_kernel<1>, grid, dim3(256), 0, st, s, q, W, none, qcodes, no_status);
    case 2: return launch_pdl(qhash_kernel<2>, grid, dim3(256), 0, st, s, q, W, none, qcodes, no_status);
    case 4: return launch_pdl(qhash_kernel<4>, grid, dim3(256), 0, st, s, q, W, none, qcodes, no_status);
    case 8: return launch_pdl(qhash_kernel<8>, grid, dim3(256), 0, st, s, q, W, none, qcodes, no_status);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace mp
