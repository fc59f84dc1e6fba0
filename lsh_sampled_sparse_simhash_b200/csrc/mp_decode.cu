// LSH-sampled decode attention for one layer (MagicPIG, Chen et al. 2024), sm_100a.
//
// Every mp_decode_attend call runs these kernels back to back on one stream
// (programmatic dependent launch between them):
//   qhash   SimHash codes of the query heads (fp32 projection of bf16 q onto W).
//   scan    counts, per token and query head, the tables whose code equals the
//           query's (bit-sliced counters saturating at 2), excludes the exact
//           set D and compacts the sampled tokens (token id | head mask) in
//           token order.  Byte codes: scan_bytes_kernel, packed fp16
//           compares of two tokens per instruction.  Bit planes:
//           scan_planes_warp_kernel, 32 tokens per logic operation.  Both
//           give each warp one chunk of one unit for all L tables, fed by
//           the warp's own cp.async ring.
//   attend  gathers the compacted K/V rows into a cp.async shared-memory
//           ring, computes q.k for all query heads of the GQA group from one
//           row load (bf16 mma.sync, fp32 accumulate), applies the -log u
//           importance correction and runs an online softmax in base 2; one
//           extra split per (b, kv head) handles D exactly (weight exp(s)).
//   merge   log-sum-exp merge of the per-split partials into out / lse, plus
//           n_sampled.
// The scan releases each chunk's candidate list with a ready flag, and the
// attention, launched as soon as every scan block is running, starts on a
// chunk once its flag is set instead of waiting for the whole scan.
// With bit planes the scan and the attention can instead run as one kernel,
// fused_planes_kernel (opt-in, MP_PATH_FUSED).
#include <math.h>

#include <algorithm>

#include "mp_common.cuh"
#include "mp_kernels.cuh"
#include "mp_kquant.cuh"
#include "mp_logu.cuh"

namespace mp {

// ------------------------------------------------------------------ qhash ---
// grid (ceil(L / TB), ceil(units / UG)), 256 threads.  A block covers TB =
// 64 / K whole tables (64 or 60 hyperplane columns) for UG units (kv heads of
// sequences); four lanes share a column, each summing 32 of the 128 products
// for all G heads of each unit (one W load serves UG G query vectors), then
// two shuffles finish the sums.
constexpr int kQhashCols = 64;
constexpr int kQhashVecs = 32;  // query vectors a block can stage (UG G)

inline int qhash_tables_per_block(int K) { return kQhashCols / K; }

template <int G>
__global__ void __launch_bounds__(256) qhash_kernel(Shape s, const uint16_t *__restrict__ q,
                                                    const uint16_t *__restrict__ W,
                                                    const uint16_t *__restrict__ qcodes_in,
                                                    uint16_t *__restrict__ qcodes, int32_t *status, int ug,
                                                    int32_t *ready, int nready)
{
    __shared__ float qs[kQhashVecs][kHeadDim + 4];  // element d at d + d / 32: the 4 quarters hit distinct banks
    __shared__ uint8_t bits[kQhashVecs][kQhashCols];
    const int tid = threadIdx.x;
    const int units = s.B * s.Hkv;
    const int u0 = blockIdx.y * ug, nu = min(ug, units - u0);  // units u0 .. u0 + nu - 1
    const int TB = kQhashCols / s.K;
    const int l0 = blockIdx.x * TB;
    const size_t vec0 = (size_t)u0 * G;  // query vectors of a unit are consecutive: (b Hkv + kvh) G + g

    // q and W are never written by this library, and every kernel that reads
    // the query codes of an earlier call has completed before this one starts
    // (see grid_launch_dependents), so the codes are computed and written
    // before the wait for the predecessor; only the status word waits.
    // After the wait: clear the call's status word, the tcgen05 attention's
    // work counter and the scan's per-chunk ready flags (word 15 of each
    // chunk's count record, i < nready), and make the clears visible before
    // the scan may launch: the attention, which starts once every scan block
    // has started, reads the flags without waiting for the scan to finish.
    auto finish = [&]() {
        grid_wait();
        if (status && blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) {
            status[0] = 0;  // the call's status word
            status[1] = 0;  // the attention kernel's work counter
        }
        const int nb = gridDim.x * gridDim.y, bid = blockIdx.y * gridDim.x + blockIdx.x;
        for (int i = bid * blockDim.x + tid; i < nready; i += nb * blockDim.x) ready[(size_t)i * 16 + 15] = 0;
        __threadfence();
        grid_launch_dependents();
    };
    if (qcodes_in) {
        for (int i = tid; i < nu * G * TB; i += blockDim.x) {
            const int v = i / TB, l = l0 + i % TB;
            if (l < s.L) qcodes[(vec0 + v) * s.L + l] = qcodes_in[(vec0 + v) * s.L + l];
        }
        finish();
        return;
    }
    // this lane's W quarter row first: its load overlaps the q staging below
    const int cl = tid >> 2, part = tid & 3;  // column within the block, quarter of the dims
    const int c = l0 * s.K + cl;
    const bool valid = cl < TB * s.K && c < s.LK;
    uint4 w4[4];
    if (valid) {
        const uint4 *wr = reinterpret_cast<const uint4 *>(W + (size_t)c * kHeadDim + part * 32);
#pragma unroll
        for (int j = 0; j < 4; j++) w4[j] = __ldg(wr + j);
    }
    for (int i = tid; i < nu * G * kHeadDim; i += blockDim.x) {
        const int d = i % kHeadDim;
        qs[i / kHeadDim][d + (d >> 5)] = bf16_to_f32(q[(vec0 + i / kHeadDim) * kHeadDim + d]);
    }
    __syncthreads();

    for (int u = 0; u < nu; u++) {
        float acc[G];
#pragma unroll
        for (int g = 0; g < G; g++) acc[g] = 0.f;
        if (valid) {
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const uint32_t wv[4] = {w4[j].x, w4[j].y, w4[j].z, w4[j].w};
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int dd = part * 33 + j * 8 + 2 * e;  // padded index of dim part * 32 + j * 8 + 2 e
                    const float w0 = bf16_lo(wv[e]), w1 = bf16_hi(wv[e]);
#pragma unroll
                    for (int g = 0; g < G; g++) {
                        acc[g] = fmaf(w0, qs[u * G + g][dd], acc[g]);
                        acc[g] = fmaf(w1, qs[u * G + g][dd + 1], acc[g]);
                    }
                }
            }
        }
#pragma unroll
        for (int g = 0; g < G; g++) {
            acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], 1);
            acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], 2);
        }
        if (part == 0) {
#pragma unroll
            for (int g = 0; g < G; g++) bits[u * G + g][cl] = valid && acc[g] > 0.f;
        }
    }
    __syncthreads();
    for (int i = tid; i < nu * G * TB; i += blockDim.x) {
        const int v = i / TB, tl = i % TB, l = l0 + tl;
        if (l < s.L) {
            unsigned code = 0;
            for (int bb = 0; bb < s.K; bb++) code |= (unsigned)bits[v][tl * s.K + bb] << bb;
            qcodes[(vec0 + v) * s.L + l] = (uint16_t)code;
        }
    }
    finish();
}

// Units per query-hash block: the most (up to kQhashVecs / G query vectors)
// that still leave at least two blocks per SM.
static int qhash_units_per_block(const Shape &s, int G)
{
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                      cudaSuccess)
            sms = 148;
    }
    const int TB = qhash_tables_per_block(s.K);
    const long long ntiles = (s.L + TB - 1) / TB, units = (long long)s.B * s.Hkv;
    int ug = 1;
    while (2 * ug * G <= kQhashVecs && ntiles * ((units + 2 * ug - 1) / (2 * ug)) >= 2LL * sms) ug *= 2;
    return ug;
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

// 16-byte read-only load that allocates in L1 (the plane scan touches each
// 32-byte sector with two consecutive loads).
__device__ __forceinline__ uint4 ld_cached_16(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
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

// Candidate list of one chunk by one warp (lane = the WIDTH tokens at t0):
// hm[g] bit i = token t0 + i is in S_g; tokens outside [lo, hi) are masked.
// Entries keep token order (lane, then bit); CHUNK = tokens per list.
template <int G, int WIDTH, int CHUNK>
__device__ __forceinline__ void compact_warp(const Shape &s, int unit, int chunk, int nchunk, int t0, int N, int lo,
                                             int hi, uint32_t (&hm)[G], const ScanOut &o, int lane)
{
    const uint32_t v = range_mask(t0, lo, hi, WIDTH);
    uint32_t any = 0u;
#pragma unroll
    for (int g = 0; g < G; g++) {
        hm[g] &= v;
        any |= hm[g];
    }
    const int mine = __popc(any);
    int incl = mine;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += t;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    int off = incl - mine;
    uint32_t *dst = o.cand + ((size_t)unit * nchunk + chunk) * CHUNK;
    while (any) {
        const int bit = __ffs(any) - 1;
        any &= any - 1u;
        uint32_t heads = 0u;
#pragma unroll
        for (int g = 0; g < G; g++) heads |= ((hm[g] >> bit) & 1u) << g;
        dst[off++] = (uint32_t)(t0 + bit) | (heads << 24);
    }
    int32_t *cnt = o.cnt + ((size_t)unit * nchunk + chunk) * 16;
    if (lane == 0) cnt[0] = total;
#pragma unroll
    for (int g = 0; g < G; g++) {
        int c = __popc(hm[g]);
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) c += __shfl_xor_sync(0xffffffffu, c, d);
        if (lane == 0) cnt[1 + g] = c;
    }
    if (o.member_out) {
        const int b = unit / s.Hkv, kvh = unit % s.Hkv;
        for (int i = 0; i < WIDTH && t0 + i < N; i++)
#pragma unroll
            for (int g = 0; g < G; g++)
                o.member_out[((size_t)b * s.Hq + kvh * G + g) * s.Ncap + t0 + i] = (hm[g] >> i) & 1u;
    }
}

// After a warp has written its chunk's candidate list and counts: every
// lane's writes are made visible, then the chunk's ready flag (word 15 of its
// count record, cleared by the query hash) is released to the attention.
__device__ __forceinline__ void mark_chunk_ready(const ScanOut &o, int unit, int chunk, int nchunk, int lane)
{
    __threadfence();
    __syncwarp();
    if (lane == 0) st_release_gpu(o.cnt + ((size_t)unit * nchunk + chunk) * 16 + 15, 1);
}

// -------------------------------------------------- scan, byte codes (K = 8) ----
// Byte codes [unit][L][Ncap].  A warp owns a 512-token chunk of one unit for
// all L tables (lane = 16 consecutive tokens, one 16-byte streaming load per
// table), so no partial counts ever cross warps; a block is 8 consecutive
// chunks of one unit and shares only the query codes.
//
// Each 16-bit half of a register holds one token's code byte c as the bit
// pattern 0x6000 | c, a normal fp16 number (512 + c/2), so two tokens are
// compared with one packed half compare against the query's 0x6000 | q:
// set.eq.f16x2 yields 1.0 per matching half, and add.f16x2 sums the matches
// per (token, head) exactly (at most L <= 255 < 2048).  Compare and add both
// run on the FMA pipe; the byte split (one lop3 for the even bytes, one prmt
// for the odd bytes of a word) is shared by the G heads.  A token is in S_h
// iff its count reaches 2.
__device__ __forceinline__ uint32_t h2_even_bytes(uint32_t w)  // halves 0x6000 | byte 0, 0x6000 | byte 2
{
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "r"(0x00FF00FFu), "r"(0x60006000u));  // (w & b) | c
    return r;
}
__device__ __forceinline__ uint32_t h2_odd_bytes(uint32_t w)  // halves 0x6000 | byte 1, 0x6000 | byte 3
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, 0x4341;" : "=r"(r) : "r"(w), "r"(0x60606060u));
    return r;
}
__device__ __forceinline__ void h2_count_eq(uint32_t &cnt, uint32_t x, uint32_t q)  // cnt += (x == q) per half
{
    uint32_t m;
    asm("set.eq.f16x2.f16x2 %0, %1, %2;" : "=r"(m) : "r"(x), "r"(q));
    asm("add.rn.f16x2 %0, %0, %1;" : "+r"(cnt) : "r"(m));
}
// Bits 0 and 1 of the result: halves of `cnt` at or above 2.0.
__device__ __forceinline__ uint32_t h2_at_least_2(uint32_t cnt)
{
    uint32_t m;
    asm("set.ge.u32.f16x2 %0, %1, %2;" : "=r"(m) : "r"(cnt), "r"(0x40004000u));  // 0xFFFF per true half (2.0)
    return (m & 1u) | ((m >> 15) & 2u);
}

constexpr int kByteWarps = 8;   // chunks (warps) per block
#ifndef MP_BYTE_RING
#define MP_BYTE_RING 12
#endif
constexpr int kByteRing = MP_BYTE_RING;  // tables in each warp's shared-memory ring (one less in flight)

// Each lane copies its own 16 code bytes of a table into its slot of the
// warp's ring (cp.async, 16 bytes, bypassing L1) and reads back only that
// slot, so the ring needs no barrier: cp.async.wait_group makes a lane's own
// copies visible to it, and a slot is refilled by the same lane only after
// the words read from it have been used (the refill is issued after the
// instructions that consume them).  The query patterns of a table are one
// 16-byte shared load for up to four heads.
template <int G>
#ifndef MP_SCAN_BLOCKS_PER_SM
#define MP_SCAN_BLOCKS_PER_SM 4
#endif
__global__ void __launch_bounds__(32 * kByteWarps, G >= 8 ? 2 : MP_SCAN_BLOCKS_PER_SM) scan_bytes_kernel(
    Shape s, const uint8_t *__restrict__ codes, const uint16_t *__restrict__ qcodes,
    const int32_t *__restrict__ seq_lens, int max_len, int nchunk, ScanOut o)
{
    extern __shared__ __align__(16) uint32_t scan_smem[];  // ring [8 warps][kByteRing][512 B], then qpat [L][GP]
    constexpr int D = kByteRing;
    constexpr int GP = G < 4 ? 4 : G;  // query patterns per table, padded to whole 16-byte loads
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t ring0 = smem_u32(scan_smem) + (uint32_t)(warp * D * kChunkBytes + lane * 16);
    const uint32_t ring_end = ring0 + D * kChunkBytes;
    uint32_t *qpat = scan_smem + kByteWarps * D * kChunkBytes / 4;  // (0x6000 | q) in both halves
    const int unit = blockIdx.y, chunk = blockIdx.x * kByteWarps + warp;
    const int b = unit / s.Hkv, kvh = unit % s.Hkv;
    grid_launch_dependents();
    // lengths and codes come from work before the query hash: read them first
    const int N = clamp_len(seq_lens, b, max_len, o.status, false);
    const bool reporter = blockIdx.x == 0 && kvh == 0 && threadIdx.x == 0;  // of a bad length of sequence b
    if (blockIdx.x * kByteWarps * kChunkBytes >= N) {  // the whole block is past the sequence
        if (reporter) {
            grid_wait();  // the status word is cleared by the query hash
            clamp_len(seq_lens, b, max_len, o.status, true);
        }
        return;
    }
    const int c0 = chunk * kChunkBytes;
    const int t0 = c0 + lane * 16;
    const bool live = c0 < N;  // warp-uniform
    const bool mine = t0 < N;  // lanes past the sequence copy nothing (their counts are masked)
    const uint8_t *src = codes + (size_t)unit * s.L * s.Ncap + t0;
    uint32_t wr = ring0;  // slot of the next copy
    if (live) {
        for (int l = 0; l < D - 1; l++) {
            if (mine && l < s.L) cp_async_16_s(wr, src, 16);
            cp_async_commit();  // one group per table, empty past L, so the group count stays uniform
            src += s.Ncap;
            wr += kChunkBytes;
        }
    }
    grid_wait();  // the query codes are the query hash's output
    if (reporter) clamp_len(seq_lens, b, max_len, o.status, true);
    for (int i = threadIdx.x; i < s.L * GP; i += blockDim.x) {
        const int l = i / GP, g = i % GP;
        qpat[i] = g < G ? ((qcodes[((size_t)b * s.Hq + kvh * G + g) * s.L + l] & 0xFFu) | 0x6000u) * 0x00010001u
                        : 0u;
    }
    __syncthreads();
    if (!live) return;

    // cnt[g][j][0]: tokens 4j and 4j + 2 (even bytes of word j), [1]: 4j + 1, 4j + 3
    uint32_t cnt[G][4][2];
#pragma unroll
    for (int g = 0; g < G; g++)
#pragma unroll
        for (int j = 0; j < 4; j++) cnt[g][j][0] = cnt[g][j][1] = 0u;

    uint32_t rd = ring0;  // slot of table l
    const uint4 *qp = reinterpret_cast<const uint4 *>(qpat);
    for (int l = 0; l < s.L; l++) {
        cp_async_wait<D - 2>();  // table l has landed (groups 0 .. l complete)
        uint4 v;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(rd)
                     : "memory");
        rd = rd + kChunkBytes == ring_end ? ring0 : rd + kChunkBytes;
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t ev[4], od[4];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            ev[j] = h2_even_bytes(w[j]);
            od[j] = h2_odd_bytes(w[j]);
        }
        // the refill of the slot of table l - 1, whose words were used last iteration
        if (mine && l + D - 1 < s.L) cp_async_16_s(wr, src, 16);
        cp_async_commit();
        src += s.Ncap;
        wr = wr + kChunkBytes == ring_end ? ring0 : wr + kChunkBytes;
        uint32_t q[GP];
#pragma unroll
        for (int k = 0; k < GP / 4; k++) {
            const uint4 t = qp[l * (GP / 4) + k];
            q[4 * k] = t.x;
            q[4 * k + 1] = t.y;
            q[4 * k + 2] = t.z;
            q[4 * k + 3] = t.w;
        }
#pragma unroll
        for (int g = 0; g < G; g++)
#pragma unroll
            for (int j = 0; j < 4; j++) {
                h2_count_eq(cnt[g][j][0], ev[j], q[g]);
                h2_count_eq(cnt[g][j][1], od[j], q[g]);
            }
    }
    cp_async_wait<0>();
    // Per-head 16-bit token masks: bit 4j + {0, 1, 2, 3} = tokens of word j.
    uint32_t hm[G];
#pragma unroll
    for (int g = 0; g < G; g++) {
        uint32_t m = 0u;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint32_t e = h2_at_least_2(cnt[g][j][0]), od = h2_at_least_2(cnt[g][j][1]);
            // e: bit 0 = token 4j, bit 1 = token 4j + 2; od: the same for 4j + 1, 4j + 3
            m |= ((e & 1u) | ((od & 1u) << 1) | ((e & 2u) << 1) | ((od & 2u) << 2)) << (4 * j);
        }
        hm[g] = m;
    }
    // Tokens eligible for S: [sink, N - window) and below N.
    compact_warp<G, 16, kChunkBytes>(s, unit, chunk, nchunk, t0, N, s.sink, min(N - s.window, N), hm, o, lane);
    mark_chunk_ready(o, unit, chunk, nchunk, lane);
}

// ---------------------------------------- bit planes: shared TMA pieces ----
// Bit-plane codes [unit][L][Ncap/32][K] (uint32).  The fused scan + attend
// kernel (fused_planes_kernel) brings them in by 3-D TMA copies: a stage is 8
// consecutive tables x one 1024-token chunk's 32 words x K planes (two copies
// for K = 10), tables past L zero-filled; a persistent block walks a
// contiguous share of the live (sequence, kv head, chunk) items.
constexpr int kScanConsumers = 8;  // consumer warps = table splits = tables per stage

template <int KB>
struct PlaneStage {
    static constexpr int kBoxWords = KB == 8 ? 256 : 160;  // inner TMA box (<= 256 elements)
    static constexpr int kBoxes = 32 * KB / kBoxWords;      // 1 or 2 copies per stage
    static constexpr int kBytes = kScanConsumers * 32 * KB * 4;
    static constexpr int kStages = KB == 8 ? 5 : 4;         // ring depth (stages of 8 tables)
};

// Live items of the plane scan: (sequence b, kv head, chunk) with chunk below
// ceil(N_b / chunk), in unit-major order.  Advanced with carries.
struct LiveCursor {
    int b, kvh, chunk, nch, N;
    __device__ __forceinline__ void load_seq(const int32_t *seq_lens, int max_len)
    {
        N = min(max(seq_lens[b], 0), max_len);
        nch = (N + kChunkPlanes - 1) / kChunkPlanes;
    }
    __device__ __forceinline__ void next(const Shape &s, const int32_t *seq_lens, int max_len)
    {
        if (++chunk < nch) return;
        chunk = 0;
        if (++kvh < s.Hkv) return;
        kvh = 0;
        do {
            if (++b >= s.B) return;
            load_seq(seq_lens, max_len);
        } while (nch == 0);
    }
    __device__ __forceinline__ int unit(const Shape &s) const { return b * s.Hkv + kvh; }
};

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y, int z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// Named barriers of the plane scan (0 is __syncthreads):
//   1  the 8 consumer warps (query-mask rewrite)
//   2  consumers arrive, producer waits: an item's split partials are written
//   3  producer arrives, consumers wait: the previous item's partials are read
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap *map, int x, int y, int z)
{
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global [%0, {%1, %2, %3}];" ::"l"(reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z)
                 : "memory");
}


// ------------------------------------------------------ scan, bit planes ----
// The bit-sliced test with the byte scan's structure: a warp owns one
// 1024-token chunk of one unit for all L tables
// (lane = one 32-token word), so no partial count ever crosses warps and no
// block-wide barrier sits in the table loop.  A table's slab of the chunk
// (32 words x K planes, 128 K contiguous bytes) goes through the warp's own
// cp.async ring: the warp copies the slab in 16-byte pieces, lane i taking
// pieces i, i + 32, .. (each copy instruction covers 512 contiguous bytes),
// and a __syncwarp after the wait makes the other lanes' pieces visible.
// Each 128-byte line of the slab stays one 128-byte line in shared memory (a
// copy instruction whose pieces scatter across lines is served twice from L2).
// K = 8: within line j the 16-byte pieces are XOR-swizzled by j & 1, so that
// the two pieces of a word that a quarter warp reads (pieces 2t + i) fall in
// distinct banks; K = 10: the slab is kept as is and lane t reads its 40 bytes
// with five 8-byte loads (a half warp's 8-byte reads at stride 40 hit
// distinct banks).
// Per (table, head): mis = OR_b (plane_b ^ qmask_b), then s2 |= s1 & ~mis,
// s1 |= ~mis; about K + 2 logic ops per 32 tokens.
constexpr int kPlaneWarps = 8;
#ifndef MP_PLANE_RING
#define MP_PLANE_RING 8
#endif
constexpr int kPlaneRing = MP_PLANE_RING;  // tables in each warp's ring (one less in flight)

template <int KB>
__host__ __device__ constexpr int plane_slot_bytes() { return 32 * KB * 4; }

// Shared-memory offset of 16-byte piece p of a K = 8 slab (line p >> 3,
// position swizzled by the line's parity).
__device__ __forceinline__ int plane_piece_k8(int p) { return ((p & ~7) | ((p ^ (p >> 3)) & 1) | (p & 6)) * 16; }

template <int G, int KB>
__global__ void __launch_bounds__(32 * kPlaneWarps) scan_planes_warp_kernel(
    Shape s, const uint32_t *__restrict__ codes, const uint16_t *__restrict__ qcodes,
    const int32_t *__restrict__ seq_lens, int max_len, int nchunk, ScanOut o)
{
    constexpr int D = kPlaneRing;
    constexpr int SLOT = plane_slot_bytes<KB>();
    constexpr int PIECES = SLOT / 16;  // 64 (K = 8) or 80 (K = 10)
    constexpr int QW = (KB + 3) & ~3;  // query masks per (table, head), padded to whole uint4s
    constexpr bool kPair = KB == 8;    // a word's planes are two 16-byte pieces
    extern __shared__ __align__(16) uint32_t pw_smem[];  // ring [warps][D][SLOT], then qm [L][G][QW]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *ring = reinterpret_cast<uint8_t *>(pw_smem) + warp * D * SLOT;
    uint32_t *qm = pw_smem + kPlaneWarps * D * SLOT / 4;
    const int unit = blockIdx.y, chunk = blockIdx.x * kPlaneWarps + warp;
    const int b = unit / s.Hkv, kvh = unit % s.Hkv;
    grid_launch_dependents();
    // lengths and codes come from work before the query hash: read them first
    const int N = clamp_len(seq_lens, b, max_len, o.status, false);
    const bool reporter = blockIdx.x == 0 && kvh == 0 && threadIdx.x == 0;  // of a bad length of sequence b
    if (blockIdx.x * kPlaneWarps * kChunkPlanes >= N) {  // the whole block is past the sequence
        if (reporter) {
            grid_wait();  // the status word is cleared by the query hash
            clamp_len(seq_lens, b, max_len, o.status, true);
        }
        return;
    }
    const int c0 = chunk * kChunkPlanes;
    const bool live = c0 < N;  // warp-uniform
    // words of this chunk that hold live tokens (the rest are zero-filled)
    const int words = s.Ncap >> 5;
    const int vw = live ? min(32, (N + 31) / 32 - chunk * 32) : 0;
    const int vbytes = vw * KB * 4;
    const uint8_t *src = reinterpret_cast<const uint8_t *>(codes) +
                         (((size_t)unit * s.L * words + (size_t)chunk * 32) * KB) * 4;
    const size_t tstride = (size_t)words * KB * 4;  // bytes between tables
    auto copy_table = [&](int slot, const uint8_t *g) {
        uint8_t *dst = ring + slot * SLOT;
#pragma unroll
        for (int i = 0; i < (PIECES + 31) / 32; i++) {
            const int p = lane + 32 * i;  // piece = 16 bytes of the slab
            if (p < PIECES) {
                const int nb = min(max(vbytes - p * 16, 0), 16);  // zero-fill past the live words
                cp_async_16(dst + (kPair ? plane_piece_k8(p) : p * 16), g + (nb ? p * 16 : 0), nb);
            }
        }
    };
    if (live) {
        for (int l = 0; l < D - 1; l++) {
            if (l < s.L) copy_table(l, src + l * tstride);
            cp_async_commit();  // one group per table, empty past L, so the group count stays uniform
        }
    }
    grid_wait();  // the query codes are the query hash's output
    if (reporter) clamp_len(seq_lens, b, max_len, o.status, true);
    for (int i = threadIdx.x; i < s.L * G; i += blockDim.x) {
        const int l = i / G, g = i % G;
        const unsigned code = qcodes[((size_t)b * s.Hq + kvh * G + g) * s.L + l];
        uint4 *dst = reinterpret_cast<uint4 *>(qm + (size_t)i * QW);
#pragma unroll
        for (int q = 0; q < QW / 4; q++) {
            uint32_t m[4];
#pragma unroll
            for (int x = 0; x < 4; x++) m[x] = 4 * q + x < KB ? 0u - ((code >> (4 * q + x)) & 1u) : 0u;
            dst[q] = make_uint4(m[0], m[1], m[2], m[3]);
        }
    }
    __syncthreads();
    if (!live) return;

    uint32_t s1[G], s2[G];
#pragma unroll
    for (int g = 0; g < G; g++) s1[g] = s2[g] = 0u;
    int rs = 0;  // slot of table l
    for (int l = 0; l < s.L; l++) {
        cp_async_wait<D - 2>();  // table l has landed (groups 0 .. l complete)
        __syncwarp();            // ... for every lane's pieces; and every lane is done with table l - 1
        uint32_t pw[KB];
        const uint8_t *rp = ring + rs * SLOT;
        if constexpr (kPair) {
#pragma unroll
            for (int i = 0; i < 2; i++) {
                const uint4 v = *reinterpret_cast<const uint4 *>(rp + plane_piece_k8(2 * lane + i));
                pw[4 * i] = v.x;
                pw[4 * i + 1] = v.y;
                pw[4 * i + 2] = v.z;
                pw[4 * i + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < KB / 2; i++) {
                const uint2 v = *reinterpret_cast<const uint2 *>(rp + lane * KB * 4 + i * 8);
                pw[2 * i] = v.x;
                pw[2 * i + 1] = v.y;
            }
        }
        // refill the slot of table l - 1 (every lane has used it) with table l + D - 1
        const int ws_ = rs == 0 ? D - 1 : rs - 1;
        if (l + D - 1 < s.L) copy_table(ws_, src + (size_t)(l + D - 1) * tstride);
        cp_async_commit();
        rs = rs + 1 == D ? 0 : rs + 1;
#pragma unroll
        for (int g = 0; g < G; g++) {
            const uint4 *m4 = reinterpret_cast<const uint4 *>(qm + (l * G + g) * QW);
            uint32_t mis = 0u;
#pragma unroll
            for (int q = 0; q < QW / 4; q++) {
                const uint4 mq = m4[q];
                const uint32_t mm[4] = {mq.x, mq.y, mq.z, mq.w};
#pragma unroll
                for (int x = 0; x < 4; x++)
                    if (4 * q + x < KB) mis |= pw[4 * q + x] ^ mm[x];
            }
            s2[g] |= s1[g] & ~mis;
            s1[g] |= ~mis;
        }
    }
    cp_async_wait<0>();
    // Tokens eligible for S: [sink, N - window) and below N.
    compact_warp<G, 32, kChunkPlanes>(s, unit, chunk, nchunk, c0 + lane * 32, N, s.sink, min(N - s.window, N), s2, o,
                                      lane);
    mark_chunk_ready(o, unit, chunk, nchunk, lane);
}

// ---------------------------------------------------------------- attend ----
constexpr int kAttThreads = 128;
constexpr int kMaxSpan = 64;                // scan chunks per attention block, at most
constexpr int kAttRows = 64;                // rows per tile (4 warps x 16)
constexpr int kAttStages = 2;               // cp.async ring depth (3 blocks fit per SM)
constexpr int kRowBytes = kHeadDim * 2;     // 256
// K / V rows in shared memory are unpadded; within each 128-byte line the
// 16-byte pieces are XOR-swizzled by row & 7 (att_piece), so that a global
// line lands in one shared line (a copy whose pieces straddle shared lines is
// fetched from L2 twice) and the 8 rows an ldmatrix reads hit distinct banks.
constexpr int kRowStride = kRowBytes;
constexpr int kStageBytes = kAttRows * kRowStride * 2;  // K rows then V rows
// int8 keys (mp_decode_attend_q8): 128-byte rows
constexpr int kRowStrideQ8 = kHeadDim;
template <bool Q8>
constexpr int att_k_stride() { return Q8 ? kRowStrideQ8 : kRowStride; }
template <bool Q8>
constexpr int att_stage_bytes() { return kAttRows * (att_k_stride<Q8>() + kRowStride); }

// Byte offset of 16-byte piece c of row `row` within the row.
__device__ __forceinline__ int att_piece(int row, int c) { return (c ^ (row & 7)) << 4; }

struct AttendArgs {
    Shape s;
    const uint16_t *q;
    const uint16_t *kc;
    const uint16_t *vc;
    const int32_t *seq_lens;
    int max_len;
    int nchunk;
    int span;   // scan chunks per attention block (their candidate lists are concatenated)
    int subs;   // blocks per span (each takes an equal share of the span's candidates)
    int ngroups;  // ceil(nchunk / span)
    int chunk_tokens;
    const uint32_t *cand;
    const int32_t *cnt;
    float *pm, *pl, *pacc;  // [B*Hq][ngroups*subs+1], [..][..][128]
    LogU lu;
    float scale;  // 1/sqrt(d)
    const int8_t *k8;      // int8 key rows [B][Hkv][Ncap][kQ8RowBytes] (attend_kernel<G, true>), else null
    int32_t *status;       // the call's status word (a ready flag that never came: MP_ERR_CUDA)
};

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3,
                                                  const void *smem_row)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(smem_row)));
}

// Transposes an 8x8 b16 matrix held one row-pair per thread (mma fragment layout).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x)
{
    uint32_t r;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(r) : "r"(x));
    return r;
}

__device__ __forceinline__ void ldmatrix_x2(uint32_t &r0, uint32_t &r1, const void *smem_row)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n"
                 : "=r"(r0), "=r"(r1)
                 : "r"(smem_u32(smem_row)));
}

// D(16x8, fp32) += A(16x16, f16, row) * B(16x8, f16, col)
__device__ __forceinline__ void mma_f16_16816(float &d0, float &d1, float &d2, float &d3, uint32_t a0, uint32_t a1,
                                              uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d0), "+f"(d1), "+f"(d2), "+f"(d3)
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four int8 values (bytes of r) -> two f16x2, exactly: byte b becomes the half
// 0x6400 | (b ^ 0x80), i.e. 1024 + b + 128, and 1152 is subtracted.
__device__ __forceinline__ void s8x4_to_f16x2(uint32_t r, uint32_t &lo, uint32_t &hi)
{
    const uint32_t x = r ^ 0x80808080u;
    asm("prmt.b32 %0, %1, %2, 0x4140;" : "=r"(lo) : "r"(x), "r"(0x64646464u));  // bytes 0, 1
    asm("prmt.b32 %0, %1, %2, 0x4342;" : "=r"(hi) : "r"(x), "r"(0x64646464u));  // bytes 2, 3
    asm("add.rn.f16x2 %0, %0, %1;" : "+r"(lo) : "r"(0xE480E480u));                // - 1152
    asm("add.rn.f16x2 %0, %0, %1;" : "+r"(hi) : "r"(0xE480E480u));
}

// {lo, hi} -> f16x2 (round to nearest even), lo in the low half.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// {lo, hi} -> bf16x2 (round to nearest even), lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// One block = 4 warps; a warp owns 16 rows of every 64-row tile.
//   scores  S^T (16 rows x 8 heads) = K rows . Q^T with bf16 mma.sync, fp32 acc;
//           |k|^2 from the same A fragments.  Lane (g, t) holds rows g, g+8 for
//           heads 2t, 2t+1 and keeps the online-softmax state of those heads.
//   log u   only for the (row, head) pairs that are sampled, compacted per warp.
//   P.V     O^T (128 dims x 8 heads) += V^T . P^T on the tensor cores: P is
//           split into bf16 hi + lo parts (error ~2^-17 relative), transposed
//           into B fragments with movmatrix, V^T comes from ldmatrix.trans.
// 2^x with the MUFU approximation (relative error about 2^-22; flushes
// subnormal results to zero).  The attention's log-weights are kept in base 2:
// s log2(e) and log2 u, so each weight is a single ex2.
__device__ __forceinline__ float fast_exp2(float x)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Attention state of one warp of a 4-warp (128-thread) group: the warp owns
// 16 rows of every 64-row tile.  Lane (g, t) holds rows g, g + 8 for heads
// 2t, 2t + 1, the B fragments of Q^T, those heads' online-softmax state (m, l)
// and O^T fragments acc[mt] (dims 16 mt + g and 16 mt + g + 8).
template <int G>
struct AttnWarp {
    uint32_t qb[8][2];
    float qi0, qi1;  // 1/|q| of heads 2t, 2t + 1
    float m0, m1, l0, l1;
    float acc[8][4];
};

// Loads the Q^T fragments of the G heads starting at query vector vec0 and
// clears the state (the 1/|q| values come later, from attn_qinv's shared array).
// With int8 keys (Q8) the fragments are f16 and follow the keys' dimension
// order inside each 16-dim step (see attn_tile): slots 2t, 2t + 1, 2t + 8,
// 2t + 9 of step ks hold dims 16 ks + 4t .. 16 ks + 4t + 3.
template <int G, bool Q8 = false>
__device__ __forceinline__ void attn_begin(AttnWarp<G> &w, const uint16_t *q, size_t vec0, int lane)
{
    const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 8; ks++) {
        if (gq < G) {
            if constexpr (Q8) {
                const uint16_t *qp = q + (vec0 + gq) * kHeadDim + ks * 16 + 4 * tq;
                w.qb[ks][0] = pack_f16x2(bf16_to_f32(qp[0]), bf16_to_f32(qp[1]));
                w.qb[ks][1] = pack_f16x2(bf16_to_f32(qp[2]), bf16_to_f32(qp[3]));
            } else {
                const uint32_t *qp = reinterpret_cast<const uint32_t *>(q + (vec0 + gq) * kHeadDim);
                w.qb[ks][0] = qp[(ks * 16 + 2 * tq) >> 1];
                w.qb[ks][1] = qp[(ks * 16 + 2 * tq + 8) >> 1];
            }
        } else {
            w.qb[ks][0] = w.qb[ks][1] = 0u;
        }
    }
    w.m0 = w.m1 = -INFINITY;
    w.l0 = w.l1 = 0.f;
#pragma unroll
    for (int mt = 0; mt < 8; mt++)
#pragma unroll
        for (int e = 0; e < 4; e++) w.acc[mt][e] = 0.f;
}

// 1/|q_h| of the G heads into qinv[G] (warp `warp` of a 4-warp group).
template <int G>
__device__ __forceinline__ void attn_qinv(const uint16_t *q, size_t vec0, int warp, int lane, float *qinv)
{
    for (int h = warp; h < G; h += 4) {
        const uint2 qv = reinterpret_cast<const uint2 *>(q + (vec0 + h) * kHeadDim)[lane];
        float x0 = bf16_lo(qv.x), x1 = bf16_hi(qv.x), x2 = bf16_lo(qv.y), x3 = bf16_hi(qv.y);
        float qq = x0 * x0 + x1 * x1 + x2 * x2 + x3 * x3;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) qq += __shfl_xor_sync(0xffffffffu, qq, o);
        if (lane == 0) qinv[h] = qq > 0.f ? rsqrtf(qq) : 0.f;
    }
}

template <int G>
__device__ __forceinline__ void attn_set_qinv(AttnWarp<G> &w, const float *qinv, int lane)
{
    const int h0 = 2 * (lane & 3), h1 = h0 + 1;
    w.qi0 = h0 < G ? qinv[h0] : 0.f;
    w.qi1 = h1 < G ? qinv[h1] : 0.f;
}

// One 64-row tile for this warp: its 16 K rows at ks_ and V rows at vs_
// (kRowStride apart, the tile's rows 16 warp ..), meta[64] = the rows' head
// masks (| 0x100 for the exact set); ucos / uval are this warp's [16 G] scratch.
//
// With int8 keys (Q8): K rows are 128 bytes (kRowStrideQ8 apart) and kq
// holds the 16 rows' {scale, squared norm} records.  One ldmatrix.x2 per
// 16-dim step gives lane (g, t) the bytes of dims 4t .. 4t + 3 of rows g and
// g + 8; widened exactly to f16 they fill fragment slots 2t, 2t + 1, 2t + 8,
// 2t + 9, a fixed permutation of the step's dims that the query fragments
// follow too (attn_begin), so the dot products are unchanged.  Scores are
// scaled by the row's scale; |k|^2 is the stored norm (no Gram products).
template <int G, bool Q8 = false>
__device__ __forceinline__ void attn_tile(AttnWarp<G> &w, const uint8_t *ks_, const uint8_t *vs_,
                                          const uint32_t *meta, int warp, int lane, float scale, const LogU &lu,
                                          float *ucos, float *uval, const float4 *kq = nullptr)
{
    const float scale2 = scale * kLog2e;  // scores in log2 units
    const int gq = lane >> 2, tq = lane & 3;
    const int h0 = 2 * tq, h1 = 2 * tq + 1;
    // ---- S^T = K rows . Q^T and |k|^2 ----
    // The A fragments of K double as B fragments of K^T, so two more MMAs
    // per k-step give the 16x16 Gram matrix K K^T, whose diagonal is |k|^2.
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    float na, nb;
    {
        if constexpr (Q8) {
            const uint8_t *arow = ks_ + (warp * 16 + (lane & 15)) * kRowStrideQ8;
            const int r7 = lane & 7;  // the row's swizzle
#pragma unroll
            for (int kst = 0; kst < 8; kst++) {
                uint32_t r0, r1, a0, a1, a2, a3;
                ldmatrix_x2(r0, r1, arow + ((kst ^ r7) << 4));
                s8x4_to_f16x2(r0, a0, a2);
                s8x4_to_f16x2(r1, a1, a3);
                mma_f16_16816(c[0], c[1], c[2], c[3], a0, a1, a2, a3, w.qb[kst][0], w.qb[kst][1]);
            }
            const float4 m0 = kq[warp * 16 + gq], m1 = kq[warp * 16 + gq + 8];
            c[0] *= m0.x;
            c[1] *= m0.x;
            c[2] *= m1.x;
            c[3] *= m1.x;
            na = m0.y;
            nb = m1.y;
        } else {
            float g0[4] = {0.f, 0.f, 0.f, 0.f}, g1[4] = {0.f, 0.f, 0.f, 0.f};
            // piece 2 kst + (lane >> 4) of row lane & 15, swizzled by lane & 7
            const uint8_t *arow = ks_ + (warp * 16 + (lane & 15)) * kRowStride;
            const int sw = (lane >> 4) ^ (lane & 7);
#pragma unroll
            for (int kst = 0; kst < 8; kst++) {
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4(a0, a1, a2, a3, arow + (((2 * kst) ^ sw) << 4));
                mma_bf16_16816(c[0], c[1], c[2], c[3], a0, a1, a2, a3, w.qb[kst][0], w.qb[kst][1]);
                mma_bf16_16816(g0[0], g0[1], g0[2], g0[3], a0, a1, a2, a3, a0, a2);  // columns: rows 0-7
                mma_bf16_16816(g1[0], g1[1], g1[2], g1[3], a0, a1, a2, a3, a1, a3);  // columns: rows 8-15
            }
            // |k_r|^2 = Gram[r][r]: row gq sits in lane 4 gq + gq/2 (g0, element gq & 1),
            // row gq + 8 in the same lane (g1, element 2 + (gq & 1)).
            const int src = 4 * gq + (gq >> 1);
            const float d0 = (gq & 1) ? g0[1] : g0[0];
            const float d1 = (gq & 1) ? g1[3] : g1[2];
            na = __shfl_sync(0xffffffffu, d0, src);
            nb = __shfl_sync(0xffffffffu, d1, src);
        }
    }

    // ---- log-weights: s (exact) or s - log u (sampled), -inf if absent ----
    const uint32_t mg = meta[warp * 16 + gq], mg8 = meta[warp * 16 + gq + 8];
    float tv[4];
    bool need[4];
    int pos[4];
    {
        const uint32_t mrow[4] = {mg, mg, mg8, mg8};
        const int hh[4] = {h0, h1, h0, h1};
        const float kinv_g = na > 0.f ? rsqrtf(na) : 0.f, kinv_g8 = nb > 0.f ? rsqrtf(nb) : 0.f;
        const float kin[4] = {kinv_g, kinv_g, kinv_g8, kinv_g8};
        const float qin[4] = {w.qi0, w.qi1, w.qi0, w.qi1};
        int base = 0;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const bool mem = hh[j] < G && ((mrow[j] >> hh[j]) & 1u);
            need[j] = mem && !(mrow[j] & 0x100u);
            tv[j] = mem ? c[j] * scale2 : -INFINITY;
            const uint32_t bal = __ballot_sync(0xffffffffu, need[j]);
            pos[j] = base + __popc(bal & ((1u << lane) - 1u));
            if (need[j]) ucos[pos[j]] = c[j] * qin[j] * kin[j];
            base += __popc(bal);
        }
        __syncwarp();
        for (int i = lane; i < base; i += 32) uval[i] = log_sampling_prob(ucos[i], lu);
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 4; j++)
            if (need[j]) tv[j] = fmaf(-kLog2e, uval[pos[j]], tv[j]);  // - log2 u
    }

    // ---- online softmax over this warp's rows (lanes with equal t share heads) ----
    float mt0 = fmaxf(tv[0], tv[2]), mt1 = fmaxf(tv[1], tv[3]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        mt0 = fmaxf(mt0, __shfl_xor_sync(0xffffffffu, mt0, o));
        mt1 = fmaxf(mt1, __shfl_xor_sync(0xffffffffu, mt1, o));
    }
    // (log2 units; a running max that stays -inf keeps weights and scale at 0 / 1)
    const float mn0 = fmaxf(w.m0, mt0), mn1 = fmaxf(w.m1, mt1);
    const float b0 = mn0 == -INFINITY ? 0.f : mn0, b1 = mn1 == -INFINITY ? 0.f : mn1;
    float p[4];
    p[0] = fast_exp2(tv[0] - b0);  // tv = -inf -> 0
    p[1] = fast_exp2(tv[1] - b1);
    p[2] = fast_exp2(tv[2] - b0);
    p[3] = fast_exp2(tv[3] - b1);
    if (__any_sync(0xffffffffu, mn0 != w.m0 || mn1 != w.m1)) {
        // some head's maximum moved: rescale its running sum and accumulators
        const float al0 = fast_exp2(w.m0 - b0), al1 = fast_exp2(w.m1 - b1);
        w.l0 *= al0;
        w.l1 *= al1;
#pragma unroll
        for (int mt = 0; mt < 8; mt++) {
            w.acc[mt][0] *= al0;
            w.acc[mt][1] *= al1;
            w.acc[mt][2] *= al0;
            w.acc[mt][3] *= al1;
        }
    }
    w.l0 += p[0] + p[2];
    w.l1 += p[1] + p[3];
    w.m0 = mn0;
    w.m1 = mn1;

    // ---- O^T += V^T . P^T (P split into bf16 hi + lo) ----
    const uint32_t hi_g = pack_bf16x2(p[0], p[1]), hi_g8 = pack_bf16x2(p[2], p[3]);
    const uint32_t lo_g = pack_bf16x2(p[0] - bf16_lo(hi_g), p[1] - bf16_hi(hi_g));
    const uint32_t lo_g8 = pack_bf16x2(p[2] - bf16_lo(hi_g8), p[3] - bf16_hi(hi_g8));
    const uint32_t bh0 = movmatrix_trans(hi_g), bh1 = movmatrix_trans(hi_g8);
    const uint32_t bl0 = movmatrix_trans(lo_g), bl1 = movmatrix_trans(lo_g8);
    {
        // piece 2 mt + (mrow & 1) of row 8 (mrow >> 1) + (lane & 7), swizzled by lane & 7
        const int mrow = lane >> 3;
        const uint8_t *vrow = vs_ + (warp * 16 + (mrow >> 1) * 8 + (lane & 7)) * kRowStride;
        const int sw = (mrow & 1) ^ (lane & 7);
#pragma unroll
        for (int mt = 0; mt < 8; mt++) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4_trans(a0, a1, a2, a3, vrow + (((2 * mt) ^ sw) << 4));
            mma_bf16_16816(w.acc[mt][0], w.acc[mt][1], w.acc[mt][2], w.acc[mt][3], a0, a1, a2, a3, bh0, bh1);
            mma_bf16_16816(w.acc[mt][0], w.acc[mt][1], w.acc[mt][2], w.acc[mt][3], a0, a1, a2, a3, bl0, bl1);
        }
    }
}

// Folds the 4 warps' states of a group (red: shared [4 G 128 + 8 G] floats,
// free for the group; bar(): the group's barrier) and writes one partial per
// head: m, l at pm/pl[(vec0 + g) nsplit + split], acc at pacc[..][128].  The
// caller keeps `red` untouched by other warps until bar() is passed again.
template <int G, typename Bar>
__device__ __forceinline__ void attn_store_partial(AttnWarp<G> &w, float *red, int warp, int lane, int tid, Bar bar,
                                                   size_t vec0, size_t nsplit, int split, float *pm, float *pl,
                                                   float *pacc)
{
    const int gq = lane >> 2, tq = lane & 3;
    const int h0 = 2 * tq, h1 = 2 * tq + 1;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        w.l0 += __shfl_xor_sync(0xffffffffu, w.l0, o);
        w.l1 += __shfl_xor_sync(0xffffffffu, w.l1, o);
    }
    float *redm = red + 4 * G * kHeadDim;
    float *redl = redm + 4 * G;
#pragma unroll
    for (int mt = 0; mt < 8; mt++) {
        if (h0 < G) {
            red[(warp * G + h0) * kHeadDim + mt * 16 + gq] = w.acc[mt][0];
            red[(warp * G + h0) * kHeadDim + mt * 16 + gq + 8] = w.acc[mt][2];
        }
        if (h1 < G) {
            red[(warp * G + h1) * kHeadDim + mt * 16 + gq] = w.acc[mt][1];
            red[(warp * G + h1) * kHeadDim + mt * 16 + gq + 8] = w.acc[mt][3];
        }
    }
    if (gq == 0) {
        if (h0 < G) {
            redm[warp * G + h0] = w.m0;
            redl[warp * G + h0] = w.l0;
        }
        if (h1 < G) {
            redm[warp * G + h1] = w.m1;
            redl[warp * G + h1] = w.l1;
        }
    }
    bar();
    const int dim = tid;  // 128 threads = head_dim
    for (int g = 0; g < G; g++) {
        float M = -INFINITY;
        for (int w = 0; w < 4; w++) M = fmaxf(M, redm[w * G + g]);
        float Ls = 0.f, A = 0.f;
        if (M != -INFINITY) {
            for (int w = 0; w < 4; w++) {
                const float mw = redm[w * G + g];
                if (mw == -INFINITY) continue;
                const float f = fast_exp2(mw - M);
                Ls += redl[w * G + g] * f;
                A += red[(w * G + g) * kHeadDim + dim] * f;
            }
        }
        const size_t bh = vec0 + g;
        const size_t pidx = bh * nsplit + split;
        pacc[pidx * kHeadDim + dim] = A;
        if (dim == 0) {
            pm[pidx] = M;
            pl[pidx] = Ls;
        }
    }
}

template <int G, bool Q8>
__global__ void __launch_bounds__(kAttThreads, 3) attend_kernel(AttendArgs a)
{
    extern __shared__ __align__(16) uint8_t smem[];
    constexpr int kWarpRows = kAttRows / 4;                   // rows of a tile per warp
    constexpr int KS = att_k_stride<Q8>();                    // K row stride in shared memory
    constexpr int kWarpStage = kWarpRows * (KS + kRowStride); // one warp's K rows then V rows
    __shared__ uint32_t meta[4][kAttStages][kWarpRows];       // per warp: headmask | exact << 8
    __shared__ float4 kq[Q8 ? 4 : 1][Q8 ? kAttStages : 1][kWarpRows];  // int8 keys: {scale, |k|^2} per row
    __shared__ float ucos[4][16 * G];                // per warp: cos of pairs needing log u
    __shared__ float uval[4][16 * G];                // per warp: their log u
    __shared__ float qinv[G];

    const Shape &s = a.s;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int unit = blockIdx.y, split = blockIdx.x;
    const int b = unit / s.Hkv, kvh = unit % s.Hkv;
    const bool dsplit = split == a.ngroups * a.subs;
    const int grp = split / a.subs, sub = split % a.subs;
    const int c_begin = grp * a.span;
    const uint32_t *lists = a.cand + ((size_t)unit * a.nchunk + c_begin) * a.chunk_tokens;
    // This kernel starts once every block of the scan has started, so all
    // work before the scan (the append's rows and lengths) is complete and
    // visible; the scan's own output is not waited for as a whole: a block
    // waits only for the ready flags of the chunks it reads (the exact-set
    // block reads none), and then lets the merge launch.  Blocks of early
    // units thus run beside the scan's last blocks.
    int N = a.seq_lens[b];
    N = N < 0 ? 0 : (N > a.max_len ? a.max_len : N);
    const int nch = (N + a.chunk_tokens - 1) / a.chunk_tokens;
    if (!dsplit && c_begin >= nch) return;
    if (!dsplit) {
        __shared__ int flags_ok;
        if (tid == 0) {
            const int c_end = min(c_begin + a.span, nch);
            bool ok = true;
            for (int c = c_begin; c < c_end && ok; c++)
                ok = flag_wait_bounded(a.cnt + ((size_t)unit * a.nchunk + c) * 16 + 15);
            if (!ok) set_status(a.status, MP_ERR_CUDA);
            flags_ok = ok;
        }
        __syncthreads();
        if (!flags_ok) return;  // a list that never became ready is not read
    }
    grid_launch_dependents();
    // A block that takes one chunk's whole list (span = subs = 1) reads the
    // list's count and the first two tiles' entries together: none of these
    // loads waits for another (entries past the count are dropped below; they
    // stay inside the chunk's list).
    const bool direct = !dsplit && a.span == 1 && a.subs == 1;
    int dcount = 0;
    uint32_t pre0 = 0xFFFFFFFFu, pre1 = 0xFFFFFFFFu;
    if (direct) {
        if (tid == 0) dcount = a.cnt[((size_t)unit * a.nchunk + c_begin) * 16];
        if (lane < kWarpRows) {  // the warp's rows of tiles 0 and 1
            pre0 = lists[warp * kWarpRows + lane];
            pre1 = lists[kAttRows + warp * kWarpRows + lane];
        }
    }

    // Rows of this block: its share of the concatenated candidate lists of
    // chunks [c_begin, c_end), or the exact set D.
    __shared__ int cpre[kMaxSpan + 1];  // prefix sums of the chunks' candidate counts
    const int n_sink = min(s.sink, N);
    const int win0 = max(n_sink, N - s.window);
    const int nc = dsplit ? 0 : min(a.span, nch - c_begin);
    int nrows, e0 = 0;
    if (dsplit) {
        nrows = n_sink + (N - win0);
    } else {
        if (direct) {
            if (tid == 0) {
                cpre[0] = 0;
                cpre[1] = dcount;
            }
        } else if (warp == 0) {
            int run = 0;
            for (int j0 = 0; j0 < nc; j0 += 32) {
                const int j = j0 + lane;
                const int v = j < nc ? a.cnt[((size_t)unit * a.nchunk + c_begin + j) * 16] : 0;
                int incl = v;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += t;
                }
                if (j < nc) cpre[j + 1] = run + incl;
                run += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) cpre[0] = 0;
        }
        __syncthreads();
        const int total = cpre[nc];
        const int per = (total + a.subs - 1) / a.subs;
        e0 = min(total, sub * per);
        nrows = min(total, e0 + per) - e0;
    }
    const uint32_t dmeta = ((1u << G) - 1u) | 0x100u;

    const size_t vec0 = (size_t)b * s.Hq + (size_t)kvh * G;
    AttnWarp<G> w;
    attn_begin<G, Q8>(w, a.q, vec0, lane);
    attn_qinv<G>(a.q, vec0, warp, lane, qinv);

    const uint16_t *kbase = Q8 ? nullptr : a.kc + (size_t)unit * s.Ncap * kHeadDim;
    const int8_t *k8base = Q8 ? a.k8 + (size_t)unit * s.Ncap * kQ8RowBytes : nullptr;
    const uint16_t *vbase = a.vc + (size_t)unit * s.Ncap * kHeadDim;
    const int ntiles = (nrows + kAttRows - 1) / kAttRows;

    // Each warp owns rows 16 warp .. 16 warp + 15 of every 64-row tile and runs
    // its own entry ring and 2-stage cp.async ring, so the warps of a block
    // meet only at the start (span prefix, q norms) and at the end (merge of
    // their states), never per tile.  Lanes 0..15 read the entries of the
    // warp's rows two tiles ahead (the load overlaps the current tile's
    // arithmetic) into a 2-slot ring; the copy issue reads its rows there.
    static_assert(kAttStages == 2, "entry ring sized for one tile of copies in flight");
    __shared__ uint32_t ents[4][2][kWarpRows];
    uint8_t *wring = smem + warp * (kAttStages * kWarpStage);
    int jc = 0;  // chunk of this lane's next candidate (rows are visited in increasing order)
    auto fetch1 = [&](int tile) -> uint32_t {
        const int e = tile * kAttRows + warp * kWarpRows + lane;
        if (e >= nrows) return 0xFFFFFFFFu;
        if (dsplit) return (uint32_t)(e < n_sink ? e : win0 + (e - n_sink));
        const int r = e0 + e;
        while (cpre[jc + 1] <= r) jc++;
        return lists[(size_t)jc * a.chunk_tokens + (r - cpre[jc])];
    };

    auto issue = [&](int tile, int stage) {
        uint8_t *ks_ = wring + stage * kWarpStage;
        uint8_t *vs_ = ks_ + kWarpRows * KS;
        const int col = lane & 15;
#pragma unroll
        for (int i = 0; i < kWarpRows / 2; i++) {
            const int r = (lane >> 4) + 2 * i;
            const uint32_t ent = ents[warp][tile & 1][r];
            const bool ok = ent != 0xFFFFFFFFu;
            const int tok = ok ? (int)(ent & 0xFFFFFFu) : 0;
            const size_t off = (size_t)tok * kHeadDim + col * 8;
            if constexpr (Q8) {  // the 9 pieces of the 144-byte row: 8 of values, then the record
                if (col < 9) {
                    void *dst = col < 8 ? (void *)(ks_ + r * KS + att_piece(r, col)) : (void *)&kq[warp][stage][r];
                    cp_async_16(dst, k8base + (size_t)tok * kQ8RowBytes + col * 16, ok ? 16 : 0);
                }
            } else {
                cp_async_16(ks_ + r * KS + att_piece(r, col), kbase + off, ok ? 16 : 0);
            }
            cp_async_16(vs_ + r * kRowStride + att_piece(r, col), vbase + off, ok ? 16 : 0);
            if (col == 0) meta[warp][stage][r] = ok ? (dsplit ? dmeta : (ent >> 24)) : 0u;
        }
    };

    if (lane < kWarpRows) {
        if (direct) {
            ents[warp][0][lane] = warp * kWarpRows + lane < nrows ? pre0 : 0xFFFFFFFFu;
            ents[warp][1][lane] = kAttRows + warp * kWarpRows + lane < nrows ? pre1 : 0xFFFFFFFFu;
        } else {
            if (ntiles > 0) ents[warp][0][lane] = fetch1(0);
            if (ntiles > 1) ents[warp][1][lane] = fetch1(1);
        }
    }
    __syncthreads();  // qinv (and this warp's entries of tiles 0 and 1)
    if (ntiles > 0) issue(0, 0);
    cp_async_commit();
    attn_set_qinv<G>(w, qinv, lane);

    for (int tile = 0; tile < ntiles; tile++) {
        if (tile + 1 < ntiles) issue(tile + 1, (tile + 1) % kAttStages);
        cp_async_commit();
        const bool fetcher = lane < kWarpRows && tile + 2 < ntiles;
        const uint32_t pend = fetcher ? fetch1(tile + 2) : 0u;
        cp_async_wait<kAttStages - 1>();
        __syncwarp();
        const int stage = tile % kAttStages;
        const uint8_t *ks_ = wring + stage * kWarpStage;
        // the warp's own 16 rows, addressed as warp 0 of a tile
        attn_tile<G, Q8>(w, ks_, ks_ + kWarpRows * KS, meta[warp][stage], 0, lane, a.scale, a.lu, ucos[warp],
                         uval[warp], kq[Q8 ? warp : 0][Q8 ? stage : 0]);
        if (fetcher) ents[warp][tile & 1][lane] = pend;  // slot of tile + 2, read after the next __syncwarp
        __syncwarp();  // the stage may be refilled next iteration
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---- merge the 4 warps' states, write this split's partial ----
    attn_store_partial<G>(w, reinterpret_cast<float *>(smem), warp, lane, tid, [] { __syncthreads(); }, vec0,
                          (size_t)a.ngroups * a.subs + 1, split, a.pm, a.pl, a.pacc);
}

// ------------------------------------------------ fused scan + attend ----
// Bit-plane codes only.  One persistent block of 14 warps per SM walks a
// contiguous share of the live (sequence, kv head, 1024-token chunk) items,
// like the bit-plane scan, and attends each item's candidates itself, so the
// candidate lists never leave shared memory and the code stream and the K/V
// row gathers of different items overlap on the same SM:
//   warp 0      TMA producer of the code stages (8 tables per 3-D copy);
//   warp 1      fold of the scan partials and compaction of each item's
//               candidates into a shared queue (sampled rows with their head
//               masks, then the exact-set rows of the chunk with an empty mask);
//   warps 2-5   scan: two tables of every stage each, bit-sliced counters;
//   warps 6-13  two attention groups of 4 warps, taking alternate items:
//               K/V rows of 64 queue entries per tile through a 2-stage
//               cp.async ring, the same per-warp tile math as attend_kernel,
//               one (m, l, acc) partial per item and head.
// Hand-offs: code stages by full/empty mbarriers, scan partials by named
// barriers 2/3 (double-buffered by item parity), queue buffers (2 per group)
// by full/empty mbarriers; each group syncs on its own named barrier.
constexpr int kFusedScanWarps = 4;
constexpr int kFusedGroups = 2;
constexpr int kFusedThreads = 32 * (2 + kFusedScanWarps + 4 * kFusedGroups);  // 448
constexpr int kFusedQueues = 2 * kFusedGroups;                                // candidate queue buffers
constexpr int kFusedPrefetch = 16;  // code stages pulled into L2 ahead of the ring

template <int KB>
struct FusedCfg {
    static constexpr int kStages = KB == 8 ? 5 : 3;  // code ring depth
};

struct FusedArgs {
    Shape s;
    const uint16_t *q, *kc, *vc, *qcodes;
    const int32_t *seq_lens;
    int max_len, nchunk;
    int32_t *cnt;         // [B*Hkv][nchunk][16]: [0] sampled union, [1+g] per head
    uint8_t *member_out;  // nullable [B][Hq][Ncap]
    int32_t *status;
    float *pm, *pl, *pacc;  // [B*Hq][nchunk + 1], [..][..][128]; split = chunk
    LogU lu;
    float scale;
};

template <int G, int KB>
constexpr size_t fused_smem_bytes(int L)
{
    return (size_t)FusedCfg<KB>::kStages * PlaneStage<KB>::kBytes + (size_t)L * G * ((KB + 3) & ~3) * 4 +
           (size_t)2 * G * 2 * (kFusedScanWarps * 32) * 4 + (size_t)kFusedQueues * kChunkPlanes * 4 +
           (size_t)kFusedGroups * kAttStages * kStageBytes;
}

__device__ __forceinline__ void bar_sync_n(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ void bar_arrive_n(int id, int n) { asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory"); }

template <int G, int KB>
__global__ void __launch_bounds__(kFusedThreads, 1) fused_planes_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                        FusedArgs a)
{
    using St = PlaneStage<KB>;
    constexpr int S = FusedCfg<KB>::kStages, QW = (KB + 3) & ~3, NSW = kFusedScanWarps, NQ = kFusedQueues;
    constexpr int SCAN_T = NSW * 32, HAND_T = SCAN_T + 32;  // scan warps; scan warps + the compaction warp
    const Shape &s = a.s;
    extern __shared__ __align__(1024) uint8_t dyn_raw[];
    uint32_t *ring = reinterpret_cast<uint32_t *>(dyn_raw);  // [S][box][8 tables][kBoxWords]
    uint32_t *qm = ring + S * St::kBytes / 4;                // [L][G][QW]
    uint32_t *part = qm + s.L * G * QW;                      // [2][G][2][SCAN_T]
    uint32_t *cq = part + 2 * G * 2 * SCAN_T;                // [NQ][1024] queue entries
    uint8_t *att = reinterpret_cast<uint8_t *>(cq + NQ * kChunkPlanes);  // [groups][stages][K rows, V rows]
    __shared__ __align__(8) uint64_t full[S], empty[S], cqf[NQ], cqe[NQ];
    __shared__ int cq_meta[NQ][4];  // unit, chunk, rows
    __shared__ int range_sh[4];
    __shared__ int gflag[kFusedGroups];
    __shared__ uint32_t meta[kFusedGroups][kAttStages][kAttRows];
    __shared__ float ucos[4 * kFusedGroups][16 * G], uval[4 * kFusedGroups][16 * G];
    __shared__ float qinv[kFusedGroups][G];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    grid_dependency_wait();

    if (threadIdx.x == 0) {
        // this block's contiguous share of the live items
        long long total = 0;
        for (int b = 0; b < s.B; b++) {
            const int n = clamp_len(a.seq_lens, b, a.max_len, a.status, blockIdx.x == 0);
            total += (long long)s.Hkv * ((n + kChunkPlanes - 1) / kChunkPlanes);
        }
        long long x = total * blockIdx.x / gridDim.x;
        const long long x1 = total * (blockIdx.x + 1) / gridDim.x;
        range_sh[3] = (int)(x1 - x);
        range_sh[0] = range_sh[1] = range_sh[2] = 0;
        for (int b = 0; b < s.B && x1 > x; b++) {
            const int n = min(max(a.seq_lens[b], 0), a.max_len);
            const long long nch = (n + kChunkPlanes - 1) / kChunkPlanes, items = nch * s.Hkv;
            if (x < items) {
                range_sh[0] = b;
                range_sh[1] = (int)(x / nch);
                range_sh[2] = (int)(x % nch);
                break;
            }
            x -= items;
        }
        for (int i = 0; i < S; i++) {
            mbar_init(smem_u32(&full[i]), 1);
            mbar_init(smem_u32(&empty[i]), NSW);
        }
        for (int i = 0; i < NQ; i++) {
            mbar_init(smem_u32(&cqf[i]), 1);
            mbar_init(smem_u32(&cqe[i]), 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const int count = range_sh[3];
    if (count <= 0) return;
    LiveCursor cur;
    cur.b = range_sh[0];
    cur.kvh = range_sh[1];
    cur.chunk = range_sh[2];
    cur.load_seq(a.seq_lens, a.max_len);
    const int nst = (s.L + 7) / 8;  // stages per item

    if (warp == 0) {
        // -------------------------------------------------- code producer ----
        if (lane == 0) {
            int e = 0;
            LiveCursor pc = cur;
            // a second cursor kFusedPrefetch stages ahead pulls stages into L2,
            // so that far more code bytes are in flight than the ring holds
            LiveCursor fc = cur;
            int fj = 0, fit = 0;
            auto prefetch_next = [&] {
                if (fit >= count) return;
#pragma unroll
                for (int bx = 0; bx < St::kBoxes; bx++)
                    tma_prefetch_3d(&tmap, fc.chunk * 32 * KB + bx * St::kBoxWords, 8 * fj, fc.unit(s));
                if (++fj == nst) {
                    fj = 0;
                    fit++;
                    fc.next(s, a.seq_lens, a.max_len);
                }
            };
            for (int i = 0; i < kFusedPrefetch; i++) prefetch_next();
            for (int it = 0; it < count; it++, pc.next(s, a.seq_lens, a.max_len)) {
                const int x0 = pc.chunk * 32 * KB, z = pc.unit(s);
                bool ok = true;
                for (int j = 0; j < nst; j++, e++) {
                    const int st = e % S;
                    prefetch_next();
                    if (e >= S && !mbar_wait_bounded(smem_u32(&empty[st]), (uint32_t)(e / S - 1) & 1u)) {
                        set_status(a.status, MP_ERR_CUDA);
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(smem_u32(&full[st]), St::kBytes);
#pragma unroll
                    for (int bx = 0; bx < St::kBoxes; bx++)
                        tma_load_3d(smem_u32(ring) + (uint32_t)(st * St::kBytes + bx * 8 * St::kBoxWords * 4), &tmap,
                                    smem_u32(&full[st]), x0 + bx * St::kBoxWords, 8 * j, z);
                }
                if (!ok) break;
            }
            // every code copy issued lands before the block exits (the last use of each stage)
            for (int st = 0; st < S && st < e; st++) {
                const int last = st + ((e - 1 - st) / S) * S;
                mbar_wait_bounded(smem_u32(&full[st]), (uint32_t)(last / S) & 1u);
            }
        }
        return;
    }

    if (warp == 1) {
        // --------------------------------------------- fold and compaction ----
        for (int ci = 0; ci < count; ci++, cur.next(s, a.seq_lens, a.max_len)) {
            const int qb = ci % NQ;
            bar_sync_n(2, HAND_T);  // the scan partials of item ci are in buffer ci & 1
            const uint32_t *pp = part + (ci & 1) * (G * 2 * SCAN_T);
            uint32_t s1[G], s2[G];
#pragma unroll
            for (int g = 0; g < G; g++) s1[g] = s2[g] = 0u;
#pragma unroll 1
            for (int t = 0; t < NSW; t++) {
#pragma unroll
                for (int g = 0; g < G; g++) {
                    const uint32_t a1 = pp[(g * 2 + 0) * SCAN_T + t * 32 + lane];
                    const uint32_t a2 = pp[(g * 2 + 1) * SCAN_T + t * 32 + lane];
                    s2[g] |= a2 | (s1[g] & a1);
                    s1[g] |= a1;
                }
            }
            if (ci + 1 < count) bar_arrive_n(3, HAND_T);  // item ci read: the scan may post item ci + 1
            // the queue buffer's previous item (ci - NQ) must have been attended
            bool free_ok = true;
            if (ci >= NQ && lane == 0)
                free_ok = mbar_wait_bounded(smem_u32(&cqe[qb]), (uint32_t)(ci / NQ - 1) & 1u);
            if (!__shfl_sync(0xffffffffu, (int)free_ok, 0) && lane == 0) set_status(a.status, MP_ERR_CUDA);
            const int unit = cur.unit(s), N = cur.N, c0 = cur.chunk * kChunkPlanes, t0 = c0 + lane * 32;
            uint32_t *q_ent = cq + qb * kChunkPlanes;
            // sampled rows: tokens in [sink, N - window) and below N, in token order
            const uint32_t v = range_mask(t0, s.sink, min(N - s.window, N), 32);
            uint32_t any = 0u;
#pragma unroll
            for (int g = 0; g < G; g++) {
                s2[g] &= v;
                any |= s2[g];
            }
            const int mine = __popc(any);
            int incl = mine;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += t;
            }
            const int nsamp = __shfl_sync(0xffffffffu, incl, 31);
            int off = incl - mine;
            while (any) {
                const int bit = __ffs(any) - 1;
                any &= any - 1u;
                uint32_t heads = 0u;
#pragma unroll
                for (int g = 0; g < G; g++) heads |= ((s2[g] >> bit) & 1u) << g;
                q_ent[off++] = (uint32_t)(t0 + bit) | (heads << 24);
            }
            // then the chunk's exact-set rows (empty head mask)
            const int n_sink = min(s.sink, N), win0 = max(n_sink, N - s.window);
            const int sink_hi = min(c0 + kChunkPlanes, n_sink);
            const int win_lo = max(c0, win0), win_hi = min(c0 + kChunkPlanes, N);
            const int na = max(0, sink_hi - c0), nb = max(0, win_hi - win_lo);
            for (int i = lane; i < na + nb; i += 32)
                q_ent[nsamp + i] = (uint32_t)(i < na ? c0 + i : win_lo + (i - na));
            int32_t *cnt = a.cnt + ((size_t)unit * a.nchunk + cur.chunk) * 16;
            if (lane == 0) cnt[0] = nsamp;
#pragma unroll
            for (int g = 0; g < G; g++) {
                int c = __popc(s2[g]);
#pragma unroll
                for (int d = 16; d > 0; d >>= 1) c += __shfl_xor_sync(0xffffffffu, c, d);
                if (lane == 0) cnt[1 + g] = c;
            }
            if (a.member_out)
                for (int i = 0; i < 32 && t0 + i < N; i++)
#pragma unroll
                    for (int g = 0; g < G; g++)
                        a.member_out[((size_t)cur.b * s.Hq + cur.kvh * G + g) * s.Ncap + t0 + i] =
                            (s2[g] >> i) & 1u;
            if (lane == 0) {
                cq_meta[qb][0] = unit;
                cq_meta[qb][1] = cur.chunk;
                cq_meta[qb][2] = nsamp + na + nb;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&cqf[qb]));  // the queue buffer is ready for its group
        }
        return;
    }

    if (warp < 2 + NSW) {
        // ------------------------------------------------------------ scan ----
        const int ts = warp - 2;  // tables 8 j + ts and 8 j + ts + 4 of stage j
        int e = 0, qm_unit = -1;
        bool dead = false;
        for (int it = 0; it < count; it++, cur.next(s, a.seq_lens, a.max_len)) {
            const int unit = cur.unit(s);
            if (unit != qm_unit) {  // uniform over the scan warps
                if (qm_unit >= 0) bar_sync_n(1, SCAN_T);  // every scan warp is done with the old masks
                for (int i = threadIdx.x - 64; i < s.L * G; i += SCAN_T) {
                    const int l = i / G, g = i % G;
                    const unsigned code = a.qcodes[((size_t)cur.b * s.Hq + cur.kvh * G + g) * s.L + l];
                    uint4 *dst = reinterpret_cast<uint4 *>(qm + (size_t)i * QW);
#pragma unroll
                    for (int q = 0; q < QW / 4; q++) {
                        uint32_t m[4];
#pragma unroll
                        for (int x = 0; x < 4; x++) m[x] = 4 * q + x < KB ? 0u - ((code >> (4 * q + x)) & 1u) : 0u;
                        dst[q] = make_uint4(m[0], m[1], m[2], m[3]);
                    }
                }
                bar_sync_n(1, SCAN_T);
                qm_unit = unit;
            }
            uint32_t s1[G], s2[G];
#pragma unroll
            for (int g = 0; g < G; g++) s1[g] = s2[g] = 0u;
            for (int j = 0; j < nst; j++, e++) {
                const int st = e % S;
                if (!dead) {
                    const bool landed = mbar_wait_bounded(smem_u32(&full[st]), (uint32_t)(e / S) & 1u);
                    if (!__all_sync(0xffffffffu, landed)) {
                        if (lane == 0) set_status(a.status, MP_ERR_CUDA);
                        dead = true;
                    }
                }
#pragma unroll
                for (int half = 0; half < 2; half++) {
                    const int r = ts + 4 * half, l = 8 * j + r;  // row of the stage, table
                    if (dead || l >= s.L) continue;
                    const int box = (lane * KB) / St::kBoxWords, in_box = lane * KB - box * St::kBoxWords;
                    const uint32_t *src = ring + st * (St::kBytes / 4) + box * 8 * St::kBoxWords + r * St::kBoxWords + in_box;
                    uint32_t pw[KB];
                    if constexpr (KB % 4 == 0) {
#pragma unroll
                        for (int q = 0; q < KB / 4; q++) {
                            const uint4 v = reinterpret_cast<const uint4 *>(src)[q];
                            pw[4 * q] = v.x;
                            pw[4 * q + 1] = v.y;
                            pw[4 * q + 2] = v.z;
                            pw[4 * q + 3] = v.w;
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < KB / 2; q++) {
                            const uint2 v = reinterpret_cast<const uint2 *>(src)[q];
                            pw[2 * q] = v.x;
                            pw[2 * q + 1] = v.y;
                        }
                    }
#pragma unroll
                    for (int g = 0; g < G; g++) {
                        const uint4 *m4 = reinterpret_cast<const uint4 *>(qm + (l * G + g) * QW);
                        uint32_t mis = 0u;
#pragma unroll
                        for (int q = 0; q < QW / 4; q++) {
                            const uint4 mq = m4[q];
                            const uint32_t mm[4] = {mq.x, mq.y, mq.z, mq.w};
#pragma unroll
                            for (int x = 0; x < 4; x++)
                                if (4 * q + x < KB) mis |= pw[4 * q + x] ^ mm[x];
                        }
                        s2[g] |= s1[g] & ~mis;
                        s1[g] |= ~mis;
                    }
                }
                // release the stage once every lane has used its words
                __syncwarp();
                if (lane == 0 && !dead) {
                    fence_proxy_async_smem();
                    mbar_arrive(smem_u32(&empty[st]));
                }
            }
            if (it >= 1) bar_sync_n(3, HAND_T);  // warp 0 has read item it - 1's partials
            uint32_t *pp = part + (it & 1) * (G * 2 * SCAN_T);
#pragma unroll
            for (int g = 0; g < G; g++) {
                pp[(g * 2 + 0) * SCAN_T + ts * 32 + lane] = s1[g];
                pp[(g * 2 + 1) * SCAN_T + ts * 32 + lane] = s2[g];
            }
            bar_arrive_n(2, HAND_T);
        }
        return;
    }

    // ------------------------------------------------------- attention ----
    const int grp = (warp - 2 - NSW) >> 2, gw = (warp - 2 - NSW) & 3, gtid = gw * 32 + lane;
    const int gbar_id = 4 + grp;
    auto gbar = [&] { bar_sync_n(gbar_id, 128); };
    uint8_t *gring = att + grp * kAttStages * kStageBytes;
    const uint32_t dmeta = ((1u << G) - 1u) | 0x100u;
    for (int k = grp; k < count; k += kFusedGroups) {
        const int qb = k % NQ;
        if (gtid == 0) gflag[grp] = mbar_wait_bounded(smem_u32(&cqf[qb]), (uint32_t)(k / NQ) & 1u) ? 1 : 0;
        gbar();  // the queue buffer (and, from the item before, the ring and qinv) is ours
        if (!gflag[grp]) {
            if (gtid == 0) set_status(a.status, MP_ERR_CUDA);
            break;
        }
        const int unit = cq_meta[qb][0], chunk = cq_meta[qb][1], rows = cq_meta[qb][2];
        const int b = unit / s.Hkv, kvh = unit % s.Hkv;
        const size_t vec0 = (size_t)b * s.Hq + (size_t)kvh * G;
        const uint16_t *kbase = a.kc + (size_t)unit * s.Ncap * kHeadDim;
        const uint16_t *vbase = a.vc + (size_t)unit * s.Ncap * kHeadDim;
        const uint32_t *ents = cq + qb * kChunkPlanes;
        AttnWarp<G> w;
        attn_begin<G>(w, a.q, vec0, lane);
        attn_qinv<G>(a.q, vec0, gw, lane, qinv[grp]);
        auto issue = [&](int tile, int stage) {
            uint8_t *ks_ = gring + stage * kStageBytes;
            uint8_t *vs_ = ks_ + kAttRows * kRowStride;
            const int col = gtid & 15;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const int r = (gtid >> 4) + 8 * i, idx = tile * kAttRows + r;
                const uint32_t ent = idx < rows ? ents[idx] : 0xFFFFFFFFu;
                const bool ok = ent != 0xFFFFFFFFu;
                const int tok = ok ? (int)(ent & 0xFFFFFFu) : 0;
                const size_t off = (size_t)tok * kHeadDim + col * 8;
                cp_async_16(ks_ + r * kRowStride + att_piece(r, col), kbase + off, ok ? 16 : 0);
                cp_async_16(vs_ + r * kRowStride + att_piece(r, col), vbase + off, ok ? 16 : 0);
                if (col == 0) meta[grp][stage][r] = ok ? ((ent >> 24) ? (ent >> 24) : dmeta) : 0u;
            }
        };
        const int ntiles = (rows + kAttRows - 1) / kAttRows;
        if (ntiles > 0) issue(0, 0);
        cp_async_commit();
        gbar();  // qinv
        attn_set_qinv<G>(w, qinv[grp], lane);
        for (int tile = 0; tile < ntiles; tile++) {
            if (tile + 1 < ntiles) issue(tile + 1, (tile + 1) % kAttStages);
            cp_async_commit();
            cp_async_wait<kAttStages - 1>();
            gbar();
            const int stage = tile % kAttStages;
            const uint8_t *ks_ = gring + stage * kStageBytes;
            attn_tile<G>(w, ks_, ks_ + kAttRows * kRowStride, meta[grp][stage], gw, lane, a.scale, a.lu,
                         ucos[grp * 4 + gw], uval[grp * 4 + gw]);
            gbar();  // the stage may be refilled
        }
        cp_async_wait<0>();
        gbar();  // every entry of the queue buffer has been read, the ring is idle
        if (gtid == 0) mbar_arrive(smem_u32(&cqe[qb]));
        attn_store_partial<G>(w, reinterpret_cast<float *>(gring), gw, lane, gtid, gbar, vec0,
                              (size_t)a.nchunk + 1, chunk, a.pm, a.pl, a.pacc);
    }
}

// ----------------------------------------------------------------- merge ----
constexpr int kMergeBatch = 8;  // splits per warp whose loads are in flight together
constexpr int kMergeWarps = 8;  // 8 kMergeBatch = 64 splits per head in one round of loads

// One block of kMergeWarps warps per (b, q head).  Warp w folds splits w,
// w + kMergeWarps, ... (lane = 4 output dims) with a running maximum,
// rescaling its sums when the maximum moves, so all loads go out in one pass
// (unrolled); the warps' (m, l, acc) are then combined in shared memory.
template <int G>
__global__ void __launch_bounds__(32 * kMergeWarps) merge_kernel(Shape s, const int32_t *__restrict__ seq_lens,
                                                         int max_len, int nchunk, int span, int subs,
                                                         int ngroups, int chunk_tokens,
                                                         const float *__restrict__ pm,
                                                         const float *__restrict__ pl,
                                                         const float *__restrict__ pacc,
                                                         const int32_t *__restrict__ cnt, float *out,
                                                         float *lse, int32_t *n_sampled, int has_d)
{
    __shared__ float red_m[kMergeWarps], red_l[kMergeWarps];
    __shared__ int red_n[kMergeWarps];
    __shared__ float4 red_acc[kMergeWarps][32];
    const int bh = blockIdx.x;
    const int b = bh / s.Hq, h = bh % s.Hq, kvh = h / G, g = h % G;
    const int unit = b * s.Hkv + kvh;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // the lengths come from work before this kernel's predecessor: that read
    // goes before the wait; the per-chunk counts (the scan's, made visible to
    // the attention by the ready flags, or the fused kernel's) after it
    int N = seq_lens[b];
    N = N < 0 ? 0 : (N > max_len ? max_len : N);
    const int nch = (N + chunk_tokens - 1) / chunk_tokens;
    grid_dependency_wait();
    int ns = 0;
    for (int j = tid; j < nch; j += blockDim.x) ns += cnt[((size_t)unit * nchunk + j) * 16 + 1 + g];
    const int nsp = ((nch + span - 1) / span) * subs;  // live chunk splits
    const int dsp = ngroups * subs;                     // the exact-set split (if has_d)
    const size_t base = (size_t)bh * (dsp + 1);
    // split j in [0, dsp] holds a partial of this call iff j < nsp or it is
    // the exact-set split; the loads below do not wait for that test (they
    // stay inside the partial arrays), only the fold does
    auto live = [&](int j) { return j < nsp || (has_d && j == dsp); };

    // each warp folds splits warp, warp + 4, ... with a running maximum; the
    // loads of kMergeBatch splits go out together before any of them is used
    float m = -INFINITY, Ls = 0.f;
    float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = warp; j0 <= dsp; j0 += kMergeWarps * kMergeBatch) {
        float mj[kMergeBatch], lj[kMergeBatch];
        float4 aj[kMergeBatch];
#pragma unroll
        for (int i = 0; i < kMergeBatch; i++) {
            const int j = j0 + kMergeWarps * i;
            mj[i] = -INFINITY;
            lj[i] = 0.f;
            aj[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j <= dsp) {
                const size_t sp = base + j;
                mj[i] = pm[sp];
                lj[i] = pl[sp];
                aj[i] = reinterpret_cast<const float4 *>(pacc + sp * kHeadDim)[lane];
            }
        }
#pragma unroll
        for (int i = 0; i < kMergeBatch; i++)
            if (!live(j0 + kMergeWarps * i)) mj[i] = -INFINITY;
#pragma unroll
        for (int i = 0; i < kMergeBatch; i++) {
            if (mj[i] == -INFINITY) continue;  // an empty or absent split (uniform across the warp)
            if (mj[i] > m) {
                const float f = m == -INFINITY ? 0.f : fast_exp2(m - mj[i]);
                Ls *= f;
                A.x *= f;
                A.y *= f;
                A.z *= f;
                A.w *= f;
                m = mj[i];
            }
            const float f = fast_exp2(mj[i] - m);
            Ls = fmaf(lj[i], f, Ls);
            A.x = fmaf(aj[i].x, f, A.x);
            A.y = fmaf(aj[i].y, f, A.y);
            A.z = fmaf(aj[i].z, f, A.z);
            A.w = fmaf(aj[i].w, f, A.w);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ns += __shfl_xor_sync(0xffffffffu, ns, o);
    red_acc[warp][lane] = A;
    if (lane == 0) {
        red_m[warp] = m;
        red_l[warp] = Ls;
        red_n[warp] = ns;
    }
    __syncthreads();
    if (warp == 0) {
        float M = red_m[0];
#pragma unroll
        for (int w = 1; w < kMergeWarps; w++) M = fmaxf(M, red_m[w]);
        float Lt = 0.f;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kMergeWarps; w++) {
                if (red_m[w] == -INFINITY) continue;
                const float f = fast_exp2(red_m[w] - M);
                const float4 t = red_acc[w][lane];
                Lt = fmaf(red_l[w], f, Lt);
                o.x = fmaf(t.x, f, o.x);
                o.y = fmaf(t.y, f, o.y);
                o.z = fmaf(t.z, f, o.z);
                o.w = fmaf(t.w, f, o.w);
            }
        }
        const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
        o.x *= inv;
        o.y *= inv;
        o.z *= inv;
        o.w *= inv;
        reinterpret_cast<float4 *>(out + (size_t)bh * kHeadDim)[lane] = o;
        if (lane == 0) {
            lse[bh] = Lt > 0.f ? (M + log2f(Lt)) * kLn2 : -INFINITY;  // partials keep log2 units
            int nt = 0;
#pragma unroll
            for (int w = 0; w < kMergeWarps; w++) nt += red_n[w];
            n_sampled[bh] = nt;
        }
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

// How attention blocks cover the scan chunks (the fused kernel instead writes
// one partial per 1024-token chunk).  Many chunks: each block takes
// `span` consecutive chunks (1200 to 2400 blocks in all, more for larger
// problems: several waves of 3 blocks per SM, so that uneven candidate counts
// even out, while the per-block set-up stays amortised and the merge sees few
// partials).  Few, large chunks:
// each chunk's list is shared by `subs` blocks.  Fixed counts, so the
// workspace size does not depend on the device.
struct SplitPlan {
    int nchunk, span, subs, ngroups, nsplit;
};

#ifndef MP_ATT_TARGET_BLOCKS
#define MP_ATT_TARGET_BLOCKS 2400
#endif
#ifndef MP_ATT_TARGET_DIV
#define MP_ATT_TARGET_DIV 6
#endif
static SplitPlan split_plan(const Shape &s, int max_len)
{
    SplitPlan p;
    const int C = chunk_tokens(s);
    p.nchunk = (max_len + C - 1) / C;
    const int blocks = p.nchunk * s.B * s.Hkv;
    // More, shorter splits pay off on large problems, fewer on small ones.
    // Measured per step (bit-plane codes, attention started by the scan's
    // ready flags): ragged16 (16512 chunk-blocks) 342 us at 2400 blocks (6
    // chunks a block) against 350 at 4128, 358 at 5504, 367 at 8256 and 355
    // at 1376; ragged4 and batch8_64k (4128 and 4160) the same within 1% from
    // 1200 to 2064 blocks.
    const int kTarget = std::min(MP_ATT_TARGET_BLOCKS, std::max(1200, blocks / MP_ATT_TARGET_DIV));
    if (blocks >= kTarget) {
        p.span = std::min(kMaxSpan, blocks / kTarget);
        p.subs = 1;
    } else {
        // few chunks: split each chunk's list so that about kTarget blocks run,
        // but give every block at least ~1024 tokens' worth of candidates
        p.span = 1;
        const int by_count = blocks > 0 ? (kTarget + blocks - 1) / blocks : 1;
        p.subs = std::max(1, std::min({8, by_count, C / 1024}));
    }
    p.ngroups = (p.nchunk + p.span - 1) / p.span;
    p.nsplit = p.ngroups * p.subs + 1;
    return p;
}

Workspace workspace_layout(const Shape &s, int max_len, void *base)
{
    const int C = chunk_tokens(s);
    const SplitPlan sp = split_plan(s, max_len);
    const int nchunk = sp.nchunk;
    // bit planes may take the fused kernel, which writes one partial per chunk
    const size_t nsplit = s.planes ? std::max((size_t)sp.nsplit, (size_t)nchunk + 1) : (size_t)sp.nsplit;
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
    u.a6 = (float)((L - 5.0) / 6.0);
    return u;
}

// Persistent plane scan: as many blocks as fit on the device at once (at
// most one per possible item); each walks its share of the live items.
template <int G, int KB>
static cudaError_t launch_scan_planes_warp(const Shape &s, const uint32_t *codes, const Workspace &ws,
                                           const int32_t *seq_lens, int max_len, int nchunk, const ScanOut &so,
                                           cudaStream_t st)
{
    const size_t sm = (size_t)kPlaneWarps * kPlaneRing * plane_slot_bytes<KB>() +
                      (size_t)s.L * G * ((KB + 3) & ~3) * sizeof(uint32_t);
    const void *fn = reinterpret_cast<const void *>(scan_planes_warp_kernel<G, KB>);
    cudaError_t e = ensure_smem(fn, (int)sm);
    if (e != cudaSuccess) return e;
    dim3 grid((nchunk + kPlaneWarps - 1) / kPlaneWarps, s.B * s.Hkv);
    return launch_pdl(scan_planes_warp_kernel<G, KB>, grid, dim3(32 * kPlaneWarps), sm, st, s, codes,
                      (const uint16_t *)ws.qcodes, seq_lens, max_len, nchunk, so);
}

// The fused scan + attend kernel, if its shared memory fits on the device
// (`used` tells the caller whether it ran).  One block per SM.
template <int G, int KB>
static cudaError_t launch_fused(const Shape &s, const uint32_t *codes, const Workspace &ws, const FusedArgs &fa,
                                cudaStream_t st, bool &used)
{
    used = false;
    const void *fn = reinterpret_cast<const void *>(fused_planes_kernel<G, KB>);
    const size_t sm = fused_smem_bytes<G, KB>(s.L);
    int dev = 0, optin = 0, sms = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cudaFuncAttributes attr;
    if ((e = cudaFuncGetAttributes(&attr, fn)) != cudaSuccess) return e;
    if (sm + attr.sharedSizeBytes > (size_t)optin) return cudaSuccess;  // does not fit: two-kernel path
    if ((e = ensure_smem(fn, (int)sm)) != cudaSuccess) return e;
    const int words = s.Ncap >> 5;
    const uint64_t dims[3] = {(uint64_t)words * KB, (uint64_t)s.L, (uint64_t)s.B * s.Hkv};
    const uint64_t strides[2] = {(uint64_t)words * KB * 4, (uint64_t)s.L * words * KB * 4};
    const uint32_t box[3] = {(uint32_t)PlaneStage<KB>::kBoxWords, 8, 1};
    CUtensorMap tmap;
    if (!encode_tensor_map(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, codes, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const long long items = (long long)fa.nchunk * s.B * s.Hkv;
    const int grid = (int)std::max(1LL, std::min(items, (long long)sms));
    e = launch_pdl(fused_planes_kernel<G, KB>, dim3(grid), dim3(kFusedThreads), sm, st, tmap, fa);
    used = e == cudaSuccess;
    return e;
}

template <int G>
static cudaError_t launch_decode_g(const Shape &s, const uint16_t *q, const uint16_t *W, const void *codes,
                                   const uint16_t *kc, const uint16_t *vc, const int32_t *seq_lens,
                                   int max_len, float *out, float *lse, int32_t *n_sampled,
                                   const Workspace &ws, const mp_decode_debug *dbg, cudaStream_t st,
                                   const int8_t *k8)
{
    const int C = chunk_tokens(s);
    const SplitPlan sp = split_plan(s, max_len);
    const int nchunk = sp.nchunk;
    const int units = s.B * s.Hkv;
    cudaError_t e;
    {
        const int TB = qhash_tables_per_block(s.K), ug = qhash_units_per_block(s, G);
        dim3 grid((s.L + TB - 1) / TB, (units + ug - 1) / ug);
        e = launch_pdl(qhash_kernel<G>, grid, dim3(256), 0, st, s, q, W,
                       (const uint16_t *)(dbg ? dbg->qcodes_in : nullptr), ws.qcodes, ws.status, ug, ws.cnt,
                       units * nchunk);
        if (e != cudaSuccess) return e;
    }
    ScanOut so{ws.cand, ws.cnt, dbg ? dbg->member_out : nullptr, ws.status};
    const LogU lu = make_logu(s);
    const float scale = 1.0f / sqrtf((float)s.d);
    const int path = dbg ? dbg->path : MP_PATH_AUTO;
    bool fused = false;
    // The fused kernel is opt-in: it shares each SM's warps and shared memory
    // between the code stream and the row gathers, and measured slower than
    // giving each phase the whole device in turn.
    if (nchunk > 0 && s.planes && path == MP_PATH_FUSED) {
        FusedArgs fa;
        fa.s = s;
        fa.q = q;
        fa.kc = kc;
        fa.vc = vc;
        fa.qcodes = ws.qcodes;
        fa.seq_lens = seq_lens;
        fa.max_len = max_len;
        fa.nchunk = nchunk;
        fa.cnt = ws.cnt;
        fa.member_out = dbg ? dbg->member_out : nullptr;
        fa.status = ws.status;
        fa.pm = ws.pm;
        fa.pl = ws.pl;
        fa.pacc = ws.pacc;
        fa.lu = lu;
        fa.scale = scale;
        e = s.K == 8 ? launch_fused<G, 8>(s, static_cast<const uint32_t *>(codes), ws, fa, st, fused)
                     : launch_fused<G, 10>(s, static_cast<const uint32_t *>(codes), ws, fa, st, fused);
        if (e != cudaSuccess) return e;
        if (!fused && path == MP_PATH_FUSED) return cudaErrorNotSupported;
    }
    if (nchunk > 0 && !fused && !(dbg && dbg->skip_scan)) {
        if (!s.planes) {
            const size_t sm = (size_t)kByteWarps * kByteRing * kChunkBytes + (size_t)s.L * std::max(G, 4) * sizeof(uint32_t);
            if ((e = ensure_smem(reinterpret_cast<const void *>(scan_bytes_kernel<G>), (int)sm)) != cudaSuccess)
                return e;
            dim3 grid((nchunk + kByteWarps - 1) / kByteWarps, units);
            e = launch_pdl(scan_bytes_kernel<G>, grid, dim3(32 * kByteWarps), sm, st, s,
                           static_cast<const uint8_t *>(codes), (const uint16_t *)ws.qcodes, seq_lens, max_len,
                           nchunk, so);
        } else if (s.K == 8) {
            e = launch_scan_planes_warp<G, 8>(s, static_cast<const uint32_t *>(codes), ws, seq_lens, max_len,
                                              nchunk, so, st);
        } else {
            e = launch_scan_planes_warp<G, 10>(s, static_cast<const uint32_t *>(codes), ws, seq_lens, max_len,
                                               nchunk, so, st);
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
    aa.span = sp.span;
    aa.subs = sp.subs;
    aa.ngroups = sp.ngroups;
    aa.chunk_tokens = C;
    aa.cand = ws.cand;
    aa.cnt = ws.cnt;
    aa.pm = ws.pm;
    aa.pl = ws.pl;
    aa.pacc = ws.pacc;

    aa.lu = lu;
    aa.scale = scale;
    aa.k8 = k8;
    aa.status = ws.status;
    if (!fused && path != MP_PATH_TC && k8) {
        const int sm = kAttStages * att_stage_bytes<true>();
        if ((e = ensure_smem(reinterpret_cast<const void *>(attend_kernel<G, true>), sm)) != cudaSuccess) return e;
        dim3 grid(sp.nsplit, units);
        if ((e = launch_pdl(attend_kernel<G, true>, grid, dim3(kAttThreads), sm, st, aa)) != cudaSuccess) return e;
    } else if (!fused && path != MP_PATH_TC) {
        const int sm = kAttStages * att_stage_bytes<false>();
        if ((e = ensure_smem(reinterpret_cast<const void *>(attend_kernel<G, false>), sm)) != cudaSuccess) return e;
        dim3 grid(sp.nsplit, units);
        if ((e = launch_pdl(attend_kernel<G, false>, grid, dim3(kAttThreads), sm, st, aa)) != cudaSuccess) return e;
    } else if (!fused) {
        AttendTcArgs ta;
        ta.s = s;
        ta.q = q;
        ta.kc = kc;
        ta.vc = vc;
        ta.seq_lens = seq_lens;
        ta.max_len = max_len;
        ta.nchunk = nchunk;
        ta.span = sp.span;
        ta.subs = sp.subs;
        ta.nsplit = sp.nsplit;
        ta.chunk_tokens = C;
        ta.cand = ws.cand;
        ta.cnt = ws.cnt;
        ta.work_counter = ws.status + 1;
        ta.status = ws.status;
        ta.pm = ws.pm;
        ta.pl = ws.pl;
        ta.pacc = ws.pacc;
        ta.lu = lu;
        ta.scale = scale;
        if ((e = launch_attend_tc(ta, st)) != cudaSuccess) return e;
    }
    // partials: per chunk (fused) or per split of the plan, then the exact set
    const int m_span = fused ? 1 : sp.span, m_subs = fused ? 1 : sp.subs, m_groups = fused ? nchunk : sp.ngroups;
    e = launch_pdl(merge_kernel<G>, dim3(s.B * s.Hq), dim3(32 * kMergeWarps), 0, st, s, seq_lens, max_len, nchunk, m_span,
                   m_subs, m_groups, C, (const float *)ws.pm, (const float *)ws.pl, (const float *)ws.pacc,
                   (const int32_t *)ws.cnt, out, lse, n_sampled, fused ? 0 : 1);
    if (e != cudaSuccess) return e;
    if (dbg && dbg->qcodes_out)
        e = cudaMemcpyAsync(dbg->qcodes_out, ws.qcodes, (size_t)s.B * s.Hq * s.L * sizeof(uint16_t),
                            cudaMemcpyDeviceToDevice, st);
    return e;
}

cudaError_t launch_decode(const Shape &s, const uint16_t *q, const uint16_t *W, const void *codes,
                          const uint16_t *kc, const uint16_t *vc, const int32_t *seq_lens, int max_len,
                          float *out, float *lse, int32_t *n_sampled, void *workspace,
                          const mp_decode_debug *dbg, cudaStream_t st, const int8_t *k8)
{
    const Workspace ws = workspace_layout(s, max_len, workspace);
    switch (s.G) {
    case 1: return launch_decode_g<1>(s, q, W, codes, kc, vc, seq_lens, max_len, out, lse, n_sampled, ws, dbg, st, k8);
    case 2: return launch_decode_g<2>(s, q, W, codes, kc, vc, seq_lens, max_len, out, lse, n_sampled, ws, dbg, st, k8);
    case 4: return launch_decode_g<4>(s, q, W, codes, kc, vc, seq_lens, max_len, out, lse, n_sampled, ws, dbg, st, k8);
    case 8: return launch_decode_g<8>(s, q, W, codes, kc, vc, seq_lens, max_len, out, lse, n_sampled, ws, dbg, st, k8);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_hash_queries(const Shape &s, const uint16_t *q, const uint16_t *W, uint16_t *qcodes,
                                cudaStream_t st)
{
    const int TB = qhash_tables_per_block(s.K), units = s.B * s.Hkv;
    const uint16_t *none = nullptr;
    int32_t *no_status = nullptr, *no_flags = nullptr;
    if (s.G != 1 && s.G != 2 && s.G != 4 && s.G != 8) return cudaErrorInvalidValue;
    const int ug = qhash_units_per_block(s, s.G);
    dim3 grid((s.L + TB - 1) / TB, (units + ug - 1) / ug);
    switch (s.G) {
    case 1: return launch_pdl(qhash_kernel<1>, grid, dim3(256), 0, st, s, q, W, none, qcodes, no_status, ug, no_flags, 0);
    case 2: return launch_pdl(qhash_kernel<2>, grid, dim3(256), 0, st, s, q, W, none, qcodes, no_status, ug, no_flags, 0);
    case 4: return launch_pdl(qhash_kernel<4>, grid, dim3(256), 0, st, s, q, W, none, qcodes, no_status, ug, no_flags, 0);
    default: return launch_pdl(qhash_kernel<8>, grid, dim3(256), 0, st, s, q, W, none, qcodes, no_status, ug, no_flags, 0);
    }
}

}  // namespace mp
