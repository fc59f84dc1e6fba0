// Sampled attention on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// The estimator of MagicPIG (Chen et al. 2024) over the candidate rows a
// collision scan found: for each (sequence, kv head) unit and every query head
// h of its GQA group, out_h = sum_i w_hi v_i / sum_i w_hi with
// w_hi = exp(s_hi - log u_hi) on the sampled set S_h and exp(s_hi) on the exact
// set D, s_hi = q_h . k_i / sqrt(d).  The work is the existing split plan: an
// item is a run of candidate rows (the concatenated lists of a few scan chunks,
// or a share of one chunk's list) or the exact set D of one unit; every item
// leaves one (m, l, acc) partial per head for the merge kernel.
//
// One persistent CTA per SM takes items from a device-wide counter and walks
// them in 128-row tiles (one row per TMEM lane):
//   warps 0-3   producers: each lane copies 16-byte pieces of the tile's K and
//               V rows (cp.async) straight into 128B-swizzled shared memory,
//               plus the item's query rows; a lane's candidate entry for the
//               next tile is loaded while the current tile's copies go out;
//               copy completion arrives on the tile's barrier
//               (cp.async.mbarrier.arrive.noinc).
//   warp 4      MMA issuer (one thread) and TMEM owner: per tile
//               S = K Q^T (M = 128 rows, N = 16 heads) and the Gram matrix
//               K K^T (N = 128), whose diagonal is |k_i|^2 for the cosine of
//               the sampling probability; then, once a row group has the
//               weights, O^T += V^T P^T (M = 128 dims, N = 16 heads, V read
//               MN-major), with P split into bf16 hi + lo parts.
//   warp 5      scheduler: takes the next item, computes its row range
//               (prefix of the chunks' candidate counts) into a slot.
//   warps 6-13  two row groups of four warps, taking alternate tiles (group =
//               tile parity), thread = row: scores and |k|^2 from TMEM, log u
//               for the sampled (row, head) pairs (compacted per warp), the
//               tile's maximum per head over the group, lazy rescaling of the
//               group's running sums (only when a head's maximum grows by more
//               than 2^8), the weights P into shared memory.  Each group has
//               its own O^T accumulator in TMEM and its own running (m, l); at
//               the end of an item group 0 merges both into the item's partial
//               (thread = output dim).
// All log-weights are kept in base 2 (scores and log u scaled by log2 e).
//
// Every mbarrier wait is bounded (1 s of %globaltimer); on expiry the kernel
// records MP_ERR_CUDA in the status word, every role leaves its loop, waits
// (bounded) for its own copies and MMAs in flight, frees TMEM and exits.
#include <cuda.h>
#include <math.h>

#include <algorithm>

#include "mp_common.cuh"
#include "mp_kernels.cuh"
#include "mp_logu.cuh"

namespace mp {
namespace atc {

constexpr int kRows = 128;                       // candidate rows per tile = TMEM lanes
constexpr int kHalf = kRows * 128;               // one 64-dim half of a tile of 128 rows: 16 KB
constexpr int kStageBytes = 4 * kHalf;           // K halves, then V halves: 64 KB
constexpr int kHeadsPad = 16;                    // N of the score and P.V MMAs (>= G)
constexpr int kOpBytes = 2 * kHeadsPad * 128;    // Q^T or P^T operand: 16 rows x 128, two 64-wide halves
constexpr int kSlots = 4;                        // work items in flight
constexpr int kQBufs = 2;                        // query operands (items whose S MMAs may be in flight)
constexpr int kProdWarps = 4;
constexpr int kWarpMma = 4, kWarpSched = 5, kWarpRow0 = 6, kRowWarps = 8;
constexpr int kThreads = 32 * (kWarpRow0 + kRowWarps);  // 448
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColGram = 32, kColO = 448;   // S at 256 g, Gram at 256 g + 32, O^T at 448 + 16 g (g = group)
constexpr int kMaxSpanC = 64;
constexpr float kRescaleMargin = 8.f;            // log2 units: weights stay below 2^8 between rescales
constexpr float kLog2e = 1.4426950408889634f;

template <int G>
struct Cfg {
    static constexpr int kStages = G <= 4 ? 3 : 2;  // K/V tile ring (shared memory bounds G = 8 to 2)
};

struct Slot {
    int item;  // -1: no more work
    int unit, split, nrows, ntiles, e0, c_begin, dsplit, n_sink, win0, live;
    int cpre[kMaxSpanC + 1];
};

// Barriers (8-byte words of `bars`); S = stages.
enum {
    B_SFULL = 0,                        // [2] S and Gram of a group's tile in TMEM (commit)
    B_SFREE = B_SFULL + 2,              // [2] the group's warps have read them (count 4)
    B_PFULL = B_SFREE + 2,              // [2] the group's P written, its O^T rescaled (count 4)
    B_PVDONE = B_PFULL + 2,             // [2] P.V of the group's tile complete (commit)
    B_SLOTFULL = B_PVDONE + 2,          // [kSlots] scheduler filled the slot (count 1)
    B_SLOTEMPTY = B_SLOTFULL + kSlots,  // [kSlots] every role is done with the item (count 13)
    B_QFREE = B_SLOTEMPTY + kSlots,     // [kQBufs] the S MMAs of the buffer's last item completed (commit)
    B_RSYNC = B_QFREE + kQBufs,         // [2] the four warps of a row group meet (count 4)
    B_XSYNC = B_RSYNC + 2,              // both row groups meet at the end of an item (count 8)
    B_FINAL = B_XSYNC + 1,              // teardown: all MMAs complete
    B_FULL = B_FINAL + 1,               // [S] producers' rows + copies landed (count 256)
    B_EMPTY_BASE = B_FULL + 3           // [S] MMA done with the stage + the group read its meta (count 5)
};
constexpr int kMaxBars = B_EMPTY_BASE + 3;

// Bounded wait on a parity phase; false on abort or timeout (then every
// role stops).
__device__ __noinline__ bool wait_slow(uint32_t a, uint32_t parity, volatile int *abort_flag, int32_t *status)
{
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(a, parity)) {
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            set_status(status, MP_ERR_CUDA);
            return false;
        }
    }
    return true;
}
__device__ __forceinline__ bool wait(uint32_t a, uint32_t parity, volatile int *abort_flag, int32_t *status)
{
    return mbar_try_wait(a, parity) || wait_slow(a, parity, abort_flag, status);
}
// Every lane of a warp waits (so each acquires what the arriving threads
// wrote); the outcome is made uniform over the warp.
__device__ __forceinline__ bool warp_wait(uint32_t a, uint32_t parity, volatile int *abort_flag, int32_t *status)
{
    const bool ok = wait(a, parity, abort_flag, status);
    return __all_sync(0xffffffffu, ok);
}
// Teardown wait: bounded by time only (it runs after an abort too).
__device__ __noinline__ void wait_teardown(uint32_t a, uint32_t parity)
{
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(a, parity))
        if (globaltimer() - t0 > kWaitLimitNs) return;
}

// K-major operand, 128B swizzle: rows of 128 B, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// MN-major operand, 128B swizzle (V read as V^T): each 128-byte row holds 64
// MN-contiguous elements of one K index, 8 K-rows form a 1024-byte swizzle
// atom (SBO = 1024 B to the next 8 rows), and the second 64 MN elements lie
// `lbo` bytes further (LBO).
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t saddr, uint32_t lbo)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// kind::f16 instruction descriptor: bf16 x bf16 -> f32, M = 128, N = n; A
// MN-major when a_mn.
__device__ __forceinline__ uint32_t idesc(int n, bool a_mn)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(kRows >> 4) << 24);
}
__device__ __forceinline__ void mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id, uint32_t accum)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
            d_tmem),
        "l"(a), "l"(b), "r"(id), "r"(accum));
}
__device__ __forceinline__ void commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&r)[8])
{
    uint32_t u[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; i++) r[i] = __uint_as_float(u[i]);
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&r)[8])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(__float_as_uint(r[0])), "r"(__float_as_uint(r[1])), "r"(__float_as_uint(r[2])),
                 "r"(__float_as_uint(r[3])), "r"(__float_as_uint(r[4])), "r"(__float_as_uint(r[5])),
                 "r"(__float_as_uint(r[6])), "r"(__float_as_uint(r[7]))
                 : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&r)[32])
{
    uint32_t u[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
        "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]),
          "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]),
          "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; i++) r[i] = __uint_as_float(u[i]);
}

// The copy-completion arrive of a producer lane: triggered once all of the
// lane's earlier cp.async copies have landed (does not count as a pending
// arrival of its own).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Swizzled byte offset of 16-byte piece c (0..7) of row r in a 128B-swizzled
// block of 128-byte rows.
__device__ __forceinline__ uint32_t sw_off(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ float fast_exp2(float x)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ uint16_t bf16_rn(float x)
{
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
    return r;
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1) attend_tc_kernel(const AttendTcArgs a)
{
    static_assert(G <= 8, "up to 8 query heads per kv head");
    constexpr int S = Cfg<G>::kStages;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[kMaxBars];
    __shared__ Slot slots[kSlots];
    __shared__ int32_t ent[S][kRows];          // token of each row (-1: none)
    __shared__ uint32_t meta[S][kRows];        // head mask | 0x100 for the exact set
    __shared__ float ucos[kRowWarps][32 * G];  // per row warp: cos, then log u, of its sampled pairs
    __shared__ float red[2][2][4][8];          // [group][tile parity][warp][head] tile maxima
    __shared__ float lsum[2][4][8];            // [group][warp][head]
    __shared__ float gstate[2][8];             // group 1's m and l per head, for the merge
    __shared__ float qinv_sh[kSlots][2][8];
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_flag;

    const Shape &s = a.s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    grid_dependency_wait();  // the candidate lists are the scan's output

    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t stage0 = base;
    const uint32_t qbuf0 = base + S * kStageBytes;       // [kQBufs] Q^T operands
    const uint32_t pbuf0 = qbuf0 + kQBufs * kOpBytes;    // [group][hi, lo] P^T operands
    const uint32_t bar0 = smem_u32(&bars[0]);
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    auto full = [&](int st) { return bar(B_FULL + st); };
    auto empty = [&](int st) { return bar(B_EMPTY_BASE + st); };

    if (tid == 0) {
        abort_flag = 0;
        for (int i = 0; i < S; i++) {
            mbar_init(full(i), 2 * 32 * kProdWarps);  // each producer lane: one plain arrive, one copy-completion arrive
            mbar_init(empty(i), 5);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(bar(B_SFULL + i), 1);
            mbar_init(bar(B_SFREE + i), 4);
            mbar_init(bar(B_PFULL + i), 4);
            mbar_init(bar(B_PVDONE + i), 1);
            mbar_init(bar(B_RSYNC + i), 4);
        }
        for (int i = 0; i < kSlots; i++) {
            mbar_init(bar(B_SLOTFULL + i), 1);
            mbar_init(bar(B_SLOTEMPTY + i), kProdWarps + 1 + kRowWarps);
        }
        for (int i = 0; i < kQBufs; i++) mbar_init(bar(B_QFREE + i), 1);
        mbar_init(bar(B_XSYNC), kRowWarps);
        mbar_init(bar(B_FINAL), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kWarpMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (warp >= kWarpRow0) {
        // the padding heads G..15 of the P^T operands stay zero
        const int rt = tid - 32 * kWarpRow0;
        for (int i = rt; i < 4 * 2 * (kHeadsPad - G) * 32; i += 32 * kRowWarps) {
            const int word = i & 31, row = G + (i >> 5) % (kHeadsPad - G), blk = i / (32 * (kHeadsPad - G));
            const uint32_t addr = pbuf0 + (uint32_t)(blk * (kOpBytes / 2)) + (uint32_t)(row * 128 + word * 4);
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(0u) : "memory");
        }
        fence_proxy_async_smem();
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = tmem_base_sh;
    const int C = a.chunk_tokens;
    const int total_items = s.B * s.Hkv * a.nsplit;
    const int n_chunk_items = s.B * s.Hkv * (a.nsplit - 1);

    if (warp == kWarpSched) {
        // ------------------------------------------------------ scheduler ----
        for (int n = 0;; n++) {
            const int slot = n % kSlots;
            if (n >= kSlots && !warp_wait(bar(B_SLOTEMPTY + slot), (n / kSlots - 1) & 1, &abort_flag, a.status))
                break;
            int item = 0;
            if (lane == 0) item = atomicAdd(a.work_counter, 1);
            item = __shfl_sync(0xffffffffu, item, 0);
            Slot &sl = slots[slot];
            if (item >= total_items) {
                if (lane == 0) {
                    sl.item = -1;
                    mbar_arrive(bar(B_SLOTFULL + slot));
                }
                break;
            }
            int unit, split;
            if (item < n_chunk_items) {
                unit = item / (a.nsplit - 1);
                split = item % (a.nsplit - 1);
            } else {
                unit = item - n_chunk_items;
                split = a.nsplit - 1;
            }
            const int b = unit / s.Hkv;
            int N = a.seq_lens[b];
            N = N < 0 ? 0 : (N > a.max_len ? a.max_len : N);
            const int nch = (N + C - 1) / C;
            const bool dsplit = split == a.nsplit - 1;
            int nrows = 0, e0 = 0, live = 1, c_begin = 0;
            const int n_sink = min(s.sink, N), win0 = max(n_sink, N - s.window);
            if (dsplit) {
                nrows = n_sink + (N - win0);
            } else {
                const int grp = split / a.subs, sub = split % a.subs;
                c_begin = grp * a.span;
                if (c_begin >= nch) {
                    live = 0;
                } else {
                    const int nc = min(a.span, nch - c_begin);
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
                        if (j < nc) sl.cpre[j + 1] = run + incl;
                        run += __shfl_sync(0xffffffffu, incl, 31);
                    }
                    const int total = run, per = (total + a.subs - 1) / a.subs;
                    e0 = min(total, sub * per);
                    nrows = min(total, e0 + per) - e0;
                    // past the item's chunks the cursor walk must stop
                    if (lane == 0) sl.cpre[0] = 0;
                    for (int j = nc + 1 + lane; j <= kMaxSpanC; j += 32) sl.cpre[j] = 0x7FFFFFFF;
                }
            }
            if (lane == 0) {
                sl.item = item;
                sl.unit = unit;
                sl.split = split;
                sl.nrows = nrows;
                sl.ntiles = live ? (nrows + kRows - 1) / kRows : 0;
                sl.e0 = e0;
                sl.c_begin = c_begin;
                sl.dsplit = dsplit ? 1 : 0;
                sl.n_sink = n_sink;
                sl.win0 = win0;
                sl.live = live;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SLOTFULL + slot));
        }
    } else if (warp < kProdWarps) {
        // ------------------------------------------------------ producers ----
        const int pw = warp, ptid = pw * 32 + lane;  // ptid: the tile row whose entry this lane fetches
        const uint32_t dmeta = ((1u << G) - 1u) | 0x100u;
        const int ck = lane & 15, kh = ck >> 3, c = ck & 7;  // this lane's 16-byte piece of a row
        int seq = 0, nq = 0;  // tiles issued, items with rows
        for (int n = 0;; n++) {
            const int slot = n % kSlots;
            if (!warp_wait(bar(B_SLOTFULL + slot), (n / kSlots) & 1, &abort_flag, a.status)) break;
            const Slot &sl = slots[slot];
            if (sl.item < 0) break;
            bool ok = true;
            if (sl.ntiles > 0) {
                const int unit = sl.unit, b = unit / s.Hkv, kvh = unit % s.Hkv;
                const uint16_t *kbase = a.kc + (size_t)unit * s.Ncap * kHeadDim;
                const uint16_t *vbase = a.vc + (size_t)unit * s.Ncap * kHeadDim;
                const uint32_t *lists = a.cand + ((size_t)unit * a.nchunk + sl.c_begin) * C;
                const size_t vec0 = (size_t)b * s.Hq + (size_t)kvh * G;
                int jc = 0;  // chunk of this lane's next candidate (rows are visited in increasing order)
                // entry of row ptid of tile t: token | head mask << 24, all ones if none
                auto fetch = [&](int t) -> uint32_t {
                    const int e = t * kRows + ptid;
                    if (e >= sl.nrows) return 0xFFFFFFFFu;
                    if (sl.dsplit) return (uint32_t)(e < sl.n_sink ? e : sl.win0 + (e - sl.n_sink));
                    const int x = sl.e0 + e;
                    while (sl.cpre[jc + 1] <= x) jc++;
                    return lists[(size_t)jc * C + (x - sl.cpre[jc])];
                };
                uint32_t en = fetch(0);
                const int qb_i = nq % kQBufs;
                if (nq >= kQBufs &&
                    !warp_wait(bar(B_QFREE + qb_i), (nq / kQBufs - 1) & 1, &abort_flag, a.status))
                    ok = false;
                for (int t = 0; ok && t < sl.ntiles; t++, seq++) {
                    const int st = seq % S, k = seq / S;
                    if (k >= 1 && !warp_wait(empty(st), (k - 1) & 1, &abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    const bool none = en == 0xFFFFFFFFu;
                    ent[st][ptid] = none ? -1 : (sl.dsplit ? (int)en : (int)(en & 0xFFFFFFu));
                    meta[st][ptid] = none ? 0u : (sl.dsplit ? dmeta : en >> 24);
                    if (t + 1 < sl.ntiles) en = fetch(t + 1);  // in flight while this tile's copies go out
                    __syncwarp();
                    mbar_arrive(full(st));  // this lane's row entry and head mask are written
                    const uint32_t sb = stage0 + (uint32_t)(st * kStageBytes);
                    if (t == 0) {
                        // the item's query rows (Q^T operand); rows G..15 zero-filled
                        const uint32_t qb = qbuf0 + (uint32_t)(qb_i * kOpBytes);
#pragma unroll
                        for (int j = 0; j < 2; j++) {
                            const int idx = ptid + 128 * j, h = idx >> 4, qk = idx & 15, qh = qk >> 3, qc = qk & 7;
                            const uint16_t *src = a.q + (vec0 + (h < G ? h : 0)) * kHeadDim + qh * 64 + qc * 8;
                            cp_async_16_s(qb + (uint32_t)(qh * (kOpBytes / 2)) + sw_off(h, qc), src, h < G ? 16 : 0);
                        }
                    }
                    // K and V rows 32 pw .. 32 pw + 31: two rows per warp-wide step
#pragma unroll 4
                    for (int it = 0; it < 16; it++) {
                        const int r = pw * 32 + 2 * it + (lane >> 4);
                        const int tok = ent[st][r];
                        const size_t off = (size_t)(tok < 0 ? 0 : tok) * kHeadDim + kh * 64 + c * 8;
                        const uint32_t d = sb + (uint32_t)(kh * kHalf) + sw_off(r, c);
                        const int nb = tok < 0 ? 0 : 16;
                        cp_async_16_s(d, kbase + off, nb);
                        cp_async_16_s(d + 2 * kHalf, vbase + off, nb);
                    }
                    cp_async_arrive_noinc(full(st));
                }
                nq++;
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SLOTEMPTY + slot));
        }
        cp_async_wait<0>();
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------------ MMA ----
        if (lane == 0) {
            const uint32_t id_s = idesc(kHeadsPad, false), id_g = idesc(kRows, false), id_pv = idesc(kHeadsPad, true);
            int seq = 0, nq = 0;
            int pend_seq = -1, pend_st = 0, pend_first = 0;
            // P.V of the pending tile into its group's O^T
            auto do_pv = [&]() -> bool {
                const int g = pend_seq & 1;
                if (!wait(bar(B_PFULL + g), (pend_seq >> 1) & 1, &abort_flag, a.status)) return false;
                fence_after();
                const uint32_t vb = stage0 + (uint32_t)(pend_st * kStageBytes) + 2 * kHalf;
                const uint32_t phi = pbuf0 + (uint32_t)((g * 2 + 0) * kOpBytes);
                const uint32_t plo = pbuf0 + (uint32_t)((g * 2 + 1) * kOpBytes);
                const uint32_t d = tmem + kColO + 16u * (uint32_t)g;
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const uint64_t ad = desc_mnmajor(vb + (uint32_t)(j * 16 * 128), kHalf);
                    const uint32_t boff = (uint32_t)((j >> 2) * (kOpBytes / 2) + (j & 3) * 32);
                    mma(d, ad, desc_kmajor(phi + boff), id_pv, (pend_first && j == 0) ? 0u : 1u);
                    mma(d, ad, desc_kmajor(plo + boff), id_pv, 1u);
                }
                commit(bar(B_PVDONE + g));
                commit(empty(pend_st));
                pend_seq = -1;
                return true;
            };
            bool ok = true;
            for (int n = 0; ok; n++) {
                const int slot = n % kSlots;
                if (!wait(bar(B_SLOTFULL + slot), (n / kSlots) & 1, &abort_flag, a.status)) break;
                const Slot &sl = slots[slot];
                if (sl.item < 0) break;
                const int ntiles = sl.ntiles;
                const uint32_t qb = qbuf0 + (uint32_t)((nq % kQBufs) * kOpBytes);
                for (int t = 0; t < ntiles; t++, seq++) {
                    const int st = seq % S, k = seq / S, g = seq & 1, kg = seq >> 1;
                    if (!wait(full(st), k & 1, &abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_smem();  // the rows arrived by cp.async (generic proxy)
                    if (kg >= 1 && !wait(bar(B_SFREE + g), (kg - 1) & 1, &abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    fence_after();
                    const uint32_t kb0 = stage0 + (uint32_t)(st * kStageBytes);
                    const uint32_t ds = tmem + (uint32_t)(g * 256), dg = ds + kColGram;
#pragma unroll
                    for (int kh = 0; kh < 2; kh++)
#pragma unroll
                        for (int ks = 0; ks < 4; ks++) {
                            const uint64_t ad = desc_kmajor(kb0 + (uint32_t)(kh * kHalf + ks * 32));
                            const uint64_t bq = desc_kmajor(qb + (uint32_t)(kh * (kOpBytes / 2) + ks * 32));
                            mma(ds, ad, bq, id_s, (kh | ks) != 0);
                            mma(dg, ad, ad, id_g, (kh | ks) != 0);
                        }
                    commit(bar(B_SFULL + g));
                    if (t == ntiles - 1) commit(bar(B_QFREE + nq % kQBufs));  // the item's last S MMAs
                    if (pend_seq >= 0 && !do_pv()) {
                        ok = false;
                        break;
                    }
                    pend_seq = seq;
                    pend_st = st;
                    pend_first = t < 2;  // the group's first tile of the item: its O^T starts over
                }
                if (!ok) break;
                if (pend_seq >= 0 && !do_pv()) break;
                if (ntiles > 0) nq++;
                commit(bar(B_SLOTEMPTY + slot));  // arrives once every MMA of the item has completed
            }
            commit(bar(B_FINAL));
            wait_teardown(bar(B_FINAL), 0);
        }
        __syncwarp();
    } else if (warp >= kWarpRow0) {
        // ------------------------------------------------------- row groups ----
        const int rw = warp - kWarpRow0, grp = rw >> 2, q4 = warp & 3;  // q4: TMEM lane quarter of this warp
        const int r = q4 * 32 + lane;
        const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
        const uint32_t o_col = kColO + 16u * (uint32_t)grp;
        const float scale2 = a.scale * kLog2e;
        float *uc = ucos[rw];
        int seq = 0, rs = 0, xs = 0;  // tiles of the CTA so far, group meetings, cross-group meetings held
        bool ok = true;
        // the four warps of the group meet (a bounded mbarrier round instead
        // of a named barrier, so that a warp leaving on a timed-out wait
        // cannot strand the others)
        auto rsync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_RSYNC + grp));
            return warp_wait(bar(B_RSYNC + grp), (rs++) & 1, &abort_flag, a.status);
        };
        auto xsync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_XSYNC));
            return warp_wait(bar(B_XSYNC), (xs++) & 1, &abort_flag, a.status);
        };
        for (int n = 0; ok; n++) {
            const int slot = n % kSlots;
            if (!warp_wait(bar(B_SLOTFULL + slot), (n / kSlots) & 1, &abort_flag, a.status)) break;
            const Slot &sl = slots[slot];
            if (sl.item < 0) break;
            if (!sl.live) {
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_SLOTEMPTY + slot));
                continue;
            }
            const int unit = sl.unit, b = unit / s.Hkv, kvh = unit % s.Hkv;
            const size_t vec0 = (size_t)b * s.Hq + (size_t)kvh * G;
            // 1 / |q_h| of the group's heads (warp q4 of the group takes heads q4, q4 + 4)
            for (int h = q4; h < G; h += 4) {
                const uint2 qv = reinterpret_cast<const uint2 *>(a.q + (vec0 + h) * kHeadDim)[lane];
                const float x0 = bf16_lo(qv.x), x1 = bf16_hi(qv.x), x2 = bf16_lo(qv.y), x3 = bf16_hi(qv.y);
                float qq = x0 * x0 + x1 * x1 + x2 * x2 + x3 * x3;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) qq += __shfl_xor_sync(0xffffffffu, qq, o);
                if (lane == 0) qinv_sh[slot][grp][h] = qq > 0.f ? rsqrtf(qq) : 0.f;
            }
            if (!rsync()) break;
            float qinv[G], m_run[G], l_part[G];
#pragma unroll
            for (int h = 0; h < G; h++) {
                qinv[h] = qinv_sh[slot][grp][h];
                m_run[h] = -INFINITY;
                l_part[h] = 0.f;
            }
            const int seq0 = seq;
            int mine = 0;  // this group's tiles of the item so far
            for (int t = 0; t < sl.ntiles; t++) {
                const int sq = seq0 + t;
                if ((sq & 1) != grp) continue;  // the other group's tile
                const int st = sq % S, k = sq / S, kg = sq >> 1;
                if (!warp_wait(full(st), k & 1, &abort_flag, a.status)) {
                    ok = false;
                    break;
                }
                const uint32_t mrow = meta[st][r];
                __syncwarp();
                if (lane == 0) mbar_arrive(empty(st));
                if (!warp_wait(bar(B_SFULL + grp), kg & 1, &abort_flag, a.status)) {
                    ok = false;
                    break;
                }
                fence_after();
                float sc[8], g32[32];
                tmem_ld8(tmem + lane_base + (uint32_t)(grp * 256), sc);
                tmem_ld32(tmem + lane_base + (uint32_t)(grp * 256) + kColGram + (uint32_t)(q4 * 32), g32);
                wait_ld();
                fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_SFREE + grp));
                // |k_r|^2 = Gram[r][r]: element `lane` of this thread's 32 columns
#pragma unroll
                for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
                    for (int j = 0; j < w; j++) g32[j] = (lane & w) ? g32[j + w] : g32[j];
                const float kn2 = g32[0];
                const float kinv = kn2 > 0.f ? rsqrtf(kn2) : 0.f;
                // log-weights (log2 units): s, minus log2 u for the sampled pairs
                float tv[G];
                int pos[G];
                bool need[G];
                int npair = 0;
#pragma unroll
                for (int h = 0; h < G; h++) {
                    const bool mem = (mrow >> h) & 1u;
                    need[h] = mem && !(mrow & 0x100u);
                    tv[h] = mem ? sc[h] * scale2 : -INFINITY;
                    const uint32_t bal = __ballot_sync(0xffffffffu, need[h]);
                    pos[h] = npair + __popc(bal & ((1u << lane) - 1u));
                    if (need[h]) uc[pos[h]] = sc[h] * qinv[h] * kinv;
                    npair += __popc(bal);
                }
                __syncwarp();
                for (int i = lane; i < npair; i += 32) uc[i] = log_sampling_prob(uc[i], a.lu);
                __syncwarp();
#pragma unroll
                for (int h = 0; h < G; h++)
                    if (need[h]) tv[h] = fmaf(-kLog2e, uc[pos[h]], tv[h]);
                // the tile's maximum per head over its 128 rows
                float mx[G];
#pragma unroll
                for (int h = 0; h < G; h++) {
                    mx[h] = tv[h];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
                }
                if (lane < G) {
                    float v = mx[0];
#pragma unroll
                    for (int h = 1; h < G; h++)
                        if (lane == h) v = mx[h];
                    red[grp][mine & 1][q4][lane] = v;
                }
                if (!rsync()) {
                    ok = false;
                    break;
                }
                float alpha[G];
                bool rescale = false;
#pragma unroll
                for (int h = 0; h < G; h++) {
                    const float (&rr)[4][8] = red[grp][mine & 1];
                    const float tm = fmaxf(fmaxf(rr[0][h], rr[1][h]), fmaxf(rr[2][h], rr[3][h]));
                    alpha[h] = 1.f;
                    if (mine == 0) {
                        m_run[h] = tm;  // the group's first P.V of the item overwrites its O^T
                    } else if (tm > m_run[h] + kRescaleMargin || (m_run[h] == -INFINITY && tm > -INFINITY)) {
                        alpha[h] = m_run[h] == -INFINITY ? 0.f : fast_exp2(m_run[h] - tm);
                        m_run[h] = tm;
                        rescale = true;
                    }
                }
                // the group's previous P.V (tile sq - 2) must be complete before its
                // O^T is rescaled or its P operand rewritten
                if (sq >= 2 && !warp_wait(bar(B_PVDONE + grp), ((sq - 2) >> 1) & 1, &abort_flag, a.status)) {
                    ok = false;
                    break;
                }
                if (rescale) {  // uniform over the group (same maxima)
                    fence_after();
                    float o[8];
                    tmem_ld8(tmem + lane_base + o_col, o);
                    wait_ld();
#pragma unroll
                    for (int h = 0; h < G; h++) o[h] *= alpha[h];
                    tmem_st8(tmem + lane_base + o_col, o);
                    wait_st();
                    fence_before();
#pragma unroll
                    for (int h = 0; h < G; h++) l_part[h] *= alpha[h];
                }
                float p[G];
#pragma unroll
                for (int h = 0; h < G; h++) {
                    p[h] = (tv[h] == -INFINITY || m_run[h] == -INFINITY) ? 0.f : fast_exp2(tv[h] - m_run[h]);
                    l_part[h] += p[h];
                }
                {
                    // P^T (bf16 hi + lo) into the group's operands
                    const uint32_t phi = pbuf0 + (uint32_t)((grp * 2 + 0) * kOpBytes);
                    const uint32_t plo = pbuf0 + (uint32_t)((grp * 2 + 1) * kOpBytes);
                    const int kh = r >> 6, kk = r & 63;
#pragma unroll
                    for (int h = 0; h < G; h++) {
                        const uint32_t off = (uint32_t)(kh * (kOpBytes / 2) + h * 128 +
                                                        (((kk >> 3) ^ (h & 7)) << 4) + (kk & 7) * 2);
                        const uint16_t hi = bf16_rn(p[h]);
                        const float hif = __uint_as_float((uint32_t)hi << 16);
                        const uint16_t lo = bf16_rn(p[h] - hif);
                        asm volatile("st.shared.u16 [%0], %1;" ::"r"(phi + off), "h"(hi) : "memory");
                        asm volatile("st.shared.u16 [%0], %1;" ::"r"(plo + off), "h"(lo) : "memory");
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_PFULL + grp));
                mine++;
            }
            if (!ok) break;
            seq = seq0 + sl.ntiles;
            // ---- the group's running sums over the item ----
#pragma unroll
            for (int h = 0; h < G; h++) {
                float v = l_part[h];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == 0) lsum[grp][q4][h] = v;
            }
            if (!rsync()) break;
            float lg[G];
#pragma unroll
            for (int h = 0; h < G; h++) lg[h] = lsum[grp][0][h] + lsum[grp][1][h] + lsum[grp][2][h] + lsum[grp][3][h];
            // the group's last P.V of the item must be complete before O^T is read
            if (mine > 0) {
                int last = seq - 1;
                if ((last & 1) != grp) last--;
                if (!warp_wait(bar(B_PVDONE + grp), (last >> 1) & 1, &abort_flag, a.status)) break;
            }
            if (grp == 1 && r < G) {
                gstate[0][r] = mine > 0 ? m_run[r] : -INFINITY;
                gstate[1][r] = mine > 0 ? lg[r] : 0.f;
            }
            fence_before();
            if (!xsync()) break;  // group 1's state is published, both groups' O^T complete
            if (grp == 0) {
                fence_after();
                const int tiles1 = sl.ntiles - (sl.ntiles + 1 - (seq0 & 1)) / 2;  // tiles of group 1
                const int tiles0 = sl.ntiles - tiles1;
                float o0[8], o1[8];
                if (tiles0 > 0) tmem_ld8(tmem + lane_base + kColO, o0);
                if (tiles1 > 0) tmem_ld8(tmem + lane_base + kColO + 16, o1);
                wait_ld();
                fence_before();
                const size_t nsp = (size_t)a.nsplit;
#pragma unroll
                for (int h = 0; h < G; h++) {
                    const float m0 = tiles0 > 0 ? m_run[h] : -INFINITY, l0 = tiles0 > 0 ? lg[h] : 0.f;
                    const float m1 = gstate[0][h], l1 = gstate[1][h];
                    const float M = fmaxf(m0, m1);
                    const float f0 = m0 == -INFINITY ? 0.f : fast_exp2(m0 - M);
                    const float f1 = m1 == -INFINITY ? 0.f : fast_exp2(m1 - M);
                    const float acc = (f0 > 0.f ? o0[h] * f0 : 0.f) + (f1 > 0.f ? o1[h] * f1 : 0.f);
                    const size_t pidx = (vec0 + h) * nsp + sl.split;
                    a.pacc[pidx * kHeadDim + r] = acc;
                    if (r == 0) {
                        a.pm[pidx] = M;
                        a.pl[pidx] = l0 * f0 + l1 * f1;
                    }
                }
            }
            if (!xsync()) break;  // O^T read: the next item's P.V may overwrite it
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SLOTEMPTY + slot));
        }
    }

    fence_before();
    __syncthreads();
    fence_after();
    if (warp == kWarpMma) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

}  // namespace atc

template <int G>
static size_t attend_tc_smem_g()
{
    return 1024 + (size_t)atc::Cfg<G>::kStages * atc::kStageBytes + (size_t)(atc::kQBufs + 4) * atc::kOpBytes;
}

size_t attend_tc_smem_bytes() { return attend_tc_smem_g<8>() > attend_tc_smem_g<4>() ? attend_tc_smem_g<8>() : attend_tc_smem_g<4>(); }

template <int G>
static cudaError_t launch_attend_tc_g(const AttendTcArgs &a, cudaStream_t st)
{
    const void *fn = reinterpret_cast<const void *>(atc::attend_tc_kernel<G>);
    const int smem = (int)attend_tc_smem_g<G>();
    cudaError_t e = ensure_smem(fn, smem);
    if (e != cudaSuccess) return e;
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    }
    const long long items = (long long)a.s.B * a.s.Hkv * a.nsplit;
    const int grid = (int)std::max(1LL, std::min(items, (long long)sms));
    return launch_pdl(atc::attend_tc_kernel<G>, dim3(grid), dim3(atc::kThreads), (size_t)smem, st, a);
}

cudaError_t launch_attend_tc(const AttendTcArgs &a, cudaStream_t st)
{
    switch (a.s.G) {
    case 1: return launch_attend_tc_g<1>(a, st);
    case 2: return launch_attend_tc_g<2>(a, st);
    case 4: return launch_attend_tc_g<4>(a, st);
    case 8: return launch_attend_tc_g<8>(a, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace mp
