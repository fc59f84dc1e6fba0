// SimHash of cached keys on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// The projection of every key row onto the L*K hyperplanes of W is a dense
// bf16 contraction (rows x 128) . (128 x L*K) with fp32 accumulation, so it
// runs as a persistent, warp-specialised GEMM whose epilogue never writes the
// fp32 product: it turns each accumulator value into a sign bit (strictly
// positive -> 1, the SimHash rule of MagicPIG, Chen et al. 2024) and packs the
// bits straight into the table-major code layout.
//
//   warp 0      TMA producer: the W column group (resident in shared memory,
//               reloaded only when a CTA moves to the next group; one barrier
//               per 256-column tile, so the first MMAs wait for one tile
//               only) and a 2-stage ring of 128-row key tiles, 128B-swizzled.
//   warp 1      MMA issuer (one thread): tcgen05.mma kind::f16, M = 128,
//               N <= 256, K = 16, into one of two TMEM accumulators (N = 256
//               keeps the operand traffic per flop within shared-memory
//               bandwidth).
//   warp 2      TMEM allocator (512 columns = 2 x 256-column accumulators).
//   warps 4..19 epilogue, four groups of four warps, each group one 64-column
//               slice of every column tile: tcgen05.ld 32x32b (thread = key
//               row, registers = columns), release of the accumulator, then
//               sign test, pack, store off the MMA's critical path.  Each
//               thread packs the sign bits of 32 columns of its row into a
//               word (one funnel shift per column; the MMA negates the keys,
//               so a set sign bit means a positive projection); byte codes then
//               swap bytes within lane quads (4 tokens of one table per 32-bit
//               store), bit planes transpose the 32x32 bit matrix across the
//               warp (one plane word per lane).
//
// Column groups: W has L*K rows (hyperplanes); a group of at most 640 rows
// (608 for K = 8, L = 75) stays resident; K = 10, L = 150 uses 3 groups of
// <= 512.  Each block keeps one group for the whole launch, and the blocks of
// the different groups walk the same key tiles side by side, so a key tile
// is read from DRAM once and from L2 by the other groups' blocks.
//
// Every wait on an mbarrier is bounded (1 s of %globaltimer); on expiry the
// kernel records MP_ERR_CUDA in the status word, skips the rest of its work,
// waits (bounded) for its own copies and MMAs in flight, frees TMEM and exits.
#include <cuda.h>

#include "mp_common.cuh"
#include "mp_kernels.cuh"

namespace mp {
namespace tc {

#ifndef MP_HASH_EPI_GROUPS
#define MP_HASH_EPI_GROUPS 4
#endif
constexpr int kEpiGroups = MP_HASH_EPI_GROUPS;  // epilogue groups of 4 warps, one column slice each
constexpr int kThreads = 128 + 128 * kEpiGroups;
constexpr int kBM = 128;                     // key rows per tile = TMEM lanes
constexpr int kAccCols = 256;                // columns per accumulator buffer
constexpr int kAccBufs = 2;                  // 2 x 256 = all 512 TMEM columns
constexpr int kLensCache = 256;              // sequence lengths kept in shared memory
constexpr int kSliceCols = kAccCols / kEpiGroups;  // columns of a tile per epilogue group
constexpr int kStages = 2;                   // key-tile ring depth
constexpr int kPrefetchAhead = 3;            // key tiles (of this block) kept in flight to L2
constexpr int kHalfBytes = kBM * 128;        // one 64-element (128 B) K half of a tile
constexpr int kTileBytes = 2 * kHalfBytes;   // 32 KB
constexpr int kMaxGroupCols = 640;
constexpr int kMaxWChunks = (kMaxGroupCols + kAccCols - 1) / kAccCols;  // column tiles of a group
constexpr int kWBox = 32;                    // W rows per TMA box

struct Params {
    Shape s;
    const int32_t *seq_lens;
    void *codes;
    int32_t *status;
    int tok0;        // first token of the hashed range (multiple of kBM)
    int n_tokens;    // tokens of the range
    int n_mt;        // 128-row tiles per unit
    int ngroups;
    int gsize;       // columns per group (multiple of 32)
    int gpad_max;    // padded width of the widest group (multiple of 32)
    int total_items; // units * n_mt (every block hashes its items for its own column group)
    uint32_t kmagic; // floor(2^32 / K) + 1: c / K = umulhi(c, kmagic) while c K < 2^32
    uint32_t hmagic; // floor(2^32 / Hkv) + 1: batch of unit u = umulhi(u, hmagic)
};

// Bounded wait for the phase of parity `parity`; false on abort or timeout.
// The first test is inline; only a phase that is not yet complete takes the
// out-of-line polling loop.
__device__ __noinline__ bool mbar_wait_slow(uint32_t a, uint32_t parity, volatile int *abort_flag, int32_t *status)
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
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity, volatile int *abort_flag, int32_t *status)
{
    if (mbar_try_wait(a, parity)) return true;
    return mbar_wait_slow(a, parity, abort_flag, status);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

// Pulls a future key tile into L2 (no shared memory, no completion tracking),
// so that the ring's real load later finds it there.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *map, int x, int y)
{
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y)
                 : "memory");
}

// K-major, 128B-swizzled operand: rows of 128 B, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::f16 instruction descriptor: bf16 x bf16 -> f32, both K-major, M = 128,
// A (the keys) negated (bit 13).  The accumulator is then -(k . w_c), computed
// exactly like k . w_c up to the sign (round-to-nearest is symmetric), and its
// sign bit is 1 iff k . w_c > 0: a projection that cancels to zero gives +0,
// sign 0, as the strict rule wants.
__device__ __forceinline__ uint32_t idesc_bf16(int n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 13) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(kBM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accum)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
            d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accum));
}
__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
        "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32-bit word whose bit c is the sign bit of v[c]: with the keys negated in
// the MMA (idesc_bf16), that bit is [k . w_c > 0].  One funnel shift per
// column moves the sign into the running word; two independent chains of 16
// columns halve the dependent latency.
__device__ __forceinline__ uint32_t pack_signs32(const uint32_t *v)
{
    uint32_t lo = 0u, hi = 0u;
#pragma unroll
    for (int c = 15; c >= 0; c--) {
        lo = __funnelshift_l(v[c], lo, 1);  // (lo << 1) | (v[c] >> 31)
        hi = __funnelshift_l(v[16 + c], hi, 1);
    }
    return __byte_perm(lo, hi, 0x5410);
}

// Within each group of 4 lanes, transposes the 4x4 byte matrix whose row r
// (lane r of the group) is the word x: afterwards lane r holds byte r of every
// lane of its group, in lane order.  sel1 / sel2 are the lane's byte
// selectors (quad_selectors).
__device__ __forceinline__ uint32_t quad_transpose(uint32_t x, uint32_t sel1, uint32_t sel2)
{
    uint32_t y = __shfl_xor_sync(0xffffffffu, x, 1);
    x = __byte_perm(x, y, sel1);
    y = __shfl_xor_sync(0xffffffffu, x, 2);
    return __byte_perm(x, y, sel2);
}
__device__ __forceinline__ void quad_selectors(int lane, uint32_t &sel1, uint32_t &sel2)
{
    sel1 = (lane & 1) ? 0x3715u : 0x6240u;
    sel2 = (lane & 2) ? 0x3276u : 0x5410u;
}

// 32x32 bit-matrix transpose across a warp: lane t holds row t; afterwards
// lane c holds column c (bit t of the result = bit c of lane t's input).
// Stage j (16, 8, 4, 2, 1) swaps j x j blocks with the lane j apart: the lane
// keeps the bits under keep[k] and takes the rest from the partner's word
// rotated by rot[k] (j or 32 - j), one shuffle, one funnel shift and one
// three-input logic op per stage.  keep / rot come from transpose_consts.
__device__ __forceinline__ uint32_t warp_transpose32(uint32_t x, const uint32_t (&keep)[5], const uint32_t (&rot)[5])
{
#pragma unroll
    for (int k = 0; k < 5; k++) {
        const uint32_t y = __shfl_xor_sync(0xffffffffu, x, 16 >> k);
        const uint32_t r = __funnelshift_r(y, y, rot[k]);
        uint32_t d;
        asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(d) : "r"(x), "r"(r), "r"(keep[k]));  // (x & keep) | (r & ~keep)
        x = d;
    }
    return x;
}
__device__ __forceinline__ void transpose_consts(int lane, uint32_t (&keep)[5], uint32_t (&rot)[5])
{
    const uint32_t masks[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
    for (int k = 0; k < 5; k++) {
        const int j = 16 >> k;
        keep[k] = (lane & j) ? ~masks[k] : masks[k];
        rot[k] = (lane & j) ? (uint32_t)j : (uint32_t)(32 - j);
    }
}

struct Item {
    int group, unit, mt, len;
    bool skip;
};

__device__ __forceinline__ Item make_item(const Params &p, int group, int unit, int mt, const int *lens_sh)
{
    Item r;
    r.group = group;
    r.unit = unit;
    r.mt = mt;
    int len = p.tok0 + p.n_tokens;  // end of the range (absolute token index)
    if (p.seq_lens) {
        const int b = (int)__umulhi((uint32_t)unit, p.hmagic);  // unit / Hkv
        len = min(len, max(b < kLensCache ? lens_sh[b] : p.seq_lens[b], 0));
    }
    r.len = len;
    r.skip = p.tok0 + r.mt * kBM >= len;
    return r;
}

// A block keeps one column group for the whole launch: block x takes group
// x % ngroups and, of the (unit, tile) items, x / ngroups + k S for k = 0,
// 1, ... (S = gridDim.x / ngroups; the grid is a multiple of ngroups).  The
// ngroups blocks x = ngroups j + g walk the same key tiles side by side, so
// each tile comes from DRAM once and from L2 for the other groups, and W is
// loaded once per block.
__device__ __forceinline__ int block_group(const Params &p) { return (int)blockIdx.x % p.ngroups; }
__device__ __forceinline__ int item_stride(const Params &p) { return (int)gridDim.x / p.ngroups; }

__device__ __forceinline__ Item item_of(const Params &p, int it, const int *lens_sh)
{
    return make_item(p, block_group(p), it / p.n_mt, it % p.n_mt, lens_sh);
}

// The (unit, tile) items of this block, advanced with carries instead of
// divisions.
struct ItemIter {
    int it, group, unit, mt;
    int step, du, dm;  // the stride in the same mixed radix
    __device__ __forceinline__ explicit ItemIter(const Params &p)
    {
        group = block_group(p);
        it = (int)blockIdx.x / p.ngroups;
        mt = it % p.n_mt;
        unit = it / p.n_mt;
        step = item_stride(p);
        dm = step % p.n_mt;
        du = step / p.n_mt;
    }
    __device__ __forceinline__ bool live(const Params &p) const { return it < p.total_items; }
    __device__ __forceinline__ void next(const Params &p)
    {
        it += step;
        mt += dm;
        unit += du;
        if (mt >= p.n_mt) {
            mt -= p.n_mt;
            unit++;
        }
    }
    __device__ __forceinline__ Item item(const Params &p, const int *lens_sh) const
    {
        return make_item(p, group, unit, mt, lens_sh);
    }
};

// Columns [c0, c0 + width) of a group; width is a multiple of 32.
__device__ __forceinline__ void group_cols(const Params &p, int g, int &c0, int &width)
{
    c0 = g * p.gsize;
    const int real = min(p.gsize, p.s.LK - c0);
    width = (real + 31) & ~31;
}

// Where an epilogue warp writes the codes of one 128-row tile.
struct TileDst {
    uint8_t *bytes;    // byte codes: this lane's 4-token group, table 0
    uint32_t *planes;  // bit planes: this warp's 32-token word, table 0, bit 0
    int t4;            // byte codes: first token of this lane's group
    int len;
    bool full4, valid, warp_live;
};

// Sign-packs and stores NCH 32-column chunks of one accumulator slice.
template <bool PLANES, int NCH>
__device__ __forceinline__ void epilogue_slice(const Params &p, const TileDst &td, uint32_t ta, uint32_t empty_bar,
                                               int col0, int lane, uint32_t sel1, uint32_t sel2,
                                               const uint32_t (&keep)[5], const uint32_t (&rot)[5])
{
    const Shape &s = p.s;
    uint32_t v[NCH][32];
#pragma unroll
    for (int q = 0; q < NCH; q++) tmem_ld32(ta + 32 * q, v[q]);
    tmem_wait_ld();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar);  // the warp's values are in registers: free the accumulator
#pragma unroll
    for (int q = 0; q < NCH; q++) {
        const int c32 = col0 + 32 * q;  // first global column of these 32
        if (!PLANES) {
            // 4 table bytes of this token -> 4 tokens of one table per lane
            const uint32_t w = quad_transpose(pack_signs32(v[q]), sel1, sel2);
            const int l = (c32 >> 3) + (lane & 3);
            if (l < s.L) {
                uint8_t *dst = td.bytes + (size_t)l * s.Ncap;
                if (td.full4) {
                    *reinterpret_cast<uint32_t *>(dst) = w;
                } else {
                    for (int k = 0; k < 4 && td.t4 + k < td.len; k++) dst[k] = (uint8_t)(w >> (8 * k));
                }
            }
        } else {
            // row word (bit c = column c32 + c) -> column word (bit t = token t)
            const uint32_t rw = td.valid ? pack_signs32(v[q]) : 0u;
            const uint32_t mine = warp_transpose32(rw, keep, rot);
            const uint32_t c = (uint32_t)(c32 + lane);
            if (td.warp_live && c < (uint32_t)s.LK) {
                const uint32_t l = __umulhi(c, p.kmagic), b = c - l * (uint32_t)s.K;
                td.planes[(size_t)l * (s.Ncap >> 5) * s.K + b] = mine;
            }
        }
    }
}

// Epilogue warps (4 .. 4 + 4 * kEpiGroups - 1).  Every epilogue warp takes
// part in every column tile: group eg owns columns [64 eg, 64 eg + 64) of the
// tile, warp quarter q4 owns rows [32 q4, 32 q4 + 32).  The accumulator is
// released as soon as its values are in registers, so packing and storing
// overlap the next MMAs.  Each slice width has its own straight-line path.
template <bool PLANES>
__device__ __forceinline__ void epilogue(const Params &p, const int *lens_sh, uint32_t tmem_base, uint32_t bar0,
                                         volatile int *abort_flag, int warp, int lane)
{
    static_assert(kSliceCols == 64, "slices of 0, 32 or 64 columns");
    const Shape &s = p.s;
    const int q4 = warp & 3;         // TMEM lane quarter of this warp
    const int eg = (warp - 4) >> 2;  // column slice of every tile
    const int row = q4 * 32 + lane;
    const int words = s.Ncap >> 5;
    int seq = 0;                     // column-tile sequence number
    uint32_t sel1, sel2, keep[5], rot[5];
    quad_selectors(lane, sel1, sel2);
    transpose_consts(lane, keep, rot);
    for (ItemIter iter(p); iter.live(p) && !*abort_flag; iter.next(p)) {
        const Item im = iter.item(p, lens_sh);
        if (im.skip) continue;
        int c0, width;
        group_cols(p, im.group, c0, width);
        TileDst td;
        td.len = im.len;
        const int tile0 = p.tok0 + im.mt * kBM;  // first token of this row tile
        td.valid = tile0 + row < im.len;
        td.warp_live = tile0 + q4 * 32 < im.len;
        td.t4 = tile0 + q4 * 32 + (lane & ~3);
        td.full4 = td.t4 + 3 < im.len;
        td.bytes = static_cast<uint8_t *>(p.codes) + (size_t)im.unit * s.L * s.Ncap + td.t4;
        td.planes = static_cast<uint32_t *>(p.codes) + (size_t)im.unit * s.L * words * s.K +
                    ((tile0 + q4 * 32) >> 5) * s.K;
        for (int n0 = 0; n0 < width; n0 += kAccCols, seq++) {
            const int acc = seq & (kAccBufs - 1);
            const int nw = min(kAccCols, width - n0);
            const int ch = eg * kSliceCols;                  // this group's slice of the tile
            const int sw = max(0, min(kSliceCols, nw - ch));  // 0, 32 or 64
            const uint32_t full = bar0 + 8u * (4 + acc), empty = bar0 + 8u * (8 + acc);
            if (!mbar_wait(full, (seq / kAccBufs) & 1, abort_flag, p.status)) return;
            tc_fence_after();
            const uint32_t ta = tmem_base + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(acc * kAccCols + ch);
            if (sw == 64) {
                epilogue_slice<PLANES, 2>(p, td, ta, empty, c0 + n0 + ch, lane, sel1, sel2, keep, rot);
            } else if (sw == 32) {
                epilogue_slice<PLANES, 1>(p, td, ta, empty, c0 + n0 + ch, lane, sel1, sel2, keep, rot);
            } else {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(empty);
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    hash_keys_tc_kernel(const __grid_constant__ CUtensorMap tmap_keys, const __grid_constant__ CUtensorMap tmap_w,
                        const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[24];
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_flag;
    __shared__ int lens_sh[kLensCache];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    grid_dependency_wait();
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t w_half = (uint32_t)p.gpad_max * 128u;  // bytes of one K half of W
    const uint32_t w_smem = base;
    const uint32_t a_smem = base + 2u * w_half;
    // barriers
    const uint32_t bar0 = smem_u32(&bars[0]);
    auto full_a = [&](int s) { return bar0 + 8u * s; };            // 0,1
    auto empty_a = [&](int s) { return bar0 + 8u * (2 + s); };     // 2,3
    auto tmem_full = [&](int b) { return bar0 + 8u * (4 + b); };   // 4..7
    auto tmem_empty = [&](int b) { return bar0 + 8u * (8 + b); };  // 8..11
    auto w_full = [&](int j) { return bar0 + 8u * (16 + j); };     // 16..18: W rows of column tile j
    const uint32_t w_empty = bar0 + 8u * 13, final_bar = bar0 + 8u * 14;

    if (tid == 0) {
        abort_flag = 0;
        for (int s = 0; s < kStages; s++) {
            mbar_init(full_a(s), 1);
            mbar_init(empty_a(s), 1);
        }
        for (int b = 0; b < kAccBufs; b++) {
            mbar_init(tmem_full(b), 1);
            mbar_init(tmem_empty(b), 4 * kEpiGroups);  // one arrival per epilogue warp
        }
        static_assert(kAccBufs * kAccCols == 512, "TMEM holds 512 columns");
        for (int j = 0; j < kMaxWChunks; j++) mbar_init(w_full(j), 1);
        mbar_init(w_empty, 1);
        mbar_init(final_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(kAccBufs * kAccCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (p.seq_lens)
        for (int i = tid; i < p.s.B && i < kLensCache; i += blockDim.x) lens_sh[i] = p.seq_lens[i];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    const Shape &s = p.s;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------ producer ----
        int stage = 0;
        uint32_t empty_par[kStages] = {0, 0};
        int last_issued_par[kStages] = {-1, -1};
        int cur_g = -1, w_loads = 0, w_rest = 0, w_width = 0, w_c0 = 0;
        int w_last_par[kMaxWChunks];
        for (int j = 0; j < kMaxWChunks; j++) w_last_par[j] = -1;
        // W rows of column tile j of the group: one barrier per tile, so the
        // first MMAs need only the first tile; every block starts at its own
        // box of the tile, which spreads the blocks' simultaneous reads of the
        // same W lines over the L2.
        auto load_w_tile = [&](int j) {
            const int n0 = j * kAccCols, cols = min(kAccCols, w_width - n0), nb = cols / kWBox;
            mbar_expect_tx(w_full(j), (uint32_t)cols * 256u);
            for (int i = 0; i < nb; i++) {
                const int rb = (i + (int)blockIdx.x) % nb;
                for (int kh = 0; kh < 2; kh++)
                    tma_load_2d(w_smem + kh * w_half + (n0 + rb * kWBox) * 128, &tmap_w, w_full(j), kh * 64,
                                w_c0 + n0 + rb * kWBox);
            }
            w_last_par[j] = (w_last_par[j] + 1) & 1;
        };
        bool first_pass = true;
        for (ItemIter iter(p); iter.live(p) && !abort_flag; iter.next(p)) {
            const Item im = iter.item(p, lens_sh);
            if (im.skip) continue;
            if (im.group != cur_g) {
                if (cur_g >= 0 && !mbar_wait(w_empty, (w_loads - 1) & 1, &abort_flag, p.status)) break;
                group_cols(p, im.group, w_c0, w_width);
                load_w_tile(0);  // the rest after this item's key tile
                w_rest = 1;
                cur_g = im.group;
                w_loads++;
            }
            if (!mbar_wait(empty_a(stage), empty_par[stage] ^ 1u, &abort_flag, p.status)) break;
            empty_par[stage] ^= 1u;
            const int row0 = im.unit * s.Ncap + p.tok0 + im.mt * kBM;
            // later tiles of this block into L2: the first pass covers 2..kPrefetchAhead
            // items ahead, every later pass the one newly kPrefetchAhead ahead
            for (int ahead = first_pass ? 2 : kPrefetchAhead; ahead <= kPrefetchAhead; ahead++) {
                const int it2 = iter.it + ahead * item_stride(p);
                if (it2 < p.total_items) {
                    const Item i2 = item_of(p, it2, lens_sh);
                    if (!i2.skip) {
                        const int r2 = i2.unit * s.Ncap + p.tok0 + i2.mt * kBM;
                        tma_prefetch_l2_2d(&tmap_keys, 0, r2);
                        tma_prefetch_l2_2d(&tmap_keys, 64, r2);
                    }
                }
            }
            first_pass = false;
            mbar_expect_tx(full_a(stage), kTileBytes);
            tma_load_2d(a_smem + stage * kTileBytes, &tmap_keys, full_a(stage), 0, row0);
            tma_load_2d(a_smem + stage * kTileBytes + kHalfBytes, &tmap_keys, full_a(stage), 64, row0);
            last_issued_par[stage] = (last_issued_par[stage] + 1) & 1;
            stage ^= 1;
            for (; w_rest > 0 && w_rest * kAccCols < w_width; w_rest++) load_w_tile(w_rest);
            w_rest = 0;
        }
        // our own copies in flight must land before the CTA exits
        for (int st = 0; st < kStages; st++)
            if (last_issued_par[st] >= 0) mbar_wait(full_a(st), (uint32_t)last_issued_par[st], &abort_flag, p.status);
        for (int j = 0; j < kMaxWChunks; j++)
            if (w_last_par[j] >= 0) mbar_wait(w_full(j), (uint32_t)w_last_par[j], &abort_flag, p.status);
    } else if (warp == 1 && lane == 0) {
        // ----------------------------------------------------------- MMA ----
        int stage = 0, seq = 0;  // seq: column-tile sequence number; buffer seq % 4, use seq / 4
        uint32_t full_par[kStages] = {0, 0};
        int cur_g = -1;
        uint32_t w_ready = 0, w_par = 0;  // bit j: tile j of the current group landed / next parity
        for (ItemIter iter(p); iter.live(p) && !abort_flag; iter.next(p)) {
            const Item im = iter.item(p, lens_sh);
            if (im.skip) continue;
            if (im.group != cur_g) {
                if (cur_g >= 0) mma_commit(w_empty);  // W free once the MMAs so far complete
                cur_g = im.group;
                w_ready = 0;
            }
            if (!mbar_wait(full_a(stage), full_par[stage], &abort_flag, p.status)) break;
            full_par[stage] ^= 1u;
            tc_fence_after();
            int c0, width;
            group_cols(p, im.group, c0, width);
            bool ok = true;
            for (int n0 = 0; n0 < width; n0 += kAccCols, seq++) {
                const int nw = min(kAccCols, width - n0);
                const int acc = seq & (kAccBufs - 1);
                const int j = n0 / kAccCols;
                if (!((w_ready >> j) & 1u)) {  // first use of W tile j in this group
                    if (!mbar_wait(w_full(j), (w_par >> j) & 1u, &abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    w_par ^= 1u << j;
                    w_ready |= 1u << j;
                }
                // wait for the epilogue to release use (seq / 4 - 1) of this buffer
                if (!mbar_wait(tmem_empty(acc), ((seq / kAccBufs) & 1) ^ 1u, &abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(acc * kAccCols);
                const uint32_t idesc = idesc_bf16(nw);
#pragma unroll
                for (int kh = 0; kh < 2; kh++) {
#pragma unroll
                    for (int ks = 0; ks < 4; ks++) {
                        const uint64_t ad = sw128_desc(a_smem + stage * kTileBytes + kh * kHalfBytes + ks * 32);
                        const uint64_t bd = sw128_desc(w_smem + kh * w_half + n0 * 128 + ks * 32);
                        mma_bf16(d, ad, bd, idesc, (kh | ks) != 0);
                    }
                }
                mma_commit(tmem_full(acc));
            }
            if (!ok) break;
            mma_commit(empty_a(stage));
            stage ^= 1;
        }
        // every MMA issued so far has completed before TMEM is released
        mma_commit(final_bar);
        mbar_wait(final_bar, 0, &abort_flag, p.status);
    } else if (warp >= 4) {
        if (s.planes)
            epilogue<true>(p, lens_sh, tmem_base, bar0, &abort_flag, warp, lane);
        else
            epilogue<false>(p, lens_sh, tmem_base, bar0, &abort_flag, warp, lane);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(kAccBufs * kAccCols));
    }
}

// ------------------------------------------------------------------ host ----
// 2-D bf16 row-major [rows][128] view, box = 64 elements x box_rows, 128B swizzle.
static bool make_map(CUtensorMap *m, const void *ptr, uint64_t rows, uint32_t box_rows)
{
    const uint64_t dims[2] = {128, rows};
    const uint64_t strides[1] = {256};
    const uint32_t box[2] = {64, box_rows};
    return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, strides, box,
                             CU_TENSOR_MAP_SWIZZLE_128B);
}

static int num_sms()
{
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

}  // namespace tc

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

bool encode_tensor_map(CUtensorMap *m, CUtensorMapDataType type, int rank, const void *ptr, const uint64_t *dims,
                       const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle swizzle)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn || rank < 1 || rank > 5) return false;
    cuuint64_t d[5], st[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; i++) {
        d[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
        if (i + 1 < rank) st[i] = strides[i];
    }
    return fn(m, type, (cuuint32_t)rank, const_cast<void *>(ptr), d, st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_hash_keys_tc(const Shape &s, const uint16_t *keys, const uint16_t *W, const int32_t *seq_lens,
                                int tok0, int n_tokens, void *codes, int32_t *status, cudaStream_t st)
{
    using namespace tc;
    if (n_tokens == 0) return cudaSuccess;
    Params p;
    p.s = s;
    p.seq_lens = seq_lens;
    p.codes = codes;
    p.status = status;
    p.tok0 = tok0;
    p.n_tokens = n_tokens;
    p.n_mt = (n_tokens + kBM - 1) / kBM;
    p.ngroups = (s.LK + kMaxGroupCols - 1) / kMaxGroupCols;
    p.gsize = (((s.LK + p.ngroups - 1) / p.ngroups) + 31) & ~31;
    p.gpad_max = p.gsize;
    p.total_items = s.B * s.Hkv * p.n_mt;  // (unit, tile) items, each hashed for every group
    p.kmagic = (uint32_t)((1ull << 32) / (uint64_t)s.K) + 1u;
    p.hmagic = (uint32_t)((1ull << 32) / (uint64_t)s.Hkv) + 1u;
    CUtensorMap mk, mw;
    if (!make_map(&mk, keys, (uint64_t)s.B * s.Hkv * s.Ncap, kBM)) return cudaErrorInvalidValue;
    if (!make_map(&mw, W, (uint64_t)s.LK, kWBox)) return cudaErrorInvalidValue;
    const int smem = 1024 + 2 * p.gpad_max * 128 + kStages * kTileBytes;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(hash_keys_tc_kernel), smem);
    if (e != cudaSuccess) return e;
    const int grid = p.ngroups * min(num_sms() / p.ngroups, p.total_items);
    return launch_pdl(hash_keys_tc_kernel, dim3(grid), dim3(kThreads), smem, st, mk, mw, p);
}

}  // namespace mp
