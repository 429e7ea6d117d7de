// Paged prefill (chunked) attention on the sm_100a tensor cores.
//
// A chunk of n new tokens at the end of a sequence of L cached tokens attends
// causally over the paged cache: chunk row i sits at position p = L - n + i
// and reads tokens 0..p.  FlashAttention's idea (attention computed in tiles
// so that K/V cross between HBM and on-chip memory once per tile, the
// "KV Cache & PagedAttention" studynote, section III) is kept; the tiles come
// through the block table.
//
// A query tile is M = 128 rows: 128 / G chunk tokens x the G query heads that
// share a KV head, so every K/V tile read feeds G heads at once.  A work item
// is two adjacent query tiles of one (sequence, KV head), whose K/V stages are
// streamed once for both.  The launch is persistent: one CTA per SM takes
// items from a counter in the caller's workspace until none is left, and the
// K/V stages of consecutive items flow through one ring, so an item's first
// copies overlap the last stages of the one before.  Per 64-key stage and tile:
//   S  = Q K^T      M = 128, N = 64, K = head_dim        (tcgen05, fp32 in TMEM)
//   P  = exp2(S * scale * log2 e - m), rounded to the input type, written
//        back into tensor memory over the S columns it came from
//   O += P V        M = 128, N = head_dim, K = 64 keys    (tcgen05, A = P from
//                   TMEM, B = V from smem, fp32 in TMEM)
// Warps: 0-3 softmax + epilogue of tile 0, 4-7 of tile 1 (thread = one row =
// one tensor-memory lane), 8 producer (work items and K/V stages), 9 and 10
// the MMA issuers of tiles 0 and 1 (one thread each), 11 the Q loader (an
// item's Q tiles, once the S MMAs of the item before are done).  The third
// warpgroup (8-11) hands registers to the softmax warps.  The two softmax
// groups run side by side (two warps per SM sub-partition); S (and the P
// written over it) is double-buffered in tensor memory per tile, so the tensor
// core computes the next stage's S while the softmax works.  The K/V ring
// holds four 64-key stages, enough to cover the copy latency (five were no
// faster).  The row maximum m is moved lazily: only when a stage
// exceeds it by 2^8 is O rescaled in tensor memory.  Keys past the row's
// position get weight 0; keys past the item's key range or in a block whose
// table entry is bad also get their V rows zeroed in shared memory (the
// product 0 * V must not meet stale or non-finite data).
//
// Every wait is bounded (2 s): a timeout sets PA_DEV_TIMEOUT, makes the other
// warps give up at their next wait, and the kernel returns.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <type_traits>

#include "pa.h"
#include "pa_common.cuh"
#include "pa_tcgen05.cuh"

namespace pa {
namespace {

constexpr int PF_KT = 64;          // keys per stage (N of S, K of PV)
constexpr int PF_M = 128;          // query rows per tile
constexpr int PF_TILES = 2;        // query tiles per CTA
// 3 warpgroups: 8 softmax warps, then producer, 2 MMA issuers and the Q
// loader.  The block is launched with 168 registers a thread; the third
// warpgroup gives registers back (setmaxnreg) and the softmax warpgroups take
// them: 256 * 208 + 128 * 80 = 63488 <= 384 * 168 = 64512.
constexpr int PF_THREADS = 384;
constexpr int PF_REGS_HIGH = 208, PF_REGS_LOW = 80;
static_assert(256 * PF_REGS_HIGH + 128 * PF_REGS_LOW <= PF_THREADS * 168, "register split");
constexpr int PF_MAX_STAGES = 4;
constexpr float kPfRescaleLog2 = 8.f;
constexpr uint32_t PF_FULL = 0xffffffffu;

struct PrefillParams {
    void* out;
    const void* q;
    const int32_t* tables;
    const int32_t* lens;
    const int32_t* cu;
    int S, total_q, max_q, npair, Hq, Hkv, mbps, NB, bs, bs_log2, nst;
    int n_items;       // npair * S * Hkv work items (pairs of query tiles)
    int out32;         // out is 32-byte aligned: rows are written 32 bytes a store
    float scale_log2e;
    int32_t* err;
    int* ws;           // [0] next item, [1] CTAs done (zero between calls)
};

// Shared memory (1024-byte aligned; every operand tile starts on a 1024-byte
// boundary, as the 128-byte swizzle wants):
//   Q        per tile NBOX boxes of [128 rows][128 B]
//   ring     nst stages of K then V, each NBOX boxes of [64 keys][128 B]
//   barriers, misc
// P never goes to shared memory: the softmax writes it into tensor memory
// over the S columns it came from, and the PV MMA reads it from there.
template <int D>
struct PfLayout {
    static constexpr int NBOX = D * 2 / 128;           // 128-byte column boxes of a row
    static constexpr int QBOX = PF_M * 128;
    static constexpr int Q_BYTES = NBOX * QBOX;        // one tile
    static constexpr int KBOX = PF_KT * 128;
    static constexpr int KV_BYTES = NBOX * KBOX;
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;
    // per tile: S x2 (64 columns each; P, 16-bit pairs, overwrites the first 32
    // columns of its S buffer) then O (head_dim columns), 256 columns
    static constexpr uint32_t TM_TILE = 256;
    static constexpr uint32_t TM_COLS = PF_TILES * TM_TILE;
    // q_full, q_empty, item_full x2, item_empty x2, then per tile s_full x2,
    // fin + spare, p_full x2, pv_done x2
    static constexpr int NBAR_FIXED = 6 + 8 * PF_TILES;
    int nst;
    __host__ __device__ explicit PfLayout(int n) : nst(n) {}
    __host__ __device__ size_t q(int t) const { return (size_t)t * Q_BYTES; }
    __host__ __device__ size_t ring(int st) const {
        return (size_t)PF_TILES * Q_BYTES + (size_t)st * STAGE_BYTES;
    }
    __host__ __device__ size_t bars() const { return ring(nst); }
    __host__ __device__ size_t misc() const { return ((bars() + (size_t)(2 * nst + NBAR_FIXED) * 8 + 15) / 16) * 16; }
    // two item slots: the item (128 bytes) and the loaded-piece masks of its
    // first 64 stages
    static constexpr int SLOT = 128 + 64 * 4;
    __host__ __device__ size_t items() const { return misc() + 64; }
    __host__ __device__ size_t total() const { return items() + 2 * SLOT; }
};

// 3-D tiled tensor copy global -> shared (box given by the tensor map).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z),
          "r"(smem_u32(bar))
        : "memory");
}

// 2-D tiled copy with the default L2 policy: K/V tiles of a sequence are read
// by every query tile of its chunk, so they should stay in L2.
__device__ __forceinline__ void tma_load_2d_keep(void* dst, const CUtensorMap* map, int x, int y,
                                                 uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y),
          "r"(smem_u32(bar))
        : "memory");
}

// Bounded wait that also gives up once another warp has given up.
__device__ __forceinline__ bool pf_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                        int32_t* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((it & 63) == 0 && global_ns() - t0 > kWaitLimitNs) {
            set_err(err, PA_DEV_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

// 64 columns of this warp's lane quarter in one load, waiting for it.
__device__ __forceinline__ void tm_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,"
        "%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,"
        "%62,%63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]),
          "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]),
          "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]),
          "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]),
          "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
}

// 16 columns to tensor memory without waiting (tm_wait_st before the result
// is handed to another thread).
__device__ __forceinline__ void tm_st16_nowait(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
          "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
          "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tm_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 bytes to global memory in one store (the address 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* dst, const uint32_t* w) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 ::"l"(dst), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]),
                   "r"(w[7])
                 : "memory");
}

// 2^x by the PTX ex2.approx instruction with subnormal results flushed to
// zero: softmax weights below 2^-126 are zero after rounding to 16 bits
// anyway (the sum they would add is far below the output's precision).
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// One work item: query tiles 2u and 2u + 1 of (sequence s, KV head j).  Items
// are numbered so that the tiles of one (s, j) are neighbours, latest pairs
// (longest key ranges) first: CTAs working at the same time share K/V in L2.
struct PfItem {
    int s, j, a, n, L, ntile, kend, nkt_all;
    int r0[PF_TILES], rows[PF_TILES], nkt[PF_TILES];
    int bad, first;    // first: u == 0 and j == 0 (a bad length is reported once)
    int q, g;          // the item's number (-1: no more), its first stage in the ring's sequence
};
static_assert(sizeof(PfItem) <= 128, "item slot");

template <int G>
__device__ __forceinline__ PfItem pf_item(const PrefillParams& p, int q) {
    constexpr int QT = PF_M / G;                   // chunk tokens per query tile
    PfItem it;
    const int sj = q / p.npair;
    const int u = p.npair - 1 - q % p.npair;
    it.s = sj / p.Hkv;
    it.j = sj % p.Hkv;
    it.first = u == 0 && it.j == 0;
    const int a = __ldg(p.cu + it.s), e = __ldg(p.cu + it.s + 1);
    int L = __ldg(p.lens + it.s);
    int n = e - a;
    bool bad = false;
    if (a < 0 || e < a || e > p.total_q) { bad = true; n = 0; }
    if (n > p.max_q) { bad = true; n = p.max_q; }
    const int hi = p.mbps * p.bs;
    if (L < 0 || L > hi) { bad = true; L = max(0, min(L, hi)); }
    if (n > L) bad = true;
    it.a = a;
    it.n = n;
    it.L = L;
    it.bad = bad;
#pragma unroll
    for (int t = 0; t < PF_TILES; ++t) {
        it.r0[t] = (PF_TILES * u + t) * QT;        // first chunk row of the tile
        it.rows[t] = max(0, min(QT, n - it.r0[t]));
        const int ke = it.rows[t] ? max(0, min(L, L - n + it.r0[t] + it.rows[t])) : 0;
        it.nkt[t] = (ke + PF_KT - 1) / PF_KT;
    }
    it.ntile = it.rows[0] == 0 ? 0 : it.rows[PF_TILES - 1] ? PF_TILES : 1;
    const int last_end = it.ntile > 1 ? it.r0[1] + it.rows[1] : it.r0[0] + it.rows[0];
    it.kend = it.ntile ? max(0, min(L, L - n + last_end)) : 0;   // keys read
    it.nkt_all = (it.kend + PF_KT - 1) / PF_KT;
    return it;
}

// Persistent: one CTA per SM takes items from a global counter until none is
// left.  The producer (warp 8) takes the tickets and hands each item on through
// a two-slot queue in shared memory; K/V stages of consecutive items flow
// through one ring, so the copies of the next item overlap the last stages and
// the epilogue of the current one.
template <typename T, int D, int G>
__global__ void __launch_bounds__(PF_THREADS, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                  const __grid_constant__ CUtensorMap qmap, PrefillParams p) {
    using LY = PfLayout<D>;
    constexpr int kItemUsers = PF_TILES + 4 * PF_TILES + 1;   // issuers, softmax warps, Q loader
    static_assert(kItemUsers == 11, "item queue arrivals");
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const LY ly(p.nst);
    const int nst = p.nst;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + ly.bars());
    uint64_t* empty = full + nst;                  // one arrival per tile's issuer
    uint64_t* q_full = empty + nst;
    uint64_t* q_empty = q_full + 1;                // an item's S MMAs of both tiles complete
    uint64_t* item_full = q_full + 2;              // [2]
    uint64_t* item_empty = q_full + 4;             // [2]
    uint64_t* tb = q_full + 6;
    // per tile t: s_full[2] (S in tensor memory), fin (its issuer's final
    // drain) and one spare, p_full[2] (P written by the 4 softmax warps),
    // pv_done[2] (PV complete)
    auto tbar = [&](int t, int kind, int b) { return tb + t * 8 + kind * 2 + b; };
    int* misc = reinterpret_cast<int*>(smem + ly.misc());
    volatile int* abort_flag = misc;
    // the two item slots of the queue (128 bytes each)
    auto item_slot = [&](int k) { return reinterpret_cast<PfItem*>(smem + ly.items() + (k & 1) * LY::SLOT); };
    auto slot_masks = [&](int k) { return reinterpret_cast<uint32_t*>(smem + ly.items() + (k & 1) * LY::SLOT + 128); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 8);

    if (tid == 0) {
        for (int k = 0; k < 2 * nst + LY::NBAR_FIXED; ++k)
            mbar_init(full + k, k >= nst && k < 2 * nst ? PF_TILES : 1);
        mbar_init(q_empty, PF_TILES);
        for (int b = 0; b < 2; ++b) mbar_init(item_empty + b, kItemUsers);
        for (int t = 0; t < PF_TILES; ++t)
            for (int b = 0; b < 2; ++b) mbar_init(tbar(t, 2, b), 4);   // p_full
        misc[0] = 0;
        fence_barrier_init();
    }
    if (warp == 9) {
        tc::alloc(tmem_slot, LY::TM_COLS);
        tc::relinquish();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tmem_slot;
    const int PR = p.bs >= 16 ? 16 : p.bs;         // rows of one TMA box (block piece)
    const int prl = p.bs >= 16 ? 4 : p.bs_log2;
    // loaded-piece mask of stage c of an item: pieces inside its key range
    // whose table entry is in range (the pieces the producer loads)
    auto piece_mask = [&](const PfItem& it, int c, int cmax) {
        const int32_t* trow = p.tables + (size_t)it.s * p.mbps;
        const int npc = PF_KT / PR;
        uint32_t mk = 0;
        for (int qq = 0; qq < npc; ++qq) {
            const int tok = c * PF_KT + qq * PR;
            if (c < cmax && tok < it.kend) {
                const int blk = __ldg(trow + (tok >> p.bs_log2));
                if (blk >= 0 && blk < p.NB) mk |= 1u << qq;
            }
        }
        return mk;
    };

    if (warp >= 8) {
    // (the whole warpgroup executes this)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(PF_REGS_LOW));
    if (warp == 8) {
        // ================================================= tickets and K/V stages
        if (lane == 0) {
            prefetch_tensormap(&kmap);
            prefetch_tensormap(&vmap);
        }
        const int npc = PF_KT / PR;                    // block pieces per stage
        const int nops = npc * 2 * LY::NBOX;           // TMA boxes per stage (<= 32)
        const int piece = lane / (2 * LY::NBOX), sub = lane % (2 * LY::NBOX);
        const int kv = sub / LY::NBOX, bx = sub % LY::NBOX;
        int g = 0, st = 0, round = 0;                  // stages issued, ring slot, ring round
        bool ok = true;
        for (int k = 0; ok;) {
            int q = 0;
            if (lane == 0) q = atomicAdd(p.ws, 1);
            q = __shfl_sync(PF_FULL, q, 0);
            PfItem it;
            uint32_t m0 = 0, m1 = 0;                   // masks of stages lane, 32 + lane
            if (q < p.n_items) {
                it = pf_item<G>(p, q);
                if (it.bad && it.first && lane == 0) set_err(p.err, PA_DEV_BAD_LEN);
                if (it.ntile == 0) continue;           // past its sequence's chunk
                m0 = piece_mask(it, lane, it.nkt_all);
                m1 = piece_mask(it, 32 + lane, it.nkt_all);
            } else {
                q = -1;
            }
            // hand it on: the slot is free once everyone took the item two back
            if (k >= 2) {
                bool w = true;
                if (lane == 0) w = pf_wait(item_empty + (k & 1), ((k - 2) >> 1) & 1, abort_flag, p.err);
                if (!__shfl_sync(PF_FULL, w, 0)) break;
            }
            slot_masks(k)[lane] = m0;
            slot_masks(k)[32 + lane] = m1;
            if (lane == 0) {
                PfItem* slot = item_slot(k);
                if (q >= 0) *slot = it;
                slot->q = q;
                slot->g = g;
            }
            __syncwarp();                              // the lanes' writes before the release
            if (lane == 0) mbar_arrive(item_full + (k & 1));
            __syncwarp();
            ++k;
            if (q < 0) break;
            const int32_t* trow = p.tables + (size_t)it.s * p.mbps;
            for (int c = 0; c < it.nkt_all; ++c) {
                if (round > 0) {
                    bool w = true;
                    if (lane == 0) w = pf_wait(empty + st, (round - 1) & 1, abort_flag, p.err);
                    if (!__shfl_sync(PF_FULL, w, 0)) { ok = false; break; }
                }
                const int tok = c * PF_KT + piece * PR;
                const bool exists = lane < nops && tok < it.kend;
                const int blk = exists ? __ldg(trow + (tok >> p.bs_log2)) : -1;
                const bool live = exists && blk >= 0 && blk < p.NB;
                const uint32_t want = __reduce_or_sync(PF_FULL, exists ? 1u << piece : 0u);
                const uint32_t got = __reduce_or_sync(PF_FULL, live ? 1u << piece : 0u);
                if (lane == 0) {
                    if (want & ~got) set_err(p.err, PA_DEV_BAD_BLOCK);
                    if (got)
                        mbar_arrive_expect_tx(full + st, (uint32_t)__popc(got) * 2u * PR * (D * 2));
                    else
                        mbar_arrive(full + st);
                }
                __syncwarp();
                if (live) {
                    const int y = ((blk * p.Hkv + it.j) << p.bs_log2) + (tok & (p.bs - 1));
                    uint8_t* dst = smem + ly.ring(st) + kv * LY::KV_BYTES + bx * LY::KBOX + piece * PR * 128;
                    tma_load_2d_keep(dst, kv ? &vmap : &kmap, bx * 64, y, full + st);
                }
                ++g;
                if (++st == nst) { st = 0; ++round; }
            }
        }
        // no copy of this CTA may still be landing when it exits
        if (lane == 0)
            for (int x = max(0, g - nst); x < g; ++x) mbar_wait(full + x % nst, (x / nst) & 1);
        __syncwarp();
    } else if (warp == 11) {
        // ================================================= Q tiles of each item
        // loaded once both issuers' S MMAs of the item before are complete
        if (lane == 0) prefetch_tensormap(&qmap);
        int last = -1;
        for (int k = 0;; ++k) {
            if (!__all_sync(PF_FULL, pf_wait(item_full + (k & 1), (k >> 1) & 1, abort_flag, p.err))) break;
            const PfItem it = *item_slot(k);
            __syncwarp();
            if (lane == 0) mbar_arrive(item_empty + (k & 1));
            if (it.q < 0) break;
            if (k >= 1) {
                // the previous Q has landed (nobody may have waited for it when
                // neither tile of that item had keys) and its S MMAs are done
                bool w = true;
                if (lane == 0)
                    w = pf_wait(q_full, (k - 1) & 1, abort_flag, p.err) &&
                        pf_wait(q_empty, (k - 1) & 1, abort_flag, p.err);
                if (!__shfl_sync(PF_FULL, w, 0)) break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(q_full, (uint32_t)(it.ntile * LY::Q_BYTES));
#pragma unroll
                for (int t = 0; t < PF_TILES; ++t)
                    if (t < it.ntile)
#pragma unroll
                        for (int b = 0; b < LY::NBOX; ++b)
                            tma_load_3d(smem + ly.q(t) + b * LY::QBOX, &qmap, b * 64, it.j * G,
                                        it.a + it.r0[t], q_full);
            }
            last = k;
        }
        // the last Q copy has landed before the CTA exits
        if (lane == 0 && last >= 0) mbar_wait(q_full, last & 1);
        __syncwarp();
    } else if (warp == 9 || warp == 10) {
        // ================================================= MMA issuers (one thread each)
        // Warp 9 issues tile 0's MMAs and warp 10 tile 1's.  Per stage c of an
        // item: S(c), then PV(c - 1).  Both issuers take part in every item and
        // every stage (an empty arrival for a tile the item does not have), so
        // each barrier they share gets one arrival per issuer and phase: the
        // stage slot is released after both committed, and Q may be replaced
        // once both tiles' S MMAs of the item are complete.
        const int t = warp - 9;
        if (lane == 0) {
            constexpr uint32_t ID_S = tc::idesc_f16<T>(false, false, PF_M, PF_KT);
            constexpr uint32_t ID_O = tc::idesc_f16<T>(false, true, PF_M, D);
            const uint64_t qd = tc::sdesc_sw128(smem_u32(smem + ly.q(t)), 16, 1024);
            const uint32_t tS = tmem + (uint32_t)(t * LY::TM_TILE);
            int st = 0, stm = 0;                       // ring slot of the stage, of the one before
            uint32_t ph = 0;
            int gs = 0;                                // this tile's S count (S buffers, phases)
            bool ok = true;
            for (int k = 0; ok; ++k) {
                ok = pf_wait(item_full + (k & 1), (k >> 1) & 1, abort_flag, p.err);
                if (!ok) break;
                const PfItem it = *item_slot(k);
                mbar_arrive(item_empty + (k & 1));
                if (it.q < 0) break;
                const int nk = t < it.ntile ? it.nkt[t] : 0;
                if (nk > 0) {
                    ok = pf_wait(q_full, k & 1, abort_flag, p.err);
                    if (!ok) break;
                } else {
                    // no S of this tile in the item: its share of q_empty, once
                    // the item before has released Q
                    if (k >= 1) {
                        ok = pf_wait(q_empty, (k - 1) & 1, abort_flag, p.err);
                        if (!ok) break;
                    }
                    mbar_arrive(q_empty);
                }
                const int gs0 = gs;
                for (int c = 0; ok && c <= it.nkt_all; ++c) {
                    if (c < it.nkt_all) {
                        ok = pf_wait(full + st, ph, abort_flag, p.err);
                        if (!ok) break;
                        if (c < nk) {
                            // S buffer b last held S of this tile's stage gs - 2,
                            // whose P the PV issued in the round before reads:
                            // this thread's MMAs run in the order issued
                            const int b = gs & 1;
                            tc::fence_after();
                            const uint64_t kd = tc::sdesc_sw128(smem_u32(smem + ly.ring(st)), 16, 1024);
#pragma unroll
                            for (int k16 = 0; k16 < D / 16; ++k16)   // descriptor start fields in 16-byte units
                                tc::mma_ss(tS + (uint32_t)(PF_KT * b),
                                           qd + (uint64_t)((k16 >> 2) * (LY::QBOX >> 4) + (k16 & 3) * 2),
                                           kd + (uint64_t)((k16 >> 2) * (LY::KBOX >> 4) + (k16 & 3) * 2),
                                           ID_S, k16 > 0 ? 1u : 0u);
                            tc::commit(tbar(t, 0, b));
                            if (c == nk - 1) tc::commit(q_empty);   // the item's last S
                            ++gs;
                        }
                    }
                    if (c >= 1) {
                        const int m = c - 1;
                        if (m < nk) {
                            const int gm = gs0 + m, bm = gm & 1;
                            ok = pf_wait(tbar(t, 2, bm), (gm >> 1) & 1, abort_flag, p.err);
                            if (!ok) break;
                            tc::fence_after();
                            // A = P in tensor memory (lane = row, column = two keys),
                            // B = the V stage (MN-major)
                            const uint64_t vd =
                                tc::sdesc_sw128(smem_u32(smem + ly.ring(stm) + LY::KV_BYTES), LY::KBOX, 1024);
#pragma unroll
                            for (int kk = 0; kk < PF_KT / 16; ++kk)
                                tc::mma_ts(tS + (uint32_t)(2 * PF_KT), tS + (uint32_t)(PF_KT * bm + kk * 8),
                                           vd + (uint64_t)(kk * 128), ID_O, (m > 0 || kk > 0) ? 1u : 0u);
                            tc::commit(tbar(t, 3, bm));
                        }
                        tc::commit(empty + stm);       // this tile is done with the stage slot
                    }
                    if (c < it.nkt_all) {
                        stm = st;
                        if (++st == nst) { st = 0; ph ^= 1u; }
                    }
                }
            }
            // every MMA of this thread completes before tensor memory is freed
            tc::commit(tbar(t, 1, 0));
            mbar_wait(tbar(t, 1, 0), 0);
        }
        __syncwarp();
    }
    } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" :: "n"(PF_REGS_HIGH));   // both warpgroups
        // ================================================= softmax + epilogue (row of tile t)
        const int t = warp >> 2;
        const int r = tid & 127;
        const int g = r % G;
        const uint32_t lq = (uint32_t)(32 * (warp & 3)) << 16;
        const uint32_t tS = tmem + (uint32_t)(t * LY::TM_TILE), tO = tS + 2 * PF_KT;
        const float sl = p.scale_log2e;
        const int npc = PF_KT / PR;
        const uint32_t all_pieces = (1u << npc) - 1u;
        // Which pieces of a stage hold loaded blocks (piece_mask, the
        // producer's rule), known here without waiting for the copy, so that
        // only stages that need their V rows zeroed wait for it themselves
        // (the S MMA already did).  Lane i holds the mask of stage 32k + i for
        // the current group k of 32 stages and the next one: the producer
        // hands the first two groups on with the item, later groups are read
        // from the table a group ahead.
        auto stage_mask = [&](const PfItem& it, int c) { return piece_mask(it, c, it.nkt[t]); };
        // take item k from the queue, with the masks of its first two groups
        // of stages (the producer's, from the slot)
        auto take = [&](int k, PfItem& it, uint32_t& mc, uint32_t& mn) {
            if (!__all_sync(PF_FULL, pf_wait(item_full + (k & 1), (k >> 1) & 1, abort_flag, p.err)))
                return false;
            it = *item_slot(k);
            mc = slot_masks(k)[lane];
            mn = slot_masks(k)[32 + lane];
            __syncwarp();
            if (lane == 0) mbar_arrive(item_empty + (k & 1));
            return true;
        };
        int gs = 0;                                    // this tile's stage count (S buffers, phases)
        PfItem it;
        uint32_t mask_cur = 0, mask_next = 0;
        bool ok = take(0, it, mask_cur, mask_next);
        for (int k = 0; ok && it.q >= 0; ++k) {
            const bool mine = t < it.ntile;            // an item may have one tile only
            const int my_nkt = mine ? it.nkt[t] : 0, kend = it.kend;
            const int crow = it.r0[t] + r / G;         // chunk row of this thread's query
            const int pos = it.L - it.n + crow;        // keys 0..pos are visible
            float m_ref = -INFINITY, l = 0.f;
            for (int c = 0; c < my_nkt; ++c, ++gs) {
                const int b = gs & 1;
                if (c > 0 && (c & 31) == 0) {
                    mask_cur = mask_next;
                    mask_next = stage_mask(it, c + 32 + lane);
                }
                const uint32_t vmask = __shfl_sync(PF_FULL, mask_cur, c & 31);
                ok = __all_sync(PF_FULL, pf_wait(tbar(t, 0, b), (gs >> 1) & 1, abort_flag, p.err));
                if (!ok) break;
                tc::fence_after();
                // keys of this stage the row may see: the first `lim` by position,
                // and only those of pieces whose block was loaded
                const int lim = pos - c * PF_KT + 1;
                const bool whole = __all_sync(PF_FULL, lim >= PF_KT && vmask == all_pieces);
                const uint32_t tSb = tS + (uint32_t)(PF_KT * b) + lq;
                // the 64 scores of the row, then their maximum (the scale is positive)
                uint32_t v[PF_KT];
                tm_ld64(tSb, v);
                float mraw = -INFINITY;
                if (whole) {                           // warp-uniform: no key is hidden
                    // eight independent chains, then a tree
                    float mx[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) mx[i] = __uint_as_float(v[i]);
#pragma unroll
                    for (int i = 8; i < PF_KT; ++i) mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(v[i]));
#pragma unroll
                    for (int w = 4; w > 0; w >>= 1)
#pragma unroll
                        for (int i = 0; i < w; ++i) mx[i] = fmaxf(mx[i], mx[i + w]);
                    mraw = mx[0];
                } else if (vmask == all_pieces) {       // causal edge only
#pragma unroll
                    for (int i = 0; i < PF_KT; ++i)
                        if (i < lim) mraw = fmaxf(mraw, __uint_as_float(v[i]));
                } else {
#pragma unroll
                    for (int i = 0; i < PF_KT; ++i)
                        if (i < lim && ((vmask >> (i >> prl)) & 1u)) mraw = fmaxf(mraw, __uint_as_float(v[i]));
                }
                const float mt = mraw * sl;
                const bool need = mt > m_ref + kPfRescaleLog2;
                if (__any_sync(PF_FULL, need)) {
                    if (c > 0) {
                        // O must hold every earlier PV before it is rescaled
                        ok = __all_sync(PF_FULL, pf_wait(tbar(t, 3, (gs - 1) & 1), ((gs - 1) >> 1) & 1,
                                                         abort_flag, p.err));
                        if (!ok) break;
                        tc::fence_after();
                        const float f = need ? exp2f(m_ref - mt) : 1.f;
#pragma unroll
                        for (int q4 = 0; q4 < D / 16; ++q4) {
                            uint32_t o[16];
                            tc::ld16(tO + (uint32_t)(16 * q4) + lq, o);
#pragma unroll
                            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                            tc::st16(tO + (uint32_t)(16 * q4) + lq, o);
                        }
                        l *= f;
                    }
                    if (need) m_ref = mt;
                }
                // P = exp2(s * scale * log2 e - m), rounded, written as 16-bit pairs
                // over columns [0, 32) of S buffer b (all 64 scores are in
                // registers); both stores complete before P is handed to the issuer
                const float nmr = m_ref == -INFINITY ? 0.f : -m_ref;
                // packed fp32x2: z = s * scale * log2 e - m for two keys at once, and
                // the row sum of the weights before their rounding to T
                const uint64_t SL2 = f2_pack(sl, sl), NM2 = f2_pack(nmr, nmr), ONE2 = f2_pack(1.f, 1.f);
                uint64_t acc2 = f2_pack(0.f, 0.f);
                // three copies of the loop (no masking; the causal edge; the causal
                // edge and missing blocks), so that the common one carries no
                // test (a per-pair test would split the unrolled loop into blocks
                // the compiler cannot interleave)
                auto exps = [&](auto mode) {
#pragma unroll
                    for (int h = 0; h < PF_KT / 32; ++h) {
                        uint32_t w[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int k0 = 32 * h + 2 * i;
                            float z0, z1;
                            f2_unpack(f2_fma(f2_pack(__uint_as_float(v[k0]), __uint_as_float(v[k0 + 1])), SL2, NM2),
                                      z0, z1);
                            if (decltype(mode)::value == 1) {
                                z0 = k0 < lim ? z0 : -INFINITY;
                                z1 = k0 + 1 < lim ? z1 : -INFINITY;
                            } else if (decltype(mode)::value == 2) {
                                if (!(k0 < lim && ((vmask >> (k0 >> prl)) & 1u))) z0 = -INFINITY;
                                if (!(k0 + 1 < lim && ((vmask >> ((k0 + 1) >> prl)) & 1u))) z1 = -INFINITY;
                            }
                            const float e0 = ex2_ftz(z0), e1 = ex2_ftz(z1);
                            w[i] = pack2<T>(e0, e1);
                            acc2 = f2_fma(f2_pack(e0, e1), ONE2, acc2);
                        }
                        tm_st16_nowait(tSb + (uint32_t)(16 * h), w);
                    }
                };
                if (whole) exps(std::integral_constant<int, 0>{});
                else if (vmask == all_pieces) exps(std::integral_constant<int, 1>{});
                else exps(std::integral_constant<int, 2>{});
                tm_wait_st();
                {
                    float a0, a1;
                    f2_unpack(acc2, a0, a1);
                    l += a0 + a1;
                }
                if ((c + 1) * PF_KT > kend || vmask != all_pieces) {
                    // rows past the item's key range or of a skipped block: zero V
                    // (both tiles' warps write the same zeros) once the stage's copy
                    // has landed, visible to the MMA's async-proxy reads
                    const int x = it.g + c, st = x % nst;
                    ok = __all_sync(PF_FULL, pf_wait(full + st, (x / nst) & 1, abort_flag, p.err));
                    if (!ok) break;
                    const int key = c * PF_KT + r;
                    if (r < PF_KT && (key >= kend || !((vmask >> (r >> prl)) & 1u))) {
                        uint8_t* vrow = smem + ly.ring(st) + LY::KV_BYTES + r * 128;
#pragma unroll
                        for (int bx = 0; bx < LY::NBOX; ++bx)
#pragma unroll
                            for (int q8 = 0; q8 < 8; ++q8)
                                *reinterpret_cast<uint4*>(vrow + bx * LY::KBOX + q8 * 16) = make_uint4(0, 0, 0, 0);
                        fence_proxy_async_smem();
                    }
                }
                tc::fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tbar(t, 2, b));
            }
            if (!ok) break;
            // the next item before this one's epilogue
            PfItem nxt;
            uint32_t nmc = 0, nmn = 0;
            ok = take(k + 1, nxt, nmc, nmn);
            if (mine && ok) {
                // epilogue: O holds every PV of the item once the last is
                // complete; the next item's first PV overwrites O only after
                // this warp's P of that item, i.e. after these loads
                if (my_nkt > 0)
                    ok = __all_sync(PF_FULL, pf_wait(tbar(t, 3, (gs - 1) & 1), ((gs - 1) >> 1) & 1,
                                                     abort_flag, p.err));
                if (!ok) break;
                tc::fence_after();
                const bool store = r / G < it.rows[t];
                const float inv = l > 0.f ? 1.f / l : 0.f;
                T* dst = reinterpret_cast<T*>(p.out) + ((size_t)(it.a + crow) * p.Hq + (size_t)it.j * G + g) * D;
#pragma unroll
                for (int h = 0; h < D / 64; ++h) {
                    uint32_t o[64];
                    if (my_nkt > 0) {
                        tm_ld64(tO + (uint32_t)(64 * h) + lq, o);
                    } else {
#pragma unroll
                        for (int i = 0; i < 64; ++i) o[i] = 0u;
                    }
                    uint32_t w[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        w[i] = pack2<T>(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
                    if (store) {
                        // each lane writes its own row: whole 32-byte sectors a
                        // store when the rows are 32-byte aligned
                        if (p.out32) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) st_global_v8(dst + 64 * h + 16 * i, &w[8 * i]);
                        } else {
                            uint4* o4 = reinterpret_cast<uint4*>(dst + 64 * h);
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                o4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                        }
                    }
                }
            }
            it = nxt;
            mask_cur = nmc;
            mask_next = nmn;
        }
    }

    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 9) tc::dealloc(tmem, LY::TM_COLS);
    // the last CTA to finish leaves the item counter at zero for the next call
    if (tid == 0) {
        __threadfence();
        if (atomicAdd(p.ws + 1, 1) == (int)gridDim.x - 1) {
            p.ws[0] = 0;
            p.ws[1] = 0;
            __threadfence();
        }
    }
}

// ------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 pf_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// Tensor map of `rank` dims (innermost first), 128-byte inner box, 128B swizzle.
int pf_map(CUtensorMap* map, const void* base, pa_dtype dt, int rank, const cuuint64_t* dims,
           const cuuint64_t* strides, const cuuint32_t* box) {
    auto fn = pf_encode_fn();
    if (!fn) return PA_ERR_CUDA;
    const CUtensorMapDataType t =
        dt == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, t, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

struct PfLaunch {
    CUtensorMap kmap, vmap, qmap;
    PrefillParams p;
    dim3 grid;
    cudaStream_t stream;
};

template <typename T, int D, int G>
int pf_run(PfLaunch& L) {
    using LY = PfLayout<D>;
    int dev = 0, optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return PA_ERR_CUDA;
    int nst = PF_MAX_STAGES;
    while (nst > 2 && LY(nst).total() + 1024 > (size_t)optin) --nst;
    const size_t smem = LY(nst).total() + 1024;
    if (smem > (size_t)optin) return PA_ERR_UNSUPPORTED;
    L.p.nst = nst;
    auto kern = prefill_tc_kernel<T, D, G>;
    static bool attr_set[64] = {};
    static std::mutex mu;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!attr_set[dev & 63]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin) !=
                cudaSuccess)
                return PA_ERR_CUDA;
            attr_set[dev & 63] = true;
        }
    }
    {
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return PA_ERR_CUDA;
        // the register split must fit in what the block is launched with, or
        // the softmax warpgroups would wait for registers for ever
        if ((long)fa.numRegs * PF_THREADS < 256L * PF_REGS_HIGH + 128L * PF_REGS_LOW) return PA_ERR_UNSUPPORTED;
    }
    kern<<<L.grid, PF_THREADS, smem, L.stream>>>(L.kmap, L.vmap, L.qmap, L.p);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <typename T, int D>
int pf_dispatch_g(PfLaunch& L, int G) {
    switch (G) {
        case 1: return pf_run<T, D, 1>(L);
        case 2: return pf_run<T, D, 2>(L);
        case 4: return pf_run<T, D, 4>(L);
        case 8: return pf_run<T, D, 8>(L);
        default: return PA_ERR_UNSUPPORTED;
    }
}

template <typename T>
int pf_dispatch(PfLaunch& L, int D, int G) {
    return D == 64 ? pf_dispatch_g<T, 64>(L, G) : pf_dispatch_g<T, 128>(L, G);
}

bool pf_aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

}  // namespace
}  // namespace pa

extern "C" {

int pa_prefill(void* out, const void* query, const void* key_cache, const void* value_cache,
               const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
               const int32_t* cu_seqlens_q, int num_seqs, int total_q, int max_query_len,
               int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
               float scale, void* workspace, size_t workspace_bytes, pa_dtype dtype,
               int32_t* err_flag, void* stream) {
    using namespace pa;
    if (num_seqs == 0 || total_q == 0) return PA_OK;
    if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens ||
        !cu_seqlens_q || !workspace)
        return PA_ERR_INVALID;
    if (workspace_bytes < PA_PREFILL_WORKSPACE_BYTES || (reinterpret_cast<uintptr_t>(workspace) & 15))
        return PA_ERR_INVALID;
    if (!(scale > 0.f) || !(scale < INFINITY)) return PA_ERR_INVALID;
    if (num_seqs < 0 || total_q < 0 || max_query_len <= 0 || num_q_heads <= 0 ||
        num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0)
        return PA_ERR_INVALID;
    if (dtype == PA_F32) return PA_ERR_UNSUPPORTED;
    if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_INVALID;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    const int G = num_q_heads / num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
    if (block_size != 8 && block_size != 16 && block_size != 32 && block_size != 64 &&
        block_size != 128)
        return PA_ERR_UNSUPPORTED;
    if (!pf_aligned16(out) || !pf_aligned16(query) || !pf_aligned16(key_cache) ||
        !pf_aligned16(value_cache))
        return PA_ERR_INVALID;
    const int64_t rows = (int64_t)num_blocks * num_kv_heads * block_size;
    if (rows >= (int64_t(1) << 31) || (int64_t)total_q * num_q_heads >= (int64_t(1) << 31))
        return PA_ERR_UNSUPPORTED;
    const int QT = PF_M / G;
    const int nqt = (max_query_len + QT - 1) / QT;
    const int npair = (nqt + PF_TILES - 1) / PF_TILES;
    const int64_t n_items = (int64_t)npair * num_seqs * num_kv_heads;
    if (n_items >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
    // persistent: one CTA per SM (no more than there are items)
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return PA_ERR_CUDA;
    const int64_t grid = std::min<int64_t>(n_items, sms);

    static thread_local PfLaunch L;
    const cuuint64_t esz = 2;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
        const cuuint64_t strides[1] = {(cuuint64_t)head_dim * esz};
        const cuuint32_t box[2] = {64, (cuuint32_t)std::min(block_size, 16)};
        int st = pf_map(&L.kmap, key_cache, dtype, 2, dims, strides, box);
        if (st == PA_OK) st = pf_map(&L.vmap, value_cache, dtype, 2, dims, strides, box);
        if (st != PA_OK) return st;
    }
    {
        // queries as [total_q][Hq][D]: a box is 64 columns x the G heads of one
        // KV head x QT chunk tokens = 128 rows of 128 bytes
        const cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_q_heads, (cuuint64_t)total_q};
        const cuuint64_t strides[2] = {(cuuint64_t)head_dim * esz,
                                       (cuuint64_t)num_q_heads * head_dim * esz};
        const cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)QT};
        int st = pf_map(&L.qmap, query, dtype, 3, dims, strides, box);
        if (st != PA_OK) return st;
    }
    PrefillParams& p = L.p;
    p.out = out;
    p.q = query;
    p.tables = block_tables;
    p.lens = context_lens;
    p.cu = cu_seqlens_q;
    p.S = num_seqs;
    p.total_q = total_q;
    p.max_q = max_query_len;
    p.npair = npair;
    p.Hq = num_q_heads;
    p.Hkv = num_kv_heads;
    p.mbps = max_blocks_per_seq;
    p.NB = num_blocks;
    p.bs = block_size;
    p.bs_log2 = __builtin_ctz((unsigned)block_size);
    p.scale_log2e = scale * 1.4426950408889634f;
    p.err = err_flag;
    p.n_items = (int)n_items;
    p.out32 = (reinterpret_cast<uintptr_t>(out) & 31) == 0 ? 1 : 0;
    p.ws = static_cast<int*>(workspace);
    L.grid = dim3((unsigned)grid);
    L.stream = (cudaStream_t)stream;
    return dtype == PA_F16 ? pf_dispatch<__half>(L, head_dim, G)
                           : pf_dispatch<__nv_bfloat16>(L, head_dim, G);
}

}  // extern "C"
