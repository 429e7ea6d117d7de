// pa_decode: paged decode attention for sm_100a (B200).
//
// What it computes ("KV Cache & PagedAttention" studynote, II-III: attention
// reads K/V scattered over blocks through the block table; "09. PagedAttention"
// (119-ai-studio), 해법: logical blocks -> physical blocks): for sequence s,
// query head h, KV head j = h / G and tokens t < L_s,
//   x_t = scale <q_h, K_t>,  out_h = sum_t softmax(x)_t V_t,
//   K_t = key_cache[block_tables[s][t / bs]][j][t % bs][:].
//
// How (one launch per decode step):
//  * Work unit = (sequence s, KV head j, partition i) covering tokens
//    [i*P, min(L_s, (i+1)*P)).  All G query heads of the group are served by
//    one pass over the group's K/V, so every K/V byte is read from HBM once.
//  * Persistent CTAs (one per SM), each running several independent
//    pipelines.  Each CTA computes the prefix sums of the partition counts
//    (tiny); then a pipeline's producer warp takes units from an atomic
//    counter in the workspace (dynamic load balance, units of at most P
//    tokens) and streams each unit as 16-token stages into its shared-memory
//    ring: 2-D tensor TMA copies of 128-byte-wide boxes with 128B swizzle, one
//    box row per token.  The block table is read 32 entries at a time by the
//    producer's lanes, ahead of use.  A 16-token stage never crosses a block
//    (bs >= 16) or covers two (bs = 8).
//  * Two compute engines read the same stages:
//      CUDA cores (fp32, and the default for G = 1): consumer warps take a
//        unit's stages round-robin and keep a per-warp online softmax in the
//        log2 domain; 8 (or 16) lanes per token and packed fp32x2 FMAs.
//      Tensor cores (tcgen05, 16-bit types, the default for G > 1): one
//        thread issues S = Q K^T (M = 64 rows = query heads, rows >= G
//        unused, N = 16 tokens) with Q and K read from shared memory through
//        swizzled matrix descriptors and S accumulated in tensor memory; a
//        softmax warp turns S into P (16-bit, in tensor memory) and the same
//        thread issues O += P V with O resident in tensor memory for the
//        whole unit.  The running max is only moved when it grows by more
//        than 2^8, so O is rescaled rarely (exact: O, l and m stay
//        consistent).
//  * A single-partition sequence writes `out` directly.  Otherwise each unit
//    writes its (m, l, o) to the workspace and a second, fully parallel
//    kernel (one CTA per sequence and query head) merges the partitions with
//    their log-sum-exp weights.  No CTA ever waits for another.
//  * Summation order depends only on logical positions (stage index within
//    the unit, warp index, partition index), never on physical block ids or
//    on which CTA ran a unit, so results are bit-identical under any
//    permutation of the pool and for block sizes 16..128.
//  * Every wait is bounded (2 s); a timeout sets PA_DEV_TIMEOUT, makes the
//    other warps give up quickly, waits (bounded) for the CTA's own copies and
//    MMAs in flight, frees its tensor memory and returns.  Bad block ids or
//    lengths set err_flag and the affected tokens are skipped.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstddef>
#include <cstring>
#include <mutex>

#include "pa_common.cuh"
#include "pa_tcgen05.cuh"

namespace pa {

constexpr int TOK = 16;           // tokens per pipeline stage
// consumer warps per pipeline of the CUDA-core engine (they take a unit's
// stages round-robin).  A ring slot stays held while its consumer computes, so
// extra consumers only pay where compute is the limit: 3 with query groups
// (G > 1), otherwise 2.
template <int G> constexpr int cons_for() { return G > 1 ? 3 : 2; }
// independent producer/consumer pipelines per CTA: 4, or 2 when a stage is
// 16 KB (fp32, head_dim 128) so that the rings still fit in shared memory
template <typename T, int D> constexpr int pipes_for() { return sizeof(T) * D > 256 ? 2 : 4; }
constexpr int NUR = 4;            // unit-descriptor slots per pipeline
constexpr int BOXB = TOK * 128;   // bytes of one 16-row x 128-byte box

struct alignas(16) UnitDesc {
    int s, j, i, t0, t1, n_p, stage_base, n_stages, end, pad0, pad1, pad2;
};

struct alignas(16) WsHeader {
    int next_unit;   // dynamic scheduler ticket
    int done_ctas;   // CTAs finished; the last one re-zeroes both
    int dirty;       // a CTA gave up: the last CTA re-zeroes the split counters too
    int pad[61];
};

struct DecodeParams {
    void* out;
    const void* q;
    const int32_t* tables;
    const int32_t* lens;
    int mbps, max_len, S, Hq, Hkv, NB, bs, bs_log2, P, n_pmax, nst;
    float scale_log2e;
    WsHeader* hdr;
    int hold_stage;    // test hook: stage of unit 0 that its producer withholds (-1: none)
    float* part_ml;    // [S*Hkv][n_pmax][G][2]
    float* part_o;     // [S*Hkv][n_pmax][G][D]
    int* split_cnt;    // [S*Hkv] partitions of a split (sequence, KV head) finished so far
    int fused_merge;   // the unit finishing a split last merges it (no merge kernel)
    int32_t* err;
    // the step's cache write done by the decode call (wslot null: none): row
    // s of wk / wv (16-byte pieces, [S][Hkv][D]) goes to slot wslot[s], which
    // must be the slot of position lens[s] - 1; kc / vc are the caches
    const uint4* wk;
    const uint4* wv;
    const int64_t* wslot;
    uint4* kc;
    uint4* vc;
};

// Shared-memory layout (dynamic, 1024-byte aligned base).  Every pipeline has
// its own stage ring, unit-descriptor ring, barriers, scratch and merge buffer.
template <typename T, int D, int G, int NCONS_ = 3>
struct Layout {
    static constexpr int NCONS = NCONS_;
    static constexpr int PIPE_WARPS = 1 + NCONS;
    static constexpr int NPIPE = pipes_for<T, D>();
    static constexpr int NTHREADS = NPIPE * PIPE_WARPS * 32;
    static constexpr int E = sizeof(T);
    static constexpr int ROWB = D * E;               // bytes per token row
    static constexpr int NBOX = ROWB / 128;          // 128-byte boxes per row
    static constexpr int KV_BYTES = NBOX * BOXB;     // one stage of K (or V)
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;
    static constexpr int QB = ((G * D * E + 127) / 128) * 128;
    static constexpr int UNIT_BYTES = (int)sizeof(UnitDesc) + QB;
    static constexpr int QF = G * D * 4;                         // per pipe: fp32 scaled q
    static constexpr int SCRATCH = NCONS * 3 * G * TOK * 4 + QF; // per pipe: xs, (p, p) pairs, q
    static constexpr int MBUF = NCONS * G * (D + 2) * 4;         // per pipe
    int nst, S;                                                  // stages per pipe
    __host__ __device__ Layout(int nst_, int S_) : nst(nst_), S(S_) {}
    __host__ __device__ size_t ring(int pipe) const { return (size_t)pipe * nst * STAGE_BYTES; }
    __host__ __device__ size_t units() const { return (size_t)NPIPE * nst * STAGE_BYTES; }
    __host__ __device__ size_t unit(int pipe, int k) const {
        return units() + (size_t)(pipe * NUR + k) * UNIT_BYTES;
    }
    __host__ __device__ size_t bars(int pipe) const {
        return units() + (size_t)NPIPE * NUR * UNIT_BYTES + (size_t)pipe * (2 * nst + 2 * NUR) * 8;
    }
    __host__ __device__ size_t stage_ok(int pipe) const { return bars(NPIPE) + (size_t)pipe * nst * 4; }
    __host__ __device__ size_t scratch(int pipe) const {
        return ((stage_ok(NPIPE) + 15) / 16) * 16 + (size_t)pipe * SCRATCH;
    }
    __host__ __device__ size_t mbuf(int pipe) const { return scratch(NPIPE) + (size_t)pipe * MBUF; }
    __host__ __device__ size_t misc() const { return mbuf(NPIPE); }              // 64 ints
    __host__ __device__ size_t lens() const { return misc() + 256; }
    __host__ __device__ size_t pre() const { return lens() + 4 * (size_t)S; }
    __host__ __device__ size_t total() const { return pre() + 4 * (size_t)(S + 1); }
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ int clamp_len(int L, const DecodeParams& p) {
    const int hi = min(p.max_len, p.mbps * p.bs);
    if (L < 0 || L > hi) {
        set_err(p.err, PA_DEV_BAD_LEN);
        L = max(0, min(L, hi));
    }
    return L;
}

__device__ __forceinline__ int n_parts(int L, int P) { return max(1, ceil_div(L, P)); }

// Orders this thread's generic-proxy global writes before later async-proxy
// (TMA) accesses of global memory.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// The step's new token of sequence s: whether wslot[s] = `slot` is to be
// written, i.e. non-negative and equal to the slot the table gives position
// pos = L - 1 (block bl, row pos % bs).  A mismatch sets PA_DEV_BAD_SLOT when
// `report`; a negative slot is a skipped write, no error.
__device__ __forceinline__ bool new_token_slot_ok(const DecodeParams& p, int64_t slot, int pos,
                                                  int bl, bool report) {
    if (slot < 0) return false;
    const bool ok = pos >= 0 && bl >= 0 && bl < p.NB &&
                    slot == (int64_t)bl * p.bs + (pos & (p.bs - 1));
    if (!ok && report) set_err(p.err, PA_DEV_BAD_SLOT);
    return ok;
}

// Copies KV head j's K and V rows of sequence s's new token into block bl,
// row pos % bs: 2 * nv 16-byte pieces, this thread's from i0 in steps of di.
__device__ __forceinline__ void put_new_token(const DecodeParams& p, int s, int j, int pos, int bl,
                                              int nv, int i0, int di) {
    const size_t src = ((size_t)s * p.Hkv + j) * nv;
    const size_t dst = (((size_t)bl * p.Hkv + j) * p.bs + (pos & (p.bs - 1))) * nv;
    for (int e = i0; e < 2 * nv; e += di) {
        const bool isv = e >= nv;
        const int x = isv ? e - nv : e;
        (isv ? p.vc : p.kc)[dst + x] = __ldg((isv ? p.wv : p.wk) + src + x);
    }
}

// The step's cache write for engines that do not do it inside the decode
// kernel: one CTA per sequence, every KV head, with the same slot check.  A
// programmatic dependent of the kernel before it; it lets the decode after it
// launch at once (it writes neither lengths nor tables), which waits for its
// completion before reading the cache.
__global__ void __launch_bounds__(128) new_token_write_kernel(DecodeParams p, int nv) {
    grid_dependency_wait();
    launch_dependents();
    const int s = blockIdx.x;
    const int64_t slot = __ldg(p.wslot + s);
    if (slot < 0) return;
    const int L = clamp_len(__ldg(p.lens + s), p);
    const int pos = L - 1;
    const int bl = pos >= 0 ? __ldg(p.tables + (size_t)s * p.mbps + (pos >> p.bs_log2)) : -1;
    if (!new_token_slot_ok(p, slot, pos, bl, threadIdx.x == 0)) return;
    for (int j = 0; j < p.Hkv; ++j) put_new_token(p, s, j, pos, bl, nv, threadIdx.x, blockDim.x);
}

// Bounded wait that also gives up as soon as another warp has given up.
// mbar_try_wait sleeps until the phase completes (suspend hint), so the abort
// flag and the clock are looked at only when a probe comes back empty.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag, int32_t* err) {
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

// Bounded wait until a ring slot's tag (2 * stage + valid, written by the
// producer before it arms the slot's barrier) names global stage `g`.  Gives
// up like wait_or_abort; on success *tag holds the value read.
__device__ __forceinline__ bool wait_tag(const volatile int* slot_tag, int g, int* tag,
                                         volatile int* abort_flag, int32_t* err) {
    if ((*tag = *slot_tag) >> 1 == g) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        if ((*tag = *slot_tag) >> 1 == g) return true;
        if (*abort_flag) return false;
        if ((it & 63) == 0 && global_ns() - t0 > kWaitLimitNs) {
            set_err(err, PA_DEV_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

// Sum over the LPT lanes of one token of v[h(lane)], h(lane) = (lane % LPT) / (LPT / G):
// a butterfly that halves the head set at each step while G > 1.
template <int G, int LPT>
__device__ __forceinline__ float reduce_scatter(float (&v)[G], int lane) {
    float a[G];
#pragma unroll
    for (int k = 0; k < G; ++k) a[k] = v[k];
    int cnt = G;
#pragma unroll
    for (int off = LPT / 2; off >= 1; off >>= 1) {
        if (cnt > 1) {
            const int half = cnt / 2;
            const bool upper = (lane & off) != 0;
#pragma unroll
            for (int k = 0; k < half; ++k) {
                const float send = upper ? a[k] : a[k + half];
                const float keep = upper ? a[k + half] : a[k];
                a[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
            }
            cnt = half;
        } else {
            a[0] += __shfl_xor_sync(0xffffffffu, a[0], off);
        }
    }
    return a[0];
}

// ------------------------------------------------------------ compute engines
// Per-warp online-softmax state and one stage's update.  Stage smem: K boxes
// then V boxes; box b holds columns [b*128, b*128+128) bytes of 16 rows, with
// the 16-byte chunk c of row r stored at chunk position c ^ (r & 7).

template <typename T, int D, int G>
struct CoreEngine {
    using LY = Layout<T, D, G, cons_for<G>()>;
    static constexpr int E = sizeof(T);
    static constexpr int VEC = 16 / E;                       // elements per 16-byte chunk
    static constexpr int NP = VEC / 2;                       // fp32 pairs per chunk
    static constexpr int CHUNKS = LY::ROWB / 16;             // chunks per row
    static constexpr int LPT = (G >= 8 && CHUNKS >= 16) ? 16 : 8;
    static constexpr int TPW = 32 / LPT;                     // tokens per warp step
    static constexpr int NCH = CHUNKS / LPT;                 // chunks per lane
    static constexpr int DPL = D / 32;                       // PV columns per lane
    static constexpr int DPP = DPL / 2;                      // PV column pairs per lane
    static constexpr int NPASS = (G + 1) / 2;
    static_assert(G <= LPT, "group larger than lanes per token");

    // All arithmetic on fp32 pairs (fma.rn.f32x2).  q lives in shared memory as
    // pre-scaled fp32, laid out [g][chunk c][k/2][lane r] in 16-byte units
    // (two pairs), so the q reads of one step are conflict-free.
    static constexpr int QUNITS = G * NCH * (NP / 2) * LPT;   // 16-byte units of q
    uint64_t o2[G][DPP];
    float m_half[NPASS], l_half[NPASS];
    const uint4* qf = nullptr;

    // Cooperative (all consumer threads of the pipeline): storage q -> fp32 scaled,
    // interleaved.  Caller synchronises before the first stage.
    static __device__ void stage_q(const T* qs, uint4* qf4, int ctid, int nthreads, float scale) {
        for (int u = ctid; u < QUNITS; u += nthreads) {
            const int r = u % LPT, kk = (u / LPT) % (NP / 2), c = (u / (LPT * (NP / 2))) % NCH;
            const int g = u / (LPT * (NP / 2) * NCH);
            const int e0 = (r + c * LPT) * VEC + 4 * kk;
            float4 f;
            f.x = DT<T>::to_float(qs[g * D + e0 + 0]) * scale;
            f.y = DT<T>::to_float(qs[g * D + e0 + 1]) * scale;
            f.z = DT<T>::to_float(qs[g * D + e0 + 2]) * scale;
            f.w = DT<T>::to_float(qs[g * D + e0 + 3]) * scale;
            qf4[u] = *reinterpret_cast<uint4*>(&f);
        }
    }

    __device__ void begin_unit(const uint4* qf4) {
        qf = qf4;
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int k = 0; k < DPP; ++k) o2[g][k] = 0ull;
#pragma unroll
        for (int k = 0; k < NPASS; ++k) { m_half[k] = -INFINITY; l_half[k] = 0.f; }
    }

    // xs: [G][TOK] logits; ps2: [TOK][G] splatted (p, p) pairs.
    __device__ void stage(const uint8_t* Ks, const uint8_t* Vs, int nv, float* xs, uint64_t* ps2,
                          int lane) {
        const int r = lane % LPT;
        // ---- x_t = <q_g, K_t> (pre-scaled to log2 units)
#pragma unroll
        for (int step = 0; step < TOK / TPW; ++step) {
            const int tok = step * TPW + lane / LPT;
            uint64_t acc2[G];
#pragma unroll
            for (int g = 0; g < G; ++g) acc2[g] = 0ull;
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                const int ch = r + c * LPT;
                const uint4 raw = *reinterpret_cast<const uint4*>(
                    Ks + (ch >> 3) * BOXB + tok * 128 + (((ch & 7) ^ (tok & 7)) << 4));
                uint64_t x2[NP];
                pairs16<T>(raw, x2);
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int kk = 0; kk < NP / 2; ++kk) {
                        const uint4 q4 = qf[((g * NCH + c) * (NP / 2) + kk) * LPT + r];
                        acc2[g] = f2_fma((uint64_t)q4.x | ((uint64_t)q4.y << 32), x2[2 * kk], acc2[g]);
                        acc2[g] = f2_fma((uint64_t)q4.z | ((uint64_t)q4.w << 32), x2[2 * kk + 1], acc2[g]);
                    }
            }
            float acc[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float lo, hi;
                f2_unpack(acc2[g], lo, hi);
                acc[g] = lo + hi;
            }
            const float v = reduce_scatter<G, LPT>(acc, lane);
            constexpr int LPH = LPT / G;           // lanes holding one head's total
            if ((r % LPH) == 0) xs[(r / LPH) * TOK + tok] = (tok < nv) ? v : -INFINITY;
        }
        __syncwarp();
        // ---- online softmax over the stage's tokens, two heads per pass
        uint64_t alpha2[G];
#pragma unroll
        for (int pass = 0; pass < NPASS; ++pass) {
            const int g = 2 * pass + (lane >> 4);
            const int t = lane & 15;
            const bool live = g < G;
            const float x = live ? xs[g * TOK + t] : -INFINITY;
            float bm = x;
#pragma unroll
            for (int off = 8; off >= 1; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
            const float mo = m_half[pass];
            const float mn = fmaxf(mo, bm);
            const float pr = live ? exp2f(x - mn) : 0.f;
            float sum = pr;
#pragma unroll
            for (int off = 8; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            const float a = live ? exp2f(mo - mn) : 1.f;
            if (live) {
                m_half[pass] = mn;
                l_half[pass] = l_half[pass] * a + sum;
                ps2[t * G + g] = f2_pack(pr, pr);
            }
            const float a0 = __shfl_sync(0xffffffffu, a, 0);
            alpha2[2 * pass] = f2_pack(a0, a0);
            if (2 * pass + 1 < G) {
                const float a1 = __shfl_sync(0xffffffffu, a, 16);
                alpha2[2 * pass + 1] = f2_pack(a1, a1);
            }
        }
        __syncwarp();
        // ---- o = alpha o + sum_t p_t V_t
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int k = 0; k < DPP; ++k) o2[g][k] = f2_mul(alpha2[g], o2[g][k]);
        const int byte = lane * DPL * E;                  // this lane's columns
        const int box = byte >> 7, cc = (byte & 127) >> 4, sub = byte & 15;
        auto pv_token = [&](int t) {
            const uint8_t* src = Vs + box * BOXB + t * 128 + (((cc ^ (t & 7)) << 4) | sub);
            uint64_t v2[DPP];
            if constexpr (DPL * E == 16) {
                pairs16<T>(*reinterpret_cast<const uint4*>(src), v2);
            } else if constexpr (DPL * E == 8) {
                const uint2 raw = *reinterpret_cast<const uint2*>(src);
                if constexpr (E == 4) {
                    v2[0] = (uint64_t)raw.x | ((uint64_t)raw.y << 32);
                } else {
                    v2[0] = Pairs<T>::from_word(raw.x);
                    v2[1] = Pairs<T>::from_word(raw.y);
                }
            } else {
                v2[0] = Pairs<T>::from_word(*reinterpret_cast<const uint32_t*>(src));
            }
            uint64_t p2[G];
#pragma unroll
            for (int g = 0; g < G; ++g) p2[g] = ps2[t * G + g];
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int k = 0; k < DPP; ++k) o2[g][k] = f2_fma(p2[g], v2[k], o2[g][k]);
        };
        if (nv == TOK) {
#pragma unroll
            for (int t = 0; t < TOK; ++t) pv_token(t);
        } else {
            for (int t = 0; t < nv; ++t) pv_token(t);
        }
        __syncwarp();
    }

    // Write this warp's (m, l, o) into the merge buffer [G][D+2].
    __device__ void dump(float* mb, int lane) const {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int k = 0; k < DPP; ++k) {
                float lo, hi;
                f2_unpack(o2[g][k], lo, hi);
                mb[g * (D + 2) + 2 + lane * DPL + 2 * k] = lo;
                mb[g * (D + 2) + 2 + lane * DPL + 2 * k + 1] = hi;
            }
#pragma unroll
        for (int pass = 0; pass < NPASS; ++pass) {
            const int g = 2 * pass + (lane >> 4);
            if ((lane & 15) == 0 && g < G) {
                mb[g * (D + 2) + 0] = m_half[pass];
                mb[g * (D + 2) + 1] = l_half[pass];
            }
        }
    }
};

// ------------------------------------------------------------ pieces shared by both kernels

// Stage format (both engines): K boxes then V boxes; box b holds byte columns
// [b*128, b*128+128) of 16 token rows, 16-byte chunk c of row r at chunk
// position c ^ (r & 7) (the TMA 128-byte swizzle).
template <typename T, int D>
struct Ring {
    static constexpr int E = sizeof(T);
    static constexpr int ROWB = D * E;               // bytes per token row
    static constexpr int NBOX = ROWB / 128;          // 128-byte boxes per row
    static constexpr int KV_BYTES = NBOX * BOXB;     // one stage of K (or V)
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;
};

// Prefix sums of the partition counts per sequence, by all threads of the CTA;
// fills lens_s[S] (clamped lengths) and pre[S + 1].  Ends with __syncthreads.
template <int NTHREADS>
__device__ void prefix_sums(const DecodeParams& p, int* lens_s, int* pre, int* wsum, int tid) {
    constexpr int NW = NTHREADS / 32;
    static_assert(NW <= 32, "one warp scans the warp totals");
    const int warp = tid >> 5, lane = tid & 31;
    const int per = (p.S + NTHREADS - 1) / NTHREADS;
    const int beg = min(p.S, tid * per), end = min(p.S, beg + per);
    int local = 0;
    for (int k = beg; k < end; ++k) {
        const int L = clamp_len(__ldg(p.lens + k), p);
        lens_s[k] = L;
        local += n_parts(L, p.P);
    }
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = (lane < NW) ? wsum[lane] : 0;
        int iv = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, iv, off);
            if (lane >= off) iv += u;
        }
        if (lane < NW) wsum[lane] = iv - v;          // exclusive warp offsets
    }
    __syncthreads();
    int run = wsum[warp] + incl - local;
    for (int k = beg; k < end; ++k) {
        pre[k] = run;
        run += n_parts(lens_s[k], p.P);
    }
    if (tid == NTHREADS - 1) pre[p.S] = run;
    __syncthreads();
}

// One pipeline's shared-memory rings, as seen by its producer.
struct PipeRings {
    uint8_t* stages;
    uint64_t *full, *empty;     // per stage slot
    uint64_t *ufull, *uempty;   // per unit slot
    int* stage_ok;              // per stage slot: tag 2 * global stage + valid
    int nst, nu;
};

// ================================================= producer warp
// Per unit: the next unit's ticket (global atomic) and its first 64 block ids
// are fetched while the current unit's stages are issued, so no global round
// trip sits between two stages.  The TMA copies of a stage are issued by
// several lanes at once.  desc_at(k) gives unit slot k's descriptor;
// load_q(k, s, j, bar) (lane 0) arms `bar` and starts the copy of the
// group's G query rows into slot k.
template <typename T, int D, class DescAt, class LoadQ>
__device__ void producer_loop(const CUtensorMap* kmap, const CUtensorMap* vmap,
                              const DecodeParams& p, const PipeRings& rg, const int* pre,
                              const int* lens_s, int U, volatile int* abort_flag, int lane,
                              DescAt desc_at, LoadQ load_q) {
    using R = Ring<T, D>;
    constexpr int BOX_ELEMS = 128 / R::E;
    const int nst = rg.nst, NU = rg.nu;
    const uint64_t policy = policy_evict_first();
    const int bs = p.bs, bsl = p.bs_log2;
    const int npiece = (bs >= TOK) ? 1 : TOK / bs;   // blocks per stage
    const int prow = (bs >= TOK) ? TOK : bs;         // box rows per block piece
    struct Plan {
        int u, s, j, i, t0, t1, nst, n_p, nblk;
        const int32_t* trow;   // block-table entries of this unit's first block
        int ids_a, ids_b;      // entries [win, win+32) and [win+32, win+64), one per lane
    };
    auto prepare = [&](int u) {
        Plan q{};
        q.u = u;
        if (u >= U) return q;
        const int x = u / p.Hkv;
        int lo = 0, hi = p.S;                      // pre[lo] <= x < pre[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (pre[mid] <= x) lo = mid; else hi = mid;
        }
        q.s = lo;
        q.i = x - pre[lo];
        q.j = u - x * p.Hkv;
        const int L = lens_s[lo];
        q.t0 = min(q.i * p.P, L);
        q.t1 = min(q.t0 + p.P, L);
        q.nst = (q.t1 - q.t0 + TOK - 1) / TOK;
        q.n_p = n_parts(L, p.P);
        const int b0 = q.t0 >> bsl;
        q.nblk = ((q.t1 + bs - 1) >> bsl) - b0;
        q.trow = p.tables + (size_t)lo * p.mbps + b0;
        q.ids_a = (lane < q.nblk) ? __ldg(q.trow + lane) : -1;
        q.ids_b = (lane + 32 < q.nblk) ? __ldg(q.trow + 32 + lane) : -1;
        return q;
    };
    int gstage = 0, st = 0, round = 0, ucount = 0;
    int ticket = 0;
    if (lane == 0) ticket = atomicAdd(&p.hdr->next_unit, 1);
    Plan cur = prepare(__shfl_sync(0xffffffffu, ticket, 0));
    bool ok = true;
    while (ok) {
        const int slot = ucount % NU;
        if (ucount >= NU) {
            bool w = true;
            if (lane == 0) w = wait_or_abort(rg.uempty + slot, ((ucount / NU) - 1) & 1, abort_flag, p.err);
            if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
        }
        UnitDesc* d = desc_at(slot);
        if (cur.u >= U) {
            if (lane == 0) {
                d->end = 1;
                mbar_arrive(rg.ufull + slot);
            }
            ++ucount;
            break;
        }
        if (lane == 0) {
            d->s = cur.s; d->j = cur.j; d->i = cur.i; d->t0 = cur.t0; d->t1 = cur.t1;
            d->n_p = cur.n_p;
            d->stage_base = gstage; d->n_stages = cur.nst; d->end = 0;
            load_q(slot, cur.s, cur.j, rg.ufull + slot);
            ticket = atomicAdd(&p.hdr->next_unit, 1);     // the unit after this one
        }
        ++ucount;
        Plan nxt{};
        bool have_next = false;
        int win = 0;                                // table index of ids_a's lane 0
        const int b0 = cur.t0 >> bsl;
        for (int c = 0; c < cur.nst; ++c) {
            const int tok0 = cur.t0 + c * TOK;
            if (round > 0) {
                bool w = true;
                if (lane == 0) w = wait_or_abort(rg.empty + st, (round - 1) & 1, abort_flag, p.err);
                if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
            }
            // physical block of each piece (one piece unless bs = 8)
            int blk0, blk1 = -2;
            const int off0 = tok0 & (bs - 1);
            {
                const int bi = (tok0 >> bsl) - b0;
                if (bi - win >= 32) {
                    win += 32;
                    cur.ids_a = cur.ids_b;
                    cur.ids_b = (lane + win + 32 < cur.nblk) ? __ldg(cur.trow + win + 32 + lane) : -1;
                }
                blk0 = __shfl_sync(0xffffffffu, cur.ids_a, (bi - win) & 31);
            }
            if (npiece == 2) {
                const int tok = tok0 + bs;
                const int bi = (tok >> bsl) - b0;
                if (bi - win >= 32) {
                    win += 32;
                    cur.ids_a = cur.ids_b;
                    cur.ids_b = (lane + win + 32 < cur.nblk) ? __ldg(cur.trow + win + 32 + lane) : -1;
                }
                const int id = __shfl_sync(0xffffffffu, cur.ids_a, (bi - win) & 31);
                if (tok < cur.t1) blk1 = id;
            }
            const bool has1 = blk1 != -2;
            const bool valid = blk0 >= 0 && blk0 < p.NB && (!has1 || (blk1 >= 0 && blk1 < p.NB));
            uint8_t* Kd = rg.stages + (size_t)st * R::STAGE_BYTES;
            if (cur.u == 0 && c == p.hold_stage) {
                // test hook: nothing will ever arrive on this stage's barrier
                ++gstage;
                if (++st == nst) { st = 0; ++round; }
                continue;
            }
            if (lane == 0) {
                rg.stage_ok[st] = 2 * gstage + (valid ? 1 : 0);   // the slot's tag
                if (!valid) {
                    set_err(p.err, PA_DEV_BAD_BLOCK);
                    mbar_arrive(rg.full + st);
                } else {
                    mbar_arrive_expect_tx(rg.full + st, (has1 ? 2u : 1u) * 2u * prow * R::ROWB);
                }
            }
            __syncwarp();
            // one TMA box per lane: (piece, K or V, 128-byte column box)
            const int nops = valid ? (has1 ? 2 : 1) * 2 * R::NBOX : 0;
            if (lane < nops) {
                const int piece = lane / (2 * R::NBOX), rem = lane % (2 * R::NBOX);
                const int kv = rem / R::NBOX, b = rem % R::NBOX;
                const int y = piece ? ((blk1 * p.Hkv + cur.j) << bsl)
                                    : (((blk0 * p.Hkv + cur.j) << bsl) + off0);
                uint8_t* dst = Kd + kv * R::KV_BYTES + b * BOXB + piece * 8 * 128;
                tma_load_2d(dst, kv ? vmap : kmap, b * BOX_ELEMS, y, rg.full + st, policy);
            }
            ++gstage;
            if (++st == nst) { st = 0; ++round; }
            if (!have_next && (c == 3 || c == cur.nst - 1)) {
                nxt = prepare(__shfl_sync(0xffffffffu, ticket, 0));
                have_next = true;
            }
        }
        if (!ok) break;
        if (!have_next) nxt = prepare(__shfl_sync(0xffffffffu, ticket, 0));
        cur = nxt;
    }
    // make sure no copy of this pipeline is still landing in shared memory
    if (lane == 0) {
        const int first = max(0, gstage - nst);
        for (int g = first; g < gstage; ++g) mbar_wait(rg.full + g % nst, (g / nst) & 1);
        const int ufirst = max(0, ucount - NU);
        for (int k = ufirst; k < ucount; ++k) mbar_wait(rg.ufull + k % NU, (k / NU) & 1);
    }
    __syncwarp();
}

// ------------------------------------------------------------ split-K merge kernels
// Launched after a decode kernel when a sequence may span several partitions.
// With the partials (m_i, l_i, o_i) of partition i (log2 domain, o not yet
// normalised), for each query head
//   M = max_i m_i,  out = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i.
// Sequences with a single partition were written by the decode kernel and are
// skipped.  Two shapes: short splits (few partitions) take one CTA per
// (sequence, KV head) with a thread per 4 output columns of all G heads;
// long splits take one CTA per (sequence, query head) with the partitions
// spread over thread slices, so no thread walks a long chain of loads.
constexpr int MERGE_THREADS = 256;
constexpr int kShortSplit = 32;     // partitions up to which the group shape is used

// Column dd of the G heads' outputs of (sequence s, KV head j) from its
// n_p <= fused_parts<G>() partials, in partition order (the same arithmetic as
// the merge kernels: exact zeros stand in for partitions past n_p).  All loads
// of a batch of heads (16 partials) are issued before any is used, so a merge
// costs G * NI / 16 round trips to L2 rather than one per partition.  Only
// short splits are merged this way: the merging unit's epilogue holds its CTA
// at the end of the schedule, where the last partitions of split sequences
// sit, so splits of more partitions are left to the merge kernel.  Reads through L2
// only: other CTAs wrote the partials.
template <int G> constexpr int fused_parts() { return 4; }
template <typename T, int D, int G>
__device__ __forceinline__ void merge_column(const DecodeParams& p, int s, int j, int dd, int n_p) {
    constexpr int NI = fused_parts<G>();
    // heads per batch: up to 16 (m, l, o) loads in flight, never past the group
    constexpr int HB = G < 16 / NI ? G : 16 / NI;
    static_assert(HB >= 1 && G % HB == 0, "batches cover the group's heads exactly");
    const size_t base = ((size_t)s * p.Hkv + j) * p.n_pmax;
#pragma unroll
    for (int h0 = 0; h0 < G; h0 += HB) {
        float2 ml[HB][NI];
        float o[HB][NI];
#pragma unroll
        for (int hh = 0; hh < HB; ++hh)
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                const size_t pi = (base + i) * G + h0 + hh;
                ml[hh][i] = i < n_p ? __ldcg(reinterpret_cast<const float2*>(p.part_ml) + pi)
                                    : make_float2(-INFINITY, 0.f);
                o[hh][i] = i < n_p ? __ldcg(p.part_o + pi * D + dd) : 0.f;
            }
#pragma unroll
        for (int hh = 0; hh < HB; ++hh) {
            float M = -INFINITY;
#pragma unroll
            for (int i = 0; i < NI; ++i) M = fmaxf(M, ml[hh][i].x);
            float acc = 0.f, Lsum = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int i = 0; i < NI; ++i) {
                    const float w = exp2f(ml[hh][i].x - M);
                    Lsum += w * ml[hh][i].y;
                    acc += w * o[hh][i];
                }
            }
            T* outp = reinterpret_cast<T*>(p.out) + ((size_t)s * p.Hq + (size_t)j * G + h0 + hh) * D + dd;
            *outp = DT<T>::from_float(acc * (Lsum > 0.f ? 1.f / Lsum : 0.f));
        }
    }
}

// atomicAdd with release and acquire semantics at GPU scope: the partials this
// CTA wrote (ordered before by a barrier) are visible to whoever sees the new
// count, and the partials of the units counted before are visible here.
__device__ __forceinline__ int atomic_add_acq_rel(int* addr, int v) {
    int old;
    asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v)
                 : "memory");
    return old;
}

template <typename T, int D>
__device__ __forceinline__ void merge_store(const DecodeParams& p, int s, int h, int col, float4 o, float inv) {
    T* outp = reinterpret_cast<T*>(p.out) + ((size_t)s * p.Hq + h) * D + 4 * col;
    outp[0] = DT<T>::from_float(o.x * inv);
    outp[1] = DT<T>::from_float(o.y * inv);
    outp[2] = DT<T>::from_float(o.z * inv);
    outp[3] = DT<T>::from_float(o.w * inv);
}

// One CTA of G * D / 4 <= MERGE_THREADS threads per (sequence, KV head):
// thread = (head g, 4 columns); every thread walks the few partitions itself.
// The loads of each pass are issued in batches before any is used (16 maxima,
// then 8 (m, l) pairs with their output columns), so a split of n_p partitions
// costs about n_p / 16 + n_p / 8 round trips to L2.  Small CTAs keep the whole
// grid resident at once.
template <typename T, int D>
__global__ void __launch_bounds__(MERGE_THREADS)
merge_group_kernel(DecodeParams p) {
    constexpr int NV = D / 4;
    constexpr int B1 = 16, B2 = 8;
    grid_dependency_wait();                          // the decode grid's partials are complete
    const int s = blockIdx.x / p.Hkv, j = blockIdx.x - s * p.Hkv;
    const int L = clamp_len(__ldg(p.lens + s), p);
    const int n_p = n_parts(L, p.P);
    if (n_p <= 1) return;                            // written by the decode kernel
    const int G = p.Hq / p.Hkv;
    const size_t base = ((size_t)s * p.Hkv + j) * p.n_pmax;
    for (int c = threadIdx.x; c < G * NV; c += blockDim.x) {
        const int g = c / NV, col = c - g * NV;
        float M = -INFINITY;
        for (int i0 = 0; i0 < n_p; i0 += B1) {
            float m[B1];
#pragma unroll
            for (int k = 0; k < B1; ++k)
                m[k] = i0 + k < n_p ? __ldcg(p.part_ml + ((base + i0 + k) * G + g) * 2) : -INFINITY;
#pragma unroll
            for (int k = 0; k < B1; ++k) M = fmaxf(M, m[k]);
        }
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float Lsum = 0.f;
        if (M != -INFINITY) {
            for (int i0 = 0; i0 < n_p; i0 += B2) {
                float2 ml[B2];
                float4 o[B2];
#pragma unroll
                for (int k = 0; k < B2; ++k) {
                    const size_t pi = (base + i0 + k) * G + g;
                    ml[k] = i0 + k < n_p ? __ldcg(reinterpret_cast<const float2*>(p.part_ml) + pi)
                                         : make_float2(-INFINITY, 0.f);
                    o[k] = i0 + k < n_p ? __ldcg(reinterpret_cast<const float4*>(p.part_o + pi * D) + col)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int k = 0; k < B2; ++k) {          // partition order
                    const float w = exp2f(ml[k].x - M);
                    Lsum += w * ml[k].y;
                    acc.x += w * o[k].x; acc.y += w * o[k].y; acc.z += w * o[k].z; acc.w += w * o[k].w;
                }
            }
        }
        merge_store<T, D>(p, s, j * G + g, col, acc, Lsum > 0.f ? 1.f / Lsum : 0.f);
    }
}

// One CTA per (sequence s, query head h); the partitions are spread over
// MERGE_THREADS / (D/4) slices, reduced in shared memory in a fixed order.
template <typename T, int D>
__global__ void __launch_bounds__(MERGE_THREADS)
merge_head_kernel(DecodeParams p) {
    constexpr int NV = D / 4;                        // float4 columns of a row
    constexpr int NS = MERGE_THREADS / NV;           // partition slices
    __shared__ float4 acc_s[NS][NV];
    __shared__ float l_s[NS], red[MERGE_THREADS / 32];
    grid_dependency_wait();                          // the decode grid's partials are complete
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int s = blockIdx.x / p.Hq, h = blockIdx.x - s * p.Hq;
    const int L = clamp_len(__ldg(p.lens + s), p);
    const int n_p = n_parts(L, p.P);
    if (n_p <= 1) return;                            // written by the decode kernel
    const int G = p.Hq / p.Hkv, j = h / G, g = h - j * G;
    const size_t base = ((size_t)s * p.Hkv + j) * p.n_pmax;
    auto ml = [&](int i, int k) { return __ldcg(p.part_ml + ((base + i) * G + g) * 2 + k); };
    float mx = -INFINITY;
    for (int i = tid; i < n_p; i += MERGE_THREADS) mx = fmaxf(mx, ml(i, 0));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    float M = red[0];
#pragma unroll
    for (int w = 1; w < MERGE_THREADS / 32; ++w) M = fmaxf(M, red[w]);
    const int col = tid % NV, slice = tid / NV;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll 4
        for (int i = slice; i < n_p; i += NS) {
            const float w = exp2f(ml(i, 0) - M);
            lsum += w * ml(i, 1);
            const float4 o = __ldcg(reinterpret_cast<const float4*>(p.part_o + ((base + i) * G + g) * D) + col);
            acc.x += w * o.x; acc.y += w * o.y; acc.z += w * o.z; acc.w += w * o.w;
        }
    }
    acc_s[slice][col] = acc;
    if (col == 0) l_s[slice] = lsum;
    __syncthreads();
    if (slice == 0) {
        float Lsum = 0.f;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < NS; ++k) {                // fixed order: deterministic
            Lsum += l_s[k];
            o.x += acc_s[k][col].x; o.y += acc_s[k][col].y; o.z += acc_s[k][col].z; o.w += acc_s[k][col].w;
        }
        merge_store<T, D>(p, s, h, col, o, Lsum > 0.f ? 1.f / Lsum : 0.f);
    }
}

// ------------------------------------------------------------ CUDA-core kernel
// Warp roles: warp w belongs to pipeline w / PIPE_WARPS; role w % PIPE_WARPS is
// 0 for the producer and 1..NCONS for the consumers.  The pipelines of a CTA
// share nothing but the prefix sums and the abort flag; each takes its own
// units from the global ticket counter.
template <typename T, int D, int G>
__global__ void __launch_bounds__(Layout<T, D, G, cons_for<G>()>::NTHREADS, 1)
decode_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
              DecodeParams p) {
    using LY = Layout<T, D, G, cons_for<G>()>;
    using Engine = CoreEngine<T, D, G>;
    constexpr int NCONS = LY::NCONS;
    constexpr int PIPE_WARPS = LY::PIPE_WARPS;
    constexpr int NPIPE = LY::NPIPE;
    constexpr int NTHREADS = LY::NTHREADS;
    constexpr int CT = NCONS * 32;               // consumer threads of a pipeline
    constexpr int E = sizeof(T);

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 128B-swizzled TMA boxes need 1024-byte aligned destinations
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const LY ly(p.nst, p.S);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int pipe = warp / PIPE_WARPS, role = warp % PIPE_WARPS;
    const int nst = p.nst;

    uint8_t* stages = smem + ly.ring(pipe);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + ly.bars(pipe));
    uint64_t* empty = full + nst;
    uint64_t* ufull = empty + nst;
    uint64_t* uempty = ufull + NUR;
    int* stage_ok = reinterpret_cast<int*>(smem + ly.stage_ok(pipe));
    float* scratch = reinterpret_cast<float*>(smem + ly.scratch(pipe));
    float* mbuf = reinterpret_cast<float*>(smem + ly.mbuf(pipe));
    int* misc = reinterpret_cast<int*>(smem + ly.misc());
    int* lens_s = reinterpret_cast<int*>(smem + ly.lens());
    int* pre = reinterpret_cast<int*>(smem + ly.pre());
    volatile int* abort_flag = misc + 0;
    int* wsum = misc + 32;
    auto desc_at = [&](int k) { return reinterpret_cast<UnitDesc*>(smem + ly.unit(pipe, k)); };
    auto q_at = [&](int k) {
        return reinterpret_cast<T*>(smem + ly.unit(pipe, k) + sizeof(UnitDesc));
    };

    if (tid == 0) {
        for (int pp = 0; pp < NPIPE; ++pp) {
            uint64_t* b = reinterpret_cast<uint64_t*>(smem + ly.bars(pp));
            for (int k = 0; k < 2 * nst + 2 * NUR; ++k) mbar_init(b + k, 1);
            int* tags = reinterpret_cast<int*>(smem + ly.stage_ok(pp));
            for (int k = 0; k < nst; ++k) tags[k] = -1;   // no stage issued yet
        }
        for (int k = 0; k < 32; ++k) misc[k] = 0;
        fence_barrier_init();
    }
    if (role == 0 && lane == 0 && pipe == 0) {
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
    }
    grid_dependency_wait();              // inputs written by the previous kernel are visible
    prefix_sums<NTHREADS>(p, lens_s, pre, wsum, tid);
    const int U = pre[p.S] * p.Hkv;

    if (role == 0) {
        const size_t qrow = (size_t)p.Hq * D * E;
        PipeRings rg{stages, full, empty, ufull, uempty, stage_ok, nst, NUR};
        producer_loop<T, D>(&kmap, &vmap, p, rg, pre, lens_s, U, abort_flag, lane, desc_at,
                            [&](int slot, int s, int j, uint64_t* bar) {
                                mbar_arrive_expect_tx(bar, G * D * E);
                                bulk_g2s(q_at(slot),
                                         reinterpret_cast<const uint8_t*>(p.q) + (size_t)s * qrow +
                                             (size_t)j * G * D * E,
                                         G * D * E, bar);
                            });
    } else {
        // ================================================= consumer warps
        const int cw = role - 1;                 // 0 .. NCONS-1
        const int ctid = cw * 32 + lane;         // 0 .. CT-1
        const int bar_id = 1 + pipe;             // named barrier of this pipeline
        Engine eng;
        float* xs = scratch + cw * 3 * G * TOK;
        uint64_t* ps = reinterpret_cast<uint64_t*>(xs + G * TOK);
        uint4* qf4 = reinterpret_cast<uint4*>(scratch + NCONS * 3 * G * TOK);   // fp32 q
        int ucount = 0;
        while (true) {
            const int slot = ucount % NUR;
            // all consumer warps give up together, so none is left at a named barrier
            const bool okw = wait_or_abort(ufull + slot, (ucount / NUR) & 1, abort_flag, p.err);
            if (named_bar_or(bar_id, CT, !okw)) break;
            const UnitDesc d = *desc_at(slot);
            if (d.end) break;
            Engine::stage_q(q_at(slot), qf4, ctid, CT, p.scale_log2e);
            named_bar_sync(bar_id, CT);                 // q in fp32 for every consumer warp
            eng.begin_unit(qf4);
            int st = (d.stage_base + cw) % nst;
            uint32_t ph = ((d.stage_base + cw) / nst) & 1;
            for (int c = cw; c < d.n_stages; c += NCONS) {
                // A slot's successive rounds may go to different consumer
                // warps, and a parity wait cannot tell round R from round
                // R - 2.  So first wait for the slot's tag to name this very
                // stage: the producer writes it only after round R - 1 was
                // consumed, and from then on the parity is unambiguous.
                int tag = -1;
                bool okt = true;
                if (lane == 0) okt = wait_tag(stage_ok + st, d.stage_base + c, &tag, abort_flag, p.err);
                okt = __shfl_sync(0xffffffffu, okt, 0);
                tag = __shfl_sync(0xffffffffu, tag, 0);
                const bool have =
                    __all_sync(0xffffffffu, okt && wait_or_abort(full + st, ph, abort_flag, p.err));
                if (have && (tag & 1)) {
                    const int nv = min(TOK, d.t1 - (d.t0 + c * TOK));
                    uint8_t* Ks = stages + (size_t)st * LY::STAGE_BYTES;
                    eng.stage(Ks, Ks + LY::KV_BYTES, nv, xs, ps, lane);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty + st);
                st += NCONS;
                while (st >= nst) { st -= nst; ph ^= 1u; }
            }
            // ---- merge the consumer warps' states of this unit
            eng.dump(mbuf + (size_t)cw * G * (D + 2), lane);   // m=-inf, l=0, o=0 if no stage
            named_bar_sync(bar_id, CT);
            if (ctid == 0) mbar_arrive(uempty + slot);          // q and the descriptor are consumed
            const size_t sj = (size_t)d.s * p.Hkv + d.j;
            for (int idx = ctid; idx < G * D; idx += CT) {
                const int g = idx / D, dd = idx % D;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < NCONS; ++w) M = fmaxf(M, mbuf[(w * G + g) * (D + 2)]);
                float Lsum = 0.f, O = 0.f;
                if (M != -INFINITY) {
#pragma unroll
                    for (int w = 0; w < NCONS; ++w) {
                        const float* e = mbuf + (w * G + g) * (D + 2);
                        const float f = exp2f(e[0] - M);
                        Lsum += e[1] * f;
                        O += e[2 + dd] * f;
                    }
                }
                if (d.n_p == 1) {
                    T* outp = reinterpret_cast<T*>(p.out) + ((size_t)d.s * p.Hq + (size_t)d.j * G + g) * D + dd;
                    *outp = DT<T>::from_float(Lsum > 0.f ? O / Lsum : 0.f);
                } else {
                    const size_t pi = (sj * p.n_pmax + d.i) * G + g;
                    p.part_o[pi * D + dd] = O;
                    if (dd == 0) {
                        p.part_ml[pi * 2 + 0] = M;
                        p.part_ml[pi * 2 + 1] = Lsum;
                    }
                }
            }
            named_bar_sync(bar_id, CT);                          // merge buffer free again
            ++ucount;
        }
        __syncwarp();
    }

    __syncthreads();
    launch_dependents();                 // the merge kernel may be scheduled
    if (tid == 0) {
        __threadfence();
        const int done = atomicAdd(&p.hdr->done_ctas, 1);
        if (done == (int)gridDim.x - 1) {
            p.hdr->next_unit = 0;
            p.hdr->done_ctas = 0;
            __threadfence();
        }
    }
}

// ------------------------------------------------------------ tensor-core (tcgen05) kernel
// A tcgen05 MMA instruction costs tens of cycles to issue whatever its size,
// so the engine is shaped to cover many tokens per instruction and to keep
// tensor memory small:
//   S^T = K Q^T   M = 64 tokens (one stage), N = 16 (query heads, G used),
//                 K = head_dim: head_dim/16 MMAs per stage
//   O^T += V^T P^T  M = head_dim, N = 16, K = 16 tokens per MMA: 4 MMAs per
//                 full stage.  O^T takes 16 columns of tensor memory.
// A CTA needs little more than 100 KB of shared memory, so two run on each
// SM: twice the stages in flight, two TMA producers and two MMA issuers, which
// is what keeps HBM busy (a ring slot stays held for the copy's latency plus
// the S -> softmax -> PV chain).
// Warps: 0-3 softmax (thread = one token of the stage: with M = 64, rows
// 16w..16w+15 sit in lanes 0-15 of warp w's lane quarter), 4-7 epilogue
// (thread = head_dim row of O^T), 8 producer, 9 MMA issuer (one thread).  Tensor memory: two S^T buffers and two O^T buffers (alternating
// per unit, so a unit's epilogue overlaps the next unit).  The softmax keeps a
// per-head reference max m that lags the true running max by at most 2^8
// (exp2 units): only when a stage exceeds it is m moved (a barrier-OR vote
// over the 128 threads), O^T rescaled in tensor memory and l rescaled.

constexpr int TTOK = 64;            // tokens per stage (a multiple of 16, at most SM_M)
constexpr int SM_M = 64;            // M of the S^T MMA (rows past TTOK are masked)
constexpr int NHP = 16;             // query heads padded to the MMA's N
constexpr float kRescaleLog2 = 8.f;
constexpr int TC_THREADS = 320;
constexpr int kTailBuckets = 16;                              // last-partition size classes
constexpr int kSchedScratch = (TC_THREADS / 32 + 1) * kTailBuckets;   // ints
constexpr int BAR_SOFTMAX = 1, BAR_EPI = 2;   // named barriers (128 threads each)

template <typename T, int D, int G>
struct TcLayout {
    static_assert(sizeof(T) == 2, "tensor-core engine takes 16-bit types");
    static_assert(G <= NHP, "query heads of a group must fit the MMA's N");
    static constexpr int E = 2;
    static constexpr int ROWB = D * E;
    static constexpr int NBOX = ROWB / 128;            // 128-byte column boxes per token row
    static constexpr int BOXT = TTOK * 128;            // one column box of a stage: 8 KB
    static constexpr int KV_BYTES = NBOX * BOXT;
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;
    static constexpr int NU = 3;                       // unit slots (descriptor + Q tile)
    static constexpr int NQ = G <= 8 ? 8 : 16;         // N of the S^T MMA (query rows read)
    static constexpr int QT = NBOX * (NQ / 8) * 1024;  // Q tile: NQ rows x head_dim, 128B swizzle
    static constexpr int PTB = TTOK * NHP * 2;         // one P^T tile (2 KB)
    static constexpr uint32_t TM_COLS = 64;            // S^T x2 then O^T x2, 16 columns each
    static constexpr int NBAR = 2 * NU + 13;           // + 2 per stage slot
    // epilogue slot: ints s, j, i, n_p, n_stages, O buffer, 2 pad; m[16]; l[4][16]
    static constexpr int ES = 32 + NHP * 4 + 4 * NHP * 4;
    static_assert(4 * kSchedScratch <= 2 * ES, "schedule scratch fits the epilogue slots");
    int nst, S;
    __host__ __device__ TcLayout(int nst_, int S_) : nst(nst_), S(S_) {}
    __host__ __device__ size_t q(int k) const { return (size_t)k * QT; }
    __host__ __device__ size_t pt(int b) const { return (size_t)NU * QT + (size_t)b * PTB; }
    __host__ __device__ size_t ring(int st) const {
        return (size_t)NU * QT + 2 * (size_t)PTB + (size_t)st * STAGE_BYTES;
    }
    __host__ __device__ size_t desc(int k) const { return ring(nst) + (size_t)k * sizeof(UnitDesc); }
    __host__ __device__ size_t bars() const { return desc(NU); }
    __host__ __device__ size_t stage_ok() const { return bars() + (size_t)(2 * nst + NBAR) * 8; }
    __host__ __device__ size_t red() const { return ((stage_ok() + (size_t)nst * 4 + 15) / 16) * 16; }
    __host__ __device__ size_t epi(int e) const { return red() + 4 * NHP * 4 + (size_t)e * ES; }
    __host__ __device__ size_t misc() const { return epi(2); }                  // 64 ints
    // the schedule's scan scratch is used only before the first unit, so it
    // shares the epilogue slots
    __host__ __device__ size_t sched() const { return epi(0); }
    __host__ __device__ size_t lens() const { return misc() + 256; }
    __host__ __device__ size_t pref() const { return lens() + 4 * (size_t)S; }
    __host__ __device__ size_t order() const { return pref() + 4 * (size_t)(S + 1); }
    __host__ __device__ size_t total() const { return order() + 4 * (size_t)S; }
};

// Unit order of the tensor-core kernel, largest first (a longest-processing-
// time order shortens the tail of the dynamic schedule): every full partition
// (P tokens) of every sequence, then each sequence's last partition by its
// stage count, most first (a stable counting sort over kTailBuckets classes;
// zero-length sequences last).  All threads of the CTA; fills lens_s[S],
// preF[S + 1] (exclusive prefix sums of the full partitions per sequence) and
// order[S]; ends with __syncthreads.  Units: (preF[S] + S) * Hkv.
template <int NTHREADS>
__device__ void schedule_units(const DecodeParams& p, int* lens_s, int* preF, int* order, int* scr,
                               int* wsum, int tid) {
    constexpr int NW = NTHREADS / 32, NB = kTailBuckets;
    static_assert((NW + 1) * NB <= kSchedScratch, "schedule scratch");
    const int warp = tid >> 5, lane = tid & 31;
    const int per = (p.S + NTHREADS - 1) / NTHREADS;
    const int beg = min(p.S, tid * per), end = min(p.S, beg + per);
    auto bucket = [&](int L) {          // 0 = the largest last partitions
        const int n_p = n_parts(L, p.P);
        const int ts = (L - (n_p - 1) * p.P + TTOK - 1) / TTOK;
        return NB - 1 - min(NB - 1, ts);
    };
    int full = 0, cnt[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) cnt[b] = 0;
    for (int k = beg; k < end; ++k) {
        const int L = clamp_len(__ldg(p.lens + k), p);
        lens_s[k] = L;
        full += n_parts(L, p.P) - 1;
        const int b = bucket(L);
#pragma unroll
        for (int q = 0; q < NB; ++q) cnt[q] += (q == b);
    }
    // block-wide exclusive scans: of `full` (-> preF) and of each bucket count
    auto warp_incl = [&](int v) {
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += u;
        }
        return v;
    };
    const int full_incl = warp_incl(full);
    int cnt_excl[NB];                   // within the warp
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const int inc = warp_incl(cnt[b]);
        cnt_excl[b] = inc - cnt[b];
        if (lane == 31) scr[warp * NB + b] = inc;
    }
    if (lane == 31) wsum[warp] = full_incl;
    __syncthreads();
    if (warp == 0) {
        const int v = (lane < NW) ? wsum[lane] : 0;
        const int iv = warp_incl(v);
        if (lane < NW) wsum[lane] = iv - v;          // exclusive warp offsets of `full`
        int run = 0;                                  // bucket `lane`: offsets over warps
        if (lane < NB) {
            for (int w = 0; w < NW; ++w) {
                const int c = scr[w * NB + lane];
                scr[w * NB + lane] = run;
                run += c;
            }
        }
        const int tot_excl = warp_incl(run) - run;    // the whole warp scans (run = 0 past NB)
        if (lane < NB) scr[NW * NB + lane] = tot_excl;    // where bucket `lane` starts in order[]
    }
    __syncthreads();
    int runF = wsum[warp] + full_incl - full;
    int pos[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) pos[b] = scr[NW * NB + b] + scr[warp * NB + b] + cnt_excl[b];
    for (int k = beg; k < end; ++k) {
        preF[k] = runF;
        runF += n_parts(lens_s[k], p.P) - 1;
        const int b = bucket(lens_s[k]);
        int at = 0;
#pragma unroll
        for (int q = 0; q < NB; ++q)
            if (q == b) at = pos[q]++;
        order[at] = k;
    }
    if (tid == NTHREADS - 1) preF[p.S] = runF;
    __syncthreads();
}

// Producer of the tensor-core engine: a 128-token stage is built from pieces of
// 16 token rows (8 when bs = 8), each inside one block; one TMA box per
// (piece, K or V, 128-byte column), at most two per lane.  stage_ok[slot] gets
// the mask of pieces that were loaded; pieces past the unit's end are not.
template <typename T, int D, int G>
__device__ void producer_tc(const CUtensorMap* kmap, const CUtensorMap* vmap,
                            const CUtensorMap* qmap, const DecodeParams& p, uint8_t* smem,
                            const TcLayout<T, D, G>& ly, uint64_t* full, uint64_t* empty,
                            uint64_t* ufull, uint64_t* uempty, int* stage_ok, const int* preF,
                            const int* order, const int* lens_s, int U, volatile int* abort_flag,
                            int lane) {
    using LY = TcLayout<T, D, G>;
    constexpr int NU = LY::NU;
    constexpr int BOX_ELEMS = 64;
    constexpr uint32_t FULL = 0xffffffffu;
    const int nst = ly.nst;
    const uint64_t policy = policy_evict_first();
    const int bs = p.bs, bsl = p.bs_log2;
    const int PR = bs >= 16 ? 16 : bs;                // rows per piece
    const int NPC = TTOK / PR;                         // pieces per stage
    const int nops = NPC * 2 * LY::NBOX;               // <= 64
    constexpr int NV = LY::ROWB / 16;                  // 16-byte pieces of a K or V row
    static_assert(2 * NV <= 32, "one piece of the new token's K and V rows per lane");
    struct Plan {
        int u, s, j, i, t0, t1, nst, n_p, nblk;
        const int32_t* trow;
        int ids_a, ids_b;
        bool wr;           // the step's new token falls in this unit (its last partition)
        bool wld;          // ... and its slot, block and row pieces are loaded
        int wbl;           // block of position L - 1 through the table
        long long wsl;     // slot_mapping entry of the sequence
        uint4 wpc;         // this lane's piece: K row (lanes < NV), V row (NV <= lanes < 2 NV)
    };
    // The new token's slot, block and row pieces, loaded into registers a unit
    // ahead (only after the dependency wait: the inputs may come from the
    // kernel before this one).
    auto load_write = [&](Plan& q) {
        const int pos = q.t1 - 1;
        q.wsl = __ldg(p.wslot + q.s);
        q.wbl = __ldg(q.trow + ((pos >> bsl) - (q.t0 >> bsl)));
        if (lane < 2 * NV)
            q.wpc = __ldg((lane < NV ? p.wk : p.wv) + ((size_t)q.s * p.Hkv + q.j) * NV + lane % NV);
        q.wld = true;
    };
    auto prepare = [&](int u, bool dep_done) {
        Plan q{};
        q.u = u;
        if (u >= U) return q;
        // unit u -> (sequence, partition): full partitions first, in sequence
        // order, then the last partitions in the largest-first order
        const int x = u / p.Hkv, F = preF[p.S];
        if (x < F) {
            int lo = 0, hi = p.S;                      // last lo with preF[lo] <= x
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (preF[mid] <= x) lo = mid; else hi = mid;
            }
            q.s = lo;
            q.i = x - preF[lo];
        } else {
            q.s = order[x - F];
            q.i = n_parts(lens_s[q.s], p.P) - 1;
        }
        q.j = u - x * p.Hkv;
        const int L = lens_s[q.s];
        q.t0 = min(q.i * p.P, L);
        q.t1 = min(q.t0 + p.P, L);
        q.nst = (q.t1 - q.t0 + TTOK - 1) / TTOK;
        q.n_p = n_parts(L, p.P);
        const int b0 = q.t0 >> bsl;
        q.nblk = ((q.t1 + bs - 1) >> bsl) - b0;
        q.trow = p.tables + (size_t)q.s * p.mbps + b0;
        q.ids_a = (lane < q.nblk) ? __ldg(q.trow + lane) : -1;
        q.ids_b = (lane + 32 < q.nblk) ? __ldg(q.trow + 32 + lane) : -1;
        q.wr = p.wslot != nullptr && q.i == q.n_p - 1 && q.nst > 0;
        if (q.wr && dep_done) load_write(q);
        return q;
    };
    // Latency hiding at unit boundaries: lane 0 holds the tickets of the two
    // units after the current one (each fetched two units ahead), and the next
    // unit's plan, whose block-table loads are then in flight, is prepared as
    // soon as the current unit's first stage is issued.  A CTA's first unit is
    // its own index (the largest units, one per CTA), planned - block-table
    // reads included - before the dependency wait; later units come from the
    // ticket counter, which hands out gridDim.x onwards.
    int gstage = 0, st = 0, round = 0, ucount = 0, t1 = 0, t2 = 0;
    Plan cur = prepare((int)blockIdx.x, false);
    // The kernel before this one has completed and its writes are visible:
    // the cache may be read, and the scheduler ticket is free (a decode call
    // just before on the same workspace has reset it).
    grid_dependency_wait();
    if (lane == 0) {
        t1 = (int)gridDim.x + atomicAdd(&p.hdr->next_unit, 1);
        t2 = (int)gridDim.x + atomicAdd(&p.hdr->next_unit, 1);
    }
    if (p.wslot != nullptr) {
        // a sequence with no tokens has no position for a new one (its slot
        // is read only now: the inputs may come from the kernel before)
        for (int k = (int)blockIdx.x * 32 + lane; k < p.S; k += (int)gridDim.x * 32)
            if (lens_s[k] == 0 && __ldg(p.wslot + k) >= 0) set_err(p.err, PA_DEV_BAD_SLOT);
    }
    bool ok = true;
    while (ok) {
        const int slot = ucount % NU;
        if (ucount >= NU) {
            bool w = true;
            if (lane == 0) w = wait_or_abort(uempty + slot, ((ucount / NU) - 1) & 1, abort_flag, p.err);
            if (!__shfl_sync(FULL, w, 0)) { ok = false; break; }
        }
        UnitDesc* d = reinterpret_cast<UnitDesc*>(smem + ly.desc(slot));
        if (cur.u >= U) {
            if (lane == 0) {
                d->end = 1;
                mbar_arrive(ufull + slot);
            }
            ++ucount;
            break;
        }
        if (lane == 0) {
            d->s = cur.s; d->j = cur.j; d->i = cur.i; d->t0 = cur.t0; d->t1 = cur.t1;
            d->n_p = cur.n_p;
            d->stage_base = gstage; d->n_stages = cur.nst; d->end = 0;
            mbar_arrive_expect_tx(ufull + slot, G * D * 2);
            uint8_t* qt = smem + ly.q(slot);
#pragma unroll
            for (int kc = 0; kc < LY::NBOX; ++kc)
                tma_load_2d(qt + kc * (LY::QT / LY::NBOX), qmap, kc * BOX_ELEMS, cur.s * p.Hq + cur.j * G,
                            ufull + slot, policy);
        }
        ++ucount;
        Plan nxt{};
        bool have_next = false;
        auto next_plan = [&]() {            // after the unit's first stage is issued
            nxt = prepare(__shfl_sync(FULL, t1, 0), true);
            have_next = true;
            if (lane == 0) {
                t1 = t2;
                t2 = (int)gridDim.x + atomicAdd(&p.hdr->next_unit, 1);
            }
        };
        if (cur.wr) {
            // The step's new token (position L - 1, in this unit's last
            // stage) goes into the cache now, with the values loaded a unit
            // ahead; the fence before the last stage's copies orders the
            // stores before them.  Only this unit reads that row: partitions
            // start at multiples of 16 tokens and pieces are at most 16 rows.
            if (!cur.wld) load_write(cur);        // a CTA's first unit
            const int pos = cur.t1 - 1;
            if (new_token_slot_ok(p, cur.wsl, pos, cur.wbl, lane == 0) && lane < 2 * NV)
                (lane < NV ? p.kc : p.vc)[(((size_t)cur.wbl * p.Hkv + cur.j) * bs + (pos & (bs - 1))) * NV +
                                          lane % NV] = cur.wpc;
        }
        int win = 0;
        const int b0 = cur.t0 >> bsl;
        for (int c = 0; c < cur.nst; ++c) {
            const int tok0 = cur.t0 + c * TTOK;
            while ((tok0 >> bsl) - b0 - win >= 32) {      // keep the stage's blocks in the window
                win += 32;
                cur.ids_a = cur.ids_b;
                cur.ids_b = (lane + win + 32 < cur.nblk) ? __ldg(cur.trow + win + 32 + lane) : -1;
            }
            if (cur.wr && c == cur.nst - 1) {
                fence_proxy_async_global();               // the new token's stores before
                __syncwarp();                             // this stage's copies
                fence_proxy_async_global();
            }
            if (round > 0) {
                bool w = true;
                if (lane == 0) w = wait_or_abort(empty + st, (round - 1) & 1, abort_flag, p.err);
                if (!__shfl_sync(FULL, w, 0)) { ok = false; break; }
            }
            int blk[2], tok[2];
            bool live[2];
            uint32_t want = 0, got = 0;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int op = lane + 32 * r;
                const int piece = op / (2 * LY::NBOX);
                tok[r] = tok0 + piece * PR;
                const bool exists = op < nops && tok[r] < cur.t1;
                const int rel = exists ? (tok[r] >> bsl) - b0 - win : 0;   // 0 <= rel < 64
                const int ia = __shfl_sync(FULL, cur.ids_a, rel & 31);
                const int ib = __shfl_sync(FULL, cur.ids_b, rel & 31);
                blk[r] = rel < 32 ? ia : ib;
                live[r] = exists && blk[r] >= 0 && blk[r] < p.NB;
                if (exists) want |= 1u << piece;
                if (live[r]) got |= 1u << piece;
            }
            want = __reduce_or_sync(FULL, want);
            got = __reduce_or_sync(FULL, got);
            uint8_t* stage = smem + ly.ring(st);
            if (cur.u == 0 && c == p.hold_stage) {
                // test hook: nothing will ever arrive on this stage's barrier
                ++gstage;
                if (++st == nst) { st = 0; ++round; }
                if (!have_next) next_plan();
                continue;
            }
            if (lane == 0) {
                stage_ok[st] = (int)got;
                if (want & ~got) set_err(p.err, PA_DEV_BAD_BLOCK);
                if (got)
                    mbar_arrive_expect_tx(full + st, (uint32_t)__popc(got) * 2u * PR * LY::ROWB);
                else
                    mbar_arrive(full + st);
            }
            __syncwarp();
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int op = lane + 32 * r;
                if (live[r]) {
                    const int piece = op / (2 * LY::NBOX), rem = op % (2 * LY::NBOX);
                    const int kv = rem / LY::NBOX, b = rem % LY::NBOX;
                    const int y = ((blk[r] * p.Hkv + cur.j) << bsl) + (tok[r] & (bs - 1));
                    uint8_t* dst = stage + kv * LY::KV_BYTES + b * LY::BOXT + piece * PR * 128;
                    tma_load_2d(dst, kv ? vmap : kmap, b * BOX_ELEMS, y, full + st, policy);
                }
            }
            ++gstage;
            if (++st == nst) { st = 0; ++round; }
            if (!have_next) next_plan();
        }
        if (!ok) break;
        if (!have_next) next_plan();
        cur = nxt;
    }
    if (lane == 0) {
        const int first = max(0, gstage - nst);
        for (int g = first; g < gstage; ++g) mbar_wait(full + g % nst, (g / nst) & 1);
        const int ufirst = max(0, ucount - NU);
        for (int k = ufirst; k < ucount; ++k) mbar_wait(ufull + k % NU, (k / NU) & 1);
    }
    __syncwarp();
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(TC_THREADS, 2)
decode_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                 const __grid_constant__ CUtensorMap qmap, DecodeParams p) {
    using LY = TcLayout<T, D, G>;
    constexpr int NU = LY::NU;
    constexpr uint32_t FULL = 0xffffffffu;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const LY ly(p.nst, p.S);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nst = p.nst;

    uint64_t* full = reinterpret_cast<uint64_t*>(smem + ly.bars());
    uint64_t* empty = full + nst;
    uint64_t* ufull = empty + nst;
    uint64_t* uempty = ufull + NU;        // 5 arrivals: MMA issuer + the 4 softmax warps
    uint64_t* s_full = uempty + NU;       // [2] S^T_g complete
    uint64_t* p_full = s_full + 2;        // [2] P^T_g written (4 softmax warps)
    uint64_t* o_done = p_full + 2;        // [2] last PV of a unit complete (per O buffer)
    uint64_t* o_free = o_done + 2;        // [2] O buffer read by the epilogue (4 warps)
    uint64_t* epi_full = o_free + 2;      // [2] epilogue slot filled (4 softmax warps)
    uint64_t* epi_empty = epi_full + 2;   // [2] epilogue slot read (4 epilogue warps)
    uint64_t* fin = epi_empty + 2;        // issuer's final drain
    int* stage_ok = reinterpret_cast<int*>(smem + ly.stage_ok());
    float* red = reinterpret_cast<float*>(smem + ly.red());      // [4][16]
    int* misc = reinterpret_cast<int*>(smem + ly.misc());
    int* lens_s = reinterpret_cast<int*>(smem + ly.lens());
    int* preF = reinterpret_cast<int*>(smem + ly.pref());
    int* order = reinterpret_cast<int*>(smem + ly.order());
    volatile int* abort_flag = misc + 0;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 60);   // outside the zeroed words
    int* wsum = misc + 32;
    volatile int* last_flag = misc + 48;     // epilogue: this unit completes its split

    if (tid == 0) {
        const int n = 2 * nst + LY::NBAR;
        for (int k = 0; k < n; ++k) mbar_init(full + k, 1);
        for (int k = 0; k < NU; ++k) mbar_init(uempty + k, 5);
        for (int k = 0; k < 2; ++k) {
            mbar_init(p_full + k, 4);
            mbar_init(o_free + k, 4);
            mbar_init(epi_full + k, 4);
            mbar_init(epi_empty + k, 4);
        }
        for (int k = 0; k < 32; ++k) misc[k] = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tc::alloc(tmem_slot, LY::TM_COLS);
        tc::relinquish();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
        prefetch_tensormap(&qmap);
    }
    // Without a merge launch after this kernel, the kernel after it in the
    // stream (e.g. the next step's decode) may be scheduled from now on: its
    // CTAs take the SM slots this grid's CTAs free in its tail and do their
    // own set-up there; they read nothing this kernel writes before their
    // griddepcontrol.wait.  (A merge kernel scheduled this early slowed the
    // split batches: it is released at the end instead.)
    const bool merge_follows = p.n_pmax > 1 && !p.fused_merge;
    if (!merge_follows) launch_dependents();
    // Launched as a programmatic dependent of the kernel before it: the
    // lengths may be read, the unit order computed and the first unit's
    // block-table entries read while that kernel still runs (no kernel of
    // this library writes lengths or tables); the scheduler ticket, the
    // queries, the new tokens, the cache and every write wait for
    // griddepcontrol.wait (in the producer before its first ticket and copy,
    // in every other warp before its loop).
    schedule_units<TC_THREADS>(p, lens_s, preF, order, reinterpret_cast<int*>(smem + ly.sched()), wsum, tid);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tO = tmem + 2 * NHP;                 // + 16 * buffer
    const uint32_t lq = (uint32_t)(32 * (warp & 3)) << 16;          // this warp's lane quarter
    const int U = (preF[p.S] + p.S) * p.Hkv;
    const int PR = p.bs >= 16 ? 16 : p.bs;

    if (warp != 8) grid_dependency_wait();
    if (warp == 8) {
        // ================================================= producer warp
        producer_tc<T, D, G>(&kmap, &vmap, &qmap, p, smem, ly, full, empty, ufull, uempty,
                             stage_ok, preF, order, lens_s, U, abort_flag, lane);
    } else if (warp == 9) {
        // ================================================= MMA issuer (one thread)
        // Event driven: the thread polls the next stage's data (-> S MMAs) and
        // the oldest pending stage's P (-> PV MMAs) and issues whichever is
        // ready, so a PV never waits for the next stage's copy.  S_g is issued
        // only once PV_{g-2} has been (its S^T and P^T buffers are reused).
        if (lane == 0) {
            constexpr uint32_t ID_S = tc::idesc_f16<T>(false, false, SM_M, LY::NQ);
            constexpr uint32_t ID_O = tc::idesc_f16<T>(true, true, D, NHP);
            struct Pending {
                int g, nv, oseq;
                bool first, last;
            };
            Pending pend0{}, pend1{};            // S issued, PV not yet (pend0 oldest)
            int npend = 0;
            int ucount = 0, ocount = 0, c = 0, oseq = 0, slot = 0;
            bool have = false, s_done = false, ok = true;
            UnitDesc d{};
            uint32_t idle = 0;
            uint64_t t_idle = 0;
            while (true) {
                bool prog = false;
                // ---- the next unit, for the S side
                if (!have && !s_done) {
                    slot = ucount % NU;
                    if (mbar_test(ufull + slot, (ucount / NU) & 1)) {
                        d = *reinterpret_cast<const UnitDesc*>(smem + ly.desc(slot));
                        prog = true;
                        if (d.end) {
                            s_done = true;
                        } else {
                            ++ucount;
                            if (d.n_stages == 0) {
                                mbar_arrive(uempty + slot);
                            } else {
                                have = true;
                                c = 0;
                                oseq = ocount++;
                            }
                        }
                    }
                }
                // ---- O^T += V^T P^T of the oldest pending stage
                if (npend > 0) {
                    const Pending r = pend0;
                    const int ob = r.oseq & 1;
                    bool ready = mbar_test(p_full + (r.g & 1), (r.g >> 1) & 1);
                    if (ready && r.first && r.oseq >= 2)   // the epilogue has read this O^T buffer
                        ready = mbar_test(o_free + ob, ((r.oseq >> 1) - 1) & 1);
                    if (ready) {
                        tc::fence_after();
                        const int st = r.g % nst;
                        const uint64_t a0 = tc::sdesc_sw128(smem_u32(smem + ly.ring(st) + LY::KV_BYTES), LY::BOXT, 1024);
                        const uint64_t b0 = tc::sdesc_none(smem_u32(smem + ly.pt(r.g & 1)), 256, 128);
                        const uint32_t od = tO + (uint32_t)(NHP * ob);
                        const int nk = (r.nv + 15) / 16;             // 16-token slices holding tokens
                        for (int kk = 0; kk < nk; ++kk)
                            tc::mma_ss(od, a0 + (uint64_t)(kk * 128), b0 + (uint64_t)(kk * 32), ID_O,
                                       (r.first && kk == 0) ? 0u : 1u);
                        tc::commit(empty + st);          // the stage slot may be refilled
                        if (r.last) tc::commit(o_done + ob);
                        pend0 = pend1;
                        --npend;
                        prog = true;
                    }
                }
                // ---- S^T of the unit's next stage
                if (have && npend < 2) {
                    const int g = d.stage_base + c, st = g % nst;
                    if (mbar_test(full + st, (g / nst) & 1)) {
                        tc::fence_after();
                        const uint64_t a0 = tc::sdesc_sw128(smem_u32(smem + ly.ring(st)), 16, 1024);
                        const uint64_t b0 = tc::sdesc_sw128(smem_u32(smem + ly.q(slot)), 16, 1024);
                        const uint32_t sd = tS + (uint32_t)(NHP * (g & 1));
#pragma unroll
                        for (int k = 0; k < D / 16; ++k)   // descriptor start fields in 16-byte units
                            tc::mma_ss(sd, a0 + (uint64_t)((k >> 2) * (LY::BOXT >> 4) + (k & 3) * 2),
                                       b0 + (uint64_t)((k >> 2) * (LY::QT / LY::NBOX >> 4) + (k & 3) * 2), ID_S,
                                       k > 0 ? 1u : 0u);
                        tc::commit(s_full + (g & 1));
                        if (c == d.n_stages - 1) tc::commit(uempty + slot);   // Q tile no longer read
                        const Pending nw{g, min(TTOK, d.t1 - (d.t0 + c * TTOK)), oseq, c == 0,
                                         c == d.n_stages - 1};
                        if (npend == 0) pend0 = nw; else pend1 = nw;
                        ++npend;
                        if (++c == d.n_stages) have = false;
                        prog = true;
                    }
                }
                if (s_done && !have && npend == 0) break;
                if (prog) {
                    idle = 0;
                } else if ((++idle & 255) == 0) {
                    // bounded: give up after kWaitLimitNs without progress, or when
                    // another warp has given up
                    if (*abort_flag) { ok = false; break; }
                    const uint64_t now = global_ns();
                    if (idle == 256) {
                        t_idle = now;
                    } else if (now - t_idle > kWaitLimitNs) {
                        set_err(p.err, PA_DEV_TIMEOUT);
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                }
            }
            (void)ok;
            // every MMA this thread issued has completed before tensor memory is freed
            tc::commit(fin);
            mbar_wait(fin, 0);
        }
        __syncwarp();
    } else if (warp < 4) {
        // ================================================= softmax warps (thread = token)
        const int t = (lane < 16 && 16 * warp + lane < TTOK) ? 16 * warp + lane : -1;   // stage token (M = 64 layout)
        const int piece = t >= 0 ? t / PR : 0;
        int ucount = 0, ocount = 0;
        while (true) {
            // Every give-up decision is taken by all four warps together (an OR
            // vote on their named barrier), so none is left waiting at a barrier.
            const int slot = ucount % NU;
            const int e = ucount & 1;
            bool okw = wait_or_abort(ufull + slot, (ucount / NU) & 1, abort_flag, p.err);
            if (ucount >= 2)
                okw = okw && wait_or_abort(epi_empty + e, ((ucount >> 1) - 1) & 1, abort_flag, p.err);
            if (named_bar_or(BAR_SOFTMAX, 128, !okw)) break;
            const UnitDesc d = *reinterpret_cast<const UnitDesc*>(smem + ly.desc(slot));
            uint8_t* es = smem + ly.epi(e);
            int* hdr = reinterpret_cast<int*>(es);
            float* em = reinterpret_cast<float*>(es + 32);
            float* el = em + NHP;
            if (d.end) {
                if (t == 0) hdr[3] = -1;                  // tells the epilogue warps to stop
                __syncwarp();
                if (lane == 0) mbar_arrive(epi_full + e);
                break;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(uempty + slot);
            const int ob = ocount & 1;
            float m_ref[G], l_part[G];
#pragma unroll
            for (int h = 0; h < G; ++h) { m_ref[h] = -INFINITY; l_part[h] = 0.f; }
            bool ok = true;
            for (int c = 0; c < d.n_stages; ++c) {
                const int g = d.stage_base + c, st = g % nst, b = g & 1;
                const bool okw = __all_sync(FULL, wait_or_abort(s_full + b, (g >> 1) & 1, abort_flag, p.err) &&
                                                      wait_or_abort(full + st, (g / nst) & 1, abort_flag, p.err));
                uint32_t sr[NHP];
                if (okw) {
                    tc::fence_after();
                    tc::ld16(tS + (uint32_t)(NHP * b) + lq, sr);
                }
                const bool valid = okw && t >= 0 && d.t0 + c * TTOK + t < d.t1 && ((stage_ok[st] >> piece) & 1);
                float x[G];
                bool over = false;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    x[h] = valid ? __uint_as_float(sr[h]) * p.scale_log2e : -INFINITY;
                    over |= x[h] > m_ref[h] + kRescaleLog2;
                }
                // one vote: some head outgrew its reference max, or a wait gave up
                if (named_bar_or(BAR_SOFTMAX, 128, over || !okw)) {
                    if (named_bar_or(BAR_SOFTMAX, 128, !okw)) {
                        ok = false;
                        break;
                    }
                    // move the reference max of the heads that outgrew it
                    float mx[G];
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        mx[h] = x[h];
#pragma unroll
                        for (int off = 16; off >= 1; off >>= 1)
                            mx[h] = fmaxf(mx[h], __shfl_xor_sync(FULL, mx[h], off));
                    }
                    if (lane == 0)
#pragma unroll
                        for (int h = 0; h < G; ++h) red[warp * NHP + h] = mx[h];
                    named_bar_sync(BAR_SOFTMAX, 128);
                    float alpha[G];
                    bool moved = false;
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float M = fmaxf(fmaxf(red[h], red[NHP + h]), fmaxf(red[2 * NHP + h], red[3 * NHP + h]));
                        alpha[h] = 1.f;
                        if (M > m_ref[h] + kRescaleLog2) {
                            alpha[h] = exp2f(m_ref[h] - M);   // 0 while m was -inf
                            m_ref[h] = M;
                            l_part[h] *= alpha[h];
                            moved = true;
                        }
                    }
                    named_bar_sync(BAR_SOFTMAX, 128);      // red[] free again
                    if (c > 0 && moved) {
                        // O^T has stage g-1's PV in it (its completion is what
                        // frees stage g-1's ring slot) and not yet stage g's
                        const int sp = (g - 1) % nst;
                        const bool okw = wait_or_abort(empty + sp, ((g - 1) / nst) & 1, abort_flag, p.err);
                        if (named_bar_or(BAR_SOFTMAX, 128, !okw)) {
                            ok = false;
                            break;
                        }
                        tc::fence_after();
                        uint32_t o[NHP];
                        tc::ld16(tO + (uint32_t)(NHP * ob) + lq, o);
#pragma unroll
                        for (int h = 0; h < G; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
                        tc::st16(tO + (uint32_t)(NHP * ob) + lq, o);
                    }
                }
                // P^T row t (16 heads, 16-bit), l sums the rounded weights the MMA uses
                uint32_t pk[NHP / 2];
#pragma unroll
                for (int k = 0; k < NHP / 2; ++k) {
                    float p0 = 0.f, p1 = 0.f;
                    if (2 * k < G && valid) p0 = exp2f(x[2 * k] - m_ref[2 * k]);
                    if (2 * k + 1 < G && valid) p1 = exp2f(x[2 * k + 1] - m_ref[2 * k + 1]);
                    pk[k] = pack2<T>(p0, p1);
                    if (2 * k < G) {
                        float r2[2];
                        Unpack<T>::run(pk[k], r2);
                        l_part[2 * k] += r2[0];
                        if (2 * k + 1 < G) l_part[2 * k + 1] += r2[1];
                    }
                }
                if (t >= 0) {
                    uint8_t* ptile = smem + ly.pt(b) + (t >> 3) * 256 + (t & 7) * 16;
                    *reinterpret_cast<uint4*>(ptile) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    *reinterpret_cast<uint4*>(ptile + 128) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
                if (t >= 0 && !valid) {
                    // this token's V row must be finite (p = 0 meets it)
                    uint8_t* vrow = smem + ly.ring(st) + LY::KV_BYTES + t * 128;
#pragma unroll
                    for (int ch = 0; ch < LY::ROWB / 16; ++ch)
                        *reinterpret_cast<uint4*>(vrow + (ch >> 3) * LY::BOXT + (((ch & 7) ^ (t & 7)) << 4)) =
                            make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
                tc::fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full + b);
            }
            if (!ok) break;
            // ---- hand (m, l partial sums, unit) to the epilogue warps
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float v = l_part[h];
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(FULL, v, off);
                if (lane == 0) el[warp * NHP + h] = v;
            }
            if (t == 0) {
                hdr[0] = d.s; hdr[1] = d.j; hdr[2] = d.i; hdr[3] = d.n_p;
                hdr[4] = d.n_stages; hdr[5] = ob;
#pragma unroll
                for (int h = 0; h < G; ++h) em[h] = m_ref[h];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(epi_full + e);
            if (d.n_stages > 0) ++ocount;
            ++ucount;
        }
        __syncwarp();
    } else {
        // ================================================= epilogue warps (thread = O^T row)
        const int et = tid - 128;
        // O^T row of this thread: M = 128 puts row r in lane r; M = 64 puts rows
        // 16q..16q+15 in lanes 32q..32q+15
        const int dd = (D == 128) ? et : ((lane < 16) ? 16 * (warp & 3) + lane : -1);
        int ucount = 0, ocount = 0;
        while (true) {
            const int e = ucount & 1;
            const bool okw = wait_or_abort(epi_full + e, (ucount >> 1) & 1, abort_flag, p.err);
            if (named_bar_or(BAR_EPI, 128, !okw)) break;
            const uint8_t* es = smem + ly.epi(e);
            const int* hdr = reinterpret_cast<const int*>(es);
            const int s = hdr[0], j = hdr[1], i = hdr[2], n_p = hdr[3], nstg = hdr[4], ob = hdr[5];
            if (n_p < 0) break;
            const float* em = reinterpret_cast<const float*>(es + 32);
            const float* el = em + NHP;
            float mh[G], lh[G], o[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                mh[h] = em[h];
                lh[h] = (el[h] + el[NHP + h]) + (el[2 * NHP + h] + el[3 * NHP + h]);
                o[h] = 0.f;
            }
            bool ok = true;
            if (nstg > 0) {
                const bool okd = wait_or_abort(o_done + ob, (ocount >> 1) & 1, abort_flag, p.err);
                if (named_bar_or(BAR_EPI, 128, !okd)) {
                    ok = false;
                } else {
                    tc::fence_after();
                    uint32_t r[NHP];
                    tc::ld16(tO + (uint32_t)(NHP * ob) + lq, r);
#pragma unroll
                    for (int h = 0; h < G; ++h) o[h] = __uint_as_float(r[h]);
                    tc::fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(o_free + ob);
                }
                ++ocount;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(epi_empty + e);   // slot copied out
            if (!ok) break;
            const size_t sj = (size_t)s * p.Hkv + j;
            if (n_p == 1) {
                if (dd >= 0)
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        T* outp = reinterpret_cast<T*>(p.out) + ((size_t)s * p.Hq + (size_t)j * G + h) * D + dd;
                        *outp = DT<T>::from_float(lh[h] > 0.f ? o[h] / lh[h] : 0.f);
                    }
            } else {
                // partials: for the merge kernel, or (fused_merge) for the unit
                // that finishes this (sequence, KV head) last
                if (dd >= 0)
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const size_t pi = (sj * p.n_pmax + i) * G + h;
                        p.part_o[pi * D + dd] = o[h];
                        if (dd == 0) {
                            p.part_ml[pi * 2 + 0] = mh[h];
                            p.part_ml[pi * 2 + 1] = lh[h];
                        }
                    }
                if (p.fused_merge) {
                    // count this unit once all 128 threads' partials are
                    // written (barrier, then one release-acquire atomic); the
                    // count that completes the split makes this group the
                    // merger, and it sees every other unit's partials
                    named_bar_sync(BAR_EPI, 128);
                    if (et == 0) *last_flag = atomic_add_acq_rel(p.split_cnt + sj, 1) == n_p - 1;
                    named_bar_sync(BAR_EPI, 128);
                    if (*last_flag) {
                        if (dd >= 0) merge_column<T, D, G>(p, s, j, dd, n_p);
                        if (et == 0) p.split_cnt[sj] = 0;   // the next call starts at zero
                    }
                }
            }
            ++ucount;
        }
        __syncwarp();
    }

    tc::fence_before();
    __syncthreads();
    if (merge_follows) launch_dependents();   // the merge kernel may be scheduled
    if (warp == 0) {
        tc::fence_after();
        tc::dealloc(tmem, LY::TM_COLS);
    }
    if (tid == 0) {
        if (*abort_flag) atomicExch(&p.hdr->dirty, 1);   // split counters may be left partial
        __threadfence();
        const int done = atomicAdd(&p.hdr->done_ctas, 1);
        if (done == (int)gridDim.x - 1) {
            if (atomicAdd(&p.hdr->dirty, 0)) {
                // only the in-kernel merge counts splits; either way the
                // header goes back to zero
                if (p.fused_merge)
                    for (int k = 0; k < p.S * p.Hkv; ++k) p.split_cnt[k] = 0;
                p.hdr->dirty = 0;
            }
            p.hdr->next_unit = 0;
            p.hdr->done_ctas = 0;
            __threadfence();
        }
    }
}

// ------------------------------------------------------------ host side
namespace {

std::mutex g_mu;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// Tensor map over a matrix of `rows` rows of D elements (a cache viewed as
// [num_blocks*Hkv*bs][D], or the queries as [S*Hq][D]); box = 128 bytes x
// box_rows, 128B swizzle.
int make_map(CUtensorMap* map, const void* base, pa_dtype dt, int D, int64_t rows, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return PA_ERR_CUDA;
    const int esz = (int)dtype_size(dt);
    CUtensorMapDataType t = dt == PA_F32   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                            : dt == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                           : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * esz};
    cuuint32_t box[2] = {(cuuint32_t)(128 / esz), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, t, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

// Tensor maps of recent calls, per host thread.  A map holds nothing but the
// base address, the element type and the shape, so an entry with the same key
// is the same map, whatever memory now sits at that address; the cache only
// saves the encoding on the host (a decode step needs three maps).
struct MapCache {
    struct Entry {
        const void* base = nullptr;
        int dt = -1, D = 0, box_rows = 0;
        int64_t rows = 0;
        CUtensorMap map;
    };
    static constexpr int N = 8;
    Entry e[N];
    int next = 0;
    int get(CUtensorMap* out, const void* base, pa_dtype dt, int D, int64_t rows, int box_rows) {
        for (int k = 0; k < N; ++k)
            if (e[k].base == base && e[k].dt == (int)dt && e[k].D == D && e[k].rows == rows &&
                e[k].box_rows == box_rows) {
                *out = e[k].map;
                return PA_OK;
            }
        const int st = make_map(out, base, dt, D, rows, box_rows);
        if (st != PA_OK) return st;
        Entry& n = e[next];
        next = (next + 1) % N;
        n.base = base; n.dt = (int)dt; n.D = D; n.rows = rows; n.box_rows = box_rows;
        n.map = *out;
        return PA_OK;
    }
};

struct DevInfo {
    int sms = 0;
    int smem_optin = 0;     // per CTA
    int smem_sm = 0;        // per SM
};

int dev_info(DevInfo* out) {
    static DevInfo cache[64];
    static bool have[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!have[dev]) {
        if (cudaDeviceGetAttribute(&cache[dev].sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&cache[dev].smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
                cudaSuccess ||
            cudaDeviceGetAttribute(&cache[dev].smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
                cudaSuccess)
            return PA_ERR_CUDA;
        have[dev] = true;
    }
    *out = cache[dev];
    return PA_OK;
}

constexpr int kMaxStages = 8;     // stages per pipeline
constexpr int kMinStages = 2;     // any count >= 1 is correct; fewer only slows the pipeline

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

// Workspace: the scheduler header; when sequences can be split, the split
// counters [S*Hkv] int, the (m, l) pairs and the unnormalised outputs of every
// partition of every query head.
size_t ws_counters(int S, int Hkv) { return round256((size_t)S * Hkv * 4); }
size_t ws_ml(int S, int Hq, int n_pmax) { return round256((size_t)S * Hq * n_pmax * 2 * 4); }
size_t ws_bytes(int S, int Hq, int Hkv, int D, int n_pmax) {
    size_t b = sizeof(WsHeader);
    if (n_pmax > 1)
        b += ws_counters(S, Hkv) + ws_ml(S, Hq, n_pmax) + (size_t)S * Hq * n_pmax * D * 4;
    return b;
}

struct Launch {
    CUtensorMap kmap, vmap, qmap;
    DecodeParams p;
    int64_t units_ub;       // upper bound on the number of work units
    dim3 grid;
    int threads;
    size_t smem;
    cudaStream_t stream;
};

// Stage count per pipeline: as many as fit in `budget` bytes of shared memory
// (at most kMaxStages).  `per_stage` is what one more stage costs in every
// pipeline (its K/V bytes, two mbarriers and a validity flag); + 1024 bytes
// of alignment slack.
template <class LY>
int pick_stages(const Launch& L, size_t budget, size_t per_stage, int* nst_out, size_t* smem_out) {
    const size_t fixed = LY(0, L.p.S).total() + 1024 + 16;
    if (budget < fixed + (size_t)kMinStages * per_stage) return PA_ERR_UNSUPPORTED;
    int nst = (int)((budget - fixed) / per_stage);
    nst = std::min(nst, kMaxStages);
    while (nst > kMinStages && LY(nst, L.p.S).total() + 1024 > budget) --nst;
    *nst_out = nst;
    *smem_out = LY(nst, L.p.S).total() + 1024;
    return *smem_out > budget ? PA_ERR_UNSUPPORTED : PA_OK;
}

// Launch as a programmatic dependent of the previous kernel in the stream:
// the decode kernel's set-up (barriers, tensor memory) overlaps that kernel's
// tail, and every thread waits (griddepcontrol.wait) before its first read of
// global memory, so whatever the previous kernel wrote is visible.
template <class Kern, class... Args>
int launch_dependent(Kern kern, dim3 grid, int threads, size_t smem, cudaStream_t stream,
                     Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <class Kern>
int set_smem_attr(Kern kern, const DevInfo& di, bool* done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    if (!done[dev & 63]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, di.smem_optin) !=
            cudaSuccess)
            return PA_ERR_CUDA;
        done[dev & 63] = true;
    }
    return PA_OK;
}

template <typename T, int D, int G>
int run_decode_core(Launch& L, const DevInfo& di) {
    using LY = Layout<T, D, G, cons_for<G>()>;
    auto kern = decode_kernel<T, D, G>;
    L.p.fused_merge = 0;     // the CUDA-core engine leaves splits to the merge kernel
    const size_t per_stage = (size_t)LY::NPIPE * (LY::STAGE_BYTES + 2 * 8 + 4);
    int st = pick_stages<LY>(L, (size_t)di.smem_optin, per_stage, &L.p.nst, &L.smem);
    if (st != PA_OK) return st;
    L.threads = LY::NTHREADS;
    static bool attr_set[64] = {};
    if ((st = set_smem_attr(kern, di, attr_set)) != PA_OK) return st;
    return launch_dependent(kern, L.grid, L.threads, L.smem, L.stream, L.kmap, L.vmap, L.p);
}

template <typename T, int D, int G>
int run_decode_tc(Launch& L, const DevInfo& di) {
    if constexpr (sizeof(T) != 2) {
        return PA_ERR_UNSUPPORTED;
    } else {
        using LY = TcLayout<T, D, G>;
        auto kern = decode_tc_kernel<T, D, G>;
        // short splits are merged by the unit that completes them
        L.p.fused_merge = (L.p.n_pmax > 1 && L.p.n_pmax <= fused_parts<G>()) ? 1 : 0;
        // two CTAs per SM: each gets half of the SM's shared memory (less the
        // 1 KB the system reserves per CTA)
        const size_t budget = std::min<size_t>((size_t)di.smem_optin, (size_t)di.smem_sm / 2 - 1024);
        const size_t per_stage = LY::STAGE_BYTES + 2 * 8 + 4;
        int st = pick_stages<LY>(L, budget, per_stage, &L.p.nst, &L.smem);
        if (st != PA_OK) return st;
        L.threads = TC_THREADS;
        static bool attr_set[64] = {};
        if ((st = set_smem_attr(kern, di, attr_set)) != PA_OK) return st;
        const dim3 grid((unsigned)std::max<int64_t>(1, std::min<int64_t>(L.units_ub, 2 * (int64_t)di.sms)));
        return launch_dependent(kern, grid, L.threads, L.smem, L.stream, L.kmap, L.vmap, L.qmap, L.p);
    }
}

template <typename T, int D, int G>
int dispatch_engine(Launch& L, const DevInfo& di, bool tensor) {
    return tensor ? run_decode_tc<T, D, G>(L, di) : run_decode_core<T, D, G>(L, di);
}

template <typename T, int D>
int dispatch_group(Launch& L, const DevInfo& di, int G, bool tensor) {
    switch (G) {
        case 1: return dispatch_engine<T, D, 1>(L, di, tensor);
        case 2: return dispatch_engine<T, D, 2>(L, di, tensor);
        case 4: return dispatch_engine<T, D, 4>(L, di, tensor);
        case 8: return dispatch_engine<T, D, 8>(L, di, tensor);
        default: return PA_ERR_UNSUPPORTED;
    }
}

template <typename T>
int dispatch_dim(Launch& L, const DevInfo& di, int D, int G, bool tensor) {
    switch (D) {
        case 64: return dispatch_group<T, 64>(L, di, G, tensor);
        case 128: return dispatch_group<T, 128>(L, di, G, tensor);
        default: return PA_ERR_UNSUPPORTED;
    }
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

// The split-K merge: the group shape for short splits, the sliced per-head
// shape for long ones.
// Launched as a programmatic dependent of the decode kernel: its CTAs may be
// scheduled while the decode grid drains and wait on the device for it.
template <typename T, int D>
int launch_merge_t(const Launch& L, bool group) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((int64_t)L.p.S * (group ? L.p.Hkv : L.p.Hq)));
    cfg.blockDim = dim3(group ? (unsigned)std::max(32, (L.p.Hq / L.p.Hkv) * D / 4) : MERGE_THREADS);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = group ? cudaLaunchKernelEx(&cfg, merge_group_kernel<T, D>, L.p)
                                : cudaLaunchKernelEx(&cfg, merge_head_kernel<T, D>, L.p);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int launch_merge(const Launch& L, pa_dtype dt, int D, int G, int n_pmax) {
    const bool group = n_pmax <= kShortSplit && G * D / 4 <= MERGE_THREADS;
    if (dt == PA_F32) return D == 64 ? launch_merge_t<float, 64>(L, group) : launch_merge_t<float, 128>(L, group);
    if (dt == PA_F16) return D == 64 ? launch_merge_t<__half, 64>(L, group) : launch_merge_t<__half, 128>(L, group);
    return D == 64 ? launch_merge_t<__nv_bfloat16, 64>(L, group) : launch_merge_t<__nv_bfloat16, 128>(L, group);
}

}  // namespace

}  // namespace pa

using namespace pa;

namespace {

// Host-side argument checks of pa_decode other than the workspace (everything
// that can be checked without touching the GPU); PA_OK or the status to return.
int validate_args(const void* out, const void* query, const void* key_cache,
                  const void* value_cache, const int32_t* block_tables, int max_blocks_per_seq,
                  const int32_t* context_lens, int max_context_len, int num_seqs, int num_q_heads,
                  int num_kv_heads, int head_dim, int block_size, int num_blocks,
                  int partition_size, pa_dtype dtype) {
    if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens)
        return PA_ERR_INVALID;
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || max_context_len < 0 || partition_size < 0 ||
        partition_size % TOK != 0 || num_q_heads % num_kv_heads != 0)
        return PA_ERR_INVALID;
    if (dtype != PA_F32 && dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_INVALID;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (block_size != 8 && block_size != 16 && block_size != 32 && block_size != 64 &&
        block_size != 128)
        return PA_ERR_UNSUPPORTED;
    const int G = num_q_heads / num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
    if (!aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) || !aligned16(out))
        return PA_ERR_INVALID;
    const int64_t rows = (int64_t)num_blocks * num_kv_heads * block_size;
    if (rows >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
    // the per-CTA prefix array must leave room for the pipeline
    if (num_seqs > 16384) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

// The workspace checks: present, 256-byte aligned, at least `need` bytes.
int validate_workspace(const void* workspace, size_t workspace_bytes, int num_seqs,
                       int num_q_heads, int num_kv_heads, int head_dim, int max_context_len,
                       int partition_size) {
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255)) return PA_ERR_INVALID;
    size_t need = 0;
    pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                             partition_size, &need);
    return workspace_bytes < need ? PA_ERR_INVALID : PA_OK;
}

// The launches of one decode call; the arguments have passed validate().
int decode_launch(void* out, const void* query, const void* key_cache, const void* value_cache,
                  const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                  int max_context_len, int num_seqs, int num_q_heads, int num_kv_heads,
                  int head_dim, int block_size, int num_blocks, float scale, int partition_size,
                  void* workspace, pa_dtype dtype, int32_t* err_flag, void* stream, int engine,
                  int hold_stage, const void* wkey, const void* wval, const int64_t* wslot) {
    const int G = num_q_heads / num_kv_heads;
    const int64_t rows = (int64_t)num_blocks * num_kv_heads * block_size;
    DevInfo di;
    if (dev_info(&di) != PA_OK) return PA_ERR_CUDA;

    static thread_local Launch L;
    static thread_local MapCache maps;
    const int box_rows = block_size >= TOK ? TOK : block_size;
    int st = maps.get(&L.kmap, key_cache, dtype, head_dim, rows, box_rows);
    if (st == PA_OK) st = maps.get(&L.vmap, value_cache, dtype, head_dim, rows, box_rows);
    if (st != PA_OK) return st;

    const int P = partition_size > 0 ? partition_size : std::max(TOK, max_context_len);
    const int n_pmax = std::max(1, (max_context_len + P - 1) / P);
    DecodeParams& p = L.p;
    p.out = out;
    p.q = query;
    p.tables = block_tables;
    p.lens = context_lens;
    p.mbps = max_blocks_per_seq;
    p.max_len = max_context_len;
    p.S = num_seqs;
    p.Hq = num_q_heads;
    p.Hkv = num_kv_heads;
    p.NB = num_blocks;
    p.bs = block_size;
    p.bs_log2 = __builtin_ctz((unsigned)block_size);
    p.P = P;
    p.n_pmax = n_pmax;
    p.scale_log2e = scale * 1.4426950408889634f;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.hdr = reinterpret_cast<WsHeader*>(ws);
    p.split_cnt = reinterpret_cast<int*>(ws + sizeof(WsHeader));
    p.part_ml = reinterpret_cast<float*>(ws + sizeof(WsHeader) + ws_counters(num_seqs, num_kv_heads));
    p.part_o = p.part_ml + ws_ml(num_seqs, num_q_heads, n_pmax) / 4;
    p.fused_merge = 0;       // set by the engine that takes it
    p.err = err_flag;
    p.hold_stage = hold_stage;
    p.wslot = wslot;
    p.wk = wslot ? static_cast<const uint4*>(wkey) : nullptr;
    p.wv = wslot ? static_cast<const uint4*>(wval) : nullptr;
    // the caches are written only with the step's cache write requested
    p.kc = static_cast<uint4*>(const_cast<void*>(key_cache));
    p.vc = static_cast<uint4*>(const_cast<void*>(value_cache));

    const int64_t units_ub = (int64_t)num_seqs * num_kv_heads * n_pmax;
    L.units_ub = units_ub;
    L.grid = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>(units_ub, di.sms)));
    L.stream = (cudaStream_t)stream;

    // tcgen05 engine: 16-bit types only (the default for them); fp32 runs on
    // CUDA cores
    const bool sixteen = dtype != PA_F32;
    if (engine == PA_ENGINE_TENSOR && !sixteen) return PA_ERR_UNSUPPORTED;
    const bool tensor = sixteen && engine != PA_ENGINE_CUDA_CORE;
    auto run = [&](bool use_tensor) {
        switch (dtype) {
            case PA_F32: return dispatch_dim<float>(L, di, head_dim, G, false);
            case PA_F16: return dispatch_dim<__half>(L, di, head_dim, G, use_tensor);
            case PA_BF16: return dispatch_dim<__nv_bfloat16>(L, di, head_dim, G, use_tensor);
        }
        return (int)PA_ERR_INVALID;
    };
    // the CUDA-core engine gets the step's cache write as a launch before it
    auto run_core = [&]() {
        if (wslot) {
            const int nv = head_dim * (dtype == PA_F32 ? 4 : 2) / 16;
            const int w = launch_dependent(new_token_write_kernel, dim3((unsigned)num_seqs), 128, 0,
                                           L.stream, L.p, nv);
            if (w != PA_OK) return w;
        }
        return run(false);
    };
    if (tensor) {
        st = maps.get(&L.qmap, query, dtype, head_dim, (int64_t)num_seqs * num_q_heads, G);
        if (st != PA_OK) return st;
        st = run(true);
        // by default, shapes whose stage ring does not fit (very many
        // sequences) go to the CUDA-core engine (nothing was launched)
        if (st == PA_ERR_UNSUPPORTED && engine == PA_ENGINE_AUTO) st = run_core();
    } else {
        st = run_core();
    }
    // sequences split into several partitions are merged by a second launch,
    // unless the decode kernel merged them itself
    if (st == PA_OK && n_pmax > 1 && !L.p.fused_merge) st = launch_merge(L, dtype, head_dim, G, n_pmax);
    return st;
}

}  // namespace

extern "C" {

int pa_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                             int max_context_len, int partition_size, size_t* bytes) {
    if (!bytes || num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        max_context_len < 0 || partition_size < 0 || (partition_size % TOK) != 0 ||
        num_q_heads % num_kv_heads != 0)
        return PA_ERR_INVALID;
    const int P = partition_size > 0 ? partition_size : std::max(TOK, max_context_len);
    const int n_pmax = std::max(1, (max_context_len + P - 1) / P);
    *bytes = ws_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, n_pmax);
    return PA_OK;
}

int pa_decode_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
    if (!workspace || workspace_bytes < sizeof(WsHeader)) return PA_ERR_INVALID;
    return cudaMemsetAsync(workspace, 0, workspace_bytes, (cudaStream_t)stream) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

int pa_decode_ex(void* out, const void* query, const void* key_cache, const void* value_cache,
                 const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                 int max_context_len, int num_seqs, int num_q_heads, int num_kv_heads,
                 int head_dim, int block_size, int num_blocks, float scale, int partition_size,
                 void* workspace, size_t workspace_bytes, pa_dtype dtype, int32_t* err_flag,
                 void* stream, const pa_decode_options* options) {
    int engine = PA_ENGINE_AUTO, hold = -1;
    const void* wkey = nullptr;
    const void* wval = nullptr;
    const int64_t* wslot = nullptr;
    if (options) {
        // fields past struct_size (a caller built against an older header) read as unset
        const int size = options->struct_size;
        auto has = [size](size_t off, size_t len) { return (size_t)size >= off + len; };
        if (!has(offsetof(pa_decode_options, test_withhold_stage), sizeof(int))) return PA_ERR_INVALID;
        engine = options->engine;
        hold = options->test_withhold_stage;
        if (engine < PA_ENGINE_AUTO || engine > PA_ENGINE_TENSOR || hold < -1) return PA_ERR_INVALID;
        if (has(offsetof(pa_decode_options, key_new), sizeof(void*))) wkey = options->key_new;
        if (has(offsetof(pa_decode_options, value_new), sizeof(void*))) wval = options->value_new;
        if (has(offsetof(pa_decode_options, slot_mapping), sizeof(void*)))
            wslot = options->slot_mapping;
        const int nset = (wkey != nullptr) + (wval != nullptr) + (wslot != nullptr);
        if (nset != 0 && nset != 3) return PA_ERR_INVALID;
        if (nset == 3 && (!aligned16(wkey) || !aligned16(wval) ||
                          (reinterpret_cast<uintptr_t>(wslot) & 7)))
            return PA_ERR_INVALID;
    }
    if (num_seqs == 0) return PA_OK;
    int st = validate_args(out, query, key_cache, value_cache, block_tables, max_blocks_per_seq,
                           context_lens, max_context_len, num_seqs, num_q_heads, num_kv_heads,
                           head_dim, block_size, num_blocks, partition_size, dtype);
    if (st == PA_OK)
        st = validate_workspace(workspace, workspace_bytes, num_seqs, num_q_heads, num_kv_heads,
                                head_dim, max_context_len, partition_size);
    if (st != PA_OK) return st;
    return decode_launch(out, query, key_cache, value_cache, block_tables, max_blocks_per_seq,
                         context_lens, max_context_len, num_seqs, num_q_heads, num_kv_heads,
                         head_dim, block_size, num_blocks, scale, partition_size, workspace, dtype,
                         err_flag, stream, engine, hold, wkey, wval, wslot);
}

int pa_decode(void* out, const void* query, const void* key_cache, const void* value_cache,
              const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
              int max_context_len, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
              int block_size, int num_blocks, float scale, int partition_size, void* workspace,
              size_t workspace_bytes, pa_dtype dtype, int32_t* err_flag, void* stream) {
    return pa_decode_ex(out, query, key_cache, value_cache, block_tables, max_blocks_per_seq,
                        context_lens, max_context_len, num_seqs, num_q_heads, num_kv_heads,
                        head_dim, block_size, num_blocks, scale, partition_size, workspace,
                        workspace_bytes, dtype, err_flag, stream, nullptr);
}

}  // extern "C"

// ------------------------------------------------------------ allocation-free entry point
// pa_decode_static: pa_decode with its workspace in a fixed array that the
// library itself holds in device memory, for callers that cannot allocate:
// plugins running inside a host that owns every device allocation, code whose
// memory budget is fixed up front, and latency-critical paths where a
// cudaMalloc (which may synchronise the device) is not acceptable.  The array
// is reserved on every GPU that loads this library and kept until exit.
namespace {

constexpr size_t kStaticWsBytes = (size_t)PA_DECODE_STATIC_WORKSPACE_BYTES;
static __device__ __align__(256) uint8_t g_static_ws[kStaticWsBytes];

// Device address of g_static_ws per device, with the context it was looked up
// in: after a device reset the module is loaded again (into a new context) and
// the array may sit elsewhere, so a different current context means a new
// lookup rather than a stale address.
struct StaticWs {
    void* ctx = nullptr;
    void* ptr = nullptr;
};
std::mutex g_static_mu;
StaticWs g_static[64];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
    });
    return fn;
}

// The array's device address on the current device (looked up with that
// device current, once per device and context); nullptr on a CUDA error.
void* static_ws_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    auto get_ctx = ctx_get_current_fn();
    CUcontext ctx = nullptr;
    if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS) return nullptr;
    if (!ctx) {
        // no context current on this thread yet: cudaSetDevice makes the
        // device's primary context current (and allocates nothing)
        if (cudaSetDevice(dev) != cudaSuccess || get_ctx(&ctx) != CUDA_SUCCESS || !ctx)
            return nullptr;
    }
    std::lock_guard<std::mutex> lk(g_static_mu);
    StaticWs& e = g_static[dev];
    if (!e.ptr || e.ctx != (void*)ctx) {
        // host code cannot use g_static_ws's name as a device address
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_static_ws) != cudaSuccess || !ptr) return nullptr;
        e.ptr = ptr;
        e.ctx = (void*)ctx;
    }
    return e.ptr;
}

}  // namespace

extern "C" int pa_decode_static(void* out, const void* query, const void* key_cache,
                                const void* value_cache, const int32_t* block_tables,
                                int max_blocks_per_seq, const int32_t* context_lens,
                                int max_context_len, int num_seqs, int num_q_heads,
                                int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                float scale, int partition_size, pa_dtype dtype,
                                int32_t* err_flag, void* stream) {
    if (num_seqs == 0) return PA_OK;
    size_t need = 0;
    int st = pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                      max_context_len, partition_size, &need);
    if (st != PA_OK) return st;
    if (need > kStaticWsBytes) return PA_ERR_INVALID;   // larger than the fixed array
    // every host check before the array is touched: a rejected call launches nothing
    st = validate_args(out, query, key_cache, value_cache, block_tables, max_blocks_per_seq,
                       context_lens, max_context_len, num_seqs, num_q_heads, num_kv_heads,
                       head_dim, block_size, num_blocks, partition_size, dtype);
    if (st != PA_OK) return st;
    void* ws = static_ws_ptr();
    if (!ws) return PA_ERR_CUDA;
    // the scheduler words and split counters must start at zero; the array
    // keeps whatever the last call left (a call that stopped early with
    // PA_DEV_TIMEOUT, or one of other sizes, may have left them dirty)
    const int P = partition_size > 0 ? partition_size : std::max(TOK, max_context_len);
    const int n_pmax = std::max(1, (max_context_len + P - 1) / P);
    const size_t clear = sizeof(WsHeader) + (n_pmax > 1 ? ws_counters(num_seqs, num_kv_heads) : 0);
    if (cudaMemsetAsync(ws, 0, clear, (cudaStream_t)stream) != cudaSuccess) return PA_ERR_CUDA;
    return decode_launch(out, query, key_cache, value_cache, block_tables, max_blocks_per_seq,
                         context_lens, max_context_len, num_seqs, num_q_heads, num_kv_heads,
                         head_dim, block_size, num_blocks, scale, partition_size, ws, dtype,
                         err_flag, stream, PA_ENGINE_AUTO, -1, nullptr, nullptr, nullptr);
}
