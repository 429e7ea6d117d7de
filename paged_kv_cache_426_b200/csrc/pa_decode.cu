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
//  * Persistent CTAs (one per SM).  Each CTA computes the prefix sums of the
//    partition counts (tiny), then one producer warp takes units from an
//    atomic counter in the workspace (dynamic load balance, units of at most
//    P tokens) and streams each unit as 16-token stages into a shared-memory
//    ring: 2-D tensor TMA copies of 128-byte-wide boxes with 128B swizzle,
//    one box row per token, so that all later shared-memory reads are free of
//    bank conflicts.  The block table is read 32 entries at a time by the
//    producer's lanes, ahead of use.  A 16-token stage never crosses a block
//    (bs >= 16) or covers two (bs = 8).
//  * Consumer warps take a unit's stages round-robin by logical stage index
//    and keep a per-warp online softmax (running max m, sum l, output o) in
//    the log2 domain.  Two compute engines (CUDA cores by default; the
//    tensor-core one on request, G = 1 only):
//      CUDA cores: 8 (or 16) lanes per token, 16-byte loads, warp-shuffle
//        reduce-scatter of the G dot products, then p*V with each lane owning
//        head_dim/32 output columns of all G heads;
//      MMA (16-bit types): S = Q K^T and O += P V with m16n8k16 tensor-core
//        MMAs; the query heads sit in the M dimension (rows >= G are zero),
//        K and V come from the swizzled stage with ldmatrix(.trans), and the
//        accumulators of S are reused directly as the A operand of P V.
//  * At the end of a unit the consumer warps merge their states in shared
//    memory.  A single-partition sequence writes `out` directly.  Otherwise
//    the unit writes (m, l, o) to the workspace and bumps a per-(s, j)
//    counter; the CTA that completes the last partition merges all partials
//    with their log-sum-exp weights and writes `out` (and re-zeroes the
//    counter).  No CTA ever waits for another.
//  * Summation order depends only on logical positions (stage index within
//    the unit, warp index, partition index), never on physical block ids or
//    on which CTA ran a unit, so results are bit-identical under any
//    permutation of the pool and for block sizes 16..128.
//  * Every wait is bounded (2 s); a timeout sets PA_DEV_TIMEOUT, makes the
//    other warps give up quickly, waits (bounded) for the CTA's own copies
//    in flight and returns.  Bad block ids or lengths set err_flag and the
//    affected tokens are skipped.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "pa_common.cuh"

namespace pa {

constexpr int TOK = 16;           // tokens per pipeline stage
// consumer warps per pipeline (they take a unit's stages round-robin).  A ring
// slot stays held while its consumer computes, so extra consumers only pay
// where compute is the limit: 3 for the CUDA-core engine with query groups
// (G > 1), otherwise 2.
template <bool MMA, int G> constexpr int cons_for() { return (!MMA && G > 1) ? 3 : 2; }
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
    int pad[62];
};

struct DecodeParams {
    void* out;
    const void* q;
    const int32_t* tables;
    const int32_t* lens;
    int mbps, max_len, S, Hq, Hkv, NB, bs, bs_log2, P, n_pmax, nst;
    float scale_log2e;
    WsHeader* hdr;
    int* counters;     // [S*Hkv]
    float* part_ml;    // [S*Hkv][n_pmax][G][2]
    float* part_o;     // [S*Hkv][n_pmax][G][D]
    int32_t* err;
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
    using LY = Layout<T, D, G, cons_for<false, G>()>;
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

template <typename T, int D, int G>
struct MmaEngine {
    static_assert(sizeof(T) == 2, "tensor-core engine takes 16-bit types");
    static_assert(G <= 8, "query heads of a group must fit 8 MMA rows");
    static constexpr int KSTEPS = D / 16;
    static constexpr int NDT = D / 8;          // 8-column output tiles

    uint32_t qa[KSTEPS][2];    // A fragments of Q (rows lane/4, k low / k high)
    float oacc[NDT][4];        // O rows lane/4 (and padding rows +8)
    float m, l;                // state of row lane/4

    __device__ void begin_unit(const T* qs, int lane, float) {
        const int r = lane >> 2, c = lane & 3;
        const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qs);
#pragma unroll
        for (int k = 0; k < KSTEPS; ++k) {
            qa[k][0] = (r < G) ? q32[(r * D + 16 * k + 2 * c) >> 1] : 0u;
            qa[k][1] = (r < G) ? q32[(r * D + 16 * k + 8 + 2 * c) >> 1] : 0u;
        }
#pragma unroll
        for (int n = 0; n < NDT; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) oacc[n][e] = 0.f;
        m = -INFINITY;
        l = 0.f;
    }

    __device__ void stage(const uint8_t* Ks, uint8_t* Vs, int nv, float scale_log2e, int lane) {
        const uint32_t kbase = smem_u32(Ks), vbase = smem_u32(Vs);
        if (nv < TOK) {
            // rows >= nv hold bytes of other tokens (or never-written memory);
            // zero them so that p = 0 never meets a NaN in the P V product
            constexpr int ROW16 = D * 2 / 16;
            for (int idx = lane; idx < (TOK - nv) * ROW16; idx += 32) {
                const int row = nv + idx / ROW16, ch = idx % ROW16;
                *reinterpret_cast<uint4*>(Vs + (ch >> 3) * BOXB + row * 128 +
                                          (((ch & 7) ^ (row & 7)) << 4)) = make_uint4(0, 0, 0, 0);
            }
            __syncwarp();
        }
        // ---- S = Q K^T  (rows: heads, columns: 16 tokens as two n-tiles)
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
        const int mi = lane >> 3, lr = lane & 7;
#pragma unroll
        for (int k = 0; k < KSTEPS; ++k) {
            const int row = (mi >> 1) * 8 + lr, ch = 2 * k + (mi & 1);
            uint32_t b00, b01, b10, b11;
            ldsm_x4(kbase + (ch >> 3) * BOXB + row * 128 + (((ch & 7) ^ (row & 7)) << 4), b00, b01,
                    b10, b11);
            mma16816<T>(s0, qa[k][0], 0u, qa[k][1], 0u, b00, b01);
            mma16816<T>(s1, qa[k][0], 0u, qa[k][1], 0u, b10, b11);
        }
        // ---- online softmax of row lane/4 over this stage's tokens
        const int c = lane & 3;
        const int t0 = 2 * c, t1 = 2 * c + 1, t2 = 8 + 2 * c, t3 = 9 + 2 * c;
        float x0 = (t0 < nv) ? s0[0] * scale_log2e : -INFINITY;
        float x1 = (t1 < nv) ? s0[1] * scale_log2e : -INFINITY;
        float x2 = (t2 < nv) ? s1[0] * scale_log2e : -INFINITY;
        float x3 = (t3 < nv) ? s1[1] * scale_log2e : -INFINITY;
        float bm = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
        const float mn = fmaxf(m, bm);
        const float a = exp2f(m - mn);
        const float p0 = exp2f(x0 - mn), p1 = exp2f(x1 - mn);
        const float p2 = exp2f(x2 - mn), p3 = exp2f(x3 - mn);
        float rs = (p0 + p1) + (p2 + p3);
        rs += __shfl_xor_sync(0xffffffffu, rs, 1);
        rs += __shfl_xor_sync(0xffffffffu, rs, 2);
        l = l * a + rs;
        m = mn;
#pragma unroll
        for (int n = 0; n < NDT; ++n) {
            oacc[n][0] *= a;
            oacc[n][1] *= a;
        }
        const uint32_t pa0 = pack2<T>(p0, p1), pa2 = pack2<T>(p2, p3);
        // ---- O += P V  (B operand = V [tokens x columns] via ldmatrix.trans)
#pragma unroll
        for (int n2 = 0; n2 < NDT / 2; ++n2) {
            const int row = (mi & 1) * 8 + lr, ch = 2 * n2 + (mi >> 1);
            uint32_t v0, v1, v2, v3;
            ldsm_x4_t(vbase + (ch >> 3) * BOXB + row * 128 + (((ch & 7) ^ (row & 7)) << 4), v0, v1,
                      v2, v3);
            mma16816<T>(oacc[2 * n2], pa0, 0u, pa2, 0u, v0, v1);
            mma16816<T>(oacc[2 * n2 + 1], pa0, 0u, pa2, 0u, v2, v3);
        }
    }

    __device__ void dump(float* mb, int lane) const {
        const int r = lane >> 2, c = lane & 3;
        if (r < G) {
#pragma unroll
            for (int n = 0; n < NDT; ++n)
                *reinterpret_cast<float2*>(&mb[r * (D + 2) + 2 + 8 * n + 2 * c]) =
                    make_float2(oacc[n][0], oacc[n][1]);
            if (c == 0) {
                mb[r * (D + 2) + 0] = m;
                mb[r * (D + 2) + 1] = l;
            }
        }
    }
};

// ------------------------------------------------------------ the kernel
// Warp roles: warp w belongs to pipeline w / PIPE_WARPS; role w % PIPE_WARPS is
// 0 for the producer and 1..NCONS for the consumers.  The pipelines of a CTA
// share nothing but the prefix sums and the abort flag; each takes its own
// units from the global ticket counter.
template <typename T, int D, int G, bool MMA>
__global__ void __launch_bounds__(Layout<T, D, G, cons_for<MMA, G>()>::NTHREADS, 1)
decode_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
              DecodeParams p) {
    using LY = Layout<T, D, G, cons_for<MMA, G>()>;
    using Engine = typename std::conditional<MMA, MmaEngine<T, D, G>, CoreEngine<T, D, G>>::type;
    constexpr int NCONS = LY::NCONS;
    constexpr int PIPE_WARPS = LY::PIPE_WARPS;
    constexpr int NPIPE = LY::NPIPE;
    constexpr int NTHREADS = LY::NTHREADS;
    constexpr int CT = NCONS * 32;               // consumer threads of a pipeline
    constexpr int E = sizeof(T);
    constexpr int BOX_ELEMS = 128 / E;

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
    volatile int* last_flag = misc + 1 + pipe;
    int* wsum = misc + 32;
    auto desc_at = [&](int k) { return reinterpret_cast<UnitDesc*>(smem + ly.unit(pipe, k)); };
    auto q_at = [&](int k) {
        return reinterpret_cast<T*>(smem + ly.unit(pipe, k) + sizeof(UnitDesc));
    };

    if (tid == 0) {
        for (int pp = 0; pp < NPIPE; ++pp) {
            uint64_t* b = reinterpret_cast<uint64_t*>(smem + ly.bars(pp));
            for (int k = 0; k < 2 * nst + 2 * NUR; ++k) mbar_init(b + k, 1);
        }
        for (int k = 0; k < 32; ++k) misc[k] = 0;
        fence_barrier_init();
    }
    if (role == 0 && lane == 0 && pipe == 0) {
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
    }

    // ---- prefix sums of partitions per sequence (each CTA, tiny)
    {
        constexpr int NW = NTHREADS / 32;
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
    }
    __syncthreads();
    const int U = pre[p.S] * p.Hkv;

    if (role == 0) {
        // ================================================= producer warp
        // Per unit: the next unit's ticket (global atomic) and its first 64
        // block ids are fetched while the current unit's stages are issued,
        // so no global round trip sits between two stages.  The TMA copies
        // of a stage are issued by several lanes at once.
        const uint64_t policy = policy_evict_first();
        const size_t qrow = (size_t)p.Hq * D * E;
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
            const int slot = ucount % NUR;
            if (ucount >= NUR) {
                bool w = true;
                if (lane == 0) w = wait_or_abort(uempty + slot, ((ucount / NUR) - 1) & 1, abort_flag, p.err);
                if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
            }
            UnitDesc* d = desc_at(slot);
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
                mbar_arrive_expect_tx(ufull + slot, G * D * E);
                bulk_g2s(q_at(slot),
                         reinterpret_cast<const uint8_t*>(p.q) + (size_t)cur.s * qrow +
                             (size_t)cur.j * G * D * E,
                         G * D * E, ufull + slot);
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
                    if (lane == 0) w = wait_or_abort(empty + st, (round - 1) & 1, abort_flag, p.err);
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
                uint8_t* Kd = stages + (size_t)st * LY::STAGE_BYTES;
                if (lane == 0) {
                    stage_ok[st] = valid ? 1 : 0;
                    if (!valid) {
                        set_err(p.err, PA_DEV_BAD_BLOCK);
                        mbar_arrive(full + st);
                    } else {
                        mbar_arrive_expect_tx(full + st, (has1 ? 2u : 1u) * 2u * prow * LY::ROWB);
                    }
                }
                __syncwarp();
                // one TMA box per lane: (piece, K or V, 128-byte column box)
                const int nops = valid ? (has1 ? 2 : 1) * 2 * LY::NBOX : 0;
                if (lane < nops) {
                    const int piece = lane / (2 * LY::NBOX), rem = lane % (2 * LY::NBOX);
                    const int kv = rem / LY::NBOX, b = rem % LY::NBOX;
                    const int y = piece ? ((blk1 * p.Hkv + cur.j) << bsl)
                                        : (((blk0 * p.Hkv + cur.j) << bsl) + off0);
                    uint8_t* dst = Kd + kv * LY::KV_BYTES + b * BOXB + piece * 8 * 128;
                    tma_load_2d(dst, kv ? &vmap : &kmap, b * BOX_ELEMS, y, full + st, policy);
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
            for (int g = first; g < gstage; ++g) mbar_wait(full + g % nst, (g / nst) & 1);
            const int ufirst = max(0, ucount - NUR);
            for (int k = ufirst; k < ucount; ++k) mbar_wait(ufull + k % NUR, (k / NUR) & 1);
        }
        __syncwarp();
    } else {
        // ================================================= consumer warps
        const int cw = role - 1;                 // 0 .. NCONS-1
        const int ctid = cw * 32 + lane;         // 0 .. CT-1
        const int bar_id = 1 + pipe;             // named barrier of this pipeline
        Engine eng;
        float* xs = scratch + cw * 3 * G * TOK;
        uint64_t* ps = reinterpret_cast<uint64_t*>(xs + G * TOK);
        uint4* qf4 = reinterpret_cast<uint4*>(scratch + NCONS * 3 * G * TOK);   // fp32 q (core engine)
        int ucount = 0;
        while (true) {
            const int slot = ucount % NUR;
            // every lane waits; __all_sync reconverges the warp (the tensor-core
            // engine's ldmatrix/mma are .aligned and need the whole warp) and
            // makes the decision the same in every lane
            if (!__all_sync(0xffffffffu, wait_or_abort(ufull + slot, (ucount / NUR) & 1, abort_flag, p.err)))
                break;
            const UnitDesc d = *desc_at(slot);
            if (d.end) break;
            if constexpr (MMA) {
                eng.begin_unit(q_at(slot), lane, p.scale_log2e);
            } else {
                Engine::stage_q(q_at(slot), qf4, ctid, CT, p.scale_log2e);
                named_bar_sync(bar_id, CT);                 // q in fp32 for every consumer warp
                eng.begin_unit(qf4);
            }
            int st = (d.stage_base + cw) % nst;
            uint32_t ph = ((d.stage_base + cw) / nst) & 1;
            for (int c = cw; c < d.n_stages; c += NCONS) {
                const bool have = __all_sync(0xffffffffu, wait_or_abort(full + st, ph, abort_flag, p.err));
                if (have && stage_ok[st]) {
                    const int nv = min(TOK, d.t1 - (d.t0 + c * TOK));
                    uint8_t* Ks = stages + (size_t)st * LY::STAGE_BYTES;
                    if constexpr (MMA) {
                        eng.stage(Ks, Ks + LY::KV_BYTES, nv, p.scale_log2e, lane);
                        if (nv < TOK) fence_proxy_async_smem();
                    } else {
                        eng.stage(Ks, Ks + LY::KV_BYTES, nv, xs, ps, lane);
                    }
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
            if (d.n_p > 1) {
                if (ctid == 0) {
                    __threadfence();                   // publish the partials before the count
                    const int prev = atomicAdd(p.counters + sj, 1);
                    const int last = (prev == d.n_p - 1);
                    if (last) {
                        p.counters[sj] = 0;            // every partition has arrived
                        __threadfence();               // see the other CTAs' partials
                    }
                    *last_flag = last;
                }
                named_bar_sync(bar_id, CT);
                if (*last_flag) {
                    const size_t base = sj * p.n_pmax;
                    for (int idx = ctid; idx < G * D; idx += CT) {
                        const int g = idx / D, dd = idx % D;
                        float M = -INFINITY;
                        for (int i = 0; i < d.n_p; ++i)
                            M = fmaxf(M, __ldcg(p.part_ml + ((base + i) * G + g) * 2));
                        float Lsum = 0.f, O = 0.f;
                        if (M != -INFINITY) {
                            int i = 0;
                            for (; i + 4 <= d.n_p; i += 4) {
                                float mm[4], ll[4], oo[4];
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    const size_t pi = (base + i + k) * G + g;
                                    mm[k] = __ldcg(p.part_ml + pi * 2);
                                    ll[k] = __ldcg(p.part_ml + pi * 2 + 1);
                                    oo[k] = __ldcg(p.part_o + pi * D + dd);
                                }
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    const float f = exp2f(mm[k] - M);
                                    Lsum += ll[k] * f;
                                    O += oo[k] * f;
                                }
                            }
                            for (; i < d.n_p; ++i) {
                                const size_t pi = (base + i) * G + g;
                                const float f = exp2f(__ldcg(p.part_ml + pi * 2) - M);
                                Lsum += __ldcg(p.part_ml + pi * 2 + 1) * f;
                                O += __ldcg(p.part_o + pi * D + dd) * f;
                            }
                        }
                        T* outp = reinterpret_cast<T*>(p.out) + ((size_t)d.s * p.Hq + (size_t)d.j * G + g) * D + dd;
                        *outp = DT<T>::from_float(Lsum > 0.f ? O / Lsum : 0.f);
                    }
                }
                named_bar_sync(bar_id, CT);                      // last_flag free again
            }
            ++ucount;
        }
        __syncwarp();
    }

    __syncthreads();
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

// ------------------------------------------------------------ host side
namespace {

int g_engine = PA_ENGINE_AUTO;
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

// Tensor map over a cache viewed as [num_blocks*Hkv*bs rows][D columns]; box =
// 128 bytes x box_rows, 128B swizzle.
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

struct DevInfo {
    int sms = 0;
    int smem_optin = 0;
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
                cudaSuccess)
            return PA_ERR_CUDA;
        have[dev] = true;
    }
    *out = cache[dev];
    return PA_OK;
}

constexpr int kMaxStages = 8;     // stages per pipeline
constexpr int kMinStages = 2;     // any count >= 1 is correct; fewer only slows the pipeline

size_t ws_bytes(int S, int Hq, int Hkv, int D, int n_pmax) {
    size_t b = sizeof(WsHeader);
    b += (((size_t)S * Hkv * 4 + 255) / 256) * 256;
    if (n_pmax > 1) {
        b += (((size_t)S * Hq * n_pmax * 2 * 4 + 255) / 256) * 256;
        b += (size_t)S * Hq * n_pmax * D * 4;
    }
    return b;
}

struct Launch {
    CUtensorMap kmap, vmap;
    DecodeParams p;
    dim3 grid;
    int threads;
    size_t smem;
    cudaStream_t stream;
};

template <typename T, int D, int G, bool MMA>
int run_decode(Launch& L, const DevInfo& di) {
    using LY = Layout<T, D, G, cons_for<MMA, G>()>;
    auto kern = decode_kernel<T, D, G, MMA>;
    // a stage costs its K/V bytes, two mbarriers and a validity flag; the
    // rest of the layout is fixed; + 1024 bytes of alignment slack
    const size_t fixed = LY(0, L.p.S).total() + 1024 + 16;
    const size_t per_stage = (size_t)LY::NPIPE * (LY::STAGE_BYTES + 2 * 8 + 4);
    if ((size_t)di.smem_optin < fixed + (size_t)kMinStages * per_stage) return PA_ERR_UNSUPPORTED;
    int nst = (int)((di.smem_optin - fixed) / per_stage);
    nst = std::min(nst, kMaxStages);
    while (nst > kMinStages && LY(nst, L.p.S).total() + 1024 > (size_t)di.smem_optin) --nst;
    L.p.nst = nst;
    L.smem = LY(nst, L.p.S).total() + 1024;
    if (L.smem > (size_t)di.smem_optin) return PA_ERR_UNSUPPORTED;
    L.threads = LY::NTHREADS;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev & 63]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, di.smem_optin) !=
            cudaSuccess)
            return PA_ERR_CUDA;
        attr_set[dev & 63] = true;
    }
    kern<<<L.grid, L.threads, L.smem, L.stream>>>(L.kmap, L.vmap, L.p);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <typename T, int D, int G>
int dispatch_engine(Launch& L, const DevInfo& di, bool mma) {
    if constexpr (sizeof(T) == 2) {
        if (mma) return run_decode<T, D, G, true>(L, di);
    }
    return run_decode<T, D, G, false>(L, di);
}

template <typename T, int D>
int dispatch_group(Launch& L, const DevInfo& di, int G, bool mma) {
    switch (G) {
        case 1: return dispatch_engine<T, D, 1>(L, di, mma);
        case 2: return dispatch_engine<T, D, 2>(L, di, mma);
        case 4: return dispatch_engine<T, D, 4>(L, di, mma);
        case 8: return dispatch_engine<T, D, 8>(L, di, mma);
        default: return PA_ERR_UNSUPPORTED;
    }
}

template <typename T>
int dispatch_dim(Launch& L, const DevInfo& di, int D, int G, bool mma) {
    switch (D) {
        case 64: return dispatch_group<T, 64>(L, di, G, mma);
        case 128: return dispatch_group<T, 128>(L, di, G, mma);
        default: return PA_ERR_UNSUPPORTED;
    }
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

}  // namespace

}  // namespace pa

using namespace pa;

extern "C" {

int pa_set_decode_engine(int engine) {
    if (engine < PA_ENGINE_AUTO || engine > PA_ENGINE_MMA) return PA_ERR_INVALID;
    std::lock_guard<std::mutex> lk(g_mu);
    const int prev = g_engine;
    g_engine = engine;
    return prev;
}

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

int pa_decode(void* out, const void* query, const void* key_cache, const void* value_cache,
              const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
              int max_context_len, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
              int block_size, int num_blocks, float scale, int partition_size, void* workspace,
              size_t workspace_bytes, pa_dtype dtype, int32_t* err_flag, void* stream) {
    if (num_seqs == 0) return PA_OK;
    if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens ||
        !workspace)
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
    if (!aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255))
        return PA_ERR_INVALID;
    const int64_t rows = (int64_t)num_blocks * num_kv_heads * block_size;
    if (rows >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
    size_t need = 0;
    pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                             partition_size, &need);
    if (workspace_bytes < need) return PA_ERR_INVALID;
    const int G = num_q_heads / num_kv_heads;

    DevInfo di;
    if (dev_info(&di) != PA_OK) return PA_ERR_CUDA;
    // the per-CTA prefix array must leave room for the pipeline
    if (num_seqs > 16384) return PA_ERR_UNSUPPORTED;

    static thread_local Launch L;
    const int box_rows = block_size >= TOK ? TOK : block_size;
    int st = make_map(&L.kmap, key_cache, dtype, head_dim, rows, box_rows);
    if (st == PA_OK) st = make_map(&L.vmap, value_cache, dtype, head_dim, rows, box_rows);
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
    p.counters = reinterpret_cast<int*>(ws + sizeof(WsHeader));
    const size_t cnt_bytes = (((size_t)num_seqs * num_kv_heads * 4 + 255) / 256) * 256;
    p.part_ml = reinterpret_cast<float*>(ws + sizeof(WsHeader) + cnt_bytes);
    p.part_o = p.part_ml + ((((size_t)num_seqs * num_q_heads * n_pmax * 2 * 4 + 255) / 256) * 256) / 4;
    p.err = err_flag;

    const int64_t units_ub = (int64_t)num_seqs * num_kv_heads * n_pmax;
    L.grid = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>(units_ub, di.sms)));
    L.stream = (cudaStream_t)stream;

    int engine;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        engine = g_engine;
    }
    // The tensor-core engine is enabled only on request and only for G = 1:
    // with G > 1 it failed (launch failure / timeouts) at full size under the
    // multi-pipeline schedule for a cause not yet found, so it is not run.
    const bool mma = engine == PA_ENGINE_MMA;
    if (mma && (dtype == PA_F32 || G != 1)) return PA_ERR_UNSUPPORTED;
    switch (dtype) {
        case PA_F32: return dispatch_dim<float>(L, di, head_dim, G, false);
        case PA_F16: return dispatch_dim<__half>(L, di, head_dim, G, mma);
        case PA_BF16: return dispatch_dim<__nv_bfloat16>(L, di, head_dim, G, mma);
    }
    return PA_ERR_INVALID;
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

std::mutex g_static_mu;
void* g_static_ptr[64] = {};   // device address of g_static_ws, per device

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
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PA_ERR_CUDA;
    void* ws = nullptr;
    {
        // first call on this device (with it current): look up the array's
        // device address; host code cannot use g_static_ws's name directly
        std::lock_guard<std::mutex> lk(g_static_mu);
        if (!g_static_ptr[dev]) {
            void* ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, g_static_ws) != cudaSuccess || !ptr) return PA_ERR_CUDA;
            g_static_ptr[dev] = ptr;
        }
        ws = g_static_ptr[dev];
    }
    // the scheduler words and partition counters must start at zero; a call
    // that stopped early (PA_DEV_TIMEOUT) may have left them dirty
    const size_t counters = sizeof(WsHeader) + (((size_t)num_seqs * num_kv_heads * 4 + 255) / 256) * 256;
    if (cudaMemsetAsync(ws, 0, counters, (cudaStream_t)stream) != cudaSuccess) return PA_ERR_CUDA;
    return pa_decode(out, query, key_cache, value_cache, block_tables, max_blocks_per_seq,
                     context_lens, max_context_len, num_seqs, num_q_heads, num_kv_heads,
                     head_dim, block_size, num_blocks, scale, partition_size, ws,
                     kStaticWsBytes, dtype, err_flag, stream);
}
