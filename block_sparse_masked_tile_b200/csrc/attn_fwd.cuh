// Block-sparse masked attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// This is the method of the tensorplay.nn.attention page (BlockMask
// "Details" items 1-2):
//   - the kernel visits only the kv blocks a BlockMask row lists;
//   - it applies mask_mod only on PARTIAL blocks;
//   - it applies score_mod (attention-gym page: a change to the score
//     before the softmax) on every visited block.
// Attention is computed tile by tile with an online softmax and the full
// score matrix is never written (L-GATr page, "Why care about Attention
// Kernels?").
//
// One persistent CTA per SM. A work unit is (b, hq, pair of adjacent
// 128-row q-blocks). Warp roles in a CTA:
//   warps 0-3  softmax for q-block 0 of the pair (one query row per thread)
//   warps 4-7  softmax for q-block 1
//   warp 8     TMA producer: Q tiles, then K and V tiles into a ring of slots
//   warp 9     allocates TMEM; issues the MMAs of q-block 0 (one elected lane)
//   warp 11    issues the MMAs of q-block 1
//   warp 10    scheduler. It merges the two rows' partial and full block
//              lists into one ascending stream of (kb, tags) in shared
//              memory, so each K/V tile is loaded once for both q-blocks.
//
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [384,384+D)
// (O1 starts at 256+D when D=64). P (bf16 pairs) overwrites the first 64
// columns of its S.
//
// The two softmax warpgroups work on their own q-blocks and fall into a
// ping-pong by themselves: while one runs its softmax, the tensor core runs
// the other's products. Two issuer warps walk the entry stream in order and,
// taking turns, issue each q-block's PV(n) as soon as its P(n) is stored,
// then its S(n+1). S overwrites the TMEM
// columns that P(n) occupies, and MMAs from one thread run in issue order.
// A tcgen05.commit fires once every earlier MMA of the thread is done, so
// when a warpgroup sees S(next) ready, its PV(n) has finished: O can be
// rescaled and P can overwrite S with no further barrier. A K/V ring slot is
// free once both q-blocks are done with it: each issuer commits after the
// MMA that read the slot, or arrives directly if its q-block skips it.
//
// The online softmax is in base 2 with a lazy reference max. O and l are
// rescaled only when a row's max grows by more than 2^8. The final
// out = O / l and lse = ln2 * (m_ref + log2 l) do not depend on when the
// reference moved, so the result is exact.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "mask_dnf.cuh"
#include "ptx.cuh"

namespace bsmt {

enum ScoreMode : int {
    kScoreNone = 0,
    kScoreSoftcap = 1,
    kScoreAlibi = 2,
    kScoreSoftcapAlibi = 3,  // softcap, then ALiBi
    kScoreAlibiSoftcap = 4,  // ALiBi, then softcap
};

struct AttnParams {
    int32_t B, Hq, Hkv, M, N, QB, KB, pairs, group;
    int32_t Bm, Hm;  // BlockMask batch / head extent (1 = broadcast)
    const int32_t* kv_num;
    const int32_t* kv_idx;
    const int32_t* full_num;
    const int32_t* full_idx;
    int32_t has_block_mask;
    int32_t num_units;
    float scale;       // natural-units softmax scale
    float scale_log2;  // scale * log2(e)
    float cap;         // soft-cap
    float inv_cap;     // 1 / cap
    const float* slopes;  // ALiBi slopes [Hq] or null (default 2^(-8(h0+h+1)/Ht))
    int32_t alibi_h0, alibi_heads;  // h0 and Ht of the default slopes
    __nv_bfloat16* out;
    float* lse;
    // out element (b, hq, i, d) sits at out + (b*Hq + hq)*out_sbh + i*out_ss + d:
    // (M*D, D) for [B, Hq, M, D], (D, Hq*D) for the packed [M, Hq, D] (B = 1)
    int64_t out_sbh, out_ss;
    // split-KV: each (b, hq, q-block pair) row of entries is cut into
    // num_splits consecutive slices, one unit each. With num_splits > 1 the
    // epilogue writes, per slice, O / l in fp32 to ws_o [S][B*Hq*M][D] and the
    // slice's lse to ws_lse [S][B*Hq*M]; splitkv_combine_kernel merges them.
    int32_t num_splits;
    float* ws_o;
    float* ws_lse;
};

constexpr int kThreads = 384;  // 12 warps: 3 warpgroups
constexpr int kWarpLoad = 8;
constexpr int kWarpMma = 9;    // also the MMA issuer for q-block 0
constexpr int kWarpMma1 = 11;  // MMA issuer for q-block 1
constexpr int kWarpSched = 10;
constexpr int kMaxKB = 1024;   // kv blocks per row supported by the schedule buffer
constexpr int kRing = 4;       // K/V ring slots (K in even slots, V in odd slots)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kRowTerms = 4;   // mask alternatives kept per row in registers

// Tags of one union entry (bits 16.. of the packed entry).
constexpr uint32_t kTagIn0 = 1u, kTagIn1 = 2u, kTagPart0 = 4u, kTagPart1 = 8u;

struct SchedHeader {
    int32_t T;      // union length; -1 marks the end of the work
    int32_t b, hq, qb0;
    int32_t n0, n1;  // tiles visited by q-block 0 / 1
    float slope;     // ALiBi slope of hq (natural units)
    int32_t split;   // slice of the entry stream (split-KV), 0 otherwise
    int32_t kb_base; // entries hold kv blocks relative to this block
    int32_t seg;     // kSegFirst | kSegLast | kSegMany
};

// Segments of a unit: the first and the last of its windows, and whether it
// has more than one. A unit of one segment carries exact tile counts (n0, n1)
// up front; the segments of a longer one carry their own counts only.
constexpr int32_t kSegFirst = 1, kSegLast = 2, kSegMany = 4;

// At D = 64 the tensor core also sums each row of P: the PV product runs with
// N = D + 16 over V followed by a block of ones, so O's column D holds the row
// sum l (of the bf16 P the product uses). TMEM has room for the wider O only
// at D = 64.
template <int D>
constexpr bool kTcRowSum = D == 64;
template <int D>
constexpr int kOCols = D + (kTcRowSum<D> ? 16 : 0);  // TMEM columns of one O accumulator

template <int D>
struct SmemLayout {
    static constexpr int kTileBytes = 128 * D * 2;          // one 128-row bf16 tile
    static constexpr int kQ0 = 0;
    static constexpr int kQ1 = kQ0 + kTileBytes;
    static constexpr int kRingBase = kQ1 + kTileBytes;
    static constexpr int kSched = kRingBase + kRing * kTileBytes;
    static constexpr int kSchedEntries = 0;                  // uint32 [kMaxKB]
    static constexpr int kSchedDocLo = kMaxKB * 4;           // int32 [256]: row's document kv interval
    static constexpr int kSchedDocHi = kSchedDocLo + 256 * 4;
    static constexpr int kSchedHeader = kSchedDocHi + 256 * 4;
    static constexpr int kSchedBytes = kSchedHeader + 64;
    static constexpr int kFlags = kSched + 2 * kSchedBytes;  // uint8 [kMaxKB]
    static constexpr int kBars = kFlags + kMaxKB;
    // barriers (8 bytes each)
    static constexpr int kBarQFull = 0, kBarQEmpty = 2, kBarSFull = 4, kBarPFull = 6, kBarOFull = 8,
                         kBarOEmpty = 10, kBarKvFull = 12, kBarKvEmpty = 12 + kRing,
                         kBarSchedFull = 12 + 2 * kRing, kBarSchedEmpty = 14 + 2 * kRing,
                         kBarDone = 16 + 2 * kRing, kBarTok = 18 + 2 * kRing, kNumBars = 20 + 2 * kRing;
    static constexpr int kTmemSlot = kBars + kNumBars * 8;
    static constexpr int kAbort = kTmemSlot + 4;
    // out staging: one 32-row x 32-column bf16 block (2 KB, 64-byte swizzle)
    // per softmax warp, written by the warp and stored by TMA
    static constexpr int kStage = (kAbort + 4 + 1023) / 1024 * 1024;
    static constexpr int kStageBytes = 32 * 32 * 2;
    // the ones block of the row-sum product (a 128 x 64 bf16 tile of 1.0)
    static constexpr int kOnes = kStage + 8 * kStageBytes;
    static constexpr int kOnesBytes = kTcRowSum<D> ? 128 * 64 * 2 : 0;
    static constexpr int kTotal = kOnes + kOnesBytes;
    static constexpr int kAlloc = kTotal + 1024;  // room to align the base to 1024 B
    static_assert(kAlloc <= 227 * 1024, "shared memory layout exceeds one CTA's limit");
};

__device__ __forceinline__ uint32_t sched_entry_kb(uint32_t e) { return e & 0xFFFFu; }
__device__ __forceinline__ uint32_t sched_entry_tags(uint32_t e) { return e >> 16; }

// Columns per 32-column chunk whose exp2 runs on the FMA pipe instead of
// MUFU. The row's exponentials are the softmax's largest cost; a small share
// on the FMA pipe shortens the MUFU-bound stretch, a larger share costs more
// issue slots than it saves (measured on B200 for D = 64 and 128).
template <int D>
constexpr int kEmuCols = 8;

// 2^x on the FMA pipe for a pair: round x to n, 2^f by a degree-3 polynomial
// for f = x - n in [-1/2, 1/2] (minimax in relative error, max 1.02e-4; the
// coefficients come from tests/fit_exp2_poly.py), and n goes straight into the
// exponent bits. Inputs are clamped at -125 so the exponent field stays
// positive; 2^-125 is far below what a bf16 P or an fp32 row sum can see.
constexpr float kExp2C1 = 0.69328314f;
constexpr float kExp2C2 = 0.24221109f;
constexpr float kExp2C3 = 0.05500825f;

__device__ __forceinline__ void exp2_poly2(float& y0, float& y1, float x0, float x1) {
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: x + kRound rounds x to an integer
    x0 = fmaxf(x0, -125.f);
    x1 = fmaxf(x1, -125.f);
    float t0, t1, n0, n1, f0, f1, q0, q1;
    add2(t0, t1, x0, x1, kRound, kRound);
    add2(n0, n1, t0, t1, -kRound, -kRound);
    fma2(f0, f1, n0, n1, -1.f, -1.f, x0, x1);
    fma2(q0, q1, kExp2C3, kExp2C3, f0, f1, kExp2C2, kExp2C2);
    fma2(q0, q1, q0, q1, f0, f1, kExp2C1, kExp2C1);
    fma2(q0, q1, q0, q1, f0, f1, 1.f, 1.f);
    // the low mantissa bits of t hold n; (bits(t) << 23) adds n to the exponent
    y0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
    y1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

// LONG: rows may span more than kMaxKB kv blocks (units in windows and
// segments). Without it the kernel assumes KB <= kMaxKB and every unit is one
// segment from block 0, and the segment logic folds away.
template <int D, int SCORE, bool LONG>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
                    const AttnParams p, const MaskDnf dnf) {
    using L = SmemLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);

    // ------------------------------------------------------------ set-up
    if (warp == kWarpLoad && lane == 0) {
        mbar_init(bar(L::kBarQFull + 0), 1);
        mbar_init(bar(L::kBarQFull + 1), 1);
        mbar_init(bar(L::kBarQEmpty + 0), 1);
        mbar_init(bar(L::kBarQEmpty + 1), 1);
        mbar_init(bar(L::kBarSFull + 0), 1);
        mbar_init(bar(L::kBarSFull + 1), 1);
        mbar_init(bar(L::kBarPFull + 0), 4);
        mbar_init(bar(L::kBarPFull + 1), 4);
        mbar_init(bar(L::kBarOFull + 0), 1);
        mbar_init(bar(L::kBarOFull + 1), 1);
        for (int s = 0; s < kRing; ++s) {
            mbar_init(bar(L::kBarKvFull + s), 1);
            mbar_init(bar(L::kBarKvEmpty + s), 2);  // one arrival per softmax warpgroup
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(L::kBarSchedFull + s), 32);
            mbar_init(bar(L::kBarSchedEmpty + s), 1 + 8 + 2);  // producer, 8 softmax warps, 2 MMA issuers
        }
        mbar_init(bar(L::kBarDone + 0), 1);
        mbar_init(bar(L::kBarDone + 1), 1);
        mbar_init(bar(L::kBarTok + 0), 1);
        mbar_init(bar(L::kBarTok + 1), 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_out);
    }
    if (warp == kWarpMma) {
        tmem_alloc(sbase + L::kTmemSlot, 512);
        tmem_relinquish();
    }
    if constexpr (kTcRowSum<D>) {
        uint4* ones = reinterpret_cast<uint4*>(smem + L::kOnes);
        for (int j = threadIdx.x; j < L::kOnesBytes / 16; j += kThreads)
            ones[j] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);  // bf16 1.0 pairs
        fence_proxy_async_smem();  // read by the tensor core (async proxy)
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tm_s[2] = {tmem + 0u, tmem + 128u};
    const uint32_t tm_o[2] = {tmem + 256u, tmem + 256u + static_cast<uint32_t>(kOCols<D>)};

    auto sched_base = [&](int buf) -> uint8_t* { return smem + L::kSched + buf * L::kSchedBytes; };


    // Register split: the launch gives every thread 168 registers (384
    // threads, one CTA per SM; build.py checks the count ptxas reports).
    // Warpgroup 2 (scheduler, producer, two MMA issuers) needs
    // few registers, so it gives them back and the two softmax warpgroups
    // take them: 128 * 72 + 256 * 216 = 64512 = 384 * 168. Each role sits
    // inside the branch of its warpgroup's setmaxnreg, so the compiler
    // allocates each region to its own limit.
    if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 72;\n" ::: "memory");
    if (warp == kWarpSched) {
        // ================================================= scheduler warp
        uint8_t* flags = smem + L::kFlags;
        for (int j = lane; j < kMaxKB; j += 32) flags[j] = 0;
        __syncwarp();
        int iter = 0;
        const uint32_t below = (1u << lane) - 1u;
        const bool ragged_kv = (p.N & 127) != 0;
        // the document searched last (batch row of the ids, id, kv interval):
        // consecutive rows, and the rows of consecutive units, mostly share it
        // (kept by the kernel for rows of at most kMaxKB kv blocks, whose
        // scheduler has the registers for it)
        int32_t cache_db = -1, cache_id = 0, cache_lo = 0, cache_hi = -1;
        // Units go out in a serpentine order: round k gives CTA c unit
        // k * G + c for even k and k * G + (G - 1 - c) for odd k (G CTAs). The
        // order runs longest first, so alternating the direction evens out
        // each CTA's total when unit lengths fall steadily (causal rows). A
        // CTA's units still increase, so the first past the end is its last.
        //
        // A unit's entries hold kv blocks relative to a window base. When the
        // unit's kv blocks span more than kMaxKB blocks (rows longer than
        // kMaxKB blocks), it goes out as several segments, one window of
        // kMaxKB blocks each, in kv order; the consumers carry the unit's
        // state from one segment to the next.
        for (int64_t k = 0;; ++k) {
            const int64_t G = gridDim.x;
            const int64_t u64 = k * G + ((k & 1) ? (G - 1 - blockIdx.x) : static_cast<int64_t>(blockIdx.x));
            const int u = u64 < p.num_units ? static_cast<int>(u64) : p.num_units;
            if (u >= p.num_units) {
                const int buf = iter & 1;
                if (!mbar_wait(bar(L::kBarSchedEmpty + buf), ((static_cast<uint32_t>(iter) >> 1) & 1u) ^ 1u,
                               abort_flag))
                    break;
                if (lane == 0) reinterpret_cast<SchedHeader*>(sched_base(buf) + L::kSchedHeader)->T = -1;
                mbar_arrive(bar(L::kBarSchedFull + buf));
                break;
            }
            // longest-first order: highest q-block pair first, then (b, hq)
            const int bh_count = p.B * p.Hq;
            const int pr = p.pairs - 1 - u / (bh_count * p.num_splits);
            const int bh = (u / p.num_splits) % bh_count;
            const int split = u % p.num_splits;
            const int b = bh / p.Hq;
            const int hq = bh % p.Hq;
            const int qb0 = 2 * pr;
            const bool has1 = qb0 + 1 < p.QB;
            // the unit's first buffer
            if (!mbar_wait(bar(L::kBarSchedEmpty + (iter & 1)), ((static_cast<uint32_t>(iter) >> 1) & 1u) ^ 1u,
                           abort_flag))
                break;
            // Each row's document interval [first, last] of kv positions with the
            // row's document id (kv ids are non-decreasing), into the unit's first
            // buffer sb0. Rows in a run usually share one id, so each distinct id
            // is searched once, with a 33-way warp search over the kv ids, and the
            // last search serves the rows that follow with the same id.
            auto doc_intervals = [&](uint8_t* sb0) {
                if (dnf.has_doc && p.has_block_mask) {
                    const int db = dnf.doc_batch > 1 ? b : 0;
                    const int32_t* qd_row = dnf.q_doc + static_cast<int64_t>(db) * p.M;
                    const int32_t* kd_row = dnf.kv_doc + static_cast<int64_t>(db) * p.N;
                    int32_t* dlo = reinterpret_cast<int32_t*>(sb0 + L::kSchedDocLo);
                    int32_t* dhi = reinterpret_cast<int32_t*>(sb0 + L::kSchedDocHi);
#pragma unroll 1
                    for (int r0 = 0; r0 < 256; r0 += 32) {
                        const int64_t q = static_cast<int64_t>(qb0) * 128 + r0 + lane;
                        const bool valid = q < p.M;
                        const int32_t d = valid ? __ldg(qd_row + q) : 0;
                        int lo = 0, hi = -1;
                        bool pending = valid;
                        if (!LONG && pending && db == cache_db && d == cache_id) {
                            lo = cache_lo;
                            hi = cache_hi;
                            pending = false;
                        }
                        unsigned todo;
                        while ((todo = __ballot_sync(0xFFFFFFFFu, pending)) != 0u) {
                            const int32_t x = __shfl_sync(0xFFFFFFFFu, d, __ffs(todo) - 1);
                            const int first = warp_lower_bound(kd_row, p.N, x, lane);
                            const int past = warp_lower_bound(kd_row, p.N, static_cast<int64_t>(x) + 1, lane);
                            if (pending && d == x) {
                                lo = first;
                                hi = past - 1;
                                pending = false;
                            }
                            if constexpr (!LONG) {  // (x and the results are the same in every lane)
                                cache_db = db;
                                cache_id = x;
                                cache_lo = first;
                                cache_hi = past - 1;
                            }
                        }
                        dlo[r0 + lane] = lo;
                        dhi[r0 + lane] = hi;
                    }
                }
            };
            if constexpr (LONG) doc_intervals(sched_base(iter & 1));
            // the two rows' partial and full lists (block mask only): list l is
            // list_at(l), l = 0 partial row0, 1 full row0, 2 partial row1, 3 full row1
            int cnt[4] = {0, 0, 0, 0};
            int64_t row0 = 0;
            auto list_at = [&](int l) -> const int32_t* {
                return ((l & 1) ? p.full_idx : p.kv_idx) + (row0 + (l >> 1)) * p.KB;
            };
            if (p.has_block_mask) {
                const int bb = p.Bm > 1 ? b : 0;
                const int hh = p.Hm > 1 ? hq : 0;
                row0 = (static_cast<int64_t>(bb) * p.Hm + hh) * p.QB + qb0;
                int v = 0;
                if (lane == 0) v = __ldg(p.kv_num + row0);
                if (lane == 1) v = __ldg(p.full_num + row0);
                if (has1 && lane == 2) v = __ldg(p.kv_num + row0 + 1);
                if (has1 && lane == 3) v = __ldg(p.full_num + row0 + 1);
                bool bad = v < 0 || v > p.KB;
                if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) record_status(BSMT_ERR_DEVICE_BOUNDS);
                v = bad ? 0 : v;
#pragma unroll
                for (int l = 0; l < 4; ++l) cnt[l] = __shfl_sync(0xFFFFFFFFu, v, l);
            }
            // Marks bit l of flags[kb - base] for each block kb of list l in
            // [base, base + span).
            auto mark = [&](int base, int span) {
                bool bad = false;
#pragma unroll
                for (int l = 0; l < 4; ++l) {
                    const int32_t* list = list_at(l);
                    for (int j = lane; j < cnt[l]; j += 32) {
                        const int kb = __ldg(list + j);
                        if (kb < 0 || kb >= p.KB) {
                            bad = true;
                        } else if (kb >= base && kb - base < span) {
                            flags[kb - base] |= static_cast<uint8_t>(1u << l);
                        }
                    }
                    __syncwarp();
                }
                if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) record_status(BSMT_ERR_DEVICE_BOUNDS);
            };
            // The unit's windows: kMaxKB blocks each from its first listed block.
            int klo = 0, nwin = 1;
            if (LONG && p.KB > kMaxKB) {
                int khi = p.KB - 1;
                if (p.has_block_mask) {
                    int mn = 0x7FFFFFFF, mx = -1;
#pragma unroll
                    for (int l = 0; l < 4; ++l) {
                        const int32_t* list = list_at(l);
                        for (int j = lane; j < cnt[l]; j += 32) {
                            const int kb = __ldg(list + j);
                            if (kb >= 0 && kb < p.KB) {
                                mn = min(mn, kb);
                                mx = max(mx, kb);
                            }
                        }
                    }
                    mn = __reduce_min_sync(0xFFFFFFFFu, mn);
                    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
                    klo = mx >= 0 ? mn : 0;
                    khi = mx;
                }
                nwin = khi >= klo ? (khi - klo) / kMaxKB + 1 : 1;
            }
            // Split-KV over several windows: the slice [g_lo, g_hi) of the
            // unit's stream needs the stream's length first.
            int g_lo = 0, g_hi = 0x7FFFFFFF;
            if (LONG && p.num_splits > 1 && nwin > 1) {
                int total = p.KB;
                if (p.has_block_mask) {
                    total = 0;
                    for (int w = 0; w < nwin; ++w) {
                        const int base = klo + w * kMaxKB;
                        const int span = min(kMaxKB, p.KB - base);
                        mark(base, span);
                        for (int c = 0; c < span; c += 32) {
                            uint32_t f = 0;
                            if (c + lane < span) {
                                f = flags[c + lane];
                                flags[c + lane] = 0;
                            }
                            total += __popc(__ballot_sync(0xFFFFFFFFu, f != 0));
                        }
                        __syncwarp();
                    }
                }
                g_lo = static_cast<int>((static_cast<int64_t>(total) * split) / p.num_splits);
                g_hi = static_cast<int>((static_cast<int64_t>(total) * (split + 1)) / p.num_splits);
            }
            int g = 0;  // stream entries before this window
            bool ok = true;
            for (int w = 0; w < nwin; ++w, ++iter) {
                const int buf = iter & 1;
                const uint32_t use = static_cast<uint32_t>(iter >> 1);
                if (w > 0 && !mbar_wait(bar(L::kBarSchedEmpty + buf), (use & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t* sb = sched_base(buf);
                SchedHeader* hdr = reinterpret_cast<SchedHeader*>(sb + L::kSchedHeader);
                uint32_t* entries = reinterpret_cast<uint32_t*>(sb + L::kSchedEntries);
                const int base = klo + w * kMaxKB;
                const int span = min(kMaxKB, p.KB - base);
                if (p.has_block_mask) mark(base, span);
                // the union of both rows' blocks in the window, ascending, with
                // tags; a block listed as both partial and full is partial, and
                // the tile crossing N is partial
                int T = 0, n0 = 0, n1 = 0;
                for (int c = 0; c < span; c += 32) {
                    const int kr = c + lane;
                    uint32_t tags = 0;
                    if (kr < span) {
                        if (p.has_block_mask) {
                            const uint32_t f = flags[kr];
                            flags[kr] = 0;
                            if (f & 3u) tags |= kTagIn0 | ((f & 1u) ? kTagPart0 : 0u);
                            if (f & 12u) tags |= kTagIn1 | ((f & 4u) ? kTagPart1 : 0u);
                        } else {
                            tags = kTagIn0 | (has1 ? kTagIn1 : 0u);
                        }
                        if (ragged_kv && base + kr == p.KB - 1) {
                            if (tags & kTagIn0) tags |= kTagPart0;
                            if (tags & kTagIn1) tags |= kTagPart1;
                        }
                    }
                    const unsigned bal = __ballot_sync(0xFFFFFFFFu, tags != 0);
                    if constexpr (LONG) {
                        // keep the stream entries g.. of the split's slice [g_lo, g_hi)
                        const int gi = g + __popc(bal & below);
                        const bool keep = tags != 0 && gi >= g_lo && gi < g_hi;
                        const unsigned kbal = __ballot_sync(0xFFFFFFFFu, keep);
                        if (keep) entries[T + __popc(kbal & below)] = static_cast<uint32_t>(kr) | (tags << 16);
                        T += __popc(kbal);
                        g += __popc(bal);
                        n0 += __popc(__ballot_sync(0xFFFFFFFFu, keep && (tags & kTagIn0)));
                        n1 += __popc(__ballot_sync(0xFFFFFFFFu, keep && (tags & kTagIn1)));
                    } else {
                        if (tags) entries[T + __popc(bal & below)] = static_cast<uint32_t>(kr) | (tags << 16);
                        T += __popc(bal);
                        n0 += __popc(__ballot_sync(0xFFFFFFFFu, (tags & kTagIn0) != 0));
                        n1 += __popc(__ballot_sync(0xFFFFFFFFu, (tags & kTagIn1) != 0));
                    }
                }
                if (p.num_splits > 1 && nwin == 1) {
                    // keep this unit's slice [lo, hi) of the stream, moved to the front
                    // (a chunk is read before it is written, and never overlaps a later
                    // chunk's source)
                    const int lo = static_cast<int>((static_cast<int64_t>(T) * split) / p.num_splits);
                    const int hi = static_cast<int>((static_cast<int64_t>(T) * (split + 1)) / p.num_splits);
                    n0 = 0;
                    n1 = 0;
                    for (int c = 0; c < hi - lo; c += 32) {
                        const bool in = c + lane < hi - lo;
                        const uint32_t e = in ? entries[lo + c + lane] : 0u;
                        __syncwarp();
                        if (in) entries[c + lane] = e;
                        __syncwarp();
                        const uint32_t tags = sched_entry_tags(e);
                        n0 += __popc(__ballot_sync(0xFFFFFFFFu, in && (tags & kTagIn0)));
                        n1 += __popc(__ballot_sync(0xFFFFFFFFu, in && (tags & kTagIn1)));
                    }
                    T = hi - lo;
                }
                if constexpr (!LONG) doc_intervals(sb);
                if (lane == 0) {
                    hdr->T = T;
                    hdr->b = b;
                    hdr->hq = hq;
                    hdr->qb0 = qb0;
                    hdr->split = split;
                    hdr->n0 = n0;
                    hdr->n1 = n1;
                    hdr->kb_base = base;
                    hdr->seg = (w == 0 ? kSegFirst : 0) | (w == nwin - 1 ? kSegLast : 0) | (nwin > 1 ? kSegMany : 0);
                    float slope = 0.f;
                    if (SCORE == kScoreAlibi || SCORE == kScoreSoftcapAlibi || SCORE == kScoreAlibiSoftcap)
                        slope = p.slopes ? __ldg(p.slopes + hq)
                                         : exp2f(-8.0f * static_cast<float>(p.alibi_h0 + hq + 1) /
                                                 static_cast<float>(p.alibi_heads));
                    hdr->slope = slope;
                    if (w == 0) {
                        // Pull this unit's Q tiles into L2 now; they are loaded into
                        // shared memory only when the unit before has finished with
                        // its own.
                        const int zq = b * p.Hq + hq;
                        for (int qq = 0; qq < 2; ++qq) {
                            if ((qq == 0 ? n0 : n1) == 0) continue;
#pragma unroll
                            for (int h = 0; h < D / 64; ++h) tma_prefetch_3d(&tm_q, h * 64, (qb0 + qq) * 128, zq);
                        }
                    }
                }
                __syncwarp();
                mbar_arrive(bar(L::kBarSchedFull + buf));
            }
            if (!ok) break;
        }
    } else if (warp == kWarpLoad) {
        // ================================================= TMA producer warp
        uint32_t kv_pos = 0;  // ring positions used so far
        uint32_t q_uses[2] = {0, 0};
        bool q_loaded[2] = {false, false};  // a unit of several segments: its Q tile i is loaded
        const uint32_t tile_bytes = L::kTileBytes;
        const uint64_t pol_kv = l2_policy_evict_last();
        const uint64_t pol_q = l2_policy_evict_first();
        // Q tile i of q-block qb of head zq, once the unit before is done with the slot
        auto load_q = [&](int i, int qb, int zq) -> bool {
            if (q_uses[i] > 0 && !mbar_wait(bar(L::kBarQEmpty + i), (q_uses[i] - 1) & 1u, abort_flag)) return false;
            ++q_uses[i];
            if (lane == 0) {
                const uint32_t qb_bar = bar(L::kBarQFull + i);
                mbar_arrive_expect_tx(qb_bar, tile_bytes);
                const uint32_t dst = sbase + (i == 0 ? L::kQ0 : L::kQ1);
#pragma unroll
                for (int h = 0; h < D / 64; ++h) tma_load_3d_hint(dst + h * 16384, &tm_q, h * 64, qb * 128, zq, qb_bar, pol_q);
            }
            return true;
        };
        for (int iter = 0;; ++iter) {
            const int buf = iter & 1;
            if (!mbar_wait(bar(L::kBarSchedFull + buf), static_cast<uint32_t>(iter >> 1) & 1u, abort_flag)) break;
            const uint8_t* sb = sched_base(buf);
            const SchedHeader hdr = *reinterpret_cast<const SchedHeader*>(sb + L::kSchedHeader);
            if (hdr.T < 0) break;
            const uint32_t* entries = reinterpret_cast<const uint32_t*>(sb + L::kSchedEntries);
            const int hkv = hdr.hq / p.group;
            const int zq = hdr.b * p.Hq + hdr.hq;
            const int zkv = hdr.b * p.Hkv + hkv;
            bool ok = true;
            // A unit of one segment knows which Q tiles it needs up front; a unit
            // of several loads each Q tile before its first K tile.
            const bool many = LONG && (hdr.seg & kSegMany) != 0;
            if (LONG && (hdr.seg & kSegFirst)) {
                q_loaded[0] = false;
                q_loaded[1] = false;
            }
            if (!many) {
                for (int i = 0; i < 2 && ok; ++i)
                    if ((i == 0 ? hdr.n0 : hdr.n1) > 0) ok = load_q(i, hdr.qb0 + i, zq);
            }
            if (!ok) break;
            for (int n = 0; n < hdr.T && ok; ++n) {
                const uint32_t e = entries[n];
                if (many) {
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        if (ok && ((sched_entry_tags(e) >> i) & 1u) && !q_loaded[i]) {
                            ok = load_q(i, hdr.qb0 + i, zq);
                            q_loaded[i] = true;
                        }
                    }
                    if (!ok) break;
                }
                const int kb = (LONG ? hdr.kb_base : 0) + static_cast<int>(sched_entry_kb(e));
#pragma unroll
                for (int kv = 0; kv < 2; ++kv) {  // 0 = K, 1 = V
                    const uint32_t s = kv_pos % kRing;
                    const uint32_t round = kv_pos / kRing;
                    if (!mbar_wait(bar(L::kBarKvEmpty + s), (round & 1u) ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = bar(L::kBarKvFull + s);
                    if (lane == 0) {
                        mbar_arrive_expect_tx(fb, tile_bytes);
                        const uint32_t dst = sbase + L::kRingBase + s * L::kTileBytes;
#pragma unroll
                        for (int h = 0; h < D / 64; ++h)
                            tma_load_3d_hint(dst + h * 16384, kv == 0 ? &tm_k : &tm_v, h * 64, kb * 128, zkv, fb,
                                             pol_kv);
                    }
                    ++kv_pos;
                }
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::kBarSchedEmpty + buf));
        }
    } else if (warp == kWarpMma || warp == kWarpMma1) {
        // ================================================= MMA issuer warps
        // One warp per q-block of the pair. Each walks the whole entry stream
        // in order; at step n it finishes entry n-1 for its q-block (O += P V
        // once the q-block's P is in TMEM, or a plain release of the V slot if
        // the q-block skips the entry) and starts entry n (S = Q K^T, or a
        // plain release of the K slot). The two issuers hand a token back and
        // forth, q-block 0 first, so the tensor pipe receives whole steps in
        // the fixed order [PV0, S0], [PV1, S1], ... and each q-block's S(n)
        // follows its PV(n-1) at once. Everything a step waits for (its P,
        // the V and K tiles, Q) is waited for before taking the token, while
        // the other issuer is issuing: a single warp issues an MMA in about as
        // long as the tensor core takes to run one, so the issuer's own waits
        // would otherwise leave the tensor pipe idle. Every wait ends: P(n-1)
        // needs only S(n-1), issued at an earlier step; a load waited for at
        // step n needs only slot releases of entries up to n-2; and the token
        // comes back after the other issuer's step, whose waits are of the
        // same kind. The whole warp runs the loop and an elected lane issues.
        const int i = warp == kWarpMma ? 0 : 1;
        constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, kOCols<D>, false, true);
        const uint64_t q_desc = sdesc_sw128(sbase + (i == 0 ? L::kQ0 : L::kQ1), 16, 1024);
        const uint32_t t_s = tm_s[i], t_o = tm_o[i];
        // Entry e of the stream (counted over all units) uses ring positions
        // 2e (K) and 2e+1 (V). Within a unit, a turn finishes entry e-1 and
        // starts entry e. A unit's last entry is finished outside the token
        // order, as soon as its P is stored: the next unit's first S then
        // waits for neither q-block's last tile of the unit before.
        uint32_t e = 0;  // entries started so far
        uint32_t q_uses = 0, pf_waits = 0, tok_waits = 0;
        bool ok = true;
        bool prev_in = false, prev_first = false, prev_last = false;  // entry e-1 for this q-block
        if (i == 1 && lane == 0) mbar_arrive(bar(L::kBarTok + 0));  // q-block 0 goes first
        auto slot_wait = [&](uint32_t pos) {
            return mbar_wait(bar(L::kBarKvFull + pos % kRing), (pos / kRing) & 1u, abort_flag);
        };
        // One step: finish entry e-1 (if has_prev) and start entry e (if has_cur),
        // in a token turn unless it only finishes.
        auto step = [&](bool has_prev, bool has_cur, bool cur_in, bool cur_first, bool cur_last) -> bool {
            const uint32_t kpos = 2u * e;
            const uint32_t vslot = (kpos - 1u) % kRing, kslot = kpos % kRing;
            // waits of this step, before the token
            if (has_prev && has_cur) {
                if (!mbar_wait2(bar(L::kBarKvFull + vslot), ((kpos - 1u) / kRing) & 1u, bar(L::kBarKvFull + kslot),
                                (kpos / kRing) & 1u, abort_flag))
                    return false;
            } else if (!slot_wait(has_prev ? kpos - 1u : kpos)) {
                return false;
            }
            if (has_prev && prev_in) {
                if (!mbar_wait(bar(L::kBarPFull + i), pf_waits & 1u, abort_flag)) return false;
                ++pf_waits;
            }
            if (has_cur && cur_in && cur_first) {  // first tile of its unit: Q
                if (!mbar_wait(bar(L::kBarQFull + i), q_uses & 1u, abort_flag)) return false;
                ++q_uses;
            }
            if (has_cur) {
                if (!mbar_wait(bar(L::kBarTok + i), tok_waits & 1u, abort_flag)) return false;
                ++tok_waits;
            }
            tc_fence_after();
            if (has_prev) {  // finish entry e-1 (V at ring position kpos - 1)
                if (prev_in) {
                    // N's second 64-column block: V's own at D = 128, the ones block at D = 64
                    const uint32_t vaddr = sbase + L::kRingBase + vslot * L::kTileBytes;
                    const uint64_t vd = sdesc_sw128(vaddr, kTcRowSum<D> ? sbase + L::kOnes - vaddr : 16384u, 1024);
                    if (elect_one()) {
                        mma_ts_run8(t_o, t_s, vd, idesc_pv, prev_first ? 0u : 1u);
                        mma_commit(bar(L::kBarKvEmpty + vslot));
                        if (prev_last) mma_commit(bar(L::kBarOFull + i));
                    }
                } else if (elect_one()) {
                    mbar_arrive(bar(L::kBarKvEmpty + vslot));
                }
                __syncwarp();
            }
            if (has_cur) {  // start entry e (K at ring position kpos)
                if (cur_in) {
                    const uint64_t kd = sdesc_sw128(sbase + L::kRingBase + kslot * L::kTileBytes, 16, 1024);
                    if (elect_one()) {
                        mma_ss_run<D / 16>(t_s, q_desc, kd, idesc_s, 0u);
                        mma_commit(bar(L::kBarSFull + i));
                        mma_commit(bar(L::kBarKvEmpty + kslot));
                        if (cur_last) mma_commit(bar(L::kBarQEmpty + i));
                    }
                } else if (elect_one()) {
                    mbar_arrive(bar(L::kBarKvEmpty + kslot));
                }
                __syncwarp();
            }
            if (has_cur && lane == 0) mbar_arrive(bar(L::kBarTok + (i ^ 1)));
            prev_in = has_cur && cur_in;
            prev_first = cur_first;
            prev_last = cur_last;
            if (has_cur) ++e;
            return true;
        };
        // A unit's state carries over its segments: s_done (this q-block's S
        // products so far) and started (an entry has started). In a unit of
        // several segments the q-block's tile count is not known ahead, so its
        // Q slot and O are released at the unit's end instead of at its last
        // tile.
        int s_done = 0;
        bool started = false;
        for (int iter = 0; ok; ++iter) {
            const int buf = iter & 1;
            if (!mbar_wait(bar(L::kBarSchedFull + buf), static_cast<uint32_t>(iter >> 1) & 1u, abort_flag)) break;
            const uint8_t* sb = sched_base(buf);
            const SchedHeader hdr = *reinterpret_cast<const SchedHeader*>(sb + L::kSchedHeader);
            if (hdr.T < 0) break;
            const uint32_t* entries = reinterpret_cast<const uint32_t*>(sb + L::kSchedEntries);
            const int ni = i == 0 ? hdr.n0 : hdr.n1;
            const bool many = LONG && (hdr.seg & kSegMany) != 0;
            if (!LONG || (hdr.seg & kSegFirst)) {
                s_done = 0;
                started = false;
            }
            for (int n = 0; n < hdr.T && ok; ++n) {
                const bool cur_in = (sched_entry_tags(entries[n]) >> i) & 1u;
                const bool cur_first = cur_in && s_done == 0;
                if (cur_in) ++s_done;
                ok = step(LONG ? started : n > 0, true, cur_in, cur_first, !many && cur_in && s_done == ni);
                started = true;
            }
            if (ok && (LONG ? (hdr.seg & kSegLast) != 0 : hdr.T > 0)) {
                if (!LONG || started) ok = step(true, false, false, false, false);  // finish the unit's last entry
                if (ok && many && s_done > 0) {
                    if (elect_one()) {
                        mma_commit(bar(L::kBarQEmpty + i));
                        mma_commit(bar(L::kBarOFull + i));
                    }
                    __syncwarp();
                }
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::kBarSchedEmpty + buf));
        }
        // every MMA of this warp must finish before TMEM is freed
        if (elect_one()) mma_commit(bar(L::kBarDone + i));
        __syncwarp();
        mbar_wait(bar(L::kBarDone + i), 0, abort_flag);
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 216;\n" ::: "memory");
        // ================================================= softmax warpgroups
        const int i = warp >> 2;              // q-block of the pair
        const int r = threadIdx.x & 127;      // row within the q-block
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_s = tm_s[i] + lane_base;
        const uint32_t t_o = tm_o[i] + lane_base;
        uint32_t s_waits = 0, o_waits = 0;
        bool ok = true;
        for (int iter = 0; ok; ++iter) {
            int buf = iter & 1;
            if (!mbar_wait(bar(L::kBarSchedFull + buf), static_cast<uint32_t>(iter >> 1) & 1u, abort_flag)) break;
            const uint8_t* sb = sched_base(buf);
            SchedHeader hdr = *reinterpret_cast<const SchedHeader*>(sb + L::kSchedHeader);
            if (hdr.T < 0) break;
            const int ni = i == 0 ? hdr.n0 : hdr.n1;  // this q-block's tiles (one-segment units)
            const int qb = hdr.qb0 + i;
            const int q = qb * 128 + r;
            const bool row_valid = qb < p.QB && q < p.M;
            int64_t row_ds = 0, row_de = p.N - 1;
            if (dnf.has_doc && p.has_block_mask) {
                row_ds = reinterpret_cast<const int32_t*>(sb + L::kSchedDocLo)[i * 128 + r];
                row_de = reinterpret_cast<const int32_t*>(sb + L::kSchedDocHi)[i * 128 + r];
            }
            const float sl2 = hdr.slope * kLog2e;
            // This row's allowed kv interval per mask alternative (document
            // leaves included), computed once per unit. Partial tiles then only
            // turn intervals into bit words. Empty intervals are stored as [1, 0].
            const bool fast_mask = p.has_block_mask && dnf.n_terms <= kRowTerms;
            int iv_lo[kRowTerms], iv_hi[kRowTerms];
#pragma unroll
            for (int t = 0; t < kRowTerms; ++t) {
                iv_lo[t] = 1;
                iv_hi[t] = 0;
                if (fast_mask && t < dnf.n_terms) {
                    int64_t lo, hi;
                    term_interval(dnf, t, q, 0, p.N - 1, row_ds, row_de, lo, hi);
                    if (hi >= lo) {  // then both lie in [0, N - 1]
                        iv_lo[t] = static_cast<int>(lo);
                        iv_hi[t] = static_cast<int>(hi);
                    }
                }
            }
            float m_ref = -INFINITY;
            float l_sum = 0.f;
            int processed = 0;
            // The unit's segments, in order: the row state above carries over;
            // every buffer but the last is released as soon as its entries are
            // done.
            for (;;) {
                const uint32_t* entries = reinterpret_cast<const uint32_t*>(sb + L::kSchedEntries);
                for (int n = 0; n < hdr.T && ok; ++n) {
                    const uint32_t e = entries[n];
                    const uint32_t tags = sched_entry_tags(e);
                    if (!((tags >> i) & 1u)) continue;  // not this q-block's tile
                    const int kb = (LONG ? hdr.kb_base : 0) + static_cast<int>(sched_entry_kb(e));
                    const bool partial = (tags >> (2 + i)) & 1u;
                    if (!mbar_wait(bar(L::kBarSFull + i), s_waits & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    ++s_waits;
                    __syncwarp();  // tcgen05.ld/st are warp-collective: reconverge after the waits
                    tc_fence_after();
                    float x[128];
                    {
                        uint32_t* xr = reinterpret_cast<uint32_t*>(x);
                        tmem_ld32(t_s + 0, *reinterpret_cast<uint32_t(*)[32]>(xr + 0));
                        tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(xr + 32));
                        tmem_ld32(t_s + 64, *reinterpret_cast<uint32_t(*)[32]>(xr + 64));
                        tmem_ld32(t_s + 96, *reinterpret_cast<uint32_t(*)[32]>(xr + 96));
                        tc_wait_ld();
                    }
                    // score_mod on every visited tile. Other modes move to base-2
                    // units here; the plain mode keeps raw scores and folds
                    // scale * log2(e) into the exponent's FFMA below.
                    // Column pairs go through the packed f32x2 FMA pipe (the same
                    // roundings as one column at a time).
                    if constexpr (SCORE != kScoreNone) {
                        const float tile_bias = sl2 * static_cast<float>(kb * 128 - q);
                        const float tile_pos = static_cast<float>(kb * 128 - q);  // exact below 2^24
                        const float u_mul = p.scale * p.inv_cap;
                        const float capl2 = p.cap * kLog2e;
#pragma unroll
                        for (int j = 0; j < 128; j += 2) {
                            const float j0 = static_cast<float>(j), j1 = static_cast<float>(j + 1);
                            if constexpr (SCORE == kScoreSoftcap) {
                                float u0, u1;
                                mul2(u0, u1, x[j], x[j + 1], u_mul, u_mul);
                                mul2(x[j], x[j + 1], capl2, capl2, tanh_approx(u0), tanh_approx(u1));
                            } else if constexpr (SCORE == kScoreAlibi) {
                                float c0, c1;
                                fma2(c0, c1, sl2, sl2, j0, j1, tile_bias, tile_bias);
                                fma2(x[j], x[j + 1], x[j], x[j + 1], p.scale_log2, p.scale_log2, c0, c1);
                            } else if constexpr (SCORE == kScoreSoftcapAlibi) {
                                float u0, u1, c0, c1;
                                mul2(u0, u1, x[j], x[j + 1], u_mul, u_mul);
                                fma2(c0, c1, sl2, sl2, j0, j1, tile_bias, tile_bias);
                                fma2(x[j], x[j + 1], capl2, capl2, tanh_approx(u0), tanh_approx(u1), c0, c1);
                            } else {  // ALiBi, then the soft-cap
                                float r0, r1, b0, b1, t0, t1;
                                add2(r0, r1, tile_pos, tile_pos, j0, j1);       // kv - q, exact
                                mul2(b0, b1, hdr.slope, hdr.slope, r0, r1);
                                fma2(t0, t1, x[j], x[j + 1], p.scale, p.scale, b0, b1);
                                mul2(t0, t1, t0, t1, p.inv_cap, p.inv_cap);
                                mul2(x[j], x[j + 1], capl2, capl2, tanh_approx(t0), tanh_approx(t1));
                            }
                        }
                    }
                    // mask_mod on partial tiles only
                    if (partial) {
                        const int64_t c0 = static_cast<int64_t>(kb) * 128;
                        const int64_t c1 = (c0 + 127 < p.N - 1) ? c0 + 127 : p.N - 1;
                        const int64_t ds = row_ds, de = row_de;
                        uint32_t w[4] = {0u, 0u, 0u, 0u};
                        if (fast_mask) {
                            const int tc0 = static_cast<int>(c0), tc1 = static_cast<int>(c1);
#pragma unroll
                            for (int t = 0; t < kRowTerms; ++t) {
                                if (t >= dnf.n_terms) break;  // uniform: the mask's own term count
                                int lo = iv_lo[t], hi = iv_hi[t];
                                lo = (lo > tc0 ? lo : tc0) - tc0;
                                hi = (hi < tc1 ? hi : tc1) - tc0;
#pragma unroll
                                for (int k = 0; k < 4; ++k) w[k] |= range_bits32(lo - 32 * k, hi - 32 * k);
                            }
                        } else if (p.has_block_mask) {
                            for (int t = 0; t < dnf.n_terms; ++t) {
                                int64_t lo, hi;
                                term_interval(dnf, t, q, c0, c1, ds, de, lo, hi);
#pragma unroll
                                for (int k = 0; k < 4; ++k) w[k] |= range_bits(lo, hi, c0 + 32 * k);
                            }
                        } else {
#pragma unroll
                            for (int k = 0; k < 4; ++k) w[k] = range_bits(c0, c1, c0 + 32 * k);
                        }
#pragma unroll
                        for (int j = 0; j < 128; ++j)
                            if (!((w[j >> 5] >> (j & 31)) & 1u)) x[j] = -INFINITY;
                    }
                    // row max: eight independent chains of three-input max
                    float mx[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        mx[k] = x[k];
#pragma unroll
                        for (int j = 8; j + 16 <= 128; j += 16) mx[k] = fmax3(mx[k], x[j + k], x[j + 8 + k]);
                        mx[k] = fmaxf(mx[k], x[120 + k]);
                    }
                    constexpr bool kRaw = SCORE == kScoreNone;
                    const float cmul = kRaw ? p.scale_log2 : 1.f;  // scale > 0, so max commutes with it
                    float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
                    if constexpr (kRaw) mt *= cmul;
                    // lazy reference update
                    bool need_rescale = false;
                    float alpha = 1.f;
                    if (mt > m_ref + kRescaleThreshold) {  // false while mt is -inf
                        if (m_ref != -INFINITY) {
                            alpha = ex2_approx(m_ref - mt);
                            need_rescale = processed > 0;
                        }
                        l_sum *= alpha;
                        m_ref = mt;
                    }
                    const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
                    // P = 2^(x * cmul - m). The first kEmuCols columns of every
                    // 32-column chunk use the FMA-pipe exp2, the rest MUFU ex2.
                    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t pk[16];
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) {
                            const int j = 32 * c + 2 * jj;
                            float a0, a1, p0, p1;
                            fma2(a0, a1, x[j], x[j + 1], cmul, cmul, neg_m, neg_m);
                            if (2 * jj < kEmuCols<D>) {
                                exp2_poly2(p0, p1, a0, a1);
                            } else {
                                p0 = ex2_approx(a0);
                                p1 = ex2_approx(a1);
                            }
                            if constexpr (!kTcRowSum<D>)
                                add2(acc[2 * (jj & 3)], acc[2 * (jj & 3) + 1], acc[2 * (jj & 3)], acc[2 * (jj & 3) + 1],
                                     p0, p1);
                            pk[jj] = pack_bf16x2(p0, p1);
                        }
                        tmem_st16(t_s + 16 * c, pk);
                    }
                    // a row whose every element in this tile is masked adds nothing
                    // (the FMA-pipe exp2 returns 2^-125 rather than 0 for -inf). With the
                    // tensor core's row sum such a row adds 2^-125 per column against its
                    // reference, which stays negligible; a row that never has an allowed
                    // key keeps m_ref = -inf and the epilogue treats it as empty.
                    if (!kTcRowSum<D> && mt != -INFINITY)
                        l_sum += ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
                    // O rescale after P is out of registers (lower register peak); with
                    // the tensor core's row sum, l (column D) is rescaled with O
                    if (__any_sync(0xFFFFFFFFu, need_rescale)) {
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t o[32];
                            tmem_ld32(t_o + 32 * c, o);
                            tc_wait_ld();
#pragma unroll
                            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                            tmem_st32(t_o + 32 * c, o);
                        }
                        if constexpr (kTcRowSum<D>) {
                            uint32_t o[16];
                            tmem_ld16(t_o + D, o);
                            tc_wait_ld();
#pragma unroll
                            for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                            tmem_st16(t_o + D, o);
                        }
                    }
                    tc_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(L::kBarPFull + i));
                    ++processed;
                }
                if (!ok || !LONG || (hdr.seg & kSegLast)) break;
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(L::kBarSchedEmpty + buf));
                ++iter;
                buf = iter & 1;
                if (!mbar_wait(bar(L::kBarSchedFull + buf), static_cast<uint32_t>(iter >> 1) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                sb = sched_base(buf);
                hdr = *reinterpret_cast<const SchedHeader*>(sb + L::kSchedHeader);
            }
            if (!ok) break;
            // epilogue: out = O / l, lse = ln2 * (m + log2 l)
            __nv_bfloat16* orow = p.out + (static_cast<int64_t>(hdr.b) * p.Hq + hdr.hq) * p.out_sbh + q * p.out_ss;
            if constexpr (kTcRowSum<D>) {
                // l is O's column D, complete once the unit's last PV is (it is
                // read again after the O-full wait below; this read only fixes
                // the row's empty case early for the lse)
                l_sum = 0.f;
                if ((LONG ? processed : ni) > 0) {
                    if (!mbar_wait(bar(L::kBarOFull + i), o_waits & 1u, abort_flag)) break;
                    __syncwarp();
                    tc_fence_after();
                    l_sum = __uint_as_float(tmem_ld1(t_o + D));
                    tc_wait_ld();
                }
                if (m_ref == -INFINITY) l_sum = 0.f;  // no allowed key in the row
            }
            const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
            const float row_lse = [&] {
                const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
                return l_sum > 0.f ? (m_use + __log2f(l_sum)) * kLn2 : -INFINITY;
            }();
            if (p.num_splits > 1) {
                // split-KV: this slice's O / l in fp32 and its lse, to the workspace
                const int64_t wrow = (static_cast<int64_t>(hdr.split) * p.B * p.Hq +
                                      static_cast<int64_t>(hdr.b) * p.Hq + hdr.hq) * p.M + q;
                float4* dst = reinterpret_cast<float4*>(p.ws_o + wrow * D);
                if ((LONG ? processed : ni) > 0) {
                    if (!mbar_wait(bar(L::kBarOFull + i), o_waits & 1u, abort_flag)) break;
                    ++o_waits;
                    __syncwarp();
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(t_o + 32 * c, o);
                        tc_wait_ld();
                        if (row_valid) {
#pragma unroll
                            for (int v = 0; v < 8; ++v)
                                dst[8 * c + v] = make_float4(__uint_as_float(o[4 * v]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                                                             __uint_as_float(o[4 * v + 2]) * inv_l, __uint_as_float(o[4 * v + 3]) * inv_l);
                        }
                    }
                    tc_fence_before();
                } else if (row_valid) {
#pragma unroll
                    for (int v = 0; v < D / 4; ++v) dst[v] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                if (row_valid) p.ws_lse[wrow] = row_lse;
            } else if ((LONG ? processed : ni) > 0) {
                if (!mbar_wait(bar(L::kBarOFull + i), o_waits & 1u, abort_flag)) break;
                ++o_waits;
                __syncwarp();
                tc_fence_after();
                // Each warp writes its 32 rows chunk by chunk (32 columns, 64 bytes a
                // row) into its staging block and TMA stores the block: coalesced
                // writes, and rows past M are clipped by the tensor map.
                const uint32_t stage = sbase + L::kStage + static_cast<uint32_t>(warp) * L::kStageBytes;
                const int y0 = qb * 128 + (warp & 3) * 32;
                const int z = hdr.b * p.Hq + hdr.hq;
                uint32_t o[D];
#pragma unroll
                for (int c = 0; c < D / 32; ++c) tmem_ld32(t_o + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(o + 32 * c));
                tc_wait_ld();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        pk[j] = pack_bf16x2(__uint_as_float(o[32 * c + 2 * j]) * inv_l,
                                            __uint_as_float(o[32 * c + 2 * j + 1]) * inv_l);
                    if (lane == 0) bulk_wait_group_read0();  // the previous block has been read
                    __syncwarp();
                    // 64-byte swizzle: 16-byte chunk k of row r sits at chunk k ^ ((r >> 1) & 3)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        st_shared_v4(stage + static_cast<uint32_t>(lane) * 64u +
                                         static_cast<uint32_t>((k ^ ((lane >> 1) & 3)) * 16),
                                     pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && y0 < p.M) {  // (a block wholly past M stores nothing)
                        tma_store_3d(&tm_out, stage, 32 * c, y0, z);
                        bulk_commit_group();
                    }
                }
                tc_fence_before();
            } else if (row_valid) {
                uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
                for (int v = 0; v < D / 8; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
            }
            if (row_valid && p.num_splits == 1) p.lse[(static_cast<int64_t>(hdr.b) * p.Hq + hdr.hq) * p.M + q] = row_lse;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::kBarSchedEmpty + buf));
        }
        if (lane == 0) bulk_wait_group0();  // staged out blocks are written before the CTA ends
        __syncwarp();
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Merges the split-KV slices of every row: with lse_s the slices' natural
// log-sum-exps and O_s their normalised outputs,
//   lse = log sum_s exp(lse_s),  out = sum_s exp(lse_s - lse) O_s,
// which is the attention over the union of the slices. A row no slice
// reaches keeps out = 0 and lse = -inf. One warp per row; lane l holds
// columns [l * D/32, (l + 1) * D/32).
template <int D>
__global__ void __launch_bounds__(256) splitkv_combine_kernel(const float* ws_o, const float* ws_lse, int splits,
                                                              int64_t rows, int64_t M, int64_t out_sbh,
                                                              int64_t out_ss, __nv_bfloat16* out, float* lse) {
    constexpr int kPer = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    float m = -INFINITY;
    for (int s = 0; s < splits; ++s) m = fmaxf(m, __ldg(ws_lse + s * rows + row));
    float acc[kPer];
#pragma unroll
    for (int c = 0; c < kPer; ++c) acc[c] = 0.f;
    float total = 0.f;
    if (m != -INFINITY) {
        for (int s = 0; s < splits; ++s) {
            const float ls = __ldg(ws_lse + s * rows + row);
            if (ls == -INFINITY) continue;
            const float w = expf(ls - m);
            total += w;
            const float* o = ws_o + (s * rows + row) * D + lane * kPer;
#pragma unroll
            for (int c = 0; c < kPer; ++c) acc[c] = fmaf(w, __ldg(o + c), acc[c]);
        }
    }
    const float inv = total > 0.f ? 1.f / total : 0.f;
    uint32_t pk[kPer / 2];
#pragma unroll
    for (int c = 0; c < kPer / 2; ++c) pk[c] = pack_bf16x2(acc[2 * c] * inv, acc[2 * c + 1] * inv);
    uint32_t* dst = reinterpret_cast<uint32_t*>(out + (row / M) * out_sbh + (row % M) * out_ss + lane * kPer);
#pragma unroll
    for (int c = 0; c < kPer / 2; ++c) dst[c] = pk[c];
    if (lane == 0) lse[row] = total > 0.f ? m + logf(total) : -INFINITY;
}

}  // namespace bsmt
