// Block-sparse masked attention backward for sm_100a (tcgen05 + TMEM + TMA).
//
// The gradients of sum(out * dout) with respect to q, k and v, for the
// forward of attn_fwd.cuh. The structure follows the tensorplay.nn.attention
// page (BlockMask "Details" items 3-4): dK and dV walk the mask along the
// query axis, using the q-side lists (q_num_blocks / q_indices and their full
// counterparts). dQ walks it along the key axis, using the kv-side lists as
// the forward does. Tiles that the lists leave out add nothing. mask_mod runs
// on PARTIAL tiles only; score_mod and its derivative run on every visited
// tile.
//
// With s = scale * q.k, z = score_mod(s), P = exp(z - lse) (lse from the
// forward), dP = dO V^T and delta = rowsum(dO * out):
//   dS = P * (dP - delta) * dz/ds,  dV = P^T dO,  dK = scale * dS^T Q,
//   dQ = scale * dS K.
// One kernel template serves both directions (flag KVSIDE):
//   KVSIDE: a unit is (b, hkv, kv-block). K and V stay in shared memory while
//     the Q and dO tiles stream in: every q-block listed for the kv-block, for
//     every query head of the GQA group. Products are taken transposed, with
//     one kv row per TMEM lane:
//     S^T = K Q^T, dP^T = V dO^T, dV += P^T dO, dK += dS^T Q.
//   !KVSIDE: a unit is (b, hq, q-block). Q and dO stay; K and V of the listed
//     kv-blocks stream in: S = Q K^T, dP = dO V^T, dQ += dS K.
// dQ has its own kernel, so it needs neither an fp32 accumulator in global
// memory nor atomics, and the result does not depend on scheduling.
//
// Pipeline. Each entry (one streamed 128-row tile pair) has one S and one
// dP buffer in TMEM, written by 128 x 128 products. The softmax warps work in
// two phases per entry: the P phase reads S and writes P (bf16, for dV), the
// dS phase reads dP and writes dS; P * dz/ds stays in registers between them.
// The MMA warp issues, for the dk/dv kernel,
//   S(n) dP(n) | dV(n) S(n+1) | dK(n) dP(n+1) | dV(n+1) S(n+2) | ...
// waiting for the P phase of n before dV(n) and for the dS phase of n before
// dK(n). So the P phase of n+1 runs while the tensor core does dK(n) and
// dP(n+1), and the dS phase while it does dV(n+1) and S(n+2). The dq kernel
// issues S(n) dP(n) | S(n+1) | dQ(n) dP(n+1) | ... the same way. MMAs issued
// by one thread run in order, so S(n+1) overwrites S (and P) only after dV(n)
// has read P, and dP(n+1) overwrites dP (and dS) only after dK(n) or dQ(n).
//
// Persistent CTAs, one per SM (every CTA takes all 512 TMEM columns), take
// units from a work counter in the workspace. 384 threads:
//   warps 0-3  columns 0-63 of each entry (thread = TMEM lane = tile row)
//   warps 4-7  columns 64-127
//   warp 8     loads tiles with TMA (the next unit's K/V or Q/dO as soon as
//              the current unit's last S and dP are issued)
//   warp 9     allocates TMEM and issues the MMAs (one elected lane)
//   warp 10    scheduler: takes the next unit and builds its entry list in
//              the other of two buffers
//   warp 11    idle; it completes the third warpgroup, whose registers
//              setmaxnreg hands to the two softmax warpgroups
// The epilogue reads the accumulators in 64-column batches, storing each, and
// releases them once the last batch is in registers, so the next unit's
// products overlap the rest of the previous unit's stores.
// TMEM columns: S [0,128), dP [128,256), acc0 [256, 256+D) (dV or dQ), acc1
// [256+D, 256+2D) (dK). Warpgroup g writes its P and dS as bf16 pairs over
// the first 32 of its own 64 columns of S and dP, so the accumulating
// products read their A operand as two runs of K = 64: columns 0-31 and
// 64-95.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "attn_fwd.cuh"
#include "mask_dnf.cuh"
#include "ptx.cuh"

namespace bsmt {

struct BwdParams {
    int32_t B, Hq, Hkv, M, N, QB, KB, group;
    int32_t Bm, Hm, has_block_mask;
    // kv-side lists (dq kernel) or q-side lists (dk/dv kernel): rows
    // [Bm, Hm, list_rows], each list list_len entries long
    const int32_t* num;
    const int32_t* idx;
    const int32_t* full_num;
    const int32_t* full_idx;
    int32_t list_rows, list_len;
    float scale, scale_log2, cap, inv_cap;
    const float* slopes;  // ALiBi slopes [Hq] or null (default 2^(-8(h0+h+1)/Ht))
    int32_t alibi_h0, alibi_heads;  // h0 and Ht of the default slopes
    // (-lse * log2(e), -delta) per query row, padded to whole q-blocks:
    // [B*Hq][QB*128]. The first is -inf for padding rows and rows with no
    // key, so that P = 2^(z2 - lse2) = 0 there.
    const float2* ld;
    __nv_bfloat16* g0;  // dq (dq kernel) or dk [B, Hkv, N, D]
    __nv_bfloat16* g1;  // dv [B, Hkv, N, D]
    // Element strides of the row-major tensors: row i of head bh of q, out,
    // dout and dq starts at bh * q_sbh + i * q_ss; of k, v, dk and dv at
    // bh * kv_sbh + i * kv_ss. (S*D, D) for [B, H, S, D]; (D, H*D) for a
    // packed [S, H, D] with B = 1.
    int64_t q_sbh, q_ss, kv_sbh, kv_ss;
    int32_t num_units;
    int32_t* next_unit;  // work counter, zero at launch (the prep kernel clears it)
};

constexpr int kBwdThreads = 384;
constexpr int kBwdWarpLoad = 8;
constexpr int kBwdWarpMma = 9;
constexpr int kBwdWarpSched = 10;
constexpr int kBwdMaxEntries = 2048;  // entries of one unit (list length x GQA group)
constexpr uint32_t kBwdPartial = 0x80000000u;
// Columns of every 32-column chunk of a full tile whose 2^x the P phase takes
// on the FMA pipe (exp2_poly2) instead of MUFU. 8 measured faster than 16 on
// B200 (the phase is bound by latency more than by MUFU).
constexpr int kBwdEmuCols = 8;

// A scheduled unit in shared memory (two buffers, filled by the scheduler warp).
struct BwdUnit {
    int32_t T;  // entries of this buffer; -1 ends the work
    int32_t b, hq, hkv, blk;
    // LONG kernels: the unit's entries and the first of this buffer's. A unit
    // of more than kBwdMaxEntries entries goes out in several buffers
    // (segments), every one full but the last.
    int32_t total, off;
};

template <int D>
struct BwdSmem {
    static constexpr int kTile = 128 * D * 2;
    static constexpr int kF0 = 0;                   // K (dk/dv) or Q (dq)
    static constexpr int kF1 = kTile;               // V or dO
    static constexpr int kStage = 2 * kTile;        // stage s: T0 at kStage + 2 s kTile, T1 one tile further
    static constexpr int kLd = kStage + 4 * kTile;  // stage s: 128 float2 (-lse2, -delta) at kLd + 1024 s
    static constexpr int kList = kLd + 2048;        // unit buffer u: entries at kList + u * kListBytes
    static constexpr int kListBytes = 4 * kBwdMaxEntries;
    static constexpr int kHdr = kList + 2 * kListBytes;  // BwdUnit[2], 32 bytes each
    static constexpr int kFlags = kHdr + 64;
    static constexpr int kBars = kFlags + kBwdMaxEntries;
    static constexpr int kBarFixedFull = 0, kBarFixedEmpty = 1, kBarTFull = 2, kBarTEmpty = 4, kBarSFull = 6,
                         kBarDpFull = 7, kBarPFull = 8, kBarDsFull = 9, kBarAccFull = 10, kBarAccEmpty = 11,
                         kBarListFull = 12, kBarListEmpty = 14, kBarDone = 16, kNumBars = 17;
    static constexpr int kTmemSlot = kBars + 8 * kNumBars;
    static constexpr int kAbort = kTmemSlot + 4;
    static constexpr int kTotal = kAbort + 4;
    // never less than 120 KB, so that a second CTA cannot share the SM (and
    // wait in tcgen05.alloc for the TMEM the first one holds)
    static constexpr int kAlloc = (kTotal + 1024 > 120 * 1024) ? kTotal + 1024 : 120 * 1024;
    static_assert(kAlloc <= 227 * 1024, "shared memory layout exceeds one CTA's limit");
};

__device__ __forceinline__ float2 mul2f(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2f(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fma2f(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// ALiBi constants of one warpgroup's 64 columns of an entry. Column j has
// kv_idx - q_idx = dkv0 + step * j (step = -1 on the dk/dv side, where
// columns are queries; +1 on the dq side).
struct BwdCols {
    float bias0, bstep;  // ALiBi bias of column 0 and its change per column (log2 units;
                         // natural units when ALiBi comes before the soft-cap)
};

// P phase of one 32-column chunk, two columns at a time on the packed f32x2
// pipe. x: raw q.k; nl: -lse2 of each column (dk/dv side, from shared memory
// as float4 (nl, nd) pairs) or of the row (dq side). For the score mods, with
// s = scale * x:
//   none         z2 = log2e * s
//   soft-cap     t = tanh(s / cap), z2 = cap * log2e * t, dz/ds = 1 - t^2
//   ALiBi        z2 = log2e * (s + slope * (kv - q))
//   both orders  the compositions of the two
// P = 2^(z2 - lse2), masked to 0 outside w (MASKED only). pk gets P as bf16
// pairs; pg keeps P * dz/ds in fp32 for the dS phase. On unmasked chunks the
// first 8 columns take 2^x on the FMA pipe (exp2_poly2), the rest on MUFU:
// the P phase is the one that has to fit in the shadow of two products.
template <int SCORE, bool KVSIDE, bool MASKED>
__device__ __forceinline__ void bwd_p_chunk(const BwdParams& p, const float* x, const float4* ld4, float2 nl_row,
                                            const BwdCols& hb, int c0, uint32_t w, float* pg, uint32_t (&pk)[16]) {
    const float2 s2 = make_float2(p.scale_log2, p.scale_log2);
    const float2 c1 = make_float2(p.scale * p.inv_cap, p.scale * p.inv_cap);
    const float2 c2 = make_float2(p.cap * kLog2e, p.cap * kLog2e);
    const float2 one = make_float2(1.f, 1.f);
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
        const int j = c0 + 2 * jj;
        float2 nl = nl_row;
        if constexpr (KVSIDE) {
            const float4 t = ld4[j >> 1];
            nl = make_float2(t.x, t.z);
        }
        const float2 X = make_float2(x[j], x[j + 1]);
        float2 A, G = one;
        if constexpr (SCORE == kScoreNone) {
            A = fma2f(X, s2, nl);
        } else if constexpr (SCORE == kScoreSoftcap) {
            const float2 u = mul2f(X, c1);
            const float2 t = make_float2(tanh_approx(u.x), tanh_approx(u.y));
            A = fma2f(c2, t, nl);
            G = fma2f(make_float2(-t.x, -t.y), t, one);
        } else if constexpr (SCORE == kScoreAlibi) {
            const float2 bias = fma2f(make_float2(static_cast<float>(j), static_cast<float>(j + 1)),
                                      make_float2(hb.bstep, hb.bstep), make_float2(hb.bias0, hb.bias0));
            A = fma2f(X, s2, add2f(bias, nl));
        } else if constexpr (SCORE == kScoreSoftcapAlibi) {
            const float2 bias = fma2f(make_float2(static_cast<float>(j), static_cast<float>(j + 1)),
                                      make_float2(hb.bstep, hb.bstep), make_float2(hb.bias0, hb.bias0));
            const float2 u = mul2f(X, c1);
            const float2 t = make_float2(tanh_approx(u.x), tanh_approx(u.y));
            A = fma2f(c2, t, add2f(bias, nl));
            G = fma2f(make_float2(-t.x, -t.y), t, one);
        } else {  // ALiBi, then soft-cap: bias in natural units, inside the tanh
            const float2 bias = fma2f(make_float2(static_cast<float>(j), static_cast<float>(j + 1)),
                                      make_float2(hb.bstep, hb.bstep), make_float2(hb.bias0, hb.bias0));
            const float2 u = mul2f(fma2f(X, make_float2(p.scale, p.scale), bias),
                                   make_float2(p.inv_cap, p.inv_cap));
            const float2 t = make_float2(tanh_approx(u.x), tanh_approx(u.y));
            A = fma2f(c2, t, nl);
            G = fma2f(make_float2(-t.x, -t.y), t, one);
        }
        float2 P;
        if constexpr (MASKED) {
            if (!((w >> (2 * jj)) & 1u)) A.x = -INFINITY;
            if (!((w >> (2 * jj + 1)) & 1u)) A.y = -INFINITY;
            P = make_float2(ex2_approx(A.x), ex2_approx(A.y));
        } else if (2 * jj < kBwdEmuCols) {
            // (an A of -inf only comes from rows past the end of the sequence
            // here, whose dO and dP rows are zero; 2^-125 there adds nothing)
            exp2_poly2(P.x, P.y, A.x, A.y);
        } else {
            P = make_float2(ex2_approx(A.x), ex2_approx(A.y));
        }
        pk[jj] = pack_bf16x2(P.x, P.y);
        if constexpr (SCORE == kScoreSoftcap || SCORE == kScoreSoftcapAlibi || SCORE == kScoreAlibiSoftcap)
            P = mul2f(P, G);
        pg[j] = P.x;
        pg[j + 1] = P.y;
    }
}

// dS phase of one 32-column chunk: dS = (P dz/ds) * (dP - delta), as bf16
// pairs. nd: -delta of each column (dk/dv side) or of the row (dq side).
template <bool KVSIDE>
__device__ __forceinline__ void bwd_ds_chunk(const float* dp, const float4* ld4, float2 nd_row, const float* pg,
                                             int c0, uint32_t (&dk)[16]) {
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
        const int j = c0 + 2 * jj;
        float2 nd = nd_row;
        if constexpr (KVSIDE) {
            const float4 t = ld4[j >> 1];
            nd = make_float2(t.y, t.w);
        }
        const float2 T = mul2f(add2f(make_float2(dp[j], dp[j + 1]), nd), make_float2(pg[j], pg[j + 1]));
        dk[jj] = pack_bf16x2(T.x, T.y);
    }
}

// The q interval [lo, hi] of term t for a fixed key kv, within [0, M - 1]
// (document leaves excluded): each leaf of mask_dnf.cuh read along the other
// axis,
//   CAUSAL kv <= q             -> q >= kv
//   WINDOW q - kv < W          -> q <= kv + W - 1
//   PREFIX_LM kv < P or q >= kv -> every q when kv < P, else q >= kv
//   SINK kv < S                -> every q when kv < S, else none
__device__ __forceinline__ void term_q_interval(const MaskDnf& m, int t, int64_t kv, int64_t M, int64_t& lo,
                                                int64_t& hi) {
    const DnfTerm& tm = m.terms[t];
    lo = 0;
    hi = M - 1;
    if (tm.flags & kTermCausal) lo = lo > kv ? lo : kv;
    if (tm.flags & kTermWindow) {
        const int64_t h = kv + static_cast<int64_t>(tm.w) - 1;
        hi = hi < h ? hi : h;
    }
    if ((tm.flags & kTermPrefix) && kv >= static_cast<int64_t>(tm.pf)) lo = lo > kv ? lo : kv;
    if ((tm.flags & kTermSink) && kv >= static_cast<int64_t>(tm.s)) hi = -1;
}

// (-lse2, -delta) per padded query row: lse2 = lse * log2(e) (+inf where lse
// is -inf and for rows past M, so that P = 0 there), delta = sum_d out * dout
// in fp32 (row i of head bh of out and dout at bh * sbh + i * ss; lse is
// [B*Hq, M]); it also zeroes the two backward kernels' work counters. A row is
// read by D/8 lanes, 16 bytes of out and of dout each; a
// warp covers kRowsPerWarp rows with all its loads issued before the sums,
// so that enough bytes are in flight to keep HBM busy.
constexpr int kPrepRowsPerWarp = 8;

template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* out, const __nv_bfloat16* dout,
                                                       const float* lse, int64_t rows_pad, int32_t M, int32_t QB,
                                                       int64_t sbh, int64_t ss, float2* ld, int32_t* counters) {
    if (blockIdx.x == 0 && threadIdx.x < 2) counters[threadIdx.x] = 0;  // work counters of the two kernels
    constexpr int kLanesPerRow = D / 8;          // 16 (D = 128) or 8 (D = 64)
    constexpr int kRowsPerIter = 32 / kLanesPerRow;
    constexpr int kIters = kPrepRowsPerWarp / kRowsPerIter;
    const int lane = threadIdx.x & 31;
    const int sub = lane / kLanesPerRow;         // row within an iteration
    const int part = lane % kLanesPerRow;        // 16-byte piece of the row
    const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * kPrepRowsPerWarp;
    const int64_t per_bh = static_cast<int64_t>(QB) * 128;
    uint4 a[kIters], g[kIters];
    bool in[kIters];
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
        const int64_t row = row0 + it * kRowsPerIter + sub;
        const int64_t bh = row / per_bh;
        const int i = static_cast<int>(row - bh * per_bh);
        in[it] = row < rows_pad && i < M;
        if (in[it]) {
            const int64_t base = bh * sbh + static_cast<int64_t>(i) * ss + part * 8;
            a[it] = __ldg(reinterpret_cast<const uint4*>(out + base));
            g[it] = __ldg(reinterpret_cast<const uint4*>(dout + base));
        } else {
            a[it] = make_uint4(0u, 0u, 0u, 0u);
            g[it] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
        const uint32_t av[4] = {a[it].x, a[it].y, a[it].z, a[it].w};
        const uint32_t gv[4] = {g[it].x, g[it].y, g[it].z, g[it].w};
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[k]));
            const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv[k]));
            acc = fmaf(x.x, y.x, fmaf(x.y, y.y, acc));
        }
#pragma unroll
        for (int o = kLanesPerRow / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
        const int64_t row = row0 + it * kRowsPerIter + sub;
        if (part == 0 && row < rows_pad) {
            const int64_t bh = row / per_bh;
            const int i = static_cast<int>(row - bh * per_bh);
            float l2 = INFINITY;
            if (in[it]) {
                const float L = __ldg(lse + bh * M + i);
                l2 = (L == -INFINITY) ? INFINITY : L * kLog2e;
            }
            ld[row] = make_float2(-l2, in[it] ? -acc : 0.f);
        }
    }
}

// LONG: lists longer than kBwdMaxEntries blocks, or units of more entries
// (GQA group x list length), handed out in segments. Without it every unit
// fits one buffer and the segment logic folds away.
template <int D, int SCORE, bool KVSIDE, bool LONG>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdParams p, const MaskDnf dnf) {
    using L = BwdSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
    auto list_of = [&](int buf) -> uint32_t* { return reinterpret_cast<uint32_t*>(smem + L::kList + buf * L::kListBytes); };
    auto hdr_of = [&](int buf) -> BwdUnit* { return reinterpret_cast<BwdUnit*>(smem + L::kHdr + 32 * buf); };

    // ------------------------------------------------------------ set-up
    if (warp == kBwdWarpLoad && lane == 0) {
        mbar_init(bar(L::kBarFixedFull), 1);
        mbar_init(bar(L::kBarFixedEmpty), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(L::kBarTFull + s), 1);
            mbar_init(bar(L::kBarTEmpty + s), 1);
            mbar_init(bar(L::kBarListFull + s), 32);     // every scheduler lane
            mbar_init(bar(L::kBarListEmpty + s), 1 + 1 + 8);  // producer, MMA warp, softmax warps
        }
        mbar_init(bar(L::kBarSFull), 1);
        mbar_init(bar(L::kBarDpFull), 1);
        mbar_init(bar(L::kBarPFull), 8);  // every softmax warp
        mbar_init(bar(L::kBarDsFull), 8);
        mbar_init(bar(L::kBarAccFull), 1);
        mbar_init(bar(L::kBarAccEmpty), 8);
        mbar_init(bar(L::kBarDone), 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_do);
    }
    if (warp == kBwdWarpMma) {
        tmem_alloc(sbase + L::kTmemSlot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlot);

    // Register split: every thread is launched with 168 registers (build.py
    // checks the count); warpgroup 2 gives some back and the softmax
    // warpgroups take them: 128 * 80 + 256 * 208 = 63488 <= 384 * 168.
    if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 80;\n" ::: "memory");
    if (warp == kBwdWarpSched) {
        // ================================================= scheduler warp
        // Takes units from the work counter in order (dk/dv: kv-blocks
        // ascending, which under a causal mask puts the longest first; dq:
        // q-blocks descending) and writes each unit's entry list: for each
        // query head of the GQA group (dk/dv) or the unit's head (dq), the
        // blocks of the partial and the full list, merged in ascending order.
        // A block in both lists counts as partial; with a ragged KV_LEN the
        // last kv block is partial (dq).
        uint8_t* flags = smem + L::kFlags;
        for (int j = lane; j < (LONG ? kBwdMaxEntries : p.list_len); j += 32) flags[j] = 0;
        __syncwarp();
        const int heads = KVSIDE ? p.group : 1;
        const bool ragged_last = !KVSIDE && (p.N & 127) != 0;
        const uint32_t below = (1u << lane) - 1u;
        for (int it = 0;; ++it) {
            const int buf = it & 1;
            if (!mbar_wait(bar(L::kBarListEmpty + buf), static_cast<uint32_t>((it >> 1) & 1) ^ 1u, abort_flag)) break;
            int u = 0;
            if (lane == 0) u = atomicAdd(p.next_unit, 1);
            u = __shfl_sync(0xFFFFFFFFu, u, 0);
            BwdUnit* hdr = hdr_of(buf);
            if (u >= p.num_units) {
                if (lane == 0) hdr->T = -1;
                __syncwarp();
                mbar_arrive(bar(L::kBarListFull + buf));
                break;
            }
            int b, hq, hkv, blk;
            if constexpr (KVSIDE) {
                const int n_bh = p.B * p.Hkv;
                blk = u / n_bh;
                const int bh = u - blk * n_bh;
                b = bh / p.Hkv;
                hkv = bh - b * p.Hkv;
                hq = hkv * p.group;
            } else {
                const int n_bh = p.B * p.Hq;
                const int r = u / n_bh;
                blk = p.QB - 1 - r;
                const int bh = u - r * n_bh;
                b = bh / p.Hq;
                hq = bh - b * p.Hq;
                hkv = hq / p.group;
            }
            if constexpr (!LONG) {
                uint32_t* entries = list_of(buf);
                int T = 0;
                bool bad = false;
                for (int g = 0; g < heads; ++g) {
                    if (!p.has_block_mask) {
                        for (int c = 0; c < p.list_len; c += 32) {
                            const int j = c + lane;
                            if (j < p.list_len) {
                                const bool part = ragged_last && j == p.list_len - 1;
                                entries[T + j] = static_cast<uint32_t>(j) | (static_cast<uint32_t>(g) << 16) |
                                                 (part ? kBwdPartial : 0u);
                            }
                        }
                        T += p.list_len;
                        continue;
                    }
                    const int hl = KVSIDE ? hq + g : hq;
                    const int bb = p.Bm > 1 ? b : 0;
                    const int hh = p.Hm > 1 ? hl : 0;
                    const int64_t row = (static_cast<int64_t>(bb) * p.Hm + hh) * p.list_rows + blk;
                    int v = 0;
                    if (lane == 0) v = __ldg(p.num + row);
                    if (lane == 1) v = __ldg(p.full_num + row);
                    if (v < 0 || v > p.list_len) {
                        bad = true;
                        v = 0;
                    }
                    const int cnt0 = __shfl_sync(0xFFFFFFFFu, v, 0);
                    const int cnt1 = __shfl_sync(0xFFFFFFFFu, v, 1);
                    const int32_t* l0 = p.idx + row * p.list_len;
                    const int32_t* l1 = p.full_idx + row * p.list_len;
                    for (int j = lane; j < cnt0; j += 32) {
                        const int x = __ldg(l0 + j);
                        if (x >= 0 && x < p.list_len) flags[x] |= 1u;
                        else bad = true;
                    }
                    __syncwarp();
                    for (int j = lane; j < cnt1; j += 32) {
                        const int x = __ldg(l1 + j);
                        if (x >= 0 && x < p.list_len) flags[x] |= 2u;
                        else bad = true;
                    }
                    __syncwarp();
                    for (int c = 0; c < p.list_len; c += 32) {
                        const int j = c + lane;
                        uint32_t f = 0;
                        if (j < p.list_len) {
                            f = flags[j];
                            flags[j] = 0;
                        }
                        const bool part = (f & 1u) || (f != 0u && ragged_last && j == p.list_len - 1);
                        const unsigned bal = __ballot_sync(0xFFFFFFFFu, f != 0u);
                        if (f)
                            entries[T + __popc(bal & below)] = static_cast<uint32_t>(j) |
                                                               (static_cast<uint32_t>(g) << 16) |
                                                               (part ? kBwdPartial : 0u);
                        T += __popc(bal);
                    }
                    __syncwarp();
                }
                if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) record_status(BSMT_ERR_DEVICE_BOUNDS);
                if (lane == 0) {
                    hdr->T = T;
                    hdr->b = b;
                    hdr->hq = hq;
                    hdr->hkv = hkv;
                    hdr->blk = blk;
                }
                __syncwarp();
                mbar_arrive(bar(L::kBarListFull + buf));
            } else {
                // Windows of kBwdMaxEntries list positions for the flags; the
                // unit's entries are counted first, so that a full buffer goes
                // out marked as continued exactly when entries remain.
                constexpr int kCap = kBwdMaxEntries;
                bool bad = false;
                auto counts = [&](int g, int& cnt0, int& cnt1, const int32_t*& l0, const int32_t*& l1) {
                    const int hl = KVSIDE ? hq + g : hq;
                    const int bb = p.Bm > 1 ? b : 0;
                    const int hh = p.Hm > 1 ? hl : 0;
                    const int64_t row = (static_cast<int64_t>(bb) * p.Hm + hh) * p.list_rows + blk;
                    int v = 0;
                    if (lane == 0) v = __ldg(p.num + row);
                    if (lane == 1) v = __ldg(p.full_num + row);
                    if (v < 0 || v > p.list_len) {
                        bad = true;
                        v = 0;
                    }
                    cnt0 = __shfl_sync(0xFFFFFFFFu, v, 0);
                    cnt1 = __shfl_sync(0xFFFFFFFFu, v, 1);
                    l0 = p.idx + row * p.list_len;
                    l1 = p.full_idx + row * p.list_len;
                };
                // bit 1: partial list, bit 2: full list, for positions [w0, w0 + span)
                auto mark = [&](int cnt0, int cnt1, const int32_t* l0, const int32_t* l1, int w0, int span) {
                    for (int j = lane; j < cnt0; j += 32) {
                        const int x = __ldg(l0 + j);
                        if (x < 0 || x >= p.list_len) bad = true;
                        else if (x >= w0 && x - w0 < span) flags[x - w0] |= 1u;
                    }
                    __syncwarp();
                    for (int j = lane; j < cnt1; j += 32) {
                        const int x = __ldg(l1 + j);
                        if (x < 0 || x >= p.list_len) bad = true;
                        else if (x >= w0 && x - w0 < span) flags[x - w0] |= 2u;
                    }
                    __syncwarp();
                };
                int total = 0;
                for (int g = 0; g < heads; ++g) {
                    if (!p.has_block_mask) {
                        total += p.list_len;
                        continue;
                    }
                    int cnt0, cnt1;
                    const int32_t *l0, *l1;
                    counts(g, cnt0, cnt1, l0, l1);
                    for (int w0 = 0; w0 < p.list_len; w0 += kCap) {
                        const int span = min(kCap, p.list_len - w0);
                        mark(cnt0, cnt1, l0, l1, w0, span);
                        for (int c = 0; c < span; c += 32) {
                            uint32_t f = 0;
                            if (c + lane < span) {
                                f = flags[c + lane];
                                flags[c + lane] = 0;
                            }
                            total += __popc(__ballot_sync(0xFFFFFFFFu, f != 0u));
                        }
                        __syncwarp();
                    }
                }
                int cur = buf, T = 0, off = 0;
                uint32_t* ents = list_of(cur);
                auto publish = [&](int t) {
                    BwdUnit* hh = hdr_of(cur);
                    if (lane == 0) {
                        hh->T = t;
                        hh->b = b;
                        hh->hq = hq;
                        hh->hkv = hkv;
                        hh->blk = blk;
                        hh->total = total;
                        hh->off = off;
                    }
                    __syncwarp();
                    mbar_arrive(bar(L::kBarListFull + cur));
                };
                bool ok = true;
                for (int g = 0; g < heads && ok; ++g) {
                    int cnt0 = 0, cnt1 = 0;
                    const int32_t *l0 = nullptr, *l1 = nullptr;
                    if (p.has_block_mask) counts(g, cnt0, cnt1, l0, l1);
                    for (int w0 = 0; w0 < p.list_len && ok; w0 += kCap) {
                        const int span = min(kCap, p.list_len - w0);
                        if (p.has_block_mask) mark(cnt0, cnt1, l0, l1, w0, span);
                        for (int c = 0; c < span; c += 32) {
                            const int j = w0 + c + lane;
                            uint32_t f = 0;
                            if (c + lane < span) {
                                if (p.has_block_mask) {
                                    f = flags[c + lane];
                                    flags[c + lane] = 0;
                                } else {
                                    f = 2u;  // every block, as full
                                }
                            }
                            const bool part = (f & 1u) || (f != 0u && ragged_last && j == p.list_len - 1);
                            const uint32_t ent = static_cast<uint32_t>(j) | (static_cast<uint32_t>(g) << 16) |
                                                 (part ? kBwdPartial : 0u);
                            const unsigned bal = __ballot_sync(0xFFFFFFFFu, f != 0u);
                            const int pos = T + __popc(bal & below);
                            if (f != 0u && pos < kCap) ents[pos] = ent;
                            T += __popc(bal);
                            if (T >= kCap && off + kCap < total) {
                                // a full buffer with entries left: it goes out, and the
                                // chunk's remaining entries open the next one
                                publish(kCap);
                                ++it;
                                cur = it & 1;
                                if (!mbar_wait(bar(L::kBarListEmpty + cur), static_cast<uint32_t>((it >> 1) & 1) ^ 1u,
                                               abort_flag)) {
                                    ok = false;
                                    break;
                                }
                                ents = list_of(cur);
                                off += kCap;
                                if (f != 0u && pos >= kCap) ents[pos - kCap] = ent;
                                T -= kCap;
                            }
                        }
                        __syncwarp();
                    }
                }
                if (!ok) break;
                if (T > kCap) {  // (the two passes read the same lists, so this does not happen)
                    bad = true;
                    T = kCap;
                }
                if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) record_status(BSMT_ERR_DEVICE_BOUNDS);
                publish(T);
            }
        }
    } else if (warp == kBwdWarpLoad) {
        // ================================================= TMA producer warp
        const uint32_t tile = L::kTile;
        uint32_t ge = 0, fixed_uses = 0;  // entries and units with entries so far
        for (int it = 0;; ++it) {
            const int buf = it & 1;
            if (!mbar_wait(bar(L::kBarListFull + buf), static_cast<uint32_t>((it >> 1) & 1), abort_flag)) break;
            const BwdUnit hdr = *hdr_of(buf);
            if (hdr.T < 0) break;
            const uint32_t* entries = list_of(buf);
            bool ok = true;
            if (hdr.T > 0) {
                // K, V (dk/dv) or Q, dO (dq) of the unit (with its first segment),
                // once the last unit's S and dP are issued
                if ((!LONG || hdr.off == 0) && fixed_uses > 0 &&
                    !mbar_wait(bar(L::kBarFixedEmpty), (fixed_uses - 1) & 1u, abort_flag))
                    break;
                const int zf = KVSIDE ? hdr.b * p.Hkv + hdr.hkv : hdr.b * p.Hq + hdr.hq;
                if (!LONG || hdr.off == 0) ++fixed_uses;
                if ((!LONG || hdr.off == 0) && lane == 0) {
                    const uint32_t fb = bar(L::kBarFixedFull);
                    mbar_arrive_expect_tx(fb, 2 * tile);
#pragma unroll
                    for (int h = 0; h < D / 64; ++h) {
                        tma_load_3d(sbase + L::kF0 + h * 16384, KVSIDE ? &tm_k : &tm_q, h * 64, hdr.blk * 128, zf, fb);
                        tma_load_3d(sbase + L::kF1 + h * 16384, KVSIDE ? &tm_v : &tm_do, h * 64, hdr.blk * 128, zf, fb);
                    }
                }
                for (int e = 0; e < hdr.T; ++e, ++ge) {
                    const uint32_t s = ge & 1u;
                    if (!mbar_wait(bar(L::kBarTEmpty + s), ((ge >> 1) & 1u) ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t ent = entries[e];
                    const int eb = static_cast<int>(ent & 0xFFFFu);
                    const int g = static_cast<int>((ent >> 16) & 0xFFu);
                    if (lane == 0) {
                        const uint32_t fb = bar(L::kBarTFull + s);
                        mbar_arrive_expect_tx(fb, 2 * tile + (KVSIDE ? 1024u : 0u));
                        const uint32_t t0 = sbase + L::kStage + s * 2u * tile;
                        const int zt = KVSIDE ? hdr.b * p.Hq + hdr.hq + g : hdr.b * p.Hkv + hdr.hkv;
#pragma unroll
                        for (int h = 0; h < D / 64; ++h) {
                            tma_load_3d(t0 + h * 16384, KVSIDE ? &tm_q : &tm_k, h * 64, eb * 128, zt, fb);
                            tma_load_3d(t0 + tile + h * 16384, KVSIDE ? &tm_do : &tm_v, h * 64, eb * 128, zt, fb);
                        }
                        if constexpr (KVSIDE)
                            bulk_load_1d(sbase + L::kLd + 1024u * s,
                                         p.ld + (static_cast<int64_t>(hdr.b * p.Hq + hdr.hq + g) * p.QB + eb) * 128,
                                         1024u, fb);
                    }
                    __syncwarp();
                }
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::kBarListEmpty + buf));
        }
    } else if (warp == kBwdWarpMma) {
        // ================================================= MMA issuer warp
        constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, false, true);
        const uint64_t f0d = sdesc_sw128(sbase + L::kF0, 16, 1024);
        const uint64_t f1d = sdesc_sw128(sbase + L::kF1, 16, 1024);
        const uint32_t tm_s = tmem, tm_dp = tmem + 128u, tm_a0 = tmem + 256u, tm_a1 = tmem + 256u + D;
        auto t0_of = [&](uint32_t g) -> uint32_t {  // streamed tile T0 of entry g (T1 one tile further)
            return sbase + L::kStage + (g & 1u) * 2u * L::kTile;
        };
        auto wait_tiles = [&](uint32_t g) -> bool {
            if (!mbar_wait(bar(L::kBarTFull + (g & 1u)), (g >> 1) & 1u, abort_flag)) return false;
            tc_fence_after();
            return true;
        };
        auto wait_phase = [&](int which, uint32_t parity) -> bool {
            if (!mbar_wait(bar(which), parity & 1u, abort_flag)) return false;
            tc_fence_after();
            return true;
        };
        // S(g) = F0 T0(g)^T and dP(g) = F1 T1(g)^T, each 128 x 128 over K = D
        auto issue_s = [&](uint32_t g) {
            if (elect_one()) {
                mma_ss_run<D / 16>(tm_s, f0d, sdesc_sw128(t0_of(g), 16, 1024), idesc_s, 0u);
                mma_commit(bar(L::kBarSFull));
            }
            __syncwarp();
        };
        auto issue_dp = [&](uint32_t g) {
            if (elect_one()) {
                mma_ss_run<D / 16>(tm_dp, f1d, sdesc_sw128(t0_of(g) + L::kTile, 16, 1024), idesc_s, 0u);
                mma_commit(bar(L::kBarDpFull));
            }
            __syncwarp();
        };
        // acc += A B over K = 128 rows of the streamed tile: A from TMEM columns
        // a, a+8, ... in two runs (columns 0-31 hold tile rows 0-63, columns
        // 64-95 rows 64-127), B MN-major from tile rows 0-63 and 64-127
        auto issue_acc = [&](uint32_t acc, uint32_t a, uint32_t tile, bool first) {
            mma_ts_run4(acc, a, sdesc_sw128(tile, 16384, 1024), idesc_acc, first ? 0u : 1u);
            mma_ts_run4(acc, a + 64u, sdesc_sw128(tile + 8192u, 16384, 1024), idesc_acc, 1u);
        };
        uint32_t ge = 0, units = 0;  // entries and units with entries so far
        bool pend_p = false;         // the P phase of entry ge - 1 is not yet waited for
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int buf = it & 1;
            if (!mbar_wait(bar(L::kBarListFull + buf), static_cast<uint32_t>((it >> 1) & 1), abort_flag)) break;
            const BwdUnit hdr = *hdr_of(buf);
            if (hdr.T < 0) break;
            const int T = hdr.T;
            // a segment's entries are entries off .. off + T - 1 of the unit's total
            const int total = LONG ? hdr.total : T;
            const int off = LONG ? hdr.off : 0;
            if (T > 0) {
                if (off == 0) {
                    // the unit's fixed tiles; S(first) overwrites S once the last P phase has read it
                    if (!(ok = wait_phase(L::kBarFixedFull, units))) break;
                    if (pend_p && !(ok = wait_phase(L::kBarPFull, ge - 1))) break;
                    if (!(ok = wait_tiles(ge))) break;
                    issue_s(ge);
                    issue_dp(ge);
                    if (total == 1 && elect_one()) mma_commit(bar(L::kBarFixedEmpty));
                    __syncwarp();
                }
                for (int n = 0; n < T && ok; ++n) {
                    const uint32_t g = ge + n;
                    const uint32_t t0 = t0_of(g);
                    const int nu = off + n;  // entry of the unit
                    const bool more = nu + 1 < total;
                    // The first accumulating product of a unit overwrites the
                    // accumulators: the previous unit's epilogue must have read them.
                    const bool acc_wait = nu == 0 && units > 0;
                    if constexpr (KVSIDE) {
                        // dV(g) += P(g)^T dO(g), S(g+1), dK(g) += dS(g)^T Q(g), dP(g+1)
                        if (!(ok = wait_phase(L::kBarPFull, g))) break;
                        if (acc_wait && !(ok = wait_phase(L::kBarAccEmpty, units - 1))) break;
                        if (elect_one()) issue_acc(tm_a0, tm_s, t0 + L::kTile, nu == 0);
                        __syncwarp();
                        if (more) {
                            if (!(ok = wait_tiles(g + 1))) break;
                            issue_s(g + 1);
                        }
                        if (!(ok = wait_phase(L::kBarDsFull, g))) break;
                        if (elect_one()) {
                            issue_acc(tm_a1, tm_dp, t0, nu == 0);
                            mma_commit(bar(L::kBarTEmpty + (g & 1u)));
                        }
                        __syncwarp();
                    } else {
                        // S(g+1) once the P phase of g has read S(g), dQ(g) += dS(g) K(g), dP(g+1)
                        if (more) {
                            if (!(ok = wait_phase(L::kBarPFull, g) && wait_tiles(g + 1))) break;
                            issue_s(g + 1);
                        }
                        if (!(ok = wait_phase(L::kBarDsFull, g))) break;
                        if (acc_wait && !(ok = wait_phase(L::kBarAccEmpty, units - 1))) break;
                        if (elect_one()) {
                            issue_acc(tm_a0, tm_dp, t0, nu == 0);
                            mma_commit(bar(L::kBarTEmpty + (g & 1u)));
                        }
                        __syncwarp();
                    }
                    if (more) {
                        issue_dp(g + 1);
                        // the unit's last S and dP are issued: its fixed tiles may be replaced
                        if (nu + 2 == total && elect_one()) mma_commit(bar(L::kBarFixedEmpty));
                        __syncwarp();
                    }
                }
                if (!ok) break;
                ge += T;
                if (off + T == total) {  // the unit's last segment
                    if (elect_one()) mma_commit(bar(L::kBarAccFull));
                    __syncwarp();
                    pend_p = !KVSIDE;  // the dq side does not wait for its last P phase
                    ++units;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::kBarListEmpty + buf));
        }
        // every MMA of this warp must finish before TMEM is freed
        if (elect_one()) mma_commit(bar(L::kBarDone));
        __syncwarp();
        mbar_wait(bar(L::kBarDone), 0, abort_flag);
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 208;\n" ::: "memory");
        // ================================================= softmax warpgroups
        const int h = warp >> 2;  // this warpgroup's 64 columns of every entry: [64 h, 64 h + 64)
        const int r = threadIdx.x & 127;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_s = tmem + 64u * static_cast<uint32_t>(h) + lane_base;
        const uint32_t t_dp = t_s + 128u;
        const int db_of = dnf.doc_batch > 1 ? 1 : 0;
        const bool masked_path = p.has_block_mask != 0;
        constexpr bool kAlibi = SCORE == kScoreAlibi || SCORE == kScoreSoftcapAlibi || SCORE == kScoreAlibiSoftcap;
        const float2* ld_smem = reinterpret_cast<const float2*>(smem + L::kLd);
        uint32_t ge = 0, units = 0;
        bool ok = true;
        // dq: the document this warp searched last (batch row of the ids, id,
        // kv span), which a later unit's rows often share
        int32_t cache_db = -1, cache_id = 0;
        int64_t cache_lo = 0, cache_hi = -1;
        for (int it = 0; ok; ++it) {
            int buf = it & 1;
            if (!mbar_wait(bar(L::kBarListFull + buf), static_cast<uint32_t>((it >> 1) & 1), abort_flag)) break;
            BwdUnit hdr = *hdr_of(buf);
            if (hdr.T < 0) break;
            const int total = LONG ? hdr.total : hdr.T;  // the unit's entries
            const int b = hdr.b, hq = hdr.hq, hkv = hdr.hkv;
            const int db = db_of ? b : 0;
            const int64_t row_idx = static_cast<int64_t>(hdr.blk) * 128 + r;  // this thread's kv (dk/dv) or q (dq)
            // Per-row data, fixed for the unit: the key's document id (dk/dv), or
            // the query's -lse2, -delta and document span (dq). Term intervals
            // are recomputed on each partial tile from the mask program.
            int32_t my_doc = 0;
            bool my_doc_ok = false;
            int64_t row_ds = 0, row_de = -1;
            float2 nl_row = make_float2(-INFINITY, -INFINITY), nd_row = make_float2(0.f, 0.f);
            float slope_unit = 0.f;
            if constexpr (KVSIDE) {
                if (dnf.has_doc && masked_path && row_idx < p.N) {
                    my_doc = __ldg(dnf.kv_doc + static_cast<int64_t>(db) * p.N + row_idx);
                    my_doc_ok = true;
                }
            } else if (total > 0) {
                const float2 ldr = p.ld[static_cast<int64_t>(b * p.Hq + hq) * p.QB * 128 + row_idx];
                nl_row = make_float2(ldr.x, ldr.x);
                nd_row = make_float2(ldr.y, ldr.y);
                if constexpr (kAlibi)
                    slope_unit = p.slopes ? __ldg(p.slopes + hq)
                                          : exp2f(-8.0f * static_cast<float>(p.alibi_h0 + hq + 1) /
                                                  static_cast<float>(p.alibi_heads));
                if (dnf.has_doc && masked_path) {
                    // the span [first, last] of kv positions with this row's document
                    // id (kv ids are non-decreasing); one warp search per distinct id
                    const int32_t* qd_row = dnf.q_doc + static_cast<int64_t>(db) * p.M;
                    const int32_t* kd_row = dnf.kv_doc + static_cast<int64_t>(db) * p.N;
                    const bool valid = row_idx < p.M;
                    const int32_t d = valid ? __ldg(qd_row + row_idx) : 0;
                    bool pending = valid;
                    if (!LONG && pending && db == cache_db && d == cache_id) {
                        row_ds = cache_lo;
                        row_de = cache_hi;
                        pending = false;
                    }
                    unsigned todo;
                    while ((todo = __ballot_sync(0xFFFFFFFFu, pending)) != 0u) {
                        const int32_t x = __shfl_sync(0xFFFFFFFFu, d, __ffs(todo) - 1);
                        const int first = warp_lower_bound(kd_row, p.N, x, lane);
                        const int past = warp_lower_bound(kd_row, p.N, static_cast<int64_t>(x) + 1, lane);
                        if (pending && d == x) {
                            row_ds = first;
                            row_de = past - 1;
                            pending = false;
                        }
                        if constexpr (!LONG) {  // (x and the results are the same in every lane)
                            cache_db = db;
                            cache_id = x;
                            cache_lo = first;
                            cache_hi = past - 1;
                        }
                    }
                }
            }
            // The unit's segments, in order (one but for LONG units of many entries);
            // each buffer but the unit's last is released once its entries are done.
            for (;;) {
                const uint32_t* entries = list_of(buf);
                const int T = hdr.T;
                for (int n = 0; n < T && ok; ++n) {
                    const uint32_t g_ent = ge + n;
                    const uint32_t ent = entries[n];
                    const int eb = static_cast<int>(ent & 0xFFFFu);
                    const int g = static_cast<int>((ent >> 16) & 0xFFu);
                    const bool partial = (ent & kBwdPartial) != 0u;
                    const int64_t c0 = static_cast<int64_t>(eb) * 128 + 64 * h;  // first column (q or kv) of this warpgroup
                    // mask words over the warpgroup's 64 columns (bit j: column c0 + j allowed)
                    uint32_t w0 = 0xFFFFFFFFu, w1 = 0xFFFFFFFFu;
                    if (partial) {
                        w0 = 0u;
                        w1 = 0u;
                        if constexpr (KVSIDE) {
                            uint32_t d0 = 0xFFFFFFFFu, d1 = 0xFFFFFFFFu;
                            if (dnf.term_has_doc) {
                                d0 = 0u;
                                d1 = 0u;
                                if (my_doc_ok) {
                                    const int32_t* qd_row = dnf.q_doc + static_cast<int64_t>(db) * p.M;
#pragma unroll 8
                                    for (int j = 0; j < 64; ++j) {
                                        const int64_t q = c0 + j;
                                        const bool m = q < p.M && __ldg(qd_row + q) == my_doc;
                                        if (j < 32) d0 |= (m ? 1u : 0u) << j;
                                        else d1 |= (m ? 1u : 0u) << (j - 32);
                                    }
                                }
                            }
                            if (row_idx < p.N) {
                                for (int t = 0; t < dnf.n_terms; ++t) {
                                    int64_t lo, hi;
                                    term_q_interval(dnf, t, row_idx, p.M, lo, hi);
                                    uint32_t a0 = range_bits(lo, hi, c0);
                                    uint32_t a1 = range_bits(lo, hi, c0 + 32);
                                    if ((dnf.term_has_doc >> t) & 1u) {
                                        a0 &= d0;
                                        a1 &= d1;
                                    }
                                    w0 |= a0;
                                    w1 |= a1;
                                }
                            }
                        } else {
                            const int64_t c1 = (c0 + 63 < p.N - 1) ? c0 + 63 : p.N - 1;
                            if (masked_path) {
                                for (int t = 0; t < dnf.n_terms; ++t) {
                                    int64_t lo, hi;
                                    term_interval(dnf, t, row_idx, c0, c1, row_ds, row_de, lo, hi);
                                    w0 |= range_bits(lo, hi, c0);
                                    w1 |= range_bits(lo, hi, c0 + 32);
                                }
                            } else {
                                w0 = range_bits(c0, c1, c0);
                                w1 = range_bits(c0, c1, c0 + 32);
                            }
                        }
                    }
                    float slope = slope_unit;
                    if constexpr (KVSIDE && kAlibi)
                        slope = p.slopes ? __ldg(p.slopes + hq + g)
                                         : exp2f(-8.0f * static_cast<float>(p.alibi_h0 + hq + g + 1) /
                                                 static_cast<float>(p.alibi_heads));
                    // kv - q at the warpgroup's column 0; it moves by -1 (dk/dv) or +1 (dq) per column
                    const float dkv0 = KVSIDE ? static_cast<float>(row_idx - c0) : static_cast<float>(c0 - row_idx);
                    constexpr float kStep = KVSIDE ? -1.f : 1.f;
                    BwdCols hb;
                    if constexpr (SCORE == kScoreAlibiSoftcap) {
                        hb.bias0 = slope * dkv0;
                        hb.bstep = slope * kStep;
                    } else {
                        hb.bias0 = slope * kLog2e * dkv0;
                        hb.bstep = slope * kLog2e * kStep;
                    }
                    const float4* ld4 = reinterpret_cast<const float4*>(ld_smem + 128 * (g_ent & 1u) + 64 * h);
                    float pg[64];  // P * dz/ds of this thread's 64 columns, from the P phase to the dS phase
                    // ---- P phase: S -> P (bf16 into TMEM for dV on the dk/dv side)
                    if (!mbar_wait(bar(L::kBarSFull), g_ent & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    __syncwarp();  // tcgen05.ld/st are warp-collective: reconverge after the wait
                    tc_fence_after();
                    {
                        // the second 32 columns load while the first are computed
                        float x[64];
                        tmem_ld32(t_s, *reinterpret_cast<uint32_t(*)[32]>(x));
                        tc_wait_ld();
                        tmem_ld32(t_s + 32u, *reinterpret_cast<uint32_t(*)[32]>(x + 32));
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            if (c == 1) tc_wait_ld();
                            uint32_t pk[16];
                            if (partial)
                                bwd_p_chunk<SCORE, KVSIDE, true>(p, x, ld4, nl_row, hb, 32 * c, c == 0 ? w0 : w1, pg, pk);
                            else
                                bwd_p_chunk<SCORE, KVSIDE, false>(p, x, ld4, nl_row, hb, 32 * c, 0u, pg, pk);
                            if constexpr (KVSIDE) tmem_st16(t_s + 16u * c, pk);
                        }
                    }
                    if constexpr (KVSIDE) tc_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(L::kBarPFull));
                    // ---- dS phase: dP -> dS (bf16 into TMEM for dK or dQ)
                    if (!mbar_wait(bar(L::kBarDpFull), g_ent & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    __syncwarp();
                    tc_fence_after();
                    {
                        float dp[64];
                        tmem_ld32(t_dp, *reinterpret_cast<uint32_t(*)[32]>(dp));
                        tc_wait_ld();
                        tmem_ld32(t_dp + 32u, *reinterpret_cast<uint32_t(*)[32]>(dp + 32));
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            if (c == 1) tc_wait_ld();
                            uint32_t dk[16];
                            bwd_ds_chunk<KVSIDE>(dp, ld4, nd_row, pg, 32 * c, dk);
                            tmem_st16(t_dp + 16u * c, dk);
                        }
                    }
                    tc_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(L::kBarDsFull));
                }
                if (!ok) break;
                ge += T;
                if (!LONG || hdr.off + T == total) break;
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(L::kBarListEmpty + buf));
                ++it;
                buf = it & 1;
                if (!mbar_wait(bar(L::kBarListFull + buf), static_cast<uint32_t>((it >> 1) & 1), abort_flag)) {
                    ok = false;
                    break;
                }
                hdr = *hdr_of(buf);
            }
            if (!ok) break;
            // -------------------------------------------------- epilogue
            // dk/dv: warpgroup 0 writes dV, warpgroup 1 writes dK (times scale).
            // dq: warpgroup h writes columns [h D/2, (h+1) D/2) of dQ (times
            // scale). The accumulator is read whole and released before the
            // stores, so that the next unit's products can start.
            constexpr int kCols = KVSIDE ? D : D / 2;
            constexpr int kBatch = kCols < 64 ? kCols : 64;  // columns read, packed and stored at a time
            const bool valid = row_idx < (KVSIDE ? p.N : p.M);
            const float mul = (KVSIDE && h == 0) ? 1.f : p.scale;
            __nv_bfloat16* dst;
            if constexpr (KVSIDE)
                dst = (h == 0 ? p.g1 : p.g0) + static_cast<int64_t>(b * p.Hkv + hkv) * p.kv_sbh + row_idx * p.kv_ss;
            else
                dst = p.g0 + static_cast<int64_t>(b * p.Hq + hq) * p.q_sbh + row_idx * p.q_ss + h * (D / 2);
            uint4* d4 = reinterpret_cast<uint4*>(dst);
            if (total > 0) {
                if (!(ok = mbar_wait(bar(L::kBarAccFull), units & 1u, abort_flag))) break;
                ++units;
                __syncwarp();
                tc_fence_after();
                const uint32_t src = tmem + 256u + (KVSIDE ? (h == 0 ? 0u : static_cast<uint32_t>(D))
                                                           : static_cast<uint32_t>(h * (D / 2))) + lane_base;
#pragma unroll
                for (int c0 = 0; c0 < kCols; c0 += kBatch) {
                    uint32_t a[kBatch];
#pragma unroll
                    for (int c = 0; c < kBatch / 32; ++c)
                        tmem_ld32(src + static_cast<uint32_t>(c0 + 32 * c), *reinterpret_cast<uint32_t(*)[32]>(a + 32 * c));
                    tc_wait_ld();
                    if (c0 + kBatch == kCols) {
                        // the whole accumulator is in registers: the next unit may overwrite it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(L::kBarAccEmpty));
                    }
                    if (valid) {
#pragma unroll
                        for (int v = 0; v < kBatch / 8; ++v) {
                            uint32_t pk[4];
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                pk[k] = pack_bf16x2(__uint_as_float(a[8 * v + 2 * k]) * mul,
                                                    __uint_as_float(a[8 * v + 2 * k + 1]) * mul);
                            d4[c0 / 8 + v] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                }
            } else if (valid) {
#pragma unroll
                for (int v = 0; v < kCols / 8; ++v) d4[v] = make_uint4(0u, 0u, 0u, 0u);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::kBarListEmpty + buf));
        }
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kBwdWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace bsmt
