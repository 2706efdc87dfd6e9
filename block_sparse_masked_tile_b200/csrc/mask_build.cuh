// Block-mask builder kernel (create_block_mask with separate_full_blocks).
//
// Reference: tensorplay.nn.attention page, create_block_mask and BlockMask
// "Details" items 1-2. One warp owns one (b, q-block) row of 128 queries;
// lane l evaluates rows l, l+32, l+64, l+96.
//
// Per row, the DNF mask gives a union of at most kMaxTerms kv intervals. The
// kernel sorts and merges them into disjoint intervals. Every interval then
// sets bit ranges over kv blocks: "any" covers the blocks the interval
// touches, "full" the blocks it covers entirely. AND-reducing "full" and
// OR-reducing "any" over the 128 rows with redux.sync classifies each tile
// exactly:
//   - FULL    = every in-range element allowed, tile inside both sequences;
//   - PARTIAL = some element allowed but not FULL;
//   - EMPTY   = no element allowed.
// Compaction is a ballot/popc prefix per 32-tile word. A mask is the same
// for every head, so the rows are computed once and written for each head
// of the block's head group. That makes the kernel a pure HBM writer.
#pragma once
#include "mask_dnf.cuh"
#include "ptx.cuh"

namespace bsmt {

struct BuildParams {
    int32_t Bm, Hm, Q_LEN, KV_LEN, QB, KB;
    int32_t heads_per_block;
    int32_t* kv_num;
    int32_t* kv_idx;
    int32_t* full_num;
    int32_t* full_idx;
};

constexpr int kBuildWarps = 4;
constexpr int kWordsPerChunk = 8;  // 256 kv blocks per pass

__global__ void __launch_bounds__(kBuildWarps * 32) mask_build_kernel(const MaskDnf dnf, const BuildParams p) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int qb = blockIdx.x * kBuildWarps + warp;
    const int b = blockIdx.y;
    if (qb >= p.QB) return;  // warp-uniform; no block-wide barrier below
    const int h0 = blockIdx.z * p.heads_per_block;
    const int h1 = min(p.Hm, h0 + p.heads_per_block);
    const int64_t N = p.KV_LEN;
    const int64_t M = p.Q_LEN;

    // Document ids: row pointers and the sortedness check of this block's
    // share of kv positions (every kv position is checked by exactly one
    // (qb, head-group 0) warp per batch row).
    const int32_t* qdoc = nullptr;
    const int32_t* kvdoc = nullptr;
    if (dnf.has_doc) {
        const int db = dnf.doc_batch > 1 ? b : 0;
        qdoc = dnf.q_doc + static_cast<int64_t>(db) * M;
        kvdoc = dnf.kv_doc + static_cast<int64_t>(db) * N;
        if (blockIdx.z == 0) {
            // kv blocks j with j % QB == qb belong to this warp
            bool bad = false;
            for (int64_t seg = static_cast<int64_t>(qb) * 128; seg < N; seg += static_cast<int64_t>(p.QB) * 128) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int64_t j = seg + lane * 4 + k;
                    if (j + 1 < N && __ldg(kvdoc + j) > __ldg(kvdoc + j + 1)) bad = true;
                }
            }
            if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) record_status(BSMT_ERR_DEVICE_PRECONDITION);
        }
    }

    // Per-row query index, validity and document interval [ds, de].
    int64_t qr[4];
    bool valid[4];
    int64_t ds[4], de[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        qr[r] = static_cast<int64_t>(qb) * 128 + lane + 32 * r;
        valid[r] = qr[r] < M;
        ds[r] = 0;
        de[r] = N - 1;
    }
    if (dnf.has_doc) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int32_t d = valid[r] ? __ldg(qdoc + qr[r]) : 0;
            bool pending = valid[r];
            unsigned todo;
            while ((todo = __ballot_sync(0xFFFFFFFFu, pending)) != 0u) {
                const int leader = __ffs(todo) - 1;
                const int32_t x = __shfl_sync(0xFFFFFFFFu, d, leader);
                const int first = warp_lower_bound(kvdoc, static_cast<int>(N), x, lane);
                const int past = warp_lower_bound(kvdoc, static_cast<int>(N), static_cast<int64_t>(x) + 1, lane);
                if (pending && d == x) {
                    ds[r] = first;
                    de[r] = past - 1;
                    pending = false;
                }
            }
        }
    }

    const bool q_tile_inside = static_cast<int64_t>(qb + 1) * 128 <= M;
    int cnt_p = 0, cnt_f = 0;

    for (int c0 = 0; c0 < p.KB; c0 += 32 * kWordsPerChunk) {
        uint32_t fw[kWordsPerChunk], aw[kWordsPerChunk];
#pragma unroll
        for (int w = 0; w < kWordsPerChunk; ++w) {
            fw[w] = 0xFFFFFFFFu;
            aw[w] = 0u;
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            if (!valid[r]) continue;  // rows past Q_LEN add nothing; their tile is never FULL (below)
            // intervals of this row, sorted by lo (insertion) and merged
            int64_t lo[kMaxTerms], hi[kMaxTerms];
            int n = 0;
            for (int t = 0; t < dnf.n_terms; ++t) {
                int64_t l, h;
                term_interval(dnf, t, qr[r], 0, N - 1, ds[r], de[r], l, h);
                if (l > h) continue;
                int j = n++;
                while (j > 0 && lo[j - 1] > l) {
                    lo[j] = lo[j - 1];
                    hi[j] = hi[j - 1];
                    --j;
                }
                lo[j] = l;
                hi[j] = h;
            }
            uint32_t rf[kWordsPerChunk], ra[kWordsPerChunk];
#pragma unroll
            for (int w = 0; w < kWordsPerChunk; ++w) rf[w] = ra[w] = 0u;
            int i = 0;
            while (i < n) {
                const int64_t cl = lo[i];
                int64_t ch = hi[i];
                ++i;
                while (i < n && lo[i] <= ch + 1) {
                    ch = hi[i] > ch ? hi[i] : ch;
                    ++i;
                }
                const int64_t a_lo = cl >> 7, a_hi = ch >> 7;
                const int64_t f_lo = (cl + 127) >> 7, f_hi = ((ch + 1) >> 7) - 1;
#pragma unroll
                for (int w = 0; w < kWordsPerChunk; ++w) {
                    const int64_t base = c0 + 32 * w;
                    ra[w] |= range_bits(a_lo, a_hi, base);
                    rf[w] |= range_bits(f_lo, f_hi, base);
                }
            }
#pragma unroll
            for (int w = 0; w < kWordsPerChunk; ++w) {
                fw[w] &= rf[w];
                aw[w] |= ra[w];
            }
        }
        // A lane whose four rows are all past Q_LEN leaves fw at all-ones;
        // the tile then cannot be FULL because q_tile_inside is false.
#pragma unroll
        for (int w = 0; w < kWordsPerChunk; ++w) {
            fw[w] = __reduce_and_sync(0xFFFFFFFFu, fw[w]);
            aw[w] = __reduce_or_sync(0xFFFFFFFFu, aw[w]);
            if (!q_tile_inside) fw[w] = 0u;
            // blocks at or past KB do not exist
            const int64_t base = c0 + 32 * w;
            const uint32_t exist = range_bits(0, p.KB - 1, base);
            fw[w] &= exist;
            aw[w] &= exist;
        }
        // write this chunk's entries for every head of the group
        const uint32_t below = (1u << lane) - 1u;
        for (int h = h0; h < h1; ++h) {
            const int64_t row = (static_cast<int64_t>(b) * p.Hm + h) * p.QB + qb;
            int32_t* pidx = p.kv_idx + row * p.KB;
            int32_t* fidx = p.full_idx + row * p.KB;
            int cp = cnt_p, cf = cnt_f;
#pragma unroll
            for (int w = 0; w < kWordsPerChunk; ++w) {
                const uint32_t pw = aw[w] & ~fw[w];
                const int kb = c0 + 32 * w + lane;
                if ((pw >> lane) & 1u) pidx[cp + __popc(pw & below)] = kb;
                if ((fw[w] >> lane) & 1u) fidx[cf + __popc(fw[w] & below)] = kb;
                cp += __popc(pw);
                cf += __popc(fw[w]);
            }
        }
#pragma unroll
        for (int w = 0; w < kWordsPerChunk; ++w) {
            cnt_p += __popc(aw[w] & ~fw[w]);
            cnt_f += __popc(fw[w]);
        }
    }

    // counts and zero tails
    for (int h = h0; h < h1; ++h) {
        const int64_t row = (static_cast<int64_t>(b) * p.Hm + h) * p.QB + qb;
        int32_t* pidx = p.kv_idx + row * p.KB;
        int32_t* fidx = p.full_idx + row * p.KB;
        for (int j = cnt_p + lane; j < p.KB; j += 32) pidx[j] = 0;
        for (int j = cnt_f + lane; j < p.KB; j += 32) fidx[j] = 0;
        if (lane == 0) {
            p.kv_num[row] = cnt_p;
            p.full_num[row] = cnt_f;
        }
    }
}

}  // namespace bsmt
