// Block-mask builder kernel (create_block_mask with separate_full_blocks).
//
// Reference: tensorplay.nn.attention page, create_block_mask and BlockMask
// "Details" items 1-2. One block of 8 warps owns one (b, q-block) row of
// 128 queries and a group of heads.
//
// Classification: warps 0-3 take one query row per lane (rows 32w + lane).
// Per row, the DNF mask gives a union of at most kMaxTerms kv intervals. The
// kernel sorts and merges them into disjoint intervals. Every interval then
// sets bit ranges over kv blocks: "any" covers the blocks the interval
// touches, "full" the blocks it covers entirely. AND-reducing "full" and
// OR-reducing "any" over the rows (redux.sync within a warp, then over the
// four warps in shared memory) classifies each tile exactly:
//   - FULL    = every in-range element allowed, tile inside both sequences;
//   - PARTIAL = some element allowed but not FULL;
//   - EMPTY   = no element allowed.
// Writing: a mask is the same for every head. With STAGED (KB a multiple of
// 4, at most kStagedMaxKB, 16-byte aligned lists), the row's two lists are
// compacted once into shared memory, zero tails included, and the bulk copy
// engine writes them to every head of the block's group: two copies per
// head, issued by one lane. Otherwise all 8 warps write the row's lists for
// the heads of the group, a head per warp at a time, and zero the tails with
// 16-byte stores. Compaction is a ballot/popc prefix per 32-tile word. The
// kernel is then an HBM writer.
#pragma once
#include "bulk_copy.cuh"
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

constexpr int kBuildWarps = 8;       // warps per block
constexpr int kClassifyWarps = 4;    // warps that classify (one row per lane)
constexpr int kWordsPerChunk = 8;    // 256 kv blocks per pass
constexpr int kStagedMaxKB = 4096;   // staged rows: 2 x 4096 int32 = 32 KB of shared memory

template <bool STAGED>
__global__ void __launch_bounds__(kBuildWarps * 32)
    mask_build_kernel(const __grid_constant__ MaskDnf dnf, const BuildParams p) {
    __shared__ uint32_t part_f[kClassifyWarps][kWordsPerChunk];
    __shared__ uint32_t part_a[kClassifyWarps][kWordsPerChunk];
    extern __shared__ __align__(16) int32_t staged[];  // STAGED: partial row [KB], then full row [KB]
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    if constexpr (STAGED) {
        uint4* z = reinterpret_cast<uint4*>(staged);
        for (int i = threadIdx.x; i < p.KB / 2; i += kBuildWarps * 32) z[i] = make_uint4(0u, 0u, 0u, 0u);
        // (ordered before the compaction's writes by the first chunk's __syncthreads)
    }
    const int qb = blockIdx.x;
    const int b = blockIdx.y;
    const int h0 = blockIdx.z * p.heads_per_block;
    const int h1 = min(p.Hm, h0 + p.heads_per_block);
    const int64_t N = p.KV_LEN;
    const int64_t M = p.Q_LEN;
    const bool classifier = warp < kClassifyWarps;

    // Document ids: row pointers and the sortedness check of this block's
    // share of kv positions (every kv position is checked by exactly one
    // (qb, head-group 0) block per batch row, in its warp 0).
    const int32_t* qdoc = nullptr;
    const int32_t* kvdoc = nullptr;
    if (dnf.has_doc) {
        const int db = dnf.doc_batch > 1 ? b : 0;
        qdoc = dnf.q_doc + static_cast<int64_t>(db) * M;
        kvdoc = dnf.kv_doc + static_cast<int64_t>(db) * N;
        if (blockIdx.z == 0 && warp == 0) {
            // kv blocks j with j % QB == qb belong to this block
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

    // This lane's query row (classifying warps), its validity and document
    // interval [ds, de].
    const int64_t qr = static_cast<int64_t>(qb) * 128 + 32 * warp + lane;
    const bool valid = classifier && qr < M;
    int64_t ds = 0, de = N - 1;
    if (dnf.has_doc && classifier) {
        const int32_t d = valid ? __ldg(qdoc + qr) : 0;
        bool pending = valid;
        unsigned todo;
        while ((todo = __ballot_sync(0xFFFFFFFFu, pending)) != 0u) {
            const int leader = __ffs(todo) - 1;
            const int32_t x = __shfl_sync(0xFFFFFFFFu, d, leader);
            const int first = warp_lower_bound(kvdoc, static_cast<int>(N), x, lane);
            const int past = warp_lower_bound(kvdoc, static_cast<int>(N), static_cast<int64_t>(x) + 1, lane);
            if (pending && d == x) {
                ds = first;
                de = past - 1;
                pending = false;
            }
        }
    }
    // The row's intervals, sorted by lo (insertion) and merged once.
    int64_t lo[kMaxTerms], hi[kMaxTerms];
    int nint = 0;
    if (valid) {
        int n = 0;
        for (int t = 0; t < dnf.n_terms; ++t) {
            int64_t l, h;
            term_interval(dnf, t, qr, 0, N - 1, ds, de, l, h);
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
        int i = 0;
        while (i < n) {
            const int64_t cl = lo[i];
            int64_t ch = hi[i];
            ++i;
            while (i < n && lo[i] <= ch + 1) {
                ch = hi[i] > ch ? hi[i] : ch;
                ++i;
            }
            lo[nint] = cl;
            hi[nint] = ch;
            ++nint;
        }
    }

    const bool q_tile_inside = static_cast<int64_t>(qb + 1) * 128 <= M;
    int cnt_p = 0, cnt_f = 0;

    for (int c0 = 0; c0 < p.KB; c0 += 32 * kWordsPerChunk) {
        if (classifier) {
            uint32_t fw[kWordsPerChunk], aw[kWordsPerChunk];
#pragma unroll
            for (int w = 0; w < kWordsPerChunk; ++w) {
                // rows past Q_LEN add nothing; their tile is never FULL (below)
                fw[w] = valid ? 0u : 0xFFFFFFFFu;
                aw[w] = 0u;
            }
            for (int i = 0; i < nint; ++i) {
                // kv-block bounds of the interval, relative to this chunk (32-bit:
                // intervals lie in [0, KV_LEN), so blocks fit easily)
                const int a_lo = static_cast<int>(lo[i] >> 7) - c0, a_hi = static_cast<int>(hi[i] >> 7) - c0;
                const int f_lo = static_cast<int>((lo[i] + 127) >> 7) - c0;
                const int f_hi = static_cast<int>((hi[i] + 1) >> 7) - 1 - c0;
#pragma unroll
                for (int w = 0; w < kWordsPerChunk; ++w) {
                    aw[w] |= range_bits32(a_lo - 32 * w, a_hi - 32 * w);
                    fw[w] |= range_bits32(f_lo - 32 * w, f_hi - 32 * w);
                }
            }
#pragma unroll
            for (int w = 0; w < kWordsPerChunk; ++w) {
                fw[w] = __reduce_and_sync(0xFFFFFFFFu, fw[w]);
                aw[w] = __reduce_or_sync(0xFFFFFFFFu, aw[w]);
            }
            if (lane == 0) {
#pragma unroll
                for (int w = 0; w < kWordsPerChunk; ++w) {
                    part_f[warp][w] = fw[w];
                    part_a[warp][w] = aw[w];
                }
            }
        }
        __syncthreads();
        uint32_t fw[kWordsPerChunk], aw[kWordsPerChunk];
#pragma unroll
        for (int w = 0; w < kWordsPerChunk; ++w) {
            fw[w] = part_f[0][w] & part_f[1][w] & part_f[2][w] & part_f[3][w];
            aw[w] = part_a[0][w] | part_a[1][w] | part_a[2][w] | part_a[3][w];
            if (!q_tile_inside) fw[w] = 0u;
            // blocks at or past KB do not exist
            const uint32_t exist = range_bits(0, p.KB - 1, c0 + 32 * w);
            fw[w] &= exist;
            aw[w] &= exist;
        }
        __syncthreads();  // the partial words may be rewritten by the next chunk
        // This lane's list positions for the chunk, the same for every head:
        // -1 where its kv block is not in the list.
        const uint32_t below = (1u << lane) - 1u;
        int pos_p[kWordsPerChunk], pos_f[kWordsPerChunk];
        {
            int cp = cnt_p, cf = cnt_f;
#pragma unroll
            for (int w = 0; w < kWordsPerChunk; ++w) {
                const uint32_t pw = aw[w] & ~fw[w];
                pos_p[w] = ((pw >> lane) & 1u) ? cp + __popc(pw & below) : -1;
                pos_f[w] = ((fw[w] >> lane) & 1u) ? cf + __popc(fw[w] & below) : -1;
                cp += __popc(pw);
                cf += __popc(fw[w]);
            }
        }
        if constexpr (STAGED) {
            // this chunk's entries, once, into the shared rows (warp 0: every
            // warp holds the same positions)
            if (warp == 0) {
#pragma unroll
                for (int w = 0; w < kWordsPerChunk; ++w) {
                    const int kb = c0 + 32 * w + lane;
                    if (pos_p[w] >= 0) staged[pos_p[w]] = kb;
                    if (pos_f[w] >= 0) staged[p.KB + pos_f[w]] = kb;
                }
            }
        }
        // write this chunk's entries for the heads of the group
        for (int h = h0 + warp; !STAGED && h < h1; h += kBuildWarps) {
            const int64_t row = (static_cast<int64_t>(b) * p.Hm + h) * p.QB + qb;
            int32_t* pidx = p.kv_idx + row * p.KB;
            int32_t* fidx = p.full_idx + row * p.KB;
#pragma unroll
            for (int w = 0; w < kWordsPerChunk; ++w) {
                const int kb = c0 + 32 * w + lane;
                if (pos_p[w] >= 0) pidx[pos_p[w]] = kb;
                if (pos_f[w] >= 0) fidx[pos_f[w]] = kb;
            }
        }
#pragma unroll
        for (int w = 0; w < kWordsPerChunk; ++w) {
            cnt_p += __popc(aw[w] & ~fw[w]);
            cnt_f += __popc(fw[w]);
        }
    }

    if constexpr (STAGED) {
        // the staged rows (entries, then zeros) to every head of the group
        fence_proxy_async_smem();
        __syncthreads();
        const uint32_t src = smem_u32(staged);
        const uint32_t row_bytes = static_cast<uint32_t>(p.KB) * 4u;
        for (int h = h0 + warp; h < h1; h += kBuildWarps) {
            const int64_t row = (static_cast<int64_t>(b) * p.Hm + h) * p.QB + qb;
            if (lane == 0) {
                bulk_store_1d(p.kv_idx + row * p.KB, src, row_bytes);
                bulk_store_1d(p.full_idx + row * p.KB, src + row_bytes, row_bytes);
                bulk_commit_group();
                p.kv_num[row] = cnt_p;
                p.full_num[row] = cnt_f;
            }
        }
        if (lane == 0) bulk_wait_group0();  // the shared rows are read before the block ends
        return;
    }
    // counts and zero tails
    for (int h = h0 + warp; h < h1; h += kBuildWarps) {
        const int64_t row = (static_cast<int64_t>(b) * p.Hm + h) * p.QB + qb;
        zero_tail(p.kv_idx + row * p.KB, cnt_p, p.KB, lane);
        zero_tail(p.full_idx + row * p.KB, cnt_f, p.KB, lane);
        if (lane == 0) {
            p.kv_num[row] = cnt_p;
            p.full_num[row] = cnt_f;
        }
    }
}

}  // namespace bsmt
