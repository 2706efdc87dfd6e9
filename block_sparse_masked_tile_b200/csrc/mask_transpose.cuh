// q-side BlockMask lists and the block-level dense map.
//
// tensorplay.nn.attention page, BlockMask "Details" items 3-4: q_num_blocks /
// q_indices and full_q_num_blocks / full_q_indices are the transpose of the
// kv-side lists. For every kv block they hold the q blocks whose partial
// (resp. full) list contains it, ascending, followed by zeros.
//
// One CTA per (b, h, chunk of kv blocks): up to kTransposeChunk kv blocks, so
// that a (b, h) is scanned by few CTAs. Its warps read every q row's two
// lists of (b, h) and set one bit per (kv block of the chunk, q block) in two
// shared-memory bitmaps. The chunk's output columns are contiguous, so the
// whole CTA first zeroes them with 16-byte stores; then each thread takes one
// column and writes its set bits in ascending order over the zeros. Columns
// with more than 32 entries are left to a second pass in which a warp takes a
// column and a popc prefix over its words places every bit. The kernel writes
// every element of its output columns, so it is bound by the writes of
// [B, H, KB, QB] x 2 lists.
//
// BlockMask "Basics" (the reconstruction loop) defines the dense map: a
// block is 1 when either list of its row holds it.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace bsmt {

constexpr int kTransposeChunk = 256;  // kv blocks per CTA (at most)
constexpr int kTransposeThreads = 512;

struct TransposeParams {
    int32_t Bm, Hm, QB, KB;
    int32_t chunk;  // kv blocks per CTA
    const int32_t* kv_num;
    const int32_t* kv_idx;
    const int32_t* full_num;
    const int32_t* full_idx;
    int32_t* q_num;
    int32_t* q_idx;
    int32_t* full_q_num;
    int32_t* full_q_idx;
};

// Kv blocks per CTA: every kv block of a (b, h) when the grid still has at
// least half a CTA per SM, else KB split into as many chunks as that takes;
// at most kTransposeChunk, and few enough for the two bitmaps to stay within
// 96 KB of shared memory. (A (b, h) is scanned once per chunk: at B2 H32 with
// 256 x 256 blocks, two chunks measured faster than one or three.)
__host__ __device__ constexpr int transpose_chunk(int64_t QB, int64_t KB, int64_t BH, int64_t nsm) {
    const int64_t want = (nsm + 1) / 2;  // CTAs
    const int64_t per_bh = BH >= want ? 1 : (want + BH - 1) / (BH > 0 ? BH : 1);  // chunks per (b, h)
    int64_t c = (KB + per_bh - 1) / per_bh;
    const int64_t fit = (96 * 1024) / (2 * 4 * ((QB + 31) / 32 > 0 ? (QB + 31) / 32 : 1));
    c = c > fit ? fit : c;
    c = c > kTransposeChunk ? kTransposeChunk : c;
    return static_cast<int>(c < 1 ? 1 : c);
}

// Shared memory: two bitmaps of chunk x ceil(QB / 32) words.
__host__ __device__ constexpr int64_t transpose_smem_bytes(int64_t QB, int chunk) {
    return 2 * static_cast<int64_t>(chunk) * ((QB + 31) / 32) * 4 + (2 * chunk + 1) * 4;
}

__global__ void __launch_bounds__(kTransposeThreads) mask_transpose_kernel(const TransposeParams p) {
    // bitmaps [2][qw][chunk] (a column's words chunk apart, so that threads
    // reading one column each read consecutive words), then the count and
    // the list of dense columns for the second pass
    extern __shared__ uint32_t bits[];
    const int qw = (p.QB + 31) / 32;
    const int C = p.chunk;
    int* n_dense = reinterpret_cast<int*>(bits + 2 * C * qw);
    int* dense_cols = n_dense + 1;
    const int kb0 = blockIdx.x * C;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = kTransposeThreads / 32;
    for (int i = threadIdx.x; i < 2 * C * qw; i += kTransposeThreads) bits[i] = 0u;
    if (threadIdx.x == 0) *n_dense = 0;
    __syncthreads();

    // scatter: q row qb's kv blocks that fall into this chunk. A warp takes 32
    // rows at a time: lane r loads row r's two counts, then the warp loads the
    // first 32 entries of 8 rows' two lists per batch (16 independent loads in
    // flight, each coalesced along a row) before using any of them. Rows with
    // more than 32 entries finish in a second loop.
    const int64_t row0 = (static_cast<int64_t>(b) * p.Hm + h) * p.QB;
    bool bad = false;
    auto take = [&](int l, int qb, int kb) {
        if (kb < 0 || kb >= p.KB) {
            bad = true;
        } else if (kb >= kb0 && kb < kb0 + C) {
            atomicOr(&bits[(l * qw + (qb >> 5)) * C + (kb - kb0)], 1u << (qb & 31));
        }
    };
    for (int base = warp * 32; base < p.QB; base += nwarps * 32) {
        const int rows = (p.QB - base) < 32 ? (p.QB - base) : 32;
        int n0 = 0, n1 = 0;
        if (lane < rows) {
            n0 = __ldg(p.kv_num + row0 + base + lane);
            n1 = __ldg(p.full_num + row0 + base + lane);
            if (n0 < 0 || n0 > p.KB) {
                bad = true;
                n0 = 0;
            }
            if (n1 < 0 || n1 > p.KB) {
                bad = true;
                n1 = 0;
            }
        }
        for (int r0 = 0; r0 < rows; r0 += 8) {
            int v0[8], v1[8];
            bool h0[8], h1[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int r = r0 + k;
                const int c0 = __shfl_sync(0xFFFFFFFFu, n0, r & 31);
                const int c1 = __shfl_sync(0xFFFFFFFFu, n1, r & 31);
                const int64_t row = row0 + base + r;
                h0[k] = r < rows && lane < c0;
                h1[k] = r < rows && lane < c1;
                v0[k] = h0[k] ? __ldg(p.kv_idx + row * p.KB + lane) : 0;
                v1[k] = h1[k] ? __ldg(p.full_idx + row * p.KB + lane) : 0;
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                if (h0[k]) take(0, base + r0 + k, v0[k]);
                if (h1[k]) take(1, base + r0 + k, v1[k]);
            }
        }
        // entries past the first 32 of a row (dense rows)
        if (__any_sync(0xFFFFFFFFu, n0 > 32 || n1 > 32)) {
            for (int r = 0; r < rows; ++r) {
                const int c0 = __shfl_sync(0xFFFFFFFFu, n0, r);
                const int c1 = __shfl_sync(0xFFFFFFFFu, n1, r);
                const int64_t row = row0 + base + r;
                for (int j = 32 + lane; j < c0; j += 32) take(0, base + r, __ldg(p.kv_idx + row * p.KB + j));
                for (int j = 32 + lane; j < c1; j += 32) take(1, base + r, __ldg(p.full_idx + row * p.KB + j));
            }
        }
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) record_status(BSMT_ERR_DEVICE_BOUNDS);
    __syncthreads();

    // zero the chunk's columns of both lists: [kb0, kb0 + cols) x QB int32,
    // contiguous in each list
    const int cols = (p.KB - kb0) < C ? (p.KB - kb0) : C;
    const int64_t base_row = (static_cast<int64_t>(b) * p.Hm + h) * p.KB + kb0;
    const int64_t n_int = static_cast<int64_t>(cols) * p.QB;
#pragma unroll 1
    for (int l = 0; l < 2; ++l) {
        int32_t* blk = (l == 0 ? p.q_idx : p.full_q_idx) + base_row * p.QB;
        const uintptr_t a = reinterpret_cast<uintptr_t>(blk);
        int64_t head = static_cast<int64_t>(((16u - (a & 15u)) & 15u) >> 2);  // int32 slots to the boundary
        head = head < n_int ? head : n_int;
        if (threadIdx.x < head) blk[threadIdx.x] = 0;
        const int64_t nv = (n_int - head) >> 2;
        uint4* v = reinterpret_cast<uint4*>(blk + head);
        for (int64_t k = threadIdx.x; k < nv; k += kTransposeThreads) v[k] = make_uint4(0u, 0u, 0u, 0u);
        const int64_t tail = head + 4 * nv;
        if (tail + threadIdx.x < n_int) blk[tail + threadIdx.x] = 0;
    }
    __syncthreads();  // the entries below overwrite the zeros

    // one thread per (list, kv column): the set bits in ascending order
    for (int c = threadIdx.x; c < 2 * cols; c += kTransposeThreads) {
        const int l = c / cols;
        const int kc = c - l * cols;
        const uint32_t* col = bits + l * qw * C + kc;
        int count = 0;
        for (int w = 0; w < qw; ++w) count += __popc(col[w * C]);
        const int64_t orow = base_row + kc;
        if (count > 32) {  // a dense column: the second pass writes it
            dense_cols[atomicAdd(n_dense, 1)] = c;
        } else {
            int32_t* out = (l == 0 ? p.q_idx : p.full_q_idx) + orow * p.QB;
            int pos = 0;
            for (int w = 0; w < qw && pos < count; ++w) {
                uint32_t rest = col[w * C];
                while (rest) {
                    out[pos++] = w * 32 + __ffs(rest) - 1;
                    rest &= rest - 1u;
                }
            }
        }
        (l == 0 ? p.q_num : p.full_q_num)[orow] = count;
    }
    __syncthreads();
    // dense columns: one warp per column; lane takes word w0 + lane, its bits'
    // positions following the set bits of the lower lanes' words
    const int nd = *n_dense;
    for (int d = warp; d < nd; d += nwarps) {
        const int c = dense_cols[d];
        const int l = c / cols;
        const int kc = c - l * cols;
        const uint32_t* col = bits + l * qw * C + kc;
        int32_t* out = (l == 0 ? p.q_idx : p.full_q_idx) + (base_row + kc) * p.QB;
        int pos = 0;
        for (int w0 = 0; w0 < qw; w0 += 32) {
            const uint32_t word = (w0 + lane < qw) ? col[(w0 + lane) * C] : 0u;
            const int cnt = __popc(word);
            int incl = cnt;
#pragma unroll
            for (int dd = 1; dd < 32; dd <<= 1) {
                const int v = __shfl_up_sync(0xFFFFFFFFu, incl, dd);
                if (lane >= dd) incl += v;
            }
            int at = pos + incl - cnt;
            uint32_t rest = word;
            while (rest) {
                out[at++] = (w0 + lane) * 32 + __ffs(rest) - 1;
                rest &= rest - 1u;
            }
            pos += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
    }
}

struct DenseParams {
    int32_t Bm, Hm, QB, KB;
    const int32_t* kv_num;
    const int32_t* kv_idx;
    const int32_t* full_num;
    const int32_t* full_idx;
    int32_t* dense;  // [B, H, QB, KB]
};

// One warp per (b, h, q row): zero the row, then set the listed blocks. The
// warp's own writes are ordered by __syncwarp.
__global__ void __launch_bounds__(128) mask_to_dense_kernel(const DenseParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t rows = static_cast<int64_t>(p.Bm) * p.Hm * p.QB;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + warp;
    if (row >= rows) return;
    int32_t* out = p.dense + row * p.KB;
    for (int j = lane; j < p.KB; j += 32) out[j] = 0;
    __syncwarp();
    bool bad = false;
#pragma unroll
    for (int l = 0; l < 2; ++l) {
        int n = __ldg((l == 0 ? p.kv_num : p.full_num) + row);
        if (n < 0 || n > p.KB) {
            bad = true;
            n = 0;
        }
        const int32_t* idx = (l == 0 ? p.kv_idx : p.full_idx) + row * p.KB;
        for (int j = lane; j < n; j += 32) {
            const int kb = __ldg(idx + j);
            if (kb < 0 || kb >= p.KB)
                bad = true;
            else
                out[kb] = 1;
        }
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) record_status(BSMT_ERR_DEVICE_BOUNDS);
}

}  // namespace bsmt
