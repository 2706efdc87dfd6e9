// Packed variable-length sequences (cu_seqlens form).
//
// The L-GATr "attention backends" page describes packing the events of a
// batch into one sequence with a block-diagonal mask, and the cu_seqlens
// form of the varlen kernels (cu_seqlens_q / max_seqlen_q). Here a packed
// batch is one sequence whose tokens carry their sequence's ordinal as a
// document id; the DOCUMENT mask (with CAUSAL for causal attention) then
// gives each token exactly the keys of its own sequence.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace bsmt {

// doc_ids[t] = i for cu[i] <= t < cu[i+1]; tokens at or past cu[num_seqs]
// get num_seqs. cu must start at 0 and not decrease, else the status word
// records BSMT_ERR_DEVICE_PRECONDITION (the ids are still written).
__global__ void __launch_bounds__(256) seqlens_to_doc_ids_kernel(const int32_t* cu, int32_t num_seqs, int64_t total,
                                                                 int32_t* doc_ids) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t first = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (first == 0) {
        bool bad = __ldg(cu) != 0;
        for (int i = 0; i < num_seqs; ++i) bad = bad || __ldg(cu + i) > __ldg(cu + i + 1);
        if (bad) record_status(BSMT_ERR_DEVICE_PRECONDITION);
    }
    for (int64_t t = first; t < total; t += stride) {
        // largest i in [0, num_seqs] with cu[i] <= t
        int lo = 0, hi = num_seqs;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (__ldg(cu + mid) <= t)
                lo = mid;
            else
                hi = mid - 1;
        }
        doc_ids[t] = lo;
    }
}

}  // namespace bsmt
