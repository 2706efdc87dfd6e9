// Mask programs in disjunctive normal form.
//
// Each primitive of the mask set (tensorplay.nn.attention: noop_mask, the
// causal example, and_masks/or_masks; L-GATr page: sliding window, PrefixLM,
// block-diagonal documents; transformerlab page: StreamingLLM sink) allows
// one contiguous interval of kv positions for a fixed query row q:
//   CAUSAL       kv <= q
//   WINDOW(W)    kv >= q - W + 1
//   PREFIX_LM(P) kv <= max(P - 1, q)
//   SINK(S)      kv <= S - 1
//   DOCUMENT     kv in [first, last] position of q's document id (kv ids sorted)
//   NOOP         everything
// The host distributes AND over OR, turning the postfix program into an OR
// of at most kMaxTerms AND-terms. Each AND-term then allows exactly one
// interval per row, so a row's allowed set is a union of at most kMaxTerms
// intervals. This is exact, and cheap to turn into tile classes (builder) or
// 32-column bit masks (attention kernel).
#pragma once
#include <cstdint>
#include <climits>

#include "bsmt.h"

namespace bsmt {

constexpr int kMaxTerms = BSMT_MAX_MASK_TERMS;

// One AND-term in canonical form: at most one leaf of each kind (the host
// keeps the strictest), so a term is a set of flags and three arguments.
constexpr uint32_t kTermCausal = 1u, kTermWindow = 2u, kTermPrefix = 4u, kTermSink = 8u, kTermDoc = 16u;

struct DnfTerm {
    uint32_t flags;    // kTerm* bits; 0 is NOOP
    int32_t w, pf, s;  // the WINDOW W, PREFIX_LM P and SINK S of the term, when flagged
};

struct MaskDnf {
    int32_t n_terms;        // 0 means "nothing allowed"
    uint32_t term_has_doc;  // bit t: term t has a DOCUMENT leaf
    DnfTerm terms[kMaxTerms];
    const int32_t* q_doc;
    const int32_t* kv_doc;
    int32_t doc_batch;
    int32_t has_doc;
};

// Interval allowed by term t for row q, clamped to [lo0, hi0], using the
// row's document interval [ds, de] when the term has a DOCUMENT leaf
// (64-bit, so that extreme W / P / S values cannot overflow). The term's
// fields are read together, with no dependence between them.
__device__ __forceinline__ void term_interval(const MaskDnf& m, int t, int64_t q, int64_t lo0, int64_t hi0,
                                              int64_t ds, int64_t de, int64_t& lo, int64_t& hi) {
    const DnfTerm tm = m.terms[t];
    lo = lo0;
    hi = hi0;
    if (tm.flags & kTermCausal) hi = hi < q ? hi : q;
    if (tm.flags & kTermWindow) {
        const int64_t l = q - static_cast<int64_t>(tm.w) + 1;
        lo = lo > l ? lo : l;
    }
    if (tm.flags & kTermPrefix) {
        const int64_t pm1 = static_cast<int64_t>(tm.pf) - 1;
        const int64_t h = pm1 > q ? pm1 : q;
        hi = hi < h ? hi : h;
    }
    if (tm.flags & kTermSink) {
        const int64_t h = static_cast<int64_t>(tm.s) - 1;
        hi = hi < h ? hi : h;
    }
    if (tm.flags & kTermDoc) {
        lo = lo > ds ? lo : ds;
        hi = hi < de ? hi : de;
    }
}

// Bits [a, b] (inclusive, relative to base) inside one 32-bit word.
__device__ __forceinline__ uint32_t range_bits(int64_t a, int64_t b, int64_t base) {
    int64_t lo = a - base;
    int64_t hi = b - base;
    lo = lo < 0 ? 0 : lo;
    hi = hi > 31 ? 31 : hi;
    if (lo > hi) return 0u;
    const uint32_t upto = (hi == 31) ? 0xFFFFFFFFu : ((1u << static_cast<uint32_t>(hi + 1)) - 1u);
    return upto & ~((1u << static_cast<uint32_t>(lo)) - 1u);
}

// Bits [a, b] of a 32-bit word (positions relative to the word; 32-bit math).
__device__ __forceinline__ uint32_t range_bits32(int a, int b) {
    a = a < 0 ? 0 : a;
    b = b > 31 ? 31 : b;
    if (a > b) return 0u;
    return (0xFFFFFFFFu >> (31 - b)) & (0xFFFFFFFFu << a);
}

// First index i in [0, n) with a[i] >= x (n if none). a is non-decreasing
// and x is uniform over the warp. 33-way split per step (32 probes).
__device__ __forceinline__ int warp_lower_bound(const int32_t* a, int n, int64_t x, int lane) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int len = hi - lo;
        const int p = lo + static_cast<int>((static_cast<int64_t>(lane + 1) * len) / 33);
        const int64_t v = (p < hi) ? static_cast<int64_t>(__ldg(a + p)) : INT64_MAX;
        const unsigned ge = __ballot_sync(0xFFFFFFFFu, v >= x);
        if (ge == 0u) {
            lo = lo + static_cast<int>((static_cast<int64_t>(32) * len) / 33) + 1;
        } else {
            const int f = __ffs(ge) - 1;
            const int pf = lo + static_cast<int>((static_cast<int64_t>(f + 1) * len) / 33);
            const int pprev = (f == 0) ? lo - 1 : lo + static_cast<int>((static_cast<int64_t>(f) * len) / 33);
            hi = pf;
            lo = pprev + 1;
        }
    }
    return lo;
}

}  // namespace bsmt
