// libbsmt: the C ABI declared in include/bsmt.h.
//
// Host side: argument checks, conversion of the postfix mask program into
// OR-of-AND form, TMA descriptor encoding and kernel launches. Nothing here
// allocates device memory and nothing synchronizes, except
// bsmt_check_device_status.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "attn_bwd.cuh"
#include "attn_fwd.cuh"
#include "bsmt.h"
#include "mask_build.cuh"
#include "mask_transpose.cuh"
#include "varlen.cuh"
#include "mask_dnf.cuh"
#include "ptx.cuh"
#include "selftest.cuh"

namespace {

thread_local std::string g_last_error;

bsmt_status fail(bsmt_status code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

bsmt_status ok() {
    g_last_error.clear();
    return BSMT_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int64_t kMaxLen = (int64_t(1) << 31) - 256;

// ------------------------------------------------------------------ DNF
// One AND-term of the mask program in canonical form. Leaves of one kind in
// a term collapse to the strictest: CAUSAL and DOCUMENT are idempotent, and
// for the others the smaller argument allows a subset of rows' keys
// (WINDOW(W): kv >= q - W + 1; PREFIX_LM(P): kv <= max(P - 1, q); SINK(S):
// kv <= S - 1). So a term is at most one leaf of each kind, and the empty
// term is NOOP.
struct Term {
    bool causal = false, doc = false, has_w = false, has_p = false, has_s = false;
    int32_t w = 0, pf = 0, s = 0;
    bool operator==(const Term& o) const {
        return causal == o.causal && doc == o.doc && has_w == o.has_w && has_p == o.has_p && has_s == o.has_s &&
               (!has_w || w == o.w) && (!has_p || pf == o.pf) && (!has_s || s == o.s);
    }
};

Term leaf_term(int32_t kind, int32_t arg) {
    Term t;
    switch (kind) {
        case BSMT_MASK_CAUSAL: t.causal = true; break;
        case BSMT_MASK_DOCUMENT: t.doc = true; break;
        case BSMT_MASK_WINDOW: t.has_w = true; t.w = arg; break;
        case BSMT_MASK_PREFIX_LM: t.has_p = true; t.pf = arg; break;
        case BSMT_MASK_SINK: t.has_s = true; t.s = arg; break;
        default: break;  // NOOP
    }
    return t;
}

// a AND b
Term term_and(const Term& a, const Term& b) {
    Term t = a;
    t.causal = a.causal || b.causal;
    t.doc = a.doc || b.doc;
    if (b.has_w) t.w = a.has_w ? std::min(a.w, b.w) : b.w;
    if (b.has_p) t.pf = a.has_p ? std::min(a.pf, b.pf) : b.pf;
    if (b.has_s) t.s = a.has_s ? std::min(a.s, b.s) : b.s;
    t.has_w = a.has_w || b.has_w;
    t.has_p = a.has_p || b.has_p;
    t.has_s = a.has_s || b.has_s;
    return t;
}

// Every key `inner` allows, `outer` allows too: each of outer's leaves has a
// leaf of the same kind in inner that is at least as strict.
bool term_within(const Term& inner, const Term& outer) {
    if (outer.causal && !inner.causal) return false;
    if (outer.doc && !inner.doc) return false;
    if (outer.has_w && !(inner.has_w && inner.w <= outer.w)) return false;
    if (outer.has_p && !(inner.has_p && inner.pf <= outer.pf)) return false;
    if (outer.has_s && !(inner.has_s && inner.s <= outer.s)) return false;
    return true;
}

// The same union of terms without repeats and without terms that another
// term contains.
void simplify(std::vector<Term>& terms) {
    std::vector<Term> uniq;
    for (const Term& t : terms)
        if (std::find(uniq.begin(), uniq.end(), t) == uniq.end()) uniq.push_back(t);
    std::vector<Term> out;
    for (size_t i = 0; i < uniq.size(); ++i) {
        bool inside = false;
        for (size_t j = 0; j < uniq.size() && !inside; ++j) inside = j != i && term_within(uniq[i], uniq[j]);
        if (!inside) out.push_back(uniq[i]);
    }
    terms = std::move(out);
}

// Terms held while the program is evaluated; only the final count must fit
// kMaxTerms, since later ANDs and ORs can merge terms again.
constexpr size_t kMaxWorkTerms = 1024;
static_assert(5 * BSMT_MAX_MASK_TERMS <= BSMT_MAX_MASK_LEAVES, "a canonical term has at most one leaf of each of 5 kinds");

bsmt_status build_dnf(const bsmt_mask_spec* spec, int64_t B, bsmt::MaskDnf* out) {
    std::memset(out, 0, sizeof(*out));
    if (spec == nullptr) {  // NOOP: one term without leaves
        out->n_terms = 1;
        return BSMT_OK;
    }
    if (spec->num_nodes < 1 || spec->num_nodes > BSMT_MAX_MASK_NODES)
        return fail(BSMT_ERR_INVALID_ARGUMENT, "mask spec: num_nodes=%d outside [1, %d]", spec->num_nodes,
                    BSMT_MAX_MASK_NODES);
    std::vector<std::vector<Term>> stack;
    bool has_doc = false;
    for (int i = 0; i < spec->num_nodes; ++i) {
        const bsmt_mask_node nd = spec->nodes[i];
        switch (nd.kind) {
            case BSMT_MASK_NOOP:
            case BSMT_MASK_CAUSAL:
            case BSMT_MASK_WINDOW:
            case BSMT_MASK_PREFIX_LM:
            case BSMT_MASK_SINK:
            case BSMT_MASK_DOCUMENT:
                if (nd.kind == BSMT_MASK_DOCUMENT) has_doc = true;
                stack.push_back({leaf_term(nd.kind, nd.arg)});
                break;
            case BSMT_MASK_AND:
            case BSMT_MASK_OR: {
                if (nd.arg < 1 || size_t(nd.arg) > stack.size())
                    return fail(BSMT_ERR_INVALID_ARGUMENT, "mask spec: node %d (%s) takes %d operands, %zu available", i,
                                nd.kind == BSMT_MASK_AND ? "AND" : "OR", nd.arg, stack.size());
                std::vector<std::vector<Term>> ops(stack.end() - nd.arg, stack.end());
                stack.resize(stack.size() - nd.arg);
                std::vector<Term> res;
                if (nd.kind == BSMT_MASK_OR) {
                    for (auto& d : ops) res.insert(res.end(), d.begin(), d.end());
                    simplify(res);
                } else {
                    res = {Term{}};
                    for (auto& d : ops) {
                        std::vector<Term> nxt;
                        for (auto& a : res)
                            for (auto& b : d) nxt.push_back(term_and(a, b));
                        simplify(nxt);
                        res = std::move(nxt);
                        if (res.size() > kMaxWorkTerms) break;
                    }
                }
                if (res.size() > kMaxWorkTerms)
                    return fail(BSMT_ERR_UNSUPPORTED, "mask spec: more than %zu alternatives while distributing AND over OR",
                                kMaxWorkTerms);
                stack.push_back(std::move(res));
                break;
            }
            default:
                return fail(BSMT_ERR_INVALID_ARGUMENT, "mask spec: node %d has unknown kind %d", i, nd.kind);
        }
    }
    if (stack.size() != 1)
        return fail(BSMT_ERR_INVALID_ARGUMENT, "mask spec: program leaves %zu values (expected 1)", stack.size());
    const std::vector<Term>& terms = stack[0];
    if (terms.size() > size_t(bsmt::kMaxTerms))
        return fail(BSMT_ERR_UNSUPPORTED, "mask spec: %zu alternatives after distributing AND over OR (at most %d)",
                    terms.size(), bsmt::kMaxTerms);
    if (has_doc) {
        if (spec->q_doc_ids == nullptr || spec->kv_doc_ids == nullptr)
            return fail(BSMT_ERR_INVALID_ARGUMENT, "mask spec: DOCUMENT needs q_doc_ids and kv_doc_ids");
        if (!aligned(spec->q_doc_ids, 4) || !aligned(spec->kv_doc_ids, 4))
            return fail(BSMT_ERR_INVALID_ARGUMENT, "mask spec: document id arrays must be 4-byte aligned");
        if (!(spec->doc_batch == 1 || spec->doc_batch == B))
            return fail(BSMT_ERR_SHAPE_MISMATCH, "mask spec: doc_batch=%d must be 1 or B=%lld", spec->doc_batch,
                        static_cast<long long>(B));
    }
    out->n_terms = static_cast<int32_t>(terms.size());
    for (size_t t = 0; t < terms.size(); ++t) {
        const Term& tm = terms[t];
        bsmt::DnfTerm& d = out->terms[t];
        d.flags = (tm.causal ? bsmt::kTermCausal : 0u) | (tm.has_w ? bsmt::kTermWindow : 0u) |
                  (tm.has_p ? bsmt::kTermPrefix : 0u) | (tm.has_s ? bsmt::kTermSink : 0u) |
                  (tm.doc ? bsmt::kTermDoc : 0u);
        d.w = tm.w;
        d.pf = tm.pf;
        d.s = tm.s;
        if (tm.doc) out->term_has_doc |= 1u << t;
    }
    // a program whose DOCUMENT leaves all fell inside other terms needs no ids
    out->has_doc = out->term_has_doc != 0u ? 1 : 0;
    out->q_doc = spec->q_doc_ids;
    out->kv_doc = spec->kv_doc_ids;
    out->doc_batch = spec->doc_batch < 1 ? 1 : spec->doc_batch;
    return BSMT_OK;
}

// ------------------------------------------------------------- device info
std::mutex g_mu;
int g_sm_count[64] = {0};
bool g_attr_set[64][32] = {{false}};

bsmt_status sm_count(int* dev_out, int* n_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return fail(BSMT_ERR_UNSUPPORTED, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_sm_count[dev] == 0) {
        int major = 0, minor = 0, n = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
        if (major != 10 || minor != 0)
            return fail(BSMT_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a (B200)", dev,
                        major, minor);
        g_sm_count[dev] = n;
    }
    *dev_out = dev;
    *n_out = g_sm_count[dev];
    return BSMT_OK;
}

// ------------------------------------------------------------ static scratch
// Device scratch of the allocation-free split-KV entry point: a file-scope
// array, so that call allocates nothing. Its address is looked up once per
// device and kept.
static __device__ __align__(256) unsigned char g_splitkv_scratch[BSMT_SPLITKV_SCRATCH_BYTES];
void* g_scratch_addr[64] = {};

bsmt_status scratch_address(int dev, void** addr) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* ptr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ptr, g_splitkv_scratch);
        if (e != cudaSuccess || ptr == nullptr)
            return fail(BSMT_ERR_CUDA, "cudaGetSymbolAddress(split-KV scratch): %s", cudaGetErrorString(e));
        g_scratch_addr[dev] = ptr;
    }
    *addr = g_scratch_addr[dev];
    return BSMT_OK;
}

// ------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bsmt_status get_encoder(EncodeTiledFn* fn) {
    static EncodeTiledFn cached = nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (cached == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q);
        if (e != cudaSuccess || ptr == nullptr || q != cudaDriverEntryPointSuccess)
            return fail(BSMT_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
        cached = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    *fn = cached;
    return BSMT_OK;
}

// bf16 tensor of (BH, S, D) as a 3-D map with 64 x 128 x 1 boxes and 128-byte
// swizzle. Row s of head bh starts at base + (bh * sbh + s * ss) elements:
// (S*D, D) for [BH, S, D], (D, H*D) for a packed [S, H, D].
bsmt_status encode_bhsd(EncodeTiledFn enc, CUtensorMap* map, const void* base, int64_t BH, int64_t S, int64_t D,
                        int64_t sbh, int64_t ss) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(ss * 2), static_cast<cuuint64_t>(sbh * 2)};
    const cuuint32_t box[3] = {64, 128, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(BSMT_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return BSMT_OK;
}

// out [BH, S, D] bf16 as a 3-D map with 32 x 32 x 1 boxes (64-byte rows) and
// 64-byte swizzle; the attention epilogue stores through it.
bsmt_status encode_out(EncodeTiledFn enc, CUtensorMap* map, void* base, int64_t BH, int64_t S, int64_t D,
                       int64_t sbh, int64_t ss) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(ss * 2), static_cast<cuuint64_t>(sbh * 2)};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(BSMT_ERR_CUDA, "cuTensorMapEncodeTiled (out) failed (%d)", static_cast<int>(r));
    return BSMT_OK;
}

// Rows with no allowed key: out = 0, lse = -inf (used when KV_LEN == 0).
__global__ void fill_empty_kernel(uint4* out, int64_t out_vec, float* lse, int64_t rows) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < out_vec; i += stride)
        out[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < rows; i += stride)
        lse[i] = -INFINITY;
}

// Score mods -> compile-time mode (kScore*), the soft-cap and the ALiBi slopes
// (explicit, or the default ones of heads h0 .. h0 + Hq - 1 of a model of
// `heads` heads).
struct ScoreArgs {
    int mode = bsmt::kScoreNone;
    float cap = 1.f;
    const float* slopes = nullptr;
    int32_t alibi_h0 = 0, alibi_heads = 1;
};

bsmt_status parse_score(const bsmt_score_spec* score, int64_t Hq, ScoreArgs* out_args) {
    int mode = bsmt::kScoreNone;
    float cap = 1.f;
    const float* slopes = nullptr;
    int32_t h0 = 0;
    int64_t heads = Hq;
    if (score != nullptr) {
        if (score->num_ops < 0 || score->num_ops > BSMT_MAX_SCORE_OPS)
            return fail(BSMT_ERR_INVALID_ARGUMENT, "score spec: num_ops=%d outside [0, %d]", score->num_ops, BSMT_MAX_SCORE_OPS);
        int kinds[2] = {0, 0};
        int nk = 0;
        for (int i = 0; i < score->num_ops; ++i) {
            const bsmt_score_op& op = score->ops[i];
            if (op.kind == BSMT_SCORE_NONE) continue;
            if (op.kind == BSMT_SCORE_SOFTCAP) {
                if (!(op.value > 0.f) || std::isinf(op.value))
                    return fail(BSMT_ERR_INVALID_ARGUMENT, "score spec: soft-cap must be finite and > 0");
                cap = op.value;
            } else if (op.kind == BSMT_SCORE_ALIBI) {
                if (op.slopes && !aligned(op.slopes, 4))
                    return fail(BSMT_ERR_INVALID_ARGUMENT, "score spec: ALiBi slopes must be 4-byte aligned");
                slopes = op.slopes;
                if (slopes == nullptr) {
                    if (op.num_heads <= 0) {
                        if (op.head_offset != 0)
                            return fail(BSMT_ERR_INVALID_ARGUMENT,
                                        "score spec: ALiBi head_offset=%d needs num_heads (the model's head count)",
                                        op.head_offset);
                    } else if (op.head_offset < 0 || op.head_offset + Hq > op.num_heads) {
                        return fail(BSMT_ERR_INVALID_ARGUMENT,
                                    "score spec: ALiBi heads [%d, %lld) outside the model's %d heads", op.head_offset,
                                    static_cast<long long>(op.head_offset + Hq), op.num_heads);
                    } else {
                        h0 = op.head_offset;
                        heads = op.num_heads;
                    }
                }
            } else {
                return fail(BSMT_ERR_INVALID_ARGUMENT, "score spec: unknown kind %d", op.kind);
            }
            if (nk == 1 && kinds[0] == op.kind)
                return fail(BSMT_ERR_UNSUPPORTED, "score spec: the same score mod twice");
            kinds[nk++] = op.kind;
        }
        if (nk == 1) mode = kinds[0] == BSMT_SCORE_SOFTCAP ? bsmt::kScoreSoftcap : bsmt::kScoreAlibi;
        if (nk == 2) mode = kinds[0] == BSMT_SCORE_SOFTCAP ? bsmt::kScoreSoftcapAlibi : bsmt::kScoreAlibiSoftcap;
    }
    out_args->mode = mode;
    out_args->cap = cap;
    out_args->slopes = slopes;
    out_args->alibi_h0 = h0;
    out_args->alibi_heads = static_cast<int32_t>(heads > 0 ? heads : 1);
    return BSMT_OK;
}

template <int D, int SCORE, bool LONG>
bsmt_status launch_attn_kind(int dev, int nsm, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to, const bsmt::AttnParams& p, const bsmt::MaskDnf& dnf,
                             cudaStream_t stream) {
    auto kern = bsmt::attn_fwd_kernel<D, SCORE, LONG>;
    const int smem = bsmt::SmemLayout<D>::kAlloc;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        const int slot = (LONG ? 16 : 0) + (D == 128 ? 8 : 0) + SCORE;
        if (!g_attr_set[dev][slot]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
            g_attr_set[dev][slot] = true;
        }
    }
    const int grid = p.num_units < nsm ? p.num_units : nsm;
    kern<<<grid, bsmt::kThreads, smem, stream>>>(tq, tk, tv, to, p, dnf);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "attention launch: %s", cudaGetErrorString(e));
    return BSMT_OK;
}

// Rows of more than kMaxKB kv blocks take the kernel's windowed variant.
template <int D, int SCORE>
bsmt_status launch_attn(int dev, int nsm, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const CUtensorMap& to, const bsmt::AttnParams& p, const bsmt::MaskDnf& dnf,
                        cudaStream_t stream) {
    if (p.KB > bsmt::kMaxKB) return launch_attn_kind<D, SCORE, true>(dev, nsm, tq, tk, tv, to, p, dnf, stream);
    return launch_attn_kind<D, SCORE, false>(dev, nsm, tq, tk, tv, to, p, dnf, stream);
}

template <int D>
bsmt_status launch_attn_score(int score, int dev, int nsm, const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv, const CUtensorMap& to, const bsmt::AttnParams& p,
                              const bsmt::MaskDnf& dnf, cudaStream_t s) {
    switch (score) {
        case bsmt::kScoreNone: return launch_attn<D, bsmt::kScoreNone>(dev, nsm, tq, tk, tv, to, p, dnf, s);
        case bsmt::kScoreSoftcap: return launch_attn<D, bsmt::kScoreSoftcap>(dev, nsm, tq, tk, tv, to, p, dnf, s);
        case bsmt::kScoreAlibi: return launch_attn<D, bsmt::kScoreAlibi>(dev, nsm, tq, tk, tv, to, p, dnf, s);
        case bsmt::kScoreSoftcapAlibi:
            return launch_attn<D, bsmt::kScoreSoftcapAlibi>(dev, nsm, tq, tk, tv, to, p, dnf, s);
        default: return launch_attn<D, bsmt::kScoreAlibiSoftcap>(dev, nsm, tq, tk, tv, to, p, dnf, s);
    }
}

}  // namespace

extern "C" {

int32_t bsmt_version(void) { return (2 << 16) | 1; }

const char* bsmt_last_error(void) { return g_last_error.c_str(); }

bsmt_status bsmt_block_mask_shape(int64_t B, int64_t H, int64_t Q_LEN, int64_t KV_LEN, int32_t BLOCK_Q,
                                  int32_t BLOCK_KV, int64_t out_shape[4]) {
    if (out_shape == nullptr) return fail(BSMT_ERR_INVALID_ARGUMENT, "out_shape is NULL");
    if (BLOCK_Q != 128 || BLOCK_KV != 128)
        return fail(BSMT_ERR_UNSUPPORTED, "BLOCK_SIZE (%d, %d): only 128 x 128 blocks are supported", BLOCK_Q, BLOCK_KV);
    if (Q_LEN < 0 || KV_LEN < 0 || Q_LEN > kMaxLen || KV_LEN > kMaxLen)
        return fail(BSMT_ERR_INVALID_ARGUMENT, "Q_LEN=%lld KV_LEN=%lld outside [0, %lld]", static_cast<long long>(Q_LEN),
                    static_cast<long long>(KV_LEN), static_cast<long long>(kMaxLen));
    out_shape[0] = B > 0 ? B : 1;
    out_shape[1] = H > 0 ? H : 1;
    out_shape[2] = (Q_LEN + BLOCK_Q - 1) / BLOCK_Q;
    out_shape[3] = (KV_LEN + BLOCK_KV - 1) / BLOCK_KV;
    return ok();
}

bsmt_status bsmt_create_block_mask(const bsmt_mask_spec* spec, int64_t B, int64_t H, int64_t Q_LEN, int64_t KV_LEN,
                                   int32_t BLOCK_Q, int32_t BLOCK_KV, bsmt_block_mask* out, void* stream) {
    int64_t shape[4];
    bsmt_status st = bsmt_block_mask_shape(B, H, Q_LEN, KV_LEN, BLOCK_Q, BLOCK_KV, shape);
    if (st != BSMT_OK) return st;
    if (spec == nullptr) return fail(BSMT_ERR_INVALID_ARGUMENT, "mask spec is NULL");
    if (out == nullptr) return fail(BSMT_ERR_INVALID_ARGUMENT, "block mask output is NULL");
    if (shape[0] > 65535) return fail(BSMT_ERR_UNSUPPORTED, "B=%lld above 65535", static_cast<long long>(shape[0]));
    if (shape[1] > (int64_t(1) << 20)) return fail(BSMT_ERR_UNSUPPORTED, "H=%lld too large", static_cast<long long>(shape[1]));
    const int64_t rows = shape[0] * shape[1] * shape[2];
    if (rows > 0) {
        if (!out->kv_num_blocks || !out->full_kv_num_blocks || (shape[3] > 0 && (!out->kv_indices || !out->full_kv_indices)))
            return fail(BSMT_ERR_INVALID_ARGUMENT, "block mask output pointers must be non-NULL");
        if (!aligned(out->kv_num_blocks, 4) || !aligned(out->kv_indices, 4) || !aligned(out->full_kv_num_blocks, 4) ||
            !aligned(out->full_kv_indices, 4))
            return fail(BSMT_ERR_INVALID_ARGUMENT, "block mask output pointers must be 4-byte aligned");
    }
    bsmt::MaskDnf dnf;
    st = build_dnf(spec, shape[0], &dnf);
    if (st != BSMT_OK) return st;
    int dev = 0, nsm = 0;
    if (rows > 0) {
        st = sm_count(&dev, &nsm);
        if (st != BSMT_OK) return st;
    }
    out->B = static_cast<int32_t>(shape[0]);
    out->H = static_cast<int32_t>(shape[1]);
    out->QB = static_cast<int32_t>(shape[2]);
    out->KB = static_cast<int32_t>(shape[3]);
    out->Q_LEN = static_cast<int32_t>(Q_LEN);
    out->KV_LEN = static_cast<int32_t>(KV_LEN);
    out->BLOCK_Q = BLOCK_Q;
    out->BLOCK_KV = BLOCK_KV;
    if (rows == 0) return ok();

    bsmt::BuildParams p;
    p.Bm = out->B;
    p.Hm = out->H;
    p.Q_LEN = out->Q_LEN;
    p.KV_LEN = out->KV_LEN;
    p.QB = out->QB;
    p.KB = out->KB;
    p.kv_num = out->kv_num_blocks;
    p.kv_idx = out->kv_indices;
    p.full_num = out->full_kv_num_blocks;
    p.full_idx = out->full_kv_indices;
    const int64_t gx = p.QB;  // one block per q-block row
    const int64_t blocks_xy = gx * p.Bm;
    int64_t groups = (2 * nsm + blocks_xy - 1) / blocks_xy;
    if (groups < 1) groups = 1;
    if (groups > p.Hm) groups = p.Hm;
    p.heads_per_block = static_cast<int32_t>((p.Hm + groups - 1) / groups);
    groups = (p.Hm + p.heads_per_block - 1) / p.heads_per_block;
    if (gx > 0x7FFFFFFF || groups > 65535) return fail(BSMT_ERR_UNSUPPORTED, "grid too large");
    dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(p.Bm), static_cast<unsigned>(groups));
    // Rows staged in shared memory and written by bulk copies when their size
    // and the lists' alignment allow it.
    const bool staged = p.KB > 0 && p.KB % 4 == 0 && p.KB <= bsmt::kStagedMaxKB && aligned(p.kv_idx, 16) &&
                        aligned(p.full_idx, 16);
    if (staged)
        bsmt::mask_build_kernel<true><<<grid, bsmt::kBuildWarps * 32, 2 * p.KB * 4, static_cast<cudaStream_t>(stream)>>>(
            dnf, p);
    else
        bsmt::mask_build_kernel<false><<<grid, bsmt::kBuildWarps * 32, 0, static_cast<cudaStream_t>(stream)>>>(dnf, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "mask builder launch: %s", cudaGetErrorString(e));
    return ok();
}

}  // extern "C"

namespace {
// The attention path. num_splits > 1 runs split-KV into the workspace
// (ws_o, ws_lse, already checked) and merges the slices into out and lse.
bsmt_status attention(const void* q, const void* k, const void* v, int64_t B, int64_t Hq, int64_t Hkv, int64_t M,
                      int64_t N, int64_t D, const bsmt_block_mask* bm, const bsmt_mask_spec* mask_spec,
                      const bsmt_score_spec* score, float scale, int32_t enable_gqa, int num_splits, float* ws_o,
                      float* ws_lse, void* out, float* lse, void* stream, bool packed = false,
                      bool dry_run = false) {
    if (B < 0 || Hq < 0 || Hkv < 0 || M < 0 || N < 0)
        return fail(BSMT_ERR_INVALID_ARGUMENT, "negative size (B=%lld Hq=%lld Hkv=%lld M=%lld N=%lld)",
                    static_cast<long long>(B), static_cast<long long>(Hq), static_cast<long long>(Hkv),
                    static_cast<long long>(M), static_cast<long long>(N));
    if (D != 64 && D != 128) return fail(BSMT_ERR_UNSUPPORTED, "head dim D=%lld (supported: 64, 128)", static_cast<long long>(D));
    if (Hkv < 1 || Hq < 1) return fail(BSMT_ERR_SHAPE_MISMATCH, "Hq=%lld and Hkv=%lld must be >= 1", static_cast<long long>(Hq), static_cast<long long>(Hkv));
    if (Hq % Hkv != 0)
        return fail(BSMT_ERR_SHAPE_MISMATCH, "Hq=%lld is not a multiple of Hkv=%lld", static_cast<long long>(Hq),
                    static_cast<long long>(Hkv));
    if (Hq != Hkv && !enable_gqa)
        return fail(BSMT_ERR_SHAPE_MISMATCH, "Hq=%lld != Hkv=%lld requires enable_gqa", static_cast<long long>(Hq),
                    static_cast<long long>(Hkv));
    if (M > kMaxLen || N > kMaxLen) return fail(BSMT_ERR_UNSUPPORTED, "sequence length above %lld", static_cast<long long>(kMaxLen));
    if (B * Hq > 0x7FFFFFFF || B * Hkv > 0x7FFFFFFF) return fail(BSMT_ERR_UNSUPPORTED, "B*H above 2^31");
    const int64_t QB = (M + 127) / 128, KB = (N + 127) / 128;
    // a tensor with no elements may be passed as NULL (its pointer is never used)
    const bool q_has = B * Hq * M > 0, kv_has = B * Hkv * N > 0;
    if ((q_has && (!q || !out || !lse)) || (kv_has && (!k || !v)))
        return fail(BSMT_ERR_INVALID_ARGUMENT, "q, k, v, out and lse must be non-NULL when they hold elements");
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
        return fail(BSMT_ERR_INVALID_ARGUMENT, "q, k, v and out must be 16-byte aligned");
    if (!aligned(lse, 4)) return fail(BSMT_ERR_INVALID_ARGUMENT, "lse must be 4-byte aligned");
    if (std::isnan(scale) || std::isinf(scale)) return fail(BSMT_ERR_INVALID_ARGUMENT, "scale must be finite");
    if (scale <= 0.f) scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));

    // score mods -> compile-time mode
    ScoreArgs sa;
    {
        const bsmt_status sst = parse_score(score, Hq, &sa);
        if (sst != BSMT_OK) return sst;
    }
    const int mode = sa.mode;

    bsmt::MaskDnf dnf;
    std::memset(&dnf, 0, sizeof(dnf));
    bsmt::AttnParams p;
    std::memset(&p, 0, sizeof(p));
    if (bm != nullptr) {
        if (bm->BLOCK_Q != 128 || bm->BLOCK_KV != 128)
            return fail(BSMT_ERR_UNSUPPORTED, "block mask BLOCK_SIZE (%d, %d): only 128 x 128", bm->BLOCK_Q, bm->BLOCK_KV);
        if (bm->Q_LEN != M || bm->KV_LEN != N || bm->QB != QB || bm->KB != KB)
            return fail(BSMT_ERR_SHAPE_MISMATCH,
                        "block mask is for (Q_LEN=%d, KV_LEN=%d, QB=%d, KB=%d) but attention has M=%lld N=%lld", bm->Q_LEN,
                        bm->KV_LEN, bm->QB, bm->KB, static_cast<long long>(M), static_cast<long long>(N));
        if (!(bm->B == 1 || bm->B == B) || !(bm->H == 1 || bm->H == Hq))
            return fail(BSMT_ERR_SHAPE_MISMATCH, "block mask (B=%d, H=%d) must broadcast to (B=%lld, Hq=%lld)", bm->B, bm->H,
                        static_cast<long long>(B), static_cast<long long>(Hq));
        if (QB > 0 && KB > 0 &&
            (!bm->kv_num_blocks || !bm->kv_indices || !bm->full_kv_num_blocks || !bm->full_kv_indices))
            return fail(BSMT_ERR_INVALID_ARGUMENT, "block mask pointers must be non-NULL");
        bsmt_status st = build_dnf(mask_spec, B, &dnf);
        if (st != BSMT_OK) return st;
        p.has_block_mask = 1;
        p.Bm = bm->B;
        p.Hm = bm->H;
        p.kv_num = bm->kv_num_blocks;
        p.kv_idx = bm->kv_indices;
        p.full_num = bm->full_kv_num_blocks;
        p.full_idx = bm->full_kv_indices;
    } else {
        dnf.n_terms = 1;
    }
    if (dry_run || B == 0 || M == 0) return ok();  // (a dry run only checks the arguments)
    int dev = 0, nsm = 0;
    bsmt_status st = sm_count(&dev, &nsm);
    if (st != BSMT_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (N == 0) {
        const int64_t out_vec = B * Hq * M * D / 8, rows = B * Hq * M;
        fill_empty_kernel<<<2 * nsm, 256, 0, s>>>(static_cast<uint4*>(out), out_vec, lse, rows);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "fill launch: %s", cudaGetErrorString(e));
        return ok();
    }
    EncodeTiledFn enc = nullptr;
    st = get_encoder(&enc);
    if (st != BSMT_OK) return st;
    CUtensorMap tq, tk, tv, to;
    // element strides (head, row): [B, H, S, D], or the packed [S, H, D] with B = 1
    const int64_t q_sbh = packed ? D : M * D, q_ss = packed ? Hq * D : D;
    const int64_t kv_sbh = packed ? D : N * D, kv_ss = packed ? Hkv * D : D;
    if ((st = encode_bhsd(enc, &tq, q, B * Hq, M, D, q_sbh, q_ss)) != BSMT_OK) return st;
    if ((st = encode_out(enc, &to, out, B * Hq, M, D, q_sbh, q_ss)) != BSMT_OK) return st;
    if ((st = encode_bhsd(enc, &tk, k, B * Hkv, N, D, kv_sbh, kv_ss)) != BSMT_OK) return st;
    if ((st = encode_bhsd(enc, &tv, v, B * Hkv, N, D, kv_sbh, kv_ss)) != BSMT_OK) return st;
    p.out_sbh = q_sbh;
    p.out_ss = q_ss;

    p.B = static_cast<int32_t>(B);
    p.Hq = static_cast<int32_t>(Hq);
    p.Hkv = static_cast<int32_t>(Hkv);
    p.M = static_cast<int32_t>(M);
    p.N = static_cast<int32_t>(N);
    p.QB = static_cast<int32_t>(QB);
    p.KB = static_cast<int32_t>(KB);
    p.pairs = static_cast<int32_t>((QB + 1) / 2);
    p.group = static_cast<int32_t>(Hq / Hkv);
    p.num_splits = num_splits;
    p.ws_o = ws_o;
    p.ws_lse = ws_lse;
    const int64_t units = B * Hq * p.pairs * num_splits;
    if (units > 0x7FFFFFFF) return fail(BSMT_ERR_UNSUPPORTED, "too many work units");
    p.num_units = static_cast<int32_t>(units);
    p.scale = scale;
    p.scale_log2 = scale * bsmt::kLog2e;
    p.cap = sa.cap;
    p.inv_cap = 1.f / sa.cap;
    p.slopes = sa.slopes;
    p.alibi_h0 = sa.alibi_h0;
    p.alibi_heads = sa.alibi_heads;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    st = D == 128 ? launch_attn_score<128>(mode, dev, nsm, tq, tk, tv, to, p, dnf, s)
                  : launch_attn_score<64>(mode, dev, nsm, tq, tk, tv, to, p, dnf, s);
    if (st != BSMT_OK) return BSMT_ERR_CUDA;
    if (num_splits > 1) {
        const int64_t rows = B * Hq * M;
        const int64_t blocks = (rows + 7) / 8;
        if (blocks > 0x7FFFFFFF) return fail(BSMT_ERR_UNSUPPORTED, "grid too large");
        if (D == 128)
            bsmt::splitkv_combine_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
                ws_o, ws_lse, num_splits, rows, M, p.out_sbh, p.out_ss, static_cast<__nv_bfloat16*>(out), lse);
        else
            bsmt::splitkv_combine_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
                ws_o, ws_lse, num_splits, rows, M, p.out_sbh, p.out_ss, static_cast<__nv_bfloat16*>(out), lse);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "split-KV combine launch: %s", cudaGetErrorString(e));
    }
    return ok();
}

// Bytes of the split-KV workspace: O slices [S][B*Hq*M][D] fp32, then the
// lse slices [S][B*Hq*M] fp32 starting at a 256-byte boundary.
int64_t splitkv_ws_o_bytes(int64_t B, int64_t Hq, int64_t M, int64_t D, int64_t S) {
    return (S * B * Hq * M * D * 4 + 255) / 256 * 256;
}
int64_t splitkv_ws_bytes(int64_t B, int64_t Hq, int64_t M, int64_t D, int64_t S) {
    return splitkv_ws_o_bytes(B, Hq, M, D, S) + S * B * Hq * M * 4;
}
}  // namespace

extern "C" {

bsmt_status bsmt_flex_attention_fwd(const void* q, const void* k, const void* v, int64_t B, int64_t Hq, int64_t Hkv,
                                    int64_t M, int64_t N, int64_t D, const bsmt_block_mask* bm,
                                    const bsmt_mask_spec* mask_spec, const bsmt_score_spec* score, float scale,
                                    int32_t enable_gqa, void* out, float* lse, void* stream) {
    return attention(q, k, v, B, Hq, Hkv, M, N, D, bm, mask_spec, score, scale, enable_gqa, 1, nullptr, nullptr, out,
                     lse, stream);
}

bsmt_status bsmt_splitkv_workspace_bytes(int64_t B, int64_t Hq, int64_t M, int64_t D, int32_t num_splits,
                                         int64_t* bytes) {
    if (bytes == nullptr) return fail(BSMT_ERR_INVALID_ARGUMENT, "bytes is NULL");
    if (B < 0 || Hq < 0 || M < 0) return fail(BSMT_ERR_INVALID_ARGUMENT, "negative size");
    if (D != 64 && D != 128) return fail(BSMT_ERR_UNSUPPORTED, "head dim D=%lld (supported: 64, 128)", static_cast<long long>(D));
    if (num_splits < 1 || num_splits > BSMT_MAX_SPLITS)
        return fail(BSMT_ERR_INVALID_ARGUMENT, "num_splits=%d outside [1, %d]", num_splits, BSMT_MAX_SPLITS);
    if (M > kMaxLen || B * Hq > 0x7FFFFFFF) return fail(BSMT_ERR_UNSUPPORTED, "sizes too large");
    *bytes = num_splits == 1 ? 0 : splitkv_ws_bytes(B, Hq, M, D, num_splits);
    return ok();
}

bsmt_status bsmt_flex_attention_fwd_splitkv(const void* q, const void* k, const void* v, int64_t B, int64_t Hq,
                                            int64_t Hkv, int64_t M, int64_t N, int64_t D, const bsmt_block_mask* bm,
                                            const bsmt_mask_spec* mask_spec, const bsmt_score_spec* score,
                                            float scale, int32_t enable_gqa, int32_t num_splits, void* workspace,
                                            int64_t workspace_bytes, void* out, float* lse, void* stream) {
    int64_t need = 0;
    bsmt_status st = bsmt_splitkv_workspace_bytes(B, Hq, M, D, num_splits, &need);
    if (st != BSMT_OK) return st;
    float* ws_o = nullptr;
    float* ws_lse = nullptr;
    if (num_splits > 1 && B * Hq * M > 0) {
        if (workspace == nullptr || !aligned(workspace, 256))
            return fail(BSMT_ERR_INVALID_ARGUMENT, "workspace must be non-NULL and 256-byte aligned");
        if (workspace_bytes < need)
            return fail(BSMT_ERR_INVALID_ARGUMENT, "workspace holds %lld bytes, %lld needed",
                        static_cast<long long>(workspace_bytes), static_cast<long long>(need));
        ws_o = static_cast<float*>(workspace);
        ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + splitkv_ws_o_bytes(B, Hq, M, D, num_splits));
    }
    return attention(q, k, v, B, Hq, Hkv, M, N, D, bm, mask_spec, score, scale, enable_gqa, num_splits, ws_o, ws_lse,
                     out, lse, stream);
}

bsmt_status bsmt_flex_attention_fwd_splitkv_static(const void* q, const void* k, const void* v, int64_t B,
                                                   int64_t Hq, int64_t Hkv, int64_t M, int64_t N, int64_t D,
                                                   const bsmt_block_mask* bm, const bsmt_mask_spec* mask_spec,
                                                   const bsmt_score_spec* score, float scale, int32_t enable_gqa,
                                                   int32_t num_splits, void* out, float* lse, void* stream) {
    int64_t need = 0;
    bsmt_status st = bsmt_splitkv_workspace_bytes(B, Hq, M, D, num_splits, &need);
    if (st != BSMT_OK) return st;
    if (need > BSMT_SPLITKV_SCRATCH_BYTES)
        return fail(BSMT_ERR_UNSUPPORTED,
                    "split-KV scratch: %lld bytes needed for B=%lld Hq=%lld M=%lld D=%lld with %d splits, the static "
                    "scratch holds %lld; use bsmt_flex_attention_fwd_splitkv with a workspace",
                    static_cast<long long>(need), static_cast<long long>(B), static_cast<long long>(Hq),
                    static_cast<long long>(M), static_cast<long long>(D), num_splits,
                    static_cast<long long>(BSMT_SPLITKV_SCRATCH_BYTES));
    void* scratch = nullptr;
    if (need > 0) {
        int dev = 0, nsm = 0;
        st = sm_count(&dev, &nsm);
        if (st != BSMT_OK) return st;
        st = scratch_address(dev, &scratch);
        if (st != BSMT_OK) return st;
    }
    // nothing in the scratch must start at zero: every slice writes each of
    // its rows (O and lse) before the merge kernel reads them
    return bsmt_flex_attention_fwd_splitkv(q, k, v, B, Hq, Hkv, M, N, D, bm, mask_spec, score, scale, enable_gqa,
                                           num_splits, scratch, BSMT_SPLITKV_SCRATCH_BYTES, out, lse, stream);
}

bsmt_status bsmt_check_device_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, bsmt::g_status, sizeof(int));
    if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "reading device status: %s", cudaGetErrorString(e));
    if (v != 0) {
        const int zero = 0;
        cudaMemcpyToSymbol(bsmt::g_status, &zero, sizeof(int));
        const char* what = v == BSMT_ERR_DEVICE_TIMEOUT     ? "a pipeline wait ran out of time"
                           : v == BSMT_ERR_DEVICE_BOUNDS    ? "a block index outside [0, KB) or a bad count"
                           : v == BSMT_ERR_DEVICE_PRECONDITION ? "kv document ids are not non-decreasing"
                                                            : "unknown device error";
        return fail(static_cast<bsmt_status>(v), "device status %d: %s", v, what);
    }
    return ok();
}

}  // extern "C"

namespace {
// Shared checks of a kv-side BlockMask passed in by the caller.
bsmt_status check_kv_side(const bsmt_block_mask* kv) {
    if (kv == nullptr) return fail(BSMT_ERR_INVALID_ARGUMENT, "block mask is NULL");
    if (kv->B < 0 || kv->H < 0 || kv->QB < 0 || kv->KB < 0)
        return fail(BSMT_ERR_INVALID_ARGUMENT, "block mask shape fields must be non-negative");
    const int64_t rows = static_cast<int64_t>(kv->B) * kv->H * kv->QB;
    if (rows > 0) {
        if (!kv->kv_num_blocks || !kv->full_kv_num_blocks || (kv->KB > 0 && (!kv->kv_indices || !kv->full_kv_indices)))
            return fail(BSMT_ERR_INVALID_ARGUMENT, "block mask pointers must be non-NULL");
        if (!aligned(kv->kv_num_blocks, 4) || !aligned(kv->kv_indices, 4) || !aligned(kv->full_kv_num_blocks, 4) ||
            !aligned(kv->full_kv_indices, 4))
            return fail(BSMT_ERR_INVALID_ARGUMENT, "block mask pointers must be 4-byte aligned");
    }
    return BSMT_OK;
}
}  // namespace

extern "C" bsmt_status bsmt_block_mask_transpose(const bsmt_block_mask* kv, bsmt_block_mask_q* out, void* stream) {
    bsmt_status st = check_kv_side(kv);
    if (st != BSMT_OK) return st;
    if (out == nullptr) return fail(BSMT_ERR_INVALID_ARGUMENT, "q-side output is NULL");
    const int64_t cols = static_cast<int64_t>(kv->B) * kv->H * kv->KB;
    if (cols == 0) return ok();
    if (!out->q_num_blocks || !out->full_q_num_blocks || (kv->QB > 0 && (!out->q_indices || !out->full_q_indices)))
        return fail(BSMT_ERR_INVALID_ARGUMENT, "q-side output pointers must be non-NULL");
    if (!aligned(out->q_num_blocks, 4) || !aligned(out->q_indices, 4) || !aligned(out->full_q_num_blocks, 4) ||
        !aligned(out->full_q_indices, 4))
        return fail(BSMT_ERR_INVALID_ARGUMENT, "q-side output pointers must be 4-byte aligned");
    if (kv->QB > 12800) return fail(BSMT_ERR_UNSUPPORTED, "QB=%d above 12800", kv->QB);
    if (kv->H > 65535 || kv->B > 65535) return fail(BSMT_ERR_UNSUPPORTED, "B or H above 65535");
    int dev = 0, nsm = 0;
    st = sm_count(&dev, &nsm);
    if (st != BSMT_OK) return st;
    const int chunk = bsmt::transpose_chunk(kv->QB, kv->KB, static_cast<int64_t>(kv->B) * kv->H, nsm);
    const int smem = static_cast<int>(bsmt::transpose_smem_bytes(kv->QB, chunk));
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(bsmt::mask_transpose_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    }
    bsmt::TransposeParams p;
    p.Bm = kv->B;
    p.Hm = kv->H;
    p.QB = kv->QB;
    p.KB = kv->KB;
    p.chunk = chunk;
    p.kv_num = kv->kv_num_blocks;
    p.kv_idx = kv->kv_indices;
    p.full_num = kv->full_kv_num_blocks;
    p.full_idx = kv->full_kv_indices;
    p.q_num = out->q_num_blocks;
    p.q_idx = out->q_indices;
    p.full_q_num = out->full_q_num_blocks;
    p.full_q_idx = out->full_q_indices;
    dim3 grid(static_cast<unsigned>((kv->KB + chunk - 1) / chunk), static_cast<unsigned>(kv->H),
              static_cast<unsigned>(kv->B));
    bsmt::mask_transpose_kernel<<<grid, bsmt::kTransposeThreads, smem, static_cast<cudaStream_t>(stream)>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "transpose launch: %s", cudaGetErrorString(e));
    return ok();
}

extern "C" bsmt_status bsmt_block_mask_to_dense(const bsmt_block_mask* kv, int32_t* dense, void* stream) {
    bsmt_status st = check_kv_side(kv);
    if (st != BSMT_OK) return st;
    const int64_t rows = static_cast<int64_t>(kv->B) * kv->H * kv->QB;
    if (rows == 0 || kv->KB == 0) return ok();
    if (dense == nullptr || !aligned(dense, 4))
        return fail(BSMT_ERR_INVALID_ARGUMENT, "dense output must be non-NULL and 4-byte aligned");
    int dev = 0, nsm = 0;
    st = sm_count(&dev, &nsm);
    if (st != BSMT_OK) return st;
    bsmt::DenseParams p;
    p.Bm = kv->B;
    p.Hm = kv->H;
    p.QB = kv->QB;
    p.KB = kv->KB;
    p.kv_num = kv->kv_num_blocks;
    p.kv_idx = kv->kv_indices;
    p.full_num = kv->full_kv_num_blocks;
    p.full_idx = kv->full_kv_indices;
    p.dense = dense;
    const int64_t blocks = (rows + 3) / 4;
    if (blocks > 0x7FFFFFFF) return fail(BSMT_ERR_UNSUPPORTED, "grid too large");
    bsmt::mask_to_dense_kernel<<<static_cast<unsigned>(blocks), 128, 0, static_cast<cudaStream_t>(stream)>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "to_dense launch: %s", cudaGetErrorString(e));
    return ok();
}

extern "C" bsmt_status bsmt_seqlens_to_doc_ids(const int32_t* cu_seqlens, int32_t num_seqs, int64_t total,
                                               int32_t* doc_ids, void* stream) {
    if (num_seqs < 0 || total < 0) return fail(BSMT_ERR_INVALID_ARGUMENT, "negative num_seqs or total");
    if (total == 0) return ok();
    if (cu_seqlens == nullptr || doc_ids == nullptr || !aligned(cu_seqlens, 4) || !aligned(doc_ids, 4))
        return fail(BSMT_ERR_INVALID_ARGUMENT, "cu_seqlens and doc_ids must be non-NULL and 4-byte aligned");
    if (total > kMaxLen) return fail(BSMT_ERR_UNSUPPORTED, "total above %lld", static_cast<long long>(kMaxLen));
    int dev = 0, nsm = 0;
    bsmt_status st = sm_count(&dev, &nsm);
    if (st != BSMT_OK) return st;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 4 * nsm) blocks = 4 * nsm;
    bsmt::seqlens_to_doc_ids_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        cu_seqlens, num_seqs, total, doc_ids);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "doc id launch: %s", cudaGetErrorString(e));
    return ok();
}

extern "C" bsmt_status bsmt_flex_attention_fwd_packed(const void* q, const void* k, const void* v, int64_t Hq,
                                                      int64_t Hkv, int64_t M, int64_t N, int64_t D,
                                                      const bsmt_block_mask* bm, const bsmt_mask_spec* mask_spec,
                                                      const bsmt_score_spec* score, float scale, int32_t enable_gqa,
                                                      void* out, float* lse, void* stream) {
    return attention(q, k, v, 1, Hq, Hkv, M, N, D, bm, mask_spec, score, scale, enable_gqa, 1, nullptr, nullptr, out,
                     lse, stream, /*packed=*/true);
}


// ------------------------------------------------------------------ backward
namespace {
bool g_bwd_attr_set[64][40] = {{false}};

__global__ void zero_kernel(uint4* p, int64_t n) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n; i += stride)
        p[i] = make_uint4(0u, 0u, 0u, 0u);
}

bsmt_status zero_bf16(void* p, int64_t elems, int nsm, cudaStream_t s) {
    if (elems == 0) return BSMT_OK;
    zero_kernel<<<2 * nsm, 256, 0, s>>>(static_cast<uint4*>(p), elems / 8);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "zero launch: %s", cudaGetErrorString(e));
    return BSMT_OK;
}

template <int D, int SCORE, bool KVSIDE, bool LONG>
bsmt_status launch_bwd_kind(int dev, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const bsmt::BwdParams& p, const bsmt::MaskDnf& dnf,
                            cudaStream_t s) {
    auto kern = bsmt::attn_bwd_kernel<D, SCORE, KVSIDE, LONG>;
    const int smem = bsmt::BwdSmem<D>::kAlloc;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        const int slot = (LONG ? 20 : 0) + (D == 128 ? 10 : 0) + 2 * SCORE + (KVSIDE ? 1 : 0);
        if (!g_bwd_attr_set[dev][slot]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
            g_bwd_attr_set[dev][slot] = true;
        }
    }
    int nsm = 0;
    cudaError_t ea = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (ea != cudaSuccess) return fail(BSMT_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(ea));
    const int grid = p.num_units < nsm ? p.num_units : nsm;  // persistent: units come from a work counter
    kern<<<static_cast<unsigned>(grid), bsmt::kBwdThreads, smem, s>>>(tq, tk, tv, tdo, p, dnf);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "backward launch: %s", cudaGetErrorString(e));
    return BSMT_OK;
}

// Units of more entries than one buffer holds (list length x heads), or lists
// longer than the flag window, take the kernel's segmented variant.
template <int D, int SCORE, bool KVSIDE>
bsmt_status launch_bwd(int dev, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const bsmt::BwdParams& p, const bsmt::MaskDnf& dnf, cudaStream_t s) {
    const int64_t per_unit = static_cast<int64_t>(p.list_len) * (KVSIDE ? p.group : 1);
    if (per_unit > bsmt::kBwdMaxEntries)
        return launch_bwd_kind<D, SCORE, KVSIDE, true>(dev, tq, tk, tv, tdo, p, dnf, s);
    return launch_bwd_kind<D, SCORE, KVSIDE, false>(dev, tq, tk, tv, tdo, p, dnf, s);
}

template <int D, bool KVSIDE>
bsmt_status launch_bwd_score(int mode, int dev, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tdo, const bsmt::BwdParams& p, const bsmt::MaskDnf& dnf,
                             cudaStream_t s) {
    switch (mode) {
        case bsmt::kScoreNone: return launch_bwd<D, bsmt::kScoreNone, KVSIDE>(dev, tq, tk, tv, tdo, p, dnf, s);
        case bsmt::kScoreSoftcap: return launch_bwd<D, bsmt::kScoreSoftcap, KVSIDE>(dev, tq, tk, tv, tdo, p, dnf, s);
        case bsmt::kScoreAlibi: return launch_bwd<D, bsmt::kScoreAlibi, KVSIDE>(dev, tq, tk, tv, tdo, p, dnf, s);
        case bsmt::kScoreSoftcapAlibi:
            return launch_bwd<D, bsmt::kScoreSoftcapAlibi, KVSIDE>(dev, tq, tk, tv, tdo, p, dnf, s);
        default: return launch_bwd<D, bsmt::kScoreAlibiSoftcap, KVSIDE>(dev, tq, tk, tv, tdo, p, dnf, s);
    }
}

// Workspace of the backward: (-lse2, -delta) per padded query row, then the
// two kernels' work counters at the next 256-byte boundary.
int64_t bwd_ld_bytes(int64_t B, int64_t Hq, int64_t M) { return (B * Hq * ((M + 127) / 128) * 128 * 8 + 255) / 256 * 256; }
int64_t bwd_ws_bytes(int64_t B, int64_t Hq, int64_t M) { return bwd_ld_bytes(B, Hq, M) + 256; }
}  // namespace

extern "C" bsmt_status bsmt_flex_attention_bwd_workspace_bytes(int64_t B, int64_t Hq, int64_t M, int64_t* bytes) {
    if (bytes == nullptr) return fail(BSMT_ERR_INVALID_ARGUMENT, "bytes is NULL");
    if (B < 0 || Hq < 0 || M < 0) return fail(BSMT_ERR_INVALID_ARGUMENT, "negative size");
    if (M > kMaxLen || B * Hq > 0x7FFFFFFF) return fail(BSMT_ERR_UNSUPPORTED, "sizes too large");
    *bytes = bwd_ws_bytes(B, Hq, M);
    return ok();
}

namespace {
// The backward path; `packed` selects the [S, H, D] layouts (B = 1).
bsmt_status backward(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
                     int64_t B, int64_t Hq, int64_t Hkv, int64_t M, int64_t N, int64_t D, const bsmt_block_mask* bm,
                     const bsmt_block_mask_q* bmq, const bsmt_mask_spec* mask_spec, const bsmt_score_spec* score,
                     float scale, int32_t enable_gqa, void* dq, void* dk, void* dv, void* workspace,
                     int64_t workspace_bytes, void* stream, bool packed) {
    if (B < 0 || Hq < 0 || Hkv < 0 || M < 0 || N < 0)
        return fail(BSMT_ERR_INVALID_ARGUMENT, "negative size (B=%lld Hq=%lld Hkv=%lld M=%lld N=%lld)",
                    static_cast<long long>(B), static_cast<long long>(Hq), static_cast<long long>(Hkv),
                    static_cast<long long>(M), static_cast<long long>(N));
    if (D != 64 && D != 128) return fail(BSMT_ERR_UNSUPPORTED, "head dim D=%lld (supported: 64, 128)", static_cast<long long>(D));
    if (Hkv < 1 || Hq < 1) return fail(BSMT_ERR_SHAPE_MISMATCH, "Hq=%lld and Hkv=%lld must be >= 1", static_cast<long long>(Hq), static_cast<long long>(Hkv));
    if (Hq % Hkv != 0)
        return fail(BSMT_ERR_SHAPE_MISMATCH, "Hq=%lld is not a multiple of Hkv=%lld", static_cast<long long>(Hq),
                    static_cast<long long>(Hkv));
    if (Hq != Hkv && !enable_gqa)
        return fail(BSMT_ERR_SHAPE_MISMATCH, "Hq=%lld != Hkv=%lld requires enable_gqa", static_cast<long long>(Hq),
                    static_cast<long long>(Hkv));
    if (M > kMaxLen || N > kMaxLen) return fail(BSMT_ERR_UNSUPPORTED, "sequence length above %lld", static_cast<long long>(kMaxLen));
    if (B * Hq > 0x7FFFFFFF || B * Hkv > 0x7FFFFFFF) return fail(BSMT_ERR_UNSUPPORTED, "B*H above 2^31");
    const int64_t QB = (M + 127) / 128, KB = (N + 127) / 128;
    const int64_t group = Hq / Hkv;
    // entries hold a block number in 16 bits and a head of the GQA group in 8
    if (KB > 65536 || QB > 65536)
        return fail(BSMT_ERR_UNSUPPORTED, "Q_LEN=%lld, KV_LEN=%lld: at most 65536 blocks of 128 per sequence",
                    static_cast<long long>(M), static_cast<long long>(N));
    if (group > 255)
        return fail(BSMT_ERR_UNSUPPORTED, "%lld query heads per kv head: at most 255", static_cast<long long>(group));
    const bool q_has = B * Hq * M > 0, kv_has = B * Hkv * N > 0;
    if ((q_has && (!q || !out || !dout || !lse || !dq)) || (kv_has && (!k || !v || !dk || !dv)))
        return fail(BSMT_ERR_INVALID_ARGUMENT, "q, k, v, out, dout, lse, dq, dk and dv must be non-NULL when they hold elements");
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(dout, 16) ||
        !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16))
        return fail(BSMT_ERR_INVALID_ARGUMENT, "q, k, v, out, dout, dq, dk and dv must be 16-byte aligned");
    if (!aligned(lse, 4)) return fail(BSMT_ERR_INVALID_ARGUMENT, "lse must be 4-byte aligned");
    if (std::isnan(scale) || std::isinf(scale)) return fail(BSMT_ERR_INVALID_ARGUMENT, "scale must be finite");
    if (scale <= 0.f) scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
    ScoreArgs sa;
    bsmt_status st = parse_score(score, Hq, &sa);
    if (st != BSMT_OK) return st;
    const int mode = sa.mode;

    bsmt::MaskDnf dnf;
    std::memset(&dnf, 0, sizeof(dnf));
    bsmt::BwdParams pq, pk;  // dq kernel (kv-side lists), dk/dv kernel (q-side lists)
    std::memset(&pq, 0, sizeof(pq));
    std::memset(&pk, 0, sizeof(pk));
    if (bm != nullptr) {
        if (bm->BLOCK_Q != 128 || bm->BLOCK_KV != 128)
            return fail(BSMT_ERR_UNSUPPORTED, "block mask BLOCK_SIZE (%d, %d): only 128 x 128", bm->BLOCK_Q, bm->BLOCK_KV);
        if (bm->Q_LEN != M || bm->KV_LEN != N || bm->QB != QB || bm->KB != KB)
            return fail(BSMT_ERR_SHAPE_MISMATCH,
                        "block mask is for (Q_LEN=%d, KV_LEN=%d, QB=%d, KB=%d) but attention has M=%lld N=%lld", bm->Q_LEN,
                        bm->KV_LEN, bm->QB, bm->KB, static_cast<long long>(M), static_cast<long long>(N));
        if (!(bm->B == 1 || bm->B == B) || !(bm->H == 1 || bm->H == Hq))
            return fail(BSMT_ERR_SHAPE_MISMATCH, "block mask (B=%d, H=%d) must broadcast to (B=%lld, Hq=%lld)", bm->B, bm->H,
                        static_cast<long long>(B), static_cast<long long>(Hq));
        if (QB > 0 && KB > 0) {
            if (!bm->kv_num_blocks || !bm->kv_indices || !bm->full_kv_num_blocks || !bm->full_kv_indices)
                return fail(BSMT_ERR_INVALID_ARGUMENT, "block mask pointers must be non-NULL");
            if (bmq == nullptr || !bmq->q_num_blocks || !bmq->q_indices || !bmq->full_q_num_blocks ||
                !bmq->full_q_indices)
                return fail(BSMT_ERR_INVALID_ARGUMENT, "the backward needs the q-side lists of the block mask");
            if (!aligned(bmq->q_num_blocks, 4) || !aligned(bmq->q_indices, 4) || !aligned(bmq->full_q_num_blocks, 4) ||
                !aligned(bmq->full_q_indices, 4))
                return fail(BSMT_ERR_INVALID_ARGUMENT, "q-side list pointers must be 4-byte aligned");
        }
        st = build_dnf(mask_spec, B, &dnf);
        if (st != BSMT_OK) return st;
        for (bsmt::BwdParams* pp : {&pq, &pk}) {
            pp->has_block_mask = 1;
            pp->Bm = bm->B;
            pp->Hm = bm->H;
        }
        pq.num = bm->kv_num_blocks;
        pq.idx = bm->kv_indices;
        pq.full_num = bm->full_kv_num_blocks;
        pq.full_idx = bm->full_kv_indices;
        if (bmq != nullptr) {
            pk.num = bmq->q_num_blocks;
            pk.idx = bmq->q_indices;
            pk.full_num = bmq->full_q_num_blocks;
            pk.full_idx = bmq->full_q_indices;
        }
    } else {
        dnf.n_terms = 1;
    }
    if (B == 0 || (M == 0 && N == 0)) return ok();
    const int64_t need = bwd_ws_bytes(B, Hq, M);
    if (need > 0 && (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need))
        return fail(BSMT_ERR_INVALID_ARGUMENT, "workspace must be non-NULL, 256-byte aligned and hold %lld bytes (has %lld)",
                    static_cast<long long>(need), static_cast<long long>(workspace_bytes));
    int dev = 0, nsm = 0;
    st = sm_count(&dev, &nsm);
    if (st != BSMT_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M == 0) {  // no queries: nothing reaches k or v
        if ((st = zero_bf16(dk, B * Hkv * N * D, nsm, s)) != BSMT_OK) return st;
        return (st = zero_bf16(dv, B * Hkv * N * D, nsm, s)) != BSMT_OK ? st : ok();
    }
    if (N == 0) return (st = zero_bf16(dq, B * Hq * M * D, nsm, s)) != BSMT_OK ? st : ok();
    if (B * Hkv * KB > 0x7FFFFFFF || B * Hq * QB > 0x7FFFFFFF) return fail(BSMT_ERR_UNSUPPORTED, "too many work units");

    // (-lse2, -delta) per padded query row, and the work counters
    float2* ld = static_cast<float2*>(workspace);
    int32_t* counters = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + bwd_ld_bytes(B, Hq, M));
    // element strides (head, row): [B, H, S, D], or the packed [S, H, D] with B = 1
    const int64_t q_sbh = packed ? D : M * D, q_ss = packed ? Hq * D : D;
    const int64_t kv_sbh = packed ? D : N * D, kv_ss = packed ? Hkv * D : D;
    const int64_t rows_pad = B * Hq * QB * 128;
    const int64_t prep_blocks = (rows_pad + 8 * bsmt::kPrepRowsPerWarp - 1) / (8 * bsmt::kPrepRowsPerWarp);
    if (prep_blocks > 0x7FFFFFFF) return fail(BSMT_ERR_UNSUPPORTED, "too many query rows");
    if (D == 128)
        bsmt::bwd_prep_kernel<128><<<static_cast<unsigned>(prep_blocks), 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), lse, rows_pad,
            static_cast<int32_t>(M), static_cast<int32_t>(QB), q_sbh, q_ss, ld, counters);
    else
        bsmt::bwd_prep_kernel<64><<<static_cast<unsigned>(prep_blocks), 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), lse, rows_pad,
            static_cast<int32_t>(M), static_cast<int32_t>(QB), q_sbh, q_ss, ld, counters);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "backward prep launch: %s", cudaGetErrorString(e));

    EncodeTiledFn enc = nullptr;
    if ((st = get_encoder(&enc)) != BSMT_OK) return st;
    CUtensorMap tq, tk, tv, tdo;
    if ((st = encode_bhsd(enc, &tq, q, B * Hq, M, D, q_sbh, q_ss)) != BSMT_OK) return st;
    if ((st = encode_bhsd(enc, &tdo, dout, B * Hq, M, D, q_sbh, q_ss)) != BSMT_OK) return st;
    if ((st = encode_bhsd(enc, &tk, k, B * Hkv, N, D, kv_sbh, kv_ss)) != BSMT_OK) return st;
    if ((st = encode_bhsd(enc, &tv, v, B * Hkv, N, D, kv_sbh, kv_ss)) != BSMT_OK) return st;
    for (bsmt::BwdParams* pp : {&pq, &pk}) {
        pp->B = static_cast<int32_t>(B);
        pp->Hq = static_cast<int32_t>(Hq);
        pp->Hkv = static_cast<int32_t>(Hkv);
        pp->M = static_cast<int32_t>(M);
        pp->N = static_cast<int32_t>(N);
        pp->QB = static_cast<int32_t>(QB);
        pp->KB = static_cast<int32_t>(KB);
        pp->group = static_cast<int32_t>(group);
        pp->scale = scale;
        pp->scale_log2 = scale * bsmt::kLog2e;
        pp->cap = sa.cap;
        pp->inv_cap = 1.f / sa.cap;
        pp->slopes = sa.slopes;
        pp->alibi_h0 = sa.alibi_h0;
        pp->alibi_heads = sa.alibi_heads;
        pp->ld = ld;
        pp->q_sbh = q_sbh;
        pp->q_ss = q_ss;
        pp->kv_sbh = kv_sbh;
        pp->kv_ss = kv_ss;
    }
    pk.list_rows = static_cast<int32_t>(KB);
    pk.list_len = static_cast<int32_t>(QB);
    pk.g0 = static_cast<__nv_bfloat16*>(dk);
    pk.g1 = static_cast<__nv_bfloat16*>(dv);
    pk.num_units = static_cast<int32_t>(B * Hkv * KB);
    pk.next_unit = counters;
    pq.list_rows = static_cast<int32_t>(QB);
    pq.list_len = static_cast<int32_t>(KB);
    pq.g0 = static_cast<__nv_bfloat16*>(dq);
    pq.num_units = static_cast<int32_t>(B * Hq * QB);
    pq.next_unit = counters + 1;
    st = D == 128 ? launch_bwd_score<128, true>(mode, dev, tq, tk, tv, tdo, pk, dnf, s)
                  : launch_bwd_score<64, true>(mode, dev, tq, tk, tv, tdo, pk, dnf, s);
    if (st != BSMT_OK) return st;
    st = D == 128 ? launch_bwd_score<128, false>(mode, dev, tq, tk, tv, tdo, pq, dnf, s)
                  : launch_bwd_score<64, false>(mode, dev, tq, tk, tv, tdo, pq, dnf, s);
    if (st != BSMT_OK) return st;
    return ok();
}
}  // namespace

extern "C" bsmt_status bsmt_flex_attention_bwd(const void* q, const void* k, const void* v, const void* out,
                                               const void* dout, const float* lse, int64_t B, int64_t Hq, int64_t Hkv,
                                               int64_t M, int64_t N, int64_t D, const bsmt_block_mask* bm,
                                               const bsmt_block_mask_q* bmq, const bsmt_mask_spec* mask_spec,
                                               const bsmt_score_spec* score, float scale, int32_t enable_gqa,
                                               void* dq, void* dk, void* dv, void* workspace, int64_t workspace_bytes,
                                               void* stream) {
    return backward(q, k, v, out, dout, lse, B, Hq, Hkv, M, N, D, bm, bmq, mask_spec, score, scale, enable_gqa, dq,
                    dk, dv, workspace, workspace_bytes, stream, false);
}

extern "C" bsmt_status bsmt_flex_attention_bwd_packed(const void* q, const void* k, const void* v, const void* out,
                                                      const void* dout, const float* lse, int64_t Hq, int64_t Hkv,
                                                      int64_t M, int64_t N, int64_t D, const bsmt_block_mask* bm,
                                                      const bsmt_block_mask_q* bmq, const bsmt_mask_spec* mask_spec,
                                                      const bsmt_score_spec* score, float scale, int32_t enable_gqa,
                                                      void* dq, void* dk, void* dv, void* workspace,
                                                      int64_t workspace_bytes, void* stream) {
    return backward(q, k, v, out, dout, lse, 1, Hq, Hkv, M, N, D, bm, bmq, mask_spec, score, scale, enable_gqa, dq,
                    dk, dv, workspace, workspace_bytes, stream, true);
}

extern "C" bsmt_status bsmt_selftest_wait_timeout(int32_t* result, void* stream) {
    if (result == nullptr || !aligned(result, 4))
        return fail(BSMT_ERR_INVALID_ARGUMENT, "result must be a non-NULL, 4-byte aligned device int32[3]");
    int dev = 0, nsm = 0;
    bsmt_status st = sm_count(&dev, &nsm);
    if (st != BSMT_OK) return st;
    bsmt::wait_timeout_selftest_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(result);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "self-test launch: %s", cudaGetErrorString(e));
    return ok();
}


// ------------------------------------------------------------ host buffers
namespace {
constexpr int kMaxHostPieces = 256;

// Per device: two copy streams and a pool of events for the host pipeline,
// created on its first call there and kept.
struct HostCtx {
    bool ready = false;
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev[2 * kMaxHostPieces + 4] = {};
};
HostCtx g_host[64];
std::mutex g_host_mu;  // held while a call enqueues (the pool is shared)

int64_t round256(int64_t x) { return (x + 255) / 256 * 256; }

// Where each device copy sits in the workspace (byte offsets, 256-aligned).
struct HostLayout {
    int64_t q, k, v, o, l, kvn, kvi, fn, fi, qdoc, kvdoc, slopes[BSMT_MAX_SCORE_OPS], total;
    int64_t Bm, QB, KB;
    bool has_doc;
    int32_t doc_batch;
};

bool spec_has_doc(const bsmt_mask_spec* spec) {
    if (spec == nullptr) return false;
    for (int i = 0; i < spec->num_nodes && i < BSMT_MAX_MASK_NODES; ++i)
        if (spec->nodes[i].kind == BSMT_MASK_DOCUMENT) return true;
    return false;
}

bsmt_status host_layout(int64_t B, int64_t Hq, int64_t Hkv, int64_t M, int64_t N, int64_t D,
                        const bsmt_mask_spec* spec, HostLayout* L) {
    if (B < 0 || Hq < 0 || Hkv < 0 || M < 0 || N < 0) return fail(BSMT_ERR_INVALID_ARGUMENT, "negative size");
    if (D != 64 && D != 128) return fail(BSMT_ERR_UNSUPPORTED, "head dim D=%lld (supported: 64, 128)", static_cast<long long>(D));
    if (M > kMaxLen || N > kMaxLen || B * Hq > 0x7FFFFFFF || B * Hkv > 0x7FFFFFFF)
        return fail(BSMT_ERR_UNSUPPORTED, "sizes too large");
    L->has_doc = spec_has_doc(spec);
    L->doc_batch = L->has_doc ? (spec->doc_batch < 1 ? 1 : spec->doc_batch) : 1;
    if (L->has_doc && !(L->doc_batch == 1 || L->doc_batch == B))
        return fail(BSMT_ERR_SHAPE_MISMATCH, "mask spec: doc_batch=%d must be 1 or B=%lld", L->doc_batch,
                    static_cast<long long>(B));
    L->Bm = (L->has_doc && L->doc_batch > 1) ? B : 1;
    L->QB = (M + 127) / 128;
    L->KB = (N + 127) / 128;
    int64_t off = 0;
    auto take = [&](int64_t bytes) {
        const int64_t at = off;
        off += round256(bytes);
        return at;
    };
    L->q = take(B * Hq * M * D * 2);
    L->k = take(B * Hkv * N * D * 2);
    L->v = take(B * Hkv * N * D * 2);
    L->o = take(B * Hq * M * D * 2);
    L->l = take(B * Hq * M * 4);
    const bool has_mask = spec != nullptr;
    L->kvn = take(has_mask ? L->Bm * L->QB * 4 : 0);
    L->fn = take(has_mask ? L->Bm * L->QB * 4 : 0);
    L->kvi = take(has_mask ? L->Bm * L->QB * L->KB * 4 : 0);
    L->fi = take(has_mask ? L->Bm * L->QB * L->KB * 4 : 0);
    L->qdoc = take(L->has_doc ? int64_t(L->doc_batch) * M * 4 : 0);
    L->kvdoc = take(L->has_doc ? int64_t(L->doc_batch) * N * 4 : 0);
    for (int i = 0; i < BSMT_MAX_SCORE_OPS; ++i) L->slopes[i] = take(Hq * 4);
    L->total = off;
    return BSMT_OK;
}

bsmt_status host_ctx(int dev, HostCtx** out) {
    HostCtx& c = g_host[dev];
    if (!c.ready) {
        cudaError_t e = cudaStreamCreateWithFlags(&c.s_in, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c.s_out, cudaStreamNonBlocking);
        for (int i = 0; e == cudaSuccess && i < 2 * kMaxHostPieces + 4; ++i)
            e = cudaEventCreateWithFlags(&c.ev[i], cudaEventDisableTiming);
        if (e != cudaSuccess) return fail(BSMT_ERR_CUDA, "host pipeline set-up: %s", cudaGetErrorString(e));
        c.ready = true;
    }
    *out = &c;
    return BSMT_OK;
}

// One piece of the host pipeline: batch rows [b0, b1) and kv heads [g0, g1)
// with their query heads (either one batch row or all heads).
struct HostPiece {
    int64_t b0, b1, g0, g1;
};

std::vector<HostPiece> host_pieces(int64_t B, int64_t Hkv, int32_t target) {
    std::vector<HostPiece> v;
    const int64_t t = target <= 0 ? 16 : (target > kMaxHostPieces ? kMaxHostPieces : target);
    if (B >= t) {
        const int64_t rows = (B + t - 1) / t;
        for (int64_t b = 0; b < B; b += rows) v.push_back({b, b + rows < B ? b + rows : B, 0, Hkv});
    } else {
        int64_t per_b = t / (B > 0 ? B : 1);
        if (per_b < 1) per_b = 1;
        if (per_b > Hkv) per_b = Hkv;
        const int64_t gs = (Hkv + per_b - 1) / per_b;
        for (int64_t b = 0; b < B; ++b)
            for (int64_t g = 0; g < Hkv; g += gs) v.push_back({b, b + 1, g, g + gs < Hkv ? g + gs : Hkv});
    }
    return v;
}
}  // namespace

extern "C" bsmt_status bsmt_flex_attention_host_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t M,
                                                                int64_t N, int64_t D, const bsmt_mask_spec* mask_spec,
                                                                int64_t* bytes) {
    if (bytes == nullptr) return fail(BSMT_ERR_INVALID_ARGUMENT, "bytes is NULL");
    HostLayout L;
    const bsmt_status st = host_layout(B, Hq, Hkv, M, N, D, mask_spec, &L);
    if (st != BSMT_OK) return st;
    *bytes = L.total;
    return ok();
}

extern "C" bsmt_status bsmt_flex_attention_host(const void* q, const void* k, const void* v, int64_t B, int64_t Hq,
                                                int64_t Hkv, int64_t M, int64_t N, int64_t D,
                                                const bsmt_mask_spec* mask_spec, const bsmt_score_spec* score,
                                                float scale, int32_t enable_gqa, int32_t pieces, void* workspace,
                                                int64_t workspace_bytes, void* out, float* lse, void* stream) {
    HostLayout L;
    bsmt_status st = host_layout(B, Hq, Hkv, M, N, D, mask_spec, &L);
    if (st != BSMT_OK) return st;
    if (Hkv < 1 || Hq < 1 || Hq % Hkv != 0)
        return fail(BSMT_ERR_SHAPE_MISMATCH, "Hq=%lld must be a positive multiple of Hkv=%lld", static_cast<long long>(Hq),
                    static_cast<long long>(Hkv));
    if (L.Bm > 65535) return fail(BSMT_ERR_UNSUPPORTED, "B=%lld above 65535", static_cast<long long>(L.Bm));
    const bool q_has = B * Hq * M > 0, kv_has = B * Hkv * N > 0;
    if ((q_has && (!q || !out || !lse)) || (kv_has && (!k || !v)))
        return fail(BSMT_ERR_INVALID_ARGUMENT, "q, k, v, out and lse must be non-NULL when they hold elements");
    if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < L.total)
        return fail(BSMT_ERR_INVALID_ARGUMENT, "workspace must be non-NULL, 256-byte aligned and hold %lld bytes (has %lld)",
                    static_cast<long long>(L.total), static_cast<long long>(workspace_bytes));
    char* ws = static_cast<char*>(workspace);
    // device-side copies of the mask and score specs: the same programs, with
    // their arrays in the workspace
    bsmt_mask_spec dspec;
    if (mask_spec != nullptr) {
        dspec = *mask_spec;
        if (L.has_doc) {
            if (mask_spec->q_doc_ids == nullptr || mask_spec->kv_doc_ids == nullptr)
                return fail(BSMT_ERR_INVALID_ARGUMENT, "mask spec: DOCUMENT needs q_doc_ids and kv_doc_ids");
            dspec.q_doc_ids = reinterpret_cast<const int32_t*>(ws + L.qdoc);
            dspec.kv_doc_ids = reinterpret_cast<const int32_t*>(ws + L.kvdoc);
            dspec.doc_batch = L.doc_batch;
        }
    }
    bsmt_score_spec dscore;
    std::memset(&dscore, 0, sizeof(dscore));
    if (score != nullptr) {
        dscore = *score;
        if (score->num_ops < 0 || score->num_ops > BSMT_MAX_SCORE_OPS)
            return fail(BSMT_ERR_INVALID_ARGUMENT, "score spec: num_ops=%d outside [0, %d]", score->num_ops,
                        BSMT_MAX_SCORE_OPS);
        for (int i = 0; i < score->num_ops; ++i)
            if (score->ops[i].kind == BSMT_SCORE_ALIBI && score->ops[i].slopes != nullptr)
                dscore.ops[i].slopes = reinterpret_cast<const float*>(ws + L.slopes[i]);
    }
    bsmt_block_mask bm;
    std::memset(&bm, 0, sizeof(bm));
    bm.kv_num_blocks = reinterpret_cast<int32_t*>(ws + L.kvn);
    bm.kv_indices = reinterpret_cast<int32_t*>(ws + L.kvi);
    bm.full_kv_num_blocks = reinterpret_cast<int32_t*>(ws + L.fn);
    bm.full_kv_indices = reinterpret_cast<int32_t*>(ws + L.fi);
    bm.B = static_cast<int32_t>(L.Bm);
    bm.H = 1;
    bm.QB = static_cast<int32_t>(L.QB);
    bm.KB = static_cast<int32_t>(L.KB);
    bm.Q_LEN = static_cast<int32_t>(M);
    bm.KV_LEN = static_cast<int32_t>(N);
    bm.BLOCK_Q = bm.BLOCK_KV = 128;
    const bsmt_block_mask* bmp = mask_spec != nullptr ? &bm : nullptr;
    const bsmt_mask_spec* dspec_p = mask_spec != nullptr ? &dspec : nullptr;
    char* const wq = ws + L.q;
    char* const wk = ws + L.k;
    char* const wv = ws + L.v;
    char* const wo = ws + L.o;
    float* const wl = reinterpret_cast<float*>(ws + L.l);
    // every argument check of the attention, at the full size, before anything is enqueued
    st = attention(wq, wk, wv, B, Hq, Hkv, M, N, D, bmp, dspec_p, &dscore, scale, enable_gqa, 1, nullptr, nullptr,
                   wo, wl, stream, false, /*dry_run=*/true);
    if (st != BSMT_OK) return st;
    if (!q_has) return ok();
    int dev = 0, nsm = 0;
    if ((st = sm_count(&dev, &nsm)) != BSMT_OK) return st;

    std::lock_guard<std::mutex> lk(g_host_mu);
    HostCtx* hc = nullptr;
    if ((st = host_ctx(dev, &hc)) != BSMT_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaEvent_t* ev = hc->ev;
    const int64_t G = Hq / Hkv;
    const std::vector<HostPiece> pcs = host_pieces(B, Hkv, pieces);
    const int np = static_cast<int>(pcs.size());
    cudaError_t ce = cudaSuccess;
    auto cuda_ok = [&](cudaError_t e) {
        if (ce == cudaSuccess && e != cudaSuccess) ce = e;
        return ce == cudaSuccess;
    };
    // `stream` waits for both copy streams at the end, error or not, so the
    // workspace is free once `stream` has passed the call
    auto join = [&]() {
        cudaEventRecord(ev[2 * kMaxHostPieces + 1], hc->s_in);
        cudaEventRecord(ev[2 * kMaxHostPieces + 2], hc->s_out);
        cudaStreamWaitEvent(s, ev[2 * kMaxHostPieces + 1], 0);
        cudaStreamWaitEvent(s, ev[2 * kMaxHostPieces + 2], 0);
    };
    cuda_ok(cudaEventRecord(ev[2 * kMaxHostPieces], s));
    cuda_ok(cudaStreamWaitEvent(hc->s_in, ev[2 * kMaxHostPieces], 0));
    cuda_ok(cudaStreamWaitEvent(hc->s_out, ev[2 * kMaxHostPieces], 0));
    // 1. document ids and slopes, then the BlockMask, on the caller's stream
    if (L.has_doc) {
        cuda_ok(cudaMemcpyAsync(ws + L.qdoc, mask_spec->q_doc_ids, int64_t(L.doc_batch) * M * 4, cudaMemcpyHostToDevice, s));
        cuda_ok(cudaMemcpyAsync(ws + L.kvdoc, mask_spec->kv_doc_ids, int64_t(L.doc_batch) * N * 4, cudaMemcpyHostToDevice, s));
    }
    for (int i = 0; score != nullptr && i < score->num_ops; ++i)
        if (score->ops[i].kind == BSMT_SCORE_ALIBI && score->ops[i].slopes != nullptr)
            cuda_ok(cudaMemcpyAsync(ws + L.slopes[i], score->ops[i].slopes, Hq * 4, cudaMemcpyHostToDevice, s));
    if (ce != cudaSuccess) {
        join();
        return fail(BSMT_ERR_CUDA, "host pipeline: %s", cudaGetErrorString(ce));
    }
    if (mask_spec != nullptr) {
        st = bsmt_create_block_mask(&dspec, L.Bm, 1, M, N, 128, 128, &bm, stream);
        if (st != BSMT_OK) {
            join();
            return st;
        }
    }
    // 2. inputs of every piece, in order, on the input copy stream
    for (int i = 0; i < np; ++i) {
        const HostPiece& pc = pcs[i];
        const int64_t qoff = (pc.b0 * Hq + pc.g0 * G) * M * D * 2;
        const int64_t qlen = (pc.b1 - pc.b0) * (pc.g1 - pc.g0) * G * M * D * 2;
        const int64_t koff = (pc.b0 * Hkv + pc.g0) * N * D * 2;
        const int64_t klen = (pc.b1 - pc.b0) * (pc.g1 - pc.g0) * N * D * 2;
        cuda_ok(cudaMemcpyAsync(wq + qoff, static_cast<const char*>(q) + qoff, qlen, cudaMemcpyHostToDevice, hc->s_in));
        if (klen > 0) {
            cuda_ok(cudaMemcpyAsync(wk + koff, static_cast<const char*>(k) + koff, klen, cudaMemcpyHostToDevice,
                                    hc->s_in));
            cuda_ok(cudaMemcpyAsync(wv + koff, static_cast<const char*>(v) + koff, klen, cudaMemcpyHostToDevice,
                                    hc->s_in));
        }
        cuda_ok(cudaEventRecord(ev[i], hc->s_in));
    }
    // 3. each piece's attention once its inputs are in, then its outputs back
    for (int i = 0; i < np && ce == cudaSuccess; ++i) {
        const HostPiece& pc = pcs[i];
        const int64_t Bp = pc.b1 - pc.b0, Hkvp = pc.g1 - pc.g0, Hqp = Hkvp * G;
        const int64_t qrow = pc.b0 * Hq + pc.g0 * G;  // first (b, hq) row of the piece
        const int64_t krow = pc.b0 * Hkv + pc.g0;
        bsmt_block_mask bmi = bm;
        bsmt_mask_spec si;
        if (mask_spec != nullptr) {
            si = dspec;
            if (L.Bm > 1) {
                bmi.kv_num_blocks += pc.b0 * L.QB;
                bmi.full_kv_num_blocks += pc.b0 * L.QB;
                bmi.kv_indices += pc.b0 * L.QB * L.KB;
                bmi.full_kv_indices += pc.b0 * L.QB * L.KB;
                bmi.B = static_cast<int32_t>(Bp);
            }
            if (L.has_doc && L.doc_batch > 1) {
                si.q_doc_ids += pc.b0 * M;
                si.kv_doc_ids += pc.b0 * N;
                si.doc_batch = static_cast<int32_t>(Bp);
            }
        }
        bsmt_score_spec sc = dscore;
        for (int j = 0; j < sc.num_ops; ++j) {
            if (sc.ops[j].kind != BSMT_SCORE_ALIBI) continue;
            if (sc.ops[j].slopes != nullptr) {
                sc.ops[j].slopes += pc.g0 * G;
            } else {
                if (sc.ops[j].num_heads <= 0) sc.ops[j].num_heads = static_cast<int32_t>(Hq);
                sc.ops[j].head_offset += static_cast<int32_t>(pc.g0 * G);
            }
        }
        cuda_ok(cudaStreamWaitEvent(s, ev[i], 0));
        if (ce != cudaSuccess) break;
        st = attention(wq + qrow * M * D * 2, wk + krow * N * D * 2, wv + krow * N * D * 2, Bp, Hqp, Hkvp, M, N, D,
                       mask_spec != nullptr ? &bmi : nullptr, mask_spec != nullptr ? &si : nullptr, &sc, scale,
                       enable_gqa, 1, nullptr, nullptr, wo + qrow * M * D * 2, wl + qrow * M, stream);
        if (st != BSMT_OK) {
            join();
            return st;
        }
        cuda_ok(cudaEventRecord(ev[kMaxHostPieces + i], s));
        cuda_ok(cudaStreamWaitEvent(hc->s_out, ev[kMaxHostPieces + i], 0));
        cuda_ok(cudaMemcpyAsync(static_cast<char*>(out) + qrow * M * D * 2, wo + qrow * M * D * 2, Bp * Hqp * M * D * 2,
                                cudaMemcpyDeviceToHost, hc->s_out));
        cuda_ok(cudaMemcpyAsync(lse + qrow * M, wl + qrow * M, Bp * Hqp * M * 4, cudaMemcpyDeviceToHost, hc->s_out));
    }
    join();
    if (ce != cudaSuccess) return fail(BSMT_ERR_CUDA, "host pipeline: %s", cudaGetErrorString(ce));
    return ok();
}
