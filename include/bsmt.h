/*
 * bsmt.h: C ABI of libbsmt, block-sparse masked-tile attention (forward and
 * backward) for NVIDIA B200 (sm_100a).
 *
 * The library builds a block-sparse BlockMask from a composable mask
 * description. It then runs scaled-dot-product attention. The attention
 * kernel skips tiles the BlockMask leaves out and applies the mask only on
 * tiles marked partial.
 *
 * Sources for the operations (page title, section):
 *   - tensorplay.nn.attention API page:
 *     - create_block_mask (signature; mask_mod(b, h, q_idx, kv_idx) -> bool;
 *       separate_full_blocks);
 *     - BlockMask "Basics" (row-wise block lists) and "Details" items 1-2
 *       (kv_num_blocks/kv_indices, full_kv_num_blocks/full_kv_indices);
 *     - and_masks, or_masks, noop_mask, and the causal example.
 *   - L-GATr "attention backends" page, "Why care about Attention Kernels?":
 *     - block-diagonal masks over packed events;
 *     - sliding window, PrefixLM, ALiBi, tanh soft-capping;
 *     - tiled attention that never writes the full matrix.
 *   - FlagAttention page, "Operator overview": layout q [B,Hq,M,D],
 *     k/v [B,Hkv,N,D], MQA/GQA.
 *   - transformerlab page, attention registry table: "sink" (StreamingLLM
 *     first-k sink tokens + window) and "alibi" (m_h * (j - i)).
 *
 * Conventions for every entry point:
 *   - Every call returns a bsmt_status. On failure, bsmt_last_error() gives
 *     a message. The message is thread-local and stays valid until the next
 *     call on the same thread.
 *   - Argument checks happen on the host, before any launch. A call that
 *     returns an error has launched nothing and written nothing.
 *   - Device pointers are owned by the caller. The library never allocates,
 *     frees or keeps device memory beyond the call. Its global device state
 *     is one status word per device and the static split-KV scratch of
 *     bsmt_flex_attention_fwd_splitkv_static (both part of the library's
 *     module, so resident on every device where the module is loaded).
 *     bsmt_flex_attention_host also keeps, per device, two copy streams and
 *     a pool of events, created on its first call there.
 *   - Work is enqueued on the caller's stream (a cudaStream_t passed as
 *     void*; NULL is the legacy default stream). Calls do not synchronize.
 *   - Errors found on the device set the status word and leave the outputs
 *     unspecified. Examples are an invalid block index in a BlockMask, kv
 *     document ids that are not sorted, or a pipeline wait that ran out of
 *     time. bsmt_check_device_status() reads and clears the word.
 *   - No C++ exception crosses this boundary.
 */
#ifndef BSMT_H
#define BSMT_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bsmt_status {
    BSMT_OK = 0,
    BSMT_ERR_INVALID_ARGUMENT = 1,   /* null or misaligned pointer, malformed spec, bad value */
    BSMT_ERR_SHAPE_MISMATCH = 2,     /* shapes that do not fit together (block mask, heads) */
    BSMT_ERR_UNSUPPORTED = 3,        /* valid request outside what this build implements */
    BSMT_ERR_CUDA = 4,               /* a CUDA runtime or driver call failed */
    BSMT_ERR_DEVICE_TIMEOUT = 5,     /* device: a pipeline wait gave up (kernel returned early) */
    BSMT_ERR_DEVICE_BOUNDS = 6,      /* device: a block index outside [0, KB) or lists not ascending */
    BSMT_ERR_DEVICE_PRECONDITION = 7 /* device: kv document ids not non-decreasing */
} bsmt_status;

/* ------------------------------------------------------------------ masks
 * A mask is a postfix (reverse Polish) program of nodes. Leaves push one
 * boolean predicate of (b, q_idx, kv_idx). BSMT_MASK_AND / BSMT_MASK_OR pop
 * `arg` operands (arg >= 1) and push their intersection / union
 * (tensorplay.nn.attention: and_masks, or_masks). A well-formed program
 * leaves exactly one value. None of the predicates depends on the head.
 *
 *   NOOP          always true                                  (noop_mask)
 *   CAUSAL        q_idx >= kv_idx                              (create_block_mask example)
 *   WINDOW  arg=W q_idx - kv_idx < W                           (sliding window)
 *   PREFIX_LM arg=P  kv_idx < P  or  q_idx >= kv_idx           (PrefixLM)
 *   SINK    arg=S kv_idx < S                                   (StreamingLLM sink tokens)
 *   DOCUMENT      q_doc_ids[b][q_idx] == kv_doc_ids[b][kv_idx] (block-diagonal)
 *
 * For DOCUMENT, each kv_doc_ids row must be non-decreasing, as it is for
 * packed documents: each document's keys are contiguous. q_doc_ids may be
 * in any order. bsmt_create_block_mask checks the kv order on the device.
 *
 * The library distributes AND over OR and simplifies as it goes: within an
 * alternative (an AND of leaves), leaves of one kind collapse to the
 * strictest (one CAUSAL, one DOCUMENT, the smallest W, P and S), repeated
 * alternatives merge, and an alternative that another one contains is
 * dropped (each of the other's leaves has one of the same kind in it, at
 * least as strict). The result is the same predicate.
 *
 * Limits: at most BSMT_MAX_MASK_NODES nodes, and at most
 * BSMT_MAX_MASK_TERMS alternatives after the simplification (1024 while
 * the program is evaluated); each alternative then has at most 5 leaves,
 * within BSMT_MAX_MASK_LEAVES. A larger program returns
 * BSMT_ERR_UNSUPPORTED.
 */
#define BSMT_MAX_MASK_NODES 64
#define BSMT_MAX_MASK_TERMS 16
#define BSMT_MAX_MASK_LEAVES 128

enum {
    BSMT_MASK_NOOP = 0,
    BSMT_MASK_CAUSAL = 1,
    BSMT_MASK_WINDOW = 2,
    BSMT_MASK_PREFIX_LM = 3,
    BSMT_MASK_SINK = 4,
    BSMT_MASK_DOCUMENT = 5,
    BSMT_MASK_AND = 6,
    BSMT_MASK_OR = 7
};

typedef struct bsmt_mask_node {
    int32_t kind;  /* BSMT_MASK_* */
    int32_t arg;   /* W, P, S, or operand count for AND/OR; ignored otherwise */
} bsmt_mask_node;

typedef struct bsmt_mask_spec {
    int32_t num_nodes;
    bsmt_mask_node nodes[BSMT_MAX_MASK_NODES];
    /* DOCUMENT only: device int32 arrays, row-major [doc_batch, Q_LEN] and
     * [doc_batch, KV_LEN], 4-byte aligned. doc_batch is 1 (shared by every
     * batch row) or B. */
    const int32_t* q_doc_ids;
    const int32_t* kv_doc_ids;
    int32_t doc_batch;
} bsmt_mask_spec;

/* ------------------------------------------------------------ score mods
 * Applied in order to the scaled score s = scale * q.k of query i, key j and
 * query head h, before masking and softmax. The source is the attention-gym
 * page, "A gallery that grew into a toolkit": score_mod changes a score
 * before the softmax.
 *   SOFTCAP  value = cap > 0:  s <- cap * tanh(s / cap)
 *   ALIBI    s <- s + m_h * (j - i) (transformerlab page, registry table,
 *            "alibi"). The slopes m_h are device float[Hq], or NULL for the
 *            default slopes m_h = 2^(-8(h0 + h + 1) / Ht): h0 = head_offset
 *            and Ht = num_heads place this call's Hq heads inside a model
 *            of Ht heads, so a call on a slice of the heads gets the slopes
 *            of those heads. num_heads <= 0 means Hq (and head_offset must
 *            then be 0); otherwise 0 <= head_offset and
 *            head_offset + Hq <= num_heads, else BSMT_ERR_INVALID_ARGUMENT.
 *            Both fields are ignored when slopes is given and for SOFTCAP.
 */
#define BSMT_MAX_SCORE_OPS 2
enum { BSMT_SCORE_NONE = 0, BSMT_SCORE_SOFTCAP = 1, BSMT_SCORE_ALIBI = 2 };

typedef struct bsmt_score_op {
    int32_t kind;          /* BSMT_SCORE_* */
    float value;           /* SOFTCAP: cap */
    const float* slopes;   /* ALIBI: device float[Hq] or NULL */
    int32_t head_offset;   /* ALIBI default slopes: model head index of this call's head 0 */
    int32_t num_heads;     /* ALIBI default slopes: the model's head count (<= 0: Hq) */
} bsmt_score_op;

typedef struct bsmt_score_spec {
    int32_t num_ops;       /* 0 .. BSMT_MAX_SCORE_OPS */
    bsmt_score_op ops[BSMT_MAX_SCORE_OPS];
} bsmt_score_spec;

/* -------------------------------------------------------------- BlockMask
 * The four int32 tensors of tensorplay.nn.attention's BlockMask ("Details"
 * items 1 and 2), with separate_full_blocks = True:
 *   kv_num_blocks       [B, H, QB]      number of PARTIAL kv blocks per q-block row
 *   kv_indices          [B, H, QB, KB]  their kv block indices, ascending, then 0s
 *   full_kv_num_blocks  [B, H, QB]      number of FULL kv blocks (no masked element)
 *   full_kv_indices     [B, H, QB, KB]  their indices, ascending, then 0s
 * QB = ceil(Q_LEN / BLOCK_Q), KB = ceil(KV_LEN / BLOCK_KV). B and H are 1
 * when the mask is shared across batch rows or heads. All four pointers
 * are caller-owned device memory, contiguous, 4-byte aligned.
 */
typedef struct bsmt_block_mask {
    int32_t* kv_num_blocks;
    int32_t* kv_indices;
    int32_t* full_kv_num_blocks;
    int32_t* full_kv_indices;
    int32_t B, H, QB, KB;
    int32_t Q_LEN, KV_LEN;
    int32_t BLOCK_Q, BLOCK_KV;
} bsmt_block_mask;

/* Shape [B, H, QB, KB] of the BlockMask tensors create_block_mask would
 * write. B <= 0 or H <= 0 means "None" and gives 1. Only 128x128 blocks are
 * supported (BSMT_ERR_UNSUPPORTED otherwise). Host-only; launches nothing. */
bsmt_status bsmt_block_mask_shape(int64_t B, int64_t H, int64_t Q_LEN, int64_t KV_LEN,
                                  int32_t BLOCK_Q, int32_t BLOCK_KV, int64_t out_shape[4]);

/* create_block_mask(mask_mod, B, H, Q_LEN, KV_LEN, BLOCK_SIZE=128) from the
 * tensorplay.nn.attention page, with separate_full_blocks = True.
 *
 * The kernel classifies every 128x128 tile of every (b, h, q-block) row
 * exactly:
 *   - FULL: all 128*128 elements allowed and inside [0,Q_LEN) x [0,KV_LEN);
 *   - EMPTY: no allowed element;
 *   - PARTIAL: otherwise.
 * It then writes the ascending lists and zero-fills their tails.
 *
 * `out` must hold the four device pointers, sized by bsmt_block_mask_shape.
 * The call fills out's shape fields. Stream-ordered on `stream`. */
bsmt_status bsmt_create_block_mask(const bsmt_mask_spec* spec, int64_t B, int64_t H,
                                   int64_t Q_LEN, int64_t KV_LEN, int32_t BLOCK_Q,
                                   int32_t BLOCK_KV, bsmt_block_mask* out, void* stream);

/* q-side lists of a BlockMask: the transpose of its kv-side lists
 * (tensorplay.nn.attention page, BlockMask "Details" items 3 and 4).
 *   q_num_blocks       [B, H, KB]      number of q blocks whose PARTIAL list holds kv block kb
 *   q_indices          [B, H, KB, QB]  those q blocks, ascending, then 0s
 *   full_q_num_blocks  [B, H, KB]      the same for the FULL lists
 *   full_q_indices     [B, H, KB, QB]
 * B, H, QB, KB are the kv-side BlockMask's. Caller-owned device memory,
 * contiguous, 4-byte aligned. */
typedef struct bsmt_block_mask_q {
    int32_t* q_num_blocks;
    int32_t* q_indices;
    int32_t* full_q_num_blocks;
    int32_t* full_q_indices;
} bsmt_block_mask_q;

/* Writes the q-side lists of `kv` (its four kv-side tensors and shape fields
 * are read; the lists may come from bsmt_create_block_mask or from the
 * caller). Every element of the four outputs is written. A kv-side count
 * outside [0, KB] or an index outside [0, KB) is skipped and reported as
 * BSMT_ERR_DEVICE_BOUNDS by bsmt_check_device_status. QB above 12800 returns
 * BSMT_ERR_UNSUPPORTED (the kernel's shared-memory bitmaps). Stream-ordered
 * on `stream`. */
bsmt_status bsmt_block_mask_transpose(const bsmt_block_mask* kv, bsmt_block_mask_q* out, void* stream);

/* Block-level dense map of a BlockMask: dense[b, h, qb, kb] = 1 when the
 * partial or the full list of row (b, h, qb) holds kb, else 0 (the
 * reconstruction loop of tensorplay.nn.attention, BlockMask "Basics").
 * dense is caller-owned device int32 [B, H, QB, KB], 4-byte aligned. Bad
 * counts or indices are skipped and reported as BSMT_ERR_DEVICE_BOUNDS.
 * Stream-ordered on `stream`. */
bsmt_status bsmt_block_mask_to_dense(const bsmt_block_mask* kv, int32_t* dense, void* stream);

/* flex_attention forward with a BlockMask:
 *   out[b,hq,i,:] = softmax_j( mod(scale * q_i . k_j) masked ) @ v
 *   lse[b,hq,i]   = natural log-sum-exp of the modified, masked scores
 *
 * kv head = hq / (Hq / Hkv). A row with no allowed key gets out = 0 and
 * lse = -inf.
 *
 * Arguments:
 *   q       device bf16 [B, Hq, M, D], contiguous, 16-byte aligned
 *   k, v    device bf16 [B, Hkv, N, D], contiguous, 16-byte aligned
 *   D       64 or 128
 *   block_mask  BlockMask for (Q_LEN, KV_LEN) = (M, N) with B in {1, B}
 *           and H in {1, Hq}. NULL means every tile is computed, with no
 *           mask. Tiles that cross the end of the sequences are then still
 *           masked to [0, N).
 *   mask_spec   the mask the BlockMask was built from. The kernel applies it
 *           on PARTIAL tiles only; FULL tiles skip it (tensorplay.nn.attention,
 *           BlockMask "Details" item 2). NULL means NOOP. Ignored when
 *           block_mask is NULL.
 *   score   score mods. NULL means none.
 *   scale   softmax scale; <= 0 selects 1/sqrt(D)
 *   enable_gqa  must be nonzero when Hq != Hkv (Hq must be a multiple of Hkv)
 *   out     device bf16 [B, Hq, M, D], 16-byte aligned
 *   lse     device float [B, Hq, M], 4-byte aligned
 *   A tensor with no elements (M == 0, N == 0 or B == 0) may be NULL.
 *
 * A block listed in both lists of a row is treated as PARTIAL; the order of
 * a list does not matter. A count outside [0, KB] or an index outside
 * [0, KB) is skipped and reported as BSMT_ERR_DEVICE_BOUNDS.
 * N is not limited beyond the int32 positions (< 2^31 - 256): a row's kv
 * blocks are visited in windows of 1024 blocks, in order.
 */
bsmt_status bsmt_flex_attention_fwd(const void* q, const void* k, const void* v,
                                    int64_t B, int64_t Hq, int64_t Hkv, int64_t M, int64_t N,
                                    int64_t D, const bsmt_block_mask* block_mask,
                                    const bsmt_mask_spec* mask_spec,
                                    const bsmt_score_spec* score, float scale,
                                    int32_t enable_gqa, void* out, float* lse, void* stream);

/* ----------------------------------------------------------- split-KV
 * Split-KV forward for rows with few q-blocks and long kv lists (decode-like
 * shapes): the kv entries of every (b, hq, q-block pair) are cut into
 * num_splits consecutive slices that run as separate work units, each
 * writing its slice's normalised output O_s (fp32) and lse_s to a
 * workspace; a second kernel merges them exactly:
 *   lse = log sum_s exp(lse_s),  out = sum_s exp(lse_s - lse) O_s.
 * This is the split reduction of Split-KV FlashAttention (FlagAttention
 * page, "Operator overview"); the result is the same attention as
 * bsmt_flex_attention_fwd, up to rounding. */
#define BSMT_MAX_SPLITS 64

/* Workspace bytes bsmt_flex_attention_fwd_splitkv needs for these sizes
 * (0 when num_splits == 1). Host-only; launches nothing. */
bsmt_status bsmt_splitkv_workspace_bytes(int64_t B, int64_t Hq, int64_t M, int64_t D, int32_t num_splits,
                                         int64_t* bytes);

/* bsmt_flex_attention_fwd with split-KV. Arguments as there, plus:
 *   num_splits       1 .. BSMT_MAX_SPLITS (1 runs the plain path)
 *   workspace        caller-owned device memory, 256-byte aligned, at least
 *                    bsmt_splitkv_workspace_bytes bytes; the call writes it
 *                    and reads it back (no part needs to start zeroed). It
 *                    may be reused once the stream has passed this call.
 *   workspace_bytes  its size
 * A workspace that is NULL, misaligned or too small returns
 * BSMT_ERR_INVALID_ARGUMENT before any launch. */
bsmt_status bsmt_flex_attention_fwd_splitkv(const void* q, const void* k, const void* v, int64_t B, int64_t Hq,
                                            int64_t Hkv, int64_t M, int64_t N, int64_t D,
                                            const bsmt_block_mask* block_mask, const bsmt_mask_spec* mask_spec,
                                            const bsmt_score_spec* score, float scale, int32_t enable_gqa,
                                            int32_t num_splits, void* workspace, int64_t workspace_bytes, void* out,
                                            float* lse, void* stream);

/* Split-KV without a caller workspace. The pages have no counterpart of this
 * entry point: it exists for callers that cannot allocate device memory,
 * such as a server whose memory manager reserves the whole device up front
 * and forbids other allocations, or a plug-in whose host framework owns
 * every allocation. It runs the same computation as
 * bsmt_flex_attention_fwd_splitkv, with the workspace taken from a static
 * device array inside the library (BSMT_SPLITKV_SCRATCH_BYTES per device),
 * and calls no cudaMalloc, cudaFree or allocating library routine.
 *   - The array is part of the library's module: every device on which the
 *     module is loaded holds its 32 MiB until the process exits, whether or
 *     not this call is used.
 *   - Sizes whose workspace (bsmt_splitkv_workspace_bytes) exceeds the
 *     scratch return BSMT_ERR_UNSUPPORTED with the sizes in the message;
 *     nothing is launched.
 *   - The scratch is shared by every call on the device and keeps the last
 *     call's contents. Nothing in it must start at zero: each split writes
 *     every row it owns before the merge reads it. Calls on one stream run
 *     in order, but calls that overlap on the GPU (other streams, other host
 *     threads) race on it and give wrong results. Serialise them, or use the
 *     workspace form.
 *   - The first call on a device does one-time set-up there, with that
 *     device current: it looks the scratch's device address up with
 *     cudaGetSymbolAddress (checked, then kept), sets the kernel's
 *     shared-memory attribute and fetches the tensor-map encoder. Make that
 *     first call before any stream capture. */
#define BSMT_SPLITKV_SCRATCH_BYTES (32LL << 20)
bsmt_status bsmt_flex_attention_fwd_splitkv_static(const void* q, const void* k, const void* v, int64_t B,
                                                   int64_t Hq, int64_t Hkv, int64_t M, int64_t N, int64_t D,
                                                   const bsmt_block_mask* block_mask,
                                                   const bsmt_mask_spec* mask_spec, const bsmt_score_spec* score,
                                                   float scale, int32_t enable_gqa, int32_t num_splits, void* out,
                                                   float* lse, void* stream);

/* --------------------------------------------------------- host buffers
 * flex_attention on inputs and outputs in host memory, end to end: the
 * create_block_mask / flex_attention example of the tensorplay.nn.attention
 * page for a caller whose tensors live on the host. One call
 *   1. copies the document ids and ALiBi slopes (if any) to the device and
 *      builds the BlockMask of mask_spec there (bsmt_create_block_mask, with
 *      B = 1 unless the document ids differ per batch row, and H = 1: the
 *      mask does not depend on the head);
 *   2. cuts the work into about `pieces` independent pieces along (batch
 *      row, group of kv heads with their query heads), and pipelines them:
 *      the host-to-device copy of piece i+1, the attention of piece i and the
 *      device-to-host copy of piece i-1 run at the same time, on two copy
 *      streams of the library and the caller's stream;
 *   3. makes `stream` wait for the last copy, so that once `stream` has
 *      passed the call, out and lse hold the result.
 * Every copy is one cudaMemcpyAsync of a contiguous range.
 *
 * Arguments:
 *   q          host bf16 [B, Hq, M, D], contiguous
 *   k, v       host bf16 [B, Hkv, N, D]
 *   mask_spec  as for bsmt_create_block_mask, but its document id arrays
 *              are HOST int32 [doc_batch, M] and [doc_batch, N]; NULL means
 *              no mask (every tile computed)
 *   score      as for bsmt_flex_attention_fwd, but ALiBi slopes are HOST
 *              float[Hq]; NULL means none
 *   scale, enable_gqa  as for bsmt_flex_attention_fwd
 *   pieces     the number of pieces to aim for (<= 0: 16); at most 256 are
 *              made
 *   workspace  caller-owned device memory, 256-byte aligned, at least
 *              bsmt_flex_attention_host_workspace_bytes bytes: it holds the
 *              device copies of q, k, v, out, lse, the BlockMask, the
 *              document ids and the slopes. Reusable once `stream` has
 *              passed the call.
 *   out        host bf16 [B, Hq, M, D]; lse host float [B, Hq, M]
 * Host buffers should be page-locked (cudaHostAlloc, or torch's
 * pin_memory) so the copies run asynchronously and overlap; pageable memory
 * gives the same result without the overlap. The host inputs must stay
 * unchanged, and out and lse unread, until `stream` has passed the call.
 * Calls on one device take a library lock while they enqueue. Argument
 * errors are returned before anything is enqueued; a CUDA error in the
 * middle returns BSMT_ERR_CUDA with the outputs unspecified. */
bsmt_status bsmt_flex_attention_host_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t M, int64_t N,
                                                     int64_t D, const bsmt_mask_spec* mask_spec, int64_t* bytes);
bsmt_status bsmt_flex_attention_host(const void* q, const void* k, const void* v, int64_t B, int64_t Hq,
                                     int64_t Hkv, int64_t M, int64_t N, int64_t D, const bsmt_mask_spec* mask_spec,
                                     const bsmt_score_spec* score, float scale, int32_t enable_gqa, int32_t pieces,
                                     void* workspace, int64_t workspace_bytes, void* out, float* lse, void* stream);

/* --------------------------------------------------- packed sequences
 * Varlen attention in the cu_seqlens form (L-GATr "attention backends" page:
 * packed events with a block-diagonal mask, and the varlen kernels'
 * cu_seqlens_q / max_seqlen_q). The sequences are packed along one token
 * axis; token t of the pack belongs to sequence i for
 * cu_seqlens[i] <= t < cu_seqlens[i+1].
 *
 * bsmt_seqlens_to_doc_ids writes doc_ids[t] = that i (device int32 [total]),
 * and num_seqs for tokens at or past cu_seqlens[num_seqs]. cu_seqlens
 * (device int32 [num_seqs + 1]) must start at 0 and not decrease; the kernel
 * checks this and reports BSMT_ERR_DEVICE_PRECONDITION. With those ids as
 * DOCUMENT ids (and CAUSAL for causal attention when q and k share
 * cu_seqlens), a BlockMask over (total_q, total_k) with B = H = 1 gives each
 * token exactly the keys of its sequence. Stream-ordered on `stream`. */
bsmt_status bsmt_seqlens_to_doc_ids(const int32_t* cu_seqlens, int32_t num_seqs, int64_t total, int32_t* doc_ids,
                                    void* stream);

/* bsmt_flex_attention_fwd on packed tensors, B = 1:
 *   q    device bf16 [M, Hq, D] (M = total query tokens), contiguous, 16-byte aligned
 *   k, v device bf16 [N, Hkv, D]
 *   out  device bf16 [M, Hq, D]
 *   lse  device float [Hq, M]
 * Everything else as in bsmt_flex_attention_fwd (block_mask has B = 1).
 * Positions seen by the mask and by ALiBi are packed token indices; they
 * equal positions within the sequence only when q and k share cu_seqlens
 * (the Python binding requires that for causal and for ALiBi). */
bsmt_status bsmt_flex_attention_fwd_packed(const void* q, const void* k, const void* v, int64_t Hq, int64_t Hkv,
                                           int64_t M, int64_t N, int64_t D, const bsmt_block_mask* block_mask,
                                           const bsmt_mask_spec* mask_spec, const bsmt_score_spec* score, float scale,
                                           int32_t enable_gqa, void* out, float* lse, void* stream);

/* ------------------------------------------------------------- backward
 * Gradients of the forward above: with dout the gradient arriving at out,
 * dq, dk and dv are the gradients of sum(out * dout) with respect to q, k
 * and v. With s = scale * q.k, z = score_mod(s), P = exp(z - lse) and
 * delta_i = sum_d out[i,d] * dout[i,d]:
 *   dS = P * (dout v^T - delta) * dz/ds
 *   dv = P^T dout,  dk = scale * dS^T q,  dq = scale * dS k
 * summed, for dk and dv, over the query heads of each kv head's GQA group.
 * Masked elements have P = 0; a row with no allowed key (lse = -inf) passes
 * no gradient. The structure follows the tensorplay.nn.attention page,
 * BlockMask "Details" items 3-4: dk and dv walk the q-side lists of the
 * block mask, dq walks its kv-side lists; mask_mod runs on PARTIAL tiles
 * only (the FlagAttention page, "Operator overview", lists forward and
 * backward for the same layouts).
 *
 * bsmt_flex_attention_bwd_workspace_bytes gives the workspace size:
 * 8 * B * Hq * ceil(M / 128) * 128 bytes (lse and delta per query row),
 * rounded up to 256, plus 256 bytes of work counters. Host-only; launches
 * nothing. */
bsmt_status bsmt_flex_attention_bwd_workspace_bytes(int64_t B, int64_t Hq, int64_t M, int64_t* bytes);

/* Arguments:
 *   q, k, v, B, Hq, Hkv, M, N, D, mask_spec, score, scale, enable_gqa
 *           as for bsmt_flex_attention_fwd (the same values as the forward)
 *   out     device bf16 [B, Hq, M, D], the forward's output, 16-byte aligned
 *   dout    device bf16 [B, Hq, M, D], 16-byte aligned
 *   lse     device float [B, Hq, M], the forward's lse, 4-byte aligned
 *   block_mask    the forward's BlockMask, or NULL for every tile
 *   block_mask_q  its q-side lists (bsmt_block_mask_transpose); required
 *           when block_mask is not NULL, ignored otherwise
 *   dq      device bf16 [B, Hq, M, D]; dk, dv device bf16 [B, Hkv, N, D];
 *           16-byte aligned, fully written (zeros where no key or query
 *           reaches)
 *   workspace  caller-owned device memory, 256-byte aligned, at least
 *           bsmt_flex_attention_bwd_workspace_bytes bytes; written and read
 *           back by the call, reusable once the stream has passed it
 * Limits: ceil(M/128) and ceil(N/128) at most 65536, Hq/Hkv at most 255,
 * else BSMT_ERR_UNSUPPORTED. Calls that share a workspace must not overlap in
 * time (it holds the kernels' work counters). Bad list entries are skipped and reported as
 * BSMT_ERR_DEVICE_BOUNDS. Stream-ordered on `stream`. */
bsmt_status bsmt_flex_attention_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
                                    const float* lse, int64_t B, int64_t Hq, int64_t Hkv, int64_t M, int64_t N,
                                    int64_t D, const bsmt_block_mask* block_mask,
                                    const bsmt_block_mask_q* block_mask_q, const bsmt_mask_spec* mask_spec,
                                    const bsmt_score_spec* score, float scale, int32_t enable_gqa, void* dq,
                                    void* dk, void* dv, void* workspace, int64_t workspace_bytes, void* stream);

/* bsmt_flex_attention_bwd on packed tensors (the layouts of
 * bsmt_flex_attention_fwd_packed), B = 1:
 *   q, out, dout, dq  device bf16 [M, Hq, D], 16-byte aligned
 *   k, v, dk, dv      device bf16 [N, Hkv, D]
 *   lse               device float [Hq, M], from the packed forward
 * Everything else as in bsmt_flex_attention_bwd (block_mask has B = 1); the
 * workspace size is bsmt_flex_attention_bwd_workspace_bytes(1, Hq, M). */
bsmt_status bsmt_flex_attention_bwd_packed(const void* q, const void* k, const void* v, const void* out,
                                           const void* dout, const float* lse, int64_t Hq, int64_t Hkv, int64_t M,
                                           int64_t N, int64_t D, const bsmt_block_mask* block_mask,
                                           const bsmt_block_mask_q* block_mask_q, const bsmt_mask_spec* mask_spec,
                                           const bsmt_score_spec* score, float scale, int32_t enable_gqa, void* dq,
                                           void* dk, void* dv, void* workspace, int64_t workspace_bytes,
                                           void* stream);

/* Self-test of the device failure path. Every pipeline wait in the kernels
 * is bounded (2 s); one that runs out records BSMT_ERR_DEVICE_TIMEOUT in the
 * status word and makes the CTA's other waits return, so the kernel ends
 * and the context stays usable. This call runs that path on purpose in a
 * one-CTA kernel: warp 0 waits on an mbarrier that nothing arrives on, warp 1
 * on another one. Afterwards bsmt_check_device_status reports
 * BSMT_ERR_DEVICE_TIMEOUT. result: device int32[3], written as
 * {warp 0 wait completed (0), warp 1 wait completed (0), warp 0 wait time in
 * microseconds (about 2e6)}. Takes about 2 s of GPU time. The pages have no
 * counterpart; it exists to test failure detection without a fault. */
bsmt_status bsmt_selftest_wait_timeout(int32_t* result, void* stream);

/* Thread-local message for the last failed call on this thread ("" if none). */
const char* bsmt_last_error(void);

/* Waits for `stream`, then reads and clears the current device's status
 * word. Returns BSMT_OK or the first BSMT_ERR_DEVICE_* recorded since the
 * last check. */
bsmt_status bsmt_check_device_status(void* stream);

/* ABI version: (major << 16) | minor. */
int32_t bsmt_version(void);

#ifdef __cplusplus
}
#endif
#endif /* BSMT_H */
