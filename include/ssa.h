/*
 * ssa.h -- C ABI of libssa: the hot path of SSA block-sparse attention on one
 * NVIDIA B200 (sm_100a).
 *
 * Method: "SSA: Sparse Sparse Attention by Aligning Full and Sparse Attention
 * Outputs in Feature Space" (arXiv 2511.20102).  Section 3 of the paper defines
 * the sparse stream: keys are cut into contiguous blocks of s tokens, each
 * block is mean-pooled, every preceding block is scored against each query,
 * the top-k blocks are kept per query and attention runs over their k*s tokens.
 * Full causal attention (section 3) runs beside it, and section 5 aligns the
 * two outputs with a bidirectional SmoothL1 loss.
 *
 * Conventions shared by every call
 *  - Tensors are DEVICE pointers allocated and owned by the caller; the library
 *    never frees or retains them.  Q, O, dO, dQ, Of, Os, dOf, dOs are
 *    contiguous [B, H, T, d] and K, V, dK, dV [B, Hkv, T, d] in the element
 *    type `dims->dtype` (bf16 or fp32).  lse / delta are fp32 [B, H, T]; Kbar
 *    is fp32 [B, Hkv, T/s, d]; idx is int32 [B, Hkv, T, k] (one selection per
 *    key/value head).
 *  - Block j covers tokens [j*s, (j+1)*s); b(t) = floor(t/s); nb = T/s.
 *  - Work is enqueued on `stream` and runs asynchronously.  Argument errors are
 *    detected on the host before anything is enqueued and return
 *    SSA_ERR_INVALID_ARG / SSA_ERR_UNSUPPORTED; a failed launch returns
 *    SSA_ERR_CUDA.  A kernel that gives up on an internal wait (a hang guard,
 *    about two seconds) records SSA_ERR_TIMEOUT, read by ssa_get_device_error().
 *  - Supported: bf16 with d == 128 on the tensor-core path; fp32 (any op) and
 *    bf16 with d == 64 on a CUDA-core path; s in {64, 128}; T % s == 0;
 *    1 <= k <= nb; nb <= 1024 for ssa_block_select; on the tensor-core sparse
 *    path also k <= 256, T < 2^23 and B*H*(T*k + 128*nb) < 2^31.
 *  - Workspace: calls that take `ws` need at least ssa_workspace_size(dims, op)
 *    bytes of device memory (16-byte aligned); its contents on entry are
 *    ignored and on exit undefined.  The library allocates nothing.
 *  - Output residual O_lo (optional, bf16 only): a bf16 forward rounds each
 *    output element o to O = bf16(o); when O_lo is not NULL it also stores
 *    O_lo = bf16(o - O), which carries o to about 16 significant bits.  A
 *    backward given O_lo forms D_t = dO_t . (O_t + O_lo_t) instead of
 *    dO_t . O_t.  D multiplies every key's contribution to dQ, so the rounding
 *    of O alone moves dQ by about 2^-9 * |dO| |o| * |mean attended key|; at
 *    long context with concentrated attention that is the largest error of the
 *    backward.  For fp32 tensors O_lo is ignored.
 */
#ifndef SSA_H_
#define SSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ABI-identical to cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *ssa_stream_t;

typedef enum {
    SSA_OK = 0,
    SSA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, inconsistent dims */
    SSA_ERR_UNSUPPORTED = 2, /* valid but outside the supported shapes listed above */
    SSA_ERR_WORKSPACE = 3,   /* ws too small or misaligned */
    SSA_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
    SSA_ERR_TIMEOUT = 5,     /* a kernel gave up on a wait (device error word) */
    SSA_ERR_BAD_INPUT = 6    /* a kernel found an invalid device-side value, e.g. a cache length (device error word) */
} ssa_status_t;

typedef enum { SSA_DT_BF16 = 0, SSA_DT_FP32 = 1 } ssa_dtype_t;

/* Problem shape.  scale is the softmax temperature applied to q.k (1/sqrt(d) is
 * the usual choice; the paper does not print it).  Hkv is the number of
 * key/value heads (0: Hkv = H).  With Hkv < H (grouped-query attention, as in
 * the two-KV-head models of the paper's Appendix C) H must be a multiple of
 * Hkv: query head h reads key/value head h / G, G = H / Hkv, and the G query
 * heads of a group share one block selection, ranked by the sum of their
 * scores q_h . Kbar_j; on the tensor-core path G must divide 128. */
typedef struct {
    int32_t B, H, T, d, s, k;
    int32_t dtype; /* ssa_dtype_t */
    float scale;
    int32_t Hkv;
} ssa_dims_t;

/* Operations that need workspace (argument `op` of ssa_workspace_size). */
enum {
    SSA_OP_SPARSE_FWD = 0,
    SSA_OP_SPARSE_BWD = 1,
    SSA_OP_FULL_FWD = 2,
    SSA_OP_FULL_BWD = 3,
    SSA_OP_ALIGN_FWD = 4,
    SSA_OP_SPARSE_INDEX = 5, /* bytes of the `index` buffer of ssa_sparse_index */
    SSA_OP_DECODE = 6        /* workspace of ssa_sparse_decode */
};

/* ssa_block_select flags. */
enum {
    /* Always keep the query's own block b(t) (counted within k).  This is the
     * only mode implemented; flags without this bit return SSA_ERR_UNSUPPORTED. */
    SSA_SEL_FORCE_CURRENT = 1u
};

/* Bytes of workspace needed by `op` for these dims (0 when none, or when the
 * dims are invalid). */
size_t ssa_workspace_size(const ssa_dims_t *dims, int op);

/*
 * Block pooling (paper section 3: each block of keys is summarised by the mean
 * of its keys, which the queries are scored against).
 * Kbar[b,h,j,:] = (1/s) * sum_{t in block j} K[b,h,t,:], fp32 accumulation,
 * unweighted.
 *   K    in   [B,H,T,d] dtype
 *   Kbar out  [B,H,T/s,d] fp32
 */
ssa_status_t ssa_block_pool(const ssa_dims_t *dims, const void *K, float *Kbar, ssa_stream_t stream);

/*
 * Per-query causal top-k block selection (paper section 3: score preceding
 * blocks with the pooled keys, keep the top-k; receptive field k*s).
 * Row t of idx holds the query's own block b(t) plus the k-1 highest-scoring
 * strictly preceding blocks, score r_j = q_t . Kbar_j evaluated in fp32; equal
 * scores go to the lower block index.  Entries are ascending; when fewer than
 * k-1 blocks precede, the row is padded with -1 at the end.  The softmax scale
 * does not affect the ranking.
 *   Q    in   [B,H,T,d] dtype
 *   Kbar in   [B,H,T/s,d] fp32 (from ssa_block_pool)
 *   idx  out  [B,H,T,k] int32
 *   flags     SSA_SEL_FORCE_CURRENT
 */
ssa_status_t ssa_block_select(const ssa_dims_t *dims, const void *Q, const float *Kbar, int32_t *idx,
                              unsigned flags, ssa_stream_t stream);

/*
 * Inverse selection index (a layout of idx, no counterpart in the paper): for
 * every head and key block j, the (query, slot) pairs whose selection row
 * holds j, in ascending query order, plus the list position of every
 * (query, slot).  The tensor-core sparse attention kernels are key-block-major
 * and read it; it depends only on idx, so one build serves the forward and
 * the backward of a step.  Deterministic (no atomics decide an order).
 *   idx    in   [B,H,T,k] int32 as produced by ssa_block_select
 *   index  out  >= ssa_workspace_size(dims, SSA_OP_SPARSE_INDEX) bytes of
 *               device memory, 16-byte aligned; opaque to the caller
 * Returns SSA_OK without work (and needs 0 bytes) for shapes that run on the
 * CUDA-core path (fp32, or d == 64), which read idx directly.
 */
ssa_status_t ssa_sparse_index(const ssa_dims_t *dims, const int32_t *idx, void *index, size_t index_bytes,
                              ssa_stream_t stream);

/*
 * Sparse attention forward (paper section 3: the selected blocks' tokens form
 * the reduced key and value matrices).  For every query t,
 *   o_t = softmax_{u in S(t)}(scale * q_t . k_u) v_u,
 * S(t) = tokens of the blocks in idx[t] with position <= t (causal inside the
 * query's own block); lse[t] = log sum_{u in S(t)} exp(scale * q_t . k_u).
 *   idx    in   [B,H,T,k] int32, rows as produced by ssa_block_select
 *               (ascending, distinct, -1 padding at the end, containing b(t))
 *   index  in   NULL, or the output of ssa_sparse_index for this idx (the call
 *               then skips its own index build)
 *   O      out  [B,H,T,d] dtype;  O_lo out (optional, see above);  lse out [B,H,T] fp32
 *   ws          >= ssa_workspace_size(dims, SSA_OP_SPARSE_FWD) bytes
 */
ssa_status_t ssa_sparse_attn_fwd(const ssa_dims_t *dims, const void *Q, const void *K, const void *V,
                                 const int32_t *idx, const void *index, void *O, void *O_lo, float *lse, void *ws,
                                 size_t ws_bytes, ssa_stream_t stream);

/* Bits of the `accumulate` argument of the attention backward calls. */
enum {
    SSA_BWD_ACCUMULATE = 1u, /* add into dQ, dK, dV instead of overwriting them */
    SSA_BWD_GRAD_FP32 = 2u   /* dQ, dK, dV are fp32 (two streams then sum without intermediate rounding) */
};

/*
 * Sparse attention backward (paper section 4.2: keys outside S(t) take no part
 * in the normalisation and receive no gradient; no gradient flows through the
 * selection or the pooling).  With P the sparse softmax weights and
 * D_t = dO_t . o_t:
 *   dQ_t = scale sum_{u in S(t)} P_tu (dO_t.v_u - D_t) k_u
 *   dK_u = scale sum_{t: u in S(t)} P_tu (dO_t.v_u - D_t) q_t
 *   dV_u = sum_{t: u in S(t)} P_tu dO_t
 *   O, O_lo, lse in  outputs of ssa_sparse_attn_fwd for the same Q, K, V, idx
 *                    (O_lo may be NULL: D is then formed from O alone)
 *   dO           in  [B,H,T,d] dtype
 *   index        in  NULL or the output of ssa_sparse_index for this idx
 *   dQ, dK, dV   out [B,H,T,d] in dtype, or fp32 with SSA_BWD_GRAD_FP32
 *   accumulate   bit set: SSA_BWD_ACCUMULATE adds to the gradients' current
 *                    contents (sum formed in fp32, then rounded once);
 *                    SSA_BWD_GRAD_FP32 makes dQ, dK, dV fp32 tensors (16-byte
 *                    aligned), which the backward reduces into directly; other
 *                    bits return SSA_ERR_INVALID_ARG
 *   ws               >= ssa_workspace_size(dims, SSA_OP_SPARSE_BWD) bytes
 */
ssa_status_t ssa_sparse_attn_bwd(const ssa_dims_t *dims, const void *Q, const void *K, const void *V,
                                 const void *O, const void *O_lo, const float *lse, const void *dO,
                                 const int32_t *idx, const void *index, void *dQ, void *dK, void *dV, int accumulate,
                                 void *ws, size_t ws_bytes, ssa_stream_t stream);

/*
 * Full causal attention forward (paper section 3: full attention uses all
 * preceding tokens): S(t) = {0..t}; outputs (O, optional O_lo, lse) as for
 * ssa_sparse_attn_fwd.
 *   ws  >= ssa_workspace_size(dims, SSA_OP_FULL_FWD) bytes (0 today; may be NULL)
 */
ssa_status_t ssa_full_attn_fwd(const ssa_dims_t *dims, const void *Q, const void *K, const void *V, void *O,
                               void *O_lo, float *lse, void *ws, size_t ws_bytes, ssa_stream_t stream);

/*
 * Full causal attention backward: the formulas of ssa_sparse_attn_bwd with
 * S(t) = {0..t}.  Same argument meaning and accumulate rule.
 */
ssa_status_t ssa_full_attn_bwd(const ssa_dims_t *dims, const void *Q, const void *K, const void *V,
                               const void *O, const void *O_lo, const float *lse, const void *dO, void *dQ, void *dK,
                               void *dV, int accumulate, void *ws, size_t ws_bytes, ssa_stream_t stream);

/*
 * Bidirectional output alignment, forward (paper section 5: full-attention
 * outputs are trained toward the sparse ones, a commitment term keeps the
 * sparse outputs near the full ones, SmoothL1 for both, weighted by alpha).
 *   loss = w_sparsity * mean l(Of - sg(Os)) + w_commit * mean l(Os - sg(Of))
 *   kind SSA_ALIGN_SMOOTH_L1: l(x) = 0.5 x^2 / beta for |x| < beta, |x| - 0.5 beta otherwise
 *   kind SSA_ALIGN_L2:        l(x) = 0.5 x^2 / beta for every x (the adjusted L2
 *                             of the section 7.5 ablation, read as SmoothL1's
 *                             quadratic branch kept everywhere)
 *   the mean runs over all B*H*T*d elements.  One-way alignment (the ablation's
 *   other variant) is w_commit = 0 or w_sparsity = 0.
 *   Of, Os   in   [B,H,T,d] dtype (full / sparse attention outputs)
 *   beta     > 0
 *   loss_dev out  one fp32 on the device
 *   ws            >= ssa_workspace_size(dims, SSA_OP_ALIGN_FWD) bytes
 */
enum { SSA_ALIGN_SMOOTH_L1 = 0, SSA_ALIGN_L2 = 1 };
ssa_status_t ssa_align_loss_fwd(const ssa_dims_t *dims, const void *Of, const void *Os, int kind, float beta,
                                float w_sparsity, float w_commit, float *loss_dev, void *ws, size_t ws_bytes,
                                ssa_stream_t stream);

/*
 * Alignment backward with the stop-gradients of section 5:
 *   dOf = g * w_sparsity * l'(Of - Os) / n
 *   dOs = g * w_commit   * l'(Os - Of) / n
 * g = *dloss_dev (device fp32 scalar), n = B*H*T*d, l as for the forward
 * (same kind and beta).  accumulate is a bit set:
 * SSA_ACC_OF adds the result into dOf, SSA_ACC_OS into dOs (sum in fp32, one
 * rounding); a clear bit overwrites.  This lets the main stream's upstream
 * gradient, preloaded into its buffer, receive the alignment gradient in place.
 */
enum { SSA_ACC_OF = 1u, SSA_ACC_OS = 2u };
ssa_status_t ssa_align_loss_bwd(const ssa_dims_t *dims, const void *Of, const void *Os, int kind, float beta,
                                float w_sparsity, float w_commit, const float *dloss_dev, void *dOf, void *dOs,
                                int accumulate, ssa_stream_t stream);

/*
 * Dropped attention mass (paper section 4.2 and Appendix B: the approximation
 * error is linear in the full-attention mass outside S(t)):
 *   delta[t] = 1 - exp(lse_sparse[t] - lse_full[t])
 *   lse_sparse, lse_full in [B,H,T] fp32;  delta out [B,H,T] fp32
 */
ssa_status_t ssa_dropped_mass(const ssa_dims_t *dims, const float *lse_sparse, const float *lse_full, float *delta,
                              ssa_stream_t stream);

/*
 * Full causal attention backward that allocates nothing and takes no workspace.
 * The paper has no counterpart: this entry point exists for callers that cannot
 * allocate device memory at the point of the call -- for example code running
 * inside a host that owns every allocation through its own pool and forbids
 * others, or a real-time path that must not call cudaMalloc (which may
 * synchronise the device).  Same arguments and results as ssa_full_attn_bwd
 * without ws / ws_bytes.
 *  - Scratch: a file-scope device array of SSA_NOALLOC_SCRATCH_BYTES (32 MiB)
 *    inside libssa, present on every GPU that loads the library until the
 *    process exits.  The call needs ssa_workspace_size(dims, SSA_OP_FULL_BWD)
 *    bytes of it (bf16, d = 128: 516 bytes per query row, so at most 65,027
 *    rows B*H*T); larger problems return SSA_ERR_WORKSPACE before anything is
 *    enqueued.
 *  - Each call looks up the array's device address in the current device's
 *    context (cudaGetSymbolAddress, which allocates nothing).  The first call
 *    on a device may load the library's device code into that context; make
 *    this first call before any stream capture begins.
 *  - Every call shares the one array and leaves its contents behind; the parts
 *    that must start at zero are cleared by the call itself on `stream`.  Calls
 *    that overlap on the GPU (other streams, other host threads) race on the
 *    scratch: serialise them.
 *  - No cudaMalloc, cudaFree or allocating library routine is called.
 */
#define SSA_NOALLOC_SCRATCH_BYTES (32u << 20)
ssa_status_t ssa_full_attn_bwd_noalloc(const ssa_dims_t *dims, const void *Q, const void *K, const void *V,
                                       const void *O, const void *O_lo, const float *lse, const void *dO, void *dQ,
                                       void *dK, void *dV, int accumulate, ssa_stream_t stream);

/* Synchronises `stream`, then reads and clears the device error word:
 * SSA_OK, SSA_ERR_TIMEOUT when a kernel gave up on a wait since the last call,
 * SSA_ERR_BAD_INPUT when a kernel found an invalid device-side value;
 * SSA_ERR_CUDA when the synchronisation itself failed. */
ssa_status_t ssa_get_device_error(ssa_stream_t stream);

/*
 * Sparse decoding with a key/value cache (paper section 3 applied to one new
 * query per sequence; the paper's own kernel keeps no cache, Appendix E).
 * Sequence b's new token sits at position L = cache_len[b] (0 <= L < T), its
 * key and value already written to row L of the caches.  The call
 *   - selects, per key/value head, the query's own block b(L) and the k-1
 *     complete preceding blocks with the highest scores (group query . Kbar_j,
 *     the group's query being the fp32 sum of its G heads' rows), ties to the
 *     lower index, written ascending with -1 padding to idx;
 *   - attends each query head over the selected blocks' tokens up to L;
 *   - when L + 1 completes block b(L), writes that block's mean key into
 *     Kbar_cache (read by the following steps; fill the complete blocks of a
 *     prompt with ssa_block_pool once).
 *   dims        B sequences, H / Hkv heads, T = cache capacity (multiple of s),
 *               d = 128, bf16, s, k, scale; nb = T/s <= 1024, H/Hkv <= 16
 *   cache_len   in   [B] int32, device
 *   q           in   [B, H, d] bf16
 *   Kcache, Vcache in [B, Hkv, T, d] bf16
 *               q, Kcache and Vcache need 16-byte aligned base addresses (the selected
 *               blocks are bulk-copied; SSA_ERR_INVALID_ARG otherwise)
 *   Kbar_cache  in/out [B, Hkv, T/s, d] fp32: rows j < b(L) are read, row b(L)
 *               is written when the token completes it
 *   idx         out  [B, Hkv, k] int32
 *   o           out  [B, H, d] bf16;  lse out [B, H] fp32
 *   ws               >= ssa_workspace_size(dims, SSA_OP_DECODE) bytes
 * A cache length outside [0, T) records SSA_ERR_BAD_INPUT in the device error
 * word (the row's outputs are then undefined).
 */
ssa_status_t ssa_sparse_decode(const ssa_dims_t *dims, const int32_t *cache_len, const void *q, const void *Kcache,
                               const void *Vcache, float *Kbar_cache, int32_t *idx, void *o, float *lse, void *ws,
                               size_t ws_bytes, ssa_stream_t stream);

/*
 * Rotary position embedding, in place (the models of the paper's section 6 put
 * rotary positions on q and k; continued training at 32k uses a scaling factor
 * of 4, Appendix K).  Rotate-half form: for i < d/2 the pair (x_i, x_{i+d/2})
 * of the row at position p = pos0 + t turns by
 *   a = p * base^(-2i/d) / factor
 * (angles in fp64); transpose != 0 turns by -a, which maps the gradient of the
 * rotated tensor to the gradient of its input.  Apply it to Q (heads = H) and
 * K (heads = Hkv) before ssa_block_pool and the attention calls, and with
 * transpose to dQ, dK after the backward calls.
 *   X      in/out  [B, heads, T, d] in dims->dtype (bf16 or fp32; fp32 also for
 *                  fp32 gradients of bf16 inputs: pass dims with dtype fp32)
 *   pos0   >= 0, position of row t = 0;  base > 1;  factor > 0
 */
ssa_status_t ssa_rope(const ssa_dims_t *dims, void *X, int heads, int pos0, float base, float factor, int transpose,
                      ssa_stream_t stream);

/*
 * Self-test of the hang guard (no counterpart in the paper).  Every wait of the
 * tensor-core kernels is bounded: one that does not complete in time records
 * SSA_ERR_TIMEOUT in the device error word, lets its CTA finish and returns,
 * so the CUDA context stays usable.  This call exercises that path on demand:
 * it launches one warp that waits on a barrier nothing completes, with the
 * same bounded wait limited to limit_ns (1 us .. 1 s, else
 * SSA_ERR_INVALID_ARG), and returns once the kernel is enqueued.  The next
 * ssa_get_device_error() returns SSA_ERR_TIMEOUT and clears the word.
 */
ssa_status_t ssa_wait_probe(uint64_t limit_ns, ssa_stream_t stream);

/* Static, human-readable name of a status code. */
const char *ssa_status_string(ssa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* SSA_H_ */
