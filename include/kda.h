/*
 * kda.h -- C ABI of libkda, the B200 (sm_100a) hot path of Kimi Delta
 * Attention (KDA).
 *
 * The operation.  For one attention head, a d_v x d_k state S maps key space
 * to value space.  Each token t updates it in five steps ("You could have come
 * up with Kimi Delta Attention", the KDA state update at the top of the
 * article; the same steps in the GeekNews summary, topic 31925, section
 * "Kimi Delta Attention: per-channel decay"):
 *
 *     S~_t   = S_{t-1} Diag(alpha_t)          forget, one rate per key channel
 *     vhat_t = S~_t k_t                       predict
 *     e_t    = beta_t (v_t - vhat_t)          correct
 *     S_t    = S~_t + e_t k_t^T               write
 *     o_t    = S_t (d_k^{-1/2} q_t)           read (post-write state)
 *
 * The gate is passed as g = log(alpha) <= 0 (GeekNews summary, end of the
 * "diagonal-plus-low-rank transition" section).  Keys are expected to be
 * L2-normalised by the caller (the pages assume normalised keys); the
 * library uses k as given and applies the d_k^{-1/2} query scale itself.
 *
 * Common conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, contiguous,
 *     row-major.  q, k, v, out, per-channel g and every state are 16-byte
 *     aligned (TMA and 128-bit loads); beta, scalar g and cu_seqlens need
 *     only their 4-byte element alignment.  Scratch comes from the caller's
 *     workspace; the one exception is kda_chunk_fwd called without one, which
 *     takes it from the device's stream-ordered memory pool (see there).  No
 *     state is kept between calls.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and never synchronise.  Host-side validation happens
 *     before any launch and returns an error status with nothing launched.
 *   - Errors only the device can see (inconsistent cu_seqlens) are reported
 *     through the optional `dev_status` device word: the kernel ORs in a
 *     KDA_DEV_* bit and skips the offending work; read it after a sync.
 *   - Outputs must not alias inputs (except S in kda_decode_step, which is
 *     updated in place by design).
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,  /* null pointer, negative or inconsistent size */
    KDA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (head size, chunk, dtype) */
    KDA_ERR_MISALIGNED = 3,   /* a pointer breaks its alignment rule (see above) */
    KDA_ERR_CUDA = 4,         /* a CUDA launch or attribute call failed */
    KDA_ERR_TIMEOUT = 5,      /* reserved: a bounded device wait expired */
    KDA_ERR_TOO_LARGE = 6     /* kda_chunk_fwd_noalloc: the shape needs more scratch than
                                 the library's static array holds */
} kda_status_t;

/* Element type of q, k, v and out.  g, beta and every state are always fp32. */
typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype_t;

/* Gate layout (GeekNews summary: "Gated DeltaNet" uses one scalar alpha per
 * token, KDA one alpha per key channel, DeltaNet none). */
typedef enum {
    KDA_GATE_CHANNEL = 0,  /* g: one value per key channel, [.., H, d_k] */
    KDA_GATE_SCALAR = 1,   /* g: one value per (token, head), [.., H]   */
    KDA_GATE_NONE = 2      /* g must be NULL; alpha = 1                  */
} kda_gate_t;

/* Device status bits written (ORed) into *dev_status. */
#define KDA_DEV_BAD_SEQLENS 1  /* cu_seqlens not monotone or beyond T; sequence skipped */
#define KDA_DEV_TIMEOUT 2      /* a bounded wait on an mbarrier expired; tile skipped */

typedef struct {
    int32_t B;          /* batch of sequences (dense); 1 for varlen; decode: N */
    int32_t T;          /* tokens per sequence (dense) or in total (varlen); decode: 1 */
    int32_t H;          /* heads */
    int32_t d_k;        /* key / query head size */
    int32_t d_v;        /* value head size */
    int32_t num_seqs;   /* sequences: B for dense, len(cu_seqlens) - 1 for varlen */
    int32_t dtype;      /* kda_dtype_t */
    int32_t gate;       /* kda_gate_t */
    int32_t chunk;      /* chunk length C of kda_chunk_fwd; ignored by decode */
    int32_t* dev_status;/* optional device int32, see KDA_DEV_*; may be NULL */
    int32_t qk_heads;   /* query/key heads Hk; 0 means H.  See "Grouped value heads". */
} kda_shape_t;

/*
 * Grouped value heads.  H counts value heads: v, out, g, beta and every
 * state have H heads.  q and k may have fewer, Hk = qk_heads, with H a
 * multiple of Hk; value head h then reads query/key head h / (H / Hk), so
 * consecutive groups of H / Hk value heads share one query/key head (the
 * value-head grid axis of the fused recurrent kernel, GeekNews summary,
 * section "fused recurrent kernel for decode").  Below, a q/k layout written
 * [.., H, d_k] means [.., Hk, d_k].  qk_heads = 0 or H is the one-to-one case;
 * any other value that does not divide H returns KDA_ERR_INVALID_ARG.
 */

/*
 * kda_chunk_fwd -- chunkwise-parallel prefill forward.
 *
 * Runs the recurrence above over every token of every sequence and head,
 * returning all outputs and (optionally) each sequence's final state.  It is
 * the chunkwise schedule of the GeekNews summary, section "Chunkwise KDA":
 * per chunk of C tokens, the log-space cumulative decay, the decay-masked
 * key/key and query/key products, a unit-lower-triangular solve for the
 * in-chunk error coupling ("pseudo-values from a triangular solve", the
 * curriculum page's objectives), and the state/output products.  The result
 * equals the token loop up to floating-point rounding.
 *
 * Layouts (tok = B*T packed token rows):
 *   q, k      [B, T, H, d_k]   dtype
 *   v, out    [B, T, H, d_v]   dtype
 *   g         [B, T, H, d_k] fp32 (CHANNEL) | [B, T, H] fp32 (SCALAR) | NULL (NONE)
 *   beta      [B, T, H] fp32
 *   S0, S_T   [num_seqs, H, d_v, d_k] fp32; row = value index, key contiguous.
 *             S0 == NULL: zero initial state.  S_T == NULL: final state not written.
 *   cu_seqlens NULL for a dense batch (num_seqs == B), else device int32
 *             [num_seqs + 1] with B == 1, cu[0] = 0, cu[n] <= cu[n+1], cu[num_seqs] <= T:
 *             sequence n is token rows [cu[n], cu[n+1]).  Chunks never cross a
 *             sequence; the state restarts from S0[n] (or zero) per sequence.
 *             Rows of out not covered by any sequence are left untouched.
 * Support:
 *   KDA_BF16: d_k = d_v = 128, chunk = 64 (tcgen05 tensor-core path), or any
 *             shape the fp32 path takes (CUDA-core path).
 *   KDA_F32:  d_k, d_v multiples of 16 in [16, 128], chunk in {16, 32, 64}.
 *   Anything else returns KDA_ERR_UNSUPPORTED.
 * Schedule and scratch (tensor-core path): every (chunk, head) first computes
 *   its state-independent operands in parallel into a scratch buffer of
 *   kda_chunk_fwd_workspace_size(shape) bytes (about 73 KB per (chunk, head)),
 *   then one sequential scan per (sequence, head) applies the state.
 *   workspace != NULL: caller-owned device memory, 256-byte aligned, at least
 *     that many bytes (else KDA_ERR_MISALIGNED / KDA_ERR_INVALID_ARG); contents
 *     need no initialisation and are garbage afterwards.
 *   workspace == NULL (workspace_bytes ignored): the scratch is allocated with
 *     cudaMallocAsync on `stream` from the current device's default memory pool
 *     and released with cudaFreeAsync on `stream` after the kernels that read it,
 *     so the call stays stream-ordered (and can be captured in a CUDA graph).  A
 *     failed allocation returns KDA_ERR_CUDA with nothing launched.  Callers
 *     that must not allocate pass a workspace or use kda_chunk_fwd_noalloc.
 *   The results do not depend on where the scratch lives.  The CUDA-core path
 *   uses no scratch and ignores the workspace.
 */
kda_status_t kda_chunk_fwd(const kda_shape_t* shape, const void* q, const void* k,
                           const void* v, const float* g, const float* beta,
                           const float* S0, const int32_t* cu_seqlens, void* out,
                           float* S_T, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * Bytes of workspace the two-kernel schedule of kda_chunk_fwd needs for this
 * shape; varlen != 0 for a packed batch (a cu_seqlens array will be passed).
 * Returns 0 for a NULL shape or for shapes whose path uses no workspace (the
 * fp32 CUDA-core path).  74,240 bytes per (chunk, head) plus bookkeeping.
 */
size_t kda_chunk_fwd_workspace_size(const kda_shape_t* shape, int varlen);

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd for callers that cannot allocate.
 *
 * The paper has no counterpart: this is an allocation-free way into the same
 * prefill.  Some callers may not call cudaMalloc (or cudaMallocAsync) at all:
 * code running under an allocator that owns all device memory, inside a
 * region where allocation is forbidden (a CUDA graph being captured by a
 * framework that does not accept allocation nodes, a real-time loop), or a
 * plugin whose host forbids it.  This entry point takes no workspace and
 * allocates nothing: the scratch is a file-scope __device__ array of 160 MiB
 * (167,772,160 bytes) inside the library, which every GPU that loads the library
 * holds until the process exits.
 *
 * Same operation, layouts, support and errors as kda_chunk_fwd, plus:
 *   - shapes whose scratch (kda_chunk_fwd_workspace_size) exceeds 160 MiB return
 *     KDA_ERR_TOO_LARGE with nothing launched (4 sequences x 16 heads x 2048
 *     tokens fit; split larger batches into calls that fit);
 *   - the first call on a device resolves the array's device address with
 *     cudaGetSymbolAddress (this may load the library's module there, which
 *     reserves the 160 MiB) and caches it; make that first call before any stream
 *     capture, as module loading cannot happen inside one;
 *   - every call on a device shares the one array and leaves its contents
 *     behind (each call overwrites what it reads, so no clearing is needed):
 *     calls that may overlap on the GPU (different streams, or several host
 *     threads) race on it and must be ordered by the caller.
 */
kda_status_t kda_chunk_fwd_noalloc(const kda_shape_t* shape, const void* q, const void* k,
                                   const void* v, const float* g, const float* beta,
                                   const float* S0, const int32_t* cu_seqlens, void* out,
                                   float* S_T, void* stream);

/*
 * kda_decode_step -- one fused recurrent token for N sequences.
 *
 * The single-token case of the recurrence (the fused recurrent schedule of the
 * GeekNews summary, section "fused recurrent kernel for decode"): each (n, h)
 * state is read once from HBM, decayed, used for the prediction and the
 * query read, corrected by the rank-1 write and stored back in place.
 *
 * Layouts (N = shape->B, shape->T must be 1):
 *   q, k   [N, H, d_k] dtype       v, out [N, H, d_v] dtype
 *   g      [N, H, d_k] fp32 (CHANNEL) | [N, H] fp32 (SCALAR) | NULL (NONE)
 *   beta   [N, H] fp32
 *   S      [N, H, d_v, d_k] fp32, read and overwritten with the new state.
 * Support: d_k = 128 (bf16 or fp32), any d_v from 1 to 65535*128.  Else
 * KDA_ERR_UNSUPPORTED.
 */
kda_status_t kda_decode_step(const kda_shape_t* shape, const void* q, const void* k,
                             const void* v, const float* g, const float* beta, float* S,
                             void* out, void* stream);

/*
 * kda_recurrent_fwd -- fused recurrent pass over a short run of tokens.
 *
 * The token loop of the recurrence for N sequences of T tokens each, with the
 * state kept in registers across the tokens: S is read from HBM once and
 * written once per call (the multi-token form of the fused recurrent decode
 * schedule, GeekNews summary, section "fused recurrent kernel for decode";
 * suited to short runs -- speculative tokens, short prefills -- where the
 * chunkwise schedule has too few tokens per chunk).  The result equals
 * kda_chunk_fwd with S0 = S_T = S up to floating-point rounding, and equals T
 * calls of kda_decode_step exactly.
 *
 * Layouts (dense batch, N = shape->B, shape->num_seqs must equal N):
 *   q, k   [N, T, H, d_k] dtype      v, out [N, T, H, d_v] dtype
 *   g      [N, T, H, d_k] fp32 (CHANNEL) | [N, T, H] fp32 (SCALAR) | NULL (NONE)
 *   beta   [N, T, H] fp32
 *   S      [N, H, d_v, d_k] fp32, read and overwritten with the state after the T tokens.
 * Alignment: q, k, per-channel g and S 16 bytes; v, out, beta, scalar g 4 bytes.
 * Support: d_k = 128 (bf16 or fp32), any d_v from 1 to 65535*128; T = 0 leaves S as is;
 * T = 1 runs the decode step's kernel (the same arithmetic, at the state-copy rate).
 * Else KDA_ERR_UNSUPPORTED.
 */
/*
 * kda_recurrent_bwd -- gradients of kda_recurrent_fwd (training).
 *
 * For the loss sum(out * d_out) + sum(S_T * d_ST), where (out, S_T) is what
 * kda_recurrent_fwd returns from the state S0 over the T tokens, writes the
 * gradients with respect to every input.  It differentiates the five-step
 * update token by token (the pages give no backward derivation; this is the
 * chain rule of the recurrence itself), walking the tokens in reverse on CUDA
 * cores with the state recomputed from checkpoints kept in the workspace.
 *
 * Layouts as kda_recurrent_fwd (dense batch, N = shape->B, num_seqs == N):
 *   q, k [N, T, Hk, d_k], v, d_out [N, T, H, d_v] dtype; g, beta, S0 as there;
 *   d_ST [N, H, d_v, d_k] fp32 or NULL (zero).
 * Outputs, all fp32 and caller-owned:
 *   dq, dk [N, T, Hk, d_k] (summed over the value heads of a group)
 *   dv     [N, T, H, d_v]
 *   dg     the shape of g (NULL when the gate is KDA_GATE_NONE, required otherwise)
 *   dbeta  [N, T, H]
 *   dS0    [N, H, d_v, d_k], or NULL when not wanted.
 * S0, d_ST and dS0 are 16-byte aligned; the workspace (>= the size below) 16 bytes.
 * dq, dk, dg and dbeta are sums over state rows accumulated with atomic adds, so
 * their last bits may differ from run to run; dv and dS0 are written directly.
 * Support: d_k = 128, d_v from 1 to 65535*16; else KDA_ERR_UNSUPPORTED.
 */
kda_status_t kda_recurrent_bwd(const kda_shape_t* shape, const void* q, const void* k,
                               const void* v, const float* g, const float* beta,
                               const float* S0, const void* d_out, const float* d_ST, float* dq,
                               float* dk, float* dv, float* dg, float* dbeta, float* dS0,
                               void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace kda_recurrent_bwd needs: the state of every (sequence, head)
 * every 8 tokens (fp32). */
size_t kda_recurrent_bwd_workspace_size(const kda_shape_t* shape);

/*
 * kda_chunk_bwd -- gradients of kda_chunk_fwd (training), chunkwise.
 *
 * For the loss sum(out * d_out) + sum(S_T * d_ST), where (out, S_T) is what
 * kda_chunk_fwd returns for the same arguments, writes the gradients with
 * respect to q, k, v, g, beta and S0.  The GeekNews summary of "You could have
 * come up with Kimi Delta Attention" (section "fused recurrent Triton kernel for
 * decode") names the chunkwise schedule as the one for training; the pages give
 * no backward derivation, so this is the chain rule of the chunk map that
 * kda_chunk_fwd computes (cumulative decay, decay-masked Gram products, the
 * triangular solve, the state and output products), undone chunk by chunk:
 *   1. the forward's records;
 *   2. in one launch, side by side: a forward state scan that keeps every chunk's
 *      incoming state (fp32, in the workspace), and a reverse state scan on the
 *      tensor cores: with dS = d_ST, per chunk from the last, dE^T = dS Kd^T +
 *      dO^T Aqk and dS <- dS Diag(e^gamma) + dO^T Qg - dE^T W (the records'
 *      operands, fp16, fp32 accumulation); the final dS is dS0;
 *   3. per (chunk, head) in parallel: the triangular solve's gradient, dv and
 *      dbeta, then dq, dk and dg.  The dense products run on the tensor cores over
 *      two-term fp16 operands; the decay-weighted Gram products and their
 *      gradients on the tensor cores over two-term bf16 operands where one decay
 *      reference holds the chunk, on CUDA cores in fp32 otherwise.
 * Arguments as kda_chunk_fwd (dense or varlen through cu_seqlens, grouped value
 * heads through shape->qk_heads), plus:
 *   d_out  [B, T, H, d_v] bf16, 16-byte aligned
 *   d_ST   [num_seqs, H, d_v, d_k] fp32 or NULL (zero)
 * Outputs, all fp32 and caller-owned, 16-byte aligned unless stated:
 *   dq, dk [B, T, Hk, d_k] (summed over the value heads of a group)
 *   dv     [B, T, H, d_v]
 *   dg     the shape of g (NULL exactly when the gate is KDA_GATE_NONE; a scalar
 *          gate's dg is 4-byte aligned)
 *   dbeta  [B, T, H], 4-byte aligned
 *   dS0    [num_seqs, H, d_v, d_k], or NULL when not wanted.
 * Rows of a packed batch that no sequence covers are left untouched.  With
 * grouped value heads (Hk < H) dq and dk are first zeroed and then summed with
 * atomic adds (their last bits may vary from run to run); otherwise every output
 * is written once and the result is deterministic.
 * Workspace: kda_chunk_bwd_workspace_size(shape, varlen) bytes, 256-byte aligned,
 *   or NULL: the scratch is then taken from the device's stream-ordered pool
 *   (cudaMallocAsync) and returned on `stream` after the last kernel.
 * Support: KDA_BF16 with d_k = d_v = 128 and chunk = 64; else KDA_ERR_UNSUPPORTED.
 * Errors as kda_chunk_fwd; a too-small workspace is KDA_ERR_INVALID_ARG.
 */
kda_status_t kda_chunk_bwd(const kda_shape_t* shape, const void* q, const void* k, const void* v,
                           const float* g, const float* beta, const float* S0,
                           const int32_t* cu_seqlens, const void* d_out, const float* d_ST, float* dq,
                           float* dk, float* dv, float* dg, float* dbeta, float* dS0, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Bytes of workspace kda_chunk_bwd needs (0 for unsupported shapes): the forward's
 * records plus, per (chunk, head), two fp32 states (the incoming state and the
 * outgoing state's gradient), one fp32 C x d_v tile, three fp16 C x d_v operand
 * images and one fp32 C x C tile: 74,240 + 131,072 + 32,768 + 49,152 + 16,384 =
 * 303,616 bytes, and a small header. */
size_t kda_chunk_bwd_workspace_size(const kda_shape_t* shape, int varlen);

kda_status_t kda_recurrent_fwd(const kda_shape_t* shape, const void* q, const void* k,
                               const void* v, const float* g, const float* beta, float* S,
                               void* out, void* stream);

/* Failure-detection self-test.  Every wait of the library's tensor-core kernels is
 * a bounded mbarrier wait: when it runs out, the kernel ORs KDA_DEV_TIMEOUT into
 * *dev_status, lets its own copies and MMAs in flight land, frees its tensor memory
 * and returns, so the context stays usable.  This call launches one 128-thread CTA
 * that takes the same bounded wait, with a budget of budget_us microseconds, on a
 * barrier of its own shared memory:
 *   complete = 0: nothing ever arrives, the wait runs out and KDA_DEV_TIMEOUT is
 *                 ORed into *dev_status;
 *   complete != 0: one thread arrives first, the wait succeeds and *dev_status is
 *                 left as it is.
 * dev_status: device int32 (required, 4-byte aligned).  budget_us: 1 to 1000000,
 * else KDA_ERR_INVALID_ARG.  Asynchronous on `stream`; read *dev_status after a
 * sync.  No other memory is touched. */
kda_status_t kda_selftest_bounded_wait(int32_t* dev_status, uint32_t budget_us, int32_t complete,
                                       void* stream);

/* Human-readable text for a status code (static storage). */
const char* kda_status_str(kda_status_t status);

/* Library version string (static storage). */
const char* kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
