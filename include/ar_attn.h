/*
 * ar_attn.h - C ABI of the QK-RMSNorm sliding-window attention core (sm_100a).
 *
 * The operation (per batch b and head h, queries i and keys j of one sequence):
 *
 *   qhat_i = q_i / sqrt(mean_d q_id^2 + eps),  khat_j likewise     (RMSNorm, no gain)
 *   s_ij   = scale * qhat_i . khat_j          for 0 <= i - j <= window, else masked
 *   lse_i  = log sum_j exp(s_ij),   o_i = sum_j exp(s_ij - lse_i) v_j
 *
 * and its exact gradient with respect to q, k and v.  Sources on the reference
 * pages: the "autoresearch" README (gitee), section 7.3 "CausalSelfAttention"
 * (norm(x) = F.rms_norm(x, (x.size(-1),)) applied to q and k, no weight) and
 * sections 5.2.1-5.2.2 (FlashAttention-3 with window_size = (window, 0); the
 * "SSSL" pattern: S = seq_len/2, L = seq_len, last layer forced to L); the
 * web3.okx.com code review, paragraphs on the QK norm and on the window pattern.
 *
 * Conventions shared by every entry point
 *   - q, k, v, o, dO, dq, dk, dv: bf16, layout [B, T, H, D] contiguous, D = 64 or
 *     128 (128 on the RoPE and no-alloc entry points).
 *   - lse: fp32 [B, H, T], natural logarithm.
 *   - window: a key j is visible to query i iff 0 <= i - j <= window.  window < 0
 *     or window >= T - 1 means full causal attention.  window = 0: each query
 *     sees only itself.
 *   - eps >= 0 and finite; scale > 0 and finite (usually 1/sqrt(D)).
 *   - All pointers are DEVICE pointers of the current CUDA device, 16-byte
 *     aligned (the kernels read them with TMA).  32-byte aligned o, dq, dk, dv
 *     (and q, k) are written (read) by the epilogues with 256-bit accesses,
 *     which is faster; results are identical either way.  The caller owns
 *     every buffer; the library never frees or retains caller memory.
 *   - stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls only enqueue work and return; results are ready when the stream is.
 *   - Return value: AR_OK (0) or a negative AR_ERR_* code.  No exception or
 *     abort crosses the ABI.  Argument errors are detected before any work is
 *     enqueued.  A device-side wait that gives up (AR_ERR_TIMEOUT) is reported
 *     by ar_attn_sync_status().
 *   - Workspace (the backward entry points and the RoPE forward; ar_attn_fwd
 *     needs none): if `workspace` is NULL
 *     the library allocates it stream-ordered (cudaMallocAsync / cudaFreeAsync
 *     on `stream`); otherwise it must hold at least the bytes returned by
 *     entry point's *_workspace_bytes() and be 256-byte aligned.  It is scratch:
 *     its contents on entry do not matter (ar_attn_bwd_rope_saved also reads a
 *     RoPE forward's workspace, as its `saved` argument).
 */
#ifndef AR_ATTN_H
#define AR_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  AR_OK = 0,
  AR_ERR_NULL = -1,        /* a required pointer is NULL */
  AR_ERR_SHAPE = -2,       /* B, T or H <= 0, or sizes overflow the index range */
  AR_ERR_UNSUPPORTED = -3, /* D other than 64 or 128 (or than 128 where only 128 is built) */
  AR_ERR_ALIGN = -4,       /* a pointer is not 16-byte aligned (workspace: 256) */
  AR_ERR_ARG = -5,         /* eps < 0, scale <= 0, or either is not finite */
  AR_ERR_DEVICE = -6,      /* current device is not compute capability 10.0 (B200) */
  AR_ERR_CUDA = -7,        /* a CUDA runtime call failed */
  AR_ERR_TIMEOUT = -8,     /* a device-side wait gave up (reported by sync_status) */
  AR_ERR_WORKSPACE = -9,   /* workspace given but smaller than required */
  AR_ERR_TOO_LARGE = -10,  /* problem exceeds ar_attn_fwd_noalloc's built-in scratch */
  AR_ERR_LAYOUT = -11      /* a kernel found its shared memory misaligned and did not run (sync_status) */
};

/* Forward pass.  Inputs q, k, v; outputs o [B,T,H,D] bf16 and lse [B,H,T] fp32
 * (lse is what ar_attn_bwd needs).  The operation is the one at the top of
 * this file: norm(q), norm(k) as in the "autoresearch" README (gitee), section
 * 7.3 "CausalSelfAttention", then the windowed causal attention of its sections
 * 5.2.1-5.2.2 (FlashAttention-3, window_size = (window, 0)).  One fused kernel
 * on `stream`; allocates nothing and needs no scratch (the per-key norm
 * factors are derived from each K tile inside the kernel).
 * lse may be NULL: the kernel then does not store it.  That is the
 * forward-only use (the README's section 9.4 "evaluate_bpb" runs the model
 * without gradients), and o is identical either way. */
int ar_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                int B, int T, int H, int D, int window, float eps, float scale, void* stream);

/* Bytes of scratch ar_attn_bwd needs (the pages do not describe the backward's
 * storage; this is this library's layout): three fp32 per-(b, h, t) vectors
 * (rounded up to whole 128-token tiles) plus a buffer of bf16 128x128 tiles G^T, one per
 * (query tile, key tile) pair of the causal band of a group of heads: for
 * nq = ceil(T/128), nq(nq+1)/2 tiles of 32 KB per head, for as many heads as
 * fit in 1 GiB (at least one, at most B*H); larger problems are processed in
 * head groups.  Sized for full causal, so it serves every window.  0 on invalid
 * sizes. */
size_t ar_attn_bwd_workspace_bytes(int B, int T, int H, int D);

/* Backward pass: the exact gradient of ar_attn_fwd's o with respect to q, k
 * and v, through the attention and through both RMSNorms.  The pages' training
 * loop runs a forward and a backward pass every step ("autoresearch" README
 * (gitee), section 5.1, the outline of train.py's training loop), through
 * FlashAttention-3's backward (section 5.2.1); the gradient itself is the
 * standard softmax-attention one, with delta = rowsum(dO * o).  Inputs q, k,
 * v, the forward's o and lse, and the upstream gradient dO; outputs dq, dk, dv
 * [B,T,H,D] bf16 (overwritten, not added to).
 * window, eps and scale must be the forward's.  Launches, on `stream`: the
 * pre-pass (delta = rowsum(dO * o), 1/rms(q), lse * log2 e), then per head
 * group the fused backward kernel (dk, dv, and the bf16 tiles G = dS rq rk
 * into the workspace) and the dq kernel (dq = G K and the q-side RMSNorm
 * backward). */
int ar_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                const float* lse, void* dq, void* dk, void* dv,
                int B, int T, int H, int D, int window, float eps, float scale,
                void* workspace, size_t workspace_bytes, void* stream);

/* Grouped K/V heads ("autoresearch" README on gitee, section 7.3: n_kv_head
 * may be smaller than n_head; section 10.2.1, item 4: n_kv_head = n_head / 2).
 * k, v, dk, dv are [B, T, Hkv, D] with Hkv dividing H; q, o, dO, dq stay
 * [B, T, H, D] and lse [B, H, T].  Query head h attends with K/V head
 * h / (H / Hkv) (consecutive query heads share a K/V head, as in
 * FlashAttention), and dk, dv of a K/V head sum the gradients of every query
 * head of its group.  Hkv = H gives exactly ar_attn_fwd / ar_attn_bwd (which
 * call these).  AR_ERR_SHAPE if Hkv < 1 or Hkv does not divide H; otherwise
 * arguments, errors and the workspace contract are those of the functions
 * above.  The backward processes whole groups per launch, so its workspace
 * holds the G tiles of at least one group of H / Hkv query heads. */
int ar_attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                    int B, int T, int H, int Hkv, int D, int window, float eps, float scale, void* stream);
size_t ar_attn_bwd_gqa_workspace_bytes(int B, int T, int H, int Hkv, int D);
int ar_attn_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* dO,
                    const float* lse, void* dq, void* dk, void* dv,
                    int B, int T, int H, int Hkv, int D, int window, float eps, float scale,
                    void* workspace, size_t workspace_bytes, void* stream);

/* The forward with the two steps the pages run just before the core
 * ("autoresearch" README (gitee), section 7.4: rotary position embedding of q
 * and k; section 5.2.3: the value embedding mixed into v on the layers that
 * have one), on the unrotated, unmixed q, k, v.  Q tiles are rotated inside the
 * forward kernel as they land in shared memory; the rotated k and the mixed v
 * are written once into the workspace by a pre-pass (a K or V tile is read by
 * every query-tile unit whose band covers it, so rotating it in each tile
 * costs more than one pass over k and v), and the kernel reads them from there.
 *   rope_cos, rope_sin: bf16 [rope_rows, D/2] (rope_rows >= T), row t holding
 *     position t's cos and sin; row t of q and k becomes
 *     (x1 cos_t + x2 sin_t, -x1 sin_t + x2 cos_t) with x1, x2 its two halves.
 *   ve, ve_gate: both NULL (no value embedding), or ve bf16 [B, T, Hkv, D] and
 *     the gate logits g bf16 [B, T, Hkv]: v becomes v + 2 sigmoid(g) ve.
 *   workspace: at least ar_attn_fwd_rope_workspace_bytes(B, T, Hkv, D, ve != NULL)
 *     bytes, 256-byte aligned (NULL: allocated stream-ordered on `stream`).  It
 *     keeps the rotated k and mixed v after the call: a caller that keeps it
 *     until the backward can pass it to ar_attn_bwd_rope_saved.
 * The rotated and mixed values are rounded to bf16 once, as the pages hold
 * them.  Everything else (layouts, lse optional, grouped K/V heads, errors) is
 * as for ar_attn_fwd_gqa.  AR_ERR_NULL if a table is NULL or only one of ve,
 * ve_gate is; AR_ERR_SHAPE if rope_rows < T; tables and ve 16-byte aligned. */
size_t ar_attn_fwd_rope_workspace_bytes(int B, int T, int Hkv, int D, int with_ve);
int ar_attn_fwd_rope(const void* q, const void* k, const void* v, void* o, float* lse, const void* rope_cos,
                     const void* rope_sin, int rope_rows, const void* ve, const void* ve_gate, int B, int T,
                     int H, int Hkv, int D, int window, float eps, float scale, void* workspace,
                     size_t workspace_bytes, void* stream);

/* Backward of ar_attn_fwd_rope: the gradients with respect to the unrotated,
 * unmixed q, k, v, and (with the value embedding) to ve and the gate logits g.
 * Arguments as for ar_attn_bwd_gqa plus the tables and ve, ve_gate of the
 * forward, and the outputs dve bf16 [B, T, Hkv, D] and dgate fp32 [B, T, Hkv]
 * (all four of ve, ve_gate, dve, dgate NULL without a value embedding).
 * A pre-pass writes the rotated q, k and the mixed v into the workspace (the
 * same bf16 values the forward formed in its tiles); the backward kernels run
 * on them and finish the chain rule in their epilogues: dq = R^T dq_rot and
 * dk = R^T dk_rot with R^T the transposed rotation of the row's position
 * (dx1 = d1 cos - d2 sin, dx2 = d1 sin + d2 cos), dv = dv_mix,
 * dve = 2 sigmoid(g) dv_mix and dgate = (dv_mix . ve) 2 sigmoid(g) (1 - sigmoid(g)).
 * The workspace must hold ar_attn_bwd_rope_workspace_bytes(..., ve != NULL)
 * bytes (NULL: allocated stream-ordered, as for ar_attn_bwd). */
size_t ar_attn_bwd_rope_workspace_bytes(int B, int T, int H, int Hkv, int D, int with_ve);
int ar_attn_bwd_rope(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                     const void* rope_cos, const void* rope_sin, int rope_rows, const void* ve, const void* ve_gate,
                     void* dq, void* dk, void* dv, void* dve, float* dgate, int B, int T, int H, int Hkv, int D,
                     int window, float eps, float scale, void* workspace, size_t workspace_bytes, void* stream);

/* ar_attn_bwd_rope given the forward's pre-pass output, as a training step
 * keeps an activation: `saved` is the workspace that ar_attn_fwd_rope was given
 * for the same k, v, ve, ve_gate and tables, not written since (it holds the
 * rotated k and, with a value embedding, the mixed v: the bf16 values the
 * backward's pre-pass would form again).  The pre-pass then rotates only q.
 * Outputs are bitwise those of ar_attn_bwd_rope.  `saved` is read only and
 * must be 256-byte aligned (AR_ERR_ALIGN otherwise); NULL means
 * ar_attn_bwd_rope.  The workspace requirement is unchanged. */
int ar_attn_bwd_rope_saved(const void* q, const void* k, const void* v, const void* o, const void* dO,
                           const float* lse, const void* rope_cos, const void* rope_sin, int rope_rows,
                           const void* ve, const void* ve_gate, void* dq, void* dk, void* dv, void* dve,
                           float* dgate, int B, int T, int H, int Hkv, int D, int window, float eps, float scale,
                           const void* saved, void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then reads and clears this device's status word.
 * Returns AR_OK, AR_ERR_TIMEOUT if a kernel abandoned a wait since the last
 * call, AR_ERR_LAYOUT if a kernel refused to run, or AR_ERR_CUDA if the
 * synchronisation itself failed.  The pages' own failure handling is at the
 * level of whole runs (the "autoresearch" README (gitee), section 6.3: a run
 * over its time budget is killed and logged as a crash); this is the library's
 * counterpart for one call: no kernel waits forever. */
int ar_attn_sync_status(void* stream);

/* Limit, in nanoseconds, of every device-side wait inside the kernels launched
 * after this call (process-wide; 0 restores the default of 2 s).  A kernel
 * whose wait runs out abandons its work, leaves its outputs unspecified and
 * sets AR_ERR_TIMEOUT for ar_attn_sync_status; the waits that let copies and
 * tensor-core work in flight finish before a CTA exits keep the default limit.
 * Meant for failure-detection tests; a limit far below a kernel's run time
 * makes every call time out.  Returns AR_OK. */
int ar_attn_set_wait_limit_ns(unsigned long long ns);

/* Static, human-readable text for a status code (never NULL). */
const char* ar_attn_strerror(int status);

/* Window of layer `layer` in a stack of n_layer layers following `pattern`
 * (characters 'S' and 'L', case-insensitive; layer l uses pattern[l mod len]):
 * 'L' -> seq_len, 'S' -> seq_len / 2, and the last layer always seq_len
 * ("autoresearch" README (gitee), section 5.2.2, the "SSSL" window pattern;
 * web3.okx.com review, paragraph on the window pattern).
 * Returns a negative AR_ERR_* code on invalid arguments. */
int ar_attn_layer_window(int layer, int n_layer, int seq_len, const char* pattern);

/* Number of visible (query, key) pairs of one head: sum_i (min(i, w) + 1),
 * w = window as above.  Used to count the FLOPs the attention really does
 * (the pages count attention work per visible key: the xyutech.top run log's
 * FLOPs-per-token figure). */
long long ar_attn_unmasked_pairs(int T, int window);

/* Kernel timing for measurement.  Kernel kinds, in launch order: */
enum {
  AR_KERNEL_FWD_PREP = 0, /* per-key norm factors (memory-bound) */
  AR_KERNEL_FWD = 1,      /* fused forward attention (tensor-core bound) */
  AR_KERNEL_BWD_PREP = 2, /* delta, 1/rms(q), lse * log2(e) (memory-bound) */
  AR_KERNEL_BWD = 3,      /* fused backward attention: dk, dv, G tiles (tensor-core bound) */
  AR_KERNEL_DQ = 4,       /* dq = G K with the q-side RMSNorm backward (reads the G tiles) */
  AR_KERNEL_ROPE_PREP = 5, /* rotated k (and q) and mixed v of the RoPE path (memory-bound) */
  AR_KERNEL_KINDS = 6
};

/* on != 0: clear the record and, until called with on == 0, bracket every
 * kernel that the forward and backward entry points launch with CUDA events on the call's
 * stream (a few microseconds of host time per kernel).  on == 0 stops
 * recording and keeps what was recorded for ar_attn_timing_read.  Returns AR_OK. */
int ar_attn_timing_enable(int on);

/* Waits for the recorded events and writes, per kernel kind, the summed device
 * time in milliseconds (ms[AR_KERNEL_KINDS]) and the number of launches
 * (count[AR_KERNEL_KINDS]); either pointer may be NULL.  Clears the record. */
int ar_attn_timing_read(double* ms, long long* count);

/* Forward pass that allocates nothing, for callers that cannot call
 * cudaMalloc: plug-ins whose host application owns the device allocator, or
 * real-time loops that forbid allocation after start-up.  It computes what
 * ar_attn_fwd computes (same arguments) in two launches: a pre-pass writes the
 * per-key norm factors into a fixed array compiled into the library, and the
 * forward kernel reads them from there.  (ar_attn_fwd itself derives the
 * factors inside its kernel and allocates nothing either; this entry point
 * keeps the two-launch form and its contract.)
 * There is no counterpart to this entry point on the reference pages.
 *
 * Limit: B * H * ceil(T / 128) * 128 <= AR_NOALLOC_MAX_KEYS (1,048,576 key
 * rows, i.e. 4 MiB of per-key norm factors); larger problems return
 * AR_ERR_TOO_LARGE without launching anything.
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before capturing a stream into a
 * graph.  Every call on a device shares the one array and leaves its contents
 * behind: calls that can overlap on the GPU (different streams, no ordering
 * between them) race on it and must be serialised by the caller.  Every entry
 * the kernels read is rewritten by the call itself, so no clearing is needed. */
#define AR_NOALLOC_MAX_KEYS (1 << 20)
int ar_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int T, int H, int D, int window, float eps, float scale, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* AR_ATTN_H */
