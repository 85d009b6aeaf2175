/*
 * vgv.h — C ABI of the B200 (sm_100a) verifier hot path of jina-ocr-v1's decoder:
 * the MoE feed-forward layer and the greedy-verify epilogue.
 *
 * Sources for what is computed:
 *  - decoder shape: 12 layers, hidden 1280, 64 routed + 2 shared experts with
 *    top-6 routing, 129,280-token vocabulary — jina-ocr-v1 model card
 *    (jina.ai/ko), architecture paragraph; "Jina OCR v1: Быстрый парсинг
 *    документов на GPU с 24 ГБ VRAM" (aikraft.ru), "01 Архитектура и
 *    эффективность";
 *  - six routed experts per token plus two shared ones — "Jina AI's 3.4B OCR
 *    model targets faster page parsing" (alphasignal.ai), "A compressed visual
 *    front end";
 *  - greedy verification, longest agreeing prefix, lossless — "jina-ocr-v1:
 *    Schnellere Dokumentenanalyse auf kostengünstigen GPUs" (jina.ai/de),
 *    "Modell und Training"; bonus token counted in tau — same page,
 *    "Spekulatives Decoding auf einer L4".
 *
 * Conventions shared by every call
 *  - All tensors are caller-owned device memory, row-major, dense. bf16 tensors
 *    are passed as void*. Pointers must be 16-byte aligned (256-byte aligned
 *    recommended); the library never allocates, frees or synchronises in the
 *    compute calls. Calls are asynchronous on the given stream and can be
 *    captured in a CUDA graph.
 *  - Every argument is validated before any launch. On a validation error
 *    nothing is launched and no output is touched.
 *  - Launch failures return VG_ERR_CUDA. Faults detected on the device (a wait
 *    that timed out, an index out of range) are recorded in a per-device status
 *    word read by vg_get_device_status; kernels never trap.
 *  - The only supported MoE shape is hidden 1280, expert width 896, 64 routed
 *    experts, 2 shared experts, top-6 (VG_ERR_UNSUPPORTED otherwise). The LM
 *    head requires hidden 1280 and any vocabulary size 1..2^31-1.
 *  - T = 0 (or B = 0) is a valid no-op returning VG_OK.
 */
#ifndef VGV_H
#define VGV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* vg_stream_t;

typedef enum vg_status {
  VG_OK = 0,
  VG_ERR_INVALID_ARG = 1,   /* null required pointer, negative size, aliasing, misalignment */
  VG_ERR_UNSUPPORTED = 2,   /* dimensions other than the supported shape */
  VG_ERR_WORKSPACE = 3,     /* workspace null, not 16-byte aligned, or smaller than the *_workspace_bytes query */
  VG_ERR_CUDA = 4,          /* a CUDA runtime/driver call or launch failed */
  VG_ERR_TIMEOUT = 5,       /* device: a bounded wait ran out (recorded in the status word) */
  VG_ERR_DEVICE_BOUNDS = 6  /* device: an index check failed (recorded in the status word) */
} vg_status;

/* MoE layer dimensions: hidden H, expert width I, routed experts E, shared
 * experts S, experts per token k. Supported: {1280, 896, 64, 2, 6}. */
typedef struct vg_moe_dims {
  int32_t hidden;
  int32_t intermediate;
  int32_t n_routed;
  int32_t n_shared;
  int32_t top_k;
} vg_moe_dims;

/* Optional views into the layer's intermediates. Each non-NULL pointer is used
 * by the layer as the storage of that intermediate (so it costs nothing extra);
 * after the call it holds the value. All are device pointers.
 *  topk_idx       int32 [T, k]   selected experts, descending router logit,
 *                                equal logits ordered by lower expert index
 *  topk_weight    fp32  [T, k]   softmax over all E logits at those experts
 *  expert_offsets int32 [E + 1]  segment start of each routed expert in the
 *                                permutation; [E] = T*k
 *  perm           int32 [T*k]    perm[p] = assignment id t*k + j at position p
 *                                (stable by assignment id within an expert)
 *  inv_perm       int32 [T*k]    inv_perm[t*k + j] = its position p
 *  act            bf16  [(k+S)*T, I]  SwiGLU activations: rows 0..T*k-1 routed
 *                                in permutation order, row k*T + s*T + t is
 *                                shared expert s on token t
 *  expert_out     bf16  [(k+S)*T, H]  unweighted expert outputs, same rows */
typedef struct vg_moe_taps {
  int32_t* topk_idx;
  float* topk_weight;
  int32_t* expert_offsets;
  int32_t* perm;
  int32_t* inv_perm;
  void* act;
  void* expert_out;
} vg_moe_taps;

/* Human-readable name of a status code (static storage). */
const char* vg_status_string(vg_status s);

/* Version of this ABI (incremented on any incompatible change). */
int32_t vg_abi_version(void);

/* Bytes of workspace vg_moe_ffn needs for up to T_max tokens; 0 if the dims
 * are unsupported or T_max < 0. */
size_t vg_moe_workspace_bytes(const vg_moe_dims* dims, int32_t T_max);

/* One MoE feed-forward layer over T tokens.
 *   logits l[t,e] = (q0 + q1) + (q2 + q3) in fp32, q_i = fp32 fma chain of
 *                   x[t,h]*router_w[e,h] over the i-th contiguous quarter of h
 *                   in increasing h, starting at +0; then + router_bias[e]
 *                   (fp32) if given;
 *   idx   = the top_k experts by (l descending, e ascending);
 *   g     = softmax over all E logits at idx (no renormalisation);
 *   y[t]  = sum_j g[t,j] * SwiGLU_{idx[t,j]}(x[t]) + sum_s SwiGLU^shared_s(x[t]),
 *           SwiGLU_W(x) = W_down (silu(W_gate x) * (W_up x)), silu(z) = z/(1+e^-z);
 *   out   = bf16(x + y) if add_residual else bf16(y).
 * Arguments:
 *   x            bf16 [T, H]
 *   router_w     bf16 [E, H]
 *   router_bias  fp32 [E] or NULL
 *   expert_w     bf16 [E][gate [I,H] | up [I,H] | down [H,I]], each expert one
 *                contiguous block of 3*I*H elements
 *   shared_w     bf16 [S][same layout]
 *   out          bf16 [T, H]; must not overlap x or the workspace
 *   taps         NULL or optional intermediate storage (above)
 *   workspace    device buffer of at least vg_moe_workspace_bytes(dims, T)
 * Errors: VG_ERR_INVALID_ARG, VG_ERR_UNSUPPORTED, VG_ERR_WORKSPACE, VG_ERR_CUDA. */
vg_status vg_moe_ffn(const vg_moe_dims* dims, int32_t T,
                     const void* x, const void* router_w, const float* router_bias,
                     const void* expert_w, const void* shared_w,
                     int32_t add_residual, void* out, const vg_moe_taps* taps,
                     void* workspace, size_t workspace_bytes, vg_stream_t stream);

/* Bytes of workspace vg_moe_ffn_stack needs for up to T_max tokens. */
size_t vg_moe_stack_workspace_bytes(const vg_moe_dims* dims, int32_t T_max);

/* The decoder's layer loop over its MoE feed-forward layers:
 * x_{l+1} = bf16(x_l + MoE_l(x_l)) for l = 0..n_layers-1, out = x_{n_layers}.
 * router_w, router_bias, expert_w, shared_w are HOST arrays of n_layers device
 * pointers (router_bias may be NULL, or hold NULL entries). out [T,H] must not
 * overlap x. n_layers >= 1. */
vg_status vg_moe_ffn_stack(const vg_moe_dims* dims, int32_t n_layers, int32_t T,
                           const void* x, const void* const* router_w,
                           const float* const* router_bias,
                           const void* const* expert_w, const void* const* shared_w,
                           void* out, void* workspace, size_t workspace_bytes,
                           vg_stream_t stream);

/* Bytes of workspace vg_verify_greedy needs (8 per verify row + 256); 0 if the
 * arguments are invalid. */
size_t vg_verify_workspace_bytes(int32_t B, int32_t K, int32_t H, int32_t V);

/* Greedy verification of B sequences with K drafted tokens each.
 *   z[r,v]   = sum_h h[r,h] * lm_head[v,h], accumulated in fp32 on tensor cores
 *              (never stored);
 *   argmax[r] = smallest v with z[r,v] = max_v z[r,v];
 *   accepted[b] = the largest a <= K with drafts[b,i] == argmax[b*(K+1)+i] for
 *              all i < a;
 *   out_tokens[b] = drafts[b, 0..a-1], then argmax[b*(K+1)+a] (the bonus
 *              token), then -1 up to K+1 entries.
 * Arguments:
 *   h          bf16 [B*(K+1), H]; row b*(K+1)+i is position i of sequence b
 *   lm_head    bf16 [V, H]
 *   drafts     int32 [B, K] (may be NULL when K == 0); drafts[b,i] proposes
 *              position i+1; values outside [0,V) are valid and never accepted
 *   argmax     int32 [B*(K+1)]   (out)
 *   accepted   int32 [B]         (out)
 *   out_tokens int32 [B, K+1]    (out)
 *   workspace  device buffer of at least vg_verify_workspace_bytes(B,K,H,V),
 *              16-byte aligned, ZERO-FILLED before its first call (e.g.
 *              cudaMemset to 0 once after allocating it); every call leaves it
 *              zero-filled again, so it can be reused by later calls (one call
 *              at a time) without clearing. It holds each row's running
 *              argmax key and a counter of finished CTAs; a counter found
 *              non-zero records VG_ERR_DEVICE_BOUNDS.
 * One kernel launch: the LM-head GEMM, the argmax and the accept; the kernel
 * starts streaming the LM head while the previous kernel in the stream is
 * still running and reads h only after that kernel has finished.
 * H must be 1280; K >= 0; B*(K+1) < 2^24.
 * Errors: VG_ERR_INVALID_ARG, VG_ERR_UNSUPPORTED, VG_ERR_WORKSPACE, VG_ERR_CUDA. */
vg_status vg_verify_greedy(int32_t B, int32_t K, int32_t H, int32_t V,
                           const void* h, const void* lm_head, const int32_t* drafts,
                           int32_t* argmax, int32_t* accepted, int32_t* out_tokens,
                           void* workspace, size_t workspace_bytes, vg_stream_t stream);

/* Kernel kinds for the timing hook. */
typedef enum vg_kernel {
  VG_KERNEL_ROUTER = 0,    /* router + top-k (+ grouping, and the previous layer's
                              combine inside a layer stack, at decode sizes) */
  VG_KERNEL_GROUPING = 1,  /* histogram, stable permutation, row gather (large T) */
  VG_KERNEL_EXPERTS = 2,   /* expert GEMMs: gate/up + SwiGLU, then down (one launch) */
  VG_KERNEL_COMBINE = 3,   /* weighted combine + shared experts + residual (a
                              layer's own output, or the stack's last layer) */
  VG_KERNEL_LM_HEAD = 4,   /* LM-head GEMM + argmax + prefix accept (one launch) */
  VG_KERNEL_ACCEPT = 5,    /* kept for numbering: the accept now runs inside the
                              LM-head launch, so nothing records this kind */
  VG_KERNEL_ATTENTION = 6, /* verifier attention: the chunk partials (scores,
                              softmax, values) of vg_attn_verify */
  VG_KERNEL_KINDS = 7
} vg_kernel;

/* Same object as cudaEvent_t. */
typedef struct CUevent_st* vg_event_t;

/* Timing hook (process-wide, for profiling; no pages' counterpart): while set,
 * the i-th launch of kernel `kind` counted from this call is bracketed by
 * cudaEventRecord(starts[i % n]) before it and cudaEventRecord(stops[i % n])
 * after it, on the stream it is launched on. The events are the caller's
 * (created with timing enabled) and must outlive the hook. n == 0 clears it.
 * The arrays are copied; the pointers need not stay valid. */
vg_status vg_profile_set_events(int32_t kind, const vg_event_t* starts, const vg_event_t* stops, int32_t n);

/* Launches of `kind` recorded since its hook was last set (-1 for a bad kind). */
int64_t vg_profile_count(int32_t kind);

/* Synchronises `stream`, then returns and clears the current device's status
 * word: VG_OK if no kernel recorded a fault, else the first recorded code;
 * *info (if non-NULL) receives a site code of where it happened. */
vg_status vg_get_device_status(vg_stream_t stream, int32_t* info);

/* Limit, in nanoseconds, for every bounded wait inside the library's kernels on
 * the current device (default 4 s). Takes effect for launches after the call. */
vg_status vg_set_wait_timeout_ns(uint64_t ns);

/* Diagnostic: one thread polls (bounded by max_ns of %globaltimer) until
 * *flag == expect. A wait that runs out records VG_ERR_TIMEOUT with site 901 in
 * the status word and returns; the context stays usable. flag is an int32
 * device pointer. */
vg_status vg_debug_wait_flag(const int32_t* flag, int32_t expect, uint64_t max_ns,
                             vg_stream_t stream);

/* Diagnostic of the two bounded waits inside the library's kernels, made to run
 * out on purpose with no copy or tensor-core work in flight, through the same
 * device functions the kernels call:
 *   VG_WAIT_MBARRIER: one thread waits for a shared-memory mbarrier phase that
 *     nothing completes (the wait of every TMA / MMA pipeline stage); site 903;
 *   VG_WAIT_GRID_BARRIER: a cooperative launch of 2 CTAs waits at the grid
 *     barrier of the layer-entry kernel for 3 arrivals, which never come;
 *     ctr is a uint32 device word that must be 0 before the call; site 902.
 * After max_ns (1 .. 60e9) the wait records VG_ERR_TIMEOUT with its site and
 * the kernel returns; the context stays usable. Errors: VG_ERR_INVALID_ARG,
 * VG_ERR_CUDA. */
#define VG_WAIT_MBARRIER 1
#define VG_WAIT_GRID_BARRIER 2
vg_status vg_debug_wait_site(int32_t which, uint32_t* ctr, uint64_t max_ns, vg_stream_t stream);

/* Allocation-free variant of vg_verify_greedy. The pages have no counterpart:
 * it exists for callers that cannot allocate device memory themselves — a
 * plugin whose device memory belongs to its host application's pool allocator,
 * or a latency-critical loop that must not call cudaMalloc because it
 * synchronises the whole device — and so cannot provide a workspace.
 * Same computation, arguments and results as vg_verify_greedy, without the
 * workspace: the running argmax keys (8 bytes per verify row) and the kernel's
 * counter of finished CTAs go to a scratch array compiled into the library
 * (VG_NOALLOC_SCRATCH_BYTES = 2 MiB of device memory that every GPU which
 * loads the library holds until the process exits). Limit: B * (K+1) <=
 * VG_NOALLOC_SCRATCH_BYTES / 8 - 1 = 262,143 verify rows; larger calls return
 * VG_ERR_WORKSPACE and launch nothing. No call allocates or frees memory.
 * The first call on each device looks up the scratch array's device address
 * (with that device current) and caches it; make that first call before any
 * stream capture. Every call uses the same array: it is zero when the library
 * is loaded and every call leaves the part it used zero again, so nothing
 * needs clearing between calls; but calls whose work overlaps on the GPU
 * (different streams, or several threads) race on the array and must be
 * serialised by the caller. */
#define VG_NOALLOC_SCRATCH_BYTES (2u << 20)
vg_status vg_verify_greedy_noalloc(int32_t B, int32_t K, int32_t H, int32_t V,
                                   const void* h, const void* lm_head, const int32_t* drafts,
                                   int32_t* argmax, int32_t* accepted, int32_t* out_tokens,
                                   vg_stream_t stream);

/* ---------------------------------------------------------------------------
 * Multi-step speculative decoding on a synthetic Markov decoder (device-side
 * bookkeeping between verify steps). The pages verify K drafted tokens per
 * step and commit the longest prefix on which draft and verifier agree plus
 * the verifier's own token, so the committed text equals plain greedy decoding
 * ("jina-ocr-v1: Schnellere Dokumentenanalyse auf kostengünstigen GPUs",
 * "Modell und Training"; "Jina AI's 3.4B OCR model targets faster page
 * parsing", "FastMTP cuts decoding work"). These calls let a loop of
 *   vg_spec_rows -> vg_embed_rows -> vg_moe_ffn_stack -> vg_verify_greedy ->
 *   vg_spec_commit
 * run step after step on the device (and be captured in one CUDA graph), for a
 * decoder whose next token is argmax(LM head(MoE stack(emb[last token]))). The
 * draft source is synthetic: the decoder's own token from a reference
 * continuation with probability p, else a uniform token (the pages' drafter is
 * a trained block that is not on this path). K = 0 is plain greedy decoding.
 * ------------------------------------------------------------------------- */

/* out[i, :] = emb[tokens[i], :] for i < n. tokens int32 [n]; emb bf16 [V, H];
 * out bf16 [n, H]; H a multiple of 8, 16-byte aligned rows. A token outside
 * [0, V) gives a zero row and records VG_ERR_DEVICE_BOUNDS in the status word.
 * Errors: VG_ERR_INVALID_ARG, VG_ERR_CUDA. */
vg_status vg_embed_rows(const int32_t* tokens, int32_t n, const void* emb, int32_t V, int32_t H, void* out,
                        vg_stream_t stream);

/* State of B sequences being decoded, all in device memory and owned by the
 * caller. last[b] starts as the prompt's last token, pos[b] as 0, *step as 0.
 * committed [B, cap] receives the committed tokens (positions >= cap are
 * counted in pos but not stored). ref [B, ref_len]: the reference continuation
 * (ref[b, j] = the token greedy decoding commits at position j), read only by
 * the draft source. Random draws: SplitMix64 on a counter of (seed, step, b,
 * draft index). */
typedef struct vg_spec_state {
  int32_t B, K, V;
  int32_t* last;        /* [B] */
  int32_t* pos;         /* [B] */
  int32_t* committed;   /* [B, cap] */
  int32_t cap;
  const int32_t* ref;   /* [B, ref_len] or NULL with ref_len = 0 (uniform drafts only) */
  int32_t ref_len;
  float p;              /* probability that a draft is the reference token, in [0, 1] */
  uint64_t seed;
  int32_t* step;        /* [1] steps taken, advanced by vg_spec_commit */
  int32_t* tokens;      /* [B, K+1] the next verify rows: last token, then the drafts */
  int32_t* drafts;      /* [B, K] the drafts alone (the verify call's input) */
} vg_spec_state;

/* Writes the next verify rows (tokens) and drafts of every sequence: draft i
 * (1..K) is ref[b, pos[b] + i - 1] with probability p (if that position is
 * below ref_len), else a uniform token in [0, V). Errors: VG_ERR_INVALID_ARG,
 * VG_ERR_CUDA. */
vg_status vg_spec_rows(const vg_spec_state* st, vg_stream_t stream);

/* After vg_verify_greedy on those rows: appends out_tokens[b, 0..accepted[b]]
 * to committed at pos[b], advances pos[b] by accepted[b] + 1, sets last[b] to
 * the bonus token and advances *step. accepted int32 [B] in [0, K] (others
 * record VG_ERR_DEVICE_BOUNDS and count as 0); out_tokens int32 [B, K+1].
 * Errors: VG_ERR_INVALID_ARG, VG_ERR_CUDA. */
vg_status vg_spec_commit(const vg_spec_state* st, const int32_t* accepted, const int32_t* out_tokens,
                         vg_stream_t stream);

/* Next verify rows from drafts the caller (e.g. vg_mtp_draft) has written to
 * st->drafts: tokens[b] = [last[b], drafts[b, 0..K-1]]; st->ref and st->p are
 * not used. Errors: VG_ERR_INVALID_ARG, VG_ERR_CUDA. */
vg_status vg_spec_rows_given(const vg_spec_state* st, vg_stream_t stream);

/* ---------------------------------------------------------------------------
 * Recursive draft block (FastMTP): one dense block reused for every draft
 * step, fed back its own hidden state and its own last token ("Jina AI's 3.4B
 * OCR model targets faster page parsing", "FastMTP cuts decoding work";
 * "jina-ocr-v1: Schnellere Dokumentenanalyse auf kostengünstigen GPUs",
 * "Modell und Training", "Erste Schritte"). The pages do not describe the
 * block; the reading computed, step i = 1..K from (g, y) = (g_{i-1}, y_{i-1}):
 *   u   = [rmsnorm(g) * gamma_h ; rmsnorm(emb[y]) * gamma_e]   bf16 [2H]
 *   z   = proj u                                              bf16 [H]
 *   g_i = bf16(z + FFN(rmsnorm(z) * gamma_f))                 bf16 [H]
 *   y_i = argmax over v of lm_head[v] . g_i (fp32 decision, lowest index on ties)
 * rmsnorm(x) = x / sqrt(mean(x^2) + 1e-6) in fp32; FFN = SwiGLU with one expert's
 * layout and width (gate [I,H] | up [I,H] | down [H,I], I = 896), its
 * activations rounded to bf16. g_0 is the given hidden row of each sequence
 * (for a verify step: the row whose argmax was the bonus token), y_0 the given
 * token (the bonus token). H = 1280.
 * ------------------------------------------------------------------------- */
typedef struct vg_mtp_weights {
  const void* proj;       /* bf16 [H, 2H] */
  const void* ffn;        /* bf16 [3 * I * H]: gate | up | down */
  const float* gamma_h;   /* fp32 [H] */
  const float* gamma_e;   /* fp32 [H] */
  const float* gamma_f;   /* fp32 [H] */
  const void* emb;        /* bf16 [V, H] token embedding */
  const void* lm_head;    /* bf16 [V, H] (the verifier's) */
  int32_t V;
} vg_mtp_weights;

/* Workspace of vg_mtp_draft for up to B sequences; 0 if B < 0 or V < 1. */
size_t vg_mtp_workspace_bytes(int32_t B, int32_t V);

/* K draft steps for B sequences. h: bf16 rows; the row of sequence b is
 * b * rows_per_seq + (accepted ? accepted[b] : 0) (pass a verify step's hidden
 * states, K+1 and its accepted lengths). y0 int32 [B]. drafts int32 [B, K]
 * receives y_1 .. y_K; hidden_out, if not NULL, bf16 [K, B, H] receives
 * g_1 .. g_K. K = 0 or B = 0 is a no-op. Stream-ordered, capturable.
 * Errors: VG_ERR_INVALID_ARG, VG_ERR_WORKSPACE (null, short or not 16-byte
 * aligned), VG_ERR_CUDA; a token outside
 * [0, V) or an accepted length outside [0, rows_per_seq) records
 * VG_ERR_DEVICE_BOUNDS. */
vg_status vg_mtp_draft(int32_t B, int32_t K, const vg_mtp_weights* w, const void* h, int32_t rows_per_seq,
                       const int32_t* accepted, const int32_t* y0, int32_t* drafts, void* hidden_out,
                       void* workspace, size_t workspace_bytes, vg_stream_t stream);

/* ---------------------------------------------------------------------------
 * Verifier attention over a KV cache (one layer of a verify step). The pages
 * give the decoder's 32,768-position limit (jina-ocr-v1 model card,
 * architecture paragraph) but not its attention; the reading computed:
 *   qkv = x W_qkv^T (W_qkv bf16 [3H, H]: q rows, k rows, v rows), bf16;
 *   10 heads of 128; RoFormer rotary positions on q and k: pair (2j, 2j+1) of a
 *   head at position p turned by p * 10000^(-2j/128); row i of sequence b sits
 *   at position lens[b] + i;
 *   the new rows' k (rotated) and v are written into the cache at positions
 *   lens[b] .. lens[b] + K;
 *   row i attends to positions 0 .. lens[b] + i, scores q.k / sqrt(128), softmax;
 *   out = bf16(x + bf16(W_o o)) (W_o bf16 [H, H]).
 * x, out bf16 [B*(K+1), H] (rows of sequence b at b*(K+1) ..); kv_cache bf16
 * [B, 2, L_max, H] (k then v, a position's heads side by side); lens int32 [B]
 * is read, not advanced (advance it by the committed tokens; a later step
 * overwrites the positions of rejected drafts). K+1 <= 8, L_max <= 32768;
 * lens[b] + K + 1 > L_max records VG_ERR_DEVICE_BOUNDS and gives o = 0 for that
 * sequence. o_out, if not NULL, bf16 [B*(K+1), H] receives the heads' output o
 * before the output projection. All pointers are device memory, the arrays
 * 16-byte aligned; out and o_out must not overlap x or each other, and none of
 * them kv_cache. Precision: both products of a head (q.k and the
 * probability-weighted sum of v) run on the tensor cores with bf16 operands and
 * fp32 accumulation, so the softmax weights enter the second product rounded to
 * bf16 (their sum is taken over the rounded weights); the projections run on
 * the tcgen05 tensor cores as fp32 sums over five 256-wide slices of the
 * reduction, added in slice order. Six launches: q/k/v projection, rotary
 * append, attention over 256-position chunks, the merge of the chunks, output
 * projection, residual. Errors: VG_ERR_INVALID_ARG, VG_ERR_UNSUPPORTED
 * (B*(K+1)*H >= 2^31 or B*2*L_max >= 2^31), VG_ERR_WORKSPACE (null, short or
 * not 16-byte aligned), VG_ERR_CUDA.
 * ------------------------------------------------------------------------- */
size_t vg_attn_workspace_bytes(int32_t B, int32_t K, int32_t L_max);
vg_status vg_attn_verify(int32_t B, int32_t K, int32_t L_max, const void* x, const void* w_qkv, const void* w_o,
                         void* kv_cache, const int32_t* lens, void* out, void* o_out, void* workspace,
                         size_t workspace_bytes, vg_stream_t stream);

/* ---------------------------------------------------------------------------
 * The whole verify step for a handful of rows in ONE kernel launch: the
 * n_layers MoE layers (x_{l+1} = bf16(x_l + MoE_l(x_l)), as vg_moe_ffn_stack),
 * then the LM-head argmax and the prefix accept (as vg_verify_greedy). For
 * T = B * (K+1) <= 16 rows (the batch-1 verify: K = 3 gives 4 rows, K = 1
 * gives 2), where a step is a stream of weights and separate launches cost as
 * much as the stream; the pages measure the speculative step at batch 1 and
 * find launch overhead dominant there ("jina-ocr-v1: Schnellere
 * Dokumentenanalyse auf kostengünstigen GPUs", "Spekulatives Decoding auf
 * einer L4"). One CTA per SM (cooperative launch): every CTA computes the
 * routing of all T rows itself (identical results, no barrier); the expert
 * products are split along K over all SMs, and the pieces of a block are
 * summed in k order by the last one to finish, so results do not depend on
 * timing. The expert outputs differ from vg_moe_ffn_stack's only in the fp32
 * summation order of the expert GEMMs.
 * Arguments as vg_moe_ffn_stack (n_layers <= 12, bf16 pointers 16-byte
 * aligned) and vg_verify_greedy (V >= 128); states_out, if not NULL, bf16
 * [n_layers+1, T, H] receives each layer's input and then the final states;
 * topk_idx_out, if not NULL, int32 [n_layers, T, 6] each layer's routed
 * experts. workspace: vg_verify_step_small_workspace_bytes() bytes, 16-byte
 * aligned, no initial contents (the call clears its control words first).
 * B = 0 is a no-op. Errors: VG_ERR_INVALID_ARG, VG_ERR_UNSUPPORTED (T > 16,
 * n_layers > 12, other dims, V < 128), VG_ERR_WORKSPACE, VG_ERR_CUDA; waits
 * that run out record VG_ERR_TIMEOUT in the device status word.
 * ------------------------------------------------------------------------- */
size_t vg_verify_step_small_workspace_bytes(void);
vg_status vg_verify_step_small(const vg_moe_dims* dims, int32_t n_layers, int32_t B, int32_t K, const void* x,
                               const void* const* router_w, const float* const* router_bias,
                               const void* const* expert_w, const void* const* shared_w, const void* lm_head,
                               int32_t V, const int32_t* drafts, int32_t* argmax, int32_t* accepted,
                               int32_t* out_tokens, void* states_out, int32_t* topk_idx_out, void* workspace,
                               size_t workspace_bytes, vg_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* VGV_H */
