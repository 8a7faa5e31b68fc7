/*
 * isa.h -- C interface of the In-context Sparse Attention (ISA) forward and
 * backward passes for NVIDIA B200 (sm_100a).
 *
 * The method is the sparse attention of "LIVEditor-14B: Lightning Unified
 * Video Editing via In-Context Sparse Attention" (arXiv:2605.04569), as the
 * paper.rainbus.top summary card states it in "Method steps in detail"
 * (steps (1)-(6)) and "Core method", with the 0th-order Taylor term of its
 * "0th-order Taylor approximate attention" section.  The model card
 * (Hugging Face mirror, "Highlights") describes ISA as a drop-in for the
 * attention call of a diffusion transformer on the concatenated
 * [source ; context] token sequence; the entry points below are that call,
 * split into planning and attention.
 *
 * Conventions shared by every entry point
 *  - Q, K, V and O are bfloat16 tensors [B, H, L, D], contiguous, on one
 *    CUDA device, with L = L_src + L_ctx and the context tokens after the
 *    source tokens.  Base addresses must be 16-byte aligned.
 *  - Each call runs on the device that holds its tensors: it looks up the
 *    device of q (of out for isa_coarse_residual, of dq for
 *    isa_coarse_residual_backward) and makes it the calling thread's
 *    current device; the stream must belong to that device.  One process
 *    may so drive several devices, from one host thread or several.
 *  - "device" pointers are CUDA device (or managed) memory; the caller owns
 *    all memory and the stream.  The library allocates no device memory,
 *    launches asynchronously on `stream` (a cudaStream_t, NULL = legacy
 *    default stream) and never synchronises the host.
 *  - Argument errors are returned synchronously before anything is
 *    launched; launch failures are returned from the launching call
 *    (ISA_ERR_CUDA); a device-side wait that exceeded its time limit sets a
 *    device status word (see isa_plan_view.status / isa_dense `status`) that
 *    the caller reads after synchronising.
 *  - isa_last_error() returns a thread-local message for the last failure.
 *
 * Supported shapes: D in {64, 128}; block in {32, 64}; L_src, L_ctx >= 1;
 * B*H*L < 2^31; alpha_s in (0, 1]; alpha_f, alpha_ns in [0, 1].
 */
#ifndef ISA_H_
#define ISA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Problem description.  The three ratios are the pages' hyper-parameters
 * (summary card "Core method"; techwalker.com section 9): alpha_s = share of
 * context blocks kept by the pre-selection, alpha_f = share of query blocks
 * sent to the Taylor ("flat") path, alpha_ns = share of kept KV blocks that a
 * flat block attends exactly.  scale <= 0 selects 1/sqrt(D). */
typedef struct isa_params {
  int32_t B, H, D;
  int32_t L_src, L_ctx;
  int32_t block;
  float alpha_s, alpha_f, alpha_ns;
  float scale;
} isa_params;

typedef enum isa_status {
  ISA_OK = 0,
  ISA_ERR_INVALID_ARG = 1,     /* null pointer, misalignment, out-of-range value   */
  ISA_ERR_UNSUPPORTED = 2,     /* valid problem outside the supported shapes        */
  ISA_ERR_WORKSPACE = 3,       /* plan workspace too small                          */
  ISA_ERR_CUDA = 4,            /* a CUDA runtime/driver call or launch failed       */
  ISA_ERR_DEVICE_TIMEOUT = 5   /* value written to a device status word, see above  */
} isa_status;

/* Sizes of the plan and device pointers into a plan workspace.  All arrays
 * are per head, heads ordered bh = b*H + h.  Block ids run over the T =
 * T_src + T_ctx blocks: source blocks 0..T_src-1 cover tokens [j*b, ...),
 * context blocks T_src..T-1 cover tokens [L_src + c*b, ...); only each
 * segment's last block may be partial. */
typedef struct isa_plan_view {
  int32_t T_src, T_ctx, T;     /* blocks per segment / in total                     */
  int32_t K_sel;               /* kept context blocks = clamp(ceil(alpha_s*T_ctx),1,T_ctx) */
  int32_t T_kv;                /* kept KV blocks = T_src + K_sel                    */
  int32_t n_flat, n_sharp;     /* n_flat = floor(alpha_f*T), n_sharp = T - n_flat   */
  int32_t n_exact;             /* exact blocks per flat block = ceil(alpha_ns*T_kv) */
  int32_t T_kv_pad;            /* rows of Kp/Vp per head (T_kv rounded up to 128)   */
  int32_t bitmap_words;        /* 32-bit words per exact bitmap = ceil(T_kv/32)     */
  const float* Qc;             /* [BH, T, D] fp32 pooled means (step (1))           */
  const float* Kc;             /* [BH, T, D]                                        */
  const float* Vc;             /* [BH, T, D]                                        */
  const float* imp;            /* [BH, T_ctx] context importance (step (2))         */
  const int32_t* ctx_sel;      /* [BH, K_sel] selected context blocks, ascending    */
  const int32_t* kept;         /* [BH, T_kv] kept block ids, ascending              */
  const float* energy;         /* [BH, T] E_i = sum_j softmax(S_i)_j^2 (step (3)); the
                                  sharpness variance is E_i/T - 1/T^2              */
  const int32_t* sharp_ids;    /* [BH, n_sharp] ascending block ids                 */
  const int32_t* flat_ids;     /* [BH, n_flat] ascending block ids                  */
  const int32_t* exact;        /* [BH, n_flat, n_exact] positions in `kept`, ascending */
  const uint32_t* exact_bits;  /* [BH, n_flat, bitmap_words] same set as a bitmap   */
  const uint16_t* Kp;          /* [BH, T_kv_pad, D] bf16 pooled K of kept blocks    */
  const uint16_t* Vp;          /* [BH, T_kv_pad, D] bf16 pooled V of kept blocks    */
  const int32_t* status;       /* device status word: ISA_OK or ISA_ERR_DEVICE_TIMEOUT */
} isa_plan_view;

/* Bytes of device workspace isa_plan needs for `p`.  Host only; launches
 * nothing.  Returns ISA_ERR_INVALID_ARG / ISA_ERR_UNSUPPORTED for bad `p`. */
isa_status isa_plan_workspace_size(const isa_params* p, size_t* bytes);

/* Planning: steps (1)-(3) of "Method steps in detail" and the exact-block
 * choice of step (5).  Pools Q/K/V into blocks (fp32 means of the valid
 * tokens), computes the coarse scores S = Qc Kc^T * scale, keeps the K_sel
 * context blocks with the largest sum of S over source query rows (ties to
 * the lower block), ranks query blocks by E_i (descending; ties: lower block
 * is sharper) into n_sharp sharp and n_flat flat blocks, and gives each flat
 * block the n_exact kept blocks with the largest S (ties to the lower block).
 *   q, k, v : device, bf16 [B,H,L,D]
 *   ws      : device, at least isa_plan_workspace_size bytes, 256-byte
 *             aligned; overwritten; holds the plan afterwards
 * Launches 6 kernels on `stream` (5 when no block is flat). */
isa_status isa_plan(const isa_params* p, const void* q, const void* k, const void* v,
                    void* ws, size_t ws_bytes, void* stream);

/* isa_rope followed by isa_plan in one pass over Q and K: the decoupled
 * RoPE of the techwalker.com article ("Decoupled RoPE": the reference
 * video's positions restart at 0) and the summary card (innovation (d)),
 * with the rotation, positions and rounding of isa_rope below, folded into
 * the pooling of step (1).  The pooling kernel rotates each Q and K row as
 * it reads it, writes the rotated bf16 row to q_rot / k_rot, and pools from
 * those values; the results (q_rot, k_rot and the plan in ws) are bit for bit
 * those of isa_rope then isa_plan, with Q and K read once instead of twice.
 *   q, k, v      : device bf16 [B,H,L,D] (before the rotation)
 *   q_rot, k_rot : device bf16 [B,H,L,D], every element written; may equal
 *                  q, k (in place).  Give them, with v, to isa_forward.
 *   base         : > 1 (10000 is the usual value)
 *   ws           : the plan workspace, as for isa_plan
 *   rope_ws      : device, >= isa_rope_workspace_size bytes, 16-byte aligned;
 *                  caller-owned scratch for the (cos, sin) table
 * Launches 7 kernels on `stream` (6 when no block is flat). */
isa_status isa_plan_rope(const isa_params* p, float base, const void* q, const void* k, const void* v, void* q_rot,
                         void* k_rot, void* ws, size_t ws_bytes, void* rope_ws, size_t rope_ws_bytes, void* stream);

/* Fills `view` with the sizes of the plan for `p` and device pointers into
 * `ws` (no launch, no copy; contents valid once isa_plan has run). */
isa_status isa_plan_view_get(const isa_params* p, const void* ws, size_t ws_bytes,
                             isa_plan_view* view);

/* Sparse attention: steps (4)-(6) of "Method steps in detail".  Sharp query
 * blocks attend exactly to every token of the kept KV blocks; flat query
 * blocks attend exactly to the tokens of their n_exact blocks and, for every
 * other kept block j, to one pooled key Kc_j with value Vc_j and weight n_j
 * (logit scale*q.Kc_j + ln n_j); one online-softmax state per query row
 * merges both parts.  Outputs go straight to token order.
 *   q, k, v : device, bf16 [B,H,L,D] (the tensors given to isa_plan)
 *   ws      : device, a workspace isa_plan filled for the same p, q, k, v
 *   out     : device, bf16 [B,H,L,D]; every row is written
 *   lse     : device fp32 [B,H,L] natural-log softmax normaliser per row, or NULL
 * One persistent launch (tcgen05/TMEM/TMA). */
isa_status isa_forward(const isa_params* p, const void* q, const void* k, const void* v,
                       const void* ws, size_t ws_bytes, void* out, float* lse, void* stream);

/* Dense reference attention: softmax(scale * Q K^T) V over all L tokens per
 * head (the full attention that ISA replaces, summary card "Background" /
 * FlashAttention baselines), with the same kernel machinery.
 *   out    : device bf16 [B,H,L,D];  lse: device fp32 [B,H,L] or NULL
 *   status : device int32 status word (set to ISA_OK by the call, raised to
 *            ISA_ERR_DEVICE_TIMEOUT by a timed-out wait), or NULL */
isa_status isa_dense(const isa_params* p, const void* q, const void* k, const void* v,
                     void* out, float* lse, int32_t* status, void* stream);

/* isa_plan + isa_forward for callers that cannot allocate device memory.
 * The pages describe nothing like it (the paper has no counterpart): it
 * serves callers that cannot hand the library a workspace -- code that must
 * not call cudaMalloc (inside an allocator or memory-pool callback, a
 * real-time loop that forbids allocation) or a binding without a device
 * allocator.  The plan lives in a fixed 16 MiB device array inside the
 * library; every GPU that loads the library holds it until the process
 * exits.  Inputs, output and lse are as for isa_forward.
 *  - A problem whose plan needs more than 16 MiB (isa_plan_workspace_size)
 *    returns ISA_ERR_WORKSPACE with a message; nothing is launched.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress), which may make the driver load the library's
 *    device code and the array with it: make that first call, per device,
 *    as a warm-up where allocation is allowed, and before any stream capture.
 *    Later calls allocate nothing (no cudaMalloc/cudaFree, no library
 *    allocation).
 *  - The looked-up address is cached per device; after cudaDeviceReset it is
 *    stale, so do not call this entry point on that device again.
 *  - All calls share the one array, which keeps the last call's contents;
 *    every plan entry is rewritten and the status word cleared by each call.
 *    Calls that overlap on the GPU race on the array: order them.
 * Device timeouts are written to the array's status word; read it with
 * isa_forward_static_status. */
isa_status isa_forward_static(const isa_params* p, const void* q, const void* k, const void* v, void* out,
                              float* lse, void* stream);

/* Copies the status word of isa_forward_static's array on CUDA device
 * `device` (ISA_OK, or ISA_ERR_DEVICE_TIMEOUT after a device wait ran out)
 * to `dst` (4 bytes of host or device memory) with one stream-ordered copy
 * on `stream`: the value is there once the stream has reached the copy (for
 * pageable host memory, when the call returns).  Like the entry point it
 * serves, it has no counterpart on the pages.  Returns ISA_ERR_INVALID_ARG
 * when dst is NULL or isa_forward_static has not run on that device. */
isa_status isa_forward_static_status(int32_t device, int32_t* dst, void* stream);

/* Workspace of isa_backward: (lse * log2 e, rowsum(dout * out)) for every
 * row of every block, padded to `block` rows per block (B*H * T * block * 8
 * bytes), and fp32 gradients of the pooled keys and values
 * (2 * B*H * T_kv_pad * D * 4 bytes), each 256-byte aligned. */
isa_status isa_backward_workspace_size(const isa_params* p, size_t* bytes);

/* Gradients of the isa_forward output with respect to Q, K and V, for the
 * loss sum(dout * out), with the plan in `ws` held fixed.  The summary card
 * ("Core method", innovation (c)) and the techwalker.com article (training
 * section) state that ISA has a forward and a backward implementation and is
 * trained end to end; they print no gradient formulas.  These are the
 * gradients of the forward as computed: the plan's choices (kept context
 * blocks, sharp/flat split, exact lists) carry no gradient, a flat block's
 * pooled key Kc_j / value Vc_j (the mean of block j's n_j tokens) passes its
 * gradient to each token of block j divided by n_j, and the count weight n_j
 * is a constant.  With P the softmax weights of a query row over its columns,
 * dP = dout V^T and Delta = rowsum(dout * out):
 *   dS = P (dP - Delta),  dq = s dS K,  dk = s dS^T Q,  dv = P^T dout.
 *   q, k, v, ws : the inputs and the plan of the forward call
 *   out         : device bf16 [B,H,L,D], the forward's output
 *   lse         : device fp32 [B,H,L], the forward's lse (isa_forward with lse != NULL)
 *   dout        : device bf16 [B,H,L,D]
 *   dq, dk, dv  : device bf16 [B,H,L,D]; every element is written (tokens of
 *                 context blocks that were not kept get dk = dv = 0)
 *   bws         : device, >= isa_backward_workspace_size bytes, 256-byte
 *                 aligned; caller-owned scratch, rewritten by every call
 * P is recomputed from lse (no attention matrix is stored); products run in
 * bf16 on the tensor cores with fp32 accumulation, P and dS rounded to bf16.
 * Launches 5 kernels: one fewer when no flat block has a pooled column
 * (every kept block exact, or no block flat), and one fewer when every
 * context block is kept (no unkept tokens to zero).
 * Device timeouts go to the plan's status word, as for isa_forward. */
isa_status isa_backward(const isa_params* p, const void* q, const void* k, const void* v, const void* ws,
                        size_t ws_bytes, const void* out, const float* lse, const void* dout, void* dq, void* dk,
                        void* dv, void* bws, size_t bws_bytes, void* stream);

/* Step (6) of "Method steps in detail" adds gamma * O_coarse to the
 * scattered output as a low-frequency residual; the summary card defines
 * neither.  Reading: O_coarse is the block-level pooling attention of its
 * "Block-sparse attention and pooling attention" background on the plan's
 * pooled means, O_coarse_i = sum_j softmax_j(scale * Qc_i . Kc_j) Vc_j over
 * all T blocks, and every token of query block i receives gamma * O_coarse_i.
 *   ws    : a workspace isa_plan filled (its Qc, Kc, Vc are used)
 *   out   : device bf16 [B,H,L,D]; out += gamma * O_coarse in place (fp32
 *           arithmetic, one rounding to bf16)
 *   gamma : finite
 * Apply it to a copy of isa_forward's output: isa_backward needs the sparse
 * output itself.  One launch (CUDA cores: T x T x D per head). */
isa_status isa_coarse_residual(const isa_params* p, float gamma, const void* ws, size_t ws_bytes, void* out,
                               void* stream);

/* Workspace of isa_coarse_residual_backward: per-block statistics and the
 * scaled block sums of dout (B*H * T * (8 + 4*D) bytes, 256-byte aligned). */
isa_status isa_coarse_residual_backward_workspace_size(const isa_params* p, size_t* bytes);

/* Gradients of sum(dout * gamma * O_coarse) (see isa_coarse_residual),
 * ADDED in place to dq, dk, dv (device bf16 [B,H,L,D], e.g. isa_backward's
 * results), through the pooled means: a block's gradient reaches each of
 * its n_j tokens divided by n_j.  dgamma: device fp32 [B*H] receiving
 * sum(dout * O_coarse) per head (zeroed by the call), or NULL.  cws:
 * caller-owned scratch of isa_coarse_residual_backward_workspace_size bytes,
 * 256-byte aligned.  Two launches. */
isa_status isa_coarse_residual_backward(const isa_params* p, float gamma, const void* ws, size_t ws_bytes,
                                        const void* dout, void* dq, void* dk, void* dv, float* dgamma, void* cws,
                                        size_t cws_bytes, void* stream);

/* Workspace of isa_rope: the cos/sin table, max(L_src, L_ctx) * D/2 float
 * pairs (8 bytes each). */
isa_status isa_rope_workspace_size(const isa_params* p, size_t* bytes);

/* Decoupled rotary position embedding of Q and K, applied before isa_plan
 * (techwalker.com article, "Decoupled RoPE": the reference video's position
 * indices restart at 0 rather than continuing after the source video;
 * summary card, innovation (d): source and context each encode positions
 * from 0).  Token l has position l in the source segment [0, L_src) and
 * l - L_src in the context segment.  The pages name no frequencies or
 * pairing; this is one-dimensional RoPE over the token index with
 * theta_i = base^(-2i/D), pair i = components (2i, 2i+1) rotated
 * counter-clockwise by position * theta_i.
 *   q, k         : device bf16 [B,H,L,D]
 *   q_out, k_out : device bf16 [B,H,L,D]; may equal q, k (in place)
 *   base         : > 1 (10000 is the usual value)
 *   ws           : device, >= isa_rope_workspace_size bytes, 16-byte aligned;
 *                  caller-owned, rewritten by every call
 * Angles and the table are computed in double precision, the rotation in
 * fp32 from bf16 inputs, rounded once to bf16 (round to nearest even).
 * Stream-ordered; argument errors return before any launch. */
isa_status isa_rope(const isa_params* p, float base, const void* q, const void* k, void* q_out, void* k_out,
                    void* ws, size_t ws_bytes, void* stream);

/* Thread-local description of the last error (never NULL). */
const char* isa_last_error(void);

/* Library version string, e.g. "isa-b200 0.1 sm_100a". */
const char* isa_version(void);

/* Time limit of every device-side wait of later launches, in nanoseconds
 * (default 2e9).  A wait that runs out writes ISA_ERR_DEVICE_TIMEOUT to the
 * status word, stops its CTA's work, drains the CTA's copies in flight and
 * returns.  0 restores the default. */
isa_status isa_set_wait_timeout_ns(uint64_t ns);

/* Host-chosen fault injection for tests of the timeout path: mode 1 makes
 * the attention kernels (forward and backward) wait on a barrier that
 * nothing arrives on, so the wait runs out; 0 turns it off.  Applies to
 * later launches. */
isa_status isa_set_fault_injection(int32_t mode);

#ifdef __cplusplus
}
#endif
#endif /* ISA_H_ */
