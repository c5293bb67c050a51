/*
 * xlpk.h - persistent single-kernel small-batch decode on one B200 (sm_100a).
 *
 * The whole greedy decode of N tokens runs as ONE cooperative kernel launch:
 * every SM holds one resident CTA that walks a statically planned list of
 * tile tasks (RMSNorm-folded QKV GEMV + RoPE + KV append, flash-decoding
 * attention split over the sequence, O-projection + residual, gate/up +
 * SwiGLU, down projection + residual, LM head + argmax) and orders them with
 * device-side dependency counters instead of kernel launches.  This follows
 * the "persistent Engine Kernel" and "tile-level pipeline" design described in
 * "TileRT speed notes" (section "TileRT's direction: from discrete kernels to
 * a resident execution pipeline") and in "Ultra-High Interactivity On NVIDIA
 * GPUs? - TileRT InferenceX" (digest, "core views": the host launches once and
 * the execution stays resident for the whole decode lifecycle).  The
 * kernel-per-op baseline the pages compare against (launch, load, compute,
 * store, synchronise per operator; "Persistent execution paradigm", section 1)
 * is xlpk_decode_unfused, built from the same tiles.  The batch-8 decode runs
 * its projections on the tcgen05 tensor cores (xlpk_tc_gemm_tile is the same
 * contraction as a stand-alone call).
 *
 * Conventions for every entry point:
 *  - Pointers named *_dev are CUDA device pointers on the handle's device;
 *    pointers named *_host are ordinary host memory.  Nothing is retained
 *    past the call except where stated (weights/KV in xlpk_create).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *  - Functions return XLPK_OK or a negative xlpk_status.  Argument errors are
 *    detected on the host before anything is enqueued.  Device-side failures
 *    of an enqueued decode (a dependency wait that exceeded its time limit)
 *    are reported by xlpk_get_status after the work has finished.
 *  - A handle is not thread-safe: calls on one handle must be serialised,
 *    and its decodes must not overlap on the GPU.
 *  - There is no CPU fallback: without a usable sm_100 device, xlpk_create
 *    returns XLPK_ERR_UNSUPPORTED or XLPK_ERR_CUDA.
 */
#ifndef XLPK_H_
#define XLPK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum xlpk_status {
  XLPK_OK = 0,
  XLPK_ERR_INVALID_ARG = -1,   /* bad pointer, size, shape or alignment */
  XLPK_ERR_UNSUPPORTED = -2,   /* shape/dtype/batch this build does not handle, or no sm_100 GPU */
  XLPK_ERR_CUDA = -3,          /* a CUDA runtime call failed (see xlpk_last_cuda_error) */
  XLPK_ERR_OOM = -4,           /* device allocation failed */
  XLPK_ERR_KV_FULL = -5,       /* n_steps would write past max_seq */
  XLPK_ERR_TIMEOUT = -6,       /* a device-side dependency wait exceeded its limit */
  XLPK_ERR_ABORTED = -7        /* the decode was abandoned after another CTA failed */
} xlpk_status;

typedef enum xlpk_dtype {
  XLPK_DTYPE_BF16 = 0,         /* bf16 weights, row-major [N][K] */
  XLPK_DTYPE_FP8_E4M3 = 1,     /* e4m3 codes, row-major [N][K], + one fp32 scale per 128x128 block;
                                  dense models only, hidden / n_q_heads*head_dim / ffn multiples
                                  of 256 and the other dims of 128 (else XLPK_ERR_UNSUPPORTED) */
  XLPK_DTYPE_NVFP4 = 2         /* weights only: e2m1 codes [N][K/2] (element 2j in the low nibble of
                                  byte j), one e4m3 scale per 16 consecutive elements of a row and one
                                  fp32 scale per matrix (xlpk_linear); dense models at batch 1, hidden /
                                  n_q_heads*head_dim / ffn multiples of 128 (else XLPK_ERR_UNSUPPORTED) */
} xlpk_dtype;

/* Model and launch shape.  All widths are element counts.
 * Dense models set n_experts = top_k = n_shared_experts = expert_ffn = 0. */
typedef struct xlpk_config {
  int32_t n_layers;
  int32_t hidden;              /* H */
  int32_t n_q_heads;           /* n_q */
  int32_t n_kv_heads;          /* n_kv; n_q % n_kv == 0; query head h reads kv head h / (n_q / n_kv) */
  int32_t head_dim;            /* d: 64 or 128 */
  int32_t ffn;                 /* F, dense SwiGLU width */
  int32_t vocab;               /* V */
  int32_t n_experts;           /* E (MoE), else 0 */
  int32_t top_k;               /* experts per token (MoE), else 0 */
  int32_t n_shared_experts;    /* always-on experts (MoE), else 0 */
  int32_t expert_ffn;          /* SwiGLU width of one expert (MoE), else 0 */
  int32_t weight_dtype;        /* xlpk_dtype of every linear weight (embedding and router stay bf16) */
  int32_t batch;               /* B sequences decoded together, 1..8 */
  int32_t max_seq;             /* KV cache capacity per sequence (positions) */
  float rope_theta;            /* RoPE base: pair (i, i + d/2) turns by pos * theta^(-2i/d) */
  float rms_eps;               /* RMSNorm epsilon */
  int32_t n_ctas;              /* persistent grid size; 0 = one CTA per SM */
  int32_t spin_limit_us;       /* limit of every device-side wait; 0 = 200000 us */
  int32_t flags;               /* XLPK_FLAG_* bits; 0 = the planner's defaults */
  int32_t window;              /* K window (columns) of the windowed projections: the down projection at
                                  batch >= 2 on CUDA cores (a multiple of its k-chunk) or every
                                  tensor-core projection at batch 8 (a multiple of 1024); 0 = chosen by
                                  the planner.  A value the planner cannot use is ignored on CUDA cores
                                  and refused (XLPK_ERR_UNSUPPORTED) on tensor cores. */
  int32_t kv_dtype;            /* xlpk_dtype of the KV cache: XLPK_DTYPE_BF16 (entries are bf16) or
                                  XLPK_DTYPE_FP8_E4M3 (entries are e4m3 codes; entry = code * scale) */
  float k_scale;               /* e4m3 cache: the scale of every K entry, a power of two in
                                  [2^-24, 2^24] (else XLPK_ERR_INVALID_ARG); ignored for bf16 */
  float v_scale;               /* e4m3 cache: the scale of every V entry, the same rule */
} xlpk_config;

/* xlpk_config::flags.  The defaults are the fast paths; the flags select the
 * alternatives they replace (both compute the same decode). */
enum {
  XLPK_FLAG_NO_FUSED_FFN = 1,      /* bf16 dense layers at batch <= 2: gate/up and down as two stages
                                      instead of one fused stage with a split-K down projection */
  XLPK_FLAG_NO_TENSOR_CORES = 2,   /* batch 8: CUDA-core GEMV tiles instead of tcgen05 MMAs */
  XLPK_FLAG_FLOAT_FFN_REDUCE = 4   /* fused FFN: add the down projection's split-K partial sums into an
                                      fp32 residual with float atomics instead of a 64-bit fixed-point
                                      accumulator with integer atomics; fewer atomic operations, but
                                      the rounding then depends on arrival order, so runs are not
                                      bit-identical */
};

/* One linear weight: y = W x with W row-major [N][K] (PyTorch Linear layout).
 * `scale_dev` is NULL for bf16; for FP8 it is fp32 [N/128][K/128], row-major;
 * for NVFP4 the e4m3 block scales, uint8 [N][K/16], and `global_scale` the
 * matrix's fp32 scale (finite, > 0): element = e2m1 code * block scale *
 * global_scale.  `global_scale` is ignored for the other types.
 * Source: the NVFP4 bytes-per-token roofline ("Ultra-High Interactivity On
 * NVIDIA GPUs? - TileRT InferenceX", digest, core views). */
typedef struct xlpk_linear {
  const void* w_dev;
  const void* scale_dev;
  float global_scale;
} xlpk_linear;

typedef struct xlpk_layer_weights {
  const float* attn_norm_dev;  /* fp32 [H] RMSNorm gain before attention */
  xlpk_linear wq;              /* [n_q*d][H] */
  xlpk_linear wk;              /* [n_kv*d][H] */
  xlpk_linear wv;              /* [n_kv*d][H] */
  xlpk_linear wo;              /* [H][n_q*d] */
  const float* ffn_norm_dev;   /* fp32 [H] RMSNorm gain before the FFN */
  xlpk_linear w_gate;          /* dense: [F][H] */
  xlpk_linear w_up;            /* dense: [F][H] */
  xlpk_linear w_down;          /* dense: [H][F] */
  const void* router_dev;      /* MoE: bf16 [E][H] */
  xlpk_linear we_gate;         /* MoE: [E][Fe][H], scale [E][Fe/128][H/128] */
  xlpk_linear we_up;           /* MoE: [E][Fe][H] */
  xlpk_linear we_down;         /* MoE: [E][H][Fe] */
  xlpk_linear ws_gate;         /* MoE shared experts: [S][Fe][H] */
  xlpk_linear ws_up;           /* MoE shared experts: [S][Fe][H] */
  xlpk_linear ws_down;         /* MoE shared experts: [S][H][Fe] */
} xlpk_layer_weights;

typedef struct xlpk_weights {
  const void* embed_dev;              /* bf16 [V][H] token embedding */
  const float* final_norm_dev;        /* fp32 [H] */
  xlpk_linear lm_head;                /* [V][H] */
  const xlpk_layer_weights* layers;   /* HOST array of n_layers entries */
} xlpk_weights;

/* Caller-owned KV cache: post-RoPE keys and values, 16-byte aligned, one
 * element per entry of the config's kv_dtype: bf16, or an e4m3 code (one byte)
 * whose value is code * k_scale (K) or code * v_scale (V).  A decode writes the
 * new token's entries rounded to that type (e4m3: x / scale rounded to nearest
 * even and saturated to +-448).
 *  - Contiguous (page_table_dev NULL): K and V each [L][B][n_kv][max_seq][d].
 *  - Paged: K and V each a pool [L][n_pages][n_kv][page_size][d] of pages of
 *    page_size positions; page_table_dev int32 [B][ceil(max_seq / page_size)]
 *    names the pool page that holds positions [j*page_size, (j+1)*page_size)
 *    of sequence b.  page_size must be the attention chunk (64 positions for
 *    head_dim 128, 128 for head_dim 64; else XLPK_ERR_UNSUPPORTED), so every
 *    attention task reads exactly one page.  Sequences may share pages (a
 *    common prefix).  The table is read by every decode; the caller may change
 *    it between calls (stream order).  An entry outside [0, n_pages) that a
 *    decode reaches is not followed: the decode stops with XLPK_ERR_INVALID_ARG
 *    from xlpk_get_status.
 * Source: the KV page planner that places each request's cache pages and the
 * decode worker that follows them ("XL-Persistent-Kernel", request lifecycle
 * steps 2-4 and the component table's KV row); a quantised (FP8) attention
 * cache read inside the persistent kernel, which the page on the persistent
 * execution paradigm names as an open combination ("持续执行范式：从 Kernel
 * Boundary Elimination 到 Ultra-Low-Latency Engine", section 7.5). */
typedef struct xlpk_kv {
  void* k_dev;
  void* v_dev;
  const int32_t* page_table_dev;   /* NULL: contiguous cache */
  int32_t page_size;               /* paged: positions per page */
  int32_t n_pages;                 /* paged: pages in each pool */
} xlpk_kv;

/* Optional per-step outputs and teacher forcing of one decode call.
 * Every pointer may be NULL. */
typedef struct xlpk_decode_io {
  const int32_t* forced_tokens_dev;   /* [n_steps][B]: next input is forced[s][b] instead of the argmax */
  float* logits_dev;                  /* [n_steps][B][V] fp32 logits of every step */
  float* hidden_dev;                  /* [n_steps][B][H] fp32 residual after the last layer */
  int32_t* experts_dev;               /* MoE: [n_steps][L][B][top_k] selected expert ids */
  uint64_t* trace_dev;                /* [n_steps][n_stages][n_ctas][16] globaltimer stamps (ns) per
                                         stage and CTA: [0] consumer entry, [1] dependency met,
                                         [2] inputs staged, [3] consumer done, [4] producer first
                                         copy, [5] producer last copy.  A library built with
                                         XLPK_TRACE_ATTN defined also records, for attention
                                         stages, totals of thread 0: [6] ns waiting for KV chunks,
                                         [7] ns of the combining CTA's wait for the partials,
                                         [8] q loads, [9] chunk math, [10] merge,
                                         [11] arrive, [12] combine, [13] the combining CTA's time to
                                         its merged output (wait + arithmetic); for the
                                         other stages, thread 0's input staging: [6] copies issued,
                                         [7] landed, [8] converted, [9] RMSNorm factor ready.
                                         n_stages = 5 * n_layers + 1 */
  int32_t withhold_release;           /* failure-detection testing only: 1 + the index (layer * 5 +
                                         stage kind, n_layers * 5 = LM head) of a stage whose
                                         completion CTA 0 does not announce at the call's first
                                         step, so the waits behind it run out; 0 = off */
} xlpk_decode_io;

/* Facts about a created handle (for measurement and tests). */
typedef struct xlpk_info {
  int32_t n_ctas;               /* persistent grid size */
  int32_t threads_per_cta;
  int32_t smem_bytes;           /* dynamic shared memory per CTA */
  int32_t ring_slots;           /* weight/KV staging slots per CTA */
  int32_t slot_bytes;
  int32_t kernels_per_step_unfused;
  int64_t packed_weight_bytes;  /* library-owned packed copy of the weights */
  int64_t workspace_bytes;
  int64_t weight_bytes_per_step;  /* weights streamed per decode step (active experts for MoE at B=1) */
} xlpk_info;

typedef struct xlpk_engine* xlpk_handle;

/* Validate `cfg`, pack the weights into a library-owned buffer laid out in
 * the order the CTAs stream them, build the RoPE table, allocate the
 * workspace and borrow the KV pointers for the handle's lifetime (the KV
 * cache is written in place).  Weight buffers may be freed afterwards.
 * Runs on the current device and synchronises it first, so weights still
 * being written by work enqueued on any stream are complete before they are
 * packed.  Returns XLPK_ERR_INVALID_ARG for a bad shape or pointer (NULL,
 * unaligned) and XLPK_ERR_UNSUPPORTED for a shape this build does not handle,
 * before any device work; *out is NULL on every error.
 * Source: the decode graph is compiled ahead of time into one resident engine
 * whose tile shapes, placement and buffers are fixed before the first token
 * ("Ultra-High Interactivity On NVIDIA GPUs? - TileRT InferenceX", digest,
 * core views and the AoT static-compilation concept; the fixed temporary-
 * tensor table of "Persistent execution paradigm", section 5.3). */
xlpk_status xlpk_create(const xlpk_config* cfg, const xlpk_weights* weights,
                        const xlpk_kv* kv, xlpk_handle* out);

/* Free everything the handle owns (not the caller's KV or weights).  Waits
 * for the device first.  (The pages are silent; resource release of the
 * handle above.) */
xlpk_status xlpk_destroy(xlpk_handle h);

/* Set the decode state: sequence b has seq_lens_host[b] positions already in
 * the KV cache and pending input token tokens_host[b] (both host arrays of B
 * entries, read during the call).  The tokens are copied to the device on
 * `stream`.  XLPK_ERR_INVALID_ARG for a token outside [0, vocab) or a length
 * outside [0, max_seq).  Host arrays let every value be checked before
 * anything is enqueued.
 * Source: the request's cache state at the start of decode ("XL-Persistent-
 * Kernel", request lifecycle: the decode worker takes over the prefilled KV
 * pages). */
xlpk_status xlpk_set_state(xlpk_handle h, const int32_t* tokens_host,
                           const int32_t* seq_lens_host, void* stream);

/* Greedy-decode n_steps tokens per sequence as ONE persistent kernel launch.
 * tokens_out_dev [n_steps][B] receives the argmax of every step.  Step s feeds
 * the pending token at position seq_len + s, appends K/V there, and makes
 * the argmax (or forced_tokens[s][b]) the next pending token.  `io` may be
 * NULL.  Asynchronous on `stream`; XLPK_ERR_KV_FULL if seq_len + n_steps >
 * max_seq; device-side failures are reported by xlpk_get_status.
 * Source: the host launches the engine once and execution stays resident on
 * the GPU for the whole decode ("Ultra-High Interactivity On NVIDIA GPUs? -
 * TileRT InferenceX", digest, core views; "TileRT speed notes", Persistent
 * Execution / Tile-Level Pipeline). */
xlpk_status xlpk_decode(xlpk_handle h, int32_t n_steps, int32_t* tokens_out_dev,
                        const xlpk_decode_io* io, void* stream);

/* The same decode as one kernel launch per operator stage, built from the same
 * tiles: the kernel-per-op baseline.  Per layer: QKV, attention, O-projection
 * and gate/up + down (one fused FFN launch where the persistent kernel fuses
 * them); per step the LM head.  Each call first clears the handle's dependency
 * counters on `stream` (an async memset) and calls nothing that synchronises,
 * so its launches may be recorded by stream capture into a CUDA graph and
 * replayed; a replay decodes the captured positions again, from the tokens the
 * device holds.  Errors as xlpk_decode.
 * Source: the launch -> load -> compute -> store -> synchronise cycle per
 * operator that persistent execution removes ("Persistent execution
 * paradigm", section 1; "Ultra-High Interactivity On NVIDIA GPUs? - TileRT
 * InferenceX", digest, section "GPU bottleneck is latency, not bandwidth"). */
xlpk_status xlpk_decode_unfused(xlpk_handle h, int32_t n_steps, int32_t* tokens_out_dev,
                                const xlpk_decode_io* io, void* stream);

/* Allocation-free decode.  The pages have no counterpart to this entry point;
 * it exists for callers that must not allocate device memory while they
 * decode: threads that must never enter the CUDA allocator, or processes whose
 * device memory is entirely owned by another framework's caching allocator.  It runs
 * the same persistent kernel as xlpk_decode, with the same arguments and
 * results, but every per-call scratch buffer of the kernel (activation vectors,
 * attention and LM-head partials, dependency counters) lives in one array
 * compiled into the library: XLPK_NOALLOC_SCRATCH_BYTES bytes of file-scope
 * __device__ memory that every GPU which loads the library holds until the
 * process exits.  It calls no cudaMalloc, cudaFree or other allocating routine.
 *  - The array's device address is looked up (cudaGetSymbolAddress) with the
 *    device current at the first call on each device, and again if the
 *    device's context has been replaced since (after cudaDeviceReset).
 *  - Returns XLPK_ERR_UNSUPPORTED (with a message in xlpk_last_cuda_error) if
 *    the handle's scratch would exceed the array.
 *  - The counters in the array are cleared on `stream` at the start of each
 *    call; every other scratch byte is written before it is read.
 *  - All calls share the one array: calls whose executions overlap on the GPU
 *    (different streams, handles or threads) race.  Serialise them.
 *  - Device-side status is reported by xlpk_get_status(h) as for xlpk_decode. */
#define XLPK_NOALLOC_SCRATCH_BYTES (8u << 20)
xlpk_status xlpk_decode_noalloc(xlpk_handle h, int32_t n_steps, int32_t* tokens_out_dev,
                                const xlpk_decode_io* io, void* stream);

/* Speculative verification: check n_draft proposed tokens in ONE persistent
 * launch and accept the longest correct prefix on the device.  The handle must
 * have batch = n_draft + 1 and a paged cache whose sequences all name the same
 * pages (one page-table row repeated): sequence b of the step feeds the pending
 * token (b = 0) or draft b - 1 at position pos + b, writes its K/V row there and
 * attends to every row up to it, including the rows the sequences before it write
 * in the same step.  argmax_dev [n_draft + 1] receives the greedy token after
 * each fed position; drafts are accepted while draft[a] == argmax[a], and the
 * tokens emitted are draft[0..a-1] followed by argmax[a] (the bonus token):
 * *emitted_host = a + 1.  The handle's state advances by a + 1 positions with
 * argmax[a] pending (the K/V rows of rejected drafts are rewritten before they
 * are read again).  Synchronises `stream`; returns the device status.  `io` may
 * name per-position logits ([1][n_draft + 1][V]) and hidden states; NULL.
 * Source: draft-token verification against the target model, accepted tokens
 * committed and the rest discarded ("XL-Persistent-Kernel", request lifecycle
 * steps 5-7; fused speculative verification among its features to implement;
 * MTP in "Persistent execution paradigm", section 3). */
xlpk_status xlpk_verify(xlpk_handle h, const int32_t* draft_dev, int32_t n_draft, int32_t* argmax_dev,
                        int32_t* emitted_host, const xlpk_decode_io* io, void* stream);

/* Parity mode: register device buffers logits_dev (fp32 [B][V]) and
 * hidden_dev (fp32 [B][H], the residual after the last layer) into which every
 * later decode call on the handle (xlpk_decode, xlpk_decode_unfused,
 * xlpk_decode_noalloc) writes each step's values, one step over the other, so
 * that after a call they hold its last step's.  A call whose `io` names its own
 * logits or hidden buffer writes those instead.  Either pointer may be NULL;
 * NULL, NULL turns parity mode off.  The buffers are borrowed until then; they
 * must be 16-byte aligned (else XLPK_ERR_INVALID_ARG).
 * Source: the oracle comparison of logits and hidden states that the decode is
 * checked by (the pages are silent; a debug output of the boundary). */
xlpk_status xlpk_debug_logits(xlpk_handle h, float* logits_dev, float* hidden_dev);

/* Device-resident request loop ("serve mode").  xlpk_serve_start launches the
 * persistent kernel once; it stays resident and decodes whatever steps the
 * host posts, with no launch per request.  The host posts a request with
 * xlpk_serve_post (a count of further greedy steps, written to a word in
 * host-mapped memory); the kernel's first CTA polls that word, forwards it to
 * the other CTAs through a device counter, decodes the steps, and publishes
 * each step's tokens and a completed-step count to host-mapped memory, which
 * xlpk_serve_wait reads.  While no request is pending the kernel waits at most
 * idle_limit_us and then leaves on its own; a later post (or a wait that finds
 * it gone) launches it again from the handle's state, transparently.  Every
 * wait on the device is bounded.  During a session the handle's other decode
 * calls and xlpk_set_state return XLPK_ERR_INVALID_ARG.
 * Source: a GPU-resident scheduler drives the decode loop and the host only
 * posts descriptors into a ring the kernel claims ("Persistent execution
 * paradigm", section 5.6); device-resident request descriptors and work queue
 * ("XL-Persistent-Kernel", features to be implemented). */

/* Open a session on `stream` from the handle's current state (xlpk_set_state):
 * allocates the mapped control words and token ring once per handle (pinned
 * host memory) and launches the loop.  idle_limit_us > 0. */
xlpk_status xlpk_serve_start(xlpk_handle h, int32_t idle_limit_us, void* stream);

/* Post a request for n_steps more greedy steps (> 0) of every sequence;
 * *first_step receives the session index of its first step (steps are
 * numbered from 0 in posting order).  Returns without waiting;
 * XLPK_ERR_KV_FULL if the session's steps would pass max_seq. */
xlpk_status xlpk_serve_post(xlpk_handle h, int32_t n_steps, int64_t* first_step);

/* Wait (host polling, at most timeout_us) until session steps
 * [first_step, first_step + n_steps) are decoded and copy their tokens
 * [n_steps][B] to tokens_out_host.  XLPK_ERR_TIMEOUT if they are not done in
 * time; a device-side failure of the loop is returned as its status. */
xlpk_status xlpk_serve_wait(xlpk_handle h, int64_t first_step, int32_t n_steps, int32_t* tokens_out_host,
                            int32_t timeout_us);

/* Ask the loop to leave once every posted step is decoded, wait for it, fold
 * the session's steps into the handle's state (a later xlpk_decode continues
 * after them) and close the session.  Returns the loop's device status. */
xlpk_status xlpk_serve_stop(xlpk_handle h);

/* End-to-end call with host buffers: uploads the state, decodes, downloads
 * tokens_out_host [n_steps][B], and synchronises `stream`.  Returns the
 * device status of the decode.
 * Source: a request submitted with its prompt state and answered with its
 * tokens ("XL-Persistent-Kernel", request lifecycle, steps 1 and 8). */
xlpk_status xlpk_generate(xlpk_handle h, const int32_t* tokens_host, const int32_t* seq_lens_host,
                          int32_t n_steps, int32_t* tokens_out_host, void* stream);

/* Synchronise the stream of the handle's last decode and return its device
 * status (XLPK_OK, XLPK_ERR_TIMEOUT or XLPK_ERR_ABORTED).  After an error the
 * handle's counters are reset; KV entries the failed call would have written
 * are unspecified.
 * Source: a persistent kernel has no per-operator failure boundary, so every
 * device-side wait is bounded and reported ("Persistent execution paradigm",
 * section 7.3, execution stability at the hardware's limits). */
xlpk_status xlpk_get_status(xlpk_handle h);

/* Facts about a created handle (grid, shared memory, ring, packed bytes).
 * (The pages are silent; measurement support.) */
xlpk_status xlpk_get_info(xlpk_handle h, xlpk_info* out);

/* Human-readable name of a status; "XLPK_ERR_UNKNOWN" for other values. */
const char* xlpk_status_string(int32_t status);

/* Text of the last CUDA error seen by this thread's calls ("" if none). */
const char* xlpk_last_cuda_error(void);

/* One batch-8 projection on the tcgen05 tensor cores:
 *     y[n][b] = sum_k w[n][k] * bf16(x[b][k]),   n < N, b < 8,
 * the dense [N x K] . [K x 8] contraction that the decoder's linear layers
 * become for 8 sequences at once, as a stand-alone call (the batch-8 decode
 * runs the same MMAs inside the persistent kernel).
 *  - w_dev: bf16 [N][K] row-major; x_dev: fp32 [8][K] row-major (rounded to
 *    bf16, round-to-nearest-even, as it enters the MMA); y_dev: fp32 [N][8]
 *    row-major, written.  All three 16-byte aligned, on the current device;
 *    nothing is retained after the call.
 *  - N >= 128 (one CTA per 128 rows; a ragged last block is fine),
 *    64 <= K <= 4096 and K a multiple of 64; else XLPK_ERR_INVALID_ARG.
 *  - Runs on `stream` and waits for it: returns XLPK_OK, XLPK_ERR_UNSUPPORTED
 *    on a device that is not sm_100, XLPK_ERR_CUDA, or XLPK_ERR_TIMEOUT if a
 *    device-side wait ran out (the kernel then leaves without writing y).
 *    One call at a time per process (the device-side error word is shared).
 * Source: tensor-core warp groups for the dense parts of the engine ("TileRT
 * speed notes", Warp / Block Specialization; "Persistent execution paradigm",
 * section 6.2, warp specialisation). */
xlpk_status xlpk_tc_gemm_tile(const void* w_dev, int32_t n, int32_t k, const float* x_dev, float* y_dev,
                              void* stream);

#ifdef __cplusplus
}
#endif

#endif /* XLPK_H_ */
