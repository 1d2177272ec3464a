/*
 * tt_denoise.h -- C ABI of the B200 (sm_100a) TwoTower denoiser refinement step.
 *
 * One refinement step of TwoTower block-autoregressive diffusion decoding, as described in
 * "Nemotron-TwoTower: Diffusion Language Modeling with Pretrained AR Context" (arXiv 2606.26493,
 * "the paper" below), has three GPU operations, each one entry point here:
 *
 *   tt_denoise_attn    layer-aligned denoiser attention, the paper §2.1 Eq. (1)
 *   tt_adaln_modulate  adaLN-single time conditioning, the paper §2.1 "Time conditioning"
 *   tt_unmask_step     confidence-threshold unmasking, the paper §2.2 "Sampling", Algorithm 2
 *   tt_block_tau       the step's time input from the mask, Algorithm 2 (its time input, the masked fraction)
 *   tt_kv_append       block commit into the paged context cache, Algorithm 1 (context update)
 *   tt_lmhead_unmask_step  the unmask step from hidden states (LM head fused, logits never stored)
 *
 * Conventions shared by every entry point
 *   - Every pointer named in an args struct is a DEVICE pointer (cudaMalloc'd or equivalent)
 *     unless its comment says "host". The caller owns all memory; the library never allocates
 *     or frees, keeps no mutable global state, and may be called from several host threads.
 *   - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default).
 *   - Tensors are dense, row-major, with the shapes written in brackets.
 *   - Argument errors are found on the host and returned before anything is launched:
 *     TT_ERR_INVALID_ARGUMENT (null pointer, bad size), TT_ERR_UNSUPPORTED (valid but not
 *     implemented, e.g. a head_dim the kernels do not handle), TT_ERR_WORKSPACE_TOO_SMALL.
 *   - A failed launch returns TT_ERR_CUDA (the CUDA error is left for cudaGetLastError()).
 *   - Errors only the device can see (a page id outside the pool, a context length beyond the
 *     page table or the contiguous stride, a wait that timed out) never trap: the kernel sets a
 *     word in the caller's workspace, skips the offending work, and tt_get_device_error()
 *     reports it as TT_ERR_DEVICE or TT_ERR_DEVICE_TIMEOUT.
 *   - Inputs must be finite. NaN/Inf inputs give unspecified (but non-faulting) results.
 *   - Early exit of a multi-step loop (Algorithm 2 finishes a block within T steps, often sooner):
 *     every args struct (and tt_block_tau) takes an optional device word `skip_if`. When it is
 *     non-NULL and holds a non-zero value once the kernel's inputs are ready, the call does
 *     nothing: no output, workspace or error word is touched. The unmask entries can set such a
 *     word (`all_done`) when no sequence of the batch has a masked position left, so the later
 *     steps of a loop captured in one CUDA graph cost only their launches.
 *   - Workspaces must be zero-filled (cudaMemset) before their first use. Their layout depends
 *     on the argument sizes; the kernels restore the merge tickets of that layout to zero, so a
 *     workspace can be reused without re-zeroing by calls with the same sizes. Zero it again
 *     before a call with different sizes. Calls sharing a workspace must be stream-ordered.
 */
#ifndef TT_DENOISE_H_
#define TT_DENOISE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* tt_stream_t;

typedef enum {
  TT_OK = 0,
  TT_ERR_INVALID_ARGUMENT = 1,
  TT_ERR_UNSUPPORTED = 2,
  TT_ERR_WORKSPACE_TOO_SMALL = 3,
  TT_ERR_CUDA = 4,
  TT_ERR_DEVICE = 5,
  TT_ERR_DEVICE_TIMEOUT = 6
} tt_status_t;

typedef enum { TT_F32 = 0, TT_BF16 = 1 } tt_dtype_t;

/* Human-readable name of a status code (static string, never NULL). */
const char* tt_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
int tt_version(void);

/* ---------------------------------------------------------------------------------------------
 * Eq. (1), the paper §2.1 "Bidirectional attention": the S queries of the noisy block b at
 * denoiser layer i attend to the concatenation of the context tower's layer-i keys/values for
 * the past blocks 0..b-1 (the prefix cache, L_b tokens) and the denoiser's own layer-i
 * keys/values of block b (S tokens):
 *     O = softmax(softmax_scale * Q [K_ctx; K_blk]^T) [V_ctx; V_blk]
 * Inside the block attention is bidirectional; every past block precedes the block, so no
 * query is masked from any key: the only mask is the ragged end of each context.
 * Grouped-query layout: query head h reads key/value head h / (Hq / Hkv).
 *
 * Layouts (E = element type given by dtype: TT_BF16 = bfloat16, TT_F32 = float):
 *   q       [B][S][Hq][d]   E
 *   k_blk   [B][S][Hkv][d]  E      (v_blk likewise)
 *   k_ctx   contiguous (page_table == NULL): [B][ctx_stride][Hkv][d] E, sequence b's token t at
 *           row t of its slab; paged: [num_pages][page_size][Hkv][d] E, token t of sequence b at
 *           page page_table[b][t / page_size], row t % page_size.  (v_ctx likewise)
 *   ctx_lens [B] int32, L_b >= 0 (0 = the first block: attention over the block alone)
 *   page_table [B][max_pages_per_seq] int32 or NULL
 *   out     [B][S][Hq][d]   E, rounded to nearest from the fp32 result
 *   lse     [B][Hq][S] float or NULL: natural-log log-sum-exp of the scaled scores per row
 * Supported: TT_BF16 with d = 128 (tensor-core path, S*Hq/Hkv rows per tile, S <= 64,
 * page_size a multiple of 128); TT_F32 with d in {64, 128} (tensor cores, tf32 with the split
 * operands). Others: TT_ERR_UNSUPPORTED.
 * ------------------------------------------------------------------------------------------- */
typedef struct {
  int32_t batch;             /* B >= 1 */
  int32_t block_size;        /* S, 1..64 */
  int32_t num_q_heads;       /* Hq, multiple of Hkv */
  int32_t num_kv_heads;      /* Hkv >= 1 */
  int32_t head_dim;          /* d */
  int32_t dtype;             /* tt_dtype_t */
  float softmax_scale;       /* > 0, multiplies Q.K (1.0 when Q is pre-scaled) */
  const void* q;
  const void* k_blk;
  const void* v_blk;
  const void* k_ctx;
  const void* v_ctx;
  const int32_t* ctx_lens;
  const int32_t* page_table; /* NULL => contiguous context */
  int32_t page_size;         /* paged: tokens per page */
  int32_t max_pages_per_seq; /* paged: row length of page_table */
  int32_t num_pages;         /* paged: pages in the pool */
  int32_t ctx_stride;        /* contiguous: rows per sequence slab (>= every L_b) */
  void* out;
  float* lse;                /* optional */
  const int32_t* skip_if;    /* optional device word: non-zero => the call does nothing */
} tt_attn_args_t;

/* Bytes of workspace tt_denoise_attn needs for these arguments (0 if the args are invalid). */
size_t tt_denoise_attn_workspace_bytes(const tt_attn_args_t* args);

/* Launch Eq. (1): the attention kernel and, stream-ordered behind it, the kernel that merges the
 * split-KV partial results. `workspace` (device) holds the partition of the tiles, the partial
 * results and the device error word. */
int tt_denoise_attn(const tt_attn_args_t* args, void* workspace, size_t workspace_bytes,
                    tt_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * adaLN-single, the paper §2.1 "Time conditioning": a global MLP maps the diffusion time to
 * shared (shift, scale, gate) parameters and a per-layer learned embedding is added; the
 * result modulates the layer's RMSNorm prologue and gates its residual.
 *
 * op TT_ADALN_COND (tau, weights -> mod):
 *   phi(tau) = [cos(1000 tau w_k), sin(1000 tau w_k)], w_k = 10000^(-k/(F/2)), k < F/2
 *   mod[b] = W3 SiLU(W2 SiLU(W1 phi(tau_b) + b1) + b2) + b3, viewed as [3][D], + layer_emb
 *   tau [B] float; w1 [W][F], b1 [W], w2 [W][W], b2 [W], w3 [3D][W], b3 [3D], layer_emb [3][D]
 *   (all float); mod [B][3][D] float (rows: shift, scale, gate). F and W multiples of 4 up to
 *   1024; w1, w2, w3 16-byte aligned.
 *   Needs workspace of tt_adaln_workspace_bytes() bytes (the MLP's hidden activations).
 * op TT_ADALN_NORM_MODULATE (h, norm_w, mod -> out):
 *   out[b][s] = h[b][s] / sqrt(mean(h[b][s]^2) + eps) * norm_w * (1 + scale[b]) + shift[b]
 *   h, out [B][S][D] E; norm_w [D] float.
 * op TT_ADALN_GATED_RESIDUAL (h, f, mod -> out):
 *   out[b][s] = h[b][s] + gate[b] * f[b][s]        h, f, out [B][S][D] E (out may alias h)
 * op TT_ADALN_NORM_MODULATE_RESIDUAL (h, f, norm_w, mod -> out, out2): both of the above from one
 *   read of h: out = NORM_MODULATE's output, out2 = GATED_RESIDUAL's output. out2 may alias h; out
 *   must not alias f or out2.
 * D must be a multiple of 8 for TT_BF16 and of 4 for TT_F32; h, f, out, out2, mod and norm_w
 * 16-byte aligned (else TT_ERR_UNSUPPORTED).
 * ------------------------------------------------------------------------------------------- */
typedef enum {
  TT_ADALN_COND = 0,
  TT_ADALN_NORM_MODULATE = 1,
  TT_ADALN_GATED_RESIDUAL = 2,
  TT_ADALN_NORM_MODULATE_RESIDUAL = 3
} tt_adaln_op_t;

typedef struct {
  int32_t op;                /* tt_adaln_op_t */
  int32_t batch;             /* B */
  int32_t block_size;        /* S (NORM_MODULATE, GATED_RESIDUAL) */
  int32_t hidden;            /* D */
  int32_t freq_dim;          /* F (COND) */
  int32_t mlp_width;         /* W (COND) */
  int32_t dtype;             /* tt_dtype_t of h, f, out */
  float eps;                 /* RMSNorm epsilon */
  const float* tau;
  const float* w1;
  const float* b1;
  const float* w2;
  const float* b2;
  const float* w3;
  const float* b3;
  const float* layer_emb;
  float* mod;                /* COND: output; other ops: input */
  const void* h;
  const float* norm_w;
  const void* f;
  void* out;
  const int32_t* skip_if;    /* optional device word: non-zero => the call does nothing */
  void* out2;                /* NORM_MODULATE_RESIDUAL: the gated residual's output */
} tt_adaln_args_t;

size_t tt_adaln_workspace_bytes(const tt_adaln_args_t* args);
int tt_adaln_modulate(const tt_adaln_args_t* args, void* workspace, size_t workspace_bytes,
                      tt_stream_t stream);

typedef enum {
  TT_SAMPLER_CONFIDENCE = 0,     /* commit every prediction with confidence >= gamma */
  TT_SAMPLER_PREDICT_NOISE = 1   /* commit all but keep_masked, the least confident re-masked */
} tt_sampler_t;

/* ---------------------------------------------------------------------------------------------
 * ConfidenceSample, the paper §2.2 "Sampling" and Algorithm 2: the denoiser predicts
 * every masked position in parallel; predictions whose confidence reaches gamma are committed,
 * the rest stay masked for later steps.
 *   conf[b][l]   = max_v softmax(inv_temperature * logits[b][l])_v
 *   argmax[b][l] = smallest v attaining max_v logits[b][l][v]
 *   For each sequence b: every position with is_masked = 1 and conf >= gamma is committed
 *   (tokens := argmax, is_masked := 0). If none qualifies and a position is still masked, the
 *   single masked position with the largest conf is committed (lowest position on ties). With
 *   remaining_steps > 0 (the T - r + 1 of Algorithm 2), at least ceil(n_masked/remaining_steps)
 *   of the most confident masked positions are committed, so a block finishes within T steps.
 *   Positions already committed are never changed.
 * sampler = TT_SAMPLER_PREDICT_NOISE selects the predict-and-noise sampler instead (the paper
 *   §2.2 "Sampling", the standard sampler of block diffusion): every masked position is
 *   predicted and the least confident ones are re-masked following the noise schedule, i.e. the
 *   (n_masked - keep_masked) most confident masked positions are committed (confidence
 *   descending, position ascending) and min(n_masked, keep_masked) stay masked; gamma and
 *   remaining_steps are ignored. With noise_steps = T > 0 the library derives keep_masked itself
 *   from the linear schedule alpha_t = 1 - t (the paper §2.2, Eq. (3)): after step r = noise_step
 *   of T the masked fraction is t = (T - r) / T, so keep_masked = floor(S * (T - r) / T)
 *   (tt_linear_schedule_keep); the keep_masked field is then ignored.
 * Layouts: logits [B][S][V] E; tokens [B][S] int32 (in/out); is_masked [B][S] uint8 (in/out,
 *   0/1); conf [B][S] float and argmax [B][S] int32 (optional outputs, may be NULL);
 *   n_committed, n_masked [B] int32 outputs. exclude_mask_token != 0 removes the logit of
 *   mask_token_id from both the softmax and the argmax. V must be a multiple of 8 (bf16) or
 *   4 (fp32); S <= 1024.
 * ------------------------------------------------------------------------------------------- */
typedef struct {
  int32_t batch;             /* B */
  int32_t block_size;        /* S */
  int32_t vocab;             /* V */
  int32_t dtype;             /* tt_dtype_t of logits */
  const void* logits;
  float gamma;               /* confidence threshold */
  float inv_temperature;     /* > 0 */
  int32_t mask_token_id;
  int32_t exclude_mask_token;
  int32_t remaining_steps;   /* 0 => commit >= gamma, else the single most confident */
  int32_t* tokens;
  uint8_t* is_masked;
  float* conf;               /* optional */
  int32_t* argmax;           /* optional */
  int32_t* n_committed;
  int32_t* n_masked;
  int32_t sampler;           /* tt_sampler_t; 0 (TT_SAMPLER_CONFIDENCE) when zero-initialised */
  int32_t keep_masked;       /* TT_SAMPLER_PREDICT_NOISE, noise_steps == 0: masked positions to keep, >= 0 */
  int32_t noise_steps;       /* TT_SAMPLER_PREDICT_NOISE: T > 0 derives keep_masked from the linear
                                schedule; 0 uses keep_masked as given */
  int32_t noise_step;        /* r in 1..noise_steps when noise_steps > 0 */
  const int32_t* skip_if;    /* optional device word: non-zero => the call does nothing */
  int32_t* all_done;         /* optional device word: set to 1 when, after this step, no sequence
                                has a masked position left (never cleared by the library) */
} tt_unmask_args_t;

/* The linear noise schedule of the predict-and-noise sampler, the paper §2.2 Eq. (3) with
 * alpha_t = 1 - t: positions of a block of block_size that stay masked after step `step` of
 * `steps`, floor(block_size * (steps - step) / steps). Host function; returns -1 unless
 * block_size >= 1, steps >= 1 and 1 <= step <= steps. */
int32_t tt_linear_schedule_keep(int32_t block_size, int32_t steps, int32_t step);

size_t tt_unmask_workspace_bytes(const tt_unmask_args_t* args);
int tt_unmask_step(const tt_unmask_args_t* args, void* workspace, size_t workspace_bytes,
                   tt_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * tt_unmask_step_noalloc: tt_unmask_step without a workspace and without any allocation.
 *
 * The paper has no counterpart: this is an interface variant of the confidence-threshold step
 * above (same arguments, same kernel, same results) for callers that cannot allocate device
 * memory when they call it, e.g. a host runtime with no CUDA allocator of its own that owns only
 * the buffers handed to it, or a decode loop that forbids allocation once running. Its scratch
 * is a fixed array in the library's static device memory (168 KiB per device).
 *
 *   - Limit: batch * block_size <= 4096. Larger sizes return TT_ERR_WORKSPACE_TOO_SMALL (the
 *     built-in scratch is too small) before anything is launched; use tt_unmask_step instead.
 *   - Setup: the first call on a device (with that device current) resolves the scratch address
 *     and enqueues on `stream` the clearing of its counters; make that first call before any
 *     stream capture begins. Later calls only launch the kernel, which leaves the counters at
 *     zero again. A failure of the setup returns TT_ERR_CUDA.
 *   - One scratch per device, shared by all callers: calls on the same device must be ordered
 *     (one stream, or events between streams). Calls that overlap on the device race on the
 *     scratch and give undefined results.
 *   - This is the one entry point that keeps library state (the scratch and its address).
 *   - The kernel sets no device error word; tt_get_device_error does not apply.
 * ------------------------------------------------------------------------------------------- */
int tt_unmask_step_noalloc(const tt_unmask_args_t* args, tt_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * tt_lmhead_unmask_step: the unmask step (either sampler, same rule and outputs as
 * tt_unmask_step) computed from the final hidden states instead of the logits, the paper §2.2:
 * the denoiser's LM head produces p_theta = softmax(x W^T) for every block position, and here the
 * logits x W^T are reduced to (confidence, argmax) tile by tile on the tensor cores without ever
 * being written to memory.
 *   x   device bf16 [batch][block_size][hidden]   (hidden states after the final norm)
 *   w   device bf16 [vocab][hidden]                (LM-head weight)
 *   the remaining fields as in tt_unmask_args_t (logits replaced by x and w; conf / argmax are
 *   optional outputs). Logits are accumulated in fp32.
 * Supported: TT_BF16; hidden a multiple of 64; vocab a multiple of 128; block_size <= 1024; x and
 * w 16-byte aligned (else TT_ERR_UNSUPPORTED). Workspace: tt_lmhead_unmask_workspace_bytes(),
 * zero-filled before first use; the kernel returns its tickets to zero, so it can be reused by
 * calls with the same sizes.
 * ------------------------------------------------------------------------------------------- */
typedef struct {
  int32_t batch, block_size, hidden, vocab;
  int32_t dtype;
  const void* x;
  const void* w;
  float gamma;
  float inv_temperature;
  int32_t mask_token_id;
  int32_t exclude_mask_token;
  int32_t remaining_steps;
  int32_t* tokens;
  uint8_t* is_masked;
  float* conf;
  int32_t* argmax;
  int32_t* n_committed;
  int32_t* n_masked;
  int32_t sampler;
  int32_t keep_masked;
  int32_t noise_steps;
  int32_t noise_step;
  const int32_t* skip_if;    /* as in tt_unmask_args_t */
  int32_t* all_done;         /* as in tt_unmask_args_t */
} tt_lmhead_unmask_args_t;

size_t tt_lmhead_unmask_workspace_bytes(const tt_lmhead_unmask_args_t* args);
int tt_lmhead_unmask_step(const tt_lmhead_unmask_args_t* args, void* workspace, size_t workspace_bytes,
                          tt_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * tt_kv_append: block commit into the paged context cache, the paper §2.2, Algorithm 1 (the
 * context update once a block is committed)
 * ("update the AR context" once block b is committed): the context tower's K and V for the S
 * tokens of the committed block are appended after each sequence's current context, taking new
 * pages from a free-page stack as needed. The context tower that produces k_new / v_new is not
 * part of this library.
 *
 * For sequence b with L = ctx_lens[b]: rows L .. L+S-1 of its context are written from
 * k_new[b] / v_new[b] through page_table[b] (position p lives in page page_table[b][p / page_size],
 * slot p % page_size); the pages holding positions >= ceil(L / page_size) * page_size are taken
 * from the top of the free stack, in order, and entered in page_table[b]; ctx_lens[b] += S.
 * Pages are claimed per sequence with a compare-and-swap on *free_count that never lowers it
 * below the claim, so a sequence that cannot be served changes nothing; which free pages a
 * sequence receives depends on the order the sequences run in (the content each sees does not).
 *
 *   k_new, v_new   device [batch][block_size][num_kv_heads][head_dim] (dtype)
 *   k_ctx, v_ctx   device paged pool [num_pages][page_size][num_kv_heads][head_dim] (dtype), written
 *   page_table     device int32 [batch][max_pages_per_seq], in/out
 *   ctx_lens       device int32 [batch], in/out
 *   free_pages     device int32 [>= *free_count]: entries [0, *free_count) are free page ids
 *   free_count     device int32 scalar, in/out (decreases by the pages taken)
 * Errors (host): TT_ERR_INVALID_ARGUMENT for null pointers or sizes < 1; TT_ERR_UNSUPPORTED unless
 * head_dim * element size is a multiple of 16 bytes and the four tensors are 16-byte aligned.
 * Errors (device, via tt_get_device_error; the failing sequence, its page_table row and the free
 * stack are left unchanged; the other sequences proceed): the free stack is too short, an entry
 * it would hand out is not a page id in [0, num_pages), or the context would need more than
 * max_pages_per_seq pages.
 * Workspace: tt_kv_append_workspace_bytes() (the error word), zero-filled before first use.
 * ------------------------------------------------------------------------------------------- */
typedef struct {
  int32_t batch, block_size, num_kv_heads, head_dim;
  int32_t dtype;                  /* tt_dtype_t */
  const void* k_new;
  const void* v_new;
  void* k_ctx;
  void* v_ctx;
  int32_t* page_table;
  int32_t* ctx_lens;
  const int32_t* free_pages;
  int32_t* free_count;
  int32_t page_size, max_pages_per_seq, num_pages;
} tt_kv_append_args_t;

size_t tt_kv_append_workspace_bytes(const tt_kv_append_args_t* args);
int tt_kv_append(const tt_kv_append_args_t* args, void* workspace, size_t workspace_bytes, tt_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * tt_block_tau: the time input of one refinement step, the paper §2.2, Algorithm 2 (the masked
 * fraction of the block):
 * tau_b = |{l : z_l = [MASK]}| / S, computed on the device from the mask so that a multi-step
 * loop (captured in one CUDA graph) needs no host round trip between steps.
 *   is_masked  device u8 [batch][block_size], 1 = still masked
 *   tau        device float [batch], written
 *   skip_if    optional device word (NULL = none): non-zero => nothing is written
 * Errors: TT_ERR_INVALID_ARGUMENT (null pointer, batch < 1, block_size < 1); TT_ERR_CUDA on a
 * failed launch. No workspace.
 * ------------------------------------------------------------------------------------------- */
int tt_block_tau(const uint8_t* is_masked, int32_t batch, int32_t block_size, float* tau, const int32_t* skip_if,
                 tt_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * tt_probe_bounded_wait: a diagnostic of the library's failure path (the paper has no
 * counterpart). Launches one thread that waits, with the same bounded wait the kernels use, on a
 * shared-memory barrier that nothing ever arrives on. After limit_us microseconds (1 ..
 * 1000000; the kernels' own limit is one second) the wait gives up, the kernel records
 * TT_ERR_DEVICE_TIMEOUT with detail TT_DETAIL_WAIT_PROBE in the workspace's error word and
 * returns: no trap, no endless wait, the context stays usable. tt_get_device_error() then
 * reports it. workspace: any workspace of >= 256 bytes (its header is used). Errors (host):
 * TT_ERR_INVALID_ARGUMENT for a null workspace or a limit outside 1 .. 1000000; TT_ERR_CUDA on
 * a failed launch.
 * ------------------------------------------------------------------------------------------- */
#define TT_DETAIL_WAIT_PROBE 0x1ffu
int tt_probe_bounded_wait(void* workspace, uint32_t limit_us, tt_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * Device-side error word of a workspace (any of the three). Synchronises `stream`, reads the
 * word and clears it. Returns TT_OK, TT_ERR_DEVICE (bad page id / context length) or
 * TT_ERR_DEVICE_TIMEOUT (a bounded wait inside a kernel gave up). *detail (host, may be NULL)
 * receives a kernel-specific code for diagnostics.
 * ------------------------------------------------------------------------------------------- */
int tt_get_device_error(void* workspace, tt_stream_t stream, uint32_t* detail);

#ifdef __cplusplus
}
#endif

#endif /* TT_DENOISE_H_ */
