/*
 * gdla.h -- C ABI of the B200 (sm_100a) GDLA forward library, libgdla.so.
 *
 * Grouped Differential Latent Attention as stated in "Motif 3: Technical
 * Report" (montaan.com/papers/2608.09119), section "Architecture", the GDLA
 * paragraphs: the compressed KV latent is RMS-normalised and expanded by one
 * up-projection W_UKV into n_kv content-key/value heads shared by the signal
 * and noise query paths; a decoupled rotary key is shared across heads and
 * RoPE touches only the rotary query/key parts; g*n_N signal heads and n_N
 * noise heads attend independently under a full causal or a sliding-window
 * mask; D_t = H_S,t - lambda_t (.) Repeat_g(H_N,t) with lambda_t = sigmoid of
 * a per-(token, signal head) logit; Y = sigmoid(G) (.) D is the element-wise
 * output gate applied before the output projection. Dimensions in that report:
 * 16 KV heads, d_qk = 192 (128 content + 64 rotary), d_v = 128, d_c = 512.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller, dense
 *    row-major in the layout stated beside them, 16-byte aligned. (The bf16
 *    attention uses 32-byte accesses when gate_logits, out and both RoPE
 *    tables are 32-byte aligned, which allocators normally give; with only
 *    16-byte alignment it returns the same bytes a little more slowly.) The library
 *    allocates no memory and keeps no per-call state; scratch comes from the
 *    caller's workspace, sized by the matching *_workspace_size function.
 *    Three entry points state their exceptions beside them: gdla_prefill_host
 *    takes its activations as host pointers and keeps its own copy and compute
 *    streams, gdla_decode_noalloc uses a fixed scratch array inside the library
 *    instead of a workspace, and the RoPE table builders write host arrays.
 *  - `stream` is a cudaStream_t passed as void*. All work is enqueued on it and
 *    the call returns without synchronising.
 *  - Argument errors (NULL pointer, misalignment, unsupported size, a too
 *    small workspace or RoPE table) are reported synchronously, BEFORE anything
 *    is launched, as GDLA_ERR_INVALID_ARG or GDLA_ERR_UNSUPPORTED. A failed
 *    launch returns GDLA_ERR_CUDA. A device-side wait that hit its iteration
 *    cap is recorded in the workspace's status word and reported by
 *    gdla_workspace_status (GDLA_ERR_TIMEOUT). Nothing is thrown across the ABI.
 *  - Element type: `dtype` selects bf16 or fp32 for every floating tensor
 *    except the lambda logits and the RoPE tables, which are always fp32.
 *    bf16 arithmetic accumulates in fp32; the softmax runs in fp32.
 */
#ifndef GDLA_H_
#define GDLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDLA_OK = 0,
  GDLA_ERR_INVALID_ARG = 1,  /* NULL/misaligned pointer, bad size, small workspace */
  GDLA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. n_noise != n_kv) */
  GDLA_ERR_CUDA = 3,         /* a CUDA launch or query failed */
  GDLA_ERR_TIMEOUT = 4,      /* a device wait hit its iteration cap */
  GDLA_ERR_SCRATCH_LIMIT = 5 /* gdla_decode_noalloc: the call needs more than its fixed scratch */
} gdla_status;

typedef enum {
  GDLA_MASK_CAUSAL = 0,  /* key j visible to query i iff j <= i */
  GDLA_MASK_SLIDING = 1  /* key j visible to query i iff i - window < j <= i */
} gdla_mask;

typedef enum { GDLA_BF16 = 0, GDLA_FP32 = 1 } gdla_dtype;

/* Shared sizes. n_signal = g * n_noise; the report pairs every noise head with
 * one KV head, so n_noise must equal n_kv. Signal head i reads KV head
 * floor(i/g) and subtracts noise head floor(i/g) (Repeat_g as
 * repeat-interleave). Supported head shapes (d_nope, d_rope, d_v):
 * (128, 64, 128), (64, 32, 64), (32, 16, 32); d_c in {64, 128, 256, 512};
 * 1 <= g <= 8. Other sizes return GDLA_ERR_UNSUPPORTED. The tensor-core kernels
 * serve bf16: prefill with (128, 64, 128) heads and any head count (e.g. the
 * report's 16 KV heads with g = 4, 80 query heads), decode with d_c = 512 and
 * d_rope = 64 and any head count (in groups of at most 48 query heads); every
 * other supported shape runs on the CUDA-core kernels, where decode holds at most
 * 64 query heads. A call whose shape selects a tensor-core kernel fails with
 * GDLA_ERR_CUDA if the driver's tensor-map encoder cannot be resolved; there is
 * no CUDA-core substitute for those shapes. */

/* ------------------------------------------------------------------ expansion
 * Steps 1-3 of the layer for a whole batch: latent RMSNorm, the single W_UKV
 * up-projection, and RoPE of the shared rotary key ("Motif 3: Technical
 * Report", Architecture: "normalized and expanded through a single
 * projection", "RoPE is applied only to the rotary query and key").
 *   c_hat[t]  = gamma (.) c_kv[t] / sqrt(mean(c_kv[t]^2) + rms_eps)
 *   kv[t, h]  = c_hat[t] @ W_UKV[:, h*(d_nope+d_v) : (h+1)*(d_nope+d_v)]
 *   k_rope_rot[t] = RoPE(k_rope[t], position t)
 * Positions restart at 0 for every sequence. */
typedef struct {
  int B, L;                  /* batch, tokens per sequence (>= 1) */
  int d_c, d_rope, n_kv, d_nope, d_v;
  gdla_dtype dtype;
  float rms_eps;             /* <= 0 selects 1e-6 */
  int rope_max_pos;          /* rows of the RoPE tables; must be >= L */
  const void* c_kv;          /* [B, L, d_c] pre-norm latent */
  const void* gamma;         /* [d_c] RMSNorm gain */
  const void* k_rope;        /* [B, L, d_rope] pre-RoPE rotary key */
  const void* w_ukv;         /* [d_c, n_kv*(d_nope+d_v)]; per KV head: d_nope key cols, then d_v value cols */
  const float* rope_cos;     /* [rope_max_pos, d_rope/2]: cos(pos * theta_k) */
  const float* rope_sin;     /* [rope_max_pos, d_rope/2]: sin(pos * theta_k) */
  void* kv_out;              /* [B, L, n_kv, d_nope+d_v] expanded key|value heads */
  void* k_rope_out;          /* [B, L, d_rope] rotated rotary key */
  void* c_hat_out;           /* [B, L, d_c] normalised latent; required (it feeds the GEMM) */
} gdla_expand_args;

gdla_status gdla_latent_expand(const gdla_expand_args* args, void* stream);

/* -------------------------------------------------------------------- prefill
 * The whole GDLA forward for B sequences of L tokens (steps 1-8): expansion as
 * above into the workspace, then per head the attention
 *   H_h,i = sum_j softmax_j( tau * (q_nope,h,i . k_nope,j + RoPE(q_rope,h,i) . k_rope_rot,j) ) v_j
 * over the visible keys, then
 *   Y_i = sigmoid(G_i) (.) ( H_S,i - sigmoid(lam_i) * H_N,floor(i/g) ).
 * Heads of q are ordered: signal heads 0..n_signal-1, then noise heads
 * 0..n_noise-1; each head holds d_nope content dims then d_rope pre-RoPE
 * rotary dims. If cache_c_hat / cache_k_rope are not NULL, the normalised
 * latent and rotated rotary key (the compact decode cache) are written there
 * too. */
typedef struct {
  int B, L, d_c, d_rope, n_kv, d_nope, d_v, n_noise, g;
  gdla_mask mask;
  int window;                /* used iff mask == GDLA_MASK_SLIDING; >= 1 */
  float softmax_scale;       /* tau; <= 0 selects 1/sqrt(d_nope + d_rope) */
  float rms_eps;             /* <= 0 selects 1e-6 */
  gdla_dtype dtype;
  int rope_max_pos;          /* >= L */
  const void* c_kv;          /* [B, L, d_c] */
  const void* gamma;         /* [d_c] */
  const void* k_rope;        /* [B, L, d_rope] pre-RoPE */
  const void* q;             /* [B, L, n_signal+n_noise, d_nope+d_rope] */
  const void* w_ukv;         /* [d_c, n_kv*(d_nope+d_v)] */
  const float* rope_cos;     /* [rope_max_pos, d_rope/2] */
  const float* rope_sin;     /* [rope_max_pos, d_rope/2] */
  const float* lam_logits;   /* [B, L, n_signal] fp32 */
  const void* gate_logits;   /* [B, L, n_signal, d_v] */
  void* out;                 /* [B, L, n_signal, d_v] = Y */
  void* cache_c_hat;         /* optional [B, L, d_c] */
  void* cache_k_rope;        /* optional [B, L, d_rope] */
  void* workspace;           /* >= gdla_prefill_workspace_size(args) bytes, 256-byte aligned */
  size_t workspace_bytes;
} gdla_prefill_args;

size_t gdla_prefill_workspace_size(const gdla_prefill_args* args);
gdla_status gdla_prefill(const gdla_prefill_args* args, void* stream);

/* --------------------------------------------------------------------- attend
 * Steps 3-8 alone over an already expanded latent (the second half of
 * gdla_prefill): RoPE of the rotary query parts, signal and noise attention
 * under the mask, differential subtraction and sigmoid gate, exactly as in
 * gdla_prefill. `kv` and `k_rope_rot` are the outputs of gdla_latent_expand
 * for the same batch. The workspace only carries the status word
 * (>= 256 bytes, 256-byte aligned).
 *
 * Query block (chunked prefill; the report has no counterpart, it is the same
 * attention restricted to some query rows): with q_len > 0 only the queries at
 * positions q_start .. q_start+q_len-1 of every sequence are computed. q,
 * lam_logits, gate_logits and out then hold q_len rows per sequence
 * ([B, q_len, ...]; row r is position q_start + r, which sets its RoPE angle
 * and its mask), while kv and k_rope_rot keep their L rows (positions 0..L-1).
 * Requires q_start >= 0 and q_start + q_len <= L, else GDLA_ERR_INVALID_ARG.
 * q_len == 0 (a zero-initialised struct) selects all L rows, and then q_start
 * must be 0. Every row's result is bit-identical to the whole-sequence call
 * when q_start is a multiple of 64. */
typedef struct {
  int B, L, d_rope, n_kv, d_nope, d_v, n_noise, g;
  gdla_mask mask;
  int window;
  float softmax_scale;       /* <= 0 selects 1/sqrt(d_nope + d_rope) */
  gdla_dtype dtype;
  int rope_max_pos;          /* >= L */
  const void* q;             /* [B, L, n_signal+n_noise, d_nope+d_rope] */
  const void* kv;            /* [B, L, n_kv, d_nope+d_v] */
  const void* k_rope_rot;    /* [B, L, d_rope] rotated */
  const float* rope_cos;     /* [rope_max_pos, d_rope/2] */
  const float* rope_sin;
  const float* lam_logits;   /* [B, L, n_signal] fp32 */
  const void* gate_logits;   /* [B, L, n_signal, d_v] */
  void* out;                 /* [B, L, n_signal, d_v] */
  void* workspace;           /* status word */
  size_t workspace_bytes;
  int q_len;                 /* query rows per sequence; 0 = L (see above) */
  int q_start;               /* position of the first query row */
} gdla_attend_args;

gdla_status gdla_attend(const gdla_attend_args* args, void* stream);

/* ------------------------------------------------------- prefill, host buffers
 * The forward of gdla_prefill for activations held in host memory (the report
 * has no counterpart; the arithmetic is gdla_prefill's, row for row). The layer's
 * parameters stay on the GPU: gamma, w_ukv, rope_cos, rope_sin, and the optional
 * cache_c_hat / cache_k_rope outputs are DEVICE pointers as in gdla_prefill. The
 * activations are HOST pointers, in gdla_prefill's layouts:
 *   inputs  c_kv, k_rope, q, lam_logits, gate_logits
 *   output  out
 * Page-locked host memory (cudaHostAlloc / cudaHostRegister) lets the copies
 * overlap the kernels; pageable memory gives the same result without the overlap.
 *
 * The call first copies the latent inputs (c_kv, k_rope) of the whole batch
 * and expands every token, as gdla_prefill does. Then every sequence's queries
 * are cut into chunks of `chunk_tokens` tokens (<= 0 selects 2048; the last
 * chunk of a sequence may be shorter). Each chunk's q, lambda and gate rows are
 * copied to the device on a copy stream, attended (the query-block form of
 * gdla_attend) on `stream`, and its rows of Y are copied back on a second copy
 * stream, so the transfers of one chunk overlap the kernels of its neighbours.
 * Chunks go latest positions first: under the causal mask they see the most
 * keys, so the cheapest chunks come last, after the final host-to-device copy.
 * The topmost chunk of a sequence is cut at its half and three-quarter marks
 * (rounded down to 64 tokens), so the first copy, which no kernel overlaps, is
 * a quarter chunk. The chunks' attention alternates over two internal compute
 * streams. With chunks of a multiple of 64 tokens the result is bit-identical
 * to gdla_prefill's.
 *
 * The device workspace (>= gdla_prefill_host_workspace_size(args,
 * chunk_tokens) bytes, 256-byte aligned) holds gdla_prefill's workspace, device
 * copies of c_kv and k_rope, and eight chunk-sized staging slots per query-side
 * tensor (q, lambda, gate, Y) that the chunks take in turn.
 *
 * The call uses two non-blocking copy streams, two compute streams and a few
 * events of its own. They are created by the first call on a device and kept by
 * the library for later calls (a call that overlaps another one on the host gets
 * a set of its own); nothing is created per call after that. All work is ordered after
 * earlier work on `stream`, and later work on `stream` waits for all of it.
 * Like every entry point, the call returns without synchronising, so `out` is
 * valid only after `stream` has been synchronised, and the host inputs must
 * stay unchanged until then. Errors as for gdla_prefill. A CUDA failure after
 * the first copy was enqueued still joins the copy streams into `stream`
 * before GDLA_ERR_CUDA is returned. */
size_t gdla_prefill_host_workspace_size(const gdla_prefill_args* args, int chunk_tokens);
gdla_status gdla_prefill_host(const gdla_prefill_args* args, int chunk_tokens, void* stream);

/* --------------------------------------------------------------------- decode
 * One new token per sequence over the compact latent cache ("Motif 3:
 * Technical Report", Architecture: GDLA "preserves MLA's compact inference
 * state"). The cache holds, per token, the normalised latent c_hat (d_c) and
 * the rotated rotary key (d_rope). The query of sequence b sits at position
 * seqlens[b]-1 and sees cache tokens 0..seqlens[b]-1 (or the last `window` of
 * them under GDLA_MASK_SLIDING). The library evaluates the same attention as
 * prefill with W_UK absorbed into the query and W_UV applied after the
 * weighted sum of latents, which is equal in exact arithmetic. */
typedef struct {
  int B, T_max, d_c, d_rope, n_kv, d_nope, d_v, n_noise, g;
  gdla_mask mask;
  int window;
  float softmax_scale;       /* <= 0 selects 1/sqrt(d_nope + d_rope) */
  gdla_dtype dtype;
  int rope_max_pos;          /* rows of the RoPE tables; must be >= T_max (the query position is at most T_max - 1) */
  const int* seqlens;        /* [B] int32 on the device, 1 <= seqlens[b] <= T_max. The host cannot check
                                them: a value outside the range is clamped into it by the kernels (every
                                access stays inside the cache and the tables) and reported as
                                GDLA_ERR_INVALID_ARG in the workspace status word (gdla_workspace_status) */
  const void* c_cache;       /* [B, T_max, d_c] normalised latent */
  const void* kr_cache;      /* [B, T_max, d_rope] rotated rotary key */
  const void* q;             /* [B, n_signal+n_noise, d_nope+d_rope], rotary part pre-RoPE */
  const void* w_ukv;         /* [d_c, n_kv*(d_nope+d_v)] */
  const float* rope_cos;     /* [rope_max_pos, d_rope/2] */
  const float* rope_sin;
  const float* lam_logits;   /* [B, n_signal] fp32 */
  const void* gate_logits;   /* [B, n_signal, d_v] */
  void* out;                 /* [B, n_signal, d_v] */
  void* workspace;           /* >= gdla_decode_workspace_size(args) bytes */
  size_t workspace_bytes;
} gdla_decode_args;

size_t gdla_decode_workspace_size(const gdla_decode_args* args);
gdla_status gdla_decode(const gdla_decode_args* args, void* stream);

/* ---------------------------------------------------------- decode, no alloc
 * Not part of the layer itself (the report has no counterpart): the same
 * decode as gdla_decode for callers that cannot provide a workspace -- code
 * that must not allocate device memory while it runs, such as a step replayed
 * from a captured CUDA graph, a latency-bound serving loop, or a plugin that
 * only receives its inputs and outputs. The scratch comes from a fixed array
 * inside the library instead of args->workspace (which is ignored):
 *  - size: GDLA_DECODE_NOALLOC_SCRATCH_BYTES (32 MiB), held on every GPU that
 *    loads the library until the process exits. A call whose
 *    gdla_decode_workspace_size() exceeds it returns GDLA_ERR_SCRATCH_LIMIT
 *    before launching anything (e.g. B=16 sequences of 4096 tokens fit,
 *    B=64 sequences of 32768 tokens do not);
 *  - the first call on a device looks up the array's device address (with that
 *    device current) and caches it: make that first call before any stream
 *    capture;
 *  - every call on a device shares the one array and leaves the previous
 *    call's data in it (the status word is cleared by each call): calls that
 *    can overlap on the GPU, from any stream or thread, race and must be
 *    serialised by the caller;
 *  - it allocates and frees nothing; errors as for gdla_decode, and
 *    gdla_workspace_status cannot be used on it. */
#define GDLA_DECODE_NOALLOC_SCRATCH_BYTES (32u << 20)
gdla_status gdla_decode_noalloc(const gdla_decode_args* args, void* stream);

/* ---------------------------------------------------------------------- gates
 * The per-token inputs of the differential epilogue, computed from the layer's
 * activations ("Motif 3: Technical Report", section "Architecture": lambda_t =
 * sigmoid(x_t W_lambda), and the output gate is computed from the normalised query
 * latent). The sigmoids stay in the attention epilogue: this call produces the
 * logits that gdla_prefill, gdla_prefill_host, gdla_attend and gdla_decode take.
 *   c_hat_q[t]     = gamma_q (.) c_q[t] / sqrt(mean(c_q[t]^2) + rms_eps)
 *   gate_logits[t] = c_hat_q[t] @ W_G       ([n_signal * d_v], in `dtype`)
 *   lam_logits[t]  = x[t] @ W_lambda        ([n_signal], fp32)
 * for the B*L tokens (a decode step: L = 1). Either half may be skipped:
 *  - c_q == NULL skips the gate (gamma_q, w_g and gate_logits are then ignored);
 *  - x == NULL skips lambda (w_lambda and lam_logits are then ignored).
 * The normalisation is the latent RMSNorm of gdla_latent_expand with its own gain.
 * Both products run on the tensor cores for bf16 when their widths (d_q, d_x,
 * n_signal*d_v, n_signal) are multiples of 8 (the report's shapes: d_q = 1536,
 * n_signal*d_v = 4096 or 6144, n_signal = 32 or 48), lambda with fp32 output, and
 * on the CUDA cores otherwise.
 * The workspace (>= gdla_gates_workspace_size(args) bytes, 256-byte aligned) holds
 * the status word and, when the gate is computed, c_hat_q [B*L, d_q]. */
typedef struct {
  int B, L;                  /* tokens = B * L */
  int d_q, d_x, n_signal, d_v;
  gdla_dtype dtype;          /* element type of c_q, gamma_q, w_g, x, w_lambda and gate_logits */
  float rms_eps;             /* <= 0 selects 1e-6 */
  const void* c_q;           /* [B, L, d_q] query latent before normalisation, or NULL */
  const void* gamma_q;       /* [d_q] its RMSNorm gain */
  const void* w_g;           /* [d_q, n_signal * d_v] */
  const void* x;             /* [B, L, d_x] layer input, or NULL */
  const void* w_lambda;      /* [d_x, n_signal] */
  void* gate_logits;         /* [B, L, n_signal, d_v] (out) */
  float* lam_logits;         /* [B, L, n_signal] fp32 (out) */
  void* workspace;
  size_t workspace_bytes;
} gdla_gates_args;

size_t gdla_gates_workspace_size(const gdla_gates_args* args);
gdla_status gdla_gates(const gdla_gates_args* args, void* stream);

/* --------------------------------------------------------------- RoPE tables
 * The cos/sin tables every entry point takes (rope_cos, rope_sin), built on the
 * host in double precision and rounded to fp32: model set-up, like loading the
 * weights (copy them to the device once). Both write [max_pos, d_rope/2] row-major
 * into caller-owned HOST arrays; entry (m, k) is cos / sin of m * theta_k.
 *
 * gdla_rope_tables: plain RoPE ("Open-Source Frontier Models: Architecture and
 * Benchmarks of Rnj-1 and Motif-2", section 2, the rotation-matrix equation),
 * theta_k = base^(-2k/d_rope), the pair (k, k + d_rope/2) rotated together.
 *
 * gdla_yarn_rope_tables: YaRN context extension (same section, the three-regime
 * Scale(i) equation) of a model trained on original_max_pos tokens by `factor`:
 * with the wavelength lambda_k = 2 pi / theta_k, a frequency is kept below
 * original_max_pos / beta_fast, divided by `factor` above original_max_pos /
 * beta_slow, and multiplied by (1 - a) + a / factor in between, where a grows
 * linearly with the wavelength from 0 to 1 across that band (the report's full
 * layers use factor 64 from 4K). Pair the tables with
 * softmax_scale = gdla_yarn_mscale(factor)^2 / sqrt(d_nope + d_rope).
 *
 * gdla_yarn_mscale: YaRN's temperature 1 + 0.1 ln(factor) (1 for factor <= 1),
 * the factor by which that section's listing scales both rotated vectors, so the
 * logits grow by its square.
 *
 * Errors: GDLA_ERR_INVALID_ARG for NULL arrays, max_pos < 1, d_rope odd, < 2 or
 * above 1024, base <= 1, factor <= 0, original_max_pos < 1 or a beta <= 0;
 * nothing is written then. */
gdla_status gdla_rope_tables(int max_pos, int d_rope, double base, float* cos_tab, float* sin_tab);
gdla_status gdla_yarn_rope_tables(int max_pos, int d_rope, double base, double factor, int original_max_pos,
                                  double beta_fast, double beta_slow, float* cos_tab, float* sin_tab);
double gdla_yarn_mscale(double factor);

/* ---------------------------------------------------------------- utilities */
const char* gdla_status_string(gdla_status s);

/* Reads (synchronously on `stream`) the device status word at the start of a
 * prefill or decode workspace: GDLA_OK, or GDLA_ERR_TIMEOUT if a device-side
 * wait of the last call hit its cap. The word is cleared by every call. */
gdla_status gdla_workspace_status(const void* workspace, void* stream);

/* Diagnostic (the report has no counterpart): launches one CTA whose device-side
 * wait can never complete (an mbarrier that nothing arrives on). The wait gives
 * up after its limit, the same ~1 s bound every wait in the kernels has, and
 * records GDLA_ERR_TIMEOUT in the status word at `status_word` (a 256-byte,
 * 256-aligned device buffer owned by the caller, cleared here first), so that a
 * caller can check, without faulting the GPU, that a stalled kernel ends and is
 * reported through gdla_workspace_status. Returns GDLA_ERR_INVALID_ARG for a NULL
 * or misaligned buffer, GDLA_ERR_CUDA if the launch fails, else GDLA_OK; the
 * kernel runs asynchronously on `stream`. */
gdla_status gdla_diag_wait_timeout(void* status_word, void* stream);

/* Build information, for checks that the native library is the one loaded. */
const char* gdla_build_info(void);

#ifdef __cplusplus
}
#endif
#endif /* GDLA_H_ */
