/*
 * gptoss.h -- C ABI of libgptoss_attn, the GPT-OSS attention core for
 * NVIDIA B200 (sm_100a).
 *
 * What the library computes (sources by page title and section):
 *   - YaRN rotary embedding of q and k: NeMo AutoModel
 *     "nemo_automodel.components.models.gpt_oss.rope_utils", class
 *     RotaryEmbedding (head_dim, base, initial_context_length, scaling_factor,
 *     ntk_alpha, ntk_beta, partial_rotary_factor) and its method
 *     _compute_concentration_and_inv_freq (YaRN paper, arXiv 2309.00071);
 *     apply_rotary_emb / apply_rotary_emb_qk (half-split pairs, tables with
 *     the concentration applied, BSHD or packed THD with cu_seqlens,
 *     arbitrary strides, independently allocated outputs).
 *   - Grouped-query causal softmax attention with a learned per-head sink
 *     logit that adds exp(sink) to the softmax denominator only, full context
 *     or a sliding window: NeMo AutoModel
 *     "nemo_automodel.components.models.gpt_oss.layers", GptOssAttention
 *     (sinks, sliding_window, softmax_scale = head_dim ** -0.5,
 *     num_attention_heads, num_key_value_heads, _has_thd_metadata);
 *     Transformers v4.55.0 release notes, "Architecture".
 *
 * Definitions used by every entry point (token i of a sequence, q-head h,
 * kv-head g = h / (Hq / Hkv)):
 *   theta(p, j) = p * inv_freq[j], j in [0, D/2), inv_freq from YaRN;
 *   x'[j]       = c * (x[j] cos theta - x[j+D/2] sin theta)
 *   x'[j+D/2]   = c * (x[j+D/2] cos theta + x[j] sin theta),  c = concentration;
 *   s_ij  = softmax_scale * <q'_i[h], k'_j[g]>;
 *   key j visible from query i iff j <= i (token order inside the sequence)
 *         and (window == 0 or i - j < window);
 *   M_i   = max(sink_h, max_visible s_ij);
 *   Z_i   = exp(sink_h - M_i) + sum_visible exp(s_ij - M_i);
 *   out_i = sum_visible exp(s_ij - M_i) v_j[g] / Z_i;   lse_i = M_i + ln Z_i.
 * sink_h = -inf gives standard softmax attention.  Positions feed RoPE only.
 *
 * Conventions:
 *   - Every tensor pointer is caller-owned DEVICE memory.  The library
 *     allocates nothing; its only state is the wait limit below.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronises.
 *   - Arguments are validated on the host before any launch; a failed check
 *     returns GPTOSS_ERR_INVALID_ARG or GPTOSS_ERR_UNSUPPORTED and launches
 *     nothing.  A failed launch returns GPTOSS_ERR_CUDA.
 *   - Device-side conditions (a bounded pipeline wait that gave up, a block
 *     index outside a paged pool) are recorded in a device status word read
 *     by gptoss_read_device_status.
 *   - bf16 tensors are IEEE bfloat16; head_dim D is 64 (128 where an entry
 *     says so) and contiguous (element stride 1); rotary_dim: see
 *     gptoss_rope_params.
 *   - No C++ exception crosses this ABI.
 */
#ifndef GPTOSS_H_
#define GPTOSS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t == struct CUstream_st* */

typedef enum gptoss_status {
  GPTOSS_OK = 0,
  GPTOSS_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad stride or alignment */
  GPTOSS_ERR_UNSUPPORTED = 2, /* valid request this build does not implement (D != 64, ...) */
  GPTOSS_ERR_CUDA = 3,        /* a CUDA runtime call or a kernel launch failed */
  GPTOSS_ERR_TIMEOUT = 4      /* a device-side bounded wait gave up (device status word) */
} gptoss_status;

/* YaRN parameters, as RotaryEmbedding on the rope_utils page names them.
 * factor <= 1 means plain RoPE (inv_freq = base^(-2j/rotary_dim), c = 1).
 * Otherwise c = 0.1 ln(factor) + 1 and pair j is kept (j <= d_lo), divided by
 * factor (j >= d_hi) or blended linearly in j between the two correction
 * dimensions d_lo / d_hi at which a pair makes ntk_beta / ntk_alpha turns
 * over initial_context tokens. */
typedef struct gptoss_rope_params {
  double base;             /* 150000 for GPT-OSS */
  double factor;           /* scaling_factor, 32 for GPT-OSS */
  int32_t initial_context; /* initial_context_length, 4096 */
  int32_t rotary_dim;      /* int(head_dim * partial_rotary_factor): features [0, rotary_dim)
                              rotate in pairs (j, j + rotary_dim/2), the rest pass through
                              unchanged; even, at most D.  gptoss_rope_qk, the decodes, the
                              append, gptoss_attn_bwd, gptoss_attn_fwd at D = 64 and its block
                              form take any multiple of 16 (partial rotary); gptoss_attn_fwd at
                              D = 128 and gptoss_qkv_rope need rotary_dim == D (else
                              UNSUPPORTED) */
  double ntk_alpha;        /* 1 */
  double ntk_beta;         /* 32 */
} gptoss_rope_params;

/* Strides in ELEMENTS.  BSHD element (b, s, h, d) sits at
 * b*batch + s*tok + h*head + d; packed THD element (t, h, d) at
 * t*tok + h*head + d (batch ignored).  tok and head must be multiples of 8
 * (16 bytes) and every base pointer 16-byte aligned. */
typedef struct gptoss_strides {
  int64_t batch;
  int64_t tok;
  int64_t head;
} gptoss_strides;

/* Human-readable name of a status code (static string, never NULL). */
const char* gptoss_status_string(gptoss_status status);

/* gptoss_rope_qk -- YaRN RoPE of q and k, out of place (in place when an
 * output aliases its input with the same strides).
 *   q      [B,S,Hq,D] (BSHD) or [T,Hq,D] (THD) bf16, strides sq; k likewise
 *          with Hkv heads, strides sk.
 *   q_out, k_out: bf16, same logical shapes, own strides (k_out may point
 *          into a KV cache slot: that is the cache-append use).
 *   positions  int32 [B*S] (row-major over b, s) or [T]; NULL -> 0..S-1 per
 *          batch row (BSHD) or restarting at 0 for every sequence (THD).
 *   cu_seqlens int32 [nseq+1], nondecreasing, cu_seqlens[0] = 0,
 *          cu_seqlens[nseq] = T; NULL -> BSHD.  With cu_seqlens, B = nseq and
 *          S_or_T = T; otherwise S_or_T = S.
 *   Angles are reduced in double precision and rotated in fp32; outputs are
 *   rounded to bf16. */
gptoss_status gptoss_rope_qk(const void* q, gptoss_strides sq, const void* k, gptoss_strides sk,
                             void* q_out, gptoss_strides sq_out, void* k_out, gptoss_strides sk_out,
                             const int32_t* positions, const int32_t* cu_seqlens, int32_t B,
                             int32_t S_or_T, int32_t Hq, int32_t Hkv, int32_t D,
                             const gptoss_rope_params* rope, struct CUstream_st* stream);

/* gptoss_attn_fwd -- prefill sink attention, causal, full (window = 0) or
 * sliding window, BSHD or packed THD.
 *   q [B,S,Hq,D] / [T,Hq,D], k and v [B,S,Hkv,D] / [T,Hkv,D], bf16, own
 *          strides.  rope != NULL: q and k are raw; q is rotated inside the
 *          attention kernel as its tiles are loaded, k once beforehand (see
 *          workspace); rope == NULL: q and k are already rotated.  Both
 *          products take fp16 operands (rotated q and k for QK^T; the
 *          unnormalised probabilities and v for P V), so the rotated q and k
 *          (c * |x|) and v must stay below 65504 in magnitude.
 *   sinks  fp32 [Hq], in the units of the scaled logits (may be -inf).
 *   positions / cu_seqlens as for gptoss_rope_qk (positions only used when
 *          rope != NULL).
 *   B      batch (BSHD) or number of sequences (THD).
 *   S      sequence length (BSHD) or the longest sequence (THD, upper bound).
 *   total_tokens  B*S (BSHD) or T (THD).
 *   window 0 = full causal; w > 0 = the last w keys including the query.
 *   softmax_scale  head_dim^-0.5 for GPT-OSS.
 *   out    bf16, q's logical shape, strides so.
 *   lse    fp32, nullable: [B,Hq,S] (BSHD) or [Hq,T] (THD), natural log.
*   workspace  device memory of at least
 *          gptoss_attn_fwd_workspace_size(total_tokens, Hkv, D) bytes, 16-byte
 *          aligned, owned by the caller, contents need not be initialised.
 *          A first kernel on the same stream writes into it k (rotated when
 *          rope != NULL) and v as dense fp16, and every token's 32 RoPE
 *          angles (c cos, c sin), which the attention kernel reads for q.
 *          NULL, too small or misaligned is GPTOSS_ERR_INVALID_ARG. */
gptoss_status gptoss_attn_fwd(const void* q, gptoss_strides sq, const void* k, gptoss_strides sk,
                              const void* v, gptoss_strides sv, const float* sinks,
                              const int32_t* positions, const int32_t* cu_seqlens, int32_t B,
                              int32_t S, int32_t total_tokens, int32_t Hq, int32_t Hkv, int32_t D,
                              int32_t window, float softmax_scale, const gptoss_rope_params* rope,
                              void* out, gptoss_strides so, float* lse, void* workspace,
                              size_t workspace_bytes, struct CUstream_st* stream);

/* Workspace bytes for gptoss_attn_fwd: k and v as fp16 (total_tokens x Hkv x
 * D values each, each rounded up to 256 bytes) and the angle table
 * (total_tokens x 32 fp32 pairs).  0 when a size is out of range. */
size_t gptoss_attn_fwd_workspace_size(int32_t total_tokens, int32_t Hkv, int32_t D);

/* gptoss_attn_fwd_block -- one key block of a query shard, for context
 * parallelism of the full-context layers (apply_rotary_emb_qk's cp_size /
 * cp_rank on the rope_utils page): the prefill over queries at global token
 * indices [q_start, q_start + Sq) against the keys at [k_start, k_start + Sk)
 * of the same sequences, causal on the global indices (key j visible from
 * query i iff k_start + j <= q_start + i), with NO sink.  Each row's output is
 * normalised over the block's visible keys and lse is their log-sum-exp;
 * gptoss_attn_merge folds the blocks and the sink together.
 *   q [B,Sq,Hq,D], k and v [B,Sk,Hkv,D], bf16, BSHD strides (raw: rope !=
 *          NULL rotates them at their global positions q_start + i and
 *          k_start + j; rope == NULL takes them as rotated).  Both products
 *          take fp16 operands, as in gptoss_attn_fwd.
 *   k_start <= q_start (a block after the shard is invisible; skip it), so
 *          every query row sees at least one key of the block.
 *   out    fp32, dense [B,Sq,Hq,D] (kept in fp32 for the merge).
 *   lse    fp32, dense [B,Hq,Sq], natural log, no sink.
 *   workspace  device memory of gptoss_attn_fwd_block_workspace_size(B, Sq,
 *          Sk, Hkv, D) bytes, 16-byte aligned (fp16 k and v of the block,
 *          the queries' angle table); contents need not be initialised.
 *   k_start > q_start or a bad size, pointer or stride: INVALID_ARG. */
gptoss_status gptoss_attn_fwd_block(const void* q, gptoss_strides sq, const void* k, gptoss_strides sk,
                                    const void* v, gptoss_strides sv, int32_t B, int32_t Sq, int32_t Sk,
                                    int32_t q_start, int32_t k_start, int32_t Hq, int32_t Hkv, int32_t D,
                                    float softmax_scale, const gptoss_rope_params* rope, float* out, float* lse,
                                    void* workspace, size_t workspace_bytes, struct CUstream_st* stream);

/* Workspace bytes for gptoss_attn_fwd_block (0 when a size is out of range). */
size_t gptoss_attn_fwd_block_workspace_size(int32_t B, int32_t Sq, int32_t Sk, int32_t Hkv, int32_t D);

/* gptoss_attn_merge -- the sink attention over the union of n_blocks key
 * blocks from their gptoss_attn_fwd_block results (same query rows):
 *   Z = exp(sink_h) + sum_b exp(lse_b),  out = sum_b exp(lse_b) out_b / Z,
 *   lse = log Z; the sink enters once, here (sinks NULL: no sink).
 *   outs   fp32 [n_blocks][B][S][Hq][D] dense (16-byte aligned).
 *   lses   fp32 [n_blocks][B][Hq][S]; a block a row sees no key of has -inf.
 *   out    bf16 [B,S,Hq,D] with BSHD strides so (8-byte aligned); lse
 *          nullable fp32 [B,Hq,S]. */
gptoss_status gptoss_attn_merge(const float* outs, const float* lses, int32_t n_blocks, const float* sinks,
                                int32_t B, int32_t S, int32_t Hq, int32_t D, void* out, gptoss_strides so,
                                float* lse, struct CUstream_st* stream);

/* Workspace bytes for gptoss_qkv_rope: every token's D/2 RoPE angles
 * (fp32 (c cos, c sin) pairs), plus 16.  0 when a size is out of range. */
size_t gptoss_qkv_rope_workspace_size(int32_t total_tokens, int32_t D);

/* gptoss_qkv_rope -- the q, k, v projections of the attention input with
 * RoPE fused into the GEMM epilogue.  GptOssAttention's q_proj, k_proj and
 * v_proj are Linear layers with bias (blog page "gpt-oss-20b 模型结构":
 * 2880 -> 4096 / 512 / 512; y = x W^T + b); q and k, viewed as
 * [token, head, D], are then rotated by the YaRN RoPE of the NeMo AutoModel
 * gpt_oss.rope_utils page (apply_rotary_emb_qk, half-split pairs).
 *   x          bf16 [T, hidden] rows of x_row_stride elements (T = B*S for
 *              BSHD, S_or_T packed tokens with cu_seqlens); hidden % 8 == 0.
 *   w_qkv      bf16 [(Hq + 2 Hkv) D, hidden], row-major: the q_proj rows,
 *              then k_proj's, then v_proj's (caller-owned, read only).
 *   b_qkv      bf16 [(Hq + 2 Hkv) D] in the same order; NULL: no bias.
 *   positions, cu_seqlens, B, S_or_T: as gptoss_rope_qk (token positions).
 *   rope       NULL: no rotation; else rotary_dim == D (full rotary;
 *              GPTOSS_ERR_UNSUPPORTED otherwise).
 *   q_out [.., Hq, D], k_out / v_out [.., Hkv, D]: bf16 with strides (D
 *              contiguous, 16-byte aligned rows), BSHD or THD like x.
 *   workspace  device, >= gptoss_qkv_rope_workspace_size(T, D) bytes when
 *              rope != NULL (the angle table); else unused.
 * D is 64 or 128 and hidden a multiple of 8 (GPTOSS_ERR_UNSUPPORTED
 * otherwise).  Products accumulate in fp32 on the
 * tensor cores; bias and rotation in fp32; outputs rounded to bf16.  Two
 * launches (angle table, GEMM), asynchronous on `stream`. */
gptoss_status gptoss_qkv_rope(const void* x, int64_t x_row_stride, const void* w_qkv, const void* b_qkv,
                              const int32_t* positions, const int32_t* cu_seqlens, int32_t B, int32_t S_or_T,
                              int32_t hidden, int32_t Hq, int32_t Hkv, int32_t D, const gptoss_rope_params* rope,
                              void* q_out, gptoss_strides sq, void* k_out, gptoss_strides sk, void* v_out,
                              gptoss_strides sv, void* workspace, size_t workspace_bytes,
                              struct CUstream_st* stream);

/* Workspace bytes gptoss_attn_bwd needs: q and k rotated once (fp16), every
 * token's 32 RoPE angles, <dout, out> and lse log2(e) per row and head (fp32),
 * and fp32 dk / dv accumulators for split sweeps.  0 when a size is out of
 * range. */
size_t gptoss_attn_bwd_workspace_size(int32_t total_tokens, int32_t Hq, int32_t Hkv, int32_t D);

/* gptoss_attn_bwd -- gradients of gptoss_attn_fwd for L = sum(dout * out):
 * the derivative of the sink attention (GptOssAttention on the NeMo
 * AutoModel gpt_oss.layers page, with RoPE of the gpt_oss.rope_utils page;
 * the pages define the forward and train with it) by the chain rule:
 *   D_i = <dout_i, out_i>, dS_ij = P_ij (<dout_i, v_j> - D_i) over the
 *   visible pairs, dv_j = sum_i P_ij dout_i, dq'_i = scale sum_j dS_ij k'_j,
 *   dk'_j = scale sum_i dS_ij q'_i, dsink_h = -sum_i exp(sink_h - lse_i) D_i
 *   (summed over every row of every sequence), and through RoPE
 *   dq = c R(theta)^T dq', dk = c R(theta)^T dk'.
 *   q, k, v, sinks, positions, cu_seqlens, B, S, total_tokens, Hq, Hkv, D,
 *          window, softmax_scale, rope: exactly as given to gptoss_attn_fwd
 *          (q and k raw with rope != NULL, already rotated with rope == NULL).
 *   out, dout  bf16, q's logical shape, own strides: the forward's output
 *          and the gradient arriving at it.
 *   lse    fp32 from the same forward call: [B,Hq,S] (BSHD) / [Hq,T] (THD).
 *   dq     [B,S,Hq,D] / [T,Hq,D] bf16 contiguous (written).
 *   dk, dv [B,S,Hkv,D] / [T,Hkv,D] bf16 contiguous (written; the sums over
 *          the query heads of each kv group).
 *   dsinks fp32 [Hq] (written, not accumulated into; zero when there are no
 *          rows).
 *   workspace  device memory of gptoss_attn_bwd_workspace_size(total_tokens,
 *          Hq, Hkv, D) bytes, 16-byte aligned, owned by the caller, contents
 *          need not be initialised.
 * Kernels on `stream`: q / k rotation; D and dsinks; dk / dv on the tcgen05
 * tensor cores (one CTA per 128-key tile and kv head; sweeps longer than 192
 * (head, 64-query tile) steps split into chunks that add into fp32
 * accumulators, then one finishing kernel); dq (one CTA per query tile and
 * head: tcgen05 for full context or windows of 1024+ keys, warp-level
 * mma.sync for shorter windows).  The rotated q / k enter the products as
 * fp16 like the forward's; P is rounded to bf16 and dS to fp16 for the
 * products, accumulation is fp32.  dsinks and split dk / dv are summed with
 * floating-point atomics (order not fixed); every other output element has
 * one writer. */
gptoss_status gptoss_attn_bwd(const void* q, gptoss_strides sq, const void* k, gptoss_strides sk,
                              const void* v, gptoss_strides sv, const void* out, gptoss_strides so,
                              const void* dout, gptoss_strides sdo, const float* lse, const float* sinks,
                              const int32_t* positions, const int32_t* cu_seqlens, int32_t B, int32_t S,
                              int32_t total_tokens, int32_t Hq, int32_t Hkv, int32_t D, int32_t window,
                              float softmax_scale, const gptoss_rope_params* rope, void* dq, void* dk,
                              void* dv, float* dsinks, void* workspace, size_t workspace_bytes,
                              struct CUstream_st* stream);

/* Workspace bytes gptoss_attn_decode needs for these sizes (split-KV
 * partial results).  0 when a size is out of range. */
size_t gptoss_attn_decode_workspace_size(int32_t B, int32_t Lmax, int32_t Hq, int32_t Hkv, int32_t D);

/* gptoss_attn_decode -- one new query token per sequence against a bf16 KV
 * cache, split over the cache length, merged with the sink folded once.
 *   q        [B,Hq,D] bf16 contiguous, raw: rotated here at position
 *            cache_seqlens[b]-1 when rope != NULL.
 *   k_cache, v_cache [B,Lmax,Hkv,D] bf16 contiguous; k_cache holds keys
 *            already rotated, v_cache raw values; the new token's k/v are
 *            already in slot cache_seqlens[b]-1.
 *   cache_seqlens int32 [B], 1 <= len <= Lmax (device memory).
 *   The query sees slots [len-window, len) (all of [0, len) when window = 0);
 *   slots past len are never read into the result and may hold anything.
 *   out      [B,Hq,D] bf16 contiguous; lse fp32 [B,Hq], nullable.
 *   workspace  device memory of at least
 *            gptoss_attn_decode_workspace_size(...) bytes, 16-byte aligned,
 *            owned by the caller; contents need not be initialised. */
gptoss_status gptoss_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* cache_seqlens, const float* sinks, int32_t B,
                                 int32_t Lmax, int32_t Hq, int32_t Hkv, int32_t D, int32_t window,
                                 float softmax_scale, const gptoss_rope_params* rope, void* out,
                                 float* lse, void* workspace, size_t workspace_bytes,
                                 struct CUstream_st* stream);

/* gptoss_attn_decode_paged -- gptoss_attn_decode over a paged KV cache.  The
 * pages describe generation with a key/value cache (Transformers v4.55.0
 * release notes, the model.generate examples and the cache entries of the
 * change list) but give no layout; this one is a block table over a pool of
 * fixed-size blocks.
 *   k_pool, v_pool [num_blocks, block_size, Hkv, D] bf16 contiguous; k_pool
 *            holds rotated keys, v_pool raw values.
 *   block_table int32 [B, max_blocks] (device memory): token p of sequence b
 *            is row p % block_size of block block_table[b * max_blocks +
 *            p / block_size].  A block index outside [0, num_blocks) reads as
 *            zeros (it never faults).
 *   block_size a multiple of 64 (whole 64-key tiles per block);
 *            num_blocks * block_size and max_blocks * block_size < 2^31.
 *   q_len    query tokens per sequence (>= 1; B * q_len <= 65535): several
 *            new tokens decoded in one call, as when draft tokens are
 *            verified.  q [B, q_len, Hq, D] (rotated by the caller, or by
 *            `rope` at positions cache_seqlens[b] - q_len + i), out
 *            [B, q_len, Hq, D], lse [B, q_len, Hq].  Token i of sequence b
 *            attends to the first cache_seqlens[b] - (q_len - 1 - i) cache
 *            rows (causal among the new tokens, which the cache must already
 *            hold); a sequence needs cache_seqlens[b] >= q_len.  The new
 *            tokens of a sequence share one pass over its cache (up to
 *            32 / (Hq / Hkv) tokens per pass: 4 at Hq / Hkv = 8).
 *   The other arguments as for gptoss_attn_decode with Lmax = max_blocks *
 *   block_size (workspace: gptoss_attn_decode_workspace_size(B * q_len,
 *   max_blocks * block_size, Hq, Hkv, D) bytes). */
gptoss_status gptoss_attn_decode_paged(const void* q, const void* k_pool, const void* v_pool,
                                       const int32_t* block_table, int32_t max_blocks, int32_t block_size,
                                       int32_t num_blocks, const int32_t* cache_seqlens, const float* sinks,
                                       int32_t B, int32_t q_len, int32_t Hq, int32_t Hkv, int32_t D,
                                       int32_t window, float softmax_scale, const gptoss_rope_params* rope,
                                       void* out, float* lse, void* workspace, size_t workspace_bytes,
                                       struct CUstream_st* stream);

/* gptoss_kv_append_paged -- writes each sequence's q_len new tokens into a
 * paged cache: the key of token i rotated at position cache_seqlens[b] -
 * q_len + i (RoPE as for gptoss_rope_qk, rounded to bf16; the cache holds
 * post-RoPE keys) and the values as given.  Run it before
 * gptoss_attn_decode_paged on the same stream.
 *   k_new, v_new [B, q_len, Hkv, D] bf16 contiguous (raw keys).
 *   q_len    new tokens per sequence (1 .. 65535).
 *   cache_seqlens int32 [B] (device memory), the new tokens included
 *            (>= q_len).
 *   block_table, max_blocks, block_size, k_pool, v_pool, num_blocks as for
 *            gptoss_attn_decode_paged.  A sequence whose block index is
 *            outside [0, num_blocks) is not written and the device status
 *            word records GPTOSS_ERR_INVALID_ARG.
 *   rope     NULL stores the key unrotated. */
gptoss_status gptoss_kv_append_paged(const void* k_new, const void* v_new, const int32_t* cache_seqlens,
                                     const int32_t* block_table, int32_t max_blocks, int32_t block_size,
                                     void* k_pool, void* v_pool, int32_t num_blocks, int32_t B, int32_t q_len,
                                     int32_t Hkv, int32_t D, const gptoss_rope_params* rope,
                                     struct CUstream_st* stream);

/* gptoss_attn_decode_noalloc -- gptoss_attn_decode for callers that cannot
 * allocate device memory when they decode (a serving loop whose memory is
 * planned once up front and must not call cudaMalloc, which may synchronise
 * the device or fail under memory pressure; a runtime whose device memory
 * comes only from its own fixed pools).  The pages have no counterpart: this
 * is a packaging variant of the decode entry point, same arguments minus the
 * workspace, same results.
 *   The split-KV partials go to one file-scope device array of 16 MiB that
 *   every GPU loading this library holds until the process exits.  Sizes
 *   whose gptoss_attn_decode_workspace_size(B, Lmax, Hq, Hkv, D) exceeds
 *   16 MiB are rejected with GPTOSS_ERR_UNSUPPORTED (B=64 x 32768 needs
 *   8.7 MB, B=8 x 131072 needs 5.0 MB).
 *   The array's device address belongs to a CUDA context: the first call in
 *   each context (the current one when the call is made) looks it up with
 *   cudaGetSymbolAddress and remembers it under the context's unique id, so a
 *   device reset or another driver context gets its own lookup, never a
 *   stale address.  Make that first call before any stream capture.  Nothing
 *   in the array needs to start at zero: each call writes every partial it
 *   later reads.
 *   All calls share the one array, which keeps the last call's contents:
 *   calls whose executions overlap on the GPU (other streams, other host
 *   threads) race and must be serialised by the caller.
 *   Allocates nothing: no cudaMalloc, no cudaFree, no allocating library. */
gptoss_status gptoss_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* cache_seqlens, const float* sinks, int32_t B,
                                         int32_t Lmax, int32_t Hq, int32_t Hkv, int32_t D, int32_t window,
                                         float softmax_scale, const gptoss_rope_params* rope, void* out,
                                         float* lse, struct CUstream_st* stream);

/* Reads (and, if reset != 0, clears) the device status word of the current
 * device: GPTOSS_OK, GPTOSS_ERR_TIMEOUT (a bounded wait gave up) or
 * GPTOSS_ERR_INVALID_ARG (gptoss_kv_append_paged skipped a block index outside
 * the pool).  Synchronises `stream`. */
gptoss_status gptoss_read_device_status(int32_t* status_out, int32_t reset, struct CUstream_st* stream);

/* Time limit, in microseconds, of every device-side pipeline wait of later
 * launches from this process (0 = the built-in default of 2 s).  A wait that
 * exceeds it records GPTOSS_ERR_TIMEOUT in the device status word and the
 * kernel winds down: it drains its own copies in flight, waits for its own
 * tensor-core work and frees its tensor memory before returning.  This limit
 * is the only state the library keeps between calls. */
gptoss_status gptoss_set_wait_limit(uint32_t microseconds);

/* Failure-path self test: launches one warp that waits, with the given limit
 * (1..1000000 us), on a barrier nothing ever arrives at.  The wait gives up,
 * records GPTOSS_ERR_TIMEOUT in the device status word and writes 0 to
 * *result_dev (1 would mean the wait was satisfied).  No fault, no trap. */
gptoss_status gptoss_selftest_wait_timeout(uint32_t limit_us, int32_t* result_dev, struct CUstream_st* stream);

#ifdef __cplusplus
}
#endif

#endif /* GPTOSS_H_ */
