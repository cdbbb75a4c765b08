/*
 * mla.h -- C-ABI of the B200 (sm_100a) multi-head latent attention hot path.
 *
 * The operations follow the eager MLA definition printed on these pages:
 *   [EQ]  "Eager latent expansion" equation page ("Read the equation", and the
 *         code under "Original context");
 *   [KQ]  Kimi-K2 "Query content heads" page ("Split content heads",
 *         "Join query parts");
 *   [GLM] GLM-5 "Normalized key-value latent" page ("Key-value compression",
 *         "KV cache");
 *   [ROT] Kimi-K2 "RoPE coefficients" page ("Generate RoPE coefficients",
 *         "Query heads", "Key heads").
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller; the library
 *     keeps no pointer after a call returns and allocates no device memory.
 *     Scratch space is the caller's `workspace` buffer, sized by the matching
 *     *_workspace_size query.
 *   - Tensors are dense and row-major (last index contiguous) unless stated.
 *   - Calls are asynchronous on `stream`; none synchronises the device except
 *     mla_check_device_status. Host-side argument errors are reported before
 *     anything is launched.
 *   - The return value is an mla_status. mla_last_error_string() gives a
 *     text for the last non-zero status of the calling thread.
 *   - MLA_BF16 runs read and write bfloat16 tensors and accumulate in fp32;
 *     MLA_FP32 runs are fp32 throughout (exact-fp32 SIMT kernels). Inside a
 *     bf16 prefill on the tensor cores the normalized latent and kv_b_proj
 *     enter the up-projection in fp16; the attention multiplies q as given
 *     with k_nope rounded to bf16 for the non-rotary scores and the rotated
 *     q_pe and k_pe rounded to fp16 for the rotary ones, and the softmax
 *     weights with the values in fp16. Values beyond the fp16 range in those
 *     fp16 buffers set the device error word.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mla_status {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad value     */
  MLA_ERR_UNSUPPORTED_SHAPE = 2,  /* head geometry / alignment not supported    */
  MLA_ERR_WORKSPACE_TOO_SMALL = 3,
  MLA_ERR_CUDA = 4,               /* a CUDA runtime call failed                 */
  MLA_ERR_DEVICE_TIMEOUT = 5      /* a bounded device-side wait gave up         */
} mla_status;

typedef enum mla_dtype { MLA_BF16 = 0, MLA_FP32 = 1 } mla_dtype;

/* Rotary configuration; field names follow config.rope_scaling ([ROT]
 * "Generate RoPE coefficients", model-args and rope excerpts).
 *   yarn = 0: default rotary embedding, inv_freq[i] = base^(-2i/rope_dim).
 *   yarn = 1: YaRN blend of base and factor-interpolated frequencies over the
 *             correction range of (beta_fast, beta_slow) turns measured over
 *             original_max_pos positions; tables multiplied by
 *             get_mscale(factor, mscale) / get_mscale(factor, mscale_all_dim). */
typedef struct mla_rope_cfg {
  int32_t rope_dim;          /* qk_rope_head_dim, even, 2..256              */
  int32_t yarn;              /* 0 or 1                                       */
  int32_t original_max_pos;  /* YaRN original_max_position_embeddings        */
  int32_t reserved;          /* must be 0                                    */
  double base;               /* rope_theta (> 1)                             */
  double factor;             /* YaRN scaling factor                          */
  double beta_fast;
  double beta_slow;
  double mscale;
  double mscale_all_dim;
} mla_rope_cfg;

/* Head geometry ([ROT] "Query heads" mla-init; [GLM] mla-init). */
typedef struct mla_dims {
  int32_t num_heads;         /* H                                            */
  int32_t kv_lora_rank;      /* R                                            */
  int32_t qk_nope;           /* N: non-rotary part of each query/key head    */
  int32_t qk_rope;           /* P: rotary part, shared key across heads      */
  int32_t v_head;            /* V                                            */
  int32_t dtype;             /* mla_dtype                                    */
  int32_t rope_interleaved;  /* 0: pair (i, i+P/2); 1: pair (2i, 2i+1)       */
  float eps;                 /* latent RMSNorm epsilon ([GLM]: 1e-6)         */
  float softmax_scale;       /* from mla_softmax_scale()                     */
} mla_dims;

/* Softmax scale ([ROT] model-args; [GLM] mla-init yarn_apply_mscale):
 * qk_head_dim^-0.5, times get_mscale(factor, mscale_all_dim)^2 when yarn = 1
 * and mscale_all_dim != 0. Host only; *scale_out is a host pointer. */
int mla_softmax_scale(const mla_rope_cfg* rope, int32_t qk_head_dim, float* scale_out);

/* Rotary cos/sin tables ([ROT] rope excerpt, _set_cos_sin_cache): for
 * pos < max_pos and pair i < rope_dim/2,
 *   cos_table[pos * rope_dim/2 + i] = cos(pos * inv_freq[i]) * table_mscale
 * (sin likewise). The angle is formed in fp64; values are stored as fp32.
 * cos_table/sin_table: device, fp32 [max_pos, rope_dim/2] each. */
int mla_init_rope_tables(const mla_rope_cfg* rope, int32_t max_pos,
                         float* cos_table, float* sin_table, cudaStream_t stream);

/* Workspace bytes mla_prefill needs for `total_tokens` packed tokens. */
int mla_prefill_workspace_size(const mla_dims* dims, int64_t total_tokens,
                               int32_t num_seqs, size_t* bytes);

/* Causal MLA prefill over packed sequences ([ROT] "Key heads" mla-kv and
 * mla-prefill; [KQ] "Join query parts"; [EQ]).
 *   latent     [Ttot, R + P]  compressed_kv before the split: latent then k_pe
 *   q          [Ttot, H, N + P]  per-head query, non-rotary part first
 *   w_kvb      [H * (N + V), R]  kv_b_proj weight (nn.Linear layout, no bias)
 *   w_norm     [R]            latent RMSNorm weight
 *   positions  int32 [Ttot]   rotary position of each token (< max_pos)
 *   cu_seqlens int32 [num_seqs + 1]  sequence boundaries, cu[0] = 0,
 *              non-decreasing, cu[num_seqs] = total_tokens; empty sequences
 *              are allowed. max_seqlen (host) >= every sequence length.
 *   cos_table, sin_table  fp32 [max_pos, P/2] from mla_init_rope_tables
 *   out        [Ttot, H, V]   attention output, token-major
 * Computes, per sequence and head: c_hat = RMSNorm(latent[:, :R]);
 * [k_nope | v] = c_hat W^T split per head; q_pe and the one shared k_pe
 * rotated at `positions`; softmax(scale * [q_nope|q_pe'][k_nope|k_pe']^T
 * with a causal mask) @ v. All tensors use dims->dtype; positions and
 * cu_seqlens are read on the device and range-checked there: a sequence with
 * bad bounds (outside 0..total_tokens, or longer than max_seqlen) is skipped
 * and a position outside the table is not used; either sets the device error
 * word (see mla_check_device_status). */
int mla_prefill(const mla_dims* dims,
                const void* latent, const void* q, const void* w_kvb, const void* w_norm,
                const int32_t* positions, const int32_t* cu_seqlens,
                int32_t num_seqs, int32_t max_seqlen, int64_t total_tokens,
                const float* cos_table, const float* sin_table, int32_t max_pos,
                void* out, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* kv_b_proj is a model constant, so its conversion for the tensor cores can
 * be done once when the weights are loaded instead of inside every prefill.
 * mla_kv_b_proj_prepared_size gives the bytes of the prepared copy for
 * `dims`; mla_prepare_kv_b_proj writes it (device buffer owned by the caller,
 * w_kvb as for mla_prefill). For the tensor-core head shapes (bf16, qk_rope =
 * 64, qk_nope and v_head multiples of 64 with qk_nope + qk_rope <= 256,
 * kv_lora_rank a multiple of 64 up to 512) the copy is w_kvb in fp16 (exact
 * for weights in fp16's normal range; a weight beyond the fp16 range sets the
 * device error word, MLA_ERR_INVALID_ARG at mla_check_device_status); for
 * other shapes it is w_kvb itself. Both pointers 16-byte aligned for the
 * tensor-core shapes (MLA_ERR_INVALID_ARG otherwise); a buffer smaller than
 * the size returns MLA_ERR_WORKSPACE_TOO_SMALL. */
int mla_kv_b_proj_prepared_size(const mla_dims* dims, size_t* bytes);
int mla_prepare_kv_b_proj(const mla_dims* dims, const void* w_kvb, void* prepared,
                          size_t prepared_bytes, cudaStream_t stream);

/* mla_prefill with the prepared kv_b_proj (w_prepared, written by
 * mla_prepare_kv_b_proj for the same dims) in place of w_kvb: the same
 * kernels and the same results (bit for bit), minus the per-call conversion.
 * For the tensor-core head shapes every tensor and the workspace must be
 * 16-byte aligned (MLA_ERR_INVALID_ARG otherwise: this entry point has no
 * fallback to the CUDA-core kernels for them), and out 32-byte aligned. */
int mla_prefill_prepared(const mla_dims* dims,
                         const void* latent, const void* q, const void* w_prepared, const void* w_norm,
                         const int32_t* positions, const int32_t* cu_seqlens,
                         int32_t num_seqs, int32_t max_seqlen, int64_t total_tokens,
                         const float* cos_table, const float* sin_table, int32_t max_pos,
                         void* out, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Workspace bytes mla_decode needs for `batch` sequences whose longest
 * cache has max_cache_len rows. */
int mla_decode_workspace_size(const mla_dims* dims, int32_t batch, int32_t max_cache_len,
                              size_t* bytes);

/* Absorbed decode: one new query per sequence over a latent cache
 * ([GLM] "KV cache": the cache holds the normalized latent and the rotated
 * shared key; [EQ] "Read the equation": the absorbed path contracts the
 * projection weights with the query and with the latent aggregate).
 *   q             [B, H, N + P]
 *   cache         [cache_num_rows, R + P]  each row = c_hat (R) || rotated k_pe (P)
 *   cache_offsets int64 [B]       first cache row of sequence b
 *   cache_lens    int32 [B]       cached rows of sequence b, 1..max_cache_len
 *   positions     int32 [B]       rotary position of the new query (< max_pos)
 *   w_kvb         [H * (N + V), R]
 *   out           [B, H, V]
 * Per (b, h): q_lat = W_UK_h^T q_nope, q_pe' = rope(q_pe, positions[b]),
 * s_t = scale (q_lat . c_hat_t + q_pe' . k_pe_t) over the sequence's rows,
 * o_lat = softmax(s) . c_hat, out = W_UV_h o_lat, where W_UK_h / W_UV_h are
 * the k_nope / value rows of head h in w_kvb. Attention is split over rows
 * and the pieces are merged by their log-sum-exp.
 * The tensor-core kernels take bf16 runs with R = 512, P = 64, N a multiple
 * of 64 and 1..64 heads (fewer than 64, e.g. one GPU's share of a
 * head-sharded model, are padded to 64 with zero queries whose outputs are
 * dropped: the call streams the same cache bytes as with 64 heads), 16-byte
 * aligned cache and workspace, and fewer than 2^31 cache rows; other calls
 * run on the CUDA cores (mla_last_dispatch says which and why).
 * Device-resident arguments are range-checked on the device: a sequence whose
 * rows fall outside the cache, whose length is outside 1..max_cache_len or
 * whose position is outside the table is skipped (its output is zero) and the
 * device error word is set (see mla_check_device_status). */
int mla_decode(const mla_dims* dims, const void* q, const void* cache, int64_t cache_num_rows,
               const int64_t* cache_offsets, const int32_t* cache_lens,
               const int32_t* positions, int32_t batch, int32_t max_cache_len,
               const void* w_kvb, const float* cos_table, const float* sin_table,
               int32_t max_pos, void* out, void* workspace, size_t workspace_bytes,
               cudaStream_t stream);

/* New cache rows ([GLM] "KV cache" and "Key-value compression": the cache is
 * written while the latent is still compressed, with the normalized latent
 * and the rotated key).
 *   latent     [n, R + P]  rows of compressed_kv
 *   w_norm     [R]
 *   positions  int32 [n]
 *   cache      [cache_num_rows, R + P]  destination; row i goes to cache_rows[i]
 *   cache_rows int64 [n]   destination row of each new token
 * Row = RMSNorm(latent[:R]) || rope(latent[R:], position). A destination
 * row or position out of range is skipped and sets the device error word. */
int mla_cache_append(const mla_dims* dims, const void* latent, const void* w_norm,
                     const int32_t* positions, int64_t n, const float* cos_table,
                     const float* sin_table, int32_t max_pos, void* cache,
                     int64_t cache_num_rows, const int64_t* cache_rows, cudaStream_t stream);

/* Workspace bytes mla_prefill_cached needs for total_tokens chunk tokens
 * whose sequences hold at most max_total_len rows once the chunk is in. */
int mla_prefill_cached_workspace_size(const mla_dims* dims, int64_t total_tokens,
                                      int32_t max_total_len, size_t* bytes);

/* Chunks of new tokens that continue cached sequences ([GLM] "KV cache": the
 * cache is updated with the new tokens' normalized latent and rotated key,
 * then the heads are expanded from every cached row and attended).
 *   latent        [Tq, R + P]   compressed_kv rows of the chunk tokens
 *   q             [Tq, H, N + P]
 *   cu_seqlens    int32 [num_seqs + 1]  chunk tokens per sequence, packed
 *                 (cu_seqlens[0] = 0, cu_seqlens[num_seqs] = Tq = total_tokens;
 *                 a sequence may have no chunk tokens)
 *   cache_offsets int64 [num_seqs]  first cache row of sequence s
 *   prefix_lens   int32 [num_seqs]  rows of sequence s cached before the call
 *   max_total_len prefix_lens[s] + chunk length of s, at most, over s
 *   cache         [cache_num_rows, R + P]  read and written (as mla_decode / mla_cache_append)
 *   w_kvb, w_norm, cos/sin tables as for mla_prefill
 *   out           [Tq, H, V]
 * Chunk token i of sequence s sits at position p + i (p = prefix_lens[s]).
 * Its row RMSNorm(latent[:R]) || rope(latent[R:], p + i) is written to cache
 * row cache_offsets[s] + p + i, and it attends to the sequence's rows
 * 0 .. p + i: its cached prefix, the chunk tokens before it, and itself (the
 * causal mask in absolute positions). Each chunk token runs as one row of
 * the absorbed decode (mla_decode), so the cost is the sum over chunk
 * tokens of the rows each attends (the absorbed form). Long chunks take the
 * eager form instead when it applies: bf16 with qk_rope 64, v_head 128,
 * qk_nope 64 or 128, at least 128 chunk tokens per sequence on average,
 * 16-byte aligned q, cache, w_kvb and workspace, 32-byte aligned out, and a workspace of at
 * least mla_prefill_cached_eager_workspace_size bytes. It expands the keys and
 * values of every row of each sequence (prefix and chunk) with the
 * up-projection and runs the prefill's attention over them, so its cost
 * grows with the rows once plus the chunk x rows attention on the tensor
 * cores; a smaller workspace keeps the absorbed form. Both give the same
 * results up to rounding; mla_last_dispatch names the form used. At most
 * 65535 chunk tokens per call
 * (MLA_ERR_UNSUPPORTED_SHAPE above). The sequences' cache regions must not
 * overlap. Device-resident arguments are range-checked on the device: a
 * token whose sequence is inconsistent with cu_seqlens, whose rows leave the
 * cache or exceed max_total_len, or whose position is outside the table is
 * neither written to the cache nor attended (its output is zero) and the
 * device error word is set. */
/* Workspace bytes of the eager form of mla_prefill_cached for num_seqs
 * sequences of total_tokens chunk tokens whose sequences hold at most
 * max_total_len rows once the chunk is in (padded key layout of
 * num_seqs x ceil(max_total_len / 128) tiles of 128 rows: keys and values of
 * every row, fp16). MLA_ERR_UNSUPPORTED_SHAPE for head shapes without the
 * eager form. */
int mla_prefill_cached_eager_workspace_size(const mla_dims* dims, int64_t total_tokens, int32_t num_seqs,
                                            int32_t max_total_len, size_t* bytes);

/* The form of a chunk call (mla_prefill_cached_form). */
typedef enum mla_chunk_form {
  MLA_CHUNK_AUTO = 0,      /* eager for long chunks when it applies and fits, else absorbed */
  MLA_CHUNK_ABSORBED = 1,  /* one absorbed decode row per chunk token */
  MLA_CHUNK_EAGER = 2      /* keys and values of every row expanded; MLA_ERR_UNSUPPORTED_SHAPE or
                              MLA_ERR_WORKSPACE_TOO_SMALL when it does not apply */
} mla_chunk_form;

int mla_prefill_cached(const mla_dims* dims, const void* latent, const void* q, const void* w_kvb,
                       const void* w_norm, const int32_t* cu_seqlens, int32_t num_seqs,
                       int64_t total_tokens, const int64_t* cache_offsets,
                       const int32_t* prefix_lens, int32_t max_total_len,
                       const float* cos_table, const float* sin_table, int32_t max_pos,
                       void* cache, int64_t cache_num_rows, void* out, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream);

/* mla_prefill_cached with the form chosen by the caller (`form`, an
 * mla_chunk_form); mla_prefill_cached is this call with MLA_CHUNK_AUTO. */
int mla_prefill_cached_form(const mla_dims* dims, const void* latent, const void* q, const void* w_kvb,
                            const void* w_norm, const int32_t* cu_seqlens, int32_t num_seqs,
                            int64_t total_tokens, const int64_t* cache_offsets,
                            const int32_t* prefix_lens, int32_t max_total_len,
                            const float* cos_table, const float* sin_table, int32_t max_pos,
                            void* cache, int64_t cache_num_rows, void* out, void* workspace,
                            size_t workspace_bytes, int32_t form, cudaStream_t stream);

/* The projections on either side of the path ([ROT] "Query heads": mla-init
 * gives the nn.Linear shapes, mla-queries the query order; "Key heads": mla-kv
 * the joint down-projection). A Linear is out[t, j] = sum_k x[t, k] w[j, k],
 * with w the nn.Linear weight [out, in]; no bias. In bf16 runs with the
 * reduced dimension K a multiple of 64, the output width a multiple of 32 and
 * 16-byte aligned tensors it runs on the tensor cores (fp32 accumulation, bf16
 * result, 128 rows by up to 256 outputs per CTA; the down-projection and
 * q_a_proj may split K into up to 4 fp32 partials, added in a fixed order by
 * the step that reads them); otherwise on the CUDA cores. At most 2^20 rows
 * (tokens) per call (MLA_ERR_UNSUPPORTED_SHAPE). */

/* Workspace bytes of mla_kv_down_append for n rows: the Linear's fp32
 * result [n, R + P] (room for 4 K-split partials) in bf16 runs, 0 in fp32
 * runs. */
int mla_kv_down_append_workspace_size(const mla_dims* dims, int64_t n, size_t* bytes);

/* kv_a_proj_with_mqa, optionally followed by the cache append:
 *   hidden     [n, hidden_size]
 *   w_kva      [R + P, hidden_size]
 *   latent     [n, R + P]  written: compressed_kv (the latent input of mla_prefill)
 * If cache and cache_rows are both non-NULL, each row is also appended as by
 * mla_cache_append (w_norm, positions and the tables are then required); if
 * both are NULL only latent is written. In bf16 runs the Linear's result stays
 * fp32 in the workspace: latent is its rounding to bf16, and the cache row's
 * RMSNorm and rotation are computed from the fp32 values (no rounding before
 * the norm); workspace may be NULL in fp32 runs. */
int mla_kv_down_append(const mla_dims* dims, int32_t hidden_size, const void* hidden,
                       const void* w_kva, const void* w_norm, const int32_t* positions, int64_t n,
                       const float* cos_table, const float* sin_table, int32_t max_pos,
                       void* latent, void* cache, int64_t cache_num_rows,
                       const int64_t* cache_rows, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream);

/* Workspace bytes of mla_q_proj: the [n, q_rank] fp32 intermediate (in bf16
 * runs room for 4 K-split partials, its normalized copy and an fp16 copy of
 * w_qb). */
int mla_q_proj_workspace_size(const mla_dims* dims, int32_t q_rank, int64_t n, size_t* bytes);

/* q = q_b_proj(q_a_layernorm(q_a_proj(hidden))):
 *   hidden  [n, hidden_size]
 *   w_qa    [q_rank, hidden_size]
 *   w_qnorm [q_rank]  RMSNorm weight (eps = dims->eps)
 *   w_qb    [H * (N + P), q_rank]
 *   q       [n, H, N + P]  written (the q input of mla_prefill / mla_decode)
 * q_a stays fp32 until its RMSNorm. In bf16 runs the normalized q_a enters
 * q_b_proj in fp16 against an fp16 copy of w_qb made in the workspace (tensor
 * cores: q_rank a multiple of 64, 16-byte aligned tensors; a w_qb value beyond
 * the fp16 range sets the device error word), or in fp32 (CUDA cores);
 * accumulation is fp32 and q is bf16. */
int mla_q_proj(const mla_dims* dims, int32_t hidden_size, int32_t q_rank, const void* hidden,
               const void* w_qa, const void* w_qnorm, const void* w_qb, int64_t n, void* q,
               void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* o_proj: attn [n, H * V] (the output of mla_prefill / mla_decode, heads
 * joined) times w_o [hidden_size, H * V]^T -> out [n, hidden_size]. */
int mla_o_proj(const mla_dims* dims, int32_t hidden_size, const void* attn, const void* w_o,
               int64_t n, void* out, cudaStream_t stream);

/* Size of the scratch array behind mla_prefill_noalloc (32 MiB). */
#define MLA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/* Prefill for callers that cannot allocate device memory. Some code that
 * calls this library owns no device allocator of its own: a plugin inside a
 * host application whose framework has already reserved the GPU's memory in
 * its caching allocator, or a latency-bound loop that may not call
 * cudaMalloc because that call can block until the whole device is idle.
 * This entry point takes the same arguments as mla_prefill except the
 * workspace, and allocates nothing: its scratch is a file-scope static
 * __device__ array of MLA_NOALLOC_SCRATCH_BYTES bytes that exists on every
 * GPU that loads this library, until the process exits. The pages have no
 * counterpart to this entry point; it changes how scratch is provided, not
 * what is computed (the results equal mla_prefill's).
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress, a host-side lookup), so a call after
 *     cudaDeviceReset finds the array in the new context. The first call on
 *     a device may load the library's device code: make it before any
 *     stream capture.
 *   - A call whose workspace need (mla_prefill_workspace_size) exceeds
 *     MLA_NOALLOC_SCRATCH_BYTES returns MLA_ERR_WORKSPACE_TOO_SMALL and
 *     launches nothing. For the Kimi-K2 head geometry half of the array
 *     holds the call's fp16 copy of kv_b_proj and the rest holds one
 *     sequence of up to 256 tokens (each sequence is padded to 128-token
 *     tiles, plus one tile per sequence of headroom).
 *   - All calls on a device share the one array, and it keeps what the last
 *     call left there (no part of it needs to start at zero: every call
 *     writes what it reads). Calls that can overlap on the GPU (different
 *     streams without ordering between them) race on it and must not be
 *     issued. */
int mla_prefill_noalloc(const mla_dims* dims,
                        const void* latent, const void* q, const void* w_kvb, const void* w_norm,
                        const int32_t* positions, const int32_t* cu_seqlens,
                        int32_t num_seqs, int32_t max_seqlen, int64_t total_tokens,
                        const float* cos_table, const float* sin_table, int32_t max_pos,
                        void* out, cudaStream_t stream);

/* Synchronises `stream`, then reads and clears the device error word that
 * the kernels' bounded waits set. Returns MLA_ERR_DEVICE_TIMEOUT if one gave
 * up since the last check, MLA_ERR_CUDA on a CUDA error, else MLA_OK. */
int mla_check_device_status(cudaStream_t stream);

/* Self-test of the failure detection (the pages have no counterpart: their
 * only error convention is the shape checks of the eager code). Every wait in
 * the library's kernels is bounded: after its time limit it sets the device
 * error word and lets the kernel return, so a lost arrival never hangs the
 * GPU. This call launches one CTA whose wait, through the same helper but with
 * a limit of `limit_us` microseconds (1 .. 1000000), is on an mbarrier that
 * nothing arrives at. It runs out, sets the device error word and writes 1 to
 * *gave_up (device int32, owned by the caller; 0 had the barrier completed).
 * The next mla_check_device_status then returns MLA_ERR_DEVICE_TIMEOUT and
 * clears the word; the context stays usable. */
int mla_selftest_wait_timeout(uint32_t limit_us, int32_t* gave_up, cudaStream_t stream);

/* Text of the calling thread's last error (static storage, never NULL). */
const char* mla_last_error_string(void);

/* Which kernels the calling thread's last prefill or decode call launched:
 * "tensor-core", or "simt: <reason>" when it ran the exact CUDA-core kernels
 * instead (a head shape or dtype outside the tensor-core kernels, a tensor
 * that is not 16-byte aligned, or a prefill output that is not 32-byte
 * aligned). Static storage, never NULL; "none" before the first call. */
const char* mla_last_dispatch(void);

/* Profiling support. Registers `pairs` pairs of host cudaEvent_t handles
 * (`events` points to 2 * pairs handles created by the caller). Every kernel
 * the calling thread's later calls launch records events[2i] on its stream
 * right before the i-th launch and events[2i+1] right after it, for
 * i < pairs; later launches are not recorded. pairs = 0 (or events = NULL)
 * stops recording. Returns the number of launches recorded so far under the
 * current registration in *recorded when `recorded` is not NULL. */
int mla_set_kernel_events(void* const* events, int32_t pairs);
int mla_recorded_kernel_events(int32_t* recorded);
/* Kernel name of the i-th recorded launch ("" when i is out of range). */
const char* mla_recorded_kernel_name(int32_t i);

/* Number of kernels this library has launched in this process. */
uint64_t mla_launch_count(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int mla_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MLA_H_ */
