/*
 * llama_b200.h -- C ABI of the B200 (sm_100a) LLaMA-style decoder-block library.
 *
 * The library computes the forward pass of a pre-norm decoder block, in
 * prefill (a whole prompt chunk at once) and KV-cached decode (one new token
 * per sequence), and optionally of a whole model (embedding, N blocks, final
 * norm, lm_head, greedy argmax).  Pages cited below by title:
 *
 *   [MLX-13B]  "iOS设备上运行LLaMA2-13B：基于苹果MLX框架的完整技术指南"
 *   [DeepDive] "LLaMA架构深度解析：从开源大模型设计到高效推理的工程实现全流程",
 *              section 二 "LLaMA架构组件"
 *   [Decoder]  "老码农和你一起学AI系列：关于LLaMA解码器"
 *   [HandsOn]  "《Hands-On Large Language Models》阅读笔记(二)"
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.  The caller owns ALL memory.  Every pointer named "device" is CUDA
 *   device memory on the current device; the library never allocates device
 *   memory and never frees what it is given.  Every device pointer must be
 *   16-byte aligned (LLAMA_ERR_ALIGNMENT otherwise).
 * Layout.  Row-major everywhere.  A Linear weight is [out_features, in_features]
 *   and computes y = x W^T with no bias ([DeepDive] nn.Linear(..., bias=False);
 *   [MLX-13B] module tree).  The residual stream x is float32 [tokens, dim],
 *   token t of sequence b at row b*seq_len + t.  Norm weights are float32 [dim].
 *   Projection weights, the embedding and lm_head are `dims.dtype`.
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  All work is enqueued on it; no call synchronises, except
 *   llama_device_status.  Layer and model calls may be captured into a CUDA
 *   graph (stream capture): they enqueue kernels only.  Positions (the cache
 *   length when the call is enqueued) are fixed in the captured work, so a
 *   replay recomputes the step at the captured position; the caller restores
 *   the cache length (and contents, if it needs them) before replaying.
 * Errors.  Calls return a llama_status and never throw.  Argument checks run
 *   before anything is enqueued; on failure nothing is enqueued and the cache
 *   length is unchanged.  Device-side failures (a bounded wait that ran out)
 *   are recorded in a status word at the start of the workspace and read with
 *   llama_device_status after the caller synchronises the stream.
 * Concurrency.  Two calls that share a workspace or a cache must not overlap
 *   on the GPU (enqueue them on one stream).
 */
#ifndef LLAMA_B200_H
#define LLAMA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LLAMA_B200_ABI_VERSION 1

typedef enum llama_status {
  LLAMA_OK = 0,
  LLAMA_ERR_INVALID_ARG = 1,         /* null pointer, bad size, bad enum, aliasing */
  LLAMA_ERR_UNSUPPORTED = 2,         /* valid but not implemented (e.g. head_dim 48) */
  LLAMA_ERR_CACHE_FULL = 3,          /* length + new tokens > capacity */
  LLAMA_ERR_ALIGNMENT = 4,           /* a device pointer is not 16-byte aligned */
  LLAMA_ERR_WORKSPACE_TOO_SMALL = 5, /* ws_bytes < the *_workspace_size query */
  LLAMA_ERR_CUDA = 6,                /* a CUDA runtime/driver call failed */
  LLAMA_ERR_DEVICE_TIMEOUT = 7,      /* a bounded device wait ran out (read via llama_device_status) */
  LLAMA_ERR_SCRATCH_LIMIT = 8        /* llama_attention_decode_noalloc: more than its fixed scratch */
} llama_status;

/* RoPE variant.  HALF: rotate-half, x*cos(emb) + cat(-x2, x1)*sin(emb) with
 * emb = cat(freqs, freqs) ([DeepDive] class LLaMARoPE).  INTERLEAVED: the
 * "traditional" variant named in [MLX-13B] "LLaMA 2 的结构分析"
 * (RoPE(128, traditional=True)); read as adjacent pairs (x[2i], x[2i+1])
 * rotated by p * theta^(-2i/head_dim). */
typedef enum llama_rope_style { LLAMA_ROPE_HALF = 0, LLAMA_ROPE_INTERLEAVED = 1 } llama_rope_style;

/* Storage / operand type of weights, projections and the KV cache.
 * LLAMA_F32: every operand fp32, CUDA-core arithmetic (no TF32).
 * LLAMA_BF16: bf16 operands on the tensor cores with fp32 accumulation.
 * The residual stream is fp32 in both. */
typedef enum llama_dtype { LLAMA_F32 = 0, LLAMA_BF16 = 1 } llama_dtype;

/* Block hyper-parameters ([MLX-13B] 模型配置 config.json; [DeepDive] LLaMAConfig).
 * Supported: head_dim in {64, 96, 128} (and 32 for LLAMA_F32);
 * n_heads % n_kv_heads == 0 (GQA group n_heads/n_kv_heads, query head h
 * reads KV head h / group, [DeepDive] LLaMAAttention); dim, ffn_dim and
 * n_heads*head_dim multiples of 8; dim <= 16384; eps > 0; rope_theta > 1. */
typedef struct llama_dims {
  int32_t dim;
  int32_t n_heads;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t ffn_dim;
  float eps;
  float rope_theta;
  int32_t rope_style; /* llama_rope_style */
  int32_t dtype;      /* llama_dtype */
} llama_dims;

/* One block's weights (device pointers, caller-owned).
 *   attn_norm, ffn_norm : float32 [dim]
 *   wq [n_heads*head_dim, dim], wk/wv [n_kv_heads*head_dim, dim]   (dtype)
 *   wo [dim, n_heads*head_dim]                                     (dtype)
 *   w1 (gate) / w3 (up) [ffn_dim, dim], w2 (down) [dim, ffn_dim]   (dtype)
 * A fused qkv weight ([HandsOn] Phi-3 qkv_proj [9216, 3072]) is passed as
 * wq = base, wk = base + nh*hd rows, wv = wk + nkv*hd rows (q, then k, then
 * v); a fused gate_up weight ([HandsOn] gate_up_proj) as w1 = base,
 * w3 = base + ffn_dim rows (gate first).  When wq, wk, wv are contiguous in
 * that order the QKV projection runs as one GEMM. */
typedef struct llama_layer_weights {
  const float* attn_norm;
  const void* wq;
  const void* wk;
  const void* wv;
  const void* wo;
  const float* ffn_norm;
  const void* w1;
  const void* w3;
  const void* w2;
} llama_layer_weights;

/* ------------------------------------------------------------------ KV cache */

/* Opaque host object describing one layer's KV cache ([MLX-13B] KV 缓存实现
 * 片段: new, already-rotated keys and values are appended after the cached
 * ones along the sequence axis; the next tokens' RoPE positions start at the
 * current length).  It holds pointers, capacity and length only.  */
typedef struct llama_kv_cache llama_kv_cache;

/* k_buf, v_buf: caller-owned device buffers, each [batch][n_kv_heads][capacity][head_dim]
 * of dims->dtype.  The new cache has length 0.
 * Errors: INVALID_ARG (null, batch/capacity <= 0, bad dims), ALIGNMENT. */
llama_status llama_kv_cache_create(const llama_dims* dims, int32_t batch, int32_t capacity, void* k_buf,
                                   void* v_buf, llama_kv_cache** out);
/* Declare that positions [0, len) of every sequence already hold valid
 * (rotated) keys and values -- e.g. a synthetic pre-filled cache.
 * Errors: INVALID_ARG (len < 0), CACHE_FULL (len > capacity). */
llama_status llama_kv_cache_set_length(llama_kv_cache* cache, int32_t len);
/* Current length (positions filled) when every sequence has the same length;
 * -2 while the sequences' lengths differ (see llama_kv_cache_lengths); -1 for a
 * null handle. */
int32_t llama_kv_cache_length(const llama_kv_cache* cache);
/* Per-sequence lengths (ragged batch; [MLX-13B] KV 缓存实现片段 keeps one
 * offset for the whole batch, here each sequence keeps its own): declare
 * that positions [0, lens[b]) of sequence b hold valid keys and values.
 *   lens   HOST int32 [batch]
 * Calls other than llama_layer_forward_ragged need equal lengths and return
 * INVALID_ARG while they differ.  Errors: INVALID_ARG, CACHE_FULL. */
llama_status llama_kv_cache_set_lengths(llama_kv_cache* cache, const int32_t* lens);
/* Copy the per-sequence lengths into lens (HOST int32 [batch]). */
llama_status llama_kv_cache_lengths(const llama_kv_cache* cache, int32_t* lens);
int32_t llama_kv_cache_capacity(const llama_kv_cache* cache);
void llama_kv_cache_destroy(llama_kv_cache* cache);

/* ------------------------------------------------------------------ workspace */

/* Bytes of device workspace a layer call with `batch` sequences of up to
 * `seq_len` new tokens needs (seq_len = 1 for decode).  0 on invalid dims.
 * The workspace is caller-owned scratch.  Zero-fill it once before its first
 * use: a fixed 4096-byte header at its start (the same for every batch and
 * seq_len) holds the device status word, the decode GEMMs' per-CTA flags,
 * the fused RMSNorm's counters and the grid-barrier counters of the
 * persistent decode-block kernel, which every launch leaves at zero; after
 * that the library keeps it consistent, also when prefill and decode calls
 * of different shapes share it.  After a
 * call that recorded LLAMA_ERR_DEVICE_TIMEOUT, zero-fill it again before
 * reusing it. */
size_t llama_workspace_size(const llama_dims* dims, int32_t batch, int32_t seq_len);

/* Byte offsets, inside the workspace of a layer call with (batch, seq_len),
 * of the intermediate tensors the call leaves behind, for inspection:
 *   out[0] qkv   [tokens, (nh + 2 nkv) hd] dtype: its q columns hold q after RoPE.
 *                The k and v columns are scratch: in bf16 prefill with head_dim
 *                64 or 128 the projection writes k and v straight into the cache;
 *                elsewhere they hold k before RoPE and v.  Read the appended k
 *                and v from the cache.
 *   out[1] h     [tokens, dim] dtype: the second RMSNorm's output
 *   out[2] attn  [tokens, nh hd] dtype: attention output (heads concatenated)
 *   out[3] m     [tokens, ffn_dim] dtype: silu(gate) * up
 * Writes min(n, 4) entries.  Errors: INVALID_ARG. */
llama_status llama_workspace_offsets(const llama_dims* dims, int32_t batch, int32_t seq_len, size_t* out,
                                     int32_t n);

/* Read (and optionally clear) the device status word at the start of
 * `workspace`.  Synchronous device-to-host copy: call after the work has
 * been synchronised.  Returns LLAMA_OK or the first device-side error
 * (LLAMA_ERR_DEVICE_TIMEOUT); LLAMA_ERR_CUDA if the copy itself fails. */
llama_status llama_device_status(const void* workspace, int32_t clear);

/* ------------------------------------------------------------------ layer calls */

/* Prefill: one decoder block over `seq_len` new tokens of each of `batch`
 * sequences, positions cache.length .. cache.length+seq_len-1 (chunked
 * prefill when the cache is not empty: query p sees keys 0..p).
 *   h   = attn_norm * x / sqrt(mean(x^2) + eps)        [MLX-13B] 4. RMSNorm; [DeepDive] LLaMARMSNorm
 *   q,k,v = h Wq^T, h Wk^T, h Wv^T; RoPE on q and k     [DeepDive] LLaMAAttention, LLaMARoPE
 *   cache <- append(k, v)                               [MLX-13B] KV 缓存实现片段
 *   o   = softmax(q k^T / sqrt(hd), causal) v, GQA     [MLX-13B] 2. 注意力机制, 5. 因果掩码
 *   x1  = x + o Wo^T                                    [DeepDive] LLaMABlock
 *   x_out = x1 + W2(silu(h2 W1^T) * (h2 W3^T)), h2 = ffn_norm-RMSNorm(x1)
 *                                                        [MLX-13B] 3. 前馈网络; [Decoder] 数据流动
 * x_in, x_out: device float32 [batch*seq_len, dim]; they must not overlap.
 * The cache length advances by seq_len when the call is enqueued.
 * Errors: INVALID_ARG (null, bad sizes, batch != cache batch, aliasing),
 *   UNSUPPORTED, ALIGNMENT, CACHE_FULL, WORKSPACE_TOO_SMALL, CUDA. */
llama_status llama_layer_prefill(const llama_dims* dims, const llama_layer_weights* w, llama_kv_cache* cache,
                                 int32_t batch, int32_t seq_len, const float* x_in, float* x_out, void* workspace,
                                 size_t ws_bytes, void* stream);

/* Decode: the same block for ONE new token per sequence at position
 * cache.length ([HandsOn] 第三章: decode reads the KV cache and processes
 * only the new token).  x_in, x_out: device float32 [batch, dim].
 * Same errors as llama_layer_prefill. */
llama_status llama_layer_decode(const llama_dims* dims, const llama_layer_weights* w, llama_kv_cache* cache,
                                int32_t batch, const float* x_in, float* x_out, void* workspace, size_t ws_bytes,
                                void* stream);

/* ------------------------------------------------------------------ ragged batches */

/* Workspace bytes of a ragged layer call: `batch` sequences, `total_tokens`
 * new tokens in all.  0 on invalid arguments (batch > 128 included). */
size_t llama_workspace_size_ragged(const llama_dims* dims, int32_t batch, int32_t total_tokens);

/* One decoder block over a ragged batch: sequence b brings n_new[b] >= 1 new
 * tokens at positions lens[b] .. lens[b] + n_new[b] - 1, lens[b] being its own
 * cache length (llama_kv_cache_set_lengths).  Decode rows (n_new = 1) and
 * prefill chunks (n_new > 1) may be mixed in one call ([HandsOn] 第三章: the
 * prefill of a prompt and the token-by-token decode are the same block); the
 * block never mixes sequences, so each sequence gets exactly what a call on it
 * alone computes ([DeepDive] LLaMAAttention attends within a batch row).
 *   n_new   HOST int32 [batch]
 *   x_in, x_out  device float32 [sum n_new, dim], the rows of sequence 0,
 *           then of sequence 1, ... (packed, no padding); must not overlap
 * Each sequence's length advances by n_new[b] when the call is enqueued.
 * dims->dtype must be LLAMA_BF16; batch <= 128.  Workspace:
 * llama_workspace_size_ragged(dims, batch, sum n_new).
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CACHE_FULL, WORKSPACE_TOO_SMALL, CUDA. */
llama_status llama_layer_forward_ragged(const llama_dims* dims, const llama_layer_weights* w, llama_kv_cache* cache,
                                        int32_t batch, const int32_t* n_new, const float* x_in, float* x_out,
                                        void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ 4-bit group-64 weights (decode) */

/* One projection [out_features, in_features] with 4-bit group-wise weights
 * ([MLX-13B] "LLaMA 2 的结构分析": every projection of the 13B block is a
 * QuantizedLinear; "模型配置": "quantization": {"group_size": 64, "bits": 4}).
 * The pages name the scheme without defining it; reading taken: each row is
 * cut into groups of 64 consecutive inputs, a group keeps a scale s and an
 * offset b, and each weight an unsigned code q in 0..15, so that the Linear
 * uses w = s * q + b (y = x W^T, no bias).
 *   codes    device uint32 [out][in / 8]: code of input 8j + k of a row in
 *            bits 4k .. 4k+3 of word j (low nibble first)
 *   scales   device bf16 [in / 64][out]: s of (row o, group g) at [g][o]
 *   offsets  device bf16 [in / 64][out]: b, same layout
 * (the scales and offsets are stored group-major so that one group's values
 * for 64 consecutive rows are one contiguous 128-byte block).  The kernel
 * forms bf16 w = fma(q, s, b) with one rounding and multiplies on the tensor
 * cores with fp32 accumulation. */
typedef struct llama_q4_weight {
  const uint32_t* codes;
  const void* scales;
  const void* offsets;
} llama_q4_weight;

/* One block's weights with every projection in the 4-bit form; norm weights
 * float32 [dim].  wq/wk/wv rows as in llama_layer_weights (three separate
 * projections); w1 gate, w3 up, w2 down. */
typedef struct llama_layer_weights_q4 {
  const float* attn_norm;
  llama_q4_weight wq, wk, wv, wo;
  const float* ffn_norm;
  llama_q4_weight w1, w3, w2;
} llama_layer_weights_q4;

/* llama_layer_decode with 4-bit group-64 weights: the same block, the same
 * cache (dims->dtype must be LLAMA_BF16: bf16 activations and KV cache) and
 * the same workspace (llama_workspace_size(dims, batch, 1)).  Requires dim,
 * ffn_dim and n_heads*head_dim multiples of 64 and batch <= 128.
 * Errors: as llama_layer_decode; UNSUPPORTED for the shapes above. */
llama_status llama_layer_decode_q4(const llama_dims* dims, const llama_layer_weights_q4* w, llama_kv_cache* cache,
                                   int32_t batch, const float* x_in, float* x_out, void* workspace, size_t ws_bytes,
                                   void* stream);

/* ------------------------------------------------------------------ whole model */

/* A whole model ([DeepDive] class LLaMA; [HandsOn] Phi3ForCausalLM tree).
 *   embed   [vocab, dim] (dtype), final_norm float32 [dim], lm_head [vocab, dim] (dtype)
 *   layers  HOST array of n_layers weight sets (device pointers inside). */
typedef struct llama_model {
  llama_dims dims;
  int32_t n_layers;
  int32_t vocab;
  const void* embed;
  const float* final_norm;
  const void* lm_head;
  const llama_layer_weights* layers;
} llama_model;

size_t llama_model_workspace_size(const llama_model* model, int32_t batch, int32_t seq_len);

/* Embedding lookup, all blocks (prefill when seq_len > 1 or the caches are
 * empty, decode otherwise), final RMSNorm, lm_head on the LAST row of each
 * sequence, greedy argmax ([HandsOn] 第三章: argmax of the last position's
 * scores; [MLX-13B] 生成过程: temp 0 is argmax).
 *   caches       HOST array of n_layers cache handles (all the same length)
 *   tokens       device int32 [batch, seq_len], each in [0, vocab)
 *   logits_or_null  device float32 [batch, vocab] or NULL
 *   next_ids     device int32 [batch]; ties resolve to the lowest index
 * Errors: as llama_layer_prefill. */
llama_status llama_model_forward(const llama_model* model, llama_kv_cache* const* caches, const int32_t* tokens,
                                 int32_t batch, int32_t seq_len, float* logits_or_null, int32_t* next_ids,
                                 void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ sampling */

/* Temperature / top-p (nucleus) sampling of the next token ([DeepDive] class
 * LLaMA, generate: logits / temperature, sorted descending, cumulative
 * softmax; a token is dropped once the probability of the tokens sorted
 * before it exceeds top_p, so the token that crosses top_p is kept; the kept
 * tokens are renormalised and one is drawn.  [MLX-13B] 生成过程: temperature 0
 * is greedy argmax).
 *   logits   device float32 [batch, vocab]
 *   u        device float32 [batch], one uniform in [0, 1) per sequence: the
 *            draw is an input; the token picked is the kept token whose
 *            interval of the cumulative renormalised distribution, in sorted
 *            order, holds u (inverse CDF)
 *   ids      device int32 [batch]
 * Sorted order is descending logit / temperature, equal values by ascending
 * index.  Probabilities are exp(z - max z) in fp32, accumulated as integers
 * in units of 2^-40 (exact, order-independent sums).  temperature 0 takes
 * the argmax (u unused, may be NULL); otherwise temperature > 0 and
 * 0 < top_p <= 1.  Allocates nothing; no workspace.
 * Errors: INVALID_ARG, ALIGNMENT, CUDA. */
llama_status llama_sample_top_p(const float* logits, int32_t batch, int32_t vocab, float temperature, float top_p,
                                const float* u, int32_t* ids, void* stream);

/* llama_model_forward with the next token chosen by llama_sample_top_p's rule
 * on the last row's logits instead of argmax (temperature 0: argmax). */
llama_status llama_model_forward_sample(const llama_model* model, llama_kv_cache* const* caches,
                                        const int32_t* tokens, int32_t batch, int32_t seq_len, float temperature,
                                        float top_p, const float* u, float* logits_or_null, int32_t* next_ids,
                                        void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ allocation-free decode attention */

/* The pages have no counterpart to this entry point: it exists for callers
 * that cannot allocate device memory -- a plug-in inside a serving framework
 * that reserved all GPU memory for its own pool and hands out no workspace,
 * or a latency-critical loop that must not call cudaMalloc (which may
 * synchronise the device).  It is the split-KV decode attention of
 * llama_layer_decode on its own, with its partial results kept in a fixed
 * 8 MiB array that is part of the library (every GPU that loads the library
 * holds it until the process exits) instead of in a workspace.  It allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library call.
 *
 *   q        device bf16 [batch, ld_q]: query head h of sequence b at
 *            q[b*ld_q + h*head_dim ...] (already rotated); ld_q >= n_heads*head_dim,
 *            ld_q % 8 == 0 (e.g. the q part of a packed q|k|v row)
 *   k_cache, v_cache  device bf16 [batch][n_kv_heads][capacity][head_dim]
 *   length   keys 0 .. length-1 are attended (1 <= length <= capacity)
 *   out      device bf16 [batch, n_heads*head_dim]
 * out[b, h] = softmax(q_bh k^T / sqrt(head_dim)) v over those keys, KV head
 * h / (n_heads/n_kv_heads).  dims->dtype must be LLAMA_BF16.
 * It runs the same kernels and key-split choice as llama_layer_decode, with
 * at least two key splits whenever the length allows.
 * Limit: batch * n_heads * (head_dim + 2) * 8 bytes <= 8 MiB (two key
 * splits), else LLAMA_ERR_SCRATCH_LIMIT; the call then enqueues nothing.
 * With no workspace there is no device status word: a device-side wait that
 * runs out is not reported by this entry point.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  All calls share the one array and nothing in it needs to start
 * at zero; two calls that overlap on the GPU (different streams, or
 * different host threads without ordering) race on it.
 * Errors: INVALID_ARG, UNSUPPORTED (fp32 dims), ALIGNMENT, SCRATCH_LIMIT, CUDA. */
llama_status llama_attention_decode_noalloc(const llama_dims* dims, int32_t batch, const void* q, int32_t ld_q,
                                            const void* k_cache, const void* v_cache, int32_t capacity,
                                            int32_t length, void* out, void* stream);

/* ------------------------------------------------------------------ misc */

const char* llama_status_string(llama_status s);
int32_t llama_abi_version(void);

/* Upper bound, in nanoseconds, on every device-side wait of later launches
 * (default 2e9).  A test may lower it.  Returns the previous value. */
uint64_t llama_set_wait_limit_ns(uint64_t ns);

/* ------------------------------------------------------------------ tracing */

/* Number of kernels the library has enqueued since it was loaded. */
uint64_t llama_launch_count(void);

/* Turn per-launch tracing on or off.  While on, every kernel launch is
 * bracketed by two CUDA events on its stream (a few microseconds of host
 * work per launch).  No page counterpart: measurement only. */
llama_status llama_profile_enable(int32_t on);

/* Accumulated device time and launch count per kernel kind of the traced
 * launches (synchronises on their events).  Fills up to n entries of each
 * non-null array; names point to static strings.  Returns the number of
 * kinds.  reset != 0 clears the accumulators afterwards. */
int32_t llama_profile_read(const char** names, double* total_ms, long long* launches, int32_t n, int32_t reset);

/* Traced launches that have not finished yet (non-blocking query of their end
 * events), oldest first: writes up to n kind names and returns the count.
 * Names a kernel that does not complete without waiting on it. */
int32_t llama_profile_inflight(const char** names, int32_t n);

/* Self-test of the failure path: launches one CTA that waits on an
 * mbarrier nothing will ever arrive on, with a limit of `limit_ns`; the wait
 * runs out, the kernel records LLAMA_ERR_DEVICE_TIMEOUT in the workspace
 * status word and returns.  No page counterpart: failure detection only. */
llama_status llama_selftest_wait_timeout(void* workspace, uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LLAMA_B200_H */
