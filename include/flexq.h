/*
 * flexq.h - C ABI of the B200 (sm_100a) group-wise int4 OPT layer library.
 *
 * What it computes comes from the FlexGen pages:
 *   - the walkthrough page «FlexGen 单 GPU 高吞吐大模型推理引擎：论文解读与源码实战指南», section 6.3 "4-bit group-wise quantisation of
 *     weights and KV cache": CompressionConfig(num_bits, group_size, group_dim,
 *     symmetric), compress / decompress, two 4-bit codes per uint8 in a data tensor of
 *     shape shape[:group_dim] + (num_groups*(group_size//2),) + shape[group_dim+1:],
 *     and an fp16 per-group scale tensor; weights use (4, 64) and the KV cache
 *     (4, 64) grouped along the head dimension.
 *   - the source-notes page «FlexGen» (PtirisNote), "Pytorch Backend": prefill attention is `mha`,
 *     the decode step is `mha_gen`; "Flex Opt": every step runs load_cache,
 *     compute_layer, store_cache, in that order.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers (cudaMalloc / torch CUDA memory) unless
 *     a parameter says otherwise. The caller owns and allocates every buffer:
 *     inputs, outputs, codes, metadata, caches and workspaces. The library keeps no
 *     per-call state; its global state is one device status word per device, created
 *     on first use (see flex_get_status), the wait limit of flex_set_wait_limit_ns, and
 *     the scratch buffer of flex_decode_attention_noalloc.
 *   - fp16 means IEEE binary16, "half2" a pair of binary16 stored as 4 bytes.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every call only enqueues work on `stream` and returns; none synchronises,
 *     except flex_get_status.
 *   - Return value: FLEX_OK (0) or a negative FLEX_ERR_*. Argument errors are found
 *     on the host before anything is enqueued; nothing is written then. No C++
 *     exception crosses this boundary.
 *   - Pointers must be 16-byte aligned. Outputs must not alias inputs unless stated.
 *   - Non-finite inputs (NaN, Inf) give unspecified results.
 */
#ifndef FLEXQ_H
#define FLEXQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------------ */
#define FLEX_OK               0
#define FLEX_ERR_INVALID_ARG (-1)  /* null pointer, negative size, bad rank       */
#define FLEX_ERR_UNSUPPORTED (-2)  /* bits not 3/4/8 (4/8 outside the codec), group
                                      not 32/64/128, head_dim not 64/128, ...     */
#define FLEX_ERR_SHAPE       (-3)  /* a weight or cache dim not a multiple of the
                                      group, pos >= max_seq, seq > max_seq, ...   */
#define FLEX_ERR_ALIGN       (-4)  /* pointer not 16-byte aligned                 */
#define FLEX_ERR_WORKSPACE   (-5)  /* workspace missing or too small              */
#define FLEX_ERR_CUDA        (-6)  /* a CUDA launch or runtime call failed        */
#define FLEX_ERR_TIMEOUT     (-7)  /* a device-side bounded wait gave up          */
#define FLEX_ERR_SCRATCH_LIMIT (-8) /* problem needs more scratch than the library's
                                       built-in buffer holds (see
                                       flex_decode_attention_noalloc)             */

/* ---- compression configuration (CompressionConfig of section 6.3) ------------ */
typedef struct {
    int32_t num_bits;    /* 4 or 8; the codec (flexq_*) also takes 3                */
    int32_t group_size;  /* 32, 64 or 128                                          */
    int32_t group_dim;   /* dimension the groups run along; negative counts back  */
    int32_t symmetric;   /* 0: the min/max form; 1 (codec only): the absmax form   */
} flexq_config;

/* A compressed tensor: the pages' (data, scale, config) triple.
 *   codes: uint8, shape shape[:gd] + (ng*gs*bits/8,) + shape[gd+1:], row-major.
 *          4-bit: byte j of a group = q[2j] | q[2j+1] << 4 (pairs along group_dim).
 *   meta : half2 {min, scale} per group, shape shape[:gd] + (ng,) + shape[gd+1:].
 *          scale = fp16((2^b - 1) / (max - min)), 0 for a constant group,
 *          65504 where that quotient overflows fp16.                              */
typedef struct {
    const void*  codes;
    const void*  meta;
    int32_t      ndim;      /* 1..4 */
    int64_t      shape[4];  /* logical (uncompressed) shape */
    flexq_config cfg;
} flexq_tensor;

/* ---- codec (compress / decompress of section 6.3) ------------------------------ */

/* Bytes of the codes / metadata buffers for a tensor of `shape` (rank ndim) under
 * `cfg`. Returns a negative FLEX_ERR_* if the configuration or shape is invalid. */
int64_t flexq_codes_bytes(int32_t ndim, const int64_t* shape, flexq_config cfg);
int64_t flexq_meta_bytes(int32_t ndim, const int64_t* shape, flexq_config cfg);

/* compress: x (fp16, row-major, `shape`) -> codes + meta, per group of group_size
 * elements along group_dim:
 *   min, max of the group; scale16 = fp16((2^b-1) / (max - min)) (0 if max == min,
 *   65504 on overflow); q = clamp(rint((x - min) * scale16), 0, 2^b - 1), the
 *   subtraction and the product each rounded in fp32, ties to even.
 * Bit-exact and deterministic. Any rank 1..4; the group dimension may be the
 * contiguous one or a strided one. Tensors of any size (64-bit indexing).
 * Variants (readings of what the pages only name: the symmetric flag and num_groups of
 * the configuration, section 6.3; "int3/int4" on the hub page «FlexLLMGen»):
 *   - num_bits 3: the codes of a group form a little-endian bit stream, code j in bits
 *     [3j, 3j+3) of the group's gs*3/8 bytes;
 *   - symmetric 1: B = 2^(b-1) - 1, scale16 = fp16(B / max|x|) (0 for an all-zero group,
 *     65504 on overflow), signed code clamp(rint(x * scale16), -B, B) stored as code + B,
 *     meta {0, scale16};
 *   - a group_dim extent that is not a multiple of group_size: ceil(extent / group_size)
 *     groups, the last one zero-padded (the padding takes part in min/max and its codes
 *     are stored; codes and meta are sized for the padded extent).
 * These variants run one thread per group (correct for any layout, not tuned); the
 * layer calls take only 4- and 8-bit min/max tensors. */
int flexq_compress(const void* x, int32_t ndim, const int64_t* shape, flexq_config cfg,
                   void* codes, void* meta, void* stream);

/* decompress: codes + meta -> y (fp16, `shape`):
 *   y = fp16(fp32(fp32(q * fp32(1/scale16)) + min)), or y = min when scale16 == 0;
 *   symmetric: y = fp16(fp32((u - B) * fp32(1/scale16))), 0 when scale16 == 0.
 * A zero-padded last group writes only the real elements. */
int flexq_decompress(const void* codes, const void* meta, int32_t ndim, const int64_t* shape,
                     flexq_config cfg, void* y, void* stream);

/* ---- OPT decoder layer ------------------------------------------------------- */

/* Parameters of one OPT pre-LayerNorm decoder layer.
 *   Weights are compressed with {4 or 8 bits, group 64, group_dim 1} and stored
 *   [out][in] (grouped along the input dimension, the contiguous one):
 *     w_qkv [3h][h]  rows ordered [q; k; v], feature = head*head_dim + j
 *     w_o   [h][h], w_fc1 [ffn][h], w_fc2 [h][ffn]
 *   Biases and LayerNorm parameters are plain fp16 vectors.                      */
typedef struct {
    int32_t h, n_heads, head_dim, ffn;
    const void *ln1_g, *ln1_b, *ln2_g, *ln2_b;   /* fp16 [h]                        */
    flexq_tensor w_qkv, w_o, w_fc1, w_fc2;       /* compressed weights              */
    const void *b_qkv, *b_o, *b_fc1, *b_fc2;     /* fp16 [3h], [h], [ffn], [h]      */
} flex_layer;

/* Compressed KV cache of one layer (section 6.3: KV grouped along the head dim).
 *   k_codes, v_codes: uint8 [batch][n_heads][max_seq][head_dim*bits/8]
 *   k_meta,  v_meta : half2 [batch][n_heads][max_seq][head_dim/group_size]
 *   cfg: num_bits 4 or 8, group_size 32/64 (dividing head_dim), group_dim = 3.
 *   valid_from: NULL, or a device int32 [batch] (4-byte aligned): prompts padded on the
 *     left to a common length (the source-notes page «FlexGen» (PtirisNote), "Flex Opt":
 *     the attention_mask buffer of the generation loop; the walkthrough page, section
 *     3.1: HELM prompts padded to pad_to_seq_len). Sequence b's real tokens start at
 *     slot valid_from[b]: no query attends to a slot below it, and a query that is
 *     itself a pad token (prefill rows below it) gets a zero attention output. The
 *     pad tokens still run through the layer and are stored in the cache. NULL (or
 *     zeros) = no padding. Read by the kernels at run time, so it may change between
 *     replays of a captured graph.                                                  */
typedef struct {
    void *k_codes, *k_meta, *v_codes, *v_meta;
    int32_t batch, n_heads, head_dim, max_seq;
    flexq_config cfg;
    const int32_t* valid_from;
} flex_kv_cache;

/* Workspace bytes that flex_prefill_layer (seq > 1) or flex_decode_layer (seq == 1)
 * needs for `batch` sequences of `seq` tokens. Negative FLEX_ERR_* on bad args. */
int64_t flex_workspace_bytes(const flex_layer* L, int32_t batch, int32_t seq);

/* Prefill (`mha` path): x_in fp16 [batch][seq][h] -> x_out fp16 [batch][seq][h].
 *   a = LN1(x); q,k,v = a Wqkv^T + b (q scaled by head_dim^-1/2); causal softmax
 *   attention on the fresh fp16 q/k/v; h1 = x + o Wo^T + b_o;
 *   out = h1 + ReLU(LN2(h1) W1^T + b1) W2^T + b2   (LayerNorm eps 1e-5).
 * Writes the quantised fp16 keys/values of tokens [0, seq) into cache slots
 * [0, seq) (store_cache). seq <= cache->max_seq, batch == cache->batch.
 * ws: device workspace of at least flex_workspace_bytes(L, batch, seq) bytes;
 * x_in and x_out must not alias. */
int flex_prefill_layer(const flex_layer* L, const flex_kv_cache* cache, const void* x_in,
                       void* x_out, int32_t batch, int32_t seq, void* ws, int64_t ws_bytes,
                       void* stream);

/* Decode step (`mha_gen` path) at position pos: x_in fp16 [batch][h] -> x_out fp16.
 *   Same layer; the new token attends to the dequantised cache slots [0, pos) and
 *   to its own fresh key/value; its quantised key/value are then in slot pos.
 * pos < cache->max_seq; batch <= cache->batch (sequences 0..batch-1 of the cache).
 * ws: at least flex_workspace_bytes(L, batch, 1) bytes. */
int flex_decode_layer(const flex_layer* L, const flex_kv_cache* cache, const void* x_in,
                      void* x_out, int32_t batch, int32_t pos, void* ws, int64_t ws_bytes,
                      void* stream);

/* Several gpu-batches through one layer with one pass over its weights (the walkthrough
 * page, sections 2.3 and 6.1: gpu_batch_size x num_gpu_batches, e.g. 48 x 3, where one
 * weight load serves every gpu-batch of the block; the source-notes page «FlexGen»
 * (PtirisNote), "Flex Opt": the loop over gpu-batches inside each layer).
 *   caches: num_batches caches (1..8) of identical geometry, cache c holding gpu-batch c.
 *   x_in, x_out: fp16 [num_batches][batch][seq][h] (prefill) or [num_batches][batch][h]
 *   (decode), gpu-batch c at rows [c*batch*seq, (c+1)*batch*seq).
 *   The LayerNorms and the four weight GEMMs run once over all num_batches * batch * seq
 *   rows; attention runs per gpu-batch on its own cache; each row's key/value go to its
 *   gpu-batch's cache. Results equal num_batches separate calls up to summation order.
 *   ws: flex_workspace_bytes(L, num_batches * batch, seq) bytes. Prefill needs
 *   batch == every cache's batch; decode batch <= every cache's batch. */
int flex_prefill_layer_batches(const flex_layer* L, const flex_kv_cache* caches, int32_t num_batches,
                               const void* x_in, void* x_out, int32_t batch, int32_t seq, void* ws,
                               int64_t ws_bytes, void* stream);
int flex_decode_layer_batches(const flex_layer* L, const flex_kv_cache* caches, int32_t num_batches,
                              const void* x_in, void* x_out, int32_t batch, int32_t pos, void* ws,
                              int64_t ws_bytes, void* stream);

/* ---- the whole model around the layers: embedding, output head, greedy choice --- */
/* The source-notes page «FlexGen» (PtirisNote), "Flex Opt": the model is an embedding,
 * N transformer layers and an output head (OptLM.generate runs the loop); "Pytorch
 * Backend": opt_input_embed / opt_output_embed are the embedding layers. The walkthrough
 * page, section 4.1: generate(..., do_sample, ...); do_sample = False is greedy.
 * E: the token table, fp16 [V_pad][h] compressed with {4 bits, group 64, group_dim 1}
 * like the layer weights (V_pad a multiple of 128 and h of 256; rows >= vocab are
 * padding that no token uses); it is also the output head (logits = LN(h) E^T). */

/* x[r] = fp16(E^[tokens[r]] + P[positions[r]]), r < n: E^ the codec's dequantisation of
 * the table row, P an fp16 position table [max_pos][h]; the sum of the two fp16 values
 * is rounded once. tokens, positions: device int32 [n]; x: fp16 [n][h]. An id outside
 * [0, vocab) or a position outside [0, max_pos) is clamped into range and reported as
 * FLEX_ERR_INVALID_ARG by flex_get_status. */
int flex_embed(const flexq_tensor* E, int32_t vocab, const void* P, int32_t max_pos,
               const int32_t* tokens, const int32_t* positions, int64_t n, void* x, void* stream);

/* Output head and greedy choice for n rows x (fp16 [n][h], natural order):
 * logits = LN(x; lnf_g, lnf_b) E^T (eps 1e-5), next[r] = the column of the largest
 * logit among columns [0, vocab), the lowest column among equal fp16 values. next:
 * device int32 [n]. logits: fp16 [n][V_pad] to keep them, or NULL (then they live in
 * the workspace). ws: flex_lm_head_ws_bytes(E, vocab, n, logits != NULL) bytes. */
int64_t flex_lm_head_ws_bytes(const flexq_tensor* E, int32_t vocab, int64_t n, int32_t with_logits);
int flex_lm_head_argmax(const flexq_tensor* E, int32_t vocab, const void* lnf_g, const void* lnf_b,
                        const void* x, int64_t n, int32_t* next, void* logits, void* ws,
                        int64_t ws_bytes, void* stream);

/* ---- hot-path steps, callable one by one ------------------------------------- */

/* store_cache: quantise k_new / v_new (fp16 [batch][n_heads][head_dim], rows of
 * `row_stride` elements between consecutive sequences; head h of sequence b starts
 * at b*row_stride + h*head_dim) into cache slot pos of sequences 0..batch-1.
 * Same quantiser as flexq_compress with group_dim = head dim. */
int flex_append_kv(const flex_kv_cache* cache, const void* k_new, const void* v_new,
                   int64_t row_stride, int32_t batch, int32_t pos, void* stream);

/* Decode attention (`mha_gen` core): per sequence b < batch and head:
 *   o = softmax([q.k_vf .. q.k_{pos-1}, q.k_new]) [v_vf .. v_{pos-1}, v_new]
 * with k_j, v_j the dequantised cache slots [vf, pos), vf = cache->valid_from[b]
 * (0 without padding; clamped to [0, pos]). q, k_new, v_new: fp16 rows of
 * `row_stride` elements per sequence (a multiple of 8, else FLEX_ERR_ALIGN), head h
 * at offset h*head_dim (q is used as given: callers pre-scale it). o: fp16
 * [batch][n_heads*head_dim].
 * ws: at least flex_decode_attention_ws_bytes(cache, batch, pos) bytes. */
int64_t flex_decode_attention_ws_bytes(const flex_kv_cache* cache, int32_t batch, int32_t pos);
int flex_decode_attention(const flex_kv_cache* cache, const void* q, const void* k_new,
                          const void* v_new, int64_t row_stride, void* o, int32_t batch,
                          int32_t pos, void* ws, int64_t ws_bytes, void* stream);

/* Decode attention that allocates nothing and takes no workspace. The pages have no
 * counterpart: it is a library convenience for callers that cannot hand over device
 * memory, e.g. a plain C host program that owns only the cache and activation buffers
 * and has no device allocator, or an out-of-memory handler that must make progress
 * when no more device memory can be had. Arguments, layouts and results are those of
 * flex_decode_attention; the split-KV partials go to a buffer compiled into the
 * library (FLEX_DECODE_ATTENTION_STATIC_MAX_BYTES per device, held for the life of
 * the process once the library's device code is loaded).
 *   - Limit: a call whose partials, flex_decode_attention_ws_bytes(cache, batch, pos),
 *     exceed FLEX_DECODE_ATTENTION_STATIC_MAX_BYTES returns FLEX_ERR_SCRATCH_LIMIT and
 *     launches nothing (8 MiB covers e.g. 144 sequences x 96 heads of 128).
 *   - Set-up: the first call on a device, made with that device current, looks up the
 *     buffer's device address with a CUDA runtime query (with lazy module loading the
 *     driver may load the library's device code, buffer included, at that moment);
 *     make that first call before any stream capture begins on the device. The address
 *     is kept for the life of the process: after cudaDeviceReset (or anything else that
 *     destroys the device's primary context) it no longer names the buffer, and this
 *     entry point must not be called again in that process.
 *   - Nothing in the buffer has to start at zero: each call writes every partial it
 *     reads.
 *   - One buffer per device, shared by all calls: two calls on one device that may run
 *     at the same time (different streams with no ordering between them) race on it and
 *     give wrong results. Calls issued on one stream are ordered and safe. */
#define FLEX_DECODE_ATTENTION_STATIC_MAX_BYTES (8LL << 20)
int flex_decode_attention_noalloc(const flex_kv_cache* cache, const void* q, const void* k_new,
                                  const void* v_new, int64_t row_stride, void* o, int32_t batch,
                                  int32_t pos, void* stream);

/* Prefill attention (`mha` core): causal softmax attention on fresh fp16 q, k, v,
 * each [batch][seq][n_heads][head_dim] inside rows of `row_stride` elements per
 * token (token t of sequence b at (b*seq + t)*row_stride). o: fp16
 * [batch][seq][n_heads*head_dim]. head_dim 64 or 128. valid_from: NULL or a device
 * int32 [batch] of left-padding starts, as in flex_kv_cache (keys below it are not
 * attended; rows below it get zeros). */
int flex_prefill_attention(const void* q, const void* k, const void* v, int64_t row_stride,
                           void* o, int32_t batch, int32_t seq, int32_t n_heads,
                           int32_t head_dim, const int32_t* valid_from, void* stream);

/* Dequant-fused weight GEMM: y[m][n] = epi( sum_k x[m][k] * W^[n][k] + bias[n] )
 *   x fp16 [M][K] row-major, W compressed [N][K] (group 64 along K, 4 or 8 bits),
 *   bias fp16 [N] or NULL, residual fp16 [M][N] or NULL (added after bias),
 *   epilogue: FLEX_EPI_NONE, FLEX_EPI_RELU (after bias), FLEX_EPI_RESIDUAL.
 *   y fp16 [M][N]; y may alias residual. ws: flex_gemm_ws_bytes(M, N, K) bytes of
 *   device memory, zero-filled before its first use (its tickets return to zero after
 *   every call); the size depends on the device. It is 0, and ws may be NULL, when the
 *   K splits of a tile reduce through distributed shared memory (thread-block
 *   clusters) or the GEMM is not split.                                          */
#define FLEX_EPI_NONE     0
#define FLEX_EPI_RELU     1
#define FLEX_EPI_RESIDUAL 2
/* OR-ed into `epilogue`: x is stored with every 8-element block of K interleaved as
 * [k0, k4, k1, k5, k2, k6, k3, k7] - the layout the layer calls hand from one kernel to
 * the next (and in which the GEMM needs no permutation of its own). */
#define FLEX_GEMM_X_INTERLEAVED 0x10
int64_t flex_gemm_ws_bytes(int32_t M, int32_t N, int32_t K);
/* The launch plan flex_dequant_gemm takes for this problem on the current device:
 * out[0] the kernel (0 the small-batch GEMV on mma.sync, 1 the 128-row tcgen05 GEMM,
 * 2 the 256-row tcgen05 GEMM), out[1] its output tiles, out[2] the K splits per tile
 * (stream-K: the CTAs that share the tiles' K steps), out[3] how split results are
 * added: 0 through workspace partials and a ticket (or no split), 1 inside a
 * thread-block cluster, 2 stream-K (a tile's first CTA adds the later pieces), 3 an
 * exchange (splits in one wave: each finishes a share of the columns). Needs a
 * current CUDA device (the plan depends on its SM count and cluster occupancy). */
int flex_gemm_plan(int32_t M, int32_t N, int32_t K, int32_t bits, int32_t* out);

/* Stream-K schedule of the 256-row GEMM (on by default): enable = 0 makes later plans
 * use K splits with workspace tickets instead, e.g. for comparison. Process-wide;
 * returns the previous setting. */
int32_t flex_set_gemm_streamk(int32_t enable);
/* The small-batch GEMV route (on by default: int4 weights, at most 32 activation rows):
 * enable = 0 sends those problems to the 128-row tcgen05 GEMM as well, e.g. for
 * comparison. Process-wide; returns the previous setting. A workspace sized under one
 * setting may be too small under the other (FLEX_ERR_WORKSPACE). */
int32_t flex_set_gemm_gemv(int32_t enable);
int flex_dequant_gemm(const void* x, const flexq_tensor* W, const void* bias,
                      const void* residual, void* y, int32_t M, int32_t epilogue,
                      void* ws, int64_t ws_bytes, void* stream);

/* LayerNorm over rows of h fp16 values: y = (x - mean)/sqrt(var + 1e-5) * g + b,
 * biased variance, fp32 statistics. x, y fp16 [rows][h]; may alias. */
int flex_layernorm(const void* x, const void* g, const void* b, void* y, int64_t rows,
                   int32_t h, void* stream);

/* ---- status ------------------------------------------------------------------ */

/* Synchronises `stream`, then returns and clears the device status word of the
 * current device: FLEX_OK, or FLEX_ERR_TIMEOUT if a kernel's bounded wait gave up
 * since the last call, or FLEX_ERR_CUDA if the stream reports an error. The word's
 * device address is looked up once per device and kept for the life of the process,
 * so the library must not be used on a device after cudaDeviceReset (or any other
 * destruction of its primary context) in the same process. */
int flex_get_status(void* stream);

/* Failure detection: limit, in nanoseconds, after which a wait inside the pipeline of
 * the tensor-core GEMM kernel (operand stages, dequantised tiles, MMA completion) gives
 * up. The kernel then records FLEX_ERR_TIMEOUT (read by flex_get_status), stops, lets
 * every copy and MMA it issued finish (those drain waits keep the default limit), and
 * exits; its outputs are unspecified, and the device stays usable. Applies to kernels
 * launched after the call (a captured CUDA graph keeps the limit of its capture time);
 * process-wide. ns = 0 restores the default of 2 s. Returns the previous limit. */
uint64_t flex_set_wait_limit_ns(uint64_t ns);

/* Failure-detection test hook: while `gate` is not NULL, every tensor-core GEMM launched
 * waits, before its first weight load, until the device int32 *gate is non-zero. The
 * wait has the limit of flex_set_wait_limit_ns; when it runs out the kernel takes the
 * timeout path described above. A flag that nothing sets thus makes that path run
 * without breaking any kernel. Process-wide; returns the previous gate. gate must stay
 * valid while kernels launched with it may run. Pass NULL to remove it. */
const int32_t* flex_set_gemm_gate(const int32_t* gate);

/* Layout of the ABI structs as this library was compiled: which = 0 flexq_config,
 * 1 flexq_tensor, 2 flex_layer, 3 flex_kv_cache; field = -1 returns sizeof, field = i
 * the byte offset of the struct's i-th field (declaration order). -1 if out of range.
 * Bindings compare these with their own declarations before any call. */
int64_t flex_abi_layout(int32_t which, int32_t field);

/* Static English text for a status code. */
const char* flex_status_string(int32_t status);

#ifdef __cplusplus
}
#endif

#endif /* FLEXQ_H */
