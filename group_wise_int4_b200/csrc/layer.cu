// OPT decoder layer: prefill (`mha` path) and decode step (`mha_gen` path).
//
// the source-notes page «FlexGen» (PtirisNote), "Flex Opt": per token, layer and gpu-batch the loop
// runs load_weight, load_cache, load_hidden, compute_layer, store_hidden, store_cache;
// compute_layer is the pre-LayerNorm OPT block. Here everything is resident on one
// GPU, so loading is a no-op and a layer call is the fixed launch sequence
//
//   LN1 -> QKV GEMM (+bias, q * d^-1/2) -> attention -> store_cache -> out-proj GEMM
//   (+bias, +x) -> LN2 -> fc1 GEMM (+bias, ReLU) -> fc2 GEMM (+bias, +h1)
//
// on one stream, without host synchronisation, so a caller can capture it in a CUDA
// graph. All intermediates live in the caller's workspace.
#include "common.cuh"

namespace flexq {

int validate_cache(const flex_kv_cache* c);
int validate_weight(const flexq_tensor* W);
int layernorm_launch(const void* x, const void* g, const void* b, void* y, int64_t rows, int h, bool perm,
                     cudaStream_t st);
int append_kv_launch(const flex_kv_cache* c, const void* k_new, const void* v_new, int64_t row_stride, int batch,
                     int seq, int pos0, cudaStream_t st);
int decode_attn_launch(const flex_kv_cache* c, const void* q, const void* k_new, const void* v_new,
                       int64_t row_stride, void* o, int batch, int pos, void* ws, bool perm, cudaStream_t st,
                       bool early_kv);
int64_t decode_attn_ws_bound(int pairs, int head_dim);
int prefill_attn_launch(const void* q, const void* k, const void* v, int64_t row_stride, void* o, int batch,
                        int seq, int n_heads, int head_dim, const int32_t* valid_from, cudaStream_t st);
int64_t gemm_ws_bytes(int M, int N, int K, int bits);
int gemm_launch(const void* x, const flexq_tensor* W, const void* bias, const void* residual, void* y, int M,
                int relu, int nq, float qscale, bool xperm, bool yperm, void* ws, int64_t ws_bytes, cudaStream_t st,
                const KvFuse* kv, bool early_w);

namespace {

inline int64_t align256(int64_t v) { return (v + 255) / 256 * 256; }

struct WsLayout {
    int64_t a, qkv, o, h1, a2, f, attn, gemm, total, gemm_bytes;
};

int check_weight_shape(const flexq_tensor& W, int64_t n, int64_t k) {
    const int rc = validate_weight(&W);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(W.shape[0] == n && W.shape[1] == k, FLEX_ERR_SHAPE);
    return FLEX_OK;
}

int validate_layer(const flex_layer* L) {
    FLEX_REQUIRE(L != nullptr, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(L->h > 0 && L->n_heads > 0 && L->head_dim > 0 && L->ffn > 0, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(L->head_dim == 64 || L->head_dim == 128, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(static_cast<int64_t>(L->n_heads) * L->head_dim == L->h, FLEX_ERR_SHAPE);
    FLEX_REQUIRE(L->h % 256 == 0 && L->ffn % 256 == 0 && L->h <= 12288, FLEX_ERR_SHAPE);
    FLEX_REQUIRE(L->ln1_g && L->ln1_b && L->ln2_g && L->ln2_b, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(L->b_qkv && L->b_o && L->b_fc1 && L->b_fc2, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(aligned16(L->ln1_g) && aligned16(L->ln1_b) && aligned16(L->ln2_g) && aligned16(L->ln2_b) &&
                     aligned16(L->b_qkv) && aligned16(L->b_o) && aligned16(L->b_fc1) && aligned16(L->b_fc2),
                 FLEX_ERR_ALIGN);
    int rc = check_weight_shape(L->w_qkv, 3LL * L->h, L->h);
    if (rc == FLEX_OK) rc = check_weight_shape(L->w_o, L->h, L->h);
    if (rc == FLEX_OK) rc = check_weight_shape(L->w_fc1, L->ffn, L->h);
    if (rc == FLEX_OK) rc = check_weight_shape(L->w_fc2, L->h, L->ffn);
    return rc;
}

WsLayout layout(const flex_layer* L, int batch, int seq) {
    const int64_t T = static_cast<int64_t>(batch) * seq;
    WsLayout w{};
    int64_t off = 0;
    w.a = off;    off += align256(T * L->h * 2);
    w.qkv = off;  off += align256(T * 3 * L->h * 2);
    w.o = off;    off += align256(T * L->h * 2);
    w.h1 = off;   off += align256(T * L->h * 2);
    w.a2 = off;   off += align256(T * L->h * 2);
    w.f = off;    off += align256(T * L->ffn * 2);
    w.attn = off;
    if (seq == 1) off += align256(decode_attn_ws_bound(batch * L->n_heads, L->head_dim));
    w.gemm = off;
    const int M = static_cast<int>(T);
    int64_t g = 0;
    const int bits[4] = {L->w_qkv.cfg.num_bits, L->w_o.cfg.num_bits, L->w_fc1.cfg.num_bits, L->w_fc2.cfg.num_bits};
    const int64_t nk[4][2] = {{3LL * L->h, L->h}, {L->h, L->h}, {L->ffn, L->h}, {L->h, L->ffn}};
    for (int i = 0; i < 4; ++i) {
        const int64_t b = gemm_ws_bytes(M, static_cast<int>(nk[i][0]), static_cast<int>(nk[i][1]), bits[i]);
        if (b > g) g = b;
    }
    w.gemm_bytes = g;
    off += align256(g);
    w.total = off;
    return w;
}

// One layer call over `nc` gpu-batches of `batch` sequences each, gpu-batch c with its
// own cache C[c]: the LayerNorms and the four weight GEMMs run once over all nc * batch
// * seq activation rows (each weight is streamed once for all gpu-batches), attention
// runs per gpu-batch on its own cache, and the QKV epilogue stores every row's key and
// value into its gpu-batch's cache.
int run_layer(const flex_layer* L, const flex_kv_cache* C, int nc, const void* x_in, void* x_out, int batch, int seq,
              int pos, void* ws, int64_t ws_bytes, cudaStream_t st) {
    const WsLayout w = layout(L, nc * batch, seq);
    FLEX_REQUIRE(ws != nullptr && ws_bytes >= w.total, FLEX_ERR_WORKSPACE);
    FLEX_REQUIRE(aligned16(ws), FLEX_ERR_ALIGN);
    char* base = static_cast<char*>(ws);
    void* a = base + w.a;
    __half* qkv = reinterpret_cast<__half*>(base + w.qkv);
    __half* o = reinterpret_cast<__half*>(base + w.o);
    void* h1 = base + w.h1;
    void* a2 = base + w.a2;
    void* f = base + w.f;
    void* gws = base + w.gemm;
    const int64_t T = static_cast<int64_t>(nc) * batch * seq;
    const int64_t Tc = static_cast<int64_t>(batch) * seq;      // rows of one gpu-batch
    const int M = static_cast<int>(T);
    const int h = L->h;
    const float qscale = 1.0f / sqrtf(static_cast<float>(L->head_dim));
    // a, a2, f and the decode attention output are written in the interleaved 8-block
    // order that the GEMM's unpack produces for its weights (see gemm.cu); h1, qkv and
    // the prefill attention output stay in natural order.
    const bool dec = (seq == 1);
    // the QKV epilogue also quantises the new keys/values into their cache slots
    // (store_cache): slot pos for a decode step, slots [0, seq) for a prompt
    const KvFuse kv{C, nc, static_cast<int>(Tc), h, seq, dec ? pos : 0};
    int rc = layernorm_launch(x_in, L->ln1_g, L->ln1_b, a, T, h, true, st);
    if (rc == FLEX_OK)
        rc = gemm_launch(a, &L->w_qkv, L->b_qkv, nullptr, qkv, M, 0, h, qscale, true, false, gws, w.gemm_bytes, st, &kv, true);
    for (int c = 0; c < nc && rc == FLEX_OK; ++c) {
        const __half* qc = qkv + c * Tc * 3 * h;
        __half* oc = o + c * Tc * h;
        if (dec)
            rc = decode_attn_launch(&C[c], qc, qc + h, qc + 2 * h, 3LL * h, oc, batch, pos, base + w.attn, true, st, true);
        else
            rc = prefill_attn_launch(qc, qc + h, qc + 2 * h, 3LL * h, oc, batch, seq, L->n_heads, L->head_dim,
                                     C[c].valid_from, st);
    }
    if (rc == FLEX_OK)
        rc = gemm_launch(o, &L->w_o, L->b_o, x_in, h1, M, 0, 0, 1.f, dec, false, gws, w.gemm_bytes, st, nullptr, true);
    if (rc == FLEX_OK) rc = layernorm_launch(h1, L->ln2_g, L->ln2_b, a2, T, h, true, st);
    if (rc == FLEX_OK)
        rc = gemm_launch(a2, &L->w_fc1, L->b_fc1, nullptr, f, M, 1, 0, 1.f, true, true, gws, w.gemm_bytes, st, nullptr, true);
    if (rc == FLEX_OK)
        rc = gemm_launch(f, &L->w_fc2, L->b_fc2, h1, x_out, M, 0, 0, 1.f, true, false, gws, w.gemm_bytes, st, nullptr, true);
    return rc;
}

int check_cache_for_layer(const flex_layer* L, const flex_kv_cache* C) {
    const int rc = validate_cache(C);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(C->n_heads == L->n_heads && C->head_dim == L->head_dim, FLEX_ERR_SHAPE);
    return FLEX_OK;
}

// Every cache valid for the layer and of the same geometry as the first; batch fits.
int check_caches(const flex_layer* L, const flex_kv_cache* C, int nc, int batch, bool exact_batch) {
    FLEX_REQUIRE(C != nullptr && nc >= 1 && nc <= kMaxKvBatches, FLEX_ERR_INVALID_ARG);
    for (int c = 0; c < nc; ++c) {
        const int rc = check_cache_for_layer(L, &C[c]);
        if (rc != FLEX_OK) return rc;
        FLEX_REQUIRE(C[c].max_seq == C[0].max_seq && C[c].cfg.num_bits == C[0].cfg.num_bits &&
                         C[c].cfg.group_size == C[0].cfg.group_size,
                     FLEX_ERR_SHAPE);
        FLEX_REQUIRE(batch > 0 && (exact_batch ? batch == C[c].batch : batch <= C[c].batch), FLEX_ERR_INVALID_ARG);
    }
    return FLEX_OK;
}

int prefill(const flex_layer* L, const flex_kv_cache* C, int nc, const void* x_in, void* x_out, int32_t batch,
            int32_t seq, void* ws, int64_t ws_bytes, void* stream) {
    int rc = validate_layer(L);
    if (rc == FLEX_OK) rc = check_caches(L, C, nc, batch, true);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(x_in && x_out && x_in != x_out, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(aligned16(x_in) && aligned16(x_out), FLEX_ERR_ALIGN);
    FLEX_REQUIRE(seq > 0 && seq <= C[0].max_seq, FLEX_ERR_SHAPE);
    FLEX_REQUIRE(static_cast<int64_t>(nc) * batch * seq < (1LL << 31), FLEX_ERR_SHAPE);
    return run_layer(L, C, nc, x_in, x_out, batch, seq, 0, ws, ws_bytes, as_stream(stream));
}

int decode(const flex_layer* L, const flex_kv_cache* C, int nc, const void* x_in, void* x_out, int32_t batch,
           int32_t pos, void* ws, int64_t ws_bytes, void* stream) {
    int rc = validate_layer(L);
    if (rc == FLEX_OK) rc = check_caches(L, C, nc, batch, false);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(x_in && x_out && x_in != x_out, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(aligned16(x_in) && aligned16(x_out), FLEX_ERR_ALIGN);
    FLEX_REQUIRE(pos >= 0 && pos < C[0].max_seq, FLEX_ERR_SHAPE);
    return run_layer(L, C, nc, x_in, x_out, batch, 1, pos, ws, ws_bytes, as_stream(stream));
}

}  // namespace
}  // namespace flexq

using namespace flexq;

extern "C" int64_t flex_workspace_bytes(const flex_layer* L, int32_t batch, int32_t seq) {
    const int rc = validate_layer(L);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(batch > 0 && seq > 0, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(static_cast<int64_t>(batch) * seq < (1LL << 31), FLEX_ERR_SHAPE);
    return layout(L, batch, seq).total;
}

extern "C" int flex_prefill_layer(const flex_layer* L, const flex_kv_cache* cache, const void* x_in, void* x_out,
                                  int32_t batch, int32_t seq, void* ws, int64_t ws_bytes, void* stream) {
    return prefill(L, cache, 1, x_in, x_out, batch, seq, ws, ws_bytes, stream);
}

extern "C" int flex_decode_layer(const flex_layer* L, const flex_kv_cache* cache, const void* x_in, void* x_out,
                                 int32_t batch, int32_t pos, void* ws, int64_t ws_bytes, void* stream) {
    return decode(L, cache, 1, x_in, x_out, batch, pos, ws, ws_bytes, stream);
}

extern "C" int flex_prefill_layer_batches(const flex_layer* L, const flex_kv_cache* caches, int32_t num_batches,
                                          const void* x_in, void* x_out, int32_t batch, int32_t seq, void* ws,
                                          int64_t ws_bytes, void* stream) {
    return prefill(L, caches, num_batches, x_in, x_out, batch, seq, ws, ws_bytes, stream);
}

extern "C" int flex_decode_layer_batches(const flex_layer* L, const flex_kv_cache* caches, int32_t num_batches,
                                         const void* x_in, void* x_out, int32_t batch, int32_t pos, void* ws,
                                         int64_t ws_bytes, void* stream) {
    return decode(L, caches, num_batches, x_in, x_out, batch, pos, ws, ws_bytes, stream);
}
