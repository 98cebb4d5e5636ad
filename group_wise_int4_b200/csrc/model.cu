// Whole-model pieces around the decoder layers: the input embedding, the output head and
// the greedy choice of the next token.
//
// the source-notes page «FlexGen» (PtirisNote), "Flex Opt": the model is an embedding, N
// transformer layers and an output head, and OptLM.generate runs the generation loop;
// "Pytorch Backend": opt_input_embed / opt_output_embed implement the embedding layers.
// The walkthrough page «FlexGen 单 GPU 高吞吐大模型推理引擎：论文解读与源码实战指南», section 4.1: generate(..., do_sample, ...);
// do_sample = False is the greedy choice. The token table E [V][h] is compressed like the
// layer weights (4 bits, group 64 along h) and also serves as the output head (logits =
// LN(h) E^T), as in OPT.
#include "common.cuh"

namespace flexq {

int validate_weight(const flexq_tensor* W);
int layernorm_launch(const void* x, const void* g, const void* b, void* y, int64_t rows, int h, bool perm,
                     cudaStream_t st);
int64_t gemm_ws_bytes(int M, int N, int K, int bits);
int gemm_launch(const void* x, const flexq_tensor* W, const void* bias, const void* residual, void* y, int M,
                int relu, int nq, float qscale, bool xperm, bool yperm, void* ws, int64_t ws_bytes, cudaStream_t st,
                const KvFuse* kv, bool early_w);

namespace {

constexpr int kThreads = 256;

// x[r][8c .. 8c+7] = fp16(E^[tokens[r]][..] + P[positions[r]][..]). E^ is the codec's
// dequantisation (fp16(fl(q * fl(1/scale)) + min), or min for a constant group); the sum
// of the two fp16 values is formed exactly (in fp64) and rounded to fp16 once. An id or
// position outside the tables is clamped into range and recorded as
// FLEX_ERR_INVALID_ARG in the status word.
__global__ void __launch_bounds__(kThreads) embed_kernel(const uint8_t* __restrict__ codes,
                                                         const uint32_t* __restrict__ meta,
                                                         const __half* __restrict__ P,
                                                         const int32_t* __restrict__ tokens,
                                                         const int32_t* __restrict__ positions, int64_t n, int h,
                                                         int V, int max_pos, __half* __restrict__ x, int* status) {
    pdl_wait();
    pdl_trigger();
    const int chunks = h / 8;
    for (int64_t it = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; it < n * chunks;
         it += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = it / chunks;
        const int c = static_cast<int>(it % chunks);
        int t = tokens[r], p = positions[r];
        if (t < 0 || t >= V || p < 0 || p >= max_pos) {
            set_status(status, FLEX_ERR_INVALID_ARG);
            t = min(max(t, 0), V - 1);
            p = min(max(p, 0), max_pos - 1);
        }
        const uint32_t w = *reinterpret_cast<const uint32_t*>(codes + static_cast<int64_t>(t) * (h / 2) + c * 4);
        const uint32_t mw = meta[static_cast<int64_t>(t) * (h / 64) + (c * 8) / 64];
        const __half mn16 = __ushort_as_half(static_cast<unsigned short>(mw & 0xFFFFu));
        const float s = h2f_hi(mw), mn = __half2float(mn16);
        const float step = s > 0.0f ? __fdiv_rn(1.0f, s) : 0.0f;
        const uint4 pv = *reinterpret_cast<const uint4*>(P + static_cast<int64_t>(p) * h + c * 8);
        const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
        __half o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t q = (w >> (4 * j)) & 15u;
            const __half e = s > 0.0f ? __float2half_rn(__fadd_rn(__fmul_rn(static_cast<float>(q), step), mn)) : mn16;
            const float pf = (j & 1) ? h2f_hi(pw[j >> 1]) : h2f_lo(pw[j >> 1]);
            o[j] = __double2half(__dadd_rn(static_cast<double>(__half2float(e)), static_cast<double>(pf)));
        }
        *reinterpret_cast<uint4*>(x + r * h + c * 8) =
            make_uint4(pack_half2_bits(o[0], o[1]), pack_half2_bits(o[2], o[3]), pack_half2_bits(o[4], o[5]),
                       pack_half2_bits(o[6], o[7]));
    }
}

// next[r] = the column of the largest of logits[r][0 .. V) (fp16 rows of `ld` values),
// the lowest column among equal ones. One CTA per row.
__global__ void __launch_bounds__(kThreads) argmax_kernel(const __half* __restrict__ logits, int64_t ld, int V,
                                                          int32_t* __restrict__ next) {
    pdl_wait();
    pdl_trigger();
    const int64_t r = blockIdx.x;
    const __half* row = logits + r * ld;
    float best = -INFINITY;
    int bi = 0x7FFFFFFF;
    for (int i = threadIdx.x; i < V; i += blockDim.x) {
        const float v = __half2float(row[i]);
        if (v > best) {               // i increases: the first maximum of this thread's columns
            best = v;
            bi = i;
        }
    }
    // (value, column) pairs: larger value wins, then the lower column
    auto better = [](float v, int i, float bv, int b) { return v > bv || (v == bv && i < b); };
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float v = __shfl_xor_sync(0xffffffffu, best, off);
        const int i = __shfl_xor_sync(0xffffffffu, bi, off);
        if (better(v, i, best, bi)) {
            best = v;
            bi = i;
        }
    }
    __shared__ float sv[kThreads / 32];
    __shared__ int si[kThreads / 32];
    if ((threadIdx.x & 31) == 0) {
        sv[threadIdx.x >> 5] = best;
        si[threadIdx.x >> 5] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kThreads / 32; ++w)
            if (better(sv[w], si[w], best, bi)) {
                best = sv[w];
                bi = si[w];
            }
        next[r] = bi == 0x7FFFFFFF ? 0 : bi;
    }
}

inline int64_t align256(int64_t v) { return (v + 255) / 256 * 256; }

int check_table(const flexq_tensor* E, int32_t vocab) {
    int rc = validate_weight(E);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(E->cfg.num_bits == 4, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(vocab > 0 && vocab <= E->shape[0], FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(E->shape[1] <= 12288, FLEX_ERR_SHAPE);            // one LayerNorm CTA per row
    return FLEX_OK;
}

struct HeadLayout {
    int64_t a, logits, gemm, total, gemm_bytes;
};

HeadLayout head_layout(const flexq_tensor* E, int64_t n, bool own_logits) {
    HeadLayout w{};
    const int64_t N = E->shape[0], h = E->shape[1];
    int64_t off = 0;
    w.a = off;
    off += align256(n * h * 2);
    w.logits = off;
    if (own_logits) off += align256(n * N * 2);
    w.gemm = off;
    w.gemm_bytes = gemm_ws_bytes(static_cast<int>(n), static_cast<int>(N), static_cast<int>(h), 4);
    off += align256(w.gemm_bytes);
    w.total = off;
    return w;
}

}  // namespace
}  // namespace flexq

using namespace flexq;

extern "C" int flex_embed(const flexq_tensor* E, int32_t vocab, const void* P, int32_t max_pos,
                          const int32_t* tokens, const int32_t* positions, int64_t n, void* x, void* stream) {
    const int rc = check_table(E, vocab);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(P && tokens && positions && x && max_pos > 0 && n >= 0, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(aligned16(P) && aligned16(x) && (reinterpret_cast<uintptr_t>(tokens) & 3u) == 0 &&
                     (reinterpret_cast<uintptr_t>(positions) & 3u) == 0,
                 FLEX_ERR_ALIGN);
    if (n == 0) return FLEX_OK;
    const int h = static_cast<int>(E->shape[1]);
    const int64_t work = n * (h / 8);
    int64_t blocks = (work + kThreads - 1) / kThreads;
    if (blocks > 8LL * sm_count()) blocks = 8LL * sm_count();
    launch_k(embed_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0, as_stream(stream), true,
             static_cast<const uint8_t*>(E->codes), static_cast<const uint32_t*>(E->meta),
             static_cast<const __half*>(P), tokens, positions, n, h, static_cast<int>(vocab), static_cast<int>(max_pos),
             static_cast<__half*>(x), status_word());
    return launch_status();
}

extern "C" int64_t flex_lm_head_ws_bytes(const flexq_tensor* E, int32_t vocab, int64_t n, int32_t with_logits) {
    const int rc = check_table(E, vocab);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(n > 0 && n < (1LL << 31), FLEX_ERR_INVALID_ARG);
    return head_layout(E, n, with_logits == 0).total;
}

extern "C" int flex_lm_head_argmax(const flexq_tensor* E, int32_t vocab, const void* lnf_g, const void* lnf_b,
                                   const void* x, int64_t n, int32_t* next, void* logits, void* ws,
                                   int64_t ws_bytes, void* stream) {
    int rc = check_table(E, vocab);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(lnf_g && lnf_b && x && next, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(n > 0 && n < (1LL << 31), FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(aligned16(lnf_g) && aligned16(lnf_b) && aligned16(x) && (!logits || aligned16(logits)) &&
                     (reinterpret_cast<uintptr_t>(next) & 3u) == 0,
                 FLEX_ERR_ALIGN);
    const HeadLayout w = head_layout(E, n, logits == nullptr);
    FLEX_REQUIRE(ws != nullptr && ws_bytes >= w.total, FLEX_ERR_WORKSPACE);
    FLEX_REQUIRE(aligned16(ws), FLEX_ERR_ALIGN);
    const cudaStream_t st = as_stream(stream);
    char* base = static_cast<char*>(ws);
    void* a = base + w.a;
    __half* lg = logits ? static_cast<__half*>(logits) : reinterpret_cast<__half*>(base + w.logits);
    const int h = static_cast<int>(E->shape[1]);
    const int64_t N = E->shape[0];
    // the final LayerNorm writes its output in the interleaved 8-block order the GEMM reads
    rc = layernorm_launch(x, lnf_g, lnf_b, a, n, h, true, st);
    if (rc == FLEX_OK)
        rc = gemm_launch(a, E, nullptr, nullptr, lg, static_cast<int>(n), 0, 0, 1.f, true, false, base + w.gemm,
                         w.gemm_bytes, st, nullptr, true);
    if (rc != FLEX_OK) return rc;
    launch_k(argmax_kernel, dim3(static_cast<unsigned>(n)), dim3(kThreads), 0, st, true,
             static_cast<const __half*>(lg), N, static_cast<int>(vocab), next);
    return launch_status();
}
