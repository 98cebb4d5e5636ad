// store_cache (flex_append_kv) and LayerNorm.
//
// store_cache: the source-notes page «FlexGen» (PtirisNote), "Flex Opt" - the step's new key/value are
// written to the cache after compute_layer; the walkthrough page «FlexGen 单 GPU 高吞吐大模型推理引擎：论文解读与源码实战指南», section 6.3 -
// with --compress-cache they are stored group-wise quantised, 4 bits, group 64, along
// the head dimension. The arithmetic is the shared quantiser (quant.cuh), so slot
// contents equal flexq_compress of the same fp16 values bit for bit.
//
// LayerNorm: the OPT block's pre-attention and pre-FFN normalisation,
// y = (x - mean) / sqrt(var + 1e-5) * g + b with biased variance; statistics in fp32,
// two passes over registers (exact mean first, then the centred second moment).
#include "quant.cuh"

namespace flexq {
namespace {

// One group of GS values per GS/8 lanes; groups enumerate (tensor, sequence, token,
// head, group). Token t of sequence b comes from row (b*seq + t) of the source and goes
// to cache slot pos0 + t.
template <int BITS, int GS>
__global__ void __launch_bounds__(256) append_kv_kernel(const __half* __restrict__ k_new,
                                                        const __half* __restrict__ v_new,
                                                        int64_t row_stride, uint8_t* __restrict__ k_codes,
                                                        uint32_t* __restrict__ k_meta,
                                                        uint8_t* __restrict__ v_codes,
                                                        uint32_t* __restrict__ v_meta, int batch, int seq,
                                                        int n_heads, int head_dim, int max_seq, int pos0) {
    constexpr int L = GS / 8;
    pdl_wait();
    pdl_trigger();
    const int gph = head_dim / GS;                              // groups per head
    const int64_t per_tensor = static_cast<int64_t>(batch) * seq * n_heads * gph;
    const int64_t total = 2 * per_tensor;
    const int lane = threadIdx.x & 31;
    const int sub = lane % L;
    const int64_t gidx = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / L;
    const bool valid = gidx < total;
    const int64_t g = valid ? gidx : 0;
    const int which = static_cast<int>(g / per_tensor);        // 0 = key, 1 = value
    int64_t r = g % per_tensor;
    const int gi = static_cast<int>(r % gph);
    r /= gph;
    const int head = static_cast<int>(r % n_heads);
    r /= n_heads;                                               // b * seq + t
    const int t = static_cast<int>(r % seq);
    const int64_t b = r / seq;
    const __half* src = (which == 0 ? k_new : v_new) + r * row_stride + head * head_dim + gi * GS + sub * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (valid) v = *reinterpret_cast<const uint4*>(src);
    __half2 hmn, hmx;
    minmax8(v, hmn, hmx);
    float mn = hmin_of(hmn), mx = hmax_of(hmx);
#pragma unroll
    for (int off = 1; off < L; off <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    const __half s16 = group_scale16<BITS>(mn, mx);
    const float s = __half2float(s16);
    if (!valid) return;
    const int64_t slot = (b * n_heads + head) * max_seq + pos0 + t;   // [b][nh][max_seq]
    uint8_t* codes = (which == 0 ? k_codes : v_codes) + slot * (head_dim * BITS / 8) + gi * (GS * BITS / 8);
    uint32_t* meta = (which == 0 ? k_meta : v_meta) + slot * gph + gi;
    if (BITS == 4)
        *reinterpret_cast<uint32_t*>(codes + sub * 4) = quant8_4bit(v, mn, s);
    else
        *reinterpret_cast<uint2*>(codes + sub * 8) = quant8_8bit(v, mn, s);
    if (sub == 0) *meta = pack_half2_bits(stored_min16(mn), s16);
}

// LayerNorm: one CTA of LN_THREADS per row, each thread keeps up to LN_VPT 16-byte
// vectors of the row in registers.
constexpr int LN_THREADS = 128;
constexpr int LN_VPT = 12;   // 128 threads * 12 vectors * 8 = 12288 values per row

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    const int w = threadIdx.x >> 5;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < LN_THREADS / 32; ++i) t += red[i];
    return t;
}

// PERM: write each 8-value block in the interleaved order [x0 x4 x1 x5 x2 x6 x3 x7] that
// the GEMM's unpack produces for the weights (see gemm.cu), so that the GEMM needs no
// re-pairing of its dequantised operand.
template <bool PERM>
__global__ void __launch_bounds__(LN_THREADS) layernorm_kernel(const __half* __restrict__ x,
                                                               const __half* __restrict__ g,
                                                               const __half* __restrict__ b,
                                                               __half* __restrict__ y, int h) {
    __shared__ float red[LN_THREADS / 32];
    const int64_t row = blockIdx.x;
    const int nvec = h / 8;
    // the gain and bias are parameters: fetched before waiting for the previous kernel
    const uint4* gr = reinterpret_cast<const uint4*>(g);
    const uint4* br = reinterpret_cast<const uint4*>(b);
    uint4 gv[LN_VPT], bv[LN_VPT];
#pragma unroll
    for (int i = 0; i < LN_VPT; ++i) {
        const int c = threadIdx.x + i * LN_THREADS;
        gv[i] = c < nvec ? __ldg(gr + c) : make_uint4(0, 0, 0, 0);
        bv[i] = c < nvec ? __ldg(br + c) : make_uint4(0, 0, 0, 0);
    }
    pdl_wait();
    pdl_trigger();
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * h);
    uint4 v[LN_VPT];
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < LN_VPT; ++i) {
        const int c = threadIdx.x + i * LN_THREADS;
        v[i] = c < nvec ? xr[c] : make_uint4(0, 0, 0, 0);
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) sum += h2f_lo(w[k]) + h2f_hi(w[k]);
    }
    const float mean = block_sum(sum, red) / static_cast<float>(h);
    float sq = 0.f;
#pragma unroll
    for (int i = 0; i < LN_VPT; ++i) {
        const int c = threadIdx.x + i * LN_THREADS;
        if (c >= nvec) continue;
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float a = h2f_lo(w[k]) - mean, bb = h2f_hi(w[k]) - mean;
            sq += a * a + bb * bb;
        }
    }
    const float var = block_sum(sq, red) / static_cast<float>(h);
    const float rstd = rsqrtf(var + 1e-5f);
    uint4* yr = reinterpret_cast<uint4*>(y + row * h);
#pragma unroll
    for (int i = 0; i < LN_VPT; ++i) {
        const int c = threadIdx.x + i * LN_THREADS;
        if (c >= nvec) continue;
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        const uint32_t gw[4] = {gv[i].x, gv[i].y, gv[i].z, gv[i].w};
        const uint32_t bw[4] = {bv[i].x, bv[i].y, bv[i].z, bv[i].w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float lo = (h2f_lo(w[k]) - mean) * rstd * h2f_lo(gw[k]) + h2f_lo(bw[k]);
            const float hi = (h2f_hi(w[k]) - mean) * rstd * h2f_hi(gw[k]) + h2f_hi(bw[k]);
            o[k] = pack_half2_bits(__float2half_rn(lo), __float2half_rn(hi));
        }
        if (PERM) {
            uint32_t t[4];
            asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(t[0]) : "r"(o[0]), "r"(o[2]));
            asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(t[1]) : "r"(o[0]), "r"(o[2]));
            asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(t[2]) : "r"(o[1]), "r"(o[3]));
            asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(t[3]) : "r"(o[1]), "r"(o[3]));
            yr[c] = make_uint4(t[0], t[1], t[2], t[3]);
        } else {
            yr[c] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

}  // namespace

int append_kv_launch(const flex_kv_cache* c, const void* k_new, const void* v_new, int64_t row_stride,
                     int batch, int seq, int pos0, cudaStream_t st) {
    const int gs = c->cfg.group_size;
    const int64_t groups = 2LL * batch * seq * c->n_heads * (c->head_dim / gs);
    const int64_t threads = groups * (gs / 8);
    if (threads == 0) return FLEX_OK;
    const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
    const __half* k = static_cast<const __half*>(k_new);
    const __half* v = static_cast<const __half*>(v_new);
    uint8_t* kc = static_cast<uint8_t*>(c->k_codes);
    uint8_t* vc = static_cast<uint8_t*>(c->v_codes);
    uint32_t* km = static_cast<uint32_t*>(c->k_meta);
    uint32_t* vm = static_cast<uint32_t*>(c->v_meta);
#define APPEND(B, G)                                                                                    \
    launch_k(append_kv_kernel<B, G>, dim3(blocks), dim3(256), 0, st, true, k, v, row_stride, kc, km, vc, vm, \
             batch, seq, c->n_heads, c->head_dim, c->max_seq, pos0)
    if (c->cfg.num_bits == 4) {
        if (gs == 32) APPEND(4, 32); else if (gs == 64) APPEND(4, 64); else APPEND(4, 128);
    } else {
        if (gs == 32) APPEND(8, 32); else if (gs == 64) APPEND(8, 64); else APPEND(8, 128);
    }
#undef APPEND
    return launch_status();
}

int validate_cache(const flex_kv_cache* c) {
    FLEX_REQUIRE(c != nullptr, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(c->k_codes && c->k_meta && c->v_codes && c->v_meta, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(c->batch > 0 && c->n_heads > 0 && c->max_seq > 0, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(c->head_dim == 64 || c->head_dim == 128, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(c->cfg.symmetric == 0, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(c->cfg.num_bits == 4 || c->cfg.num_bits == 8, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(c->cfg.group_size == 32 || c->cfg.group_size == 64, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(c->head_dim % c->cfg.group_size == 0, FLEX_ERR_SHAPE);
    FLEX_REQUIRE(c->cfg.group_dim == 3 || c->cfg.group_dim == -1, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(aligned16(c->k_codes) && aligned16(c->v_codes) && aligned16(c->k_meta) &&
                     aligned16(c->v_meta),
                 FLEX_ERR_ALIGN);
    FLEX_REQUIRE(c->valid_from == nullptr || (reinterpret_cast<uintptr_t>(c->valid_from) & 3u) == 0, FLEX_ERR_ALIGN);
    return FLEX_OK;
}

int layernorm_launch(const void* x, const void* g, const void* b, void* y, int64_t rows, int h, bool perm,
                     cudaStream_t st) {
    if (rows == 0) return FLEX_OK;
    const __half* xh = static_cast<const __half*>(x);
    const __half* gh = static_cast<const __half*>(g);
    const __half* bh = static_cast<const __half*>(b);
    __half* yh = static_cast<__half*>(y);
    const dim3 grid(static_cast<unsigned>(rows));
    if (perm)
        launch_k(layernorm_kernel<true>, grid, dim3(LN_THREADS), 0, st, true, xh, gh, bh, yh, h);
    else
        launch_k(layernorm_kernel<false>, grid, dim3(LN_THREADS), 0, st, true, xh, gh, bh, yh, h);
    return launch_status();
}

}  // namespace flexq

using namespace flexq;

extern "C" int flex_append_kv(const flex_kv_cache* cache, const void* k_new, const void* v_new,
                              int64_t row_stride, int32_t batch, int32_t pos, void* stream) {
    int rc = validate_cache(cache);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(k_new && v_new, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(batch > 0 && batch <= cache->batch, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(pos >= 0 && pos < cache->max_seq, FLEX_ERR_SHAPE);
    FLEX_REQUIRE(row_stride >= static_cast<int64_t>(cache->n_heads) * cache->head_dim, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(row_stride % 8 == 0, FLEX_ERR_ALIGN);
    FLEX_REQUIRE(aligned16(k_new) && aligned16(v_new), FLEX_ERR_ALIGN);
    return append_kv_launch(cache, k_new, v_new, row_stride, batch, 1, pos, as_stream(stream));
}

extern "C" int flex_layernorm(const void* x, const void* g, const void* b, void* y, int64_t rows, int32_t h,
                              void* stream) {
    FLEX_REQUIRE(x && g && b && y, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(rows >= 0 && h > 0, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(h % 8 == 0 && h <= LN_THREADS * LN_VPT * 8, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(aligned16(x) && aligned16(g) && aligned16(b) && aligned16(y), FLEX_ERR_ALIGN);
    return layernorm_launch(x, g, b, y, rows, h, false, as_stream(stream));
}
