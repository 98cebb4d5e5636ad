// Oracle in plain C++17, IEEE binary32 - TEST INFRASTRUCTURE ONLY.
//
// Nothing in the product path may link, load or call this file. Only the test-suite,
// the smoke check and the CPU-baseline / reference legs of the benchmark use it. It
// shares no code, header, table or helper with the CUDA library; it is a second,
// independent statement of what the hot path computes, written as plain loops.
//
// Sources (the web pages on FlexGen's group-wise int4 method):
//   - the walkthrough page «FlexGen 单 GPU 高吞吐大模型推理引擎：论文解读与源码实战指南», section 6.3
//     (4-bit group-wise quantisation of weights and KV cache): groups of group_size
//     along group_dim, min/max quantisation to unsigned num_bits codes, two 4-bit codes
//     per byte, a per-group fp16 scale;
//   - the source-notes page «FlexGen» (PtirisNote), "Pytorch Backend" (mha is the prefill
//     attention, mha_gen the decode step) and "Flex Opt" (each step runs load_cache,
//     compute_layer, store_cache: the new token's key/value enter the cache after the
//     layer has used them).
//
// Readings where the pages leave a step open (the same as the numpy oracle's):
//   codes q = clamp(rint(fl(fl(x - min) * s)), 0, 2^b - 1) with s = fp16((2^b - 1) / (max - min))
//   (the stored scale; 0 for a constant group, 65504 on overflow), ties to even; metadata
//   {fp16 min, fp16 scale} per group; the even element of a pair in the low nibble;
//   x^ = fp16(fl(fl(q * fl(1/s)) + min)), or min when s = 0.
//   OPT pre-LayerNorm block, LayerNorm eps 1e-5 with the biased variance; fused QKV rows
//   [q; k; v] with feature = head * head_dim + j; q = (a Wq^T + bq) / sqrt(head_dim);
//   keys/values rounded to fp16 before they are quantised into the cache; prefill
//   attends to the fresh keys/values of the prompt, a decode step at pos to the
//   dequantised cache slots [0, pos) and to its own fresh key/value.
//
// Arithmetic: every operation is a single binary32 operation rounded to nearest even.
// Build with -ffp-contract=off so that no multiply-add is fused. Sums run in index order
// (sequentially over the reduced index). Matrix products process several tokens per
// weight row at once only to reuse the row from cache; each output element is still one
// sequential sum over the input features, so the results do not depend on that blocking
// nor on the number of threads.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ---- IEEE binary16 <-> binary32 ------------------------------------------------------
float half_to_float(uint16_t h) {
    const uint32_t sign = (h >> 15) & 1u, exp = (h >> 10) & 0x1Fu, man = h & 0x3FFu;
    float v;
    if (exp == 0) {
        v = std::ldexp(static_cast<float>(man), -24);          // zero or subnormal: man * 2^-24, exact
    } else if (exp == 31) {
        v = man ? std::nanf("") : INFINITY;
    } else {
        const uint32_t bits = ((exp + 112u) << 23) | (man << 13);
        std::memcpy(&v, &bits, 4);
    }
    return sign ? -v : v;
}

// Round to nearest, ties to even.
uint16_t float_to_half(float f) {
    uint32_t x;
    std::memcpy(&x, &f, 4);
    const uint16_t sign = static_cast<uint16_t>((x >> 16) & 0x8000u);
    const uint32_t ax = x & 0x7FFFFFFFu;
    if (ax >= 0x7F800000u) return sign | (ax > 0x7F800000u ? 0x7E00u : 0x7C00u);   // NaN, Inf
    if (ax >= 0x477FF000u) return sign | 0x7C00u;              // >= 65520 rounds to infinity
    if (ax < 0x38800000u) {                                    // below 2^-14: a subnormal (or 0)
        float a;
        std::memcpy(&a, &ax, 4);
        const float units = std::nearbyint(a * 16777216.0f);   // a / 2^-24, exact scaling, then RNE
        return sign | static_cast<uint16_t>(units);            // 1024 units = the smallest normal
    }
    uint32_t h = (((ax >> 23) - 112u) << 10) | ((ax & 0x7FFFFFu) >> 13);
    const uint32_t rem = ax & 0x1FFFu;
    if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) ++h;   // a carry moves into the exponent
    return sign | static_cast<uint16_t>(h);
}

struct HalfTable {
    float v[65536];
    HalfTable() {
        for (uint32_t i = 0; i < 65536; ++i) v[i] = half_to_float(static_cast<uint16_t>(i));
    }
};
const HalfTable& table() {
    static const HalfTable t;
    return t;
}
inline float hf(uint16_t h) { return table().v[h]; }

template <class F>
void parallel_for(int64_t n, int nthreads, F fn) {
    if (nthreads <= 1 || n < 2) {
        fn(int64_t(0), n);
        return;
    }
    const int64_t T = std::min<int64_t>(nthreads, n);
    const int64_t chunk = (n + T - 1) / T;
    std::vector<std::thread> th;
    for (int64_t t = 0; t < T; ++t) {
        const int64_t b = t * chunk, e = std::min(n, b + chunk);
        if (b < e) th.emplace_back(fn, b, e);
    }
    for (auto& x : th) x.join();
}

// ---- the quantiser -------------------------------------------------------------------
// One group of gs values (fp16 values as floats) -> codes q[gs] and {min, scale} bits.
void quantise_group(const float* v, int gs, int bits, uint8_t* q, uint16_t* mn16, uint16_t* s16) {
    const float levels = static_cast<float>((1 << bits) - 1);
    float mn = v[0], mx = v[0];
    for (int j = 1; j < gs; ++j) {
        mn = std::min(mn, v[j]);
        mx = std::max(mx, v[j]);
    }
    const float r = mx - mn;
    uint16_t sc = 0;
    if (r > 0.0f) {
        const float s32 = levels / r;
        sc = float_to_half(s32);
        if ((sc & 0x7FFFu) == 0x7C00u) sc = 0x7BFFu;           // overflow: saturate to 65504
    }
    const float s = hf(sc);
    for (int j = 0; j < gs; ++j) {
        const float d = v[j] - mn;
        const float t = d * s;
        float c = std::nearbyint(t);
        if (c < 0.0f) c = 0.0f;
        if (c > levels) c = levels;
        q[j] = static_cast<uint8_t>(c);
    }
    *mn16 = float_to_half(mn + 0.0f);                          // exact; a zero minimum is stored as +0
    *s16 = sc;
}

// x^ of one code under {min, scale}.
inline uint16_t dequantise_one(uint32_t q, uint16_t mn16, uint16_t s16) {
    const float s = hf(s16);
    if (!(s > 0.0f)) return mn16;
    const float step = 1.0f / s;
    const float p = static_cast<float>(q) * step;
    const float x = p + hf(mn16);
    return float_to_half(x);
}

struct Dims {
    int64_t outer, G, inner;
};

bool dims_of(int ndim, const int64_t* shape, int gd, int gs, Dims* d) {
    if (ndim < 1 || ndim > 4) return false;
    if (gd < 0) gd += ndim;
    if (gd < 0 || gd >= ndim) return false;
    d->outer = 1;
    d->inner = 1;
    for (int i = 0; i < gd; ++i) d->outer *= shape[i];
    for (int i = gd + 1; i < ndim; ++i) d->inner *= shape[i];
    d->G = shape[gd];
    return d->G % gs == 0;
}

bool config_ok(int bits, int gs) { return (bits == 4 || bits == 8) && (gs == 32 || gs == 64 || gs == 128); }

}  // namespace

extern "C" {

float fo_half_to_float(uint16_t h) { return half_to_float(h); }
uint16_t fo_float_to_half(float f) { return float_to_half(f); }
void fo_float_to_half_n(const float* f, int64_t n, uint16_t* h) {
    for (int64_t i = 0; i < n; ++i) h[i] = float_to_half(f[i]);
}

// compress: x fp16 (bits) of `shape` -> codes (the pages' packed shape) and meta
// (shape[:gd] + (ng,) + shape[gd+1:] + (2,) fp16 bits {min, scale}). 0 or -1.
int fo_compress(const uint16_t* x, int ndim, const int64_t* shape, int bits, int gs, int gd, uint8_t* codes,
                uint16_t* meta, int nthreads) {
    Dims D;
    if (!config_ok(bits, gs) || !dims_of(ndim, shape, gd, gs, &D)) return -1;
    const int64_t ng = D.G / gs, bpg = gs * bits / 8, cG = ng * bpg;
    parallel_for(D.outer * ng, nthreads, [&](int64_t b, int64_t e) {
        std::vector<float> v(gs);
        std::vector<uint8_t> q(gs);
        for (int64_t og = b; og < e; ++og) {
            const int64_t o = og / ng, g = og % ng;
            for (int64_t i = 0; i < D.inner; ++i) {
                for (int j = 0; j < gs; ++j) v[j] = hf(x[(o * D.G + g * gs + j) * D.inner + i]);
                uint16_t mn16, s16;
                quantise_group(v.data(), gs, bits, q.data(), &mn16, &s16);
                for (int64_t c = 0; c < bpg; ++c) {
                    const uint8_t byte = bits == 4 ? static_cast<uint8_t>(q[2 * c] | (q[2 * c + 1] << 4)) : q[c];
                    codes[(o * cG + g * bpg + c) * D.inner + i] = byte;
                }
                uint16_t* m = meta + ((o * ng + g) * D.inner + i) * 2;
                m[0] = mn16;
                m[1] = s16;
            }
        }
    });
    return 0;
}

int fo_decompress(const uint8_t* codes, const uint16_t* meta, int ndim, const int64_t* shape, int bits, int gs,
                  int gd, uint16_t* y, int nthreads) {
    Dims D;
    if (!config_ok(bits, gs) || !dims_of(ndim, shape, gd, gs, &D)) return -1;
    const int64_t ng = D.G / gs, bpg = gs * bits / 8, cG = ng * bpg;
    parallel_for(D.outer * ng, nthreads, [&](int64_t b, int64_t e) {
        for (int64_t og = b; og < e; ++og) {
            const int64_t o = og / ng, g = og % ng;
            for (int64_t i = 0; i < D.inner; ++i) {
                const uint16_t* m = meta + ((o * ng + g) * D.inner + i) * 2;
                for (int j = 0; j < gs; ++j) {
                    const uint8_t byte = codes[(o * cG + g * bpg + (bits == 4 ? j / 2 : j)) * D.inner + i];
                    const uint32_t q = bits == 4 ? ((j & 1) ? byte >> 4 : byte & 0xF) : byte;
                    y[(o * D.G + g * gs + j) * D.inner + i] = dequantise_one(q, m[0], m[1]);
                }
            }
        }
    });
    return 0;
}

}  // extern "C"

// ---- the OPT layer -----------------------------------------------------------------------
namespace {

struct Layer {
    int h, nh, d, ffn;
    std::vector<float> ln1_g, ln1_b, ln2_g, ln2_b, b_qkv, b_o, b_fc1, b_fc2;
    std::vector<uint16_t> w[4];       // dequantised fp16 weights [rows][cols]: qkv, o, fc1, fc2
    int rows[4], cols[4];
};

struct Cache {                        // [batch][n_heads][max_seq][...] like the library's
    uint8_t *k_codes, *v_codes;
    uint16_t *k_meta, *v_meta;
    int batch, n_heads, head_dim, max_seq, bits, gs;
};

std::vector<float> vec(const uint16_t* p, int n) {
    std::vector<float> v(n);
    for (int i = 0; i < n; ++i) v[i] = hf(p[i]);
    return v;
}

void layer_norm(const float* x, const std::vector<float>& g, const std::vector<float>& b, int h, float* y) {
    float sum = 0.0f;
    for (int i = 0; i < h; ++i) sum += x[i];
    const float mean = sum / static_cast<float>(h);
    float ss = 0.0f;
    for (int i = 0; i < h; ++i) {
        const float c = x[i] - mean;
        ss += c * c;
    }
    const float var = ss / static_cast<float>(h);
    const float den = std::sqrt(var + 1e-5f);
    for (int i = 0; i < h; ++i) y[i] = (x[i] - mean) / den * g[i] + b[i];
}

// out[t][n] = sum_k a[t][k] * w[n][k] + bias[n], t < T. Each sum runs over k in order.
constexpr int kTB = 16;               // tokens per pass over a weight row (cache reuse only)
void linear(const float* a, int T, int K, const std::vector<uint16_t>& w, int N, const std::vector<float>& bias,
            float* out, int nthreads) {
    const float* tab = table().v;
    for (int t0 = 0; t0 < T; t0 += kTB) {
        const int tb = std::min(kTB, T - t0);
        std::vector<float> at(static_cast<size_t>(K) * kTB, 0.0f);    // [k][token] of this block
        for (int t = 0; t < tb; ++t)
            for (int k = 0; k < K; ++k) at[static_cast<size_t>(k) * kTB + t] = a[static_cast<size_t>(t0 + t) * K + k];
        parallel_for(N, nthreads, [&](int64_t nb, int64_t ne) {
            for (int64_t n = nb; n < ne; ++n) {
                const uint16_t* wr = w.data() + n * K;
                float acc[kTB];
                for (int t = 0; t < kTB; ++t) acc[t] = 0.0f;
                for (int k = 0; k < K; ++k) {
                    const float wv = tab[wr[k]];
                    const float* ak = at.data() + static_cast<size_t>(k) * kTB;
                    for (int t = 0; t < kTB; ++t) acc[t] += ak[t] * wv;
                }
                for (int t = 0; t < tb; ++t) out[static_cast<size_t>(t0 + t) * N + n] = acc[t] + bias[n];
            }
        });
    }
}

// Softmax attention of one query over `n` keys/values (float rows of d): max-subtracted,
// p_j = e_j / z, o = sum_j p_j v_j.
void attend(const float* q, int d, const std::vector<const float*>& keys, const std::vector<const float*>& vals,
            float* o) {
    const size_t n = keys.size();
    std::vector<float> sc(n);
    for (size_t j = 0; j < n; ++j) {
        float s = 0.0f;
        for (int e = 0; e < d; ++e) s += q[e] * keys[j][e];
        sc[j] = s;
    }
    float m = sc[0];
    for (size_t j = 1; j < n; ++j) m = std::max(m, sc[j]);
    float z = 0.0f;
    for (size_t j = 0; j < n; ++j) {
        sc[j] = std::exp(sc[j] - m);
        z += sc[j];
    }
    for (size_t j = 0; j < n; ++j) sc[j] = sc[j] / z;
    for (int e = 0; e < d; ++e) {
        float acc = 0.0f;
        for (size_t j = 0; j < n; ++j) acc += sc[j] * vals[j][e];
        o[e] = acc;
    }
}

// Quantise the fp16-rounded key (or value) vector of one head into slot `slot`.
void store_slot(const Cache& c, bool value, int b, int head, int slot, const float* kv) {
    const int d = c.head_dim, gs = c.gs, bits = c.bits;
    const int64_t base = (static_cast<int64_t>(b) * c.n_heads + head) * c.max_seq + slot;
    uint8_t* codes = (value ? c.v_codes : c.k_codes) + base * (d * bits / 8);
    uint16_t* meta = (value ? c.v_meta : c.k_meta) + base * (d / gs) * 2;
    std::vector<float> v(gs);
    std::vector<uint8_t> q(gs);
    for (int g = 0; g < d / gs; ++g) {
        for (int j = 0; j < gs; ++j) v[j] = hf(float_to_half(kv[g * gs + j]));
        quantise_group(v.data(), gs, bits, q.data(), meta + 2 * g, meta + 2 * g + 1);
        const int bpg = gs * bits / 8;
        for (int cb = 0; cb < bpg; ++cb)
            codes[g * bpg + cb] = bits == 4 ? static_cast<uint8_t>(q[2 * cb] | (q[2 * cb + 1] << 4)) : q[cb];
    }
}

// Dequantised key (or value) of slot `slot` as floats.
void load_slot(const Cache& c, bool value, int b, int head, int slot, float* out) {
    const int d = c.head_dim, gs = c.gs, bits = c.bits;
    const int64_t base = (static_cast<int64_t>(b) * c.n_heads + head) * c.max_seq + slot;
    const uint8_t* codes = (value ? c.v_codes : c.k_codes) + base * (d * bits / 8);
    const uint16_t* meta = (value ? c.v_meta : c.k_meta) + base * (d / gs) * 2;
    for (int j = 0; j < d; ++j) {
        const uint32_t q = bits == 4 ? ((j & 1) ? codes[j / 2] >> 4 : codes[j / 2] & 0xF) : codes[j];
        out[j] = hf(dequantise_one(q, meta[2 * (j / gs)], meta[2 * (j / gs) + 1]));
    }
}

// The block after attention: h1 = x + o Wo^T + bo; out = h1 + ReLU(LN(h1) W1^T + b1) W2^T + b2.
void mlp_block(const Layer& L, const std::vector<float>& x, const std::vector<float>& o, int T, uint16_t* out,
               int nthreads) {
    const int h = L.h, ffn = L.ffn;
    std::vector<float> h1(static_cast<size_t>(T) * h), a2(static_cast<size_t>(T) * h), f(static_cast<size_t>(T) * ffn),
        y(static_cast<size_t>(T) * h);
    linear(o.data(), T, h, L.w[1], h, L.b_o, h1.data(), nthreads);
    for (size_t i = 0; i < h1.size(); ++i) h1[i] = x[i] + h1[i];
    for (int t = 0; t < T; ++t) layer_norm(h1.data() + static_cast<size_t>(t) * h, L.ln2_g, L.ln2_b, h, a2.data() + static_cast<size_t>(t) * h);
    linear(a2.data(), T, h, L.w[2], ffn, L.b_fc1, f.data(), nthreads);
    for (auto& v : f) v = std::max(v, 0.0f);
    linear(f.data(), T, ffn, L.w[3], h, L.b_fc2, y.data(), nthreads);
    for (size_t i = 0; i < y.size(); ++i) out[i] = float_to_half(h1[i] + y[i]);
}

// LN1 and the fused QKV projection of T tokens: qkv [T][3h], q already scaled.
void qkv_block(const Layer& L, const std::vector<float>& x, int T, std::vector<float>& qkv, int nthreads) {
    const int h = L.h;
    std::vector<float> a(static_cast<size_t>(T) * h);
    for (int t = 0; t < T; ++t) layer_norm(x.data() + static_cast<size_t>(t) * h, L.ln1_g, L.ln1_b, h, a.data() + static_cast<size_t>(t) * h);
    qkv.assign(static_cast<size_t>(T) * 3 * h, 0.0f);
    linear(a.data(), T, h, L.w[0], 3 * h, L.b_qkv, qkv.data(), nthreads);
    const float rs = std::sqrt(static_cast<float>(L.d));
    for (int t = 0; t < T; ++t)
        for (int i = 0; i < h; ++i) qkv[static_cast<size_t>(t) * 3 * h + i] /= rs;
}

}  // namespace

extern "C" {

typedef struct {
    int h, n_heads, head_dim, ffn, w_bits;
    const uint16_t *ln1_g, *ln1_b, *ln2_g, *ln2_b, *b_qkv, *b_o, *b_fc1, *b_fc2;
    const uint8_t* w_codes[4];        // qkv [3h][h], o [h][h], fc1 [ffn][h], fc2 [h][ffn]; group 64 along in
    const uint16_t* w_meta[4];
} fo_layer_desc;

typedef struct {
    uint8_t *k_codes, *v_codes;
    uint16_t *k_meta, *v_meta;
    int batch, n_heads, head_dim, max_seq, bits, gs;
} fo_cache;

// A layer with its weights dequantised once (fp16 values). NULL on bad arguments.
void* fo_layer_new(const fo_layer_desc* D, int nthreads) {
    if (!D || D->n_heads <= 0 || D->head_dim <= 0 || D->n_heads * D->head_dim != D->h) return nullptr;
    if (D->w_bits != 4 && D->w_bits != 8) return nullptr;
    Layer* L = new Layer;
    L->h = D->h;
    L->nh = D->n_heads;
    L->d = D->head_dim;
    L->ffn = D->ffn;
    const int h = D->h, ffn = D->ffn;
    L->ln1_g = vec(D->ln1_g, h);
    L->ln1_b = vec(D->ln1_b, h);
    L->ln2_g = vec(D->ln2_g, h);
    L->ln2_b = vec(D->ln2_b, h);
    L->b_qkv = vec(D->b_qkv, 3 * h);
    L->b_o = vec(D->b_o, h);
    L->b_fc1 = vec(D->b_fc1, ffn);
    L->b_fc2 = vec(D->b_fc2, h);
    const int rows[4] = {3 * h, h, ffn, h}, cols[4] = {h, h, h, ffn};
    for (int i = 0; i < 4; ++i) {
        L->rows[i] = rows[i];
        L->cols[i] = cols[i];
        L->w[i].resize(static_cast<size_t>(rows[i]) * cols[i]);
        const int64_t shape[2] = {rows[i], cols[i]};
        if (fo_decompress(D->w_codes[i], D->w_meta[i], 2, shape, D->w_bits, 64, 1, L->w[i].data(), nthreads) != 0) {
            delete L;
            return nullptr;
        }
    }
    return L;
}

void fo_layer_free(void* L) { delete static_cast<Layer*>(L); }

// Prefill (mha): x fp16 [batch][seq][h] -> out fp16; writes cache slots [0, seq) of
// sequences 0..batch-1.
int fo_prefill_layer(void* Lp, const fo_cache* C, const uint16_t* x16, int batch, int seq, uint16_t* out,
                     int nthreads) {
    const Layer& L = *static_cast<Layer*>(Lp);
    const Cache c{C->k_codes, C->v_codes, C->k_meta, C->v_meta, C->batch, C->n_heads, C->head_dim, C->max_seq,
                  C->bits, C->gs};
    if (batch > c.batch || seq > c.max_seq || c.head_dim != L.d || c.n_heads != L.nh) return -1;
    const int h = L.h, d = L.d, T = batch * seq;
    std::vector<float> x(static_cast<size_t>(T) * h);
    for (size_t i = 0; i < x.size(); ++i) x[i] = hf(x16[i]);
    std::vector<float> qkv;
    qkv_block(L, x, T, qkv, nthreads);
    std::vector<float> o(static_cast<size_t>(T) * h);
    parallel_for(static_cast<int64_t>(batch) * L.nh, nthreads, [&](int64_t pb, int64_t pe) {
        for (int64_t p = pb; p < pe; ++p) {
            const int b = static_cast<int>(p / L.nh), hd = static_cast<int>(p % L.nh);
            std::vector<const float*> keys, vals;
            for (int i = 0; i < seq; ++i) {
                const float* row = qkv.data() + static_cast<size_t>(b * seq + i) * 3 * h;
                keys.push_back(row + h + hd * d);
                vals.push_back(row + 2 * h + hd * d);
                attend(row + hd * d, d, keys, vals, o.data() + static_cast<size_t>(b * seq + i) * h + hd * d);
            }
            for (int i = 0; i < seq; ++i) {
                store_slot(c, false, b, hd, i, keys[i]);
                store_slot(c, true, b, hd, i, vals[i]);
            }
        }
    });
    mlp_block(L, x, o, T, out, nthreads);
    return 0;
}

// Decode step (mha_gen) at pos: x fp16 [batch][h] -> out fp16; attends to cache slots
// [0, pos) and the fresh key/value, then quantises the fresh key/value into slot pos.
int fo_decode_layer(void* Lp, const fo_cache* C, const uint16_t* x16, int batch, int pos, uint16_t* out,
                    int nthreads) {
    const Layer& L = *static_cast<Layer*>(Lp);
    const Cache c{C->k_codes, C->v_codes, C->k_meta, C->v_meta, C->batch, C->n_heads, C->head_dim, C->max_seq,
                  C->bits, C->gs};
    if (batch > c.batch || pos < 0 || pos >= c.max_seq || c.head_dim != L.d || c.n_heads != L.nh) return -1;
    const int h = L.h, d = L.d;
    std::vector<float> x(static_cast<size_t>(batch) * h);
    for (size_t i = 0; i < x.size(); ++i) x[i] = hf(x16[i]);
    std::vector<float> qkv;
    qkv_block(L, x, batch, qkv, nthreads);
    std::vector<float> o(static_cast<size_t>(batch) * h);
    parallel_for(static_cast<int64_t>(batch) * L.nh, nthreads, [&](int64_t pb, int64_t pe) {
        std::vector<float> kc(static_cast<size_t>(pos) * d), vc(static_cast<size_t>(pos) * d);
        for (int64_t p = pb; p < pe; ++p) {
            const int b = static_cast<int>(p / L.nh), hd = static_cast<int>(p % L.nh);
            const float* row = qkv.data() + static_cast<size_t>(b) * 3 * h;
            std::vector<const float*> keys, vals;
            for (int j = 0; j < pos; ++j) {
                load_slot(c, false, b, hd, j, kc.data() + static_cast<size_t>(j) * d);
                load_slot(c, true, b, hd, j, vc.data() + static_cast<size_t>(j) * d);
                keys.push_back(kc.data() + static_cast<size_t>(j) * d);
                vals.push_back(vc.data() + static_cast<size_t>(j) * d);
            }
            keys.push_back(row + h + hd * d);
            vals.push_back(row + 2 * h + hd * d);
            attend(row + hd * d, d, keys, vals, o.data() + static_cast<size_t>(b) * h + hd * d);
        }
    });
    mlp_block(L, x, o, batch, out, nthreads);
    for (int b = 0; b < batch; ++b)
        for (int hd = 0; hd < L.nh; ++hd) {
            const float* row = qkv.data() + static_cast<size_t>(b) * 3 * h;
            store_slot(c, false, b, hd, pos, row + h + hd * d);
            store_slot(c, true, b, hd, pos, row + 2 * h + hd * d);
        }
    return 0;
}

// Decode attention alone: q, k_new, v_new fp16 [batch][n_heads][head_dim] (q already
// scaled) -> o float [batch][n_heads][head_dim].
int fo_decode_attention(const fo_cache* C, const uint16_t* q16, const uint16_t* k16, const uint16_t* v16, int batch,
                        int pos, float* o) {
    const Cache c{C->k_codes, C->v_codes, C->k_meta, C->v_meta, C->batch, C->n_heads, C->head_dim, C->max_seq,
                  C->bits, C->gs};
    if (batch > c.batch || pos < 0 || pos >= c.max_seq) return -1;
    const int d = c.head_dim;
    std::vector<float> kc(static_cast<size_t>(pos) * d), vc(static_cast<size_t>(pos) * d), q(d), kn(d), vn(d);
    for (int b = 0; b < batch; ++b)
        for (int hd = 0; hd < c.n_heads; ++hd) {
            const size_t off = (static_cast<size_t>(b) * c.n_heads + hd) * d;
            std::vector<const float*> keys, vals;
            for (int j = 0; j < pos; ++j) {
                load_slot(c, false, b, hd, j, kc.data() + static_cast<size_t>(j) * d);
                load_slot(c, true, b, hd, j, vc.data() + static_cast<size_t>(j) * d);
                keys.push_back(kc.data() + static_cast<size_t>(j) * d);
                vals.push_back(vc.data() + static_cast<size_t>(j) * d);
            }
            for (int e = 0; e < d; ++e) {
                q[e] = hf(q16[off + e]);
                kn[e] = hf(k16[off + e]);
                vn[e] = hf(v16[off + e]);
            }
            keys.push_back(kn.data());
            vals.push_back(vn.data());
            attend(q.data(), d, keys, vals, o + off);
        }
    return 0;
}

}  // extern "C"
