// Attention of the OPT layer.
//
// Decode (`mha_gen`, FlexGen source-reading notes, "Pytorch Backend"): one new token per
// sequence attends to the compressed cache slots [0, pos) - written by earlier
// store_cache calls - and to its own fresh key/value (the loop runs load_cache,
// compute_layer, store_cache, so the current token's key/value are not in the cache
// yet). The int4 cache (FlexGen source walkthrough, section 6.3: 4 bits, group 64
// along the head dimension) is streamed once and dequantised in registers; the sum
// over a group is factored as  sum_i q_i * (c_i*step + min) = step*sum_i q_i c_i +
// min*sum_i q_i,  and likewise for the value side, so each code costs one extract and
// one FMA. Work is split across the KV length (flash-decoding): every CTA keeps an
// online softmax per key lane, merges its lanes, and writes (max, sum, o) partials;
// a combine kernel folds the partials together with the fresh key/value.
//
// Prefill (`mha`): causal softmax attention over the prompt on the fresh fp16
// q/k/v, flash-attention style: 64 queries per CTA, 64-key tiles double-buffered in
// shared memory with cp.async, QK^T and PV on the tensor cores (mma.sync m16n8k16,
// fp32 accumulation), online softmax in registers.
#include <float.h>

#include "quant.cuh"

namespace flexq {
namespace {

constexpr int DA_THREADS = 128;

// ---------------------------------------------------------------------------------
// decode attention, split-KV partials
template <int D, int BITS, int GS>
__global__ void __launch_bounds__(DA_THREADS) decode_attn_split_kernel(
    const __half* __restrict__ q, int64_t row_stride, const uint8_t* __restrict__ k_codes,
    const uint32_t* __restrict__ k_meta, const uint8_t* __restrict__ v_codes,
    const uint32_t* __restrict__ v_meta, int n_heads, int max_seq, int pos, int chunk,
    float* __restrict__ part) {
    constexpr int KB = D * BITS / 8;        // code bytes per key
    constexpr int TPK = KB / 4;             // threads per key (one u32 of codes each)
    constexpr int EPT = 32 / BITS;          // dims per thread
    constexpr int KPI = DA_THREADS / TPK;   // keys per iteration
    constexpr int GPK = D / GS;             // groups per key
    const int pair = blockIdx.x;            // b * n_heads + head
    const int split = blockIdx.y;
    const int nsplit = gridDim.y;
    const int b = pair / n_heads, head = pair % n_heads;
    const int tid = threadIdx.x;
    const int kl = tid / TPK, wl = tid % TPK;
    const int d0 = wl * EPT;
    const int grp = d0 / GS;

    float qv[EPT];
    float qsum = 0.f;
    {
        const __half* qp = q + static_cast<int64_t>(b) * row_stride + head * D + d0;
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
            qv[e] = __half2float(qp[e]);
            qsum += qv[e];
        }
    }
    const int j0 = split * chunk;
    const int j1 = min(pos, j0 + chunk);
    const int64_t slot0 = static_cast<int64_t>(pair) * max_seq;

    float m = -FLT_MAX, l = 0.f, U = 0.f;
    float acc[EPT];
#pragma unroll
    for (int e = 0; e < EPT; ++e) acc[e] = 0.f;

    // the trip count is uniform across the CTA: lanes past the end of the split load
    // nothing and skip the update, but still take part in the shuffles
    for (int jb = j0; jb < j1; jb += KPI) {
        const int j = jb + kl;
        const bool valid = j < j1;
        const int64_t slot = slot0 + (valid ? j : j0);
        const uint32_t kw = __ldg(reinterpret_cast<const uint32_t*>(k_codes + slot * KB) + wl);
        const uint32_t vw = __ldg(reinterpret_cast<const uint32_t*>(v_codes + slot * KB) + wl);
        const uint32_t km = __ldg(k_meta + slot * GPK + grp);
        const uint32_t vm = __ldg(v_meta + slot * GPK + grp);
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
            const uint32_t c = (kw >> (BITS * e)) & ((1u << BITS) - 1u);
            dot = fmaf(qv[e], static_cast<float>(c), dot);
        }
        const float kstep = group_step(__ushort_as_half(static_cast<unsigned short>(km >> 16)));
        const float kmn = h2f_lo(km);
        float s = (kstep == 0.f) ? kmn * qsum : fmaf(kstep, dot, kmn * qsum);
#pragma unroll
        for (int off = TPK / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (!valid) continue;
        if (s > m) {
            const float alpha = __expf(m - s);
            m = s;
            l *= alpha;
            U *= alpha;
#pragma unroll
            for (int e = 0; e < EPT; ++e) acc[e] *= alpha;
        }
        const float p = __expf(s - m);
        l += p;
        const float vstep = group_step(__ushort_as_half(static_cast<unsigned short>(vm >> 16)));
        const float vmn = h2f_lo(vm);
        const float w = p * vstep;
        U = fmaf(p, vmn, U);
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
            const uint32_t c = (vw >> (BITS * e)) & ((1u << BITS) - 1u);
            acc[e] = fmaf(w, static_cast<float>(c), acc[e]);
        }
    }

    // merge the KPI key lanes of this CTA
    __shared__ float sm_m[KPI], sm_l[KPI];
    __shared__ float sm_o[KPI][D];
    if (wl == 0) {
        sm_m[kl] = m;
        sm_l[kl] = l;
    }
#pragma unroll
    for (int e = 0; e < EPT; ++e) sm_o[kl][d0 + e] = acc[e] + U;
    __syncthreads();
    float M = -FLT_MAX;
#pragma unroll
    for (int i = 0; i < KPI; ++i) M = fmaxf(M, sm_m[i]);
    float* out = part + (static_cast<int64_t>(pair) * nsplit + split) * (D + 2);
    for (int d = tid; d < D; d += DA_THREADS) {
        float o = 0.f;
#pragma unroll
        for (int i = 0; i < KPI; ++i) {
            const float f = sm_l[i] > 0.f ? __expf(sm_m[i] - M) : 0.f;
            o = fmaf(f, sm_o[i][d], o);
        }
        out[2 + d] = o;
    }
    if (tid == 0) {
        float L = 0.f;
#pragma unroll
        for (int i = 0; i < KPI; ++i) L += sm_l[i] > 0.f ? __expf(sm_m[i] - M) * sm_l[i] : 0.f;
        out[0] = M;
        out[1] = L;
    }
}

// combine the split partials with the fresh key/value of the current token
template <int D>
__global__ void __launch_bounds__(D) decode_attn_combine_kernel(const __half* __restrict__ q,
                                                                const __half* __restrict__ k_new,
                                                                const __half* __restrict__ v_new,
                                                                int64_t row_stride, int n_heads,
                                                                int nsplit,
                                                                const float* __restrict__ part,
                                                                __half* __restrict__ o) {
    const int pair = blockIdx.x;
    const int b = pair / n_heads, head = pair % n_heads;
    const int d = threadIdx.x;
    const int64_t off = static_cast<int64_t>(b) * row_stride + head * D + d;
    float s = __half2float(q[off]) * __half2float(k_new[off]);
#pragma unroll
    for (int w = 16; w > 0; w >>= 1) s += __shfl_xor_sync(0xffffffffu, s, w);
    __shared__ float red[D / 32];
    if ((d & 31) == 0) red[d >> 5] = s;
    __syncthreads();
    float snew = 0.f;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) snew += red[i];
    const float* pp = part + static_cast<int64_t>(pair) * nsplit * (D + 2);
    float M = snew;
    for (int i = 0; i < nsplit; ++i)
        if (pp[i * (D + 2) + 1] > 0.f) M = fmaxf(M, pp[i * (D + 2)]);
    const float fn = __expf(snew - M);
    float L = fn;
    float acc = fn * __half2float(v_new[off]);
    for (int i = 0; i < nsplit; ++i) {
        const float* p = pp + i * (D + 2);
        if (!(p[1] > 0.f)) continue;
        const float f = __expf(p[0] - M);
        L = fmaf(f, p[1], L);
        acc = fmaf(f, p[2 + d], acc);
    }
    o[static_cast<int64_t>(b) * n_heads * D + head * D + d] = __float2half_rn(acc / L);
}

// ---------------------------------------------------------------------------------
// prefill attention (causal), mma.sync m16n8k16
constexpr int PA_BQ = 64, PA_BK = 64, PA_THREADS = 128;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool pred) {
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const int n = pred ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* p) {
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(s));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void* p) {
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(s));
}

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f2h2(float lo, float hi) {
    return pack_half2_bits(__float2half_rn(lo), __float2half_rn(hi));
}

template <int D>
__global__ void __launch_bounds__(PA_THREADS) prefill_attn_kernel(const __half* __restrict__ q,
                                                                  const __half* __restrict__ k,
                                                                  const __half* __restrict__ v,
                                                                  int64_t row_stride,
                                                                  __half* __restrict__ o, int seq,
                                                                  int n_heads) {
    constexpr int LD = D + 8;                  // padded smem row (halves): conflict-free ldmatrix
    constexpr int CPR = D / 8;                 // 16-byte chunks per row
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __half* sQ = reinterpret_cast<__half*>(smem_raw);
    __half* sK = sQ + PA_BQ * LD;              // [2][BK][LD]
    __half* sV = sK + 2 * PA_BK * LD;          // [2][BK][LD]

    const int nqb = gridDim.x;
    const int qb = nqb - 1 - blockIdx.x;       // heaviest blocks first
    const int head = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int q0 = qb * PA_BQ;
    const int64_t base = static_cast<int64_t>(b) * seq;

    // Q tile
    for (int c = tid; c < PA_BQ * CPR; c += PA_THREADS) {
        const int r = c / CPR, cc = c % CPR;
        const int tok = q0 + r;
        const bool ok = tok < seq;
        cp_async16(sQ + r * LD + cc * 8, q + (base + (ok ? tok : 0)) * row_stride + head * D + cc * 8, ok);
    }
    auto load_kv = [&](int kb, int buf) {
        const int k0 = kb * PA_BK;
        for (int c = tid; c < PA_BK * CPR; c += PA_THREADS) {
            const int r = c / CPR, cc = c % CPR;
            const int tok = k0 + r;
            const bool ok = tok < seq;
            const int64_t off = (base + (ok ? tok : 0)) * row_stride + head * D + cc * 8;
            cp_async16(sK + (buf * PA_BK + r) * LD + cc * 8, k + off, ok);
            cp_async16(sV + (buf * PA_BK + r) * LD + cc * 8, v + off, ok);
        }
    };
    const int nkb = min((q0 + PA_BQ + PA_BK - 1) / PA_BK, (seq + PA_BK - 1) / PA_BK);
    load_kv(0, 0);
    cp_async_commit();

    uint32_t qa[D / 16][4];
    float oacc[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    float mrow[2] = {-FLT_MAX, -FLT_MAX}, lrow[2] = {0.f, 0.f};
    constexpr float LOG2E = 1.4426950408889634f;

    for (int kb = 0; kb < nkb; ++kb) {
        const int buf = kb & 1;
        if (kb + 1 < nkb) load_kv(kb + 1, buf ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (kb == 0) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int c = ks * 16 + (lane >> 4) * 8;
                ldmatrix_x4(qa[ks], sQ + r * LD + c);
            }
        }
        // S = Q K^T for 64 keys
        float s[PA_BK / 8][4];
#pragma unroll
        for (int i = 0; i < PA_BK / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
        const __half* Kt = sK + buf * PA_BK * LD;
#pragma unroll
        for (int nt = 0; nt < PA_BK / 16; ++nt) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t bk[4];
                const int r = nt * 16 + (lane & 7) + (lane >> 4) * 8;
                const int c = ks * 16 + ((lane >> 3) & 1) * 8;
                ldmatrix_x4(bk, Kt + r * LD + c);
                mma16816(s[2 * nt], qa[ks], bk[0], bk[1]);
                mma16816(s[2 * nt + 1], qa[ks], bk[2], bk[3]);
            }
        }
        // mask, online softmax
        const int k0 = kb * PA_BK;
        const int qrow0 = q0 + warp * 16 + g;
        float bmax[2] = {-FLT_MAX, -FLT_MAX};
#pragma unroll
        for (int nt = 0; nt < PA_BK / 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = k0 + nt * 8 + 2 * t + (e & 1);
                const int qi = qrow0 + (e >> 1) * 8;
                float val = s[nt][e] * LOG2E;
                if (key > qi || key >= seq) val = -FLT_MAX;
                s[nt][e] = val;
                bmax[e >> 1] = fmaxf(bmax[e >> 1], val);
            }
        }
        float scale[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            bmax[r] = fmaxf(bmax[r], __shfl_xor_sync(0xffffffffu, bmax[r], 1));
            bmax[r] = fmaxf(bmax[r], __shfl_xor_sync(0xffffffffu, bmax[r], 2));
            const float mnew = fmaxf(mrow[r], bmax[r]);
            scale[r] = exp2f(mrow[r] - mnew);
            mrow[r] = mnew;
            lrow[r] *= scale[r];
        }
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            oacc[i][0] *= scale[0];
            oacc[i][1] *= scale[0];
            oacc[i][2] *= scale[1];
            oacc[i][3] *= scale[1];
        }
        uint32_t pa[PA_BK / 16][4];
#pragma unroll
        for (int nt = 0; nt < PA_BK / 8; ++nt) {
            float p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                p[e] = s[nt][e] == -FLT_MAX ? 0.f : exp2f(s[nt][e] - mrow[e >> 1]);
                lrow[e >> 1] += p[e];
            }
            pa[nt >> 1][(nt & 1) * 2 + 0] = pack_f2h2(p[0], p[1]);
            pa[nt >> 1][(nt & 1) * 2 + 1] = pack_f2h2(p[2], p[3]);
        }
        // O += P V
        const __half* Vt = sV + buf * PA_BK * LD;
#pragma unroll
        for (int ks = 0; ks < PA_BK / 16; ++ks) {
            // A regs order for m16n8k16: {row g k0-7, row g+8 k0-7, row g k8-15, row g+8 k8-15}
            const uint32_t a[4] = {pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3]};
#pragma unroll
            for (int nt = 0; nt < D / 16; ++nt) {
                uint32_t bv[4];
                const int r = ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int c = nt * 16 + (lane >> 4) * 8;
                ldmatrix_x4_trans(bv, Vt + r * LD + c);
                mma16816(oacc[2 * nt], a, bv[0], bv[1]);
                mma16816(oacc[2 * nt + 1], a, bv[2], bv[3]);
            }
        }
        __syncthreads();
    }
    // finalise
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
        lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
    }
    const int hD = n_heads * D;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int tok = q0 + warp * 16 + g + r * 8;
        if (tok >= seq) continue;
        const float inv = 1.f / lrow[r];
        __half* dst = o + (base + tok) * hD + head * D;
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
            *reinterpret_cast<uint32_t*>(dst + nt * 8 + 2 * t) =
                pack_f2h2(oacc[nt][2 * r] * inv, oacc[nt][2 * r + 1] * inv);
        }
    }
}

}  // namespace

int validate_cache(const flex_kv_cache* c);

int decode_attn_nsplit(int pairs, int pos) {
    if (pos <= 0) return 0;
    const int target = 4 * sm_count();
    int ns = (target + pairs - 1) / pairs;
    const int max_by_len = (pos + 31) / 32;          // at least 32 keys per split
    if (ns > max_by_len) ns = max_by_len;
    return ns < 1 ? 1 : ns;
}

int64_t decode_attn_ws_bytes(int pairs, int head_dim, int pos) {
    const int ns = decode_attn_nsplit(pairs, pos);
    return static_cast<int64_t>(pairs) * (ns > 0 ? ns : 1) * (head_dim + 2) * 4;
}

// Bound on decode_attn_ws_bytes over every pos.
int64_t decode_attn_ws_bound(int pairs, int head_dim) {
    const int target = 4 * sm_count();
    const int ns = (target + pairs - 1) / pairs;
    return static_cast<int64_t>(pairs) * (ns > 0 ? ns : 1) * (head_dim + 2) * 4;
}

int decode_attn_launch(const flex_kv_cache* c, const void* q, const void* k_new, const void* v_new,
                       int64_t row_stride, void* o, int batch, int pos, void* ws, cudaStream_t st) {
    const int pairs = batch * c->n_heads;
    const int ns = decode_attn_nsplit(pairs, pos);
    const int chunk = ns > 0 ? (pos + ns - 1) / ns : 0;
    float* part = static_cast<float*>(ws);
    const __half* qh = static_cast<const __half*>(q);
    const uint8_t* kc = static_cast<const uint8_t*>(c->k_codes);
    const uint8_t* vc = static_cast<const uint8_t*>(c->v_codes);
    const uint32_t* km = static_cast<const uint32_t*>(c->k_meta);
    const uint32_t* vm = static_cast<const uint32_t*>(c->v_meta);
    if (ns > 0) {
        const dim3 grid(pairs, ns);
#define SPLIT(D_, B_, G_)                                                                                 \
    decode_attn_split_kernel<D_, B_, G_><<<grid, DA_THREADS, 0, st>>>(qh, row_stride, kc, km, vc, vm,     \
                                                                      c->n_heads, c->max_seq, pos, chunk, \
                                                                      part)
        const int D = c->head_dim, B = c->cfg.num_bits, G = c->cfg.group_size;
        if (D == 64 && B == 4 && G == 64) SPLIT(64, 4, 64);
        else if (D == 64 && B == 4 && G == 32) SPLIT(64, 4, 32);
        else if (D == 64 && B == 8 && G == 64) SPLIT(64, 8, 64);
        else if (D == 64 && B == 8 && G == 32) SPLIT(64, 8, 32);
        else if (D == 128 && B == 4 && G == 64) SPLIT(128, 4, 64);
        else if (D == 128 && B == 4 && G == 32) SPLIT(128, 4, 32);
        else if (D == 128 && B == 8 && G == 64) SPLIT(128, 8, 64);
        else SPLIT(128, 8, 32);
#undef SPLIT
    }
    const __half* kn = static_cast<const __half*>(k_new);
    const __half* vn = static_cast<const __half*>(v_new);
    __half* oh = static_cast<__half*>(o);
    if (c->head_dim == 64)
        decode_attn_combine_kernel<64><<<pairs, 64, 0, st>>>(qh, kn, vn, row_stride, c->n_heads, ns, part, oh);
    else
        decode_attn_combine_kernel<128><<<pairs, 128, 0, st>>>(qh, kn, vn, row_stride, c->n_heads, ns, part, oh);
    return launch_status();
}

size_t prefill_attn_smem(int D) { return static_cast<size_t>(PA_BQ + 4 * PA_BK) * (D + 8) * 2; }

int prefill_attn_launch(const void* q, const void* k, const void* v, int64_t row_stride, void* o, int batch,
                        int seq, int n_heads, int head_dim, cudaStream_t st) {
    if (batch == 0 || seq == 0) return FLEX_OK;
    const dim3 grid((seq + PA_BQ - 1) / PA_BQ, n_heads, batch);
    const size_t smem = prefill_attn_smem(head_dim);
    const __half* qh = static_cast<const __half*>(q);
    const __half* kh = static_cast<const __half*>(k);
    const __half* vh = static_cast<const __half*>(v);
    __half* oh = static_cast<__half*>(o);
    if (head_dim == 64) {
        cudaFuncSetAttribute(prefill_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        prefill_attn_kernel<64><<<grid, PA_THREADS, smem, st>>>(qh, kh, vh, row_stride, oh, seq, n_heads);
    } else {
        cudaFuncSetAttribute(prefill_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        prefill_attn_kernel<128><<<grid, PA_THREADS, smem, st>>>(qh, kh, vh, row_stride, oh, seq, n_heads);
    }
    return launch_status();
}

}  // namespace flexq

using namespace flexq;

extern "C" int64_t flex_decode_attention_ws_bytes(const flex_kv_cache* cache, int32_t batch, int32_t pos) {
    const int rc = validate_cache(cache);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(batch > 0 && batch <= cache->batch, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(pos >= 0 && pos < cache->max_seq, FLEX_ERR_SHAPE);
    return decode_attn_ws_bytes(batch * cache->n_heads, cache->head_dim, pos);
}

extern "C" int flex_decode_attention(const flex_kv_cache* cache, const void* q, const void* k_new,
                                     const void* v_new, int64_t row_stride, void* o, int32_t batch,
                                     int32_t pos, void* ws, int64_t ws_bytes, void* stream) {
    const int rc = validate_cache(cache);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(q && k_new && v_new && o, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(batch > 0 && batch <= cache->batch, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(pos >= 0 && pos < cache->max_seq, FLEX_ERR_SHAPE);
    FLEX_REQUIRE(row_stride >= static_cast<int64_t>(cache->n_heads) * cache->head_dim, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(aligned16(q) && aligned16(k_new) && aligned16(v_new) && aligned16(o), FLEX_ERR_ALIGN);
    const int64_t need = decode_attn_ws_bytes(batch * cache->n_heads, cache->head_dim, pos);
    FLEX_REQUIRE(ws != nullptr && ws_bytes >= need, FLEX_ERR_WORKSPACE);
    FLEX_REQUIRE(aligned16(ws), FLEX_ERR_ALIGN);
    return decode_attn_launch(cache, q, k_new, v_new, row_stride, o, batch, pos, ws, as_stream(stream));
}

extern "C" int flex_prefill_attention(const void* q, const void* k, const void* v, int64_t row_stride, void* o,
                                      int32_t batch, int32_t seq, int32_t n_heads, int32_t head_dim,
                                      void* stream) {
    FLEX_REQUIRE(q && k && v && o, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(batch >= 0 && seq >= 0 && n_heads > 0, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(head_dim == 64 || head_dim == 128, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(row_stride >= static_cast<int64_t>(n_heads) * head_dim && row_stride % 8 == 0,
                 FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(o), FLEX_ERR_ALIGN);
    return prefill_attn_launch(q, k, v, row_stride, o, batch, seq, n_heads, head_dim, as_stream(stream));
}
