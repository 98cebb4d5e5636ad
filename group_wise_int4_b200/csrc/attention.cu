// Attention of the OPT layer.
//
// Decode (`mha_gen`, the source-notes page «FlexGen» (PtirisNote), "Pytorch Backend"): one new token per
// sequence attends to the compressed cache slots [0, pos) - written by earlier
// store_cache calls - and to its own fresh key/value (the loop runs load_cache,
// compute_layer, store_cache, so the current token's key/value are not in the cache
// yet). The int4 cache (the walkthrough page «FlexGen 单 GPU 高吞吐大模型推理引擎：论文解读与源码实战指南», section 6.3: 4 bits, group 64
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

#include <mutex>

#include "quant.cuh"

namespace flexq {
namespace {
// 1/scale of a group with the hardware reciprocal (rcp.approx, relative error below
// 2^-22): attention uses the step only inside fp32 sums checked against a tolerance,
// so the correctly rounded division of the codec is not needed here. Scale 0 (a
// constant group) gives step 0.
__device__ __forceinline__ float group_step_fast(__half s16) {
    const float s = __half2float(s16);
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
    return s > 0.0f ? r : 0.0f;
}
}  // namespace
}  // namespace flexq

namespace flexq {
namespace {

constexpr int DA_THREADS = 128;

// ---------------------------------------------------------------------------------
// prefill attention (causal), mma.sync m16n8k16
constexpr int PA_BQ = 64, PA_BK = 64, PA_THREADS = 128;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool pred) {
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const int n = pred ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(n) : "memory");
}
// unpredicated forms (the whole 16 / 4 bytes are always copied)
__device__ __forceinline__ void cp_async16u(uint32_t s, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4u(uint32_t s, const void* gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s), "l"(gmem) : "memory");
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

// ---------------------------------------------------------------------------------
// decode attention, split-KV partials.
//
// A thread owns 16 bytes of every key it touches (32 dims at 4 bits, 16 at 8 bits);
// TPK = key bytes / 16 threads share a key. Each CTA iteration covers DA_U keys per
// thread: all their code and metadata loads are issued first (memory-level
// parallelism), then the scores, one online-softmax update for the block, and the
// value accumulation.
constexpr int DA_U = 8;

// Exact integer -> float of a code: place it in the mantissa of 2^23 and subtract 2^23
// (an integer-pipe OR and one fp32 add, instead of the slower conversion unit).
__device__ __forceinline__ float code_f(uint32_t w, int shift, uint32_t mask) {
    return __int_as_float(0x4B000000u | ((w >> shift) & mask)) - 8388608.0f;
}

template <int D, int BITS, int GS>
__global__ void __launch_bounds__(DA_THREADS) decode_attn_split_kernel(
    const __half* __restrict__ q, int64_t row_stride, const uint8_t* __restrict__ k_codes,
    const uint32_t* __restrict__ k_meta, const uint8_t* __restrict__ v_codes,
    const uint32_t* __restrict__ v_meta, int n_heads, int max_seq, int pos, int chunk,
    float* __restrict__ part, const int32_t* __restrict__ valid_from) {
    constexpr int KB = D * BITS / 8;        // code bytes per key
    constexpr int TPK = KB / 16;            // threads per key (16 bytes each)
    constexpr int EPT = 128 / BITS;         // dims per thread
    constexpr int KPI = DA_THREADS / TPK;   // keys per CTA and unroll step
    constexpr int GPK = D / GS;             // groups per key
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    pdl_wait();
    pdl_trigger();
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
        const uint4* qp = reinterpret_cast<const uint4*>(q + static_cast<int64_t>(b) * row_stride + head * D + d0);
#pragma unroll
        for (int v = 0; v < EPT / 8; ++v) {
            const uint4 w = qp[v];
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                qv[8 * v + 2 * k] = h2f_lo(ww[k]);
                qv[8 * v + 2 * k + 1] = h2f_hi(ww[k]);
            }
        }
#pragma unroll
        for (int e = 0; e < EPT; ++e) qsum += qv[e];
    }
    // keys [split * chunk, +chunk) of [0, pos), minus the left padding [0, valid_from[b])
    const int vf = valid_from ? valid_from[b] : 0;
    const int j0 = max(split * chunk, vf);
    const int j1 = min(pos, split * chunk + chunk);
    const int64_t slot0 = static_cast<int64_t>(pair) * max_seq;

    float m = -FLT_MAX, l = 0.f, U = 0.f;
    float acc[EPT];
#pragma unroll
    for (int e = 0; e < EPT; ++e) acc[e] = 0.f;

    // the trip count is uniform across the CTA: lanes past the end of the split load
    // slot j0 instead and skip the update, but still take part in the shuffles
    for (int jb = j0; jb < j1; jb += DA_U * KPI) {
        uint4 kc[DA_U], vc[DA_U];
        uint32_t km[DA_U], vm[DA_U];
#pragma unroll
        for (int u = 0; u < DA_U; ++u) {
            const int j = jb + u * KPI + kl;
            const int64_t slot = slot0 + (j < j1 ? j : j0);
            kc[u] = __ldg(reinterpret_cast<const uint4*>(k_codes + slot * KB) + wl);
            vc[u] = __ldg(reinterpret_cast<const uint4*>(v_codes + slot * KB) + wl);
            km[u] = __ldg(k_meta + slot * GPK + grp);
            vm[u] = __ldg(v_meta + slot * GPK + grp);
        }
        float s[DA_U];
        float bmax = -FLT_MAX;
#pragma unroll
        for (int u = 0; u < DA_U; ++u) {
            const uint32_t w[4] = {kc[u].x, kc[u].y, kc[u].z, kc[u].w};
            float dot = 0.f;
#pragma unroll
            for (int e = 0; e < EPT; ++e) dot = fmaf(qv[e], code_f(w[e * BITS / 32], (e * BITS) % 32, MASK), dot);
            const float kstep = group_step_fast(__ushort_as_half(static_cast<unsigned short>(km[u] >> 16)));
            const float kmn = h2f_lo(km[u]);
            float su = fmaf(kstep, dot, kmn * qsum);
#pragma unroll
            for (int off = TPK / 2; off > 0; off >>= 1) su += __shfl_xor_sync(0xffffffffu, su, off);
            const int j = jb + u * KPI + kl;
            s[u] = j < j1 ? su : -FLT_MAX;
            bmax = fmaxf(bmax, s[u]);
        }
        if (bmax > m) {
            const float alpha = __expf(m - bmax);
            m = bmax;
            l *= alpha;
            U *= alpha;
#pragma unroll
            for (int e = 0; e < EPT; ++e) acc[e] *= alpha;
        }
#pragma unroll
        for (int u = 0; u < DA_U; ++u) {
            if (s[u] == -FLT_MAX) continue;
            const float p = __expf(s[u] - m);
            l += p;
            const float vstep = group_step_fast(__ushort_as_half(static_cast<unsigned short>(vm[u] >> 16)));
            const float w = p * vstep;
            U = fmaf(p, h2f_lo(vm[u]), U);
            const uint32_t vw[4] = {vc[u].x, vc[u].y, vc[u].z, vc[u].w};
#pragma unroll
            for (int e = 0; e < EPT; ++e) acc[e] = fmaf(w, code_f(vw[e * BITS / 32], (e * BITS) % 32, MASK), acc[e]);
        }
    }

    // merge the KPI key lanes of this CTA
    __shared__ float sm_m[KPI], sm_l[KPI];
    __shared__ float sm_o[KPI][D + 1];
    if (wl == 0) {
        sm_m[kl] = m;
        sm_l[kl] = l;
    }
#pragma unroll
    for (int e = 0; e < EPT; ++e) sm_o[kl][d0 + e] = acc[e] + U;
    __syncthreads();
    float M = -FLT_MAX;
    for (int i = 0; i < KPI; ++i) M = fmaxf(M, sm_m[i]);
    float* out = part + (static_cast<int64_t>(pair) * nsplit + split) * (D + 2);
    for (int d = tid; d < D; d += DA_THREADS) {
        float o = 0.f;
        for (int i = 0; i < KPI; ++i) {
            const float f = sm_l[i] > 0.f ? __expf(sm_m[i] - M) : 0.f;
            o = fmaf(f, sm_o[i][d], o);
        }
        out[2 + d] = o;
    }
    if (tid == 0) {
        float L = 0.f;
        for (int i = 0; i < KPI; ++i) L += sm_l[i] > 0.f ? __expf(sm_m[i] - M) * sm_l[i] : 0.f;
        out[0] = M;
        out[1] = L;
    }
}

// ---------------------------------------------------------------------------------
// decode attention on the tensor cores (4-bit cache), mma.sync m16n8k16, fp32 accumulate.
//
// Codes enter the MMAs raw, as exact fp16 values built with one LOP3 per two codes:
// the low nibble of a byte (the even dim) as 1024 + c, the high nibble (the odd dim)
// as 1024 + 16 c, so no shifts are needed. The group dequantisation x^ = step c + min
// (step = 1/scale) is applied to the small results instead of to every element:
//   scores: the query operand holds q[dim] for even dims and q[dim]/16 for odd ones,
//           in column n = the dim's group (zero elsewhere), so the QK MMA gives per
//           key j and group n  R[j][n] = sum_{dim in n} c_j[dim] q[dim] + QC_n  with
//           QC_n = 1024 sum_{even dim in n} q + 64 sum_{odd dim in n} q, and
//           s_j = sum_n step_jn (R[j][n] - QC_n) + min_jn Q_n,  Q_n = sum_{dim in n} q;
//   values: the PV MMA multiplies the transposed codes by B[j][n] = w_jn = fp16(p_j
//           step_jn), so for dim d of group n: D'[d] = 1024 W_n + f_d sum_j w_jn c_j[d]
//           (f_d = 1 for even, 16 for odd dims) and
//           o[d] = (D'[d] - 1024 W_n) / f_d + U_n,  W_n = sum_j w_jn,  U_n = sum_j p_j min_jn.
// Both MMAs are free to permute their K dimension (dims for QK, keys for PV) as long as
// A and B agree; the layouts below let every thread load contiguous code bytes.
__device__ __forceinline__ uint32_t nib_lo(uint32_t x) {
    // (x & 0x000F000F) | 0x64006400: low nibbles of bytes 0 and 2 as fp16 1024 + c
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(0x000F000Fu), "r"(0x64006400u));
    return r;
}
__device__ __forceinline__ uint32_t nib_hi(uint32_t x) {
    // (x & 0x00F000F0) | 0x64006400: high nibbles of bytes 0 and 2 as fp16 1024 + 16 c
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(0x00F000F0u), "r"(0x64006400u));
    return r;
}
// a[n] for a runtime n without dynamic register indexing (which would go to local memory)
template <int N>
__device__ __forceinline__ float pick(const float (&a)[N], int n) {
    float r = a[0];
#pragma unroll
    for (int i = 1; i < N; ++i) r = (n == i) ? a[i] : r;
    return r;
}
__device__ __forceinline__ uint32_t prmt_sel(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem, bool pred) {
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const int n = pred ? 4 : 0;
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(s), "l"(gmem), "r"(n) : "memory");
}

// One CTA (4 warps) streams the key range [j0, j1) of one (sequence, head) in stages of
// DT_KEYS keys through a cp.async ring of DT_STAGES stages; in a stage warp w owns keys
// [32 w, 32 w + 32) as two 16-key tiles, with one online-softmax update per stage.
// Writes the split's partial {max, sum, unnormalised output} for the combine kernel;
// with a single split (gridDim.y == 1) it does the combine step itself: it folds in the
// fresh key/value of the current token and writes the normalised output o (in the
// interleaved 8-block order when perm != 0).
constexpr int DT_KEYS = 128;

// Position, in 16-byte chunks, of chunk u (key u / 4, chunk u % 4) of a stage's value
// codes at head_dim 128. In the PV step the 16 lanes of a half-warp read 8 bytes each
// from chunks 0-1 (or 2-3) of four keys of one parity; stored in key order those all
// fall in the same 8 banks (a 4-way conflict). Swapping keys 2j and 2j+1 when bit 1 of
// the key is set, and chunks c and c ^ 2 when bit 2 is set, spreads them over all 32
// banks. Bits 1 and 2 of the key index are the same in the stage and in its 16-key
// tile, so the reader applies the same map to its tile-local key. head_dim 64 keeps the
// plain order.
template <int D>
__device__ __forceinline__ int v_chunk(int u) {
    if (D != 128) return u;
    const int key = u >> 2, c = u & 3;
    return ((key ^ ((key >> 1) & 1)) << 2) | (c ^ (((key >> 2) & 1) << 1));
}
#ifndef FLEXQ_DT_STAGES
#define FLEXQ_DT_STAGES 2
#endif
constexpr int DT_STAGES = FLEXQ_DT_STAGES;  // stages of DT_KEYS keys in flight per CTA
static_assert(DT_STAGES >= 2, "the stage loop refills the slot of the previous stage");

// Dynamic shared memory of decode_attn_tc_kernel<D, GS>: the ring of stages, each the
// codes and metadata of DT_KEYS keys and values.
constexpr int dt_smem_bytes(int D, int GS) {
    return DT_STAGES * (2 * DT_KEYS * (D / 2) + 2 * DT_KEYS * (D / GS) * 4);
}

// 7 CTAs per SM at head_dim 64 (all 1024 CTAs of a 32 x 32-head decode in one wave);
// at head_dim 128 FLEXQ_DT_MINB_128 (a build constant, tuned by measurement)
#ifndef FLEXQ_DT_MINB_128
#define FLEXQ_DT_MINB_128 4
#endif
template <int D, int GS>
__global__ void __launch_bounds__(DA_THREADS, D == 64 ? 7 : FLEXQ_DT_MINB_128) decode_attn_tc_kernel(
    const __half* __restrict__ q, int64_t row_stride, const uint8_t* __restrict__ k_codes,
    const uint32_t* __restrict__ k_meta, const uint8_t* __restrict__ v_codes,
    const uint32_t* __restrict__ v_meta, int n_heads, int max_seq, int pos, int chunk,
    float* __restrict__ part, const __half* __restrict__ k_new, const __half* __restrict__ v_new,
    __half* __restrict__ o, int perm, int early_kv, const int32_t* __restrict__ valid_from) {
    constexpr int G = D / GS;              // groups per key: 1, 2 or 4
    constexpr int KB = D / 2;              // code bytes per key
    constexpr int KW = D / 32;             // QK: code words per key and thread (D/4 dims)
    constexpr int VW = D / 64;             // PV: code words per key and thread (D/8 dims)
    constexpr int NMT = D / 16;            // PV M-tiles (16 dims each)
    constexpr int NW = DA_THREADS / 32;
    constexpr int CODE = DT_KEYS * KB;     // code bytes of a stage (keys or values)
    constexpr int META = DT_KEYS * G;      // metadata words of a stage (keys or values)
    constexpr int STAGE = 2 * CODE + 2 * META * 4;
    constexpr int DT_NS = DT_STAGES;       // ring depth (dynamic shared memory, dt_smem_bytes)
    static_assert(NW * 32 == DT_KEYS, "32 keys per warp and stage");
    static_assert((32 * KB / 16) % 32 == 0 && (32 * G) % 32 == 0, "whole copy rounds per warp");
    extern __shared__ __align__(16) uint8_t dt_ring[];
    auto ring = reinterpret_cast<uint8_t (*)[STAGE]>(dt_ring);
    __shared__ float sm_m[NW], sm_l[NW];
    // the warps' output rows reuse the ring once every warp is done with its stages
    float (*const sm_o)[D] = reinterpret_cast<float (*)[D]>(dt_ring);
    static_assert(NW * D * 4 <= DT_NS * STAGE, "the output rows fit in the ring");
    __shared__ float sm_red[NW];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int pair = blockIdx.x, split = blockIdx.y, nsplit = gridDim.y;
    const int b = pair / n_heads, head = pair % n_heads;
    const int64_t slot0 = static_cast<int64_t>(pair) * max_seq;
    // keys [split * chunk, +chunk) of [0, pos), minus the left padding [0, valid_from[b]);
    // valid_from is the caller's, written before the layer call (safe before the launch wait)
    const int vf = valid_from ? valid_from[b] : 0;
    const int j0 = max(split * chunk, vf);
    const int nkeys = min(pos, split * chunk + chunk) - j0;       // keys of this split (may be <= 0)
    static_assert(D <= DA_THREADS, "one thread per output dim");
    const int nst = nkeys > 0 ? (nkeys + DT_KEYS - 1) / DT_KEYS : 0;

    // ---- stage copies: every thread moves CODE/16/128 16-byte units of each code tensor
    // and META/128 metadata words of each metadata tensor; keys past the range are
    // zero-filled (a zero scale gives step 0, so they contribute nothing)
    const uint8_t* kc_src = k_codes + (slot0 + j0) * KB;
    const uint8_t* vc_src = v_codes + (slot0 + j0) * KB;
    const uint32_t* km_src = k_meta + (slot0 + j0) * G;
    const uint32_t* vm_src = v_meta + (slot0 + j0) * G;
    // Each warp copies and later reads only its own 32 keys of a stage (the K and V code
    // rows and metadata of keys [32 w, 32 w + 32)), so a stage needs no CTA barrier: the
    // warp's own copies are waited for, then shared across its lanes by __syncwarp.
    constexpr int WCH = 32 * KB / 16;                 // 16-byte code chunks per warp and stage
    constexpr int WMETA = 32 * G;                     // metadata words per warp and stage
    auto load_stage = [&](int s) {
        uint8_t* st = ring[s % DT_NS];
        const int kbase = s * DT_KEYS + warp * 32;    // this warp's first key of the stage
        const int c0 = warp * WCH, m0w = warp * WMETA;
        if (kbase + 32 <= nkeys) {
            // all 32 keys present: no per-copy predicate or clamped address
            const uint32_t s0 = static_cast<uint32_t>(__cvta_generic_to_shared(st));
            const uint8_t* kc = kc_src + static_cast<int64_t>(kbase) * KB;
            const uint8_t* vc = vc_src + static_cast<int64_t>(kbase) * KB;
            const uint32_t* km = km_src + static_cast<int64_t>(kbase) * G;
            const uint32_t* vm = vm_src + static_cast<int64_t>(kbase) * G;
#pragma unroll
            for (int i = 0; i < WCH / 32; ++i) {
                const int ul = lane + i * 32;
                cp_async16u(s0 + (c0 + ul) * 16, kc + ul * 16);
                cp_async16u(s0 + CODE + v_chunk<D>(c0 + ul) * 16, vc + ul * 16);
            }
#pragma unroll
            for (int i = 0; i < WMETA / 32; ++i) {
                const int ul = lane + i * 32;
                cp_async4u(s0 + 2 * CODE + (m0w + ul) * 4, km + ul);
                cp_async4u(s0 + 2 * CODE + META * 4 + (m0w + ul) * 4, vm + ul);
            }
            return;
        }
#pragma unroll
        for (int i = 0; i < WCH / 32; ++i) {
            const int ul = lane + i * 32;
            const bool ok = kbase + (ul * 16) / KB < nkeys;
            const int64_t off = ok ? static_cast<int64_t>(kbase) * KB + ul * 16 : 0;
            cp_async16(st + (c0 + ul) * 16, kc_src + off, ok);
            cp_async16(st + CODE + v_chunk<D>(c0 + ul) * 16, vc_src + off, ok);
        }
#pragma unroll
        for (int i = 0; i < WMETA / 32; ++i) {
            const int ul = lane + i * 32;
            const bool ok = kbase + ul / G < nkeys;
            const int64_t off = ok ? static_cast<int64_t>(kbase) * G + ul : 0;
            cp_async4(st + 2 * CODE + (m0w + ul) * 4, km_src + off, ok);
            cp_async4(st + 2 * CODE + META * 4 + (m0w + ul) * 4, vm_src + off, ok);
        }
    };
    // Inside a layer call (early_kv) the cached keys/values [0, pos) were written by
    // kernels that completed before the previous kernel's own launch wait, and the
    // previous kernel (the QKV projection) writes only position pos and the query: the
    // first stages are then requested before waiting for it.
    auto prologue = [&]() {
#pragma unroll
        for (int s = 0; s < DT_NS - 1; ++s) {
            if (s < nst) load_stage(s);
            cp_async_commit();
        }
    };
    if (early_kv) prologue();
    pdl_wait();
    pdl_trigger();
    if (!early_kv) prologue();

    // ---- query: group sums (Qg = sum of q, QC = sum of 1024 q_even + 64 q_odd over the
    // group's dims), shared out by the warp: lane l takes dims [DPL l, DPL l + DPL), the
    // LPG lanes of a group add theirs, and every lane reads each group's total
    const __half* qp = q + static_cast<int64_t>(b) * row_stride + head * D;
    constexpr int DPL = D / 32;            // dims per lane (4 or 2)
    constexpr int LPG = GS / DPL;          // lanes per group
    float qg_l = 0.f, qc_l = 0.f;
    if (DPL == 4) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(qp) + lane);
        const float e0 = h2f_lo(w.x), o0 = h2f_hi(w.x), e1 = h2f_lo(w.y), o1 = h2f_hi(w.y);
        qg_l = (e0 + o0) + (e1 + o1);
        qc_l = 1024.f * (e0 + e1) + 64.f * (o0 + o1);
    } else {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(qp) + lane);
        const float e0 = h2f_lo(w), o0 = h2f_hi(w);
        qg_l = e0 + o0;
        qc_l = 1024.f * e0 + 64.f * o0;
    }
#pragma unroll
    for (int off = LPG / 2; off > 0; off >>= 1) {
        qg_l += __shfl_xor_sync(0xffffffffu, qg_l, off);
        qc_l += __shfl_xor_sync(0xffffffffu, qc_l, off);
    }
    float Qg[G], QC[G];
#pragma unroll
    for (int n = 0; n < G; ++n) {
        Qg[n] = __shfl_sync(0xffffffffu, qg_l, n * LPG);
        QC[n] = __shfl_sync(0xffffffffu, qc_l, n * LPG);
    }
    const int tgrp = (t * (D / 4)) / GS;   // group of this thread's QK dims
    const __half sixteenth = __float2half(0.0625f);
    uint32_t bq[2 * KW][2];
#pragma unroll
    for (int ks = 0; ks < 2 * KW; ++ks) {
        // k-step ks uses word ks/2; its registers hold dims (d, d+4) and (d+1, d+5)
        const int d = t * (D / 4) + 8 * (ks / 2) + 2 * (ks % 2);
        if (g == tgrp) {
            bq[ks][0] = pack_half2_bits(qp[d], qp[d + 4]);
            bq[ks][1] = pack_half2_bits(__hmul(qp[d + 1], sixteenth), __hmul(qp[d + 5], sixteenth));
        } else {
            bq[ks][0] = bq[ks][1] = 0u;
        }
    }

    // ---- PV: owner lanes of the w values and the lanes they are gathered from.
    // Lane (g, t) owns group own_n of key g + 8 own_h (G = 1: t < 2; G = 2: all; G = 4:
    // both halves of group t).
    const int own_n = (G == 4) ? t : t % G;
    const int own_h = (G == 4) ? 0 : t / G;
    const bool owner = (G == 4) || (t < 2 * G);
    // b0 needs keys 2t, 2t+1 (half 0) and b1 keys 2t+8, 2t+9 (half 1), group g
    const int gn = g < G ? g : 0;
    const int src_a0 = 4 * (2 * t) + gn;                              // half 0: owner t = n
    const int src_a1 = 4 * (2 * t + 1) + gn;
    const int src_b0 = 4 * (2 * t) + ((G == 4) ? gn : G + gn);        // half 1: t = G + n (G < 4)
    const int src_b1 = 4 * (2 * t + 1) + ((G == 4) ? gn : G + gn);

    float m = -FLT_MAX, lsum = 0.f, Wl = 0.f, Ul = 0.f;
    float oacc[NMT][4];
#pragma unroll
    for (int i = 0; i < NMT; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;

    // Per warp and stage: after __syncwarp, stage s has landed for every lane and every
    // lane has finished stage s - 1, whose slot then takes stage s + DT_NS - 1.
    for (int s = 0; s < nst; ++s) {
        cp_async_wait<DT_NS - 2>();
        __syncwarp();
        if (s + DT_NS - 1 < nst) load_stage(s + DT_NS - 1);
        cp_async_commit();
        const int kw0 = s * DT_KEYS + warp * 32;                 // the warp's first key
        if (kw0 < nkeys) {
            const uint8_t* st = ring[s % DT_NS];
            const uint32_t* kmeta = reinterpret_cast<const uint32_t*>(st + 2 * CODE) + warp * 32 * G;
            const uint32_t* vmeta = reinterpret_cast<const uint32_t*>(st + 2 * CODE + META * 4) + warp * 32 * G;
            // ---- scores of the two tiles: keys (tile 16 + g) and (tile 16 + g + 8)
            float sc[2][2];
#pragma unroll
            for (int tile = 0; tile < 2; ++tile) {
                const uint8_t* kc = st + (warp * 32 + tile * 16) * KB + t * (D / 8);
                uint32_t x0[KW], x8[KW];
                if (KW == 4) {
                    const uint4 a = *reinterpret_cast<const uint4*>(kc + g * KB);
                    const uint4 c = *reinterpret_cast<const uint4*>(kc + (g + 8) * KB);
                    x0[0] = a.x; x0[1 % KW] = a.y; x0[2 % KW] = a.z; x0[3 % KW] = a.w;
                    x8[0] = c.x; x8[1 % KW] = c.y; x8[2 % KW] = c.z; x8[3 % KW] = c.w;
                } else {
                    const uint2 a = *reinterpret_cast<const uint2*>(kc + g * KB);
                    const uint2 c = *reinterpret_cast<const uint2*>(kc + (g + 8) * KB);
                    x0[0] = a.x; x0[1 % KW] = a.y;
                    x8[0] = c.x; x8[1 % KW] = c.y;
                }
                // two accumulator sets (even and odd k-steps) halve the dependent MMA chain
                float sacc[4] = {0.f, 0.f, 0.f, 0.f}, sacc2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int w = 0; w < KW; ++w) {
                    const uint32_t y0 = x0[w] >> 8, y8 = x8[w] >> 8;
                    const uint32_t a0[4] = {nib_lo(x0[w]), nib_lo(x8[w]), nib_hi(x0[w]), nib_hi(x8[w])};
                    mma16816(sacc, a0, bq[2 * w][0], bq[2 * w][1]);
                    const uint32_t a1[4] = {nib_lo(y0), nib_lo(y8), nib_hi(y0), nib_hi(y8)};
                    mma16816(sacc2, a1, bq[2 * w + 1][0], bq[2 * w + 1][1]);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) sacc[i] += sacc2[i];
                // per key: sum over the groups this lane holds (columns 2t, 2t+1)
                float s0 = 0.f, s8 = 0.f;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int n = 2 * t + u;
                    if (n < G) {
                        const uint32_t m0 = kmeta[(tile * 16 + g) * G + n], m8 = kmeta[(tile * 16 + g + 8) * G + n];
                        const float qc = pick(QC, n), qg = pick(Qg, n);
                        const float st0 = group_step_fast(__ushort_as_half(static_cast<unsigned short>(m0 >> 16)));
                        const float st8 = group_step_fast(__ushort_as_half(static_cast<unsigned short>(m8 >> 16)));
                        s0 += fmaf(st0, sacc[u] - qc, h2f_lo(m0) * qg);
                        s8 += fmaf(st8, sacc[2 + u] - qc, h2f_lo(m8) * qg);
                    }
                }
                if (G == 4) {
                    s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
                    s8 += __shfl_xor_sync(0xffffffffu, s8, 1);
                }
                s0 = __shfl_sync(0xffffffffu, s0, lane & ~3);
                s8 = __shfl_sync(0xffffffffu, s8, lane & ~3);
                const int kt = kw0 + tile * 16;
                sc[tile][0] = (kt + g < nkeys) ? s0 : -FLT_MAX;
                sc[tile][1] = (kt + g + 8 < nkeys) ? s8 : -FLT_MAX;
            }
            // ---- one online-softmax update for the 32 keys
            float tmax = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
            if (tmax > m) {                        // warp-uniform
                const float alpha = __expf(m - tmax);
                m = tmax;
                lsum *= alpha;
                Wl *= alpha;
                Ul *= alpha;
#pragma unroll
                for (int i = 0; i < NMT; ++i) {
                    oacc[i][0] *= alpha;
                    oacc[i][1] *= alpha;
                    oacc[i][2] *= alpha;
                    oacc[i][3] *= alpha;
                }
            }
            float pr[2][2];
#pragma unroll
            for (int tile = 0; tile < 2; ++tile)
#pragma unroll
                for (int h = 0; h < 2; ++h) pr[tile][h] = sc[tile][h] == -FLT_MAX ? 0.f : __expf(sc[tile][h] - m);
            if (t == 0) lsum += (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
            // ---- values
#pragma unroll
            for (int tile = 0; tile < 2; ++tile) {
                // owner lanes: w = fp16(p step) of (key g + 8 h, group n); running W, U
                uint32_t wb[2] = {0u, 0u};
#pragma unroll
                for (int hh = 0; hh < ((G == 4) ? 2 : 1); ++hh) {
                    const int h = (G == 4) ? hh : own_h;
                    if (owner) {
                        const uint32_t mv = vmeta[(tile * 16 + g + 8 * h) * G + own_n];
                        const float stp = group_step_fast(__ushort_as_half(static_cast<unsigned short>(mv >> 16)));
                        const float pk = h ? pr[tile][1] : pr[tile][0];
                        const __half w16 = __float2half_rn(pk * stp);
                        Wl += __half2float(w16);
                        Ul = fmaf(pk, h2f_lo(mv), Ul);
                        wb[hh] = static_cast<uint32_t>(__half_as_ushort(w16));
                    }
                }
                // gather the B operand: keys 2t, 2t+1 (b0) and 2t+8, 2t+9 (b1) of group g
                const uint32_t lo_a = __shfl_sync(0xffffffffu, wb[0], src_a0);
                const uint32_t lo_b = __shfl_sync(0xffffffffu, wb[0], src_a1);
                const uint32_t hi_a = __shfl_sync(0xffffffffu, wb[(G == 4) ? 1 : 0], src_b0);
                const uint32_t hi_b = __shfl_sync(0xffffffffu, wb[(G == 4) ? 1 : 0], src_b1);
                const uint32_t b0 = g < G ? (lo_a | (lo_b << 16)) : 0u;
                const uint32_t b1 = g < G ? (hi_a | (hi_b << 16)) : 0u;
                // A: transposed codes; thread g holds D/16 bytes (dims D/8 g ..) of keys
                // 2t, 2t+1, 2t+8, 2t+9
                const uint8_t* vc = st + CODE + (warp * 32 + tile * 16) * KB + g * (D / 16);
                uint32_t vk[4][VW > 0 ? VW : 1];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int key = 2 * t + (u & 1) + 8 * (u >> 1);
                    if (VW == 2) {
                        // 16-byte chunk g/2 of the key sits where v_chunk put it
                        const int pk = key ^ ((key >> 1) & 1), pc = (g >> 1) ^ (((key >> 2) & 1) << 1);
                        const uint2 a = *reinterpret_cast<const uint2*>(st + CODE + (warp * 32 + tile * 16 + pk) * KB +
                                                                        pc * 16 + (g & 1) * 8);
                        vk[u][0] = a.x;
                        vk[u][1 % (VW > 0 ? VW : 1)] = a.y;
                    } else {
                        vk[u][0] = *reinterpret_cast<const uint32_t*>(vc + key * KB);
                    }
                }
#pragma unroll
                for (int mt = 0; mt < NMT; ++mt) {
                    const int wi = mt / 4, by = mt % 4;
                    // byte `by` of key 2t -> bytes 0,1 and of key 2t+1 -> bytes 2,3
                    const uint32_t sel = static_cast<uint32_t>(by * 0x11 + (4 + by) * 0x1100);
                    const uint32_t x1 = prmt_sel(vk[0][wi], vk[1][wi], sel);
                    const uint32_t x2 = prmt_sel(vk[2][wi], vk[3][wi], sel);
                    const uint32_t a[4] = {nib_lo(x1), nib_hi(x1), nib_lo(x2), nib_hi(x2)};
                    mma16816(oacc[mt], a, b0, b1);
                }
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();                       // every warp is done with the ring (sm_o reuses it)

    // ---- warp result: W_n, U_n per group (sum over the owner lanes), then the rows
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
        Wl += __shfl_xor_sync(0xffffffffu, Wl, off);
        Ul += __shfl_xor_sync(0xffffffffu, Ul, off);
    }
    if (G == 1) {                          // owners t = 0, 1 (t = 2, 3 hold 0)
        Wl += __shfl_xor_sync(0xffffffffu, Wl, 1);
        Ul += __shfl_xor_sync(0xffffffffu, Ul, 1);
        Wl += __shfl_xor_sync(0xffffffffu, Wl, 2);
        Ul += __shfl_xor_sync(0xffffffffu, Ul, 2);
    } else if (G == 2) {                   // owners of group t % 2: t and t ^ 2
        Wl += __shfl_xor_sync(0xffffffffu, Wl, 2);
        Ul += __shfl_xor_sync(0xffffffffu, Ul, 2);
    }
    // now lane t of every quad holds W, U of group t (G = 1: all lanes hold group 0)
    float Wn[2], Un[2];                    // groups 2t and 2t + 1
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int n = (2 * t + u) < G ? 2 * t + u : 0;
        Wn[u] = __shfl_sync(0xffffffffu, Wl, (lane & ~3) | (G == 1 ? 0 : n));
        Un[u] = __shfl_sync(0xffffffffu, Ul, (lane & ~3) | (G == 1 ? 0 : n));
    }
#pragma unroll
    for (int mt = 0; mt < NMT; ++mt) {
        const int de = 2 * (g * (D / 16) + mt);        // even dim of row g; row g + 8 is de + 1
        const int n = de / GS;
        if (n / 2 == t) {
            // static register indices only (a runtime index would move oacc to local memory)
            const bool odd_col = (n % 2) != 0;
            const float ev = odd_col ? oacc[mt][1] : oacc[mt][0];
            const float od = odd_col ? oacc[mt][3] : oacc[mt][2];
            const float W = odd_col ? Wn[1] : Wn[0], U = odd_col ? Un[1] : Un[0];
            sm_o[warp][de] = ev - 1024.f * W + U;
            sm_o[warp][de + 1] = (od - 1024.f * W) * 0.0625f + U;
        }
    }
    if (lane == 0) {
        sm_m[warp] = m;
        sm_l[warp] = lsum;
    }
    __syncthreads();
    if (nsplit == 1) {
        // single split: the combine step here. Fresh score q . k_new (one dim per thread).
        const int d = threadIdx.x;
        const int64_t off = static_cast<int64_t>(b) * row_stride + head * D + d;
        float sn = d < D ? __half2float(qp[d]) * __half2float(k_new[off]) : 0.f;
#pragma unroll
        for (int w = 16; w > 0; w >>= 1) sn += __shfl_xor_sync(0xffffffffu, sn, w);
        if (lane == 0) sm_red[warp] = sn;
        __syncthreads();
        float snew = 0.f;
#pragma unroll
        for (int i = 0; i < NW; ++i) snew += sm_red[i];
        float M = snew;
#pragma unroll
        for (int i = 0; i < NW; ++i)
            if (sm_l[i] > 0.f) M = fmaxf(M, sm_m[i]);
        if (d < D) {
            const float fn = __expf(snew - M);
            float L = fn, acc = fn * __half2float(v_new[off]);
#pragma unroll
            for (int i = 0; i < NW; ++i) {
                if (!(sm_l[i] > 0.f)) continue;
                const float f = __expf(sm_m[i] - M);
                L = fmaf(f, sm_l[i], L);
                acc = fmaf(f, sm_o[i][d], acc);
            }
            // perm: interleaved 8-block order for the next GEMM (element k -> 2(k%4) + (k/4)%2)
            const int dd = perm ? ((d & ~7) | ((d & 3) << 1) | ((d >> 2) & 1)) : d;
            o[static_cast<int64_t>(b) * n_heads * D + head * D + dd] = __float2half_rn(acc / L);
        }
        return;
    }
    float M = -FLT_MAX;
#pragma unroll
    for (int i = 0; i < NW; ++i) M = fmaxf(M, sm_m[i]);
    float* out = part + (static_cast<int64_t>(pair) * nsplit + split) * (D + 2);
    for (int d = threadIdx.x; d < D; d += DA_THREADS) {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < NW; ++i) {
            const float f = sm_l[i] > 0.f ? __expf(sm_m[i] - M) : 0.f;
            acc = fmaf(f, sm_o[i][d], acc);
        }
        out[2 + d] = acc;
    }
    if (threadIdx.x == 0) {
        float L = 0.f;
#pragma unroll
        for (int i = 0; i < NW; ++i) L += sm_l[i] > 0.f ? __expf(sm_m[i] - M) * sm_l[i] : 0.f;
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
                                                                __half* __restrict__ o, int perm) {
    pdl_wait();
    pdl_trigger();
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
    // perm: interleaved 8-block order for the next GEMM (element k -> 2(k%4) + (k/4)%2)
    const int dd = perm ? ((d & ~7) | ((d & 3) << 1) | ((d >> 2) & 1)) : d;
    o[static_cast<int64_t>(b) * n_heads * D + head * D + dd] = __float2half_rn(acc / L);
}

template <int D>
__global__ void __launch_bounds__(PA_THREADS) prefill_attn_kernel(const __half* __restrict__ q,
                                                                  const __half* __restrict__ k,
                                                                  const __half* __restrict__ v,
                                                                  int64_t row_stride,
                                                                  __half* __restrict__ o, int seq,
                                                                  int n_heads,
                                                                  const int32_t* __restrict__ valid_from) {
    constexpr int LD = D + 8;                  // padded smem row (halves): conflict-free ldmatrix
    pdl_wait();
    pdl_trigger();
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
    // left padding: keys below valid_from[b] are never attended; a query row with no
    // visible key (a pad row) gets a zero output
    const int vf = valid_from ? min(max(valid_from[b], 0), seq) : 0;

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
    const int kb0 = vf / PA_BK;                // first key block holding a real token
    if (kb0 < nkb) load_kv(kb0, kb0 & 1);
    cp_async_commit();

    uint32_t qa[D / 16][4];
    float oacc[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    float mrow[2] = {-FLT_MAX, -FLT_MAX}, lrow[2] = {0.f, 0.f};
    constexpr float LOG2E = 1.4426950408889634f;

    for (int kb = kb0; kb < nkb; ++kb) {
        const int buf = kb & 1;
        if (kb + 1 < nkb) load_kv(kb + 1, buf ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (kb == kb0) {
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
                if (key > qi || key >= seq || key < vf) val = -FLT_MAX;
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
    cp_async_wait<0>();                        // a tile of pad rows visits no key block
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
        const float inv = lrow[r] > 0.f ? 1.f / lrow[r] : 0.f;     // a pad row: zero output
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
    const int max_by_len = (pos + 127) / 128;        // at least 128 keys per split
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
                       int64_t row_stride, void* o, int batch, int pos, void* ws, bool perm, cudaStream_t st,
                       bool early_kv) {
    const int pairs = batch * c->n_heads;
    const int ns = decode_attn_nsplit(pairs, pos);
    const int chunk = ns > 0 ? (pos + ns - 1) / ns : 0;
    float* part = static_cast<float*>(ws);
    const __half* qh = static_cast<const __half*>(q);
    const uint8_t* kc = static_cast<const uint8_t*>(c->k_codes);
    const uint8_t* vc = static_cast<const uint8_t*>(c->v_codes);
    const uint32_t* km = static_cast<const uint32_t*>(c->k_meta);
    const uint32_t* vm = static_cast<const uint32_t*>(c->v_meta);
    const __half* kn = static_cast<const __half*>(k_new);
    const __half* vn = static_cast<const __half*>(v_new);
    __half* oh = static_cast<__half*>(o);
    const int D = c->head_dim, B = c->cfg.num_bits, G = c->cfg.group_size;
    // 4-bit caches with a single split finish in the split kernel (no combine launch)
    bool combined = false;
    if (ns > 0) {
        const dim3 grid(pairs, ns);
#define SPLIT(D_, B_, G_)                                                                                 \
    launch_k(decode_attn_split_kernel<D_, B_, G_>, grid, dim3(DA_THREADS), 0, st, true, qh, row_stride, kc, km, vc, \
             vm, c->n_heads, c->max_seq, pos, chunk, part, c->valid_from)
#define MMA(D_, G_)                                                                                      \
    do {                                                                                                 \
        set_smem_once(decode_attn_tc_kernel<D_, G_>, dt_smem_bytes(D_, G_));                            \
        launch_k(decode_attn_tc_kernel<D_, G_>, grid, dim3(DA_THREADS), dt_smem_bytes(D_, G_), st, true, qh, \
                 row_stride, kc, km, vc, vm, c->n_heads, c->max_seq, pos, chunk, part, kn, vn, oh, perm ? 1 : 0, \
                 early_kv ? 1 : 0, c->valid_from);                                                       \
    } while (0)
        if (B == 4) {
            if (D == 64 && G == 64) MMA(64, 64);
            else if (D == 64) MMA(64, 32);
            else if (G == 64) MMA(128, 64);
            else MMA(128, 32);
            combined = (ns == 1);
        } else {
            if (D == 64 && G == 64) SPLIT(64, 8, 64);
            else if (D == 64) SPLIT(64, 8, 32);
            else if (G == 64) SPLIT(128, 8, 64);
            else SPLIT(128, 8, 32);
        }
#undef SPLIT
#undef MMA
    }
    if (!combined) {
        if (D == 64)
            launch_k(decode_attn_combine_kernel<64>, dim3(pairs), dim3(64), 0, st, true, qh, kn, vn, row_stride,
                     c->n_heads, ns, static_cast<const float*>(part), oh, perm ? 1 : 0);
        else
            launch_k(decode_attn_combine_kernel<128>, dim3(pairs), dim3(128), 0, st, true, qh, kn, vn, row_stride,
                     c->n_heads, ns, static_cast<const float*>(part), oh, perm ? 1 : 0);
    }
    return launch_status();
}

size_t prefill_attn_smem(int D) { return static_cast<size_t>(PA_BQ + 4 * PA_BK) * (D + 8) * 2; }

int prefill_attn_launch(const void* q, const void* k, const void* v, int64_t row_stride, void* o, int batch,
                        int seq, int n_heads, int head_dim, const int32_t* valid_from, cudaStream_t st) {
    if (batch == 0 || seq == 0) return FLEX_OK;
    const dim3 grid((seq + PA_BQ - 1) / PA_BQ, n_heads, batch);
    const size_t smem = prefill_attn_smem(head_dim);
    const __half* qh = static_cast<const __half*>(q);
    const __half* kh = static_cast<const __half*>(k);
    const __half* vh = static_cast<const __half*>(v);
    __half* oh = static_cast<__half*>(o);
    if (head_dim == 64) {
        set_smem_once(prefill_attn_kernel<64>, (int)smem);
        launch_k(prefill_attn_kernel<64>, grid, dim3(PA_THREADS), smem, st, true, qh, kh, vh, row_stride, oh, seq,
                 n_heads, valid_from);
    } else {
        set_smem_once(prefill_attn_kernel<128>, (int)smem);
        launch_k(prefill_attn_kernel<128>, grid, dim3(PA_THREADS), smem, st, true, qh, kh, vh, row_stride, oh, seq,
                 n_heads, valid_from);
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
    FLEX_REQUIRE(row_stride % 8 == 0, FLEX_ERR_ALIGN);                  // 16-byte rows (vector loads)
    const int64_t need = decode_attn_ws_bytes(batch * cache->n_heads, cache->head_dim, pos);
    FLEX_REQUIRE(ws != nullptr && ws_bytes >= need, FLEX_ERR_WORKSPACE);
    FLEX_REQUIRE(aligned16(ws), FLEX_ERR_ALIGN);
    return decode_attn_launch(cache, q, k_new, v_new, row_stride, o, batch, pos, ws, false, as_stream(stream), false);
}

extern "C" int flex_prefill_attention(const void* q, const void* k, const void* v, int64_t row_stride, void* o,
                                      int32_t batch, int32_t seq, int32_t n_heads, int32_t head_dim,
                                      const int32_t* valid_from, void* stream) {
    FLEX_REQUIRE(q && k && v && o, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(batch >= 0 && seq >= 0 && n_heads > 0, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(head_dim == 64 || head_dim == 128, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(row_stride >= static_cast<int64_t>(n_heads) * head_dim && row_stride % 8 == 0,
                 FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(o), FLEX_ERR_ALIGN);
    FLEX_REQUIRE(valid_from == nullptr || (reinterpret_cast<uintptr_t>(valid_from) & 3u) == 0, FLEX_ERR_ALIGN);
    return prefill_attn_launch(q, k, v, row_stride, o, batch, seq, n_heads, head_dim, valid_from, as_stream(stream));
}

// ---- decode attention with library-owned scratch ---------------------------------------
//
// Same kernels and launch as flex_decode_attention; only the split-KV partials live in a
// buffer inside this library instead of a caller-supplied workspace, so the call itself
// allocates nothing. Every partial the combine kernel reads is written earlier in the same
// call by the split kernel, so the buffer needs no clearing, at load time or between calls.
namespace flexq {
namespace {

constexpr int64_t kDecodeScratchBytes = FLEX_DECODE_ATTENTION_STATIC_MAX_BYTES;
__device__ __align__(256) unsigned char g_decode_scratch[kDecodeScratchBytes];

constexpr int kScratchDevices = 64;
void* g_decode_scratch_ptr[kScratchDevices];
std::mutex g_decode_scratch_mu;

// Device address of this device's copy of g_decode_scratch, looked up on the first call
// made with the device current and cached for the life of the process. nullptr if the
// lookup fails.
void* decode_scratch() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kScratchDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_decode_scratch_mu);
    if (g_decode_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return nullptr;
        g_decode_scratch_ptr[dev] = p;
    }
    return g_decode_scratch_ptr[dev];
}

}  // namespace
}  // namespace flexq

extern "C" int flex_decode_attention_noalloc(const flex_kv_cache* cache, const void* q, const void* k_new,
                                             const void* v_new, int64_t row_stride, void* o, int32_t batch,
                                             int32_t pos, void* stream) {
    const int rc = validate_cache(cache);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(q && k_new && v_new && o, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(batch > 0 && batch <= cache->batch, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(pos >= 0 && pos < cache->max_seq, FLEX_ERR_SHAPE);
    FLEX_REQUIRE(row_stride >= static_cast<int64_t>(cache->n_heads) * cache->head_dim, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(aligned16(q) && aligned16(k_new) && aligned16(v_new) && aligned16(o), FLEX_ERR_ALIGN);
    FLEX_REQUIRE(row_stride % 8 == 0, FLEX_ERR_ALIGN);                  // 16-byte rows (vector loads)
    const int64_t need = decode_attn_ws_bytes(batch * cache->n_heads, cache->head_dim, pos);
    FLEX_REQUIRE(need <= kDecodeScratchBytes, FLEX_ERR_SCRATCH_LIMIT);
    void* scratch = decode_scratch();
    FLEX_REQUIRE(scratch != nullptr, FLEX_ERR_CUDA);
    return decode_attn_launch(cache, q, k_new, v_new, row_stride, o, batch, pos, scratch, false,
                              as_stream(stream), false);
}
