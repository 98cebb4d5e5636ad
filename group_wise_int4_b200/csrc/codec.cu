// Group-wise int4/int8 compression and decompression (the walkthrough page «FlexGen 单 GPU 高吞吐大模型推理引擎：论文解读与源码实战指南»,
// section 6.3: compress / decompress of a CompressionConfig(num_bits, group_size,
// group_dim, symmetric=False) with a packed uint8 data tensor and an fp16 per-group
// scale).
//
// Both directions are pure HBM streams (2 + bits/8 + 4/group_size bytes per element),
// so the kernels are shaped for bandwidth: 16-byte vector loads that bypass L1,
// streaming stores, several independent vectors in flight per thread, and a
// grid-stride loop sized to the SM count.
//
// Two layouts:
//   contiguous - the group dimension is the last one: the tensor is a flat sequence of
//                groups; a group's lanes (one or two vectors each) reduce min/max
//                with shuffles.
//   strided    - the group dimension has inner extent `inner` > 1 after it: gs/8
//                lanes share 8 adjacent columns (one 16-byte vector per row), each
//                holding 8 of the group's rows in registers; they combine min/max with
//                shuffles and quantise their rows without reading them again (one column
//                per thread when the width is not a multiple of 8).
#include "quant.cuh"

namespace flexq {
namespace {

constexpr int kThreads = 256;
// Pairs of vectors in flight per thread (contiguous compress) and resident blocks per SM
// the register budget is sized for: build constants, tuned by measurement.
#ifndef FLEXQ_CODEC_UNROLL
#define FLEXQ_CODEC_UNROLL 1
#endif
#ifndef FLEXQ_CODEC_MINB
#define FLEXQ_CODEC_MINB 4
#endif
#ifndef FLEXQ_DEC_UNROLL
#define FLEXQ_DEC_UNROLL 8
#endif
constexpr int kUnroll = FLEXQ_CODEC_UNROLL;
constexpr int kMinBlocks = FLEXQ_CODEC_MINB;

// Division by a divisor d fixed for a launch (groups per row, column items per group
// row): Granlund and Montgomery's unsigned division by a run-time invariant integer
// ("Division by Invariant Integers using Multiplication", 1994, figure 4.1). With
// l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1, every 32-bit n gives
//   n / d = (t + ((n - t) >> 1)) >> (l - 1),  t = umulhi(m, n)   (d >= 2).
struct DivU32 {
    uint32_t m = 0;
    int l = 0;                                 // 0: ng == 1
};
inline DivU32 make_div(int64_t dd) {
    DivU32 d;
    if (dd < 2 || dd >= 0x7FFFFFFF) return d;
    const uint32_t dv = static_cast<uint32_t>(dd);
    int l = 0;
    while ((1ull << l) < dv) ++l;
    d.l = l;
    d.m = static_cast<uint32_t>(((1ull << 32) * ((1ull << l) - dv)) / dv + 1);
    return d;
}
__device__ __forceinline__ uint32_t div_u32(uint32_t n, const DivU32& d) {
    const uint32_t t = __umulhi(d.m, n);
    return (t + ((n - t) >> 1)) >> (d.l - 1);
}

// n / d and n % d for 0 <= n; the 32-bit form when n fits, else 64-bit division.
__device__ __forceinline__ void divmod(int64_t n, int64_t d, const DivU32& dv, int64_t& quo, int64_t& rem) {
    if (d == 1) {
        quo = n;
        rem = 0;
        return;
    }
    quo = (dv.l > 0 && n < 0x7FFFFFFF) ? static_cast<int64_t>(div_u32(static_cast<uint32_t>(n), dv)) : n / d;
    rem = n - quo * d;
}

// ---------------------------------------------------------------------------------
// contiguous compress: G groups of GS fp16, codes G x (GS*BITS/8) bytes, meta G half2.
// With 4-bit codes a lane holds two 16-byte vectors of one group, vectors sub and
// sub + L, so that each load instruction of a warp still covers whole 32-byte sectors,
// while the group's min/max shuffle reduction and its scale (an fp32 division) are
// computed once per 16 values instead of once per 8: the 4-bit kernel is bound by instruction
// issue about as much as by HBM, and those two steps were a fifth of its instructions
// (76% -> 92% of HBM at group 64, 72% -> 95% at group 128). With 8-bit codes, whose
// stores are twice as wide, splitting a lane's codes in two cost 4%, so there a lane
// holds one vector of each of two groups.
template <int BITS>
constexpr int contig_vpl() { return BITS == 4 ? 2 : 1; }

template <int BITS, int GS>
__global__ void __launch_bounds__(kThreads, kMinBlocks) compress_contig_kernel(const __half* __restrict__ x,
                                                                   uint8_t* __restrict__ codes,
                                                                   uint32_t* __restrict__ meta,
                                                                   int64_t G) {
    constexpr int V = contig_vpl<BITS>();   // vectors per lane and group
    constexpr int L = GS / (8 * V);         // lanes per group
    constexpr int GPW = 32 / L;             // groups per warp and step
    constexpr int U = kUnroll * 2 / V;      // groups per lane and step
    const int lane = threadIdx.x & 31;
    const int sub = lane % L;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    const int64_t stride = nwarps * GPW;

    auto load = [&](uint4 (&v)[U][V], int64_t base) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t g = base + u * stride + lane / L;
            const __half* p = x + g * GS + sub * 8;
#pragma unroll
            for (int j = 0; j < V; ++j) v[u][j] = g < G ? ld_stream_v4(p + j * L * 8) : make_uint4(0, 0, 0, 0);
        }
    };
    auto process = [&](const uint4 (&v)[U][V], int64_t base) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t g = base + u * stride + lane / L;
            __half2 hmn, hmx;
            minmax8(v[u][0], hmn, hmx);
#pragma unroll
            for (int j = 1; j < V; ++j) {
                __half2 mn1, mx1;
                minmax8(v[u][j], mn1, mx1);
                hmn = __hmin2(hmn, mn1);
                hmx = __hmax2(hmx, mx1);
            }
            float mn, mx;
            group_minmax<L>(hmn, hmx, mn, mx);
            const __half s16 = group_scale16<BITS>(mn, mx);
            const float s = __half2float(s16);
            if (g < G) {
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    if (BITS == 4) {
                        st_stream_u32(codes + g * (GS / 2) + (sub + j * L) * 4, quant8_4bit(v[u][j], mn, s));
                    } else {
                        st_stream_v2(codes + g * GS + (sub + j * L) * 8, quant8_8bit(v[u][j], mn, s));
                    }
                }
                if (sub == 0) meta[g] = pack_half2_bits(stored_min16(mn), s16);
            }
        }
    };
    // software pipelined: the next step's vectors are requested before this step's are
    // quantised, so the loads of one step overlap the arithmetic of the previous one
    int64_t base = warp * GPW;
    uint4 v[U][V];
    load(v, base);
    while (base < G) {
        const int64_t next = base + stride * U;
        uint4 nv[U][V];
        load(nv, next);
        process(v, base);
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int j = 0; j < V; ++j) v[u][j] = nv[u][j];
        base = next;
    }
}

// contiguous decompress: one item = 8 consecutive values (4 or 8 code bytes in, one
// 16-byte vector out), so a warp's loads and stores each cover one contiguous span.
constexpr int kDecUnroll = FLEXQ_DEC_UNROLL;

template <int BITS, int GS>
__global__ void __launch_bounds__(kThreads, kMinBlocks) decompress_contig_kernel(const uint8_t* __restrict__ codes,
                                                                     const uint32_t* __restrict__ meta,
                                                                     __half* __restrict__ y,
                                                                     int64_t items) {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
    for (int64_t base = tid; base < items; base += nthreads * kDecUnroll) {
        // codes and the group's metadata word are both requested before any is used: the
        // metadata of a tensor larger than L2 comes from DRAM too, and a load issued only
        // when its item is converted would add one memory round trip per item
        uint2 c[kDecUnroll];
        uint32_t mw[kDecUnroll];
#pragma unroll
        for (int u = 0; u < kDecUnroll; ++u) {
            const int64_t it = base + u * nthreads;
            c[u] = make_uint2(0u, 0u);
            mw[u] = 0u;
            if (it < items) {
                if (BITS == 4) {
                    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(c[u].x) : "l"(codes + it * 4));
                } else {
                    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                                 : "=r"(c[u].x), "=r"(c[u].y)
                                 : "l"(codes + it * 8));
                }
                // the 8 values lie in one group (GS >= 32)
                mw[u] = __ldg(meta + (it * 8) / GS);
            }
        }
#pragma unroll
        for (int u = 0; u < kDecUnroll; ++u) {
            const int64_t it = base + u * nthreads;
            if (it >= items) continue;
            const uint32_t m = mw[u];
            const float mn = h2f_lo(m);
            const float step = group_step(__ushort_as_half(static_cast<unsigned short>(m >> 16)));
            uint32_t out[4];
            if (step == 0.0f) {                  // constant group: every value is min
#pragma unroll
                for (int k = 0; k < 4; ++k) out[k] = (m & 0xFFFFu) * 0x10001u;
            } else if (BITS == 4) {
                const uint32_t w = c[u].x;       // byte k = q[2k] | q[2k+1] << 4
#pragma unroll
                for (int k = 0; k < 4; ++k) out[k] = dequant_two((w >> (8 * k)) & 15u, (w >> (8 * k + 4)) & 15u, step, mn);
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t w = k < 2 ? c[u].x : c[u].y;
                    const int sh = 16 * (k & 1);
                    out[k] = dequant_two((w >> sh) & 0xFFu, (w >> (sh + 8)) & 0xFFu, step, mn);
                }
            }
            st_stream_v4(y + it * 8, make_uint4(out[0], out[1], out[2], out[3]));
        }
    }
}

// ---------------------------------------------------------------------------------
// strided compress, one pass: x viewed as [outer][ng*GS][inner]; a work item is (o, g,
// 8 columns) and NS = GS/RPS lanes share it, each holding RPS of the group's rows in
// registers. Lane = IPW slice + ci: a warp covers IPW = 32/NS adjacent items (ci), so
// every load instruction reads 16 IPW contiguous bytes per row slice. The slices combine
// min/max with shuffles (lane offsets IPW, 2 IPW, ...) and then quantise their own rows
// with no second read.
// Rows per slice: 8, or 16 for groups of 128 rows, so that a slice still spans at most 8
// lanes and a warp reads at least 64 contiguous bytes of every row (with 8 rows per slice
// a 128-row group took 16 lanes and left 32-byte row pieces: about 1.3-2.3 TB/s).
// 8-bit codes take 16 rows per slice at every group size: with 8 (and a register budget for
// 4 blocks per SM) the kernel spilled and fell from 5.0 to 2.9 TB/s between 1 and 4 GiB
// tensors at g64; with 16 rows per slice (and 2 blocks per SM) it holds 5.1-5.6 TB/s.
template <int BITS>
constexpr int strided_rps(int gs) { return (gs >= 128 || BITS == 8) ? 16 : 8; }

template <int BITS, int GS>
__global__ void __launch_bounds__(kThreads, (GS >= 128 || BITS == 8) ? 2 : kMinBlocks) compress_strided_1pass_kernel(const __half* __restrict__ x,
                                                                          uint8_t* __restrict__ codes,
                                                                          uint32_t* __restrict__ meta, int64_t outer,
                                                                          int64_t ng, int64_t inner) {
    constexpr int RPS = strided_rps<BITS>(GS);       // rows per slice
    constexpr int NS = GS / RPS;               // slices (lanes) per item
    constexpr int IPW = 32 / NS;               // items per warp
    constexpr int CB = GS * BITS / 8;          // code rows per group
    const int lane = threadIdx.x & 31, ci = lane % IPW, slice = lane / IPW;
    const int64_t cols = inner / 8;
    const int64_t items = outer * ng * cols;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    for (int64_t base = warp * IPW; base < items; base += nwarps * IPW) {
        const int64_t it = base + ci;
        const bool ok = it < items;            // the lanes of an item agree
        // the item's group row and column: one division for 8-bit codes (2-5% faster);
        // the 4-bit kernels keep % and / (with one division they were 7-9% slower)
        int64_t og = 0, cv = 0;
        if constexpr (BITS == 8) {
            og = ok ? it / cols : 0;
            cv = ok ? it - og * cols : 0;
        } else {
            cv = ok ? it % cols : 0;
            og = ok ? it / cols : 0;
        }
        const int64_t c0 = cv * 8;
        const __half* src = x + (og * GS + slice * RPS) * inner + c0;
        uint4 v[RPS];
#pragma unroll
        for (int r = 0; r < RPS; ++r) v[r] = ok ? ld_stream_v4(src + r * inner) : make_uint4(0u, 0u, 0u, 0u);
        __half2 m2[4], M2[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t w0 = k == 0 ? v[0].x : (k == 1 ? v[0].y : (k == 2 ? v[0].z : v[0].w));
            m2[k] = M2[k] = *reinterpret_cast<const __half2*>(&w0);
        }
#pragma unroll
        for (int r = 1; r < RPS; ++r) {
            const __half2* h = reinterpret_cast<const __half2*>(&v[r]);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                m2[k] = __hmin2(m2[k], h[k]);
                M2[k] = __hmax2(M2[k], h[k]);
            }
        }
#pragma unroll
        for (int off = IPW; off < 32; off <<= 1) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t a = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<const uint32_t*>(&m2[k]), off);
                const uint32_t b = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<const uint32_t*>(&M2[k]), off);
                m2[k] = __hmin2(m2[k], *reinterpret_cast<const __half2*>(&a));
                M2[k] = __hmax2(M2[k], *reinterpret_cast<const __half2*>(&b));
            }
        }
        if (!ok) continue;
        float mn[8], s[8];
        uint32_t mw[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            mn[2 * k] = __low2float(m2[k]);
            mn[2 * k + 1] = __high2float(m2[k]);
            const float mx0 = __low2float(M2[k]), mx1 = __high2float(M2[k]);
            const __half s0 = group_scale16<BITS>(mn[2 * k], mx0), s1 = group_scale16<BITS>(mn[2 * k + 1], mx1);
            s[2 * k] = __half2float(s0);
            s[2 * k + 1] = __half2float(s1);
            mw[2 * k] = pack_half2_bits(stored_min16(mn[2 * k]), s0);
            mw[2 * k + 1] = pack_half2_bits(stored_min16(mn[2 * k + 1]), s1);
        }
        uint64_t mn2[4], s2[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            mn2[k] = f2_pack(mn[2 * k], mn[2 * k + 1]);
            s2[k] = f2_pack(s[2 * k], s[2 * k + 1]);
        }
        uint8_t* dst = codes + og * CB * inner + c0;
        if (BITS == 4) {
#pragma unroll
            for (int r = 0; r < RPS; r += 2) {
                const uint32_t wa[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
                const uint32_t wb[4] = {v[r + 1].x, v[r + 1].y, v[r + 1].z, v[r + 1].w};
                uint32_t p[8];                 // column c: q[row r] + 16 q[row r + 1] in the low byte
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint32_t a0, a1, b0, b1;
                    quant_bits_pair(wa[k], mn2[k], s2[k], a0, a1);
                    quant_bits_pair(wb[k], mn2[k], s2[k], b0, b1);
                    p[2 * k] = a0 + (b0 << 4);
                    p[2 * k + 1] = a1 + (b1 << 4);
                }
                st_stream_v2(dst + ((slice * RPS + r) / 2) * inner,
                             make_uint2(pack_low_bytes(p[0], p[1], p[2], p[3]), pack_low_bytes(p[4], p[5], p[6], p[7])));
            }
        } else {
#pragma unroll
            for (int r = 0; r < RPS; ++r) {
                const uint32_t wa[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
                uint32_t p[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) quant_bits_pair(wa[k], mn2[k], s2[k], p[2 * k], p[2 * k + 1]);
                st_stream_v2(dst + (slice * RPS + r) * inner,
                             make_uint2(pack_low_bytes(p[0], p[1], p[2], p[3]), pack_low_bytes(p[4], p[5], p[6], p[7])));
            }
        }
        if (slice == 0) {
            uint32_t* md = meta + og * inner + c0;
            st_stream_v4(md, make_uint4(mw[0], mw[1], mw[2], mw[3]));
            st_stream_v4(md + 4, make_uint4(mw[4], mw[5], mw[6], mw[7]));
        }
    }
}

// strided compress, one column per thread: x viewed as [outer][ng*GS][inner], a work
// item is (o, g, 1 column); serves widths that are not a multiple of 8 columns.
template <int BITS, int GS>
__global__ void __launch_bounds__(kThreads) compress_strided_kernel(const __half* __restrict__ x,
                                                                    uint8_t* __restrict__ codes,
                                                                    uint32_t* __restrict__ meta,
                                                                    int64_t outer, int64_t ng,
                                                                    int64_t inner) {
    const int64_t items = outer * ng * inner;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
    constexpr int CB = GS * BITS / 8;  // code rows per group
    for (int64_t it = tid; it < items; it += nthreads) {
        const int64_t c0 = it % inner;
        const int64_t og = it / inner;  // o * ng + g
        const __half* src = x + og * GS * inner + c0;
        float mn = __half2float(src[0]), mx = mn;
        for (int r = 1; r < GS; ++r) {
            const float v = __half2float(src[r * inner]);
            mn = fminf(mn, v);
            mx = fmaxf(mx, v);
        }
        const __half s16 = group_scale16<BITS>(mn, mx);
        const float s = __half2float(s16);
        uint8_t* dst = codes + og * CB * inner + c0;
        for (int r = 0; r < GS; r += (BITS == 4 ? 2 : 1)) {
            uint32_t q = quant_one<BITS>(__half2float(src[r * inner]), mn, s);
            if (BITS == 4) q |= quant_one<4>(__half2float(src[(r + 1) * inner]), mn, s) << 4;
            dst[(BITS == 4 ? r / 2 : r) * inner] = static_cast<uint8_t>(q);
        }
        meta[og * inner + c0] = pack_half2_bits(stored_min16(mn), s16);
    }
}

// Resident blocks per SM the strided decompress is compiled for, and code rows in flight
// per thread: measured per configuration. 4-bit codes at group 32 / 64 gain 2-5% from a
// fifth block per SM (a few registers spill) and lose 3% at group 128; 8-bit codes gain 4%
// from 8 rows in flight, 4-bit ones lose 2-7%. (The other counts only keep each kernel at
// the registers it takes without a bound: an explicit bound of 1 lets it take ~95.)
template <int BITS, int GS, int VEC>
constexpr int strided_dec_minb() {
    return VEC == 1 ? (BITS == 4 ? 8 : 6) : BITS == 8 ? 5 : GS < 128 ? 5 : 4;
}
template <int BITS>
constexpr int strided_dec_rows() { return BITS == 8 ? 8 : 4; }

template <int BITS, int GS, int VEC>
__global__ void __launch_bounds__(kThreads, strided_dec_minb<BITS, GS, VEC>()) decompress_strided_kernel(const uint8_t* __restrict__ codes,
                                                                      const uint32_t* __restrict__ meta,
                                                                      __half* __restrict__ y,
                                                                      int64_t outer, int64_t ng,
                                                                      int64_t inner, DivU32 dcols) {
    const int64_t cols = inner / VEC;
    const int64_t items = outer * ng * cols;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
    constexpr int CB = GS * BITS / 8;
    for (int64_t it = tid; it < items; it += nthreads) {
        // 4-bit codes: the reciprocal division (the item's work is short enough for a 64-bit
        // division to show: g32 71% -> 78% of HBM at 4 GiB); 8-bit: plain division (the
        // reciprocal form made those 8-15% slower)
        int64_t og, cv;
        if constexpr (BITS == 4) {
            divmod(it, cols, dcols, og, cv);
        } else {
            (void)dcols;
            og = it / cols;
            cv = it - og * cols;
        }
        const int64_t c0 = cv * VEC;
        float mn[VEC], step[VEC];
        const uint32_t* ms = meta + og * inner + c0;
        if (VEC == 8) {
            const uint4 a = ld_stream_v4(ms);
            const uint4 b = ld_stream_v4(ms + 4);
            const uint32_t m[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                mn[k] = h2f_lo(m[k]);
                step[k] = group_step(__ushort_as_half(static_cast<unsigned short>(m[k] >> 16)));
            }
        } else {
            mn[0] = h2f_lo(ms[0]);
            step[0] = group_step(__ushort_as_half(static_cast<unsigned short>(ms[0] >> 16)));
        }
        const uint8_t* src = codes + og * CB * inner + c0;
        __half* dst = y + og * GS * inner + c0;
        if (VEC == 8) {
            constexpr int JU = strided_dec_rows<BITS>();
#pragma unroll JU
            for (int j = 0; j < CB; ++j) {
                uint2 cw;
                asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                             : "=r"(cw.x), "=r"(cw.y)
                             : "l"(src + j * inner));
                const uint32_t w[2] = {cw.x, cw.y};
                if (BITS == 4) {
                    uint32_t r0[4], r1[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t b0 = (w[k / 2] >> (16 * (k % 2))) & 0xFFu;
                        const uint32_t b1 = (w[k / 2] >> (16 * (k % 2) + 8)) & 0xFFu;
                        r0[k] = pack_half2_bits(dequant_one(b0 & 15u, step[2 * k], mn[2 * k]),
                                                dequant_one(b1 & 15u, step[2 * k + 1], mn[2 * k + 1]));
                        r1[k] = pack_half2_bits(dequant_one(b0 >> 4, step[2 * k], mn[2 * k]),
                                                dequant_one(b1 >> 4, step[2 * k + 1], mn[2 * k + 1]));
                    }
                    st_stream_v4(dst + (2 * j) * inner, make_uint4(r0[0], r0[1], r0[2], r0[3]));
                    st_stream_v4(dst + (2 * j + 1) * inner, make_uint4(r1[0], r1[1], r1[2], r1[3]));
                } else {
                    uint32_t r0[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t b0 = (w[k / 2] >> (16 * (k % 2))) & 0xFFu;
                        const uint32_t b1 = (w[k / 2] >> (16 * (k % 2) + 8)) & 0xFFu;
                        r0[k] = pack_half2_bits(dequant_one(b0, step[2 * k], mn[2 * k]),
                                                dequant_one(b1, step[2 * k + 1], mn[2 * k + 1]));
                    }
                    st_stream_v4(dst + j * inner, make_uint4(r0[0], r0[1], r0[2], r0[3]));
                }
            }
        } else {
            for (int j = 0; j < CB; ++j) {
                const uint32_t b = src[j * inner];
                if (BITS == 4) {
                    dst[(2 * j) * inner] = dequant_one(b & 15u, step[0], mn[0]);
                    dst[(2 * j + 1) * inner] = dequant_one(b >> 4, step[0], mn[0]);
                } else {
                    dst[j * inner] = dequant_one(b, step[0], mn[0]);
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------------
// Codec variants (one thread per group): 3-bit codes, the symmetric (absmax) form and a
// group dimension that is not a multiple of the group size. Readings of what the pages
// only name - the symmetric flag and num_groups of the compression configuration (the
// walkthrough page, section 6.3), int3/int4 group-wise quantisation (the hub page):
//   - symmetric: B = 2^(b-1) - 1, scale = fp16(B / max|x|) (0 for an all-zero group,
//     65504 on overflow), signed code q = clamp(rint(x * scale), -B, B) stored as q + B,
//     metadata {0, scale}, x^ = fp16((u - B) * fp32(1/scale));
//   - 3 bits: the codes of a group form a little-endian bit stream (code j in bits
//     [3j, 3j + 3)), 8 codes in every 3 bytes;
//   - a partial last group is zero-padded: the padding takes part in min/max (or
//     max|x|) and its codes are stored; decompression writes only the real elements.
// Item (o, g, i): group g of the dimension, outer index o, inner index i.
__global__ void __launch_bounds__(kThreads) compress_generic_kernel(const __half* __restrict__ x,
                                                                     uint8_t* __restrict__ codes,
                                                                     uint32_t* __restrict__ meta, int64_t outer,
                                                                     int64_t G, int64_t ng, int64_t inner, int gs,
                                                                     int bits, int sym) {
    const int64_t items = outer * ng * inner;
    const int64_t bpg = gs * bits / 8;
    const int levels = (1 << bits) - 1, B = (1 << (bits - 1)) - 1;
    for (int64_t it = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; it < items;
         it += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = it % inner, og = it / inner, g = og % ng, o = og / ng;
        const __half* src = x + (o * G + g * gs) * inner + i;
        const int real = G - g * gs < gs ? static_cast<int>(G - g * gs) : gs;
        auto val = [&](int j) { return j < real ? __half2float(src[static_cast<int64_t>(j) * inner]) : 0.0f; };
        float s = 0.0f, mn = 0.0f;
        __half s16 = __ushort_as_half(0);
        if (sym) {
            float a = 0.0f;
            for (int j = 0; j < gs; ++j) a = fmaxf(a, fabsf(val(j)));
            if (a > 0.0f) {
                s16 = __float2half_rn(__fdiv_rn(static_cast<float>(B), a));
                if (__hisinf(s16)) s16 = __ushort_as_half(0x7BFF);
            }
        } else {
            float mx = val(0);
            mn = mx;
            for (int j = 1; j < gs; ++j) {
                const float v = val(j);
                mn = fminf(mn, v);
                mx = fmaxf(mx, v);
            }
            const float r = __fsub_rn(mx, mn);
            if (r > 0.0f) {
                s16 = __float2half_rn(__fdiv_rn(static_cast<float>(levels), r));
                if (__hisinf(s16)) s16 = __ushort_as_half(0x7BFF);
            }
        }
        s = __half2float(s16);
        uint8_t* dst = codes + (o * ng * bpg + g * bpg) * inner + i;
        uint32_t acc = 0;          // pending bits of the 3-bit stream, or the low nibble
        int nacc = 0;
        int64_t byte = 0;
        for (int j = 0; j < gs; ++j) {
            int q;
            if (sym) {
                q = __float2int_rn(__fmul_rn(val(j), s));
                q = min(max(q, -B), B) + B;
            } else {
                q = __float2int_rn(__fmul_rn(__fsub_rn(val(j), mn), s));
                q = min(max(q, 0), levels);
            }
            if (bits == 8) {
                dst[(byte++) * inner] = static_cast<uint8_t>(q);
            } else {
                acc |= static_cast<uint32_t>(q) << nacc;
                nacc += bits;
                while (nacc >= 8) {
                    dst[(byte++) * inner] = static_cast<uint8_t>(acc & 0xFFu);
                    acc >>= 8;
                    nacc -= 8;
                }
            }
        }
        meta[(o * ng + g) * inner + i] = pack_half2_bits(sym ? __ushort_as_half(0) : stored_min16(mn), s16);
    }
}

__global__ void __launch_bounds__(kThreads) decompress_generic_kernel(const uint8_t* __restrict__ codes,
                                                                       const uint32_t* __restrict__ meta,
                                                                       __half* __restrict__ y, int64_t outer,
                                                                       int64_t G, int64_t ng, int64_t inner, int gs,
                                                                       int bits, int sym) {
    const int64_t items = outer * ng * inner;
    const int64_t bpg = gs * bits / 8;
    const int B = (1 << (bits - 1)) - 1;
    const uint32_t mask = (1u << bits) - 1u;
    for (int64_t it = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; it < items;
         it += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = it % inner, og = it / inner, g = og % ng, o = og / ng;
        const uint32_t mw = meta[(o * ng + g) * inner + i];
        const __half mn16 = __ushort_as_half(static_cast<unsigned short>(mw & 0xFFFFu));
        const float s = h2f_hi(mw), mn = __half2float(mn16);
        const float step = s > 0.0f ? __fdiv_rn(1.0f, s) : 0.0f;
        const uint8_t* src = codes + (o * ng * bpg + g * bpg) * inner + i;
        __half* dst = y + (o * G + g * gs) * inner + i;
        const int real = G - g * gs < gs ? static_cast<int>(G - g * gs) : gs;
        uint32_t acc = 0;
        int nacc = 0;
        int64_t byte = 0;
        for (int j = 0; j < real; ++j) {
            while (nacc < bits) {
                acc |= static_cast<uint32_t>(src[(byte++) * inner]) << nacc;
                nacc += 8;
            }
            const int q = static_cast<int>(acc & mask);
            acc >>= bits;
            nacc -= bits;
            __half v;
            if (sym)
                v = __float2half_rn(__fmul_rn(static_cast<float>(q - B), step));
            else
                v = s > 0.0f ? __float2half_rn(__fadd_rn(__fmul_rn(static_cast<float>(q), step), mn)) : mn16;
            dst[static_cast<int64_t>(j) * inner] = v;
        }
    }
}

// ---------------------------------------------------------------------------------
// Codec variants on contiguous groups (group_dim the last one, its extent G a multiple of
// 8): the layout of the main contiguous kernels - 8 values per 16-byte load, the lanes of
// a group reducing min/max (or max|x|) with shuffles; compress with 3- and 4-bit codes
// gives a lane two vectors of its group - with the variants' arithmetic, bit for bit
// that of the one-thread-per-group kernels above. A vector whose 8 values lie past G (the
// padding of a partial last group; G % 8 == 0, so a vector is wholly in or out) is taken
// as zeros, which count in min/max and max|x|, and its codes are stored like any other.
// 3-bit codes: the 8 codes of vector l of a group are bits [24 l, 24 l + 24) of the
// group's little-endian stream, i.e. 3 whole bytes at byte 3 l.
template <int BITS, int SYM>
__device__ __forceinline__ uint32_t var_quant8(uint4 v, float mn, float s) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t q[8];
    if (SYM) {
        // q = rint(fl(x * s)) in [-B, B] (|x * s| <= B (1 + 2^-10) < B + 0.5 by the
        // choice of s), stored as q + B; a NaN product gives q = 0 like the conversion
        constexpr int B = (1 << (BITS - 1)) - 1;
        const uint64_t s2 = f2_pack(s, s);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float a, b;
            f2_unpack(f2_mul(f2_pack(h2f_lo(w[k]), h2f_hi(w[k])), s2), a, b);
            a = (a == a) ? a : 0.0f;
            b = (b == b) ? b : 0.0f;
            f2_unpack(f2_add(f2_pack(a, b), f2_pack(12582912.0f, 12582912.0f)), a, b);
            q[2 * k] = (__float_as_uint(a) + B) & ((1u << BITS) - 1u);
            q[2 * k + 1] = (__float_as_uint(b) + B) & ((1u << BITS) - 1u);
        }
    } else {
        const uint64_t mn2 = f2_pack(mn, mn), s2 = f2_pack(s, s);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            quant_bits_pair(w[k], mn2, s2, q[2 * k], q[2 * k + 1]);
            q[2 * k] &= (1u << BITS) - 1u;
            q[2 * k + 1] &= (1u << BITS) - 1u;
        }
    }
    uint32_t u = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) u |= q[k] << (BITS * k);     // BITS <= 4: fits 32 bits
    return u;
}

// Group q of the [rows][ng] grid of groups, with its row o = q / ng and its index gi = q %
// ng in the row. A thread's groups form an arithmetic sequence (its grid stride is a
// multiple of the lanes per group), so the walk advances (o, gi) by (D / ng, D % ng), taken
// once per thread, and one conditional subtraction, instead of dividing for every group.
// When every group is whole (ng GS == G, the WHOLE instantiation) the address is flat and
// only q is kept: the row state would cost registers and resident blocks (3-11% measured).
// (gi + dr < 2 ng and the stride fit 31 bits: the stride is at most the threads of a
// resident grid, and the launcher routes ng >= 2^30 to the generic kernels.)
template <int GS, bool WHOLE>
struct GroupWalk {
    int64_t q, o;
    int32_t gi, dq, dr, D;
    __device__ __forceinline__ GroupWalk(int64_t q0, int64_t stride, int64_t ng) : q(q0), D(static_cast<int32_t>(stride)) {
        if constexpr (!WHOLE) {
            o = q0 / ng;
            gi = static_cast<int32_t>(q0 - o * ng);
            dq = static_cast<int32_t>(stride / ng);
            dr = static_cast<int32_t>(stride - static_cast<int64_t>(dq) * ng);
        }
    }
    __device__ __forceinline__ void step(int64_t ng) {
        q += D;
        if constexpr (!WHOLE) {
            o += dq;
            gi += dr;
            if (gi >= static_cast<int32_t>(ng)) {
                gi -= static_cast<int32_t>(ng);
                ++o;
            }
        }
    }
    // Element offset of the 8 values at position `sub` (in units of 8) of the walk's group,
    // passed again as gq (a caller that knows it saves the walk's copy), and whether they
    // lie inside the row (a partial last group leaves padding).
    __device__ __forceinline__ int64_t at(int64_t gq, int sub, int64_t G, bool& ok) const {
        if constexpr (WHOLE) {
            ok = true;
            return gq * GS + sub * 8;
        } else {
            const int64_t col = static_cast<int64_t>(gi) * GS + sub * 8;
            ok = col < G;
            return o * G + col;
        }
    }
};

// Like the main 4-bit kernel, a lane holds two vectors of its group (vectors sub and
// sub + L), so the group's reduction and scale division are done once per 16 values.
template <int BITS, int GS, int SYM, bool WHOLE>
__global__ void __launch_bounds__(kThreads) compress_var_contig_kernel(const __half* __restrict__ x,
                                                                        uint8_t* __restrict__ codes,
                                                                        uint32_t* __restrict__ meta, int64_t rows,
                                                                        int64_t G, int64_t ng) {
    constexpr int L = GS / 16;                 // lanes per group
    constexpr int GPW = 32 / L;                // groups per warp and step
    constexpr int CB = GS * BITS / 8;          // code bytes per group
    const int lane = threadIdx.x & 31, sub = lane % L;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    const int64_t total = rows * ng;
    GroupWalk<GS, WHOLE> walk(warp * GPW + lane / L, nwarps * GPW, ng);   // the group of the next load
    auto load = [&](uint4 (&v)[2], int64_t base) {
        const int64_t q = base + lane / L;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            bool ok = false;
            const int64_t at = q < total ? walk.at(q, sub + j * L, G, ok) : 0;
            v[j] = (q < total && ok) ? ld_stream_v4(x + at) : make_uint4(0u, 0u, 0u, 0u);
        }
        walk.step(ng);
    };
    // software pipelined: the next step's vectors are requested before these are quantised
    int64_t base = warp * GPW;
    uint4 v[2];
    load(v, base);
    while (base < total) {
        const int64_t next = base + nwarps * GPW;
        uint4 nv[2];
        load(nv, next);
        const int64_t q = base + lane / L;
        float mn = 0.0f;
        __half s16 = __ushort_as_half(0);
        if (SYM) {
            const __half2* h = reinterpret_cast<const __half2*>(&v[0]);
            const __half2* k = reinterpret_cast<const __half2*>(&v[1]);
            __half2 a2 = __hmax2(__hmax2(__hmax2(__habs2(h[0]), __habs2(h[1])), __hmax2(__habs2(h[2]), __habs2(h[3]))),
                                 __hmax2(__hmax2(__habs2(k[0]), __habs2(k[1])), __hmax2(__habs2(k[2]), __habs2(k[3]))));
#pragma unroll
            for (int off = 1; off < L; off <<= 1) {
                const uint32_t o2 = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<const uint32_t*>(&a2), off);
                a2 = __hmax2(a2, *reinterpret_cast<const __half2*>(&o2));
            }
            const float a = fmaxf(__low2float(a2), __high2float(a2));
            if (a > 0.0f) {
                s16 = __float2half_rn(__fdiv_rn(static_cast<float>((1 << (BITS - 1)) - 1), a));
                if (__hisinf(s16)) s16 = __ushort_as_half(0x7BFF);
            }
        } else {
            __half2 hmn, hmx, mn1, mx1;
            minmax8(v[0], hmn, hmx);
            minmax8(v[1], mn1, mx1);
            float mx;
            group_minmax<L>(__hmin2(hmn, mn1), __hmax2(hmx, mx1), mn, mx);
            s16 = group_scale16<BITS>(mn, mx);
        }
        if (q < total) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint32_t u = var_quant8<BITS, SYM>(v[j], mn, __half2float(s16));
                uint8_t* dst = codes + q * CB + (sub + j * L) * BITS;
                if (BITS == 4) {
                    *reinterpret_cast<uint32_t*>(dst) = u;
                } else {                           // 3 bytes, little-endian
                    dst[0] = static_cast<uint8_t>(u);
                    dst[1] = static_cast<uint8_t>(u >> 8);
                    dst[2] = static_cast<uint8_t>(u >> 16);
                }
            }
            if (sub == 0) meta[q] = pack_half2_bits(SYM ? __ushort_as_half(0) : stored_min16(mn), s16);
        }
        v[0] = nv[0];
        v[1] = nv[1];
        base = next;
    }
}

// 8-bit codes of the contiguous variants (8 code bytes per lane): the symmetric form, or
// the min/max form of a partial last group.
template <int GS, int SYM, bool WHOLE>
__global__ void __launch_bounds__(kThreads) compress_var8_contig_kernel(const __half* __restrict__ x,
                                                                         uint8_t* __restrict__ codes,
                                                                         uint32_t* __restrict__ meta, int64_t rows,
                                                                         int64_t G, int64_t ng) {
    constexpr int L = GS / 8, GPW = 32 / L, B = 127;
    const int lane = threadIdx.x & 31, sub = lane % L;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    const int64_t total = rows * ng;
    GroupWalk<GS, WHOLE> walk(warp * GPW + lane / L, nwarps * GPW, ng);   // the group of the next load
    auto load = [&](int64_t base) {
        const int64_t q = base + lane / L;
        bool okv = false;
        const int64_t at = q < total ? walk.at(q, sub, G, okv) : 0;
        walk.step(ng);
        return (q < total && okv) ? ld_stream_v4(x + at) : make_uint4(0u, 0u, 0u, 0u);
    };
    // software pipelined: the next step's vector is requested before this one is quantised
    int64_t base = warp * GPW;
    uint4 v = load(base);
    while (base < total) {
        const int64_t next = base + nwarps * GPW;
        const uint4 nv = load(next);
        const int64_t q = base + lane / L;
        const bool okg = q < total;
        float mn = 0.0f;
        __half s16 = __ushort_as_half(0);
        if (SYM) {
            const __half2* h = reinterpret_cast<const __half2*>(&v);
            __half2 a2 = __hmax2(__hmax2(__habs2(h[0]), __habs2(h[1])), __hmax2(__habs2(h[2]), __habs2(h[3])));
#pragma unroll
            for (int off = 1; off < L; off <<= 1) {
                const uint32_t o2 = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<const uint32_t*>(&a2), off);
                a2 = __hmax2(a2, *reinterpret_cast<const __half2*>(&o2));
            }
            const float a = fmaxf(__low2float(a2), __high2float(a2));
            if (a > 0.0f) {
                s16 = __float2half_rn(__fdiv_rn(static_cast<float>(B), a));
                if (__hisinf(s16)) s16 = __ushort_as_half(0x7BFF);
            }
        } else {
            __half2 hmn, hmx;
            minmax8(v, hmn, hmx);
            float mx;
            group_minmax<L>(hmn, hmx, mn, mx);
            s16 = group_scale16<8>(mn, mx);
        }
        if (okg) {
            const float s = __half2float(s16);
            uint2 out;
            if (SYM) {
                const uint64_t s2 = f2_pack(s, s);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                uint32_t b8[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float p0, p1;
                    f2_unpack(f2_mul(f2_pack(h2f_lo(w[k]), h2f_hi(w[k])), s2), p0, p1);
                    p0 = (p0 == p0) ? p0 : 0.0f;
                    p1 = (p1 == p1) ? p1 : 0.0f;
                    f2_unpack(f2_add(f2_pack(p0, p1), f2_pack(12582912.0f, 12582912.0f)), p0, p1);
                    b8[2 * k] = (__float_as_uint(p0) + B) & 0xFFu;
                    b8[2 * k + 1] = (__float_as_uint(p1) + B) & 0xFFu;
                }
                out = make_uint2(pack_low_bytes(b8[0], b8[1], b8[2], b8[3]), pack_low_bytes(b8[4], b8[5], b8[6], b8[7]));
            } else {
                out = quant8_8bit(v, mn, s);
            }
            *reinterpret_cast<uint2*>(codes + q * GS + sub * 8) = out;
            if (sub == 0) meta[q] = pack_half2_bits(SYM ? __ushort_as_half(0) : stored_min16(mn), s16);
        }
        v = nv;
        base = next;
    }
}

// Decompression of the contiguous variants: one item = vectors sub and sub + L of one
// group (L = GS / 16 lanes per group; BITS bytes of codes in and one 16-byte store out per
// vector), so the group's step (an fp32 division) and the index arithmetic are done once
// per 16 values, as in compression: the kernel is bound by instruction issue. A vector
// past G (padding) writes nothing. Two items per thread and step, their codes and
// metadata requested before any is converted.
template <int BITS, int GS, int SYM, bool WHOLE>
__global__ void __launch_bounds__(kThreads) decompress_var_contig_kernel(const uint8_t* __restrict__ codes,
                                                                          const uint32_t* __restrict__ meta,
                                                                          __half* __restrict__ y, int64_t rows,
                                                                          int64_t G, int64_t ng) {
    constexpr int L = GS / 16;
    constexpr int CB = GS * BITS / 8;
    constexpr int B = (1 << (BITS - 1)) - 1;
    constexpr int U = 2;
    const int64_t items = rows * ng * L;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
    // item it = tid + m nthreads (m = 0, 1, ...): group tid / L + m (nthreads / L), position
    // tid % L in it (nthreads is a multiple of L, a power of two)
    const int sub = static_cast<int>(tid & (L - 1));
    GroupWalk<GS, WHOLE> walk(tid / L, nthreads / L, ng);
    for (int64_t base = tid; base < items; base += nthreads * U) {
        uint2 c[U][2];
        uint32_t mw[U];
        int64_t at[U][2];
        bool ok[U][2];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t it = base + u * nthreads;
            const int64_t q = WHOLE ? it / L : walk.q;      // L is a power of two
            const bool in = it < items;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                ok[u][j] = false;
                at[u][j] = in ? walk.at(q, sub + j * L, G, ok[u][j]) : 0;
                ok[u][j] = ok[u][j] && in;
                c[u][j] = make_uint2(0u, 0u);
                if (ok[u][j]) {
                    const uint8_t* src = codes + q * CB + (sub + j * L) * BITS;
                    if (BITS == 8) {
                        c[u][j] = __ldg(reinterpret_cast<const uint2*>(src));
                    } else if (BITS == 4) {
                        c[u][j].x = __ldg(reinterpret_cast<const uint32_t*>(src));
                    } else {
                        c[u][j].x = static_cast<uint32_t>(__ldg(src)) | (static_cast<uint32_t>(__ldg(src + 1)) << 8) |
                                    (static_cast<uint32_t>(__ldg(src + 2)) << 16);
                    }
                }
            }
            // vector sub + L lies further along the row than vector sub: if sub is padding,
            // so is sub + L
            mw[u] = ok[u][0] ? __ldg(meta + q) : 0u;
            walk.step(ng);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (!ok[u][0]) continue;
            const uint32_t m = mw[u];
            const float step = group_step(__ushort_as_half(static_cast<unsigned short>(m >> 16)));
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                if (!ok[u][j]) continue;
                const uint32_t cw[2] = {c[u][j].x, c[u][j].y};
                uint32_t out[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint32_t q0, q1;
                    if (BITS == 8) {
                        q0 = (cw[k / 2] >> (16 * (k % 2))) & 0xFFu;
                        q1 = (cw[k / 2] >> (16 * (k % 2) + 8)) & 0xFFu;
                    } else {
                        q0 = (cw[0] >> (BITS * 2 * k)) & ((1u << BITS) - 1u);
                        q1 = (cw[0] >> (BITS * (2 * k + 1))) & ((1u << BITS) - 1u);
                    }
                    if (SYM) {
                        // x^ = fp16(fl((u - B) * step)); an all-zero group (step 0) gives 0
                        const __half2 hv =
                            __floats2half2_rn(__fmul_rn(static_cast<float>(static_cast<int>(q0) - B), step),
                                              __fmul_rn(static_cast<float>(static_cast<int>(q1) - B), step));
                        out[k] = *reinterpret_cast<const uint32_t*>(&hv);
                    } else if (step == 0.0f) {
                        out[k] = (m & 0xFFFFu) * 0x10001u;
                    } else {
                        out[k] = dequant_two(q0, q1, step, h2f_lo(m));
                    }
                }
                st_stream_v4(y + at[u][j], make_uint4(out[0], out[1], out[2], out[3]));
            }
        }
    }
}

// ---------------------------------------------------------------------------------
struct Geometry {
    int64_t outer = 1, ng = 0, inner = 1, n = 0, G = 0;
    int gd = 0;
    bool generic = false;      // a variant configuration (compress_/decompress_generic_kernel)
};

int validate(int32_t ndim, const int64_t* shape, const flexq_config& cfg, Geometry& geo) {
    FLEX_REQUIRE(shape != nullptr, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(ndim >= 1 && ndim <= 4, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(cfg.symmetric == 0 || cfg.symmetric == 1, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(cfg.num_bits == 3 || cfg.num_bits == 4 || cfg.num_bits == 8, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(cfg.group_size == 32 || cfg.group_size == 64 || cfg.group_size == 128,
                 FLEX_ERR_UNSUPPORTED);
    int gd = cfg.group_dim;
    if (gd < 0) gd += ndim;
    FLEX_REQUIRE(gd >= 0 && gd < ndim, FLEX_ERR_INVALID_ARG);
    int64_t n = 1;
    for (int i = 0; i < ndim; ++i) {
        FLEX_REQUIRE(shape[i] >= 0, FLEX_ERR_INVALID_ARG);
        n *= shape[i];
    }
    geo.gd = gd;
    geo.n = n;
    geo.G = shape[gd];
    geo.outer = 1;
    for (int i = 0; i < gd; ++i) geo.outer *= shape[i];
    geo.inner = 1;
    for (int i = gd + 1; i < ndim; ++i) geo.inner *= shape[i];
    geo.ng = (shape[gd] + cfg.group_size - 1) / cfg.group_size;      // a partial last group is padded
    geo.generic = cfg.num_bits == 3 || cfg.symmetric != 0 || shape[gd] % cfg.group_size != 0;
    return FLEX_OK;
}


// Grid of a grid-stride kernel: enough blocks for `work_threads`, capped at what the
// device holds resident at once (blocks per SM from the kernel's registers, times the SM
// count), so that no block waits for a second wave while the others stream.
template <auto Kernel>
unsigned grid_for(int64_t work_threads) {
    static int per_sm = 0;   // one cached value per kernel (all devices are one type)
    if (per_sm == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, Kernel, kThreads, 0) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = 1;
        }
        per_sm = n;
    }
    const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm;
    int64_t blocks = (work_threads + kThreads - 1) / kThreads;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return static_cast<unsigned>(blocks);
}

int launch_generic(const Geometry& g, const flexq_config& cfg, const __half* x, uint8_t* codes, uint32_t* meta,
                   const uint8_t* ccodes, const uint32_t* cmeta, __half* y, cudaStream_t st) {
    const int64_t items = g.outer * g.ng * g.inner;
    if (x != nullptr) {
        const unsigned grid = grid_for<compress_generic_kernel>(items);
        compress_generic_kernel<<<grid, kThreads, 0, st>>>(x, codes, meta, g.outer, g.G, g.ng, g.inner,
                                                           cfg.group_size, cfg.num_bits, cfg.symmetric);
    } else {
        const unsigned grid = grid_for<decompress_generic_kernel>(items);
        decompress_generic_kernel<<<grid, kThreads, 0, st>>>(ccodes, cmeta, y, g.outer, g.G, g.ng, g.inner,
                                                             cfg.group_size, cfg.num_bits, cfg.symmetric);
    }
    return launch_status();
}

template <int BITS, int GS>
int launch_compress(const Geometry& g, const __half* x, uint8_t* codes, uint32_t* meta,
                    cudaStream_t st) {
    if (g.inner == 1) {
        const int64_t G = g.outer * g.ng;
        constexpr int U = kUnroll * 2 / contig_vpl<BITS>();     // groups per lane and step
        const int64_t lanes = G * (GS / (8 * contig_vpl<BITS>()));
        const unsigned grid = grid_for<compress_contig_kernel<BITS, GS>>((lanes + U - 1) / U);
        compress_contig_kernel<BITS, GS><<<grid, kThreads, 0, st>>>(x, codes, meta, G);
    } else {
        const bool vec = (g.inner % 8 == 0);
        const int64_t items = g.outer * g.ng * (vec ? g.inner / 8 : g.inner);
        if (vec)   // GS / strided_rps<BITS>(GS) lanes per item
            compress_strided_1pass_kernel<BITS, GS>
                <<<grid_for<compress_strided_1pass_kernel<BITS, GS>>(items * (GS / strided_rps<BITS>(GS))), kThreads, 0, st>>>(
                    x, codes, meta, g.outer, g.ng, g.inner);
        else
            compress_strided_kernel<BITS, GS>
                <<<grid_for<compress_strided_kernel<BITS, GS>>(items), kThreads, 0, st>>>(x, codes, meta, g.outer, g.ng, g.inner);
    }
    return launch_status();
}

template <int BITS, int GS>
int launch_decompress(const Geometry& g, const uint8_t* codes, const uint32_t* meta, __half* y,
                      cudaStream_t st) {
    if (g.inner == 1) {
        const int64_t items = g.n / 8;       // n is a multiple of the group size (>= 32)
        const unsigned grid = grid_for<decompress_contig_kernel<BITS, GS>>((items + kDecUnroll - 1) / kDecUnroll);
        decompress_contig_kernel<BITS, GS><<<grid, kThreads, 0, st>>>(codes, meta, y, items);
    } else {
        const bool vec = (g.inner % 8 == 0);
        const int64_t items = g.outer * g.ng * (vec ? g.inner / 8 : g.inner);
        if (vec)
            decompress_strided_kernel<BITS, GS, 8>
                <<<grid_for<decompress_strided_kernel<BITS, GS, 8>>(items), kThreads, 0, st>>>(codes, meta, y, g.outer, g.ng,
                                                                                                g.inner, make_div(g.inner / 8));
        else
            decompress_strided_kernel<BITS, GS, 1>
                <<<grid_for<decompress_strided_kernel<BITS, GS, 1>>(items), kThreads, 0, st>>>(codes, meta, y, g.outer, g.ng,
                                                                                                g.inner, make_div(g.inner));
    }
    return launch_status();
}

// The contiguous-group variants (3-bit, symmetric, partial last group with G % 8 == 0).
template <int BITS, int GS, int SYM, bool WHOLE>
int launch_var_w(const Geometry& g, const __half* x, uint8_t* codes, uint32_t* meta, const uint8_t* ccodes,
                 const uint32_t* cmeta, __half* y, cudaStream_t st) {
    const int64_t lanes = g.outer * g.ng * (GS / 8);
    if (x != nullptr) {
        if constexpr (BITS == 8) {
            compress_var8_contig_kernel<GS, SYM, WHOLE>
                <<<grid_for<compress_var8_contig_kernel<GS, SYM, WHOLE>>(lanes), kThreads, 0, st>>>(x, codes, meta, g.outer,
                                                                                                     g.G, g.ng);
        } else {                               // two vectors per lane
            compress_var_contig_kernel<BITS, GS, SYM, WHOLE>
                <<<grid_for<compress_var_contig_kernel<BITS, GS, SYM, WHOLE>>(lanes / 2), kThreads, 0, st>>>(
                    x, codes, meta, g.outer, g.G, g.ng);
        }
    } else {
        decompress_var_contig_kernel<BITS, GS, SYM, WHOLE>      // two vectors per lane
            <<<grid_for<decompress_var_contig_kernel<BITS, GS, SYM, WHOLE>>(lanes / 2), kThreads, 0, st>>>(ccodes, cmeta, y,
                                                                                                        g.outer, g.G, g.ng);
    }
    return launch_status();
}

template <int BITS, int GS, int SYM>
int launch_var(const Geometry& g, const __half* x, uint8_t* codes, uint32_t* meta, const uint8_t* ccodes,
               const uint32_t* cmeta, __half* y, cudaStream_t st) {
    if (g.ng * GS == g.G) return launch_var_w<BITS, GS, SYM, true>(g, x, codes, meta, ccodes, cmeta, y, st);
    return launch_var_w<BITS, GS, SYM, false>(g, x, codes, meta, ccodes, cmeta, y, st);
}

template <int BITS, int SYM>
int launch_var_gs(const Geometry& g, int gs, const __half* x, uint8_t* codes, uint32_t* meta, const uint8_t* ccodes,
                  const uint32_t* cmeta, __half* y, cudaStream_t st) {
    if (gs == 32) return launch_var<BITS, 32, SYM>(g, x, codes, meta, ccodes, cmeta, y, st);
    if (gs == 64) return launch_var<BITS, 64, SYM>(g, x, codes, meta, ccodes, cmeta, y, st);
    return launch_var<BITS, 128, SYM>(g, x, codes, meta, ccodes, cmeta, y, st);
}

// A variant configuration: the contiguous-group kernels when the group dimension is the
// last one and its extent a multiple of 8, else the one-thread-per-group kernels.
int launch_variant(const Geometry& g, const flexq_config& cfg, const __half* x, uint8_t* codes, uint32_t* meta,
                   const uint8_t* ccodes, const uint32_t* cmeta, __half* y, cudaStream_t st) {
    if (g.inner != 1 || g.G % 8 != 0 || g.ng >= (int64_t{1} << 30))
        return launch_generic(g, cfg, x, codes, meta, ccodes, cmeta, y, st);
    const int gs = cfg.group_size;
    if (cfg.symmetric) {
        if (cfg.num_bits == 3) return launch_var_gs<3, 1>(g, gs, x, codes, meta, ccodes, cmeta, y, st);
        if (cfg.num_bits == 4) return launch_var_gs<4, 1>(g, gs, x, codes, meta, ccodes, cmeta, y, st);
        return launch_var_gs<8, 1>(g, gs, x, codes, meta, ccodes, cmeta, y, st);
    }
    if (cfg.num_bits == 3) return launch_var_gs<3, 0>(g, gs, x, codes, meta, ccodes, cmeta, y, st);
    if (cfg.num_bits == 4) return launch_var_gs<4, 0>(g, gs, x, codes, meta, ccodes, cmeta, y, st);
    return launch_var_gs<8, 0>(g, gs, x, codes, meta, ccodes, cmeta, y, st);
}

}  // namespace
}  // namespace flexq

using namespace flexq;

extern "C" int64_t flexq_codes_bytes(int32_t ndim, const int64_t* shape, flexq_config cfg) {
    Geometry g;
    const int rc = validate(ndim, shape, cfg, g);
    if (rc != FLEX_OK) return rc;
    return g.outer * g.ng * cfg.group_size * cfg.num_bits / 8 * g.inner;
}

extern "C" int64_t flexq_meta_bytes(int32_t ndim, const int64_t* shape, flexq_config cfg) {
    Geometry g;
    const int rc = validate(ndim, shape, cfg, g);
    if (rc != FLEX_OK) return rc;
    return g.outer * g.ng * g.inner * 4;
}

extern "C" int flexq_compress(const void* x, int32_t ndim, const int64_t* shape, flexq_config cfg,
                              void* codes, void* meta, void* stream) {
    Geometry g;
    const int rc = validate(ndim, shape, cfg, g);
    if (rc != FLEX_OK) return rc;
    if (g.n == 0) return FLEX_OK;
    FLEX_REQUIRE(x && codes && meta, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(aligned16(x) && aligned16(codes) && aligned16(meta), FLEX_ERR_ALIGN);
    const cudaStream_t st = as_stream(stream);
    const __half* xh = static_cast<const __half*>(x);
    uint8_t* c = static_cast<uint8_t*>(codes);
    uint32_t* m = static_cast<uint32_t*>(meta);
    if (g.generic) return launch_variant(g, cfg, xh, c, m, nullptr, nullptr, nullptr, st);
#define CALL_C(B, S) launch_compress<B, S>(g, xh, c, m, st)
    if (cfg.num_bits == 4) {
        if (cfg.group_size == 32) return CALL_C(4, 32);
        if (cfg.group_size == 64) return CALL_C(4, 64);
        return CALL_C(4, 128);
    }
    if (cfg.group_size == 32) return CALL_C(8, 32);
    if (cfg.group_size == 64) return CALL_C(8, 64);
    return CALL_C(8, 128);
#undef CALL_C
}

extern "C" int flexq_decompress(const void* codes, const void* meta, int32_t ndim, const int64_t* shape,
                                flexq_config cfg, void* y, void* stream) {
    Geometry g;
    const int rc = validate(ndim, shape, cfg, g);
    if (rc != FLEX_OK) return rc;
    if (g.n == 0) return FLEX_OK;
    FLEX_REQUIRE(y && codes && meta, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(aligned16(y) && aligned16(codes) && aligned16(meta), FLEX_ERR_ALIGN);
    const cudaStream_t st = as_stream(stream);
    const uint8_t* c = static_cast<const uint8_t*>(codes);
    const uint32_t* m = static_cast<const uint32_t*>(meta);
    __half* yh = static_cast<__half*>(y);
    if (g.generic) return launch_variant(g, cfg, nullptr, nullptr, nullptr, c, m, yh, st);
#define CALL_D(B, S) launch_decompress<B, S>(g, c, m, yh, st)
    if (cfg.num_bits == 4) {
        if (cfg.group_size == 32) return CALL_D(4, 32);
        if (cfg.group_size == 64) return CALL_D(4, 64);
        return CALL_D(4, 128);
    }
    if (cfg.group_size == 32) return CALL_D(8, 32);
    if (cfg.group_size == 64) return CALL_D(8, 64);
    return CALL_D(8, 128);
#undef CALL_D
}
