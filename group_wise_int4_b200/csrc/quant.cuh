// Group-wise min/max quantiser arithmetic, shared by every kernel that writes codes
// (compression, store_cache, the fused QKV epilogue) so that all of them produce the
// same bits.
//
// the walkthrough page «FlexGen 单 GPU 高吞吐大模型推理引擎：论文解读与源码实战指南», section 6.3: per group of group_size values along
// group_dim keep {min, scale} with an fp16 scale and store unsigned num_bits codes;
// q = round((x - min) * (2^b - 1) / (max - min)).  Every fp32 operation below is an
// explicitly rounded intrinsic, so the compiler cannot contract or reorder it.
#pragma once

#include "common.cuh"

namespace flexq {

// Scale of a group from its exact min/max: fp16((2^b-1)/(max-min)), 0 for a constant
// group, 65504 (largest finite fp16) when the quotient overflows fp16.
template <int BITS>
__device__ __forceinline__ __half group_scale16(float mn, float mx) {
    const float r = __fsub_rn(mx, mn);
    if (!(r > 0.0f)) return __ushort_as_half(0);
    const float s32 = __fdiv_rn(static_cast<float>((1 << BITS) - 1), r);
    __half s16 = __float2half_rn(s32);
    if (__hisinf(s16)) s16 = __ushort_as_half(0x7BFF);
    return s16;
}

template <int BITS>
__device__ __forceinline__ uint32_t quant_one(float x, float mn, float s) {
    int q = __float2int_rn(__fmul_rn(__fsub_rn(x, mn), s));
    q = q < 0 ? 0 : q;
    q = q > ((1 << BITS) - 1) ? ((1 << BITS) - 1) : q;
    return static_cast<uint32_t>(q);
}

// Eight consecutive fp16 values (one 16-byte vector) -> 4-bit codes packed in a u32
// (byte k = q[2k] | q[2k+1] << 4).
__device__ __forceinline__ uint32_t quant8_4bit(uint4 v, float mn, float s) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t lo = quant_one<4>(h2f_lo(w[k]), mn, s);
        const uint32_t hi = quant_one<4>(h2f_hi(w[k]), mn, s);
        out |= (lo | (hi << 4)) << (8 * k);
    }
    return out;
}

// Eight consecutive fp16 values -> eight 8-bit codes.
__device__ __forceinline__ uint2 quant8_8bit(uint4 v, float mn, float s) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t b[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        b[k] = quant_one<8>(h2f_lo(w[k]), mn, s) | (quant_one<8>(h2f_hi(w[k]), mn, s) << 8);
    }
    return make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
}

// min and max (as half2 lanes) of a 16-byte vector of 8 fp16 values.
__device__ __forceinline__ void minmax8(uint4 v, __half2& mn, __half2& mx) {
    const __half2 a = *reinterpret_cast<const __half2*>(&v.x);
    const __half2 b = *reinterpret_cast<const __half2*>(&v.y);
    const __half2 c = *reinterpret_cast<const __half2*>(&v.z);
    const __half2 d = *reinterpret_cast<const __half2*>(&v.w);
    mn = __hmin2(__hmin2(a, b), __hmin2(c, d));
    mx = __hmax2(__hmax2(a, b), __hmax2(c, d));
}

// Reduce a half2 min/max pair to scalars (exact: min/max select, no rounding).
__device__ __forceinline__ float hmin_of(__half2 m) { return fminf(__low2float(m), __high2float(m)); }
__device__ __forceinline__ float hmax_of(__half2 m) { return fmaxf(__low2float(m), __high2float(m)); }

// Dequantisation step of a group: fp32(1/scale16); 0 marks a constant group.
__device__ __forceinline__ float group_step(__half s16) {
    const float s = __half2float(s16);
    return s > 0.0f ? __fdiv_rn(1.0f, s) : 0.0f;
}

// x^ = fp16(fp32(fp32(q * step) + min)); a constant group (step 0) returns min.
__device__ __forceinline__ __half dequant_one(uint32_t q, float step, float mn) {
    if (step == 0.0f) return __float2half_rn(mn);
    return __float2half_rn(__fadd_rn(__fmul_rn(static_cast<float>(q), step), mn));
}

}  // namespace flexq
