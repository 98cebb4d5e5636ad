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

// The stored fp16 minimum of a group: a zero minimum is stored as +0. A group holding
// both +0 and -0 has no defined sign for its smallest value; +0 is the one kept, so
// every kernel writes the same bits (dequantised values do not depend on it).
__device__ __forceinline__ __half stored_min16(float mn) { return __float2half_rn(__fadd_rn(mn, 0.0f)); }

// ---- packed fp32 pairs ---------------------------------------------------------------
// sm_100 executes add / mul on two fp32 lanes held in one 64-bit register, each lane
// rounded like the scalar instruction; the quantiser's per-value arithmetic runs on pairs
// of values this way.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// q = clamp(rint(fl(fl(x - min) * scale)), 0, 2^b - 1) (round half to even), returned
// as the bit pattern of the fp32 value 1.5 * 2^23 + q. Adding 1.5 * 2^23 (where the fp32
// spacing is 1) rounds exactly like a float-to-int conversion, on the FP32 pipe rather
// than the conversion unit; q is the low byte and the rest of the low 22 bits are zero.
// Only the lower clamp is needed. Every non-NaN x of the group lies in [min, max], so
// fl(x - min) <= fl(max - min) = r; and the fp16 scale is at most (2^b - 1)/r times
// (1 + 2^-11)(1 + 2^-24), or 65504 < (2^b - 1)/r when it saturates. The product is thus
// below 2^b - 1 + 0.13 and rounds to at most 2^b - 1, while a NaN (a NaN x, or inf * 0
// in a group holding an infinity) becomes 0 through fmaxf, as the conversion gives.
template <int BITS>
__device__ __forceinline__ uint32_t quant_bits(float x, float mn, float s) {
    const float v = fmaxf(__fmul_rn(__fsub_rn(x, mn), s), 0.0f);
    return __float_as_uint(__fadd_rn(v, 12582912.0f));
}

// quant_bits of the two fp16 values of a half2 word (low value first), with min and
// scale given as packed pairs {min_lo, min_hi} and {scale_lo, scale_hi} (the two values
// may belong to different groups).
// fl(x - min) is formed by the mixed-precision subtract (fp16 operand, fp32 operand and
// result): the fp16 value enters exactly, as after a conversion, and the difference is
// rounded once - the same bits as converting first, one instruction fewer per value.
__device__ __forceinline__ void quant_bits_pair(uint32_t w, uint64_t mn2, uint64_t s2, uint32_t& lo, uint32_t& hi) {
    float a, b, mn, mn_hi;
    f2_unpack(mn2, mn, mn_hi);
    asm("{.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\tsub.rn.f32.f16 %0, l, %3;\n\tsub.rn.f32.f16 %1, h, %4;}"
        : "=f"(a), "=f"(b)
        : "r"(w), "f"(mn), "f"(mn_hi));
    f2_unpack(f2_mul(f2_pack(a, b), s2), a, b);
    f2_unpack(f2_add(f2_pack(fmaxf(a, 0.0f), fmaxf(b, 0.0f)), f2_pack(12582912.0f, 12582912.0f)), a, b);
    lo = __float_as_uint(a);
    hi = __float_as_uint(b);
}

template <int BITS>
__device__ __forceinline__ uint32_t quant_one(float x, float mn, float s) {
    return quant_bits<BITS>(x, mn, s) & ((1u << BITS) - 1u);
}

// Four byte-valued words (code in the low byte of each) -> one u32, byte k from word k.
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
    return __byte_perm(__byte_perm(b0, b1, 0x0040u), __byte_perm(b2, b3, 0x0040u), 0x5410u);
}

// Eight consecutive fp16 values (one 16-byte vector) -> 4-bit codes packed in a u32
// (byte k = q[2k] | q[2k+1] << 4).
__device__ __forceinline__ uint32_t quant8_4bit(uint4 v, float mn, float s) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const uint64_t mn2 = f2_pack(mn, mn), s2 = f2_pack(s, s);
    uint32_t p[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t lo, hi;
        quant_bits_pair(w[k], mn2, s2, lo, hi);
        p[k] = lo + (hi << 4);   // low byte: q_lo + 16 q_hi (the rest of both low bytes is zero)
    }
    return pack_low_bytes(p[0], p[1], p[2], p[3]);
}

// Eight consecutive fp16 values -> eight 8-bit codes.
__device__ __forceinline__ uint2 quant8_8bit(uint4 v, float mn, float s) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const uint64_t mn2 = f2_pack(mn, mn), s2 = f2_pack(s, s);
    uint32_t b[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) quant_bits_pair(w[k], mn2, s2, b[2 * k], b[2 * k + 1]);
    return make_uint2(pack_low_bytes(b[0], b[1], b[2], b[3]), pack_low_bytes(b[4], b[5], b[6], b[7]));
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

// min and max over the L lanes of a group (L a power of two, lanes aligned to L) from
// each lane's half2 min/max pair: {min, -max} travel as one half2 word, so every
// shuffle round is one shuffle and one packed min (exact: selects and a negation).
template <int L>
__device__ __forceinline__ void group_minmax(__half2 hmn, __half2 hmx, float& mn, float& mx) {
    const __half2 a = __halves2half2(__low2half(hmn), __hneg(__low2half(hmx)));
    const __half2 b = __halves2half2(__high2half(hmn), __hneg(__high2half(hmx)));
    __half2 r = __hmin2(a, b);
#pragma unroll
    for (int off = 1; off < L; off <<= 1) {
        const uint32_t o = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<const uint32_t*>(&r), off);
        r = __hmin2(r, *reinterpret_cast<const __half2*>(&o));
    }
    mn = __low2float(r);
    mx = -__high2float(r);
}

// Reduce a half2 min/max pair to scalars (exact: min/max select, no rounding).
__device__ __forceinline__ float hmin_of(__half2 m) { return fminf(__low2float(m), __high2float(m)); }
__device__ __forceinline__ float hmax_of(__half2 m) { return fmaxf(__low2float(m), __high2float(m)); }

// Dequantisation step of a group: fp32(1/scale16); 0 marks a constant group.
__device__ __forceinline__ float group_step(__half s16) {
    const float s = __half2float(s16);
    return s > 0.0f ? __fdiv_rn(1.0f, s) : 0.0f;
}

// A code q < 2^23 as an exact fp32: the mantissa of 2^23 + q minus 2^23 (no conversion
// unit involved).
__device__ __forceinline__ float code_to_float(uint32_t q) {
    return __fsub_rn(__uint_as_float(0x4B000000u | q), 8388608.0f);
}

// x^ = fp16(fp32(fp32(q * step) + min)); a constant group (step 0) returns min.
__device__ __forceinline__ __half dequant_one(uint32_t q, float step, float mn) {
    if (step == 0.0f) return __float2half_rn(mn);
    return __float2half_rn(__fadd_rn(__fmul_rn(code_to_float(q), step), mn));
}

// Two codes of a group with a nonzero step -> their fp16 values as one half2 word
// (low half from q0), with the rounding of dequant_one. This stays scalar: with the
// product and the sum on packed fp32 pairs, the decompressed values differed from the
// scalar path at fp16 rounding boundaries (consistent with the two being fused).
__device__ __forceinline__ uint32_t dequant_two(uint32_t q0, uint32_t q1, float step, float mn) {
    const __half2 h = __floats2half2_rn(__fadd_rn(__fmul_rn(code_to_float(q0), step), mn),
                                        __fadd_rn(__fmul_rn(code_to_float(q1), step), mn));
    return *reinterpret_cast<const uint32_t*>(&h);
}

}  // namespace flexq
