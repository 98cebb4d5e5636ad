// Dequant-fused weight GEMM on the 5th-generation tensor cores (tcgen05).
//
//   y[m][n] = epilogue( sum_k x[m][k] * W^[n][k] + bias[n] )
//
// W is a group-wise compressed weight (the walkthrough page «FlexGen 单 GPU 高吞吐大模型推理引擎：论文解读与源码实战指南», section 6.3:
// 4-bit codes, group 64, per-group fp16 {min, scale}), stored [N][K] and grouped along
// K, so a 64-wide K chunk is exactly one group per row. The kernel never materialises
// W^ in global memory:
//
//   warp 0      TMA: code tiles [128 rows][128 B] (one step = 4 K chunks at 4 bits, 2
//               at 8 bits) and metadata tiles [128 rows][4 groups] into a shared ring
//   warp 1      TMA: activation tiles [BN rows][64] fp16 with the 128-byte swizzle, a
//               step (or half a step for BN > 128) per stage
//   warp 2      allocates all 512 TMEM columns and issues tcgen05.mma (one thread):
//               A (the dequantised weights) from TMEM, B (activations) from shared
//               memory, one wait and one commit per step
//   warps 4-11  unpack the codes to fp16 (q*step + min, one half2 FMA per pair) and
//               store them into the step's A slot in TMEM (tcgen05.st), then run the
//               epilogue from the TMEM accumulator (bias, 1/sqrt(d) on the query
//               columns, ReLU, residual, fp16 store, fused store_cache)
//
// TMEM: columns [0, 256) hold the fp32 accumulator (BN <= 256 columns), [256, 512) the
// A slots (two steps at 4 bits), so dequantisation of step j+1 overlaps the MMAs of
// step j and the dequantised weights never go through shared memory.
//
// Swap-AB orientation: the weight rows are the MMA's M side (128 per CTA) and the
// activation rows (batch in decode, tokens in prefill) its N side (BN = 16..256), so a
// decode batch of a few sequences still fills an M=128 instruction. Small grids are
// split along K into up to 8 splits per tile. When every tile's splits fit on the GPU
// at once as one thread-block cluster each, they are launched so: each split leaves its
// fp32 partial tile in its own shared memory and the CTAs of the cluster each finish a
// share of the tile, reading all partials over distributed shared memory. Otherwise
// the splits write fp32 partials to the workspace and the last CTA of a tile (atomic
// ticket) finishes it. Both add the partials in split order, so results do not depend
// on scheduling. Every mbarrier wait is bounded: on
// expiry the CTA records FLEX_ERR_TIMEOUT in the device status word, drains its own
// copies and MMAs, frees TMEM and exits (still taking part in the cluster barriers).
#include <atomic>
#include <map>
#include <mutex>
#include <tuple>

#include "quant.cuh"
#include "tc.cuh"

namespace flexq {

namespace {

constexpr int kBM = 128;           // weight rows per CTA (MMA M)
constexpr int kBK = 64;            // K per stage = one quantisation group
// 14 warps: 0 code TMA, 1 activation TMA, 2 TMEM allocation, 4-11 dequantisation into
// TMEM and then the epilogue (a warp reaches only the TMEM lane quarter warp % 4, so each
// quarter has two of them, one per K half). One thread each of warps 2, 3, 12, 13
// issues the MMAs of one accumulator (as many issuers as accumulators), so the issue
// latency of tcgen05.mma is paid in parallel.
constexpr int kThreads = 448;
constexpr int kDequantThreads = 256;
constexpr int kMetaChunks = 4;     // groups per metadata tile
constexpr int kDoneRing = 8;       // mma_done barriers, one per step (more than any ring's look-ahead)
constexpr int kTmemCols = 512;     // whole TMEM of the SM (one CTA per SM)
constexpr int kACol0 = 256;        // TMEM columns [0, 256): accumulator; [256, 512): dequantised A slots
constexpr int kACols = kTmemCols - kACol0;
constexpr int kMaxSplits = 8;      // K splits of a tile form one cluster (portable size)
// Split-K tickets: a fixed region at the start of every GEMM workspace (the partials
// follow it), so that GEMMs of different tile counts sharing one workspace never write
// partials over each other's tickets. A split plan has at most kTicketBytes / 4 tiles.
constexpr int64_t kTicketBytes = 2048;

struct GemmParams {
    uint64_t wait_ns;      // limit of the pipeline waits (drain waits keep tc::kWaitLimitNs)
    // nullptr, or a device flag the code producer waits on (bounded by wait_ns) before its
    // first weight load (flex_set_gemm_gate)
    const volatile int* gate;
    const __half* bias;
    const __half* residual;
    __half* y;
    int* status;
    int M, N, K;
    int BN;
    int splits, cps;       // K splits, chunks per split (multiple of kMetaChunks)
    int nq;                // columns n < nq are multiplied by qscale
    float qscale;
    int relu;
    // weights may be read before the previous kernel on the stream has completed: set
    // only by the layer calls, whose kernels never write weights (every kernel of this
    // library signals its dependents only after its own wait, so everything before the
    // immediately preceding kernel is complete whenever this grid runs)
    int early_w;
    int yperm;             // write y in the interleaved 8-block order
    int nsx, nsc;          // activation / code ring depths
    int xu;                // K chunks per activation stage
    int nacc, acc_stride;  // independent TMEM accumulators and their column spacing
    int nslot, a_col0;     // gemm_tc2_kernel: A slots (one chunk per tile) and their first TMEM column
    // K splits (splits > 1): cluster = 1 reduces them through distributed shared memory
    // inside one thread-block cluster per tile; cluster = 0 through fp32 partials in the
    // workspace, the last CTA of a tile (atomic ticket) finishing it
    int cluster;
    float* part;
    int* counters;
    // gemm_tc2_kernel stream-K schedule (sk = 1): the tiles' K steps laid end to end,
    // sk_total of them, shared out evenly over the grid; tiles numbered tm * sk_tiles_n + tn
    int sk, sk_tiles_n;
    int64_t sk_total;
    // gemm_tc2_kernel, splits in one wave without a cluster: the splits of a tile exchange
    // their partials and each finishes a share of the columns (xchg = 1) instead of a ticket
    int xchg;
    uint32_t off_x, off_c, off_m, off_bar;
    uint32_t tmem_cols;
    // fused store_cache (QKV projection): output features [kv.h, 2 kv.h) are the keys and
    // [2 kv.h, 3 kv.h) the values; row m is row r = m % kv.rows of cache m / kv.rows, and
    // r = b * kv.seq + t goes to slot kv.pos0 + t of that cache's sequence b
    KvTarget kv;
};

struct Bars {
    uint32_t codes_full, codes_empty, x_full, a_full, mma_done, acc_full, drain;   // drain: one per issuer
    uint32_t red;          // gemm_tc2_kernel: two barriers of the split-K reduction's bulk loads
};

__device__ __forceinline__ uint32_t dequant_pair(uint32_t raw_pair_bits, uint32_t step2, uint32_t mn2) {
    // raw_pair_bits holds two integers q in the low mantissa bits of 1024.0h: (1024+q)
    const uint32_t bias2 = 0x64006400u;
    __half2 v = __hsub2(*reinterpret_cast<const __half2*>(&raw_pair_bits), *reinterpret_cast<const __half2*>(&bias2));
    v = __hfma2(v, *reinterpret_cast<const __half2*>(&step2), *reinterpret_cast<const __half2*>(&mn2));
    return *reinterpret_cast<uint32_t*>(&v);
}

// Hardware reciprocal (rcp.approx, relative error below 2^-22); the result is rounded
// to fp16 right after, so it matches the correctly rounded reciprocal except at rare
// fp16 rounding ties.
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ uint32_t lop_nib(uint32_t w) {
    // (w & 0x000F000F) | 0x64006400
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "r"(0x000F000Fu), "r"(0x64006400u));
    return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ uint32_t lop_nib_hi(uint32_t w) {
    // (w & 0x00F000F0) | 0x64006400: the high nibbles of bytes 0 and 2 left in place, as
    // fp16 1024 + 16 q
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "r"(0x00F000F0u), "r"(0x64006400u));
    return r;
}

// Dequantisation constants of one group from its metadata word {min, scale}, each packed
// twice: step = fp16(1/scale) (0 for a constant group, which then decodes to min), step/16
// for codes read in place from a byte's high nibble (fp16 16 q: 16 q * step/16 = q * step,
// exactly while step/16 is a normal fp16), and min.
struct DqConst {
    uint32_t step2, step2_16, mn2;
};
__device__ __forceinline__ DqConst dq_const(uint32_t mw) {
    const __half mn = __ushort_as_half(static_cast<unsigned short>(mw & 0xFFFFu));
    const float sc32 = __half2float(__ushort_as_half(static_cast<unsigned short>(mw >> 16)));
    const float r = sc32 > 0.f ? rcp_approx(sc32) : 0.f;
    const __half2 s = __float2half2_rn(r), s16 = __float2half2_rn(r * 0.0625f), m = __half2half2(mn);
    DqConst k;
    k.step2 = *reinterpret_cast<const uint32_t*>(&s);
    k.step2_16 = *reinterpret_cast<const uint32_t*>(&s16);
    k.mn2 = *reinterpret_cast<const uint32_t*>(&m);
    return k;
}

// 8 codes of 4 bits (one u32, element e in bits 4e..4e+3) as the four pairs (e0,e4)
// (e1,e5) (e2,e6) (e3,e7): low nibbles masked out directly, high nibbles in place, one
// shift for the upper byte of each half.
__device__ __forceinline__ void dequant8_4bit_pairs(uint32_t w, const DqConst& k, uint32_t (&p)[4]) {
    const uint32_t w8 = w >> 8;
    p[0] = dequant_pair(lop_nib(w), k.step2, k.mn2);           // (e0, e4)
    p[1] = dequant_pair(lop_nib_hi(w), k.step2_16, k.mn2);     // (e1, e5)
    p[2] = dequant_pair(lop_nib(w8), k.step2, k.mn2);          // (e2, e6)
    p[3] = dequant_pair(lop_nib_hi(w8), k.step2_16, k.mn2);    // (e3, e7)
}

// 8 codes of 4 bits -> 8 fp16 in natural order.
__device__ __forceinline__ uint4 dequant8_4bit(uint32_t w, const DqConst& k) {
    uint32_t p[4];
    dequant8_4bit_pairs(w, k, p);
    return make_uint4(prmt(p[0], p[1], 0x5410u), prmt(p[2], p[3], 0x5410u), prmt(p[0], p[1], 0x7632u),
                      prmt(p[2], p[3], 0x7632u));
}

// Same 8 codes, left in the pair order the unpack produces: (e0,e4) (e1,e5) (e2,e6)
// (e3,e7), i.e. positions [e0 e4 e1 e5 e2 e6 e3 e7]. The activation operand must then
// use the same order inside every 8-block of K (the "interleaved" activation layout the
// layer kernels write), and the MMA sees matching K positions on both sides.
__device__ __forceinline__ uint4 dequant8_4bit_il(uint32_t w, const DqConst& k) {
    uint32_t p[4];
    dequant8_4bit_pairs(w, k, p);
    return make_uint4(p[0], p[1], p[2], p[3]);
}

__device__ __forceinline__ uint32_t lop_byte(uint32_t x) {
    // (x & 0x00FF00FF) | 0x64006400
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(0x00FF00FFu), "r"(0x64006400u));
    return r;
}

// 8 codes of 8 bits (two u32: k0..k3, k4..k7) -> 8 fp16 in the interleaved order.
__device__ __forceinline__ uint4 dequant8_8bit_il(uint32_t w0, uint32_t w1, uint32_t step2, uint32_t mn2) {
    return make_uint4(dequant_pair(lop_byte(prmt(w0, w1, 0x0400u)), step2, mn2),
                      dequant_pair(lop_byte(prmt(w0, w1, 0x0501u)), step2, mn2),
                      dequant_pair(lop_byte(prmt(w0, w1, 0x0602u)), step2, mn2),
                      dequant_pair(lop_byte(prmt(w0, w1, 0x0703u)), step2, mn2));
}

// 4 codes of 8 bits (one u32) -> 4 fp16 as two half2.
__device__ __forceinline__ uint2 dequant4_8bit(uint32_t w, uint32_t step2, uint32_t mn2) {
    const uint32_t hi = 0x64646464u;
    return make_uint2(dequant_pair(prmt(w, hi, 0x4140u), step2, mn2), dequant_pair(prmt(w, hi, 0x4342u), step2, mn2));
}

// Fused store_cache for 8 token columns of the epilogue. Thread (warp, lane) holds output
// feature n (= one dimension of one head) for the columns col..col+7, already rounded to
// fp16. A quantisation group is gs consecutive features: one warp (gs = 32) or the two
// warps of a pair (gs = 64: warps 4/5, 6/7, 8/9, 10/11 hold rows 0-63 / 64-127 of the
// same column half). min/max are reduced over the group, then every thread quantises its
// own value with the shared quantiser (bit-identical to flexq_compress of the same
// fp16 values); even lanes write the byte of two 4-bit codes, the group's first row its
// {min, scale}.
template <int BITS>
__device__ __forceinline__ void kv_store8_bits(const GemmParams& p, const __half (&o16)[8], int col, int m0, int n0,
                                               int n, int warp, int lane, uint32_t* kv_red) {
    const int sec = (n0 - p.kv.h) / p.kv.h;                // 0 keys, 1 values
    const int f = n - p.kv.h - sec * p.kv.h;
    const int head = f / p.kv.hd, dim = f % p.kv.hd;
    // {min, max} of each of the 8 columns over the warp's 32 rows, as half2 (min low, max
    // high), reduced and scattered: after the xor-16/8/4 rounds lane l holds column
    // (l >> 2) & 7 over 8 lanes, and the xor-2/1 rounds finish it over all 32
    auto comb = [](uint32_t a, uint32_t b) -> uint32_t {
        const __half2 lo = __hmin2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
        const __half2 hi = __hmax2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
        return prmt(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi), 0x7610u);
    };
    uint32_t v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = pack_half2_bits(o16[j], o16[j]);
    const bool b4 = (lane & 16) != 0, b3 = (lane & 8) != 0, b2 = (lane & 4) != 0;
    uint32_t w[4], x[2];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t got = __shfl_xor_sync(0xffffffffu, b4 ? v[k] : v[k + 4], 16);
        w[k] = comb(b4 ? v[k + 4] : v[k], got);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const uint32_t got = __shfl_xor_sync(0xffffffffu, b3 ? w[k] : w[k + 2], 8);
        x[k] = comb(b3 ? w[k + 2] : w[k], got);
    }
    uint32_t y = comb(b2 ? x[1] : x[0], __shfl_xor_sync(0xffffffffu, b2 ? x[0] : x[1], 4));
    y = comb(y, __shfl_xor_sync(0xffffffffu, y, 2));
    y = comb(y, __shfl_xor_sync(0xffffffffu, y, 1));
    const int jc = (lane >> 2) & 7;                        // the column this lane now holds
    if (p.kv.gs == 64) {
        // a group of 64 rows spans the two warps of a pair: add the partner's column
        const int wi = warp - 4, pairbar = 2 + (wi >> 1);
        if ((lane & 3) == 0) kv_red[wi * 8 + jc] = y;
        asm volatile("bar.sync %0, 64;" ::"r"(pairbar) : "memory");
        y = comb(y, kv_red[(wi ^ 1) * 8 + jc]);
        asm volatile("bar.sync %0, 64;" ::"r"(pairbar) : "memory");   // kv_red is reused by the next call
    }
    // this lane's column: scale (one division per lane), then every column's {min, scale}
    // to every lane
    const __half mnh = __ushort_as_half(static_cast<unsigned short>(y & 0xFFFFu));
    const __half mxh = __ushort_as_half(static_cast<unsigned short>(y >> 16));
    const __half s16c = group_scale16<BITS>(__half2float(mnh), __half2float(mxh));
    const uint32_t ms = pack_half2_bits(mnh, s16c);
    const int gph = p.kv.hd / p.kv.gs;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t msj = __shfl_sync(0xffffffffu, ms, 4 * j);
        const int m = m0 + col + j;
        const float mn = h2f_lo(msj);
        const __half s16 = __ushort_as_half(static_cast<unsigned short>(msj >> 16));
        const uint32_t q = quant_one<BITS>(__half2float(o16[j]), mn, __half2float(s16));
        const uint32_t qn = __shfl_down_sync(0xffffffffu, q, 1);
        if (m >= p.M) continue;
        const int c = m / p.kv.rows, r = m - c * p.kv.rows;
        const int b = r / p.kv.seq, t = r - b * p.kv.seq;
        uint8_t* codes = p.kv.codes[c][sec];
        uint32_t* meta = p.kv.meta[c][sec];
        const int64_t slot = (static_cast<int64_t>(b) * p.kv.nh + head) * p.kv.max_seq + p.kv.pos0 + t;
        if (BITS == 4) {
            if ((lane & 1) == 0) codes[slot * (p.kv.hd / 2) + dim / 2] = static_cast<uint8_t>(q | (qn << 4));
        } else {
            codes[slot * p.kv.hd + dim] = static_cast<uint8_t>(q);
        }
        if (dim % p.kv.gs == 0) meta[slot * gph + dim / p.kv.gs] = pack_half2_bits(stored_min16(mn), s16);
    }
}

__device__ __forceinline__ void kv_store8(const GemmParams& p, const __half (&o16)[8], int col, int m0, int n0, int n,
                                          int warp, int lane, uint32_t* kv_red) {
    if (p.kv.bits == 4)
        kv_store8_bits<4>(p, o16, col, m0, n0, n, warp, lane, kv_red);
    else
        kv_store8_bits<8>(p, o16, col, m0, n0, n, warp, lane, kv_red);
}

// The MMAs of one K chunk (4 k-steps of 16) that belong to issuer ii of NI: k-steps ii,
// ii + NI, ... into accumulator d_acc (unrolled, so the issue loop has no branches).
template <int NI>
__device__ __forceinline__ void issue_ksteps(uint32_t d_acc, uint32_t a_chunk, uint64_t b_desc, uint32_t idesc, int ii,
                                             bool first) {
#pragma unroll
    for (int q = 0; q < kBK / 16 / NI; ++q) {
        const int kk = ii + q * NI;
        tc::mma_f16_ts(d_acc, a_chunk + kk * 8, b_desc + 2 * kk, idesc, (first && q == 0) ? 0u : 1u);
    }
}

// Split-K partials in the workspace: per (tile, split) a block of BN x R fp32 (R = the
// tile's weight rows) laid out [col / 8][row][8], so a thread (one row) moves 8 columns
// as two 16-byte accesses and a warp (32 consecutive rows) covers 1 KB contiguously.
__device__ __forceinline__ void part_store8(float* blk, int R, int row, int col, const float (&v)[8]) {
    float4* d = reinterpret_cast<float4*>(blk + (static_cast<int64_t>(col >> 3) * R + row) * 8);
    __stcg(d, make_float4(v[0], v[1], v[2], v[3]));
    __stcg(d + 1, make_float4(v[4], v[5], v[6], v[7]));
}
// Requests the 8 columns (col..col+7) of `row` of splits s0..s0+3 (zeros past `splits`).
__device__ __forceinline__ void part_load4(const float* all, int64_t split_stride, int splits, int s0, int R, int row,
                                           int col, float4 (&t)[4][2]) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        if (s0 + u < splits) {
            const float4* q = reinterpret_cast<const float4*>(all + (s0 + u) * split_stride +
                                                              (static_cast<int64_t>(col >> 3) * R + row) * 8);
            t[u][0] = __ldcg(q);
            t[u][1] = __ldcg(q + 1);
        } else {
            t[u][0] = t[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
}
__device__ __forceinline__ void part_add4(float (&acc)[8], const float4 (&t)[4][2]) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {           // split order
        acc[0] += t[u][0].x;
        acc[1] += t[u][0].y;
        acc[2] += t[u][0].z;
        acc[3] += t[u][0].w;
        acc[4] += t[u][1].x;
        acc[5] += t[u][1].y;
        acc[6] += t[u][1].z;
        acc[7] += t[u][1].w;
    }
}
// The last split of a tile: for every 8-column group in [cbeg, cend) of `row`, the sum of
// all splits' partials in split order, handed to finish(col, acc). With at most 4 splits
// the next group's partials are requested before the current group is finished, so the
// loop pays about one memory round trip per two groups instead of one per group.
template <typename Finish>
__device__ __forceinline__ void part_reduce(const float* all, int64_t split_stride, int splits, int R, int row,
                                            int cbeg, int cend, Finish&& finish) {
    if (splits <= 4) {
        float4 nx[4][2];
        if (cbeg < cend) part_load4(all, split_stride, splits, 0, R, row, cbeg, nx);
        for (int col = cbeg; col < cend; col += 8) {
            float4 cu[4][2];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                cu[u][0] = nx[u][0];
                cu[u][1] = nx[u][1];
            }
            if (col + 8 < cend) part_load4(all, split_stride, splits, 0, R, row, col + 8, nx);
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
            part_add4(acc, cu);
            finish(col, acc);
        }
    } else {
        for (int col = cbeg; col < cend; col += 8) {
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
            for (int s0 = 0; s0 < splits; s0 += 4) {
                float4 t[4][2];
                part_load4(all, split_stride, splits, s0, R, row, col, t);
                part_add4(acc, t);
            }
            finish(col, acc);
        }
    }
}

template <int BITS, bool XPERM>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_codes,
                                                              const __grid_constant__ CUtensorMap tm_meta,
                                                              const __grid_constant__ CUtensorMap tm_x,
                                                              const GemmParams p) {
    constexpr int CROW = kBK * BITS / 8;          // code bytes per row and K chunk (32 or 64)
    constexpr int KU = 128 / CROW;                // K chunks per step = per code stage (4 or 2)
    constexpr int CSTAGE = kBM * 128;             // code bytes per stage: 128 rows x 128 B
    constexpr int MSTAGE = kBM * kMetaChunks * 4; // metadata bytes per stage: 128 rows x 4 groups
    constexpr int SLOT_COLS = KU * 32;            // TMEM columns of one A slot: KU chunks x 64 fp16
    constexpr int NSLOT = kACols / SLOT_COLS;     // A slots (2 at 4 bits, 4 at 8 bits)
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const gbase = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kBM, m0 = blockIdx.y * p.BN, split = blockIdx.z;
    const int nk_total = p.K / kBK;
    const int c_begin = split * p.cps;                            // multiple of kMetaChunks
    const int nk = min(nk_total, c_begin + p.cps) - c_begin;      // multiple of kMetaChunks
    const int nsteps = nk / KU;
    const int XU = p.xu;                                          // K chunks per activation stage
    const int nxu = nk / XU;

    const uint32_t sX = base, sC = base + p.off_c, sM = base + p.off_m;
    const uint32_t sb = base + p.off_bar;
    const int NSX = p.nsx, NSC = p.nsc;
    const uint32_t xbytes = static_cast<uint32_t>(p.BN) * 128;   // one activation chunk: BN rows x 64 fp16
    Bars B;
    B.codes_full = sb;
    B.codes_empty = B.codes_full + 8 * NSC;
    B.x_full = B.codes_empty + 8 * NSC;
    B.a_full = B.x_full + 8 * NSX;
    B.mma_done = B.a_full + 8 * NSLOT;
    B.acc_full = B.mma_done + 8 * kDoneRing;
    B.drain = B.acc_full + 8;
    const uint32_t misc = B.drain + 8 * 4;                    // tmem slot, abort flag, last flag
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + (misc - base));
    volatile int* abort = reinterpret_cast<volatile int*>(gbase + (misc - base) + 4);
    volatile int* last_flag = reinterpret_cast<volatile int*>(gbase + (misc - base) + 8);
    uint32_t* kv_red = reinterpret_cast<uint32_t*>(gbase + (misc - base) + 16);   // [8 warps][4 pairs][2]

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSC; ++s) {
            tc::bar_init(B.codes_full + 8 * s, 1);
            tc::bar_init(B.codes_empty + 8 * s, kDequantThreads);
        }
        for (int s = 0; s < NSX; ++s) tc::bar_init(B.x_full + 8 * s, 1);
        for (int s = 0; s < NSLOT; ++s) tc::bar_init(B.a_full + 8 * s, kDequantThreads);
        // every issuer commits each step once
        for (int s = 0; s < kDoneRing; ++s) tc::bar_init(B.mma_done + 8 * s, p.nacc);
        tc::bar_init(B.acc_full, p.nacc);
        for (int i = 0; i < 4; ++i) tc::bar_init(B.drain + 8 * i, 1);
        *abort = 0;
        *last_flag = 0;
        tc::bar_fence_init();
    }
    if (warp == 2) {
        tc::tmem_alloc(misc, kTmemCols);
        tc::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tc::tma_prefetch(&tm_codes);
        tc::tma_prefetch(&tm_meta);
    }
    if (warp == 1 && lane == 0) tc::tma_prefetch(&tm_x);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;             // accumulator: columns [0, BN); A slots from kACol0

    // epilogue mapping (warps 4-11): TMEM lane quarter lq = row block, column half ch
    const int lq = warp & 3, ch = (warp - 4) >> 2;
    const int irow = lq * 32 + lane;
    const int n = n0 + irow;
    const float scale_n = n < p.nq ? p.qscale : 1.f;
    // interleaved output: element k of every 8-block goes to position 2(k%4) + (k/4)%2
    const int n_out = p.yperm ? ((n & ~7) | ((n & 3) << 1) | ((n >> 2) & 1)) : n;
    // fused store_cache: this tile lies inside the key or the value block (h % 128 == 0)
    const bool kv_on = p.kv.codes[0][0] != nullptr && n0 >= p.kv.h;
    float bias_n = 0.f;                           // read by the epilogue after its PDL wait
    uint32_t all_ok = 0;                          // epilogue warps: the main loop completed
    // bias, q-scale, ReLU, residual, fp16 store (and store_cache) of 8 columns of row n
    auto finish8 = [&](int col, const float (&v)[8]) {
        float r[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int m = m0 + col + j;
            r[j] = (p.residual && m < p.M) ? __half2float(p.residual[static_cast<int64_t>(m) * p.N + n]) : 0.f;
        }
        __half o16[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int m = m0 + col + j;
            float x = (v[j] + bias_n) * scale_n;
            if (p.relu) x = fmaxf(x, 0.f);
            o16[j] = __float2half_rn(x + r[j]);
            if (m < p.M) p.y[static_cast<int64_t>(m) * p.N + n_out] = o16[j];
        }
        if (kv_on) kv_store8(p, o16, col, m0, n0, n, warp, lane, kv_red);
    };
    // Dependencies on the previous kernel (programmatic dependent launch): the
    // activation producer and the epilogue wait for it before touching global memory;
    // the code producer also waits unless early_w; the MMA and dequant roles only touch
    // shared memory and TMEM.

    if (warp == 0) {
        // ---------------- code + metadata producer: one stage = one step of KU chunks ----------------
        if (lane == 0) {
            if (!p.early_w) pdl_wait();
            // ring position kept incrementally (stage s, phase bit ph): no integer division
            // by the runtime ring depth on this thread's path
            int st = 0, s = 0;
            uint32_t ph = 0;
            const bool go = p.gate == nullptr || tc::gate_wait(p.gate, abort, p.status, p.wait_ns);
            for (; go && st < nsteps; ++st) {
                if (st >= NSC && !tc::bar_wait(B.codes_empty + 8 * s, ph ^ 1, abort, p.status, p.wait_ns)) break;
                const int c = c_begin + st * KU;
                tc::bar_arrive_expect_tx(B.codes_full + 8 * s, CSTAGE + MSTAGE);
                tc::tma_load_2d(sC + s * CSTAGE, &tm_codes, c * CROW, n0, B.codes_full + 8 * s);
                tc::tma_load_2d(sM + s * MSTAGE, &tm_meta, c & ~(kMetaChunks - 1), n0, B.codes_full + 8 * s);
                if (++s == NSC) { s = 0; ph ^= 1; }
            }
            // drain: every copy this thread issued has landed before the CTA can exit
            for (int s = 0; s < NSC && s < st; ++s) {
                const int last = s + ((st - 1 - s) / NSC) * NSC;
                volatile int never = 0;
                tc::bar_wait(B.codes_full + 8 * s, (last / NSC) & 1, &never, p.status);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- activation producer: one stage = XU chunks ----------------
        if (lane == 0) {
            pdl_wait();                           // the activations come from the previous kernel
            int u = 0, s = 0;
            for (; u < nxu; ++u) {
                if (u >= NSX) {
                    // the stage last held unit u - NSX: wait for the MMAs of the step that read it
                    const int pj = ((u - NSX) * XU) / KU;
                    if (!tc::bar_wait(B.mma_done + 8 * (pj % kDoneRing), (pj / kDoneRing) & 1, abort, p.status,
                                      p.wait_ns))
                        break;
                }
                tc::bar_arrive_expect_tx(B.x_full + 8 * s, XU * xbytes);
                for (int c = 0; c < XU; ++c)
                    tc::tma_load_2d(sX + (s * XU + c) * xbytes, &tm_x, (c_begin + u * XU + c) * kBK, m0,
                                    B.x_full + 8 * s);
                if (++s == NSX) s = 0;
            }
            const int issued = u;
            for (int s = 0; s < NSX && s < issued; ++s) {
                const int last = s + ((issued - 1 - s) / NSX) * NSX;
                volatile int never = 0;
                tc::bar_wait(B.x_full + 8 * s, (last / NSX) & 1, &never, p.status);
            }
        }
        __syncwarp();
    } else if (warp == 2 || warp == 3 || warp >= 12) {
        // ---------------- MMA issuers: one per accumulator ----------------
        // Issuer ii issues the k-steps kk = ii, ii + nacc, ... of every chunk into
        // accumulator ii, with one wait per step (A slot) and per activation stage and one
        // commit per step. Each thread's loop is free of integer division by runtime
        // values: its instruction latency is part of the issue rate.
        const int ii = warp == 2 ? 0 : (warp == 3 ? 1 : warp - 10);
        if (lane == 0 && ii < p.nacc) {
            const int NI = p.nacc;
            const uint32_t idesc = tc::idesc_f16_f32(kBM, p.BN);
            const uint32_t d_acc = tmem + static_cast<uint32_t>(ii * p.acc_stride);
            int xs = 0;
            uint32_t xph = 0;
            bool ok = true;
            int j = 0;
            for (; j < nsteps && ok; ++j) {
                const int sa = j % NSLOT;
                if (!tc::bar_wait(B.a_full + 8 * sa, (j / NSLOT) & 1, abort, p.status, p.wait_ns)) { ok = false; break; }
                tc::fence_after_sync();
                const uint32_t a_tm = tmem + kACol0 + sa * SLOT_COLS;
                for (int c0 = 0; c0 < KU && ok; c0 += XU) {
                    if (!tc::bar_wait(B.x_full + 8 * xs, xph, abort, p.status, p.wait_ns)) { ok = false; break; }
                    const uint32_t xb = sX + static_cast<uint32_t>(xs * XU) * xbytes;
                    for (int c2 = 0; c2 < XU; ++c2) {
                        const int c = c0 + c2;
                        const uint64_t bd = tc::desc_k_sw128(xb + c2 * xbytes);
                        const bool first = (j == 0 && c == 0);
                        if (NI == 4) issue_ksteps<4>(d_acc, a_tm + c * 32, bd, idesc, ii, first);
                        else if (NI == 2) issue_ksteps<2>(d_acc, a_tm + c * 32, bd, idesc, ii, first);
                        else issue_ksteps<1>(d_acc, a_tm + c * 32, bd, idesc, ii, first);
                    }
                    if (++xs == NSX) { xs = 0; xph ^= 1; }
                }
                if (!ok) break;
                // exactly one commit per step and issuer: a commit covers the MMAs this
                // thread issued since its previous one, so a second commit here would
                // complete at once. The A slot and the activation stages of this step are
                // reused once every issuer's commit has landed; the last step's commits
                // are the accumulator-ready signal.
                tc::mma_commit(j + 1 < nsteps ? B.mma_done + 8 * (j % kDoneRing) : B.acc_full);
            }
            // Every commit's mbarrier arrival must have landed before the CTA exits: a late
            // arrival would hit the barriers of the next CTA on this SM, which live at the
            // same shared-memory addresses. Steps [0, committed) were committed to the
            // mma_done ring; after an abort a final commit drains whatever is still on the
            // tensor cores.
            volatile int never = 0;
            const int committed = ok ? nsteps - 1 : j;   // (the last step of a full run went to acc_full)
            if (!ok) {
                tc::mma_commit(B.drain + 8 * ii);
                tc::bar_wait(B.drain + 8 * ii, 0, &never, p.status);
            }
            for (int c = committed - kDoneRing > 0 ? committed - kDoneRing : 0; c < committed; ++c)
                tc::bar_wait(B.mma_done + 8 * (c % kDoneRing), (c / kDoneRing) & 1, &never, p.status);
            if (ok) tc::bar_wait(B.acc_full, 0, &never, p.status);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------- dequantisation into TMEM ----------------
        // Warp w writes TMEM lanes 32 (w % 4) .. +31 (a warp may only access its own lane
        // quarter): thread (row = 32 (w % 4) + lane, half h) turns half of the row's codes
        // of each K chunk (16 code bytes at 4 bits, 32 at 8 bits) into 32 fp16 = 16
        // columns of the step's A slot.
        const int q = warp & 3, h = (warp - 4) >> 2;
        const int row = q * 32 + lane;
        const int sw = row & 7;
        const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16) + kACol0 + h * 16;
        bool ok = true;
        int s = 0;
        uint32_t cph = 0;
        for (int st = 0; st < nsteps && ok; ++st) {
            if (!tc::bar_wait(B.codes_full + 8 * s, cph, abort, p.status, p.wait_ns)) { ok = false; break; }
            // codes of the stage (the tile was stored with the 128-byte swizzle: 16-byte
            // unit u of row r sits at unit u ^ (r % 8))
            const uint32_t crow = sC + s * CSTAGE + row * 128;
            uint4 cw[KU][BITS / 4];
#pragma unroll
            for (int c = 0; c < KU; ++c)
#pragma unroll
                for (int v = 0; v < BITS / 4; ++v) {
                    const int u = c * (CROW / 16) + h * (BITS / 4) + v;
                    cw[c][v] = tc::lds128(crow + ((u ^ sw) << 4));
                }
            const uint4 mrow = tc::lds128(sM + s * MSTAGE + row * 16);
            const int moff = (c_begin + st * KU) & (kMetaChunks - 1);
            // the A slot must have been read by the MMAs of step st - NSLOT
            const int sa = st % NSLOT;
            if (st >= NSLOT) {
                const int pj = st - NSLOT;
                if (!tc::bar_wait(B.mma_done + 8 * (pj % kDoneRing), (pj / kDoneRing) & 1, abort, p.status,
                                  p.wait_ns)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
            }
            // the step's groups (moff + c) % 4 of the metadata tile, decoded together (a
            // select per word: a runtime array index would put them in local memory)
            DqConst kc[KU];
#pragma unroll
            for (int c = 0; c < KU; ++c) {
                const int mi = (moff + c) & 3;
                kc[c] = dq_const(mi == 0 ? mrow.x : (mi == 1 ? mrow.y : (mi == 2 ? mrow.z : mrow.w)));
            }
#pragma unroll
            for (int c = 0; c < KU; ++c) {
                const uint32_t step2 = kc[c].step2, mnv2 = kc[c].mn2;
                uint32_t r[16];
                if (BITS == 4) {
                    const uint32_t w[4] = {cw[c][0].x, cw[c][0].y, cw[c][0].z, cw[c][0].w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint4 v = XPERM ? dequant8_4bit_il(w[j], kc[c]) : dequant8_4bit(w[j], kc[c]);
                        r[4 * j] = v.x;
                        r[4 * j + 1] = v.y;
                        r[4 * j + 2] = v.z;
                        r[4 * j + 3] = v.w;
                    }
                } else {
                    const uint4 q0 = cw[c][0], q1 = cw[c][BITS / 4 - 1];
                    const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint4 v;
                        if (XPERM) {
                            v = dequant8_8bit_il(w[2 * j], w[2 * j + 1], step2, mnv2);
                        } else {
                            const uint2 a = dequant4_8bit(w[2 * j], step2, mnv2);
                            const uint2 b = dequant4_8bit(w[2 * j + 1], step2, mnv2);
                            v = make_uint4(a.x, a.y, b.x, b.y);
                        }
                        r[4 * j] = v.x;
                        r[4 * j + 1] = v.y;
                        r[4 * j + 2] = v.z;
                        r[4 * j + 3] = v.w;
                    }
                }
                tc::tmem_st16(t_row + sa * SLOT_COLS + c * 32, r);
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            tc::bar_arrive(B.a_full + 8 * sa);
            // the code stage's values are all consumed: the next TMA may refill it
            tc::bar_arrive(B.codes_empty + 8 * s);
            if (++s == NSC) { s = 0; cph ^= 1; }
        }
        // ---------------- epilogue ----------------
        pdl_wait();                               // residual, bias and y
        pdl_trigger();                            // dependents may start their prologue
        bias_n = p.bias ? __half2float(p.bias[n]) : 0.f;
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (ok && !*abort) ok = tc::bar_wait(B.acc_full, 0, abort, p.status);
        // one decision for all 256 threads (they share the named barriers below)
        asm volatile(
            "{\n\t.reg .pred p, q;\n\t"
            "setp.ne.u32 p, %1, 0;\n\t"
            "barrier.cta.red.and.pred q, 1, 256, p;\n\t"
            "selp.u32 %0, 1, 0, q;\n\t}"
            : "=r"(all_ok)
            : "r"((ok && !*abort) ? 1u : 0u)
            : "memory");
        if (all_ok) {
            tc::fence_after_sync();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(lq * 32) << 16);
            const int cbeg = ch * (p.BN / 2), cend = cbeg + p.BN / 2;
            // 8 columns of row n: the sum of the accumulators, in accumulator order
            auto acc8 = [&](int col, float (&v)[8]) {
                tc::tmem_ld8(taddr + col, v);
                for (int a = 1; a < p.nacc; ++a) {
                    float w[8];
                    tc::tmem_ld8(taddr + a * p.acc_stride + col, w);
#pragma unroll
                    for (int j = 0; j < 8; ++j) v[j] += w[j];
                }
            };
            if (p.splits == 1) {
                for (int col = cbeg; col < cend; col += 8) {
                    float v[8];
                    acc8(col, v);
                    finish8(col, v);
                }
            } else if (p.cluster) {
                // this split's fp32 partial tile into this CTA's shared memory, column-major
                // [BN][128] (it reuses the activation ring: every MMA has completed)
                for (int col = cbeg; col < cend; col += 8) {
                    float v[8];
                    acc8(col, v);
#pragma unroll
                    for (int j = 0; j < 8; ++j) tc::st_shared_f32(sX + ((col + j) * kBM + irow) * 4, v[j]);
                }
            } else {
                // partial tile to the workspace (the ticket exchange follows below)
                float* mine = p.part + (static_cast<int64_t>(blockIdx.y * gridDim.x + blockIdx.x) * p.splits + split) *
                                           p.BN * kBM;
                for (int col = cbeg; col < cend; col += 8) {
                    float v[8];
                    acc8(col, v);
                    part_store8(mine, kBM, irow, col, v);
                }
            }
        }
        if (p.splits > 1 && !p.cluster) {
            // Ticket: every split of the tile takes one, also a split whose main loop gave
            // up, so that the tile's counter always returns to zero; the last split to
            // arrive adds all partials in split order and finishes the tile (all_ok is one
            // value for the 256 threads, so the named barriers stay uniform).
            const int et = (warp - 4) * 32 + lane;
            const int tile = blockIdx.y * gridDim.x + blockIdx.x;
            __threadfence();
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (et == 0) *last_flag = (atomicAdd(p.counters + tile, 1) == p.splits - 1);
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (*last_flag) {
                __threadfence();
                if (all_ok) {
                    const int cbeg = ch * (p.BN / 2), cend = cbeg + p.BN / 2;
                    const float* all = p.part + static_cast<int64_t>(tile) * p.splits * p.BN * kBM;
                    part_reduce(all, static_cast<int64_t>(p.BN) * kBM, p.splits, kBM, irow, cbeg, cend,
                                [&](int col, const float (&acc)[8]) { finish8(col, acc); });
                }
                if (et == 0) p.counters[tile] = 0;
            }
        }
    }

    if (p.splits > 1 && p.cluster) {
        // ---------------- split-K reduction across the cluster ----------------
        // The K splits of a tile are one thread-block cluster. After the barrier every
        // split's partial tile is visible; CTA r finishes the 8-column groups v with
        // v % splits == r, adding the partials in split order (deterministic), and the
        // second barrier keeps every CTA's shared memory alive until its peers are done.
        // All threads of every CTA take part in both barriers.
        tc::cluster_sync();
        if (warp >= 4 && all_ok) {
            const int S = p.splits;
            const int rank = static_cast<int>(tc::cluster_rank());
            int idx = 0;
            for (int v = rank; v < p.BN / 8; v += S, ++idx) {
                if ((idx & 1) != ch) continue;    // the two column halves alternate
                const int col = v * 8;
                float acc[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = 0.f;
                for (int sp = 0; sp < S; ++sp) {
                    const uint32_t peer = tc::map_peer(sX + (col * kBM + irow) * 4, static_cast<uint32_t>(sp));
                    float t[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) t[j] = tc::ld_peer_f32(peer + j * kBM * 4);
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[j] += t[j];
                }
                finish8(col, acc);
            }
        }
        tc::cluster_sync();
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 2) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------------------
// 256 weight rows per CTA (two 128-row tiles, t = 0, 1), for N a multiple of 256 and up
// to 192 activation rows per tile (BN). Each activation tile brought in from L2 feeds
// both weight tiles (half the activation traffic per weight row of the 128-row kernel),
// and the two tiles' MMA issuers run side by side. Above 128 activation rows this kernel
// was the faster of the two at every OPT-175B weight shape measured.
//
//   warp 0      TMA: code tiles [256 rows][128 B] and metadata [256 rows][4 groups]
//   warp 1      TMA: activation tiles [BN rows][64] fp16 (128-byte swizzle), XU chunks per stage
//   warps 2, 3  one thread each issues the MMAs of tile 0 / tile 1 into its own TMEM
//               accumulator (warp 2 also allocates TMEM)
//   warps 4-11  warp w dequantises rows 128 t + 32 (w % 4) + lane, t = (w - 4) / 4, one
//               whole 64-wide K chunk at a time into that tile's A slot in TMEM
//               (tcgen05.st), then runs the epilogue of the same rows
//
// TMEM: accumulator of tile t at columns [t acc_stride, t acc_stride + BN); from a_col0 on,
// nslot A slots of one chunk per tile (slot s of tile t at a_col0 + (s * 2 + t) * 32). A
// "unit" is one chunk: one A slot fill, one MMA issue round per tile, one commit per
// issuer (the mma_done ring counts units, across all segments of the CTA). The A-slot and
// mma_done barriers are per tile: a tile's issuer waits only for its own 4 dequantising
// warps, and they only for its commits, so one tile's issuer keeps the tensor pipe busy
// while the other waits (two threads issuing back to back are what it takes to keep the
// pipe full at these N: one thread issues an MMA every ~130-160 cycles, a 128 x 144 x 16
// MMA occupies the pipe for 72). A CTA works
// through one or more segments (see SegWalk); between segments the issuers wait for the
// epilogue to have read the accumulators (acc_full, one phase per segment). Bounded waits,
// abort and drain, split-K through clusters or tickets and the fused store_cache are as
// in gemm_tc_kernel.
constexpr int kRT = 2;                  // 128-row tiles per CTA
// 12 warps: 0 code TMA, 1 activation TMA, 2 and 3 the MMA issuers of tiles 0 and 1,
// 4-11 dequantisation and the epilogue. One CTA per SM, so a thread may hold up to 168
// registers (the epilogue with the fused store_cache needs about 140).
constexpr int kThreads2 = 384;
constexpr int kRows2 = kRT * kBM;       // 256
constexpr int kDoneRing2 = 16;          // mma_done barriers (units)
constexpr int kMaxPieces = 8;           // stream-K: later pieces of one tile that its owner adds

// A CTA's work, as segments of K steps of one tile. A classic launch gives each CTA one
// segment: tile (blockIdx.x, blockIdx.y), the steps of K split blockIdx.z. A stream-K
// launch (p.sk) lays the tiles' steps end to end and gives CTA c the contiguous share
// [c total / G, (c + 1) total / G): a run of segments that may start and end inside a
// tile. A segment that covers its whole tile finishes it directly. A tile shared by
// several CTAs is finished by the CTA holding its first steps (the owner; always its
// CTA's last segment), after the later pieces - each the first segment of one of the
// next CTAs, written to that CTA's partial slot early in its run - have been published.
struct Seg {
    int tn, tm;            // tile (256-row block of N, BN-column block of M)
    int k0, k1;            // steps [k0, k1) of the tile's nst steps
    bool whole, owner;     // covers the tile / first piece of a shared tile
};

struct SegWalk {
    int64_t pos, end;      // stream-K: the next step and the end of this CTA's share
    int nst, tiles_n;
    bool sk, done;
    __device__ SegWalk(const GemmParams& p, int nst_) : nst(nst_), tiles_n(p.sk_tiles_n), sk(p.sk != 0), done(false) {
        if (sk) {
            pos = static_cast<int64_t>(blockIdx.x) * p.sk_total / gridDim.x;
            end = static_cast<int64_t>(blockIdx.x + 1) * p.sk_total / gridDim.x;
        } else {
            pos = end = 0;
        }
    }
    __device__ bool next(const GemmParams& p, int KU, Seg& sg) {
        if (done) return false;
        if (!sk) {
            done = true;
            sg.tn = blockIdx.x;
            sg.tm = blockIdx.y;
            sg.k0 = blockIdx.z * (p.cps / KU);
            sg.k1 = min(nst, sg.k0 + p.cps / KU);
            sg.whole = p.splits == 1;
            sg.owner = false;
            return sg.k1 > sg.k0;
        }
        if (pos >= end) {
            done = true;
            return false;
        }
        const int t = static_cast<int>(pos / nst);
        sg.tn = t % tiles_n;
        sg.tm = t / tiles_n;
        sg.k0 = static_cast<int>(pos - static_cast<int64_t>(t) * nst);
        const int64_t room = end - pos;
        sg.k1 = room < static_cast<int64_t>(nst - sg.k0) ? sg.k0 + static_cast<int>(room) : nst;
        sg.whole = sg.k0 == 0 && sg.k1 == nst;
        sg.owner = sg.k0 == 0 && sg.k1 < nst;
        pos += sg.k1 - sg.k0;
        return true;
    }
};

template <int BITS, bool XPERM>
__global__ void __launch_bounds__(kThreads2, 1) gemm_tc2_kernel(const __grid_constant__ CUtensorMap tm_codes,
                                                               const __grid_constant__ CUtensorMap tm_meta,
                                                               const __grid_constant__ CUtensorMap tm_x,
                                                               const GemmParams p) {
    constexpr int CROW = kBK * BITS / 8;          // code bytes per row and K chunk (32 or 64)
    constexpr int KU = 128 / CROW;                // K chunks (units) per step = per code stage (4 or 2)
    constexpr int CSTAGE = kRows2 * 128;          // code bytes per stage: 256 rows x 128 B
    constexpr int MSTAGE = kRows2 * kMetaChunks * 4;
    constexpr int WPC = CROW / 16;                // 16-byte code vectors per row and chunk (2 or 4)
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const gbase = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nst = p.K / (kBK * KU);             // steps per tile
    const int XU = p.xu;
    const int NSLOT = p.nslot;

    const uint32_t sX = base, sC = base + p.off_c, sM = base + p.off_m;
    const uint32_t sb = base + p.off_bar;
    const int NSX = p.nsx, NSC = p.nsc;
    const uint32_t xbytes = static_cast<uint32_t>(p.BN) * 128;
    Bars B;
    B.codes_full = sb;
    B.codes_empty = B.codes_full + 8 * NSC;
    B.x_full = B.codes_empty + 8 * NSC;
    // per tile: a_full of (slot s, tile t) at a_full + 8 (2 s + t); mma_done of (unit u, tile t)
    // at mma_done + 8 (2 (u % kDoneRing2) + t)
    B.a_full = B.x_full + 8 * NSX;
    B.mma_done = B.a_full + 8 * kRT * NSLOT;
    B.acc_full = B.mma_done + 8 * kRT * kDoneRing2;   // here: the accumulators are free again (one phase per segment)
    B.drain = B.acc_full + 8;
    B.red = B.drain + 8 * 4;
    const uint32_t misc = B.red + 8 * 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + (misc - base));
    volatile int* abort = reinterpret_cast<volatile int*>(gbase + (misc - base) + 4);
    volatile int* last_flag = reinterpret_cast<volatile int*>(gbase + (misc - base) + 8);
    uint32_t* kv_red = reinterpret_cast<uint32_t*>(gbase + (misc - base) + 16);   // [8 warps][4 pairs][2]

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSC; ++s) {
            tc::bar_init(B.codes_full + 8 * s, 1);
            tc::bar_init(B.codes_empty + 8 * s, kDequantThreads);
        }
        for (int s = 0; s < NSX; ++s) tc::bar_init(B.x_full + 8 * s, 1);
        for (int s = 0; s < kRT * NSLOT; ++s) tc::bar_init(B.a_full + 8 * s, kDequantThreads / kRT);   // a tile's 4 warps
        for (int s = 0; s < kRT * kDoneRing2; ++s) tc::bar_init(B.mma_done + 8 * s, 1);   // the tile's issuer
        tc::bar_init(B.acc_full, kDequantThreads);
        for (int i = 0; i < 4; ++i) tc::bar_init(B.drain + 8 * i, 1);
        tc::bar_init(B.red, 1);
        tc::bar_init(B.red + 8, 1);
        *abort = 0;
        *last_flag = 0;
        tc::bar_fence_init();
    }
    if (warp == 2) {
        tc::tmem_alloc(misc, kTmemCols);
        tc::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tc::tma_prefetch(&tm_codes);
        tc::tma_prefetch(&tm_meta);
    }
    if (warp == 1 && lane == 0) tc::tma_prefetch(&tm_x);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    // epilogue / dequantisation mapping (warps 4-11): TMEM lane quarter lq, tile tt
    const int lq = warp & 3, tt = (warp - 4) >> 2;
    const int row = tt * kBM + lq * 32 + lane;                    // row of the CTA's 256
    uint32_t all_ok = 0;
    // the rings hold a whole fp32 partial (staged for one bulk store) once they are drained
    const bool stage_ok = static_cast<uint32_t>(p.BN) * kRows2 * 4 <= p.off_bar;

    if (warp == 0) {
        // ---------------- code + metadata producer: one stage = one step (KU chunks of 256 rows) ----------------
        if (lane == 0) {
            if (!p.early_w) pdl_wait();
            int s = 0, issued = 0;
            uint32_t ph = 0;
            bool go = p.gate == nullptr || tc::gate_wait(p.gate, abort, p.status, p.wait_ns);
            SegWalk walk(p, nst);
            Seg sg;
            while (go && walk.next(p, KU, sg)) {
                const int n0 = sg.tn * kRows2;
                for (int st = sg.k0; st < sg.k1; ++st) {
                    if (issued >= NSC && !tc::bar_wait(B.codes_empty + 8 * s, ph ^ 1, abort, p.status, p.wait_ns)) {
                        go = false;
                        break;
                    }
                    const int c = st * KU;
                    tc::bar_arrive_expect_tx(B.codes_full + 8 * s, CSTAGE + MSTAGE);
                    tc::tma_load_2d(sC + s * CSTAGE, &tm_codes, c * CROW, n0, B.codes_full + 8 * s);
                    tc::tma_load_2d(sM + s * MSTAGE, &tm_meta, c & ~(kMetaChunks - 1), n0, B.codes_full + 8 * s);
                    ++issued;
                    if (++s == NSC) { s = 0; ph ^= 1; }
                }
            }
            // drain: every copy this thread issued has landed before the CTA can exit
            for (int s2 = 0; s2 < NSC && s2 < issued; ++s2) {
                const int last = s2 + ((issued - 1 - s2) / NSC) * NSC;
                volatile int never = 0;
                tc::bar_wait(B.codes_full + 8 * s2, (last / NSC) & 1, &never, p.status);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- activation producer: one stage = XU chunks ----------------
        if (lane == 0) {
            pdl_wait();
            int s = 0, gx = 0;                    // ring slot; stages issued so far (all segments)
            bool go = true;
            SegWalk walk(p, nst);
            Seg sg;
            while (go && walk.next(p, KU, sg)) {
                const int m0 = sg.tm * p.BN;
                for (int xi = sg.k0 * KU / XU; xi < sg.k1 * KU / XU; ++xi) {
                    if (gx >= NSX) {
                        // the slot last held units [(gx - NSX) XU, +XU): wait for the MMAs of its
                        // last unit, both tiles
                        const int ul = (gx - NSX) * XU + XU - 1;
                        const uint32_t md = B.mma_done + 8 * (kRT * (ul % kDoneRing2));
                        const uint32_t par = (ul / kDoneRing2) & 1;
                        if (!tc::bar_wait(md, par, abort, p.status, p.wait_ns) ||
                            !tc::bar_wait(md + 8, par, abort, p.status, p.wait_ns)) {
                            go = false;
                            break;
                        }
                    }
                    tc::bar_arrive_expect_tx(B.x_full + 8 * s, XU * xbytes);
                    for (int c = 0; c < XU; ++c)
                        tc::tma_load_2d(sX + (s * XU + c) * xbytes, &tm_x, (xi * XU + c) * kBK, m0, B.x_full + 8 * s);
                    ++gx;
                    if (++s == NSX) s = 0;
                }
            }
            for (int s2 = 0; s2 < NSX && s2 < gx; ++s2) {
                const int last = s2 + ((gx - 1 - s2) / NSX) * NSX;
                volatile int never = 0;
                tc::bar_wait(B.x_full + 8 * s2, (last / NSX) & 1, &never, p.status);
            }
        }
        __syncwarp();
    } else if (warp == 2 || warp == 3) {
        // ---------------- MMA issuers: warp 2 tile 0, warp 3 tile 1 ----------------
        // Each issuer waits only for its own tile's A slot and commits to its own tile's
        // mma_done ring, so the two tiles' pipelines need not wait for each other.
        const int t = warp - 2;
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_f16_f32(kBM, p.BN);
            const uint32_t d_acc = tmem + static_cast<uint32_t>(t * p.acc_stride);
            int xs = 0, xc = 0;                 // activation stage and chunk within it
            uint32_t xph = 0;
            int sa = 0;                         // A slot of the next unit and its phase bit
            uint32_t aph = 0;
            bool ok = true;
            int g = 0;                          // units committed so far (all segments)
            int seg_i = 0;
            SegWalk walk(p, nst);
            Seg sg;
            while (ok && walk.next(p, KU, sg)) {
                // the previous segment's epilogue has read the accumulators
                if (seg_i > 0 && !tc::bar_wait(B.acc_full, (seg_i - 1) & 1, abort, p.status, p.wait_ns)) {
                    ok = false;
                    break;
                }
                const int nu = (sg.k1 - sg.k0) * KU;
                for (int u = 0; u < nu; ++u) {
                    if (!tc::bar_wait(B.a_full + 8 * (kRT * sa + t), aph, abort, p.status, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    if (xc == 0 && !tc::bar_wait(B.x_full + 8 * xs, xph, abort, p.status, p.wait_ns)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t a_tm = tmem + static_cast<uint32_t>(p.a_col0 + (sa * kRT + t) * 32);
                    const uint64_t bd = tc::desc_k_sw128(sX + static_cast<uint32_t>(xs * XU + xc) * xbytes);
                    issue_ksteps<1>(d_acc, a_tm, bd, idesc, 0, u == 0);
                    if (++xc == XU) {
                        xc = 0;
                        if (++xs == NSX) { xs = 0; xph ^= 1; }
                    }
                    tc::mma_commit(B.mma_done + 8 * (kRT * (g % kDoneRing2) + t));
                    ++g;
                    if (++sa == NSLOT) { sa = 0; aph ^= 1; }
                }
                ++seg_i;
            }
            volatile int never = 0;
            if (!ok) {
                tc::mma_commit(B.drain + 8 * t);
                tc::bar_wait(B.drain + 8 * t, 0, &never, p.status);
            }
            // every commit arrival lands before the CTA exits
            for (int c = g - kDoneRing2 > 0 ? g - kDoneRing2 : 0; c < g; ++c)
                tc::bar_wait(B.mma_done + 8 * (kRT * (c % kDoneRing2) + t), (c / kDoneRing2) & 1, &never, p.status);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 12) {
        // ---------------- dequantisation into TMEM, one chunk (unit) at a time; epilogues ----------------
        const int sw = row & 7;
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(lq * 32) << 16);
        const uint32_t taddr = t_lane + static_cast<uint32_t>(tt * p.acc_stride);
        const int et = (warp - 4) * 32 + lane;
        bool ok = true;
        int s = 0;
        uint32_t cph = 0;
        int dq_slot = 0;                   // A slot of the next unit
        int g = 0;                         // units dequantised so far (all segments)
        int seg_i = 0;
        bool pdl_done = false;
        SegWalk walk(p, nst);
        Seg sg;
        while (walk.next(p, KU, sg)) {
            for (int st = sg.k0; st < sg.k1 && ok; ++st) {
                if (!tc::bar_wait(B.codes_full + 8 * s, cph, abort, p.status, p.wait_ns)) { ok = false; break; }
                const uint32_t crow = sC + s * CSTAGE + row * 128;
                uint4 cw[KU][WPC];
#pragma unroll
                for (int c = 0; c < KU; ++c)
#pragma unroll
                    for (int v = 0; v < WPC; ++v) cw[c][v] = tc::lds128(crow + (((c * WPC + v) ^ sw) << 4));
                const uint4 mrow = tc::lds128(sM + s * MSTAGE + row * 16);
                const int moff = (st * KU) & (kMetaChunks - 1);
                // the step's groups, decoded together before the first unit
                DqConst kc[KU];
#pragma unroll
                for (int c = 0; c < KU; ++c) {
                    const int mi = (moff + c) & 3;
                    kc[c] = dq_const(mi == 0 ? mrow.x : (mi == 1 ? mrow.y : (mi == 2 ? mrow.z : mrow.w)));
                }
#pragma unroll
                for (int c = 0; c < KU; ++c) {
                    const int u = g;
                    const int sa = dq_slot;
                    if (++dq_slot == NSLOT) dq_slot = 0;
                    if (u >= NSLOT) {
                        const int pu = u - NSLOT;
                        if (!tc::bar_wait(B.mma_done + 8 * (kRT * (pu % kDoneRing2) + tt), (pu / kDoneRing2) & 1,
                                          abort, p.status, p.wait_ns)) {
                            ok = false;
                            break;
                        }
                        tc::fence_after_sync();
                    }
                    const uint32_t step2 = kc[c].step2, mnv2 = kc[c].mn2;
                    const uint32_t a_col = p.a_col0 + (sa * kRT + tt) * 32;
                    // the whole chunk (64 values, 32 columns) goes to TMEM in one store: a
                    // tcgen05.st costs about as much issue time as two of half the width
                    uint32_t r32[32];
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {          // two halves of the chunk: 32 values each
                        uint32_t (&r)[16] = *reinterpret_cast<uint32_t (*)[16]>(&r32[16 * hh]);
                        if (BITS == 4) {
                            const uint4 q = cw[c][hh];
                            const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const uint4 v = XPERM ? dequant8_4bit_il(w[j], kc[c]) : dequant8_4bit(w[j], kc[c]);
                                r[4 * j] = v.x;
                                r[4 * j + 1] = v.y;
                                r[4 * j + 2] = v.z;
                                r[4 * j + 3] = v.w;
                            }
                        } else {
                            const uint4 q0 = cw[c][2 * hh], q1 = cw[c][2 * hh + 1];
                            const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                uint4 v;
                                if (XPERM) {
                                    v = dequant8_8bit_il(w[2 * j], w[2 * j + 1], step2, mnv2);
                                } else {
                                    const uint2 a = dequant4_8bit(w[2 * j], step2, mnv2);
                                    const uint2 b = dequant4_8bit(w[2 * j + 1], step2, mnv2);
                                    v = make_uint4(a.x, a.y, b.x, b.y);
                                }
                                r[4 * j] = v.x;
                                r[4 * j + 1] = v.y;
                                r[4 * j + 2] = v.z;
                                r[4 * j + 3] = v.w;
                            }
                        }
                    }
                    tc::tmem_st32(t_lane + a_col, r32);
                    tc::tmem_wait_st();
                    tc::fence_before_sync();
                    tc::bar_arrive(B.a_full + 8 * (kRT * sa + tt));
                    ++g;
                }
                if (!ok) break;
                // every value of the code stage has been used: the next TMA may refill it
                tc::bar_arrive(B.codes_empty + 8 * s);
                if (++s == NSC) { s = 0; cph ^= 1; }
            }

            // ---------------- epilogue of this segment ----------------
            const int n0 = sg.tn * kRows2, m0 = sg.tm * p.BN;
            const int n = n0 + row;
            const int n0t = n0 + tt * kBM;                            // first row of this thread's tile
            const float scale_n = n < p.nq ? p.qscale : 1.f;
            const int n_out = p.yperm ? ((n & ~7) | ((n & 3) << 1) | ((n >> 2) & 1)) : n;
            const bool kv_on = p.kv.codes[0][0] != nullptr && n0t >= p.kv.h;
            if (!pdl_done) {
                pdl_wait();
                pdl_trigger();
                pdl_done = true;
            }
            const float bias_n = p.bias ? __half2float(p.bias[n]) : 0.f;
            auto finish8 = [&](int col, const float (&v)[8]) {
                float r[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int m = m0 + col + j;
                    r[j] = (p.residual && m < p.M) ? __half2float(p.residual[static_cast<int64_t>(m) * p.N + n]) : 0.f;
                }
                __half o16[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int m = m0 + col + j;
                    float x = (v[j] + bias_n) * scale_n;
                    if (p.relu) x = fmaxf(x, 0.f);
                    o16[j] = __float2half_rn(x + r[j]);
                    if (m < p.M) p.y[static_cast<int64_t>(m) * p.N + n_out] = o16[j];
                }
                if (kv_on) kv_store8(p, o16, col, m0, n0t, n, warp, lane, kv_red);
            };
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (ok && !*abort && g > 0) {
                const int gl = g - 1;                                 // the segment's last unit: both tiles' MMAs done
                const uint32_t md = B.mma_done + 8 * (kRT * (gl % kDoneRing2));
                ok = tc::bar_wait(md, (gl / kDoneRing2) & 1, abort, p.status) &&
                     tc::bar_wait(md + 8, (gl / kDoneRing2) & 1, abort, p.status);
            }
            asm volatile(
                "{\n\t.reg .pred p, q;\n\t"
                "setp.ne.u32 p, %1, 0;\n\t"
                "barrier.cta.red.and.pred q, 1, 256, p;\n\t"
                "selp.u32 %0, 1, 0, q;\n\t}"
                : "=r"(all_ok)
                : "r"((ok && !*abort) ? 1u : 0u)
                : "memory");
            if (all_ok) tc::fence_after_sync();
            const int64_t pstride = static_cast<int64_t>(p.BN) * kRows2;     // floats per partial

            // Sum, for every 8-column group of `row`, of `own` (this CTA's accumulator, when
            // set) and the partial blocks src[0..np) in that order, handed to finish8. The
            // blocks pass through the drained rings in batches of C column groups, bulk-
            // loaded into two alternating halves. Returns false if a wait gave up.
            auto reduce_blocks = [&](const float* const* src, int np, bool own) -> bool {
                const int ng = p.BN / 8;
                const uint32_t half = (p.off_bar / 2) & ~15u;
                int C = static_cast<int>(half / (static_cast<uint32_t>(np) * kRows2 * 32));
                if (C > ng) C = ng;
                const int nb = (ng + C - 1) / C;
                auto issue = [&](int bi) {
                    const int g0 = bi * C, gc = min(C, ng - g0);
                    const uint32_t dst = base + (bi & 1) * half;
                    const uint32_t bytes = static_cast<uint32_t>(gc) * kRows2 * 32;
                    tc::bar_arrive_expect_tx(B.red + 8 * (bi & 1), bytes * np);
                    for (int sp = 0; sp < np; ++sp)
                        tc::bulk_load(dst + sp * static_cast<uint32_t>(C) * kRows2 * 32,
                                      src[sp] + static_cast<int64_t>(g0) * kRows2 * 8, bytes, B.red + 8 * (bi & 1));
                };
                if (et == 0) {
                    tc::fence_proxy_async_global();
                    issue(0);
                    if (nb > 1) issue(1);
                }
                int waited = 0;
                bool rok = true;
                for (int bi = 0; bi < nb; ++bi) {
                    const bool w = tc::bar_wait(B.red + 8 * (bi & 1), (bi >> 1) & 1, abort, p.status, p.wait_ns);
                    uint32_t wall;                                    // one decision for the 256 threads
                    asm volatile(
                        "{\n\t.reg .pred p, q;\n\t"
                        "setp.ne.u32 p, %1, 0;\n\t"
                        "barrier.cta.red.and.pred q, 1, 256, p;\n\t"
                        "selp.u32 %0, 1, 0, q;\n\t}"
                        : "=r"(wall)
                        : "r"(w ? 1u : 0u)
                        : "memory");
                    if (!wall) {
                        rok = false;
                        break;
                    }
                    waited = bi + 1;
                    const uint32_t sbuf = base + (bi & 1) * half;
                    const int g0 = bi * C, gc = min(C, ng - g0);
                    for (int gi = 0; gi < gc; ++gi) {
                        float acc[8];
                        if (own) {
                            tc::tmem_ld8(taddr + (g0 + gi) * 8, acc);
                        } else {
#pragma unroll
                            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
                        }
                        for (int sp = 0; sp < np; ++sp) {                 // block order
                            const uint32_t q = sbuf + ((sp * C + gi) * kRows2 + row) * 32;
                            const float4 lo = tc::lds128f(q), hi = tc::lds128f(q + 16);
                            acc[0] += lo.x;
                            acc[1] += lo.y;
                            acc[2] += lo.z;
                            acc[3] += lo.w;
                            acc[4] += hi.x;
                            acc[5] += hi.y;
                            acc[6] += hi.z;
                            acc[7] += hi.w;
                        }
                        finish8((g0 + gi) * 8, acc);
                    }
                    asm volatile("bar.sync 1, 256;" ::: "memory");       // this half is free again
                    if (et == 0 && bi + 2 < nb) issue(bi + 2);
                }
                // a wait that gave up: the copies already issued land before the CTA exits
                const int issued = rok ? nb : min(nb, waited + 2);
                for (int bi = waited; bi < issued; ++bi) {
                    volatile int never = 0;
                    tc::bar_wait(B.red + 8 * (bi & 1), (bi >> 1) & 1, &never, p.status);
                }
                return rok;
            };

            if (p.sk) {
                // (every CTA keeps the flag protocol even after a wait gave up, so the flags
                // are back at zero when the kernel ends; the data is then unspecified)
                if (sg.whole) {
                    if (all_ok)
                        for (int col = 0; col < p.BN; col += 8) {
                            float v[8];
                            tc::tmem_ld8(taddr + col, v);
                            finish8(col, v);
                        }
                } else if (!sg.owner) {
                    // a later piece of a shared tile (this CTA's first segment): partial to this
                    // CTA's slot, then published (the rings still feed the next segment, so the
                    // partial goes straight from the accumulator to the workspace)
                    if (all_ok) {
                        float* mine = p.part + static_cast<int64_t>(blockIdx.x) * pstride;
                        for (int col = 0; col < p.BN; col += 8) {
                            float v[8];
                            tc::tmem_ld8(taddr + col, v);
                            part_store8(mine, kRows2, row, col, v);
                        }
                    }
                    __threadfence();
                    asm volatile("bar.sync 1, 256;" ::: "memory");
                    if (et == 0) atomicExch(p.counters + blockIdx.x, 1);
                } else {
                    // the owner: its accumulator plus the later pieces, CTAs blockIdx.x + 1, ...
                    // up to the tile's last step, in K order
                    const int64_t tile_end = (static_cast<int64_t>(sg.tm) * p.sk_tiles_n + sg.tn + 1) * nst;
                    const float* srcs[kMaxPieces];
                    int np = 0;
                    for (int c2 = blockIdx.x + 1; c2 < static_cast<int>(gridDim.x) && np < kMaxPieces; ++c2) {
                        if (static_cast<int64_t>(c2) * p.sk_total / gridDim.x >= tile_end) break;
                        srcs[np++] = p.part + static_cast<int64_t>(c2) * pstride;
                    }
                    // wait until every piece is published (its CTA started earlier in K order
                    // and runs on another SM; the wait is bounded all the same)
                    bool pub = true;
                    if (et == 0) {
                        const uint64_t t0 = tc::globaltimer_ns();
                        for (int i = 0; i < np && pub; ++i) {
                            volatile int* f = p.counters + blockIdx.x + 1 + i;
                            while (*f == 0) {
                                if (tc::globaltimer_ns() - t0 > p.wait_ns) {     // (peers publish even after an abort)
                                    *abort = 1;
                                    set_status(p.status, FLEX_ERR_TIMEOUT);
                                    pub = false;
                                    break;
                                }
                                __nanosleep(256);
                            }
                        }
                        __threadfence();
                    }
                    uint32_t pall;
                    asm volatile(
                        "{\n\t.reg .pred p, q;\n\t"
                        "setp.ne.u32 p, %1, 0;\n\t"
                        "barrier.cta.red.and.pred q, 1, 256, p;\n\t"
                        "selp.u32 %0, 1, 0, q;\n\t}"
                        : "=r"(pall)
                        : "r"((pub && all_ok) ? 1u : 0u)
                        : "memory");
                    if (pall && stage_ok && (p.off_bar / 2) >= static_cast<uint32_t>(np) * kRows2 * 32) {
                        __threadfence();
                        reduce_blocks(srcs, np, true);
                    } else if (pall) {
                        __threadfence();
                        for (int col = 0; col < p.BN; col += 8) {
                            float acc[8];
                            tc::tmem_ld8(taddr + col, acc);
                            for (int i = 0; i < np; ++i) {
                                const float4* q = reinterpret_cast<const float4*>(
                                    srcs[i] + (static_cast<int64_t>(col >> 3) * kRows2 + row) * 8);
                                const float4 lo = __ldcg(q), hi = __ldcg(q + 1);
                                acc[0] += lo.x;
                                acc[1] += lo.y;
                                acc[2] += lo.z;
                                acc[3] += lo.w;
                                acc[4] += hi.x;
                                acc[5] += hi.y;
                                acc[6] += hi.z;
                                acc[7] += hi.w;
                            }
                            finish8(col, acc);
                        }
                    }
                    asm volatile("bar.sync 1, 256;" ::: "memory");
                    if (et == 0)
                        for (int i = 0; i < np; ++i) p.counters[blockIdx.x + 1 + i] = 0;   // ready for the next call
                }
            } else if (all_ok) {
                if (p.splits == 1) {
                    for (int col = 0; col < p.BN; col += 8) {
                        float v[8];
                        tc::tmem_ld8(taddr + col, v);
                        finish8(col, v);
                    }
                } else if (p.cluster) {
                    // this split's fp32 partial [BN][256] into this CTA's shared memory (the rings
                    // are drained: every copy has landed and every MMA has completed)
                    for (int col = 0; col < p.BN; col += 8) {
                        float v[8];
                        tc::tmem_ld8(taddr + col, v);
#pragma unroll
                        for (int j = 0; j < 8; ++j) tc::st_shared_f32(base + ((col + j) * kRows2 + row) * 4, v[j]);
                    }
                } else if (p.xchg) {
                    // the column groups other splits finish (v % splits != this split), in
                    // workspace layout, packed into the drained rings for the bulk stores below
                    int j = 0;
                    for (int v = 0; v < p.BN / 8; ++v) {
                        if (v % p.splits == static_cast<int>(blockIdx.z)) continue;
                        float x8[8];
                        tc::tmem_ld8(taddr + v * 8, x8);
                        const uint32_t sa = base + (j * kRows2 + row) * 32;
                        tc::sts128(sa, x8[0], x8[1], x8[2], x8[3]);
                        tc::sts128(sa + 16, x8[4], x8[5], x8[6], x8[7]);
                        ++j;
                    }
                    tc::fence_proxy_async_smem();
                } else if (stage_ok) {
                    // the partial, in its workspace layout, into the drained rings; one bulk
                    // store (issued with the ticket below) moves it to the workspace
                    for (int col = 0; col < p.BN; col += 8) {
                        float v[8];
                        tc::tmem_ld8(taddr + col, v);
                        const uint32_t sa = base + ((col >> 3) * kRows2 + row) * 32;
                        tc::sts128(sa, v[0], v[1], v[2], v[3]);
                        tc::sts128(sa + 16, v[4], v[5], v[6], v[7]);
                    }
                    tc::fence_proxy_async_smem();
                } else {
                    float* mine = p.part + (static_cast<int64_t>(blockIdx.y * gridDim.x + blockIdx.x) * p.splits +
                                            blockIdx.z) * pstride;
                    for (int col = 0; col < p.BN; col += 8) {
                        float v[8];
                        tc::tmem_ld8(taddr + col, v);
                        part_store8(mine, kRows2, row, col, v);
                    }
                }
            }
            if (!p.sk && p.splits > 1 && !p.cluster && p.xchg) {
                // Exchange (all of the grid is resident at once: one wave, one CTA per SM):
                // split z finishes the column groups v with v % S == z. Each split publishes
                // the groups the others finish, waits for the others' copies of its own
                // groups and adds all splits in split order (its own from TMEM). A split that
                // gave up still publishes and counts itself done, so nobody waits for it.
                const int tile = blockIdx.y * gridDim.x + blockIdx.x;
                const int S = p.splits, z = blockIdx.z, ng = p.BN / 8;
                const int nown = (ng - z + S - 1) / S;                // groups z, z + S, ...
                const int nmax = (ng + S - 1) / S;                    // slots per peer in the load area
                int* flags = p.counters + tile * S;
                int* done = p.counters + gridDim.x * gridDim.y * S + tile;
                float* mine = p.part + (static_cast<int64_t>(tile) * S + z) * pstride;
                asm volatile("bar.sync 1, 256;" ::: "memory");
                if (et == 0) {
                    if (all_ok) {
                        int j = 0;
                        for (int v = 0; v < ng; ++v) {
                            if (v % S == z) continue;
                            tc::bulk_store(mine + static_cast<int64_t>(v) * kRows2 * 8, base + j * kRows2 * 32,
                                           kRows2 * 32);
                            ++j;
                        }
                        tc::bulk_commit();
                        tc::bulk_wait_all();
                        tc::fence_proxy_async_global();
                    }
                    __threadfence();
                    atomicExch(flags + z, 1);
                }
                bool pub = true;
                if (et == 0) {
                    const uint64_t t0 = tc::globaltimer_ns();
                    for (int s2 = 0; s2 < S && pub; ++s2) {
                        if (s2 == z) continue;
                        volatile int* f = flags + s2;
                        while (*f == 0) {
                            if (tc::globaltimer_ns() - t0 > p.wait_ns) {         // (peers publish even after an abort)
                                *abort = 1;
                                set_status(p.status, FLEX_ERR_TIMEOUT);
                                pub = false;
                                break;
                            }
                            __nanosleep(128);
                        }
                    }
                    __threadfence();
                }
                uint32_t pall;
                asm volatile(
                    "{\n\t.reg .pred p, q;\n\t"
                    "setp.ne.u32 p, %1, 0;\n\t"
                    "barrier.cta.red.and.pred q, 1, 256, p;\n\t"
                    "selp.u32 %0, 1, 0, q;\n\t}"
                    : "=r"(pall)
                    : "r"((pub && all_ok) ? 1u : 0u)
                    : "memory");
                if (pall && nown > 0) {
                    // the peers' copies of this split's groups: peer slot k (peers in split
                    // order, skipping z), group i at base + (k nmax + i) 8 KB
                    if (et == 0) {
                        tc::fence_proxy_async_global();
                        tc::bar_arrive_expect_tx(B.red, static_cast<uint32_t>((S - 1) * nown) * kRows2 * 32);
                        int k = 0;
                        for (int s2 = 0; s2 < S; ++s2) {
                            if (s2 == z) continue;
                            const float* peer = p.part + (static_cast<int64_t>(tile) * S + s2) * pstride;
                            for (int i = 0; i < nown; ++i)
                                tc::bulk_load(base + (k * nmax + i) * kRows2 * 32,
                                              peer + static_cast<int64_t>(z + i * S) * kRows2 * 8, kRows2 * 32, B.red);
                            ++k;
                        }
                    }
                    const bool w = tc::bar_wait(B.red, 0, abort, p.status, p.wait_ns);
                    uint32_t wall;
                    asm volatile(
                        "{\n\t.reg .pred p, q;\n\t"
                        "setp.ne.u32 p, %1, 0;\n\t"
                        "barrier.cta.red.and.pred q, 1, 256, p;\n\t"
                        "selp.u32 %0, 1, 0, q;\n\t}"
                        : "=r"(wall)
                        : "r"(w ? 1u : 0u)
                        : "memory");
                    if (wall) {
                        for (int i = 0; i < nown; ++i) {
                            const int v = z + i * S;
                            float acc[8];
#pragma unroll
                            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
                            int k = 0;
                            for (int s2 = 0; s2 < S; ++s2) {              // split order
                                float t8[8];
                                if (s2 == z) {
                                    tc::tmem_ld8(taddr + v * 8, t8);
                                } else {
                                    const uint32_t q = base + ((k * nmax + i) * kRows2 + row) * 32;
                                    const float4 lo = tc::lds128f(q), hi = tc::lds128f(q + 16);
                                    t8[0] = lo.x; t8[1] = lo.y; t8[2] = lo.z; t8[3] = lo.w;
                                    t8[4] = hi.x; t8[5] = hi.y; t8[6] = hi.z; t8[7] = hi.w;
                                    ++k;
                                }
#pragma unroll
                                for (int j = 0; j < 8; ++j) acc[j] += t8[j];
                            }
                            finish8(v * 8, acc);
                        }
                    } else {
                        volatile int never = 0;                         // the copies land before exit
                        tc::bar_wait(B.red, 0, &never, p.status);
                    }
                }
                asm volatile("bar.sync 1, 256;" ::: "memory");
                if (et == 0 && atomicAdd(done, 1) == S - 1) {            // the last split out resets
                    for (int s2 = 0; s2 < S; ++s2) flags[s2] = 0;
                    *done = 0;
                }
            } else if (!p.sk && p.splits > 1 && !p.cluster) {
                // ticket, taken by every split (see gemm_tc_kernel); the last adds the partials in split order
                const int tile = blockIdx.y * gridDim.x + blockIdx.x;
                __threadfence();
                asm volatile("bar.sync 1, 256;" ::: "memory");
                if (et == 0) {
                    if (all_ok && stage_ok) {
                        tc::bulk_store(p.part + (static_cast<int64_t>(tile) * p.splits + blockIdx.z) * pstride, base,
                                       static_cast<uint32_t>(pstride * 4));
                        tc::bulk_commit();
                        tc::bulk_wait_all();
                        tc::fence_proxy_async_global();
                        __threadfence();
                    }
                    *last_flag = (atomicAdd(p.counters + tile, 1) == p.splits - 1);
                }
                asm volatile("bar.sync 1, 256;" ::: "memory");
                if (*last_flag) {
                    __threadfence();
                    const float* all = p.part + static_cast<int64_t>(tile) * p.splits * pstride;
                    if (all_ok && stage_ok && (p.off_bar / 2) >= static_cast<uint32_t>(p.splits) * kRows2 * 32) {
                        const float* srcs[kMaxSplits];
                        for (int sp = 0; sp < p.splits; ++sp) srcs[sp] = all + sp * pstride;
                        reduce_blocks(srcs, p.splits, false);
                    } else if (all_ok) {
                        part_reduce(all, pstride, p.splits, kRows2, row, 0, p.BN,
                                    [&](int col, const float (&acc)[8]) { finish8(col, acc); });
                    }
                    if (et == 0) p.counters[tile] = 0;
                }
            }
            // the accumulators are free for the next segment's MMAs
            tc::fence_before_sync();
            tc::bar_arrive(B.acc_full);
            ++seg_i;
            if (!all_ok) break;
        }
        (void)seg_i;
    }

    if (!p.sk && p.splits > 1 && p.cluster) {
        // split-K across the cluster: CTA r finishes the 8-column groups v = r, r + S, ...
        // of every row, adding the splits' partials in split order; the second barrier keeps
        // each CTA's shared memory alive until its peers are done. All threads of every CTA
        // take part in both barriers.
        tc::cluster_sync();
        if (warp >= 4 && warp < 12 && all_ok) {
            const int S = p.splits;
            const int rank = static_cast<int>(tc::cluster_rank());
            const int n = blockIdx.x * kRows2 + row;
            const int n0t = blockIdx.x * kRows2 + tt * kBM;
            const int m0 = blockIdx.y * p.BN;
            const float scale_n = n < p.nq ? p.qscale : 1.f;
            const int n_out = p.yperm ? ((n & ~7) | ((n & 3) << 1) | ((n >> 2) & 1)) : n;
            const bool kv_on = p.kv.codes[0][0] != nullptr && n0t >= p.kv.h;
            const float bias_n = p.bias ? __half2float(p.bias[n]) : 0.f;
            for (int v = rank; v < p.BN / 8; v += S) {
                const int col = v * 8;
                float acc[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = 0.f;
                for (int sp = 0; sp < S; ++sp) {
                    const uint32_t peer = tc::map_peer(base + (col * kRows2 + row) * 4, static_cast<uint32_t>(sp));
                    float tv[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) tv[j] = tc::ld_peer_f32(peer + j * kRows2 * 4);
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[j] += tv[j];
                }
                float r[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int m = m0 + col + j;
                    r[j] = (p.residual && m < p.M) ? __half2float(p.residual[static_cast<int64_t>(m) * p.N + n]) : 0.f;
                }
                __half o16[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int m = m0 + col + j;
                    float x = (acc[j] + bias_n) * scale_n;
                    if (p.relu) x = fmaxf(x, 0.f);
                    o16[j] = __float2half_rn(x + r[j]);
                    if (m < p.M) p.y[static_cast<int64_t>(m) * p.N + n_out] = o16[j];
                }
                if (kv_on) kv_store8(p, o16, col, m0, n0t, n, warp, lane, kv_red);
            }
        }
        tc::cluster_sync();
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 2) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------------------
// Small-batch path (up to 32 activation rows, 4-bit weights): dequant-fused GEMV on
// mma.sync m16n8k16.
//
// A CTA owns kGvRows = 64 weight rows and a range of K groups (all of K, or 1/splits of
// it). Its warps form a kGvRowWarps x kGvKq grid: warp (rb, kq) owns kGvMt m16 tiles of
// rows (16 kGvMt rows from 16 kGvMt rb; the tiles share each activation fragment) and the
// kq-th share of the 8 code words of every group, so each warp's dependent chain per
// stage is 8/kGvKq words long and the SM holds enough warps to hide the latencies. The
// group's codes, metadata and activation slice pass through a kGvStages-deep cp.async
// ring in shared memory, so several groups are always in flight. A warp turns each
// 32-bit word of codes into 4 fp16 pairs in registers (lop3, hsub2, hfma2; the pairs come out in the order (e0,e4)
// (e1,e5) (e2,e6) (e3,e7)) and uses them directly as A fragments - thread (g, t) holds
// K positions [16t, 16t+16) of rows g and g+8 - with the activations of the same K
// positions as B fragments (an interleaved activation row gives them as plain 16-byte
// loads). No single issuing thread and no staging of dequantised weights.
// The kGvKq partial tiles of a CTA are added in shared memory. With K splits each split
// writes its partial tile to the workspace and the last split of a tile to finish
// (atomic ticket) adds them in split order, so results do not depend on scheduling. The epilogue is the GEMM's (bias, q-scale, ReLU, residual,
// interleaved output, fused store_cache).
constexpr int kGvMt = 1;                   // m16 row tiles per warp (they share the B fragments)
constexpr int kGvRowWarps = 4 / kGvMt;     // warps across the rows (16 kGvMt rows each)
constexpr int kGvKq = 4;                   // warps across the 8 code words of a group
constexpr int kGvWords = 8 / kGvKq;        // code words per warp per group
constexpr int kGvThreads = kGvRowWarps * kGvKq * 32;
constexpr int kGvCtasPerSm = 1;
constexpr int kGvRows = 16 * kGvMt * kGvRowWarps;  // 64 weight rows per CTA
static_assert(kGvRows == 64, "the epilogue and the fused store_cache assume 64-row tiles");
constexpr int kGvStages = 5;               // ring of stages of 4 groups (256 K)
static_assert(8 * 32 <= kGvThreads, "every epilogue item (activation row, 8 rows) has its own thread");

struct GemvParams {
    const uint8_t* codes;                  // [N][K/2]
    const uint32_t* meta;                  // [N][K/64] half2 {min, scale}
    const __half* x;                       // [M][K]
    const __half* bias;
    const __half* residual;
    __half* y;
    float* part;                           // split partials [tiles][splits][kGvRows][32]
    int* counters;                         // [tiles] tickets
    int M, N, K, splits, gps;              // gps: groups per split
    int nq;
    float qscale;
    int relu, yperm, xperm, early_w;
    int cluster;                           // K splits reduced inside a thread-block cluster
    KvTarget kv;                           // fused store_cache, as in GemmParams
};

__device__ __forceinline__ void hmma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void gv_cp16(uint32_t dst, const void* src, bool pred) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(pred ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void gv_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void gv_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(kGvStages - 2) : "memory");
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds128v(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

// Epilogue of the small-batch path for activation row m and weight rows n0 + 8c .. +7:
// bias, q-scale, ReLU, residual, fp16 store (interleaved 8-block order when yperm) and
// the fused store_cache. The 8 lanes sharing m are consecutive (item = 8 m + c); rows
// past M return without touching anything. bv / rv are the 8 bias and residual values,
// loaded by the caller ahead of time (zeros where there are none).
__device__ __forceinline__ void gemv_finish(const GemvParams& p, int n0, int c, int m, int lane, const float (&v)[8],
                                            const uint4 bv, const uint4 rv) {
    const bool valid = m < p.M;
    const int nb = n0 + 8 * c;
    __half o16[8];
    if (valid) {
        const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w}, rw[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float bi = (i & 1) ? h2f_hi(bw[i >> 1]) : h2f_lo(bw[i >> 1]);
            const float ri = (i & 1) ? h2f_hi(rw[i >> 1]) : h2f_lo(rw[i >> 1]);
            float xo = (v[i] + bi) * (nb + i < p.nq ? p.qscale : 1.f);
            if (p.relu) xo = fmaxf(xo, 0.f);
            o16[i] = __float2half_rn(xo + ri);
        }
        // interleaved output: element k of the 8-block goes to position 2(k%4) + (k/4)%2
        __half op[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) op[p.yperm ? (2 * (i & 3) + ((i >> 2) & 1)) : i] = o16[i];
        *reinterpret_cast<uint4*>(p.y + static_cast<int64_t>(m) * p.N + nb) =
            make_uint4(pack_half2_bits(op[0], op[1]), pack_half2_bits(op[2], op[3]), pack_half2_bits(op[4], op[5]),
                       pack_half2_bits(op[6], op[7]));
    }
    if (p.kv.codes[0][0] != nullptr && n0 >= p.kv.h && valid) {
        // fused store_cache: the 8 values are dims [dim, dim+8) of one head; a group of gs
        // dims is the gs/8 lanes of consecutive c for this m (all 8 lanes of m are here)
        const uint4 nv = make_uint4(pack_half2_bits(o16[0], o16[1]), pack_half2_bits(o16[2], o16[3]),
                                    pack_half2_bits(o16[4], o16[5]), pack_half2_bits(o16[6], o16[7]));
        const int sec = (n0 - p.kv.h) / p.kv.h;                 // 0 keys, 1 values
        const int f = nb - p.kv.h - sec * p.kv.h;
        const int head = f / p.kv.hd, dim = f % p.kv.hd;
        __half2 mn2, mx2;
        minmax8(nv, mn2, mx2);
        float mn = hmin_of(mn2), mx = hmax_of(mx2);
        const unsigned lanes = 0xFFu << (lane & 24);
        const unsigned gmask = p.kv.gs == 64 ? 7u : 3u;
        for (unsigned off = 1; off <= gmask; off <<= 1) {
            mn = fminf(mn, __shfl_xor_sync(lanes, mn, off));
            mx = fmaxf(mx, __shfl_xor_sync(lanes, mx, off));
        }
        const int c = m / p.kv.rows, r = m - c * p.kv.rows;
        const int b = r / p.kv.seq, tt = r - b * p.kv.seq;
        const int64_t slot = (static_cast<int64_t>(b) * p.kv.nh + head) * p.kv.max_seq + p.kv.pos0 + tt;
        uint8_t* codes = p.kv.codes[c][sec];
        uint32_t* meta = p.kv.meta[c][sec];
        const int gph = p.kv.hd / p.kv.gs;
        if (p.kv.bits == 4) {
            const __half s16 = group_scale16<4>(mn, mx);
            *reinterpret_cast<uint32_t*>(codes + slot * (p.kv.hd / 2) + dim / 2) = quant8_4bit(nv, mn, __half2float(s16));
            if (dim % p.kv.gs == 0) meta[slot * gph + dim / p.kv.gs] = pack_half2_bits(stored_min16(mn), s16);
        } else {
            const __half s16 = group_scale16<8>(mn, mx);
            *reinterpret_cast<uint2*>(codes + slot * p.kv.hd + dim) = quant8_8bit(nv, mn, __half2float(s16));
            if (dim % p.kv.gs == 0) meta[slot * gph + dim / p.kv.gs] = pack_half2_bits(stored_min16(mn), s16);
        }
    }
}

template <int NT>                          // n-tiles of 8 activation rows (M <= 8 NT)
__global__ void __launch_bounds__(kGvThreads, kGvCtasPerSm) gemv_kernel(const GemvParams p) {
    constexpr int MC = 8 * NT;             // activation rows of the tile
    // stage = 4 groups (256 K): codes [64 rows][128 B + 16 pad], metadata [64][4 groups],
    // activations [MC rows][4 groups][128 B + 16 pad] (the pads spread the fragment loads
    // over all banks)
    constexpr int CROW = 128 + 16;
    constexpr int XSEG = 128 + 16;
    constexpr int CODES = kGvRows * CROW;
    constexpr int META = kGvRows * 16;
    constexpr int STAGE = CODES + META + MC * 4 * XSEG;
    extern __shared__ __align__(16) uint8_t gv_smem[];
    __shared__ int last;
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(gv_smem));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int rb = warp % kGvRowWarps, kq = warp / kGvRowWarps;
    const int tile = blockIdx.x, split = blockIdx.y;
    const int n0 = tile * kGvRows;
    const int ngroups = p.K / 64;
    const int gb = split * p.gps;                       // multiple of 4
    const int nst = (min(ngroups, gb + p.gps) - gb) / 4;  // stages of this CTA (> 0)
    const int64_t krow = p.K / 2;                       // code bytes per weight row

    auto load_weights = [&](int i) {       // groups gb + 4i .. +3 into stage i % kGvStages
        const uint32_t st = sbase + (i % kGvStages) * STAGE;
        const int G = gb + 4 * i;
#pragma unroll
        for (int j = 0; j < (kGvRows * 8 + kGvThreads - 1) / kGvThreads; ++j) {
            const int u = threadIdx.x + j * kGvThreads, row = u >> 3, c16 = u & 7;
            if ((kGvRows * 8) % kGvThreads == 0 || u < kGvRows * 8)
                gv_cp16(st + row * CROW + c16 * 16, p.codes + (n0 + row) * krow + G * 32 + c16 * 16, true);
        }
        if (threadIdx.x < kGvRows)
            gv_cp16(st + CODES + threadIdx.x * 16, p.meta + static_cast<int64_t>(n0 + threadIdx.x) * ngroups + G, true);
    };
    auto load_x = [&](int i) {
        const uint32_t st = sbase + (i % kGvStages) * STAGE + CODES + META;
        const int G = gb + 4 * i;
#pragma unroll
        for (int j = 0; j < (MC * 32 + kGvThreads - 1) / kGvThreads; ++j) {
            const int u = threadIdx.x + j * kGvThreads;
            const int m = u >> 5, q = (u >> 3) & 3, c16 = u & 7;
            const bool ok = m < p.M;
            if ((MC * 32) % kGvThreads == 0 || u < MC * 32)
                gv_cp16(st + (m * 4 + q) * XSEG + c16 * 16,
                        p.x + static_cast<int64_t>(ok ? m : 0) * p.K + (G + q) * 64 + c16 * 8, ok);
        }
    };
    // weights do not depend on the previous kernel: inside a layer call their first
    // stages are requested before the programmatic-launch wait
    if (p.early_w) {
#pragma unroll
        for (int i = 0; i < kGvStages - 1; ++i)
            if (i < nst) load_weights(i);
    }
    // this thread's epilogue item, if any: rows n0 + 8 (tid % 8) .. +7 of activation row
    // m_fin (the cluster reduction gives rank r the rows m = r, r + S, ...); its bias
    // (a weight) is fetched now, its residual once the previous kernel has finished
    const int c_fin = threadIdx.x & 7;
    const int m_fin = (p.splits > 1 && p.cluster) ? split + p.splits * (threadIdx.x >> 3) : (threadIdx.x >> 3);
    const bool has_fin = m_fin < p.M && (p.splits > 1 && p.cluster ? true : threadIdx.x < 8 * MC);
    const uint4 bias_v = (has_fin && p.bias) ? __ldg(reinterpret_cast<const uint4*>(p.bias + n0 + 8 * c_fin))
                                             : make_uint4(0u, 0u, 0u, 0u);
    pdl_wait();                            // the activations come from the previous kernel
    pdl_trigger();
    const uint4 res_v = (has_fin && p.residual)
                            ? *reinterpret_cast<const uint4*>(p.residual + static_cast<int64_t>(m_fin) * p.N + n0 + 8 * c_fin)
                            : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int i = 0; i < kGvStages - 1; ++i) {
        if (i < nst) {
            if (!p.early_w) load_weights(i);
            load_x(i);
        }
        gv_commit();
    }

    // two accumulator sets (the two MMAs of every code word go to different sets), so
    // each set's dependent mma.sync chain is half as long
    float acc[kGvMt][NT][4], acc2[kGvMt][NT][4];
#pragma unroll
    for (int mt = 0; mt < kGvMt; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[mt][nt][j] = acc2[mt][nt][j] = 0.f;
    // thread (g, t): rows r0 and r0 + 8 of the tile, group t of every stage, code words
    // [kq kGvWords, (kq + 1) kGvWords) of it (8 K positions each); the MMA's K order is
    // free as long as A and B agree
    const int r0 = 16 * kGvMt * rb + g;       // rows r0 + 16 mt and r0 + 16 mt + 8
    for (int i = 0; i < nst; ++i) {
        // stage i has landed once all but the newest kGvStages - 2 copy groups are done;
        // the barrier publishes it and also tells that every warp has finished stage
        // i - 1, whose slot is refilled right after (one barrier per stage)
        gv_wait();
        __syncthreads();
        if (i + kGvStages - 1 < nst) {
            load_weights(i + kGvStages - 1);
            load_x(i + kGvStages - 1);
        }
        gv_commit();
        const uint32_t st = sbase + (i % kGvStages) * STAGE;
        uint32_t wa[kGvMt][kGvWords], wb[kGvMt][kGvWords];
        DqConst kd[kGvMt][2];
#pragma unroll
        for (int mt = 0; mt < kGvMt; ++mt) {
            const int ra_row = r0 + 16 * mt;
            const uint32_t ra = st + ra_row * CROW + t * 32 + kq * kGvWords * 4, rbb = ra + 8 * CROW;
#pragma unroll
            for (int v = 0; v < kGvWords; v += 4) {
                if (kGvWords >= 4) {
                    const uint4 a = lds128v(ra + 4 * v), b = lds128v(rbb + 4 * v);
                    wa[mt][v] = a.x; wa[mt][v + 1] = a.y; wa[mt][v + 2] = a.z; wa[mt][v + 3] = a.w;
                    wb[mt][v] = b.x; wb[mt][v + 1] = b.y; wb[mt][v + 2] = b.z; wb[mt][v + 3] = b.w;
                }
            }
            if (kGvWords == 2) {
                const uint2 a = lds64(ra), b = lds64(rbb);
                wa[mt][0] = a.x; wa[mt][kGvWords - 1] = a.y; wb[mt][0] = b.x; wb[mt][kGvWords - 1] = b.y;
            }
            if (kGvWords == 1) { wa[mt][0] = lds32(ra); wb[mt][0] = lds32(rbb); }
            const uint32_t mw0 = lds32(st + CODES + ra_row * 16 + t * 4), mw1 = lds32(st + CODES + (ra_row + 8) * 16 + t * 4);
            kd[mt][0] = dq_const(mw0);
            kd[mt][1] = dq_const(mw1);
        }
        const uint32_t xs = st + CODES + META + (g * 4 + t) * XSEG + kq * kGvWords * 16;
#pragma unroll
        for (int w = 0; w < kGvWords; ++w) {
            // K positions 8w .. 8w+7 of group t: A pairs (e0,e4) (e1,e5) (e2,e6) (e3,e7)
            uint4 d0[kGvMt], d1[kGvMt];
#pragma unroll
            for (int mt = 0; mt < kGvMt; ++mt) {
                d0[mt] = dequant8_4bit_il(wa[mt][w], kd[mt][0]);    // row r0 + 16 mt
                d1[mt] = dequant8_4bit_il(wb[mt][w], kd[mt][1]);    // row r0 + 16 mt + 8
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                // activations of row 8 nt + g at the same K positions, as the pairs
                // (k0,k4) (k1,k5) (k2,k6) (k3,k7)
                uint4 xv = lds128v(xs + nt * 8 * 4 * XSEG + w * 16);
                if (!p.xperm)
                    xv = make_uint4(prmt(xv.x, xv.z, 0x5410u), prmt(xv.x, xv.z, 0x7632u), prmt(xv.y, xv.w, 0x5410u),
                                    prmt(xv.y, xv.w, 0x7632u));
#pragma unroll
                for (int mt = 0; mt < kGvMt; ++mt) {
                    hmma16816(acc[mt][nt], d0[mt].x, d1[mt].x, d0[mt].y, d1[mt].y, xv.x, xv.y);
                    hmma16816(acc2[mt][nt], d0[mt].z, d1[mt].z, d0[mt].w, d1[mt].w, xv.z, xv.w);
                }
            }
        }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
    for (int mt = 0; mt < kGvMt; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[mt][nt][j] += acc2[mt][nt][j];

    // ---- the tile (64 rows x MC activation rows) through shared memory: one
    // [64][MC + 1] partial per word share kq, added in kq order
    float* red = reinterpret_cast<float*>(gv_smem);
    constexpr int RED = kGvRows * (MC + 1);
    static_assert(kGvKq * RED * 4 <= STAGE * kGvStages, "reduction tile exceeds the ring");
    __syncthreads();
#pragma unroll
    for (int mt = 0; mt < kGvMt; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                red[kq * RED + (r0 + 16 * mt + 8 * (j >> 1)) * (MC + 1) + 8 * nt + 2 * t + (j & 1)] = acc[mt][nt][j];
    __syncthreads();
    // (activation row m, rows 8c .. 8c+7): 8 MC items
    for (int item = threadIdx.x; item < 8 * MC; item += kGvThreads) {
        const int c = item & 7, m = item >> 3;
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = red[(8 * c + i) * (MC + 1) + m];
#pragma unroll
        for (int q = 1; q < kGvKq; ++q)
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] += red[q * RED + (8 * c + i) * (MC + 1) + m];
        if (p.splits == 1) {
            gemv_finish(p, n0, c, m, lane, v, bias_v, res_v);
        } else if (p.cluster) {
#pragma unroll
            for (int i = 0; i < 8; ++i) red[(8 * c + i) * (MC + 1) + m] = v[i];   // this item's own elements
        } else {
            float* mine = p.part + (static_cast<int64_t>(tile) * p.splits + split) * kGvRows * 32;
#pragma unroll
            for (int i = 0; i < 8; ++i) mine[(8 * c + i) * 32 + m] = v[i];
        }
    }
    if (p.splits == 1) return;
    if (p.cluster) {
        // The K splits of a tile are one cluster (rank = split). After the barrier every
        // split's summed partial tile (the kq = 0 slot of its `red`) is visible; rank r
        // finishes activation rows m = r, r + S, ... adding the partials in split order,
        // and the second barrier keeps every CTA's shared memory alive until its peers
        // are done. Every thread of every CTA takes part in both barriers.
        tc::cluster_sync();
        const int S = p.splits;
        if (has_fin) {
            const int m = m_fin, c = c_fin;
            const uint32_t own = static_cast<uint32_t>(__cvta_generic_to_shared(red + (8 * c) * (MC + 1) + m));
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = 0.f;
            for (int sp0 = 0; sp0 < S; sp0 += 4) {
                float t4[4][8];
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4) {
                    const uint32_t peer = tc::map_peer(own, static_cast<uint32_t>(sp0 + s4 < S ? sp0 + s4 : 0));
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        t4[s4][i] = sp0 + s4 < S ? tc::ld_peer_f32(peer + i * (MC + 1) * 4) : 0.f;
                }
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4)
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[i] += t4[s4][i];
            }
            gemv_finish(p, n0, c, m, lane, v, bias_v, res_v);
        }
        tc::cluster_sync();
        return;
    }
    // ticket: the barrier orders every thread's partial stores before thread 0's fence
    // and atomic (release); the last split's thread 0 fences again before the barrier
    // that lets its CTA read the other splits' partials (acquire)
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        last = (atomicAdd(p.counters + tile, 1) == p.splits - 1);
        if (last) __threadfence();
    }
    __syncthreads();
    if (!last) return;
    const float* all = p.part + static_cast<int64_t>(tile) * p.splits * kGvRows * 32;
    for (int item = threadIdx.x; item < 8 * MC; item += kGvThreads) {
        const int c = item & 7, m = item >> 3;
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.f;
        // four splits' loads in flight at a time, added in split order
        for (int sp0 = 0; sp0 < p.splits; sp0 += 4) {
            float t4[4][8];
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4)
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    t4[s4][i] = sp0 + s4 < p.splits
                                    ? __ldcg(all + (static_cast<int64_t>(sp0 + s4) * kGvRows + 8 * c + i) * 32 + m)
                                    : 0.f;
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4)
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] += t4[s4][i];
        }
        gemv_finish(p, n0, c, m, lane, v, bias_v, res_v);
    }
    if (threadIdx.x == 0) p.counters[tile] = 0;
}

// ---------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// Thread-block clusters of `splits` CTAs of this kernel that can be resident at once on
// the current device (cached per device and size); 0 if the query fails.
int max_active_clusters(int splits, uint32_t smem, bool rows256 = false) {
    static std::map<std::tuple<int, int, uint32_t, bool>, int> cache;
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_tuple(dev, splits, smem, rows256);
    const auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    const void* kfn = rows256 ? reinterpret_cast<const void*>(gemm_tc2_kernel<4, true>)
                              : reinterpret_cast<const void*>(gemm_tc_kernel<4, true>);
    set_smem_once(gemm_tc_kernel<4, true>, 227 * 1024);
    set_smem_once(gemm_tc2_kernel<4, true>, 227 * 1024);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, splits);
    cfg.blockDim = dim3(rows256 ? kThreads2 : kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = splits;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kfn, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    cache[key] = n;
    return n;
}

// K splits per tile: the count whose waves of (tile, split) units take the least time,
// one unit costing its K steps plus a fixed overhead (prologue, pipeline fill, epilogue;
// more when partials must be added). One CTA per SM.
int choose_splits(int tiles, int nk, int bits) {
    const int sms = sm_count();
    int max_splits = nk / kMetaChunks;
    if (max_splits > kMaxSplits) max_splits = kMaxSplits;
    if (max_splits < 1) max_splits = 1;
    const double steps_total = static_cast<double>(nk) / (128 / (kBK * bits / 8));
    int splits = 1;
    double best = 0.0;
    for (int s = 1; s <= max_splits; ++s) {
        if (s > 1 && tiles > static_cast<int>(kTicketBytes / sizeof(int))) break;   // one ticket per tile
        const int64_t units = static_cast<int64_t>(tiles) * s;
        const int64_t waves = (units + sms - 1) / sms;
        const double t = static_cast<double>(waves) * (steps_total / s + (s > 1 ? 5.0 : 3.0));
        if (s == 1 || t < best * 0.97) {
            best = t;
            splits = s;
        }
    }
    return splits;
}

struct Plan2 {
    int BN, tiles_n, tiles_m, splits, cps, nsx, nsc, xu, nslot, acc_stride, a_col0, cluster;
    int sk, grid;                          // stream-K schedule over `grid` CTAs
    int64_t sk_total;
    int xchg;                              // one-wave splits exchange partials (no ticket)
    uint32_t off_c, off_m, off_bar, smem;
    int64_t ws_bytes, counters_bytes;
};

// Stream-K for the 256-row kernel (flex_set_gemm_streamk): on unless switched off.
std::atomic<int> g_streamk{1};

// gemm_tc2_kernel serves weights with N a multiple of 256 (two 128-row tiles per CTA)
// for more than 128 activation rows; its activation tile is at most 192 rows (M <= 192
// in one tile, else tiles of 128). Up to 128 rows the 128-row kernel was faster in every
// weight shape of the OPT-175B layer (its CTAs are half as long, so split-K and the
// waves over 148 SMs come out better).
bool tc2_eligible(int M, int N) {
#ifdef FLEXQ_GEMM_ROWS128_ONLY
    (void)M;
    (void)N;
    return false;
#else
    return M > 128 && N % kRows2 == 0;
#endif
}

Plan2 make_plan2(int M, int N, int K, int bits) {
    Plan2 P{};
    P.BN = M <= 192 ? ((M + 15) / 16) * 16 : 128;
    if (P.BN < 16) P.BN = 16;
    P.tiles_n = N / kRows2;
    P.tiles_m = (M + P.BN - 1) / P.BN;
    const int nk = K / kBK;
    const int tiles = P.tiles_n * P.tiles_m;
    int splits = choose_splits(tiles, nk, bits);
    int cps = (nk + splits - 1) / splits;
    cps = ((cps + kMetaChunks - 1) / kMetaChunks) * kMetaChunks;
    P.splits = (nk + cps - 1) / cps;
    P.cps = cps;
    P.acc_stride = ((P.BN + 31) / 32) * 32;
    P.a_col0 = kRT * P.acc_stride;
    P.nslot = (kTmemCols - P.a_col0) / (kRT * 32);
    // shared memory: code stages (256 rows x 128 B + metadata) and activation stages of
    // XU chunks (BN rows x 128 B each), within about 220 KB
    const int ku = 128 / (kBK * bits / 8);
    const uint32_t cstage = kRows2 * 128 + kRows2 * kMetaChunks * 4;
    int xu = ku;
    while (xu > 1 && static_cast<uint32_t>(xu) * P.BN * 128 > 56u * 1024u) xu >>= 1;
    const uint32_t xstage = static_cast<uint32_t>(xu) * P.BN * 128;
    const uint32_t budget = 220u * 1024u;
    int nsc = 3;
    int nsx = static_cast<int>((budget - nsc * cstage) / xstage);
    if (nsx < 2) {
        nsc = 2;
        nsx = static_cast<int>((budget - nsc * cstage) / xstage);
    }
    if (nsx > 6) nsx = 6;
    P.xu = xu;
    P.nsx = nsx;
    P.nsc = nsc;
    P.off_c = nsx * xstage;
    P.off_m = P.off_c + nsc * kRows2 * 128;
    P.off_bar = P.off_m + nsc * kRows2 * kMetaChunks * 4;
    P.smem = P.off_bar + 8 * (2 * nsc + nsx + kRT * P.nslot + kRT * kDoneRing2 + 1 + 4 + 2) + 16 + 256 + 1024;
    // split-K through distributed shared memory when the partial tile fits in the drained
    // rings and every tile's cluster can be resident at once, else workspace and tickets
    const bool fits = static_cast<uint32_t>(P.BN) * kRows2 * 4 <= P.off_bar;
    P.cluster = (P.splits > 1 && fits && max_active_clusters(P.splits, P.smem, true) >= tiles) ? 1 : 0;
    P.counters_bytes = kTicketBytes;
    P.ws_bytes = (P.splits > 1 && !P.cluster)
                     ? P.counters_bytes + static_cast<int64_t>(tiles) * P.splits * P.BN * kRows2 * 4
                     : 0;
    // Where the split plan would reduce through the workspace in more than one wave of
    // CTAs, a stream-K schedule instead: one CTA per SM, each taking an equal share of all
    // tiles' K steps; a tile is cut only where one CTA's share ends, so at most one partial
    // per CTA crosses the workspace, and the CTAs' fills and epilogues are paid once per CTA,
    // not once per (tile, split). Taken when every CTA gets at least 8 steps and no tile is
    // spread over more than kMaxPieces + 1 CTAs. (With the splits in one wave the ticket
    // plan measured faster: at OPT-175B shapes, 48 tiles x 3 splits, 62 against 72 us.)
    P.sk = 0;
    P.grid = tiles * P.splits;
    P.sk_total = 0;
    // Splits that all run in one wave (one CTA per SM, so every CTA of the grid is resident
    // at once) exchange partials: each split finishes 1/splits of the columns, instead of
    // the last split adding all of them after the others.
    {
        const int ng = P.BN / 8, nmax = (ng + P.splits - 1) / P.splits;
        P.xchg = (P.splits > 1 && !P.cluster && tiles * P.splits <= sm_count() &&
                  static_cast<uint32_t>(P.BN) * kRows2 * 4 <= P.off_bar &&
                  static_cast<uint32_t>((P.splits - 1) * nmax) * kRows2 * 32 <= P.off_bar &&
                  tiles * (P.splits + 1) <= static_cast<int>(kTicketBytes / sizeof(int)))
                     ? 1
                     : 0;
    }
    if (g_streamk.load(std::memory_order_relaxed) && P.splits > 1 && !P.cluster && tiles * P.splits > sm_count()) {
        const int sms = sm_count();
        const int nst = nk / ku;
        const int64_t total = static_cast<int64_t>(tiles) * nst;
        const int64_t qmin = total / sms;
        if (qmin >= 8 && (nst + qmin - 1) / qmin <= kMaxPieces) {
            P.sk = 1;
            P.grid = sms;
            P.sk_total = total;
            P.ws_bytes = P.counters_bytes + static_cast<int64_t>(sms) * P.BN * kRows2 * 4;
        }
    }
    return P;
}

struct Plan {
    int BN, tiles_n, tiles_m, splits, cps, nsx, nsc, xu, nacc, acc_stride, cluster;
    uint32_t off_x, off_c, off_m, off_bar, smem, tmem_cols;
    int64_t ws_bytes, counters_bytes;
};

Plan make_plan(int M, int N, int K, int bits) {
    Plan P{};
    P.BN = M <= 256 ? ((M + 15) / 16) * 16 : 256;
    if (P.BN < 16) P.BN = 16;
    P.tiles_n = N / kBM;
    P.tiles_m = (M + P.BN - 1) / P.BN;
    const int nk = K / kBK;
    const int tiles = P.tiles_n * P.tiles_m;
    int splits = choose_splits(tiles, nk, bits);
    int cps = (nk + splits - 1) / splits;
    cps = ((cps + kMetaChunks - 1) / kMetaChunks) * kMetaChunks;
    splits = (nk + cps - 1) / cps;
    P.splits = splits;
    P.cps = cps;
    // activation stages: a whole step (KU chunks) when it fits in 64 KB, else half a step;
    // up to 128 KB of them, 2..6 deep
    const int ku = 128 / (kBK * bits / 8);
    int xu = ku;
    while (xu > 1 && xu * P.BN * 128 > 64 * 1024) xu >>= 1;
    const uint32_t xstage = static_cast<uint32_t>(xu) * P.BN * 128;
    int nsx = static_cast<int>((128u * 1024u) / xstage);
    if (nsx > 6) nsx = 6;
    if (nsx < 2) nsx = 2;
    P.xu = xu;
    P.nsx = nsx;
    P.nsc = 4;                                    // code stages of 128 rows x 128 B (+ metadata)
    P.off_x = 0;
    P.off_c = nsx * xstage;
    P.off_m = P.off_c + P.nsc * kBM * 128;
    P.off_bar = P.off_m + P.nsc * kBM * kMetaChunks * 4;
    const int nslot = kACols / (ku * 32);
    uint32_t smem = P.off_bar + 8 * (2 * P.nsc + P.nsx + nslot + kDoneRing + 1 + 4) + 16 + 256 + 1024;
    if (smem < 120 * 1024) smem = 120 * 1024;   // at most one CTA per SM: the CTA takes all of TMEM
    P.smem = smem;
    P.tmem_cols = kTmemCols;
    // up to 4 accumulators in TMEM columns [0, 256), 32-column aligned
    P.acc_stride = ((P.BN + 31) / 32) * 32;
    P.nacc = kACol0 / P.acc_stride >= 4 ? 4 : (kACol0 / P.acc_stride >= 2 ? 2 : 1);   // a power of two
    // split-K: through distributed shared memory when every tile's cluster can be
    // resident at once (one wave), else through workspace partials and a ticket
    P.cluster = (splits > 1 && max_active_clusters(splits, P.smem) >= tiles) ? 1 : 0;
    P.counters_bytes = kTicketBytes;
    P.ws_bytes = (splits > 1 && !P.cluster)
                     ? P.counters_bytes + static_cast<int64_t>(tiles) * splits * P.BN * kBM * 4
                     : 0;
    return P;
}

// The register-dequant GEMV serves int4 weights for up to 32 activation rows (one tile
// of n-tiles) unless switched off (flex_set_gemm_gemv); larger batches and prefill go to
// the tcgen05 GEMM.
std::atomic<int> g_gemv{1};
bool gemv_eligible(int M, int N, int bits) {
    return g_gemv.load(std::memory_order_relaxed) && bits == 4 && M >= 1 && M <= 32 && N % kGvRows == 0;
}

struct GemvPlan {
    int nt, tiles, splits, gps, cluster;
    uint32_t smem;
    int64_t ws_bytes, counters_bytes;
};

// Clusters of `splits` GEMV CTAs that can be resident at once (cached per device, size
// and shared memory); 0 if the query fails.
int gemv_max_active_clusters(int splits, uint32_t smem) {
    static std::map<std::tuple<int, int, uint32_t>, int> cache;
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_tuple(dev, splits, smem);
    const auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    set_smem_once(gemv_kernel<4>, static_cast<int>(smem));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, splits, 1);
    cfg.blockDim = dim3(kGvThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = splits;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemv_kernel<4>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    cache[key] = n;
    return n;
}

GemvPlan gemv_plan(int M, int N, int K) {
    GemvPlan P{};
    P.nt = (M + 7) / 8;
    P.tiles = N / kGvRows;
    const int nstages = K / 256;          // stages of 4 groups
    // split K while the grid fits kGvCtasPerSm CTAs per SM and every split keeps >= 2 stages
    int splits = 1;
    while (P.tiles * (splits + 1) <= kGvCtasPerSm * sm_count() && nstages / (splits + 1) >= 2) ++splits;
    const int sps = (nstages + splits - 1) / splits;   // stages per split
    P.gps = 4 * sps;
    P.splits = (nstages + sps - 1) / sps;
    P.smem = static_cast<uint32_t>((kGvRows * 144 + kGvRows * 16 + 8 * P.nt * 4 * 144) * kGvStages);
    // K splits: reduced through distributed shared memory when the splits of every tile
    // fit one portable cluster and all clusters are resident at once, else through
    // workspace partials and a ticket
    P.cluster = (P.splits > 1 && P.splits <= kMaxSplits && gemv_max_active_clusters(P.splits, P.smem) >= P.tiles) ? 1 : 0;
    P.counters_bytes = kTicketBytes;
    P.ws_bytes = (P.splits > 1 && !P.cluster)
                     ? P.counters_bytes + static_cast<int64_t>(P.tiles) * P.splits * kGvRows * 32 * 4
                     : 0;
    return P;
}

}  // namespace

int make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                 uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return FLEX_ERR_CUDA;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FLEX_OK : FLEX_ERR_CUDA;
}

int64_t gemm_ws_bytes(int M, int N, int K, int bits) {
    if (gemv_eligible(M, N, bits)) return gemv_plan(M, N, K).ws_bytes;
    return tc2_eligible(M, N) ? make_plan2(M, N, K, bits).ws_bytes : make_plan(M, N, K, bits).ws_bytes;
}

namespace {
int gemv_launch(const void* x, const flexq_tensor* W, const void* bias, const void* residual, void* y, int M,
                int relu, int nq, float qscale, bool xperm, bool yperm, void* ws, int64_t ws_bytes, cudaStream_t st,
                const KvFuse* kv, bool early_w) {
    const int N = static_cast<int>(W->shape[0]), K = static_cast<int>(W->shape[1]);
    const GemvPlan P = gemv_plan(M, N, K);
    if (P.ws_bytes > 0 && (ws == nullptr || ws_bytes < P.ws_bytes)) return FLEX_ERR_WORKSPACE;
    GemvParams gp{};
    gp.codes = static_cast<const uint8_t*>(W->codes);
    gp.meta = static_cast<const uint32_t*>(W->meta);
    gp.x = static_cast<const __half*>(x);
    gp.bias = static_cast<const __half*>(bias);
    gp.residual = static_cast<const __half*>(residual);
    gp.y = static_cast<__half*>(y);
    gp.counters = static_cast<int*>(ws);
    gp.part = reinterpret_cast<float*>(static_cast<char*>(ws) + P.counters_bytes);
    gp.M = M;
    gp.N = N;
    gp.K = K;
    gp.splits = P.splits;
    gp.gps = P.gps;
    gp.nq = nq;
    gp.qscale = qscale;
    gp.relu = relu;
    gp.yperm = yperm ? 1 : 0;
    gp.xperm = xperm ? 1 : 0;
    gp.early_w = early_w ? 1 : 0;
    gp.cluster = P.cluster;
    fill_kv_target(gp.kv, kv);
    // programmatic dependent launch, and the K splits of a tile as one cluster
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P.tiles, P.splits);
    cfg.blockDim = dim3(kGvThreads);
    cfg.dynamicSmemBytes = P.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = P.splits;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = P.cluster ? 2 : 1;
#define GEMV_LAUNCH(NT_)                                         \
    do {                                                         \
        set_smem_once(gemv_kernel<NT_>, static_cast<int>(P.smem)); \
        cudaLaunchKernelEx(&cfg, gemv_kernel<NT_>, gp);          \
    } while (0)
    switch (P.nt) {
        case 1: GEMV_LAUNCH(1); break;
        case 2: GEMV_LAUNCH(2); break;
        case 3: GEMV_LAUNCH(3); break;
        default: GEMV_LAUNCH(4); break;
    }
#undef GEMV_LAUNCH
    return launch_status();
}
}  // namespace

namespace {
// The 256-row tensor-core GEMM (gemm_tc2_kernel); same arguments as gemm_launch.
int gemm2_launch(const void* x, const flexq_tensor* W, const void* bias, const void* residual, void* y, int M,
                 int relu, int nq, float qscale, bool xperm, bool yperm, void* ws, int64_t ws_bytes, cudaStream_t st,
                 const KvFuse* kv, bool early_w) {
    const int N = static_cast<int>(W->shape[0]), K = static_cast<int>(W->shape[1]);
    const int bits = W->cfg.num_bits;
    const Plan2 P = make_plan2(M, N, K, bits);
    if (P.ws_bytes > 0 && (ws == nullptr || ws_bytes < P.ws_bytes)) return FLEX_ERR_WORKSPACE;
    CUtensorMap tm_codes, tm_meta, tm_x;
    // code tiles: 256 rows x 128 bytes (4 K chunks at 4 bits, 2 at 8 bits), 128-byte swizzle
    int rc = make_tmap_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->codes, static_cast<uint64_t>(K) * bits / 8,
                          N, static_cast<uint64_t>(K) * bits / 8, 128, kRows2, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != FLEX_OK) return rc;
    rc = make_tmap_2d(&tm_meta, CU_TENSOR_MAP_DATA_TYPE_UINT32, W->meta, K / kBK, N,
                      static_cast<uint64_t>(K / kBK) * 4, kMetaChunks, kRows2, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc != FLEX_OK) return rc;
    rc = make_tmap_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, K, M, static_cast<uint64_t>(K) * 2, kBK, P.BN,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != FLEX_OK) return rc;
    GemmParams gp{};
    gp.wait_ns = pipeline_wait_ns();
    gp.gate = reinterpret_cast<const volatile int*>(gemm_gate());
    gp.bias = static_cast<const __half*>(bias);
    gp.residual = static_cast<const __half*>(residual);
    gp.y = static_cast<__half*>(y);
    gp.status = status_word();
    gp.M = M;
    gp.N = N;
    gp.K = K;
    gp.BN = P.BN;
    gp.splits = P.splits;
    gp.cps = P.cps;
    gp.nq = nq;
    gp.qscale = qscale;
    gp.relu = relu;
    gp.early_w = early_w ? 1 : 0;
    gp.yperm = yperm ? 1 : 0;
    gp.nsx = P.nsx;
    gp.nsc = P.nsc;
    gp.xu = P.xu;
    gp.cluster = P.cluster;
    gp.counters = static_cast<int*>(ws);
    gp.part = reinterpret_cast<float*>(static_cast<char*>(ws) + P.counters_bytes);
    gp.nacc = 1;
    gp.acc_stride = P.acc_stride;
    gp.nslot = P.nslot;
    gp.a_col0 = P.a_col0;
    gp.off_x = 0;
    gp.off_c = P.off_c;
    gp.off_m = P.off_m;
    gp.off_bar = P.off_bar;
    gp.tmem_cols = kTmemCols;
    gp.sk = P.sk;
    gp.sk_tiles_n = P.tiles_n;
    gp.sk_total = P.sk_total;
    gp.xchg = P.sk ? 0 : P.xchg;
    fill_kv_target(gp.kv, kv);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = P.sk ? dim3(P.grid, 1, 1) : dim3(P.tiles_n, P.tiles_m, P.splits);
    cfg.blockDim = dim3(kThreads2);
    cfg.dynamicSmemBytes = P.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = P.splits;
    cfg.attrs = attr;
    cfg.numAttrs = P.cluster ? 2 : 1;
#define GEMM2_LAUNCH(B_, XP_)                                                                \
    do {                                                                                     \
        set_smem_once(gemm_tc2_kernel<B_, XP_>, 227 * 1024);                                 \
        cudaLaunchKernelEx(&cfg, gemm_tc2_kernel<B_, XP_>, tm_codes, tm_meta, tm_x, gp);     \
    } while (0)
    if (bits == 4) {
        if (xperm) GEMM2_LAUNCH(4, true); else GEMM2_LAUNCH(4, false);
    } else {
        if (xperm) GEMM2_LAUNCH(8, true); else GEMM2_LAUNCH(8, false);
    }
#undef GEMM2_LAUNCH
    return launch_status();
}
}  // namespace

int validate_weight(const flexq_tensor* W) {
    FLEX_REQUIRE(W != nullptr && W->codes && W->meta, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(W->ndim == 2, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(W->cfg.symmetric == 0, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(W->cfg.num_bits == 4 || W->cfg.num_bits == 8, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(W->cfg.group_size == 64, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(W->cfg.group_dim == 1 || W->cfg.group_dim == -1, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(W->shape[0] > 0 && W->shape[1] > 0, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(W->shape[0] % kBM == 0 && W->shape[1] % 256 == 0, FLEX_ERR_SHAPE);
    FLEX_REQUIRE(W->shape[0] < (1LL << 31) && W->shape[1] < (1LL << 31), FLEX_ERR_SHAPE);
    FLEX_REQUIRE(aligned16(W->codes) && aligned16(W->meta), FLEX_ERR_ALIGN);
    return FLEX_OK;
}

// y = epilogue(x W^T + bias); see flex_dequant_gemm. nq/qscale: columns n < nq scaled.
int gemm_launch(const void* x, const flexq_tensor* W, const void* bias, const void* residual, void* y, int M,
                int relu, int nq, float qscale, bool xperm, bool yperm, void* ws, int64_t ws_bytes, cudaStream_t st,
                const KvFuse* kv, bool early_w) {
    if (M == 0) return FLEX_OK;
    const int N = static_cast<int>(W->shape[0]), K = static_cast<int>(W->shape[1]);
    const int bits = W->cfg.num_bits;
    // small batches of int4 weights: the register-dequant GEMV on mma.sync
    if (gemv_eligible(M, N, bits))
        return gemv_launch(x, W, bias, residual, y, M, relu, nq, qscale, xperm, yperm, ws, ws_bytes, st, kv, early_w);
    if (tc2_eligible(M, N))
        return gemm2_launch(x, W, bias, residual, y, M, relu, nq, qscale, xperm, yperm, ws, ws_bytes, st, kv, early_w);
    const Plan P = make_plan(M, N, K, bits);
    if (P.ws_bytes > 0 && (ws == nullptr || ws_bytes < P.ws_bytes)) return FLEX_ERR_WORKSPACE;
    CUtensorMap tm_codes, tm_meta, tm_x;
    // code tiles: 128 rows x 128 bytes (4 K chunks at 4 bits, 2 at 8 bits), 128-byte swizzle
    int rc = make_tmap_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->codes, static_cast<uint64_t>(K) * bits / 8,
                          N, static_cast<uint64_t>(K) * bits / 8, 128, kBM, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != FLEX_OK) return rc;
    rc = make_tmap_2d(&tm_meta, CU_TENSOR_MAP_DATA_TYPE_UINT32, W->meta, K / kBK, N,
                      static_cast<uint64_t>(K / kBK) * 4, kMetaChunks, kBM, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc != FLEX_OK) return rc;
    rc = make_tmap_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, K, M, static_cast<uint64_t>(K) * 2, kBK, P.BN,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != FLEX_OK) return rc;
    GemmParams gp{};
    gp.wait_ns = pipeline_wait_ns();
    gp.gate = reinterpret_cast<const volatile int*>(gemm_gate());
    gp.bias = static_cast<const __half*>(bias);
    gp.residual = static_cast<const __half*>(residual);
    gp.y = static_cast<__half*>(y);
    gp.status = status_word();
    gp.M = M;
    gp.N = N;
    gp.K = K;
    gp.BN = P.BN;
    gp.splits = P.splits;
    gp.cps = P.cps;
    gp.nq = nq;
    gp.qscale = qscale;
    gp.relu = relu;
    gp.early_w = early_w ? 1 : 0;
    gp.yperm = yperm ? 1 : 0;
    gp.nsx = P.nsx;
    gp.nsc = P.nsc;
    gp.xu = P.xu;
    gp.cluster = P.cluster;
    gp.counters = static_cast<int*>(ws);
    gp.part = reinterpret_cast<float*>(static_cast<char*>(ws) + P.counters_bytes);
    gp.nacc = P.nacc;
    gp.acc_stride = P.acc_stride;
    gp.off_x = P.off_x;
    gp.off_c = P.off_c;
    gp.off_m = P.off_m;
    gp.off_bar = P.off_bar;
    gp.tmem_cols = P.tmem_cols;
    fill_kv_target(gp.kv, kv);
    const dim3 grid(P.tiles_n, P.tiles_m, P.splits);
    // programmatic dependent launch, and the K splits of a tile as one cluster
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = P.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = P.splits;
    cfg.attrs = attr;
    cfg.numAttrs = P.cluster ? 2 : 1;
#define GEMM_LAUNCH(B_, XP_)                                                                 \
    do {                                                                                     \
        set_smem_once(gemm_tc_kernel<B_, XP_>, 227 * 1024);                                  \
        cudaLaunchKernelEx(&cfg, gemm_tc_kernel<B_, XP_>, tm_codes, tm_meta, tm_x, gp);      \
    } while (0)
    if (bits == 4) {
        if (xperm) GEMM_LAUNCH(4, true); else GEMM_LAUNCH(4, false);
    } else {
        if (xperm) GEMM_LAUNCH(8, true); else GEMM_LAUNCH(8, false);
    }
#undef GEMM_LAUNCH
    return launch_status();
}

}  // namespace flexq

using namespace flexq;

extern "C" int64_t flex_gemm_ws_bytes(int32_t M, int32_t N, int32_t K) {
    FLEX_REQUIRE(M >= 0 && N > 0 && K > 0, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(N % kBM == 0 && K % 256 == 0, FLEX_ERR_SHAPE);
    const int64_t a = gemm_ws_bytes(M, N, K, 4), b = gemm_ws_bytes(M, N, K, 8);
    return a > b ? a : b;
}

extern "C" int32_t flex_set_gemm_streamk(int32_t enable) { return g_streamk.exchange(enable ? 1 : 0); }

extern "C" int32_t flex_set_gemm_gemv(int32_t enable) { return g_gemv.exchange(enable ? 1 : 0); }

extern "C" int flex_gemm_plan(int32_t M, int32_t N, int32_t K, int32_t bits, int32_t* out) {
    FLEX_REQUIRE(out != nullptr && M > 0 && N > 0 && K > 0, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(bits == 4 || bits == 8, FLEX_ERR_UNSUPPORTED);
    FLEX_REQUIRE(N % kBM == 0 && K % 256 == 0, FLEX_ERR_SHAPE);
    if (gemv_eligible(M, N, bits)) {
        const GemvPlan P = gemv_plan(M, N, K);
        out[0] = 0;
        out[1] = P.tiles;
        out[2] = P.splits;
        out[3] = P.cluster;
    } else if (tc2_eligible(M, N)) {
        const Plan2 P = make_plan2(M, N, K, bits);
        out[0] = 2;
        out[1] = P.tiles_n * P.tiles_m;
        out[2] = P.sk ? P.grid : P.splits;
        out[3] = P.sk ? 2 : (P.cluster ? 1 : (P.xchg && P.splits > 1 ? 3 : 0));
    } else {
        const Plan P = make_plan(M, N, K, bits);
        out[0] = 1;
        out[1] = P.tiles_n * P.tiles_m;
        out[2] = P.splits;
        out[3] = P.cluster;
    }
    return FLEX_OK;
}

extern "C" int flex_dequant_gemm(const void* x, const flexq_tensor* W, const void* bias, const void* residual,
                                 void* y, int32_t M, int32_t epilogue, void* ws, int64_t ws_bytes, void* stream) {
    int rc = validate_weight(W);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(x && y, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(M >= 0, FLEX_ERR_INVALID_ARG);
    const bool xil = (epilogue & FLEX_GEMM_X_INTERLEAVED) != 0;
    epilogue &= ~FLEX_GEMM_X_INTERLEAVED;
    FLEX_REQUIRE(epilogue == FLEX_EPI_NONE || epilogue == FLEX_EPI_RELU || epilogue == FLEX_EPI_RESIDUAL,
                 FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(epilogue != FLEX_EPI_RESIDUAL || residual != nullptr, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(aligned16(x) && aligned16(y) && (!bias || aligned16(bias)) && (!residual || aligned16(residual)),
                 FLEX_ERR_ALIGN);
    FLEX_REQUIRE(ws == nullptr || aligned16(ws), FLEX_ERR_ALIGN);
    return gemm_launch(x, W, bias, epilogue == FLEX_EPI_RESIDUAL ? residual : nullptr, y, M,
                       epilogue == FLEX_EPI_RELU ? 1 : 0, 0, 1.0f, xil, false, ws, ws_bytes, as_stream(stream),
                       nullptr, false);
}
