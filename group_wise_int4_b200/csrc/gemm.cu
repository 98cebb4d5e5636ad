// Dequant-fused weight GEMM on the 5th-generation tensor cores (tcgen05).
//
//   y[m][n] = epilogue( sum_k x[m][k] * W^[n][k] + bias[n] )
//
// W is a group-wise compressed weight (FlexGen source walkthrough, section 6.3:
// 4-bit codes, group 64, per-group fp16 {min, scale}), stored [N][K] and grouped along
// K, so a 64-wide K chunk is exactly one group per row. The kernel never materialises
// W^ in global memory:
//
//   warp 0      TMA: int4 code tiles [128 rows][32 B] and metadata tiles
//               [128 rows][4 groups] into shared-memory rings
//   warp 1      TMA: activation tiles [BN rows][64] fp16 with the 128-byte swizzle
//   warp 2      allocates the TMEM accumulator and issues tcgen05.mma (one thread)
//   warps 4-11  unpack the codes in shared memory to fp16 (q*step + min, one half2 FMA
//               per pair) in the canonical K-major 128-byte-swizzled layout, then run
//               the epilogue from TMEM (bias, 1/sqrt(d) on the query columns, ReLU,
//               residual, fp16 store)
//
// Swap-AB orientation: the weight rows are the MMA's M side (128 per CTA) and the
// activation rows (batch in decode, tokens in prefill) its N side (BN = 16..256), so a
// decode batch of a few sequences still fills an M=128 instruction. Small grids are
// split along K; each split writes fp32 partials and the last CTA of a tile (atomic
// ticket) reduces them in a fixed order and runs the epilogue, so results do not
// depend on scheduling. Every mbarrier wait is bounded: on expiry the CTA records
// FLEX_ERR_TIMEOUT in the device status word, drains its own copies and MMAs, frees
// TMEM and exits.
#include "tc.cuh"

namespace flexq {

namespace {

constexpr int kBM = 128;           // weight rows per CTA (MMA M)
constexpr int kBK = 64;            // K per stage = one quantisation group
constexpr int kThreads = 384;      // 12 warps
constexpr int kDequantThreads = 256;
constexpr int kNSA = 4;            // dequantised A stages
constexpr int kMetaChunks = 4;     // groups per metadata tile

struct GemmParams {
    const __half* bias;
    const __half* residual;
    __half* y;
    float* part;
    int* counters;
    int* status;
    int M, N, K;
    int BN;
    int splits, cps;       // K splits, chunks per split (multiple of kMetaChunks)
    int nq;                // columns n < nq are multiplied by qscale
    float qscale;
    int relu;
    int nsx, nsc;          // activation / code ring depths
    uint32_t off_x, off_c, off_m, off_bar;
    uint32_t tmem_cols;
};

struct Bars {
    uint32_t codes_full, codes_empty, x_full, x_empty, a_full, a_empty, meta_full, meta_empty, acc_full, drain;
};

__device__ __forceinline__ uint32_t dequant_pair(uint32_t raw_pair_bits, uint32_t step2, uint32_t mn2) {
    // raw_pair_bits holds two integers q in the low mantissa bits of 1024.0h: (1024+q)
    const uint32_t bias2 = 0x64006400u;
    __half2 v = __hsub2(*reinterpret_cast<const __half2*>(&raw_pair_bits), *reinterpret_cast<const __half2*>(&bias2));
    v = __hfma2(v, *reinterpret_cast<const __half2*>(&step2), *reinterpret_cast<const __half2*>(&mn2));
    return *reinterpret_cast<uint32_t*>(&v);
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

// 8 codes of 4 bits (one u32, element e in bits 4e..4e+3) -> 8 fp16 in natural order.
__device__ __forceinline__ uint4 dequant8_4bit(uint32_t w, uint32_t step2, uint32_t mn2) {
    const uint32_t p0 = dequant_pair(lop_nib(w), step2, mn2);         // (e0, e4)
    const uint32_t p1 = dequant_pair(lop_nib(w >> 4), step2, mn2);    // (e1, e5)
    const uint32_t p2 = dequant_pair(lop_nib(w >> 8), step2, mn2);    // (e2, e6)
    const uint32_t p3 = dequant_pair(lop_nib(w >> 12), step2, mn2);   // (e3, e7)
    return make_uint4(prmt(p0, p1, 0x5410u), prmt(p2, p3, 0x5410u), prmt(p0, p1, 0x7632u), prmt(p2, p3, 0x7632u));
}

// 4 codes of 8 bits (one u32) -> 4 fp16 as two half2.
__device__ __forceinline__ uint2 dequant4_8bit(uint32_t w, uint32_t step2, uint32_t mn2) {
    const uint32_t hi = 0x64646464u;
    return make_uint2(dequant_pair(prmt(w, hi, 0x4140u), step2, mn2), dequant_pair(prmt(w, hi, 0x4342u), step2, mn2));
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_codes,
                                                              const __grid_constant__ CUtensorMap tm_meta,
                                                              const __grid_constant__ CUtensorMap tm_x,
                                                              const GemmParams p) {
    constexpr int CB = kBM * kBK * BITS / 8;     // code bytes per stage
    constexpr int CROW = kBK * BITS / 8;         // code bytes per row and stage
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const gbase = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kBM, m0 = blockIdx.y * p.BN, split = blockIdx.z;
    const int nk_total = p.K / kBK;
    const int c_begin = split * p.cps;
    const int nk = min(nk_total, c_begin + p.cps) - c_begin;

    const uint32_t sA = base, sX = base + p.off_x, sC = base + p.off_c, sM = base + p.off_m;
    const uint32_t sb = base + p.off_bar;
    const int NSX = p.nsx, NSC = p.nsc;
    Bars B;
    B.codes_full = sb;
    B.codes_empty = B.codes_full + 8 * NSC;
    B.x_full = B.codes_empty + 8 * NSC;
    B.x_empty = B.x_full + 8 * NSX;
    B.a_full = B.x_empty + 8 * NSX;
    B.a_empty = B.a_full + 8 * kNSA;
    B.meta_full = B.a_empty + 8 * kNSA;
    B.meta_empty = B.meta_full + 16;
    B.acc_full = B.meta_empty + 16;
    B.drain = B.acc_full + 8;
    const uint32_t misc = B.drain + 8;                        // tmem slot, abort flag, last flag
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + (misc - base));
    volatile int* abort = reinterpret_cast<volatile int*>(gbase + (misc - base) + 4);
    volatile int* last_flag = reinterpret_cast<volatile int*>(gbase + (misc - base) + 8);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSC; ++s) {
            tc::bar_init(B.codes_full + 8 * s, 1);
            tc::bar_init(B.codes_empty + 8 * s, kDequantThreads);
        }
        for (int s = 0; s < NSX; ++s) {
            tc::bar_init(B.x_full + 8 * s, 1);
            tc::bar_init(B.x_empty + 8 * s, 1);
        }
        for (int s = 0; s < kNSA; ++s) {
            tc::bar_init(B.a_full + 8 * s, kDequantThreads);
            tc::bar_init(B.a_empty + 8 * s, 1);
        }
        for (int s = 0; s < 2; ++s) {
            tc::bar_init(B.meta_full + 8 * s, 1);
            tc::bar_init(B.meta_empty + 8 * s, kDequantThreads);
        }
        tc::bar_init(B.acc_full, 1);
        tc::bar_init(B.drain, 1);
        *abort = 0;
        *last_flag = 0;
        tc::bar_fence_init();
    }
    if (warp == 2) {
        tc::tmem_alloc(misc, p.tmem_cols);
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

    if (warp == 0) {
        // ---------------- codes + metadata producer ----------------
        if (lane == 0) {
            int i = 0, mi = 0;   // code tiles and metadata tiles issued
            for (; i < nk; ++i) {
                const int c = c_begin + i;
                if (i % kMetaChunks == 0) {
                    const int blk = i / kMetaChunks, sm = blk & 1;
                    if (!tc::bar_wait(B.meta_empty + 8 * sm, ((blk >> 1) & 1) ^ 1, abort, p.status)) break;
                    tc::bar_arrive_expect_tx(B.meta_full + 8 * sm, kBM * kMetaChunks * 4);
                    tc::tma_load_2d(sM + sm * (kBM * kMetaChunks * 4), &tm_meta, c, n0, B.meta_full + 8 * sm);
                    ++mi;
                }
                const int s = i % NSC;
                if (!tc::bar_wait(B.codes_empty + 8 * s, ((i / NSC) & 1) ^ 1, abort, p.status)) break;
                tc::bar_arrive_expect_tx(B.codes_full + 8 * s, CB);
                tc::tma_load_2d(sC + s * CB, &tm_codes, c * CROW, n0, B.codes_full + 8 * s);
            }
            // drain: every copy this thread issued has landed before the CTA can exit
            const int issued = i;
            for (int s = 0; s < NSC && s < issued; ++s) {
                const int last = s + ((issued - 1 - s) / NSC) * NSC;
                volatile int never = 0;
                tc::bar_wait(B.codes_full + 8 * s, (last / NSC) & 1, &never, p.status);
            }
            for (int sm = 0; sm < 2 && sm < mi; ++sm) {
                const int last = sm + ((mi - 1 - sm) / 2) * 2;
                volatile int never = 0;
                tc::bar_wait(B.meta_full + 8 * sm, (last >> 1) & 1, &never, p.status);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- activation producer ----------------
        if (lane == 0) {
            int i = 0;
            for (; i < nk; ++i) {
                const int s = i % NSX;
                if (!tc::bar_wait(B.x_empty + 8 * s, ((i / NSX) & 1) ^ 1, abort, p.status)) break;
                tc::bar_arrive_expect_tx(B.x_full + 8 * s, p.BN * 128);
                tc::tma_load_2d(sX + s * (p.BN * 128), &tm_x, (c_begin + i) * kBK, m0, B.x_full + 8 * s);
            }
            const int issued = i;
            for (int s = 0; s < NSX && s < issued; ++s) {
                const int last = s + ((issued - 1 - s) / NSX) * NSX;
                volatile int never = 0;
                tc::bar_wait(B.x_full + 8 * s, (last / NSX) & 1, &never, p.status);
            }
        }
        __syncwarp();
    } else if (warp == 2) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_f16_f32(kBM, p.BN);
            bool ok = true;
            for (int i = 0; i < nk; ++i) {
                const int sa = i % kNSA, sx = i % NSX;
                if (!tc::bar_wait(B.a_full + 8 * sa, (i / kNSA) & 1, abort, p.status)) { ok = false; break; }
                if (!tc::bar_wait(B.x_full + 8 * sx, (i / NSX) & 1, abort, p.status)) { ok = false; break; }
                tc::fence_after_sync();
                const uint64_t ad = tc::desc_k_sw128(sA + sa * (kBM * 128));
                const uint64_t bd = tc::desc_k_sw128(sX + sx * (p.BN * 128));
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk)
                    tc::mma_f16(tmem, ad + 2 * kk, bd + 2 * kk, idesc, (i > 0 || kk > 0) ? 1u : 0u);
                tc::mma_commit(B.a_empty + 8 * sa);
                tc::mma_commit(B.x_empty + 8 * sx);
            }
            if (ok) {
                tc::mma_commit(B.acc_full);
            } else {
                // nothing of ours may still run on the tensor cores at exit
                tc::mma_commit(B.drain);
                volatile int never = 0;
                tc::bar_wait(B.drain, 0, &never, p.status);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------- dequantisation ----------------
        const int dt = threadIdx.x - 128;
        const int row = dt & 127, half_ = dt >> 7;
        bool ok = true;
        uint4 mrow = make_uint4(0, 0, 0, 0);
        for (int i = 0; i < nk; ++i) {
            if (i % kMetaChunks == 0) {
                const int blk = i / kMetaChunks;
                if (!tc::bar_wait(B.meta_full + 8 * (blk & 1), (blk >> 1) & 1, abort, p.status)) { ok = false; break; }
                mrow = *reinterpret_cast<const uint4*>(gbase + (sM - base) + (blk & 1) * (kBM * kMetaChunks * 4) + row * 16);
            }
            const int sc = i % NSC;
            if (!tc::bar_wait(B.codes_full + 8 * sc, (i / NSC) & 1, abort, p.status)) { ok = false; break; }
            const uint8_t* crow = gbase + (sC - base) + sc * CB + row * CROW + half_ * (CROW / 2);
            uint4 cw0 = *reinterpret_cast<const uint4*>(crow);
            uint4 cw1 = make_uint4(0, 0, 0, 0);
            if (BITS == 8) cw1 = *reinterpret_cast<const uint4*>(crow + 16);
            tc::bar_arrive(B.codes_empty + 8 * sc);
            if (i % kMetaChunks == kMetaChunks - 1 || i == nk - 1) tc::bar_arrive(B.meta_empty + 8 * ((i / kMetaChunks) & 1));

            const uint32_t mw = (i % 4 == 0) ? mrow.x : (i % 4 == 1) ? mrow.y : (i % 4 == 2) ? mrow.z : mrow.w;
            const __half mn = __ushort_as_half(static_cast<unsigned short>(mw & 0xFFFFu));
            const float sc32 = __half2float(__ushort_as_half(static_cast<unsigned short>(mw >> 16)));
            const __half step = __float2half_rn(sc32 > 0.f ? 1.0f / sc32 : 0.f);
            const __half2 step2h = __half2half2(step), mn2h = __half2half2(mn);
            const uint32_t step2 = *reinterpret_cast<const uint32_t*>(&step2h);
            const uint32_t mn2 = *reinterpret_cast<const uint32_t*>(&mn2h);

            const int sa = i % kNSA;
            if (!tc::bar_wait(B.a_empty + 8 * sa, ((i / kNSA) & 1) ^ 1, abort, p.status)) { ok = false; break; }
            uint8_t* arow = gbase + sa * (kBM * 128) + row * 128;
            const int sw = row & 7;
            if (BITS == 4) {
                const uint32_t w[4] = {cw0.x, cw0.y, cw0.z, cw0.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 v = dequant8_4bit(w[j], step2, mn2);
                    *reinterpret_cast<uint4*>(arow + (((half_ * 4 + j) ^ sw) << 4)) = v;
                }
            } else {
                const uint32_t w[8] = {cw0.x, cw0.y, cw0.z, cw0.w, cw1.x, cw1.y, cw1.z, cw1.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint2 a = dequant4_8bit(w[2 * j], step2, mn2);
                    const uint2 b = dequant4_8bit(w[2 * j + 1], step2, mn2);
                    *reinterpret_cast<uint4*>(arow + (((half_ * 4 + j) ^ sw) << 4)) = make_uint4(a.x, a.y, b.x, b.y);
                }
            }
            tc::fence_proxy_async_smem();
            tc::bar_arrive(B.a_full + 8 * sa);
        }
        // ---------------- epilogue ----------------
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (ok && !*abort) ok = tc::bar_wait(B.acc_full, 0, abort, p.status);
        // one decision for all 256 threads (they share the named barriers below)
        uint32_t all_ok;
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
            const int lq = warp & 3, ch = (warp - 4) >> 2;
            const int irow = lq * 32 + lane;
            const int n = n0 + irow;
            const uint32_t taddr = tmem + (static_cast<uint32_t>(lq * 32) << 16);
            const int cbeg = ch * (p.BN / 2), cend = cbeg + p.BN / 2;
            const float bias_n = p.bias ? __half2float(p.bias[n]) : 0.f;
            const float scale_n = n < p.nq ? p.qscale : 1.f;
            auto finish = [&](int col, float v) {
                const int m = m0 + col;
                if (m >= p.M) return;
                v = (v + bias_n) * scale_n;
                if (p.relu) v = fmaxf(v, 0.f);
                const int64_t o = static_cast<int64_t>(m) * p.N + n;
                if (p.residual) v += __half2float(p.residual[o]);
                p.y[o] = __float2half_rn(v);
            };
            if (p.splits == 1) {
                for (int col = cbeg; col < cend; col += 8) {
                    float v[8];
                    tc::tmem_ld8(taddr + col, v);
#pragma unroll
                    for (int j = 0; j < 8; ++j) finish(col + j, v[j]);
                }
            } else {
                const int tile = blockIdx.y * gridDim.x + blockIdx.x;
                float* mine = p.part + (static_cast<int64_t>(tile) * p.splits + split) * p.BN * kBM;
                for (int col = cbeg; col < cend; col += 8) {
                    float v[8];
                    tc::tmem_ld8(taddr + col, v);
#pragma unroll
                    for (int j = 0; j < 8; ++j) mine[(col + j) * kBM + irow] = v[j];
                }
                __threadfence();
                asm volatile("bar.sync 1, 256;" ::: "memory");
                if (dt == 0) *last_flag = (atomicAdd(p.counters + tile, 1) == p.splits - 1);
                asm volatile("bar.sync 1, 256;" ::: "memory");
                if (*last_flag) {
                    __threadfence();
                    const float* all = p.part + static_cast<int64_t>(tile) * p.splits * p.BN * kBM;
                    for (int col = cbeg; col < cend; ++col) {
                        float acc = 0.f;
                        for (int s = 0; s < p.splits; ++s)
                            acc += __ldcg(all + (static_cast<int64_t>(s) * p.BN + col) * kBM + irow);
                        finish(col, acc);
                    }
                    if (dt == 0) p.counters[tile] = 0;
                }
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 2) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, p.tmem_cols);
    }
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

struct Plan {
    int BN, tiles_n, tiles_m, splits, cps, nsx, nsc;
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
    const int sms = sm_count();
    int splits = 1;
    if (tiles < sms) splits = sms / tiles;
    int max_splits = nk / kMetaChunks;
    if (max_splits < 1) max_splits = 1;
    if (splits > max_splits) splits = max_splits;
    int cps = (nk + splits - 1) / splits;
    cps = ((cps + kMetaChunks - 1) / kMetaChunks) * kMetaChunks;
    splits = (nk + cps - 1) / cps;
    P.splits = splits;
    P.cps = cps;
    P.nsx = P.BN <= 64 ? 6 : (P.BN <= 160 ? 4 : 3);
    P.nsc = bits == 4 ? 8 : 4;
    const uint32_t cb = kBM * kBK * bits / 8;
    P.off_x = kNSA * kBM * 128;
    P.off_c = P.off_x + P.nsx * P.BN * 128;
    P.off_m = P.off_c + P.nsc * cb;
    P.off_bar = P.off_m + 2 * kBM * kMetaChunks * 4;
    uint32_t smem = P.off_bar + 8 * (2 * P.nsc + 2 * P.nsx + 2 * kNSA + 4 + 2) + 16 + 1024;
    if (smem < 120 * 1024) smem = 120 * 1024;   // at most one CTA per SM: TMEM is never contended
    P.smem = smem;
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(P.BN)) cols <<= 1;
    P.tmem_cols = cols;
    P.counters_bytes = ((static_cast<int64_t>(tiles) * 4 + 255) / 256) * 256;
    P.ws_bytes = splits > 1 ? P.counters_bytes + static_cast<int64_t>(tiles) * splits * P.BN * kBM * 4 : 0;
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

int64_t gemm_ws_bytes(int M, int N, int K, int bits) { return make_plan(M, N, K, bits).ws_bytes; }

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
                int relu, int nq, float qscale, void* ws, int64_t ws_bytes, cudaStream_t st) {
    if (M == 0) return FLEX_OK;
    const int N = static_cast<int>(W->shape[0]), K = static_cast<int>(W->shape[1]);
    const int bits = W->cfg.num_bits;
    const Plan P = make_plan(M, N, K, bits);
    if (P.ws_bytes > 0 && (ws == nullptr || ws_bytes < P.ws_bytes)) return FLEX_ERR_WORKSPACE;
    CUtensorMap tm_codes, tm_meta, tm_x;
    int rc = make_tmap_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->codes, static_cast<uint64_t>(K) * bits / 8,
                          N, static_cast<uint64_t>(K) * bits / 8, kBK * bits / 8, kBM, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc != FLEX_OK) return rc;
    rc = make_tmap_2d(&tm_meta, CU_TENSOR_MAP_DATA_TYPE_UINT32, W->meta, K / kBK, N,
                      static_cast<uint64_t>(K / kBK) * 4, kMetaChunks, kBM, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc != FLEX_OK) return rc;
    rc = make_tmap_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, K, M, static_cast<uint64_t>(K) * 2, kBK, P.BN,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != FLEX_OK) return rc;
    GemmParams gp{};
    gp.bias = static_cast<const __half*>(bias);
    gp.residual = static_cast<const __half*>(residual);
    gp.y = static_cast<__half*>(y);
    gp.counters = static_cast<int*>(ws);
    gp.part = reinterpret_cast<float*>(static_cast<char*>(ws) + P.counters_bytes);
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
    gp.nsx = P.nsx;
    gp.nsc = P.nsc;
    gp.off_x = P.off_x;
    gp.off_c = P.off_c;
    gp.off_m = P.off_m;
    gp.off_bar = P.off_bar;
    gp.tmem_cols = P.tmem_cols;
    const dim3 grid(P.tiles_n, P.tiles_m, P.splits);
    if (bits == 4) {
        cudaFuncSetAttribute(gemm_tc_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.smem);
        gemm_tc_kernel<4><<<grid, kThreads, P.smem, st>>>(tm_codes, tm_meta, tm_x, gp);
    } else {
        cudaFuncSetAttribute(gemm_tc_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.smem);
        gemm_tc_kernel<8><<<grid, kThreads, P.smem, st>>>(tm_codes, tm_meta, tm_x, gp);
    }
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

extern "C" int flex_dequant_gemm(const void* x, const flexq_tensor* W, const void* bias, const void* residual,
                                 void* y, int32_t M, int32_t epilogue, void* ws, int64_t ws_bytes, void* stream) {
    int rc = validate_weight(W);
    if (rc != FLEX_OK) return rc;
    FLEX_REQUIRE(x && y, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(M >= 0, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(epilogue == FLEX_EPI_NONE || epilogue == FLEX_EPI_RELU || epilogue == FLEX_EPI_RESIDUAL,
                 FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(epilogue != FLEX_EPI_RESIDUAL || residual != nullptr, FLEX_ERR_INVALID_ARG);
    FLEX_REQUIRE(aligned16(x) && aligned16(y) && (!bias || aligned16(bias)) && (!residual || aligned16(residual)),
                 FLEX_ERR_ALIGN);
    FLEX_REQUIRE(ws == nullptr || aligned16(ws), FLEX_ERR_ALIGN);
    return gemm_launch(x, W, bias, epilogue == FLEX_EPI_RESIDUAL ? residual : nullptr, y, M,
                       epilogue == FLEX_EPI_RELU ? 1 : 0, 0, 1.0f, ws, ws_bytes, as_stream(stream));
}
