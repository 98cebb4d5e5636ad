// Shared host/device helpers of the flexq library (sm_100a only).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/flexq.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "flexq is built for sm_100a (B200) only"
#endif

namespace flexq {

// ---- host-side argument checks ---------------------------------------------------
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define FLEX_REQUIRE(cond, err) \
    do {                        \
        if (!(cond)) return (err); \
    } while (0)

inline int launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FLEX_OK : FLEX_ERR_CUDA;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Raise a kernel's dynamic shared-memory limit once per (kernel, device), so that it is
// not called again while a stream is being captured into a graph.
bool smem_attr_needed(const void* kernel, int bytes);
template <typename K>
inline void set_smem_once(K kernel, int bytes) {
    if (smem_attr_needed(reinterpret_cast<const void*>(kernel), bytes))
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// Launch `kernel` on `st`, with programmatic stream serialisation when pdl is true.
template <typename... KArgs, typename... Args>
inline void launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                     Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// store_cache fused into the QKV projection's epilogue (see gemm.cu). The activation
// rows may belong to several gpu-batches, each with its own cache: row m is row
// m % rows of the cache m / rows.
constexpr int kMaxKvBatches = 8;
struct KvFuse {
    const flex_kv_cache* caches;   // ncaches caches of identical geometry
    int ncaches;
    int rows;    // activation rows per cache (its batch * seq)
    int h;       // hidden size: features [h, 2h) keys, [2h, 3h) values
    int seq;     // tokens per sequence in this call
    int pos0;    // cache slot of token 0
};

// Kernel-side form of KvFuse. codes[0][0] == nullptr: no fused store.
struct KvTarget {
    uint8_t* codes[kMaxKvBatches][2];      // [cache][keys, values]
    uint32_t* meta[kMaxKvBatches][2];
    int rows, h, hd, nh, max_seq, seq, pos0, bits, gs;
};

inline void fill_kv_target(KvTarget& t, const KvFuse* kv) {
    t = KvTarget{};
    if (kv == nullptr) return;
    for (int c = 0; c < kv->ncaches && c < kMaxKvBatches; ++c) {
        t.codes[c][0] = static_cast<uint8_t*>(kv->caches[c].k_codes);
        t.codes[c][1] = static_cast<uint8_t*>(kv->caches[c].v_codes);
        t.meta[c][0] = static_cast<uint32_t*>(kv->caches[c].k_meta);
        t.meta[c][1] = static_cast<uint32_t*>(kv->caches[c].v_meta);
    }
    const flex_kv_cache& c0 = kv->caches[0];
    t.rows = kv->rows;
    t.h = kv->h;
    t.hd = c0.head_dim;
    t.nh = c0.n_heads;
    t.max_seq = c0.max_seq;
    t.seq = kv->seq;
    t.pos0 = kv->pos0;
    t.bits = c0.cfg.num_bits;
    t.gs = c0.cfg.group_size;
}

// Number of SMs of the current device (cached per device).
int sm_count();
// Limit of the tensor-core GEMM's pipeline waits for kernels launched from now on
// (flex_set_wait_limit_ns).
uint64_t pipeline_wait_ns();
// Gate of the tensor-core GEMM's weight loads for kernels launched from now on
// (flex_set_gemm_gate; nullptr = none).
const int32_t* gemm_gate();
// Device status word of the current device (created on first use; see flex_get_status).
int* status_word();

// ---- device helpers --------------------------------------------------------------
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_stream_v4(void* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_stream_u32(void* p, uint32_t v) {
    asm volatile("st.global.cs.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void st_stream_v2(void* p, uint2 v) {
    asm volatile("st.global.cs.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

__device__ __forceinline__ float h2f_lo(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xFFFFu)));
}
__device__ __forceinline__ float h2f_hi(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
}

__device__ __forceinline__ uint32_t pack_half2_bits(__half lo, __half hi) {
    return static_cast<uint32_t>(__half_as_ushort(lo)) |
           (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
}

// Programmatic dependent launch: a kernel launched with launch_k(..., pdl = true) may
// start while its predecessor in the stream is still running. pdl_wait() blocks until
// the predecessor grid has completed and its writes are visible (it returns at once
// when there is no such dependency); pdl_trigger() lets this kernel's own dependents
// start their prologues.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void set_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

}  // namespace flexq
