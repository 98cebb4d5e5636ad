// Library-wide state and status reporting.
//
// The only global state is one `int` status word per device, a file-scope __device__
// variable whose address is looked up once per device. Kernels with bounded waits
// record FLEX_ERR_TIMEOUT there instead of trapping; flex_get_status reads and clears
// it.
#include <atomic>
#include <cstddef>
#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"

namespace flexq {

namespace {
__device__ int g_status_word;

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];
int* g_status_ptr[kMaxDevices];
std::mutex g_mu;

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev < kMaxDevices ? dev : -1;
}
}  // namespace

bool smem_attr_needed(const void* kernel, int bytes) {
    static std::map<std::pair<const void*, int>, int> done;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(g_mu);
    int& have = done[std::make_pair(kernel, dev)];
    if (have >= bytes) return false;
    have = bytes;
    return true;
}

int sm_count() {
    const int dev = current_device();
    if (dev < 0) return 148;
    if (g_sm_count[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        g_sm_count[dev] = n;
    }
    return g_sm_count[dev];
}

namespace {
constexpr uint64_t kDefaultWaitNs = 2000000000ull;     // the drain waits' limit, tc::kWaitLimitNs
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
}  // namespace

uint64_t pipeline_wait_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

namespace {
std::atomic<const int32_t*> g_gate{nullptr};
}  // namespace

const int32_t* gemm_gate() { return g_gate.load(std::memory_order_relaxed); }

int* status_word() {
    const int dev = current_device();
    if (dev < 0) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_status_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    return g_status_ptr[dev];
}

}  // namespace flexq

extern "C" int flex_get_status(void* stream) {
    using namespace flexq;
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return FLEX_ERR_CUDA;
    int* p = status_word();
    if (p == nullptr) return FLEX_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FLEX_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return FLEX_ERR_CUDA;
    }
    return v;
}

extern "C" uint64_t flex_set_wait_limit_ns(uint64_t ns) {
    return flexq::g_wait_ns.exchange(ns == 0 ? flexq::kDefaultWaitNs : ns);
}

extern "C" const int32_t* flex_set_gemm_gate(const int32_t* gate) { return flexq::g_gate.exchange(gate); }

extern "C" int64_t flex_abi_layout(int32_t which, int32_t field) {
#define FLEX_FIELDS(T, ...)                                              \
    {                                                                    \
        const int64_t offs[] = {__VA_ARGS__};                            \
        if (field == -1) return static_cast<int64_t>(sizeof(T));        \
        if (field >= 0 && field < static_cast<int32_t>(sizeof(offs) / sizeof(offs[0]))) return offs[field]; \
        return -1;                                                       \
    }
    switch (which) {
        case 0:
            FLEX_FIELDS(flexq_config, offsetof(flexq_config, num_bits), offsetof(flexq_config, group_size),
                        offsetof(flexq_config, group_dim), offsetof(flexq_config, symmetric))
        case 1:
            FLEX_FIELDS(flexq_tensor, offsetof(flexq_tensor, codes), offsetof(flexq_tensor, meta),
                        offsetof(flexq_tensor, ndim), offsetof(flexq_tensor, shape), offsetof(flexq_tensor, cfg))
        case 2:
            FLEX_FIELDS(flex_layer, offsetof(flex_layer, h), offsetof(flex_layer, n_heads),
                        offsetof(flex_layer, head_dim), offsetof(flex_layer, ffn), offsetof(flex_layer, ln1_g),
                        offsetof(flex_layer, ln1_b), offsetof(flex_layer, ln2_g), offsetof(flex_layer, ln2_b),
                        offsetof(flex_layer, w_qkv), offsetof(flex_layer, w_o), offsetof(flex_layer, w_fc1),
                        offsetof(flex_layer, w_fc2), offsetof(flex_layer, b_qkv), offsetof(flex_layer, b_o),
                        offsetof(flex_layer, b_fc1), offsetof(flex_layer, b_fc2))
        case 3:
            FLEX_FIELDS(flex_kv_cache, offsetof(flex_kv_cache, k_codes), offsetof(flex_kv_cache, k_meta),
                        offsetof(flex_kv_cache, v_codes), offsetof(flex_kv_cache, v_meta),
                        offsetof(flex_kv_cache, batch), offsetof(flex_kv_cache, n_heads),
                        offsetof(flex_kv_cache, head_dim), offsetof(flex_kv_cache, max_seq),
                        offsetof(flex_kv_cache, cfg), offsetof(flex_kv_cache, valid_from))
        default:
            return -1;
    }
#undef FLEX_FIELDS
}

extern "C" const char* flex_status_string(int32_t status) {
    switch (status) {
        case FLEX_OK: return "ok";
        case FLEX_ERR_INVALID_ARG: return "invalid argument";
        case FLEX_ERR_UNSUPPORTED: return "unsupported configuration";
        case FLEX_ERR_SHAPE: return "shape error";
        case FLEX_ERR_ALIGN: return "pointer not 16-byte aligned";
        case FLEX_ERR_WORKSPACE: return "workspace missing or too small";
        case FLEX_ERR_CUDA: return "CUDA error";
        case FLEX_ERR_TIMEOUT: return "device wait timed out";
        case FLEX_ERR_SCRATCH_LIMIT: return "problem needs more scratch than the built-in buffer holds";
        default: return "unknown status";
    }
}
