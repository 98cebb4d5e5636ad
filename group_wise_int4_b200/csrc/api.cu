// Library-wide state and status reporting.
//
// The only global state is one `int` status word per device, a file-scope __device__
// variable whose address is looked up once per device. Kernels with bounded waits
// record FLEX_ERR_TIMEOUT there instead of trapping; flex_get_status reads and clears
// it.
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
