// Status strings and the device error word.
//
// Every GPU that runs a kernel of this library holds one int (a module-scope
// __device__ variable). Kernels record the first error they meet there with an
// atomic compare-and-swap; pkv_get_device_error reads and clears it. Host code
// only knows the variable's host-side shadow, so the device address is looked
// up once per device (with that device current) and cached.
#include <atomic>
#include <mutex>

#include "common.cuh"

namespace {

__device__ int g_error_word = 0;

constexpr int kMaxDevices = 64;
std::atomic<int*> g_word_ptr[kMaxDevices];
std::mutex g_word_mutex;

}  // namespace

namespace pkv {

int* device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    int* p = g_word_ptr[dev].load(std::memory_order_acquire);
    if (p) return p;
    std::lock_guard<std::mutex> lock(g_word_mutex);
    p = g_word_ptr[dev].load(std::memory_order_relaxed);
    if (!p) {
        void* addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_error_word) != cudaSuccess) return nullptr;
        p = static_cast<int*>(addr);
        g_word_ptr[dev].store(p, std::memory_order_release);
    }
    return p;
}

// One-shot test hook: the next launch of the named kernel withholds one copy in
// its first CTA and uses a short wait limit (pkv_test_withhold_copy).
namespace {
std::mutex g_hook_mutex;
int g_hook_index[2] = {-1, -1};
unsigned long long g_hook_wait_ns[2] = {0, 0};
}  // namespace

void take_wait_hook(int kernel, int* withhold, unsigned long long* wait_ns) {
    *withhold = -1;
    *wait_ns = kDefaultWaitNs;
    std::lock_guard<std::mutex> lock(g_hook_mutex);
    if (g_hook_index[kernel] >= 0) {
        *withhold = g_hook_index[kernel];
        *wait_ns = g_hook_wait_ns[kernel];
        g_hook_index[kernel] = -1;
    }
}

}  // namespace pkv

extern "C" {

pkv_status pkv_test_withhold_copy(int kernel, int index, unsigned long long wait_limit_ns) {
    if (kernel != 0 && kernel != 1) return PKV_ERR_INVALID_ARG;
    if (index < -1 || (index >= 0 && (wait_limit_ns < 100000ull || wait_limit_ns > pkv::kDefaultWaitNs)))
        return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(pkv::g_hook_mutex);
    pkv::g_hook_index[kernel] = index;
    pkv::g_hook_wait_ns[kernel] = index >= 0 ? wait_limit_ns : 0;
    return PKV_OK;
}

const char* pkv_status_string(int status) {
    switch (status) {
        case PKV_OK: return "ok";
        case PKV_ERR_INVALID_ARG: return "invalid argument";
        case PKV_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case PKV_ERR_CUDA: return "CUDA runtime error";
        case PKV_ERR_DEVICE_BOUNDS: return "device: block id, slot or context length out of range";
        case PKV_ERR_OUT_OF_BLOCKS: return "block manager: no free block";
        case PKV_ERR_DEVICE_TIMEOUT: return "device: bounded wait timed out";
        default: return "unknown status";
    }
}

pkv_status pkv_get_device_error(int* code, void* stream) {
    if (!code) return PKV_ERR_INVALID_ARG;
    *code = 0;
    int* word = pkv::device_error_word();
    if (!word) return PKV_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int host = 0;
    const int zero = 0;
    if (cudaMemcpyAsync(&host, word, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return PKV_ERR_CUDA;
    if (cudaMemcpyAsync(word, &zero, sizeof(int), cudaMemcpyHostToDevice, s) != cudaSuccess)
        return PKV_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return PKV_ERR_CUDA;
    *code = host;
    return PKV_OK;
}

}  // extern "C"
