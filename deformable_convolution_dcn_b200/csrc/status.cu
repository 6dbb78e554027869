// Device status word of libdcn_b200: kernels with bounded waits record a
// non-zero code here instead of hanging; dcn_check_status() reads and clears it.
// Also the per-device host-side caches the launchers share (SM count, status
// word address, shared-memory attributes), each safe under concurrent callers.
#include <mutex>

#include "kernels.h"

namespace dcn {

__device__ unsigned int g_status_word;
// Where take_status_kernel leaves the word it took.
__device__ unsigned int g_status_taken;

namespace {
std::mutex g_setup_mu;  // serialises the slow path of every per-device set-up below

__global__ void take_status_kernel() { g_status_taken = atomicExch(&g_status_word, 0u); }
}  // namespace

cudaError_t status_word_ptr(unsigned int** ptr) {
    static std::atomic<unsigned int*> cache[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    unsigned int* p = cache[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_setup_mu);
        p = cache[dev].load(std::memory_order_relaxed);
        if (!p) {
            e = cudaGetSymbolAddress((void**)&p, g_status_word);
            if (e != cudaSuccess) return e;
            cache[dev].store(p, std::memory_order_release);
        }
    }
    *ptr = p;
    return cudaSuccess;
}

cudaError_t read_and_clear_status(unsigned int* out, cudaStream_t st) {
    // taking the word with one atomic exchange on the device loses no bit that
    // a kernel on another stream sets meanwhile
    take_status_kernel<<<1, 1, 0, st>>>();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbolAsync(out, g_status_taken, sizeof(unsigned int), 0, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(st);
}

cudaError_t max_dynamic_smem_once(const void* func, int bytes, DeviceFlags& flags) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (flags.done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (flags.done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) flags.done[dev].store(true, std::memory_order_release);
    return e;
}

cudaError_t smem_carveout_for(const void* func, uint32_t smem_bytes, DeviceCarveout& cache) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    int per_sm = 0;
    e = cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (e != cudaSuccess || per_sm <= 0) return e != cudaSuccess ? e : cudaErrorInvalidValue;
    // the block's dynamic shared memory plus the 1 KB the system reserves per block
    int pct = (int)(((long long)smem_bytes + 1024) * 100 / per_sm) + 1;
    pct = pct > 100 ? 100 : pct;
    if (cache.pct[dev].load(std::memory_order_acquire) == pct + 1) return cudaSuccess;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (cache.pct[dev].load(std::memory_order_relaxed) == pct + 1) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, pct);
    if (e == cudaSuccess) cache.pct[dev].store(pct + 1, std::memory_order_release);
    return e;
}

int num_sms() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev].store(n, std::memory_order_relaxed);  // every thread computes the same value
    }
    return n;
}

}  // namespace dcn
