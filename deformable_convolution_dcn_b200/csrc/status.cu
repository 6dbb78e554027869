// Device status word of libdcn_b200: kernels with bounded waits record a
// non-zero code here instead of hanging; dcn_check_status() reads and clears it.
#include "kernels.h"

namespace dcn {

__device__ unsigned int g_status_word;

cudaError_t status_word_ptr(unsigned int** ptr) {
    static unsigned int* cache[64] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!cache[dev]) {
        e = cudaGetSymbolAddress((void**)&cache[dev], g_status_word);
        if (e != cudaSuccess) return e;
    }
    *ptr = cache[dev];
    return cudaSuccess;
}

cudaError_t read_and_clear_status(unsigned int* out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_status_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_status_word, &zero, sizeof(unsigned int));
}

int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

}  // namespace dcn
