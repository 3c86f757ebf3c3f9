// Scratch for ckv_sparse_decode_noalloc: a fixed array inside the library, so
// that callers who cannot allocate device memory can still run the sparse
// attention.  Host code only ever sees a host-side stand-in for the name
// g_decode_scratch; the real device address is looked up once per device
// with cudaGetSymbolAddress while that device is current, and passed to the
// kernels as an ordinary pointer.
#include <mutex>

#include "ckv_internal.cuh"

namespace ckv {

static __device__ __align__(256) unsigned char g_decode_scratch[CKV_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;
}  // namespace

cudaError_t static_decode_scratch(void** ptr, size_t* bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *ptr = g_scratch_addr[dev];
    *bytes = CKV_NOALLOC_SCRATCH_BYTES;
    return cudaSuccess;
}

}  // namespace ckv
