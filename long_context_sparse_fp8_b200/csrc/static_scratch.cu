// static_scratch.cu -- the fixed device array behind dsa_sparse_mla_decode_noalloc.
//
// The array lives in this translation unit alone, so its module (and the memory the
// CUDA runtime reserves for it on each device) is loaded only by processes that make
// that call, not by every user of the library.
#include <mutex>

#include "kernels.h"

namespace dsa {
namespace {

__device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ptr[kMaxDevices];

}  // namespace

cudaError_t static_scratch(void** ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_ptr[dev]) {
        // first call on this device, with the device current: look the address up once
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        g_ptr[dev] = p;
    }
    *ptr = g_ptr[dev];
    return cudaSuccess;
}

}  // namespace dsa
