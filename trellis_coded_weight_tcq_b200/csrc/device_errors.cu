// device_errors.cu -- the device-side error word and tcq_device_errors.
//
// Kernels report failures that do not fault the GPU by OR-ing a flag into one
// 32-bit word per device: a bounded wait that gave up (the tensor-core feedback
// product of tcq_ldlq), and, in the TCQ_DEBUG build, an index that failed its
// bounds check (the access is skipped).  The host reads and clears the word
// with tcq_device_errors, which synchronises the caller's stream first.
#include <mutex>

#include "common.cuh"

namespace tcq {

// In the TCQ_DEBUG build (relocatable device code) the word is visible to the
// bounds checks of every kernel file; otherwise only through its address.
#ifdef TCQ_DEBUG
__device__ unsigned int g_tcq_device_errors = 0;
#else
static __device__ unsigned int g_tcq_device_errors = 0;
#endif

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mutex;
unsigned int* g_addr[kMaxDevices] = {};
}  // namespace

unsigned int* device_error_word(cudaStream_t stream)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    // looked up on every call made outside stream capture (a host query that
    // allocates nothing); during capture the last address looked up is used,
    // since a lookup may have to load the module, which capture forbids
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
        cudaGetLastError();
        cap = cudaStreamCaptureStatusActive;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    if (cap == cudaStreamCaptureStatusNone || !g_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_tcq_device_errors) != cudaSuccess) {
            cudaGetLastError();
            return g_addr[dev];
        }
        g_addr[dev] = static_cast<unsigned int*>(p);
    }
    return g_addr[dev];
}

}  // namespace tcq

extern "C" tcq_status tcq_device_errors(tcq_stream_t stream, uint32_t* flags)
{
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (flags) *flags = 0;
    unsigned int* word = tcq::device_error_word(st);
    if (!word) return TCQ_ERR_CUDA;
    unsigned int host = 0;
    // host is pageable: the copy completes before cudaMemcpyAsync returns to
    // the synchronised stream below
    if (cudaStreamSynchronize(st) != cudaSuccess ||
        cudaMemcpyAsync(&host, word, sizeof(host), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemsetAsync(word, 0, sizeof(unsigned int), st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return TCQ_ERR_CUDA;
    }
    if (flags) *flags = host;
    return host ? TCQ_ERR_INTERNAL : TCQ_OK;
}
