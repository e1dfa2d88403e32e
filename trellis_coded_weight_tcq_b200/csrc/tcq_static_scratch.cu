// tcq_static_scratch.cu -- tcq_encode for callers that cannot allocate device
// memory.
//
// The regular encoder needs a caller-provided workspace for its Viterbi
// backpointers.  Some callers cannot get one: a host program that hands all of
// the GPU's memory to its own pool allocator (so a raw cudaMalloc fails or
// fragments that pool), code running under a fixed device-memory budget, or a
// latency-critical path that must not call cudaMalloc because it can
// synchronise the device and take unbounded time.  This entry point gives them
// an encoder that allocates nothing: its scratch is one file-scope device array
// of TCQ_STATIC_SCRATCH_BYTES, which exists on every GPU that loads the library
// for as long as the process lives.
#include <mutex>

#include "common.cuh"

namespace {

// 256 bytes of slack: the address is rounded up to the encoder's 256-byte
// workspace alignment at set-up, whatever alignment the loader gave the array.
static __device__ __align__(256) unsigned char g_tcq_scratch[TCQ_STATIC_SCRATCH_BYTES + 256];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_tcq_scratch on the current device.  In host code the
// array's name only stands in for the symbol; the address a kernel may use is
// looked up with that device current.  Outside stream capture it is looked up
// on every call (a host-side query that allocates nothing), so a module reload
// after cudaDeviceReset in the caller's process is picked up; during capture
// the address cached by the last call outside capture is used, because a
// lookup may have to load the module, which capture forbids.
tcq_status scratch_address(cudaStream_t stream, void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return TCQ_ERR_CUDA;
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
        cudaGetLastError();  // e.g. the legacy stream while another stream captures
        cap = cudaStreamCaptureStatusActive;
    }
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (cap == cudaStreamCaptureStatusNone || !g_scratch_addr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_tcq_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return TCQ_ERR_CUDA;
        }
        const uintptr_t a = (reinterpret_cast<uintptr_t>(p) + 255) & ~static_cast<uintptr_t>(255);
        g_scratch_addr[dev] = reinterpret_cast<void*>(a);
    }
    *out = g_scratch_addr[dev];
    return TCQ_OK;
}

}  // namespace

extern "C" tcq_status tcq_encode_static_scratch(const float* x, const float* d,
                                                const void* codebook, tcq_dtype cb_dtype, int L,
                                                int k, int T, int64_t n_blocks,
                                                uint32_t* start_state, uint32_t* bits,
                                                float* path_cost, tcq_stream_t stream)
{
    if (n_blocks == 0)  // nothing to do; the regular entry point answers without scratch
        return tcq_encode(x, d, codebook, cb_dtype, L, k, T, n_blocks, start_state, bits,
                          path_cost, nullptr, 0, stream);
    // one CTA's share must fit, else the problem is too large for the static array
    const size_t one_cta = tcq_encode_workspace_bytes(L, k, T, 1, cb_dtype);
    if (one_cta > (size_t)TCQ_STATIC_SCRATCH_BYTES) return TCQ_ERR_WORKSPACE;
    void* scratch = nullptr;
    const tcq_status st = scratch_address(reinterpret_cast<cudaStream_t>(stream), &scratch);
    if (st != TCQ_OK) return st;
    // Nothing in the scratch has to start at zero: every byte the encoder reads
    // was written earlier in the same call, so the previous call's leftovers
    // are harmless.
    return tcq_encode(x, d, codebook, cb_dtype, L, k, T, n_blocks, start_state, bits, path_cost,
                      scratch, (size_t)TCQ_STATIC_SCRATCH_BYTES, stream);
}
