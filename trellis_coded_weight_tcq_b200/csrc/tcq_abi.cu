// tcq_abi.cu -- the C ABI declared in include/tcq.h: host-side argument checks,
// kernel selection, grid sizing from the workspace, and launches.  No entry
// point allocates, frees, synchronises or keeps state between calls.
#include <stdint.h>

#include "codes.cuh"

using namespace tcq;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

tcq_status check_shape(int L, int k, int T)
{
    if (k < 1 || k > TCQ_MAX_K || L < k || L > TCQ_MAX_L) return TCQ_ERR_UNSUPPORTED;
    if (T < 1 || T > TCQ_MAX_T) return TCQ_ERR_UNSUPPORTED;
    return TCQ_OK;
}

bool valid_dtype(tcq_dtype dt) { return dt == TCQ_F32 || dt == TCQ_F16 || dt == TCQ_MAD; }

// A table codebook must be present and aligned to its entry; the computed code has none.
bool codebook_ok(const void* cb, tcq_dtype dt)
{
    return dt == TCQ_MAD || (cb && aligned(cb, dt == TCQ_F16 ? 2 : 4));
}

// The kernels' codebook mode: 0 binary32 table, 1 binary16 table, 2 computed code.
int code_mode(tcq_dtype dt) { return dt == TCQ_F16 ? 1 : dt == TCQ_MAD ? kMadCodebook : 0; }

// Workspace bytes of the binary16 table a computed code is written to for the
// table-based kernels (encoders, soft quantizer); 0 for a table codebook.
size_t mad_table_bytes(int L, tcq_dtype dt)
{
    return dt == TCQ_MAD ? ((((size_t)2) << L) + 255) & ~(size_t)255 : 0;
}

// The dtype the table-based kernels run with.
tcq_dtype table_dtype(tcq_dtype dt) { return dt == TCQ_MAD ? TCQ_F16 : dt; }

// For the table-based kernels: writes the computed code's table to the front of
// the workspace and points (cb, dt) at it; the workspace shrinks by its size.
tcq_status resolve_table(const void*& cb, tcq_dtype& dt, int L, unsigned char*& ws,
                         size_t& ws_bytes, cudaStream_t stream)
{
    if (dt != TCQ_MAD) return TCQ_OK;
    const size_t tb = mad_table_bytes(L, dt);
    if (ws_bytes < tb) return TCQ_ERR_WORKSPACE;
    if (launch_mad_table(L, ws, stream) != cudaSuccess) return TCQ_ERR_CUDA;
    cb = ws;
    dt = TCQ_F16;
    ws += tb;
    ws_bytes -= tb;
    return TCQ_OK;
}

// The encoder for (L, k, T, dtype): the one-warp-per-block kernel for small
// trellises with blocks it holds, else a grouped kernel, else the generic one.
const EncodeKernelInfo* select_kernel(int L, int k, int T, tcq_dtype dt)
{
    if (const EncodeKernelInfo* w = find_warp_kernel(L, k, T)) return w;
    const EncodeKernelInfo* g = find_grouped_kernel(L, k, table_dtype(dt) == TCQ_F16 ? 1 : 0);
    return g ? g : generic_kernel_info(L, k);
}

// Streaming multiprocessors of the current device, or 0 without a device.
int current_sms()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return sms;
}

// Resident CTAs per SM for this kernel (at least 1).
int ctas_per_sm(const EncodeKernelInfo* info, int L, int k, int T)
{
    int n = 0;
    const size_t smem = info->smem_bytes(L, k, T);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, info->kernel, info->threads, smem) !=
        cudaSuccess) {
        cudaGetLastError();
        n = 1;
    }
    if (info->max_ctas_per_sm > 0 && n > info->max_ctas_per_sm) n = info->max_ctas_per_sm;
    return n > 0 ? n : 1;
}

// CTAs the encoder wants: enough for every block, at most what stays resident.
long long wanted_ctas(const EncodeKernelInfo* info, int L, int k, int T, long long n_blocks,
                      int sms)
{
    const long long by_blocks = (n_blocks + info->nteam - 1) / info->nteam;
    const long long resident = (long long)(sms > 0 ? sms : 148) * ctas_per_sm(info, L, k, T);
    return by_blocks < resident ? by_blocks : resident;
}

long long bcjr_grid(int L, int k, long long n_blocks, tcq_dtype dt, int sms)
{
    const long long resident =
        (long long)(sms > 0 ? sms : 148) * bcjr_ctas_per_sm(L, k, table_dtype(dt) == TCQ_F16 ? 1 : 0);
    return n_blocks < resident ? n_blocks : resident;
}

// Plans the grid for an encode whose arguments are filled in (all but the
// workspace) and launches it.
tcq_status run_encode(EncodeArgs& a, tcq_dtype cb_dtype, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream)
{
    const EncodeKernelInfo* info = select_kernel(a.L, a.K, a.T, cb_dtype);
    if (!info) return TCQ_ERR_INTERNAL;
    const size_t slot = info->slot_bytes(a.L, a.K, a.T);
    const int sms = current_sms();
    if (sms <= 0) return TCQ_ERR_CUDA;
    long long grid = wanted_ctas(info, a.L, a.K, a.T, a.n_blocks, sms);
    if (slot > 0) {
        const long long fit = (long long)(workspace_bytes / slot);
        if (fit < 1) return TCQ_ERR_WORKSPACE;
        if (grid > fit) grid = fit;
    }
    if (grid < 1) grid = 1;
    a.ws = static_cast<unsigned char*>(workspace);
    a.slot_bytes = slot;
    cudaError_t e = info->launch(a, (int)grid, stream);
    // the backpointers are dead once traced: drop them from L2 unwritten
    if (e == cudaSuccess) e = launch_discard_l2(workspace, (size_t)grid * slot, sms, stream);
    return e == cudaSuccess ? TCQ_OK : TCQ_ERR_CUDA;
}

// Vector trellis shapes: V weights per step, k V bits per step (at most 8,
// one backpointer byte), V | T.
tcq_status check_vec_shape(int L, int k, int V, int T)
{
    if (V < 1 || V > 8 || k < 1 || k > TCQ_MAX_K || k * V > 8 || k * V > L || L > TCQ_MAX_L)
        return TCQ_ERR_UNSUPPORTED;
    if (T < 1 || T > TCQ_MAX_T || T % V != 0) return TCQ_ERR_UNSUPPORTED;
    return TCQ_OK;
}

// run_encode for a caller's codebook of any dtype (a computed code is written
// to the front of the workspace first).
tcq_status resolve_and_encode(EncodeArgs& a, tcq_dtype dt, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream)
{
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    const tcq_status r = resolve_table(a.cb, dt, a.L, ws, workspace_bytes, stream);
    if (r != TCQ_OK) return r;
    a.cb_f16 = code_mode(dt);
    return run_encode(a, dt, ws, workspace_bytes, stream);
}

}  // namespace

extern "C" {

int tcq_words_per_block(int k, int T)
{
    if (k < 1 || k > TCQ_MAX_K || T < 1 || T > TCQ_MAX_T) return -1;
    return (int)(((long long)T * k + 31) / 32);
}

size_t tcq_encode_workspace_bytes(int L, int k, int T, int64_t n_blocks, tcq_dtype cb_dtype)
{
    if (check_shape(L, k, T) != TCQ_OK || n_blocks <= 0 || !valid_dtype(cb_dtype)) return 0;
    const EncodeKernelInfo* info = select_kernel(L, k, T, cb_dtype);
    const long long ctas = wanted_ctas(info, L, k, T, n_blocks, current_sms());
    return mad_table_bytes(L, cb_dtype) + (size_t)ctas * info->slot_bytes(L, k, T);
}

const char* tcq_encode_path(int L, int k, tcq_dtype cb_dtype)
{
    if (check_shape(L, k, 1) != TCQ_OK || !valid_dtype(cb_dtype)) return "unsupported";
    return select_kernel(L, k, 1, cb_dtype)->name;  // blocks of few steps
}

tcq_status tcq_encode(const float* x, const float* d, const void* codebook, tcq_dtype cb_dtype,
                      int L, int k, int T, int64_t n_blocks, uint32_t* start_state,
                      uint32_t* bits, float* path_cost, void* workspace, size_t workspace_bytes,
                      tcq_stream_t stream)
{
    if (n_blocks < 0) return TCQ_ERR_INVALID_ARG;
    if (!valid_dtype(cb_dtype)) return TCQ_ERR_INVALID_ARG;
    const tcq_status shape = check_shape(L, k, T);
    if (shape != TCQ_OK) return shape;
    if (n_blocks == 0) return TCQ_OK;
    if (!x || !codebook_ok(codebook, cb_dtype) || !start_state || !bits || !path_cost ||
        !workspace)
        return TCQ_ERR_INVALID_ARG;
    if (!aligned(x, 4) || (d && !aligned(d, 4)) || !aligned(start_state, 4) ||
        !aligned(bits, 4) || !aligned(path_cost, 4) || !aligned(workspace, 256))
        return TCQ_ERR_INVALID_ARG;
    if ((unsigned long long)n_blocks > (1ull << 40)) return TCQ_ERR_INVALID_ARG;

    EncodeArgs a;
    a.x = x;
    a.d = d;
    a.cb = codebook;
    a.cb_f16 = cb_dtype == TCQ_F16 ? 1 : 0;
    a.L = L;
    a.K = k;
    a.T = T;
    a.W = tcq_words_per_block(k, T);
    a.n_blocks = n_blocks;
    a.start_state = start_state;
    a.bits = bits;
    a.path_cost = path_cost;
    a.x_stride = T;
    a.d_stride = T;
    a.out_stride = 1;
    a.fixed_start = nullptr;
    return resolve_and_encode(a, cb_dtype, workspace, workspace_bytes,
                              reinterpret_cast<cudaStream_t>(stream));
}

tcq_status tcq_encode_fixed_start(const float* x, const float* d, const void* codebook,
                                  tcq_dtype cb_dtype, int L, int k, int T, int64_t n_blocks,
                                  const uint32_t* fixed_start, uint32_t* start_state,
                                  uint32_t* bits, float* path_cost, void* workspace,
                                  size_t workspace_bytes, tcq_stream_t stream)
{
    if (n_blocks > 0 && (!fixed_start || !aligned(fixed_start, 4))) return TCQ_ERR_INVALID_ARG;
    if (n_blocks < 0) return TCQ_ERR_INVALID_ARG;
    if (!valid_dtype(cb_dtype)) return TCQ_ERR_INVALID_ARG;
    const tcq_status shape = check_shape(L, k, T);
    if (shape != TCQ_OK) return shape;
    if (n_blocks == 0) return TCQ_OK;
    if (!x || !codebook_ok(codebook, cb_dtype) || !start_state || !bits || !path_cost ||
        !workspace)
        return TCQ_ERR_INVALID_ARG;
    if (!aligned(x, 4) || (d && !aligned(d, 4)) || !aligned(start_state, 4) ||
        !aligned(bits, 4) || !aligned(path_cost, 4) || !aligned(workspace, 256))
        return TCQ_ERR_INVALID_ARG;
    if ((unsigned long long)n_blocks > (1ull << 40)) return TCQ_ERR_INVALID_ARG;
    EncodeArgs a;
    a.x = x;
    a.d = d;
    a.cb = codebook;
    a.cb_f16 = cb_dtype == TCQ_F16 ? 1 : 0;
    a.L = L;
    a.K = k;
    a.T = T;
    a.W = tcq_words_per_block(k, T);
    a.n_blocks = n_blocks;
    a.start_state = start_state;
    a.bits = bits;
    a.path_cost = path_cost;
    a.x_stride = T;
    a.d_stride = T;
    a.out_stride = 1;
    a.fixed_start = fixed_start;
    return resolve_and_encode(a, cb_dtype, workspace, workspace_bytes,
                              reinterpret_cast<cudaStream_t>(stream));
}

tcq_status tcq_decode(const uint32_t* bits, const uint32_t* start_state, const void* codebook,
                      tcq_dtype cb_dtype, int L, int k, int T, int64_t n_blocks, float* y,
                      tcq_stream_t stream)
{
    if (n_blocks < 0) return TCQ_ERR_INVALID_ARG;
    if (!valid_dtype(cb_dtype)) return TCQ_ERR_INVALID_ARG;
    const tcq_status shape = check_shape(L, k, T);
    if (shape != TCQ_OK) return shape;
    if (n_blocks == 0) return TCQ_OK;
    if (!bits || !start_state || !codebook_ok(codebook, cb_dtype) || !y) return TCQ_ERR_INVALID_ARG;
    if (!aligned(bits, 4) || !aligned(start_state, 4) || !aligned(y, 4)) return TCQ_ERR_INVALID_ARG;
    if ((unsigned long long)n_blocks > (1ull << 40)) return TCQ_ERR_INVALID_ARG;
    const int sms = current_sms();
    if (sms <= 0) return TCQ_ERR_CUDA;

    DecodeArgs a;
    a.bits = bits;
    a.start_state = start_state;
    a.cb = codebook;
    a.cb_f16 = code_mode(cb_dtype);
    a.L = L;
    a.K = k;
    a.T = T;
    a.W = tcq_words_per_block(k, T);
    a.n_blocks = n_blocks;
    a.y = y;
    a.in_stride = 1;
    a.y_stride = T;
    const cudaError_t e = launch_decode(a, sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TCQ_OK : TCQ_ERR_CUDA;
}

tcq_status tcq_gemv(const uint32_t* bits, const uint32_t* start_state, const float* scale,
                    const void* codebook, tcq_dtype cb_dtype, int L, int k, int T, int64_t rows,
                    int64_t cols, const float* x, float* y, tcq_stream_t stream)
{
    if (rows < 0 || cols < 0) return TCQ_ERR_INVALID_ARG;
    if (!valid_dtype(cb_dtype)) return TCQ_ERR_INVALID_ARG;
    const tcq_status shape = check_shape(L, k, T);
    if (shape != TCQ_OK) return shape;
    if (T % 4 != 0) return TCQ_ERR_UNSUPPORTED;
    if (cb_dtype == TCQ_F32 && L >= 15) return TCQ_ERR_UNSUPPORTED;  // table must fit in smem
    if (cols % T != 0) return TCQ_ERR_INVALID_ARG;
    if (rows == 0) return TCQ_OK;
    if (cols > ((int64_t)1 << 31)) return TCQ_ERR_INVALID_ARG;
    if (!bits || !start_state || !codebook_ok(codebook, cb_dtype) || !x || !y)
        return TCQ_ERR_INVALID_ARG;
    if (!aligned(bits, 4) || !aligned(start_state, 4) || (scale && !aligned(scale, 4)) ||
        !aligned(x, 16) || !aligned(y, 4))
        return TCQ_ERR_INVALID_ARG;
    if ((unsigned long long)rows * (unsigned long long)(cols / T) > (1ull << 40))
        return TCQ_ERR_INVALID_ARG;
    const int sms = current_sms();
    if (sms <= 0) return TCQ_ERR_CUDA;
    GemvArgs a;
    a.bits = bits;
    a.start_state = start_state;
    a.scale = scale;
    a.cb = codebook;
    a.cb_f16 = code_mode(cb_dtype);
    a.L = L;
    a.K = k;
    a.T = T;
    a.W = tcq_words_per_block(k, T);
    a.rows = rows;
    a.cols = cols;
    a.x = x;
    a.y = y;
    const cudaError_t e = launch_gemv(a, sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TCQ_OK : TCQ_ERR_CUDA;
}

size_t tcq_ldlq_workspace_bytes(int L, int k, int T, int64_t rows, int64_t cols,
                                tcq_dtype cb_dtype)
{
    if (check_shape(L, k, T) != TCQ_OK || rows <= 0 || cols <= 0 || cols % T != 0 ||
        !valid_dtype(cb_dtype))
        return 0;
    const size_t enc = tcq_encode_workspace_bytes(L, k, T, rows, cb_dtype);
    const size_t targets = ((size_t)rows * (size_t)T * sizeof(float) + 255) & ~(size_t)255;
    return targets + enc;
}

tcq_status tcq_ldlq(const float* w, const float* u, const float* d, const void* codebook,
                    tcq_dtype cb_dtype, int L, int k, int T, int64_t rows, int64_t cols, float* q,
                    float* x, uint32_t* start_state, uint32_t* bits, float* path_cost,
                    void* workspace, size_t workspace_bytes, tcq_stream_t stream)
{
    if (rows < 0 || cols < 0) return TCQ_ERR_INVALID_ARG;
    if (!valid_dtype(cb_dtype)) return TCQ_ERR_INVALID_ARG;
    const tcq_status shape = check_shape(L, k, T);
    if (shape != TCQ_OK) return shape;
    if (cols % T != 0) return TCQ_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return TCQ_OK;
    if (!w || !u || !codebook_ok(codebook, cb_dtype) || !q || !start_state || !bits ||
        !path_cost || !workspace)
        return TCQ_ERR_INVALID_ARG;
    if (!aligned(w, 4) || !aligned(u, 4) || (d && !aligned(d, 4)) || !aligned(q, 4) ||
        (x && !aligned(x, 4)) || !aligned(start_state, 4) || !aligned(bits, 4) ||
        !aligned(path_cost, 4) || !aligned(workspace, 256))
        return TCQ_ERR_INVALID_ARG;
    // grid rows of the feedback product, and the block count of the code
    if (rows > 65535LL * 128 || cols >= ((int64_t)1 << 31)) return TCQ_ERR_INVALID_ARG;
    const size_t targets = ((size_t)rows * (size_t)T * sizeof(float) + 255) & ~(size_t)255;
    if (workspace_bytes <= targets + mad_table_bytes(L, cb_dtype)) return TCQ_ERR_WORKSPACE;
    const int sms = current_sms();
    if (sms <= 0) return TCQ_ERR_CUDA;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    const tcq_status rt = resolve_table(codebook, cb_dtype, L, ws, workspace_bytes, st);
    if (rt != TCQ_OK) return rt;
    const int64_t nb = cols / T;
    const int W = tcq_words_per_block(k, T);
    // targets of the current column block: x[:, B] when the caller keeps them,
    // else the front of the workspace
    float* xbuf = x ? x : reinterpret_cast<float*>(ws);
    const long long x_ld = x ? cols : T;
    unsigned int* err = device_error_word(st);  // where a feedback give-up is reported

    for (int64_t j = 0; j < nb; ++j) {
        const long long c0 = j * (long long)T;
        FeedbackArgs f;
        f.w = w;
        f.q = q;
        f.u = u;
        f.rows = rows;
        f.cols = cols;
        f.c0 = c0;
        f.n = T;
        f.x = x ? xbuf + c0 : xbuf;
        f.x_ld = x_ld;
        f.err = err;
        if (launch_feedback(f, st) != cudaSuccess) return TCQ_ERR_CUDA;

        EncodeArgs a;
        a.x = f.x;
        a.d = d ? d + c0 : nullptr;
        a.cb = codebook;
        a.cb_f16 = code_mode(cb_dtype);
        a.L = L;
        a.K = k;
        a.T = T;
        a.W = W;
        a.n_blocks = rows;
        a.start_state = start_state + j;
        a.bits = bits + j * W;
        a.path_cost = path_cost + j;
        a.x_stride = x_ld;
        a.d_stride = 0;
        a.out_stride = nb;
        a.fixed_start = nullptr;
        const tcq_status es = run_encode(a, cb_dtype, ws + targets, workspace_bytes - targets, st);
        if (es != TCQ_OK) return es;

        DecodeArgs dq;
        dq.bits = bits + j * W;
        dq.start_state = start_state + j;
        dq.cb = codebook;
        dq.cb_f16 = a.cb_f16;
        dq.L = L;
        dq.K = k;
        dq.T = T;
        dq.W = W;
        dq.n_blocks = rows;
        dq.y = q + c0;
        dq.in_stride = nb;
        dq.y_stride = cols;
        if (launch_decode(dq, sms, st) != cudaSuccess) return TCQ_ERR_CUDA;
    }
    return TCQ_OK;
}

size_t tcq_bcjr_workspace_bytes(int L, int k, int T, int64_t n_blocks, tcq_dtype cb_dtype)
{
    if (check_shape(L, k, T) != TCQ_OK || n_blocks <= 0 || !valid_dtype(cb_dtype)) return 0;
    return mad_table_bytes(L, cb_dtype) +
           (size_t)bcjr_grid(L, k, n_blocks, cb_dtype, current_sms()) * bcjr_slot_bytes(L, k, T);
}

tcq_status tcq_bcjr(const float* x, const float* d, const void* codebook, tcq_dtype cb_dtype,
                    int L, int k, int T, int64_t n_blocks, float tau, float* y_soft,
                    float* free_energy, void* workspace, size_t workspace_bytes,
                    tcq_stream_t stream)
{
    if (n_blocks < 0) return TCQ_ERR_INVALID_ARG;
    if (!valid_dtype(cb_dtype)) return TCQ_ERR_INVALID_ARG;
    const tcq_status shape = check_shape(L, k, T);
    if (shape != TCQ_OK) return shape;
    if (!(tau > 0.f) || !(tau < INFINITY)) return TCQ_ERR_INVALID_ARG;
    if (n_blocks == 0) return TCQ_OK;
    if (!x || !codebook_ok(codebook, cb_dtype) || !y_soft || !workspace) return TCQ_ERR_INVALID_ARG;
    if (!aligned(x, 4) || (d && !aligned(d, 4)) || !aligned(y_soft, 4) ||
        (free_energy && !aligned(free_energy, 4)) || !aligned(workspace, 256))
        return TCQ_ERR_INVALID_ARG;
    if ((unsigned long long)n_blocks > (1ull << 40)) return TCQ_ERR_INVALID_ARG;
    const float w_scale = (float)(1.4426950408889634 / (double)tau);
    if (!(w_scale < INFINITY)) return TCQ_ERR_INVALID_ARG;
    const int sms = current_sms();
    if (sms <= 0) return TCQ_ERR_CUDA;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    const tcq_status rt = resolve_table(codebook, cb_dtype, L, ws, workspace_bytes,
                                        reinterpret_cast<cudaStream_t>(stream));
    if (rt != TCQ_OK) return rt;
    const size_t slot = bcjr_slot_bytes(L, k, T);
    long long grid = bcjr_grid(L, k, n_blocks, cb_dtype, sms);
    const long long fit = (long long)(workspace_bytes / slot);
    if (fit < 1) return TCQ_ERR_WORKSPACE;
    if (grid > fit) grid = fit;
    if (grid < 1) grid = 1;
    BcjrArgs a;
    a.x = x;
    a.d = d;
    a.cb = codebook;
    a.cb_f16 = cb_dtype == TCQ_F16 ? 1 : 0;
    a.L = L;
    a.K = k;
    a.T = T;
    a.n_blocks = n_blocks;
    a.w_scale = w_scale;
    a.tau_ln2 = (double)tau * 0.6931471805599453;
    a.y = y_soft;
    a.free_energy = free_energy;
    a.ws = ws;
    a.slot_bytes = slot;
    const cudaError_t e = launch_bcjr(a, (int)grid, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TCQ_OK : TCQ_ERR_CUDA;
}

size_t tcq_encode_vec_workspace_bytes(int L, int k, int V, int T, int64_t n_blocks,
                                      tcq_dtype cb_dtype)
{
    if (V == 1) return tcq_encode_workspace_bytes(L, k, T, n_blocks, cb_dtype);
    if (check_vec_shape(L, k, V, T) != TCQ_OK || n_blocks <= 0 ||
        (cb_dtype != TCQ_F32 && cb_dtype != TCQ_F16))
        return 0;
    // enough for whichever kernel the encode picks (the compile-time one needs a
    // 4-byte aligned codebook, which the query cannot see)
    size_t need = 0;
    for (const EncodeKernelInfo* info : {find_vec_kernel(L, k, V, cb_dtype == TCQ_F16 ? 1 : 0),
                                         generic_kernel_info(L, k * V)}) {
        if (!info) continue;
        const long long ctas = wanted_ctas(info, L, k * V, T / V, n_blocks, current_sms());
        const size_t b = (size_t)ctas * info->slot_bytes(L, k * V, T / V);
        if (b > need) need = b;
    }
    return need;
}

tcq_status tcq_encode_vec(const float* x, const float* d, const void* codebook, tcq_dtype cb_dtype,
                          int L, int k, int V, int T, int64_t n_blocks, uint32_t* start_state,
                          uint32_t* bits, float* path_cost, void* workspace,
                          size_t workspace_bytes, tcq_stream_t stream)
{
    if (V == 1)
        return tcq_encode(x, d, codebook, cb_dtype, L, k, T, n_blocks, start_state, bits,
                          path_cost, workspace, workspace_bytes, stream);
    if (n_blocks < 0) return TCQ_ERR_INVALID_ARG;
    if (cb_dtype == TCQ_MAD) return TCQ_ERR_UNSUPPORTED;  // the computed code is scalar
    if (!valid_dtype(cb_dtype)) return TCQ_ERR_INVALID_ARG;
    const tcq_status shape = check_vec_shape(L, k, V, T);
    if (shape != TCQ_OK) return shape;
    if (n_blocks == 0) return TCQ_OK;
    if (!x || !codebook_ok(codebook, cb_dtype) || !start_state || !bits || !path_cost ||
        !workspace)
        return TCQ_ERR_INVALID_ARG;
    if (!aligned(x, 4) || (d && !aligned(d, 4)) || !aligned(start_state, 4) ||
        !aligned(bits, 4) || !aligned(path_cost, 4) || !aligned(workspace, 256))
        return TCQ_ERR_INVALID_ARG;
    if ((unsigned long long)n_blocks > (1ull << 40)) return TCQ_ERR_INVALID_ARG;
    const EncodeKernelInfo* info =
        find_vec_kernel(L, k, V, cb_dtype == TCQ_F16 && aligned(codebook, 4) ? 1 : 0);
    if (!info) info = generic_kernel_info(L, k * V);
    if (!info) return TCQ_ERR_INTERNAL;
    const int sms = current_sms();
    if (sms <= 0) return TCQ_ERR_CUDA;
    const size_t slot = info->slot_bytes(L, k * V, T / V);
    long long grid = wanted_ctas(info, L, k * V, T / V, n_blocks, sms);
    const long long fit = (long long)(workspace_bytes / slot);
    if (fit < 1) return TCQ_ERR_WORKSPACE;
    if (grid > fit) grid = fit;
    if (grid < 1) grid = 1;
    EncodeArgs a;
    a.x = x;
    a.d = d;
    a.cb = codebook;
    a.cb_f16 = cb_dtype == TCQ_F16 ? 1 : 0;
    a.L = L;
    a.K = k;
    a.T = T;
    a.W = tcq_words_per_block(k, T);
    a.n_blocks = n_blocks;
    a.start_state = start_state;
    a.bits = bits;
    a.path_cost = path_cost;
    a.x_stride = T;
    a.d_stride = T;
    a.out_stride = 1;
    a.fixed_start = nullptr;
    a.V = V;
    a.ws = static_cast<unsigned char*>(workspace);
    a.slot_bytes = slot;
    cudaError_t e = info->launch(a, (int)grid, reinterpret_cast<cudaStream_t>(stream));
    if (e == cudaSuccess)  // dead backpointers: drop them from L2 unwritten
        e = launch_discard_l2(workspace, (size_t)grid * slot, sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TCQ_OK : TCQ_ERR_CUDA;
}

tcq_status tcq_decode_vec(const uint32_t* bits, const uint32_t* start_state, const void* codebook,
                          tcq_dtype cb_dtype, int L, int k, int V, int T, int64_t n_blocks,
                          float* y, tcq_stream_t stream)
{
    if (V == 1) return tcq_decode(bits, start_state, codebook, cb_dtype, L, k, T, n_blocks, y, stream);
    if (n_blocks < 0) return TCQ_ERR_INVALID_ARG;
    if (cb_dtype == TCQ_MAD) return TCQ_ERR_UNSUPPORTED;
    if (!valid_dtype(cb_dtype)) return TCQ_ERR_INVALID_ARG;
    const tcq_status shape = check_vec_shape(L, k, V, T);
    if (shape != TCQ_OK) return shape;
    if (n_blocks == 0) return TCQ_OK;
    if (!bits || !start_state || !codebook_ok(codebook, cb_dtype) || !y) return TCQ_ERR_INVALID_ARG;
    if (!aligned(bits, 4) || !aligned(start_state, 4) || !aligned(y, 4)) return TCQ_ERR_INVALID_ARG;
    if ((unsigned long long)n_blocks > (1ull << 40)) return TCQ_ERR_INVALID_ARG;
    const int sms = current_sms();
    if (sms <= 0) return TCQ_ERR_CUDA;
    DecodeArgs a;
    a.bits = bits;
    a.start_state = start_state;
    a.cb = codebook;
    a.cb_f16 = cb_dtype == TCQ_F16 ? 1 : 0;
    a.L = L;
    a.K = k * V;
    a.T = T;
    a.W = tcq_words_per_block(k, T);
    a.n_blocks = n_blocks;
    a.y = y;
    a.in_stride = 1;
    a.y_stride = T;
    const cudaError_t e = launch_decode_vec(a, V, sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TCQ_OK : TCQ_ERR_CUDA;
}

tcq_status tcq_gemv_vec(const uint32_t* bits, const uint32_t* start_state, const float* scale,
                        const void* codebook, tcq_dtype cb_dtype, int L, int k, int V, int T,
                        int64_t rows, int64_t cols, const float* x, float* y, tcq_stream_t stream)
{
    if (V == 1)
        return tcq_gemv(bits, start_state, scale, codebook, cb_dtype, L, k, T, rows, cols, x, y,
                        stream);
    if (rows < 0 || cols < 0) return TCQ_ERR_INVALID_ARG;
    if (cb_dtype == TCQ_MAD) return TCQ_ERR_UNSUPPORTED;  // the computed code is scalar
    if (!valid_dtype(cb_dtype)) return TCQ_ERR_INVALID_ARG;
    const tcq_status shape = check_vec_shape(L, k, V, T);
    if (shape != TCQ_OK) return shape;
    if (cols % T != 0) return TCQ_ERR_INVALID_ARG;
    if (rows == 0) return TCQ_OK;
    if (cols > ((int64_t)1 << 31)) return TCQ_ERR_INVALID_ARG;
    if (!bits || !start_state || !codebook_ok(codebook, cb_dtype) || !x || !y)
        return TCQ_ERR_INVALID_ARG;
    if (!aligned(bits, 4) || !aligned(start_state, 4) || (scale && !aligned(scale, 4)) ||
        !aligned(x, 16) || !aligned(y, 4))
        return TCQ_ERR_INVALID_ARG;
    if ((unsigned long long)rows * (unsigned long long)(cols / T) > (1ull << 40))
        return TCQ_ERR_INVALID_ARG;
    const int sms = current_sms();
    if (sms <= 0) return TCQ_ERR_CUDA;
    GemvArgs a;
    a.bits = bits;
    a.start_state = start_state;
    a.scale = scale;
    a.cb = codebook;
    a.cb_f16 = cb_dtype == TCQ_F16 ? 1 : 0;
    a.L = L;
    a.K = k * V;
    a.T = T;
    a.W = tcq_words_per_block(k, T);
    a.rows = rows;
    a.cols = cols;
    a.x = x;
    a.y = y;
    const cudaError_t e = launch_gemv_vec(a, V, sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TCQ_OK : TCQ_ERR_CUDA;
}

int tcq_ub8_words_per_block(int V, int m, int T)
{
    if (V < 1 || V > TCQ_UB8_MAX_V || m < 0 || m > TCQ_UB8_MAX_M || T < 1 || T % V != 0 ||
        T / V > TCQ_UB8_MAX_STEPS)
        return -1;
    return (T / V * (1 + m) + 31) / 32;
}

tcq_status tcq_ub8_encode(const float* x, const float* d, const void* codebook, tcq_dtype cb_dtype,
                          int V, int m, int T, int64_t n_blocks, const uint32_t* fixed_start,
                          uint32_t* start_state, uint32_t* bits, float* path_cost,
                          tcq_stream_t stream)
{
    if (n_blocks < 0) return TCQ_ERR_INVALID_ARG;
    if (!valid_dtype(cb_dtype)) return TCQ_ERR_INVALID_ARG;
    if (cb_dtype == TCQ_MAD) return TCQ_ERR_UNSUPPORTED;  // the union codebook is a table
    const int W = tcq_ub8_words_per_block(V, m, T);
    if (W < 0) return TCQ_ERR_UNSUPPORTED;
    if (n_blocks == 0) return TCQ_OK;
    if (!x || !codebook_ok(codebook, cb_dtype) || !start_state || !bits || !path_cost)
        return TCQ_ERR_INVALID_ARG;
    if (!aligned(x, 4) || (d && !aligned(d, 4)) || (fixed_start && !aligned(fixed_start, 4)) ||
        !aligned(start_state, 4) || !aligned(bits, 4) || !aligned(path_cost, 4))
        return TCQ_ERR_INVALID_ARG;
    if ((unsigned long long)n_blocks > (1ull << 40)) return TCQ_ERR_INVALID_ARG;
    const int sms = current_sms();
    if (sms <= 0) return TCQ_ERR_CUDA;
    Ub8EncodeArgs a;
    a.x = x;
    a.d = d;
    a.cb = codebook;
    a.cb_f16 = cb_dtype == TCQ_F16 ? 1 : 0;
    a.V = V;
    a.m = m;
    a.T = T;
    a.W = W;
    a.n_blocks = n_blocks;
    a.fixed_start = fixed_start;
    a.start_state = start_state;
    a.bits = bits;
    a.path_cost = path_cost;
    const cudaError_t e = launch_ub8_encode(a, sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TCQ_OK : TCQ_ERR_CUDA;
}

tcq_status tcq_ub8_decode(const uint32_t* bits, const uint32_t* start_state, const void* codebook,
                          tcq_dtype cb_dtype, int V, int m, int T, int64_t n_blocks, float* y,
                          tcq_stream_t stream)
{
    if (n_blocks < 0) return TCQ_ERR_INVALID_ARG;
    if (!valid_dtype(cb_dtype)) return TCQ_ERR_INVALID_ARG;
    if (cb_dtype == TCQ_MAD) return TCQ_ERR_UNSUPPORTED;
    const int W = tcq_ub8_words_per_block(V, m, T);
    if (W < 0) return TCQ_ERR_UNSUPPORTED;
    if (n_blocks == 0) return TCQ_OK;
    if (!bits || !start_state || !codebook_ok(codebook, cb_dtype) || !y) return TCQ_ERR_INVALID_ARG;
    if (!aligned(bits, 4) || !aligned(start_state, 4) || !aligned(y, 4)) return TCQ_ERR_INVALID_ARG;
    if ((unsigned long long)n_blocks > (1ull << 40)) return TCQ_ERR_INVALID_ARG;
    const int sms = current_sms();
    if (sms <= 0) return TCQ_ERR_CUDA;
    Ub8DecodeArgs a;
    a.bits = bits;
    a.start_state = start_state;
    a.cb = codebook;
    a.cb_f16 = cb_dtype == TCQ_F16 ? 1 : 0;
    a.V = V;
    a.m = m;
    a.T = T;
    a.W = W;
    a.n_blocks = n_blocks;
    a.y = y;
    const cudaError_t e = launch_ub8_decode(a, sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TCQ_OK : TCQ_ERR_CUDA;
}

const char* tcq_status_string(tcq_status status)
{
    switch (status) {
    case TCQ_OK: return "TCQ_OK";
    case TCQ_ERR_INVALID_ARG: return "TCQ_ERR_INVALID_ARG: null or misaligned pointer, or bad size";
    case TCQ_ERR_UNSUPPORTED: return "TCQ_ERR_UNSUPPORTED: L, k or T outside the supported ranges";
    case TCQ_ERR_WORKSPACE: return "TCQ_ERR_WORKSPACE: workspace smaller than one CTA's share";
    case TCQ_ERR_CUDA: return "TCQ_ERR_CUDA: a CUDA runtime call or kernel launch failed";
    case TCQ_ERR_INTERNAL: return "TCQ_ERR_INTERNAL: library invariant violated";
    }
    return "unknown tcq_status";
}

}  // extern "C"
