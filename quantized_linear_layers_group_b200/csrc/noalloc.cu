// noalloc.cu -- qlin_scaled_mm_noalloc: the scaled GEMM for callers that
// cannot allocate device memory.
//
// Who needs it: code that must not call cudaMalloc -- for example a kernel
// plugin loaded into a serving engine that owns the whole device-memory pool
// and forbids (or cannot account for) allocations made behind its back.  Such
// callers cannot hand qlin_scaled_mm a workspace, so the Split-K variants
// would be closed to them.
//
// What it does instead: the Split-K ticket words and partial tiles live in a
// file-scope device array of a fixed size, QLIN_NOALLOC_SCRATCH_BYTES.  Every
// GPU that loads the library holds that array until the process exits.  The
// array's host-side name is only a stand-in for the device symbol, so the
// device address is looked up once per device (with that device current) and
// cached; the first call on a device does this set-up.  Every call shares the
// one array: the ticket words are cleared on the caller's stream before each
// launch, and two calls whose kernels overlap on the GPU (different streams,
// or one stream with overlapping launches) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace qlin {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[QLIN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once per
// device).  Returns nullptr (and a CUDA status) if the lookup fails.
void* scratch_for_current_device(cudaError_t* err) {
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= kMaxDevices) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(g_setup_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (*err != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace qlin

using namespace qlin;

extern "C" qlin_status qlin_scaled_mm_noalloc(int fmt, int variant, int tile_n, int k_segments, int64_t M, int64_t N,
                                              int64_t K, const void* a_q, const float* s_a, const void* w_q,
                                              const float* s_w, const void* bias, void* c_out, uint32_t flags,
                                              qlin_stream_t stream) {
    if (fmt == QLIN_FMT_BF16 || is_block_scaled(fmt)) return QLIN_ERR_INVALID_ARG;  // as qlin_scaled_mm
    qlin_status st = check_fmt_shape(fmt, M, N, K);
    if (st != QLIN_OK) return st;
    if (flags & ~(QLIN_OUT_I32ACC | QLIN_PDL | QLIN_SPLITK_CLUSTER)) return QLIN_ERR_INVALID_ARG;
    const bool out_i32 = (flags & QLIN_OUT_I32ACC) != 0;
    if (out_i32 && fmt != QLIN_FMT_INT8) return QLIN_ERR_INVALID_ARG;
    if (fmt == QLIN_FMT_FP8_BLOCK && bias) return QLIN_ERR_INVALID_ARG;
    if (variant < QLIN_VAR_AUTO || variant > QLIN_VAR_PAIR || tile_n < 0 || k_segments < 0)
        return QLIN_ERR_INVALID_ARG;
    if (M == 0) return QLIN_OK;  // a no-op, as for qlin_scaled_mm
    if (!a_q || !s_a || !w_q || !s_w || !c_out) return QLIN_ERR_INVALID_ARG;
    if (!aligned16(a_q) || !aligned16(w_q) || !aligned16(c_out)) return QLIN_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(s_a) & 3u) || (reinterpret_cast<uintptr_t>(s_w) & 3u) ||
        (reinterpret_cast<uintptr_t>(bias) & 1u))
        return QLIN_ERR_ALIGNMENT;
    const int sms = current_device_sms();
    if (sms <= 0) return QLIN_ERR_NO_DEVICE;
    GemmPlan p;
    st = make_gemm_plan(fmt, variant, tile_n, k_segments, M, N, K, sms,
                        (flags & QLIN_SPLITK_CLUSTER) ? kModeCluster : kModeStd, &p);
    if (st != QLIN_OK) return st;
    if (p.workspace_bytes > QLIN_NOALLOC_SCRATCH_BYTES) return QLIN_ERR_WORKSPACE;  // beyond the fixed maximum
    void* scratch = nullptr;
    if (p.workspace_bytes) {
        cudaError_t err;
        scratch = scratch_for_current_device(&err);
        if (!scratch) return QLIN_ERR_CUDA;
        // the array keeps the previous call's contents: the tickets must start at zero
        if (cudaMemsetAsync(scratch, 0, p.ticket_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return QLIN_ERR_CUDA;
    }
    GemmOperands ops{a_q, s_a, w_q, s_w, bias, c_out, out_i32, scratch, (flags & QLIN_PDL) != 0};
    return launch_gemm(p, ops, static_cast<cudaStream_t>(stream));
}
