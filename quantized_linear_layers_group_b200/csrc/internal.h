// internal.h -- declarations shared by the library's translation units (not
// part of the public ABI; see include/qlin.h for that).
#pragma once
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "qlin.h"

namespace qlin {

constexpr int kNumSMsB200 = 148;
// Split-K tickets live in a fixed-size prefix of the workspace, so that no
// call's partial tiles ever overlap another call's ticket words.
constexpr size_t kTicketBytes = 65536;
constexpr int64_t kMaxSplitTiles = kTicketBytes / 4;
// Cluster Split-K (Swap-AB): the S segments of a tile run on the S CTAs of a
// thread-block cluster and meet in rank 0's shared memory; the receive area
// holds S-1 segments, so S is bounded per tile width.
#define QLIN_MAX_CLUSTER 8
__host__ __device__ constexpr int cluster_split_max(int tile_n) {
    return tile_n == 16 ? 8 : (tile_n == 32 || tile_n == 64) ? 4 : 0;
}

// Kernel variants of one (format, orientation, tile_n).
enum GemmMode : int {
    kModeStd = 0,      // operands from global memory by TMA; Split-K through the workspace
    kModeCluster = 1,  // Swap-AB Split-K reduced through a thread-block cluster
    kModeFused = 2,    // Swap-AB with the activation quantisation done by the GEMM itself
    kModePair = 3,     // plain 256-row tiles on a pair of CTAs (cluster of 2, cta_group::2 MMA)
};
// Fused mode keeps the unit's activation codes resident: 64 KiB of shared
// memory, so at most this many K blocks per unit.
__host__ __device__ constexpr int fused_max_kblocks(int tile_n) { return tile_n > 0 ? 65536 / (tile_n * 128) : 0; }

// ---------------------------------------------------------------- quantise
cudaError_t launch_quantize_per_token(int fmt, const void* x, int64_t rows, int64_t cols, int64_t ld, void* q,
                                      float* s, bool pdl, cudaStream_t st);
cudaError_t launch_quantize_block(const void* x, int64_t rows, int64_t cols, int64_t ld, int block_rows, void* q,
                                  float* s, bool pdl, cudaStream_t st);
// MXFP8 / NVFP4 codes and tiled scale factors (g: NVFP4's device-side decode scale)
cudaError_t launch_quantize_block_scaled(int fmt, const void* x, int64_t rows, int64_t cols, int64_t ld,
                                         const float* g, void* q, void* sf, bool pdl, cudaStream_t st);
__host__ __device__ constexpr bool is_block_scaled(int fmt) { return fmt == QLIN_FMT_MXFP8 || fmt == QLIN_FMT_NVFP4; }

// ------------------------------------------------------------------- GEMM
// A fully resolved GEMM launch: which operand feeds the 128-row MMA side
// ("P") and which the narrow side ("Q", tile_n rows), how K is segmented and
// whether the segments of one tile run in separate CTAs.
struct GemmPlan {
    int fmt = 0;
    bool swap = false;    // P = W (rows of N), Q = A (rows of M)
    bool spread = false;  // Split-K: one work unit per (tile, segment)
    int mode = kModeStd;  // GemmMode
    int tile_n = 0;       // Q rows per tile (MMA N)
    int k_segments = 1;   // S
    int stages = 0;
    int64_t M = 0, N = 0, K = 0;
    int64_t p_rows = 0, q_rows = 0;
    int64_t p_tiles = 0, q_tiles = 0, num_tiles = 0, units = 0;
    int64_t k_bytes = 0;   // bytes of one operand row: K (8-bit) or 2K (bf16)
    int kblocks = 0;       // k_bytes / 128: K blocks of 128 bytes
    int kb_per_seg = 0;    // kblocks / S
    int kb_per_unit = 0;   // K blocks one work unit covers
    int grid = 0;          // persistent CTAs
    size_t smem_bytes = 0;
    size_t ticket_bytes = 0;   // workspace prefix holding the per-tile tickets
    size_t workspace_bytes = 0;
    int moe_E = 0;             // MoE grouped GEMM: experts (units counted on the device)
};

// Grouped GEMM over experts (MoE): R rows of A / C grouped by expert, W [E N,
// K]; the per-expert tile counts are only known on the device.
qlin_status make_moe_plan(int fmt, int variant, int tile_n, int64_t R, int E, int64_t N, int64_t K, int num_sms,
                          GemmPlan* plan);
constexpr int kMoeMaxE = 255;  // experts the kernel's shared-memory table holds

// Validates the (fmt, tile_n, S, variant) combination and fills the plan.
// want_mode kModeCluster: a Swap-AB Split-K whose S fits one cluster reduces
// through the cluster; kModeFused: a Swap-AB plan whose units fit the
// resident activation operand quantises its own activations (otherwise the
// plan keeps kModeStd).  Returns QLIN_OK or an error status; touches no
// device state.
qlin_status make_gemm_plan(int fmt, int variant, int tile_n, int k_segments, int64_t M, int64_t N, int64_t K,
                           int num_sms, int want_mode, GemmPlan* plan);

// Shared-memory pipeline depth and dynamic smem size of the GEMM kernel
// instantiation for (fmt, orientation, tile_n, mode); false if none exists.
bool gemm_kernel_info(int fmt, bool swap, int tile_n, int mode, int* stages, size_t* smem_bytes);

struct GemmOperands {
    const void* a_q;   // fused mode: written (codes), not read
    const float* s_a;  // fused mode: written (scales), not read
    const void* w_q;
    const float* s_w;
    const void* bias;
    void* c;
    bool out_i32;
    void* workspace;
    bool pdl;  // launch as a programmatic dependent of the previous kernel
    const void* x = nullptr;  // fused mode: bf16 activations [M, K], row stride ld_x elements
    int64_t ld_x = 0;
    const int32_t* moe_offsets = nullptr;  // MoE: expert row offsets [E + 1] (device)
    // block-scaled formats: tiled scale factors of A and W (s_a / s_w then
    // point at the NVFP4 per-tensor decode scales, or are null for MXFP8)
    const void* sf_a = nullptr;
    const void* sf_w = nullptr;
};

// ------------------------------------------------------------------- MoE
cudaError_t launch_moe_route(const float* logits, int T, int E, int k, int32_t* ids, float* w, int32_t* offsets,
                             int32_t* rows, bool pdl, cudaStream_t st);
cudaError_t launch_moe_quantize_scatter(const void* x, int T, int H, int k, const int32_t* rows, void* a_q,
                                        float* s_a, bool pdl, cudaStream_t st);
cudaError_t launch_moe_act_quantize(const void* g, int R, int I, void* h_q, float* s_h, bool pdl, cudaStream_t st);
cudaError_t launch_moe_combine(const void* y, const float* w, const int32_t* rows, int T, int H, int k, void* out,
                               bool pdl, cudaStream_t st);

qlin_status launch_gemm(const GemmPlan& plan, const GemmOperands& ops, cudaStream_t st);

// Reads and clears the device status word that bounded waits set on timeout.
cudaError_t device_status_read_clear(int* value);

// Launches the failure-path self-test (a bounded wait that must give up).
cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t st);

// Shape / format preconditions shared by the GEMM entry points (M >= 0).
qlin_status check_fmt_shape(int fmt, int64_t M, int64_t N, int64_t K);

// Number of SMs of the current device (cached per device); 0 if none.
int current_device_sms();

}  // namespace qlin
