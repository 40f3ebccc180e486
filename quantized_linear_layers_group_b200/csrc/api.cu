// api.cu -- the extern "C" entry points of include/qlin.h: host-side argument
// validation, GEMM planning, the per-shape dispatch table and status codes.
//
// Dispatch follows the page "[Kernel][Perf] Add Hopper (SM90) tuned config for
// batch-invariant persistent matmul" (section "Summary": a per-shape config is
// looked up at kernel launch; the table is keyed by architecture family and
// split into M buckets) and "Helion in vLLM: A Unified Route to Tunable Linear
// Kernels" ("Algorithm choice becomes part of tuning": the variant is part of
// each per-shape entry).  The table is plain text written by the offline
// sweep:
//
//   qlin-dispatch 1
//   device <sm_count> <cc_major> <cc_minor> <device name ...>
//   # fmt N K m_max variant tile_n k_segments
//   entry fp8 4096 2048 16 swapab_splitk 16 4
//   ...
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <fstream>
#include <mutex>
#include <sstream>
#include <string>
#include <vector>

#include "internal.h"

namespace qlin {

namespace {

struct TableEntry {
    int fmt;
    int64_t N, K, m_max;
    int variant, tile_n, k_segments;
};

std::mutex g_table_mu;
std::vector<TableEntry> g_table;  // sorted by (fmt, N, K, m_max)

bool g_log = [] {
    const char* e = std::getenv("QLIN_LOG");
    return e && e[0] == '1';
}();

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

const char* fmt_name(int f) {
    switch (f) {
        case QLIN_FMT_INT8: return "int8";
        case QLIN_FMT_FP8: return "fp8";
        case QLIN_FMT_FP8_BLOCK: return "fp8_block";
        case QLIN_FMT_BF16: return "bf16";
        case QLIN_FMT_MXFP8: return "mxfp8";
        case QLIN_FMT_NVFP4: return "nvfp4";
    }
    return "?";
}

int parse_fmt(const std::string& s) {
    if (s == "int8") return QLIN_FMT_INT8;
    if (s == "fp8") return QLIN_FMT_FP8;
    if (s == "fp8_block") return QLIN_FMT_FP8_BLOCK;
    if (s == "bf16") return QLIN_FMT_BF16;
    if (s == "mxfp8") return QLIN_FMT_MXFP8;
    if (s == "nvfp4") return QLIN_FMT_NVFP4;
    return -1;
}

const char* variant_name(int v) {
    switch (v) {
        case QLIN_VAR_PLAIN: return "plain";
        case QLIN_VAR_SPLITK: return "splitk";
        case QLIN_VAR_SWAPAB: return "swapab";
        case QLIN_VAR_SWAPAB_SPLITK: return "swapab_splitk";
        case QLIN_VAR_PAIR: return "pair";
    }
    return "auto";
}

int parse_variant(const std::string& s) {
    if (s == "plain") return QLIN_VAR_PLAIN;
    if (s == "splitk") return QLIN_VAR_SPLITK;
    if (s == "swapab") return QLIN_VAR_SWAPAB;
    if (s == "swapab_splitk") return QLIN_VAR_SWAPAB_SPLITK;
    if (s == "pair") return QLIN_VAR_PAIR;
    return -1;
}

bool is_swap(int v) { return v == QLIN_VAR_SWAPAB || v == QLIN_VAR_SWAPAB_SPLITK; }
int base_mode(int v) { return v == QLIN_VAR_PAIR ? kModePair : kModeStd; }
bool is_spread(int v) { return v == QLIN_VAR_SPLITK || v == QLIN_VAR_SWAPAB_SPLITK; }
// Swap-AB Split-K whose segments fit one cluster may reduce through it.
bool runs_as_cluster(int variant, int tile_n, int S) {
    return variant == QLIN_VAR_SWAPAB_SPLITK && S > 1 && S <= cluster_split_max(tile_n);
}

bool tile_supported(int fmt, bool swap, int tile_n, bool pair = false) {
    if (is_block_scaled(fmt)) return !pair && (swap ? (tile_n == 32 || tile_n == 64) : tile_n == 128);
    if (pair) return fmt != QLIN_FMT_FP8_BLOCK && tile_n == 256;
    if (swap) return tile_n == 16 || tile_n == 32 || tile_n == 64;
    if (fmt == QLIN_FMT_FP8_BLOCK) return tile_n == 128;
    return tile_n == 128 || tile_n == 256;
}

// K segmentation of the built-in rule: the largest S <= 8 dividing K/128 such
// that the Swap-AB tiles of the shape (ceil(N/128)) times S still fit in one
// wave of CTAs.  Fixed per (format, N, K), independent of M.
int default_segments(int fmt, int64_t N, int64_t K, int num_sms) {
    (void)fmt;
    const int64_t kblocks = K / 128;
    const int64_t tiles = (N + 127) / 128;
    int best = 1;
    for (int s = 2; s <= 8; ++s)
        if (kblocks % s == 0 && tiles * s <= num_sms) best = s;
    return best;
}

// Bytes of one operand row and 128-byte K blocks: 8-bit formats 1 B/element,
// bf16 2, packed NVFP4 1/2.
int64_t row_bytes(int fmt, int64_t K) { return fmt == QLIN_FMT_BF16 ? 2 * K : (fmt == QLIN_FMT_NVFP4 ? K / 2 : K); }

qlin_config default_config(int fmt, int64_t M, int64_t N, int64_t K, int num_sms) {
    qlin_config c{};
    if (is_block_scaled(fmt)) {
        // block-scaled: one K segment (measured fastest at every M for the
        // attention and down-projection shapes: the running total and the
        // Split-K partials cost more than they gain); Swap-AB 32 / 64 tiles
        // for small M, plain 128 x 128 tiles above
        c.k_segments = 1;
        c.from_table = 0;
        c.m_max = 0;
        c.variant = M <= 64 ? QLIN_VAR_SWAPAB : QLIN_VAR_PLAIN;
        c.tile_n = M <= 32 ? 32 : (M <= 64 ? 64 : 128);
        size_t smem = 0;
        gemm_kernel_info(fmt, is_swap(c.variant), c.tile_n, kModeStd, &c.stages, &smem);
        return c;
    }
    c.k_segments = default_segments(fmt, N, row_bytes(fmt, K), num_sms);
    c.from_table = 0;
    c.m_max = 0;
    if (M <= 64 && !is_block_scaled(fmt)) {
        c.tile_n = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
        c.variant = c.k_segments > 1 ? QLIN_VAR_SWAPAB_SPLITK : QLIN_VAR_SWAPAB;
    } else {
        const bool multi = fmt == QLIN_FMT_FP8_BLOCK || is_block_scaled(fmt) ||
                           ((fmt == QLIN_FMT_FP8 || fmt == QLIN_FMT_BF16) && c.k_segments > 1);
        c.tile_n = multi ? 128 : 256;
        const int64_t tiles = ((M + 127) / 128) * ((N + c.tile_n - 1) / c.tile_n);
        c.variant = (c.k_segments > 1 && tiles * 2 <= num_sms) ? QLIN_VAR_SPLITK : QLIN_VAR_PLAIN;
    }
    size_t smem = 0;
    gemm_kernel_info(fmt, is_swap(c.variant), c.tile_n, kModeStd, &c.stages, &smem);
    return c;
}

bool lookup_table(int fmt, int64_t M, int64_t N, int64_t K, qlin_config* out) {
    std::lock_guard<std::mutex> lk(g_table_mu);
    const TableEntry* best = nullptr;
    const TableEntry* largest = nullptr;
    for (const auto& e : g_table) {
        if (e.fmt != fmt || e.N != N || e.K != K) continue;
        if (!largest || e.m_max > largest->m_max) largest = &e;
        if (e.m_max >= M && (!best || e.m_max < best->m_max)) best = &e;
    }
    if (!best) best = largest;
    if (!best) return false;
    out->variant = best->variant;
    out->tile_n = best->tile_n;
    out->k_segments = best->k_segments;
    size_t smem = 0;
    gemm_kernel_info(fmt, is_swap(best->variant), best->tile_n, base_mode(best->variant), &out->stages, &smem);
    out->m_max = best->m_max;
    out->from_table = 1;
    return true;
}


qlin_status resolve_config(int fmt, int variant, int tile_n, int k_segments, int64_t M, int64_t N, int64_t K,
                           int num_sms, qlin_config* cfg) {
    if (variant < QLIN_VAR_AUTO || variant > QLIN_VAR_PAIR) return QLIN_ERR_INVALID_ARG;
    if (tile_n < 0 || k_segments < 0) return QLIN_ERR_INVALID_ARG;
    qlin_config base{};
    if (!lookup_table(fmt, M, N, K, &base)) base = default_config(fmt, M, N, K, num_sms);
    if (variant != QLIN_VAR_AUTO) {
        // a forced variant keeps the shape's segmentation; its tile defaults
        // to the rule's choice for that orientation
        const qlin_config d = default_config(fmt, is_swap(variant) ? 1 : 65, N, K, num_sms);
        const bool same_orientation = is_swap(variant) == is_swap(base.variant);
        base.tile_n = same_orientation ? base.tile_n : d.tile_n;
        if (is_swap(variant) && !same_orientation)
            base.tile_n = M <= 16 && !is_block_scaled(fmt) ? 16 : (M <= 32 ? 32 : 64);
        if (variant == QLIN_VAR_PAIR) base.tile_n = 256;
        base.variant = variant;
    }
    if (tile_n) base.tile_n = tile_n;
    if (k_segments) base.k_segments = k_segments;
    size_t smem = 0;
    base.stages = 0;
    gemm_kernel_info(fmt, is_swap(base.variant), base.tile_n, base_mode(base.variant), &base.stages, &smem);
    *cfg = base;
    return QLIN_OK;
}

}  // namespace

qlin_status check_fmt_shape(int fmt, int64_t M, int64_t N, int64_t K) {
    if (fmt < QLIN_FMT_INT8 || fmt > QLIN_FMT_NVFP4) return QLIN_ERR_INVALID_ARG;
    // elements per 128-byte K block
    const int64_t kunit = fmt == QLIN_FMT_BF16 ? 64 : (fmt == QLIN_FMT_NVFP4 ? 256 : 128);
    if (M < 0 || N < 16 || K < kunit) return QLIN_ERR_INVALID_ARG;
    if (N % 16 != 0 || K % kunit != 0) return QLIN_ERR_UNSUPPORTED;
    if (fmt == QLIN_FMT_FP8_BLOCK && N % 128 != 0) return QLIN_ERR_UNSUPPORTED;
    if (M > (int64_t)1 << 30 || N > (int64_t)1 << 30 || K > (int64_t)1 << 24) return QLIN_ERR_UNSUPPORTED;
    return QLIN_OK;
}

int current_device_sms() {
    static int cached_dev = -1, cached_sms = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev != cached_dev) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cached_sms = sms;
        cached_dev = dev;
    }
    return cached_sms;
}

qlin_status make_gemm_plan(int fmt, int variant, int tile_n, int k_segments, int64_t M, int64_t N, int64_t K,
                           int num_sms, int want_mode, GemmPlan* plan) {
    qlin_status st = check_fmt_shape(fmt, M, N, K);
    if (st != QLIN_OK) return st;
    if (num_sms <= 0) num_sms = kNumSMsB200;
    qlin_config cfg{};
    st = resolve_config(fmt, variant, tile_n, k_segments, M, N, K, num_sms, &cfg);
    if (st != QLIN_OK) return st;
    GemmPlan p;
    p.fmt = fmt;
    p.swap = is_swap(cfg.variant);
    p.spread = is_spread(cfg.variant);
    p.tile_n = cfg.tile_n;
    p.k_segments = cfg.k_segments;
    p.M = M;
    p.N = N;
    p.K = K;
    p.k_bytes = row_bytes(fmt, K);
    p.kblocks = (int)(p.k_bytes / 128);
    const bool pair = cfg.variant == QLIN_VAR_PAIR;
    if (!tile_supported(fmt, p.swap, p.tile_n, pair)) return QLIN_ERR_UNSUPPORTED;
    // block-scaled Swap-AB: one activation tile (its scale rows are rows
    // 0 .. tile_n - 1 of the first 128-row atom; see the kernel's Cfg)
    if (is_block_scaled(fmt) && p.swap && M > p.tile_n) return QLIN_ERR_UNSUPPORTED;
    if (p.k_segments < 1 || p.kblocks % p.k_segments != 0) return QLIN_ERR_UNSUPPORTED;
    if (p.k_segments == 1) p.spread = false;
    p.kb_per_seg = p.kblocks / p.k_segments;
    // units with more than one accumulator chunk keep tile_n fp32 values per
    // thread and a TMEM running total: only tiles up to 128 columns do that
    const bool multi_chunk =
        (fmt == QLIN_FMT_FP8_BLOCK && (p.spread ? p.kb_per_seg : p.kblocks) > 1) ||
        ((fmt == QLIN_FMT_FP8 || fmt == QLIN_FMT_BF16 || is_block_scaled(fmt)) && !p.spread && p.k_segments > 1);
    if (multi_chunk && p.tile_n > 128) return QLIN_ERR_UNSUPPORTED;
    p.kb_per_unit = p.spread ? p.kb_per_seg : p.kblocks;
    p.mode = pair ? kModePair : kModeStd;
    if (want_mode == kModeCluster && p.spread && runs_as_cluster(cfg.variant, p.tile_n, p.k_segments))
        p.mode = kModeCluster;
    if (want_mode == kModeFused && p.swap && p.kb_per_unit <= fused_max_kblocks(p.tile_n)) p.mode = kModeFused;
    if (!gemm_kernel_info(fmt, p.swap, p.tile_n, p.mode, &p.stages, &p.smem_bytes)) return QLIN_ERR_UNSUPPORTED;
    p.p_rows = p.swap ? N : M;
    p.q_rows = p.swap ? M : N;
    p.p_tiles = (p.p_rows + 127) / 128;
    p.q_tiles = (p.q_rows + p.tile_n - 1) / p.tile_n;
    // PAIR: one unit per 256-row tile (two 128-row halves on the two CTAs)
    p.num_tiles = (pair ? (p.p_tiles + 1) / 2 : p.p_tiles) * p.q_tiles;
    p.units = p.num_tiles * (p.spread ? p.k_segments : 1);
    if (p.units > (int64_t)INT32_MAX / 2) return QLIN_ERR_UNSUPPORTED;
    p.grid = (int)std::min<int64_t>(p.units, num_sms);
    if (p.mode == kModeCluster)  // whole clusters; the launcher also caps them by co-residency
        p.grid = (int)std::min<int64_t>(p.num_tiles, std::max(1, num_sms / p.k_segments)) * p.k_segments;
    if (p.mode == kModePair) p.grid = (int)std::min<int64_t>(p.num_tiles, std::max(1, num_sms / 2)) * 2;
    if (p.grid < 1) p.grid = 1;
    const bool workspace_split = p.spread && p.mode != kModeCluster;
    if (workspace_split && p.num_tiles > kMaxSplitTiles) return QLIN_ERR_UNSUPPORTED;
    if (workspace_split) {
        p.ticket_bytes = kTicketBytes;
        p.workspace_bytes = p.ticket_bytes + (size_t)p.k_segments * p.num_tiles * 128 * p.tile_n * 4;
    } else {
        p.ticket_bytes = 0;
        p.workspace_bytes = 0;
    }
    *plan = p;
    return QLIN_OK;
}

qlin_status make_moe_plan(int fmt, int variant, int tile_n, int64_t R, int E, int64_t N, int64_t K, int num_sms,
                          GemmPlan* plan) {
    if (fmt != QLIN_FMT_INT8 && fmt != QLIN_FMT_FP8) return QLIN_ERR_UNSUPPORTED;
    if (E < 1 || E > kMoeMaxE) return QLIN_ERR_UNSUPPORTED;
    qlin_status st = check_fmt_shape(fmt, R, N, K);
    if (st != QLIN_OK) return st;
    if ((int64_t)E * N > (int64_t)1 << 31) return QLIN_ERR_UNSUPPORTED;
    if (num_sms <= 0) num_sms = kNumSMsB200;
    const int64_t avg = (R + E - 1) / E;  // rows per expert, on average
    if (variant == QLIN_VAR_AUTO) variant = avg <= 64 ? QLIN_VAR_SWAPAB : QLIN_VAR_PLAIN;
    if (variant != QLIN_VAR_SWAPAB && variant != QLIN_VAR_PLAIN) return QLIN_ERR_UNSUPPORTED;
    GemmPlan p;
    p.fmt = fmt;
    p.swap = variant == QLIN_VAR_SWAPAB;
    p.spread = false;
    p.mode = kModeStd;
    p.tile_n = tile_n ? tile_n : (p.swap ? (avg <= 16 ? 16 : avg <= 32 ? 32 : 64) : 128);
    if (!tile_supported(fmt, p.swap, p.tile_n)) return QLIN_ERR_UNSUPPORTED;
    p.k_segments = 1;
    p.M = R;
    p.N = N;
    p.K = K;
    p.k_bytes = K;
    p.kblocks = (int)(K / 128);
    p.kb_per_seg = p.kblocks;
    p.kb_per_unit = p.kblocks;
    if (!gemm_kernel_info(fmt, p.swap, p.tile_n, p.mode, &p.stages, &p.smem_bytes)) return QLIN_ERR_UNSUPPORTED;
    p.p_rows = p.swap ? (int64_t)E * N : R;
    p.q_rows = p.swap ? R : (int64_t)E * N;
    // upper bound on the units the device will count (each expert's last tile may be partial)
    const int64_t bound = p.swap ? ((N + 127) / 128) * (R / p.tile_n + E) : ((N + p.tile_n - 1) / p.tile_n) * (R / 128 + E);
    p.p_tiles = 0;
    p.q_tiles = 0;
    p.num_tiles = bound;
    p.units = 0;
    p.grid = (int)std::max<int64_t>(1, std::min<int64_t>(bound, num_sms));
    p.moe_E = E;
    *plan = p;
    return QLIN_OK;
}

}  // namespace qlin

using namespace qlin;

extern "C" {

int qlin_abi_version(void) { return QLIN_ABI_VERSION; }

const char* qlin_status_string(qlin_status s) {
    switch (s) {
        case QLIN_OK: return "ok";
        case QLIN_ERR_INVALID_ARG: return "invalid argument";
        case QLIN_ERR_UNSUPPORTED: return "unsupported shape, format or variant";
        case QLIN_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
        case QLIN_ERR_WORKSPACE: return "workspace missing or too small";
        case QLIN_ERR_TABLE_IO: return "dispatch table file unreadable";
        case QLIN_ERR_TABLE_FORMAT: return "dispatch table malformed";
        case QLIN_ERR_TABLE_DEVICE: return "dispatch table made for another device";
        case QLIN_ERR_CUDA: return "CUDA call failed";
        case QLIN_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case QLIN_ERR_NO_DEVICE: return "no sm_100 device";
    }
    return "unknown status";
}

qlin_status qlin_quantize_per_token(int fmt, const void* x, int64_t rows, int64_t cols, int64_t ld_x, void* q_out,
                                    float* scale_out, uint32_t flags, qlin_stream_t stream) {
    if (fmt != QLIN_FMT_INT8 && fmt != QLIN_FMT_FP8) return QLIN_ERR_INVALID_ARG;
    if (flags & ~QLIN_PDL) return QLIN_ERR_INVALID_ARG;
    if (rows < 0 || cols < 1 || ld_x < cols) return QLIN_ERR_INVALID_ARG;
    if (rows == 0) return QLIN_OK;
    if (!x || !q_out || !scale_out) return QLIN_ERR_INVALID_ARG;
    if (cols % 8 != 0 || ld_x % 8 != 0) return QLIN_ERR_ALIGNMENT;
    if (!aligned16(x) || !aligned16(q_out) || (reinterpret_cast<uintptr_t>(scale_out) & 3u))
        return QLIN_ERR_ALIGNMENT;
    if (rows > (int64_t)1 << 34) return QLIN_ERR_UNSUPPORTED;
    cudaError_t e = launch_quantize_per_token(fmt, x, rows, cols, ld_x, q_out, scale_out, (flags & QLIN_PDL) != 0,
                                              static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QLIN_OK : QLIN_ERR_CUDA;
}

qlin_status qlin_quantize_block(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int block_rows,
                                int block_cols, void* q_out, float* scale_out, uint32_t flags, qlin_stream_t stream) {
    if (rows < 0 || cols < 1 || ld_x < cols) return QLIN_ERR_INVALID_ARG;
    if (flags & ~QLIN_PDL) return QLIN_ERR_INVALID_ARG;
    if (block_cols != 128 || (block_rows != 1 && block_rows != 128)) return QLIN_ERR_UNSUPPORTED;
    if (cols % 128 != 0) return QLIN_ERR_UNSUPPORTED;
    if (rows == 0) return QLIN_OK;
    if (!x || !q_out || !scale_out) return QLIN_ERR_INVALID_ARG;
    if (ld_x % 8 != 0) return QLIN_ERR_ALIGNMENT;
    if (!aligned16(x) || !aligned16(q_out) || (reinterpret_cast<uintptr_t>(scale_out) & 3u))
        return QLIN_ERR_ALIGNMENT;
    if (block_rows == 128 && (rows + 127) / 128 > 65535) return QLIN_ERR_UNSUPPORTED;
    cudaError_t e = launch_quantize_block(x, rows, cols, ld_x, block_rows, q_out, scale_out, (flags & QLIN_PDL) != 0,
                                          static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QLIN_OK : QLIN_ERR_CUDA;
}

qlin_status qlin_scaled_mm_workspace_size(int fmt, int variant, int tile_n, int k_segments, int64_t M, int64_t N,
                                          int64_t K, size_t* bytes_out) {
    if (!bytes_out) return QLIN_ERR_INVALID_ARG;
    *bytes_out = 0;
    if (M == 0) {
        qlin_status s = check_fmt_shape(fmt, 1, N, K);
        return s;
    }
    GemmPlan p;
    qlin_status st = make_gemm_plan(fmt, variant, tile_n, k_segments, M, N, K, current_device_sms(), kModeStd, &p);
    if (st != QLIN_OK) return st;
    *bytes_out = p.workspace_bytes;
    return QLIN_OK;
}

qlin_status qlin_scaled_mm(int fmt, int variant, int tile_n, int k_segments, int64_t M, int64_t N, int64_t K,
                           const void* a_q, const float* s_a, const void* w_q, const float* s_w, const void* bias,
                           void* c_out, uint32_t flags, void* workspace, size_t workspace_bytes,
                           qlin_stream_t stream) {
    if (fmt == QLIN_FMT_BF16 || is_block_scaled(fmt)) return QLIN_ERR_INVALID_ARG;  // qlin_matmul_bf16 / _block_scaled_mm
    qlin_status st = check_fmt_shape(fmt, M, N, K);
    if (st != QLIN_OK) return st;
    if (flags & ~(QLIN_OUT_I32ACC | QLIN_PDL | QLIN_SPLITK_CLUSTER)) return QLIN_ERR_INVALID_ARG;
    const bool out_i32 = (flags & QLIN_OUT_I32ACC) != 0;
    if (out_i32 && fmt != QLIN_FMT_INT8) return QLIN_ERR_INVALID_ARG;
    if (fmt == QLIN_FMT_FP8_BLOCK && bias) return QLIN_ERR_INVALID_ARG;
    if (variant < QLIN_VAR_AUTO || variant > QLIN_VAR_PAIR || tile_n < 0 || k_segments < 0)
        return QLIN_ERR_INVALID_ARG;
    if (M == 0) return QLIN_OK;
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
    if (p.workspace_bytes) {
        if (!workspace || workspace_bytes < p.workspace_bytes) return QLIN_ERR_WORKSPACE;
        if (!aligned16(workspace)) return QLIN_ERR_ALIGNMENT;
    }
    if (g_log)
        std::fprintf(stderr, "[qlin] scaled_mm %s M=%lld N=%lld K=%lld -> %s%s tile_n=%d S=%d grid=%d\n",
                     fmt_name(fmt), (long long)M, (long long)N, (long long)K,
                     variant_name(p.mode == kModePair ? QLIN_VAR_PAIR
                                  : p.swap ? (p.spread ? QLIN_VAR_SWAPAB_SPLITK : QLIN_VAR_SWAPAB)
                                           : (p.spread ? QLIN_VAR_SPLITK : QLIN_VAR_PLAIN)),
                     p.mode == kModeCluster ? " (cluster)" : "", p.tile_n, p.k_segments, p.grid);
    GemmOperands ops{a_q, s_a, w_q, s_w, bias, c_out, out_i32, workspace, (flags & QLIN_PDL) != 0};
    return launch_gemm(p, ops, static_cast<cudaStream_t>(stream));
}

qlin_status qlin_linear(int fmt, int variant, int tile_n, int k_segments, int64_t M, int64_t N, int64_t K,
                        const void* x, int64_t ld_x, void* a_q, float* s_a, const void* w_q, const float* s_w,
                        const void* bias, void* c_out, uint32_t flags, void* workspace, size_t workspace_bytes,
                        qlin_stream_t stream) {
    if (fmt == QLIN_FMT_BF16 || is_block_scaled(fmt)) return QLIN_ERR_INVALID_ARG;  // per-token / Block-FP8 only
    qlin_status st = check_fmt_shape(fmt, M, N, K);
    if (st != QLIN_OK) return st;
    if (flags & ~(QLIN_OUT_I32ACC | QLIN_PDL | QLIN_FUSED)) return QLIN_ERR_INVALID_ARG;
    const bool out_i32 = (flags & QLIN_OUT_I32ACC) != 0;
    if (out_i32 && fmt != QLIN_FMT_INT8) return QLIN_ERR_INVALID_ARG;
    if (fmt == QLIN_FMT_FP8_BLOCK && bias) return QLIN_ERR_INVALID_ARG;
    if (variant < QLIN_VAR_AUTO || variant > QLIN_VAR_PAIR || tile_n < 0 || k_segments < 0)
        return QLIN_ERR_INVALID_ARG;
    if (ld_x < K) return QLIN_ERR_INVALID_ARG;
    if (M == 0) return QLIN_OK;
    if (!x || !a_q || !s_a || !w_q || !s_w || !c_out) return QLIN_ERR_INVALID_ARG;
    if (ld_x % 8 != 0 || !aligned16(x) || !aligned16(a_q) || !aligned16(w_q) || !aligned16(c_out))
        return QLIN_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(s_a) & 3u) || (reinterpret_cast<uintptr_t>(s_w) & 3u) ||
        (reinterpret_cast<uintptr_t>(bias) & 1u))
        return QLIN_ERR_ALIGNMENT;
    const int sms = current_device_sms();
    if (sms <= 0) return QLIN_ERR_NO_DEVICE;
    GemmPlan p;
    st = make_gemm_plan(fmt, variant, tile_n, k_segments, M, N, K, sms,
                        (flags & QLIN_FUSED) ? kModeFused : kModeStd, &p);
    if (st != QLIN_OK) return st;
    if (p.workspace_bytes) {
        if (!workspace || workspace_bytes < p.workspace_bytes) return QLIN_ERR_WORKSPACE;
        if (!aligned16(workspace)) return QLIN_ERR_ALIGNMENT;
    }
    const bool pdl = (flags & QLIN_PDL) != 0;
    const auto cst = static_cast<cudaStream_t>(stream);
    if (g_log)
        std::fprintf(stderr, "[qlin] linear %s M=%lld N=%lld K=%lld -> %s%s tile_n=%d S=%d grid=%d\n", fmt_name(fmt),
                     (long long)M, (long long)N, (long long)K,
                     variant_name(p.mode == kModePair ? QLIN_VAR_PAIR
                                  : p.swap ? (p.spread ? QLIN_VAR_SWAPAB_SPLITK : QLIN_VAR_SWAPAB)
                                           : (p.spread ? QLIN_VAR_SPLITK : QLIN_VAR_PLAIN)),
                     p.mode == kModeFused ? " (fused)" : "", p.tile_n, p.k_segments, p.grid);
    if (p.mode == kModeFused) {
        GemmOperands ops{a_q, s_a, w_q, s_w, bias, c_out, out_i32, workspace, pdl, x, ld_x};
        return launch_gemm(p, ops, cst);
    }
    // two kernels: the quantiser, then the GEMM as its programmatic dependent
    // (the quantiser writes neither the weights nor anything the GEMM's
    // early weight prefetch reads)
    cudaError_t e = fmt == QLIN_FMT_FP8_BLOCK ? launch_quantize_block(x, M, K, ld_x, 1, a_q, s_a, pdl, cst)
                                              : launch_quantize_per_token(fmt, x, M, K, ld_x, a_q, s_a, pdl, cst);
    if (e != cudaSuccess) return QLIN_ERR_CUDA;
    GemmOperands ops{a_q, s_a, w_q, s_w, bias, c_out, out_i32, workspace, true};
    return launch_gemm(p, ops, cst);
}

qlin_status qlin_matmul_bf16(int variant, int tile_n, int k_segments, int64_t M, int64_t N, int64_t K, const void* a,
                             const void* w, const void* bias, void* c_out, uint32_t flags, void* workspace,
                             size_t workspace_bytes, qlin_stream_t stream) {
    const int fmt = QLIN_FMT_BF16;
    qlin_status st = check_fmt_shape(fmt, M, N, K);
    if (st != QLIN_OK) return st;
    if (flags & ~(QLIN_PDL | QLIN_SPLITK_CLUSTER)) return QLIN_ERR_INVALID_ARG;
    if (variant < QLIN_VAR_AUTO || variant > QLIN_VAR_PAIR || tile_n < 0 || k_segments < 0)
        return QLIN_ERR_INVALID_ARG;
    if (M == 0) return QLIN_OK;
    if (!a || !w || !c_out) return QLIN_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(w) || !aligned16(c_out) || (reinterpret_cast<uintptr_t>(bias) & 1u))
        return QLIN_ERR_ALIGNMENT;
    const int sms = current_device_sms();
    if (sms <= 0) return QLIN_ERR_NO_DEVICE;
    GemmPlan p;
    st = make_gemm_plan(fmt, variant, tile_n, k_segments, M, N, K, sms,
                        (flags & QLIN_SPLITK_CLUSTER) ? kModeCluster : kModeStd, &p);
    if (st != QLIN_OK) return st;
    if (p.workspace_bytes) {
        if (!workspace || workspace_bytes < p.workspace_bytes) return QLIN_ERR_WORKSPACE;
        if (!aligned16(workspace)) return QLIN_ERR_ALIGNMENT;
    }
    if (g_log)
        std::fprintf(stderr, "[qlin] matmul_bf16 M=%lld N=%lld K=%lld -> %s%s tile_n=%d S=%d grid=%d\n",
                     (long long)M, (long long)N, (long long)K,
                     variant_name(p.mode == kModePair ? QLIN_VAR_PAIR
                                  : p.swap ? (p.spread ? QLIN_VAR_SWAPAB_SPLITK : QLIN_VAR_SWAPAB)
                                           : (p.spread ? QLIN_VAR_SPLITK : QLIN_VAR_PLAIN)),
                     p.mode == kModeCluster ? " (cluster)" : "", p.tile_n, p.k_segments, p.grid);
    GemmOperands ops{a, nullptr, w, nullptr, bias, c_out, false, workspace, (flags & QLIN_PDL) != 0};
    return launch_gemm(p, ops, static_cast<cudaStream_t>(stream));
}

qlin_status qlin_quantize_block_scaled(int fmt, const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                                       const float* g, void* q_out, void* sf_out, uint32_t flags,
                                       qlin_stream_t stream) {
    if (!is_block_scaled(fmt)) return QLIN_ERR_INVALID_ARG;
    if (flags & ~QLIN_PDL) return QLIN_ERR_INVALID_ARG;
    if (rows < 0 || cols < 1 || ld_x < cols) return QLIN_ERR_INVALID_ARG;
    if ((fmt == QLIN_FMT_NVFP4) != (g != nullptr)) return QLIN_ERR_INVALID_ARG;
    if (cols % 128 != 0) return QLIN_ERR_UNSUPPORTED;
    if (rows > (int64_t)1 << 34 || cols > (int64_t)1 << 24) return QLIN_ERR_UNSUPPORTED;
    if (rows == 0) return QLIN_OK;
    if (!x || !q_out || !sf_out) return QLIN_ERR_INVALID_ARG;
    if (ld_x % 8 != 0 || !aligned16(x) || !aligned16(q_out) || !aligned16(sf_out) ||
        (reinterpret_cast<uintptr_t>(g) & 3u))
        return QLIN_ERR_ALIGNMENT;
    cudaError_t e = launch_quantize_block_scaled(fmt, x, rows, cols, ld_x, g, q_out, sf_out, (flags & QLIN_PDL) != 0,
                                                 static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QLIN_OK : QLIN_ERR_CUDA;
}

qlin_status qlin_block_scaled_mm(int fmt, int variant, int tile_n, int k_segments, int64_t M, int64_t N, int64_t K,
                                 const void* a_q, const void* a_sf, const void* w_q, const void* w_sf,
                                 const float* g_a, const float* g_w, const void* bias, void* c_out, uint32_t flags,
                                 void* workspace, size_t workspace_bytes, qlin_stream_t stream) {
    if (!is_block_scaled(fmt)) return QLIN_ERR_INVALID_ARG;
    qlin_status st = check_fmt_shape(fmt, M, N, K);
    if (st != QLIN_OK) return st;
    if (flags & ~QLIN_PDL) return QLIN_ERR_INVALID_ARG;
    if (variant < QLIN_VAR_AUTO || variant > QLIN_VAR_PAIR) return QLIN_ERR_INVALID_ARG;
    if (variant == QLIN_VAR_PAIR) return QLIN_ERR_UNSUPPORTED;
    if (tile_n < 0 || k_segments < 0) return QLIN_ERR_INVALID_ARG;
    const bool nv = fmt == QLIN_FMT_NVFP4;
    if (nv != (g_a != nullptr) || nv != (g_w != nullptr)) return QLIN_ERR_INVALID_ARG;
    if (M == 0) return QLIN_OK;
    if (!a_q || !a_sf || !w_q || !w_sf || !c_out) return QLIN_ERR_INVALID_ARG;
    if (!aligned16(a_q) || !aligned16(a_sf) || !aligned16(w_q) || !aligned16(w_sf) || !aligned16(c_out))
        return QLIN_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(g_a) & 3u) || (reinterpret_cast<uintptr_t>(g_w) & 3u) ||
        (reinterpret_cast<uintptr_t>(bias) & 1u))
        return QLIN_ERR_ALIGNMENT;
    const int sms = current_device_sms();
    if (sms <= 0) return QLIN_ERR_NO_DEVICE;
    GemmPlan p;
    st = make_gemm_plan(fmt, variant, tile_n, k_segments, M, N, K, sms, kModeStd, &p);
    if (st != QLIN_OK) return st;
    if (p.workspace_bytes) {
        if (!workspace || workspace_bytes < p.workspace_bytes) return QLIN_ERR_WORKSPACE;
        if (!aligned16(workspace)) return QLIN_ERR_ALIGNMENT;
    }
    if (g_log)
        std::fprintf(stderr, "[qlin] block_scaled_mm %s M=%lld N=%lld K=%lld -> %s tile_n=%d S=%d grid=%d\n",
                     fmt_name(fmt), (long long)M, (long long)N, (long long)K,
                     variant_name(p.swap ? (p.spread ? QLIN_VAR_SWAPAB_SPLITK : QLIN_VAR_SWAPAB)
                                         : (p.spread ? QLIN_VAR_SPLITK : QLIN_VAR_PLAIN)),
                     p.tile_n, p.k_segments, p.grid);
    GemmOperands ops{a_q, g_a, w_q, g_w, bias, c_out, false, workspace, (flags & QLIN_PDL) != 0};
    ops.sf_a = a_sf;
    ops.sf_w = w_sf;
    return launch_gemm(p, ops, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------- MoE
namespace {
bool moe_dims_ok(int64_t T, int E, int topk) { return T >= 0 && E >= 1 && E <= kMoeMaxE && topk >= 1 && topk <= 32 && topk <= E; }
size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
struct MoeLayout {
    size_t ids, w, rows, offsets, a_q, s_a, g, h_q, s_h, y, total;
};
MoeLayout moe_layout(int64_t T, int64_t H, int64_t I, int E, int topk) {
    const size_t R = (size_t)T * topk;
    MoeLayout l;
    size_t o = 0;
    l.ids = o; o = align256(o + R * 4);
    l.w = o; o = align256(o + R * 4);
    l.rows = o; o = align256(o + R * 4);
    l.offsets = o; o = align256(o + ((size_t)E + 1) * 4);
    l.a_q = o; o = align256(o + R * (size_t)H);
    l.s_a = o; o = align256(o + R * 4);
    l.g = o; o = align256(o + R * 2 * (size_t)I * 2);
    l.h_q = o; o = align256(o + R * (size_t)I);
    l.s_h = o; o = align256(o + R * 4);
    l.y = o; o = align256(o + R * (size_t)H * 2);
    l.total = o;
    return l;
}
}  // namespace

qlin_status qlin_moe_route(int64_t T, int E, int topk, const float* logits, int32_t* topk_ids, float* topk_w,
                           int32_t* rows, int32_t* offsets, uint32_t flags, qlin_stream_t stream) {
    if (!moe_dims_ok(T, E, topk) || (flags & ~QLIN_PDL)) return QLIN_ERR_INVALID_ARG;
    if (T * topk > (int64_t)1 << 30) return QLIN_ERR_UNSUPPORTED;
    if (!offsets) return QLIN_ERR_INVALID_ARG;
    if (current_device_sms() <= 0) return QLIN_ERR_NO_DEVICE;
    if (T == 0) return cudaMemsetAsync(offsets, 0, ((size_t)E + 1) * 4, static_cast<cudaStream_t>(stream)) == cudaSuccess
                           ? QLIN_OK : QLIN_ERR_CUDA;
    if (!logits || !topk_ids || !topk_w || !rows) return QLIN_ERR_INVALID_ARG;
    return launch_moe_route(logits, (int)T, E, topk, topk_ids, topk_w, offsets, rows, (flags & QLIN_PDL) != 0,
                            static_cast<cudaStream_t>(stream)) == cudaSuccess ? QLIN_OK : QLIN_ERR_CUDA;
}

qlin_status qlin_moe_quantize_scatter(int64_t T, int64_t H, int topk, const void* x, const int32_t* rows, void* a_q,
                                      float* s_a, uint32_t flags, qlin_stream_t stream) {
    if (T < 0 || H < 16 || topk < 1 || topk > 32 || (flags & ~QLIN_PDL)) return QLIN_ERR_INVALID_ARG;
    if (H % 16 != 0) return QLIN_ERR_UNSUPPORTED;
    if (T == 0) return QLIN_OK;
    if (!x || !rows || !a_q || !s_a) return QLIN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(a_q)) return QLIN_ERR_ALIGNMENT;
    if (current_device_sms() <= 0) return QLIN_ERR_NO_DEVICE;
    return launch_moe_quantize_scatter(x, (int)T, (int)H, topk, rows, a_q, s_a, (flags & QLIN_PDL) != 0,
                                       static_cast<cudaStream_t>(stream)) == cudaSuccess ? QLIN_OK : QLIN_ERR_CUDA;
}

qlin_status qlin_moe_grouped_mm(int fmt, int variant, int tile_n, int E, int64_t R, int64_t N, int64_t K,
                                const void* a_q, const float* s_a, const int32_t* offsets, const void* w_q,
                                const float* s_w, void* c_out, uint32_t flags, qlin_stream_t stream) {
    if (flags & ~QLIN_PDL) return QLIN_ERR_INVALID_ARG;
    if (variant < QLIN_VAR_AUTO || variant > QLIN_VAR_PAIR || tile_n < 0) return QLIN_ERR_INVALID_ARG;
    if (R < 0 || E < 1) return QLIN_ERR_INVALID_ARG;
    if (R == 0) return QLIN_OK;
    if (!a_q || !s_a || !offsets || !w_q || !s_w || !c_out) return QLIN_ERR_INVALID_ARG;
    if (!aligned16(a_q) || !aligned16(w_q) || !aligned16(c_out)) return QLIN_ERR_ALIGNMENT;
    const int sms = current_device_sms();
    if (sms <= 0) return QLIN_ERR_NO_DEVICE;
    GemmPlan p;
    qlin_status st = make_moe_plan(fmt, variant, tile_n, R, E, N, K, sms, &p);
    if (st != QLIN_OK) return st;
    GemmOperands ops{a_q, s_a, w_q, s_w, nullptr, c_out, false, nullptr, (flags & QLIN_PDL) != 0};
    ops.moe_offsets = offsets;
    return launch_gemm(p, ops, static_cast<cudaStream_t>(stream));
}

qlin_status qlin_moe_act_quantize(int64_t R, int64_t I, const void* g, void* h_q, float* s_h, uint32_t flags,
                                  qlin_stream_t stream) {
    if (R < 0 || I < 16 || (flags & ~QLIN_PDL)) return QLIN_ERR_INVALID_ARG;
    if (I % 16 != 0) return QLIN_ERR_UNSUPPORTED;
    if (R == 0) return QLIN_OK;
    if (!g || !h_q || !s_h) return QLIN_ERR_INVALID_ARG;
    if (!aligned16(h_q) || (reinterpret_cast<uintptr_t>(g) & 3u)) return QLIN_ERR_ALIGNMENT;
    if (current_device_sms() <= 0) return QLIN_ERR_NO_DEVICE;
    return launch_moe_act_quantize(g, (int)R, (int)I, h_q, s_h, (flags & QLIN_PDL) != 0,
                                   static_cast<cudaStream_t>(stream)) == cudaSuccess ? QLIN_OK : QLIN_ERR_CUDA;
}

qlin_status qlin_moe_combine(int64_t T, int64_t H, int topk, const void* y, const float* topk_w, const int32_t* rows,
                             void* out, uint32_t flags, qlin_stream_t stream) {
    if (T < 0 || H < 16 || topk < 1 || topk > 32 || (flags & ~QLIN_PDL)) return QLIN_ERR_INVALID_ARG;
    if (H % 16 != 0) return QLIN_ERR_UNSUPPORTED;
    if (T == 0) return QLIN_OK;
    if (!y || !topk_w || !rows || !out) return QLIN_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(out)) return QLIN_ERR_ALIGNMENT;
    if (current_device_sms() <= 0) return QLIN_ERR_NO_DEVICE;
    return launch_moe_combine(y, topk_w, rows, (int)T, (int)H, topk, out, (flags & QLIN_PDL) != 0,
                              static_cast<cudaStream_t>(stream)) == cudaSuccess ? QLIN_OK : QLIN_ERR_CUDA;
}

qlin_status qlin_moe_workspace_size(int64_t T, int64_t H, int64_t I, int E, int topk, size_t* bytes_out) {
    if (!bytes_out || !moe_dims_ok(T, E, topk) || H < 16 || I < 16) return QLIN_ERR_INVALID_ARG;
    *bytes_out = moe_layout(T, H, I, E, topk).total;
    return QLIN_OK;
}

qlin_status qlin_moe_forward(int64_t T, int64_t H, int64_t I, int E, int topk, const void* x, const float* logits,
                             const void* w1_q, const float* s_w1, const void* w2_q, const float* s_w2, void* out,
                             uint32_t flags, void* workspace, size_t workspace_bytes, qlin_stream_t stream) {
    if (!moe_dims_ok(T, E, topk) || (flags & ~QLIN_PDL)) return QLIN_ERR_INVALID_ARG;
    if (H < 128 || I < 128) return QLIN_ERR_INVALID_ARG;
    if (H % 128 != 0 || I % 128 != 0) return QLIN_ERR_UNSUPPORTED;
    if (T == 0) return QLIN_OK;
    if (!x || !logits || !w1_q || !s_w1 || !w2_q || !s_w2 || !out) return QLIN_ERR_INVALID_ARG;
    const MoeLayout l = moe_layout(T, H, I, E, topk);
    if (!workspace || workspace_bytes < l.total) return QLIN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return QLIN_ERR_ALIGNMENT;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    auto* ids = reinterpret_cast<int32_t*>(ws + l.ids);
    auto* w = reinterpret_cast<float*>(ws + l.w);
    auto* rows = reinterpret_cast<int32_t*>(ws + l.rows);
    auto* offsets = reinterpret_cast<int32_t*>(ws + l.offsets);
    auto* s_a = reinterpret_cast<float*>(ws + l.s_a);
    auto* s_h = reinterpret_cast<float*>(ws + l.s_h);
    const int64_t R = T * topk;
    const uint32_t pdl = flags & QLIN_PDL;
    qlin_status st;
    if ((st = qlin_moe_route(T, E, topk, logits, ids, w, rows, offsets, pdl, stream)) != QLIN_OK) return st;
    if ((st = qlin_moe_quantize_scatter(T, H, topk, x, rows, ws + l.a_q, s_a, QLIN_PDL, stream)) != QLIN_OK) return st;
    if ((st = qlin_moe_grouped_mm(QLIN_FMT_FP8, QLIN_VAR_AUTO, 0, E, R, 2 * I, H, ws + l.a_q, s_a, offsets, w1_q, s_w1,
                                  ws + l.g, QLIN_PDL, stream)) != QLIN_OK)
        return st;
    if ((st = qlin_moe_act_quantize(R, I, ws + l.g, ws + l.h_q, s_h, QLIN_PDL, stream)) != QLIN_OK) return st;
    if ((st = qlin_moe_grouped_mm(QLIN_FMT_FP8, QLIN_VAR_AUTO, 0, E, R, H, I, ws + l.h_q, s_h, offsets, w2_q, s_w2,
                                  ws + l.y, QLIN_PDL, stream)) != QLIN_OK)
        return st;
    return qlin_moe_combine(T, H, topk, ws + l.y, w, rows, out, QLIN_PDL, stream);
}

qlin_status qlin_dispatch_query(int fmt, int64_t M, int64_t N, int64_t K, qlin_config* out) {
    if (!out) return QLIN_ERR_INVALID_ARG;
    qlin_status st = check_fmt_shape(fmt, M < 1 ? 1 : M, N, K);
    if (st != QLIN_OK) return st;
    int sms = current_device_sms();
    if (sms <= 0) sms = kNumSMsB200;
    return resolve_config(fmt, QLIN_VAR_AUTO, 0, 0, M < 1 ? 1 : M, N, K, sms, out);
}

qlin_status qlin_dispatch_table_clear(void) {
    std::lock_guard<std::mutex> lk(g_table_mu);
    g_table.clear();
    return QLIN_OK;
}

qlin_status qlin_dispatch_table_load(const char* path) {
    if (!path) return QLIN_ERR_INVALID_ARG;
    std::ifstream f(path);
    if (!f) return QLIN_ERR_TABLE_IO;
    std::string line;
    bool have_magic = false, have_device = false;
    int t_sms = 0, t_major = 0, t_minor = 0;
    std::string t_name;
    std::vector<TableEntry> entries;
    while (std::getline(f, line)) {
        if (line.empty() || line[0] == '#') continue;
        std::istringstream ss(line);
        std::string key;
        ss >> key;
        if (key == "qlin-dispatch") {
            int ver = 0;
            if (!(ss >> ver) || ver != 1) return QLIN_ERR_TABLE_FORMAT;
            have_magic = true;
        } else if (key == "device") {
            if (!(ss >> t_sms >> t_major >> t_minor)) return QLIN_ERR_TABLE_FORMAT;
            std::getline(ss, t_name);
            const size_t b = t_name.find_first_not_of(" \t");
            t_name = b == std::string::npos ? "" : t_name.substr(b);
            have_device = true;
        } else if (key == "entry") {
            std::string fs, vs;
            TableEntry e{};
            if (!(ss >> fs >> e.N >> e.K >> e.m_max >> vs >> e.tile_n >> e.k_segments)) return QLIN_ERR_TABLE_FORMAT;
            e.fmt = parse_fmt(fs);
            e.variant = parse_variant(vs);
            if (e.fmt < 0 || e.variant < 0 || e.m_max < 1) return QLIN_ERR_TABLE_FORMAT;
            if (check_fmt_shape(e.fmt, 1, e.N, e.K) != QLIN_OK) return QLIN_ERR_TABLE_FORMAT;
            if (!tile_supported(e.fmt, is_swap(e.variant), e.tile_n)) return QLIN_ERR_TABLE_FORMAT;
            if (e.k_segments < 1 || (row_bytes(e.fmt, e.K) / 128) % e.k_segments != 0) return QLIN_ERR_TABLE_FORMAT;
            entries.push_back(e);
        } else {
            return QLIN_ERR_TABLE_FORMAT;
        }
    }
    if (!have_magic || !have_device) return QLIN_ERR_TABLE_FORMAT;
    // every M bucket of one (format, N, K) must share the segmentation, or
    // results would change with the batch size
    for (size_t i = 0; i < entries.size(); ++i)
        for (size_t j = i + 1; j < entries.size(); ++j) {
            const auto &a = entries[i], &b = entries[j];
            if (a.fmt == b.fmt && a.N == b.N && a.K == b.K) {
                if (a.m_max == b.m_max) return QLIN_ERR_TABLE_FORMAT;
                if (a.fmt != QLIN_FMT_INT8 && a.k_segments != b.k_segments) return QLIN_ERR_TABLE_FORMAT;
            }
        }
    // every entry must be launchable (validates tile / segmentation / chunking)
    for (const auto& e : entries) {
        GemmPlan p;
        if (make_gemm_plan(e.fmt, e.variant, e.tile_n, e.k_segments, e.m_max, e.N, e.K, t_sms > 0 ? t_sms : 148,
                           kModeStd, &p) != QLIN_OK)
            return QLIN_ERR_TABLE_FORMAT;
    }
    // device guard: the table must have been measured on this kind of device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QLIN_ERR_NO_DEVICE;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return QLIN_ERR_CUDA;
    if (prop.multiProcessorCount != t_sms || prop.major != t_major || prop.minor != t_minor ||
        t_name != std::string(prop.name))
        return QLIN_ERR_TABLE_DEVICE;
    for (const auto& e : entries) {
        int stages = 0;
        size_t smem = 0;
        if (!gemm_kernel_info(e.fmt, is_swap(e.variant), e.tile_n, base_mode(e.variant), &stages, &smem) ||
            smem > prop.sharedMemPerBlockOptin)
            return QLIN_ERR_TABLE_FORMAT;
    }
    std::sort(entries.begin(), entries.end(), [](const TableEntry& a, const TableEntry& b) {
        if (a.fmt != b.fmt) return a.fmt < b.fmt;
        if (a.N != b.N) return a.N < b.N;
        if (a.K != b.K) return a.K < b.K;
        return a.m_max < b.m_max;
    });
    {
        std::lock_guard<std::mutex> lk(g_table_mu);
        g_table.swap(entries);
    }
    if (g_log) std::fprintf(stderr, "[qlin] loaded %zu dispatch entries from %s\n", g_table.size(), path);
    return QLIN_OK;
}

qlin_status qlin_selftest_wait_timeout(uint32_t limit_us, qlin_stream_t stream) {
    if (limit_us == 0 || limit_us > 1000000u) return QLIN_ERR_INVALID_ARG;
    if (current_device_sms() <= 0) return QLIN_ERR_NO_DEVICE;
    return launch_wait_selftest((uint64_t)limit_us * 1000u, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? QLIN_OK
               : QLIN_ERR_CUDA;
}

qlin_status qlin_sync_status(qlin_stream_t stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return QLIN_ERR_CUDA;
    int v = 0;
    if (device_status_read_clear(&v) != cudaSuccess) return QLIN_ERR_CUDA;
    return v != 0 ? (qlin_status)v : QLIN_OK;
}

}  // extern "C"
