// quantize.cu -- dynamic activation (and offline weight) quantisation kernels.
//
// Per-token INT8 / FP8 and Block-FP8 (1x128 groups, 128x128 blocks), the
// formats named on the page "Helion in vLLM: A Unified Route to Tunable Linear
// Kernels", section "What the integration changes".  Each kernel makes ONE
// pass over HBM: a row (or block) is loaded with 16-byte vector loads into
// registers, its absolute maximum is reduced with warp shuffles, and the codes
// are produced from the registers.
//
// Arithmetic (bit-exact by construction, no fast-math anywhere):
//   scale = amax / Qmax          IEEE binary32 division (__fdiv_rn)
//   v     = x / scale            correctly rounded quotient (Markstein-corrected
//                                reciprocal, or __fdiv_rn; see quotient())
//   INT8: q = clamp(rint_half_even(v), -127, 127)
//   FP8 : q = e4m3_rn_satfinite(clamp(v, -448, 448))
//   amax == 0 -> scale = 0, q = 0.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "pdl.cuh"
#include "quant_math.cuh"

namespace qlin {

namespace {

using namespace qm;

constexpr int kQuantWarps = 8;  // rows per CTA for the warp-per-row kernels

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ----------------------------------------------------------------------------
// Per-token: WPR warps per row (WPR = 1, 2 or 8; 8 / WPR rows per 256-thread
// CTA).  Thread t of a row's group owns vectors t, t + 32*WPR, ... (16 bytes =
// 8 bf16 each), held in registers (VPL per thread).  The row maximum is a warp
// shuffle reduction, then (WPR > 1) a reduction over the row's warps through
// shared memory.
template <int FMT, int VPL, int WPR>
__global__ void __launch_bounds__(kQuantWarps * 32)
    quantize_per_token_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                              uint8_t* __restrict__ q, float* __restrict__ s) {
    __shared__ float warp_max[kQuantWarps];
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * (kQuantWarps / WPR) + warp / WPR;
    const int t = (warp % WPR) * 32 + lane;
    const bool live = row < rows;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (live ? row : 0) * ld);
    const int nvec = (int)(cols >> 3);
    constexpr float QMAX = (FMT == QLIN_FMT_INT8) ? 127.f : 448.f;

    uint4 v[VPL];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int idx = i * 32 * WPR + t;
        if (live && idx < nvec) {
            v[i] = ld_stream(xr + idx);
            amax = fmaxf(amax, absmax8(v[i]));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if constexpr (WPR > 1) {
        if (lane == 0) warp_max[warp] = amax;
        __syncthreads();
        const int w0 = (warp / WPR) * WPR;
#pragma unroll
        for (int w = 0; w < WPR; ++w) amax = fmaxf(amax, warp_max[w0 + w]);
    }
    if (!live) return;
    const float sc = __fdiv_rn(amax, QMAX);
    if (t == 0) s[row] = sc;
    const Divisor dv = make_divisor(sc);
    uint2* qr = reinterpret_cast<uint2*>(q + row * cols);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int idx = i * 32 * WPR + t;
        if (idx < nvec) qr[idx] = quant8<FMT>(v[i], dv);
    }
}

// Per-token, rows too long to hold in registers: two passes over the row
// (the second one hits L2), one warp per row.
template <int FMT>
__global__ void __launch_bounds__(kQuantWarps * 32)
    quantize_per_token_long_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                                   uint8_t* __restrict__ q, float* __restrict__ s) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
    if (row >= rows) return;
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * ld);
    const int64_t nvec = cols >> 3;
    constexpr float QMAX = (FMT == QLIN_FMT_INT8) ? 127.f : 448.f;
    float amax = 0.f;
    for (int64_t idx = lane; idx < nvec; idx += 32) amax = fmaxf(amax, absmax8(xr[idx]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = __fdiv_rn(amax, QMAX);
    if (lane == 0) s[row] = sc;
    const Divisor dv = make_divisor(sc);
    uint2* qr = reinterpret_cast<uint2*>(q + row * cols);
    for (int64_t idx = lane; idx < nvec; idx += 32) qr[idx] = quant8<FMT>(xr[idx], dv);
}

// ----------------------------------------------------------------------------
// Block-FP8 activations, 1x128 groups, few rows (latency first): 8 warps per
// row.  Thread t of the row owns vectors t, t + 256, ...; in each step lanes
// 0-15 and 16-31 of a warp hold one whole group each (16 vectors x 8 = 128),
// so the group maximum is a 16-lane shuffle reduction.  A row is spread over
// all 256 threads, so each lane's chain of work is short.
template <int VPL, int WPR>
__global__ void __launch_bounds__(kQuantWarps * 32)
    quantize_group128_wide_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                             uint8_t* __restrict__ q, float* __restrict__ s) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * (kQuantWarps / WPR) + warp / WPR;
    const int t = (warp % WPR) * 32 + lane;
    if (row >= rows) return;
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * ld);
    const int nvec = (int)(cols >> 3);  // multiple of 16
    const int ngroups = (int)(cols >> 7);
    uint2* qr = reinterpret_cast<uint2*>(q + row * cols);
    float* sr = s + row * ngroups;
    for (int base = 0; base < nvec; base += VPL * 32 * WPR) {
        uint4 v[VPL];
        float gmax[VPL];
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int idx = base + i * 32 * WPR + t;
            gmax[i] = 0.f;
            if (idx < nvec) {
                v[i] = ld_stream(xr + idx);
                gmax[i] = absmax8(v[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) gmax[i] = fmaxf(gmax[i], __shfl_xor_sync(0xffffffffu, gmax[i], o));
        }
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int idx = base + i * 32 * WPR + t;
            if (idx < nvec) {
                const float sc = __fdiv_rn(gmax[i], 448.f);
                if ((lane & 15) == 0) sr[idx >> 4] = sc;
                const Divisor dv = make_divisor(sc);
                qr[idx] = quant8<QLIN_FMT_FP8>(v[i], dv);
            }
        }
    }
}

// ----------------------------------------------------------------------------
// Block-FP8 activations, 1x128 groups, many rows (instructions first): WPR warps per row.  A group's 16
// vectors (8 elements each) belong to 4 consecutive lanes: lane l takes group
// slot l / 4 and vectors l % 4, l % 4 + 4, l % 4 + 8 and l % 4 + 12 of it, so
// one warp instruction of the scale computation serves 8 groups and the group
// maximum is a 4-lane shuffle.  The row's WPR warps cover 8 * WPR groups per
// slot; a lane takes PASSES slots per round and issues all their loads before
// the first reduction, so a row of up to 8 * WPR * PASSES groups costs one
// memory round trip.
template <int PASSES, int WPR>
__global__ void __launch_bounds__(kQuantWarps * 32)
    quantize_group128_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                             uint8_t* __restrict__ q, float* __restrict__ s) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * (kQuantWarps / WPR) + warp / WPR;
    if (row >= rows) return;  // warp-uniform: the shuffles below stay converged
    const int gw = (warp % WPR) * 8 + (lane >> 2);  // this lane's group within a slot of the row
    const int sub = lane & 3;
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * ld);
    const int ngroups = (int)(cols >> 7);
    uint2* qr = reinterpret_cast<uint2*>(q + row * cols);
    float* sr = s + row * ngroups;
    constexpr int GPS = 8 * WPR;  // groups of the row per slot
    for (int g0 = 0; g0 < ngroups; g0 += GPS * PASSES) {
        uint4 v[PASSES][4];
#pragma unroll
        for (int p = 0; p < PASSES; ++p) {
            const int g = g0 + p * GPS + gw;
            if (g < ngroups) {
#pragma unroll
                for (int j = 0; j < 4; ++j) v[p][j] = ld_stream(xr + g * 16 + sub + 4 * j);
            }
        }
#pragma unroll
        for (int p = 0; p < PASSES; ++p) {
            const int g = g0 + p * GPS + gw;
            float gmax = 0.f;
            if (g < ngroups) {
#pragma unroll
                for (int j = 0; j < 4; ++j) gmax = fmaxf(gmax, absmax8(v[p][j]));
            }
            gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, 1));
            gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, 2));
            if (g < ngroups) {
                const float sc = __fdiv_rn(gmax, 448.f);
                if (sub == 0) sr[g] = sc;
                const Divisor dv = make_divisor(sc);
#pragma unroll
                for (int j = 0; j < 4; ++j) qr[g * 16 + sub + 4 * j] = quant8<QLIN_FMT_FP8>(v[p][j], dv);
            }
        }
    }
}

// Block-FP8 weights, 128x128 blocks: one CTA (256 threads) per block.  Thread
// t owns column vector t%16 of rows t/16 + 16*i, i = 0..7.
__global__ void __launch_bounds__(256)
    quantize_block128_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                             uint8_t* __restrict__ q, float* __restrict__ s) {
    __shared__ float warp_max[8];
    pdl_wait();
    pdl_launch_dependents();
    const int t = threadIdx.x;
    const int64_t br = blockIdx.y, bc = blockIdx.x;
    const int64_t nbc = cols >> 7;
    const int cv = t & 15;
    uint4 v[8];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t r = br * 128 + (t >> 4) + 16 * i;
        if (r < rows) {
            v[i] = ld_stream(reinterpret_cast<const uint4*>(x + r * ld + bc * 128) + cv);
            amax = fmaxf(amax, absmax8(v[i]));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((t & 31) == 0) warp_max[t >> 5] = amax;
    __syncthreads();
    amax = warp_max[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, warp_max[w]);
    const float sc = __fdiv_rn(amax, 448.f);
    if (t == 0) s[br * nbc + bc] = sc;
    const Divisor dv = make_divisor(sc);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t r = br * 128 + (t >> 4) + 16 * i;
        if (r < rows) reinterpret_cast<uint2*>(q + r * cols + bc * 128)[cv] = quant8<QLIN_FMT_FP8>(v[i], dv);
    }
}

// Launch with the programmatic-stream-serialization attribute when `pdl`.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, bool pdl, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Warps per row: wide rows over few tokens get more threads per row.
int warps_per_row(int64_t rows) { return rows <= 512 ? 8 : (rows <= 2048 ? 2 : 1); }

template <int FMT, int WPR>
cudaError_t launch_per_token_wpr(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* q, float* s,
                                 bool pdl, cudaStream_t st) {
    const int64_t per_thread = ((cols >> 3) + 32 * WPR - 1) / (32 * WPR);
    const dim3 grid((unsigned)((rows + (kQuantWarps / WPR) - 1) / (kQuantWarps / WPR))), block(kQuantWarps * 32);
    if (per_thread <= 1) return launch_k(quantize_per_token_kernel<FMT, 1, WPR>, grid, block, pdl, st, x, rows, cols, ld, q, s);
    if (per_thread <= 2) return launch_k(quantize_per_token_kernel<FMT, 2, WPR>, grid, block, pdl, st, x, rows, cols, ld, q, s);
    if (per_thread <= 4) return launch_k(quantize_per_token_kernel<FMT, 4, WPR>, grid, block, pdl, st, x, rows, cols, ld, q, s);
    if (per_thread <= 8) return launch_k(quantize_per_token_kernel<FMT, 8, WPR>, grid, block, pdl, st, x, rows, cols, ld, q, s);
    if (per_thread <= 16) return launch_k(quantize_per_token_kernel<FMT, 16, WPR>, grid, block, pdl, st, x, rows, cols, ld, q, s);
    if (per_thread <= 32) return launch_k(quantize_per_token_kernel<FMT, 32, WPR>, grid, block, pdl, st, x, rows, cols, ld, q, s);
    const dim3 g1((unsigned)((rows + kQuantWarps - 1) / kQuantWarps));
    return launch_k(quantize_per_token_long_kernel<FMT>, g1, block, pdl, st, x, rows, cols, ld, q, s);
}

template <int FMT>
cudaError_t launch_per_token_fmt(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* q, float* s,
                                 bool pdl, cudaStream_t st) {
    switch (warps_per_row(rows)) {
        case 8: return launch_per_token_wpr<FMT, 8>(x, rows, cols, ld, q, s, pdl, st);
        case 2: return launch_per_token_wpr<FMT, 2>(x, rows, cols, ld, q, s, pdl, st);
        default: return launch_per_token_wpr<FMT, 1>(x, rows, cols, ld, q, s, pdl, st);
    }
}

// Few rows: the row spread over the 256 threads of a CTA (16 lanes per group).
cudaError_t launch_group_wide(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* q, float* s,
                              bool pdl, cudaStream_t st) {
    constexpr int WPR = 8;
    const int64_t per_thread = ((cols >> 3) + 32 * WPR - 1) / (32 * WPR);
    const dim3 grid((unsigned)rows), block(kQuantWarps * 32);
    if (per_thread <= 1) return launch_k(quantize_group128_wide_kernel<1, WPR>, grid, block, pdl, st, x, rows, cols, ld, q, s);
    if (per_thread <= 4) return launch_k(quantize_group128_wide_kernel<4, WPR>, grid, block, pdl, st, x, rows, cols, ld, q, s);
    return launch_k(quantize_group128_wide_kernel<8, WPR>, grid, block, pdl, st, x, rows, cols, ld, q, s);
}

// Many rows: 4 lanes per group.
template <int WPR>
cudaError_t launch_group_wpr(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* q, float* s,
                             bool pdl, cudaStream_t st) {
    const int64_t slots = ((cols >> 7) + 8 * WPR - 1) / (8 * WPR);  // group slots per lane
    const dim3 grid((unsigned)((rows + (kQuantWarps / WPR) - 1) / (kQuantWarps / WPR))), block(kQuantWarps * 32);
    if (slots <= 1) return launch_k(quantize_group128_kernel<1, WPR>, grid, block, pdl, st, x, rows, cols, ld, q, s);
    if (slots <= 2) return launch_k(quantize_group128_kernel<2, WPR>, grid, block, pdl, st, x, rows, cols, ld, q, s);
    if (slots <= 3) return launch_k(quantize_group128_kernel<3, WPR>, grid, block, pdl, st, x, rows, cols, ld, q, s);
    return launch_k(quantize_group128_kernel<4, WPR>, grid, block, pdl, st, x, rows, cols, ld, q, s);  // rounds of 4
}

}  // namespace

cudaError_t launch_quantize_per_token(int fmt, const void* x, int64_t rows, int64_t cols, int64_t ld, void* q,
                                      float* s, bool pdl, cudaStream_t st) {
    const auto* xb = static_cast<const uint16_t*>(x);
    auto* qb = static_cast<uint8_t*>(q);
    if (fmt == QLIN_FMT_INT8) return launch_per_token_fmt<QLIN_FMT_INT8>(xb, rows, cols, ld, qb, s, pdl, st);
    return launch_per_token_fmt<QLIN_FMT_FP8>(xb, rows, cols, ld, qb, s, pdl, st);
}

cudaError_t launch_quantize_block(const void* x, int64_t rows, int64_t cols, int64_t ld, int block_rows, void* q,
                                  float* s, bool pdl, cudaStream_t st) {
    const auto* xb = static_cast<const uint16_t*>(x);
    auto* qb = static_cast<uint8_t*>(q);
    if (block_rows == 1) {
        // Few rows are latency-bound: the short per-lane chains of the wide
        // kernel win (Block-FP8 K = 6144: 2.8 against 4.1 us at M <= 64).
        // Many rows are issue-bound: 4 lanes per group cut the instructions
        // per element (M = 2048: 14.4 against 16.4 us).
        if (warps_per_row(rows) == 8) return launch_group_wide(xb, rows, cols, ld, qb, s, pdl, st);
        // no more warps on a row than it has slots of 8 groups for
        int wpr = warps_per_row(rows);
        while (wpr > 1 && 8 * wpr > (cols >> 7)) wpr >>= 1;
        return wpr == 2 ? launch_group_wpr<2>(xb, rows, cols, ld, qb, s, pdl, st)
                        : launch_group_wpr<1>(xb, rows, cols, ld, qb, s, pdl, st);
    }
    const dim3 grid((unsigned)(cols >> 7), (unsigned)((rows + 127) / 128));
    return launch_k(quantize_block128_kernel, grid, dim3(256), pdl, st, xb, rows, cols, ld, qb, s);
}

}  // namespace qlin
