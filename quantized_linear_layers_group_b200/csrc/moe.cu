// moe.cu -- the FP8 MoE layer as one chain of kernels: routing, expert row
// layout, per-token quantisation scattered into the expert rows, the grouped
// scaled GEMMs (gemm.cu, MoE mode), SiLU(gate) * up with per-token
// quantisation, and the top-k reduction.
//
// The page "vLLM and Tencent Hunyuan upstream two HPC backends for NVIDIA
// Hopper GPUs" (section "FP8 MoE pipeline as a single execution path") lists
// the steps -- routing, Gate-Up GEMM, activation function, quantisation, Down
// GEMM, top-k reduction -- and runs them as one path chained with
// programmatic dependent launch, so no step waits for a host round trip.  Each
// kernel here launches as the previous one's programmatic dependent: it waits
// (griddepcontrol.wait) before touching the previous step's output and lets
// the next one start early.
//
// Arithmetic (the plainest readings; identical in the oracle):
//   routing   the k largest fp32 logits of a token, descending, ties to the
//             lower expert; w_j = e_j / (e_0 + ... + e_{k-1}) in fp32 with
//             e_j = fp32(exp_binary64(l_j - l_0))
//   rows      expert groups in expert order (offsets = prefix sums of the
//             counts); inside a group any order (rows are independent)
//   act       h = (g / (1 + fp32(exp_binary64(-g)))) * up in fp32, then the
//             per-token FP8 quantisation of the row (quant_math.cuh)
//   combine   out = bf16(sum_j w_j * y_j), fp32 from +0 in routing order,
//             products and adds separately rounded
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "pdl.cuh"
#include "quant_math.cuh"

namespace qlin {
namespace {

using namespace qm;

__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// ----------------------------------------------------------------- routing
// One warp per token: k rounds of a warp arg-max over the token's E logits
// (each lane holds logits lane, lane + 32, ...), ties to the lower index.
template <int PER_LANE>
__global__ void __launch_bounds__(256) moe_route_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                        int32_t* __restrict__ ids, float* __restrict__ w) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    float v[PER_LANE];
    uint32_t taken = 0;  // bit i: logit lane + 32 i already chosen
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? logits[(size_t)t * E + e] : 0.f;
    }
    float my_val = 0.f;  // lane j keeps the j-th chosen logit
    int my_id = 0;
    for (int j = 0; j < k; ++j) {
        float bv = 0.f;
        int bi = -1;
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u) && (bi < 0 || v[i] > bv)) {
                bv = v[i];
                bi = e;
            }
        }
        // warp arg-max: larger value first, then the lower index
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (oi >= 0 && (bi < 0 || ov > bv || (ov == bv && oi < bi))) {
                bv = ov;
                bi = oi;
            }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == j) {
            my_val = bv;
            my_id = bi;
        }
    }
    const float m = __shfl_sync(0xffffffffu, my_val, 0);
    const float ej = lane < k ? (float)exp((double)__fsub_rn(my_val, m)) : 0.f;
    float s = 0.f;
    for (int j = 0; j < k; ++j) s = __fadd_rn(s, __shfl_sync(0xffffffffu, ej, j));  // routing order
    if (lane < k) {
        ids[(size_t)t * k + lane] = my_id;
        w[(size_t)t * k + lane] = __fdiv_rn(ej, s);
    }
}

// One CTA: expert counts, offsets (prefix sums) and a row for every (t, j).
__global__ void __launch_bounds__(1024) moe_rows_kernel(const int32_t* __restrict__ ids, int n, int E,
                                                        int32_t* __restrict__ offsets, int32_t* __restrict__ rows) {
    extern __shared__ int32_t sh[];  // counts[E], then cursors[E]
    int32_t* cnt = sh;
    int32_t* cur = sh + E;
    __shared__ int32_t warp_tot[32];
    pdl_wait();
    pdl_launch_dependents();
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) atomicAdd(&cnt[ids[i]], 1);
    __syncthreads();
    // exclusive scan over the experts, in chunks of blockDim.x
    int32_t carry = 0;
    for (int base = 0; base < E; base += blockDim.x) {
        const int e = base + threadIdx.x;
        const int32_t c = e < E ? cnt[e] : 0;
        int32_t x = c;  // inclusive scan within the warp
        const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[wid] = x;
        __syncthreads();
        int32_t before = 0;
        for (int w2 = 0; w2 < wid; ++w2) before += warp_tot[w2];
        int32_t chunk = 0;
        for (int w2 = 0; w2 < (int)(blockDim.x >> 5); ++w2) chunk += warp_tot[w2];
        if (e < E) {
            const int32_t off = carry + before + x - c;
            offsets[e] = off;
            cur[e] = off;
        }
        carry += chunk;
        __syncthreads();
    }
    if (threadIdx.x == 0) offsets[E] = carry;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) rows[i] = atomicAdd(&cur[ids[i]], 1);
}

// -------------------------------------------------- quantise and scatter
// One warp per token: the per-token FP8 quantisation of x[t] (the stand-alone
// quantiser's arithmetic), written to each of the token's k expert rows.
__global__ void __launch_bounds__(256) moe_quantize_scatter_kernel(const uint16_t* __restrict__ x, int T, int H,
                                                                   int k, const int32_t* __restrict__ rows,
                                                                   uint8_t* __restrict__ a_q,
                                                                   float* __restrict__ s_a) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    const int nvec = H >> 3;
    float amax = 0.f;
    for (int i = lane; i < nvec; i += 32) amax = fmaxf(amax, absmax8(xr[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = __fdiv_rn(amax, 448.f);
    const Divisor dv = make_divisor(sc);
    int32_t dst[32];
    for (int j = 0; j < k; ++j) dst[j] = rows[(size_t)t * k + j];
    if (lane < k) s_a[rows[(size_t)t * k + lane]] = sc;
    for (int i = lane; i < nvec; i += 32) {
        const uint2 q = quant8<QLIN_FMT_FP8>(xr[i], dv);
        for (int j = 0; j < k; ++j) reinterpret_cast<uint2*>(a_q + (size_t)dst[j] * H)[i] = q;
    }
}

// ------------------------------------------------ SiLU(gate) * up, quantise
__device__ __forceinline__ float silu_up(uint16_t gate, uint16_t up) {
    const float g = bf16f(gate);
    const float q = (float)exp(-(double)g);
    return __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, q)), bf16f(up));
}

// One warp per row: h = silu(G[:, :I]) * G[:, I:], then its per-token FP8
// quantisation (two passes; the second recomputes h identically).
__global__ void __launch_bounds__(256) moe_act_quantize_kernel(const uint16_t* __restrict__ g, int R, int I,
                                                               uint8_t* __restrict__ h_q, float* __restrict__ s_h) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= R) return;
    const uint16_t* gr = g + (size_t)r * 2 * I;
    float amax = 0.f;
    for (int i = lane; i < I; i += 32) amax = fmaxf(amax, fabsf(silu_up(gr[i], gr[I + i])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = __fdiv_rn(amax, 448.f);
    if (lane == 0) s_h[r] = sc;
    const Divisor dv = make_divisor(sc);
    uint8_t* hr = h_q + (size_t)r * I;
    for (int i0 = lane * 4; i0 < I; i0 += 128) {  // 4 codes per lane per step (I % 4 == 0)
        float f[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) f[c] = silu_up(gr[i0 + c], gr[I + i0 + c]);
        *reinterpret_cast<uint32_t*>(hr + i0) = quant_e4m3_x4(f, dv);
    }
}

// ----------------------------------------------------------------- combine
// One thread per (token, 8 columns): out = bf16(sum_j w_j * y[row(t, j)]).
__global__ void __launch_bounds__(256) moe_combine_kernel(const uint16_t* __restrict__ y, const float* __restrict__ w,
                                                          const int32_t* __restrict__ rows, int T, int H, int k,
                                                          uint16_t* __restrict__ out) {
    pdl_wait();
    pdl_launch_dependents();
    const int per_row = H >> 3;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)T * per_row) return;
    const int t = (int)(idx / per_row), c8 = (int)(idx % per_row);
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.f;
    for (int j = 0; j < k; ++j) {
        const float wj = w[(size_t)t * k + j];
        const uint4 v = reinterpret_cast<const uint4*>(y + (size_t)rows[(size_t)t * k + j] * H)[c8];
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            acc[2 * c] = __fadd_rn(acc[2 * c], __fmul_rn(wj, bf16f((uint16_t)(u[c] & 0xFFFFu))));
            acc[2 * c + 1] = __fadd_rn(acc[2 * c + 1], __fmul_rn(wj, bf16f((uint16_t)(u[c] >> 16))));
        }
    }
    uint4 o;
    uint32_t* op = &o.x;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const __nv_bfloat162 p = __floats2bfloat162_rn(acc[2 * c], acc[2 * c + 1]);
        op[c] = *reinterpret_cast<const uint32_t*>(&p);
    }
    reinterpret_cast<uint4*>(out + (size_t)t * H)[c8] = o;
}

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, bool pdl, cudaStream_t st,
                   Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace

cudaError_t launch_moe_route(const float* logits, int T, int E, int k, int32_t* ids, float* w, int32_t* offsets,
                             int32_t* rows, bool pdl, cudaStream_t st) {
    const dim3 grid((unsigned)((T + 7) / 8)), block(256);
    cudaError_t e;
    if (E <= 64)
        e = launch(moe_route_kernel<2>, grid, block, 0, pdl, st, logits, T, E, k, ids, w);
    else if (E <= 256)
        e = launch(moe_route_kernel<8>, grid, block, 0, pdl, st, logits, T, E, k, ids, w);
    else
        e = launch(moe_route_kernel<32>, grid, block, 0, pdl, st, logits, T, E, k, ids, w);
    if (e != cudaSuccess) return e;
    return launch(moe_rows_kernel, dim3(1), dim3(1024), (size_t)2 * E * sizeof(int32_t), true, st,
                  (const int32_t*)ids, T * k, E, offsets, rows);
}

cudaError_t launch_moe_quantize_scatter(const void* x, int T, int H, int k, const int32_t* rows, void* a_q,
                                        float* s_a, bool pdl, cudaStream_t st) {
    return launch(moe_quantize_scatter_kernel, dim3((unsigned)((T + 7) / 8)), dim3(256), 0, pdl, st,
                  static_cast<const uint16_t*>(x), T, H, k, rows, static_cast<uint8_t*>(a_q), s_a);
}

cudaError_t launch_moe_act_quantize(const void* g, int R, int I, void* h_q, float* s_h, bool pdl, cudaStream_t st) {
    return launch(moe_act_quantize_kernel, dim3((unsigned)((R + 7) / 8)), dim3(256), 0, pdl, st,
                  static_cast<const uint16_t*>(g), R, I, static_cast<uint8_t*>(h_q), s_h);
}

cudaError_t launch_moe_combine(const void* y, const float* w, const int32_t* rows, int T, int H, int k, void* out,
                               bool pdl, cudaStream_t st) {
    const int64_t n = (int64_t)T * (H / 8);
    return launch(moe_combine_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, pdl, st,
                  static_cast<const uint16_t*>(y), w, rows, T, H, k, static_cast<uint16_t*>(out));
}

}  // namespace qlin
