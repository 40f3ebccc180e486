// quantize_bs.cu -- quantisation into the block-scaled formats MXFP8 and NVFP4.
//
// The page "Helion in vLLM: A Unified Route to Tunable Linear Kernels"
// (introduction) lists NVFP4 among the formats vLLM's linear layers serve;
// the formats themselves follow their public definitions (OCP Microscaling
// Formats v1.0 for MXFP8; NVIDIA's two-level E2M1 / E4M3 / fp32 scheme for
// NVFP4):
//
//   MXFP8  block of 32 along K, E8M0 scale 2^e with e = floor(log2 amax) - 8
//          (clamped to [-127, 127]); q = e4m3_rn_satfinite(x * 2^-e)
//          (x * 2^-e is exact, so the conversion is the only rounding)
//   NVFP4  block of 16 along K, s = e4m3_rn_satfinite((amax / 6) / g),
//          d = s * g, q = e2m1_rn_satfinite(x / d), g the tensor's decode scale
//   amax == 0 (MXFP8) or d == 0 (NVFP4): every code +0.
//
// One pass over HBM: a warp takes U chunks of 256 elements of one row, one
// 16-byte vector (8 bf16) per lane per chunk, all loads issued before any
// arithmetic.  The block maximum is a 4-lane (MXFP8) or 2-lane (NVFP4)
// shuffle reduction.  Each 128-element (MXFP8) or 64-element (NVFP4) atom's
// four scale bytes are gathered into one lane and written as one 32-bit word
// at the atom's place in the tiled scale layout the GEMM's tensor cores read:
// 512 bytes per (128-row group, atom), row r's word at (r%32)*16 + ((r/32)%4)*4.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "internal.h"
#include "pdl.cuh"
#include "quant_math.cuh"

namespace qlin {

namespace {

using namespace qm;

constexpr int kBsThreads = 256;
constexpr int kBsChunks = 4;  // 256-element chunks per warp task (loads in flight per lane)

__device__ __forceinline__ uint4 ld_stream_bs(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Byte offset of row r's scale word of atom a in the tiled layout.
__device__ __forceinline__ size_t sf_word_offset(int64_t r, int64_t atoms, int64_t a) {
    return ((size_t)(r >> 7) * (size_t)atoms + (size_t)a) * 512u + (size_t)(r & 31) * 16u + (size_t)((r >> 5) & 3) * 4u;
}

// Exact value of an E4M3 code with the sign bit clear (a block scale).
__device__ __forceinline__ float e4m3_pos_value(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    if (e == 0) return __fmul_rn((float)m, 0x1p-9f);
    return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Two floats -> one byte of two E2M1 codes, lo in the low nibble.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
    uint32_t out;
    asm("{\n\t.reg .b8 b;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\t"
        "cvt.u32.u8 %0, b;\n\t}"
        : "=r"(out)
        : "f"(hi), "f"(lo));
    return out;
}

// Gather the byte held by lanes base, base+step, base+2 step, base+3 step
// (base = this lane rounded down to 4 step) into one little-endian word.
__device__ __forceinline__ uint32_t gather4(uint32_t byte, int lane, int step) {
    const int base = lane & ~(4 * step - 1);
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) w |= (__shfl_sync(0xffffffffu, byte, base + j * step) & 0xFFu) << (8 * j);
    return w;
}

template <int U>
__global__ void __launch_bounds__(kBsThreads)
    quantize_mxfp8_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                          uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t groups = (cols + 256 * U - 1) / (256 * U);  // warp tasks per row
    const int64_t tasks = rows * groups;
    const int64_t atoms = cols / 128;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < tasks; t += nwarps) {
        const int64_t r = t / groups;
        const int64_t c0 = (t % groups) * (256 * U) + lane * 8;
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = c0 + u * 256;
            v[u] = c < cols ? ld_stream_bs(x + r * ld + c) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = c0 + u * 256;
            float f[8];
            unpack8(v[u], f);
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            // e = floor(log2 amax) - 8 from the exponent field (a subnormal
            // amax has floor(log2) <= -127, so its e clamps to -127)
            const int ef = (int)(__float_as_uint(amax) >> 23);
            const int e = max(ef - 135, -127);
            const float mul = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, exact
            uint2 codes = make_uint2(0u, 0u);
            if (amax != 0.f) {
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    w[i] = __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(f[2 * i], mul), __fmul_rn(f[2 * i + 1], mul)),
                                                    __NV_SATFINITE, __NV_E4M3);
                codes.x = w[0] | (w[1] << 16);
                codes.y = w[2] | (w[3] << 16);
            }
            const uint32_t code_byte = amax != 0.f ? (uint32_t)(e + 127) : 0u;
            const uint32_t word = gather4(code_byte, lane, 4);  // the 4 blocks of this lane's 128-element atom
            if (c < cols) {
                *reinterpret_cast<uint2*>(q + r * cols + c) = codes;
                if ((lane & 15) == 0) *reinterpret_cast<uint32_t*>(sf + sf_word_offset(r, atoms, c >> 7)) = word;
            }
        }
    }
}

template <int U>
__global__ void __launch_bounds__(kBsThreads)
    quantize_nvfp4_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                          const float* __restrict__ gp, uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
    pdl_wait();
    pdl_launch_dependents();
    const float g = __ldg(gp);
    const int lane = threadIdx.x & 31;
    const int64_t groups = (cols + 256 * U - 1) / (256 * U);
    const int64_t tasks = rows * groups;
    const int64_t atoms = cols / 64;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < tasks; t += nwarps) {
        const int64_t r = t / groups;
        const int64_t c0 = (t % groups) * (256 * U) + lane * 8;
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = c0 + u * 256;
            v[u] = c < cols ? ld_stream_bs(x + r * ld + c) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = c0 + u * 256;
            float f[8];
            unpack8(v[u], f);
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            float tq = __fdiv_rn(amax, 6.0f);
            tq = __fdiv_rn(tq, g);
            const uint32_t s = (uint32_t)__nv_cvt_float_to_fp8(tq, __NV_SATFINITE, __NV_E4M3);
            const float d = __fmul_rn(e4m3_pos_value(s), g);
            uint32_t codes = 0;
            if (d != 0.f) {
                const Divisor dv = make_divisor(d);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    codes |= e2m1x2(quotient(f[2 * i], dv), quotient(f[2 * i + 1], dv)) << (8 * i);
            }
            const uint32_t word = gather4(s, lane, 2);  // the 4 blocks of this lane's 64-element atom
            if (c < cols) {
                *reinterpret_cast<uint32_t*>(q + r * (cols / 2) + c / 2) = codes;
                if ((lane & 7) == 0) *reinterpret_cast<uint32_t*>(sf + sf_word_offset(r, atoms, c >> 6)) = word;
            }
        }
    }
}

template <typename... KArgs, typename... Args>
cudaError_t launch_bs(void (*kern)(KArgs...), int64_t tasks, bool pdl, cudaStream_t st, Args... args) {
    int dev = 0, sms = kNumSMsB200;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t warps_per_cta = kBsThreads / 32;
    const int64_t want = (tasks + warps_per_cta - 1) / warps_per_cta;
    const int64_t cap = (int64_t)sms * 8;  // 8 CTAs of 256 threads fill an SM
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::max<int64_t>(1, std::min(want, cap)));
    cfg.blockDim = dim3(kBsThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace

cudaError_t launch_quantize_block_scaled(int fmt, const void* x, int64_t rows, int64_t cols, int64_t ld,
                                         const float* g, void* q, void* sf, bool pdl, cudaStream_t st) {
    const auto* xb = static_cast<const uint16_t*>(x);
    auto* qb = static_cast<uint8_t*>(q);
    auto* sb = static_cast<uint8_t*>(sf);
    const int64_t tasks = rows * ((cols + 256 * kBsChunks - 1) / (256 * kBsChunks));
    if (fmt == QLIN_FMT_MXFP8)
        return launch_bs(quantize_mxfp8_kernel<kBsChunks>, tasks, pdl, st, xb, rows, cols, ld, qb, sb);
    return launch_bs(quantize_nvfp4_kernel<kBsChunks>, tasks, pdl, st, xb, rows, cols, ld, g, qb, sb);
}

}  // namespace qlin
