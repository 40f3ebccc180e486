// gemm.cu -- persistent sm_100a scaled GEMM for the quantized linear layer.
//
// C = (A_q W_q^T) * s_a * s_w + bias in bf16, INT8 (kind::i8, int32 TMEM
// accumulators), FP8 e4m3 per-token/per-channel and Block-FP8 (kind::f8f6f4,
// fp32 TMEM accumulators), with the three strategies the page "Helion in vLLM:
// A Unified Route to Tunable Linear Kernels" lists in "What the integration
// changes": ordinary GEMM, Split-K ("divides the K dimension across more
// thread blocks") and Swap-AB ("rewrites the multiplication through
// transposes": C^T = W A^T, so a small M becomes the narrow MMA side).
//
// One CTA per SM runs a static round-robin over work units.  Warp roles:
//   warp 4  TMA producer: 128-byte-swizzled K-major tiles of both operands
//           into a STAGES-deep shared-memory ring (mbarrier full/empty pairs)
//   warp 5  TMEM allocator + MMA issuer: one thread issues tcgen05.mma
//           (M = 128, N = tile_n, K = 32 per instruction) into one of two
//           TMEM accumulator buffers and commits to mbarriers
//   warps 0-3  epilogue: tcgen05.ld of the accumulator (warp w owns TMEM
//           lanes 32w..32w+31), scales, bias, bf16 convert, global store.
//
// Fixed reduction order (batch invariance).  K is cut into S segments fixed
// per (format, N, K).  Each segment is accumulated on its own in TMEM
// (Block-FP8: each 128-wide K block is, and is promoted into an fp32 segment
// sum in registers with one fma per block), and the per-segment values are
// added in order s = 0..S-1 starting from +0.  The plain variant keeps the
// running total in a third TMEM region, the Split-K variant writes each
// segment to a workspace and the last CTA to arrive on the tile's ticket adds
// them in the same order; so every variant gives bitwise the same C, and a
// row of C never depends on the other rows.  INT8 sums are exact, so the
// plain INT8 variant simply accumulates all of K in one TMEM buffer.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "internal.h"

namespace qlin {
__device__ int g_device_status = 0;
}

#include "ptx.cuh"

namespace qlin {

namespace {

struct GemmArgs {
    const float* s_a;
    const float* s_w;
    const uint16_t* bias;
    void* c;
    int32_t* tickets;
    uint32_t* partials;
    int M, N;
    int kblocks, S, kb_per_seg;
    int p_tiles, units;
    int spread, out_i32;
};

constexpr int kThreads = 192;  // 4 epilogue warps + producer warp + MMA warp
constexpr int kSmemBudget = 232448 - 1024 - 256;

__host__ __device__ constexpr int pow2_at_least(int v) {
    int p = 32;
    while (p < v) p <<= 1;
    return p;
}

template <int FMT, bool SWAP, int BN>
struct Cfg {
    static constexpr bool INT8 = (FMT == QLIN_FMT_INT8);
    static constexpr bool BLOCK = (FMT == QLIN_FMT_FP8_BLOCK);
    static constexpr int BM = 128;                 // P rows per tile (MMA M)
    static constexpr int BK = 128;                 // K bytes per stage: one swizzle atom
    static constexpr int P_BYTES = BM * BK;
    static constexpr int Q_BYTES = BN * BK;
    static constexpr int STAGE_BYTES = P_BYTES + Q_BYTES;
    static constexpr int STAGES_FIT = kSmemBudget / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
    static constexpr int SW = BN < 32 ? BN : 32;   // columns per TMEM load
    static constexpr int NSLICE = BN / SW;
    static constexpr int ACC_COLS = BN < 32 ? 32 : BN;
    static constexpr bool MULTI = BN <= 128;       // may run multi-chunk units
    static constexpr int TOTAL_COL = 2 * ACC_COLS; // running-total region
    static constexpr int TMEM_COLS = pow2_at_least(2 * ACC_COLS + (MULTI ? ACC_COLS : 0));
    static constexpr uint32_t IDESC = make_idesc(INT8, 128, BN);
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
    static_assert(TMEM_COLS <= 512, "TMEM overflow");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
};

struct Unit {
    int tile, seg, pt, qt, kb0, kb1, chunk_kb;
};

template <int FMT>
__device__ __forceinline__ Unit decode_unit(const GemmArgs& a, int u) {
    Unit r;
    if (a.spread) {
        r.seg = u % a.S;
        r.tile = u / a.S;
        r.kb0 = r.seg * a.kb_per_seg;
        r.kb1 = r.kb0 + a.kb_per_seg;
    } else {
        r.seg = 0;
        r.tile = u;
        r.kb0 = 0;
        r.kb1 = a.kblocks;
    }
    r.pt = r.tile % a.p_tiles;
    r.qt = r.tile / a.p_tiles;
    if (FMT == QLIN_FMT_FP8_BLOCK)
        r.chunk_kb = 1;
    else if (FMT == QLIN_FMT_INT8)
        r.chunk_kb = r.kb1 - r.kb0;
    else
        r.chunk_kb = a.kb_per_seg;
    return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat16 l = __float2bfloat16_rn(lo);
    const __nv_bfloat16 h = __float2bfloat16_rn(hi);
    return (uint32_t)__bfloat16_as_ushort(l) | ((uint32_t)__bfloat16_as_ushort(h) << 16);
}

// Final epilogue of one slice of SW accumulator columns.  `v` holds fp32 bits
// (FP8 formats: the summed value) or int32 (INT8: the exact accumulator).
template <int FMT, bool SWAP, int BN>
__device__ __forceinline__ void store_slice(const GemmArgs& a, const Unit& un, int j, int row_lane,
                                            const uint32_t* v) {
    using C = Cfg<FMT, SWAP, BN>;
    constexpr int SW = C::SW;
    if constexpr (!SWAP) {
        const int m = un.pt * 128 + row_lane;
        if (m >= a.M) return;
        const int n0 = un.qt * BN + j * SW;
        if (a.out_i32) {
            int32_t* out = static_cast<int32_t*>(a.c) + (size_t)m * a.N + n0;
#pragma unroll
            for (int h = 0; h < SW / 16; ++h) {
                if (n0 + h * 16 + 16 <= a.N) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        reinterpret_cast<uint4*>(out + h * 16)[q4] =
                            make_uint4(v[h * 16 + q4 * 4], v[h * 16 + q4 * 4 + 1], v[h * 16 + q4 * 4 + 2],
                                       v[h * 16 + q4 * 4 + 3]);
                }
            }
            return;
        }
        float sa = 0.f;
        if constexpr (!C::BLOCK) sa = __ldg(a.s_a + m);
        uint16_t* out = reinterpret_cast<uint16_t*>(a.c) + (size_t)m * a.N + n0;
#pragma unroll
        for (int h = 0; h < SW / 16; ++h) {
            if (n0 + h * 16 + 16 > a.N) continue;
            uint32_t packed[8];
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                float y[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int c = h * 16 + i + e;
                    const int n = n0 + c;
                    float t;
                    if constexpr (C::INT8)
                        t = __int2float_rn((int)v[c]);
                    else
                        t = __uint_as_float(v[c]);
                    if constexpr (!C::BLOCK) {
                        t = __fmul_rn(t, sa);
                        t = __fmul_rn(t, __ldg(a.s_w + n));
                        if (a.bias) t = __fadd_rn(t, __uint_as_float((uint32_t)__ldg(a.bias + n) << 16));
                    }
                    y[e] = t;
                }
                packed[i / 2] = pack_bf16x2(y[0], y[1]);
            }
            reinterpret_cast<uint4*>(out + h * 16)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            reinterpret_cast<uint4*>(out + h * 16)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        }
    } else {
        const int n = un.pt * 128 + row_lane;
        if (n >= a.N) return;
        const int m0 = un.qt * BN + j * SW;
        if (a.out_i32) {
            int32_t* out = static_cast<int32_t*>(a.c);
#pragma unroll
            for (int c = 0; c < SW; ++c)
                if (m0 + c < a.M) out[(size_t)(m0 + c) * a.N + n] = (int32_t)v[c];
            return;
        }
        float swv = 0.f, bv = 0.f;
        if constexpr (!C::BLOCK) {
            swv = __ldg(a.s_w + n);
            if (a.bias) bv = __uint_as_float((uint32_t)__ldg(a.bias + n) << 16);
        }
        uint16_t* out = reinterpret_cast<uint16_t*>(a.c);
#pragma unroll
        for (int c = 0; c < SW; ++c) {
            const int m = m0 + c;
            if (m >= a.M) break;
            float t;
            if constexpr (C::INT8)
                t = __int2float_rn((int)v[c]);
            else
                t = __uint_as_float(v[c]);
            if constexpr (!C::BLOCK) {
                t = __fmul_rn(t, __ldg(a.s_a + m));
                t = __fmul_rn(t, swv);
                if (a.bias) t = __fadd_rn(t, bv);
            }
            out[(size_t)m * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(t));
        }
    }
}

template <int SW>
__device__ __forceinline__ void tmem_load_slice(uint32_t taddr, uint32_t (&r)[SW]) {
    if constexpr (SW == 32)
        tmem_ld32(taddr, r);
    else
        tmem_ld16(taddr, r);
}

template <int SW>
__device__ __forceinline__ void tmem_store_slice(uint32_t taddr, const uint32_t (&r)[SW]) {
    if constexpr (SW == 32)
        tmem_st32(taddr, r);
    else
        tmem_st16(taddr, r);
}

// Split-K: write this unit's segment value for slice j to the workspace.
template <int SW>
__device__ __forceinline__ uint32_t* partial_ptr(const GemmArgs& a, int tile, int seg, int j, int nslice,
                                                 int row_lane) {
    return a.partials + ((((size_t)tile * a.S + seg) * nslice + j) * 128 + row_lane) * SW;
}

template <int SW>
__device__ __forceinline__ void store_partial(uint32_t* p, const uint32_t (&v)[SW]) {
#pragma unroll
    for (int q = 0; q < SW / 4; ++q)
        reinterpret_cast<uint4*>(p)[q] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// Split-K: after every segment of a tile has been written, the last CTA to
// arrive adds them in segment order and runs the final epilogue.
template <int FMT, bool SWAP, int BN>
__device__ __forceinline__ void splitk_finish(const GemmArgs& a, const Unit& un, int row_lane, int* bcast) {
    using C = Cfg<FMT, SWAP, BN>;
    constexpr int SW = C::SW;
    __threadfence();
    named_bar_sync(1, 128);
    if (threadIdx.x == 0) {
        const int old = atomicAdd(a.tickets + un.tile, 1);
        *bcast = (old == a.S - 1) ? 1 : 0;
    }
    named_bar_sync(1, 128);
    const bool last = *(volatile int*)bcast != 0;
    if (!last) return;
    __threadfence();
#pragma unroll 1
    for (int j = 0; j < C::NSLICE; ++j) {
        uint32_t acc[SW];
        if constexpr (C::INT8) {
            int32_t t[SW];
#pragma unroll
            for (int c = 0; c < SW; ++c) t[c] = 0;
#pragma unroll 1
            for (int s = 0; s < a.S; ++s) {
                const uint4* p = reinterpret_cast<const uint4*>(partial_ptr<SW>(a, un.tile, s, j, C::NSLICE, row_lane));
#pragma unroll
                for (int q = 0; q < SW / 4; ++q) {
                    const uint4 w = __ldcg(p + q);
                    t[4 * q] += (int32_t)w.x;
                    t[4 * q + 1] += (int32_t)w.y;
                    t[4 * q + 2] += (int32_t)w.z;
                    t[4 * q + 3] += (int32_t)w.w;
                }
            }
#pragma unroll
            for (int c = 0; c < SW; ++c) acc[c] = (uint32_t)t[c];
        } else {
            float t[SW];
#pragma unroll
            for (int c = 0; c < SW; ++c) t[c] = 0.f;
#pragma unroll 1
            for (int s = 0; s < a.S; ++s) {
                const uint4* p = reinterpret_cast<const uint4*>(partial_ptr<SW>(a, un.tile, s, j, C::NSLICE, row_lane));
#pragma unroll
                for (int q = 0; q < SW / 4; ++q) {
                    const uint4 w = __ldcg(p + q);
                    t[4 * q] = __fadd_rn(t[4 * q], __uint_as_float(w.x));
                    t[4 * q + 1] = __fadd_rn(t[4 * q + 1], __uint_as_float(w.y));
                    t[4 * q + 2] = __fadd_rn(t[4 * q + 2], __uint_as_float(w.z));
                    t[4 * q + 3] = __fadd_rn(t[4 * q + 3], __uint_as_float(w.w));
                }
            }
#pragma unroll
            for (int c = 0; c < SW; ++c) acc[c] = __float_as_uint(t[c]);
        }
        store_slice<FMT, SWAP, BN>(a, un, j, row_lane, acc);
    }
    if (threadIdx.x == 0) a.tickets[un.tile] = 0;  // leave the ticket zeroed for the next call
}

// Hand one segment value (slice j, SW columns) to the running sum: Split-K
// writes it out; the plain variant adds it to the TMEM total (or, on the last
// segment, finishes the tile).
template <int FMT, bool SWAP, int BN>
__device__ __forceinline__ void consume_segment_slice(const GemmArgs& a, const Unit& un, int seg_no, int j,
                                                      int row_lane, uint32_t t_total,
                                                      const uint32_t (&segv)[Cfg<FMT, SWAP, BN>::SW]) {
    using C = Cfg<FMT, SWAP, BN>;
    constexpr int SW = C::SW;
    if (a.spread) {
        store_partial<SW>(partial_ptr<SW>(a, un.tile, un.seg, j, C::NSLICE, row_lane), segv);
        return;
    }
    uint32_t t[SW];
    if constexpr (C::INT8) {
#pragma unroll
        for (int c = 0; c < SW; ++c) t[c] = segv[c];  // exact: whole K in one accumulator
        store_slice<FMT, SWAP, BN>(a, un, j, row_lane, t);
        return;
    } else {
        if (seg_no == 0) {
#pragma unroll
            for (int c = 0; c < SW; ++c) t[c] = __float_as_uint(__fadd_rn(0.f, __uint_as_float(segv[c])));
        } else {
            uint32_t prev[SW];
            tmem_load_slice<SW>(t_total + j * SW, prev);
            tc_wait_ld();
#pragma unroll
            for (int c = 0; c < SW; ++c)
                t[c] = __float_as_uint(__fadd_rn(__uint_as_float(prev[c]), __uint_as_float(segv[c])));
        }
        if (seg_no == a.S - 1) {
            store_slice<FMT, SWAP, BN>(a, un, j, row_lane, t);
        } else {
            if constexpr (C::MULTI) tmem_store_slice<SW>(t_total + j * SW, t);
        }
    }
}

template <int FMT, bool SWAP, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    qlin_gemm_kernel(const __grid_constant__ CUtensorMap tmap_p, const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ GemmArgs args) {
    using C = Cfg<FMT, SWAP, BN>;
    constexpr int STAGES = C::STAGES;
    constexpr int SW = C::SW;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sP = smem;
    uint8_t* sQ = smem + (size_t)STAGES * C::P_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sQ + (size_t)STAGES * C::Q_BYTES);
    const uint32_t full0 = smem_u32(bars);
    const uint32_t empty0 = smem_u32(bars + STAGES);
    const uint32_t tfull0 = smem_u32(bars + 2 * STAGES);
    const uint32_t tempty0 = smem_u32(bars + 2 * STAGES + 2);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
    int* bcast = reinterpret_cast<int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (warp == 4 && lane == 0) {
        prefetch_tmap(&tmap_p);
        prefetch_tmap(&tmap_q);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull0 + 8 * b, 1);
            mbar_init(tempty0 + 8 * b, 128);
        }
        fence_mbarrier_init();
    }
    if (warp == 5) {
        tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 4) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_a = policy_evict_last();
            const uint64_t pol_p = SWAP ? pol_w : pol_a;
            const uint64_t pol_q = SWAP ? pol_a : pol_w;
            uint32_t stage = 0, phase = 0;
            for (int u = blockIdx.x; u < args.units; u += gridDim.x) {
                const Unit un = decode_unit<FMT>(args, u);
                for (int kb = un.kb0; kb < un.kb1; ++kb) {
                    if (!mbar_wait(empty0 + 8 * stage, phase ^ 1)) goto done;
                    mbar_arrive_expect_tx(full0 + 8 * stage, C::STAGE_BYTES);
                    tma_load_2d(smem_u32(sP + (size_t)stage * C::P_BYTES), &tmap_p, kb * 128, un.pt * 128,
                                full0 + 8 * stage, pol_p);
                    tma_load_2d(smem_u32(sQ + (size_t)stage * C::Q_BYTES), &tmap_q, kb * 128, un.qt * BN,
                                full0 + 8 * stage, pol_q);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
    } else if (warp == 5) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0, abuf = 0, aphase = 0;
            for (int u = blockIdx.x; u < args.units; u += gridDim.x) {
                const Unit un = decode_unit<FMT>(args, u);
                for (int c0 = un.kb0; c0 < un.kb1; c0 += un.chunk_kb) {
                    if (!mbar_wait(tempty0 + 8 * abuf, aphase ^ 1)) goto done;
                    tc_fence_after();
                    const uint32_t d = tmem_base + abuf * C::ACC_COLS;
                    for (int kb = c0; kb < c0 + un.chunk_kb; ++kb) {
                        if (!mbar_wait(full0 + 8 * stage, phase)) goto done;
                        tc_fence_after();
                        const uint64_t adesc = smem_desc_k_sw128(smem_u32(sP + (size_t)stage * C::P_BYTES));
                        const uint64_t bdesc = smem_desc_k_sw128(smem_u32(sQ + (size_t)stage * C::Q_BYTES));
#pragma unroll
                        for (int k = 0; k < 4; ++k)  // 4 x K=32 bytes per 128-byte stage
                            tc_mma<C::INT8>(d, adesc + 2 * k, bdesc + 2 * k, C::IDESC,
                                            (kb > c0 || k > 0) ? 1u : 0u);
                        tc_commit(empty0 + 8 * stage);
                        if (++stage == STAGES) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                    tc_commit(tfull0 + 8 * abuf);
                    abuf ^= 1;
                    if (abuf == 0) aphase ^= 1;
                }
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int row_lane = warp * 32 + lane;
        const uint32_t t_lane = tmem_base + ((uint32_t)(warp * 32) << 16);
        const uint32_t t_total = t_lane + C::TOTAL_COL;
        uint32_t abuf = 0, aphase = 0;
        for (int u = blockIdx.x; u < args.units; u += gridDim.x) {
            const Unit un = decode_unit<FMT>(args, u);
            const int nchunks = (un.kb1 - un.kb0) / un.chunk_kb;
            if (nchunks == 1 && !C::BLOCK) {
                // one accumulator holds the whole unit: stream it slice by slice
                if (!mbar_wait(tfull0 + 8 * abuf, aphase)) goto done;
                tc_fence_after();
                const uint32_t tacc = t_lane + abuf * C::ACC_COLS;
#pragma unroll 1
                for (int j = 0; j < C::NSLICE; ++j) {
                    uint32_t v[SW];
                    tmem_load_slice<SW>(tacc + j * SW, v);
                    tc_wait_ld();
                    if (j == C::NSLICE - 1) {  // accumulator fully read: hand it back
                        tc_fence_before();
                        mbar_arrive(tempty0 + 8 * abuf);
                    }
                    consume_segment_slice<FMT, SWAP, BN>(args, un, un.seg, j, row_lane, t_total, v);
                }
                abuf ^= 1;
                if (abuf == 0) aphase ^= 1;
            } else if constexpr (C::MULTI) {
                if constexpr (C::BLOCK) {
                    // Block-FP8: promote every 128-wide K block into the fp32
                    // segment sum: seg = fma(P_kb, s_a[m,kb] * s_w[n/128,kb], seg)
                    float seg[BN];
                    for (int c0 = un.kb0; c0 < un.kb1; ++c0) {
                        const int rel = c0 - (args.spread ? un.kb0 : 0);
                        const int seg_no = args.spread ? un.seg : rel / args.kb_per_seg;
                        const bool seg_start = (rel % args.kb_per_seg) == 0;
                        const bool seg_end = ((rel + 1) % args.kb_per_seg) == 0;
                        float row_scale = 0.f, swv;
                        if constexpr (!SWAP) {
                            const int m = un.pt * 128 + row_lane;
                            swv = __ldg(args.s_w + (size_t)((un.qt * BN) >> 7) * args.kblocks + c0);
                            if (m < args.M) row_scale = __fmul_rn(__ldg(args.s_a + (size_t)m * args.kblocks + c0), swv);
                        } else {
                            swv = __ldg(args.s_w + (size_t)un.pt * args.kblocks + c0);
                        }
                        if (seg_start) {
#pragma unroll
                            for (int c = 0; c < BN; ++c) seg[c] = 0.f;
                        }
                        if (!mbar_wait(tfull0 + 8 * abuf, aphase)) goto done;
                        tc_fence_after();
                        const uint32_t tacc = t_lane + abuf * C::ACC_COLS;
#pragma unroll
                        for (int j = 0; j < C::NSLICE; ++j) {
                            uint32_t v[SW];
                            tmem_load_slice<SW>(tacc + j * SW, v);
                            tc_wait_ld();
#pragma unroll
                            for (int c = 0; c < SW; ++c) {
                                float sc;
                                if constexpr (!SWAP) {
                                    sc = row_scale;
                                } else {
                                    const int m = un.qt * BN + j * SW + c;
                                    sc = (m < args.M)
                                             ? __fmul_rn(__ldg(args.s_a + (size_t)m * args.kblocks + c0), swv)
                                             : 0.f;
                                }
                                seg[j * SW + c] = __fmaf_rn(__uint_as_float(v[c]), sc, seg[j * SW + c]);
                            }
                        }
                        tc_fence_before();
                        mbar_arrive(tempty0 + 8 * abuf);
                        abuf ^= 1;
                        if (abuf == 0) aphase ^= 1;
                        if (seg_end) {
#pragma unroll
                            for (int j = 0; j < C::NSLICE; ++j) {
                                uint32_t sv[SW];
#pragma unroll
                                for (int c = 0; c < SW; ++c) sv[c] = __float_as_uint(seg[j * SW + c]);
                                consume_segment_slice<FMT, SWAP, BN>(args, un, seg_no, j, row_lane, t_total, sv);
                            }
                            tc_wait_st();
                        }
                    }
                } else {
                    // FP8 per-token, plain variant with S > 1: one chunk per
                    // segment, summed into the TMEM running total in order.
                    int seg_no = 0;
                    for (int c0 = un.kb0; c0 < un.kb1; c0 += un.chunk_kb, ++seg_no) {
                        if (!mbar_wait(tfull0 + 8 * abuf, aphase)) goto done;
                        tc_fence_after();
                        const uint32_t tacc = t_lane + abuf * C::ACC_COLS;
#pragma unroll 1
                        for (int j = 0; j < C::NSLICE; ++j) {
                            uint32_t v[SW];
                            tmem_load_slice<SW>(tacc + j * SW, v);
                            tc_wait_ld();
                            consume_segment_slice<FMT, SWAP, BN>(args, un, seg_no, j, row_lane, t_total, v);
                        }
                        tc_wait_st();
                        tc_fence_before();
                        mbar_arrive(tempty0 + 8 * abuf);
                        abuf ^= 1;
                        if (abuf == 0) aphase ^= 1;
                    }
                }
            }
            if (args.spread) splitk_finish<FMT, SWAP, BN>(args, un, row_lane, bcast);
        }
    }
done:
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// K-major 8-bit operand [rows, K] as a 2-D tensor map with a (128 B x box_rows) box.
bool make_operand_tmap(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int FMT, bool SWAP, int BN>
qlin_status launch_instance(const GemmPlan& plan, const GemmOperands& ops, cudaStream_t st) {
    using C = Cfg<FMT, SWAP, BN>;
    auto kern = qlin_gemm_kernel<FMT, SWAP, BN>;
    // one attribute set per device is enough; repeating it is cheap and safe
    static int configured_device = -1;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QLIN_ERR_CUDA;
    if (configured_device != dev) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM) != cudaSuccess)
            return QLIN_ERR_CUDA;
        configured_device = dev;
    }
    alignas(64) CUtensorMap tp, tq;
    const void* p_base = SWAP ? ops.w_q : ops.a_q;
    const void* q_base = SWAP ? ops.a_q : ops.w_q;
    if (!make_operand_tmap(&tp, p_base, plan.p_rows, plan.K, 128)) return QLIN_ERR_CUDA;
    if (!make_operand_tmap(&tq, q_base, plan.q_rows, plan.K, BN)) return QLIN_ERR_CUDA;
    GemmArgs a;
    a.s_a = ops.s_a;
    a.s_w = ops.s_w;
    a.bias = static_cast<const uint16_t*>(ops.bias);
    a.c = ops.c;
    a.tickets = plan.spread ? static_cast<int32_t*>(ops.workspace) : nullptr;
    a.partials = plan.spread ? reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ops.workspace) + plan.ticket_bytes)
                             : nullptr;
    a.M = (int)plan.M;
    a.N = (int)plan.N;
    a.kblocks = plan.kblocks;
    a.S = plan.k_segments;
    a.kb_per_seg = plan.kb_per_seg;
    a.p_tiles = (int)plan.p_tiles;
    a.units = (int)plan.units;
    a.spread = plan.spread ? 1 : 0;
    a.out_i32 = ops.out_i32 ? 1 : 0;
    kern<<<plan.grid, kThreads, C::SMEM, st>>>(tp, tq, a);
    return cudaGetLastError() == cudaSuccess ? QLIN_OK : QLIN_ERR_CUDA;
}

template <int FMT>
qlin_status launch_fmt(const GemmPlan& p, const GemmOperands& ops, cudaStream_t st) {
    if (p.swap) {
        switch (p.tile_n) {
            case 16: return launch_instance<FMT, true, 16>(p, ops, st);
            case 32: return launch_instance<FMT, true, 32>(p, ops, st);
            case 64: return launch_instance<FMT, true, 64>(p, ops, st);
            default: return QLIN_ERR_UNSUPPORTED;
        }
    }
    switch (p.tile_n) {
        case 128: return launch_instance<FMT, false, 128>(p, ops, st);
        case 256:
            if constexpr (FMT != QLIN_FMT_FP8_BLOCK) return launch_instance<FMT, false, 256>(p, ops, st);
            return QLIN_ERR_UNSUPPORTED;
        default: return QLIN_ERR_UNSUPPORTED;
    }
}

}  // namespace

int gemm_stages_for(int tile_n) {
    const int stage = 128 * 128 + tile_n * 128;
    const int s = kSmemBudget / stage;
    return s > 12 ? 12 : s;
}

size_t gemm_smem_bytes_for(int tile_n) {
    return 1024 + (size_t)gemm_stages_for(tile_n) * (128 * 128 + tile_n * 128) + 256;
}

cudaError_t device_status_read_clear(int* value) {
    cudaError_t e = cudaMemcpyFromSymbol(value, g_device_status, sizeof(int));
    if (e != cudaSuccess || *value == 0) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
}

qlin_status launch_gemm(const GemmPlan& plan, const GemmOperands& ops, cudaStream_t st) {
    switch (plan.fmt) {
        case QLIN_FMT_INT8: return launch_fmt<QLIN_FMT_INT8>(plan, ops, st);
        case QLIN_FMT_FP8: return launch_fmt<QLIN_FMT_FP8>(plan, ops, st);
        case QLIN_FMT_FP8_BLOCK: return launch_fmt<QLIN_FMT_FP8_BLOCK>(plan, ops, st);
        default: return QLIN_ERR_INVALID_ARG;
    }
}

}  // namespace qlin
