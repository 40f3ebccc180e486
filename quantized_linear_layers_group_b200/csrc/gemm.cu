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
//   warp 8  TMA producer: 128-byte-swizzled K-major tiles of both operands
//           into a STAGES-deep shared-memory ring (mbarrier full/empty pairs)
//   warp 9  TMEM allocator + MMA issuer: one thread issues tcgen05.mma
//           (M = 128, N = tile_n, K = 32 per instruction) into one of two
//           TMEM accumulator buffers and commits to mbarriers
//   warps 0-7  epilogue: warp w reads TMEM lanes 32(w%4)..32(w%4)+31 (the
//           hardware's lane quadrant for that warp) and the 32-column slices
//           j with j % 2 == w / 4, so two warps share each quadrant; scales
//           and bias are staged once per tile in shared memory.  Plain tiles
//           leave through bulk tensor stores of 32 x 32 bf16 boxes.
// Plain 256 x 256 tiles may also run on the two CTAs of a cluster
// (cta_group::2): each CTA loads its 128 rows of A and half of the W tile,
// and rank 0 issues M = 256 MMAs that fill both CTAs' accumulators.
//
// Fixed reduction order (batch invariance).  K is cut into S segments fixed
// per (format, N, K).  Each segment is accumulated on its own in TMEM
// (Block-FP8: each 128-wide K block is, and is promoted into an fp32 segment
// sum kept in TMEM with one fma per block), and the per-segment values are
// added in order s = 0..S-1 starting from +0.  The plain variant keeps the
// running total in a third TMEM region, the Split-K variant writes each
// segment to a workspace and the last CTA to arrive on the tile's ticket adds
// them in the same order (Swap-AB Split-K with few segments instead runs the
// S segment CTAs of a tile as one thread-block cluster: ranks 1..S-1 store
// their segments into rank 0's shared memory over the cluster's distributed
// shared memory and rank 0 adds them in order); so every variant gives
// bitwise the same C, and a
// row of C never depends on the other rows.  INT8 sums are exact, so the
// plain INT8 variant simply accumulates all of K in one TMEM buffer.
//
// Programmatic dependent launch: with QLIN_PDL the kernel starts while the
// previous kernel of the stream (normally the activation quantiser) is still
// running; the producer streams the first weight tiles before pdl_wait(), and
// everything that reads activations, scales or writes C waits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <algorithm>
#include <cstring>
#include <mutex>

#include "internal.h"

namespace qlin {
__device__ int g_device_status = 0;
}

#include "ptx.cuh"
#include "quant_math.cuh"

namespace qlin {

namespace {

struct GemmArgs {
    const float* s_a;
    const float* s_w;
    const uint16_t* bias;
    void* c;  // bf16 C, or int32 C when out_i32
    int32_t* tickets;
    uint32_t* partials;
    int M, N;
    int kblocks, S, kb_per_seg;
    int p_tiles, units;
    int spread, out_i32;
    // fused activation quantisation: bf16 x [M, K] (row stride ld_x) in,
    // codes and scales also written out (by the CTAs of the first W tile)
    const uint16_t* x;
    int64_t ld_x;
    uint8_t* a_q_out;
    float* s_a_out;
    // grouped GEMM over experts (MoE): A and C rows are grouped by expert,
    // expert e's rows [moe_offsets[e], moe_offsets[e+1]) multiply W rows
    // [e N, e N + N); nullptr / 0 for an ordinary GEMM
    const int32_t* moe_offsets;
    int moe_E;
    // block-scaled formats (MXFP8, NVFP4): tiled scale factors of A and W,
    // 512-byte atoms [row group][atom], sf_atoms atoms per 128-row group
    const uint8_t* sf_a;
    const uint8_t* sf_w;
    int sf_atoms;
};

constexpr int kMoeMaxExperts = kMoeMaxE;
constexpr int kMoeBytes = 2 * (kMoeMaxExperts + 1) * 4;  // expert row offsets and unit prefix sums

// Three warpgroups: warps 0-7 (two warpgroups) run the epilogue; warpgroup 2
// holds the TMA producer (warp 8), the MMA issuer (warp 9) and two idle warps.
// After set-up the register file is rebalanced with setmaxnreg: the epilogue
// warpgroups get kEpiRegs per thread, warpgroup 2 keeps kAuxRegs.  The sum
// must not exceed the CTA's launch allocation (kThreads x the kernel's
// register count), or the increase would wait forever; the host refuses to
// launch a kernel whose register count is below kLaunchRegs.
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kProducerWarp = kEpiWarps;
constexpr int kMmaWarp = kEpiWarps + 1;
constexpr int kThreads = (kEpiWarps + 4) * 32;
constexpr int kEpiRegs = 216;
constexpr int kAuxRegs = 72;
constexpr int kLaunchRegs = (kEpiThreads * kEpiRegs + (kThreads - kEpiThreads) * kAuxRegs + kThreads - 1) / kThreads;
static_assert(kLaunchRegs <= 168, "register split above what a 384-thread CTA is launched with");
static_assert(kEpiRegs % 8 == 0 && kAuxRegs % 8 == 0 && kAuxRegs >= 24 && kEpiRegs <= 256, "setmaxnreg values");
constexpr int kStagingBytes = kEpiWarps * 2048;  // per epilogue warp: one 32x32 bf16 box
constexpr int kScaleBytes = 2 * 256 * 4;         // column scale + column bias of one tile
constexpr int kBarBytes = 512;                  // mbarriers and the TMEM holder
constexpr int kStageBudget = 232448 - 1024 - kBarBytes - kStagingBytes - kScaleBytes - 2112;  // 2112: MoE table

__host__ __device__ constexpr int pow2_at_least(int v) {
    int p = 32;
    while (p < v) p <<= 1;
    return p;
}

template <int FMT, bool SWAP, int BN, bool CSK = false, bool FUSE = false, bool PAIR = false>
struct Cfg {
    // CSK: cluster Split-K (Swap-AB tiles): the K segments of a tile run on the
    // CTAs of one cluster and are reduced in the leader's shared memory.
    // FUSE: (Swap-AB tiles) the epilogue warps quantise the unit's activation
    // rows from bf16 into a resident shared-memory operand; no A loads.
    static_assert(!CSK || SWAP, "cluster Split-K is built for Swap-AB tiles");
    static_assert(!FUSE || (SWAP && !CSK), "fused quantisation is built for Swap-AB tiles");
    // PAIR: plain tiles of 256 P rows on the two CTAs of a cluster; each CTA
    // loads its own 128 rows of A and half (BN/2 rows) of the W tile, and CTA
    // rank 0 issues M=256 MMAs that fill both CTAs' accumulators.
    static_assert(!PAIR || (!SWAP && !CSK && !FUSE && BN == 256 && FMT != QLIN_FMT_FP8_BLOCK),
                  "CTA pairs are built for plain 256-column tiles");
    static_assert(!FUSE || FMT != QLIN_FMT_BF16, "bf16 activations need no quantisation");
    static constexpr int CSK_MAXS = CSK ? cluster_split_max(BN) : 1;  // segments per cluster
    static constexpr int RECV_BYTES = CSK ? (CSK_MAXS - 1) * 128 * BN * 4 : 0;
    static constexpr bool INT8 = (FMT == QLIN_FMT_INT8);
    static constexpr bool BLOCK = (FMT == QLIN_FMT_FP8_BLOCK);
    static constexpr bool BF16 = (FMT == QLIN_FMT_BF16);  // bf16 operands: no scales
    // block-scaled (MXFP8, NVFP4): the tensor core applies per-block scale
    // factors that the MMA thread copies from shared memory into TMEM
    static constexpr bool BS = is_block_scaled(FMT);
    // plain 128 x 128 tiles, or Swap-AB tiles of 32 / 64 activation rows.  The
    // MMA reads the scale of its column n from TMEM column base + n / 32 of a
    // copied 128-row atom, and its scale address must not be offset inside
    // the atom's four columns, so a Swap-AB tile uses rows 0 .. tile_n - 1 of
    // atom 0: the host plans Swap-AB only for M <= tile_n (one activation tile)
    static_assert(!BS || (!CSK && !FUSE && !PAIR && (SWAP ? (BN == 32 || BN == 64) : BN == 128)),
                  "block-scaled formats: plain 128 x 128 or Swap-AB 32 / 64 tiles");
    static constexpr int KIND =
        BS ? (FMT == QLIN_FMT_MXFP8 ? kKindMXF8 : kKindNVF4) : (INT8 ? kKindI8 : (BF16 ? kKindF16 : kKindF8));
    // scale-factor atoms (512 B: 128 rows x 4 scales) per 128-byte K block of
    // one 128-row group: MXFP8 1 (128 elements), NVFP4 4 (256 elements).  The
    // "A" slot holds the P operand's atoms (the MMA's A: activations, or W in
    // Swap-AB), the "B" slot the Q operand's (SF_RGQ row groups: whole atoms,
    // also for a Swap-AB tile that uses 32 or 64 of their rows)
    static constexpr int SF_APK = FMT == QLIN_FMT_NVFP4 ? 4 : 1;
    static constexpr int SF_RGQ = (BN + 127) / 128;
    static constexpr int SFA_BYTES = BS ? 512 * SF_APK : 0;
    static constexpr int SFB_BYTES = BS ? 512 * SF_APK * SF_RGQ : 0;
    static constexpr int SF_BYTES = SFA_BYTES + SFB_BYTES;
    static constexpr int BM = 128;                 // P rows per tile (MMA M)
    static constexpr int BK = 128;                 // K bytes per stage: one swizzle atom
    static constexpr int P_BYTES = BM * BK;
    static constexpr int Q_BYTES = (PAIR ? BN / 2 : BN) * BK;
    static constexpr int STAGE_BYTES = P_BYTES + (FUSE ? 0 : Q_BYTES) + SF_BYTES;
    // FUSE: A codes of one unit, [K block][BN rows x 128 B] in the 128-byte
    // swizzled K-major layout, and the unit's activation scales (2 buffers)
    static constexpr int A_BYTES = FUSE ? 65536 : 0;
    static constexpr int A_MAXKB = FUSE ? A_BYTES / (BN * 128) : 0;  // K blocks per unit, at most
    static constexpr int SA_FLOATS = FUSE ? (FMT == QLIN_FMT_FP8_BLOCK ? BN * A_MAXKB : BN) : 0;
    static constexpr int SA_BYTES = FUSE ? ((2 * SA_FLOATS * 4 + BN * 4 + 1023) / 1024) * 1024 : 0;
    // Block-FP8: per-unit table of scale products s_a*s_w, [K block][P row or Q column]
    static constexpr int BS_KB = 48;                           // K blocks per staged window
    static constexpr int BS_PITCH = (SWAP ? BN : 128) + 1;     // floats; 1 mod 32: no bank conflicts
    static constexpr int BSCALE_BYTES = BLOCK ? ((BS_KB * BS_PITCH * 4 + 1023) / 1024) * 1024 : 0;
    static constexpr int STAGES_FIT = (kStageBudget - BSCALE_BYTES - RECV_BYTES - A_BYTES - SA_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 11 ? 11 : STAGES_FIT;
    static constexpr int SW = BN < 32 ? BN : 32;   // columns per TMEM load / per store box
    static constexpr int NSLICE = BN / SW;
    static constexpr int MY_SLICES = (NSLICE + 1) / 2;  // slices per epilogue warp (at most)
    static constexpr int ACC_COLS = BN < 32 ? 32 : BN;
    static constexpr bool MULTI = BN <= 128;       // may run multi-chunk units
    // TMEM accumulator buffers the MMA fills in turn.  Block-FP8 plain tiles
    // keep their segment sum in registers and use three: the epilogue folds two
    // K blocks in per accumulator wait and the MMA still has a buffer to run
    // ahead into.  (The same pairing on the Swap-AB Block tiles, whose segment
    // sum lives in TMEM, was measured: 3 % faster at tile 32, 20 % slower at
    // tile 64; not used.)
    static constexpr int NACC = (BLOCK && !SWAP) ? 3 : 2;
    static constexpr int SEG_COL = NACC * ACC_COLS;  // Block-FP8 Swap-AB: running segment sum
    static constexpr int TOTAL_COL = (BLOCK ? (SWAP ? NACC + 1 : 3) : 2) * ACC_COLS;  // running total over segments
    // block-scaled: two copies (alternate K blocks) of one K block's scale
    // factors, 4 columns per atom, after the accumulators and running total
    static constexpr int SF_COL = NACC * ACC_COLS + (MULTI ? ACC_COLS : 0) + ((BLOCK && SWAP) ? ACC_COLS : 0);
    static constexpr int SF_COLS = BS ? 4 * SF_APK * (1 + SF_RGQ) : 0;
    static constexpr int TMEM_COLS = pow2_at_least(SF_COL + 2 * SF_COLS);
    static_assert(NACC * ACC_COLS <= TOTAL_COL, "accumulators overlap the running total");
    static_assert(!MULTI || TOTAL_COL + ACC_COLS <= TMEM_COLS, "running total outside the TMEM allocation");
    static_assert(!(BLOCK && SWAP) || (SEG_COL + ACC_COLS <= TOTAL_COL), "segment sum overlaps the running total");
    static constexpr uint32_t IDESC = BS ? make_idesc_bs(KIND, 128, BN) : make_idesc(KIND, PAIR ? 256 : 128, BN);
    // K blocks the MMA thread takes per pass (measured; the MMAs and their order
    // are the same, so C is bitwise the same): 4 for Swap-AB tiles with rings of
    // 8+ stages, fused ones included (3-8 % less time at small M; a fused
    // tile-16 layer at M = 1 1.2 us less), 2 for plain 128-column tiles
    // (6-stage rings, 3-5 %), 1 for the 256-column tiles, whose 4-stage rings
    // need each stage released at once (grouping them cost 10-50 %)
    // Block-FP8 plain tiles: K blocks the epilogue folds in per accumulator wait
    // (at most NACC - 1, so the MMA always has a free buffer)
    static constexpr int BLOCK_PASS = 2;
    static constexpr int MMA_GROUP = (BLOCK || PAIR) ? 1
                                     : (SWAP && STAGES >= 8) ? 4
                                     : (!SWAP && BN == 128 && STAGES >= 6) ? 2 : 1;
    static constexpr size_t STAGING_OFF = (size_t)STAGES * STAGE_BYTES;
    static constexpr size_t SCALE_OFF = STAGING_OFF + kStagingBytes;
    static constexpr size_t BSCALE_OFF = SCALE_OFF + kScaleBytes;
    static constexpr size_t RECV_OFF = BSCALE_OFF + BSCALE_BYTES;
    static constexpr size_t A_OFF = RECV_OFF + RECV_BYTES;
    static constexpr size_t SA_OFF = A_OFF + A_BYTES;
    static constexpr size_t MOE_OFF = SA_OFF + SA_BYTES;
    static constexpr size_t BAR_OFF = MOE_OFF + ((kMoeBytes + 63) / 64) * 64;
    static constexpr size_t SMEM = 1024 + BAR_OFF + kBarBytes;
    // barriers: full/empty per stage, tfull/tempty per accumulator buffer,
    // recv_full/free, a_full/empty; then the TMEM holder and a broadcast word
    static_assert((2 * STAGES + 2 * NACC + 4) * 8 + 8 <= kBarBytes, "barrier area");
    static_assert(!FUSE || A_MAXKB <= BS_KB, "scale window");
    static_assert(TMEM_COLS <= 512, "TMEM overflow");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
    static_assert(SMEM <= 232448, "shared memory");
};

struct Unit {
    int tile, seg, pt, qt, kb0, kb1, chunk_kb;
    // rows of A / C this unit's tile indexes from (row0 ..), how many exist
    // (rows), and the first W row (wrow0): 0, M, 0 for an ordinary GEMM,
    // the expert's group and weight slice for MoE
    int row0, rows, wrow0;
};

// MoE: unit u lies in the expert e with pref[e] <= u < pref[e + 1] (pref =
// prefix sums of the experts' tile counts); within it, tiles go P-side first.
template <bool SWAP, int BN>
__device__ __forceinline__ void decode_moe(const GemmArgs& a, int u, const int32_t* tab, Unit& r) {
    const int32_t* off = tab;
    const int32_t* pref = tab + kMoeMaxExperts + 1;
    int lo = 0, hi = a.moe_E - 1;  // largest e with pref[e] <= u
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pref[mid] <= u) lo = mid; else hi = mid - 1;
    }
    const int e = lo, local = u - pref[e];
    r.row0 = off[e];
    r.rows = off[e + 1] - off[e];
    r.wrow0 = e * a.N;
    const int p_tiles = SWAP ? (a.N + 127) / 128 : (r.rows + 127) / 128;
    r.pt = local % p_tiles;
    r.qt = local / p_tiles;
}

// Pair tiles (PAIR): unit = 256-row tile; pt is this CTA's 128-row half of it.
template <int FMT, bool PAIR = false, bool SWAP = false, int BN = 128>
__device__ __forceinline__ Unit decode_unit(const GemmArgs& a, int u, int rank = 0, const int32_t* moe_tab = nullptr) {
    Unit r;
    r.row0 = 0;
    r.rows = a.M;
    r.wrow0 = 0;
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
    if constexpr (PAIR) {
        const int pairs = (a.p_tiles + 1) >> 1;
        r.pt = 2 * (r.tile % pairs) + rank;
        r.qt = r.tile / pairs;
    } else {
        if (moe_tab != nullptr) {
            decode_moe<SWAP, BN>(a, u, moe_tab, r);
        } else {
            r.pt = r.tile % a.p_tiles;
            r.qt = r.tile / a.p_tiles;
        }
    }
    if (FMT == QLIN_FMT_FP8_BLOCK)
        r.chunk_kb = 1;
    else if (FMT == QLIN_FMT_INT8)
        r.chunk_kb = r.kb1 - r.kb0;
    else
        r.chunk_kb = a.kb_per_seg;
    return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), .y = hi
    return *reinterpret_cast<const uint32_t*>(&p);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ void sts_u4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ void sts_u2(uint32_t addr, uint2 v) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(v.x), "r"(v.y) : "memory");
}
__device__ __forceinline__ uint4 lds_u4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

// Warp-level mbarrier use by the epilogue: one lane polls and the warp then
// proceeds together; one lane arrives for the whole warp once every lane is
// done (the barrier counts warps).  256 threads polling or arriving one by
// one on the same barrier serialise on it.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait_idle(bar, parity) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Next TMEM accumulator buffer (NACC in turn); the parity flips per round.
template <int NACC>
__device__ __forceinline__ void next_acc(uint32_t& abuf, uint32_t& aphase) {
    if (++abuf == NACC) {
        abuf = 0;
        aphase ^= 1;
    }
}

__device__ __forceinline__ void warp_arrive(uint32_t bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Per-thread epilogue context.
struct EpiCtx {
    int quad, half, lane, row_lane;  // TMEM lane quadrant, slice parity, lane, TMEM lane (row of P)
    float row_scale;                 // s_a[m] (plain) or s_w[n] (Swap-AB)
    float row_bias;                  // bias[n] (Swap-AB only)
    uint32_t s_col;                  // shared address of the tile's column scales
    uint32_t b_col;                  // shared address of the tile's column bias
    uint32_t staging;                // shared address of this warp's 2 KB transpose buffer
    const CUtensorMap* tmap_c;       // plain tiles: bf16 C as a tensor of 32 x 32 boxes (64-byte swizzle)
    bool has_bias;
    // cluster Split-K only
    int rank;                        // CTA rank in the cluster = K segment
    uint32_t recv;                   // this CTA's receive area (read by rank 0)
    uint32_t recv_remote;            // rank 0's receive area, cluster address
    uint32_t recv_full, recv_free;   // local mbarriers
    uint32_t xphase;                 // phase of the per-tile exchange
};

// Warp-level wait on an mbarrier that other CTAs of the cluster arrive on.
// The __syncwarp extends lane 0's acquire to the whole warp.
__device__ __forceinline__ bool warp_wait_cluster(uint32_t bar, uint32_t parity) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait_cluster(bar, parity) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// Final epilogue of one slice of SW accumulator columns.  `v` holds fp32 bits
// (FP8 formats: the summed value) or int32 (INT8: the exact accumulator).
//   y = ((float)acc * s_a[m]) * s_w[n] + bias[n]   (Block-FP8: y = acc)
template <int FMT, bool SWAP, int BN>
__device__ __forceinline__ void finish_slice(const GemmArgs& a, const Unit& un, int j, EpiCtx& e,
                                             const uint32_t* v) {
    using C = Cfg<FMT, SWAP, BN>;
    constexpr int SW = C::SW;
    if (a.out_i32) {  // raw INT8 accumulators (test path): direct stores
        int32_t* out = static_cast<int32_t*>(a.c);
        if constexpr (!SWAP) {
            const int m = un.pt * 128 + e.row_lane;
            const int n0 = un.qt * BN + j * SW;
            if (m < a.M) {
#pragma unroll
                for (int c = 0; c < SW; ++c)
                    if (n0 + c < a.N) out[(size_t)m * a.N + n0 + c] = (int32_t)v[c];
            }
        } else {
            const int n = un.pt * 128 + e.row_lane;
            const int m0 = un.qt * BN + j * SW;
            if (n < a.N) {
#pragma unroll
                for (int c = 0; c < SW; ++c)
                    if (m0 + c < a.M) out[(size_t)(m0 + c) * a.N + n] = (int32_t)v[c];
            }
        }
        return;
    }
    float y[SW];
#pragma unroll
    for (int c4 = 0; c4 < SW; c4 += 4) {
        float4 sc = make_float4(0.f, 0.f, 0.f, 0.f), bc = make_float4(0.f, 0.f, 0.f, 0.f);
        if constexpr (!C::BLOCK) {
            if constexpr (!C::BF16) sc = lds_f4(e.s_col + (uint32_t)(j * SW + c4) * 4u);
            if (!SWAP && e.has_bias) bc = lds_f4(e.b_col + (uint32_t)(j * SW + c4) * 4u);
        }
        const float scv[4] = {sc.x, sc.y, sc.z, sc.w};
        const float bcv[4] = {bc.x, bc.y, bc.z, bc.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int c = c4 + i;
            float t;
            if constexpr (C::INT8)
                t = __int2float_rn((int)v[c]);
            else
                t = __uint_as_float(v[c]);
            if constexpr (C::BF16) {
                if (e.has_bias) t = __fadd_rn(t, SWAP ? e.row_bias : bcv[i]);  // + bias[n]
            } else if constexpr (!C::BLOCK) {
                if constexpr (!SWAP) {
                    t = __fmul_rn(t, e.row_scale);  // * s_a[m]
                    t = __fmul_rn(t, scv[i]);       // * s_w[n]
                    if (e.has_bias) t = __fadd_rn(t, bcv[i]);
                } else {
                    t = __fmul_rn(t, scv[i]);       // * s_a[m]
                    t = __fmul_rn(t, e.row_scale);  // * s_w[n]
                    if (e.has_bias) t = __fadd_rn(t, e.row_bias);
                }
            }
            y[c] = t;
        }
    }
    uint16_t* cb = static_cast<uint16_t*>(a.c);
    if constexpr (SWAP) {
        // lane = column n of C; each store instruction writes 64 contiguous bytes of row m
        const int n = un.pt * 128 + e.row_lane;
        const int m0 = un.qt * BN + j * SW;
        if (n < a.N) {
#pragma unroll
            for (int c = 0; c < SW; ++c)
                if (m0 + c < un.rows)
                    cb[(size_t)(un.row0 + m0 + c) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y[c]));
        }
    } else {
        // The warp's 32 x 32 box of C goes to shared memory row by row (lane =
        // row, 64 bytes, chunk q of row r at q ^ ((r >> 1) & 3): the 64-byte
        // swizzle) and from there to global memory as one bulk tensor store,
        // which also leaves out the rows and columns past the edges of C.
        const int bx = un.qt * BN + j * SW;
        const int by = un.pt * 128 + e.quad * 32;
        if (bx >= a.N || by >= un.rows) return;  // warp-uniform: the whole box is outside C
        uint32_t packed[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) packed[c / 2] = pack_bf16x2(y[c], y[c + 1]);
        if (a.moe_E > 0) {
            // MoE: the box may reach into the next expert's rows, so each
            // thread stores its own row, 16 bytes at a time (N % 16 == 0)
            const int m = by + e.lane;
            if (m < un.rows) {
                uint4* dst = reinterpret_cast<uint4*>(cb + (size_t)(un.row0 + m) * a.N + bx);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (bx + 8 * q < a.N)
                        dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
            }
            return;
        }
        if (e.lane == 0) bulk_wait_read_all();  // the previous box has left the buffer
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 4; ++q)
            sts_u4(e.staging + e.lane * 64 + ((q ^ ((e.lane >> 1) & 3)) * 16),
                   make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]));
        fence_proxy_async_shared();
        __syncwarp();
        if (e.lane == 0) {
            tma_store_2d(e.tmap_c, bx, by, e.staging);
            bulk_commit_group();
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

// Split-K workspace: [tile][segment][slice][SW/4 column groups][128 lanes]
// 16-byte vectors, so the 32 lanes of a warp touch 512 contiguous bytes per
// access.  partial_ptr returns this lane's first vector; group q is 128
// vectors further on.
template <int SW>
__device__ __forceinline__ uint4* partial_ptr(const GemmArgs& a, int tile, int seg, int j, int nslice,
                                              int row_lane) {
    return reinterpret_cast<uint4*>(a.partials) + (((size_t)tile * a.S + seg) * nslice + j) * (SW / 4) * 128 +
           row_lane;
}

template <int SW>
__device__ __forceinline__ void store_partial(uint4* p, const uint32_t (&v)[SW]) {
#pragma unroll
    for (int q = 0; q < SW / 4; ++q) p[q * 128] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// Split-K: after every segment of a tile has been written, the last CTA to
// arrive adds them in segment order and runs the final epilogue.  One thread
// publishes the CTA's partial (release) and takes the ticket (acquire).
template <int FMT, bool SWAP, int BN>
__device__ __forceinline__ void splitk_finish(const GemmArgs& a, const Unit& un, EpiCtx& e, int* bcast) {
    using C = Cfg<FMT, SWAP, BN>;
    constexpr int SW = C::SW;
    constexpr int SB = 64 / SW;  // segments loaded per round trip: 64 registers of partials
    named_bar_sync(1, kEpiThreads);
    if (threadIdx.x == 0) {
        // acq_rel: releases this CTA's partial stores (ordered before it by the
        // barrier above) and, for the last arriver, acquires everyone else's
        const int old = atom_add_acq_rel_gpu(a.tickets + un.tile, 1);
        *bcast = (old == a.S - 1) ? 1 : 0;
    }
    named_bar_sync(1, kEpiThreads);
    const bool last = *(volatile int*)bcast != 0;
    if (!last) return;
#pragma unroll 1
    for (int j = e.half; j < C::NSLICE; j += 2) {
        uint32_t acc[SW];
        if constexpr (C::INT8) {
            int32_t t[SW];
#pragma unroll
            for (int c = 0; c < SW; ++c) t[c] = 0;
#pragma unroll 1
            for (int s0 = 0; s0 < a.S; s0 += SB) {
                uint4 w[SB][SW / 4];
#pragma unroll
                for (int i = 0; i < SB; ++i)
                    if (s0 + i < a.S) {
                        const uint4* p =
                            reinterpret_cast<const uint4*>(partial_ptr<SW>(a, un.tile, s0 + i, j, C::NSLICE, e.row_lane));
#pragma unroll
                        for (int q = 0; q < SW / 4; ++q) w[i][q] = __ldcg(p + q * 128);
                    }
#pragma unroll
                for (int i = 0; i < SB; ++i)
                    if (s0 + i < a.S) {
#pragma unroll
                        for (int q = 0; q < SW / 4; ++q) {
                            t[4 * q] += (int32_t)w[i][q].x;
                            t[4 * q + 1] += (int32_t)w[i][q].y;
                            t[4 * q + 2] += (int32_t)w[i][q].z;
                            t[4 * q + 3] += (int32_t)w[i][q].w;
                        }
                    }
            }
#pragma unroll
            for (int c = 0; c < SW; ++c) acc[c] = (uint32_t)t[c];
        } else {
            float t[SW];
#pragma unroll
            for (int c = 0; c < SW; ++c) t[c] = 0.f;
#pragma unroll 1
            for (int s0 = 0; s0 < a.S; s0 += SB) {
                uint4 w[SB][SW / 4];
#pragma unroll
                for (int i = 0; i < SB; ++i)
                    if (s0 + i < a.S) {
                        const uint4* p =
                            reinterpret_cast<const uint4*>(partial_ptr<SW>(a, un.tile, s0 + i, j, C::NSLICE, e.row_lane));
#pragma unroll
                        for (int q = 0; q < SW / 4; ++q) w[i][q] = __ldcg(p + q * 128);
                    }
#pragma unroll
                for (int i = 0; i < SB; ++i)  // fixed segment order
                    if (s0 + i < a.S) {
#pragma unroll
                        for (int q = 0; q < SW / 4; ++q) {
                            t[4 * q] = __fadd_rn(t[4 * q], __uint_as_float(w[i][q].x));
                            t[4 * q + 1] = __fadd_rn(t[4 * q + 1], __uint_as_float(w[i][q].y));
                            t[4 * q + 2] = __fadd_rn(t[4 * q + 2], __uint_as_float(w[i][q].z));
                            t[4 * q + 3] = __fadd_rn(t[4 * q + 3], __uint_as_float(w[i][q].w));
                        }
                    }
            }
#pragma unroll
            for (int c = 0; c < SW; ++c) acc[c] = __float_as_uint(t[c]);
        }
        finish_slice<FMT, SWAP, BN>(a, un, j, e, acc);
    }
    named_bar_sync(1, kEpiThreads);  // every warp has read its partials
    if (threadIdx.x == 0) a.tickets[un.tile] = 0;  // leave the ticket zeroed for the next call
}

// Cluster Split-K: the S CTAs of a cluster hold the S segments of one tile
// (rank = segment).  Ranks 1..S-1 store their segment values into rank 0's
// shared memory, [rank-1][slice][SW/4 column groups][128 lanes] 16-byte
// vectors; rank 0 adds them to its own in segment order, exactly as the
// workspace Split-K reducer does, and runs the final epilogue.
template <int FMT, bool SWAP, int BN>
__device__ __forceinline__ bool csk_slice(const GemmArgs& a, const Unit& un, int j, EpiCtx& e,
                                          const uint32_t (&segv)[Cfg<FMT, SWAP, BN>::SW]) {
    using C = Cfg<FMT, SWAP, BN>;
    constexpr int SW = C::SW;
    constexpr uint32_t kGroup = 128u * 16u;  // bytes between column groups
    if (e.rank != 0) {
        // the receive slot is free once rank 0 has read the previous tile
        if (!warp_wait_cluster(e.recv_free, e.xphase ^ 1u)) return false;
        const uint32_t dst =
            e.recv_remote + ((uint32_t)((e.rank - 1) * C::NSLICE + j) * (SW / 4)) * kGroup + (uint32_t)e.row_lane * 16u;
#pragma unroll
        for (int q = 0; q < SW / 4; ++q)
            st_cluster_v4(dst + q * kGroup, make_uint4(segv[4 * q], segv[4 * q + 1], segv[4 * q + 2], segv[4 * q + 3]));
        return true;
    }
    if (!warp_wait_cluster(e.recv_full, e.xphase)) return false;
    uint32_t acc[SW];
    if constexpr (C::INT8) {
        int32_t t[SW];
#pragma unroll
        for (int c = 0; c < SW; ++c) t[c] = (int32_t)segv[c];
#pragma unroll 1
        for (int r = 1; r < a.S; ++r) {
            const uint32_t src = e.recv + ((uint32_t)((r - 1) * C::NSLICE + j) * (SW / 4)) * kGroup + e.row_lane * 16u;
#pragma unroll
            for (int q = 0; q < SW / 4; ++q) {
                const uint4 w = lds_u4(src + q * kGroup);
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
        for (int c = 0; c < SW; ++c) t[c] = __fadd_rn(0.f, __uint_as_float(segv[c]));
#pragma unroll 1
        for (int r = 1; r < a.S; ++r) {  // fixed segment order
            const uint32_t src = e.recv + ((uint32_t)((r - 1) * C::NSLICE + j) * (SW / 4)) * kGroup + e.row_lane * 16u;
#pragma unroll
            for (int q = 0; q < SW / 4; ++q) {
                const uint4 w = lds_u4(src + q * kGroup);
                t[4 * q] = __fadd_rn(t[4 * q], __uint_as_float(w.x));
                t[4 * q + 1] = __fadd_rn(t[4 * q + 1], __uint_as_float(w.y));
                t[4 * q + 2] = __fadd_rn(t[4 * q + 2], __uint_as_float(w.z));
                t[4 * q + 3] = __fadd_rn(t[4 * q + 3], __uint_as_float(w.w));
            }
        }
#pragma unroll
        for (int c = 0; c < SW; ++c) acc[c] = __float_as_uint(t[c]);
    }
    finish_slice<FMT, SWAP, BN>(a, un, j, e, acc);
    return true;
}

// Hand one segment value (slice j, SW columns) to the running sum: Split-K
// writes it out (workspace, or rank 0's shared memory); the plain variant adds
// it to the TMEM total (or, on the last segment, finishes the tile).  False
// only when a bounded wait gave up.
template <int FMT, bool SWAP, int BN, bool CSK>
__device__ __forceinline__ bool consume_segment_slice(const GemmArgs& a, const Unit& un, int seg_no, int j,
                                                      uint32_t t_total, EpiCtx& e,
                                                      const uint32_t (&segv)[Cfg<FMT, SWAP, BN>::SW]) {
    using C = Cfg<FMT, SWAP, BN>;
    constexpr int SW = C::SW;
    if (a.spread) {
        if constexpr (CSK) return csk_slice<FMT, SWAP, BN>(a, un, j, e, segv);
        store_partial<SW>(partial_ptr<SW>(a, un.tile, un.seg, j, C::NSLICE, e.row_lane), segv);
        return true;
    }
    if constexpr (C::INT8) {
        finish_slice<FMT, SWAP, BN>(a, un, j, e, segv);  // exact: whole K in one accumulator
    } else {
        uint32_t t[SW];
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
            finish_slice<FMT, SWAP, BN>(a, un, j, e, t);
        } else {
            if constexpr (C::MULTI) tmem_store_slice<SW>(t_total + j * SW, t);
        }
    }
    return true;
}

// End of a fused unit: rows past M get zero codes (what the TMA's
// out-of-bounds fill gives), then the generic-proxy stores are made visible
// to the tensor core.  sA as in fused_quantize_unit; cpr: 16-byte chunks per
// row of the unit.
template <int BN>
__device__ __forceinline__ void finish_fused_rows(uint32_t sA, int rows, int cpr) {
    for (int i = threadIdx.x; i < (BN - rows) * cpr; i += kEpiThreads) {
        const int r = rows + i / cpr, ch = i % cpr;
        const int kbl = ch >> 3, c = ch & 7;
        sts_u4(sA + (uint32_t)(kbl * BN * 128 + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)),
               make_uint4(0u, 0u, 0u, 0u));
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Fused activation quantisation of one Swap-AB unit (the 256 epilogue
// threads, which all call it): rows m0..m0+BN-1 of x, K blocks kb0..kb1-1,
// into the resident operand sA ([K block][BN rows x 128 B], 16-byte chunk c of
// row r stored at chunk c ^ (r % 8): the 128-byte swizzle the MMA descriptors
// describe) and the unit's scales into sa (per token: [BN]; Block-FP8:
// [BN][MAXKB]).  The arithmetic is the stand-alone quantisers'
// (quant_math.cuh), so codes and scales are theirs bit for bit.  Only rows
// below M are read; the work is spread over all threads by element, not by
// row.  Per token: when a thread's share of its row fits in registers (rows
// of up to 16 x 256 x 8 elements per unit), all its loads go out at once and
// the codes are made from the registers, so a unit costs one L2 round trip;
// longer rows take two passes.  Rows past M get zero codes.
// rmax: BN words of scratch shared memory (per-token formats).  xs: a
// shared-memory buffer of xs_bytes; when the unit's slice of x (rows x its K
// range in bf16) fits, pass 1 keeps that slice there and pass 2 reads it back
// instead of going to memory a second time.
template <int FMT, int BN, int MAXKB, bool IN_REGS = false>
__device__ __forceinline__ void fused_quantize_unit(const GemmArgs& a, const Unit& un, uint32_t sA, float* sa,
                                                    uint32_t* rmax, uint32_t xs, int xs_bytes) {
    constexpr int T = kEpiThreads;
    constexpr int UNROLL1 = 4;  // 16-byte vectors in flight per thread, pass 1
    constexpr int UNROLL2 = 2;  // 16-element chunks in flight per thread, pass 2
    const int tid = threadIdx.x;  // 0 .. T-1
    const int m0 = un.qt * BN;
    const int rows = min(BN, a.M - m0);  // >= 1
    const int nkb = un.kb1 - un.kb0;
    const int cpr = nkb * 8;  // 16-element chunks per row in this unit
    const bool write_out = un.pt == 0 && a.a_q_out != nullptr;
    const int64_t K = (int64_t)a.kblocks * 128;
    auto sa_addr = [&](int r, int ch) -> uint32_t {
        const int kbl = ch >> 3, c = ch & 7;
        return sA + (uint32_t)(kbl * BN * 128 + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
    };
    auto xrow = [&](int r) { return reinterpret_cast<const uint4*>(a.x + (size_t)(m0 + r) * a.ld_x); };
    if constexpr (FMT != QLIN_FMT_FP8_BLOCK) {
        constexpr float QMAX = (FMT == QLIN_FMT_INT8) ? 127.f : 448.f;
        constexpr int RV = 16;  // 16-byte vectors of a row one thread may hold
        // TPR consecutive threads per row: the largest power of two with
        // TPR * rows <= T (so a batch of one row has all 256 threads on it)
        int tpr = T;
        while (tpr * rows > T) tpr >>= 1;
        const int r = tid / tpr, sub = tid % tpr;
        const bool live = r < rows;
        const uint4* xr = xrow(live ? r : 0);
        const int nvec = (int)(K >> 3);
        const int uv0 = un.kb0 * 16, uvn = nkb * 16;  // the unit's vectors of a row
        uint8_t* qrow = write_out ? a.a_q_out + (size_t)(m0 + r) * K : nullptr;
        // The row maximum from the threads' partial maxima: within the warp
        // (a row's lanes are consecutive), then across warps for rows wider
        // than a warp (|x| >= 0, so float order = bit order).  Writes the
        // unit's scales (and, once per row, s_a) and returns row r's scale.
        auto row_scale_from = [&](float amax) -> float {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float other = __shfl_xor_sync(0xffffffffu, amax, o);
                if (o < tpr) amax = fmaxf(amax, other);
            }
            for (int i = tid; i < BN; i += T) rmax[i] = 0u;
            named_bar_sync(1, T);
            if (live && ((tid % tpr) & 31) == 0) atomicMax(&rmax[r], __float_as_uint(amax));
            named_bar_sync(1, T);
            for (int i = tid; i < BN; i += T) {
                const float s = i < rows ? __fdiv_rn(__uint_as_float(rmax[i]), QMAX) : 0.f;
                sa[i] = s;
                if (i < rows && un.pt == 0 && un.seg == 0 && a.s_a_out) a.s_a_out[m0 + i] = s;
            }
            return live ? __fdiv_rn(__uint_as_float(rmax[r]), QMAX) : 0.f;
        };
        if (IN_REGS && (nvec + tpr - 1) / tpr <= RV) {
            // A thread's share of its row fits in registers (RV vectors): one
            // batch of loads, the row maximum, then the codes straight from
            // the registers (8 codes = half a swizzled 16-byte chunk each).
            uint4 v[RV];
            float amax = 0.f;
            if (live) {
#pragma unroll
                for (int j = 0; j < RV; ++j)
                    if (sub + j * tpr < nvec) v[j] = __ldg(xr + sub + j * tpr);
#pragma unroll
                for (int j = 0; j < RV; ++j)
                    if (sub + j * tpr < nvec) amax = fmaxf(amax, qm::absmax8(v[j]));
            }
            const float sc = row_scale_from(amax);
            const qm::Divisor dv = qm::make_divisor(sc);
            auto put = [&](int vu, uint2 q) {  // vu: vector within the unit's K range
                sts_u2(sa_addr(r, vu >> 1) + (uint32_t)((vu & 1) * 8), q);
                if (qrow) *reinterpret_cast<uint2*>(qrow + (size_t)(uv0 + vu) * 8) = q;
            };
            if (live && dv.fast) {
#pragma unroll
                for (int j = 0; j < RV; ++j) {
                    const int vu = sub + j * tpr - uv0;
                    if (vu >= 0 && vu < uvn) put(vu, qm::quant8<FMT, true>(v[j], dv));
                }
            } else if (live) {
                // a scale outside the reciprocal's range: the IEEE division,
                // one vector at a time, read again from memory
#pragma unroll 1
                for (int vu = sub - uv0 + ((uv0 - sub + tpr - 1) / tpr) * tpr; vu < uvn; vu += tpr)
                    put(vu, qm::quant8<FMT>(__ldg(xr + uv0 + vu), dv));
            }
            finish_fused_rows<BN>(sA, rows, cpr);
            return;
        }
        // Longer rows. pass 1: the row maximum over all of K, 16-byte vectors,
        // loads first; the vectors of this unit's K range are kept in xs when
        // they fit
        const bool staged = rows * uvn * 16 <= xs_bytes;
        float amax = 0.f;
        if (live) {
            for (int v0 = sub; v0 < nvec; v0 += tpr * UNROLL1) {
                uint4 v[UNROLL1];
#pragma unroll
                for (int j = 0; j < UNROLL1; ++j)
                    if (v0 + j * tpr < nvec) v[j] = __ldg(xr + v0 + j * tpr);
#pragma unroll
                for (int j = 0; j < UNROLL1; ++j) {
                    const int vi = v0 + j * tpr;
                    if (vi < nvec) {
                        amax = fmaxf(amax, qm::absmax8(v[j]));
                        if (staged && vi >= uv0 && vi < uv0 + uvn)
                            sts_u4(xs + (uint32_t)((r * uvn + vi - uv0) * 16), v[j]);
                    }
                }
            }
        }
        const float sc = row_scale_from(amax);
        // pass 2: the unit's K range, 16 elements -> one 16-byte chunk of codes
        if (live) {
            const qm::Divisor dv = qm::make_divisor(sc);
            const uint4* xsrc = xr + (((int64_t)un.kb0 * 128) >> 3);
            uint8_t* qout = write_out ? a.a_q_out + (size_t)(m0 + r) * K + (int64_t)un.kb0 * 128 : nullptr;
            for (int c0 = sub; c0 < cpr; c0 += tpr * UNROLL2) {
                uint4 v[UNROLL2][2];
#pragma unroll
                for (int j = 0; j < UNROLL2; ++j) {
                    const int ch = c0 + j * tpr;
                    if (ch < cpr) {
                        if (staged) {
                            v[j][0] = lds_u4(xs + (uint32_t)((r * uvn + 2 * ch) * 16));
                            v[j][1] = lds_u4(xs + (uint32_t)((r * uvn + 2 * ch + 1) * 16));
                        } else {
                            v[j][0] = __ldg(xsrc + 2 * ch);
                            v[j][1] = __ldg(xsrc + 2 * ch + 1);
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < UNROLL2; ++j) {
                    const int ch = c0 + j * tpr;
                    if (ch < cpr) {
                        const uint2 q0 = qm::quant8<FMT>(v[j][0], dv), q1 = qm::quant8<FMT>(v[j][1], dv);
                        const uint4 codes = make_uint4(q0.x, q0.y, q1.x, q1.y);
                        sts_u4(sa_addr(r, ch), codes);
                        if (qout) *reinterpret_cast<uint4*>(qout + ch * 16) = codes;
                    }
                }
            }
        }
    } else {
        // 1x128 groups: 8 consecutive lanes per (row, K block) group, 16 elements each
        constexpr int GPP = T / 8;  // groups per pass
        const int ngroups = rows * nkb;
        const int c = tid & 7;
        for (int g0 = 0; g0 < ngroups; g0 += GPP * 2) {  // uniform trip count: the shuffles stay converged
            uint4 v[2][2];
            int gr[2], gk[2];
            bool live[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int g = g0 + j * GPP + (tid >> 3);
                live[j] = g < ngroups;
                gr[j] = live[j] ? g / nkb : 0;
                gk[j] = live[j] ? g % nkb : 0;
                if (live[j]) {
                    const uint4* src = xrow(gr[j]) + (((int64_t)(un.kb0 + gk[j]) * 128 + c * 16) >> 3);
                    v[j][0] = __ldg(src);
                    v[j][1] = __ldg(src + 1);
                } else {
                    v[j][0] = v[j][1] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float gmax = fmaxf(qm::absmax8(v[j][0]), qm::absmax8(v[j][1]));
#pragma unroll
                for (int o = 4; o > 0; o >>= 1) gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
                if (!live[j]) continue;
                const float sc = __fdiv_rn(gmax, 448.f);
                const int r = gr[j], kbl = gk[j];
                if (c == 0) {
                    sa[r * MAXKB + kbl] = sc;
                    if (un.pt == 0 && a.s_a_out) a.s_a_out[(size_t)(m0 + r) * a.kblocks + un.kb0 + kbl] = sc;
                }
                const qm::Divisor dv = qm::make_divisor(sc);
                const uint2 q0 = qm::quant8<QLIN_FMT_FP8>(v[j][0], dv), q1 = qm::quant8<QLIN_FMT_FP8>(v[j][1], dv);
                const uint4 codes = make_uint4(q0.x, q0.y, q1.x, q1.y);
                sts_u4(sa_addr(r, kbl * 8 + c), codes);
                if (write_out)
                    *reinterpret_cast<uint4*>(a.a_q_out + (size_t)(m0 + r) * K + (int64_t)(un.kb0 + kbl) * 128 + c * 16) =
                        codes;
            }
        }
    }
    finish_fused_rows<BN>(sA, rows, cpr);
}

// Block-FP8: stage the scale products s_a[m,kb] * s_w[n/128,kb] of a window of
// up to BS_KB K blocks from win0 into shared memory, [kb][row] (plain tiles) or
// [kb][column] (Swap-AB), by coalesced cooperative loads of the 256 epilogue
// threads (which all call it).  Fused mode reads s_a from the unit's own
// scales (sa_cur).
template <int FMT, bool SWAP, int BN, bool CSK, bool FUSE, bool PAIR>
__device__ __forceinline__ void stage_block_scales(const GemmArgs& args, const Unit& un, int win0, uint32_t bsc,
                                                   const float* sa_cur) {
    using C = Cfg<FMT, SWAP, BN, CSK, FUSE, PAIR>;
    const int kbc = min(C::BS_KB, un.kb1 - win0);
    constexpr int NIDX = SWAP ? BN : 128;
    const int nb = SWAP ? un.pt : ((un.qt * BN) >> 7);
    const int mbase = SWAP ? un.qt * BN : un.pt * 128;
    named_bar_sync(1, kEpiThreads);  // the previous window is no longer read
    constexpr int BATCH = 24;        // loads in flight per thread: a 128 x 48 window in one round trip
    for (int i0 = threadIdx.x; i0 < NIDX * kbc; i0 += kEpiThreads * BATCH) {
        float va[BATCH], vw[BATCH];
        int off[BATCH];
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
            const int i = i0 + b * kEpiThreads;
            const int idx = i / kbc, kbl = i - idx * kbc;
            const int m = mbase + idx, kb = win0 + kbl;
            off[b] = -1;
            va[b] = 0.f;
            vw[b] = 0.f;
            if (i < NIDX * kbc) {
                off[b] = kbl * C::BS_PITCH + idx;
                if (m < args.M) {
                    if constexpr (FUSE)
                        va[b] = sa_cur[idx * C::A_MAXKB + (kb - un.kb0)];
                    else
                        va[b] = __ldg(args.s_a + (size_t)m * args.kblocks + kb);
                    vw[b] = __ldg(args.s_w + (size_t)nb * args.kblocks + kb);
                }
            }
        }
#pragma unroll
        for (int b = 0; b < BATCH; ++b)
            if (off[b] >= 0)
                asm volatile("st.shared.f32 [%0], %1;" ::"r"(bsc + (uint32_t)off[b] * 4u), "f"(__fmul_rn(va[b], vw[b]))
                             : "memory");
    }
    named_bar_sync(1, kEpiThreads);
}

template <int FMT, bool SWAP, int BN, bool CSK, bool FUSE, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    qlin_gemm_kernel(const __grid_constant__ CUtensorMap tmap_p, const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_c, const __grid_constant__ GemmArgs args) {
    using C = Cfg<FMT, SWAP, BN, CSK, FUSE, PAIR>;
    constexpr int STAGES = C::STAGES;
    constexpr int SW = C::SW;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sP = smem;
    uint8_t* sQ = smem + (size_t)STAGES * C::P_BYTES;
    uint8_t* sF = sQ + (size_t)STAGES * C::Q_BYTES;  // block-scaled: per stage, A's then W's scale atoms
    float* s_col = reinterpret_cast<float*>(smem + C::SCALE_OFF);
    float* b_col = s_col + 256;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    const uint32_t full0 = smem_u32(bars);
    const uint32_t empty0 = smem_u32(bars + STAGES);
    constexpr int NACC = C::NACC;
    uint64_t* bars_x = bars + 2 * STAGES + 2 * NACC;
    const uint32_t tfull0 = smem_u32(bars + 2 * STAGES);
    const uint32_t tempty0 = smem_u32(bars + 2 * STAGES + NACC);
    const uint32_t recv_full = smem_u32(bars_x + 0);  // cluster Split-K, rank 0
    const uint32_t recv_free = smem_u32(bars_x + 1);  // cluster Split-K, ranks > 0
    const uint32_t a_full = smem_u32(bars_x + 2);     // fused: unit's A codes written
    const uint32_t a_empty = smem_u32(bars_x + 3);    // fused: MMA done with them
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars_x + 4);
    int32_t* moe_tab = reinterpret_cast<int32_t*>(smem + C::MOE_OFF);  // offsets [E+1], then unit prefixes
    const uint32_t sA = smem_u32(smem + C::A_OFF);
    float* sa_tile = reinterpret_cast<float*>(smem + C::SA_OFF);
    uint32_t* rmax = reinterpret_cast<uint32_t*>(sa_tile + 2 * C::SA_FLOATS);  // fused per-token row maxima
    // fused: the epilogue's transpose buffers (unused by Swap-AB tiles) hold x slices
    const uint32_t xstage = smem_u32(smem + C::STAGING_OFF);
    int* bcast = reinterpret_cast<int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // PAIR: both CTAs of a cluster walk the same pair tiles; rank 0 leads
    const int rank = PAIR ? (int)cluster_ctarank() : 0;
    const int u_first = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int u_step = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

    if (warp == kProducerWarp && lane == 0) {
        prefetch_tmap(&tmap_p);
        if constexpr (!FUSE) prefetch_tmap(&tmap_q);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int b = 0; b < NACC; ++b) {
            mbar_init(tfull0 + 8 * b, 1);
            // one arrival per epilogue warp (PAIR: of both CTAs, on rank 0's barrier)
            mbar_init(tempty0 + 8 * b, PAIR ? 2 * kEpiWarps : kEpiWarps);
        }
        if constexpr (CSK) {
            mbar_init(recv_full, (args.S - 1) * kEpiWarps);  // every epilogue warp of every other rank
            mbar_init(recv_free, 1);                         // rank 0's thread 0
        }
        if constexpr (FUSE) {
            mbar_init(a_full, kEpiWarps);
            mbar_init(a_empty, 1);
        }
        fence_mbarrier_init();
    }
    if (warp == kMmaWarp) {
        if constexpr (PAIR) {
            tmem_alloc_pair(smem_u32(tmem_holder), C::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
            tmem_relinquish();
        }
    }
    if (args.moe_E > 0 && warp == kEpiWarps + 2) {
        // MoE: the expert row offsets come from the previous kernel (routing);
        // wait for it, then the experts' tile counts and their prefix sums
        pdl_wait();
        int32_t* off = moe_tab;
        int32_t* pref = moe_tab + kMoeMaxExperts + 1;
        const int E = args.moe_E;
        const int per = (E + 32) / 32;  // experts per lane (E + 1 offsets)
        int32_t sum = 0;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e <= E) off[e] = args.moe_offsets[e];
        }
        __syncwarp();
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) {
                const int rows = off[e + 1] - off[e];
                const int p_tiles = SWAP ? (args.N + 127) / 128 : (rows + 127) / 128;
                const int q_tiles = SWAP ? (rows + BN - 1) / BN : (args.N + BN - 1) / BN;
                sum += rows > 0 ? p_tiles * q_tiles : 0;
            }
        }
        int32_t incl = sum;  // inclusive scan of the lanes' sums
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int32_t run = incl - sum;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) {
                pref[e] = run;
                const int rows = off[e + 1] - off[e];
                const int p_tiles = SWAP ? (args.N + 127) / 128 : (rows + 127) / 128;
                const int q_tiles = SWAP ? (rows + BN - 1) / BN : (args.N + BN - 1) / BN;
                run += rows > 0 ? p_tiles * q_tiles : 0;
            }
        }
        if (lane == 31) pref[E] = incl;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int32_t* moe = args.moe_E > 0 ? moe_tab : nullptr;
    const int units = moe ? moe_tab[kMoeMaxExperts + 1 + args.moe_E] : args.units;
    // every rank's barriers are initialised before any remote arrive or load signal
    if constexpr (CSK || PAIR) cluster_sync();
    const uint32_t tmem_base = *tmem_holder;
    pdl_launch_dependents();

    // Each role rebalances its registers first thing in its own branch (the
    // compiler applies a warp's register limit to the code that setmaxnreg
    // dominates, so no role's code may follow a merge of the two limits).
    if (warp == kProducerWarp) {
        regs_decrease<kAuxRegs>();
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_a = policy_evict_last();
            const CUtensorMap* tm_w = SWAP ? &tmap_p : &tmap_q;
            const CUtensorMap* tm_a = SWAP ? &tmap_q : &tmap_p;
            // PAIR: both CTAs' loads of a stage are counted on rank 0's full
            // barrier, which rank 0 alone arms with the bytes of both
            const uint32_t stage_tx = PAIR ? 2 * C::STAGE_BYTES : C::STAGE_BYTES;
            const int w_row_off = PAIR ? rank * (BN / 2) : 0;  // this CTA's half of the W tile
            auto arm = [&](uint32_t fb) {
                if (!PAIR || rank == 0) mbar_arrive_expect_tx(fb, stage_tx);
            };
            auto load = [&](uint32_t dst, const CUtensorMap* m, int x, int y, uint32_t fb, uint64_t pol) {
                if constexpr (PAIR)
                    tma_load_2d_pair(dst, m, x, y, mapa_shared(fb, 0), pol);
                else
                    tma_load_2d(dst, m, x, y, fb, pol);
            };
            auto load_w = [&](uint32_t stage, const Unit& un, int kb, uint32_t fb) {
                if constexpr (SWAP) {
                    load(smem_u32(sP + (size_t)stage * C::P_BYTES), tm_w, kb * 128, un.wrow0 + un.pt * 128, fb,
                         pol_w);
                    if constexpr (C::BS)  // W is the MMA's A: its scale atoms go to the A slot
                        bulk_load(smem_u32(sF + (size_t)stage * C::SF_BYTES),
                                  args.sf_w + ((size_t)un.pt * args.sf_atoms + (size_t)kb * C::SF_APK) * 512u,
                                  (uint32_t)C::SFA_BYTES, fb, pol_w);
                } else {
                    load(smem_u32(sQ + (size_t)stage * C::Q_BYTES), tm_w, kb * 128,
                         un.wrow0 + un.qt * BN + w_row_off, fb, pol_w);
                    if constexpr (C::BS) {  // the W tile's scale atoms of this K block
#pragma unroll
                        for (int j = 0; j < BN / 128; ++j)
                            bulk_load(smem_u32(sF + (size_t)stage * C::SF_BYTES + C::SFA_BYTES + j * 512 * C::SF_APK),
                                      args.sf_w + ((size_t)(un.qt * (BN / 128) + j) * args.sf_atoms +
                                                   (size_t)kb * C::SF_APK) * 512u,
                                      512u * C::SF_APK, fb, pol_w);
                    }
                }
            };
            // weights do not depend on the previous kernel: start streaming the
            // first unit's weight tiles before waiting for it
            int pre = 0;
            if (u_first < units) {
                const Unit un = decode_unit<FMT, PAIR, SWAP, BN>(args, u_first, rank, moe);
                for (int kb = un.kb0; kb < un.kb1 && pre < STAGES; ++kb, ++pre) {
                    arm(full0 + 8 * pre);
                    load_w(pre, un, kb, full0 + 8 * pre);
                }
            }
            pdl_wait();
            uint32_t stage = 0, phase = 0;
            int it = 0;
            for (int u = u_first; u < units; u += u_step) {
                const Unit un = decode_unit<FMT, PAIR, SWAP, BN>(args, u, rank, moe);
                for (int kb = un.kb0; kb < un.kb1; ++kb, ++it) {
                    const uint32_t fb = full0 + 8 * stage;
                    if (it >= pre) {
                        const bool freed = PAIR ? mbar_wait_cluster(empty0 + 8 * stage, phase ^ 1)
                                                : mbar_wait(empty0 + 8 * stage, phase ^ 1);
                        if (!freed) goto done;
                        arm(fb);
                        load_w(stage, un, kb, fb);
                    }
                    if constexpr (FUSE)
                        (void)pol_a;  // the activation operand is quantised in place
                    else if constexpr (SWAP)
                        load(smem_u32(sQ + (size_t)stage * C::Q_BYTES), tm_a, kb * 128, un.row0 + un.qt * BN, fb,
                             pol_a);
                    else
                        load(smem_u32(sP + (size_t)stage * C::P_BYTES), tm_a, kb * 128, un.row0 + un.pt * 128, fb,
                             pol_a);
                    if constexpr (C::BS && SWAP)  // the activation rows' 128-row atom group, B slot
                        bulk_load(smem_u32(sF + (size_t)stage * C::SF_BYTES + C::SFA_BYTES),
                                  args.sf_a + ((size_t)((un.qt * BN) >> 7) * args.sf_atoms +
                                               (size_t)kb * C::SF_APK) * 512u,
                                  (uint32_t)C::SFB_BYTES, fb, pol_a);
                    else if constexpr (C::BS)  // the A tile's scale atoms of this K block
                        bulk_load(smem_u32(sF + (size_t)stage * C::SF_BYTES),
                                  args.sf_a + ((size_t)un.pt * args.sf_atoms + (size_t)kb * C::SF_APK) * 512u,
                                  (uint32_t)C::SFA_BYTES, fb, pol_a);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        regs_decrease<kAuxRegs>();
        // -------------------------------------------------------- MMA issuer
        // (PAIR: rank 0 issues for both CTAs; rank 1's MMA warp only holds TMEM)
        if (lane == 0 && (!PAIR || rank == 0)) {
            uint32_t stage = 0, phase = 0, abuf = 0, aphase = 0, uphase = 0;
            uint32_t sfi = 0;  // block-scaled: K blocks issued, picks the TMEM copy of the scale factors
            for (int u = u_first; u < units; u += u_step) {
                const Unit un = decode_unit<FMT, PAIR, SWAP, BN>(args, u, rank, moe);
                if constexpr (FUSE) {
                    if (!mbar_wait(a_full, uphase)) goto done;
                    tc_fence_after();
                }
                for (int c0 = un.kb0; c0 < un.kb1; c0 += un.chunk_kb) {
                    const bool acc_free = PAIR ? mbar_wait_cluster(tempty0 + 8 * abuf, aphase ^ 1)
                                               : mbar_wait(tempty0 + 8 * abuf, aphase ^ 1);
                    if (!acc_free) goto done;
                    tc_fence_after();
                    const uint32_t d = tmem_base + abuf * C::ACC_COLS;
                    // the four MMAs (32 bytes of K each) of K block kb from stage st
                    auto issue_stage = [&](uint32_t st, int kb) {
                        const uint64_t adesc = smem_desc_k_sw128(smem_u32(sP + (size_t)st * C::P_BYTES));
                        const uint64_t bdesc =
                            FUSE ? smem_desc_k_sw128(sA + (uint32_t)((kb - un.kb0) * BN * 128))
                                 : smem_desc_k_sw128(smem_u32(sQ + (size_t)st * C::Q_BYTES));
                        if constexpr (C::BS) {
                            // this K block's scale factors into TMEM (the tensor pipe runs the
                            // copies and the MMAs in issue order); A's atoms, then W's, 4
                            // columns each: [atom][row group]
                            constexpr int RG = C::SF_RGQ;
                            const uint32_t sfa_t = tmem_base + C::SF_COL + (sfi & 1u) * C::SF_COLS;
                            const uint32_t sfb_t = sfa_t + 4 * C::SF_APK;
                            const uint32_t sfs = smem_u32(sF + (size_t)st * C::SF_BYTES);
#pragma unroll
                            for (int at = 0; at < C::SF_APK; ++at) {
                                tc_cp_sf(sfa_t + 4 * at, smem_desc_sf(sfs + 512 * at));
#pragma unroll
                                for (int j = 0; j < RG; ++j)
                                    tc_cp_sf(sfb_t + 4 * (at * RG + j),
                                             smem_desc_sf(sfs + C::SFA_BYTES + 512 * (j * C::SF_APK + at)));
                            }
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const uint32_t accum = (kb > c0 || k > 0) ? 1u : 0u;
                                if constexpr (C::KIND == kKindMXF8)  // byte k of the atom's column: sub-block k
                                    tc_mma_bs<C::KIND>(d, adesc + 2 * k, bdesc + 2 * k,
                                                       idesc_sf_ids(C::IDESC, (uint32_t)k, (uint32_t)k), sfa_t, sfb_t,
                                                       accum);
                                else  // one atom (four 16-element blocks) per MMA
                                    tc_mma_bs<C::KIND>(d, adesc + 2 * k, bdesc + 2 * k, C::IDESC, sfa_t + 4 * k,
                                                       sfb_t + 4 * k * RG, accum);
                            }
                            ++sfi;
                        } else {
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const uint32_t accum = (kb > c0 || k > 0) ? 1u : 0u;
                                if constexpr (PAIR)
                                    tc_mma_pair<C::KIND>(d, adesc + 2 * k, bdesc + 2 * k, C::IDESC, accum);
                                else
                                    tc_mma<C::KIND>(d, adesc + 2 * k, bdesc + 2 * k, C::IDESC, accum);
                            }
                        }
                    };
                    for (int kb = c0; kb < c0 + un.chunk_kb; ++kb) {
                        if constexpr (C::MMA_GROUP > 1) {
                            // G K blocks per pass (G waits, 4G MMAs, G commits): the
                            // issuing thread's per-K-block work (barrier test, fence,
                            // loop) sets the pace of narrow tiles; one pass over G
                            // stages spends it once.  Same MMAs in the same order.
                            constexpr int G = C::MMA_GROUP;
                            if (((kb - c0) % G) == 0 && kb + G <= c0 + un.chunk_kb) {
                                uint32_t sg[G], pg[G];
                                sg[0] = stage;
                                pg[0] = phase;
#pragma unroll
                                for (int g = 1; g < G; ++g) {
                                    const bool wrap = sg[g - 1] + 1 == STAGES;
                                    sg[g] = wrap ? 0u : sg[g - 1] + 1;
                                    pg[g] = wrap ? (pg[g - 1] ^ 1u) : pg[g - 1];
                                }
#pragma unroll
                                for (int g = 0; g < G; ++g)
                                    if (!mbar_wait(full0 + 8 * sg[g], pg[g])) goto done;
                                tc_fence_after();
#pragma unroll
                                for (int g = 0; g < G; ++g) issue_stage(sg[g], kb + g);
#pragma unroll
                                for (int g = 0; g < G; ++g) tc_commit(empty0 + 8 * sg[g]);
                                const bool wrap = sg[G - 1] + 1 == STAGES;
                                stage = wrap ? 0u : sg[G - 1] + 1;
                                phase = wrap ? (pg[G - 1] ^ 1u) : pg[G - 1];
                                kb += G - 1;
                                continue;
                            }
                        }
                        const bool landed = PAIR ? mbar_wait_cluster(full0 + 8 * stage, phase)
                                                 : mbar_wait(full0 + 8 * stage, phase);
                        if (!landed) goto done;
                        tc_fence_after();
                        issue_stage(stage, kb);
                        if constexpr (PAIR)
                            tc_commit_pair(empty0 + 8 * stage, 0x3);  // both CTAs may refill the stage
                        else
                            tc_commit(empty0 + 8 * stage);
                        if (++stage == STAGES) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                    if constexpr (PAIR)
                        tc_commit_pair(tfull0 + 8 * abuf, 0x3);  // both CTAs' accumulators are ready
                    else
                        tc_commit(tfull0 + 8 * abuf);
                    next_acc<NACC>(abuf, aphase);
                }
                if constexpr (FUSE) {
                    tc_commit(a_empty);  // arrives once every MMA of the unit has read sA
                    uphase ^= 1;
                }
            }
        }
    } else if (warp < kEpiWarps) {
        regs_increase<kEpiRegs>();
        // ---------------------------------------------------------- epilogue
        pdl_wait();  // scales are written by the previous kernel; C may be read by it
        EpiCtx e;
        e.quad = warp & 3;
        e.half = warp >> 2;
        e.lane = lane;
        e.row_lane = e.quad * 32 + lane;
        e.s_col = smem_u32(s_col);
        e.b_col = smem_u32(b_col);
        e.staging = smem_u32(smem + C::STAGING_OFF) + warp * 2048;
        e.tmap_c = &tmap_c;
        e.has_bias = args.bias != nullptr;
        e.row_scale = 0.f;
        e.row_bias = 0.f;
        e.rank = 0;
        e.recv = smem_u32(smem + C::RECV_OFF);
        e.recv_remote = 0;
        e.recv_full = recv_full;
        e.recv_free = recv_free;
        e.xphase = 0;
        if constexpr (CSK) {
            e.rank = (int)cluster_ctarank();
            e.recv_remote = mapa_shared(e.recv, 0);
        }
        const uint32_t t_lane = tmem_base + ((uint32_t)(e.quad * 32) << 16);
        const uint32_t t_total = t_lane + C::TOTAL_COL;
        const uint32_t t_seg = t_lane + C::SEG_COL;
        uint32_t abuf = 0, aphase = 0;
        // accumulator hand-over; PAIR: rank 0's MMAs fill both CTAs' TMEM and
        // both CTAs' epilogue warps hand the buffer back on rank 0's barrier
        auto acc_wait = [&](uint32_t bar, uint32_t parity) {
            return PAIR ? warp_wait_cluster(bar, parity) : warp_wait(bar, parity);
        };
        auto acc_release = [&](uint32_t bar) {
            if constexpr (PAIR) {
                __syncwarp();
                if (lane == 0) {
                    if (rank == 0)
                        mbar_arrive(bar);
                    else
                        mbar_arrive_remote(mapa_shared(bar, 0));
                }
            } else {
                warp_arrive(bar);
            }
        };
        if constexpr (FUSE) {
            if (u_first < units) {
                fused_quantize_unit<FMT, BN, C::A_MAXKB, true>(args, decode_unit<FMT>(args, u_first), sA, sa_tile,
                                                         rmax, xstage, kStagingBytes);
                warp_arrive(a_full);
            }
        }
        int ui = 0;  // this CTA's unit count so far (fused: scale buffer ui % 2)
        for (int u = u_first; u < units; u += u_step, ++ui) {
            const Unit un = decode_unit<FMT, PAIR, SWAP, BN>(args, u, rank, moe);
            const float* sa_cur = sa_tile + (ui & 1) * C::SA_FLOATS;
            // Fused: the next unit's rows are quantised once the MMA is done
            // with this unit's.  A unit whose MMAs fill one accumulator is
            // finished before its epilogue starts, so the next unit is
            // quantised first and its MMAs overlap this epilogue; a unit of
            // several accumulator chunks needs this epilogue to drain them
            // first, so its successor waits until after it.
            const int nxt = u + u_step;
            const bool quantise_next = FUSE && nxt < units;
            const bool next_first = (un.kb1 - un.kb0) == un.chunk_kb;
            if (quantise_next && next_first) {
                if (!warp_wait(a_empty, (uint32_t)(ui & 1))) goto done;
                fused_quantize_unit<FMT, BN, C::A_MAXKB>(args, decode_unit<FMT>(args, nxt), sA,
                                                         sa_tile + ((ui + 1) & 1) * C::SA_FLOATS, rmax, xstage,
                                                         kStagingBytes);
                warp_arrive(a_full);
            }
            if constexpr (!C::BLOCK) {
                // stage the tile's column scales (and bias) once; row values in registers
                named_bar_sync(1, kEpiThreads);
                for (int c = threadIdx.x; c < BN; c += kEpiThreads) {
                    const int q = un.qt * BN + c;
                    if constexpr (!SWAP) {
                        if constexpr (C::BS)  // NVFP4: W's decode scale; MXFP8: none (exact * 1)
                            s_col[c] = FMT == QLIN_FMT_NVFP4 ? __ldg(args.s_w) : 1.f;
                        else if constexpr (!C::BF16)
                            s_col[c] = q < args.N ? __ldg(args.s_w + un.wrow0 + q) : 0.f;
                        b_col[c] = (e.has_bias && q < args.N) ? bf16_to_f32(__ldg(args.bias + q)) : 0.f;
                    } else if constexpr (FUSE) {
                        s_col[c] = sa_cur[c];
                    } else if constexpr (C::BS) {  // NVFP4: the activations' decode scale
                        s_col[c] = FMT == QLIN_FMT_NVFP4 ? __ldg(args.s_a) : 1.f;
                    } else if constexpr (!C::BF16) {
                        s_col[c] = q < un.rows ? __ldg(args.s_a + un.row0 + q) : 0.f;
                    }
                }
                if constexpr (!SWAP) {
                    const int m = un.pt * 128 + e.row_lane;
                    if constexpr (C::BS)
                        e.row_scale = FMT == QLIN_FMT_NVFP4 ? __ldg(args.s_a) : 1.f;
                    else if constexpr (!C::BF16)
                        e.row_scale = m < un.rows ? __ldg(args.s_a + un.row0 + m) : 0.f;
                } else {
                    const int n = un.pt * 128 + e.row_lane;
                    if constexpr (C::BS)
                        e.row_scale = FMT == QLIN_FMT_NVFP4 ? __ldg(args.s_w) : 1.f;
                    else if constexpr (!C::BF16)
                        e.row_scale = n < args.N ? __ldg(args.s_w + un.wrow0 + n) : 0.f;
                    e.row_bias = (e.has_bias && n < args.N) ? bf16_to_f32(__ldg(args.bias + n)) : 0.f;
                }
                named_bar_sync(1, kEpiThreads);
            }
            const int nchunks = (un.kb1 - un.kb0) / un.chunk_kb;
            if (nchunks == 1 && !C::BLOCK) {
                // one accumulator holds the whole unit: stream this warp's slices
                if (!acc_wait(tfull0 + 8 * abuf, aphase)) goto done;
                tc_fence_after();
                const uint32_t tacc = t_lane + abuf * C::ACC_COLS;
                if (e.half >= C::NSLICE) {  // no slice for this warp: hand the buffer back
                    tc_fence_before();
                    acc_release(tempty0 + 8 * abuf);
                }
#pragma unroll 1
                for (int j = e.half; j < C::NSLICE; j += 2) {
                    uint32_t v[SW];
                    tmem_load_slice<SW>(tacc + j * SW, v);
                    tc_wait_ld();
                    if (j + 2 >= C::NSLICE) {  // this warp's last read of the accumulator
                        tc_fence_before();
                        acc_release(tempty0 + 8 * abuf);
                    }
                    if (!consume_segment_slice<FMT, SWAP, BN, CSK>(args, un, un.seg, j, t_total, e, v)) goto done;
                }
                next_acc<NACC>(abuf, aphase);
            } else if constexpr (C::MULTI) {
                if constexpr (C::BLOCK && !SWAP) {
                    // Block-FP8, plain tiles: one 128-wide K block per
                    // accumulator.  Each thread loads its row's 64 columns of
                    // the K block's products P_kb (slices 2h and 2h+1 for slice
                    // parity h), hands the buffer straight back (the MMA runs
                    // ahead into the other buffers), and promotes them into the
                    // segment sum it keeps in registers,
                    //   seg = fma(P_kb, s_a[m,kb] * s_w[n/128,kb], seg)  from +0,
                    // two lanes per instruction.  The tile's 128 columns lie in
                    // one 128-block of N, so the scale product is one value per
                    // row and K block, read from the staged table.
                    static_assert(C::NSLICE == 4 && SW == 32, "128-column tiles");
                    const uint32_t bsc = smem_u32(smem + C::BSCALE_OFF);
                    const int kbps = args.kb_per_seg;
                    int win0 = -C::BS_KB;
                    int kin = 0;                          // K block within the segment
                    int seg_no = args.spread ? un.seg : 0;
                    float sg[2 * SW];                     // the segment sum of this thread's 64 columns
                    for (int c0 = un.kb0; c0 < un.kb1; ++c0) {
                        const bool seg_start = kin == 0;
                        if (c0 - win0 >= C::BS_KB) {
                            win0 = c0;
                            stage_block_scales<FMT, SWAP, BN, CSK, FUSE, PAIR>(args, un, win0, bsc, nullptr);
                        }
                        float row_scale;
                        asm volatile("ld.shared.f32 %0, [%1];"
                                     : "=f"(row_scale)
                                     : "r"(bsc + (uint32_t)((c0 - win0) * C::BS_PITCH + e.row_lane) * 4u));
                        constexpr int P = C::BLOCK_PASS;
                        if (kin + P - 1 < kbps && c0 + P - 1 < un.kb1 && c0 + P - 1 - win0 < C::BS_KB) {
                            // P K blocks of the segment in one pass: one accumulator
                            // wait covers them all (the last buffer's commit arrives
                            // only after every earlier MMA has completed); each block
                            // is then loaded, released and folded in, the same fmas in
                            // the same order
                            float rs[P];
                            rs[0] = row_scale;
#pragma unroll
                            for (int q = 1; q < P; ++q)
                                asm volatile("ld.shared.f32 %0, [%1];"
                                             : "=f"(rs[q])
                                             : "r"(bsc + (uint32_t)((c0 + q - win0) * C::BS_PITCH + e.row_lane) * 4u));
                            uint32_t bl = abuf, pl = aphase;
#pragma unroll
                            for (int q = 1; q < P; ++q) next_acc<NACC>(bl, pl);
                            if (!acc_wait(tfull0 + 8 * bl, pl)) goto done;
                            tc_fence_after();
#pragma unroll
                            for (int q = 0; q < P; ++q) {
                                uint32_t v[2 * SW];
                                tmem_ld64(t_lane + abuf * C::ACC_COLS + e.half * 2 * SW, v);
                                tc_wait_ld();
                                tc_fence_before();
                                acc_release(tempty0 + 8 * abuf);
                                next_acc<NACC>(abuf, aphase);
                                if (q == 0 && seg_start) {
#pragma unroll
                                    for (int c = 0; c < 2 * SW; c += 2)
                                        fma2_rn(sg[c], sg[c + 1], __uint_as_float(v[c]), __uint_as_float(v[c + 1]),
                                                rs[q], 0.f, 0.f);
                                } else {
#pragma unroll
                                    for (int c = 0; c < 2 * SW; c += 2)
                                        fma2_rn(sg[c], sg[c + 1], __uint_as_float(v[c]), __uint_as_float(v[c + 1]),
                                                rs[q], sg[c], sg[c + 1]);
                                }
                            }
                            c0 += P - 1;
                            kin += P;
                            if (kin < kbps) continue;
                        } else {
                            if (!acc_wait(tfull0 + 8 * abuf, aphase)) goto done;
                            tc_fence_after();
                            uint32_t v[2 * SW];
                            tmem_ld64(t_lane + abuf * C::ACC_COLS + e.half * 2 * SW, v);
                            tc_wait_ld();
                            tc_fence_before();
                            acc_release(tempty0 + 8 * abuf);
                            next_acc<NACC>(abuf, aphase);
                            if (seg_start) {
#pragma unroll
                                for (int c = 0; c < 2 * SW; c += 2)
                                    fma2_rn(sg[c], sg[c + 1], __uint_as_float(v[c]), __uint_as_float(v[c + 1]), row_scale,
                                            0.f, 0.f);
                            } else {
#pragma unroll
                                for (int c = 0; c < 2 * SW; c += 2)
                                    fma2_rn(sg[c], sg[c + 1], __uint_as_float(v[c]), __uint_as_float(v[c + 1]), row_scale,
                                            sg[c], sg[c + 1]);
                            }
                            if (++kin < kbps) continue;
                        }
                        kin = 0;
                        // segment end: Split-K writes the segment out; otherwise
                        // total = total + seg in segment order from +0 (the total
                        // lives in TMEM between segments), and the last segment
                        // finishes the tile
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const int j = 2 * e.half + i;
                            uint32_t out[SW];
                            if (args.spread) {
#pragma unroll
                                for (int c = 0; c < SW; ++c) out[c] = __float_as_uint(sg[i * SW + c]);
                                store_partial<SW>(partial_ptr<SW>(args, un.tile, un.seg, j, C::NSLICE, e.row_lane), out);
                                continue;
                            }
                            if (seg_no == 0) {
#pragma unroll
                                for (int c = 0; c < SW; ++c) out[c] = __float_as_uint(__fadd_rn(0.f, sg[i * SW + c]));
                            } else {
                                tmem_load_slice<SW>(t_total + j * SW, out);
                                tc_wait_ld();
#pragma unroll
                                for (int c = 0; c < SW; ++c)
                                    out[c] = __float_as_uint(__fadd_rn(__uint_as_float(out[c]), sg[i * SW + c]));
                            }
                            if (seg_no == args.S - 1)
                                finish_slice<FMT, SWAP, BN>(args, un, j, e, out);
                            else
                                tmem_store_slice<SW>(t_total + j * SW, out);
                        }
                        tc_wait_st();  // the running total is read again at the next segment end
                        ++seg_no;
                    }
                } else if constexpr (C::BLOCK) {
                    // Block-FP8, Swap-AB tiles: promote every 128-wide K block
                    // into the fp32 segment sum kept in TMEM,
                    // seg = fma(P_kb, s_a[m,kb] * s_w[n/128,kb], seg); the scale
                    // product is one value per column m (the tile's 128 lanes
                    // lie in one 128-block of N), read from the staged table.
                    const uint32_t bsc = smem_u32(smem + C::BSCALE_OFF);
                    int win0 = -C::BS_KB;
                    for (int c0 = un.kb0; c0 < un.kb1; ++c0) {
                        const int rel = c0 - (args.spread ? un.kb0 : 0);
                        const int seg_no = args.spread ? un.seg : rel / args.kb_per_seg;
                        const bool seg_start = (rel % args.kb_per_seg) == 0;
                        const bool seg_end = ((rel + 1) % args.kb_per_seg) == 0;
                        if (c0 - win0 >= C::BS_KB) {
                            win0 = c0;
                            stage_block_scales<FMT, SWAP, BN, CSK, FUSE, PAIR>(args, un, win0, bsc, sa_cur);
                        }
                        const uint32_t bsrow = bsc + (uint32_t)((c0 - win0) * C::BS_PITCH) * 4u;
                        if (!acc_wait(tfull0 + 8 * abuf, aphase)) goto done;
                        tc_fence_after();
                        const uint32_t tacc = t_lane + abuf * C::ACC_COLS;
#pragma unroll 1
                        for (int j = e.half; j < C::NSLICE; j += 2) {
                            // this K block's accumulator and (after the first block of
                            // the segment) the segment's running sum, both from TMEM
                            uint32_t v[SW], sg[SW];
                            tmem_load_slice<SW>(tacc + j * SW, v);
                            if (!seg_start) tmem_load_slice<SW>(t_seg + j * SW, sg);
                            tc_wait_ld();
#pragma unroll
                            for (int c = 0; c < SW; ++c) {
                                float sc;  // column scale, same address for the whole warp
                                asm volatile("ld.shared.f32 %0, [%1];" : "=f"(sc) : "r"(bsrow + (uint32_t)(j * SW + c) * 4u));
                                const float prev = seg_start ? 0.f : __uint_as_float(sg[c]);
                                sg[c] = __float_as_uint(__fmaf_rn(__uint_as_float(v[c]), sc, prev));
                            }
                            if (seg_end) {
                                if (!consume_segment_slice<FMT, SWAP, BN, CSK>(args, un, seg_no, j, t_total, e, sg))
                                    goto done;
                            } else {
                                tmem_store_slice<SW>(t_seg + j * SW, sg);
                            }
                        }
                        tc_wait_st();
                        tc_fence_before();
                        acc_release(tempty0 + 8 * abuf);
                        next_acc<NACC>(abuf, aphase);
                    }
                } else {
                    // FP8 per-token, plain variant with S > 1: one chunk per
                    // segment, summed into the TMEM running total in order.
                    int seg_no = 0;
                    for (int c0 = un.kb0; c0 < un.kb1; c0 += un.chunk_kb, ++seg_no) {
                        if (!acc_wait(tfull0 + 8 * abuf, aphase)) goto done;
                        tc_fence_after();
                        const uint32_t tacc = t_lane + abuf * C::ACC_COLS;
#pragma unroll 1
                        for (int j = e.half; j < C::NSLICE; j += 2) {
                            uint32_t v[SW];
                            tmem_load_slice<SW>(tacc + j * SW, v);
                            tc_wait_ld();
                            if (!consume_segment_slice<FMT, SWAP, BN, CSK>(args, un, seg_no, j, t_total, e, v))
                                goto done;
                        }
                        tc_wait_st();
                        tc_fence_before();
                        acc_release(tempty0 + 8 * abuf);
                        next_acc<NACC>(abuf, aphase);
                    }
                }
            }
            if constexpr (CSK) {
                // per-tile exchange: ranks > 0 tell rank 0 their slices are in
                // place; rank 0 hands the receive area back once it has read it
                if (e.rank != 0) {
                    if (e.half >= C::NSLICE && !warp_wait_cluster(e.recv_free, e.xphase ^ 1u)) goto done;
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote(mapa_shared(e.recv_full, 0));
                } else {
                    // warps without a slice wait too, so that a wait that gives
                    // up sends every epilogue warp out together
                    if (e.half >= C::NSLICE && !warp_wait_cluster(e.recv_full, e.xphase)) goto done;
                    named_bar_sync(1, kEpiThreads);
                    if (threadIdx.x == 0)
                        for (int r = 1; r < args.S; ++r) mbar_arrive_remote(mapa_shared(e.recv_free, (uint32_t)r));
                }
                e.xphase ^= 1u;
            } else {
                if (args.spread) splitk_finish<FMT, SWAP, BN>(args, un, e, bcast);
            }
            if (quantise_next && !next_first) {
                if (!warp_wait(a_empty, (uint32_t)(ui & 1))) goto done;
                fused_quantize_unit<FMT, BN, C::A_MAXKB>(args, decode_unit<FMT>(args, nxt), sA,
                                                         sa_tile + ((ui + 1) & 1) * C::SA_FLOATS, rmax, xstage,
                                                         kStagingBytes);
                warp_arrive(a_full);
            }
        }
    } else {
        regs_decrease<kAuxRegs>();  // warps 10 and 11: idle members of warpgroup 2
    }
done:
    // the bulk stores of C have completed (and left the staging buffers)
    if (!SWAP && warp < kEpiWarps && lane == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if constexpr (PAIR) {
        // both CTAs are done with the TMEM that rank 0's MMAs wrote, and with
        // each other's barriers, before the pair frees its columns
        cluster_sync();
        tc_fence_after();
        if (warp == kMmaWarp) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    } else {
        if (warp == kMmaWarp) tmem_dealloc(tmem_base, C::TMEM_COLS);
        // no CTA leaves while another rank may still arrive on its barriers or
        // store into its shared memory
        if constexpr (CSK) cluster_sync();
    }
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

// K-major operand [rows, K] (8-bit or bf16 elements) as a 2-D tensor map over
// its bytes, K_bytes per row, with a (128 B x box_rows) box and the 128-byte
// swizzle (the layout the MMA descriptors describe).
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

// bf16 C [M, N] (row stride N) as a 2-D tensor map with a 32 x 32 box and the
// 64-byte swizzle (the layout the epilogue writes into its staging buffer).
bool make_output_tmap(CUtensorMap* map, const void* base, int64_t M, int64_t N) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)N * 2};
    cuuint32_t box[2] = {32u, 32u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int FMT, bool SWAP, int BN, bool CSK, bool FUSE, bool PAIR>
qlin_status launch_instance(const GemmPlan& plan, const GemmOperands& ops, cudaStream_t st) {
    using C = Cfg<FMT, SWAP, BN, CSK, FUSE, PAIR>;
    auto kern = qlin_gemm_kernel<FMT, SWAP, BN, CSK, FUSE, PAIR>;
    static int configured_device = -1;
    static int max_clusters[QLIN_MAX_CLUSTER + 1];  // co-resident clusters per cluster size, this device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QLIN_ERR_CUDA;
    const int S = plan.k_segments;
    if (CSK && (S < 2 || S > C::CSK_MAXS)) return QLIN_ERR_UNSUPPORTED;
    if (configured_device != dev) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM) != cudaSuccess)
            return QLIN_ERR_CUDA;
        // the in-kernel register split must fit the launch allocation
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return QLIN_ERR_CUDA;
        if (fa.numRegs < kLaunchRegs) return QLIN_ERR_UNSUPPORTED;
        for (int& m : max_clusters) m = -1;
        configured_device = dev;
    }
    if (FUSE && plan.kb_per_unit > C::A_MAXKB) return QLIN_ERR_UNSUPPORTED;
    alignas(64) CUtensorMap tp, tq;
    const void* p_base = SWAP ? ops.w_q : ops.a_q;
    const void* q_base = SWAP ? ops.a_q : ops.w_q;
    if (!make_operand_tmap(&tp, p_base, plan.p_rows, plan.k_bytes, 128)) return QLIN_ERR_CUDA;
    if (FUSE)
        tq = tp;  // unused: the kernel quantises its activation operand in place
    else if (!make_operand_tmap(&tq, q_base, plan.q_rows, plan.k_bytes, PAIR ? BN / 2 : BN))  // PAIR: half a W tile
        return QLIN_ERR_CUDA;
    alignas(64) CUtensorMap tc;  // plain tiles: bf16 C in 32 x 32 boxes
    if (!SWAP && !ops.out_i32) {
        if (!make_output_tmap(&tc, ops.c, plan.M, plan.N)) return QLIN_ERR_CUDA;
    } else {
        tc = tp;  // unused (Swap-AB stores columns of C directly; int32 output stores directly)
    }
    GemmArgs a;
    a.s_a = ops.s_a;
    a.s_w = ops.s_w;
    a.bias = static_cast<const uint16_t*>(ops.bias);
    a.c = ops.c;
    const bool global_split = plan.spread && !CSK;
    a.tickets = global_split ? static_cast<int32_t*>(ops.workspace) : nullptr;
    a.partials = global_split
                     ? reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ops.workspace) + plan.ticket_bytes)
                     : nullptr;
    a.M = (int)plan.M;
    a.N = (int)plan.N;
    a.kblocks = plan.kblocks;
    a.S = S;
    a.kb_per_seg = plan.kb_per_seg;
    a.p_tiles = (int)plan.p_tiles;
    a.units = (int)plan.units;
    a.spread = plan.spread ? 1 : 0;
    a.out_i32 = ops.out_i32 ? 1 : 0;
    a.x = FUSE ? static_cast<const uint16_t*>(ops.x) : nullptr;
    a.ld_x = FUSE ? ops.ld_x : 0;
    a.a_q_out = FUSE ? static_cast<uint8_t*>(const_cast<void*>(ops.a_q)) : nullptr;
    a.s_a_out = FUSE ? const_cast<float*>(ops.s_a) : nullptr;
    a.moe_offsets = ops.moe_offsets;
    a.moe_E = plan.moe_E;
    a.sf_a = static_cast<const uint8_t*>(ops.sf_a);
    a.sf_w = static_cast<const uint8_t*>(ops.sf_w);
    a.sf_atoms = plan.kblocks * C::SF_APK;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)plan.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int nattr = 0;
    const int csize = PAIR ? 2 : S;  // CTAs per cluster
    if (CSK || PAIR) {
        attr[nattr].id = cudaLaunchAttributeClusterDimension;
        attr[nattr].val.clusterDim.x = (unsigned)csize;
        attr[nattr].val.clusterDim.y = 1;
        attr[nattr].val.clusterDim.z = 1;
        ++nattr;
        cfg.attrs = attr;
        cfg.numAttrs = nattr;
        if (max_clusters[csize] < 0) {
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) return QLIN_ERR_CUDA;
            max_clusters[csize] = n;
        }
        if (max_clusters[csize] < 1) return QLIN_ERR_UNSUPPORTED;
        // every CTA of a cluster walks the same tiles: grid = clusters x cluster size
        const int64_t clusters = std::min<int64_t>(plan.num_tiles, max_clusters[csize]);
        cfg.gridDim = dim3((unsigned)(clusters * csize));
    }
    if (ops.pdl) {
        attr[nattr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[nattr].val.programmaticStreamSerializationAllowed = 1;
        ++nattr;
    }
    cfg.attrs = attr;
    cfg.numAttrs = nattr;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tp, tq, tc, a);
    return e == cudaSuccess ? QLIN_OK : QLIN_ERR_CUDA;
}

template <int FMT, bool SWAP, int BN, bool CSK, bool FUSE, bool PAIR>
void cfg_info(int* stages, size_t* smem) {
    *stages = Cfg<FMT, SWAP, BN, CSK, FUSE, PAIR>::STAGES;
    *smem = Cfg<FMT, SWAP, BN, CSK, FUSE, PAIR>::SMEM;
}

// One switch over every kernel instantiation: OP<FMT, SWAP, BN, CSK, FUSE, PAIR>
// is applied to the one matching (swap, tile_n, mode); false if none exists.
template <int FMT, template <int, bool, int, bool, bool, bool> class OP, typename... A>
bool dispatch_instance(bool swap, int tile_n, int mode, A&&... args) {
    if constexpr (is_block_scaled(FMT)) {  // plain 128 x 128 and Swap-AB 32 / 64 tiles (with Split-K)
        if (mode != kModeStd) return false;
        switch ((swap ? 1000 : 0) + tile_n) {
            case 128: OP<FMT, false, 128, false, false, false>::run(args...); return true;
            case 1032: OP<FMT, true, 32, false, false, false>::run(args...); return true;
            case 1064: OP<FMT, true, 64, false, false, false>::run(args...); return true;
        }
        return false;
    } else {
    if (swap) {
        switch (mode * 1000 + tile_n) {
            case kModeStd * 1000 + 16: OP<FMT, true, 16, false, false, false>::run(args...); return true;
            case kModeStd * 1000 + 32: OP<FMT, true, 32, false, false, false>::run(args...); return true;
            case kModeStd * 1000 + 64: OP<FMT, true, 64, false, false, false>::run(args...); return true;
            case kModeCluster * 1000 + 16: OP<FMT, true, 16, true, false, false>::run(args...); return true;
            case kModeCluster * 1000 + 32: OP<FMT, true, 32, true, false, false>::run(args...); return true;
            case kModeCluster * 1000 + 64: OP<FMT, true, 64, true, false, false>::run(args...); return true;
        }
        if constexpr (FMT != QLIN_FMT_BF16) {
            switch (mode * 1000 + tile_n) {
                case kModeFused * 1000 + 16: OP<FMT, true, 16, false, true, false>::run(args...); return true;
                case kModeFused * 1000 + 32: OP<FMT, true, 32, false, true, false>::run(args...); return true;
                case kModeFused * 1000 + 64: OP<FMT, true, 64, false, true, false>::run(args...); return true;
            }
        }
        return false;
    }
    if (mode == kModePair) {
        if constexpr (FMT != QLIN_FMT_FP8_BLOCK) {
            if (tile_n == 256) {
                OP<FMT, false, 256, false, false, true>::run(args...);
                return true;
            }
        }
        return false;
    }
    if (mode != kModeStd) return false;
    if (tile_n == 128) {
        OP<FMT, false, 128, false, false, false>::run(args...);
        return true;
    }
    if constexpr (FMT != QLIN_FMT_FP8_BLOCK) {
        if (tile_n == 256) {
            OP<FMT, false, 256, false, false, false>::run(args...);
            return true;
        }
    }
    return false;
    }
}

template <int FMT, bool SWAP, int BN, bool CSK, bool FUSE, bool PAIR>
struct LaunchOp {
    static void run(const GemmPlan& p, const GemmOperands& ops, cudaStream_t st, qlin_status* out) {
        *out = launch_instance<FMT, SWAP, BN, CSK, FUSE, PAIR>(p, ops, st);
    }
};

template <int FMT, bool SWAP, int BN, bool CSK, bool FUSE, bool PAIR>
struct InfoOp {
    static void run(int* stages, size_t* smem) { cfg_info<FMT, SWAP, BN, CSK, FUSE, PAIR>(stages, smem); }
};

template <int FMT>
qlin_status launch_fmt(const GemmPlan& p, const GemmOperands& ops, cudaStream_t st) {
    qlin_status r = QLIN_ERR_UNSUPPORTED;
    if (!dispatch_instance<FMT, LaunchOp>(p.swap, p.tile_n, p.mode, p, ops, st, &r)) return QLIN_ERR_UNSUPPORTED;
    return r;
}

}  // namespace

bool gemm_kernel_info(int fmt, bool swap, int tile_n, int mode, int* stages, size_t* smem_bytes) {
    switch (fmt) {
        case QLIN_FMT_INT8: return dispatch_instance<QLIN_FMT_INT8, InfoOp>(swap, tile_n, mode, stages, smem_bytes);
        case QLIN_FMT_FP8: return dispatch_instance<QLIN_FMT_FP8, InfoOp>(swap, tile_n, mode, stages, smem_bytes);
        case QLIN_FMT_FP8_BLOCK:
            return dispatch_instance<QLIN_FMT_FP8_BLOCK, InfoOp>(swap, tile_n, mode, stages, smem_bytes);
        case QLIN_FMT_BF16: return dispatch_instance<QLIN_FMT_BF16, InfoOp>(swap, tile_n, mode, stages, smem_bytes);
        case QLIN_FMT_MXFP8: return dispatch_instance<QLIN_FMT_MXFP8, InfoOp>(swap, tile_n, mode, stages, smem_bytes);
        case QLIN_FMT_NVFP4: return dispatch_instance<QLIN_FMT_NVFP4, InfoOp>(swap, tile_n, mode, stages, smem_bytes);
    }
    return false;
}


// Failure-path self-test: one thread waits, with the given limit, on an
// mbarrier that nothing ever arrives on; the wait gives up, records
// QLIN_ERR_DEVICE_TIMEOUT and the kernel returns normally.
__global__ void qlin_wait_selftest_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbarrier_init();
        (void)mbar_wait_for(smem_u32(&bar), 0, limit_ns);
    }
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t st) {
    qlin_wait_selftest_kernel<<<1, 32, 0, st>>>(limit_ns);
    return cudaGetLastError();
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
        case QLIN_FMT_BF16: return launch_fmt<QLIN_FMT_BF16>(plan, ops, st);
        case QLIN_FMT_MXFP8: return launch_fmt<QLIN_FMT_MXFP8>(plan, ops, st);
        case QLIN_FMT_NVFP4: return launch_fmt<QLIN_FMT_NVFP4>(plan, ops, st);
        default: return QLIN_ERR_INVALID_ARG;
    }
}

}  // namespace qlin
