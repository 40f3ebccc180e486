// qlin_sweep.cu -- offline sweep that writes the per-shape dispatch table.
//
// The page "Helion in vLLM: A Unified Route to Tunable Linear Kernels"
// ("Algorithm choice becomes part of tuning") has the GEMM variant chosen per
// shape by an ahead-of-time search, and "[Kernel][Perf] Add Hopper (SM90) tuned
// config for batch-invariant persistent matmul" keys such tables by device and
// M bucket.  This program is that search for this library, over a bounded grid
// (minutes, not hours):
//
//   for each (format, N, K):
//     for each K segmentation S dividing K/128 (S in {1,2,3,4,6,8}):
//       for each M bucket: time every variant / tile the library offers,
//         keep only those whose output is bitwise equal to the plain variant
//         with the same S (every variant must sum segments in the same order)
//     pick the S with the smallest summed best time over the buckets (one S
//     per shape, so results never depend on the batch size), and for each
//     bucket the fastest variant under that S
//
// Timing: a CUDA graph of `iters` launches (each reading a different weight
// copy, with enough copies that the bytes between two uses of one copy exceed
// 2x L2), launched with QLIN_PDL as the hot path runs, CUDA events around the
// graph, median of `reps` replays.
//
// Usage: qlin_sweep [--quick] <out.qlt> [shape ...]   shape = fmt:N:K (fmt int8|fp8|fp8_block|bf16|mxfp8|nvfp4)
// Without shapes it sweeps the five workload shapes.  --quick (for tests):
// buckets {1, 16, 256} only, two weight copies, short timing loops.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "qlin.h"

#define CK(x)                                                                                     \
    do {                                                                                          \
        cudaError_t e_ = (x);                                                                     \
        if (e_ != cudaSuccess) {                                                                  \
            std::fprintf(stderr, "CUDA error %s at %s:%d\n", cudaGetErrorString(e_), __FILE__, __LINE__); \
            std::exit(2);                                                                         \
        }                                                                                         \
    } while (0)

namespace {

struct Shape {
    int fmt;
    int64_t N, K;
};

struct Cand {
    int variant, tile_n;
};

const char* fmt_name(int f) {
    switch (f) {
        case QLIN_FMT_INT8: return "int8";
        case QLIN_FMT_FP8: return "fp8";
        case QLIN_FMT_FP8_BLOCK: return "fp8_block";
        case QLIN_FMT_MXFP8: return "mxfp8";
        case QLIN_FMT_NVFP4: return "nvfp4";
    }
    return "bf16";
}
bool block_scaled(int f) { return f == QLIN_FMT_MXFP8 || f == QLIN_FMT_NVFP4; }
// bytes of one operand row of K elements
int64_t row_bytes(int f, int64_t K) { return f == QLIN_FMT_BF16 ? 2 * K : (f == QLIN_FMT_NVFP4 ? K / 2 : K); }
// bytes of the tiled scale factors of a [rows, K] block-scaled operand
size_t sf_bytes(int f, int64_t rows, int64_t K) {
    return (size_t)((rows + 127) / 128) * (size_t)(K / (f == QLIN_FMT_MXFP8 ? 128 : 64)) * 512u;
}
const char* var_name(int v) {
    switch (v) {
        case QLIN_VAR_PLAIN: return "plain";
        case QLIN_VAR_SPLITK: return "splitk";
        case QLIN_VAR_SWAPAB: return "swapab";
        case QLIN_VAR_SWAPAB_SPLITK: return "swapab_splitk";
        case QLIN_VAR_PAIR: return "pair";
    }
    return "auto";
}

// Deterministic filler: int8 bytes, or finite e4m3 codes (no 0x7F / 0xFF NaNs).
__global__ void fill_codes(uint8_t* p, size_t n, uint32_t seed, int e4m3) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        uint32_t h = (uint32_t)i * 2654435761u ^ seed;
        h ^= h >> 13;
        h *= 0x5bd1e995u;
        h ^= h >> 15;
        uint8_t v = (uint8_t)h;
        if (e4m3) v = (uint8_t)((v & 0x80) | ((v & 0x7F) % 0x77));  // |code| <= 0x76 (240)
        p[i] = v;
    }
}

// Deterministic bf16 filler: values of magnitude below 2 (exponent field 112..127).
__global__ void fill_bf16(uint16_t* p, size_t n, uint32_t seed) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        uint32_t h = (uint32_t)i * 2654435761u ^ seed;
        h ^= h >> 13;
        h *= 0x5bd1e995u;
        h ^= h >> 15;
        p[i] = (uint16_t)((h & 0x807Fu) | ((112u + ((h >> 8) & 15u)) << 7));
    }
}

// Block scale codes: E8M0 2^-7 .. 2^7 (MXFP8) or E4M3 0.5 .. 1.875 (NVFP4), never NaN.
__global__ void fill_sf(uint8_t* p, size_t n, uint32_t seed, int e8m0) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        uint32_t h = (uint32_t)i * 2246822519u ^ seed;
        h ^= h >> 15;
        p[i] = e8m0 ? (uint8_t)(120u + h % 15u) : (uint8_t)(0x30u + h % 16u);
    }
}

__global__ void fill_scales(float* p, size_t n, uint32_t seed) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        uint32_t h = (uint32_t)i * 747796405u + seed;
        h ^= h >> 16;
        p[i] = 1e-3f * (1.0f + (float)(h & 1023) / 1024.0f);
    }
}

struct Problem {
    Shape s;
    int64_t M;
    void* a_q = nullptr;
    float* s_a = nullptr;    // block-scaled formats: the tiled scale bytes
    float* g = nullptr;      // NVFP4: the two per-tensor decode scales
    std::vector<void*> w_q;
    std::vector<float*> s_w;
    uint16_t* c = nullptr;
    uint16_t* c_ref = nullptr;
    void* ws = nullptr;
    size_t ws_bytes = 0;
};

std::vector<int> segment_choices(int fmt, int64_t K) {
    std::vector<int> out;
    const int kb = (int)(row_bytes(fmt, K) / 128);
    for (int s : {1, 2, 3, 4, 6, 8})
        if (kb % s == 0 && kb / s >= 1) out.push_back(s);
    return out;
}

std::vector<Cand> candidates(int fmt, int64_t M) {
    std::vector<Cand> c;
    if (block_scaled(fmt)) {  // Swap-AB 32 / 64 for one activation tile; plain 128
        for (int t : {32, 64}) {
            if (M > t || (t == 64 && M <= 32)) continue;
            c.push_back({QLIN_VAR_SWAPAB, t});
            c.push_back({QLIN_VAR_SWAPAB_SPLITK, t});
        }
        c.push_back({QLIN_VAR_PLAIN, 128});
        c.push_back({QLIN_VAR_SPLITK, 128});
        return c;
    }
    for (int t : {16, 32, 64}) {
        if (t >= 2 * M && t > 16) continue;  // a tile more than twice M only wastes the narrow side
        if (M > 64 && t < 64) continue;
        c.push_back({QLIN_VAR_SWAPAB, t});
        c.push_back({QLIN_VAR_SWAPAB_SPLITK, t});
    }
    if (M >= 16) {
        for (int t : {128, 256}) {
            if (fmt == QLIN_FMT_FP8_BLOCK && t == 256) continue;
            c.push_back({QLIN_VAR_PLAIN, t});
            c.push_back({QLIN_VAR_SPLITK, t});
        }
        // 256-row tiles on CTA pairs: only worth a try once M fills two 128-row halves
        if (fmt != QLIN_FMT_FP8_BLOCK && M >= 256) c.push_back({QLIN_VAR_PAIR, 256});
    }
    return c;
}

// One GEMM call of the problem's format on weight copy w.
qlin_status run_gemm(Problem& P, int variant, int tile, int S, size_t w, uint16_t* c, uint32_t flags,
                     cudaStream_t st) {
    if (P.s.fmt == QLIN_FMT_BF16)
        return qlin_matmul_bf16(variant, tile, S, P.M, P.s.N, P.s.K, P.a_q, P.w_q[w], nullptr, c, flags, P.ws,
                                P.ws_bytes, st);
    if (block_scaled(P.s.fmt)) {
        const bool nv = P.s.fmt == QLIN_FMT_NVFP4;
        return qlin_block_scaled_mm(P.s.fmt, variant, tile, S, P.M, P.s.N, P.s.K, P.a_q, P.s_a, P.w_q[w], P.s_w[w],
                                    nv ? P.g : nullptr, nv ? P.g + 1 : nullptr, nullptr, c, flags, P.ws, P.ws_bytes,
                                    st);
    }
    return qlin_scaled_mm(P.s.fmt, variant, tile, S, P.M, P.s.N, P.s.K, P.a_q, P.s_a, P.w_q[w], P.s_w[w], nullptr, c,
                          flags, P.ws, P.ws_bytes, st);
}

float time_config(Problem& P, int variant, int tile, int S, int iters, int reps, cudaStream_t st, bool* ok) {
    *ok = false;
    size_t need = 0;
    if (qlin_scaled_mm_workspace_size(P.s.fmt, variant, tile, S, P.M, P.s.N, P.s.K, &need) != QLIN_OK) return -1.f;
    if (need > P.ws_bytes) return -1.f;
    // correctness / warm-up launch on copy 0
    if (run_gemm(P, variant, tile, S, 0, P.c, QLIN_PDL, st) != QLIN_OK) return -1.f;
    cudaGraph_t graph;
    cudaGraphExec_t exec;
    CK(cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal));
    for (int i = 0; i < iters; ++i) {
        const size_t w = (size_t)(i + 1) % P.w_q.size();
        if (run_gemm(P, variant, tile, S, w, P.c, QLIN_PDL, st) != QLIN_OK) {
            cudaStreamEndCapture(st, &graph);
            cudaGraphDestroy(graph);
            return -1.f;
        }
    }
    CK(cudaStreamEndCapture(st, &graph));
    CK(cudaGraphInstantiate(&exec, graph, 0));
    cudaEvent_t e0, e1;
    CK(cudaEventCreate(&e0));
    CK(cudaEventCreate(&e1));
    CK(cudaGraphLaunch(exec, st));
    std::vector<float> ts;
    for (int r = 0; r < reps; ++r) {
        CK(cudaEventRecord(e0, st));
        CK(cudaGraphLaunch(exec, st));
        CK(cudaEventRecord(e1, st));
        CK(cudaEventSynchronize(e1));
        float ms = 0.f;
        CK(cudaEventElapsedTime(&ms, e0, e1));
        ts.push_back(ms * 1000.f / iters);
    }
    CK(cudaEventDestroy(e0));
    CK(cudaEventDestroy(e1));
    CK(cudaGraphExecDestroy(exec));
    CK(cudaGraphDestroy(graph));
    if (qlin_sync_status(st) != QLIN_OK) return -1.f;
    std::sort(ts.begin(), ts.end());
    *ok = true;
    return ts[ts.size() / 2];
}

bool same_output(Problem& P, int variant, int tile, int S, cudaStream_t st) {
    if (run_gemm(P, variant, tile, S, 0, P.c, 0, st) != QLIN_OK) return false;
    CK(cudaStreamSynchronize(st));
    const size_t bytes = (size_t)P.M * P.s.N * 2;
    std::vector<uint16_t> a(bytes / 2), b(bytes / 2);
    CK(cudaMemcpy(a.data(), P.c, bytes, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(b.data(), P.c_ref, bytes, cudaMemcpyDeviceToHost));
    return std::memcmp(a.data(), b.data(), bytes) == 0;
}

}  // namespace

int main(int argc, char** argv) {
    bool quick = false;
    int first = 1;
    if (argc > 1 && std::strcmp(argv[1], "--quick") == 0) {
        quick = true;
        first = 2;
    }
    if (argc < first + 1) {
        std::fprintf(stderr, "usage: %s [--quick] out.qlt [fmt:N:K ...]\n", argv[0]);
        return 1;
    }
    const char* out_path = argv[first];
    std::vector<Shape> shapes;
    for (int i = first + 1; i < argc; ++i) {
        char f[32];
        long long n, k;
        if (std::sscanf(argv[i], "%31[^:]:%lld:%lld", f, &n, &k) != 3) return 1;
        const std::string fs(f);
        shapes.push_back({fs == "int8"    ? QLIN_FMT_INT8
                          : fs == "fp8"   ? QLIN_FMT_FP8
                          : fs == "bf16"  ? QLIN_FMT_BF16
                          : fs == "mxfp8" ? QLIN_FMT_MXFP8
                          : fs == "nvfp4" ? QLIN_FMT_NVFP4
                                          : QLIN_FMT_FP8_BLOCK,
                          n, k});
    }
    if (shapes.empty())
        shapes = {{QLIN_FMT_FP8, 4096, 2048},
                  {QLIN_FMT_FP8_BLOCK, 2048, 6144},
                  {QLIN_FMT_FP8, 151936, 2048},
                  {QLIN_FMT_FP8, 12288, 2048},
                  {QLIN_FMT_INT8, 2048, 2048}};
    const std::vector<int64_t> buckets =
        quick ? std::vector<int64_t>{1, 16, 256} : std::vector<int64_t>{1, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048};
    int dev = 0;
    CK(cudaGetDevice(&dev));
    cudaDeviceProp prop;
    CK(cudaGetDeviceProperties(&prop, dev));
    qlin_dispatch_table_clear();
    cudaStream_t st;
    CK(cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking));
    const size_t l2 = (size_t)prop.l2CacheSize;

    FILE* out = std::fopen(out_path, "w");
    if (!out) return 1;
    std::fprintf(out, "qlin-dispatch 1\n");
    std::fprintf(out, "device %d %d %d %s\n", prop.multiProcessorCount, prop.major, prop.minor, prop.name);
    std::fprintf(out, "# written by qlin_sweep; per bucket: fmt N K m_max variant tile_n k_segments\n");

    for (const Shape& s : shapes) {
        const int64_t M_max = buckets.back();
        Problem P;
        P.s = s;
        const bool bsf = block_scaled(s.fmt);
        const size_t wbytes = (size_t)s.N * (size_t)row_bytes(s.fmt, s.K);
        const size_t abytes = (size_t)M_max * (size_t)row_bytes(s.fmt, s.K);
        const size_t ncopy = quick ? 2 : std::max<size_t>(2, (2 * l2 + wbytes - 1) / wbytes + 1);
        const size_t sw_elems = s.fmt == QLIN_FMT_FP8_BLOCK ? (size_t)((s.N + 127) / 128) * (s.K / 128) : (size_t)s.N;
        const size_t sa_elems = s.fmt == QLIN_FMT_FP8_BLOCK ? (size_t)M_max * (s.K / 128) : (size_t)M_max;
        // scale storage in bytes: fp32 scales, or the tiled block-scale bytes
        const size_t sa_bytes = bsf ? sf_bytes(s.fmt, M_max, s.K) : sa_elems * 4;
        const size_t sw_bytes = bsf ? sf_bytes(s.fmt, s.N, s.K) : sw_elems * 4;
        CK(cudaMalloc(&P.a_q, abytes));
        CK(cudaMalloc(&P.s_a, sa_bytes));
        if (s.fmt == QLIN_FMT_BF16)
            fill_bf16<<<1024, 256, 0, st>>>(static_cast<uint16_t*>(P.a_q), abytes / 2, 17u);
        else
            fill_codes<<<1024, 256, 0, st>>>(static_cast<uint8_t*>(P.a_q), abytes, 17u,
                                             s.fmt != QLIN_FMT_INT8 && s.fmt != QLIN_FMT_NVFP4);
        if (bsf) {
            fill_sf<<<256, 256, 0, st>>>(reinterpret_cast<uint8_t*>(P.s_a), sa_bytes, 5u, s.fmt == QLIN_FMT_MXFP8);
            const float g[2] = {1e-2f, 2e-3f};
            CK(cudaMalloc(&P.g, sizeof g));
            CK(cudaMemcpy(P.g, g, sizeof g, cudaMemcpyHostToDevice));
        } else {
            fill_scales<<<256, 256, 0, st>>>(P.s_a, sa_elems, 5u);
        }
        for (size_t i = 0; i < ncopy; ++i) {
            void* w;
            float* sw;
            CK(cudaMalloc(&w, wbytes));
            CK(cudaMalloc(&sw, sw_bytes));
            if (s.fmt == QLIN_FMT_BF16)
                fill_bf16<<<2048, 256, 0, st>>>(static_cast<uint16_t*>(w), wbytes / 2, 1000u + (uint32_t)i);
            else
                fill_codes<<<2048, 256, 0, st>>>(static_cast<uint8_t*>(w), wbytes, 1000u + (uint32_t)i,
                                                 s.fmt != QLIN_FMT_INT8 && s.fmt != QLIN_FMT_NVFP4);
            if (bsf)
                fill_sf<<<256, 256, 0, st>>>(reinterpret_cast<uint8_t*>(sw), sw_bytes, 77u + (uint32_t)i,
                                             s.fmt == QLIN_FMT_MXFP8);
            else
                fill_scales<<<256, 256, 0, st>>>(sw, sw_elems, 77u);
            P.w_q.push_back(w);
            P.s_w.push_back(sw);
        }
        CK(cudaMalloc(&P.c, (size_t)M_max * s.N * 2));
        CK(cudaMalloc(&P.c_ref, (size_t)M_max * s.N * 2));
        P.ws_bytes = 256u << 20;
        CK(cudaMalloc(&P.ws, P.ws_bytes));
        CK(cudaMemsetAsync(P.ws, 0, P.ws_bytes, st));
        CK(cudaStreamSynchronize(st));

        const std::vector<int> segs = segment_choices(s.fmt, s.K);
        // best[si][bi] = (time, cand)
        std::vector<std::vector<std::pair<float, Cand>>> best(segs.size(),
                                                              std::vector<std::pair<float, Cand>>(buckets.size()));
        for (size_t si = 0; si < segs.size(); ++si) {
            const int S = segs[si];
            for (size_t bi = 0; bi < buckets.size(); ++bi) {
                P.M = buckets[bi];
                const int iters =
                    quick ? 4 : std::max(4, std::min(40, (int)(40 * 64 / std::max<int64_t>(P.M, 64))));
                // reference output: plain tile 128 with this S (the canonical order)
                bool have_ref = run_gemm(P, QLIN_VAR_PLAIN, 128, S, 0, P.c_ref, 0, st) == QLIN_OK;
                CK(cudaStreamSynchronize(st));
                float bt = 1e30f;
                Cand bc{0, 0};
                for (const Cand& c : candidates(s.fmt, P.M)) {
                    if (S == 1 && (c.variant == QLIN_VAR_SPLITK || c.variant == QLIN_VAR_SWAPAB_SPLITK)) continue;
                    bool ok = false;
                    const float t = time_config(P, c.variant, c.tile_n, S, iters, quick ? 2 : 5, st, &ok);
                    if (!ok) continue;
                    const bool same = !have_ref || s.fmt == QLIN_FMT_INT8 || same_output(P, c.variant, c.tile_n, S, st);
                    std::printf("%s N=%lld K=%lld S=%d M=%lld %-14s tile=%3d  %9.2f us%s\n", fmt_name(s.fmt),
                                (long long)s.N, (long long)s.K, S, (long long)P.M, var_name(c.variant), c.tile_n, t,
                                same ? "" : "  (NOT bitwise equal: rejected)");
                    std::fflush(stdout);
                    if (same && t < bt) {
                        bt = t;
                        bc = c;
                    }
                }
                best[si][bi] = {bt, bc};
            }
        }
        // one segmentation per shape: smallest summed best time over the buckets
        size_t bs = 0;
        double bsum = 1e300;
        for (size_t si = 0; si < segs.size(); ++si) {
            double sum = 0;
            for (size_t bi = 0; bi < buckets.size(); ++bi) sum += best[si][bi].first;
            std::printf("%s N=%lld K=%lld: S=%d total %.2f us\n", fmt_name(s.fmt), (long long)s.N, (long long)s.K,
                        segs[si], sum);
            if (sum < bsum) {
                bsum = sum;
                bs = si;
            }
        }
        for (size_t bi = 0; bi < buckets.size(); ++bi) {
            const auto& b = best[bs][bi];
            if (b.second.variant == 0) continue;
            std::fprintf(out, "entry %s %lld %lld %lld %s %d %d   # %.2f us\n", fmt_name(s.fmt), (long long)s.N,
                         (long long)s.K, (long long)buckets[bi], var_name(b.second.variant), b.second.tile_n,
                         segs[bs], b.first);
        }
        std::fflush(out);
        cudaFree(P.a_q);
        cudaFree(P.s_a);
        if (P.g) cudaFree(P.g);
        for (auto p : P.w_q) cudaFree(p);
        for (auto p : P.s_w) cudaFree(p);
        cudaFree(P.c);
        cudaFree(P.c_ref);
        cudaFree(P.ws);
    }
    std::fclose(out);
    CK(cudaStreamDestroy(st));
    return 0;
}
