// gemm_sm100.cu — the bf16 GEMM of gemm_sm100.cuh.  One CTA per 128 x 256 output tile: a
// TMA warp streams 64-wide K slabs of A and B through a 4-stage ring (128-byte swizzle), one
// thread issues tcgen05.mma M=128 N=256 K=16 into a 256-column TMEM accumulator, and four
// epilogue warps (thread = output row) apply alpha, beta and D and store bf16 into the output
// part the tile's columns belong to.  Either operand may be K-major or MN-major (the
// transpose stored); A's parts are picked per K slab (split along K) or per tile (along M).
// Every wait is bounded; on expiry the CTA records the site, drains and frees TMEM.
#include <cudaTypedefs.h>

#include "gemm_sm100.cuh"
#include "sm100.cuh"

namespace zgcm {
using namespace sm100;

namespace {

constexpr int BM = GEMM_BM, BN = GEMM_BN, BK = GEMM_BK;
constexpr int STAGES = 4;
constexpr uint32_t A_STAGE = BM * BK * 2;   // 16 KB
constexpr uint32_t B_STAGE = BN * BK * 2;   // 32 KB
constexpr uint32_t CHUNK = BK * 128;        // MN-major operand: one 64-wide chunk of a stage, 8 KB
constexpr int THREADS = 256;                // w0 TMA, w1 MMA + TMEM, w2-3 idle, w4-7 epilogue

struct GemmParams {
    CUtensorMap tm_a[GEMM_MAX_SEG];  // K-major part: box {64 (K), 128}; MN-major: box {64 (M), 64 (K)}
    CUtensorMap tm_b;                // [N, K]: box {64 (K), 256}; [K, N]: box {64 (N), 64 (K)}
    int a_start[GEMM_MAX_SEG];
    int a_nseg, a_split, a_mn;
    bf16* c[GEMM_MAX_SEG];
    int c_ld[GEMM_MAX_SEG];
    int c_start[GEMM_MAX_SEG];
    int c_nseg;
    const bf16* d;
    int M, N, K;
    float alpha, beta;
    int b_kn, upper;
    int* err;
};

enum { BAR_FULL = 0, BAR_EMPTY = STAGES, BAR_DONE = 2 * STAGES, NBAR = 2 * STAGES + 1 };

struct GemmSmem {
    alignas(1024) unsigned char A[STAGES][A_STAGE];
    alignas(1024) unsigned char B[STAGES][B_STAGE];
    uint64_t bar[NBAR];
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(GemmSmem) + 1024 <= 232448, "beyond the 227 KB of shared memory a CTA can have");

// the part holding position x of a split dimension (parts in ascending start order)
__device__ __forceinline__ int seg_of(const int* start, int nseg, int x) {
    int s = 0;
    while (s + 1 < nseg && x >= start[s + 1]) ++s;
    return s;
}

__global__ void __launch_bounds__(THREADS, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
    extern __shared__ unsigned char smem_raw[];
    GemmSmem& sm = *reinterpret_cast<GemmSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int* abort = &sm.abort;
    const int n0 = (int)blockIdx.x * BN, m0 = (int)blockIdx.y * BM;
    const int nk = (p.K + BK - 1) / BK;
    if (p.upper && n0 + BN <= m0) return;  // every column of the tile left of its first row

    if (tid == 0) {
        sm.abort = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.bar[BAR_FULL + s], 1);
            mbar_init(&sm.bar[BAR_EMPTY + s], 1);
        }
        mbar_init(&sm.bar[BAR_DONE], 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, BN);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        for (int s = 0; s < p.a_nseg; ++s) prefetch_tmap(&p.tm_a[s]);
        prefetch_tmap(&p.tm_b);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        // ================================================ TMA producer: the K slabs of A and B
        if (lane == 0) {
            const int mseg = p.a_split == 2 ? seg_of(p.a_start, p.a_nseg, m0) : 0;
            int issued = 0;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % STAGES, k0 = kb * BK;
                if (kb >= STAGES && !mbar_wait(&sm.bar[BAR_EMPTY + s], ((kb / STAGES) - 1) & 1, abort, 601)) break;
                mbar_expect_tx(&sm.bar[BAR_FULL + s], A_STAGE + B_STAGE);
                if (p.a_mn) {  // [K, M] part: two 64-column chunks of the tile's 128 rows
                    const int ml = m0 - p.a_start[mseg];
                    tma_load_2d(sm.A[s], &p.tm_a[mseg], &sm.bar[BAR_FULL + s], ml, k0);
                    tma_load_2d(sm.A[s] + CHUNK, &p.tm_a[mseg], &sm.bar[BAR_FULL + s], ml + 64, k0);
                } else {
                    const int ks = p.a_split == 1 ? seg_of(p.a_start, p.a_nseg, k0) : 0;
                    tma_load_2d(sm.A[s], &p.tm_a[ks], &sm.bar[BAR_FULL + s], k0 - p.a_start[ks], m0);
                }
                if (p.b_kn) {
                    for (int j = 0; j < BN / 64; ++j)
                        tma_load_2d(sm.B[s] + j * CHUNK, &p.tm_b, &sm.bar[BAR_FULL + s], n0 + 64 * j, k0);
                } else {
                    tma_load_2d(sm.B[s], &p.tm_b, &sm.bar[BAR_FULL + s], k0, n0);
                }
                issued = kb + 1;
            }
            // every copy issued lands before the CTA exits (matters after an abort)
            for (int kb = issued > STAGES ? issued - STAGES : 0; kb < issued; ++kb)
                mbar_wait_drain(&sm.bar[BAR_FULL + kb % STAGES], (kb / STAGES) & 1);
        }
    } else if (warp == 1) {
        // ================================================ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(BM, BN, p.b_kn != 0) | ((p.a_mn ? 1u : 0u) << 15);
            bool ok = true;
            for (int kb = 0; kb < nk && ok; ++kb) {
                const int s = kb % STAGES;
                if (!(ok = mbar_wait(&sm.bar[BAR_FULL + s], (kb / STAGES) & 1, abort, 602))) break;
                tc_fence_after();
                const uint32_t a0 = smem_u32(sm.A[s]), b0 = smem_u32(sm.B[s]);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    // K-major: 16 elements = 32 bytes along the swizzled row; MN-major: 16 K rows =
                    // 2 KB on, 64-wide chunks 8 KB apart
                    const uint64_t ad = p.a_mn ? sdesc_sw128(a0 + kk * 16 * 128, CHUNK, 1024)
                                               : sdesc_sw128(a0 + kk * 32, 16, 1024);
                    const uint64_t bd = p.b_kn ? sdesc_sw128(b0 + kk * 16 * 128, CHUNK, 1024)
                                               : sdesc_sw128(b0 + kk * 32, 16, 1024);
                    mma_ss(tmem, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&sm.bar[BAR_EMPTY + s]);  // the stage is free once these products are done
            }
            // every MMA issued completes before TMEM is read or released
            mma_commit(&sm.bar[BAR_DONE]);
            if (!mbar_wait(&sm.bar[BAR_DONE], 0, abort, 603)) mbar_wait_drain(&sm.bar[BAR_DONE], 0);
        }
    } else if (warp >= 4) {
        // ================================================ epilogue: thread = output row m0 + r
        const int wq = warp - 4, r = 32 * wq + lane, row = m0 + r;
        const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
        const int cs = seg_of(p.c_start, p.c_nseg, n0);  // the tile's columns lie in one part
        bf16* cbase = p.c[cs] + (size_t)row * p.c_ld[cs] - p.c_start[cs];
        const bool got = mbar_wait(&sm.bar[BAR_DONE], 0, abort, 604);
        if (__all_sync(0xffffffffu, got)) {  // tcgen05.ld is warp-collective: one decision per warp
            tc_fence_after();
            for (int c = 0; c < BN / 32; ++c) {
                float v[32];
                tmem_ld32f(tmem + lane_off + 32 * c, v);
                tmem_wait_ld();
                if (row >= p.M) continue;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int col = n0 + 32 * c + 8 * q;  // N is a multiple of 8: whole chunks
                    if (col >= p.N) break;
                    float dv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    if (p.d) {
                        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p.d + (size_t)row * p.N + col));
                        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = unpack_bf16(w[e]);
                            dv[2 * e] = f.x;
                            dv[2 * e + 1] = f.y;
                        }
                    }
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        o[e] = pack_bf16(fmaf(p.alpha, v[8 * q + 2 * e], p.beta * dv[2 * e]),
                                         fmaf(p.alpha, v[8 * q + 2 * e + 1], p.beta * dv[2 * e + 1]));
                    *reinterpret_cast<uint4*>(cbase + col) = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
        }
    }

    // ------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, BN);
    if (tid == 0 && sm.abort && p.err) atomicExch(p.err, sm.abort);
}

// C[r][c] = C[c][r] for every c < r of a symmetric p x p matrix whose upper triangle (and
// diagonal) is computed: 32 x 32 tiles of the lower triangle through shared memory.
__global__ void __launch_bounds__(256) gemm_mirror_kernel(bf16* __restrict__ C, int n) {
    __shared__ bf16 tile[32][34];
    const int bx = (int)blockIdx.x, by = (int)blockIdx.y;  // destination tile: rows by*32, columns bx*32
    if (bx > by) return;
    for (int y = threadIdx.y; y < 32; y += 8) {  // source: rows bx*32.., columns by*32..
        const int r = bx * 32 + y, c = by * 32 + threadIdx.x;
        if (r < n && c < n) tile[y][threadIdx.x] = C[(size_t)r * n + c];
    }
    __syncthreads();
    for (int y = threadIdx.y; y < 32; y += 8) {
        const int r = by * 32 + y, c = bx * 32 + threadIdx.x;
        if (r < n && c < r) C[(size_t)r * n + c] = tile[threadIdx.x][y];
    }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 2-D bf16 map of a row-major [rows, cols] tensor, box {64 columns, box_rows rows}, 128-byte swizzle
bool make_map(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
    auto enc = get_encode();
    if (!enc || !base || rows < 1 || cols < 8 || cols % 8 != 0) return false;
    if (reinterpret_cast<uintptr_t>(base) & 15u) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

cudaError_t launch_gemm(const GemmDesc& g, int* err_word, cudaStream_t stream) {
    if (g.M < 1 || g.N < 8 || g.K < 1 || g.N % 8 != 0) return cudaErrorInvalidValue;
    // K is a contiguous dimension (16-byte row strides) unless both operands store it as rows
    if ((!g.a_mn || !g.b_kn) && g.K % 8 != 0) return cudaErrorInvalidValue;
    if (g.a_nseg < 1 || g.a_nseg > GEMM_MAX_SEG || g.c_nseg < 1 || g.c_nseg > GEMM_MAX_SEG) return cudaErrorInvalidValue;
    if ((g.a_split == 1 && g.a_mn) || (g.a_split == 2 && !g.a_mn) || g.a_split < 0 || g.a_split > 2 ||
        (g.a_split == 0 && g.a_nseg != 1))
        return cudaErrorInvalidValue;
    if ((g.upper || g.d) && (g.c_nseg != 1 || (g.upper && (g.M != g.N || g.c_ld[0] != g.N))))
        return cudaErrorInvalidValue;
    GemmParams p;
    p.a_nseg = g.a_nseg;
    p.a_split = g.a_split;
    p.a_mn = g.a_mn;
    for (int s = 0; s < g.a_nseg; ++s) {
        const GemmSeg& a = g.a[s];
        const int align = g.a_split == 1 ? BK : BM;  // a part never straddles a slab or a tile
        if (g.a_split && (a.start % align != 0 || (s == 0 && a.start != 0) || (s > 0 && a.start <= g.a[s - 1].start)))
            return cudaErrorInvalidValue;
        p.a_start[s] = a.start;
        if (!make_map(&p.tm_a[s], a.ptr, a.rows, a.cols, g.a_mn ? BK : BM)) return cudaErrorInvalidValue;
    }
    if (g.b_kn ? !make_map(&p.tm_b, g.b, g.K, g.N, BK) : !make_map(&p.tm_b, g.b, g.N, g.K, BN))
        return cudaErrorInvalidValue;
    p.c_nseg = g.c_nseg;
    for (int s = 0; s < g.c_nseg; ++s) {
        if (!g.c[s] || !aligned16(g.c[s]) || g.c_ld[s] % 8 != 0 || g.c_start[s] % BN != 0 ||
            (s == 0 && g.c_start[s] != 0) || (s > 0 && g.c_start[s] <= g.c_start[s - 1]))
            return cudaErrorInvalidValue;
        p.c[s] = static_cast<bf16*>(g.c[s]);
        p.c_ld[s] = g.c_ld[s];
        p.c_start[s] = g.c_start[s];
    }
    if (g.d && !aligned16(g.d)) return cudaErrorInvalidValue;
    p.d = static_cast<const bf16*>(g.d);
    p.M = g.M;
    p.N = g.N;
    p.K = g.K;
    p.alpha = g.alpha;
    p.beta = g.d ? g.beta : 0.0f;
    p.b_kn = g.b_kn ? 1 : 0;
    p.upper = g.upper ? 1 : 0;
    p.err = err_word;
    const size_t smem = sizeof(GemmSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((g.N + BN - 1) / BN, (g.M + BM - 1) / BM);
    gemm_kernel<<<grid, THREADS, smem, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess || !g.upper) return e;
    gemm_mirror_kernel<<<dim3((g.M + 31) / 32, (g.M + 31) / 32), dim3(32, 8), 0, stream>>>(p.c[0], g.M);
    return cudaGetLastError();
}

}  // namespace zgcm
