// hq_gemm.cu -- int8 tensor-core GEMM over the weight's lattice codes with one binary32 scale per
// tile (tcgen05 MMA, TMEM accumulators, TMA operand loads).
//
// Y[m, r] = sa_m * sum_t g[t, r] S_{m,r,t},  S_{m,r,t} = sum_{j in group t} A[m, j] V[r, j]
// with A int8 [M, K] (activations after the same RHT as the weight), V int8 [N, K] (the weight's
// integer codes in the RHT domain) and g [K / 128, N] the per-tile scales.  The group sums are
// exact int32 MMA results; the scales are applied in binary32 as acc = fma(S, g, acc) over the
// groups in order, then y = acc * sa_m.  This is the int8 MMA path of the method (abstract: 8-bit
// tensor-core MMA paths, int8 ahead of fp8 on the post-RHT lattice output), with the group scale
// the decoder would otherwise apply.
//
// Persistent CTAs (one per SM) walk the 128 x GN tiles of Y (GN = 128 columns; 64 or 32 when the
// 128-wide tiles are too few to occupy the SMs, i.e. at small M): warp 0 streams 128 x 128-byte
// boxes of A, GN x 128-byte boxes of V and the group's GN scales into a ring with TMA (128-byte
// swizzle, the canonical K-major layout of the MMA); warp 1 issues four
// tcgen05.mma.kind::i8 (M 128, N GN, K 32) per group into one of 512 / GN TMEM accumulator slots
// of GN columns; the epilogue warps (warpgroups of 32 columns each) read each finished slot
// (tcgen05.ld), release it, convert the int32 sums and apply the group scales with paired binary32
// fma, so MMA and scaling overlap; a tile's result leaves through a staging buffer and TMA stores
// while the next tile's MMAs run.  Every wait is bounded: on a timeout the kernel records HQ_ERR_TIMEOUT and winds down.
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/hq.h"
#include "hq_common.cuh"
#include "hq_launch.h"
#include "hq_tc.cuh"

namespace hq {
namespace {

constexpr float kMagicGemm = 12582912.0f;  // 1.5 * 2^23
constexpr int kMagicBits = 0x4B400000;

constexpr int GM = 128, GK = 128;  // CTA tile rows and K group

// Tile width GN (128, 64 or 32 output columns): one epilogue warpgroup per 32 columns (a 128-wide
// tile has 16 epilogue warps; 256 columns were measured slower: 64 accumulators per epilogue
// thread exceed the register budget), the TMEM's 512 columns as 512 / GN accumulator slots.
template <int GN>
struct GemmCfg {
    static constexpr int STAGES = GN == 128 ? 4 : (GN == 64 ? 6 : 8);  // operand ring
    static constexpr int ACC = 512 / GN;
    static constexpr int OUT = GN;          // columns staged per output store
    static constexpr int EPI = GN / 8;      // epilogue warps: GN / 32 warpgroups of 32 columns
    static constexpr int THREADS = 64 + 32 * EPI;
    static constexpr uint32_t IDESC = idesc_i8(GM, GN);  // s8 x s8 -> s32, both K-major, M = GM, N = GN
};

template <int GN>
struct GemmSmem {
    using C = GemmCfg<GN>;
    alignas(1024) int8_t a[C::STAGES][GM * GK];
    alignas(1024) int8_t b[C::STAGES][GN * GK];
    alignas(1024) unsigned char out[C::OUT / 32][GM * 128];  // output staging: 32-column boxes
    alignas(16) float g[C::STAGES][GN];                     // the group's scales, loaded with the operands
    alignas(8) uint64_t full[C::STAGES];
    uint64_t empty[C::STAGES];
    uint64_t acc_full[C::ACC];
    uint64_t acc_empty[C::ACC];
    uint32_t tmem_base;
};

struct GemmArgs {
    int64_t M, N, K;
    const float* sa;
    const float* g;
    WsHeader* ws;
};

template <int GN>
__global__ void __launch_bounds__(GemmCfg<GN>::THREADS, 1)
    gemm_i8_grouped_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tB,
                           const __grid_constant__ CUtensorMap tY)
{
    using C = GemmCfg<GN>;
    constexpr int GSTAGES = C::STAGES, GACC = C::ACC, GOUT = C::OUT, GEPI = C::EPI;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    GemmSmem<GN>& sm =
        *reinterpret_cast<GemmSmem<GN>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = (int)(a.K / GK);
    const int NT = (int)(a.N / GN);  // N is a multiple of 128, so of GN
    const int tiles = (int)(a.M / GM) * NT;  // persistent: tiles blockIdx.x, + gridDim.x, ...

    if (threadIdx.x == 0) {
        for (int s = 0; s < GSTAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1 + GEPI);  // the MMAs' commit and every epilogue warp's read of g
        }
        for (int s = 0; s < GACC; ++s) {
            mbar_init(&sm.acc_full[s], 1);
            mbar_init(&sm.acc_empty[s], GEPI);  // one arrival per epilogue warp
        }
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&sm.tmem_base, GACC * GN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer: A, V boxes and the group's scales ----------------
        if (lane == 0) {
            int it = 0;
            bool alive = true;
            for (int tile = blockIdx.x; alive && tile < tiles; tile += gridDim.x) {
                const int m0 = (tile / NT) * GM, n0 = (tile % NT) * GN;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % GSTAGES;
                    if (it >= GSTAGES && !mbar_wait_sleep(&sm.empty[s], (uint32_t)((it / GSTAGES - 1) & 1))) {
                        status_set(a.ws, kStTimeout);
                        alive = false;
                        break;
                    }
                    // rows of V past N read as zeros (TMA fill); the scales of those columns stay unset
                    // and their results are clipped by the TMA store
                    const uint32_t gbytes = (uint32_t)(a.N - n0 < GN ? a.N - n0 : GN) * 4u;
                    mbar_arrive_expect_tx(&sm.full[s], (uint32_t)(GM * GK + GN * GK) + gbytes);
                    tma_load_2d(sm.a[s], &tA, kb * GK, m0, &sm.full[s]);
                    tma_load_2d(sm.b[s], &tB, kb * GK, n0, &sm.full[s]);
                    bulk_load_1d(sm.g[s], a.g + (int64_t)kb * a.N + n0, gbytes, &sm.full[s]);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int it = 0;
            bool alive = true;
            for (int tile = blockIdx.x; alive && tile < tiles; tile += gridDim.x) {
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % GSTAGES, slot = it % GACC;
                    if (it >= GACC && !mbar_wait_sleep(&sm.acc_empty[slot], (uint32_t)((it / GACC - 1) & 1))) {
                        status_set(a.ws, kStTimeout);
                        alive = false;
                        break;
                    }
                    if (!mbar_wait_sleep(&sm.full[s], (uint32_t)((it / GSTAGES) & 1))) {
                        status_set(a.ws, kStTimeout);
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(sm.a[s]), bd = sw128_desc(sm.b[s]);
#pragma unroll
                    for (int kk = 0; kk < GK / 32; ++kk)  // K 32 per MMA: the start address moves 32 bytes
                        mma_i8(tbase + (uint32_t)(slot * GN), ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk),
                               C::IDESC, kk > 0 ? 1u : 0u);
                    mma_commit(&sm.empty[s]);
                    mma_commit(&sm.acc_full[slot]);
                }
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: scale and accumulate each group, store each tile ----------------
        // warpgroup h (warps 2 + 4h .. 5 + 4h) takes columns HC h .. HC h + HC - 1 of each slot; a
        // warp reads the TMEM lane quarter warp % 4, one accumulator row per thread
        const int q = warp & 3;
        const int h = (warp - 2) >> 2;
        const int row = q * 32 + lane;
        constexpr int HC = GN / (GEPI / 4);  // columns per warpgroup
        static_assert(HC % 32 == 0, "TMEM loads take 32 columns");
        const float2 nm = make_float2(-kMagicGemm, -kMagicGemm);
        int it = 0;
        bool alive = true;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const int m0 = (tile / NT) * GM, n0 = (tile % NT) * GN;
            float2 acc[HC / 2];
#pragma unroll
            for (int c = 0; c < HC / 2; ++c) acc[c] = make_float2(0.0f, 0.0f);
            // after a timeout a warp keeps walking the loops without waiting, so that every
            // epilogue warp still reaches each named barrier below
            for (int kb = 0; kb < KB; ++kb, ++it) {
                if (!alive) continue;
                const int slot = it % GACC, s = it % GSTAGES;
                const bool got = mbar_wait_sleep(&sm.acc_full[slot], (uint32_t)((it / GACC) & 1));
                __syncwarp();  // the warp-wide TMEM loads below need the whole warp converged
                if (!__all_sync(0xffffffffu, got)) {
                    if (lane == 0) status_set(a.ws, kStTimeout);
                    alive = false;
                    continue;
                }
                tc_fence_after();
                // 32 columns at a time: load, then scale with the group's scales read from the stage
#pragma unroll
                for (int c = 0; c < HC / 32; ++c) {
                    uint32_t S[32];
                    const uint32_t ta = tbase + ((uint32_t)(q * 32) << 16) + (uint32_t)(slot * GN + h * HC + 32 * c);
                    tmem_ld32_nowait(ta, S);
                    tmem_wait_ld();
                    if (c == HC / 32 - 1) {  // the slot is read: release it before the arithmetic
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm.acc_empty[slot]);
                    }
                    const float4* gp = reinterpret_cast<const float4*>(&sm.g[s][h * HC + 32 * c]);
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 g4 = gp[c4];
                        // |S| < 2^22: adding 1.5 * 2^23 in the integer domain gives an exact float
                        const float2 f0 = __fadd2_rn(make_float2(__int_as_float((int)S[4 * c4] + kMagicBits),
                                                                 __int_as_float((int)S[4 * c4 + 1] + kMagicBits)), nm);
                        const float2 f1 = __fadd2_rn(make_float2(__int_as_float((int)S[4 * c4 + 2] + kMagicBits),
                                                                 __int_as_float((int)S[4 * c4 + 3] + kMagicBits)), nm);
                        acc[16 * c + 2 * c4] = __ffma2_rn(f0, make_float2(g4.x, g4.y), acc[16 * c + 2 * c4]);
                        acc[16 * c + 2 * c4 + 1] = __ffma2_rn(f1, make_float2(g4.z, g4.w), acc[16 * c + 2 * c4 + 1]);
                    }
                }
                // the stage's scales are read
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.empty[s]);
            }
            // ---------------- output: y = acc * sa through the swizzled staging boxes, TMA store ----------------
            // GOUT columns at a time; warpgroup h's columns HC h .. belong to part HC h / GOUT
            const float sa = a.sa[m0 + row];
#pragma unroll
            for (int part = 0; part < GN / GOUT; ++part) {
                if (threadIdx.x == 64) bulk_wait_read0();  // the previous store has read the staging
                named_sync(1, 32 * GEPI);
                if ((h * HC) / GOUT == part) {
#pragma unroll
                    for (int bb = 0; bb < HC / 32; ++bb)
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int b = (h * HC - part * GOUT) / 32 + bb;  // 32-column box of this part
                            const float2 p0 = acc[bb * 16 + 2 * j], p1 = acc[bb * 16 + 2 * j + 1];
                            *reinterpret_cast<float4*>(&sm.out[b][swz(row, j)]) = make_float4(
                                __fmul_rn(p0.x, sa), __fmul_rn(p0.y, sa), __fmul_rn(p1.x, sa), __fmul_rn(p1.y, sa));
                        }
                }
                fence_proxy_async();
                named_sync(1, 32 * GEPI);
                if (threadIdx.x == 64 && alive && n0 + part * GOUT < a.N) {  // no store starts past N
#pragma unroll
                    for (int b = 0; b < GOUT / 32; ++b)
                        tma_store_2d(&tY, n0 + part * GOUT + b * 32, m0, &sm.out[b][0]);
                    bulk_commit();
                }
            }
        }
        if (threadIdx.x == 64) bulk_wait0();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, GACC * GN);
}

template <int GN>
cudaError_t launch_gemm(const GemmArgs& a, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& ty,
                        cudaStream_t st)
{
    const size_t smem = sizeof(GemmSmem<GN>) + 1024;
    // set on every call: the attribute belongs to the current device's context
    cudaError_t e = cudaFuncSetAttribute(gemm_i8_grouped_kernel<GN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (a.M / GM) * (a.N / GN);
    const int grid = (int)(tiles < num_sms() ? tiles : num_sms());  // persistent: one CTA per SM
    gemm_i8_grouped_kernel<GN><<<grid, GemmCfg<GN>::THREADS, smem, st>>>(a, ta, tb, ty);
    return cudaGetLastError();
}

}  // namespace
}  // namespace hq

using namespace hq;

// tile width: 128 columns when the 128-wide tiles fill the SMs, else the widest of 64 / 32 whose
// tiles do (32 when none does); N is a multiple of 128, so every width divides it
static int gemm_tile_width(int64_t M, int64_t N)
{
    const int64_t sms = num_sms();
    for (int gn = 128; gn > 32; gn /= 2)
        if ((M / GM) * (N / gn) >= sms) return gn;
    return 32;
}

extern "C" hq_status_t hq_gemm_int8(const int8_t* A, const float* sa, int64_t M, const int8_t* V, const float* g,
                                    int64_t N, int64_t K, int32_t group, float* Y, void* ws, size_t ws_bytes,
                                    void* stream)
{
    if (!A || !sa || !V || !g || !Y || !ws) return HQ_ERR_ARG;
    if (group != GK) return HQ_ERR_UNSUPPORTED;
    if (M < GM || N < 128 || K < GK || M % GM || N % 128 || K % GK) return HQ_ERR_ARG;
    if (K > ((int64_t)1 << 20) || M > ((int64_t)1 << 31) || N > ((int64_t)1 << 31)) return HQ_ERR_UNSUPPORTED;
    if ((M / GM) * (N / 32) > ((int64_t)1 << 30)) return HQ_ERR_UNSUPPORTED;
    if (ws_bytes < sizeof(WsHeader)) return HQ_ERR_ARG;
    const uintptr_t al = reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(V) |
                         reinterpret_cast<uintptr_t>(Y) | reinterpret_cast<uintptr_t>(ws) |
                         reinterpret_cast<uintptr_t>(g) | reinterpret_cast<uintptr_t>(sa);
    if (al & 15u) return HQ_ERR_ARG;
    if (!device_of(A)) return HQ_ERR_ARG;
    const int gn = gemm_tile_width(M, N);
    CUtensorMap ta, tb, ty;
    if (!tensor_map_2d(&ta, A, M, K, 1, GM) || !tensor_map_2d(&tb, V, N, K, 1, gn) || !tensor_map_2d(&ty, Y, M, N, 4, GM))
        return HQ_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), st) != cudaSuccess) return HQ_ERR_CUDA;
    const GemmArgs a{M, N, K, sa, g, static_cast<WsHeader*>(ws)};
    const cudaError_t e = gn == 128 ? launch_gemm<128>(a, ta, tb, ty, st)
                                    : (gn == 64 ? launch_gemm<64>(a, ta, tb, ty, st) : launch_gemm<32>(a, ta, tb, ty, st));
    return e == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}
