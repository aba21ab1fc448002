// hq_dense.cu -- dense-rotation KV variant: a caller-given orthogonal 128 x 128 matrix Q in place
// of the sign diagonal and Hadamard transform (Methodology step 4, "Bias Correction for KV Cache":
// the per-layer rotation may be a dense Haar-random orthogonal matrix instead of the sign
// diagonal).  Two kernels around the codec's lattice / Rice stages:
//
//   rotate    u = (Q x) / (s_hat beta) per head vector, s_hat the bf16 RMS (the codec's scale);
//             every u_j is the binary32 fma chain over i = 0 .. 127 of Q[j][i] x_i from 0, so the
//             lattice decisions that follow are those of the reference arithmetic bit for bit.
//             One register-tiled binary32 product Y = A B over K = 128 (A = x, B = Q^T): persistent
//             blocks keep B in shared memory (64 KB), stage 64 rows of A per step, and each of the
//             128 threads accumulates an 8 x 8 block of Y with k ascending (paired binary32 fma:
//             two independent fma per instruction, each rounded once); the next step's rows are
//             loaded into registers while the current step's FMAs run, two blocks per SM.  It stays
//             on the FP32 pipe: its outputs decide integer codes, and tensor-core accumulation
//             (order and internal precision unspecified) could not reproduce the reference chain.
//   unrotate  x_hat = (Q^T p) (s_hat beta) per head vector, p the decoded lattice point minus the
//             dither in u units.  Only a tolerance applies here, so it runs on the tensor cores
//             (tcgen05, fp16 two-term splits of p and Q, binary32 accumulation in TMEM).
#include <cuda_runtime.h>

#include <type_traits>

#include "../../include/hq.h"
#include "hq_common.cuh"
#include "hq_launch.h"
#include "hq_tc.cuh"

#include <cuda_fp16.h>

namespace hq {
namespace {

constexpr int kDN = 128;             // vector length (head dimension)
constexpr int kDBM = 64;             // rows staged per step
constexpr int kDThreads = 128;
constexpr int kDWarps = kDThreads / 32;
constexpr int kRW = kDBM / kDWarps;  // rows each warp stages per step
constexpr int kTR = kDBM / 8;        // rows per thread in the product (row groups of 8)
constexpr int kDLD = kDN + 4;        // padded row of the staged tile (floats)

struct DenseSmem {
    float B[kDN][kDN];   // B[k][c]
    float A[kDBM][kDLD];  // A[r][k]
    float rs[kDBM];       // per-row factor: forward 1 / (s_hat beta), inverse s_hat beta
};

// B into shared memory: forward B[k][c] = Q[c][k], inverse B[k][c] = Q[k][c]
template <bool FWD>
__device__ __forceinline__ void load_rotation(DenseSmem& sm, const float* Q)
{
#pragma unroll 16
    for (int idx = threadIdx.x; idx < kDN * kDN; idx += kDThreads) {
        const int k = idx / kDN, c = idx % kDN;
        sm.B[k][c] = FWD ? Q[c * kDN + k] : Q[k * kDN + c];
    }
}

// acc[i][0..3] += A[r_i][k] B[k][4 tx + 0..3], acc[i][4..7] += A[r_i][k] B[k][64 + 4 tx + 0..3] for
// k = 0 .. 127 in order; rows r_i = ty + 8 i.  Lane l of warp w: tx = 4 w + l % 4, ty = l / 4, so a
// warp reads 8 consecutive rows of A (row pitch 132 floats: 32 distinct banks) and 64 contiguous
// bytes of each half of B[k].
__device__ __forceinline__ void thread_tile(int tid, int& ty, int& tx)
{
    const int lane = tid & 31, warp = tid >> 5;
    tx = 4 * warp + (lane & 3);
    ty = lane >> 2;
}

__device__ __forceinline__ void product(const DenseSmem& sm, int ty, int tx, float (&acc)[kTR][8])
{
    // paired binary32 fma (two independent fma, each rounded once: the same values as scalar fma)
    float2 c[kTR][4];
#pragma unroll
    for (int i = 0; i < kTR; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) c[i][j] = make_float2(0.0f, 0.0f);
#pragma unroll 2
    for (int k = 0; k < kDN; k += 4) {
        float4 a[kTR];
#pragma unroll
        for (int i = 0; i < kTR; ++i) a[i] = *reinterpret_cast<const float4*>(&sm.A[ty + 8 * i][k]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const float4 b0 = *reinterpret_cast<const float4*>(&sm.B[k + kk][4 * tx]);
            const float4 b1 = *reinterpret_cast<const float4*>(&sm.B[k + kk][64 + 4 * tx]);
            const float2 bp[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w), make_float2(b1.x, b1.y),
                                  make_float2(b1.z, b1.w)};
#pragma unroll
            for (int i = 0; i < kTR; ++i) {
                const float av = kk == 0 ? a[i].x : (kk == 1 ? a[i].y : (kk == 2 ? a[i].z : a[i].w));
                const float2 a2 = make_float2(av, av);
#pragma unroll
                for (int j = 0; j < 4; ++j) c[i][j] = __ffma2_rn(a2, bp[j], c[i][j]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kTR; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc[i][2 * j] = c[i][j].x;
            acc[i][2 * j + 1] = c[i][j].y;
        }
}

// Rows of one step in registers: warp w holds rows kRW w .. kRW w + kRW - 1 of the step, lane l
// elements 4 l .. 4 l + 3 of each (bf16 kept packed).  The next step's rows are loaded before the
// current step's product, so the loads are in flight while the FMAs run.
template <bool BF16>
struct RowRegs {
    using T = typename std::conditional<BF16, uint2, float4>::type;
    T w[kRW];
};

template <bool BF16>
__device__ __forceinline__ void prefetch_rows(RowRegs<BF16>& rg, const void* base, int64_t r0, int64_t rows)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int rr = 0; rr < kRW; ++rr) {
        const int64_t gr = r0 + warp * kRW + rr;
        if constexpr (BF16) {
            rg.w[rr] = gr < rows ? *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + gr * kDN + 4 * lane)
                                 : make_uint2(0u, 0u);
        } else {
            rg.w[rr] = gr < rows ? *reinterpret_cast<const float4*>(static_cast<const float*>(base) + gr * kDN + 4 * lane)
                                 : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
    }
}

template <bool BF16>
__device__ __forceinline__ float4 row_value(const RowRegs<BF16>& rg, int rr)
{
    if constexpr (BF16) {
        const uint2 w = rg.w[rr];
        return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u), __uint_as_float(w.y << 16),
                           __uint_as_float(w.y & 0xFFFF0000u));
    } else {
        return rg.w[rr];
    }
}

// forward: x (bf16 or fp32) -> u fp32, scale bf16 bits; non-finite vectors counted in *nonfinite
template <bool BF16>
__global__ void __launch_bounds__(kDThreads, 2) rotate_kernel(const void* __restrict__ x, const float* __restrict__ Q,
                                                             float beta, int64_t rows, float* __restrict__ u,
                                                             uint16_t* __restrict__ scale, uint32_t* nonfinite)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    DenseSmem& sm = *reinterpret_cast<DenseSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int ty, tx;
    thread_tile(tid, ty, tx);
    const int64_t steps = (rows + kDBM - 1) / kDBM;
    RowRegs<BF16> rg;
    if ((int64_t)blockIdx.x < steps) prefetch_rows<BF16>(rg, x, (int64_t)blockIdx.x * kDBM, rows);
    load_rotation<true>(sm, Q);
    for (int64_t st = blockIdx.x; st < steps; st += gridDim.x) {
        const int64_t r0 = st * kDBM;
        // ---- stage the rows; RMS of each by the pairwise tree (q_i = x_i^2; q[i] += q[i + h] for
        // h = 1, 2 in-thread, then h = 4 .. 64 across lanes), the warp's trees interleaved
        constexpr int RW = kRW;
        float q[RW];
        uint32_t bad = 0u;  // bit rr: row rr holds a non-finite element
#pragma unroll
        for (int rr = 0; rr < RW; ++rr) {
            const float4 f = row_value<BF16>(rg, rr);
            q[rr] = __fadd_rn(__fadd_rn(__fmul_rn(f.x, f.x), __fmul_rn(f.y, f.y)),
                              __fadd_rn(__fmul_rn(f.z, f.z), __fmul_rn(f.w, f.w)));
            const bool fin = isfinite(f.x) && isfinite(f.y) && isfinite(f.z) && isfinite(f.w);
            bad |= (__all_sync(0xffffffffu, fin) ? 0u : 1u) << rr;
        }
#pragma unroll
        for (int m = 1; m < 32; m *= 2) {
#pragma unroll
            for (int rr = 0; rr < RW; ++rr) {
                const float o = __shfl_down_sync(0xffffffffu, q[rr], m);
                if ((lane & (2 * m - 1)) == 0) q[rr] = __fadd_rn(q[rr], o);
            }
        }
        // lane rr < RW finishes row rr: scale bits and 1 / (s_hat beta)
        float tot = 0.0f;
#pragma unroll
        for (int rr = 0; rr < RW; ++rr) {
            const float t = __shfl_sync(0xffffffffu, q[rr], 0);
            if (lane == rr) tot = t;
        }
        bool zero = false, nonfin = false;
        if (lane < RW) {
            const int rl = warp * RW + lane;
            const int64_t gr = r0 + rl;
            const bool all_fin = ((bad >> lane) & 1u) == 0u;
            const float s = all_fin ? __fsqrt_rn(__fmul_rn(tot, 1.0f / (float)kDN)) : 0.0f;
            uint16_t sb = f32_to_bf16_bits(s);
            const float sh = __uint_as_float((uint32_t)sb << 16);
            if (!all_fin || !isfinite(sh)) {
                sb = 0;
                zero = true;
                nonfin = gr < rows;
            } else if (sh < 1.2621774483536189e-29f) {  // 2^-96: coded as an all-zero tile
                sb = 0;
                zero = true;
            }
            sm.rs[rl] = zero ? 0.0f : __fdiv_rn(1.0f, __fmul_rn(sh, beta));
            if (gr < rows) scale[gr] = sb;
        }
        const uint32_t nf = __popc(__ballot_sync(0xffffffffu, nonfin));
        if (lane == 0 && nf) atomicAdd(nonfinite, nf);
        // rows coded as zeros are staged as zeros: their products are +0 exactly, and so is u
        const uint32_t zmask = __ballot_sync(0xffffffffu, zero);
#pragma unroll
        for (int rr = 0; rr < RW; ++rr) {
            const float4 f = ((zmask >> rr) & 1u) ? make_float4(0.0f, 0.0f, 0.0f, 0.0f) : row_value<BF16>(rg, rr);
            *reinterpret_cast<float4*>(&sm.A[warp * RW + rr][4 * lane]) = f;
        }
        __syncthreads();
        if (st + gridDim.x < steps) prefetch_rows<BF16>(rg, x, (st + gridDim.x) * kDBM, rows);
        float acc[kTR][8];
        product(sm, ty, tx, acc);
#pragma unroll
        for (int i = 0; i < kTR; ++i) {
            const int rl = ty + 8 * i;
            const int64_t gr = r0 + rl;
            if (gr >= rows) continue;
            const float g = sm.rs[rl];
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = __fmul_rn(acc[i][j], g);
            float* dst = u + gr * kDN;
            *reinterpret_cast<float4*>(dst + 4 * tx) = make_float4(v[0], v[1], v[2], v[3]);
            *reinterpret_cast<float4*>(dst + 64 + 4 * tx) = make_float4(v[4], v[5], v[6], v[7]);
        }
        __syncthreads();  // the staged rows are read: the next step may overwrite them
    }
}

// ------------------------------------------------------------------------------------------------
// inverse on the tensor cores: x_hat (bf16 or fp32) = (Q^T p) (s_hat beta).  Only a tolerance
// applies here (the codes are already decided), so the product runs as tcgen05.mma.kind::f16 on a
// two-term fp16 split of each operand: p = ph + pl, Q = qh + ql with ph = fp16(p),
// pl = fp16(p - ph) (22 significant bits in all), and D = ph qh + ph ql + pl qh accumulated in
// binary32 in TMEM (the dropped pl ql and the split's rounding are below 2^-22 of each product).
// One CTA of 128 threads per SM: the split Q^T (K-major, 128-byte swizzle) stays in shared
// memory; each 128-row tile of p arrives by TMA in binary32, every thread splits its row into the
// fp16 operand stage, one thread issues the 24 MMAs (M 128, N 128, K 16) into one of two TMEM
// accumulators, and while they run the threads read the previous tile's accumulator (one row per
// thread), scale it and store it.
// ------------------------------------------------------------------------------------------------
constexpr int kTM = 128;  // rows per tile
struct UnrotSmem {
    alignas(1024) unsigned char b[2][2][kTM * 128];   // split Q^T: [hi / lo][K half][row c: 64 fp16]
    alignas(1024) unsigned char a[2][2][kTM * 128];   // split p:   [hi / lo][K half][row m: 64 fp16]
    alignas(1024) unsigned char st[4][kTM * 128];     // p tile as loaded: [K quarter][row m: 32 fp32]
    alignas(8) uint64_t tma_bar;
    uint64_t mma_bar[2];
    uint32_t tmem_base;
};

// element k of row r in a K-major 128-byte-swizzled fp16 operand of two K halves: byte offset
__device__ __forceinline__ uint32_t f16_off(int r, int k) { return (uint32_t)((k >> 6) * (kTM * 128)) + swz(r, (k & 63) >> 3) + 2u * (uint32_t)(k & 7); }

__device__ __forceinline__ uint32_t split_pair(float x0, float x1, uint32_t& lo)
{
    const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
    const __half l0 = __float2half_rn(__fadd_rn(x0, -__half2float(h0)));
    const __half l1 = __float2half_rn(__fadd_rn(x1, -__half2float(h1)));
    lo = (uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1) << 16);
    return (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
}

constexpr uint32_t kIdescF16 = (1u << 4) | ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(kTM >> 4) << 24);  // f16 x f16 -> f32

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate)
{
    const uint32_t z = 0u;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(kIdescF16), "r"(accumulate), "r"(z), "r"(z), "r"(z), "r"(z)
        : "memory");
}

template <bool BF16>
__global__ void __launch_bounds__(kDThreads, 1) unrotate_tc_kernel(const __grid_constant__ CUtensorMap tP,
                                                                   const float* __restrict__ Q,
                                                                   const uint16_t* __restrict__ scale, float beta,
                                                                   int64_t rows, void* __restrict__ y, WsHeader* ws)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    UnrotSmem& sm = *reinterpret_cast<UnrotSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t tiles = (rows + kTM - 1) / kTM;
    if (tid == 0) {
        mbar_init(&sm.tma_bar, 1);
        mbar_init(&sm.mma_bar[0], 1);
        mbar_init(&sm.mma_bar[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&sm.tmem_base, 2 * 128);
    // split Q^T: operand row c holds Q[k][c], k = 0 .. 127 (thread c builds row c)
    {
        const int c = tid;
#pragma unroll 4
        for (int k = 0; k < 128; k += 2) {
            uint32_t lo;
            const uint32_t hi = split_pair(Q[k * 128 + c], Q[(k + 1) * 128 + c], lo);
            *reinterpret_cast<uint32_t*>(&sm.b[0][0][0] + f16_off(c, k)) = hi;
            *reinterpret_cast<uint32_t*>(&sm.b[1][0][0] + f16_off(c, k)) = lo;
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;
    const uint64_t bd0 = sw128_desc(&sm.b[0][0][0]), bd1 = sw128_desc(&sm.b[1][0][0]);
    const uint64_t ad0 = sw128_desc(&sm.a[0][0][0]), ad1 = sw128_desc(&sm.a[1][0][0]);
    constexpr uint64_t kHalf = (kTM * 128) >> 4;  // descriptor units of one K half

    auto issue_load = [&](int64_t tile) {
        mbar_arrive_expect_tx(&sm.tma_bar, 4u * kTM * 128u);
#pragma unroll
        for (int q = 0; q < 4; ++q) tma_load_2d(sm.st[q], &tP, 32 * q, (int)(tile * kTM), &sm.tma_bar);
    };
    // epilogue of one tile: accumulator slot s -> scaled row of y
    auto epilogue = [&](int64_t tile, int s, int i) -> bool {
        const bool got = mbar_wait(&sm.mma_bar[s], (uint32_t)((i >> 1) & 1));
        __syncwarp();
        if (!__all_sync(0xffffffffu, got)) return false;
        tc_fence_after();
        const int64_t r = tile * kTM + tid;
        const float h = r < rows ? __fmul_rn(__uint_as_float((uint32_t)scale[r] << 16), beta) : 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t v[32];
            tmem_ld32_nowait(tbase + ((uint32_t)(warp * 32) << 16) + (uint32_t)(s * 128 + 32 * c), v);
            tmem_wait_ld();
            if (r < rows) {
                if constexpr (BF16) {
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(y) + r * 128 + 32 * c);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(v[8 * q + 2 * e]), h),
                                                                            __fmul_rn(__uint_as_float(v[8 * q + 2 * e + 1]), h));
                            w[e] = *reinterpret_cast<const uint32_t*>(&b2);
                        }
                        dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                } else {
                    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(y) + r * 128 + 32 * c);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        dst[q] = make_float4(__fmul_rn(__uint_as_float(v[4 * q]), h), __fmul_rn(__uint_as_float(v[4 * q + 1]), h),
                                             __fmul_rn(__uint_as_float(v[4 * q + 2]), h), __fmul_rn(__uint_as_float(v[4 * q + 3]), h));
                }
            }
        }
        tc_fence_before();
        return true;
    };

    bool alive = true;
    if (tid == 0 && (int64_t)blockIdx.x < tiles) issue_load(blockIdx.x);
    int i = 0;
    int64_t prev = -1;
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++i) {
        const bool arrived = mbar_wait(&sm.tma_bar, (uint32_t)(i & 1));
        // the previous tile's MMAs read the operand stage: they must be complete before it is rewritten
        bool free = true;
        if (i > 0) free = mbar_wait(&sm.mma_bar[(i - 1) & 1], (uint32_t)(((i - 1) >> 1) & 1));
        if (__syncthreads_or(!(arrived && free))) {
            if (tid == 0) {
                status_set(ws, kStTimeout);
                if (!arrived) mbar_wait(&sm.tma_bar, (uint32_t)(i & 1));  // no copy may outlive the block
            }
            alive = false;
            break;
        }
        // split row tid of the tile into the fp16 operand stage
        {
            const int m = tid;
#pragma unroll 4
            for (int k = 0; k < 128; k += 4) {
                const float4 x = *reinterpret_cast<const float4*>(sm.st[k >> 5] + swz(m, (k & 31) >> 2));
                uint32_t l0, l1;
                const uint32_t h0 = split_pair(x.x, x.y, l0), h1 = split_pair(x.z, x.w, l1);
                *reinterpret_cast<uint2*>(&sm.a[0][0][0] + f16_off(m, k)) = make_uint2(h0, h1);
                *reinterpret_cast<uint2*>(&sm.a[1][0][0] + f16_off(m, k)) = make_uint2(l0, l1);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            const int64_t next = tile + gridDim.x;
            if (next < tiles) issue_load(next);  // the staging was read by every thread
            const int s = i & 1;
            const uint32_t d = tbase + (uint32_t)(s * 128);
            int n = 0;
            // D = ph qh + ph ql + pl qh, K in steps of 16 (32 bytes within a 128-byte swizzle row)
#pragma unroll
            for (int term = 0; term < 3; ++term) {
                const uint64_t ad = term == 2 ? ad1 : ad0, bd = term == 1 ? bd1 : bd0;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk, ++n) {
                    const uint64_t off = (uint64_t)(kk >> 2) * kHalf + (uint64_t)(2 * (kk & 3));
                    mma_f16(d, ad + off, bd + off, n > 0 ? 1u : 0u);
                }
            }
            mma_commit(&sm.mma_bar[s]);
        }
        if (prev >= 0 && !epilogue(prev, (i - 1) & 1, i - 1)) {
            if ((tid & 31) == 0) status_set(ws, kStTimeout);
        }
        prev = tile;
    }
    if (alive && prev >= 0 && !epilogue(prev, (i - 1) & 1, i - 1)) {
        if ((tid & 31) == 0) status_set(ws, kStTimeout);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, 2 * 128);
}

// the rotation's non-finite count into the workspace status (after the encode cleared it)
__global__ void merge_nonfinite(WsHeader* h, const uint32_t* nonfinite)
{
    const uint32_t c = *nonfinite;
    if (c) {
        atomicOr(&h->status, 1u << HQ_ERR_NONFINITE);
        atomicAdd(&h->nonfinite, c);
    }
}

template <typename K>
cudaError_t grid_for(K kernel, int64_t rows, int& grid)
{
    const int smem = (int)sizeof(DenseSmem);
    cudaError_t e = cudaFuncSetAttribute((const void*)kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, (const void*)kernel, kDThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t steps = (rows + kDBM - 1) / kDBM;
    int64_t g = (int64_t)per_sm * num_sms();
    grid = (int)(g < steps ? g : steps);
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_rotate(const void* x, bool bf16, const float* Q, float beta, int64_t rows, float* u,
                          uint16_t* scale, uint32_t* nonfinite, cudaStream_t st)
{
    int grid = 0;
    cudaError_t e;
    if (bf16) {
        if ((e = grid_for(rotate_kernel<true>, rows, grid)) != cudaSuccess) return e;
        rotate_kernel<true><<<grid, kDThreads, sizeof(DenseSmem), st>>>(x, Q, beta, rows, u, scale, nonfinite);
    } else {
        if ((e = grid_for(rotate_kernel<false>, rows, grid)) != cudaSuccess) return e;
        rotate_kernel<false><<<grid, kDThreads, sizeof(DenseSmem), st>>>(x, Q, beta, rows, u, scale, nonfinite);
    }
    return cudaGetLastError();
}

cudaError_t launch_unrotate(const float* p, const float* Q, const uint16_t* scale, float beta, int64_t rows, void* y,
                            bool bf16, void* ws, cudaStream_t st)
{
    CUtensorMap tp;
    if (!tensor_map_2d(&tp, p, rows, kDN, 4, kTM)) return cudaErrorInvalidValue;
    const int smem = (int)sizeof(UnrotSmem) + 1024;
    const int64_t tiles = (rows + kTM - 1) / kTM;
    const int grid = (int)(tiles < num_sms() ? tiles : num_sms());  // persistent: one CTA per SM
    cudaError_t e;
    if (bf16) {
        if ((e = cudaFuncSetAttribute(unrotate_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
            return e;
        unrotate_tc_kernel<true><<<grid, kDThreads, smem, st>>>(tp, Q, scale, beta, rows, y, static_cast<WsHeader*>(ws));
    } else {
        if ((e = cudaFuncSetAttribute(unrotate_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
            return e;
        unrotate_tc_kernel<false><<<grid, kDThreads, smem, st>>>(tp, Q, scale, beta, rows, y, static_cast<WsHeader*>(ws));
    }
    return cudaGetLastError();
}

cudaError_t launch_merge_nonfinite(void* ws, const uint32_t* nonfinite, cudaStream_t st)
{
    merge_nonfinite<<<1, 1, 0, st>>>(static_cast<WsHeader*>(ws), nonfinite);
    return cudaGetLastError();
}

}  // namespace hq
