// hq_dense.cu -- dense-rotation KV variant: a caller-given orthogonal 128 x 128 matrix Q in place
// of the sign diagonal and Hadamard transform (Methodology step 4, "Bias Correction for KV Cache":
// the per-layer rotation may be a dense Haar-random orthogonal matrix instead of the sign
// diagonal).  Two kernels around the codec's lattice / Rice stages:
//
//   rotate    u = (Q x) / (s_hat beta) per head vector, s_hat the bf16 RMS (the codec's scale);
//             every u_j is the binary32 fma chain over i = 0 .. 127 of Q[j][i] x_i from 0, so the
//             lattice decisions that follow are those of the reference arithmetic bit for bit.
//   unrotate  x_hat = (Q^T p) (s_hat beta) per head vector, p the decoded lattice point minus the
//             dither in u units.
//
// Both are one register-tiled binary32 product Y = A B over K = 128 (forward: A = x, B = Q^T;
// inverse: A = p, B = Q): persistent blocks keep B in shared memory (64 KB), stage 64 rows of A
// per step, and each of the 128 threads accumulates an 8 x 8 block of Y with k ascending (paired
// binary32 fma: two independent fma per instruction, each rounded once).  Eight rows per thread
// halve the shared-memory loads per fma against four, which kept shared memory busier than the
// FMA pipes.  The next step's rows are loaded into registers while the current step's FMAs run,
// and two blocks share an SM.  The product stays on the FP32 pipe: its outputs decide integer
// codes, and tensor-core accumulation (order and internal precision unspecified) could not
// reproduce the reference chain.
#include <cuda_runtime.h>

#include <type_traits>

#include "../../include/hq.h"
#include "hq_common.cuh"
#include "hq_launch.h"

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

// inverse: p fp32 -> x_hat (bf16 or fp32) = (Q^T p) (s_hat beta)
template <bool BF16>
__global__ void __launch_bounds__(kDThreads, 2) unrotate_kernel(const float* __restrict__ p, const float* __restrict__ Q,
                                                               const uint16_t* __restrict__ scale, float beta,
                                                               int64_t rows, void* __restrict__ y)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    DenseSmem& sm = *reinterpret_cast<DenseSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int ty, tx;
    thread_tile(tid, ty, tx);
    const int64_t steps = (rows + kDBM - 1) / kDBM;
    RowRegs<false> rg;
    if ((int64_t)blockIdx.x < steps) prefetch_rows<false>(rg, p, (int64_t)blockIdx.x * kDBM, rows);
    load_rotation<false>(sm, Q);
    for (int64_t st = blockIdx.x; st < steps; st += gridDim.x) {
        const int64_t r0 = st * kDBM;
#pragma unroll
        for (int rr = 0; rr < kRW; ++rr) {
            const int rl = warp * kRW + rr;
            *reinterpret_cast<float4*>(&sm.A[rl][4 * lane]) = rg.w[rr];
        }
        if (tid < kDBM) {
            const int64_t gr = r0 + tid;
            sm.rs[tid] = gr < rows ? __fmul_rn(__uint_as_float((uint32_t)scale[gr] << 16), beta) : 0.0f;
        }
        __syncthreads();
        if (st + gridDim.x < steps) prefetch_rows<false>(rg, p, (st + gridDim.x) * kDBM, rows);
        float acc[kTR][8];
        product(sm, ty, tx, acc);
#pragma unroll
        for (int i = 0; i < kTR; ++i) {
            const int rl = ty + 8 * i;
            const int64_t gr = r0 + rl;
            if (gr >= rows) continue;
            const float h = sm.rs[rl];
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = __fmul_rn(acc[i][j], h);
            if constexpr (BF16) {
                uint16_t* dst = static_cast<uint16_t*>(y) + gr * kDN;
                uint32_t w[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
                    w[q] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                *reinterpret_cast<uint2*>(dst + 4 * tx) = make_uint2(w[0], w[1]);
                *reinterpret_cast<uint2*>(dst + 64 + 4 * tx) = make_uint2(w[2], w[3]);
            } else {
                float* dst = static_cast<float*>(y) + gr * kDN;
                *reinterpret_cast<float4*>(dst + 4 * tx) = make_float4(v[0], v[1], v[2], v[3]);
                *reinterpret_cast<float4*>(dst + 64 + 4 * tx) = make_float4(v[4], v[5], v[6], v[7]);
            }
        }
        __syncthreads();
    }
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
                            bool bf16, cudaStream_t st)
{
    int grid = 0;
    cudaError_t e;
    if (bf16) {
        if ((e = grid_for(unrotate_kernel<true>, rows, grid)) != cudaSuccess) return e;
        unrotate_kernel<true><<<grid, kDThreads, sizeof(DenseSmem), st>>>(p, Q, scale, beta, rows, y);
    } else {
        if ((e = grid_for(unrotate_kernel<false>, rows, grid)) != cudaSuccess) return e;
        unrotate_kernel<false><<<grid, kDThreads, sizeof(DenseSmem), st>>>(p, Q, scale, beta, rows, y);
    }
    return cudaGetLastError();
}

cudaError_t launch_merge_nonfinite(void* ws, const uint32_t* nonfinite, cudaStream_t st)
{
    merge_nonfinite<<<1, 1, 0, st>>>(static_cast<WsHeader*>(ws), nonfinite);
    return cudaGetLastError();
}

}  // namespace hq
