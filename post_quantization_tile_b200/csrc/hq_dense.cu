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
// per step, and each of the 256 threads accumulates a 4 x 8 block of Y with k ascending.  Two
// blocks share an SM, so one block's staging overlaps the other's FMAs.  The product stays on the
// FP32 pipe: its outputs decide integer codes, and tensor-core accumulation (order and internal
// precision unspecified) could not reproduce the reference chain.
#include <cuda_runtime.h>

#include "../../include/hq.h"
#include "hq_common.cuh"
#include "hq_launch.h"

namespace hq {
namespace {

constexpr int kDN = 128;       // vector length (head dimension)
constexpr int kDBM = 64;       // rows staged per step
constexpr int kDThreads = 256;
constexpr int kDLD = kDN + 4;  // padded row of the staged tile (floats)

struct DenseSmem {
    float B[kDN][kDN];   // B[k][c]
    float A[kDBM][kDLD];  // A[r][k]
    float rs[kDBM];       // per-row factor: forward 1 / (s_hat beta), inverse s_hat beta
    int zr[kDBM];         // forward: the row is coded as zeros (zero or non-finite vector)
};

// 4 consecutive elements of a row as binary32
template <bool BF16>
__device__ __forceinline__ float4 load4(const void* base, int64_t row, int col)
{
    if constexpr (BF16) {
        const uint2 w = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + row * kDN + col);
        return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u), __uint_as_float(w.y << 16),
                           __uint_as_float(w.y & 0xFFFF0000u));
    } else {
        return *reinterpret_cast<const float4*>(static_cast<const float*>(base) + row * kDN + col);
    }
}

// B into shared memory: forward B[k][c] = Q[c][k], inverse B[k][c] = Q[k][c]
template <bool FWD>
__device__ __forceinline__ void load_rotation(DenseSmem& sm, const float* Q)
{
    for (int idx = threadIdx.x; idx < kDN * kDN; idx += kDThreads) {
        const int k = idx / kDN, c = idx % kDN;
        sm.B[k][c] = FWD ? Q[c * kDN + k] : Q[k * kDN + c];
    }
}

// acc[i][0..3] += A[r_i][k] B[k][c0 + 0..3], acc[i][4..7] += A[r_i][k] B[k][c0 + 64 + 0..3] for
// k = 0 .. 127 in order; rows r_i = 4 ty + i
__device__ __forceinline__ void product(const DenseSmem& sm, int ty, int tx, float (&acc)[4][8])
{
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
#pragma unroll 2
    for (int k = 0; k < kDN; k += 4) {
        float4 a[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(&sm.A[4 * ty + i][k]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const float4 b0 = *reinterpret_cast<const float4*>(&sm.B[k + kk][4 * tx]);
            const float4 b1 = *reinterpret_cast<const float4*>(&sm.B[k + kk][64 + 4 * tx]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float av = kk == 0 ? a[i].x : (kk == 1 ? a[i].y : (kk == 2 ? a[i].z : a[i].w));
                acc[i][0] = __fmaf_rn(av, b0.x, acc[i][0]);
                acc[i][1] = __fmaf_rn(av, b0.y, acc[i][1]);
                acc[i][2] = __fmaf_rn(av, b0.z, acc[i][2]);
                acc[i][3] = __fmaf_rn(av, b0.w, acc[i][3]);
                acc[i][4] = __fmaf_rn(av, b1.x, acc[i][4]);
                acc[i][5] = __fmaf_rn(av, b1.y, acc[i][5]);
                acc[i][6] = __fmaf_rn(av, b1.z, acc[i][6]);
                acc[i][7] = __fmaf_rn(av, b1.w, acc[i][7]);
            }
        }
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
    const int ty = tid / 16, tx = tid % 16;
    load_rotation<true>(sm, Q);
    const int64_t steps = (rows + kDBM - 1) / kDBM;
    for (int64_t st = blockIdx.x; st < steps; st += gridDim.x) {
        const int64_t r0 = st * kDBM;
        // ---- stage 8 rows per warp, lane l holding elements 4l .. 4l + 3; RMS by the pairwise tree
#pragma unroll 1
        for (int rr = 0; rr < kDBM / 8; ++rr) {
            const int rl = warp * (kDBM / 8) + rr;
            const int64_t gr = r0 + rl;
            float4 f = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (gr < rows) f = load4<BF16>(x, gr, 4 * lane);
            *reinterpret_cast<float4*>(&sm.A[rl][4 * lane]) = f;
            const bool fin = isfinite(f.x) && isfinite(f.y) && isfinite(f.z) && isfinite(f.w);
            const bool all_fin = __all_sync(0xffffffffu, fin);
            // q_i = x_i^2; q[i] += q[i + h] for h = 1, 2 in-thread, then h = 4 .. 64 across lanes
            float q = __fadd_rn(__fadd_rn(__fmul_rn(f.x, f.x), __fmul_rn(f.y, f.y)),
                                __fadd_rn(__fmul_rn(f.z, f.z), __fmul_rn(f.w, f.w)));
#pragma unroll
            for (int m = 1; m < 32; m *= 2) {
                const float o = __shfl_down_sync(0xffffffffu, q, m);
                if ((lane & (2 * m - 1)) == 0) q = __fadd_rn(q, o);
            }
            if (lane == 0) {
                const float s = all_fin ? __fsqrt_rn(__fmul_rn(q, 1.0f / (float)kDN)) : 0.0f;
                uint16_t sb = f32_to_bf16_bits(s);
                const float sh = __uint_as_float((uint32_t)sb << 16);
                int zero = 0;
                if (!all_fin || !isfinite(sh)) {
                    sb = 0;
                    zero = 1;
                    if (gr < rows) atomicAdd(nonfinite, 1u);
                } else if (sh < 1.2621774483536189e-29f) {  // 2^-96: coded as an all-zero tile
                    sb = 0;
                    zero = 1;
                }
                sm.zr[rl] = zero;
                sm.rs[rl] = zero ? 0.0f : __fdiv_rn(1.0f, __fmul_rn(sh, beta));
                if (gr < rows) scale[gr] = sb;
            }
        }
        __syncthreads();
        float acc[4][8];
        product(sm, ty, tx, acc);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int rl = 4 * ty + i;
            const int64_t gr = r0 + rl;
            if (gr >= rows) continue;
            const float g = sm.rs[rl];
            const bool z = sm.zr[rl] != 0;
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = z ? 0.0f : __fmul_rn(acc[i][j], g);
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
    const int ty = tid / 16, tx = tid % 16;
    load_rotation<false>(sm, Q);
    const int64_t steps = (rows + kDBM - 1) / kDBM;
    for (int64_t st = blockIdx.x; st < steps; st += gridDim.x) {
        const int64_t r0 = st * kDBM;
#pragma unroll 2
        for (int rr = 0; rr < kDBM / 8; ++rr) {
            const int rl = warp * (kDBM / 8) + rr;
            const int64_t gr = r0 + rl;
            float4 f = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (gr < rows) f = load4<false>(p, gr, 4 * lane);
            *reinterpret_cast<float4*>(&sm.A[rl][4 * lane]) = f;
            if (lane == 0) sm.rs[rl] = gr < rows ? __fmul_rn(__uint_as_float((uint32_t)scale[gr] << 16), beta) : 0.0f;
        }
        __syncthreads();
        float acc[4][8];
        product(sm, ty, tx, acc);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int rl = 4 * ty + i;
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
