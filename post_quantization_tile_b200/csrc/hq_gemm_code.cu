// hq_gemm_code.cu -- the grouped int8 tensor-core GEMM with the decode of the weight's code fused
// into its producer warps: the weight's int8 lattice codes never exist outside shared memory.
//
// Y[m, r] = sa_m * sum_t g[t, r] S_{m,r,t},  S_{m,r,t} = sum_{j in group t} A[m, j] V[r, j], exactly
// the product of hq_decode_int8 followed by hq_gemm_int8 (same codes, same zeroed tiles, same
// binary32 order acc = fma(S, g, acc) over the groups from 0, then y = acc * sa_m).
//
// One CTA per SM walks work units (activation tile of 128 rows, weight tile of 128 rows = one
// encoder item of one tile column per K group, a range of K groups):
//   warp 0       TMA loads of the activation boxes (rows past M read as zeros);
//   warp 1       tcgen05.mma.kind::i8 (M 128, N 128, K 32) x 4 per group into one of four TMEM slots;
//   warps 2-9    epilogue: TMEM loads, int32 -> binary32, fma with the group scales, output;
//   warps 10-17  two decoder groups of 128 threads, alternating K groups: a bulk copy of the item's
//                words, per-chunk scans of the tile lengths, then one thread per weight row reads
//                its tile's Rice codes from both ends, unstrips each lattice block and writes the
//                int8 codes straight into the MMA's K-major 128-byte-swizzled operand stage, and the
//                tile's group scale next to it.
// At small M the weight's 128-row tiles alone give too few units to occupy every SM, so the K
// groups are split into ranges; the range s of an output tile continues the binary32 chain of
// range s - 1 (published through the workspace with a flag), which keeps the result bit-exact.
// Units are ordered range-major and every CTA takes its units in increasing order, so a unit's
// predecessor is always on an earlier position of a resident CTA.  Every wait is bounded: on a
// timeout the kernel records HQ_ERR_TIMEOUT and winds down.
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/hq.h"
#include "hq_common.cuh"
#include "hq_launch.h"
#include "hq_lattice.cuh"
#include "hq_tc.cuh"

namespace hq {
namespace {

constexpr int FM = 128, FN = 128, FK = 128;  // activation rows, weight rows per tile; K group = code tile
constexpr int FST = 3;                        // operand stages
constexpr int FACC = 4;                       // TMEM accumulator slots of FN columns
constexpr int FEPI = 8;                       // epilogue warps: two warpgroups of 64 columns
constexpr int FDEC = 2;                       // decoder groups of 128 threads
constexpr int FHC = FN / (FEPI / 4);          // columns per epilogue warpgroup
constexpr int FOUT = 64;                      // output columns staged per store
constexpr int FTHREADS = 64 + 32 * FEPI + 128 * FDEC;
constexpr int FDEC0 = 64 + 32 * FEPI;         // first decoder thread
constexpr int F_LMAX = FK / 8 + 12 * FK + 2 * FK;  // bits of a tile the input buffer takes (k <= 11)
constexpr int F_GUARD = 4;
constexpr int F_IN_WORDS = (FN * ((F_LMAX + 31) / 32) + 4 + 8 + 2 * F_GUARD + 3) / 4 * 4;
constexpr uint32_t kIdescF = idesc_i8(FM, FN);
constexpr float kMagicF = 12582912.0f;  // 1.5 * 2^23
constexpr int kMagicBitsF = 0x4B400000;

struct FusedSmem {
    alignas(1024) int8_t a[FST][FM * FK];
    alignas(1024) int8_t v[FST][FN * FK];
    alignas(1024) unsigned char out[FOUT / 32][FM * 128];
    alignas(16) uint32_t in[FDEC][F_IN_WORDS];
    alignas(16) float g[FST][FN];
    uint32_t Ls[FDEC][FN];
    uint32_t chunkbase[FDEC][FN / 32 + 1];
    int32_t in_ok[FDEC];
    alignas(8) uint64_t full[FST];
    uint64_t empty[FST];
    uint64_t acc_full[FACC];
    uint64_t acc_empty[FACC];
    uint64_t in_bar[FDEC];
    uint32_t tmem_base;
};

struct FusedArgs {
    int64_t M, N, K;            // activation rows, weight rows, inner dimension
    int64_t KB, MT, NT, S, KS;  // K groups, activation tiles, weight tiles, K ranges, groups per range
    int64_t units;
    float beta;
    const float* sa;
    const uint16_t* scale;
    const uint16_t* meta;
    const uint32_t* chunk_word;
    const uint32_t* bits;
    int64_t cap_words, RB, IB;
    WsHeader* ws;
    uint32_t* flags;            // per output tile: K ranges finished
    float* partial;             // per output tile: 128 x 128 binary32 chain, between ranges
};

struct Unit {
    int64_t mt, nt, s;
};

__device__ __forceinline__ Unit unit_of(const FusedArgs& a, int64_t u)
{
    const int64_t per = a.MT * a.NT;
    Unit w;
    w.s = u / per;
    const int64_t t = u % per;
    w.mt = t / a.NT;
    w.nt = t % a.NT;
    return w;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// 8 lattice codes as int8 bytes into two words; `out` collects codes outside [-127, 127]
__device__ __forceinline__ uint2 pack8(const int32_t (&v)[8], uint32_t& out)
{
    uint32_t w0 = 0, w1 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        out |= (uint32_t)(v[i] + 127) > 254u ? 1u : 0u;
        out |= (uint32_t)(v[4 + i] + 127) > 254u ? 1u : 0u;
        w0 |= ((uint32_t)v[i] & 0xFFu) << (8 * i);
        w1 |= ((uint32_t)v[4 + i] & 0xFFu) << (8 * i);
    }
    return make_uint2(w0, w1);
}

// zig-zag symbols of one block of eight coefficients -> integer lattice codes (E8 doubled)
template <int LAT>
__device__ __forceinline__ void unstrip8(const uint32_t (&z)[8], uint32_t cbit, int32_t (&v)[8])
{
    int32_t sym[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) sym[j] = unzigzag(z[j]);
    constexpr int D = Lat<LAT>::d;
#pragma unroll
    for (int b = 0; b < 8 / D; ++b) unstrip_block<LAT>(sym + b * D, cbit, v + b * D);
}

// One decoder thread: weight row `row` of the item (tile column jt, rows nt*128 ..), its tile's
// Rice codes from both ends into the stage's row `row`; returns the tile's group scale.
template <int LAT>
__device__ __forceinline__ float decode_row(const FusedArgs& a, FusedSmem& sm, int d, int st, int row, int64_t jt,
                                            int64_t nt, bool stage_ok)
{
    constexpr int COSB = LAT == HQ_E8 ? FK / 8 : 0;
    const int64_t r = nt * FN + row;
    const int64_t t = jt * a.N + r;
    const uint32_t mt = a.meta[t];
    const uint16_t sbits = a.scale[t];
    const int k = (int)(mt & 15u);
    const uint32_t L = (uint32_t)COSB + (uint32_t)FK * (uint32_t)(k + 1) + (mt >> 4);
    const int ch = row / kChunkTiles;
    // the tile's first bit: its chunk's word, then the lengths of the chunk's earlier tiles
    uint32_t before = 0;
    for (int i = ch * kChunkTiles; i < row; ++i) before += sm.Ls[d][i];
    const int tile0 = (int)(sm.chunkbase[d][ch] * 32u + before);
    const uint32_t* in = sm.in[d];
    int8_t* vrow = sm.v[st];
    bool ok = stage_ok;
    uint32_t out8 = 0;
    if (ok) {
        uint32_t cosbits = 0;
        if constexpr (LAT == HQ_E8) {
            const int cw = min(max(tile0 >> 5, 0), F_IN_WORDS - 2);
            const unsigned long long two = ((unsigned long long)in[cw + 1] << 32) | in[cw];
            cosbits = (uint32_t)(two >> (tile0 & 31)) & 0xFFFFu;
        }
        const uint32_t pow2k = 1u << k, sq_meta = mt >> 4;
        BitReader<true> rf;
        BitReader<false> rb;
        rf.begin(in, tile0 + COSB, F_IN_WORDS - 1);
        rb.begin(in, tile0 + (int)L - 1, F_IN_WORDS - 1);
#pragma unroll 1
        for (int g = 0; g < FK / 16; ++g) {
            uint32_t zf[8], zb[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if ((j & 3) == 0) {
                    rf.refill();
                    rb.refill();
                }
                zf[j] = get_code<true>(rf, k, pow2k, sq_meta, ok);
                zb[7 - j] = get_code<false>(rb, k, pow2k, sq_meta, ok);
            }
            int32_t vf[8], vb[8];
            const int bf = g, bb = FK / 8 - 1 - g;  // the forward block g, the backward block 15 - g
            unstrip8<LAT>(zf, (cosbits >> bf) & 1u, vf);
            unstrip8<LAT>(zb, (cosbits >> bb) & 1u, vb);
            *reinterpret_cast<uint2*>(vrow + swz(row, bf >> 1) + 8 * (bf & 1)) = pack8(vf, out8);
            *reinterpret_cast<uint2*>(vrow + swz(row, bb >> 1) + 8 * (bb & 1)) = pack8(vb, out8);
        }
        const uint32_t sq = (uint32_t)(rf.consumed() + rb.consumed() - FK * (k + 1));
        if (sq != sq_meta) ok = false;
    }
    if (!ok) status_set(a.ws, kStCorrupt);
    else if (out8) status_set(a.ws, kStRange);
    if (!ok || out8) {
        // a corrupt tile, or a code outside int8: the tile's codes are zero (as hq_decode_int8)
#pragma unroll
        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(vrow + swz(row, c)) = make_uint4(0u, 0u, 0u, 0u);
    }
    const float sh = __uint_as_float((uint32_t)sbits << 16);
    float gs = __fmul_rn(__fmul_rn(sh, a.beta), __uint_as_float(0x3DB504F3u));  // c_128 = RN(2^-3.5)
    if constexpr (LAT == HQ_E8) gs = __fmul_rn(gs, 0.5f);
    return gs;
}

template <int LAT>
__global__ void __launch_bounds__(FTHREADS, 1)
    gemm_code_kernel(const FusedArgs a, const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tY)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    FusedSmem& sm = *reinterpret_cast<FusedSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < FST; ++s) {
            mbar_init(&sm.full[s], 2);             // the activation box's TMA and the decoder group
            mbar_init(&sm.empty[s], 1 + FEPI);     // the MMAs' commit and every epilogue warp's read of g
        }
        for (int s = 0; s < FACC; ++s) {
            mbar_init(&sm.acc_full[s], 1);
            mbar_init(&sm.acc_empty[s], FEPI);
        }
        for (int d = 0; d < FDEC; ++d) mbar_init(&sm.in_bar[d], 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&sm.tmem_base, FACC * FN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer: activation boxes ----------------
        if (lane == 0) {
            int it = 0;
            bool alive = true;
            for (int64_t u = blockIdx.x; alive && u < a.units; u += gridDim.x) {
                const Unit w = unit_of(a, u);
                for (int64_t kb = w.s * a.KS; kb < (w.s + 1) * a.KS; ++kb, ++it) {
                    const int s = it % FST;
                    if (it >= FST && !mbar_wait_sleep(&sm.empty[s], (uint32_t)((it / FST - 1) & 1))) {
                        status_set(a.ws, kStTimeout);
                        alive = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.full[s], (uint32_t)(FM * FK));
                    tma_load_2d(sm.a[s], &tA, (int)(kb * FK), (int)(w.mt * FM), &sm.full[s]);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int it = 0;
            bool alive = true;
            for (int64_t u = blockIdx.x; alive && u < a.units; u += gridDim.x) {
                for (int64_t kb = 0; kb < a.KS; ++kb, ++it) {
                    const int s = it % FST, slot = it % FACC;
                    if (it >= FACC && !mbar_wait_sleep(&sm.acc_empty[slot], (uint32_t)((it / FACC - 1) & 1))) {
                        status_set(a.ws, kStTimeout);
                        alive = false;
                        break;
                    }
                    if (!mbar_wait_sleep(&sm.full[s], (uint32_t)((it / FST) & 1))) {
                        status_set(a.ws, kStTimeout);
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(sm.a[s]), bd = sw128_desc(sm.v[s]);
#pragma unroll
                    for (int kk = 0; kk < FK / 32; ++kk)
                        mma_i8(tbase + (uint32_t)(slot * FN), ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), kIdescF,
                               kk > 0 ? 1u : 0u);
                    mma_commit(&sm.empty[s]);
                    mma_commit(&sm.acc_full[slot]);
                }
            }
        }
        __syncwarp();
    } else if (threadIdx.x < FDEC0) {
        // ---------------- epilogue ----------------
        const int q = warp & 3;
        const int h = (warp - 2) >> 2;
        const int row = q * 32 + lane;
        const float2 nm = make_float2(-kMagicF, -kMagicF);
        int it = 0;
        bool alive = true;
        for (int64_t u = blockIdx.x; u < a.units; u += gridDim.x) {
            const Unit w = unit_of(a, u);
            const int64_t tile = w.mt * a.NT + w.nt;
            float2 acc[FHC / 2];
#pragma unroll
            for (int c = 0; c < FHC / 2; ++c) acc[c] = make_float2(0.0f, 0.0f);
            if (w.s > 0) {
                // continue the chain of the previous K range of this output tile
                if (threadIdx.x == 64) {
                    uint32_t spins = 0;
                    while (ld_acquire_u32(a.flags + tile) < (uint32_t)w.s) {
                        if (++spins > kSpinLimit) {
                            status_set(a.ws, kStTimeout);
                            break;
                        }
                        __nanosleep(128);
                    }
                }
                named_sync(1, 32 * FEPI);
                asm volatile("fence.acq_rel.gpu;" ::: "memory");
                const float4* src = reinterpret_cast<const float4*>(a.partial + tile * (int64_t)(FM * FN) +
                                                                    (int64_t)row * FN + h * FHC);
#pragma unroll
                for (int c = 0; c < FHC / 4; ++c) {
                    const float4 p = src[c];
                    acc[2 * c] = make_float2(p.x, p.y);
                    acc[2 * c + 1] = make_float2(p.z, p.w);
                }
            }
            for (int64_t kb = 0; kb < a.KS; ++kb, ++it) {
                if (!alive) continue;
                const int slot = it % FACC, s = it % FST;
                const bool got = mbar_wait_sleep(&sm.acc_full[slot], (uint32_t)((it / FACC) & 1));
                __syncwarp();
                if (!__all_sync(0xffffffffu, got)) {
                    if (lane == 0) status_set(a.ws, kStTimeout);
                    alive = false;
                    continue;
                }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < FHC / 32; ++c) {
                    uint32_t S[32];
                    const uint32_t ta = tbase + ((uint32_t)(q * 32) << 16) + (uint32_t)(slot * FN + h * FHC + 32 * c);
                    tmem_ld32_nowait(ta, S);
                    tmem_wait_ld();
                    if (c == FHC / 32 - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm.acc_empty[slot]);
                    }
                    const float4* gp = reinterpret_cast<const float4*>(&sm.g[s][h * FHC + 32 * c]);
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 g4 = gp[c4];
                        // |S| < 2^22: adding 1.5 * 2^23 in the integer domain gives an exact float
                        const float2 f0 = __fadd2_rn(make_float2(__int_as_float((int)S[4 * c4] + kMagicBitsF),
                                                                 __int_as_float((int)S[4 * c4 + 1] + kMagicBitsF)), nm);
                        const float2 f1 = __fadd2_rn(make_float2(__int_as_float((int)S[4 * c4 + 2] + kMagicBitsF),
                                                                 __int_as_float((int)S[4 * c4 + 3] + kMagicBitsF)), nm);
                        acc[16 * c + 2 * c4] = __ffma2_rn(f0, make_float2(g4.x, g4.y), acc[16 * c + 2 * c4]);
                        acc[16 * c + 2 * c4 + 1] = __ffma2_rn(f1, make_float2(g4.z, g4.w), acc[16 * c + 2 * c4 + 1]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.empty[s]);
            }
            if (w.s + 1 < a.S) {
                // hand the chain to the next K range of this output tile
                float4* dst = reinterpret_cast<float4*>(a.partial + tile * (int64_t)(FM * FN) + (int64_t)row * FN + h * FHC);
#pragma unroll
                for (int c = 0; c < FHC / 4; ++c)
                    dst[c] = make_float4(acc[2 * c].x, acc[2 * c].y, acc[2 * c + 1].x, acc[2 * c + 1].y);
                __threadfence();
                named_sync(1, 32 * FEPI);
                if (threadIdx.x == 64) st_release_u32(a.flags + tile, (uint32_t)(w.s + 1));
                continue;
            }
            // ---------------- output: y = acc * sa through the swizzled staging boxes ----------------
            const int64_t m0 = w.mt * FM, n0 = w.nt * FN;
            const float sa = m0 + row < a.M ? a.sa[m0 + row] : 0.0f;
#pragma unroll
            for (int part = 0; part < FN / FOUT; ++part) {
                if (threadIdx.x == 64) bulk_wait_read0();
                named_sync(1, 32 * FEPI);
                if ((h * FHC) / FOUT == part) {
#pragma unroll
                    for (int bb = 0; bb < FHC / 32; ++bb)
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int b = (h * FHC - part * FOUT) / 32 + bb;
                            const float2 p0 = acc[bb * 16 + 2 * j], p1 = acc[bb * 16 + 2 * j + 1];
                            *reinterpret_cast<float4*>(&sm.out[b][swz(row, j)]) = make_float4(
                                __fmul_rn(p0.x, sa), __fmul_rn(p0.y, sa), __fmul_rn(p1.x, sa), __fmul_rn(p1.y, sa));
                        }
                }
                fence_proxy_async();
                named_sync(1, 32 * FEPI);
                if (threadIdx.x == 64 && alive) {
#pragma unroll
                    for (int b = 0; b < FOUT / 32; ++b)
                        tma_store_2d(&tY, (int)(n0 + part * FOUT + b * 32), (int)m0, &sm.out[b][0]);
                    bulk_commit();
                }
            }
        }
        if (threadIdx.x == 64) bulk_wait0();
    } else {
        // ---------------- decoder groups: the weight's codes -> int8 operand stages ----------------
        const int d = (threadIdx.x - FDEC0) / 128;
        const int t = (threadIdx.x - FDEC0) % 128;  // weight row within the tile
        const int dwarp = t >> 5;
        int it = 0, j = 0;
        bool alive = true;
        for (int64_t u = blockIdx.x; u < a.units; u += gridDim.x) {
            const Unit w = unit_of(a, u);
            for (int64_t kb = w.s * a.KS; kb < (w.s + 1) * a.KS; ++kb, ++it) {
                if ((it % FDEC) != d) continue;
                const int s = it % FST;
                if (alive && it >= FST) {
                    bool got = true;
                    if (t == 0) got = mbar_wait_sleep(&sm.empty[s], (uint32_t)((it / FST - 1) & 1));
                    named_sync(2 + d, 128);
                    if (t == 0 && !got) sm.in_ok[d] = -1;
                    named_sync(2 + d, 128);
                    if (sm.in_ok[d] < 0) {
                        if (t == 0) status_set(a.ws, kStTimeout);
                        alive = false;
                    }
                }
                if (!alive) continue;
                // the item's words: chunks (kb, 4 nt .. 4 nt + 3), one bulk copy of their 16-byte range
                const int64_t c0 = kb * a.RB + w.nt * (FN / kChunkTiles);
                if (t == 0) {
                    const int64_t w0 = a.chunk_word[c0];
                    const int64_t w1 = a.chunk_word[c0 + FN / kChunkTiles];
                    const int64_t lo = w0 & ~(int64_t)3, hi = (w1 + 3) & ~(int64_t)3;
                    const bool good = w1 >= w0 && hi <= a.cap_words && (hi - lo) <= (int64_t)(F_IN_WORDS - 2 * F_GUARD);
                    for (int ch = 0; ch <= FN / kChunkTiles; ++ch)
                        sm.chunkbase[d][ch] = good ? (uint32_t)(a.chunk_word[c0 + ch] - lo + F_GUARD) : 0u;
                    sm.in_ok[d] = good ? 1 : 0;
                    if (!good) status_set(a.ws, kStCorrupt);
                    const uint32_t bytes = good ? (uint32_t)((hi - lo) * 4) : 0u;
                    if (bytes) {
                        mbar_arrive_expect_tx(&sm.in_bar[d], bytes);
                        bulk_load_1d(sm.in[d] + F_GUARD, a.bits + lo, bytes, &sm.in_bar[d]);
                    } else {
                        mbar_arrive(&sm.in_bar[d]);
                    }
                }
                {
                    // tile lengths of this row's chunk (read by decode_row)
                    const int64_t tt = kb * a.N + w.nt * FN + t;
                    const uint32_t mt = a.meta[tt];
                    constexpr int COSB = LAT == HQ_E8 ? FK / 8 : 0;
                    sm.Ls[d][t] = (uint32_t)COSB + (uint32_t)FK * ((mt & 15u) + 1u) + (mt >> 4);
                }
                named_sync(2 + d, 128);
                bool arrived = true;
                if (t == 0) arrived = mbar_wait(&sm.in_bar[d], (uint32_t)(j & 1));
                ++j;
                named_sync(2 + d, 128);
                if (t == 0 && !arrived) {
                    status_set(a.ws, kStTimeout);
                    sm.in_ok[d] = 0;
                }
                named_sync(2 + d, 128);
                const bool stage_ok = sm.in_ok[d] == 1;
                const float gs = decode_row<LAT>(a, sm, d, s, t, kb, w.nt, stage_ok);
                sm.g[s][t] = gs;
                fence_proxy_async();  // the stage is read by the tensor cores (async proxy)
                named_sync(2 + d, 128);
                if (t == 0) mbar_arrive(&sm.full[s]);
                (void)dwarp;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, FACC * FN);
}

}  // namespace
}  // namespace hq

using namespace hq;

namespace {

// K ranges per output tile: enough units to cover the SMs of a B200 (148), each range at least
// one group and the ranges equal (a divisor of the group count)
int64_t k_splits(int64_t tiles, int64_t KB)
{
    if (tiles >= 120) return 1;
    const int64_t want = (148 + tiles - 1) / tiles;
    int64_t S = 1;
    for (int64_t c = 1; c <= KB && c <= want; ++c)
        if (KB % c == 0) S = c;
    return S;
}

size_t gemm_code_ws(int64_t M, int64_t N, int64_t K)
{
    const int64_t MT = (M + FM - 1) / FM, NT = N / FN, KB = K / FK;
    const int64_t S = k_splits(MT * NT, KB);
    size_t b = 256 + (((size_t)(MT * NT) * 4u + 255u) & ~(size_t)255u);
    if (S > 1) b += (size_t)(MT * NT) * FM * FN * 4u;
    return b;
}

}  // namespace

extern "C" size_t hq_gemm_code_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || N < FN || N % FN || K < FK || K % FK || M > ((int64_t)1 << 31) || N > ((int64_t)1 << 31) ||
        K > ((int64_t)1 << 20))
        return 0;
    return gemm_code_ws(M, N, K);
}

extern "C" hq_status_t hq_gemm_code(const int8_t* A, const float* sa, int64_t M, const hq_code_t* code, float* Y,
                                    void* ws, size_t ws_bytes, void* stream)
{
    if (!A || !sa || !code || !Y || !ws) return HQ_ERR_ARG;
    if (code->version != HQ_FORMAT_VERSION || code->kv != 0) return HQ_ERR_ARG;
    const hq_params_t& p = code->p;
    if (p.tile != FK || (p.lattice != HQ_Z && p.lattice != HQ_D4 && p.lattice != HQ_E8)) return HQ_ERR_UNSUPPORTED;
    if (!(p.step >= 0.00390625f && p.step <= 64.0f)) return HQ_ERR_ARG;
    const int64_t N = code->rows, K = code->cols;
    const size_t need = hq_gemm_code_workspace_bytes(M, N, K);
    if (need == 0 || ws_bytes < need) return HQ_ERR_ARG;
    if (!code->scale || !code->meta || !code->chunk_word || !code->bits || code->cap_words < 1) return HQ_ERR_ARG;
    const uintptr_t al = reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(Y) |
                         reinterpret_cast<uintptr_t>(ws) | reinterpret_cast<uintptr_t>(code->bits);
    if (al & 15u) return HQ_ERR_ARG;
    if (!device_of(A)) return HQ_ERR_ARG;
    CUtensorMap ta, ty;
    if (!tensor_map_2d(&ta, A, M, K, 1, FM) || !tensor_map_2d(&ty, Y, M, N, 4, FM)) return HQ_ERR_CUDA;
    const int64_t MT = (M + FM - 1) / FM, NT = N / FN, KB = K / FK;
    const int64_t S = k_splits(MT * NT, KB);
    FusedArgs a{};
    a.M = M;
    a.N = N;
    a.K = K;
    a.KB = KB;
    a.MT = MT;
    a.NT = NT;
    a.S = S;
    a.KS = KB / S;
    a.units = MT * NT * S;
    a.beta = p.step;
    a.sa = sa;
    a.scale = code->scale;
    a.meta = code->meta;
    a.chunk_word = code->chunk_word;
    a.bits = code->bits;
    a.cap_words = code->cap_words;
    a.RB = (N + kChunkTiles - 1) / kChunkTiles;
    a.IB = (N + FN - 1) / FN;
    a.ws = static_cast<WsHeader*>(ws);
    a.flags = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + 256);
    a.partial = S > 1 ? reinterpret_cast<float*>(static_cast<char*>(ws) + 256 +
                                                 ((((size_t)(MT * NT) * 4u) + 255u) & ~(size_t)255u))
                      : nullptr;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // header and flags start at zero; the partial chains are written before they are read
    if (cudaMemsetAsync(ws, 0, 256 + (size_t)(MT * NT) * 4u, st) != cudaSuccess) return HQ_ERR_CUDA;
    const size_t smem = sizeof(FusedSmem) + 1024;
    const int64_t grid64 = a.units < num_sms() ? a.units : num_sms();
    const int grid = (int)grid64;
    cudaError_t e;
    switch (p.lattice) {
    case HQ_Z:
        e = cudaFuncSetAttribute(gemm_code_kernel<HQ_Z>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess) gemm_code_kernel<HQ_Z><<<grid, FTHREADS, smem, st>>>(a, ta, ty);
        break;
    case HQ_D4:
        e = cudaFuncSetAttribute(gemm_code_kernel<HQ_D4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess) gemm_code_kernel<HQ_D4><<<grid, FTHREADS, smem, st>>>(a, ta, ty);
        break;
    default:
        e = cudaFuncSetAttribute(gemm_code_kernel<HQ_E8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess) gemm_code_kernel<HQ_E8><<<grid, FTHREADS, smem, st>>>(a, ta, ty);
        break;
    }
    if (e != cudaSuccess) return HQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}
