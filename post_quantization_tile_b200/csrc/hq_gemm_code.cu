// hq_gemm_code.cu -- the grouped int8 tensor-core GEMM with the decode of the weight's code fused
// into its producer warps: the weight's int8 lattice codes never exist outside shared memory.
//
// Y[m, r] = sa_m * sum_t g[t, r] S_{m,r,t},  S_{m,r,t} = sum_{j in group t} A[m, j] V[r, j], exactly
// the product of hq_decode_int8 followed by hq_gemm_int8 (same codes, same zeroed tiles, same
// binary32 order acc = fma(S, g, acc) over the groups from 0, then y = acc * sa_m).
//
// A work unit is R activation tiles of 128 rows (R = 1, or 2 once M > 128) against one weight
// slab of 32 rows -- one chunk of the code per K group -- over all K groups, so each output
// element's binary32 chain runs in one CTA from start to end and each decoded chunk feeds R
// tiles; the slabs give 128 units per activation row block of a 4096-row weight, enough to occupy
// the SMs at small M without splitting K.  One CTA per SM walks units:
//   warp 0       TMA loads of the activation boxes (rows past M read as zeros) into a ring;
//   warp 1       tcgen05.mma.kind::i8 (M 128, N 32, K 32) x 4 per group and tile into a TMEM slot;
//   warps 2 ..   epilogue, one warpgroup per activation tile: TMEM loads, int32 -> binary32, fma
//                with the group scales, output;
//   the rest     decoder warps (16 when R = 1, 12 when R = 2), K group kb on warp kb mod their
//                count: a bulk copy of the chunk's words (read in place when longer than 4 KB), a
//                warp scan of its tile lengths, then one lane per weight row reads its
//                tile's Rice codes from both ends, unstrips each lattice block and writes the int8
//                codes straight into the MMA's K-major 128-byte-swizzled operand stage (one per
//                decoder warp), and the tile's group scale next to it.
// Every wait is bounded: on a timeout the kernel records HQ_ERR_TIMEOUT and winds down.
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/hq.h"
#include "hq_common.cuh"
#include "hq_launch.h"
#include "hq_lattice.cuh"
#include "hq_tc.cuh"

namespace hq {
namespace {

constexpr int FM = 128, FN = 32, FK = 128;  // activation rows, weight rows per unit (one chunk), K group

// R activation tiles per unit: the ring, the decoder warps (= weight-code stages), the epilogue
// warpgroups and the TMEM slots (R x 32 columns each, all 512) follow from it; 704 threads either way
template <int R>
struct FusedCfg {
    static constexpr int SA = R == 1 ? 4 : 2;      // activation stages (R boxes each)
    static constexpr int DW = R == 1 ? 16 : 12;    // decoder warps
    static constexpr int EPI = 4 * R;              // epilogue warps
    static constexpr int ACC = 512 / (FN * R);     // TMEM accumulator slots
    static constexpr int THREADS = 32 * (2 + EPI + DW);
    static constexpr int DEC0 = 32 * (2 + EPI);    // first decoder thread
};
// a decoder warp's copy of one chunk: up to 1024 words (8 bits per weight); a longer chunk is
// read from global memory where it lies
constexpr int F_GUARD = 4;
constexpr int F_IN_WORDS = 1024 + 8 + 2 * F_GUARD;
constexpr uint32_t kIdescF = idesc_i8(FM, FN);  // per activation tile
constexpr float kMagicF = 12582912.0f;  // 1.5 * 2^23
constexpr int kMagicBitsF = 0x4B400000;

template <int R>
struct FusedSmem {
    using C = FusedCfg<R>;
    alignas(1024) int8_t a[C::SA][R][FM * FK];
    alignas(1024) int8_t v[C::DW][FN * FK];
    alignas(1024) unsigned char out[R][FM * 128];  // output staging: one 32-column box per tile
    alignas(16) uint32_t in[C::DW][F_IN_WORDS];     // each decoder warp's chunk words
    alignas(16) float g[C::DW][FN];
    alignas(8) uint64_t a_full[C::SA];
    uint64_t a_empty[C::SA];
    uint64_t b_full[C::DW];
    uint64_t b_empty[C::DW];
    uint64_t acc_full[C::ACC];
    uint64_t acc_empty[C::ACC];
    uint64_t in_bar[C::DW];
    uint32_t tmem_base;
};

struct FusedArgs {
    int64_t M, N, K;     // activation rows, weight rows, inner dimension
    int64_t KB, MT, NS;  // K groups, activation tiles, weight slabs
    int64_t MP;          // activation row blocks of R tiles
    int64_t units;
    float beta;
    const float* sa;
    const uint16_t* scale;
    const uint16_t* meta;
    const uint32_t* chunk_word;
    const uint32_t* bits;
    int64_t cap_words, RB;
    WsHeader* ws;
};

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

// One decoder lane: weight row `row` of the slab, its tile's Rice codes (starting at bit tile0 of
// the copied words `in`, L bits long) from both ends into row `row` of the operand stage `vst`.
// Returns the tile's group scale.
template <int LAT>
__device__ __forceinline__ float decode_row(const FusedArgs& a, const uint32_t* in, int lim, int8_t* vst, int row,
                                            int tile0, uint32_t L, uint32_t mt, uint16_t sbits, bool ok)
{
    constexpr int COSB = LAT == HQ_E8 ? FK / 8 : 0;
    const int k = (int)(mt & 15u);
    uint32_t out8 = 0;
    if (ok) {
        uint32_t cosbits = 0;
        if constexpr (LAT == HQ_E8) {
            const int cw = min(max(tile0 >> 5, 0), lim);
            const unsigned long long two = ((unsigned long long)in[min(cw + 1, lim)] << 32) | in[cw];
            cosbits = (uint32_t)(two >> (tile0 & 31)) & 0xFFFFu;
        }
        const uint32_t pow2k = 1u << k, sq_meta = mt >> 4;
        BitReader<true> rf;
        BitReader<false> rb;
        rf.begin(in, tile0 + COSB, lim);
        rb.begin(in, tile0 + (int)L - 1, lim);
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
            *reinterpret_cast<uint2*>(vst + swz(row, bf >> 1) + 8 * (bf & 1)) = pack8(vf, out8);
            *reinterpret_cast<uint2*>(vst + swz(row, bb >> 1) + 8 * (bb & 1)) = pack8(vb, out8);
        }
        const uint32_t sq = (uint32_t)(rf.consumed() + rb.consumed() - FK * (k + 1));
        if (sq != sq_meta) ok = false;
    }
    if (!ok) status_set(a.ws, kStCorrupt);
    else if (out8) status_set(a.ws, kStRange);
    if (!ok || out8) {
        // a corrupt tile, or a code outside int8: the tile's codes are zero (as hq_decode_int8)
#pragma unroll
        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(vst + swz(row, c)) = make_uint4(0u, 0u, 0u, 0u);
    }
    const float sh = __uint_as_float((uint32_t)sbits << 16);
    float gs = __fmul_rn(__fmul_rn(sh, a.beta), __uint_as_float(0x3DB504F3u));  // c_128 = RN(2^-3.5)
    if constexpr (LAT == HQ_E8) gs = __fmul_rn(gs, 0.5f);
    return gs;
}

template <int LAT, int R>
__global__ void __launch_bounds__(FusedCfg<R>::THREADS, 1)
    gemm_code_kernel(const FusedArgs a, const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tY)
{
    using C = FusedCfg<R>;
    constexpr int FSA = C::SA, FDW = C::DW, FEPI = C::EPI, FACC = C::ACC, FDEC0 = C::DEC0;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    FusedSmem<R>& sm =
        *reinterpret_cast<FusedSmem<R>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = (int)a.KB;

    if (threadIdx.x == 0) {
        for (int s = 0; s < FSA; ++s) {
            mbar_init(&sm.a_full[s], 1);   // the activation box's TMA
            mbar_init(&sm.a_empty[s], 1);  // the MMAs' commit
        }
        for (int s = 0; s < FDW; ++s) {
            mbar_init(&sm.b_full[s], 1);          // the decoder warp
            mbar_init(&sm.b_empty[s], 1 + FEPI);  // the MMAs' commit and every epilogue warp's read of g
            mbar_init(&sm.in_bar[s], 1);
        }
        for (int s = 0; s < FACC; ++s) {
            mbar_init(&sm.acc_full[s], 1);
            mbar_init(&sm.acc_empty[s], FEPI);
        }
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&sm.tmem_base, 512);
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
                const int64_t mp = u / a.NS;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % FSA;
                    if (it >= FSA && !mbar_wait_sleep(&sm.a_empty[s], (uint32_t)((it / FSA - 1) & 1))) {
                        status_set(a.ws, kStTimeout);
                        alive = false;
                        break;
                    }
                    // a box whose rows all lie past M reads as zeros and still brings its bytes
                    mbar_arrive_expect_tx(&sm.a_full[s], (uint32_t)(R * FM * FK));
#pragma unroll
                    for (int r = 0; r < R; ++r)
                        tma_load_2d(sm.a[s][r], &tA, kb * FK, (int)((mp * R + r) * FM), &sm.a_full[s]);
                }
            }
            // no copy outlives the block: the last boxes of each stage have landed (at once, unless
            // the MMA side stopped on a timeout)
            for (int j = it > FSA ? it - FSA : 0; j < it; ++j)
                if (!mbar_wait_sleep(&sm.a_full[j % FSA], (uint32_t)((j / FSA) & 1))) status_set(a.ws, kStTimeout);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int it = 0;
            bool alive = true;
            for (int64_t u = blockIdx.x; alive && u < a.units; u += gridDim.x) {
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int sa = it % FSA, sb = it % FDW, slot = it % FACC;
                    bool ok = it < FACC || mbar_wait_sleep(&sm.acc_empty[slot], (uint32_t)((it / FACC - 1) & 1));
                    ok = ok && mbar_wait_sleep(&sm.a_full[sa], (uint32_t)((it / FSA) & 1));
                    ok = ok && mbar_wait_sleep(&sm.b_full[sb], (uint32_t)((it / FDW) & 1));
                    if (!ok) {
                        status_set(a.ws, kStTimeout);
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t bd = sw128_desc(sm.v[sb]);
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const uint64_t ad = sw128_desc(sm.a[sa][r]);
#pragma unroll
                        for (int kk = 0; kk < FK / 32; ++kk)
                            mma_i8(tbase + (uint32_t)((slot * R + r) * FN), ad + (uint64_t)(2 * kk),
                                   bd + (uint64_t)(2 * kk), kIdescF, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&sm.a_empty[sa]);
                    mma_commit(&sm.b_empty[sb]);
                    mma_commit(&sm.acc_full[slot]);
                }
            }
        }
        __syncwarp();
    } else if (threadIdx.x < FDEC0) {
        // ---------------- epilogue: warpgroup r takes activation tile r; one row per thread ----------------
        const int q = warp & 3;          // TMEM lane quarter of this warp
        const int r = (warp - 2) >> 2;   // activation tile of the unit
        const int lead = 64 + 128 * r;   // the warpgroup's first thread: staging and stores
        const int row = q * 32 + lane;
        const float2 nm = make_float2(-kMagicF, -kMagicF);
        int it = 0;
        bool alive = true;
        for (int64_t u = blockIdx.x; u < a.units; u += gridDim.x) {
            const int64_t mt = (u / a.NS) * R + r, ns = u % a.NS;
            float2 acc[FN / 2];
#pragma unroll
            for (int c = 0; c < FN / 2; ++c) acc[c] = make_float2(0.0f, 0.0f);
            // after a timeout a warp keeps walking the loops without waiting, so that every
            // epilogue warp still reaches each named barrier below
            for (int kb = 0; kb < KB; ++kb, ++it) {
                if (!alive) continue;
                const int slot = it % FACC, sb = it % FDW;
                const bool got = mbar_wait_sleep(&sm.acc_full[slot], (uint32_t)((it / FACC) & 1));
                __syncwarp();  // the warp-wide TMEM load below needs the whole warp converged
                if (!__all_sync(0xffffffffu, got)) {
                    if (lane == 0) status_set(a.ws, kStTimeout);
                    alive = false;
                    continue;
                }
                tc_fence_after();
                uint32_t S[32];
                tmem_ld32_nowait(tbase + ((uint32_t)(q * 32) << 16) + (uint32_t)((slot * R + r) * FN), S);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.acc_empty[slot]);  // the slot is read
                const float4* gp = reinterpret_cast<const float4*>(&sm.g[sb][0]);
#pragma unroll
                for (int c4 = 0; c4 < 8; ++c4) {
                    const float4 g4 = gp[c4];
                    // |S| < 2^22: adding 1.5 * 2^23 in the integer domain gives an exact float
                    const float2 f0 = __fadd2_rn(make_float2(__int_as_float((int)S[4 * c4] + kMagicBitsF),
                                                             __int_as_float((int)S[4 * c4 + 1] + kMagicBitsF)), nm);
                    const float2 f1 = __fadd2_rn(make_float2(__int_as_float((int)S[4 * c4 + 2] + kMagicBitsF),
                                                             __int_as_float((int)S[4 * c4 + 3] + kMagicBitsF)), nm);
                    acc[2 * c4] = __ffma2_rn(f0, make_float2(g4.x, g4.y), acc[2 * c4]);
                    acc[2 * c4 + 1] = __ffma2_rn(f1, make_float2(g4.z, g4.w), acc[2 * c4 + 1]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.b_empty[sb]);  // the stage's scales are read
            }
            // ---------------- output: y = acc * sa through the swizzled staging box ----------------
            const int64_t m0 = mt * FM, n0 = ns * FN;
            if (m0 >= a.M) continue;  // the unit's second tile lies past M: nothing to store
            const float sa = m0 + row < a.M ? a.sa[m0 + row] : 0.0f;
            if (threadIdx.x == lead) bulk_wait_read0();  // the previous store has read the staging
            named_sync(1 + r, 128);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float2 p0 = acc[2 * j], p1 = acc[2 * j + 1];
                *reinterpret_cast<float4*>(&sm.out[r][swz(row, j)]) =
                    make_float4(__fmul_rn(p0.x, sa), __fmul_rn(p0.y, sa), __fmul_rn(p1.x, sa), __fmul_rn(p1.y, sa));
            }
            fence_proxy_async();
            named_sync(1 + r, 128);
            if (threadIdx.x == lead && alive) {
                tma_store_2d(&tY, (int)n0, (int)m0, &sm.out[r][0]);
                bulk_commit();
            }
        }
        if (threadIdx.x == lead) bulk_wait0();
    } else {
        // ---------------- decoder warps: the weight's codes -> int8 operand stages ----------------
        constexpr int COSB = LAT == HQ_E8 ? FK / 8 : 0;
        const int w = warp - FDEC0 / 32;  // decoder warp = its operand stage
        uint32_t* in = sm.in[w];
        int it = 0, j = 0;
        bool alive = true;
        for (int64_t u = blockIdx.x; u < a.units; u += gridDim.x) {
            const int64_t ns = u % a.NS;
            for (int kb = 0; kb < KB; ++kb, ++it) {
                if ((it % FDW) != w || !alive) continue;
                // the stage is free once the MMAs and the epilogue of its previous group are done
                if (it >= FDW) {
                    bool got = true;
                    if (lane == 0) got = mbar_wait_sleep(&sm.b_empty[w], (uint32_t)((it / FDW - 1) & 1));
                    got = __shfl_sync(0xffffffffu, got, 0);
                    if (!got) {
                        if (lane == 0) status_set(a.ws, kStTimeout);
                        alive = false;
                        continue;
                    }
                }
                // the chunk's words: one bulk copy of their 16-byte range, or (a chunk too long for
                // the copy) read in place
                const int64_t c = (int64_t)kb * a.RB + ns;
                const int64_t w0 = a.chunk_word[c], w1 = a.chunk_word[c + 1];
                const int64_t lo = w0 & ~(int64_t)3, hi = (w1 + 3) & ~(int64_t)3;
                const bool good = w1 > w0 && w1 <= a.cap_words;
                const bool copied = good && (hi - lo) <= (int64_t)(F_IN_WORDS - 2 * F_GUARD);
                const uint32_t cb = copied ? (uint32_t)(w0 - lo + F_GUARD) : 0u;
                const uint32_t* src = copied ? in : a.bits + (good ? w0 : 0);
                const int lim = copied ? F_IN_WORDS - 1 : (good ? (int)(w1 - w0 - 1) : 0);
                if (lane == 0) {
                    if (!good) status_set(a.ws, kStCorrupt);
                    if (copied) {
                        mbar_arrive_expect_tx(&sm.in_bar[w], (uint32_t)((hi - lo) * 4));
                        bulk_load_1d(in + F_GUARD, a.bits + lo, (uint32_t)((hi - lo) * 4), &sm.in_bar[w]);
                    } else {
                        mbar_arrive(&sm.in_bar[w]);
                    }
                }
                // this lane's tile: header, length, and its first bit (a scan of the chunk's lengths)
                const int64_t t = (int64_t)kb * a.N + ns * FN + lane;
                const uint32_t mt = a.meta[t];
                const uint16_t sbits = a.scale[t];
                const uint32_t L = (uint32_t)COSB + (uint32_t)FK * ((mt & 15u) + 1u) + (mt >> 4);
                uint32_t incl = L;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                bool arrived = true;
                if (lane == 0) arrived = mbar_wait(&sm.in_bar[w], (uint32_t)(j & 1));
                ++j;
                arrived = __shfl_sync(0xffffffffu, arrived, 0);
                if (!arrived && lane == 0) status_set(a.ws, kStTimeout);
                const int tile0 = (int)(cb * 32u + (incl - L));
                const float gs = decode_row<LAT>(a, src, lim, sm.v[w], lane, tile0, L, mt, sbits, good && arrived);
                sm.g[w][lane] = gs;
                fence_proxy_async();  // the stage is read by the tensor cores (async proxy)
                __syncwarp();
                if (!arrived) {
                    // a copy that did not complete may still land in `in`: give it one more bounded
                    // wait and stop decoding (the stage is published, zeroed, so the MMA side finishes)
                    if (lane == 0) mbar_wait(&sm.in_bar[w], (uint32_t)((j - 1) & 1));
                    alive = false;
                }
                if (lane == 0) mbar_arrive(&sm.b_full[w]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, 512);
}

template <int LAT, int R>
cudaError_t launch_fused(const FusedArgs& a, const CUtensorMap& ta, const CUtensorMap& ty, cudaStream_t st)
{
    const size_t smem = sizeof(FusedSmem<R>) + 1024;
    const cudaError_t e =
        cudaFuncSetAttribute(gemm_code_kernel<LAT, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = (int)(a.units < num_sms() ? a.units : num_sms());
    gemm_code_kernel<LAT, R><<<grid, FusedCfg<R>::THREADS, smem, st>>>(a, ta, ty);
    return cudaGetLastError();
}

}  // namespace
}  // namespace hq

using namespace hq;

extern "C" size_t hq_gemm_code_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || N < 128 || N % 128 || K < FK || K % FK || M > ((int64_t)1 << 31) || N > ((int64_t)1 << 31) ||
        K > ((int64_t)1 << 20))
        return 0;
    return 256;  // the status word
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
    FusedArgs a{};
    a.M = M;
    a.N = N;
    a.K = K;
    a.KB = K / FK;
    a.MT = (M + FM - 1) / FM;
    a.NS = N / FN;
    const int R = a.MT > 1 ? 2 : 1;  // two activation tiles per decoded slab once there are two
    a.MP = (a.MT + R - 1) / R;
    a.units = a.MP * a.NS;
    // the roles count K groups over their units in 32-bit integers, and TMA coordinates are 32-bit
    if (a.units * a.KB >= ((int64_t)1 << 31) || a.MP * R * FM >= ((int64_t)1 << 31)) return HQ_ERR_UNSUPPORTED;
    a.beta = p.step;
    a.sa = sa;
    a.scale = code->scale;
    a.meta = code->meta;
    a.chunk_word = code->chunk_word;
    a.bits = code->bits;
    a.cap_words = code->cap_words;
    a.RB = (N + kChunkTiles - 1) / kChunkTiles;
    a.ws = static_cast<WsHeader*>(ws);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), st) != cudaSuccess) return HQ_ERR_CUDA;
    cudaError_t e;
    switch (p.lattice) {
    case HQ_Z: e = R == 1 ? launch_fused<HQ_Z, 1>(a, ta, ty, st) : launch_fused<HQ_Z, 2>(a, ta, ty, st); break;
    case HQ_D4: e = R == 1 ? launch_fused<HQ_D4, 1>(a, ta, ty, st) : launch_fused<HQ_D4, 2>(a, ta, ty, st); break;
    default: e = R == 1 ? launch_fused<HQ_E8, 1>(a, ta, ty, st) : launch_fused<HQ_E8, 2>(a, ta, ty, st); break;
    }
    return e == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}
