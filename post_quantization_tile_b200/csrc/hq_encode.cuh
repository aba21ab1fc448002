// hq_encode.cuh -- encode kernel of the HyperQuant tile codec (Methodology steps 1-4).
//
// One block of 128 threads works on an "item": TI consecutive rows of one tile column, i.e.
// TI tiles = TI/32 chunks.  Threads own whole tiles in registers (two threads per tile when
// n = 256), so the RMS, the sign flip, the Walsh-Hadamard butterflies, the lattice decision and
// the Rice parameter need no cross-thread traffic.  Tiles arrive through 2-D TMA boxes with
// 128-byte swizzle (conflict-free row reads) in a two-stage ring; items are claimed from a
// global counter so that the single-pass chunk-offset scan (decoupled look-back over items) only
// ever waits on blocks that are already running.
#pragma once
#include "hq_common.cuh"
#include "hq_lattice.cuh"

namespace hq {

struct EncodeArgs {
    int64_t rows, cols;
    float beta;
    uint64_t seed;
    int64_t kv_S;
    int64_t items;   // number of items
    int64_t IB;      // items per tile column
    int64_t RB;      // chunks per tile column
    int64_t C;       // chunks
    uint16_t* scale;
    uint16_t* meta;
    uint32_t* chunk_word;
    uint32_t* bits;
    int64_t cap_words;
    int32_t* v_out;
    WsHeader* ws;
    unsigned long long* states;
    uint32_t rk[20];  // Philox round keys of `seed` (key words 0, 1 of rounds 0 .. 9), for the dither
    const RateSearch* search;  // count-only passes of a step search: the step comes from here
    int64_t kv_s0;             // KV: position of the call's first token in every sequence
    int64_t test_silent_item;  // read only by the test build (HQ_TEST_HOOKS): this item never publishes
                               // its offset (-1: none), so its successor's bounded look-back must run
                               // out and report a timeout
};

// Several tensors in one launch: tensor t takes the global items item0[t] .. item0[t + 1] - 1,
// in its own order, with its own look-back chain, outputs and tensor map; the header (work
// counter, status) is shared.  One launch of one tensor is the batch of one.
constexpr int kEncodeBatchMax = 16;
template <int MAXB>
struct EncodeBatch {
    CUtensorMap map[MAXB];
    EncodeArgs arg[MAXB];
    int64_t item0[MAXB + 1];
    int32_t count;
};

template <int MAXB>
__device__ __forceinline__ int batch_tensor(const int64_t (&item0)[MAXB + 1], int32_t count, int64_t g)
{
    int t = 0;
#pragma unroll
    for (int i = 1; i < MAXB; ++i)
        if (i < count && g >= item0[i]) t = i;
    return t;
}

// SRC: 0 bf16 weight, 1 fp32 weight, 2 fp32 normalised coefficients (no RMS / RHT)
template <int N, int SRC>
struct EncGeom {
    static constexpr int TPT = enc_tpt(N, SRC);
    static constexpr int V = N / TPT;      // coefficients per thread
    static constexpr int H = V / 2;        // float2 pairs per thread: P[m] = (c[m], c[m + H])
    static constexpr int TI = kThreads / TPT;  // tiles (rows) per item
    static constexpr int ES = SRC == 0 ? 2 : 4;
    static constexpr int ROWB = N * ES;    // bytes per tile row
    static constexpr int NB = ROWB / 128;  // 128-byte boxes per row
    static constexpr int STAGE = NB * TI * 128;
    static constexpr int ZZ = V * 2 * kThreads;  // zig-zag symbol scratch (uint16)
    // the scratch aliases the TMA stage (smaller footprint, 3 blocks per SM, the next item is
    // loaded after packing) or has its own buffer (next item loaded as soon as the stage is read)
    static constexpr bool SEPARATE_ZZ = HQ_ENC_SEPARATE_ZZ != 0;
    static constexpr int BUF = SEPARATE_ZZ ? STAGE : (STAGE > ZZ ? STAGE : ZZ);
    static constexpr int ZZBUF = SEPARATE_ZZ ? ZZ : 16;
    static constexpr int CH = TI / kChunkTiles;  // chunks per item
    // staging bound per tile: n/8 coset bits + n (k + 1) + sum q with k <= 11 and sum q < 2n.
    // The step range keeps k <= 9; longer tiles are reported (HQ_ERR_RANGE) and left out.
    static constexpr int KMAX = 11;
    static constexpr int LMAX = N / 8 + (KMAX + 1) * N + 2 * N;
    static constexpr int STG_WORDS = TI * ((LMAX + 31) / 32) + CH + 8;
    static constexpr int LOG2N = N == 64 ? 6 : (N == 128 ? 7 : 8);
    static constexpr int MASKS = SRC == 0 ? N / 2 : N;  // sign-mask words per tile column
};

template <int N, int SRC>
struct EncSmem {
    using G = EncGeom<N, SRC>;
    alignas(1024) unsigned char buf[G::BUF];  // TMA stage (and the zig-zag scratch when aliased)
    alignas(16) unsigned char zzbuf[G::ZZBUF];
    uint32_t stg[G::STG_WORDS];
    alignas(16) uint32_t mask[G::MASKS];
    uint32_t Ls[G::TI];
    uint32_t rowoff[G::TI];
    uint32_t chunkoff[G::CH + 1];
    int64_t item_cur;
    int64_t mask_jt;
    uint32_t item_words;
    uint32_t base;
    alignas(8) uint64_t bar;
};

// zig-zag scratch: symbols 8g .. 8g+7 of thread t at byte (g * kThreads + t) * 16
__device__ __forceinline__ uint4* zz_slot(unsigned char* buf, int g, int tid)
{
    return reinterpret_cast<uint4*>(buf + ((size_t)g * kThreads + tid) * 16);
}

// ------------------------------------------------------------------------------------------------
// sign masks of tile column jt: D_jj = -1 where bit (J & 31) of Philox(seed, (J >> 7, 0, 0, 0))
// word (J & 127) >> 5 is set (J = jt n + j, the transformed-axis index).
// bf16 rows: one word per element pair (bits 15 / 31); fp32 rows: one word per element.
// ------------------------------------------------------------------------------------------------
template <int N, int SRC>
__device__ __forceinline__ void build_masks(uint32_t* mask, int64_t jt, uint64_t seed)
{
    using G = EncGeom<N, SRC>;
    for (int w = threadIdx.x; w < G::MASKS; w += kThreads) {
        const int per = SRC == 0 ? 2 : 1;
        uint32_t m = 0;
#pragma unroll
        for (int e = 0; e < per; ++e) {
            const int64_t J = jt * N + (int64_t)w * per + e;
            const uint4 ph = philox4x32_10(make_uint4((uint32_t)((uint64_t)J >> 7), 0u, 0u, 0u), (uint32_t)seed,
                                           (uint32_t)(seed >> 32));
            const int wsel = (int)((J & 127) >> 5);
            const uint32_t word = wsel == 0 ? ph.x : (wsel == 1 ? ph.y : (wsel == 2 ? ph.z : ph.w));
            const uint32_t bit = (word >> (J & 31)) & 1u;
            m |= bit << (SRC == 0 ? (e ? 31 : 15) : 31);
        }
        mask[w] = m;
    }
}

// ------------------------------------------------------------------------------------------------
// load a thread's coefficients from the swizzled stage into float2 pairs
// TPT == 1: P[m] = (x_m, x_{m+H});  TPT == 2: the first butterfly (stride n/2) is taken here,
// thread tau computes y_{tau n/2 + i} = x_i +- x_{i + n/2} and P[m] = (y'_m, y'_{m+H}).
// Also returns the thread's share of the RMS sum (ascending pairwise tree over its raw x).
// ------------------------------------------------------------------------------------------------
template <int N, int SRC>
__device__ __forceinline__ void load_row(const unsigned char* stage, const uint32_t* mask, int row, int tau,
                                         float2 (&P)[EncGeom<N, SRC>::H], float& sumsq)
{
    using G = EncGeom<N, SRC>;
    constexpr int H = G::H;
    // element e of the row -> (box, 16-byte chunk, offset)
    auto chunk_ptr = [&](int c) -> const uint4* {
        const int b = c >> 3;
        return reinterpret_cast<const uint4*>(stage + b * (G::TI * 128) + swz(row, c & 7));
    };
    if constexpr (SRC == 0) {
        // bf16: chunk c = elements 8c .. 8c+7
        if constexpr (G::TPT == 1) {
            float2 Q[H];
#pragma unroll
            for (int c = 0; c < H / 8; ++c) {
                const uint4 A = *chunk_ptr(c);
                const uint4 B = *chunk_ptr(c + H / 8);
                const uint4 MA = *reinterpret_cast<const uint4*>(mask + 4 * c);
                const uint4 MB = *reinterpret_cast<const uint4*>(mask + 4 * (c + H / 8));
                const uint32_t a[4] = {A.x ^ MA.x, A.y ^ MA.y, A.z ^ MA.z, A.w ^ MA.w};
                const uint32_t b[4] = {B.x ^ MB.x, B.y ^ MB.y, B.z ^ MB.z, B.w ^ MB.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    P[8 * c + 2 * q] = make_float2(bf16lo_to_f32(a[q]), bf16lo_to_f32(b[q]));
                    P[8 * c + 2 * q + 1] = make_float2(bf16hi_to_f32(a[q]), bf16hi_to_f32(b[q]));
                }
            }
#pragma unroll
            for (int m = 0; m < H; ++m) Q[m] = f2mul(P[m], P[m]);
#pragma unroll
            for (int h = 1; h < H; h *= 2)
#pragma unroll
                for (int m = 0; m < H; m += 2 * h) Q[m] = f2add(Q[m], Q[m + h]);
            sumsq = __fadd_rn(Q[0].x, Q[0].y);
        } else {
            // quarter k (0..3) of the row = elements k n/4 .. (k+1) n/4 - 1 = chunks k QC .. (k+1) QC - 1
            constexpr int QC = N / 32;
            float2 Q[H];
            const float2 sgn = tau ? make_float2(-1.0f, -1.0f) : make_float2(1.0f, 1.0f);
#pragma unroll
            for (int c = 0; c < QC; ++c) {
                uint4 X[4];
                uint32_t x[4][4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    X[k] = *chunk_ptr(c + QC * k);
                    const uint4 M = *reinterpret_cast<const uint4*>(mask + 4 * (c + QC * k));
                    x[k][0] = X[k].x ^ M.x; x[k][1] = X[k].y ^ M.y; x[k][2] = X[k].z ^ M.z; x[k][3] = X[k].w ^ M.w;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int m = 8 * c + 2 * q + hh;
                        const float2 lo = hh ? make_float2(bf16hi_to_f32(x[0][q]), bf16hi_to_f32(x[1][q]))
                                             : make_float2(bf16lo_to_f32(x[0][q]), bf16lo_to_f32(x[1][q]));
                        const float2 hi = hh ? make_float2(bf16hi_to_f32(x[2][q]), bf16hi_to_f32(x[3][q]))
                                             : make_float2(bf16lo_to_f32(x[2][q]), bf16lo_to_f32(x[3][q]));
                        // this thread's half of the RMS: tau 0 sums x[0, n/2), tau 1 x[n/2, n)
                        Q[m] = tau ? f2mul(hi, hi) : f2mul(lo, lo);
                        // first butterfly, stride n/2: tau 0 keeps sums, tau 1 differences
                        P[m] = __ffma2_rn(hi, sgn, lo);
                    }
                }
            }
#pragma unroll
            for (int h = 1; h < H; h *= 2)
#pragma unroll
                for (int m = 0; m < H; m += 2 * h) Q[m] = f2add(Q[m], Q[m + h]);
            sumsq = __fadd_rn(Q[0].x, Q[0].y);
        }
    } else {
        // fp32: chunk c = elements 4c .. 4c+3  (TPT == 1 only: N <= 128 for fp32 weights)
        static_assert(SRC == 2 || G::TPT == 1 || true, "");
        if constexpr (G::TPT == 1) {
            float2 Q[H];
#pragma unroll
            for (int c = 0; c < H / 4; ++c) {
                uint4 A = *chunk_ptr(c);
                uint4 B = *chunk_ptr(c + H / 4);
                if constexpr (SRC == 1) {
                    const uint4 MA = *reinterpret_cast<const uint4*>(mask + 4 * c);
                    const uint4 MB = *reinterpret_cast<const uint4*>(mask + 4 * (c + H / 4));
                    A.x ^= MA.x; A.y ^= MA.y; A.z ^= MA.z; A.w ^= MA.w;
                    B.x ^= MB.x; B.y ^= MB.y; B.z ^= MB.z; B.w ^= MB.w;
                }
                P[4 * c + 0] = make_float2(__uint_as_float(A.x), __uint_as_float(B.x));
                P[4 * c + 1] = make_float2(__uint_as_float(A.y), __uint_as_float(B.y));
                P[4 * c + 2] = make_float2(__uint_as_float(A.z), __uint_as_float(B.z));
                P[4 * c + 3] = make_float2(__uint_as_float(A.w), __uint_as_float(B.w));
            }
            if constexpr (SRC == 1) {
#pragma unroll
                for (int m = 0; m < H; ++m) Q[m] = f2mul(P[m], P[m]);
#pragma unroll
                for (int h = 1; h < H; h *= 2)
#pragma unroll
                    for (int m = 0; m < H; m += 2 * h) Q[m] = f2add(Q[m], Q[m + h]);
                sumsq = __fadd_rn(Q[0].x, Q[0].y);
            } else {
                sumsq = 0.0f;
            }
        } else {
            // coefficients, two threads per tile: thread tau holds positions tau V + [0, V)
#pragma unroll
            for (int c = 0; c < H / 4; ++c) {
                const uint4 A = *chunk_ptr(tau * (G::V / 4) + c);
                const uint4 B = *chunk_ptr(tau * (G::V / 4) + c + H / 4);
                P[4 * c + 0] = make_float2(__uint_as_float(A.x), __uint_as_float(B.x));
                P[4 * c + 1] = make_float2(__uint_as_float(A.y), __uint_as_float(B.y));
                P[4 * c + 2] = make_float2(__uint_as_float(A.z), __uint_as_float(B.z));
                P[4 * c + 3] = make_float2(__uint_as_float(A.w), __uint_as_float(B.w));
            }
            sumsq = 0.0f;
        }
    }
}

// in-thread Walsh-Hadamard butterflies on P[m] = (c_m, c_{m+H}), descending strides:
// H (within each pair), then H/2, ..., 1 (between pairs)
template <int H>
__device__ __forceinline__ void fwht_pairs(float2 (&P)[H])
{
#pragma unroll
    for (int m = 0; m < H; ++m) P[m] = make_float2(__fadd_rn(P[m].x, P[m].y), __fadd_rn(P[m].x, -P[m].y));
#pragma unroll
    for (int h = H / 2; h >= 1; h /= 2)
#pragma unroll
        for (int m = 0; m < H; ++m)
            if ((m & h) == 0) {
                const float2 a = P[m], b = P[m + h];
                P[m] = f2add(a, b);
                P[m + h] = f2sub(a, b);
            }
}

template <int N, int SRC>
__device__ __forceinline__ void issue_tma(EncSmem<N, SRC>& sm, const CUtensorMap* tmap, const EncodeArgs& a, int64_t it)
{
    using G = EncGeom<N, SRC>;
    if (it >= a.items) return;
    const int64_t jt = it / a.IB, ib = it % a.IB;
    mbar_arrive_expect_tx(&sm.bar, G::STAGE);
#pragma unroll
    for (int b = 0; b < G::NB; ++b)
        tma_load_2d(sm.buf + b * G::TI * 128, tmap, (int)(jt * N + b * (128 / G::ES)), (int)(ib * G::TI), &sm.bar);
}

// the TMA copy of global item g of a batch
template <int N, int SRC, int MAXB>
__device__ __forceinline__ void issue_tma_batch(EncSmem<N, SRC>& sm, const EncodeBatch<MAXB>& B, int64_t g)
{
    if (g >= B.item0[B.count]) return;
    const int t = batch_tensor<MAXB>(B.item0, B.count, g);
    issue_tma<N, SRC>(sm, &B.map[t], B.arg[t], g - B.item0[t]);
}

template <int N, int LAT, bool KV, int SRC, bool COUNT, int MAXB>
__global__ void __launch_bounds__(kThreads, kMinBlocks) encode_kernel(const __grid_constant__ EncodeBatch<MAXB> B)
{
    using G = EncGeom<N, SRC>;
    using SM = EncSmem<N, SRC>;
    constexpr int TPT = G::TPT, V = G::V, H = G::H, TI = G::TI, D = Lat<LAT>::d;
    constexpr int COSB = LAT == HQ_E8 ? N / 8 : 0;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // TMA boxes with 128-byte swizzle need 1024-byte aligned shared memory: align by hand
    SM& sm = *reinterpret_cast<SM*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);

    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int row_l = tid / TPT;   // row within the item
    const int tau = tid % TPT;
    unsigned char* const zzs = G::SEPARATE_ZZ ? sm.zzbuf : sm.buf;

    // the header (work counter, status) and a step search are shared by the batch's tensors
    WsHeader* const hdr = B.arg[0].ws;
    const int64_t total = B.item0[B.count];
    // a count-only pass of a finished step search does nothing (block-uniform)
    float beta_s = B.arg[0].beta;
    if constexpr (COUNT) {
        if (B.arg[0].search) {
            if (*(volatile const int32_t*)&B.arg[0].search->done) return;
            beta_s = *(volatile const float*)&B.arg[0].search->probe;
        }
    }

    for (int w = tid; w < G::STG_WORDS; w += kThreads) sm.stg[w] = 0u;
    if (tid == 0) {
        mbar_init(&sm.bar, 1);
        fence_mbar_init();
        sm.mask_jt = -1;
        const int64_t it = (int64_t)atomicAdd(&hdr->counter, 1u);
        sm.item_cur = it;
        issue_tma_batch<N, SRC, MAXB>(sm, B, it);
    }
    __syncthreads();

    for (int iter = 0;; ++iter) {
        const int64_t gitem = sm.item_cur;
        if (gitem >= total) break;
        // this item's tensor; below, `item` is its index within that tensor
        const int tb = MAXB == 1 ? 0 : batch_tensor<MAXB>(B.item0, B.count, gitem);
        const EncodeArgs& a = B.arg[tb];
        const int64_t item = gitem - B.item0[tb];
        const float beta = MAXB == 1 ? beta_s : a.beta;
        const int64_t jt = item / a.IB, ib = item % a.IB;
        const int64_t r0 = ib * TI;
        const int rows_valid = (int)min((int64_t)TI, a.rows - r0);
        const bool valid = row_l < rows_valid;

        if constexpr (SRC != 2) {
            const int64_t mkey = ((int64_t)tb << 48) | jt;  // tensor and tile column
            if (sm.mask_jt != mkey) {                       // block-uniform
                build_masks<N, SRC>(sm.mask, jt, a.seed);
                __syncthreads();
                if (tid == 0) sm.mask_jt = mkey;
            }
        }
        const bool arrived = mbar_wait(&sm.bar, (uint32_t)(iter & 1));
        if (!arrived) status_set(a.ws, kStTimeout);
        if (__syncthreads_or(!arrived)) {
            // the input copy did not complete in time: one more bounded wait (the copy may not
            // outlive the block), then leave; items after this one time out in their look-back
            if (tid == 0) mbar_wait(&sm.bar, (uint32_t)(iter & 1));
            break;
        }

        float2 P[H];
        float sumsq;
        load_row<N, SRC>(sm.buf, sm.mask, row_l, tau, P, sumsq);
        unsigned int next_claim = 0;
        if (tid == 0) next_claim = atomicAdd(&hdr->counter, 1u);  // used once the stage is free
        __syncthreads();  // [A] the stage is consumed (and, aliased, becomes the zig-zag scratch)
        if constexpr (G::SEPARATE_ZZ) {
            if (tid == 0) {
                sm.item_cur = next_claim;
                issue_tma_batch<N, SRC, MAXB>(sm, B, next_claim);
            }
        }

        // ---------------- per-tile scale, RHT, normalisation ----------------
        uint16_t sbits = 0;
        if constexpr (SRC != 2) {
            if constexpr (TPT == 2) {
                const float other = __shfl_xor_sync(0xffffffffu, sumsq, 1);
                sumsq = tau ? __fadd_rn(other, sumsq) : __fadd_rn(sumsq, other);  // first half + second half
            }
            const float s_rms = __fsqrt_rn(__fmul_rn(sumsq, 1.0f / (float)N));
            sbits = f32_to_bf16_bits(s_rms);
            const float sh = __uint_as_float((uint32_t)sbits << 16);
            const bool finite = isfinite(sh);
            if (!finite && valid && tau == 0) {
                status_set(a.ws, kStNonfinite);
                atomicAdd(&a.ws->nonfinite, 1u);
            }
            const bool zero_tile = !finite || sh < 1.2621774483536189e-29f;  // 2^-96
            if (zero_tile) sbits = 0;
            fwht_pairs<H>(P);
            const float t = __fmul_rn(sh, beta);
            const float rinv = __frcp_rn(t);
            const float cn = N == 64 ? 0.125f : (N == 128 ? __uint_as_float(0x3DB504F3u) : 0.0625f);
            const float g = zero_tile ? 0.0f : __fmul_rn(cn, rinv);
            const float2 g2 = make_float2(g, g);
#pragma unroll
            for (int m = 0; m < H; ++m) P[m] = f2mul(P[m], g2);
            // zero (and non-finite) tiles code as all zeros; a warp-uniform test keeps the
            // per-coefficient selects off the common path
            if (__any_sync(0xffffffffu, zero_tile)) {
#pragma unroll
                for (int m = 0; m < H; ++m) P[m] = zero_tile ? make_float2(0.0f, 0.0f) : P[m];
            }
        }

        // ---------------- dither counter words: KV row (b H + h, s), or (row, tile column) ----------------
        uint64_t dc = 0;
        uint32_t dc1 = 0;
        if constexpr (KV) {
            const int64_t r = r0 + row_l;
            const uint64_t Sv = (uint64_t)a.kv_S;
            dc = Sv ? (uint64_t)r % Sv + (uint64_t)a.kv_s0 : (uint64_t)r;
            dc1 = Sv ? (uint32_t)((uint64_t)r / Sv) : (uint32_t)jt;
        }

        // ---------------- (dither,) lattice + strip -> zig-zag scratch ----------------
        // Pair-block g8 is P[8 g8 .. 8 g8 + 8): lane x holds positions 8 g8 .., lane y positions
        // H + 8 g8 ...  The pair-blocks run in ROT rounds of one unrolled body over P[0 .. H/ROT):
        // after each round the next part of P moves down, so the instruction stream of the
        // quantizer is 1/ROT as long (unrolled over a whole tile it overflows the instruction cache).
        uint32_t A = 0, zor = 0;
        uint32_t cosbits = 0;  // coset bit of local block lb at bit lb (E8)
        auto store_group = [&](int group, const int32_t (&sym)[8]) {
            uint32_t z[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                z[i] = zigzag(sym[i]);
                A += z[i];
                if constexpr (SRC == 2) zor |= z[i];
            }
            *zz_slot(zzs, group, tid) =
                make_uint4(z[0] | (z[1] << 16), z[2] | (z[3] << 16), z[4] | (z[5] << 16), z[6] | (z[7] << 16));
        };
        constexpr int ROT = H >= 16 ? HQ_QUANT_ROT : 1;
        constexpr int PB = H / 8 / ROT;  // pair-blocks per round
#pragma unroll 1
        for (int rr = 0; rr < ROT; ++rr) {
            uint32_t rare = 0;  // E8: blocks of this round to redo with the plain rule (bit 2 gb + lane)
#pragma unroll
            for (int gb = 0; gb < PB; ++gb) {
                const int g8 = rr * PB + gb;
                if constexpr (LAT == HQ_E8) {
                    float2 p8[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) p8[i] = P[gb * 8 + i];
                    if constexpr (KV) {
                        // dither: the block of lane x is groups 2 g8, 2 g8 + 1 of this thread's
                        // positions, lane y the same H/4 groups further on
                        float Ux[8], Uy[8];
                        dither_e8(a.rk, dc1, dc, (uint32_t)(tau * (V / 4) + 2 * g8), Ux);
                        dither_e8(a.rk, dc1, dc, (uint32_t)(tau * (V / 4) + H / 4 + 2 * g8), Uy);
#pragma unroll
                        for (int i = 0; i < 8; ++i) p8[i] = make_float2(__fadd_rn(p8[i].x, Ux[i]), __fadd_rn(p8[i].y, Uy[i]));
                    }
                    int32_t sx[8], sy[8], vx[8], vy[8];
                    uint32_t cx, cy, rare2;
                    e8_pair_symbols<SRC == 2>(p8, sx, sy, cx, cy, vx, vy, rare2);
                    rare |= rare2 << (2 * gb);
                    if constexpr (SRC == 2) {
                        if (valid && a.v_out) {
                            int32_t* vo = a.v_out + (r0 + row_l) * (int64_t)N + tau * V;
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                vo[g8 * 8 + i] = vx[i];
                                vo[H + g8 * 8 + i] = vy[i];
                            }
                        }
                    }
                    cosbits |= (cx << g8) | (cy << (H / 8 + g8));
                    store_group(g8, sx);
                    store_group(H / 8 + g8, sy);
                } else {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float u8[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) u8[i] = half ? P[gb * 8 + i].y : P[gb * 8 + i].x;
                        // dither of the two groups (positions half H + 8 g8 + 4 bb ..): added to u,
                        // or for A2 to (P, Q) = (2 u0, u1 K), the coordinates of its quantizer
                        float U8[8];
                        if constexpr (KV) {
                            // groups 2 (g8 + ...) and the next one: one Philox block
                            dither_pair<LAT>(a.rk, dc1, dc, (uint32_t)(tau * (V / 4) + half * (H / 4) + 2 * g8) >> 1, U8);
                            if constexpr (LAT != HQ_A2) {
#pragma unroll
                                for (int i = 0; i < 8; ++i) u8[i] = __fadd_rn(u8[i], U8[i]);
                            }
                        }
                        int32_t sym[8];
#pragma unroll
                        for (int b = 0; b < 8 / D; ++b) {
                            int32_t v[D];
                            if constexpr (KV && LAT == HQ_A2) {
                                int32_t v2[2];
                                q_a2_pq(__fadd_rn(__fmul_rn(2.0f, u8[2 * b]), U8[2 * b]),
                                        __fadd_rn(__fmul_rn(u8[2 * b + 1], kA2K), U8[2 * b + 1]), v2);
                                v[0] = v2[0];
                                v[1] = v2[1];
                                strip_block<LAT>(v, sym + b * D);
                            } else {
                                quantize_strip<LAT, SRC == 2>(u8 + b * D, sym + b * D, v);
                            }
                            if constexpr (SRC == 2) {
                                if (valid && a.v_out) {
                                    int32_t* vo =
                                        a.v_out + (r0 + row_l) * (int64_t)N + tau * V + half * H + g8 * 8 + b * D;
#pragma unroll
                                    for (int i = 0; i < D; ++i) vo[i] = v[i];
                                }
                            }
                        }
                        store_group(half * (H / 8) + g8, sym);
                    }
                }
            }
            if constexpr (LAT == HQ_E8) {
                // blocks within 2^-16 of a coset tie, or whose fix-up meets the key floor: redo
                // them with the plain rule and replace their symbols, coset bit and codes
                if (rare) {
#pragma unroll
                    for (int gb = 0; gb < PB; ++gb) {
#pragma unroll
                        for (int ln = 0; ln < 2; ++ln) {
                            if (!((rare >> (2 * gb + ln)) & 1u)) continue;
                            const int g8 = rr * PB + gb;
                            float u8[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) u8[i] = ln ? P[gb * 8 + i].y : P[gb * 8 + i].x;
                            if constexpr (KV) {
                                float U[8];
                                dither_e8(a.rk, dc1, dc, (uint32_t)(tau * (V / 4) + ln * (H / 4) + 2 * g8), U);
#pragma unroll
                                for (int i = 0; i < 8; ++i) u8[i] = __fadd_rn(u8[i], U[i]);
                            }
                            int32_t s8[8], v8[8];
                            const uint32_t c = e8_symbols<SRC == 2>(u8, s8, v8);
                            const int slot = ln * (H / 8) + g8;
                            const uint4 old = *zz_slot(zzs, slot, tid);
                            A -= (old.x & 0xFFFFu) + (old.x >> 16) + (old.y & 0xFFFFu) + (old.y >> 16) +
                                 (old.z & 0xFFFFu) + (old.z >> 16) + (old.w & 0xFFFFu) + (old.w >> 16);
                            store_group(slot, s8);
                            const int cb = ln * (H / 8) + g8;
                            cosbits = (cosbits & ~(1u << cb)) | (c << cb);
                            if constexpr (SRC == 2) {
                                if (valid && a.v_out) {
                                    int32_t* vo = a.v_out + (r0 + row_l) * (int64_t)N + tau * V + ln * H + g8 * 8;
#pragma unroll
                                    for (int i = 0; i < 8; ++i) vo[i] = v8[i];
                                }
                            }
                        }
                    }
                }
            }
            if (ROT > 1 && rr + 1 < ROT) {
#pragma unroll
                for (int m = 0; m < H - H / ROT; ++m) P[m] = P[m + H / ROT];
            }
        }

        // ---------------- Rice parameter and tile length ----------------
        if constexpr (TPT == 2) A += __shfl_xor_sync(0xffffffffu, A, 1);
        const int k = rice_k(A, G::LOG2N);
        // sum q = sum (zz >> k) on both 16-bit halves of the packed scratch words at once: the k rule
        // keeps the tile's sum below 2n (at most n when k is capped), so neither half carries over
        const uint32_t hm = (0xFFFFu >> k) * 0x00010001u;
        uint32_t sq2 = 0;
#pragma unroll 4
        for (int g = 0; g < V / 8; ++g) {
            const uint4 w = *zz_slot(zzs, g, tid);
            sq2 += ((w.x >> k) & hm) + ((w.y >> k) & hm) + ((w.z >> k) & hm) + ((w.w >> k) & hm);
        }
        const uint32_t sq = (sq2 & 0xFFFFu) + (sq2 >> 16);
        uint32_t sq_tile = sq;
        if constexpr (TPT == 2) sq_tile += __shfl_xor_sync(0xffffffffu, sq, 1);
        const uint32_t L = (uint32_t)COSB + (uint32_t)N * (uint32_t)(k + 1) + sq_tile;
        // the staging stream holds at most LMAX bits per tile; longer tiles (only reachable with
        // caller-given coefficients of huge magnitude) are reported and left out
        bool fits_tile = L <= (uint32_t)G::LMAX && k <= G::KMAX;
        if constexpr (SRC == 2) {
            if constexpr (TPT == 2) zor |= __shfl_xor_sync(0xffffffffu, zor, 1);
            fits_tile = fits_tile && zor <= 0xFFFFu;
        }
        if (!fits_tile && valid && tau == 0) status_set(a.ws, kStRange);
        const bool emit = valid && fits_tile;
        if (tau == 0) sm.Ls[row_l] = emit ? L : 0u;
        __syncthreads();  // [B]

        // ---------------- chunk layout of the item (warp 0) ----------------
        if (warp == 0) {
            uint32_t acc_words = 0;
#pragma unroll
            for (int ch = 0; ch < G::CH; ++ch) {
                const uint32_t v = sm.Ls[ch * 32 + lane];
                uint32_t incl = v;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                sm.rowoff[ch * 32 + lane] = incl - v;
                const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
                if (lane == 0) sm.chunkoff[ch] = acc_words;
                acc_words += (tot + 31) >> 5;
            }
            uint32_t bits = 0;
            if constexpr (COUNT) {
#pragma unroll
                for (int ch = 0; ch < G::CH; ++ch) bits += sm.Ls[ch * 32 + lane];
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) bits += __shfl_xor_sync(0xffffffffu, bits, o);
            }
            if (lane == 0) {
                sm.chunkoff[G::CH] = acc_words;
                sm.item_words = acc_words;
                if constexpr (COUNT) {
                    atomicAdd(&a.ws->count_bits, (unsigned long long)bits);
                } else {
                    const unsigned long long st = ((item == 0 ? 2ull : 1ull) << 32) | acc_words;
#ifdef HQ_TEST_HOOKS
                    if (item != a.test_silent_item)
#endif
                        st_relaxed_u64(a.states + item, st);
                }
            }
        }
        __syncthreads();  // [C]
        if constexpr (COUNT) {
            if (!G::SEPARATE_ZZ && tid == 0) {
                sm.item_cur = next_claim;
                issue_tma_batch<N, SRC, MAXB>(sm, B, next_claim);
            }
            __syncthreads();
            continue;
        }

        // the staging stream is all zero here: cleared once at start, then by each copy-out
        const uint32_t item_words = sm.item_words;

        // ---------------- Rice bits into the staging stream ----------------
        if (emit) {
            const int ch = row_l / kChunkTiles;
            const int tile0 = (int)(sm.chunkoff[ch] * 32u + sm.rowoff[row_l]);  // tile start bit
            if constexpr (LAT == HQ_E8) {
                const int cpos = tile0 + tau * (V / 8);
                const uint32_t lo = cosbits << (cpos & 31);
                const uint32_t hi = (cpos & 31) ? (cosbits >> (32 - (cpos & 31))) : 0u;
                if (lo) atomicOr(&sm.stg[cpos >> 5], lo);
                if (hi) atomicOr(&sm.stg[(cpos >> 5) + 1], hi);
            }
            const uint32_t km = (1u << k) - 1u;
            const uint32_t one = 1u << k;
            if constexpr (TPT == 1) {
                // both halves in one loop: the forward writer (first half, from the tile start)
                // and the backward writer (second half, from the tile's last bit) are independent
                BitWriter<true> bf;
                BitWriter<false> bb;
                bf.begin(sm.stg, tile0 + COSB);
                bb.begin(sm.stg, tile0 + (int)L - 1);
#pragma unroll 1
                for (int g = 0; g < N / 16; ++g) {
                    const uint4 wf = *zz_slot(zzs, g, tid);
                    const uint4 wb = *zz_slot(zzs, V / 8 - 1 - g, tid);
                    put4<true>(bf, wf.x & 0xFFFFu, wf.x >> 16, wf.y & 0xFFFFu, wf.y >> 16, k, km, one);
                    put4<false>(bb, wb.w >> 16, wb.w & 0xFFFFu, wb.z >> 16, wb.z & 0xFFFFu, k, km, one);
                    put4<true>(bf, wf.z & 0xFFFFu, wf.z >> 16, wf.w & 0xFFFFu, wf.w >> 16, k, km, one);
                    put4<false>(bb, wb.y >> 16, wb.y & 0xFFFFu, wb.x >> 16, wb.x & 0xFFFFu, k, km, one);
                }
                bf.finish();
                bb.finish();
            } else if (tau == 0) {
                // first half, forward from the tile start
                BitWriter<true> bw;
                bw.begin(sm.stg, tile0 + COSB);
                constexpr int G8 = V / 8;
#pragma unroll 1
                for (int g = 0; g < G8; ++g) {
                    const uint4 w = *zz_slot(zzs, g, tid);
                    put4<true>(bw, w.x & 0xFFFFu, w.x >> 16, w.y & 0xFFFFu, w.y >> 16, k, km, one);
                    put4<true>(bw, w.z & 0xFFFFu, w.z >> 16, w.w & 0xFFFFu, w.w >> 16, k, km, one);
                }
                bw.finish();
            }
            else {
                // second half, backward from the tile's last bit (symbols in decreasing order)
                BitWriter<false> bw;
                bw.begin(sm.stg, tile0 + (int)L - 1);
                constexpr int G0 = 0;
#pragma unroll 1
                for (int g = V / 8 - 1; g >= G0; --g) {
                    const uint4 w = *zz_slot(zzs, g, tid);
                    put4<false>(bw, w.w >> 16, w.w & 0xFFFFu, w.z >> 16, w.z & 0xFFFFu, k, km, one);
                    put4<false>(bw, w.y >> 16, w.y & 0xFFFFu, w.x >> 16, w.x & 0xFFFFu, k, km, one);
                }
                bw.finish();
            }
        }
        __syncthreads();  // [E] scratch free: load the next item (aliased scratch)
        if (!G::SEPARATE_ZZ && tid == 0) {
            sm.item_cur = next_claim;
            issue_tma_batch<N, SRC, MAXB>(sm, B, next_claim);
        }

        // ---------------- look-back for the item's word offset (warp 0) ----------------
        if (warp == 0) {
            uint32_t excl = 0;
            if (item > 0) {
                int64_t j = item - 1;
                uint32_t spins = 0;
                while (true) {
                    const int64_t idx = j - lane;
                    const unsigned long long st = idx >= 0 ? ld_relaxed_u64(a.states + idx) : (2ull << 32);
                    const uint32_t flag = (uint32_t)(st >> 32);
                    const uint32_t pmask = __ballot_sync(0xffffffffu, flag == 2u);
                    const uint32_t xmask = __ballot_sync(0xffffffffu, flag == 0u);
                    const int firstP = pmask ? __ffs(pmask) - 1 : 32;
                    const uint32_t need = firstP >= 31 ? 0xffffffffu : ((2u << firstP) - 1u);
                    if (xmask & need) {
                        if (++spins > kSpinLimit) {
                            if (lane == 0) status_set(a.ws, kStTimeout);
                            break;
                        }
                        __nanosleep(32);
                        continue;
                    }
                    uint32_t val = lane <= firstP ? (uint32_t)st : 0u;
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1) val += __shfl_xor_sync(0xffffffffu, val, o);
                    excl += val;
                    if (firstP < 32) break;
                    j -= 32;
                }
            }
            if (lane == 0) {
#ifdef HQ_TEST_HOOKS
                if (item > 0 && item != a.test_silent_item)
#else
                if (item > 0)
#endif
                    st_relaxed_u64(a.states + item, (2ull << 32) | (unsigned long long)(excl + item_words));
                sm.base = excl;
            }
        }
        __syncthreads();  // [F]

        // ---------------- store: bits, chunk offsets, scale, meta ----------------
        const uint32_t base = sm.base;
        const bool fits = (int64_t)base + (int64_t)item_words <= a.cap_words;
        if (fits) {
            for (uint32_t w = tid; w < item_words; w += kThreads) {
                a.bits[base + w] = sm.stg[w];
                sm.stg[w] = 0u;
            }
        } else {
            for (uint32_t w = tid; w < item_words; w += kThreads) sm.stg[w] = 0u;
            if (tid == 0) status_set(a.ws, kStCapacity);
        }
        const int nch = (rows_valid + kChunkTiles - 1) / kChunkTiles;
        const int64_t c0 = jt * a.RB + ib * G::CH;
        if (tid < nch) a.chunk_word[c0 + tid] = base + sm.chunkoff[tid];
        if (item == a.items - 1 && tid == 0) {
            a.chunk_word[a.C] = base + item_words;
            atomicMax(&a.ws->needed, (unsigned long long)(base + item_words));
        }
        if (valid && tau == 0) {
            const int64_t t = jt * a.rows + r0 + row_l;
            if (a.scale) a.scale[t] = sbits;
            a.meta[t] = (uint16_t)((uint32_t)k | (sq_tile << 4));
        }
    }
}

}  // namespace hq
