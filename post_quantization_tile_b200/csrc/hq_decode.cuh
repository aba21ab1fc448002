// hq_decode.cuh -- decode kernel of the HyperQuant tile codec (inverse of Methodology steps 1-4).
//
// A block decodes one item (TI rows of one tile column = TI/32 chunks) at a time.  The item's
// words are independent of every other item thanks to the stored chunk offsets, so items are
// assigned statically.  Thread 0 bulk-copies the item's 16-byte-aligned word range into shared
// memory (two-stage ring); every thread parses its tile's Rice codes -- the first half forward
// from the tile start, the second half backward from the tile end, so two threads can share a
// 256-tile -- rebuilds the integer lattice codes, applies the inverse transform D H_n p and the
// scale, and writes its row into a swizzled staging box that one TMA store sends to HBM.
#pragma once
#include "hq_common.cuh"
#include "hq_encode.cuh"
#include "hq_lattice.cuh"

namespace hq {

struct DecodeArgs {
    int64_t rows, cols;
    float beta;
    uint64_t seed;
    int64_t kv_S;
    int64_t items, IB, RB, C;
    const uint16_t* scale;
    const uint16_t* meta;
    const uint32_t* chunk_word;
    const uint32_t* bits;
    int64_t cap_words;
    WsHeader* ws;
    uint32_t rk[20];  // Philox round keys of `seed` (key words 0, 1 of rounds 0 .. 9), for the dither
    float* g_out;     // int8-code output: group scale of tile (r, jt) at g_out[jt rows + r]
    int64_t kv_s0;    // KV: position of the code's first token in every sequence
};

// Several codes in one launch, as EncodeBatch: code t takes the global items item0[t] ..
// item0[t + 1] - 1 (assigned to the blocks in turn); the header (status) is shared.
template <int MAXB>
struct DecodeBatch {
    CUtensorMap map[MAXB];
    DecodeArgs arg[MAXB];
    int64_t item0[MAXB + 1];
    int32_t count;
};

// DST: 0 bf16, 1 fp32, 2 int8 lattice codes (RHT domain, no transform), 3 fp32 lattice points minus
// the dither in u units (no transform, no scale: the input of a dense inverse rotation)
template <int N, int DST>
struct DecGeom {
    static constexpr int TPT = dec_tpt(N);
    static constexpr int V = N / TPT;
    static constexpr int H = V / 2;
    static constexpr int TI = kThreads / TPT;
    static constexpr int CH = TI / kChunkTiles;
    static constexpr int ES = DST == 0 ? 2 : (DST == 2 ? 1 : 4);
    static constexpr int ROWB = N * ES;
    static constexpr int NB = ROWB / 128;
    static constexpr int OUT = NB * TI * 128;
    static constexpr int ZZ = V * 2 * kThreads;  // zig-zag scratch, aliases the output box
    static constexpr int BUF = OUT > ZZ ? OUT : ZZ;
    // streams written by the encoder have k <= 9 (step range); the buffer takes k <= 11 and
    // larger items are reported as corrupt
    static constexpr int LMAX = N / 8 + 12 * N + 2 * N;
    static constexpr int GUARD = 4;  // words before and after the copied range
    static constexpr int IN_WORDS = (TI * ((LMAX + 31) / 32) + CH + 8 + 2 * GUARD + 3) / 4 * 4;
    static constexpr int MASKS = DST == 0 ? N / 2 : (DST == 1 ? N : 4);
    static constexpr int LOG2N = N == 64 ? 6 : (N == 128 ? 7 : 8);
    // input stages: one (the next item is fetched once this one is parsed) or two (fetched a
    // whole item ahead, at the cost of shared memory)
    static constexpr int STAGES = HQ_DEC_STAGES;
};

template <int N, int DST>
struct DecSmem {
    using G = DecGeom<N, DST>;
    alignas(1024) unsigned char buf[G::BUF];       // zig-zag scratch, then the output TMA box
    alignas(16) uint32_t in[G::STAGES][G::IN_WORDS];  // the items' words
    alignas(16) uint32_t mask[G::MASKS];
    uint32_t Ls[G::TI];
    uint32_t rowoff[G::TI];
    uint32_t chunkbase[G::STAGES][G::CH + 1];  // chunk start word relative to the copied range
    int64_t item_ring[G::STAGES];
    int32_t ok_ring[G::STAGES];
    int64_t mask_jt;
    alignas(8) uint64_t bar[G::STAGES];
};

template <int N, int DST>
__device__ __forceinline__ void build_masks_out(uint32_t* mask, int64_t jt, uint64_t seed)
{
    using G = DecGeom<N, DST>;
    for (int w = threadIdx.x; w < G::MASKS; w += kThreads) {
        const int per = DST == 0 ? 2 : 1;
        uint32_t m = 0;
#pragma unroll
        for (int e = 0; e < per; ++e) {
            const int64_t J = jt * N + (int64_t)w * per + e;
            const uint4 ph = philox4x32_10(make_uint4((uint32_t)((uint64_t)J >> 7), 0u, 0u, 0u), (uint32_t)seed,
                                           (uint32_t)(seed >> 32));
            const int wsel = (int)((J & 127) >> 5);
            const uint32_t word = wsel == 0 ? ph.x : (wsel == 1 ? ph.y : (wsel == 2 ? ph.z : ph.w));
            m |= ((word >> (J & 31)) & 1u) << (DST == 0 ? (e ? 31 : 15) : 31);
        }
        mask[w] = m;
    }
}

// Producer (one thread): copy the words of item `it` into the input stage.  An item whose
// chunk offsets are inconsistent with the buffers is flagged and decoded as zeros.
template <int N, int DST>
__device__ __forceinline__ void issue_item(DecSmem<N, DST>& sm, const DecodeArgs& a, int s, int64_t it)
{
    using G = DecGeom<N, DST>;
    sm.item_ring[s] = it;
    sm.ok_ring[s] = 0;
    if (it >= a.items) return;
    const int64_t jt = it / a.IB, ib = it % a.IB;
    const int64_t r0 = ib * G::TI;
    const int rows_valid = (int)min((int64_t)G::TI, a.rows - r0);
    const int nch = (rows_valid + kChunkTiles - 1) / kChunkTiles;
    const int64_t c0 = jt * a.RB + ib * G::CH;
    const int64_t w0 = a.chunk_word[c0];
    const int64_t w1 = a.chunk_word[c0 + nch];
    const int64_t lo = w0 & ~(int64_t)3;
    const int64_t hi = (w1 + 3) & ~(int64_t)3;
    const bool good = w1 >= w0 && hi <= a.cap_words && (hi - lo) <= (int64_t)(G::IN_WORDS - 2 * G::GUARD);
    for (int ch = 0; ch <= nch; ++ch) sm.chunkbase[s][ch] = (uint32_t)(a.chunk_word[c0 + ch] - lo + G::GUARD);
    if (!good) status_set(a.ws, kStCorrupt);
    const uint32_t bytes = (uint32_t)((hi - lo) * 4);
    if (good && bytes) {
        sm.ok_ring[s] = 1;
        mbar_arrive_expect_tx(&sm.bar[s], bytes);
        bulk_load_1d(sm.in[s] + G::GUARD, a.bits + lo, bytes, &sm.bar[s]);
    } else {
        sm.ok_ring[s] = good ? 1 : 0;
        mbar_arrive(&sm.bar[s]);  // complete the phase without data
    }
}

// the copy of global item g of a batch into stage s (the ring holds global item numbers)
template <int N, int DST, int MAXB>
__device__ __forceinline__ void issue_item_batch(DecSmem<N, DST>& sm, const DecodeBatch<MAXB>& B, int s, int64_t g)
{
    if (g >= B.item0[B.count]) {
        sm.item_ring[s] = g;
        sm.ok_ring[s] = 0;
        return;
    }
    const int t = MAXB == 1 ? 0 : batch_tensor<MAXB>(B.item0, B.count, g);
    issue_item<N, DST>(sm, B.arg[t], s, g - B.item0[t]);
    sm.item_ring[s] = g;
}

template <int N, int LAT, bool KV, int DST, int MAXB>
__global__ void __launch_bounds__(kThreads, kMinBlocks) decode_kernel(const __grid_constant__ DecodeBatch<MAXB> B)
{
    using G = DecGeom<N, DST>;
    using SM = DecSmem<N, DST>;
    constexpr int TPT = G::TPT, V = G::V, H = G::H, TI = G::TI, D = Lat<LAT>::d;
    constexpr int COSB = LAT == HQ_E8 ? N / 8 : 0;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // TMA boxes with 128-byte swizzle need 1024-byte aligned shared memory: align by hand
    SM& sm = *reinterpret_cast<SM*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);

    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int row_l = tid / TPT;
    const int tau = tid % TPT;

    if (tid == 0) {
        for (int s = 0; s < G::STAGES; ++s) mbar_init(&sm.bar[s], 1);
        fence_mbar_init();
        sm.mask_jt = -1;
        for (int s = 0; s < G::STAGES; ++s)
            issue_item_batch<N, DST, MAXB>(sm, B, s, (int64_t)blockIdx.x + (int64_t)s * gridDim.x);
    }
    __syncthreads();
    const int64_t total = B.item0[B.count];

    for (int iter = 0;; ++iter) {
        const int st = iter % G::STAGES;
        const uint32_t parity = (uint32_t)((iter / G::STAGES) & 1);
        const int64_t gitem = sm.item_ring[st];
        if (gitem >= total) break;
        // this item's code; below, `item` is its index within that code
        const int tb = MAXB == 1 ? 0 : batch_tensor<MAXB>(B.item0, B.count, gitem);
        const DecodeArgs& a = B.arg[tb];
        const CUtensorMap& tmap = B.map[tb];
        const int64_t item = gitem - B.item0[tb];
        const int64_t jt = item / a.IB, ib = item % a.IB;
        const int64_t r0 = ib * TI;
        const int rows_valid = (int)min((int64_t)TI, a.rows - r0);
        const bool valid = row_l < rows_valid;
        const bool stage_ok = sm.ok_ring[st] != 0;

        const int64_t mkey = ((int64_t)tb << 48) | jt;  // code and tile column
        if (DST < 2 && sm.mask_jt != mkey) {
            build_masks_out<N, DST>(sm.mask, jt, a.seed);
            __syncthreads();
            if (tid == 0) sm.mask_jt = mkey;
        }

        // tile lengths from meta -> bit offsets within the chunks (warp 0 scans each chunk)
        const int64_t t = jt * a.rows + r0 + row_l;
        uint32_t L = 0, mt = 0;
        if (valid) {
            mt = a.meta[t];
            L = (uint32_t)COSB + (uint32_t)N * ((mt & 15u) + 1u) + (mt >> 4);
        }
        const uint16_t sbits = valid ? a.scale[t] : (uint16_t)0;
        if (tau == 0) sm.Ls[row_l] = L;
        if (tid == 0) bulk_wait_read0();  // the previous output box has left shared memory
        __syncthreads();
        if (warp == 0) {
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
            }
        }
        const bool arrived = mbar_wait(&sm.bar[st], parity);
        if (!arrived) status_set(a.ws, kStTimeout);
        if (__syncthreads_or(!arrived)) {
            // a copy did not complete in time: issue nothing more, give every copy still in flight
            // one more bounded wait (no copy may outlive the block), and leave
            if (tid == 0) {
                for (int k = 0; k < G::STAGES; ++k) {
                    const int sk = (iter + k) % G::STAGES;
                    if (sm.item_ring[sk] < total) mbar_wait(&sm.bar[sk], (uint32_t)(((iter + k) / G::STAGES) & 1));
                }
            }
            break;
        }

        // ---------------- parse: Rice codes -> zig-zag scratch ----------------
        uint32_t cosbits = 0;
        bool ok = valid && stage_ok;
        uint32_t sq_part = 0, sq_want = 0;
        const int k = (int)(mt & 15u);
        if (ok) {
            const uint32_t sq_meta = mt >> 4;
            const uint32_t pow2k = 1u << k;
            sq_want = sq_meta;
            const int ch = row_l / kChunkTiles;
            const int tile0 = (int)(sm.chunkbase[st][ch] * 32u + sm.rowoff[row_l]);
            const uint32_t* in = sm.in[st];
            if constexpr (LAT == HQ_E8) {
                const int cpos = tile0 + tau * (V / 8);
                const int cw = min(max(cpos >> 5, 0), G::IN_WORDS - 2);
                const unsigned long long two = ((unsigned long long)in[cw + 1] << 32) | in[cw];
                cosbits = (uint32_t)(two >> (cpos & 31)) & ((V / 8) >= 32 ? 0xffffffffu : ((1u << (V / 8)) - 1u));
            }
            uint32_t sq = 0;
            if constexpr (TPT == 1) {
                // both halves in one loop: independent forward and backward readers
                BitReader<true> rf;
                BitReader<false> rb;
                rf.begin(in, tile0 + COSB, G::IN_WORDS - 1);
                rb.begin(in, tile0 + (int)L - 1, G::IN_WORDS - 1);
#pragma unroll 1
                for (int g = 0; g < N / 8; ++g) {
                    uint32_t zf[4], zb[4];
                    rf.refill();
                    rb.refill();
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        zf[j] = get_code<true>(rf, k, pow2k, sq_meta, ok);
                        zb[3 - j] = get_code<false>(rb, k, pow2k, sq_meta, ok);
                    }
                    uint2* pf = reinterpret_cast<uint2*>(zz_slot(sm.buf, g >> 1, tid)) + (g & 1);
                    uint2* pb = reinterpret_cast<uint2*>(zz_slot(sm.buf, V / 8 - 1 - (g >> 1), tid)) + (1 - (g & 1));
                    *pf = make_uint2(zf[0] | (zf[1] << 16), zf[2] | (zf[3] << 16));
                    *pb = make_uint2(zb[0] | (zb[1] << 16), zb[2] | (zb[3] << 16));
                }
                // the codes' unary parts: the bits taken minus one stop bit and k remainder bits per code
                sq = (uint32_t)(rf.consumed() + rb.consumed() - N * (k + 1));
            } else if (tau == 0) {
                BitReader<true> br;
                br.begin(in, tile0 + COSB, G::IN_WORDS - 1);
                constexpr int G8 = V / 8;
#pragma unroll 1
                for (int g = 0; g < G8; ++g) {
                    uint32_t z[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if ((j & 3) == 0) br.refill();
                        z[j] = get_code<true>(br, k, pow2k, sq_meta, ok);
                    }
                    *zz_slot(sm.buf, g, tid) = make_uint4(z[0] | (z[1] << 16), z[2] | (z[3] << 16),
                                                          z[4] | (z[5] << 16), z[6] | (z[7] << 16));
                }
                sq = (uint32_t)(br.consumed() - V * (k + 1));
            }
            else {
                BitReader<false> br;
                br.begin(in, tile0 + (int)L - 1, G::IN_WORDS - 1);
                constexpr int G0 = 0;
#pragma unroll 1
                for (int g = V / 8 - 1; g >= G0; --g) {
                    uint32_t z[8];
#pragma unroll
                    for (int j = 7; j >= 0; --j) {
                        if ((j & 3) == 3) br.refill();
                        z[j] = get_code<false>(br, k, pow2k, sq_meta, ok);
                    }
                    *zz_slot(sm.buf, g, tid) = make_uint4(z[0] | (z[1] << 16), z[2] | (z[3] << 16),
                                                          z[4] | (z[5] << 16), z[6] | (z[7] << 16));
                }
                sq = (uint32_t)(br.consumed() - V * (k + 1));
            }
            sq_part = sq;
        }
        if constexpr (TPT == 2) sq_part += __shfl_xor_sync(0xffffffffu, sq_part, 1);
        if (ok && sq_part != sq_want) ok = false;
        if constexpr (TPT == 2) {
            const int other = __shfl_xor_sync(0xffffffffu, (int)ok, 1);
            ok = ok && other;
        }
        if (valid && stage_ok && !ok) status_set(a.ws, kStCorrupt);
        __syncthreads();  // the input stage is consumed: fetch the next item's words
        if (tid == 0) issue_item_batch<N, DST, MAXB>(sm, B, st, gitem + (int64_t)G::STAGES * gridDim.x);

        // ---------------- codes -> lattice point (float pairs) ----------------
        float2 P[H];
        uint32_t out_of_int8 = 0u;  // int8-code output: some code of the tile is outside [-127, 127]
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int g8 = 0; g8 < H / 8; ++g8) {
                const uint4 w = *zz_slot(sm.buf, half * (H / 8) + g8, tid);
                const uint32_t zw[4] = {w.x, w.y, w.z, w.w};
                if constexpr (LAT == HQ_E8 && DST != 2) {
                    // zig-zag -> doubled E8 point in one pass: 2 unzigzag(z) = z ^ -(z & 1), so
                    // v_i = 2 w_i + c = (z_i ^ -(z_i & 1)) + c for i < 7, the parity p of w_0 .. w_6
                    // is bit 1 of the XOR of those, and v_7 = 2 (2 h + p) + c; the binary32 value
                    // comes from adding 1.5 * 2^23 in the integer domain (exact, |v| < 2^22)
                    const int cm = (int)((cosbits >> (half * (H / 8) + g8)) & 1u) + __float_as_int(kMagic);
                    int t[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t z = (zw[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
                        t[j] = (int)(z ^ (0u - (z & 1u)));
                    }
                    const int p2 = (t[0] ^ t[1] ^ t[2] ^ t[3] ^ t[4] ^ t[5] ^ t[6]) & 2;  // 2 p
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int vb = i < 7 ? t[i] + cm : 2 * t[7] + p2 + cm;
                        const float f = __int_as_float(vb) - kMagic;  // !ok: zeroed below
                        if (half) P[g8 * 8 + i].y = f;
                        else P[g8 * 8 + i].x = f;
                    }
                } else {
                    int32_t sym[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) sym[j] = unzigzag((zw[j >> 1] >> (16 * (j & 1))) & 0xFFFFu);  // !ok: zeroed below
#pragma unroll
                    for (int b = 0; b < 8 / D; ++b) {
                        const int pos = half * H + g8 * 8 + b * D;
                        int32_t v[D];
                        unstrip_block<LAT>(sym + b * D, (cosbits >> (pos / 8)) & 1u, v);
#pragma unroll
                        for (int i = 0; i < D; ++i) {
                            if constexpr (DST == 2) out_of_int8 |= (uint32_t)(v[i] + 127) > 254u ? 1u : 0u;
                            float f = __int_as_float(v[i] + __float_as_int(kMagic)) - kMagic;  // exact, |v| < 2^22
                            // A2: (P, Q) -> u after the dither is taken off (in P, Q coordinates)
                            if constexpr (LAT == HQ_A2 && !KV) f = (i & 1) ? __fmul_rn(f, 0.866025403784438647f) : __fmul_rn(f, 0.5f);
                            if (half) P[g8 * 8 + b * D + i].y = f;
                            else P[g8 * 8 + b * D + i].x = f;
                        }
                    }
                }
            }
        }
        if constexpr (DST == 2) {
            // ---------------- int8 lattice codes + group scale (no transform) ----------------
            if constexpr (TPT == 2) out_of_int8 |= __shfl_xor_sync(0xffffffffu, out_of_int8, 1);
            const bool keep = ok && out_of_int8 == 0u;
            if (valid && ok && out_of_int8 && tau == 0) status_set(a.ws, kStRange);
            if (valid && tau == 0) {
                const float sh = __uint_as_float((uint32_t)sbits << 16);
                const float cn = N == 64 ? 0.125f : (N == 128 ? __uint_as_float(0x3DB504F3u) : 0.0625f);
                float gs = __fmul_rn(__fmul_rn(sh, a.beta), cn);
                if constexpr (LAT == HQ_E8) gs = __fmul_rn(gs, 0.5f);
                a.g_out[jt * a.rows + r0 + row_l] = gs;
            }
            __syncthreads();  // every thread has read its scratch: the box may be overwritten
            // 16 codes per 16-byte chunk; chunk c of this thread's half-row holds elements 16 c ..
#pragma unroll
            for (int c = 0; c < H / 16; ++c) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int e0 = tau * V + half * H + 16 * c;
                    uint32_t w[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t b4 = 0u;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float f = half ? P[16 * c + 4 * q + e].y : P[16 * c + 4 * q + e].x;
                            b4 |= ((uint32_t)__float2int_rn(f) & 0xFFu) << (8 * e);
                        }
                        w[q] = keep ? b4 : 0u;
                    }
                    const int cg = e0 / 16;
                    *reinterpret_cast<uint4*>(sm.buf + (cg >> 3) * (TI * 128) + swz(row_l, cg & 7)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        } else {
            if constexpr (KV) {
                // the dither of this tile, taken off in the quantizer's coordinates: doubled u for E8
                // (minus 2U), (P, Q) for A2 (then scaled to u), u for Z and D4
                const int64_t r = r0 + row_l;
                const uint64_t Sv = (uint64_t)a.kv_S;
                const uint64_t dc = Sv ? (uint64_t)r % Sv + (uint64_t)a.kv_s0 : (uint64_t)r;
                const uint32_t dc1 = Sv ? (uint32_t)((uint64_t)r / Sv) : (uint32_t)jt;
                if constexpr (LAT == HQ_E8) {
    #pragma unroll
                    for (int g8 = 0; g8 < H / 8; ++g8) {
    #pragma unroll 1
                        for (int half = 0; half < 2; ++half) {  // rolled: half the Philox code
                            float U[8];
                            dither_e8(a.rk, dc1, dc, (uint32_t)(tau * (V / 4) + half * (H / 4) + 2 * g8), U);
    #pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                float2& q = P[8 * g8 + i];
                                if (half) q.y = __fadd_rn(q.y, -__fmul_rn(2.0f, U[i]));
                                else q.x = __fadd_rn(q.x, -__fmul_rn(2.0f, U[i]));
                            }
                        }
                    }
                } else {
    #pragma unroll
                    for (int b2 = 0; b2 < H / 8; ++b2) {
    #pragma unroll 1
                        for (int half = 0; half < 2; ++half) {  // rolled: half the Philox code
                            // groups 2 b2, 2 b2 + 1 of this half: one Philox block
                            float U[8];
                            dither_pair<LAT>(a.rk, dc1, dc, (uint32_t)(tau * (V / 4) + half * (H / 4) + 2 * b2) >> 1, U);
    #pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                float2& q = P[8 * b2 + i];
                                float f = __fadd_rn(half ? q.y : q.x, -U[i]);
                                if constexpr (LAT == HQ_A2) f = (i & 1) ? __fmul_rn(f, 0.866025403784438647f) : __fmul_rn(f, 0.5f);
                                if (half) q.y = f;
                                else q.x = f;
                            }
                        }
                    }
                }
            }
            if (__any_sync(0xffffffffu, !ok)) {
    #pragma unroll
                for (int m = 0; m < H; ++m) P[m] = ok ? P[m] : make_float2(0.0f, 0.0f);
            }

            if constexpr (DST == 3) {
                // the E8 codes are doubled points: halve (exact)
                if constexpr (LAT == HQ_E8) {
    #pragma unroll
                    for (int m = 0; m < H; ++m) P[m] = f2mul(P[m], make_float2(0.5f, 0.5f));
                }
            } else {
                // ---------------- inverse transform: H_n p, exact for integer points ----------------
                // in-thread strides (H within pairs, then H/2 .. 1); with two threads per tile the
                // stride n/2 butterfly between the pair comes last
        #pragma unroll
                for (int m = 0; m < H; ++m) P[m] = make_float2(__fadd_rn(P[m].x, P[m].y), __fadd_rn(P[m].x, -P[m].y));
        #pragma unroll
                for (int h = H / 2; h >= 1; h /= 2)
        #pragma unroll
                    for (int m = 0; m < H; ++m)
                        if ((m & h) == 0) {
                            const float2 x = P[m], y = P[m + h];
                            P[m] = f2add(x, y);
                            P[m + h] = f2sub(x, y);
                        }
                if constexpr (TPT == 2) {
        #pragma unroll
                    for (int m = 0; m < H; ++m) {
                        const float ox = __shfl_xor_sync(0xffffffffu, P[m].x, 1);
                        const float oy = __shfl_xor_sync(0xffffffffu, P[m].y, 1);
                        // tau 0 holds a (positions < n/2), tau 1 holds b: a + b -> tau 0, a - b -> tau 1
                        P[m] = tau ? make_float2(__fadd_rn(ox, -P[m].x), __fadd_rn(oy, -P[m].y))
                                   : make_float2(__fadd_rn(P[m].x, ox), __fadd_rn(P[m].y, oy));
                    }
                }

                // ---------------- scale, sign, store into the staging box ----------------
                const float sh = __uint_as_float((uint32_t)sbits << 16);
                const float cn = N == 64 ? 0.125f : (N == 128 ? __uint_as_float(0x3DB504F3u) : 0.0625f);
                float ht = __fmul_rn(__fmul_rn(sh, a.beta), cn);
                if constexpr (LAT == HQ_E8) ht = __fmul_rn(ht, 0.5f);
                const float2 h2 = make_float2(ht, ht);
        #pragma unroll
                for (int m = 0; m < H; ++m) P[m] = f2mul(P[m], h2);
            }

            __syncthreads();  // every thread has read its scratch: the box may be overwritten
            if constexpr (DST == 0) {
                // bf16: 8 elements per 16-byte chunk; chunk c holds elements 8c .. 8c+7
    #pragma unroll
                for (int c = 0; c < H / 8; ++c) {
    #pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int e0 = tau * V + half * H + 8 * c;  // first element of the chunk
                        uint32_t w[4];
    #pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float lo = half ? P[8 * c + 2 * q].y : P[8 * c + 2 * q].x;
                            const float hi = half ? P[8 * c + 2 * q + 1].y : P[8 * c + 2 * q + 1].x;
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(lo, hi);  // one packed RNE conversion
                            w[q] = *reinterpret_cast<const uint32_t*>(&b2) ^ sm.mask[e0 / 2 + q];
                        }
                        const int cg = e0 / 8;
                        *reinterpret_cast<uint4*>(sm.buf + (cg >> 3) * (TI * 128) + swz(row_l, cg & 7)) =
                            make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            } else {
    #pragma unroll
                for (int c = 0; c < H / 4; ++c) {
    #pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int e0 = tau * V + half * H + 4 * c;
                        uint32_t w[4];
    #pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float f = half ? P[4 * c + q].y : P[4 * c + q].x;
                            w[q] = DST == 1 ? __float_as_uint(f) ^ sm.mask[e0 + q] : __float_as_uint(f);
                        }
                        const int cg = e0 / 4;
                        *reinterpret_cast<uint4*>(sm.buf + (cg >> 3) * (TI * 128) + swz(row_l, cg & 7)) =
                            make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
        }
        fence_proxy_async();
        __syncthreads();
        if (tid == 0) {
#pragma unroll
            for (int b = 0; b < G::NB; ++b)
                tma_store_2d(&tmap, (int)(jt * N + b * (128 / G::ES)), (int)r0, sm.buf + b * TI * 128);
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait0();
}

}  // namespace hq
